// K1 fused RoPE + append, K2 re-rotation / rotate-copy.
//
// Both are HBM-bound streaming kernels: each thread moves one 16-byte chunk
// (8 bf16 = 4 rotation pairs) of one (token, head) row with 128-bit loads and
// stores; consecutive threads touch consecutive chunks of the token-major
// input, so reads are fully coalesced and every write is a whole 256-byte
// (d=128) row segment of the head-major cache.
//
// RoPE (Causal-Forcing walkthrough, section 3: causal_rope_apply with the
// absolute start frame; LingBot explainer, two easily-missed details): pair m
// of a head vector rotates by angle pos * omega_m, pos = time index for the
// first pt pairs, latent row for the next ph, latent column for the last pw.
// cos/sin come from fp32 tables computed on the host in fp64. The rotation
// uses separately rounded products (no fused multiply-add) so that a CPU fp32
// restatement reproduces it bit for bit.
#include "kernels.cuh"
#include "df_compact.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>

#include <algorithm>

namespace rc {

namespace {

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(bf16x2_rn(f[0], f[1]), bf16x2_rn(f[2], f[3]), bf16x2_rn(f[4], f[5]),
                    bf16x2_rn(f[6], f[7]));
}

__device__ __forceinline__ float2 rope_cs(const RopeTables& rt, int m, int t, int hr, int wc) {
  if (m < rt.pt) return __ldg(rt.t + (size_t)t * rt.pt + m);
  m -= rt.pt;
  if (m < rt.ph) return __ldg(rt.h + (size_t)hr * rt.ph + m);
  m -= rt.ph;
  return __ldg(rt.w + (size_t)wc * rt.pw + m);
}

// Element offset of (head h, token row t, 16-byte chunk c8) in a ring
// buffer. K and V keep each head in d/64 planes of 64 dims, [H][d/64][cap][64],
// so the time pairs (the first 2 P_t < 64 dims) of consecutive tokens sit in
// dense 128-byte rows of plane 0 and an in-place time rotation reads and
// writes 96 of every 128 bytes instead of 96 of every 256.
__device__ __forceinline__ size_t cache_off(int h, int planes, int cap, int t, int c8) {
  return (((size_t)h * planes + (c8 >> 3)) * cap + t) * 64 + (c8 & 7) * 8;
}

// (x, y) -> (x c - y s, x s + y c), products rounded separately.
__device__ __forceinline__ void rot(float& x, float& y, float c, float s) {
  float nx = __fsub_rn(__fmul_rn(x, c), __fmul_rn(y, s));
  float ny = __fadd_rn(__fmul_rn(x, s), __fmul_rn(y, c));
  x = nx;
  y = ny;
}

// Thread layout of both kernels: threadIdx.x = 16-byte chunk of a head row
// (d/8 lanes cover one row), threadIdx.y = row within the block; rows are
// walked grid-stride in 32-bit arithmetic.
__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendParams p) {
  const int c8 = threadIdx.x;
  const int rows = p.n_tok * p.H;  // (token, head) rows in input order
  for (int row = blockIdx.x * blockDim.y + threadIdx.y; row < rows; row += gridDim.x * blockDim.y) {
    const int tok = row / p.H;
    const int h = row - tok * p.H;
    const int r = tok / p.F;
    const int n_in = tok - r * p.F;
    const int hr = n_in / p.rt.grid_w;
    const int wc = n_in - hr * p.rt.grid_w;
    const size_t src = (size_t)row * p.d + c8 * 8;
    uint4 uq = __ldg(reinterpret_cast<const uint4*>(p.q + src));
    uint4 uk = __ldg(reinterpret_cast<const uint4*>(p.k + src));
    uint4 uv = __ldg(reinterpret_cast<const uint4*>(p.v + src));
    float fq[8], fk[8];
    unpack8(uq, fq);
    unpack8(uk, fk);
    const int t = p.sigma[r];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 cs = rope_cs(p.rt, c8 * 4 + j, t, hr, wc);
      rot(fq[2 * j], fq[2 * j + 1], cs.x, cs.y);
      rot(fk[2 * j], fk[2 * j + 1], cs.x, cs.y);
    }
    const size_t qdst = ((size_t)h * p.q_stride + tok) * p.d + c8 * 8;
    const size_t cdst = cache_off(h, p.d / 64, p.cap, p.slot[r] * p.F + n_in, c8);
    *reinterpret_cast<uint4*>(p.q_rot + qdst) = pack8(fq);
    *reinterpret_cast<uint4*>(p.kc + cdst) = pack8(fk);
    *reinterpret_cast<uint4*>(p.vc + cdst) = uv;
    const int rf = p.raw_frame[r];
    if (rf >= 0) {
      const size_t rdst = ((size_t)h * p.raw_cap + (size_t)rf * p.F + n_in) * p.d + c8 * 8;
      *reinterpret_cast<uint4*>(p.raw_k + rdst) = uk;
      if (p.raw_v) *reinterpret_cast<uint4*>(p.raw_v + rdst) = uv;
    }
  }
}

// One job per blockIdx.y; rows ordered (head, token in frame) so a warp
// writes whole consecutive rows of one head's slot. Rotate-copy rewrites the
// key row from the pristine raw source at the job's target time (and copies
// V when the slot's content changes); in-place composes R_t(delta) onto the
// stored key and touches only the chunks that hold time pairs.
__global__ void __launch_bounds__(256) rerotate_kernel(const __grid_constant__ RerotateParams p) {
  const RerotateJob& jb = p.job[blockIdx.y];
  const int rows = p.F * p.H;
  if (jb.mode == 1) {
    // in place: only the ct chunks holding time pairs; the block's threads
    // are packed densely over (row, chunk) so every lane has work
    const int ct = (2 * p.rt.pt + 7) / 8;
    const float sgn = jb.delta < 0 ? -1.f : 1.f;
    const int adelta = jb.delta < 0 ? -jb.delta : jb.delta;
    const int nthr = blockDim.x * blockDim.y;
    const int total = rows * ct;
    for (int i = blockIdx.x * nthr + threadIdx.y * blockDim.x + threadIdx.x; i < total; i += gridDim.x * nthr) {
      const int row = i / ct;
      const int c8 = i - row * ct;
      const int h = row / p.F;
      const int n_in = row - h * p.F;
      const size_t dst = cache_off(h, p.d / 64, p.cap, jb.dst_slot * p.F + n_in, c8);
      float f[8];
      uint4 u = *reinterpret_cast<const uint4*>(p.kc + dst);
      unpack8(u, f);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int m = c8 * 4 + j;
        if (m < p.rt.pt) {
          float2 cs = __ldg(p.rt.t + (size_t)adelta * p.rt.pt + m);
          rot(f[2 * j], f[2 * j + 1], cs.x, sgn * cs.y);
        }
      }
      *reinterpret_cast<uint4*>(p.kc + dst) = pack8(f);
    }
    return;
  }
  const int c8 = threadIdx.x;
  for (int row = blockIdx.x * blockDim.y + threadIdx.y; row < rows; row += gridDim.x * blockDim.y) {
    const int h = row / p.F;
    const int n_in = row - h * p.F;
    const size_t dst = cache_off(h, p.d / 64, p.cap, jb.dst_slot * p.F + n_in, c8);
    float f[8];
    {
      const int hr = n_in / p.rt.grid_w;
      const int wc = n_in - hr * p.rt.grid_w;
      const size_t src = ((size_t)h * p.raw_cap + (size_t)jb.src_frame * p.F + n_in) * p.d + c8 * 8;
      uint4 u = __ldg(reinterpret_cast<const uint4*>(p.raw_k + src));
      unpack8(u, f);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 cs = rope_cs(p.rt, c8 * 4 + j, jb.sigma, hr, wc);
        rot(f[2 * j], f[2 * j + 1], cs.x, cs.y);
      }
      *reinterpret_cast<uint4*>(p.kc + dst) = pack8(f);
      if (jb.copy_v)
        *reinterpret_cast<uint4*>(p.vc + dst) = __ldg(reinterpret_cast<const uint4*>(p.raw_v + src));
    }
  }
}

// K2 in place, TMA-staged. The time pairs of a key row are its first 2 pt
// dims, which sit in plane 0: ct 16-byte chunks (96 of the row's 128 bytes
// at pt = 22). Each work item is one (job, head, block of R rows) of a slot;
// a TMA box brings the item's R x 8 ct dims into a ring of kStages
// shared-memory stages, so every CTA keeps kStages boxes of reads in flight
// instead of one 16-byte load per thread. Threads rotate their chunks from
// shared memory and store them back with 16-byte stores, only the rows of
// the slot (a box past the slot's last row reads rows it never writes).
// Thread t always handles chunk t % ct of a row, so its four (cos, sin)
// pairs are loaded once per item. Bounded waits; on give-up the CTA waits
// (bounded) for its loads in flight and returns with RC_ETIMEOUT recorded.
constexpr int kInplaceStages = 4;

__global__ void __launch_bounds__(256) rerotate_inplace_kernel(const __grid_constant__ InplaceParams p) {
  extern __shared__ __align__(128) uint8_t ip_smem[];
  __shared__ uint64_t full[kInplaceStages];
  __shared__ int abort_sh;
  const int tid = threadIdx.x;
  const int stage_bytes = (p.R * p.ct * 16 + 127) & ~127;
  const int n_items = p.n_jobs * p.H * p.tiles_per_head;
  const int G = gridDim.x;
  const int n_local = blockIdx.x < n_items ? (n_items - blockIdx.x + G - 1) / G : 0;
  if (tid == 0) {
    for (int s = 0; s < kInplaceStages; ++s) ptx::mbar_init(&full[s], 1);
    abort_sh = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &abort_sh;
  auto issue = [&](int i) {  // local item i into stage i % kInplaceStages (thread 0)
    const int item = blockIdx.x + i * G;
    const int j = item / (p.H * p.tiles_per_head);
    const int rem = item - j * p.H * p.tiles_per_head;
    const int h = rem / p.tiles_per_head;
    const int b = rem - h * p.tiles_per_head;
    uint64_t* bar = &full[i % kInplaceStages];
    ptx::mbar_arrive_expect_tx(bar, (uint32_t)(p.R * p.ct * 16));
    ptx::tma_load_3d(&p.tm, bar, ip_smem + (i % kInplaceStages) * stage_bytes, 0, p.slot[j] * p.F + b * p.R,
                     h * p.planes);
  };
  if (tid == 0) {
    ptx::fence_proxy_async_smem();
    for (int i = 0; i < n_local && i < kInplaceStages; ++i) issue(i);
  }
  const int c8 = tid % p.ct;
  const int row_step = blockDim.x / p.ct;
  const bool active = tid < row_step * p.ct;
  int i = 0;
  for (; i < n_local; ++i) {
    const int st = i % kInplaceStages;
    const bool ok = ptx::mbar_wait(&full[st], (i / kInplaceStages) & 1, abort, p.status, RC_ETIMEOUT);
    if (ok && active) {
      const int item = blockIdx.x + i * G;
      const int j = item / (p.H * p.tiles_per_head);
      const int rem = item - j * p.H * p.tiles_per_head;
      const int h = rem / p.tiles_per_head;
      const int b = rem - h * p.tiles_per_head;
      const int r0 = b * p.R;
      const int nrows = min(p.R, p.F - r0);
      const int delta = p.delta[j];
      const float sgn = delta < 0 ? -1.f : 1.f;
      const int adelta = delta < 0 ? -delta : delta;
      float cs_c[4], cs_s[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int m = c8 * 4 + jj;
        const float2 cs = m < p.pt ? __ldg(p.tab_t + (size_t)adelta * p.pt + m) : make_float2(1.f, 0.f);
        cs_c[jj] = cs.x;
        cs_s[jj] = sgn * cs.y;
      }
      const uint4* src = reinterpret_cast<const uint4*>(ip_smem + st * stage_bytes);
      uint16_t* dst0 = p.kc + cache_off(h, p.planes, p.cap, p.slot[j] * p.F + r0, c8);
      for (int row = tid / p.ct; row < nrows; row += row_step) {
        float f[8];
        unpack8(src[row * p.ct + c8], f);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          if (c8 * 4 + jj < p.pt) rot(f[2 * jj], f[2 * jj + 1], cs_c[jj], cs_s[jj]);
        *reinterpret_cast<uint4*>(dst0 + (size_t)row * 64) = pack8(f);
      }
    }
    // every thread reaches this barrier (the waits are bounded): stage st is
    // consumed, and all leave together if any wait gave up
    if (__syncthreads_or(!ok)) break;
    if (tid == 0 && i + kInplaceStages < n_local) {
      ptx::fence_proxy_async_smem();
      issue(i + kInplaceStages);
    }
  }
  if (i < n_local && tid == 0) {
    // gave up: wait (bounded, ignoring the abort flag) for the loads still in flight
    int dummy = 0;
    volatile int* noabort = reinterpret_cast<volatile int*>(&dummy);
    for (int k = i; k < n_local && k < i + kInplaceStages; ++k)
      ptx::mbar_wait(&full[k % kInplaceStages], (k / kInplaceStages) & 1, noabort, p.status, RC_ETIMEOUT);
  }
}

// K7 Deep Forcing compaction (rCM guide, strategy 4: keep the top-C scored
// tokens, then rewrite their time encoding so no holes remain). One thread
// per 16-byte chunk of a (head, new region token) row, rows head-major so a
// warp writes consecutive rows of one head; sources are gathered.
__global__ void __launch_bounds__(256) df_compact_kernel(const __grid_constant__ DfCompactParams p) {
  const int c8 = threadIdx.x;
  const int rows = p.H * p.n_new;
  const int planes = p.d / 64;
  for (int r = blockIdx.x * blockDim.y + threadIdx.y; r < rows; r += gridDim.x * blockDim.y) {
    const int h = r / p.n_new;
    const int i = r - h * p.n_new;
    const int pi = p.sel ? __ldg(p.sel + i) : i;
    int src_row;
    int2 meta;
    if (pi < p.n_old) {
      src_row = p.src_row0 + pi;
      meta = p.meta_src[pi];
    } else {
      const int q = pi - p.n_old;
      const int e = q / p.F;
      const int t = q - e * p.F;
      src_row = p.e_slot[e] * p.F + t;
      meta = make_int2(p.e_frame[e], t);
    }
    const int dst_row = p.dst_row0 + i;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.vc + cache_off(h, planes, p.cap, src_row, c8)));
    if (p.keep_time) {
      // Relax Forcing: the key already sits at its frame's time; move it and
      // the frame's descriptor (by the thread rows of the frame's first token)
      *reinterpret_cast<uint4*>(p.kc + cache_off(h, planes, p.cap, dst_row, c8)) =
          *reinterpret_cast<const uint4*>(p.kc + cache_off(h, planes, p.cap, src_row, c8));
      if (i % p.F == 0) {
        const int src_vs = pi < p.n_old ? p.src_vslot0 + pi / p.F : p.e_slot[(pi - p.n_old) / p.F];
        const float4* sd = reinterpret_cast<const float4*>(p.desc + ((size_t)src_vs * p.H + h) * p.d + c8 * 8);
        float4* dd = reinterpret_cast<float4*>(p.desc + ((size_t)(p.dst_vslot0 + i / p.F) * p.H + h) * p.d + c8 * 8);
        dd[0] = sd[0];
        dd[1] = sd[1];
      }
    } else {
      const int hr = meta.y / p.rt.grid_w;
      const int wc = meta.y - hr * p.rt.grid_w;
      const int tau = p.tau_new0 + i / p.F;
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p.raw_k + ((size_t)h * p.cap + src_row) * p.d + c8 * 8));
      float f[8];
      unpack8(raw, f);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 cs = rope_cs(p.rt, c8 * 4 + j, tau, hr, wc);
        rot(f[2 * j], f[2 * j + 1], cs.x, cs.y);
      }
      *reinterpret_cast<uint4*>(p.kc + cache_off(h, planes, p.cap, dst_row, c8)) = pack8(f);
      *reinterpret_cast<uint4*>(p.raw_k + ((size_t)h * p.cap + dst_row) * p.d + c8 * 8) = raw;
    }
    *reinterpret_cast<uint4*>(p.vc + cache_off(h, planes, p.cap, dst_row, c8)) = v;
    if (h == 0 && c8 == 0) p.meta_dst[i] = meta;
  }
}

// MemRoPE update: one thread per 16-byte chunk of a (memory, token, head)
// row; the EMA runs in fp32 with separately rounded products so a CPU fp32
// restatement reproduces it bit for bit.
__global__ void __launch_bounds__(256) mem_update_kernel(const __grid_constant__ MemUpdateParams p) {
  const int c8 = threadIdx.x;
  const int per_mem = p.F * p.H;
  const int rows = 2 * per_mem;
  const int planes = p.d / 64;
  for (int r = blockIdx.x * blockDim.y + threadIdx.y; r < rows; r += gridDim.x * blockDim.y) {
    const int m = r >= per_mem;          // 0 long-term, 1 short-term
    const int rr = r - m * per_mem;
    const int t = rr / p.H;
    const int h = rr - t * p.H;
    float* sk = p.mem + (((size_t)(0 * 2 + m) * p.F + t) * p.H + h) * p.d + c8 * 8;
    float* sv = p.mem + (((size_t)(1 * 2 + m) * p.F + t) * p.H + h) * p.d + c8 * 8;
    float k[8], v[8];
    if (p.initialised) {
      const float4* k4 = reinterpret_cast<const float4*>(sk);
      const float4* v4 = reinterpret_cast<const float4*>(sv);
      const float4 k0 = k4[0], k1 = k4[1], v0 = v4[0], v1 = v4[1];
      k[0] = k0.x; k[1] = k0.y; k[2] = k0.z; k[3] = k0.w; k[4] = k1.x; k[5] = k1.y; k[6] = k1.z; k[7] = k1.w;
      v[0] = v0.x; v[1] = v0.y; v[2] = v0.z; v[3] = v0.w; v[4] = v1.x; v[5] = v1.y; v[6] = v1.z; v[7] = v1.w;
    }
    for (int e = 0; e < p.n_e; ++e) {
      const int row = p.e_slot[e] * p.F + t;
      float xk[8], xv[8];
      unpack8(__ldg(reinterpret_cast<const uint4*>(p.raw_k + ((size_t)h * p.raw_cap + row) * p.d + c8 * 8)), xk);
      unpack8(__ldg(reinterpret_cast<const uint4*>(p.vc + cache_off(h, planes, p.cap, row, c8))), xv);
      const bool first = !p.initialised && e == 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        k[j] = first ? xk[j] : __fadd_rn(__fmul_rn(p.a[m], k[j]), __fmul_rn(p.b[m], xk[j]));
        v[j] = first ? xv[j] : __fadd_rn(__fmul_rn(p.a[m], v[j]), __fmul_rn(p.b[m], xv[j]));
      }
    }
    if (p.n_e > 0) {
      float4* k4 = reinterpret_cast<float4*>(sk);
      float4* v4 = reinterpret_cast<float4*>(sv);
      k4[0] = make_float4(k[0], k[1], k[2], k[3]);
      k4[1] = make_float4(k[4], k[5], k[6], k[7]);
      v4[0] = make_float4(v[0], v[1], v[2], v[3]);
      v4[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
    const int hr = t / p.rt.grid_w;
    const int wc = t - hr * p.rt.grid_w;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 cs = rope_cs(p.rt, c8 * 4 + j, p.tau[m], hr, wc);
      rot(k[2 * j], k[2 * j + 1], cs.x, cs.y);
    }
    const int dst = p.row0 + m * p.F + t;
    *reinterpret_cast<uint4*>(p.kc + cache_off(h, planes, p.cap, dst, c8)) = pack8(k);
    *reinterpret_cast<uint4*>(p.vc + cache_off(h, planes, p.cap, dst, c8)) = pack8(v);
  }
}

// Blocks of 256 threads of `kernel` resident at once on the current GPU
// (blocks per SM from the occupancy API x SMs). The grid-stride kernels below
// launch at most one full wave: blocks beyond it would only start when others
// finish their whole loops and leave the tail of the launch to a few SMs.
template <typename Kernel>
int one_wave(Kernel kernel, PerDevice& cache) {
  int n = 0;
  const cudaError_t e = cache.get(&n, [kernel](int dev, int* x) {
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess || per_sm < 1)
      per_sm = 4;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;
    *x = per_sm * sms;
    return cudaSuccess;
  });
  return e == cudaSuccess && n > 0 ? n : 4 * 148;
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
  const int rows = p.n_tok * p.H;
  if (rows == 0) return cudaSuccess;
  const dim3 block(p.d / 8, 256 / (p.d / 8));
  static PerDevice wave;
  int blocks = (rows + block.y - 1) / block.y;
  const int cap = one_wave(append_kernel, wave);
  if (blocks > cap) blocks = cap;
  append_kernel<<<blocks, block, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_rerotate(const RerotateParams& p, cudaStream_t s) {
  if (p.n_jobs == 0) return cudaSuccess;
  const dim3 block(p.d / 8, 256 / (p.d / 8));
  const int rows = p.F * p.H;
  int bx = (rows + block.y - 1) / block.y;
  static PerDevice wave;
  const int cap = one_wave(rerotate_kernel, wave) / p.n_jobs;
  if (bx > cap) bx = cap;
  if (bx < 1) bx = 1;
  rerotate_kernel<<<dim3(bx, p.n_jobs), block, 0, s>>>(p);
  return cudaGetLastError();
}

int inplace_box_rows(int F) {
  if (F <= 256) return F;
  for (int r = 128; r >= 64; --r)
    if (F % r == 0) return r;
  return 128;
}

cudaError_t launch_rerotate_inplace(const InplaceParams& p, cudaStream_t s) {
  const int n_items = p.n_jobs * p.H * p.tiles_per_head;
  if (n_items == 0) return cudaSuccess;
  const int threads = 32 * p.ct;
  const int smem = kInplaceStages * ((p.R * p.ct * 16 + 127) & ~127);
  static PerDevice attr_set;
  static PerDevice wave;
  int done = 0;
  cudaError_t e = attr_set.get(&done, [](int, int* x) {
    *x = 1;
    return cudaFuncSetAttribute(rerotate_inplace_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 1024);
  });
  if (e != cudaSuccess) return e;
  int cap = 0;
  e = wave.get(&cap, [](int dev, int* x) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;
    *x = sms;
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  // a few CTAs per SM: each keeps kInplaceStages boxes in flight
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rerotate_inplace_kernel, threads, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int blocks = std::min(n_items, cap * std::min(per_sm, 4));
  rerotate_inplace_kernel<<<blocks, threads, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_mem_update(const MemUpdateParams& p, cudaStream_t s) {
  const int rows = 2 * p.F * p.H;
  const dim3 block(p.d / 8, 256 / (p.d / 8));
  static PerDevice wave;
  int blocks = (rows + block.y - 1) / block.y;
  const int cap = one_wave(mem_update_kernel, wave);
  if (blocks > cap) blocks = cap;
  mem_update_kernel<<<blocks, block, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_df_compact(const DfCompactParams& p, cudaStream_t s) {
  const int rows = p.H * p.n_new;
  if (rows == 0) return cudaSuccess;
  const dim3 block(p.d / 8, 256 / (p.d / 8));
  static PerDevice wave;
  int blocks = (rows + block.y - 1) / block.y;
  const int cap = one_wave(df_compact_kernel, wave);
  if (blocks > cap) blocks = cap;
  df_compact_kernel<<<blocks, block, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace rc
