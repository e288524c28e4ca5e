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

#include <cuda_bf16.h>

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

// (x, y) -> (x c - y s, x s + y c), products rounded separately.
__device__ __forceinline__ void rot(float& x, float& y, float c, float s) {
  float nx = __fsub_rn(__fmul_rn(x, c), __fmul_rn(y, s));
  float ny = __fadd_rn(__fmul_rn(x, s), __fmul_rn(y, c));
  x = nx;
  y = ny;
}

__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendParams p) {
  const int chunks = p.d >> 3;
  const long long total = (long long)p.n_tok * p.H * chunks;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int c8 = (int)(i % chunks);
    const long long th = i / chunks;
    const int h = (int)(th % p.H);
    const int tok = (int)(th / p.H);
    const int r = tok / p.F;
    const int n_in = tok - r * p.F;
    const int hr = n_in / p.rt.grid_w;
    const int wc = n_in - hr * p.rt.grid_w;
    const size_t src = ((size_t)tok * p.H + h) * p.d + c8 * 8;
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
    const size_t cdst = ((size_t)h * p.cap + (size_t)p.slot[r] * p.F + n_in) * p.d + c8 * 8;
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

// One job per blockIdx.y. Rotate-copy rewrites the whole key row from the
// pristine raw source at the job's target time (and copies V when the slot's
// content changes); in-place composes R_t(delta) onto the stored key, touching
// only the chunks that hold time pairs.
__global__ void __launch_bounds__(256) rerotate_kernel(const __grid_constant__ RerotateParams p) {
  const RerotateJob& jb = p.job[blockIdx.y];
  const bool inplace = jb.mode == 1;
  const int chunks = inplace ? (2 * p.rt.pt + 7) / 8 : p.d / 8;
  const long long total = (long long)p.F * p.H * chunks;
  const float sgn = jb.delta < 0 ? -1.f : 1.f;
  const int adelta = jb.delta < 0 ? -jb.delta : jb.delta;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int c8 = (int)(i % chunks);
    const long long th = i / chunks;
    const int h = (int)(th % p.H);
    const int n_in = (int)(th / p.H);
    const size_t dst = ((size_t)h * p.cap + (size_t)jb.dst_slot * p.F + n_in) * p.d + c8 * 8;
    float f[8];
    if (inplace) {
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
    } else {
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

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
  const long long total = (long long)p.n_tok * p.H * (p.d / 8);
  if (total == 0) return cudaSuccess;
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)sm_count() * 8;  // 8 resident 256-thread blocks per SM
  if (blocks > cap) blocks = cap;
  append_kernel<<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_rerotate(const RerotateParams& p, cudaStream_t s) {
  if (p.n_jobs == 0) return cudaSuccess;
  const long long per_job = (long long)p.F * p.H * (p.d / 8);
  long long bx = (per_job + 255) / 256;
  const long long cap = ((long long)sm_count() * 8 + p.n_jobs - 1) / p.n_jobs;
  if (bx > cap) bx = cap;
  if (bx < 1) bx = 1;
  rerotate_kernel<<<dim3((unsigned)bx, (unsigned)p.n_jobs), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace rc
