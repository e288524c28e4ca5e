// K4 chunk attention and K6a column scores for sm_100a.
//
// O = softmax(Q K^T / sqrt(d) + mask) V for one chunk's queries over the
// cache's valid slots (LingBot explainer, sliding-window section: the query
// reads the window up to local_end; Causal-Forcing walkthrough, section 3:
// only the current block's queries are computed). Masking applies only inside
// the current chunk (reading M1): a query of chunk frame r sees cached keys
// and the chunk's keys of mask class <= its own.
//
// One CTA = one 128-query tile of one head. Warp roles:
//   warp 0      TMA producer: Q tile once, then K/V tiles into a 2-stage ring
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 4..7  softmax: one query row per thread (TMEM lane = row)
// TMEM: S = Q K^T at columns [0,128) (fp32); P overwrites S's first 64
// columns as packed bf16 pairs and is the A operand of O += P V; O at columns
// [128, 128+d). Shared memory tiles use the 128-byte swizzle TMA writes and
// the UMMA descriptors read: K-major for Q and K, MN-major for V.
//
// The KV tile list is the plan's segment list (runs of valid slots with one
// mask class) cut into 128-token tiles; a tile of a segment whose mask class
// no query of this tile reaches is skipped, a ragged last tile is masked by
// column. Every wait is bounded (2 s) and reports RC_ETIMEOUT through the
// status word instead of hanging; no trap.
#include "kernels.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>

namespace rc {

namespace {

constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kTileRows = 128;
constexpr uint32_t kSubTileBytes = 128 * 64 * 2;  // 128 rows x 64 bf16
constexpr int kStatusTimeout = RC_ETIMEOUT;

template <int D>
struct Layout {
  static constexpr int kSub = D / 64;
  static constexpr uint32_t kTile = kSubTileBytes * kSub;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTile;           // 2 stages
  static constexpr uint32_t kV = kK + 2 * kTile;       // 2 stages
  static constexpr uint32_t kBytes = kV + 2 * kTile;
  static constexpr uint32_t kDynSmem = kBytes + 1024;  // alignment slack
};

struct Tile {
  int tok, nvalid, rank;
};

// Walks the plan's segments in order, yielding 128-token tiles a query tile
// with mask classes in [.., rq_hi] can see. Identical in every role.
struct TileWalker {
  const KvSegment* seg;
  int n_segs, rq_hi;
  int s = 0, off = 0;
  __device__ bool next(Tile& t) {
    while (s < n_segs) {
      const KvSegment& g = seg[s];
      if (g.rank >= 0 && g.rank > rq_hi) { ++s; off = 0; continue; }
      if (off >= g.len) { ++s; off = 0; continue; }
      t.tok = g.tok_start + off;
      t.nvalid = min(kTileRows, g.len - off);
      t.rank = g.rank;
      off += kTileRows;
      return true;
    }
    return false;
  }
};

__device__ __forceinline__ int count_tiles(const KvSegment* seg, int n, int rq_hi) {
  int c = 0;
  for (int s = 0; s < n; ++s)
    if (!(seg[s].rank >= 0 && seg[s].rank > rq_hi)) c += (seg[s].len + kTileRows - 1) / kTileRows;
  return c;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ AttnParams p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_k[2], bar_v[2], bar_kv_free[2], bar_s, bar_p, bar_o, bar_fin;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y;
  const uint32_t base_u32 = (ptx::smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - ptx::smem_u32(smem_raw));

  const int q0 = qt * kTileRows;
  const int q_last = min(q0 + kTileRows, p.Nq) - 1;
  const int rq_hi = (q_last / p.F) / p.mask_block;
  const int T = count_tiles(p.seg, p.n_segs, rq_hi);

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bar_k[i], 1);
      ptx::mbar_init(&bar_v[i], 1);
      ptx::mbar_init(&bar_kv_free[i], 1);
    }
    ptx::mbar_init(&bar_s, 1);
    ptx::mbar_init(&bar_p, 128);
    ptx::mbar_init(&bar_o, 1);
    ptx::mbar_init(&bar_fin, 1);
    abort_sh = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&tmem_base_sh, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t tS = tmem, tO = tmem + 128;
  volatile int* abort = &abort_sh;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- producer
    ptx::tma_prefetch_desc(&p.tm_q);
    ptx::tma_prefetch_desc(&p.tm_k);
    ptx::tma_prefetch_desc(&p.tm_v);
    ptx::mbar_arrive_expect_tx(&bar_q, L::kTile);
    for (int j = 0; j < L::kSub; ++j)
      ptx::tma_load_3d(&p.tm_q, &bar_q, base + L::kQ + j * kSubTileBytes, 64 * j, q0, h);
    TileWalker wk{p.seg, p.n_segs, rq_hi};
    Tile t;
    int issued[2] = {0, 0};
    for (int i = 0; wk.next(t); ++i) {
      const int st = i & 1;
      if (i >= 2 && !ptx::mbar_wait(&bar_kv_free[st], ((i >> 1) - 1) & 1, abort, p.status, kStatusTimeout))
        break;
      ptx::mbar_arrive_expect_tx(&bar_k[st], L::kTile);
      for (int j = 0; j < L::kSub; ++j)
        ptx::tma_load_3d(&p.tm_k, &bar_k[st], base + L::kK + st * L::kTile + j * kSubTileBytes, 64 * j,
                         t.tok, h);
      ptx::mbar_arrive_expect_tx(&bar_v[st], L::kTile);
      for (int j = 0; j < L::kSub; ++j)
        ptx::tma_load_3d(&p.tm_v, &bar_v[st], base + L::kV + st * L::kTile + j * kSubTileBytes, 64 * j,
                         t.tok, h);
      issued[st]++;
    }
    // never leave a copy in flight: wait (bounded, ignoring abort) for the last ones
    int dummy = 0;
    volatile int* noabort = reinterpret_cast<volatile int*>(&dummy);
    ptx::mbar_wait(&bar_q, 0, noabort, p.status, kStatusTimeout);
    for (int st = 0; st < 2; ++st)
      if (issued[st]) {
        ptx::mbar_wait(&bar_k[st], (issued[st] - 1) & 1, noabort, p.status, kStatusTimeout);
        ptx::mbar_wait(&bar_v[st], (issued[st] - 1) & 1, noabort, p.status, kStatusTimeout);
      }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc_s = ptx::idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t idesc_o = ptx::idesc_bf16(128, D, 0, 1);
    const uint32_t sQ = base_u32 + L::kQ;
    bool ok = ptx::mbar_wait(&bar_q, 0, abort, p.status, kStatusTimeout);
    for (int i = 0; ok && i < T; ++i) {
      const int st = i & 1;
      const uint32_t sK = base_u32 + L::kK + st * L::kTile;
      const uint32_t sV = base_u32 + L::kV + st * L::kTile;
      if (!ptx::mbar_wait(&bar_k[st], (i >> 1) & 1, abort, p.status, kStatusTimeout)) break;
      if (i > 0 && !ptx::mbar_wait(&bar_o, (i - 1) & 1, abort, p.status, kStatusTimeout)) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = (ks >> 2) * kSubTileBytes + (ks & 3) * 32;
        ptx::mma_ss(tS, ptx::sdesc_sw128(sQ + off, 16, 1024), ptx::sdesc_sw128(sK + off, 16, 1024), idesc_s,
                    ks > 0);
      }
      ptx::mma_commit(&bar_s);
      if (!ptx::mbar_wait(&bar_p, i & 1, abort, p.status, kStatusTimeout)) break;
      if (!ptx::mbar_wait(&bar_v[st], (i >> 1) & 1, abort, p.status, kStatusTimeout)) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 128 / 16; ++ks)
        ptx::mma_ts(tO, tS + ks * 8, ptx::sdesc_sw128(sV + ks * 2048, kSubTileBytes, 1024), idesc_o,
                    (i > 0 || ks > 0));
      ptx::mma_commit(&bar_o);
      ptx::mma_commit(&bar_kv_free[st]);
    }
    // all issued MMAs complete before TMEM is released
    int dummy = 0;
    ptx::mma_commit(&bar_fin);
    ptx::mbar_wait(&bar_fin, 0, reinterpret_cast<volatile int*>(&dummy), p.status, kStatusTimeout);
  } else if (warp >= kSoftmaxWarp0) {
    // ---------------------------------------------------------- softmax
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int qtok = q0 + row;
    const int my_rank = (min(qtok, p.Nq - 1) / p.F) / p.mask_block;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    float row_m = -INFINITY, row_l = 0.f;
    TileWalker wk{p.seg, p.n_segs, rq_hi};
    Tile t;
    bool ok = true;
    for (int i = 0; wk.next(t); ++i) {
      if (!ptx::mbar_wait(&bar_s, i & 1, abort, p.status, kStatusTimeout)) { ok = false; break; }
      ptx::tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tS + lane_off + c * 32, s[c]);
      ptx::tmem_ld_wait();
      const bool vis = t.rank < 0 || t.rank <= my_rank;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = c * 32 + j;
          float x = (vis && col < t.nvalid) ? __uint_as_float(s[c][j]) * p.scale_log2 : -INFINITY;
          s[c][j] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
      const float m_new = fmaxf(row_m, mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = ptx::ex2(row_m - m_use);
      if (i > 0) {
        if (!ptx::mbar_wait(&bar_o, (i - 1) & 1, abort, p.status, kStatusTimeout)) { ok = false; break; }
        ptx::tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            ptx::tmem_ld32(tO + lane_off + c * 32, o);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            ptx::tmem_st32(tO + lane_off + c * 32, o);
          }
        }
      }
      float sum = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = half * 64 + 2 * j;
          const float a = ptx::ex2(__uint_as_float(s[col >> 5][col & 31]) - m_use);
          const float b = ptx::ex2(__uint_as_float(s[(col + 1) >> 5][(col + 1) & 31]) - m_use);
          sum += a + b;
          pk[j] = ptx::pack_bf16x2(a, b);
        }
        ptx::tmem_st32(tS + lane_off + half * 32, pk);
      }
      ptx::tmem_st_wait();
      row_l = row_l * alpha + sum;
      row_m = m_new;
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bar_p);
    }
    // epilogue: O / l -> bf16 [Nq][H][D]; lse natural log
    bool have_o = ok && T > 0 &&
                  ptx::mbar_wait(&bar_o, (T - 1) & 1, abort, p.status, kStatusTimeout);
    ptx::tc_fence_after();
    const float inv_l = row_l > 0.f ? 1.f / row_l : 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (have_o) {
        ptx::tmem_ld32(tO + lane_off + c * 32, o);
        ptx::tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = 0u;
      }
      if (qtok < p.Nq) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)qtok * p.H + h) * D + c * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 u;
          u.x = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
          u.y = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
          u.z = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
          u.w = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
          dst[v] = u;
        }
      }
    }
    if (p.lse && qtok < p.Nq) {
      const float lse2 = row_l > 0.f ? row_m + __log2f(row_l) : -INFINITY;
      p.lse[(size_t)h * p.Nq + qtok] = lse2 * 0.69314718055994531f;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------ scores
// Column sums of softmax probabilities over history tiles: a second Q K^T
// pass that uses the attention's final LSE, p = 2^(s*c - lse*log2e). Each
// softmax warp reduces its 32 rows per column with a transpose-reduce
// (31 shuffles per 32 columns), the 4 warps combine through shared memory
// and one atomicAdd per column per CTA accumulates over query tiles and heads.
template <int D>
__global__ void __launch_bounds__(kThreads, 1) score_kernel(const __grid_constant__ ScoreParams p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_k[2], bar_kv_free[2], bar_s, bar_sfree, bar_fin;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float red[4][128];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y;
  const uint32_t base_u32 = (ptx::smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - ptx::smem_u32(smem_raw));
  const int q0 = qt * kTileRows;
  const int T = count_tiles(p.seg, p.n_segs, 0x7fffffff);

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bar_k[i], 1);
      ptx::mbar_init(&bar_kv_free[i], 1);
    }
    ptx::mbar_init(&bar_s, 1);
    ptx::mbar_init(&bar_sfree, 128);
    ptx::mbar_init(&bar_fin, 1);
    abort_sh = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&tmem_base_sh, 128);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort = &abort_sh;

  if (warp == 0 && lane == 0) {
    ptx::mbar_arrive_expect_tx(&bar_q, L::kTile);
    for (int j = 0; j < L::kSub; ++j)
      ptx::tma_load_3d(&p.tm_q, &bar_q, base + L::kQ + j * kSubTileBytes, 64 * j, q0, h);
    TileWalker wk{p.seg, p.n_segs, 0x7fffffff};
    Tile t;
    int issued[2] = {0, 0};
    for (int i = 0; wk.next(t); ++i) {
      const int st = i & 1;
      if (i >= 2 && !ptx::mbar_wait(&bar_kv_free[st], ((i >> 1) - 1) & 1, abort, p.status, kStatusTimeout))
        break;
      ptx::mbar_arrive_expect_tx(&bar_k[st], L::kTile);
      for (int j = 0; j < L::kSub; ++j)
        ptx::tma_load_3d(&p.tm_k, &bar_k[st], base + L::kK + st * L::kTile + j * kSubTileBytes, 64 * j,
                         t.tok, h);
      issued[st]++;
    }
    int dummy = 0;
    volatile int* noabort = reinterpret_cast<volatile int*>(&dummy);
    ptx::mbar_wait(&bar_q, 0, noabort, p.status, kStatusTimeout);
    for (int st = 0; st < 2; ++st)
      if (issued[st]) ptx::mbar_wait(&bar_k[st], (issued[st] - 1) & 1, noabort, p.status, kStatusTimeout);
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc_s = ptx::idesc_bf16(128, 128, 0, 0);
    const uint32_t sQ = base_u32 + L::kQ;
    bool ok = ptx::mbar_wait(&bar_q, 0, abort, p.status, kStatusTimeout);
    for (int i = 0; ok && i < T; ++i) {
      const int st = i & 1;
      const uint32_t sK = base_u32 + L::kK + st * L::kTile;
      if (!ptx::mbar_wait(&bar_k[st], (i >> 1) & 1, abort, p.status, kStatusTimeout)) break;
      if (i > 0 && !ptx::mbar_wait(&bar_sfree, (i - 1) & 1, abort, p.status, kStatusTimeout)) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = (ks >> 2) * kSubTileBytes + (ks & 3) * 32;
        ptx::mma_ss(tmem, ptx::sdesc_sw128(sQ + off, 16, 1024), ptx::sdesc_sw128(sK + off, 16, 1024), idesc_s,
                    ks > 0);
      }
      ptx::mma_commit(&bar_s);
      ptx::mma_commit(&bar_kv_free[st]);
    }
    int dummy = 0;
    ptx::mma_commit(&bar_fin);
    ptx::mbar_wait(&bar_fin, 0, reinterpret_cast<volatile int*>(&dummy), p.status, kStatusTimeout);
  } else if (warp >= kSoftmaxWarp0) {
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int qtok = q0 + row;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float lse2 = qtok < p.Nq ? p.lse[(size_t)h * p.Nq + qtok] * 1.4426950408889634f : INFINITY;
    TileWalker wk{p.seg, p.n_segs, 0x7fffffff};
    Tile t;
    for (int i = 0; wk.next(t); ++i) {
      if (!ptx::mbar_wait(&bar_s, i & 1, abort, p.status, kStatusTimeout)) break;
      ptx::tc_fence_after();
      float colsum[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t s[32];
        ptx::tmem_ld32(tmem + lane_off + c * 32, s);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) colsum[c * 32 + j] = ptx::ex2(__uint_as_float(s[j]) * p.scale_log2 - lse2);
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bar_sfree);
      // transpose-reduce over the warp's 32 rows: afterwards lane l holds
      // the 32-row sum of column (c*32 + l) in colsum[c*32]
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float* v = colsum + c * 32;
#pragma unroll
        for (int k = 16; k >= 1; k >>= 1) {
          const bool upper = (lane & k) != 0;
#pragma unroll
          for (int j = 0; j < k; ++j) {
            const float send = upper ? v[j] : v[j + k];
            const float keep = upper ? v[j + k] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, k);
          }
        }
        red[wq][c * 32 + lane] = v[0];
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      {
        const float tot = red[0][row] + red[1][row] + red[2][row] + red[3][row];
        if (row < t.nvalid) atomicAdd(p.score_phys + t.tok + row, tot);
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 128);
  }
}

template <int D>
cudaError_t launch_attn_d(const AttnParams& p, cudaStream_t s) {
  using L = Layout<D>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::kDynSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((p.Nq + kTileRows - 1) / kTileRows, p.H);
  attn_kernel<D><<<grid, kThreads, L::kDynSmem, s>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_scores_d(const ScoreParams& p, cudaStream_t s) {
  using L = Layout<D>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::kDynSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((p.Nq + kTileRows - 1) / kTileRows, p.H);
  score_kernel<D><<<grid, kThreads, L::kDynSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnParams& p, int head_dim, cudaStream_t s) {
  if (p.Nq <= 0) return cudaSuccess;
  return head_dim == 64 ? launch_attn_d<64>(p, s) : launch_attn_d<128>(p, s);
}

cudaError_t launch_scores(const ScoreParams& p, int head_dim, cudaStream_t s) {
  if (p.Nq <= 0 || p.n_segs == 0) return cudaSuccess;
  return head_dim == 64 ? launch_scores_d<64>(p, s) : launch_scores_d<128>(p, s);
}

}  // namespace rc
