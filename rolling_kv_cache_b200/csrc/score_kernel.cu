// K6a: Deep-Forcing token scores for sm_100a.
//
// rCM guide, strategy 4: every cached token is scored by the attention its
// key receives from the current chunk's queries. Reading S1: score[j] = sum
// over heads and queries of the softmax probability the attention used,
// p = exp(q.k_j / sqrt(d) - LSE), with the attention's final LSE. This is a
// second Q K^T pass over the history tiles only (sink and current chunk are
// not candidates).
//
// One CTA = one 128-query tile of one head; warp 0 loads Q and K tiles
// (TMA, 2-stage ring), warp 1 issues S = Q K^T into TMEM, warps 4..7 turn a
// row of S into probabilities and reduce columns. Bounded waits, no trap.
#include "attn_common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>

namespace rc {

namespace {

constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
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

cudaError_t launch_scores(const ScoreParams& p, int head_dim, cudaStream_t s) {
  if (p.Nq <= 0 || p.n_segs == 0) return cudaSuccess;
  return head_dim == 64 ? launch_scores_d<64>(p, s) : launch_scores_d<128>(p, s);
}

}  // namespace rc
