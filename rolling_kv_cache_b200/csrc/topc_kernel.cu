// K6b: Deep-Forcing top-C over the history tokens' scores.
//
// rCM guide, strategy 4: each cached token is scored by the attention it
// receives and the top-C tokens of the candidate range are kept. One CTA of
// 1024 threads: (1) gathers the per-physical-token scores into logical order
// (oldest frame first, token in frame), (2) finds the C-th largest score by a
// 4-pass 8-bit radix select on order-preserving fp32 keys, (3) compacts the
// selected logical indices in index order, taking every score above the
// threshold and the lowest-index ties at it. Output is ascending; missing
// entries (fewer candidates than C) are -1.
#include "kernels.cuh"
#include "ptx.cuh"

namespace rc {

namespace {

constexpr int kTopcThreads = 1024;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exclusive block-wide scan of one int per thread; returns the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_tot[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_tot[warp - 1] : 0) + x - v;
  total = warp_tot[31];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kTopcThreads) topc_kernel(const __grid_constant__ TopCParams p) {
  __shared__ int hist[256];
  __shared__ int warp_tot[32];
  __shared__ uint32_t sh_prefix, sh_mask;
  __shared__ int sh_k;
  const int n = p.n_cand_frames * p.F;
  float* lg = p.scores_out;
  for (int i = threadIdx.x; i < n; i += kTopcThreads) {
    const int fi = i / p.F, t = i - fi * p.F;
    lg[i] = p.score_phys[(size_t)p.cand_slot[fi] * p.F + t];
  }
  __syncthreads();
  if (!p.topc || p.C <= 0) return;
  const int take = min(p.C, n);
  if (threadIdx.x == 0) {
    sh_prefix = 0;
    sh_mask = 0;
    sh_k = take;
  }
  __syncthreads();
  if (take > 0) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += kTopcThreads) hist[i] = 0;
      __syncthreads();
      const uint32_t prefix = sh_prefix, mask = sh_mask;
      for (int i = threadIdx.x; i < n; i += kTopcThreads) {
        const uint32_t key = order_key(lg[i]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int k = sh_k, cum = 0, d = 255;
        for (; d > 0; --d) {
          if (cum + hist[d] >= k) break;
          cum += hist[d];
        }
        sh_k = k - cum;
        sh_prefix = prefix | (static_cast<uint32_t>(d) << shift);
        sh_mask = mask | (255u << shift);
      }
      __syncthreads();
    }
  }
  const uint32_t thr = sh_prefix;
  const int k_eq = sh_k;  // ties at the threshold to take, lowest index first
  int eq_base = 0, out_base = 0;
  for (int c0 = 0; c0 < n && take > 0; c0 += kTopcThreads) {
    const int i = c0 + threadIdx.x;
    uint32_t key = 0;
    if (i < n) key = order_key(lg[i]);
    const int gt = (i < n && key > thr) ? 1 : 0;
    const int eq = (i < n && key == thr) ? 1 : 0;
    int eq_tot, sel_tot;
    const int eq_rank = eq_base + block_exclusive_scan(eq, warp_tot, eq_tot);
    const int sel = gt || (eq && eq_rank < k_eq);
    const int pos = out_base + block_exclusive_scan(sel, warp_tot, sel_tot);
    if (sel && pos < p.C) {
      const int fi = i / p.F, t = i - fi * p.F;
      p.topc[pos] = p.cand_lpos[fi] * p.F + t;
    }
    eq_base += eq_tot;
    out_base += sel_tot;
  }
  for (int i = take + threadIdx.x; i < p.C; i += kTopcThreads) p.topc[i] = -1;
}

// A bounded wait on a barrier that nothing completes: exercises the same
// give-up path every pipeline wait uses, without faulting the GPU.
__global__ void watchdog_kernel(int* status, unsigned limit_us) {
  __shared__ uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_sh = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    ptx::mbar_wait(&bar, 0, &abort_sh, status, RC_ETIMEOUT, (uint64_t)limit_us * 1000ull);
  __syncthreads();
}

}  // namespace

cudaError_t launch_watchdog_selftest(int* status, unsigned limit_us, cudaStream_t s) {
  watchdog_kernel<<<1, 32, 0, s>>>(status, limit_us);
  return cudaGetLastError();
}

cudaError_t launch_topc(const TopCParams& p, cudaStream_t s) {
  topc_kernel<<<1, kTopcThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace rc
