// K6b: Deep-Forcing top-C over the history tokens' scores.
//
// rCM guide, strategy 4: each cached token is scored by the attention it
// receives and the top-C tokens of the candidate range are kept. One cluster
// of kTopcCluster CTAs x 1024 threads, each CTA owning a contiguous slice of
// the candidates in logical order: (1) each gathers its slice's
// per-physical-token scores into logical order (oldest frame first, token in
// frame), (2) together they find the C-th largest score by a 4-pass 8-bit
// radix select on order-preserving fp32 keys: every CTA counts its slice,
// then reads the other CTAs' counts through distributed shared memory and
// takes the same decision, (3) each compacts the selected logical indices of
// its slice in index order after the slices before it, taking every score
// above the threshold and the lowest-index ties at it. Output is ascending;
// missing entries (fewer candidates than C) are -1.
// A few CTAs run on latency, not bandwidth: the gather keeps eight loads in
// flight per thread, and a slice's order keys stay in shared memory for the
// passes and the compaction (up to kTopcSmemKeys per CTA; a larger candidate
// set reads its keys back from the logical-order scores in global memory).
// The scores of one step share their top bytes, so a warp adds the count of
// its lanes that fall in the first valid lane's bin with one atomic (the
// rest add their own), each warp into its own histogram; one warp finds the
// threshold digit by a shuffle scan over the 256 bins; the compaction gives
// each thread a contiguous run of candidates and places them with one block
// scan of (above, tied) counts plus the counts of the slices before: the
// selected elements before a thread are the above ones plus min(ties before
// it, ties taken).
#include <cooperative_groups.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace rc {

namespace {

constexpr int kTopcThreads = 1024;
constexpr int kTopcCluster = 8;       // CTAs (one cluster), each owning a slice of the candidates
constexpr int kTopcSmemKeys = 45056;  // 176 KB of order keys per CTA
constexpr int kTopcGather = 8;        // gather loads in flight per thread
static_assert(kTopcThreads == 1024, "the histogram sum maps 1024 threads onto 256 bins x 4 warp groups");

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exclusive block-wide scan of one 64-bit value per thread; returns the
// block total in `total`.
__device__ __forceinline__ long long block_exclusive_scan(long long v, long long* warp_tot, long long& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_tot[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const long long before = (warp > 0 ? warp_tot[warp - 1] : 0) + x - v;
  total = warp_tot[31];
  __syncthreads();
  return before;
}

__global__ void __cluster_dims__(kTopcCluster, 1, 1) __launch_bounds__(kTopcThreads)
    topc_kernel(const __grid_constant__ TopCParams p, int keys_in_smem) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  extern __shared__ uint32_t skey[];  // [slice] order keys, when keys_in_smem
  __shared__ int hist[2][256];        // this slice's counts, double buffered across passes
  __shared__ int ghist[256];          // every slice's counts
  __shared__ int whist[kTopcThreads / 32][257];  // per-warp histograms (padded row: no bank conflicts in the sum)
  __shared__ long long warp_tot[32];
  __shared__ long long slice_tot;     // (above << 32 | tied) of this slice
  __shared__ uint32_t sh_prefix, sh_mask;
  __shared__ int sh_k;
  const int n = p.n_cand_frames * p.F;
  const int rank = (int)cl.block_rank();
  const int chunk = (n + kTopcCluster - 1) / kTopcCluster;
  const int lo = min(n, rank * chunk), hi = min(n, lo + chunk), nl = hi - lo;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* lg = p.scores_out;
  // this thread's candidates i = lo + threadIdx.x + m kTopcThreads, as (frame
  // fi, token t) advanced by a fixed step instead of a division per element
  const int step_f = kTopcThreads / p.F, step_t = kTopcThreads - step_f * p.F;
  int fi = (lo + threadIdx.x) / p.F, t = lo + threadIdx.x - fi * p.F;
  for (int b = threadIdx.x; b < nl; b += kTopcGather * kTopcThreads) {
    float v[kTopcGather];
#pragma unroll
    for (int u = 0; u < kTopcGather; ++u) {
      const int i = b + u * kTopcThreads;
      if (i < nl) v[u] = p.score_phys[(size_t)p.cand_slot[fi] * p.F + t];
      fi += step_f;
      t += step_t;
      if (t >= p.F) {
        t -= p.F;
        ++fi;
      }
    }
#pragma unroll
    for (int u = 0; u < kTopcGather; ++u) {
      const int i = b + u * kTopcThreads;
      if (i < nl) {
        lg[lo + i] = v[u];
        if (keys_in_smem) skey[i] = order_key(v[u]);
      }
    }
  }
  __syncthreads();
  // key of the slice's i-th candidate
  auto key_at = [&](int i) -> uint32_t { return keys_in_smem ? skey[i] : order_key(lg[lo + i]); };
  if (!p.topc || p.C <= 0) return;  // the same for every CTA: no shared memory is read remotely
  const int take = min(p.C, n);
  if (threadIdx.x == 0) {
    sh_prefix = 0;
    sh_mask = 0;
    sh_k = take;
  }
  __syncthreads();
  if (take > 0) {
    for (int shift = 24, pass = 0; shift >= 0; shift -= 8, ++pass) {
      // each warp counts into its own histogram (no contention between warps
      // on the few bins the scores of one step share); summed below
      for (int i = lane; i < 256; i += 32) whist[warp][i] = 0;
      __syncwarp();
      const uint32_t prefix = sh_prefix, mask = sh_mask;
      // whole warps step together (b is warp-uniform) so the votes see every lane
      for (int b = warp * 32; b < nl; b += kTopcThreads) {
        const int i = b + lane;
        int digit = -1;
        if (i < nl) {
          const uint32_t key = key_at(i);
          if ((key & mask) == prefix) digit = (int)((key >> shift) & 255u);
        }
        const uint32_t valid = __ballot_sync(0xffffffffu, digit >= 0);
        if (valid == 0) continue;
        const int src = __ffs(valid) - 1;
        const int lead = __shfl_sync(0xffffffffu, digit, src);
        const uint32_t same = __ballot_sync(0xffffffffu, digit == lead);
        if (lane == src) atomicAdd(&whist[warp][lead], __popc(same));
        else if (digit >= 0 && digit != lead) atomicAdd(&whist[warp][digit], 1);
      }
      __syncthreads();
      int* h = hist[pass & 1];
      {  // bin t / 4 summed over warps 8 (t % 4) .. 8 (t % 4) + 7, then over the 4 threads
        const int bin = threadIdx.x >> 2, w0 = (threadIdx.x & 3) * 8;
        int c = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) c += whist[w0 + w][bin];
        c += __shfl_xor_sync(0xffffffffu, c, 1);
        c += __shfl_xor_sync(0xffffffffu, c, 2);
        if ((threadIdx.x & 3) == 0) h[bin] = c;
      }
      // every slice's counts are written; this pass's buffer is not written
      // again before the next pass's barrier, after every CTA has read it
      cl.sync();
      {  // bin t / 4 summed over CTAs 2 (t % 4), 2 (t % 4) + 1, then over the 4 threads
        const int bin = threadIdx.x >> 2, r0 = (threadIdx.x & 3) * (kTopcCluster / 4);
        int c = 0;
#pragma unroll
        for (int r = 0; r < kTopcCluster / 4; ++r) c += cl.map_shared_rank(h, r0 + r)[bin];
        c += __shfl_xor_sync(0xffffffffu, c, 1);
        c += __shfl_xor_sync(0xffffffffu, c, 2);
        if ((threadIdx.x & 3) == 0) ghist[bin] = c;
      }
      __syncthreads();
      if (warp == 0) {
        // lane l holds bins 255 - 8 l - j (j = 0..7): counts from the top
        int cnt[8], tot = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          cnt[j] = ghist[255 - 8 * lane - j];
          tot += cnt[j];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int excl = incl - tot;
        const int k = sh_k;
        // the first bin, from the top, at which the running count reaches k
        // (bin 0 if none does)
        const uint32_t hit = __ballot_sync(0xffffffffu, excl < k && k <= incl);
        const int hl = hit ? __ffs(hit) - 1 : 31;
        if (lane == hl) {
          int cum = excl, d = 0;
          for (int j = 0; j < 8; ++j) {
            d = 255 - 8 * lane - j;
            if (cum + cnt[j] >= k || d == 0) break;
            cum += cnt[j];
          }
          sh_k = k - cum;
          sh_prefix = prefix | (static_cast<uint32_t>(d) << shift);
          sh_mask = mask | (255u << shift);
        }
      }
      __syncthreads();
    }
    const uint32_t thr = sh_prefix;
    const int k_eq = sh_k;  // ties at the threshold to take, lowest index first
    const int per = (nl + kTopcThreads - 1) / kTopcThreads;
    const int i0 = min(nl, threadIdx.x * per), i1 = min(nl, i0 + per);
    int gt = 0, eq = 0;
    for (int i = i0; i < i1; ++i) {
      const uint32_t key = key_at(i);
      gt += key > thr;
      eq += key == thr;
    }
    long long tot;
    const long long before = block_exclusive_scan(((long long)gt << 32) | (long long)eq, warp_tot, tot);
    if (threadIdx.x == 0) slice_tot = tot;
    cl.sync();  // every slice's totals are written
    long long base = 0;  // (above, tied) of the slices before this one
    for (int r = 0; r < rank; ++r) base += *cl.map_shared_rank(&slice_tot, r);
    const int gt_before = (int)(before >> 32) + (int)(base >> 32);
    const int eq_before = (int)(before & 0xffffffffll) + (int)(base & 0xffffffffll);
    int pos = gt_before + min(eq_before, k_eq);
    int eq_seen = eq_before;
    for (int i = i0; i < i1; ++i) {
      const uint32_t key = key_at(i);
      bool sel = key > thr;
      if (key == thr) sel = eq_seen++ < k_eq;
      if (sel) {
        if (pos < p.C) {
          const int g = lo + i;
          const int fi2 = g / p.F, t2 = g - fi2 * p.F;
          p.topc[pos] = p.cand_lpos[fi2] * p.F + t2;
        }
        ++pos;
      }
    }
  }
  if (rank == 0)
    for (int i = take + threadIdx.x; i < p.C; i += kTopcThreads) p.topc[i] = -1;
  cl.sync();  // no CTA leaves while another may still read its shared memory
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
  static PerDevice attr_set;
  int done = 0;
  cudaError_t e = attr_set.get(&done, [](int, int* x) {
    *x = 1;
    return cudaFuncSetAttribute(topc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kTopcSmemKeys * (int)sizeof(uint32_t));
  });
  if (e != cudaSuccess) return e;
  const long long n = (long long)p.n_cand_frames * p.F;
  const long long chunk = (n + kTopcCluster - 1) / kTopcCluster;
  const int in_smem = chunk <= kTopcSmemKeys ? 1 : 0;
  topc_kernel<<<kTopcCluster, kTopcThreads, in_smem ? (size_t)chunk * sizeof(uint32_t) : 0, s>>>(p, in_smem);
  return cudaGetLastError();
}

}  // namespace rc
