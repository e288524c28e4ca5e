// K6a: Deep-Forcing token scores for sm_100a.
//
// rCM guide, strategy 4: every cached token is scored by the attention its
// key receives from the current chunk's queries. Reading S1: score[j] = sum
// over heads and queries of the softmax probability the attention used,
// p = exp(q.k_j / sqrt(d) - LSE), with the attention's final LSE. This is a
// second Q K^T pass over the history tiles only (sink and current chunk are
// not candidates, and every query sees every candidate).
//
// The LSE is known before the pass starts, so no row maximum is needed and
// the pass is computed transposed: S^T = K Q^T puts one key per TMEM lane
// (M = 128 keys, N = 128 queries), and each thread turns its key's row of
// S^T into exp2(s c - lse2[q]) and sums it over the queries in registers.
// There is no P tile, no column-sum GEMM and no exchange between warps.
//
// Persistent CTAs walk (head, query pair, KV tile) items in equal contiguous
// ranges; the sums go to global memory with atomics, so a pair cut between
// CTAs needs no merge. Per CTA, two 128-query tiles share each K tile:
//   warps 0-7 / 8-15  exponentials of Q0 / Q1: warp w reads TMEM lane quarter
//                     w % 4 (32 keys) and query half (w / 4) % 2 (64 columns),
//                     so four such warps share each SM sub-partition's exp2
//                     unit
//   warp 16           TMA producer (Q pair per job, K tiles in a 3-stage ring)
//   warps 17 / 18     one MMA issuer per query tile (warp 17 also owns TMEM)
// TMEM: two S^T buffers per query tile, S_g,b at columns [(2g + b) 128, +128):
// the issuer computes tile t + 1 into one while the exponential warps read
// tile t from the other. Each job's lse2 (log2 units, +inf past the last
// query) is staged in shared memory by the exponential warps, one buffer per
// job parity.
// Bounded waits (RC_ETIMEOUT in the status word), no trap.
#include "attn_common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rc {

namespace {

constexpr int kSoftmaxWarps = 16;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;  // and 18
constexpr int kScoreThreads = 19 * 32;
constexpr int kKStages = 3;

template <int D>
struct ScoreLayout {
  static constexpr int kSub = D / 64;
  static constexpr uint32_t kTile = kSubTileBytes * kSub;  // Q or K tile: 128 rows x D
  static constexpr uint32_t kQ = 0;                         // Q0, Q1
  static constexpr uint32_t kK = 2 * kTile;                 // kKStages stages
  static constexpr uint32_t kBytes = kK + kKStages * kTile;
  static constexpr uint32_t kDynSmem = kBytes + 1024;
};

struct ScoreJob {
  int h, q0, kv_lo, kv_hi;
};

// Equal contiguous ranges of the W = H * NP * T work items (head, pair, tile).
struct ScoreScheduler {
  const ScoreParams* p;
  long long pos, end;
  __device__ void init(const ScoreParams& prm) {
    p = &prm;
    const long long W = (long long)prm.H * prm.n_pairs * prm.tiles;
    pos = (long long)blockIdx.x * W / gridDim.x;
    end = (long long)(blockIdx.x + 1) * W / gridDim.x;
  }
  // Both query tiles of a pair always run: rows past Nq load as zeros and
  // get lse2 = +inf, so their terms are 0 (at most 2^-126 where the
  // exponential runs on the FMA pipe).
  __device__ bool next(ScoreJob& j) {
    if (pos >= end) return false;
    const long long unit = pos / p->tiles;
    const int off = (int)(pos - unit * p->tiles);
    const int len = (int)min((long long)(p->tiles - off), end - pos);
    pos += len;
    j.h = (int)(unit / p->n_pairs);
    j.q0 = (int)(unit % p->n_pairs) * 2 * kTileRows;
    j.kv_lo = off;
    j.kv_hi = off + len;
    return true;
  }
};

// 2^x for a pair of lanes on the FMA pipe, for the share of the exponentials
// the exp2 unit (16 per clock per SM, the binding pipe of this kernel) should
// not take: x = n + f with n the nearest integer (added to the exponent bits)
// and 2^f on [-1/2, 1/2] by a quartic: the minimax fit of the relative error
// of 2^f (Remez exchange in fp64, degree 4, equioscillating error 2.59e-6),
// each coefficient rounded to fp32 (max relative error 2.7e-6 in fp32
// arithmetic; tests/test_kernel_math.py re-derives the coefficients and
// checks the bound). Every step is a packed f32x2 instruction: as scalar
// code the nine dependent steps stall the few warps a sub-partition holds.
// x is clamped at -126, so -inf (a query past the chunk) gives at most
// 2^-126 instead of 0.
__device__ __forceinline__ float2 exp2_quartic2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = ptx::fadd2(x, make_float2(12582912.f, 12582912.f));  // 1.5 * 2^23: round(x) in the low bits
  const float2 n = ptx::fadd2(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = ptx::ffma2(n, make_float2(-1.f, -1.f), x);
  float2 q = ptx::ffma2(make_float2(0.009570101276040077f, 0.009570101276040077f), f,
                        make_float2(0.05591785907745361f, 0.05591785907745361f));
  q = ptx::ffma2(q, f, make_float2(0.240247443318367f, 0.240247443318367f));
  q = ptx::ffma2(q, f, make_float2(0.6931217908859253f, 0.6931217908859253f));
  q = ptx::ffma2(q, f, make_float2(0.9999992847442627f, 0.9999992847442627f));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

// Sum over 32 queries of exp2(s c - lse2): r holds S^T columns (queries)
// q .. q + 31 of this thread's key, nlse the matching -lse2 values. The scale
// and the sums are packed f32x2 instructions; two pairs in eight take
// exp2_quartic2 (measured on B200: the exponential phase alone 20 % shorter
// than with the exp2 unit only, where one scalar exponential in eight on the
// FMA pipe gained 6 %).
__device__ __forceinline__ float exp_sum32(const uint32_t (&r)[32], const float* nlse, float c) {
  const float2 c2 = make_float2(c, c);
  float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    const float4 l = *reinterpret_cast<const float4*>(nlse + k);
    const float2 x0 = ptx::ffma2(make_float2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), c2,
                                 make_float2(l.x, l.y));
    const float2 x1 = ptx::ffma2(make_float2(__uint_as_float(r[k + 2]), __uint_as_float(r[k + 3])), c2,
                                 make_float2(l.z, l.w));
    float2 e0, e1;
    if ((k & 15) == 0) {  // pairs 8 i and 8 i + 1 of every eight
      e0 = exp2_quartic2(x0);
      e1 = exp2_quartic2(x1);
    } else {
      e0 = make_float2(ptx::ex2(x0.x), ptx::ex2(x0.y));
      e1 = make_float2(ptx::ex2(x1.x), ptx::ex2(x1.y));
    }
    a0 = ptx::fadd2(a0, e0);
    a1 = ptx::fadd2(a1, e1);
  }
  return (a0.x + a0.y) + (a1.x + a1.y);
}

template <int D>
__global__ void __launch_bounds__(kScoreThreads, 1) score_kernel(const __grid_constant__ ScoreParams p) {
  using L = ScoreLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_qe, bar_kf[kKStages], bar_ke[kKStages], bar_s[2][2], bar_sfree[2][2],
      bar_lse[2], bar_fin[2];
  __shared__ __align__(16) float s_lse[2][2][kTileRows];  // -lse2: [job parity][query tile][query]
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base_u32 = (ptx::smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - ptx::smem_u32(smem_raw));

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar_q, 1);
    ptx::mbar_init(&bar_qe, 2);
    for (int i = 0; i < kKStages; ++i) {
      ptx::mbar_init(&bar_kf[i], 1);
      ptx::mbar_init(&bar_ke[i], 2);
    }
    for (int g = 0; g < 2; ++g) {
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(&bar_s[g][b], 1);
        ptx::mbar_init(&bar_sfree[g][b], 256);
      }
      ptx::mbar_init(&bar_lse[g], 256);
      ptx::mbar_init(&bar_fin[g], 1);
    }
    abort_sh = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(&tmem_base_sh, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort = &abort_sh;
  int dummy_abort = 0;
  volatile int* noabort = reinterpret_cast<volatile int*>(&dummy_abort);
  ScoreScheduler sc;
  sc.init(p);
  ScoreJob jb;

  if (warp == kProducerWarp && lane == 0) {
    // ---------------------------------------------------------- producer
    int nq = 0, g = 0, nk[kKStages] = {0, 0, 0};
    bool ok = true;
    while (ok && sc.next(jb)) {
      if (nq > 0 && !ptx::mbar_wait(&bar_qe, (nq - 1) & 1, abort, p.status, RC_ETIMEOUT)) break;
      ptx::mbar_arrive_expect_tx(&bar_q, 2 * L::kTile);
      for (int i = 0; i < 2; ++i)
        for (int k = 0; k < L::kSub; ++k)
          ptx::tma_load_3d(&p.tm_q, &bar_q, base + L::kQ + i * L::kTile + k * kSubTileBytes, 64 * k,
                           jb.q0 + i * kTileRows, jb.h);
      ++nq;
      TileWalker wk{p.seg, p.n_segs, 0x7fffffff};
      wk.seek(jb.kv_lo);
      Tile t;
      for (int j = jb.kv_lo; j < jb.kv_hi && wk.next(t); ++j, ++g) {
        const int st = g % kKStages, use = g / kKStages;
        if (use > 0 && !ptx::mbar_wait(&bar_ke[st], (use - 1) & 1, abort, p.status, RC_ETIMEOUT)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(&bar_kf[st], L::kTile);
        for (int k = 0; k < L::kSub; ++k)
          ptx::tma_load_3d(&p.tm_k, &bar_kf[st], base + L::kK + st * L::kTile + k * kSubTileBytes, 0, t.tok,
                           jb.h * L::kSub + k);
        nk[st]++;
      }
    }
    // copies still in flight complete before the CTA leaves
    if (nq) ptx::mbar_wait(&bar_q, (nq - 1) & 1, noabort, p.status, RC_ETIMEOUT);
    for (int st = 0; st < kKStages; ++st)
      if (nk[st]) ptx::mbar_wait(&bar_kf[st], (nk[st] - 1) & 1, noabort, p.status, RC_ETIMEOUT);
  } else if ((warp == kMmaWarp || warp == kMmaWarp + 1) && lane == 0) {
    // ---------------------------------------------------------- MMA issuers
    // one thread per query tile, so the two groups' pipelines never wait on
    // each other; K stages and the Q pair are released by both (count 2).
    // S^T(t) = K(t) Q_g^T goes to buffer t & 1 once the exponential warps
    // have read tile t - 2 from it.
    const int g = warp - kMmaWarp;
    constexpr uint32_t idesc = ptx::idesc_bf16(128, 128, 0, 0);
    const uint32_t sQg = base_u32 + L::kQ + g * L::kTile;
    const uint32_t tSg = tmem + g * 256;
    int nq = 0, gk = 0, t = 0;  // Q pairs waited for, K tiles consumed, S tiles issued
    bool ok = true;
    while (ok && sc.next(jb)) {
      if (!ptx::mbar_wait(&bar_q, nq & 1, abort, p.status, RC_ETIMEOUT)) break;
      ++nq;
      const int n = jb.kv_hi - jb.kv_lo;
      for (int j = 0; j < n; ++j, ++gk, ++t) {
        const int st = gk % kKStages, b = t & 1;
        if (!ptx::mbar_wait(&bar_kf[st], (gk / kKStages) & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
        if (t >= 2 && !ptx::mbar_wait(&bar_sfree[g][b], ((t >> 1) - 1) & 1, abort, p.status, RC_ETIMEOUT)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t sK = base_u32 + L::kK + st * L::kTile;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kSubTileBytes + (ks & 3) * 32;
          ptx::mma_ss(tSg + b * 128, ptx::sdesc_sw128(sK + off, 16, 1024), ptx::sdesc_sw128(sQg + off, 16, 1024),
                      idesc, ks > 0);
        }
        ptx::mma_commit(&bar_s[g][b]);
        ptx::mma_commit(&bar_ke[st]);
        if (j + 1 == n) ptx::mma_commit(&bar_qe);
      }
    }
    ptx::mma_commit(&bar_fin[g]);
    ptx::mbar_wait(&bar_fin[g], 0, noabort, p.status, RC_ETIMEOUT);
  } else if (warp < kSoftmaxWarps) {
    // ---------------------------------------------------------- exponentials
    const int grp = warp >> 3;
    const int ch = (warp >> 2) & 1;
    const int wq = warp & 3;
    const int key = wq * 32 + lane;  // TMEM lane = key within the tile
    const uint32_t tSg = tmem + (static_cast<uint32_t>(wq * 32) << 16) + grp * 256 + ch * 64;
    const float c = p.scale_log2;
    int gs = 0;  // this group's tiles read so far
    int nj = 0;  // jobs so far (lse2 buffer parity)
    bool ok = true;
    while (ok && sc.next(jb)) {
      if (*abort) break;
      // this job's -lse2, written by the first column half (one query each)
      float* lse = s_lse[nj & 1][grp];
      if (ch == 0) {
        const int qtok = jb.q0 + grp * kTileRows + key;
        lse[key] = qtok < p.Nq ? -(p.lse[(size_t)jb.h * p.Nq + qtok] * 1.4426950408889634f) : -INFINITY;
      }
      ptx::mbar_arrive(&bar_lse[grp]);
      if (!ptx::mbar_wait(&bar_lse[grp], nj & 1, abort, p.status, RC_ETIMEOUT)) break;
      ++nj;
      const float* lse_h = lse + ch * 64;
      TileWalker wk{p.seg, p.n_segs, 0x7fffffff};
      wk.seek(jb.kv_lo);
      Tile t;
      for (int j = jb.kv_lo; j < jb.kv_hi && wk.next(t); ++j, ++gs) {
        const int b = gs & 1;
        if (!ptx::mbar_wait(&bar_s[grp][b], (gs >> 1) & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t tS = tSg + b * 128;
        float sum;
        {
          uint32_t r[32];
          ptx::tmem_ld32(tS, r);
          ptx::tmem_ld_wait();
          sum = exp_sum32(r, lse_h, c);
        }
        {
          uint32_t r[32];
          ptx::tmem_ld32(tS + 32, r);
          ptx::tmem_ld_wait();
          ptx::tc_fence_before();
          ptx::mbar_arrive(&bar_sfree[grp][b]);  // S^T read: the next-but-one tile may overwrite it
          sum += exp_sum32(r, lse_h + 32, c);
        }
        if (key < t.nvalid) atomicAdd(p.score_phys + t.tok + key, sum);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_scores_d(const ScoreParams& p, cudaStream_t s) {
  using L = ScoreLayout<D>;
  static PerDevice attr_set;
  int done = 0;
  cudaError_t e = attr_set.get(&done, [](int, int* x) {
    *x = 1;
    return cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kDynSmem);
  });
  if (e != cudaSuccess) return e;
  score_kernel<D><<<p.n_ctas, kScoreThreads, L::kDynSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scores(const ScoreParams& p, int head_dim, cudaStream_t s) {
  if (p.Nq <= 0 || p.n_segs == 0 || p.tiles == 0 || p.n_ctas <= 0) return cudaSuccess;
  return head_dim == 64 ? launch_scores_d<64>(p, s) : launch_scores_d<128>(p, s);
}

}  // namespace rc
