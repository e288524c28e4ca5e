// K6a: Deep-Forcing token scores for sm_100a.
//
// rCM guide, strategy 4: every cached token is scored by the attention its
// key receives from the current chunk's queries. Reading S1: score[j] = sum
// over heads and queries of the softmax probability the attention used,
// p = exp(q.k_j / sqrt(d) - LSE), with the attention's final LSE. This is a
// second Q K^T pass over the history tiles only (sink and current chunk are
// not candidates, and every query sees every candidate).
//
// Persistent CTAs walk (head, query pair, KV tile) items in equal contiguous
// ranges; column sums go to global memory with atomics, so a pair cut
// between CTAs needs no merge. Per CTA, two 128-query tiles share each K tile:
//   warps 0-7 / 8-15  softmax of Q0 / Q1: P = 2^(s c - lse2) as bf16 into
//                     shared memory ([query][key], 128-byte swizzle); each
//                     warp takes 32 rows x 64 keys, so four softmax warps
//                     share each SM sub-partition's exp2 unit
//   warp 16           TMA producer (Q pair per job, K tiles in a 2-stage ring)
//   warps 17 / 18     one MMA issuer per query tile (warp 17 also owns TMEM)
// The column sum itself runs on the tensor core: D'_g = P_g^T 1 with P_g^T
// read MN-major from shared memory (M = 128 keys, N = 16, K = 128 queries);
// lane j of D'_g holds key j's sum over the tile's queries, which group g
// reads one tile later (its two column halves in turn) and adds to the score
// buffer.
// TMEM: S0 [0,128), S1 [128,256), D'_0 [256,288), D'_1 [288,320) (2 buffers each).
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
constexpr uint32_t kPTileBytes = 128 * 128 * 2;  // P: 128 queries x 128 keys bf16
constexpr uint32_t kOnesBytes = 16 * 128 * 2;    // B = ones: 16 x 128 bf16

template <int D>
struct ScoreLayout {
  static constexpr int kSub = D / 64;
  static constexpr uint32_t kTile = kSubTileBytes * kSub;  // Q or K tile: 128 rows x D
  static constexpr uint32_t kQ = 0;                         // Q0, Q1
  static constexpr uint32_t kK = 2 * kTile;                 // 2 stages
  static constexpr uint32_t kP = 4 * kTile;                 // P0, P1
  static constexpr uint32_t kOnes = kP + 2 * kPTileBytes;
  static constexpr uint32_t kBytes = kOnes + kOnesBytes;
  static constexpr uint32_t kDynSmem = kBytes + 1024;
};

struct ScoreJob {
  int h, q0, kv_lo, kv_hi;
  bool has1;
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
    // both tiles always: rows past Nq load as zeros and get lse2 = +inf, so
    // their P is exactly 0 (keeps the two issuers' barrier phases in step)
    j.has1 = true;
    return true;
  }
};

// P = 2^(s c - lse2) of 32 keys of one row (S columns c0 .. c0 + 31 of this
// warp's half) as bf16, into the row's four 16-byte chunks c0/8 .. c0/8 + 3 of
// the 128-byte-swizzled sub-tile. Keys at or past lim (ragged tile end) get 0.
template <bool kCheck>
__device__ __forceinline__ void exp_store(const uint32_t (&r)[32], int c0, int lim, float c, float lse2,
                                          uint8_t* sProw, int row) {
  uint32_t pk[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float a = ptx::ex2(fmaf(__uint_as_float(r[2 * k]), c, -lse2));
    float b = ptx::ex2(fmaf(__uint_as_float(r[2 * k + 1]), c, -lse2));
    if (kCheck) {
      if (c0 + 2 * k >= lim) a = 0.f;
      if (c0 + 2 * k + 1 >= lim) b = 0.f;
    }
    pk[k] = ptx::pack_bf16x2(a, b);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(sProw + (((c0 / 8 + q) ^ (row & 7)) << 4)) =
        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
}

template <int D>
__global__ void __launch_bounds__(kScoreThreads, 1) score_kernel(const __grid_constant__ ScoreParams p) {
  using L = ScoreLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_qe, bar_kf[2], bar_ke[2], bar_s[2], bar_sfree[2], bar_p[2], bar_pfree[2],
      bar_dfull[2][2], bar_dfree[2][2], bar_fin[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base_u32 = (ptx::smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - ptx::smem_u32(smem_raw));

  // B operand of the column sum: all ones (layout-free)
  for (uint32_t i = threadIdx.x; i < kOnesBytes / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(base + L::kOnes)[i] = 0x3F803F80u;
  ptx::fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar_q, 1);
    ptx::mbar_init(&bar_qe, 2);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bar_kf[i], 1);
      ptx::mbar_init(&bar_ke[i], 2);
      ptx::mbar_init(&bar_s[i], 1);
      ptx::mbar_init(&bar_sfree[i], 256);
      ptx::mbar_init(&bar_p[i], 256);
      ptx::mbar_init(&bar_pfree[i], 1);
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(&bar_dfull[i][b], 1);
        ptx::mbar_init(&bar_dfree[i][b], 128);
      }
      ptx::mbar_init(&bar_fin[i], 1);
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
    int nq = 0, g = 0, nk[2] = {0, 0};
    bool ok = true;
    while (ok && sc.next(jb)) {
      if (nq > 0 && !ptx::mbar_wait(&bar_qe, (nq - 1) & 1, abort, p.status, RC_ETIMEOUT)) break;
      ptx::mbar_arrive_expect_tx(&bar_q, (jb.has1 ? 2 : 1) * L::kTile);
      for (int i = 0; i < (jb.has1 ? 2 : 1); ++i)
        for (int k = 0; k < L::kSub; ++k)
          ptx::tma_load_3d(&p.tm_q, &bar_q, base + L::kQ + i * L::kTile + k * kSubTileBytes, 64 * k,
                           jb.q0 + i * kTileRows, jb.h);
      ++nq;
      TileWalker wk{p.seg, p.n_segs, 0x7fffffff};
      wk.seek(jb.kv_lo);
      Tile t;
      for (int j = jb.kv_lo; j < jb.kv_hi && wk.next(t); ++j, ++g) {
        const int st = g & 1;
        if (g >= 2 && !ptx::mbar_wait(&bar_ke[st], ((g >> 1) - 1) & 1, abort, p.status, RC_ETIMEOUT)) {
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
    if (nq) ptx::mbar_wait(&bar_q, (nq - 1) & 1, noabort, p.status, RC_ETIMEOUT);
    for (int st = 0; st < 2; ++st)
      if (nk[st]) ptx::mbar_wait(&bar_kf[st], (nk[st] - 1) & 1, noabort, p.status, RC_ETIMEOUT);
  } else if ((warp == kMmaWarp || warp == kMmaWarp + 1) && lane == 0) {
    // ---------------------------------------------------------- MMA issuers
    // one thread per query tile, so the two groups' pipelines never wait on
    // each other; K stages and the Q pair are released by both (count 2)
    const int g = warp - kMmaWarp;
    constexpr uint32_t idesc_s = ptx::idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t idesc_c = ptx::idesc_bf16(128, 16, 1, 0);  // A = P^T (MN-major), B = ones (K-major)
    const uint32_t sQg = base_u32 + L::kQ + g * L::kTile;
    const uint32_t sP = base_u32 + L::kP + g * kPTileBytes;
    const uint32_t sOnes = base_u32 + L::kOnes;
    auto issue_s = [&](int st) {
      const uint32_t sK = base_u32 + L::kK + st * L::kTile;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = (ks >> 2) * kSubTileBytes + (ks & 3) * 32;
        ptx::mma_ss(tmem + g * 128, ptx::sdesc_sw128(sQg + off, 16, 1024), ptx::sdesc_sw128(sK + off, 16, 1024),
                    idesc_s, ks > 0);
      }
      ptx::mma_commit(&bar_s[g]);
    };
    int nq = 0, gk = 0, gt = 0, gd = 0;
    bool ok = true;
    while (ok && sc.next(jb)) {
      const int n = jb.kv_hi - jb.kv_lo;
      if (!ptx::mbar_wait(&bar_q, nq & 1, abort, p.status, RC_ETIMEOUT)) break;
      ++nq;
      if (!ptx::mbar_wait(&bar_kf[gk & 1], (gk >> 1) & 1, abort, p.status, RC_ETIMEOUT)) break;
      if (gt > 0 && !ptx::mbar_wait(&bar_sfree[g], (gt - 1) & 1, abort, p.status, RC_ETIMEOUT)) break;
      ptx::tc_fence_after();
      issue_s(gk & 1);
      ptx::mma_commit(&bar_ke[gk & 1]);
      if (n == 1) ptx::mma_commit(&bar_qe);
      for (int j = 0; j < n; ++j, ++gk, ++gt, ++gd) {
        if (j + 1 < n) {  // S of the next tile once this one's S has been read
          const int st1 = (gk + 1) & 1;
          if (!ptx::mbar_wait(&bar_kf[st1], ((gk + 1) >> 1) & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
          if (!ptx::mbar_wait(&bar_sfree[g], gt & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
          ptx::tc_fence_after();
          issue_s(st1);
          ptx::mma_commit(&bar_ke[st1]);
          if (j + 2 == n) ptx::mma_commit(&bar_qe);
        }
        const int db = gd & 1;
        if (gd >= 2 && !ptx::mbar_wait(&bar_dfree[g][db], ((gd >> 1) - 1) & 1, abort, p.status, RC_ETIMEOUT)) {
          ok = false;
          break;
        }
        if (!ptx::mbar_wait(&bar_p[g], gt & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
        ptx::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kTileRows / 16; ++ks)
          ptx::mma_ss(tmem + 256 + g * 32 + db * 16, ptx::sdesc_sw128(sP + ks * 2048, kSubTileBytes, 1024),
                      ptx::sdesc_sw128(sOnes + (ks >> 2) * 2048 + (ks & 3) * 32, 16, 1024), idesc_c, ks > 0);
        ptx::mma_commit(&bar_pfree[g]);
        ptx::mma_commit(&bar_dfull[g][db]);
      }
    }
    ptx::mma_commit(&bar_fin[g]);
    ptx::mbar_wait(&bar_fin[g], 0, noabort, p.status, RC_ETIMEOUT);
  } else if (warp < kSoftmaxWarps) {
    // ---------------------------------------------------------- softmax
    // group g = warp / 8 owns query tile g; within it warp w reads TMEM lane
    // quarter w % 4 (rows) and column half (w / 4) % 2 (keys [64 ch, 64 ch + 64))
    const int grp = warp >> 3;
    const int ch = (warp >> 2) & 1;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + grp * 128 + ch * 64;
    uint8_t* sProw = base + L::kP + grp * kPTileBytes + ch * kSubTileBytes + row * 128;
    const float c = p.scale_log2;
    int gs = 0;            // this group's tiles (phases of s / sfree / p / pfree)
    int gd = 0;            // D' sums of this group (drained by the two column halves in turn)
    int prev_tok = 0, prev_nvalid = 0;
    bool have_prev = false;
    // add the previous tile's key sums (lane j of this group's D' = key j) to the scores
    auto drain = [&]() -> bool {
      if (!have_prev) return true;
      have_prev = false;
      const int db = gd & 1;  // buffer db is drained by column half db
      const uint32_t phase = (gd >> 1) & 1;
      ++gd;
      if (db != ch) return true;
      if (!ptx::mbar_wait(&bar_dfull[grp][db], phase, abort, p.status, RC_ETIMEOUT)) return false;
      ptx::tc_fence_after();
      const uint32_t v = ptx::tmem_ld1(tmem + lane_off + 256 + grp * 32 + db * 16);
      ptx::tmem_ld_wait();
      if (row < prev_nvalid) atomicAdd(p.score_phys + prev_tok + row, __uint_as_float(v));
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bar_dfree[grp][db]);
      return true;
    };
    bool ok = true;
    while (ok && sc.next(jb)) {
      if (*abort) break;
      const int qtok = jb.q0 + grp * kTileRows + row;
      const float lse2 = qtok < p.Nq ? p.lse[(size_t)jb.h * p.Nq + qtok] * 1.4426950408889634f : INFINITY;
      TileWalker wk{p.seg, p.n_segs, 0x7fffffff};
      wk.seek(jb.kv_lo);
      Tile t;
      for (int j = jb.kv_lo; j < jb.kv_hi && wk.next(t); ++j) {
        if (!ptx::mbar_wait(&bar_s[grp], gs & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
        ptx::tc_fence_after();
        // P smem of the previous tile must have been read by its column-sum MMA
        if (gs > 0 && !ptx::mbar_wait(&bar_pfree[grp], (gs - 1) & 1, abort, p.status, RC_ETIMEOUT)) {
          ok = false;
          break;
        }
        const int lim = t.nvalid - ch * 64;  // valid keys in this half
        {
          uint32_t r[32];
          ptx::tmem_ld32(tS, r);
          ptx::tmem_ld_wait();
          if (lim >= 64) exp_store<false>(r, 0, lim, c, lse2, sProw, row);
          else exp_store<true>(r, 0, lim, c, lse2, sProw, row);
        }
        {
          uint32_t r[32];
          ptx::tmem_ld32(tS + 32, r);
          ptx::tmem_ld_wait();
          ptx::tc_fence_before();
          ptx::mbar_arrive(&bar_sfree[grp]);  // S read: the MMA may overwrite it
          if (lim >= 64) exp_store<false>(r, 32, lim, c, lse2, sProw, row);
          else exp_store<true>(r, 32, lim, c, lse2, sProw, row);
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&bar_p[grp]);
        ++gs;
        if (!drain()) { ok = false; break; }
        prev_tok = t.tok;
        prev_nvalid = t.nvalid;
        have_prev = true;
      }
    }
    if (ok) drain();
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
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(score_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::kDynSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  score_kernel<D><<<p.n_ctas, kScoreThreads, L::kDynSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scores(const ScoreParams& p, int head_dim, cudaStream_t s) {
  if (p.Nq <= 0 || p.n_segs == 0 || p.tiles == 0 || p.n_ctas <= 0) return cudaSuccess;
  return head_dim == 64 ? launch_scores_d<64>(p, s) : launch_scores_d<128>(p, s);
}

}  // namespace rc
