// K4: chunk attention for sm_100a (tcgen05 + TMEM + TMA).
//
// O = softmax(Q K^T / sqrt(d) + mask) V for the current chunk's queries over
// every valid slot of the ring buffer (LingBot explainer, sliding-window
// section: the query reads the window up to local_end; Causal-Forcing
// walkthrough, section 3: only the current block's queries are computed).
// The mask acts only inside the current chunk (reading M1).
//
// One CTA = two 128-query tiles (Q0, Q1) of one head sharing every K/V tile.
//   warps 0-7   softmax of Q0 and epilogue: 32 query rows (TMEM lanes) x
//               64 keys per warp, so four softmax warps share each SM
//               sub-partition's exp2 unit
//   warps 8-15  softmax of Q1, epilogue
//   warp 16     TMA producer: Q0/Q1 once, K and V into separate 2-stage rings
//   warp 17     TMEM allocator; one thread issues every tcgen05.mma
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d), O1 [384,384+d).
// P_i (packed bf16) overwrites columns [0,32) and [64,96) of S_i, each key
// half in the half of S its softmax warp read, and is the A operand of
// O_i += P_i V.
//
// MMA issue order per KV tile j (FA-style ping-pong):
//   PV0(j), S0(j+1), PV1(j), S1(j+1)
// so while one softmax group turns S into P the tensor core runs the other
// group's two GEMMs. S0(j+1) may overwrite P0(j) because tcgen05.mma ops of
// one thread execute in issue order. K stage j is released after S1(j), V
// stage j after PV1(j), so the next loads start early.
//
// Online softmax keeps a stale row maximum and rescales O only when the
// maximum grows by more than 2^8 (in exp2 units); numerator and denominator
// carry the same factor, so the result is unchanged and P stays below 256.
// A rescale waits for the group's previous PV; otherwise the softmax never
// waits on the PV path.
//
// Every wait is bounded (2 s) and reports RC_ETIMEOUT through the status
// word; no trap.
#include "attn_common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rc {

namespace {

// 2^x for a pair of lanes on the FMA pipe, in packed f32x2 steps: n =
// round(x) by the 1.5 * 2^23 shift, f = x - n in [-1/2, 1/2], 2^f by a cubic,
// n added to the exponent field. The cubic's coefficients are the minimax fit
// of the relative error on [-1/2, 1/2] (Remez exchange in fp64, each rounded
// to fp32): relative error within 7.5e-5, below the 2^-9 of the bf16 P it
// feeds. x is clamped at -126 so the exponent field cannot wrap; below that
// the result is at most 2^-126, as the SFU's flush-to-zero gives 0.
__device__ __forceinline__ float2 exp2_cubic2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = ptx::fadd2(x, make_float2(12582912.f, 12582912.f));
  const float2 n = ptx::fadd2(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = ptx::ffma2(n, make_float2(-1.f, -1.f), x);
  float2 q = ptx::ffma2(make_float2(5.517166853e-02f, 5.517166853e-02f), f,
                        make_float2(2.426111251e-01f, 2.426111251e-01f));
  q = ptx::ffma2(q, f, make_float2(6.932609677e-01f, 6.932609677e-01f));
  q = ptx::ffma2(q, f, make_float2(9.999280572e-01f, 9.999280572e-01f));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}
// pairs k of a 16-pair chunk with (k % 8) < kCubicPairs take exp2_cubic2;
// the rest the SFU's ex2 (16 per clock per SM, the bound of the exponential
// phase when it runs alone)
constexpr int kCubicPairs = 2;

constexpr int kSoftmaxWarps = 16;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kFwdThreads = 18 * 32;
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct FwdLayout {
  static constexpr int kSub = D / 64;
  static constexpr uint32_t kTile = kSubTileBytes * kSub;
  static constexpr uint32_t kQ = 0;              // Q0, Q1
  static constexpr uint32_t kK = 2 * kTile;      // 2 stages
  static constexpr uint32_t kV = 4 * kTile;      // 2 stages
  static constexpr uint32_t kBytes = 6 * kTile;
  static constexpr uint32_t kDynSmem = kBytes + 1024;
};

// One unit of work: query pair (rows q0 .. q0+255) of head h over the KV
// tiles [kv_lo, kv_hi) of the pair's tile walk. slot >= 0: the job covers
// part of its pair's tiles and leaves (O / l, log2-sum-exp) in the partial
// workspace for the combine kernel; slot < 0: it writes the output.
struct Job {
  int h, q0, kv_lo, kv_hi, slot, rq_hi;
  bool has1;
};

__device__ __forceinline__ int pair_rq_hi(const AttnParams& p, int pair) {
  const int q_last = min((pair + 1) * 2 * kTileRows, p.Nq) - 1;
  return (q_last / p.F) / p.mask_block;
}

// Persistent schedule over units u = h * NP + pair (head-major), each with
// T(pair) KV tiles (pair_prefix). Rounds first: CTA c takes whole units
// c, c + G, ... for R = U / G rounds; the G CTAs of a round all start at KV
// tile 0 together, so the query pairs of a head read each K/V tile about
// when the others do and it comes from DRAM once. The U mod G units left
// over (the last heads) are then cut stream-K style: their tiles, in (unit,
// tile) order, are split into G ranges, one per CTA, sized by the host so
// that every CTA's round tiles plus range tiles come out equal (units differ
// in length under the in-chunk mask); a unit cut between CTAs leaves partial
// rows for the combine kernel. Their K/V spans only a few heads, so it stays
// in L2 whatever the offsets.
// Without a partial workspace the grid has one CTA per unit.
struct Scheduler {
  const AttnParams* p;
  int NP, T_head, c, G, rounds, r;
  long long pos, end, base;
  bool split, first_sk;

  __device__ void init(const AttnParams& prm) {
    p = &prm;
    NP = prm.n_pairs;
    c = blockIdx.x;
    G = gridDim.x;
    split = prm.part_o != nullptr;
    T_head = split ? prm.pair_prefix[NP] : 0;  // the prefix table is filled for persistent launches
    first_sk = true;
    r = 0;
    const long long U = (long long)NP * prm.H;
    rounds = split ? (int)(U / G) : 1;
    pos = end = 0;
    if (split) {
      pos = prm.sk_start[c];
      end = prm.sk_start[c + 1];
    }
  }

  __device__ void fill(Job& j, int h, int pair, int off, int len, int T_u, int slot) const {
    j.h = h;
    j.q0 = pair * 2 * kTileRows;
    j.kv_lo = off;
    j.kv_hi = off + len;
    j.rq_hi = pair_rq_hi(*p, pair);
    j.has1 = j.q0 + kTileRows < p->Nq;
    j.slot = (off > 0 || off + len < T_u) ? slot : -1;
  }

  __device__ bool next(Job& j) {
    if (r < rounds) {
      const int u = c + r * G;
      ++r;
      const int pair = u % NP;
      const int T_u = split ? p->pair_prefix[pair + 1] - p->pair_prefix[pair]
                            : count_tiles(p->seg, p->n_segs, pair_rq_hi(*p, pair));
      fill(j, u / NP, pair, 0, T_u, T_u, -1);
      return true;
    }
    if (pos >= end) return false;
    const int h = (int)(pos / T_head);
    const int rem = (int)(pos - (long long)h * T_head);
    int pair = 0;
    while (p->pair_prefix[pair + 1] <= rem) ++pair;
    const int T_u = p->pair_prefix[pair + 1] - p->pair_prefix[pair];
    const int off = rem - p->pair_prefix[pair];
    const int len = (int)min((long long)(T_u - off), end - pos);
    pos += len;
    fill(j, h, pair, off, len, T_u, 2 * c + (first_sk ? 0 : 1));
    first_sk = false;
    return true;
  }
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_qe, bar_kf[2], bar_vf[2], bar_ke[2], bar_ve[2], bar_s[2], bar_p[2], bar_o[2],
      bar_fin, bar_pair[8];
  __shared__ float swap_buf[2][2][2][kTileRows];  // [group][exchange parity][column half][row]
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base_u32 = (ptx::smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - ptx::smem_u32(smem_raw));

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar_q, 1);
    ptx::mbar_init(&bar_qe, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bar_kf[i], 1);
      ptx::mbar_init(&bar_vf[i], 1);
      ptx::mbar_init(&bar_ke[i], 1);
      ptx::mbar_init(&bar_ve[i], 1);
      ptx::mbar_init(&bar_s[i], 1);
      ptx::mbar_init(&bar_p[i], 256);
      ptx::mbar_init(&bar_o[i], 1);
    }
    ptx::mbar_init(&bar_fin, 1);
    for (int i = 0; i < 8; ++i) ptx::mbar_init(&bar_pair[i], 64);
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
  Scheduler sc_mem;
  sc_mem.init(p);
  // the schedule's state lives in local memory (read once per unit), keeping
  // registers for the per-tile work
  Scheduler* volatile sc_ptr = &sc_mem;
  Scheduler& sc = *sc_ptr;
  Job jb;

  if (warp == kProducerWarp && lane == 0) {
    // ---------------------------------------------------------- producer
    ptx::tma_prefetch_desc(&p.tm_q);
    ptx::tma_prefetch_desc(&p.tm_k);
    ptx::tma_prefetch_desc(&p.tm_v);
    int nq = 0, g = 0;
    int nk[2] = {0, 0}, nv[2] = {0, 0};  // loads issued per stage
    // K/V tiles are read by every query pair of their head, whose CTAs walk
    // them at about the same time: keep them in L2; Q is read by one CTA
    const uint64_t pol_q = ptx::l2_policy(false), pol_kv = ptx::l2_policy(true);
    bool ok = true;
    while (ok && sc.next(jb)) {
      if (nq > 0 && !ptx::mbar_wait(&bar_qe, (nq - 1) & 1, abort, p.status, RC_ETIMEOUT)) break;
      ptx::mbar_arrive_expect_tx(&bar_q, (jb.has1 ? 2 : 1) * L::kTile);
      for (int i = 0; i < (jb.has1 ? 2 : 1); ++i)
        for (int j = 0; j < L::kSub; ++j)
          ptx::tma_load_3d_hint(&p.tm_q, &bar_q, base + L::kQ + i * L::kTile + j * kSubTileBytes, 64 * j,
                                jb.q0 + i * kTileRows, jb.h, pol_q);
      ++nq;
      TileWalker wk{p.seg, p.n_segs, jb.rq_hi};
      wk.seek(jb.kv_lo);
      Tile t;
      for (int j = jb.kv_lo; j < jb.kv_hi && wk.next(t); ++j, ++g) {
        const int st = g & 1;
        const uint32_t free_par = ((g >> 1) - 1) & 1;
        if (g >= 2 && !ptx::mbar_wait(&bar_ke[st], free_par, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
        ptx::mbar_arrive_expect_tx(&bar_kf[st], L::kTile);
        for (int k = 0; k < L::kSub; ++k)
          ptx::tma_load_3d_hint(&p.tm_k, &bar_kf[st], base + L::kK + st * L::kTile + k * kSubTileBytes,
                                0, t.tok, jb.h * L::kSub + k, pol_kv);
        nk[st]++;
        if (g >= 2 && !ptx::mbar_wait(&bar_ve[st], free_par, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
        ptx::mbar_arrive_expect_tx(&bar_vf[st], L::kTile);
        for (int k = 0; k < L::kSub; ++k)
          ptx::tma_load_3d_hint(&p.tm_v, &bar_vf[st], base + L::kV + st * L::kTile + k * kSubTileBytes,
                                0, t.tok, jb.h * L::kSub + k, pol_kv);
        nv[st]++;
      }
    }
    // never leave a copy in flight: wait (bounded, ignoring abort) for the last ones
    if (nq) ptx::mbar_wait(&bar_q, (nq - 1) & 1, noabort, p.status, RC_ETIMEOUT);
    for (int st = 0; st < 2; ++st) {
      if (nk[st]) ptx::mbar_wait(&bar_kf[st], (nk[st] - 1) & 1, noabort, p.status, RC_ETIMEOUT);
      if (nv[st]) ptx::mbar_wait(&bar_vf[st], (nv[st] - 1) & 1, noabort, p.status, RC_ETIMEOUT);
    }
  } else if (warp == kMmaWarp && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc_s = ptx::idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t idesc_o = ptx::idesc_bf16(128, D, 0, 1);
    const uint32_t sQ = base_u32 + L::kQ;
    auto issue_s = [&](int i, int st) {
      const uint32_t sQi = sQ + i * L::kTile;
      const uint32_t sK = base_u32 + L::kK + st * L::kTile;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = (ks >> 2) * kSubTileBytes + (ks & 3) * 32;
        ptx::mma_ss(tmem + i * 128, ptx::sdesc_sw128(sQi + off, 16, 1024), ptx::sdesc_sw128(sK + off, 16, 1024),
                    idesc_s, ks > 0);
      }
      ptx::mma_commit(&bar_s[i]);
    };
    // O_i += P_i V; the commit that tells the epilogue O_i is final goes only
    // after a job's last PV (a softmax that rescales O at tile j has already
    // waited for S_i(j), issued after PV_i(j-1), and tcgen05 work completes in
    // issue order). Each commit costs the issuing thread about 46 cycles,
    // during which the tensor pipe, fed one MMA at a time, has nothing queued.
    auto issue_pv = [&](int i, int st, bool acc, bool last) {
      const uint32_t sV = base_u32 + L::kV + st * L::kTile;
      // P of keys [16 ks, 16 ks + 16): column (ks / 4) * 64 + (ks % 4) * 8 of S_i
#pragma unroll
      for (int ks = 0; ks < kTileRows / 16; ++ks)
        ptx::mma_ts(tmem + 256 + i * 128, tmem + i * 128 + (ks >> 2) * 64 + (ks & 3) * 8,
                    ptx::sdesc_sw128(sV + ks * 2048, kSubTileBytes, 1024), idesc_o, acc || ks > 0);
      if (last) ptx::mma_commit(&bar_o[i]);
    };
    int nq = 0, g = 0, gp[2] = {0, 0};
    bool ok = true;
    while (ok && sc.next(jb)) {
      const int n = jb.kv_hi - jb.kv_lo;
      const bool two = jb.has1;
      if (!ptx::mbar_wait(&bar_q, nq & 1, abort, p.status, RC_ETIMEOUT)) break;
      ++nq;
      if (!ptx::mbar_wait(&bar_kf[g & 1], (g >> 1) & 1, abort, p.status, RC_ETIMEOUT)) break;
      ptx::tc_fence_after();
      issue_s(0, g & 1);
      if (two) issue_s(1, g & 1);
      ptx::mma_commit(&bar_ke[g & 1]);
      if (n == 1) ptx::mma_commit(&bar_qe);
      for (int j = 0; j < n; ++j, ++g) {
        const int st = g & 1, st1 = (g + 1) & 1;
        const bool more = j + 1 < n;
        if (!ptx::mbar_wait(&bar_p[0], gp[0] & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
        if (!ptx::mbar_wait(&bar_vf[st], (g >> 1) & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
        ptx::tc_fence_after();
        issue_pv(0, st, j > 0, !more);
        ++gp[0];
        if (!two) ptx::mma_commit(&bar_ve[st]);
        if (more) {
          if (!ptx::mbar_wait(&bar_kf[st1], ((g + 1) >> 1) & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
          ptx::tc_fence_after();
          issue_s(0, st1);
          if (!two) {
            ptx::mma_commit(&bar_ke[st1]);
            if (j + 2 == n) ptx::mma_commit(&bar_qe);
          }
        }
        if (two) {
          if (!ptx::mbar_wait(&bar_p[1], gp[1] & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
          ptx::tc_fence_after();
          issue_pv(1, st, j > 0, !more);
          ++gp[1];
          ptx::mma_commit(&bar_ve[st]);
          if (more) {
            issue_s(1, st1);
            ptx::mma_commit(&bar_ke[st1]);
            if (j + 2 == n) ptx::mma_commit(&bar_qe);
          }
        }
      }
    }
    ptx::mma_commit(&bar_fin);
    ptx::mbar_wait(&bar_fin, 0, noabort, p.status, RC_ETIMEOUT);
  } else if (warp < kSoftmaxWarps) {
    // ---------------------------------------------------------- softmax
    // group g = warp / 8 owns query tile g. Warp w reads TMEM lane quarter
    // w % 4 (32 query rows) and column half ch = (w / 4) % 2: keys
    // [64 ch, 64 ch + 64) of S and output columns [ch D/2, ch D/2 + D/2) of O.
    // The two warps of a row block (partners) swap their partial row maxima
    // every tile and their partial row sums once per unit through shared
    // memory and a 64-thread mbarrier.
    const int grp = warp >> 3;
    const int ch = (warp >> 2) & 1;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + grp * 128 + ch * 64;
    const uint32_t tO = tmem + lane_off + 256 + grp * 128 + ch * (D / 2);
    uint64_t* pbar = &bar_pair[grp * 4 + wq];
    const float c = p.scale_log2;
    const float thresh = kRescaleLog2 / c;
    int gs = 0;  // this group's tiles so far (phase of bar_s / bar_p)
    int nj = 0;  // this group's jobs so far (phase of bar_o: one commit per job)
    int nx = 0;  // partner exchanges so far (phase of pbar, slot of swap_buf)
    // writes v, returns the partner's value (bounded wait)
    auto swap = [&](float v, float& other) -> bool {
      float(*buf)[128] = swap_buf[grp][nx & 1];
      buf[ch][row] = v;
      ptx::mbar_arrive(pbar);
      if (!ptx::mbar_wait(pbar, nx & 1, abort, p.status, RC_ETIMEOUT)) return false;
      ++nx;
      other = buf[ch ^ 1][row];
      return true;
    };
    while (sc.next(jb)) {
      if (*abort) break;
      if (grp == 1 && !jb.has1) continue;
      const int qtok = jb.q0 + grp * kTileRows + row;
      const int my_rank = (min(qtok, p.Nq - 1) / p.F) / p.mask_block;
      float m = -INFINITY, l = 0.f;  // l: this half's share of the row sum
      TileWalker wk{p.seg, p.n_segs, jb.rq_hi};
      wk.seek(jb.kv_lo);
      Tile t;
      bool ok = true;
      int done = 0;
      for (int j = jb.kv_lo; j < jb.kv_hi && wk.next(t); ++j) {
        if (!ptx::mbar_wait(&bar_s[grp], gs & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
        ptx::tc_fence_after();
        // keys [0, lim) of this row are visible (the whole row or a ragged tail is masked);
        // lim_h of them fall in this warp's half
        const int lim = (t.rank < 0 || t.rank <= my_rank) ? t.nvalid : 0;
        const int lim_h = lim - ch * 64;
        uint32_t ra[32], rb[32];
        ptx::tmem_ld32(tS, ra);
        ptx::tmem_ld32(tS + 32, rb);
        ptx::tmem_ld_wait();
        float mx = -INFINITY;
        if (lim_h >= 64) {
#pragma unroll
          for (int k = 0; k < 32; ++k) mx = ptx::fmax3(mx, __uint_as_float(ra[k]), __uint_as_float(rb[k]));
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            mx = ptx::fmax3(mx, k < lim_h ? __uint_as_float(ra[k]) : -INFINITY,
                            32 + k < lim_h ? __uint_as_float(rb[k]) : -INFINITY);
        }
        float mo;
        if (!swap(mx, mo)) { ok = false; break; }
        const float m_new = ptx::fmax3(m, mx, mo);
        const bool need = m_new > m + thresh;       // also true for the first visible tile
        const bool real = need && m != -INFINITY;   // O already holds weighted values
        if (__any_sync(0xffffffffu, real)) {
          // PV of the previous tile is complete: it was issued before this
          // tile's S, which the wait above saw complete
          const float alpha = real ? ptx::ex2((m - m_new) * c) : 1.f;
#pragma unroll
          for (int cc = 0; cc < D / 64; ++cc) {
            uint32_t o[32];
            ptx::tmem_ld32(tO + cc * 32, o);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            ptx::tmem_st32(tO + cc * 32, o);
          }
          ptx::tmem_st_wait();
          l *= alpha;
        }
        if (need) m = m_new;
        const float mc = (m == -INFINITY ? 0.f : m) * c;
        // P = 2^(s c - m c) as packed bf16 pairs over the first 32 columns of
        // this half of S (already read): keys 64 ch + 2i, 64 ch + 2i + 1 -> column i
        float sum = 0.f;
        auto emit = [&](const uint32_t (&r)[32], int k0) {
          uint32_t pk[16];
          if (lim_h >= 64) {
            const float2 c2 = make_float2(c, c), nmc2 = make_float2(-mc, -mc);
            float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float2 x =
                  ptx::ffma2(make_float2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), c2, nmc2);
              float2 e;
              if ((k & 7) < kCubicPairs) {
                e = exp2_cubic2(x);
              } else {
                e.x = ptx::ex2(x.x);
                e.y = ptx::ex2(x.y);
              }
              s2 = ptx::fadd2(s2, e);
              pk[k] = ptx::pack_bf16x2(e.x, e.y);
            }
            sum += s2.x + s2.y;
          } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float a = k0 + 2 * k < lim_h ? ptx::ex2(fmaf(__uint_as_float(r[2 * k]), c, -mc)) : 0.f;
              const float b =
                  k0 + 2 * k + 1 < lim_h ? ptx::ex2(fmaf(__uint_as_float(r[2 * k + 1]), c, -mc)) : 0.f;
              sum += a + b;
              pk[k] = ptx::pack_bf16x2(a, b);
            }
          }
          ptx::tmem_st16(tS + k0 / 2, pk);
        };
        // S is read again rather than kept in registers across the exchange
        ptx::tmem_ld32(tS, ra);
        ptx::tmem_ld_wait();
        emit(ra, 0);
        ptx::tmem_ld32(tS + 32, rb);
        ptx::tmem_ld_wait();
        emit(rb, 32);
        ptx::tmem_st_wait();
        l += sum;
        ptx::tc_fence_before();
        ptx::mbar_arrive(&bar_p[grp]);
        ++gs;
        ++done;
      }
      // epilogue: O / l, to the output (bf16 [Nq][H][D], lse in natural log)
      // or to this CTA's partial slot (fp32, log2-sum-exp); each warp writes
      // its D/2 columns
      float l_other = 0.f;
      if (ok && !swap(l, l_other)) ok = false;
      const float lt = l + l_other;
      const bool have_o =
          ok && done > 0 && ptx::mbar_wait(&bar_o[grp], nj & 1, abort, p.status, RC_ETIMEOUT);
      if (done > 0) ++nj;
      ptx::tc_fence_after();
      const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
      const float lse2 = lt > 0.f ? m * c + __log2f(lt) : -INFINITY;
      const int prow = grp * kTileRows + row;
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t o[32];
        if (have_o) {
          ptx::tmem_ld32(tO + cc * 32, o);
          ptx::tmem_ld_wait();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        if (qtok >= p.Nq) continue;
        const int col = ch * (D / 2) + cc * 32;
        if (jb.slot < 0) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)qtok * p.H + jb.h) * D + col);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 u;
            u.x = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
            u.y = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
            u.z = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
            u.w = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
            __stcs(dst + v, u);  // streamed: leaves L2 before the next launch has to evict it
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(p.part_o + ((size_t)jb.slot * 2 * kTileRows + prow) * D + col);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv_l, __uint_as_float(o[4 * v + 1]) * inv_l,
                                 __uint_as_float(o[4 * v + 2]) * inv_l, __uint_as_float(o[4 * v + 3]) * inv_l);
        }
      }
      if (qtok < p.Nq && ch == 0) {
        if (jb.slot < 0) {
          if (p.lse) p.lse[(size_t)jb.h * p.Nq + qtok] = lse2 * 0.69314718055994531f;
        } else {
          p.part_lse[(size_t)jb.slot * 2 * kTileRows + prow] = lse2;
        }
      }
      if (!ok) break;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// K5: merges the partial results of the (head, pair) units the stream-K
// schedule split between CTAs: O = sum_i 2^(lse_i - lse) O_i with
// lse = log2 sum_i 2^(lse_i). Block (unit, y) takes 32 query rows of the
// unit; 8 consecutive threads share a row, D/8 columns each, so every warp
// reads 4 whole rows of a partial at once.
// The CTA whose stream-K range holds tile position pos: the largest c with
// sk_start[c] <= pos (empty ranges before it share its start).
__device__ __forceinline__ int owner_of(const AttnParams& p, int G, long long pos) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.sk_start[mid] <= pos) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

constexpr int kCombineRowsPerBlock = 32;

template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const __grid_constant__ AttnParams p, int G) {
  constexpr int kCols = D / 8;
  const int NP = p.n_pairs;
  const long long T_head = p.pair_prefix[NP];
  const long long U = (long long)NP * p.H;
  const long long first_rem = (U / G) * G;  // units before it ran in whole-unit rounds
  const long long u = first_rem + blockIdx.x;
  if (u >= U) return;
  const int h = (int)(u / NP), pair = (int)(u % NP);
  auto cum = [&](long long v) { return (v / NP) * T_head + p.pair_prefix[v % NP]; };
  const long long C_u = cum(u);  // unit start (tile position)
  const int T_u = p.pair_prefix[pair + 1] - p.pair_prefix[pair];
  const int c_lo = owner_of(p, G, C_u), c_hi = owner_of(p, G, C_u + T_u - 1);
  if (c_lo == c_hi) return;  // written directly by one CTA
  const int prow = blockIdx.y * kCombineRowsPerBlock + (threadIdx.x >> 3);
  const int col0 = (threadIdx.x & 7) * kCols;
  const int qtok = pair * 2 * kTileRows + prow;
  if (qtok >= p.Nq) return;
  // slot of CTA c's job on this unit: its first job iff its range starts inside the unit
  auto slot_of = [&](int cc) { return 2 * cc + ((p.sk_start[cc] >= C_u) ? 0 : 1); };
  // a CTA whose stream-K range is empty holds no part
  auto has_part = [&](int cc) { return p.sk_start[cc + 1] > p.sk_start[cc]; };
  float mx = -INFINITY;
  for (int cc = c_lo; cc <= c_hi; ++cc)
    if (has_part(cc)) mx = fmaxf(mx, p.part_lse[(size_t)slot_of(cc) * 2 * kTileRows + prow]);
  float acc[kCols];
#pragma unroll
  for (int k = 0; k < kCols; ++k) acc[k] = 0.f;
  float den = 0.f;
  for (int cc = c_lo; cc <= c_hi; ++cc) {
    if (!has_part(cc)) continue;
    const int sl = slot_of(cc);
    const float ls = p.part_lse[(size_t)sl * 2 * kTileRows + prow];
    const float w = ls == -INFINITY ? 0.f : exp2f(ls - mx);
    den += w;
    const float4* src =
        reinterpret_cast<const float4*>(p.part_o + ((size_t)sl * 2 * kTileRows + prow) * D + col0);
#pragma unroll
    for (int v = 0; v < kCols / 4; ++v) {
      const float4 x = src[v];
      acc[4 * v] += w * x.x;
      acc[4 * v + 1] += w * x.y;
      acc[4 * v + 2] += w * x.z;
      acc[4 * v + 3] += w * x.w;
    }
  }
  // the partial rows are dead once merged: drop their L2 lines (each 128-byte
  // line by the first of the threads that read it) instead of letting them
  // be written back to HBM during a later launch. The lanes still here are
  // whole 8-lane row groups (a row past Nq left as a group), converged.
  __syncwarp(__activemask());
  if ((col0 & 31) == 0)
    for (int cc = c_lo; cc <= c_hi; ++cc)
      if (has_part(cc)) ptx::discard_l2(p.part_o + ((size_t)slot_of(cc) * 2 * kTileRows + prow) * D + col0);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)qtok * p.H + h) * D + col0);
#pragma unroll
  for (int v = 0; v < kCols / 8; ++v) {
    uint4 x;
    x.x = ptx::pack_bf16x2(acc[8 * v] * inv, acc[8 * v + 1] * inv);
    x.y = ptx::pack_bf16x2(acc[8 * v + 2] * inv, acc[8 * v + 3] * inv);
    x.z = ptx::pack_bf16x2(acc[8 * v + 4] * inv, acc[8 * v + 5] * inv);
    x.w = ptx::pack_bf16x2(acc[8 * v + 6] * inv, acc[8 * v + 7] * inv);
    __stcs(dst + v, x);
  }
  if (p.lse && (threadIdx.x & 7) == 0)
    p.lse[(size_t)h * p.Nq + qtok] = (den > 0.f ? mx + log2f(den) : -INFINITY) * 0.69314718055994531f;
}

template <int D>
cudaError_t launch_fwd_d(const AttnParams& p, cudaStream_t s) {
  using L = FwdLayout<D>;
  static PerDevice attr_set;
  int done = 0;
  cudaError_t e = attr_set.get(&done, [](int, int* x) {
    *x = 1;
    return cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kDynSmem);
  });
  if (e != cudaSuccess) return e;
  attn_fwd_kernel<D><<<p.n_ctas, kFwdThreads, L::kDynSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnParams& p, int head_dim, cudaStream_t s) {
  if (p.Nq <= 0 || p.n_ctas <= 0) return cudaSuccess;
  return head_dim == 64 ? launch_fwd_d<64>(p, s) : launch_fwd_d<128>(p, s);
}

cudaError_t launch_attention_combine(const AttnParams& p, int head_dim, cudaStream_t s) {
  if (p.Nq <= 0 || !p.part_o) return cudaSuccess;
  const int units = p.n_pairs * p.H;
  const int rem = units % p.n_ctas;  // units of the stream-K remainder
  if (rem == 0) return cudaSuccess;
  const dim3 grid(rem, 2 * kTileRows / kCombineRowsPerBlock);
  if (head_dim == 64)
    attn_combine_kernel<64><<<grid, 256, 0, s>>>(p, p.n_ctas);
  else
    attn_combine_kernel<128><<<grid, 256, 0, s>>>(p, p.n_ctas);
  return cudaGetLastError();
}

}  // namespace rc
