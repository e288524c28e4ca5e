// K4: chunk attention for sm_100a (tcgen05 + TMEM + TMA).
//
// O = softmax(Q K^T / sqrt(d) + mask) V for the current chunk's queries over
// every valid slot of the ring buffer (LingBot explainer, sliding-window
// section: the query reads the window up to local_end; Causal-Forcing
// walkthrough, section 3: only the current block's queries are computed).
// The mask acts only inside the current chunk (reading M1).
//
// One CTA = two 128-query tiles (Q0, Q1) of one head sharing every K/V tile.
//   warps 0-3   softmax of Q0 (thread = query row = TMEM lane), epilogue
//   warps 4-7   softmax of Q1, epilogue
//   warp 8      TMA producer: Q0/Q1 once, K and V into separate 2-stage rings
//   warp 9      TMEM allocator; one thread issues every tcgen05.mma
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d), O1 [384,384+d).
// P_i overwrites the first 64 columns of S_i as packed bf16 and is the A
// operand of O_i += P_i V.
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

constexpr int kFwdThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
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

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using L = FwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q, bar_kf[2], bar_vf[2], bar_ke[2], bar_ve[2], bar_s[2], bar_p[2], bar_o[2], bar_fin;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int q0 = blockIdx.x * 2 * kTileRows;
  const bool has1 = q0 + kTileRows < p.Nq;
  const int q_last = min(q0 + 2 * kTileRows, p.Nq) - 1;
  const int rq_hi = (q_last / p.F) / p.mask_block;
  const int T = count_tiles(p.seg, p.n_segs, rq_hi);
  const uint32_t base_u32 = (ptx::smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - ptx::smem_u32(smem_raw));

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bar_kf[i], 1);
      ptx::mbar_init(&bar_vf[i], 1);
      ptx::mbar_init(&bar_ke[i], 1);
      ptx::mbar_init(&bar_ve[i], 1);
      ptx::mbar_init(&bar_s[i], 1);
      ptx::mbar_init(&bar_p[i], 128);
      ptx::mbar_init(&bar_o[i], 1);
    }
    ptx::mbar_init(&bar_fin, 1);
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

  if (warp == kProducerWarp && lane == 0) {
    // ---------------------------------------------------------- producer
    ptx::tma_prefetch_desc(&p.tm_q);
    ptx::tma_prefetch_desc(&p.tm_k);
    ptx::tma_prefetch_desc(&p.tm_v);
    ptx::mbar_arrive_expect_tx(&bar_q, (has1 ? 2 : 1) * L::kTile);
    for (int i = 0; i < (has1 ? 2 : 1); ++i)
      for (int j = 0; j < L::kSub; ++j)
        ptx::tma_load_3d(&p.tm_q, &bar_q, base + L::kQ + i * L::kTile + j * kSubTileBytes, 64 * j,
                         q0 + i * kTileRows, h);
    TileWalker wk{p.seg, p.n_segs, rq_hi};
    Tile t;
    int nk[2] = {0, 0}, nv[2] = {0, 0};  // loads issued per stage
    for (int it = 0; wk.next(t); ++it) {
      const int st = it & 1;
      const uint32_t free_par = ((it >> 1) - 1) & 1;
      if (it >= 2 && !ptx::mbar_wait(&bar_ke[st], free_par, abort, p.status, RC_ETIMEOUT)) break;
      ptx::mbar_arrive_expect_tx(&bar_kf[st], L::kTile);
      for (int j = 0; j < L::kSub; ++j)
        ptx::tma_load_3d(&p.tm_k, &bar_kf[st], base + L::kK + st * L::kTile + j * kSubTileBytes, 64 * j,
                         t.tok, h);
      nk[st]++;
      if (it >= 2 && !ptx::mbar_wait(&bar_ve[st], free_par, abort, p.status, RC_ETIMEOUT)) break;
      ptx::mbar_arrive_expect_tx(&bar_vf[st], L::kTile);
      for (int j = 0; j < L::kSub; ++j)
        ptx::tma_load_3d(&p.tm_v, &bar_vf[st], base + L::kV + st * L::kTile + j * kSubTileBytes, 64 * j,
                         t.tok, h);
      nv[st]++;
    }
    // never leave a copy in flight: wait (bounded, ignoring abort) for the last ones
    int dummy = 0;
    volatile int* noabort = reinterpret_cast<volatile int*>(&dummy);
    ptx::mbar_wait(&bar_q, 0, noabort, p.status, RC_ETIMEOUT);
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
    auto issue_pv = [&](int i, int st, bool acc) {
      const uint32_t sV = base_u32 + L::kV + st * L::kTile;
#pragma unroll
      for (int ks = 0; ks < kTileRows / 16; ++ks)
        ptx::mma_ts(tmem + 256 + i * 128, tmem + i * 128 + ks * 8,
                    ptx::sdesc_sw128(sV + ks * 2048, kSubTileBytes, 1024), idesc_o, acc || ks > 0);
      ptx::mma_commit(&bar_o[i]);
    };
    bool ok = ptx::mbar_wait(&bar_q, 0, abort, p.status, RC_ETIMEOUT);
    if (ok && T > 0) {
      ok = ptx::mbar_wait(&bar_kf[0], 0, abort, p.status, RC_ETIMEOUT);
      if (ok) {
        ptx::tc_fence_after();
        issue_s(0, 0);
        if (has1) issue_s(1, 0);
        ptx::mma_commit(&bar_ke[0]);
      }
    }
    for (int j = 0; ok && j < T; ++j) {
      const int st = j & 1, st1 = (j + 1) & 1;
      const uint32_t par = j & 1;
      if (!ptx::mbar_wait(&bar_p[0], par, abort, p.status, RC_ETIMEOUT)) break;
      if (!ptx::mbar_wait(&bar_vf[st], (j >> 1) & 1, abort, p.status, RC_ETIMEOUT)) break;
      ptx::tc_fence_after();
      issue_pv(0, st, j > 0);
      if (!has1) ptx::mma_commit(&bar_ve[st]);
      const bool more = j + 1 < T;
      if (more) {
        if (!ptx::mbar_wait(&bar_kf[st1], ((j + 1) >> 1) & 1, abort, p.status, RC_ETIMEOUT)) break;
        ptx::tc_fence_after();
        issue_s(0, st1);
        if (!has1) ptx::mma_commit(&bar_ke[st1]);
      }
      if (has1) {
        if (!ptx::mbar_wait(&bar_p[1], par, abort, p.status, RC_ETIMEOUT)) break;
        ptx::tc_fence_after();
        issue_pv(1, st, j > 0);
        ptx::mma_commit(&bar_ve[st]);
        if (more) {
          issue_s(1, st1);
          ptx::mma_commit(&bar_ke[st1]);
        }
      }
    }
    int dummy = 0;
    ptx::mma_commit(&bar_fin);
    ptx::mbar_wait(&bar_fin, 0, reinterpret_cast<volatile int*>(&dummy), p.status, RC_ETIMEOUT);
  } else if (warp < 8 && (warp < 4 || has1)) {
    // ---------------------------------------------------------- softmax
    const int grp = warp >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int qtok = q0 + grp * kTileRows + row;
    const int my_rank = (min(qtok, p.Nq - 1) / p.F) / p.mask_block;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + grp * 128;
    const uint32_t tO = tmem + lane_off + 256 + grp * 128;
    const float c = p.scale_log2;
    const float thresh = kRescaleLog2 / c;
    float m = -INFINITY, l = 0.f;
    TileWalker wk{p.seg, p.n_segs, rq_hi};
    Tile t;
    bool ok = true;
    for (int j = 0; wk.next(t); ++j) {
      if (!ptx::mbar_wait(&bar_s[grp], j & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
      ptx::tc_fence_after();
      // columns [0, lim) of this row are visible (the whole row or a ragged tail is masked)
      const int lim = (t.rank < 0 || t.rank <= my_rank) ? t.nvalid : 0;
      // pass 1: row maximum of the raw scores
      float mx = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        ptx::tmem_ld32(tS + cc * 32, r);
        ptx::tmem_ld_wait();
        if (lim == kTileRows) {
#pragma unroll
          for (int k = 0; k < 32; ++k) mx = fmaxf(mx, __uint_as_float(r[k]));
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) mx = fmaxf(mx, cc * 32 + k < lim ? __uint_as_float(r[k]) : -INFINITY);
        }
      }
      const float m_new = fmaxf(m, mx);
      const bool need = m_new > m + thresh;       // also true for the first visible tile
      const bool real = need && m != -INFINITY;   // O already holds weighted values
      if (__any_sync(0xffffffffu, real)) {
        if (!ptx::mbar_wait(&bar_o[grp], (j - 1) & 1, abort, p.status, RC_ETIMEOUT)) { ok = false; break; }
        ptx::tc_fence_after();
        const float alpha = real ? ptx::ex2((m - m_new) * c) : 1.f;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
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
      // pass 2: P = 2^(s c - m c), packed bf16 pairs written over S's first
      // 64 columns; chunk cc's P columns [16cc, 16cc+16) lie in S columns
      // already read, so the overwrite never races a later read.
      float sum = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        ptx::tmem_ld32(tS + cc * 32, r);
        ptx::tmem_ld_wait();
        uint32_t pk[16];
        if (lim == kTileRows) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float a = ptx::ex2(fmaf(__uint_as_float(r[2 * k]), c, -mc));
            const float b = ptx::ex2(fmaf(__uint_as_float(r[2 * k + 1]), c, -mc));
            sum += a + b;
            pk[k] = ptx::pack_bf16x2(a, b);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float a = cc * 32 + 2 * k < lim ? ptx::ex2(fmaf(__uint_as_float(r[2 * k]), c, -mc)) : 0.f;
            const float b = cc * 32 + 2 * k + 1 < lim ? ptx::ex2(fmaf(__uint_as_float(r[2 * k + 1]), c, -mc)) : 0.f;
            sum += a + b;
            pk[k] = ptx::pack_bf16x2(a, b);
          }
        }
        ptx::tmem_st16(tS + cc * 16, pk);
      }
      ptx::tmem_st_wait();
      l += sum;
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bar_p[grp]);
    }
    // epilogue: O / l -> bf16 [Nq][H][D]; lse in natural log
    const int T_done = ok ? T : 0;
    bool have_o = T_done > 0 && ptx::mbar_wait(&bar_o[grp], (T_done - 1) & 1, abort, p.status, RC_ETIMEOUT);
    ptx::tc_fence_after();
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      if (have_o) {
        ptx::tmem_ld32(tO + cc * 32, o);
        ptx::tmem_ld_wait();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = 0u;
      }
      if (qtok < p.Nq) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)qtok * p.H + h) * D + cc * 32);
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
      const float lse2 = l > 0.f ? m * c + __log2f(l) : -INFINITY;
      p.lse[(size_t)h * p.Nq + qtok] = lse2 * 0.69314718055994531f;
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
cudaError_t launch_fwd_d(const AttnParams& p, cudaStream_t s) {
  using L = FwdLayout<D>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::kDynSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((p.Nq + 2 * kTileRows - 1) / (2 * kTileRows), p.H);
  attn_fwd_kernel<D><<<grid, kFwdThreads, L::kDynSmem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnParams& p, int head_dim, cudaStream_t s) {
  if (p.Nq <= 0) return cudaSuccess;
  return head_dim == 64 ? launch_fwd_d<64>(p, s) : launch_fwd_d<128>(p, s);
}

}  // namespace rc
