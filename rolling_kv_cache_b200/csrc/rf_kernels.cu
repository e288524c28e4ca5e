// Relax Forcing frame selection (rCM guide, strategy 5): the cache keeps a
// sink, K history frames chosen by cosine similarity and the recent tail;
// score = w * alignment + (1 - w) * complement, Top-K.
//
// RF-a (two launches, fixed summation order, so a descriptor is the same bits
// on every run): the descriptor of a chunk frame is, per head, the mean over
// its tokens of the raw key. rf_desc_partial sums token ranges, rf_desc_final
// adds the ranges in order and scales by 1/F.
// RF-b (one CTA): alignment of every pool frame with the mean descriptor of
// the tail, complement = 1 - its mean cosine with the other pool frames, the
// score, and the K best (ties to the older frame) as token-level pool indices
// for the region gather.
#include "df_compact.cuh"
#include "kernels.cuh"

#include <cuda_bf16.h>

namespace rc {

namespace {

constexpr int kDescSplits = 32;
constexpr int kSelThreads = 256;
constexpr int kMaxPool = 64;   // pool frames one selection scores (validated on the host)

__global__ void rf_desc_partial_kernel(const __grid_constant__ RfDescParams p, float* partial) {
  const int rh = blockIdx.x;  // frame * H + head
  const int r = rh / p.H, h = rh - r * p.H;
  const int s = blockIdx.y;
  const int j = threadIdx.x;  // dim
  const int t0 = s * p.F / p.splits, t1 = (s + 1) * p.F / p.splits;
  float acc = 0.f;
  for (int t = t0; t < t1; ++t) {
    const uint16_t b = p.k[((size_t)(r * p.F + t) * p.H + h) * p.d + j];
    acc += __uint_as_float((uint32_t)b << 16);
  }
  partial[((size_t)s * gridDim.x + rh) * p.d + j] = acc;
}

__global__ void rf_desc_final_kernel(const __grid_constant__ RfDescParams p, const float* partial) {
  const int rh = blockIdx.x, j = threadIdx.x;
  float acc = 0.f;
  for (int s = 0; s < p.splits; ++s) acc += partial[((size_t)s * gridDim.x + rh) * p.d + j];
  p.desc_cur[(size_t)rh * p.d + j] = acc / (float)p.F;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One CTA; each warp takes whole dot products (lane-strided, then a shuffle
// reduction), so every sum has a fixed order.
__global__ void __launch_bounds__(kSelThreads) rf_select_kernel(const __grid_constant__ RfSelectParams p) {
  extern __shared__ float tail[];            // [H * d]: mean descriptor of the tail
  __shared__ float nrm[kMaxPool], al[kMaxPool], cs[kMaxPool][kMaxPool], sc[kMaxPool];
  __shared__ float tail_norm;
  __shared__ int keep[kMaxPool];
  const int D = p.H * p.d, n = p.n_pool, nt = p.n_tail + p.n_cur;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = kSelThreads / 32;
  for (int x = threadIdx.x; x < D; x += kSelThreads) {
    float a = 0.f;
    for (int f = 0; f < p.n_tail; ++f) a += p.desc[(size_t)p.tail_vslot[f] * D + x];
    for (int f = 0; f < p.n_cur; ++f) a += p.desc_cur[(size_t)f * D + x];
    tail[x] = a / (float)nt;
  }
  __syncthreads();
  if (warp == 0) {
    float v = 0.f;
    for (int x = lane; x < D; x += 32) v += tail[x] * tail[x];
    v = warp_sum(v);
    if (lane == 0) tail_norm = sqrtf(v);
  }
  __syncthreads();
  // norms and alignment, one pool frame per warp
  for (int i = warp; i < n; i += nw) {
    const float* di = p.desc + (size_t)p.pool_vslot[i] * D;
    float vv = 0.f, vt = 0.f;
    for (int x = lane; x < D; x += 32) {
      vv += di[x] * di[x];
      vt += di[x] * tail[x];
    }
    vv = warp_sum(vv);
    vt = warp_sum(vt);
    if (lane == 0) {
      nrm[i] = sqrtf(vv);
      al[i] = (nrm[i] > 0.f && tail_norm > 0.f) ? vt / (nrm[i] * tail_norm) : 0.f;
    }
  }
  __syncthreads();
  // pairwise cosines among the pool, one pair per warp
  for (int i = 0, cnt = 0; i < n; ++i)
    for (int j = i + 1; j < n; ++j, ++cnt) {
      if (cnt % nw != warp) continue;
      const float* di = p.desc + (size_t)p.pool_vslot[i] * D;
      const float* dj = p.desc + (size_t)p.pool_vslot[j] * D;
      float v = 0.f;
      for (int x = lane; x < D; x += 32) v += di[x] * dj[x];
      v = warp_sum(v);
      if (lane == 0) {
        const float c = (nrm[i] > 0.f && nrm[j] > 0.f) ? v / (nrm[i] * nrm[j]) : 0.f;
        cs[i][j] = c;
        cs[j][i] = c;
      }
    }
  __syncthreads();
  if (threadIdx.x < n) {
    const int i = threadIdx.x;
    float m = 0.f;
    for (int j = 0; j < n; ++j)
      if (j != i) m += cs[i][j];
    const float comp = n > 1 ? 1.f - m / (float)(n - 1) : 1.f;
    sc[i] = p.weight * al[i] + (1.f - p.weight) * comp;
    p.pool_scores[i] = sc[i];
  }
  if (threadIdx.x == 0) *p.n_scored = n;
  __syncthreads();
  // K best: frame i is kept if fewer than K frames rank before it
  // (higher score, or equal score and older); kept frames in pool order
  if (threadIdx.x < n) {
    const int i = threadIdx.x;
    int rank = 0;
    for (int j = 0; j < n; ++j) rank += (sc[j] > sc[i]) || (sc[j] == sc[i] && j < i);
    keep[i] = rank < p.K;
  }
  __syncthreads();
  for (int i = 0, k = 0; i < n; ++i) {
    if (!keep[i]) continue;
    for (int t = threadIdx.x; t < p.F; t += kSelThreads) p.sel[k * p.F + t] = i * p.F + t;
    ++k;
  }
}

}  // namespace

cudaError_t launch_rf_desc(const RfDescParams& p, cudaStream_t s) {
  // the partial sums live in the tail of desc_cur's scratch: the caller passes
  // desc_cur with room for kDescSplits more copies behind it
  float* partial = p.desc_cur + (size_t)p.n_frames * p.H * p.d;
  RfDescParams q = p;
  q.splits = kDescSplits;
  rf_desc_partial_kernel<<<dim3(p.n_frames * p.H, kDescSplits), p.d, 0, s>>>(q, partial);
  if (cudaError_t e = cudaGetLastError()) return e;
  rf_desc_final_kernel<<<p.n_frames * p.H, p.d, 0, s>>>(q, partial);
  return cudaGetLastError();
}

cudaError_t launch_rf_select(const RfSelectParams& p, cudaStream_t s) {
  // pool <= 64 frames and H * d <= 6144 are checked when the config is validated
  if (p.n_pool > kMaxPool || p.H * p.d > 6144) return cudaErrorInvalidValue;
  rf_select_kernel<<<1, kSelThreads, (size_t)p.H * p.d * sizeof(float), s>>>(p);
  return cudaGetLastError();
}

}  // namespace rc
