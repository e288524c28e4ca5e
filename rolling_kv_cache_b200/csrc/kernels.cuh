// Kernel parameter blocks and launchers. Every kernel receives its metadata
// by value (a __grid_constant__ struct), so a step does no host-to-device
// copy of plans.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/rc.h"

namespace rc {

constexpr int kMaxJobs = 64;
constexpr int kMaxSegs = 48;  // == kEngineMaxSegs
constexpr int kMaxCandFrames = RC_MAX_SLOTS;
// Most CTAs a persistent attention launch uses (>= the B200's 148 SMs); sizes
// the partial-result workspace: 2 slots per CTA.
constexpr int kMaxPersistentCtas = 160;
// Most 256-query pairs a persistent attention launch schedules (per head).
constexpr int kMaxPairs = 128;

// Values the launchers look up once per device: a kernel's dynamic shared
// memory attribute (cudaFuncSetAttribute acts on the current device only), the
// SM count, a grid-stride kernel's resident blocks. One entry per device
// ordinal, so a process that drives several GPUs gets each device's own
// value; lock-free, and two threads that race compute the same value.
constexpr int kMaxDevices = 64;
struct PerDevice {
  std::atomic<int> v[kMaxDevices];
  // *out = the current device's value; `compute(dev, &x)` fills it the first
  // time (x must come out nonzero).
  template <typename Fn>
  cudaError_t get(int* out, Fn compute) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    int x = v[dev].load(std::memory_order_acquire);
    if (x == 0) {
      e = compute(dev, &x);
      if (e != cudaSuccess) return e;
      v[dev].store(x, std::memory_order_release);
    }
    *out = x;
    return cudaSuccess;
  }
};

struct RopeTables {
  const float2* t;  // [t_max][pt]   (cos, sin)
  const float2* h;  // [grid_h][ph]
  const float2* w;  // [grid_w][pw]
  int pt, ph, pw;
  int grid_w;
  int t_max;
};

// K1: fused RoPE + append of one chunk.
struct AppendParams {
  const uint16_t* q;   // [n_tok][H][d]
  const uint16_t* k;
  const uint16_t* v;
  uint16_t* q_rot;     // [H][q_stride][d]
  uint16_t* kc;        // [H][d/64][cap][64]: 64-dim planes (cache_off)
  uint16_t* vc;
  uint16_t* raw_k;     // pristine [H][raw_cap][d] or null
  uint16_t* raw_v;     // pristine V (Rolling Sink bank) or null
  int n_tok, H, d, F, cap, q_stride, raw_cap;
  int n_frames;
  int slot[RC_MAX_CHUNK_FRAMES];
  int sigma[RC_MAX_CHUNK_FRAMES];
  int raw_frame[RC_MAX_CHUNK_FRAMES];
  RopeTables rt;
};

// K2: re-rotation jobs (rotate-copy from a pristine source, or in place).
struct RerotateJob {
  int dst_slot;
  int mode;       // 0 rotate-copy, 1 in place (t pairs only)
  int src_frame;  // pristine frame
  int sigma;      // target time (rotate-copy)
  int delta;      // time delta (in place)
  int copy_v;
};
struct RerotateParams {
  uint16_t* kc;
  uint16_t* vc;
  const uint16_t* raw_k;
  const uint16_t* raw_v;
  int H, d, F, cap, raw_cap;
  int n_jobs;
  RerotateJob job[kMaxJobs];
  RopeTables rt;
};

// K2 in place, staged by TMA: R_t(delta_j) composed onto the time pairs of
// every key row of slot slot[j], for each job j. The tensor map covers the
// K ring [H * d/64][cap][64] with a box of the first 8 ct dims (the 16-byte
// chunks that hold time pairs) x R rows of one plane-0 row block.
struct InplaceParams {
  CUtensorMap tm;      // K ring as (64, cap, H * d/64), box {8 ct, R, 1}, no swizzle
  uint16_t* kc;
  const float2* tab_t; // time table [t_max][pt] (cos, sin)
  int* status;
  int pt, ct, planes, F, H, cap, R;
  int tiles_per_head;  // ceil(F / R)
  int n_jobs;
  int slot[kMaxJobs];
  int delta[kMaxJobs];
};

struct KvSegment {
  int tok_start;
  int len;
  int rank;  // -1 history, else mask class of the run
};

// K4: chunk attention (one CTA per 128-query tile and head).
struct alignas(64) AttnParams {
  CUtensorMap tm_q;    // q_rot [H][Nq][d], box {64, 128, 1}, 128B swizzle
  CUtensorMap tm_k;    // K cache [H][d/64][cap][64] as (64, cap, H*d/64), box {64, 128, 1}
  CUtensorMap tm_v;    // V cache, same layout
  uint16_t* out;       // [Nq][H][d] bf16
  float* lse;          // [H][Nq] or null
  int* status;         // device status word
  float* part_o;       // null, or stream-K partials [2 * n_ctas][256][d] fp32 (O / l)
  float* part_lse;     // [2 * n_ctas][256] fp32, log2-sum-exp of each partial row
  int n_ctas;          // grid size: persistent CTAs (with partials) or one per (head, pair)
  int Nq, H, F, mask_block;
  float scale_log2;    // log2(e) / sqrt(d)
  int n_segs;
  KvSegment seg[kMaxSegs];
  int n_pairs;                      // query pairs per head (persistent launches)
  int pair_prefix[kMaxPairs + 1];   // KV tiles of pairs [0, q) (same for every head)
  // stream-K range of CTA c, in (unit, tile) positions: [sk_start[c], sk_start[c + 1]);
  // sized so that round work + range is the same for every CTA
  int sk_start[kMaxPersistentCtas + 1];
};

// K6a: column scores over history tokens (second QK^T pass with final LSE).
struct alignas(64) ScoreParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  const float* lse;    // [H][Nq] natural log
  float* score_phys;   // [cap] fp32, accumulated with atomics
  int* status;
  int Nq, H;
  float scale_log2;
  int n_segs;
  KvSegment seg[kMaxSegs];
  int n_pairs;   // 256-query pairs per head
  int tiles;     // candidate KV tiles (every pair walks all of them)
  int n_ctas;    // persistent grid
};

// K6b: gather scores to logical order + top-C.
struct TopCParams {
  const float* score_phys;
  float* scores_out;   // [n_cand] or null
  int32_t* topc;       // [C] or null
  int C, F, n_cand_frames;
  int cand_slot[kMaxCandFrames];
  int cand_lpos[kMaxCandFrames];
};

cudaError_t launch_append(const AppendParams& p, cudaStream_t s);
cudaError_t launch_rerotate(const RerotateParams& p, cudaStream_t s);
cudaError_t launch_rerotate_inplace(const InplaceParams& p, cudaStream_t s);
// Rows per TMA box of the in-place kernel for frames of F tokens.
int inplace_box_rows(int F);
cudaError_t launch_attention(const AttnParams& p, int head_dim, cudaStream_t s);
// K5: merges the partial rows of split (head, pair) units; only after a launch with partials.
cudaError_t launch_attention_combine(const AttnParams& p, int head_dim, cudaStream_t s);
cudaError_t launch_scores(const ScoreParams& p, int head_dim, cudaStream_t s);
cudaError_t launch_topc(const TopCParams& p, cudaStream_t s);
cudaError_t launch_watchdog_selftest(int* status, unsigned limit_us, cudaStream_t s);
// Device address and size of the static step scratch on the current device
// (looked up once per device).
cudaError_t static_step_scratch(void** ptr, size_t* bytes);

}  // namespace rc
