// Deep Forcing compaction kernel: parameter block and launcher.
#pragma once

#include "kernels.cuh"

namespace rc {

// K7: Deep Forcing compaction. New region token i comes from pool index
// p = sel[i] (sel == null: p = i); p < n_old is old region token p, else
// token (p - n_old) % F of leaving tail frame (p - n_old) / F. Its key is
// rotated again from its raw copy to time tau_new0 + i / F at its own (h, w)
// position; raw key and value are copied along, and meta records its
// (frame, token). Rows are physical rows of the layer's buffers.
struct DfCompactParams {
  uint16_t* kc;            // [H][d/64][cap][64]
  uint16_t* vc;
  uint16_t* raw_k;         // [H][cap][d] raw keys, same row indexing as the cache
  const int2* meta_src;    // (frame, token) of the old region's tokens
  int2* meta_dst;
  const int* sel;          // [n_new] ascending pool indices, or null
  int H, d, F, cap;
  int src_row0, dst_row0, n_old, n_new;
  int n_e;
  int e_slot[RC_MAX_CHUNK_FRAMES];
  int e_frame[RC_MAX_CHUNK_FRAMES];
  int tau_new0;
  // Relax Forcing: tokens keep their frame's time (keys copied, not rotated;
  // raw_k unused) and each region frame's descriptor moves with it
  int keep_time;
  float* desc;             // [vslots][H][d] fp32 frame descriptors (ring slots, then region slots)
  int src_vslot0, dst_vslot0;  // descriptor slot of region frame 0 in the old / new buffer
  RopeTables rt;
};

// Relax Forcing (rCM guide, strategy 5) frame selection.
// RF-a: desc_cur[r][h][:] = mean over frame r's tokens of the chunk's raw key.
struct RfDescParams {
  const uint16_t* k;   // [n_frames * F][H][d] bf16, the chunk's raw keys
  float* desc_cur;     // [n_frames][H][d], followed by room for the partial sums
  int n_frames, F, H, d, splits;
};
// RF-b: scores of the pool frames and the top-K of them, one CTA.
struct RfSelectParams {
  const float* desc;       // [vslots][H][d]
  const float* desc_cur;   // [n_cur][H][d]
  int n_pool;              // pool frames: pool_vslot[i]
  int pool_vslot[RC_MAX_SLOTS];
  int n_tail;              // tail frames that stay: tail_vslot[i]; then the n_cur chunk frames
  int tail_vslot[RC_MAX_SLOTS];
  int n_cur;
  int K, F, H, d;
  float weight;
  int* sel;                // [K * F] token-level pool indices, ascending
  float* pool_scores;      // [RC_MAX_SLOTS]
  int* n_scored;           // pool size of this selection
};
// MemRoPE (rCM guide, MemRoPE tip): fold the frames leaving the window into
// the long- and short-term EMA memories (fp32 state, raw keys and values)
// and write both memory frames, keys rotated to their times, into the cache.
struct MemUpdateParams {
  uint16_t* kc;            // [H][d/64][cap][64]
  uint16_t* vc;
  const uint16_t* raw_k;   // [H][raw_cap][d] raw keys of the ring slots
  float* mem;              // [2 (k, v)][2 (long, short)][F][H][d] fp32 state
  int H, d, F, cap, raw_cap;
  int n_e;                 // frames leaving the window, oldest first
  int e_slot[RC_MAX_CHUNK_FRAMES];
  int initialised;         // the state holds a folded frame already
  float a[2], b[2];        // alpha, 1 - alpha of the long- and short-term memory
  int tau[2];              // their times
  int row0;                // cache row of memory token 0 (long), row0 + F (short)
  RopeTables rt;
};
cudaError_t launch_mem_update(const MemUpdateParams& p, cudaStream_t s);

cudaError_t launch_rf_desc(const RfDescParams& p, cudaStream_t s);
cudaError_t launch_rf_select(const RfSelectParams& p, cudaStream_t s);

cudaError_t launch_df_compact(const DfCompactParams& p, cudaStream_t s);

}  // namespace rc
