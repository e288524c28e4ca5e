// Policy engine: the integer side of one rc_step.
//
// Host-only C++ (no CUDA). Per layer it keeps the stream history (virtual
// time of every committed frame, flush points, cut total) and the ring
// buffer's slot table (which stream frame each physical frame slot holds and
// the time index its keys are rotated to). A step recomputes the kept frames
// from the history with the page rules, maps them to slots, and diffs the
// wanted slot table against the current one to produce the device work:
// append jobs (fused RoPE + write of the new chunk), re-rotation jobs for
// kept frames whose time index or content changed, and the attention's KV
// segment list. Eviction is a slot-table update; no bytes move.
#pragma once

#include <algorithm>
#include <cstdint>
#include <string>
#include <vector>

#include "../../include/rc.h"

namespace rc {

// Largest number of KV runs one attention launch takes (kernel parameter space).
constexpr int kEngineMaxSegs = 48;

enum Region { kSink = 0, kHist = 1, kCur = 2 };

struct Kept {
  int content;  // stream frame index of the raw k/v
  int tau;      // policy time index
  int region;   // Region
  int rank;     // chunk-relative frame for kCur, -1 otherwise
};

struct Slot {
  int valid = 0;
  int content = -1;
  int sigma = 0;  // time index the stored keys are rotated to
};

enum JobMode { kRotCopy = 0, kInPlace = 1 };

struct Job {
  int dst_slot;
  int mode;       // JobMode
  int src_frame;  // pristine frame index (kRotCopy)
  int sigma;      // target time (kRotCopy)
  int delta;      // time delta (kInPlace)
  int copy_v;     // kRotCopy also copies V from the pristine source
};

struct AppendFrame {
  int slot;
  int sigma;
  int raw_frame;  // frame index in the pristine buffer, -1 = none
};

struct Segment {
  int tok_start;  // first token (physical, per head) of the run
  int len;        // tokens
  int rank;       // mask class of the run: -1 history, else (chunk frame)/mask_block
};

struct CandFrame {
  int slot;       // physical slot of a history-region frame
  int lpos;       // its position in the logical kept list
};

// Deep Forcing compaction of one new chunk: the new compressed region is
// gathered from the pool (old region tokens, then the tokens of the frames
// that left the tail) into the other region buffer, each key re-rotated from
// its old time to its new one.
struct DfCompact {
  bool active = false;
  int src_row0 = 0, dst_row0 = 0;  // first physical row of the old / new region buffer
  int src_buf = 0, dst_buf = 0;
  int n_old = 0, n_new = 0;        // region tokens before / after
  int n_e = 0;                     // frames that left the tail
  int e_slot[RC_MAX_CHUNK_FRAMES];
  int e_frame[RC_MAX_CHUNK_FRAMES];
  int e_sigma[RC_MAX_CHUNK_FRAMES];
  bool use_sel = false;            // pool > budget: region = the device top-C selection
  int tau_old0 = 0, tau_new0 = 0;  // region token i: tau = tau0 + i / F (Deep Forcing)
  bool keep_time = false;          // Relax Forcing: tokens keep their frame's time, no rotation
  int n_tail_kept = 0;             // Relax Forcing: tail frames that stay (ring slots)
  int tail_slot[RC_MAX_SLOTS];
};

// MemRoPE memory update of one new chunk: fold the frames leaving the window
// into the two EMA memories and rotate both to their positions.
struct MemUpdate {
  bool active = false;
  bool initialised = false;        // a frame was folded before this chunk
  int n_e = 0;                     // frames leaving the window, oldest first
  int e_slot[RC_MAX_CHUNK_FRAMES];
  int tau[2] = {0, 0};             // long-term, short-term memory time
};

struct StepPlan {
  bool repeat = false;
  int frame_start = 0;
  int n_frames = 0;
  AppendFrame append[RC_MAX_CHUNK_FRAMES];
  std::vector<Job> jobs;
  std::vector<Segment> segs;
  std::vector<CandFrame> cand;  // logical order
  // Deep Forcing
  DfCompact df;
  std::vector<CandFrame> df_pool;  // next new chunk's pool (lpos = pool frame index)
  bool df_select = false;          // that pool exceeds the budget: select top-C now
  // MemRoPE
  MemUpdate mem;
};

struct LayerState {
  int end = 0;
  int cur_start = -1;
  int cur_n = 0;
  std::vector<int> vtime;
  int cut_total = 0;
  std::vector<int> flush_points;
  int sink_delta = 0;
  int shift = 0;
  std::vector<Slot> slots;
  std::vector<Kept> kept;
  std::vector<int> kept_slot;
  std::vector<int> evicted;
  int n_jobs = 0;
  // Deep Forcing compressed region
  int comp_n = 0;     // tokens
  int comp_buf = 0;   // which of the two region buffers holds it
  int comp_tau0 = 0;  // region token i has tau = comp_tau0 + i / F
  // MemRoPE: a frame has been folded into the memories
  bool mem_folded = false;
};

class Engine {
 public:
  // cfg must already be validated (ValidateConfig).
  explicit Engine(const rc_config& cfg);

  // Plans and commits one step of `layer`. On failure the layer is unchanged.
  rc_status Step(int layer, int frame_start, int n_frames, StepPlan* plan, std::string* err);
  rc_status Reindex(int t_delta, unsigned flags, std::string* err);

  const LayerState& layer(int l) const { return layers_[l]; }
  int slots() const { return P_; }
  // Tokens per head the device buffers hold: the ring plus, under Deep
  // Forcing, two compressed-region buffers of df_budget_tokens each.
  long long capacity_tokens() const { return (long long)P_ * F_ + 2LL * C_ + (mem() ? 2LL * F_ : 0); }
  bool mem() const { return cfg_.policy == RC_MEMROPE; }
  int df_budget() const { return C_; }
  // Frames of the pristine (raw, unrotated) source a policy keeps: Rolling
  // Sink's bank of the first K blocks (K and V), Infinity-RoPE's sink (K).
  int pristine_frames() const;
  bool pristine_has_v() const { return cfg_.policy == RC_ROLLING_SINK; }

 private:
  std::vector<Kept> KeptSet(const LayerState& L) const;
  int SlotOf(const LayerState& L, const Kept& k) const;
  int ShiftOf(const LayerState& L) const;

  int TailStart(int end) const { return std::max(S_f_, end - W_f_); }

  rc_config cfg_;
  int B_, S_f_, W_f_, P_, F_, C_;
  std::vector<LayerState> layers_;
};

// Returns RC_OK or RC_EINVAL with a message.
rc_status ValidateConfig(const rc_config& cfg, std::string* err);
// Default RoPE pair split of head_dim/2 pairs.
void DefaultPairs(int head_dim, int* pt, int* ph, int* pw);

}  // namespace rc
