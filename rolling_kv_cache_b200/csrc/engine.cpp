// Policy engine (see engine.hpp). Rules, with the passages they restate:
//
// Sliding window + sink -- LingBot-World 2.0 explainer, "local_attn_size
//   滑动窗口" / "sink_size 注意力汇聚": the first sink frames never move; once
//   the cache is full every new block evicts as many of the oldest non-sink
//   frames (num_evicted = new + local_end - capacity); rolling fires only when
//   the forward adds new content, so a repeated pass overwrites in place.
//   RoPE uses the absolute frame number ("两个容易忽略的细节"): tau = g.
// Rolling Sink -- Rolling Sink digest, method-step details: at step i >= K the
//   sink shows a length-S segment of Roll(x_[0,K)) at the sliding times
//   [i-K, i-K+S); the K-S blocks before i keep their own time.
// Infinity-RoPE -- rCM guide, strategy 3: newest block ends at f_limit, older
//   blocks shift back by the same amount, times below 0 clamp to 0; KV flush
//   keeps the global sink and the last block; RoPE cut adds a jump to the
//   time of everything after the switch point.
// Deep Forcing -- rCM guide, strategy 4: deep sink + the top-C scored tokens
//   + the recent tail; after compaction the sink's and the compressed
//   region's time encodings are rewritten so no empty time positions remain
//   (the readings are spelled out in include/rc.h, RC_DEEP_FORCING). The
//   engine plans the region by counts and time formulas only; which tokens it
//   holds is decided on the device from the scores.
//
// The ring buffer replaces the pages' left-shift of the cache: frame g of the
// window lives in slot sink + (g - sink) mod window, so eviction is a table
// update. Keys are stored rotated to sigma = tau + shift, where shift is the
// Infinity-RoPE back-shift (0 elsewhere); a uniform offset of every time
// index leaves q.k unchanged, so only frames whose tau is clamped or whose
// content changes need a re-rotation job.
#include "engine.hpp"

#include <algorithm>
#include <map>
#include <sstream>

namespace rc {

void DefaultPairs(int head_dim, int* pt, int* ph, int* pw) {
  int c = head_dim / 2;
  *ph = *pw = c / 3;
  *pt = c - 2 * (c / 3);
}

static rc_status Fail(std::string* err, const std::string& m) {
  if (err) *err = m;
  return RC_EINVAL;
}

rc_status ValidateConfig(const rc_config& c, std::string* err) {
  if (c.layers < 1 || c.layers > 4096) return Fail(err, "layers must be in [1, 4096]");
  if (c.heads < 1 || c.heads > 1024) return Fail(err, "heads must be in [1, 1024]");
  if (c.head_dim != 64 && c.head_dim != 128) return Fail(err, "head_dim must be 64 or 128");
  if (c.grid_h < 1 || c.grid_w < 1 || (long long)c.grid_h * c.grid_w != c.frame_seqlen)
    return Fail(err, "frame_seqlen must equal grid_h * grid_w");
  if (c.chunk_frames < 1 || c.chunk_frames > RC_MAX_CHUNK_FRAMES)
    return Fail(err, "chunk_frames must be in [1, 16]");
  if (c.sink_frames < 0 || c.window_frames < 1) return Fail(err, "bad sink/window frames");
  if (c.sink_frames + c.window_frames > RC_MAX_SLOTS) return Fail(err, "sink + window exceeds 256 frames");
  if (c.df_budget_tokens != 0 && c.policy != RC_DEEP_FORCING)
    return Fail(err, "df_budget_tokens is a Deep Forcing parameter");
  if (c.rf_history_frames != 0 && c.policy != RC_RELAX_FORCING)
    return Fail(err, "rf_history_frames is a Relax Forcing parameter");
  long long cap = (long long)(c.sink_frames + c.window_frames) * c.frame_seqlen + 2LL * c.df_budget_tokens +
                  2LL * c.rf_history_frames * c.frame_seqlen + (c.policy == RC_MEMROPE ? 2LL * c.frame_seqlen : 0);
  if (cap * c.heads * c.head_dim >= (1LL << 31)) return Fail(err, "cache too large for 32-bit indexing");
  if ((long long)c.chunk_frames * c.frame_seqlen * c.heads * c.head_dim >= (1LL << 31))
    return Fail(err, "chunk too large for 32-bit indexing");
  if (c.mask_block_frames < 1) return Fail(err, "mask_block_frames must be >= 1");
  int pt = c.rope_t_pairs, ph = c.rope_h_pairs, pw = c.rope_w_pairs;
  if (pt == 0 && ph == 0 && pw == 0) DefaultPairs(c.head_dim, &pt, &ph, &pw);
  if (pt < 0 || ph < 0 || pw < 0 || pt + ph + pw != c.head_dim / 2)
    return Fail(err, "rope pairs must sum to head_dim / 2");
  if (!(c.theta > 1.0)) return Fail(err, "theta must be > 1");
  if (c.t_max < 1 || c.t_max > (1 << 20)) return Fail(err, "t_max must be in [1, 2^20]");
  const int B = c.chunk_frames;
  switch (c.policy) {
    case RC_NONE:
    case RC_SLIDING:
      if (c.window_frames < B) return Fail(err, "window must hold a whole chunk");
      break;
    case RC_ROLLING_SINK:
      if (c.rs_sink_blocks < 1 || c.rs_bank_blocks <= c.rs_sink_blocks)
        return Fail(err, "rolling sink needs K > S >= 1");
      if (c.sink_frames != c.rs_sink_blocks * B ||
          c.window_frames != (c.rs_bank_blocks - c.rs_sink_blocks + 1) * B)
        return Fail(err, "rolling sink needs sink = S*chunk and window = (K-S+1)*chunk frames");
      break;
    case RC_INFINITY_ROPE:
      if (c.ir_sink_blocks < 0 || c.ir_cache_blocks <= c.ir_sink_blocks)
        return Fail(err, "infinity-rope needs cache_blocks > sink_blocks >= 0");
      if (c.sink_frames != c.ir_sink_blocks * B ||
          c.window_frames != (c.ir_cache_blocks - c.ir_sink_blocks + 1) * B)
        return Fail(err, "infinity-rope needs sink = sink_blocks*chunk and window = "
                         "(cache - sink + 1)*chunk frames");
      if (c.ir_f_limit < B) return Fail(err, "f_limit must be >= chunk_frames");
      break;
    case RC_DEEP_FORCING:
      if (c.window_frames < 2 * B) return Fail(err, "deep forcing needs a tail of at least two chunks");
      if (c.df_budget_tokens < 0 || c.df_budget_tokens % c.frame_seqlen)
        return Fail(err, "df_budget_tokens must be a non-negative multiple of frame_seqlen");
      if (c.sink_frames + c.window_frames + c.df_budget_tokens / c.frame_seqlen > RC_MAX_SLOTS)
        return Fail(err, "sink + tail + budget frames exceed 256");
      break;
    case RC_MEMROPE:
      if (c.window_frames < B) return Fail(err, "window must hold a whole chunk");
      if (c.sink_frames + c.window_frames + 2 > RC_MAX_SLOTS) return Fail(err, "sink + window + memory exceed 256");
      if (!(c.mr_alpha_long >= 0.0 && c.mr_alpha_long <= 1.0 && c.mr_alpha_short >= 0.0 &&
            c.mr_alpha_short <= 1.0))
        return Fail(err, "mr_alpha_long / mr_alpha_short must be in [0, 1]");
      break;
    case RC_RELAX_FORCING:
      if (c.window_frames < B) return Fail(err, "the tail must hold a whole chunk");
      if (c.rf_history_frames < 0) return Fail(err, "rf_history_frames must be >= 0");
      if (c.sink_frames + c.window_frames + c.rf_history_frames > RC_MAX_SLOTS)
        return Fail(err, "sink + tail + history frames exceed 256");
      if (!(c.rf_weight >= 0.0 && c.rf_weight <= 1.0)) return Fail(err, "rf_weight must be in [0, 1]");
      if (c.rf_history_frames + B > 64) return Fail(err, "history frames + chunk frames must be <= 64");
      if (c.heads * c.head_dim > 6144) return Fail(err, "relax forcing needs heads * head_dim <= 6144");
      break;
    default:
      return Fail(err, "unknown policy");
  }
  return RC_OK;
}

Engine::Engine(const rc_config& cfg) : cfg_(cfg) {
  B_ = cfg.chunk_frames;
  S_f_ = cfg.sink_frames;
  W_f_ = cfg.window_frames;
  P_ = S_f_ + W_f_;
  F_ = cfg.frame_seqlen;
  // tokens of one selected-region buffer (Deep Forcing budget, Relax Forcing history)
  C_ = cfg.policy == RC_DEEP_FORCING ? cfg.df_budget_tokens
       : cfg.policy == RC_RELAX_FORCING ? cfg.rf_history_frames * cfg.frame_seqlen : 0;
  layers_.resize(cfg.layers);
  for (auto& L : layers_) L.slots.assign(P_, Slot());
}

int Engine::pristine_frames() const {
  if (cfg_.policy == RC_ROLLING_SINK) return cfg_.rs_bank_blocks * B_;
  if (cfg_.policy == RC_INFINITY_ROPE) return S_f_;
  // Deep Forcing: raw keys of every ring slot and both region buffers, indexed
  // like the cache's rows, so sink and region keys are always rotated from raw
  if (cfg_.policy == RC_DEEP_FORCING) return P_ + 2 * (C_ / F_);
  if (cfg_.policy == RC_MEMROPE) return P_;  // raw keys of the ring, folded when a frame leaves
  return 0;
}

static int RollIndex(int p, int K) {
  int q = p % (2 * K);
  return q < K ? q : 2 * K - 1 - q;
}

int Engine::ShiftOf(const LayerState& L) const {
  if (cfg_.policy != RC_INFINITY_ROPE) return 0;
  int g_end_v = L.vtime[L.cur_start + L.cur_n - 1] + 1;
  return std::max(0, g_end_v - cfg_.ir_f_limit);
}

std::vector<Kept> Engine::KeptSet(const LayerState& L) const {
  const int g0 = L.cur_start, n = L.cur_n, end = g0 + n, B = B_;
  std::vector<Kept> out;
  switch (cfg_.policy) {
    case RC_NONE:
    case RC_SLIDING: {
      int window = cfg_.policy == RC_NONE ? end : W_f_;
      for (int g = 0; g < std::min(S_f_, end); ++g)
        if (g < g0) out.push_back({g, g + L.sink_delta, kSink, -1});
      for (int g = std::max(S_f_, end - window); g < g0; ++g) out.push_back({g, g, kHist, -1});
      for (int g = g0; g < end; ++g)
        out.push_back({g, g + (g < S_f_ ? L.sink_delta : 0), kCur, g - g0});
      break;
    }
    case RC_ROLLING_SINK: {
      const int K = cfg_.rs_bank_blocks, S = cfg_.rs_sink_blocks, i = g0 / B;
      if (i < K) {
        for (int b = 0; b < i; ++b)
          for (int o = 0; o < B; ++o) out.push_back({b * B + o, b * B + o, b < S ? kSink : kHist, -1});
      } else {
        for (int j = 0; j < S; ++j) {
          int p = i - K + j;
          int cb = cfg_.rs_static_semantics ? j : RollIndex(p, K);
          for (int o = 0; o < B; ++o) out.push_back({cb * B + o, p * B + o, kSink, -1});
        }
        for (int b = i - (K - S); b < i; ++b)
          for (int o = 0; o < B; ++o) out.push_back({b * B + o, b * B + o, kHist, -1});
      }
      for (int o = 0; o < B; ++o) out.push_back({i * B + o, i * B + o, kCur, o});
      break;
    }
    case RC_INFINITY_ROPE: {
      const int sink_end = cfg_.ir_sink_blocks * B;
      int lo = std::max(sink_end, g0 - (cfg_.ir_cache_blocks - cfg_.ir_sink_blocks) * B);
      int last_flush = -1;
      for (int f : L.flush_points)
        if (f <= g0) last_flush = std::max(last_flush, f);
      if (last_flush >= 0) lo = std::max(lo, last_flush - B);
      const int shift = ShiftOf(L);
      auto tau = [&](int g) { return std::max(0, L.vtime[g] - shift); };
      for (int g = 0; g < std::min(sink_end, g0); ++g) out.push_back({g, tau(g), kSink, -1});
      for (int g = lo; g < g0; ++g) out.push_back({g, tau(g), kHist, -1});
      for (int g = g0; g < end; ++g) out.push_back({g, tau(g), kCur, g - g0});
      break;
    }
    case RC_MEMROPE: {
      // sliding window with the two memory frames (virtual slots P, P + 1) in
      // place of the evicted frames: long term after the sink, short term
      // right before the window
      const int g_w = TailStart(end);
      for (int g = 0; g < std::min(S_f_, g0); ++g) out.push_back({g, g, kSink, -1});
      if (L.mem_folded) {
        out.push_back({-1, S_f_, kHist, -1});
        out.push_back({-2, g_w - 1, kHist, -1});
      }
      for (int g = g_w; g < g0; ++g) out.push_back({g, g, kHist, -1});
      for (int g = g0; g < end; ++g) out.push_back({g, g, kCur, g - g0});
      break;
    }
    case RC_RELAX_FORCING: {
      // every frame at its own index; the history frames sit in the region
      for (int g = 0; g < std::min(S_f_, g0); ++g) out.push_back({g, g, kSink, -1});
      for (int g = TailStart(end); g < g0; ++g) out.push_back({g, g, kHist, -1});
      for (int g = g0; g < end; ++g) out.push_back({g, g, kCur, g - g0});
      break;
    }
    case RC_DEEP_FORCING: {
      // sink right before the region, region right before the tail (no holes)
      const int g_t = TailStart(end), V = L.comp_n / F_;
      for (int j = 0; j < std::min(S_f_, g0); ++j) out.push_back({j, g_t - V - S_f_ + j, kSink, -1});
      for (int g = g_t; g < g0; ++g) out.push_back({g, g, kHist, -1});
      for (int g = g0; g < end; ++g) out.push_back({g, g, kCur, g - g0});
      break;
    }
  }
  return out;
}

int Engine::SlotOf(const LayerState& L, const Kept& k) const {
  const int B = B_;
  if (cfg_.policy == RC_ROLLING_SINK) {
    const int K = cfg_.rs_bank_blocks, S = cfg_.rs_sink_blocks;
    const int i = L.cur_start / B;
    if (k.region == kSink && i >= K) {
      int p = k.tau / B, o = k.tau % B;
      return (p % S) * B + o;
    }
    int b = k.content / B, o = k.content % B;
    if (b < S) return k.content;
    return S_f_ + ((b - S) % (K - S + 1)) * B + o;
  }
  if (cfg_.policy == RC_NONE) return k.content;
  if (k.content < S_f_) return k.content;
  return S_f_ + (k.content - S_f_) % W_f_;
}

rc_status Engine::Step(int layer, int frame_start, int n_frames, StepPlan* plan, std::string* err) {
  if (layer < 0 || layer >= (int)layers_.size()) return Fail(err, "layer out of range");
  if (n_frames < 1 || n_frames > B_) return Fail(err, "n_frames must be in [1, chunk_frames]");
  LayerState L = layers_[layer];  // work on a copy; commit on success
  DfCompact df;
  MemUpdate mem;
  const bool repeat = L.cur_start >= 0 && frame_start == L.cur_start;
  if (repeat) {
    if (n_frames != L.cur_n) return Fail(err, "a repeated pass must cover the same frames");
  } else {
    if (frame_start != L.end) {
      if (err) {
        std::ostringstream s;
        s << "frame_start " << frame_start << " neither repeats the last chunk (" << L.cur_start
          << ") nor continues the stream (" << L.end << ")";
        *err = s.str();
      }
      return RC_ESTATE;
    }
    if (cfg_.policy == RC_ROLLING_SINK || cfg_.policy == RC_INFINITY_ROPE || cfg_.policy == RC_DEEP_FORCING ||
        cfg_.policy == RC_RELAX_FORCING || cfg_.policy == RC_MEMROPE) {
      if (n_frames != B_ || frame_start % B_) return Fail(err, "block policies step whole blocks");
    }
    if (cfg_.policy == RC_NONE && frame_start + n_frames > P_) {
      if (err) *err = "history exceeds the unbounded cache's capacity";
      return RC_ERANGE;
    }
    for (int g = frame_start; g < frame_start + n_frames; ++g) L.vtime.push_back(g + L.cut_total);
    if (cfg_.policy == RC_DEEP_FORCING || cfg_.policy == RC_RELAX_FORCING) {
      // pool = region tokens + the tokens of the frames leaving the tail (Relax
      // Forcing selects whole frames of it, Deep Forcing single tokens)
      DfCompact& d = df;
      const int new_end = frame_start + n_frames;
      d.n_old = L.comp_n;
      d.n_e = 0;
      for (int g = TailStart(L.end); g < TailStart(new_end) && g < L.end; ++g) {
        const int s = S_f_ + (g - S_f_) % W_f_;
        if (!L.slots[s].valid || L.slots[s].content != g) {
          if (err) *err = "internal: a leaving tail frame is not in its slot";
          return RC_EINVAL;
        }
        d.e_slot[d.n_e] = s;
        d.e_frame[d.n_e] = g;
        d.e_sigma[d.n_e] = L.slots[s].sigma;
        ++d.n_e;
      }
      const int pool = d.n_old + d.n_e * F_;
      d.n_new = std::min(C_, pool);
      d.use_sel = C_ > 0 && pool > C_;
      d.active = d.n_new > 0;
      d.src_buf = L.comp_buf;
      d.dst_buf = d.active ? 1 - L.comp_buf : L.comp_buf;
      d.src_row0 = P_ * F_ + d.src_buf * C_;
      d.dst_row0 = P_ * F_ + d.dst_buf * C_;
      d.tau_old0 = L.comp_tau0;
      d.tau_new0 = cfg_.policy == RC_RELAX_FORCING ? -1 : TailStart(new_end) - d.n_new / F_;
      d.keep_time = cfg_.policy == RC_RELAX_FORCING;
      // the tail after this chunk (Relax Forcing's alignment target): ring slots
      // of the frames that stay, then the chunk's own frames
      d.n_tail_kept = 0;
      for (int g = TailStart(new_end); g < frame_start; ++g) d.tail_slot[d.n_tail_kept++] = S_f_ + (g - S_f_) % W_f_;
      L.comp_n = d.n_new;
      L.comp_buf = d.dst_buf;
      L.comp_tau0 = d.tau_new0;
    }
    if (cfg_.policy == RC_MEMROPE) {
      MemUpdate& mu = mem;
      const int new_end = frame_start + n_frames;
      mu.initialised = L.mem_folded;
      for (int g = TailStart(L.end); g < TailStart(new_end) && g < L.end; ++g)
        mu.e_slot[mu.n_e++] = S_f_ + (g - S_f_) % W_f_;
      if (mu.n_e > 0) L.mem_folded = true;
      mu.active = L.mem_folded;
      mu.tau[0] = S_f_;
      mu.tau[1] = TailStart(new_end) - 1;
    }
    L.end = frame_start + n_frames;
    L.cur_start = frame_start;
    L.cur_n = n_frames;
  }

  std::vector<Kept> kept = KeptSet(L);
  const int shift = ShiftOf(L);
  std::vector<int> kslot(kept.size());
  std::vector<Slot> want(P_);
  for (size_t e = 0; e < kept.size(); ++e) {
    if (kept[e].content < 0) {  // a MemRoPE memory frame: rows past the ring, written by its own kernel
      kslot[e] = P_ + (kept[e].content == -1 ? 0 : 1);
      if (kept[e].tau < 0 || kept[e].tau >= cfg_.t_max) {
        if (err) *err = "memory time index outside [0, t_max)";
        return RC_ERANGE;
      }
      continue;
    }
    int s = SlotOf(L, kept[e]);
    int sigma = kept[e].tau + shift;
    if (s < 0 || s >= P_ || want[s].valid) {
      if (err) *err = "internal: slot collision";
      return RC_EINVAL;
    }
    if (sigma < 0 || sigma >= cfg_.t_max) {
      if (err) {
        std::ostringstream m;
        m << "time index " << sigma << " outside [0, t_max=" << cfg_.t_max << ")";
        *err = m.str();
      }
      return RC_ERANGE;
    }
    want[s] = Slot{1, kept[e].content, sigma};
    kslot[e] = s;
  }

  StepPlan p;
  p.df = df;
  p.mem = mem;
  p.repeat = repeat;
  p.frame_start = frame_start;
  p.n_frames = n_frames;
  const int npr = pristine_frames();
  for (size_t e = 0; e < kept.size(); ++e) {
    const Kept& k = kept[e];
    if (k.content < 0) continue;  // MemRoPE memory: updated by the memory kernel
    const Slot& have = L.slots[kslot[e]];
    const Slot& w = want[kslot[e]];
    if (k.region == kCur) {
      const int raw = (cfg_.policy == RC_DEEP_FORCING || cfg_.policy == RC_MEMROPE) ? kslot[e]
                      : (k.content < npr ? k.content : -1);
      p.append[k.rank] = AppendFrame{kslot[e], w.sigma, raw};
      continue;
    }
    if (have.valid && have.content == w.content && have.sigma == w.sigma) continue;
    const bool same = have.valid && have.content == w.content;
    if (cfg_.policy == RC_DEEP_FORCING && same) {
      // sink moved in time: rotate again from its raw keys (raw row = slot row)
      p.jobs.push_back(Job{kslot[e], kRotCopy, kslot[e], w.sigma, 0, 0});
    } else if (k.content < npr && (same || pristine_has_v())) {
      p.jobs.push_back(Job{kslot[e], kRotCopy, k.content, w.sigma, 0, same ? 0 : 1});
    } else if (same) {
      int delta = w.sigma - have.sigma;
      if (delta <= -cfg_.t_max || delta >= cfg_.t_max) {
        if (err) *err = "re-rotation delta exceeds t_max";
        return RC_ERANGE;
      }
      p.jobs.push_back(Job{kslot[e], kInPlace, -1, 0, delta, 0});
    } else {
      if (err) *err = "internal: kept content has no source";
      return RC_EINVAL;
    }
  }

  // KV runs for the attention: maximal runs of valid slots with one mask class.
  std::vector<int> cls(P_, -2);
  for (size_t e = 0; e < kept.size(); ++e)
    if (kslot[e] < P_) cls[kslot[e]] = kept[e].region == kCur ? kept[e].rank / cfg_.mask_block_frames : -1;
  for (int s = 0; s < P_;) {
    if (!want[s].valid) { ++s; continue; }
    int t = s + 1;
    while (t < P_ && want[t].valid && cls[t] == cls[s]) ++t;
    p.segs.push_back(Segment{s * F_, (t - s) * F_, cls[s]});
    s = t;
  }
  if (L.mem_folded) p.segs.push_back(Segment{P_ * F_, 2 * F_, -1});  // the two MemRoPE memory frames
  // Deep Forcing: the region (logically between the sink and the history
  // frames) is one more always-visible run; its V = comp_n / F "frames" are
  // candidates with virtual slots past the ring (slot * F = its first row)
  const int V = L.comp_n / F_;
  const int vslot0 = P_ + L.comp_buf * (C_ / std::max(1, F_));
  int n_sink = 0;
  for (const Kept& k : kept) n_sink += k.region == kSink;
  if (L.comp_n > 0) {
    p.segs.push_back(Segment{P_ * F_ + L.comp_buf * C_, L.comp_n, -1});
    for (int v = 0; v < V; ++v) p.cand.push_back(CandFrame{vslot0 + v, n_sink + v});
  }
  for (size_t e = 0; e < kept.size(); ++e)
    if (kept[e].region == kHist) p.cand.push_back(CandFrame{kslot[e], (int)e + V});
  if (cfg_.policy == RC_DEEP_FORCING) {
    // the next new chunk's pool: region + the tail frames it will push out
    const int end = L.cur_start + L.cur_n;
    for (int v = 0; v < V; ++v) p.df_pool.push_back(CandFrame{vslot0 + v, v});
    int k = 0;
    for (int g = TailStart(end); g < TailStart(end + B_); ++g, ++k)
      p.df_pool.push_back(CandFrame{S_f_ + (g - S_f_) % W_f_, V + k});
    p.df_select = C_ > 0 && L.comp_n + k * F_ > C_;
  }
  if ((int)p.segs.size() > kEngineMaxSegs) {
    if (err) *err = "cache holds more KV runs than one attention launch takes";
    return RC_ERANGE;
  }

  // evictions (multiset difference of contents) at a new chunk
  L.evicted.clear();
  if (!repeat) {
    std::map<int, int> cnt;
    for (const Kept& k : L.kept) cnt[k.content]++;
    for (const Kept& k : kept) cnt[k.content]--;
    for (auto& kv : cnt)
      for (int r = 0; r < kv.second; ++r) L.evicted.push_back(kv.first);
  }
  L.slots = want;
  L.kept = kept;
  L.kept_slot = kslot;
  L.shift = shift;
  L.n_jobs = (int)p.jobs.size();
  layers_[layer] = std::move(L);
  if (plan) *plan = std::move(p);
  return RC_OK;
}

rc_status Engine::Reindex(int t_delta, unsigned flags, std::string* err) {
  if (flags == 0 || (flags & ~7u)) return Fail(err, "unknown reindex flags");
  const bool ir = cfg_.policy == RC_INFINITY_ROPE;
  if ((flags & (RC_REINDEX_FLUSH | RC_REINDEX_CUT)) && !ir)
    return Fail(err, "flush and cut are Infinity-RoPE operations");
  if ((flags & RC_REINDEX_SINK) && !(cfg_.policy == RC_SLIDING || cfg_.policy == RC_NONE))
    return Fail(err, "sink time shift applies to the sliding and unbounded policies");
  if ((flags & RC_REINDEX_CUT) && t_delta < 0) return Fail(err, "a RoPE cut moves time forward");
  for (auto& L : layers_) {
    if (flags & RC_REINDEX_FLUSH) L.flush_points.push_back(L.end);
    if (flags & RC_REINDEX_CUT) L.cut_total += t_delta;
    if (flags & RC_REINDEX_SINK) L.sink_delta += t_delta;
  }
  return RC_OK;
}

}  // namespace rc
