// C ABI (include/rc.h): memory plan, RoPE tables, TMA descriptors and the
// launch sequence of one step. Host code; kernels live in the other .cu files.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <memory>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/rc.h"
#include "engine.hpp"
#include "kernels.cuh"
#include "df_compact.cuh"

namespace {

thread_local std::string g_err;

rc_status set_err(rc_status st, const std::string& m) {
  g_err = m;
  return st;
}

rc_status cuda_err(cudaError_t e, const char* what) {
  return set_err(RC_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Raw (unrotated) source buffers a policy keeps per layer: K and V for
// Rolling Sink's bank, K for Infinity-RoPE's sink and for Deep Forcing.
int raw_buffers(const rc_config& c) {
  if (c.policy == RC_ROLLING_SINK) return 2;
  return (c.policy == RC_INFINITY_ROPE || c.policy == RC_DEEP_FORCING || c.policy == RC_MEMROPE) ? 1 : 0;
}

struct MemPlan {
  size_t kv_bytes, raw_bytes, q_bytes, lse_bytes, score_bytes, tab_t, tab_h, tab_w, status_bytes,
      part_o_bytes, part_lse_bytes, df_meta_bytes, df_sel_bytes, rf_desc_bytes, rf_pool_bytes,
      rf_cur_bytes, mem_bytes;
  size_t off_kv, off_raw, off_q, off_lse, off_score_phys, off_score_logical, off_tab_t, off_tab_h,
      off_tab_w, off_status, off_part_o, off_part_lse, off_df, off_rf_cur, total;
  int pt, ph, pw, cap, raw_frames, q_stride;
};

MemPlan plan_memory(const rc_config& c, int raw_frames) {
  MemPlan m{};
  m.pt = c.rope_t_pairs;
  m.ph = c.rope_h_pairs;
  m.pw = c.rope_w_pairs;
  if (m.pt == 0 && m.ph == 0 && m.pw == 0) rc::DefaultPairs(c.head_dim, &m.pt, &m.ph, &m.pw);
  // ring rows, then two selected-region buffers (Deep Forcing tokens, Relax Forcing frames)
  const int region = c.df_budget_tokens + c.rf_history_frames * c.frame_seqlen;
  m.cap = (c.sink_frames + c.window_frames) * c.frame_seqlen + 2 * region +
          (c.policy == RC_MEMROPE ? 2 * c.frame_seqlen : 0);  // MemRoPE: the two memory frames
  m.raw_frames = raw_frames;
  m.q_stride = c.chunk_frames * c.frame_seqlen;
  const size_t row = (size_t)c.head_dim * 2;
  m.kv_bytes = align_up((size_t)c.heads * m.cap * row);                     // one of K/V, one layer
  m.raw_bytes = align_up((size_t)c.heads * raw_frames * c.frame_seqlen * row);
  m.q_bytes = align_up((size_t)c.heads * m.q_stride * row);
  m.lse_bytes = align_up((size_t)c.heads * m.q_stride * 4);
  m.score_bytes = align_up((size_t)m.cap * 4);
  m.tab_t = align_up((size_t)c.t_max * m.pt * 8);
  m.tab_h = align_up((size_t)c.grid_h * m.ph * 8);
  m.tab_w = align_up((size_t)c.grid_w * m.pw * 8);
  m.status_bytes = kAlign;
  // stream-K partial rows of the attention: 2 slots per persistent CTA, 256 query rows each
  m.part_o_bytes = align_up((size_t)2 * rc::kMaxPersistentCtas * 256 * c.head_dim * 4);
  m.part_lse_bytes = align_up((size_t)2 * rc::kMaxPersistentCtas * 256 * 4);
  // Deep / Relax Forcing per layer: (frame, token) of both region buffers' tokens, and the selection
  m.df_meta_bytes = align_up((size_t)2 * region * 8);
  m.df_sel_bytes = align_up((size_t)region * 4);
  // Relax Forcing per layer: frame descriptors [ring + 2 K slots][H][d] fp32, pool scores;
  // per step: the chunk's descriptors and their partial sums
  const bool rf = c.policy == RC_RELAX_FORCING;
  m.rf_desc_bytes = rf ? align_up((size_t)(c.sink_frames + c.window_frames + 2 * c.rf_history_frames) *
                                  c.heads * c.head_dim * 4) : 0;
  m.rf_pool_bytes = rf ? align_up((RC_MAX_SLOTS + 1) * 4) : 0;
  m.rf_cur_bytes = rf ? align_up((size_t)(1 + 32) * c.chunk_frames * c.heads * c.head_dim * 4) : 0;
  // MemRoPE per layer: fp32 EMA state of keys and values of both memories
  m.mem_bytes = c.policy == RC_MEMROPE ? align_up((size_t)4 * c.frame_seqlen * c.heads * c.head_dim * 4) : 0;
  const int nraw = raw_buffers(c);
  size_t o = 0;
  m.off_kv = o;
  o += 2 * m.kv_bytes * c.layers;
  m.off_raw = o;
  o += (size_t)nraw * m.raw_bytes * c.layers;
  m.off_q = o;
  o += m.q_bytes;
  m.off_lse = o;
  o += m.lse_bytes;
  m.off_score_phys = o;
  o += m.score_bytes;
  m.off_score_logical = o;
  o += m.score_bytes;
  m.off_tab_t = o;
  o += m.tab_t;
  m.off_tab_h = o;
  o += m.tab_h;
  m.off_tab_w = o;
  o += m.tab_w;
  m.off_status = o;
  o += m.status_bytes;
  m.off_part_o = o;
  o += m.part_o_bytes;
  m.off_part_lse = o;
  o += m.part_lse_bytes;
  m.off_df = o;
  o += (m.df_meta_bytes + m.df_sel_bytes + m.rf_desc_bytes + m.rf_pool_bytes + m.mem_bytes) * c.layers;
  m.off_rf_cur = o;
  o += m.rf_cur_bytes;
  m.total = o;
  return m;
}

// fp64 cos/sin of pos * theta^(-2j / (2 P)) for pos in [0, n_pos), rounded to fp32.
void build_table(std::vector<float>& out, int n_pos, int pairs, double theta) {
  out.assign((size_t)n_pos * pairs * 2, 0.f);
  for (int j = 0; j < pairs; ++j) {
    const double omega = std::pow(theta, -2.0 * j / (2.0 * pairs));
    for (int t = 0; t < n_pos; ++t) {
      const double a = t * omega;
      out[((size_t)t * pairs + j) * 2] = (float)std::cos(a);
      out[((size_t)t * pairs + j) * 2 + 1] = (float)std::sin(a);
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [heads][rows][d] bf16, head stride `head_stride_rows` rows; box {box_x, box_rows, 1}.
rc_status make_map(CUtensorMap* map, void* base, int d, int rows, int heads, long long head_stride_rows,
                   int box_x = 64, int box_rows = 128, bool swizzle128 = true) {
  auto fn = encode_fn();
  if (!fn) return set_err(RC_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)head_stride_rows * d * 2};
  cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_err(RC_ECUDA, "cuTensorMapEncodeTiled failed: " + std::to_string(r));
  return RC_OK;
}

// Optional per-kernel event timing (rc_profile_begin / rc_profile_end).
struct Profiler {
  bool on = false;
  int max = 0, used = 0;
  std::vector<cudaEvent_t> ev;  // 2 per timed launch
  std::vector<int> kind;
  int64_t launches[RC_KERNEL_KINDS] = {};
  double flops[RC_KERNEL_KINDS] = {}, bytes[RC_KERNEL_KINDS] = {};
  void release() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
    ev.clear();
    kind.clear();
    on = false;
    max = used = 0;
  }
  ~Profiler() { release(); }
};

// Brackets one launch with events when profiling is armed.
struct Timed {
  Profiler& p;
  int k, slot = -1;
  cudaStream_t s;
  Timed(Profiler& pr, int kind, cudaStream_t st, double flops, double bytes) : p(pr), k(kind), s(st) {
    if (!p.on) return;
    p.launches[k]++;
    p.flops[k] += flops;
    p.bytes[k] += bytes;
    if (p.used < p.max) {
      slot = p.used++;
      p.kind[slot] = k;
      cudaEventRecord(p.ev[2 * slot], s);
    }
  }
  ~Timed() {
    if (slot >= 0) cudaEventRecord(p.ev[2 * slot + 1], s);
  }
};

struct Cache {
  Profiler prof;
  rc_config cfg{};
  std::unique_ptr<rc::Engine> engine;
  bool device = false;
  uint8_t* mem = nullptr;
  MemPlan mp{};
  std::vector<uint16_t*> kc, vc, rawk, rawv;
  std::vector<CUtensorMap> tm_k, tm_v;
  // K ring boxes of the time-pair chunks for the TMA in-place re-rotation
  // (empty when the time pairs do not all sit in the first 64 dims)
  std::vector<CUtensorMap> tm_kt;
  int ip_ct = 0, ip_rows = 0;
  CUtensorMap tm_q{};
  int tm_q_rows = -1;
  std::vector<float> tab[3];
  rc::RopeTables rt{};
  uint16_t* qrot = nullptr;
  float* lse_scratch = nullptr;
  float* score_phys = nullptr;
  float* score_logical = nullptr;
  int* status = nullptr;
  float* part_o = nullptr;
  float* part_lse = nullptr;
  int sm_count = 148;
  int dev_id = -1;  // CUDA device ordinal the block was created on (device handles)
  // candidate frames (slot, logical position) of each layer's last step, for rc_select_topc
  std::vector<std::vector<std::pair<int, int>>> last_cand;
  // Deep Forcing per layer: region token sources [2][budget] and the pool selection [budget]
  std::vector<int2*> df_meta;
  std::vector<int*> df_sel;
  // Relax Forcing per layer: frame descriptors and the last pool scores ([RC_MAX_SLOTS] + count)
  std::vector<float*> rf_desc;
  std::vector<float*> rf_pool;
  float* rf_cur = nullptr;  // the chunk's descriptors + partial sums (per step)
  // MemRoPE per layer: fp32 EMA state [2 (k, v)][2 (long, short)][F][H][d]
  std::vector<float*> mem_state;
};

rc_status check_handle(const void* h) {
  if (!h) return set_err(RC_EINVAL, "null handle");
  return RC_OK;
}

// A device handle's kernels and copies must run on the GPU that holds its
// memory block: with another device current they would be launched there
// against memory of another GPU. Checked before anything is planned or
// enqueued.
rc_status check_device(const Cache* c) {
  if (!c->device) return RC_OK;
  int dev = -1;
  if (cudaError_t e = cudaGetDevice(&dev)) return cuda_err(e, "cudaGetDevice");
  if (dev != c->dev_id)
    return set_err(RC_EINVAL, "the current CUDA device (" + std::to_string(dev) +
                                  ") is not the device the cache was created on (" +
                                  std::to_string(c->dev_id) + ")");
  return RC_OK;
}

}  // namespace

extern "C" {

const char* rc_last_error(void) { return g_err.c_str(); }

rc_status rc_config_init(rc_config* cfg, int layers, int heads, int head_dim, int frame_seqlen,
                         int sink_frames, int window_frames) {
  if (!cfg) return set_err(RC_EINVAL, "null config");
  std::memset(cfg, 0, sizeof(*cfg));
  cfg->layers = layers;
  cfg->heads = heads;
  cfg->head_dim = head_dim;
  cfg->frame_seqlen = frame_seqlen;
  cfg->grid_h = 1;
  cfg->grid_w = frame_seqlen;
  cfg->sink_frames = sink_frames;
  cfg->window_frames = window_frames;
  cfg->chunk_frames = 3;
  cfg->mask_block_frames = 1;
  cfg->theta = 10000.0;
  cfg->t_max = 4096;
  cfg->policy = RC_SLIDING;
  return RC_OK;
}

rc_status rc_cache_bytes(const rc_config* cfg, size_t* bytes) {
  if (!cfg || !bytes) return set_err(RC_EINVAL, "null argument");
  std::string err;
  if (rc_status st = rc::ValidateConfig(*cfg, &err)) return set_err(st, err);
  rc::Engine e(*cfg);
  *bytes = plan_memory(*cfg, e.pristine_frames()).total;
  return RC_OK;
}

rc_status rc_cache_create(const rc_config* cfg, void* dev_mem, size_t bytes, void** out_handle) {
  if (!cfg || !out_handle) return set_err(RC_EINVAL, "null argument");
  *out_handle = nullptr;
  std::string err;
  if (rc_status st = rc::ValidateConfig(*cfg, &err)) return set_err(st, err);
  auto c = std::make_unique<Cache>();
  c->cfg = *cfg;
  c->engine = std::make_unique<rc::Engine>(*cfg);
  c->mp = plan_memory(*cfg, c->engine->pristine_frames());
  const MemPlan& m = c->mp;
  build_table(c->tab[0], cfg->t_max, m.pt, cfg->theta);
  build_table(c->tab[1], cfg->grid_h, m.ph, cfg->theta);
  build_table(c->tab[2], cfg->grid_w, m.pw, cfg->theta);
  if (dev_mem) {
    if (bytes < m.total) return set_err(RC_ENOMEM, "memory block smaller than rc_cache_bytes()");
    if (reinterpret_cast<uintptr_t>(dev_mem) % kAlign) return set_err(RC_EINVAL, "memory block must be 256-byte aligned");
    c->device = true;
    c->mem = static_cast<uint8_t*>(dev_mem);
    uint8_t* b = c->mem;
    const int L = cfg->layers;
    const int nraw = raw_buffers(*cfg);
    for (int l = 0; l < L; ++l) {
      c->kc.push_back(reinterpret_cast<uint16_t*>(b + m.off_kv + (2 * (size_t)l) * m.kv_bytes));
      c->vc.push_back(reinterpret_cast<uint16_t*>(b + m.off_kv + (2 * (size_t)l + 1) * m.kv_bytes));
      c->rawk.push_back(nraw >= 1 ? reinterpret_cast<uint16_t*>(b + m.off_raw + (nraw * (size_t)l) * m.raw_bytes)
                                  : nullptr);
      c->rawv.push_back(nraw == 2 ? reinterpret_cast<uint16_t*>(b + m.off_raw + (nraw * (size_t)l + 1) * m.raw_bytes)
                                  : nullptr);
      uint8_t* df = b + m.off_df + (m.df_meta_bytes + m.df_sel_bytes + m.rf_desc_bytes + m.rf_pool_bytes +
                                    m.mem_bytes) * l;
      c->df_meta.push_back(reinterpret_cast<int2*>(df));
      c->df_sel.push_back(reinterpret_cast<int*>(df + m.df_meta_bytes));
      c->rf_desc.push_back(reinterpret_cast<float*>(df + m.df_meta_bytes + m.df_sel_bytes));
      c->rf_pool.push_back(reinterpret_cast<float*>(df + m.df_meta_bytes + m.df_sel_bytes + m.rf_desc_bytes));
      c->mem_state.push_back(reinterpret_cast<float*>(df + m.df_meta_bytes + m.df_sel_bytes + m.rf_desc_bytes +
                                                      m.rf_pool_bytes));
    }
    c->qrot = reinterpret_cast<uint16_t*>(b + m.off_q);
    c->lse_scratch = reinterpret_cast<float*>(b + m.off_lse);
    c->score_phys = reinterpret_cast<float*>(b + m.off_score_phys);
    c->score_logical = reinterpret_cast<float*>(b + m.off_score_logical);
    c->status = reinterpret_cast<int*>(b + m.off_status);
    c->part_o = reinterpret_cast<float*>(b + m.off_part_o);
    c->part_lse = reinterpret_cast<float*>(b + m.off_part_lse);
    c->rf_cur = reinterpret_cast<float*>(b + m.off_rf_cur);
    int dev = 0, sms = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return cuda_err(e, "cudaGetDevice");
    c->dev_id = dev;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
      c->sm_count = sms;
    cudaError_t e = cudaMemset(c->mem, 0, m.total);
    if (e != cudaSuccess) return cuda_err(e, "cudaMemset");
    float* tabs[3] = {reinterpret_cast<float*>(b + m.off_tab_t), reinterpret_cast<float*>(b + m.off_tab_h),
                      reinterpret_cast<float*>(b + m.off_tab_w)};
    for (int a = 0; a < 3; ++a) {
      if (c->tab[a].empty()) continue;
      e = cudaMemcpy(tabs[a], c->tab[a].data(), c->tab[a].size() * 4, cudaMemcpyHostToDevice);
      if (e != cudaSuccess) return cuda_err(e, "cudaMemcpy tables");
    }
    c->rt = rc::RopeTables{reinterpret_cast<const float2*>(tabs[0]), reinterpret_cast<const float2*>(tabs[1]),
                           reinterpret_cast<const float2*>(tabs[2]), m.pt, m.ph, m.pw, cfg->grid_w, cfg->t_max};
    c->tm_k.resize(L);
    c->tm_v.resize(L);
    for (int l = 0; l < L; ++l) {
      // K/V rings: [H][d/64][cap][64], mapped as H*d/64 planes of cap x 64
      const int planes = cfg->heads * (cfg->head_dim / 64);
      if (rc_status st = make_map(&c->tm_k[l], c->kc[l], 64, m.cap, planes, m.cap)) return st;
      if (rc_status st = make_map(&c->tm_v[l], c->vc[l], 64, m.cap, planes, m.cap)) return st;
    }
    if (m.pt > 0 && 2 * m.pt <= 64) {
      c->ip_ct = (2 * m.pt + 7) / 8;
      c->ip_rows = rc::inplace_box_rows(cfg->frame_seqlen);
      c->tm_kt.resize(L);
      const int planes = cfg->heads * (cfg->head_dim / 64);
      for (int l = 0; l < L; ++l)
        if (rc_status st = make_map(&c->tm_kt[l], c->kc[l], 64, m.cap, planes, m.cap, 8 * c->ip_ct, c->ip_rows,
                                    false))
          return st;
    }
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_err(e, "cache init");
  }
  *out_handle = c.release();
  return RC_OK;
}

rc_status rc_cache_destroy(void* handle) {
  delete static_cast<Cache*>(handle);
  return RC_OK;
}

rc_status rc_reindex(void* handle, rc_policy policy, int t_delta, unsigned flags, void* stream) {
  (void)stream;
  if (rc_status st = check_handle(handle)) return st;
  Cache* c = static_cast<Cache*>(handle);
  if (policy != c->cfg.policy) return set_err(RC_EINVAL, "policy differs from the cache's policy");
  std::string err;
  if (rc_status st = c->engine->Reindex(t_delta, flags, &err)) return set_err(st, err);
  return RC_OK;
}

rc_status rc_step(void* handle, int layer, const void* q, const void* k_new, const void* v_new, int frame_start,
                  int n_frames, rc_policy policy, void* out, float* lse, float* scores, int32_t* topc, int C,
                  void* stream) {
  if (rc_status st = check_handle(handle)) return st;
  Cache* c = static_cast<Cache*>(handle);
  const rc_config& cfg = c->cfg;
  if (policy != cfg.policy) return set_err(RC_EINVAL, "policy differs from the cache's policy");
  if (C < 0 || (C > 0 && !topc) || (topc && C == 0)) return set_err(RC_EINVAL, "topc needs C > 0");
  if (rc_status st = check_device(c)) return st;
  if (c->device) {
    if (!q || !k_new || !v_new || !out) return set_err(RC_EINVAL, "null tensor");
    for (const void* ptr : {q, k_new, v_new, (const void*)out})
      if (reinterpret_cast<uintptr_t>(ptr) % 16) return set_err(RC_EINVAL, "tensors must be 16-byte aligned");
  } else if (q || k_new || v_new || out || lse || scores || topc) {
    return set_err(RC_EINVAL, "a host-only handle takes no tensors");
  }
  rc::StepPlan plan;
  std::string err;
  if (rc_status st = c->engine->Step(layer, frame_start, n_frames, &plan, &err)) return set_err(st, err);
  if ((int)c->last_cand.size() < cfg.layers) c->last_cand.resize(cfg.layers);
  c->last_cand[layer].clear();
  for (auto& cf : plan.cand) c->last_cand[layer].emplace_back(cf.slot, cf.lpos);
  if (!c->device) return RC_OK;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const MemPlan& m = c->mp;
  const int F = cfg.frame_seqlen, H = cfg.heads, d = cfg.head_dim;
  const int Nq = n_frames * F;

  // Relax Forcing: the chunk's frame descriptors, then (pool over K frames) the selection
  const bool rf_policy = cfg.policy == RC_RELAX_FORCING;
  if (rf_policy) {
    rc::RfDescParams dp{};
    dp.k = static_cast<const uint16_t*>(k_new);
    dp.desc_cur = c->rf_cur;
    dp.n_frames = n_frames;
    dp.F = F;
    dp.H = H;
    dp.d = d;
    Timed tm(c->prof, RC_KERNEL_COMPACT, s, 0.0, (double)n_frames * F * H * d * 2);
    if (cudaError_t e = rc::launch_rf_desc(dp, s)) return cuda_err(e, "descriptor launch");
  }
  const int vslots_ring = cfg.sink_frames + cfg.window_frames;
  const int region_frames = c->engine->df_budget() / F;  // K for Relax Forcing
  if (rf_policy && !plan.repeat) {  // no pool scores unless this chunk selects
    if (cudaError_t e = cudaMemsetAsync(c->rf_pool[layer] + RC_MAX_SLOTS, 0, 4, s)) return cuda_err(e, "memset");
  }
  if (rf_policy && plan.df.use_sel) {
    const rc::DfCompact& df = plan.df;
    rc::RfSelectParams sp{};
    sp.desc = c->rf_desc[layer];
    sp.desc_cur = c->rf_cur;
    sp.n_pool = df.n_old / F + df.n_e;
    for (int v = 0; v < df.n_old / F; ++v) sp.pool_vslot[v] = vslots_ring + df.src_buf * region_frames + v;
    for (int e = 0; e < df.n_e; ++e) sp.pool_vslot[df.n_old / F + e] = df.e_slot[e];
    sp.n_tail = df.n_tail_kept;
    for (int t = 0; t < df.n_tail_kept; ++t) sp.tail_vslot[t] = df.tail_slot[t];
    sp.n_cur = n_frames;
    sp.K = region_frames;
    sp.F = F;
    sp.H = H;
    sp.d = d;
    sp.weight = (float)cfg.rf_weight;
    sp.sel = c->df_sel[layer];
    sp.pool_scores = c->rf_pool[layer];
    sp.n_scored = reinterpret_cast<int*>(c->rf_pool[layer] + RC_MAX_SLOTS);
    Timed tm(c->prof, RC_KERNEL_COMPACT, s, 0.0, 0.0);
    if (cudaError_t e = rc::launch_rf_select(sp, s)) return cuda_err(e, "frame selection launch");
  }

  // MemRoPE: fold the frames leaving the window into the memories (before the
  // append reuses their slots) and place both memory frames at their times
  if (plan.mem.active) {
    const rc::MemUpdate& mu = plan.mem;
    rc::MemUpdateParams up{};
    up.kc = c->kc[layer];
    up.vc = c->vc[layer];
    up.raw_k = c->rawk[layer];
    up.mem = c->mem_state[layer];
    up.H = H;
    up.d = d;
    up.F = F;
    up.cap = m.cap;
    up.raw_cap = m.raw_frames * F;
    up.n_e = mu.n_e;
    for (int e = 0; e < mu.n_e; ++e) up.e_slot[e] = mu.e_slot[e];
    up.initialised = mu.initialised ? 1 : 0;
    up.a[0] = (float)cfg.mr_alpha_long;
    up.b[0] = (float)(1.0 - cfg.mr_alpha_long);
    up.a[1] = (float)cfg.mr_alpha_short;
    up.b[1] = (float)(1.0 - cfg.mr_alpha_short);
    up.tau[0] = mu.tau[0];
    up.tau[1] = mu.tau[1];
    up.row0 = (cfg.sink_frames + cfg.window_frames) * F;
    up.rt = c->rt;
    // per evicted frame: raw key + value read; state read + written; two memory rows written
    const double bytes = (double)F * H * d * (mu.n_e * 2.0 * 2 + 2 * 2 * 4 * 2 + 2 * 2 * 2);
    Timed tm(c->prof, RC_KERNEL_COMPACT, s, 0.0, bytes);
    if (cudaError_t e = rc::launch_mem_update(up, s)) return cuda_err(e, "memory update launch");
  }

  // K7: Deep / Relax Forcing region gather (before the append reuses the leaving frames' slots)
  if (plan.df.active) {
    const rc::DfCompact& df = plan.df;
    rc::DfCompactParams cp{};
    cp.kc = c->kc[layer];
    cp.vc = c->vc[layer];
    cp.raw_k = c->rawk[layer];
    const int budget = c->engine->df_budget();
    cp.meta_src = c->df_meta[layer] + (size_t)df.src_buf * budget;
    cp.meta_dst = c->df_meta[layer] + (size_t)df.dst_buf * budget;
    cp.sel = df.use_sel ? c->df_sel[layer] : nullptr;
    cp.H = H;
    cp.d = d;
    cp.F = F;
    cp.cap = m.cap;
    cp.src_row0 = df.src_row0;
    cp.dst_row0 = df.dst_row0;
    cp.n_old = df.n_old;
    cp.n_new = df.n_new;
    cp.n_e = df.n_e;
    for (int e = 0; e < df.n_e; ++e) {
      cp.e_slot[e] = df.e_slot[e];
      cp.e_frame[e] = df.e_frame[e];
    }
    cp.tau_new0 = df.tau_new0;
    cp.keep_time = df.keep_time ? 1 : 0;
    cp.desc = rf_policy ? c->rf_desc[layer] : nullptr;
    cp.src_vslot0 = vslots_ring + df.src_buf * region_frames;
    cp.dst_vslot0 = vslots_ring + df.dst_buf * region_frames;
    cp.rt = c->rt;
    // raw key read + rotated key, raw key and value written, value read: 5 rows of d bf16
    // (a Relax Forcing frame move: key and value read and written, 4 rows)
    Timed tm(c->prof, RC_KERNEL_COMPACT, s, 0.0, (df.keep_time ? 4.0 : 5.0) * df.n_new * H * d * 2);
    if (cudaError_t e = rc::launch_df_compact(cp, s)) return cuda_err(e, "compact launch");
  }

  // K2: re-rotation jobs (before the append; they touch other slots). In-place
  // time deltas go to the TMA-staged kernel, rotate-copies to the other; the
  // jobs of one step target distinct slots.
  std::vector<const rc::Job*> inplace, rotcopy;
  for (const rc::Job& jb : plan.jobs) (jb.mode == rc::kInPlace && !c->tm_kt.empty() ? inplace : rotcopy).push_back(&jb);
  for (size_t j0 = 0; j0 < inplace.size(); j0 += rc::kMaxJobs) {
    rc::InplaceParams ip;
    std::memset(&ip, 0, sizeof(ip));
    ip.tm = c->tm_kt[layer];
    ip.kc = c->kc[layer];
    ip.tab_t = c->rt.t;
    ip.status = c->status;
    ip.pt = m.pt;
    ip.ct = c->ip_ct;
    ip.planes = d / 64;
    ip.F = F;
    ip.H = H;
    ip.cap = m.cap;
    ip.R = c->ip_rows;
    ip.tiles_per_head = (F + c->ip_rows - 1) / c->ip_rows;
    ip.n_jobs = (int)std::min<size_t>(rc::kMaxJobs, inplace.size() - j0);
    for (int j = 0; j < ip.n_jobs; ++j) {
      ip.slot[j] = inplace[j0 + j]->dst_slot;
      ip.delta[j] = inplace[j0 + j]->delta;
    }
    // the time pairs of every row read and written: 2 F H (2 pt) x 2 B per job
    Timed tm(c->prof, RC_KERNEL_REROTATE, s, 0.0, (double)ip.n_jobs * F * H * 2 * (2 * m.pt) * 2);
    if (cudaError_t e = rc::launch_rerotate_inplace(ip, s)) return cuda_err(e, "in-place rerotate launch");
  }
  for (size_t j0 = 0; j0 < rotcopy.size(); j0 += rc::kMaxJobs) {
    rc::RerotateParams rp{};
    rp.kc = c->kc[layer];
    rp.vc = c->vc[layer];
    rp.raw_k = c->rawk[layer];
    rp.raw_v = c->rawv[layer];
    rp.H = H;
    rp.d = d;
    rp.F = F;
    rp.cap = m.cap;
    rp.raw_cap = m.raw_frames * F;
    rp.n_jobs = (int)std::min<size_t>(rc::kMaxJobs, rotcopy.size() - j0);
    for (int j = 0; j < rp.n_jobs; ++j) {
      const rc::Job& jb = *rotcopy[j0 + j];
      rp.job[j] = rc::RerotateJob{jb.dst_slot, jb.mode, jb.src_frame, jb.sigma, jb.delta, jb.copy_v};
    }
    rp.rt = c->rt;
    double bytes = 0;
    for (int j = 0; j < rp.n_jobs; ++j) {
      const rc::RerotateJob& jb = rp.job[j];
      const double rows = (double)F * H;
      bytes += jb.mode == 1 ? rows * 2 * (2 * m.pt) * 2 : rows * 2 * d * 2 * (jb.copy_v ? 2 : 1);
    }
    Timed tm(c->prof, RC_KERNEL_REROTATE, s, 0.0, bytes);
    if (cudaError_t e = rc::launch_rerotate(rp, s)) return cuda_err(e, "rerotate launch");
  }

  // K1: fused RoPE + append
  rc::AppendParams ap{};
  ap.q = static_cast<const uint16_t*>(q);
  ap.k = static_cast<const uint16_t*>(k_new);
  ap.v = static_cast<const uint16_t*>(v_new);
  ap.q_rot = c->qrot;
  ap.kc = c->kc[layer];
  ap.vc = c->vc[layer];
  ap.raw_k = c->rawk[layer];
  ap.raw_v = c->rawv[layer];
  ap.n_tok = Nq;
  ap.H = H;
  ap.d = d;
  ap.F = F;
  ap.cap = m.cap;
  ap.q_stride = m.q_stride;
  ap.raw_cap = m.raw_frames * F;
  ap.n_frames = n_frames;
  for (int r = 0; r < n_frames; ++r) {
    ap.slot[r] = plan.append[r].slot;
    ap.sigma[r] = plan.append[r].sigma;
    ap.raw_frame[r] = plan.append[r].raw_frame;
  }
  ap.rt = c->rt;
  {
    double bytes = 6.0 * Nq * H * d * 2;
    for (int r = 0; r < n_frames; ++r)
      if (ap.raw_frame[r] >= 0) bytes += (double)F * H * d * 2 * (ap.raw_v ? 2 : 1);
    Timed tm(c->prof, RC_KERNEL_APPEND, s, 0.0, bytes);
    if (cudaError_t e = rc::launch_append(ap, s)) return cuda_err(e, "append launch");
  }
  if (rf_policy) {  // the chunk's descriptors go with its frames' slots
    const size_t fb = (size_t)H * d * 4;
    for (int r = 0; r < n_frames; ++r)
      if (cudaError_t e = cudaMemcpyAsync(c->rf_desc[layer] + (size_t)ap.slot[r] * H * d, c->rf_cur + (size_t)r * H * d,
                                          fb, cudaMemcpyDeviceToDevice, s))
        return cuda_err(e, "descriptor copy");
  }

  // K4: attention
  if (c->tm_q_rows != Nq) {
    if (rc_status st = make_map(&c->tm_q, c->qrot, d, Nq, H, m.q_stride)) return st;
    c->tm_q_rows = Nq;
  }
  const bool df_policy = cfg.policy == RC_DEEP_FORCING;
  const bool want_scores = scores || topc || df_policy;
  float* lse_buf = lse ? lse : (want_scores ? c->lse_scratch : nullptr);
  rc::AttnParams at;
  std::memset(&at, 0, sizeof(at));
  at.tm_q = c->tm_q;
  at.tm_k = c->tm_k[layer];
  at.tm_v = c->tm_v[layer];
  at.out = static_cast<uint16_t*>(out);
  at.lse = lse_buf;
  at.status = c->status;
  {
    // KV tiles each 256-query pair walks: the runs whose mask class the pair
    // reaches, each cut into 128-token tiles (the kernels' tile walk)
    const int NP = (Nq + 255) / 256;
    at.n_pairs = NP;
    if (NP <= rc::kMaxPairs) {
      at.pair_prefix[0] = 0;
      for (int q = 0; q < NP; ++q) {
        const int q_last = std::min((q + 1) * 256, Nq) - 1;
        const int rq_hi = (q_last / F) / cfg.mask_block_frames;
        int t = 0;
        for (const rc::Segment& g : plan.segs)
          if (g.rank < 0 || g.rank <= rq_hi) t += (g.len + 127) / 128;
        at.pair_prefix[q + 1] = at.pair_prefix[q] + t;
      }
    }
    // persistent grid (whole-unit rounds, then stream-K over the remainder)
    // when there are more (head, query pair) units than SMs
    const int units = NP * H;
    const int G = std::min(std::min(c->sm_count, rc::kMaxPersistentCtas), units);
    const bool split = c->part_o != nullptr && units > G && NP <= rc::kMaxPairs;
    at.part_o = split ? c->part_o : nullptr;
    at.part_lse = split ? c->part_lse : nullptr;
    at.n_ctas = split ? G : units;
    if (split) {
      // stream-K ranges that level the work: CTA c ran round units c, c + G, ...;
      // give it the share of the remainder that brings it to the average
      const long long T_head = at.pair_prefix[NP];
      auto cum = [&](long long v) { return (v / NP) * T_head + at.pair_prefix[v % NP]; };
      auto len = [&](long long u) { return (long long)at.pair_prefix[u % NP + 1] - at.pair_prefix[u % NP]; };
      const long long rounds = units / G;
      const long long base = cum(rounds * G), W_rem = cum(units) - base;
      std::vector<double> want(G);
      double total = (double)W_rem, wsum = 0;
      for (int cc = 0; cc < G; ++cc) {
        long long rt = 0;
        for (long long r = 0; r < rounds; ++r) rt += len(cc + r * G);
        want[cc] = (double)rt;
        total += (double)rt;
      }
      for (int cc = 0; cc < G; ++cc) {
        want[cc] = std::max(0.0, total / G - want[cc]);
        wsum += want[cc];
      }
      double acc = 0;
      for (int cc = 0; cc <= G; ++cc) {
        at.sk_start[cc] = (int)(base + (wsum > 0 ? (long long)std::floor(W_rem * acc / wsum)
                                                  : (long long)cc * W_rem / G));
        if (cc < G) acc += wsum > 0 ? want[cc] : 0;
      }
      at.sk_start[G] = (int)(base + W_rem);
    }
  }
  at.Nq = Nq;
  at.H = H;
  at.F = F;
  at.mask_block = cfg.mask_block_frames;
  at.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
  if (plan.segs.size() > (size_t)rc::kMaxSegs) return set_err(RC_ERANGE, "too many KV segments");
  at.n_segs = (int)plan.segs.size();
  for (int i = 0; i < at.n_segs; ++i)
    at.seg[i] = rc::KvSegment{plan.segs[i].tok_start, plan.segs[i].len, plan.segs[i].rank};
  {
    // algorithmic FLOPs: 4 d H per visible (query, key) pair
    const rc::LayerState& Ls = c->engine->layer(layer);
    double n_hist = Ls.comp_n;  // the Deep / Relax Forcing region, always visible
    for (const rc::Kept& k : Ls.kept) n_hist += k.region != rc::kCur ? F : 0;
    double pairs = 0;
    for (int r = 0; r < n_frames; ++r) {
      int vis = 0;
      for (int r2 = 0; r2 < n_frames; ++r2) vis += (r2 / cfg.mask_block_frames) <= (r / cfg.mask_block_frames);
      pairs += (double)F * (n_hist + (double)vis * F);
    }
    {
      Timed tm(c->prof, RC_KERNEL_ATTENTION, s, 4.0 * d * H * pairs, 0.0);
      if (cudaError_t e = rc::launch_attention(at, d, s)) return cuda_err(e, "attention launch");
    }
    if (at.part_o && (at.n_pairs * H) % at.n_ctas != 0) {
      Timed tm(c->prof, RC_KERNEL_COMBINE, s, 0.0, (double)2 * at.n_ctas * 256 * (d + 1) * 4);
      if (cudaError_t e = rc::launch_attention_combine(at, d, s)) return cuda_err(e, "combine launch");
    }
  }

  // K6: scores over history tokens + top-C
  if (want_scores) {
    std::vector<int> slots;
    for (auto& cf : plan.cand) slots.push_back(cf.slot);
    std::sort(slots.begin(), slots.end());
    rc::ScoreParams sp;
    std::memset(&sp, 0, sizeof(sp));
    for (size_t i = 0; i < slots.size();) {
      size_t j = i + 1;
      while (j < slots.size() && slots[j] == slots[j - 1] + 1) ++j;
      if (sp.n_segs == rc::kMaxSegs) return set_err(RC_ERANGE, "too many candidate segments");
      sp.seg[sp.n_segs++] = rc::KvSegment{slots[i] * F, (int)(j - i) * F, -1};
      i = j;
    }
    if (cudaError_t e = cudaMemsetAsync(c->score_phys, 0, (size_t)m.cap * 4, s)) return cuda_err(e, "memset");
    sp.tm_q = c->tm_q;
    sp.tm_k = c->tm_k[layer];
    sp.lse = lse_buf;
    sp.score_phys = c->score_phys;
    sp.status = c->status;
    sp.Nq = Nq;
    sp.H = H;
    sp.scale_log2 = at.scale_log2;
    sp.n_pairs = (Nq + 255) / 256;
    sp.tiles = 0;
    for (int i = 0; i < sp.n_segs; ++i) sp.tiles += (sp.seg[i].len + 127) / 128;
    {
      const long long work = (long long)H * sp.n_pairs * sp.tiles;
      sp.n_ctas = (int)std::min<long long>(c->sm_count, work);
    }
    {
      Timed tm(c->prof, RC_KERNEL_SCORES, s, 2.0 * d * H * Nq * (double)plan.cand.size() * F, 0.0);
      if (cudaError_t e = rc::launch_scores(sp, d, s)) return cuda_err(e, "scores launch");
    }
    rc::TopCParams tp;
    std::memset(&tp, 0, sizeof(tp));
    tp.score_phys = c->score_phys;
    tp.scores_out = scores ? scores : c->score_logical;
    tp.topc = topc;
    tp.C = C;
    tp.F = F;
    tp.n_cand_frames = (int)plan.cand.size();
    for (size_t i = 0; i < plan.cand.size(); ++i) {
      tp.cand_slot[i] = plan.cand[i].slot;
      tp.cand_lpos[i] = plan.cand[i].lpos;
    }
    if (scores || topc) {
      Timed tm(c->prof, RC_KERNEL_TOPC, s, 0.0, (double)plan.cand.size() * F * 4 * 2);
      if (cudaError_t e = rc::launch_topc(tp, s)) return cuda_err(e, "topc launch");
    }
    // Deep Forcing: the next new chunk's region, chosen now from this step's scores
    if (df_policy && plan.df_select) {
      rc::TopCParams sp2;
      std::memset(&sp2, 0, sizeof(sp2));
      sp2.score_phys = c->score_phys;
      sp2.scores_out = c->score_logical;
      sp2.topc = c->df_sel[layer];
      sp2.C = c->engine->df_budget();
      sp2.F = F;
      sp2.n_cand_frames = (int)plan.df_pool.size();
      for (size_t i = 0; i < plan.df_pool.size(); ++i) {
        sp2.cand_slot[i] = plan.df_pool[i].slot;
        sp2.cand_lpos[i] = plan.df_pool[i].lpos;
      }
      Timed tm(c->prof, RC_KERNEL_TOPC, s, 0.0, (double)plan.df_pool.size() * F * 4 * 2);
      if (cudaError_t e = rc::launch_topc(sp2, s)) return cuda_err(e, "pool top-C launch");
    }
  }
  return RC_OK;
}

rc_status rc_select_topc(void* handle, int layer, const float* scores, int C, int32_t* topc, void* stream) {
  if (rc_status st = check_handle(handle)) return st;
  Cache* c = static_cast<Cache*>(handle);
  if (!c->device) return set_err(RC_EINVAL, "rc_select_topc needs a device handle");
  if (rc_status st = check_device(c)) return st;
  if (layer < 0 || layer >= c->cfg.layers) return set_err(RC_EINVAL, "layer out of range");
  if (!scores || !topc || C <= 0) return set_err(RC_EINVAL, "scores, topc and C > 0 are required");
  if ((int)c->last_cand.size() <= layer) return set_err(RC_ESTATE, "no step has run on this layer");
  const auto& cand = c->last_cand[layer];
  rc::TopCParams tp;
  std::memset(&tp, 0, sizeof(tp));
  tp.score_phys = scores;  // already logical: candidate frame i sits at [i F, i F + F)
  tp.scores_out = c->score_logical;
  tp.topc = topc;
  tp.C = C;
  tp.F = c->cfg.frame_seqlen;
  tp.n_cand_frames = (int)cand.size();
  for (size_t i = 0; i < cand.size(); ++i) {
    tp.cand_slot[i] = (int)i;
    tp.cand_lpos[i] = cand[i].second;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Timed tm(c->prof, RC_KERNEL_TOPC, s, 0.0, (double)cand.size() * tp.F * 4 * 2);
  if (cudaError_t e = rc::launch_topc(tp, s)) return cuda_err(e, "topc launch");
  return RC_OK;
}

// rc_step with its per-call scratch (rotated queries, log-sum-exps, token
// score work buffers) placed in the library's static device array instead of
// the caller's block: the handle's scratch pointers and query descriptor are
// pointed there for the duration of one rc_step and restored afterwards.
rc_status rc_step_noalloc(void* handle, int layer, const void* q, const void* k_new, const void* v_new,
                          int frame_start, int n_frames, rc_policy policy, void* out, float* lse,
                          float* scores, int32_t* topc, int C, void* stream) {
  if (rc_status st = check_handle(handle)) return st;
  Cache* c = static_cast<Cache*>(handle);
  if (!c->device) return set_err(RC_EINVAL, "rc_step_noalloc needs a device handle");
  if (rc_status st = check_device(c)) return st;
  const rc_config& cfg = c->cfg;
  const MemPlan& m = c->mp;
  const size_t q_bytes = align_up((size_t)cfg.heads * m.q_stride * cfg.head_dim * 2);
  const size_t lse_bytes = align_up((size_t)cfg.heads * m.q_stride * 4);
  const size_t score_bytes = align_up((size_t)m.cap * 4);
  const size_t need = q_bytes + lse_bytes + 2 * score_bytes;
  void* base = nullptr;
  size_t have = 0;
  if (cudaError_t e = rc::static_step_scratch(&base, &have)) return cuda_err(e, "static scratch lookup");
  if (need > have)
    return set_err(RC_ERANGE, "rc_step_noalloc needs " + std::to_string(need) +
                                  " bytes of step scratch; the static maximum is " + std::to_string(have) +
                                  " (heads * chunk_frames * frame_seqlen * head_dim * 2 plus scores)");
  uint8_t* b = static_cast<uint8_t*>(base);
  uint16_t* const saved_q = c->qrot;
  float* const saved_lse = c->lse_scratch;
  float* const saved_phys = c->score_phys;
  float* const saved_logical = c->score_logical;
  float* const saved_part_o = c->part_o;
  float* const saved_part_lse = c->part_lse;
  const CUtensorMap saved_map = c->tm_q;
  const int saved_rows = c->tm_q_rows;
  c->part_o = nullptr;  // one CTA per (head, query pair): no partial rows to stage
  c->part_lse = nullptr;
  c->qrot = reinterpret_cast<uint16_t*>(b);
  c->lse_scratch = reinterpret_cast<float*>(b + q_bytes);
  c->score_phys = reinterpret_cast<float*>(b + q_bytes + lse_bytes);
  c->score_logical = reinterpret_cast<float*>(b + q_bytes + lse_bytes + score_bytes);
  c->tm_q_rows = -1;  // re-encode the query descriptor over the static array
  const rc_status st = rc_step(handle, layer, q, k_new, v_new, frame_start, n_frames, policy, out, lse,
                               scores, topc, C, stream);
  c->qrot = saved_q;
  c->lse_scratch = saved_lse;
  c->score_phys = saved_phys;
  c->score_logical = saved_logical;
  c->part_o = saved_part_o;
  c->part_lse = saved_part_lse;
  c->tm_q = saved_map;
  c->tm_q_rows = saved_rows;
  return st;
}

rc_status rc_get_state(const void* handle, int layer, rc_state* out) {
  if (rc_status st = check_handle(handle)) return st;
  if (!out) return set_err(RC_EINVAL, "null state");
  const Cache* c = static_cast<const Cache*>(handle);
  if (layer < 0 || layer >= c->cfg.layers) return set_err(RC_EINVAL, "layer out of range");
  const rc::LayerState& L = c->engine->layer(layer);
  std::memset(out, 0, sizeof(*out));
  out->n_kept = (int)L.kept.size();
  out->frames_committed = L.end;
  out->chunk_start = L.cur_start;
  out->chunk_frames = L.cur_n;
  out->valid_tokens = (int)L.kept.size() * c->cfg.frame_seqlen;
  out->shift = L.shift;
  out->n_jobs = L.n_jobs;
  int nc = 0;
  for (size_t e = 0; e < L.kept.size(); ++e) {
    const rc::Kept& k = L.kept[e];
    out->kept[e] = rc_frame_state{k.content, k.tau, k.region, k.rank, L.kept_slot[e], k.tau + L.shift};
    if (k.region == rc::kHist) nc += c->cfg.frame_seqlen;
  }
  out->n_candidates = nc + L.comp_n;
  out->valid_tokens += L.comp_n;
  out->comp_tokens = L.comp_n;
  out->comp_tau0 = L.comp_tau0;
  out->comp_row0 = (c->cfg.sink_frames + c->cfg.window_frames) * c->cfg.frame_seqlen +
                   L.comp_buf * c->engine->df_budget();
  out->n_evicted = (int)L.evicted.size();
  for (size_t i = 0; i < L.evicted.size() && i < RC_MAX_SLOTS; ++i) out->evicted[i] = L.evicted[i];
  return RC_OK;
}

rc_status rc_comp_tokens(void* handle, int layer, int32_t* frame, int32_t* tok, void* stream) {
  if (rc_status st = check_handle(handle)) return st;
  Cache* c = static_cast<Cache*>(handle);
  if ((c->cfg.policy != RC_DEEP_FORCING && c->cfg.policy != RC_RELAX_FORCING) || !c->device)
    return set_err(RC_EINVAL, "rc_comp_tokens needs a Deep or Relax Forcing device handle");
  if (layer < 0 || layer >= c->cfg.layers) return set_err(RC_EINVAL, "layer out of range");
  if (rc_status st = check_device(c)) return st;
  const rc::LayerState& L = c->engine->layer(layer);
  if (L.comp_n == 0) return RC_OK;
  if (!frame || !tok) return set_err(RC_EINVAL, "null output array");
  std::vector<int2> meta(L.comp_n);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int2* src = c->df_meta[layer] + (size_t)L.comp_buf * c->engine->df_budget();
  if (cudaError_t e = cudaMemcpyAsync(meta.data(), src, meta.size() * sizeof(int2), cudaMemcpyDeviceToHost, s))
    return cuda_err(e, "region metadata copy");
  if (cudaError_t e = cudaStreamSynchronize(s)) return cuda_err(e, "stream sync");
  for (int i = 0; i < L.comp_n; ++i) {
    frame[i] = meta[i].x;
    tok[i] = meta[i].y;
  }
  return RC_OK;
}

rc_status rc_pool_scores(void* handle, int layer, float* scores, int32_t* n, void* stream) {
  if (rc_status st = check_handle(handle)) return st;
  Cache* c = static_cast<Cache*>(handle);
  if (c->cfg.policy != RC_RELAX_FORCING || !c->device)
    return set_err(RC_EINVAL, "rc_pool_scores needs a Relax Forcing device handle");
  if (layer < 0 || layer >= c->cfg.layers) return set_err(RC_EINVAL, "layer out of range");
  if (rc_status st = check_device(c)) return st;
  if (!scores || !n) return set_err(RC_EINVAL, "null output");
  std::vector<float> buf(RC_MAX_SLOTS + 1);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaError_t e = cudaMemcpyAsync(buf.data(), c->rf_pool[layer], buf.size() * 4, cudaMemcpyDeviceToHost, s))
    return cuda_err(e, "pool score copy");
  if (cudaError_t e = cudaStreamSynchronize(s)) return cuda_err(e, "stream sync");
  int cnt = 0;
  std::memcpy(&cnt, &buf[RC_MAX_SLOTS], 4);
  *n = cnt;
  for (int i = 0; i < cnt && i < RC_MAX_SLOTS; ++i) scores[i] = buf[i];
  return RC_OK;
}

rc_status rc_device_status(void* handle, void* stream) {
  if (rc_status st = check_handle(handle)) return st;
  Cache* c = static_cast<Cache*>(handle);
  if (!c->device) return RC_OK;
  if (rc_status st = check_device(c)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaError_t e = cudaStreamSynchronize(s)) return cuda_err(e, "stream sync");
  int word = 0;
  if (cudaError_t e = cudaMemcpy(&word, c->status, 4, cudaMemcpyDeviceToHost)) return cuda_err(e, "status read");
  if (word) {
    cudaMemset(c->status, 0, 4);
    return set_err(RC_ETIMEOUT, "a device-side wait gave up (status word " + std::to_string(word) + ")");
  }
  return RC_OK;
}

rc_status rc_cache_layout(const void* handle, rc_layout* out) {
  if (rc_status st = check_handle(handle)) return st;
  if (!out) return set_err(RC_EINVAL, "null layout");
  const Cache* c = static_cast<const Cache*>(handle);
  const MemPlan& m = c->mp;
  const int nraw = raw_buffers(c->cfg);
  std::memset(out, 0, sizeof(*out));
  out->kv_layer_stride = 2 * m.kv_bytes;
  out->k_offset = m.off_kv;
  out->v_offset = m.off_kv + m.kv_bytes;
  out->raw_layer_stride = nraw * m.raw_bytes;
  out->raw_k_offset = nraw >= 1 ? m.off_raw : 0;
  out->raw_v_offset = nraw == 2 ? m.off_raw + m.raw_bytes : 0;
  out->q_offset = m.off_q;
  out->capacity = m.cap;
  out->raw_frames = m.raw_frames;
  out->total = m.total;
  return RC_OK;
}

rc_status rc_watchdog_selftest(void* handle, unsigned limit_us, void* stream) {
  if (rc_status st = check_handle(handle)) return st;
  Cache* c = static_cast<Cache*>(handle);
  if (!c->device) return set_err(RC_EINVAL, "host-only handle");
  if (rc_status st = check_device(c)) return st;
  if (limit_us == 0 || limit_us > 5000000u) return set_err(RC_EINVAL, "limit_us must be in (0, 5e6]");
  if (cudaError_t e = rc::launch_watchdog_selftest(c->status, limit_us, static_cast<cudaStream_t>(stream)))
    return cuda_err(e, "watchdog launch");
  return RC_OK;
}

rc_status rc_profile_begin(void* handle, int max_launches) {
  if (rc_status st = check_handle(handle)) return st;
  Cache* c = static_cast<Cache*>(handle);
  if (!c->device) return set_err(RC_EINVAL, "host-only handle");
  if (rc_status st = check_device(c)) return st;
  if (max_launches < 0 || max_launches > (1 << 20)) return set_err(RC_EINVAL, "max_launches out of range");
  Profiler& p = c->prof;
  p.release();
  p.ev.resize(2 * (size_t)max_launches);
  for (auto& e : p.ev)
    if (cudaError_t err = cudaEventCreate(&e)) {
      p.ev.clear();
      return cuda_err(err, "cudaEventCreate");
    }
  p.kind.assign(max_launches, 0);
  p.max = max_launches;
  p.used = 0;
  std::fill(p.launches, p.launches + RC_KERNEL_KINDS, 0);
  std::fill(p.flops, p.flops + RC_KERNEL_KINDS, 0.0);
  std::fill(p.bytes, p.bytes + RC_KERNEL_KINDS, 0.0);
  p.on = true;
  return RC_OK;
}

rc_status rc_profile_end(void* handle, rc_profile* out) {
  if (rc_status st = check_handle(handle)) return st;
  if (!out) return set_err(RC_EINVAL, "null profile");
  Cache* c = static_cast<Cache*>(handle);
  Profiler& p = c->prof;
  std::memset(out, 0, sizeof(*out));
  for (int k = 0; k < RC_KERNEL_KINDS; ++k) {
    out->launches[k] = p.launches[k];
    out->flops[k] = p.flops[k];
    out->bytes[k] = p.bytes[k];
  }
  for (int i = 0; i < p.used; ++i) {
    if (cudaError_t e = cudaEventSynchronize(p.ev[2 * i + 1])) {
      p.release();
      return cuda_err(e, "event sync");
    }
    float ms = 0.f;
    cudaEventElapsedTime(&ms, p.ev[2 * i], p.ev[2 * i + 1]);
    out->ms[p.kind[i]] += ms;
    out->timed[p.kind[i]]++;
  }
  p.release();
  return RC_OK;
}

rc_status rc_rope_table(const void* handle, int axis, float* dst, size_t* count) {
  if (rc_status st = check_handle(handle)) return st;
  if (axis < 0 || axis > 2 || !count) return set_err(RC_EINVAL, "bad axis or count");
  const Cache* c = static_cast<const Cache*>(handle);
  const std::vector<float>& t = c->tab[axis];
  if (!dst) {
    *count = t.size();
    return RC_OK;
  }
  size_t n = std::min(*count, t.size());
  std::memcpy(dst, t.data(), n * 4);
  *count = n;
  return RC_OK;
}

}  // extern "C"
