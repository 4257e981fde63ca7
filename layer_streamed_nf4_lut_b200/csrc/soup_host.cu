// libsoup host side: model state, NF4 layer stack in page-locked host memory, the
// double-buffered layer streamer, per-layer forward/backward orchestration, the SFT and
// DPO steps, and the extern "C" boundary declared in include/soup.h.
//
// Streaming (rug.gal radar "Soup ... layer streaming", "En detalle"): the base stays in host
// RAM; each decoder layer is copied to one of n_layer_buffers device buffers on a side copy
// stream right before it is needed, so the copy of layer i+1 overlaps the compute of layer i.
// Fences: the compute stream waits on copy_done[b] before touching buffer b; the copy stream
// waits on buf_free[b] (recorded after the last kernel that read buffer b) before overwriting.
// The same kernels with the same launch configurations run in streamed and resident mode,
// so both produce identical bits (the pages' "difference 0.0").
#include "../../include/soup.h"
#include "common.cuh"
#include "internal.h"
#include "layer_file.h"

#include <nvtx3/nvToolsExt.h>

#include <unistd.h>

#include <chrono>
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>
#include <algorithm>
#include <mutex>
#include <unordered_map>

namespace soup {
namespace {

// ------------------------------------------------------------------ NF4 codebook
// QLoRA's 4-bit NormalFloat levels: N(0,1) quantiles at probabilities evenly spaced from
// 1 - delta to 1/2 (8 positive, 7 negative, plus 0), delta = (1/30 + 1/32)/2, scaled so the
// extremes are -1 and +1.  The inverse CDF is solved in float64 by bisection then Newton on
// Phi(x) = erfc(-x/sqrt 2)/2; the levels are rounded to float32 once.
double phi_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }
double normal_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200 && hi - lo > 1e-300; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (phi_cdf(mid) < p) lo = mid; else hi = mid;
    if (mid == lo && mid == hi) break;
  }
  double x = 0.5 * (lo + hi);
  for (int i = 0; i < 4; ++i) {
    const double f = phi_cdf(x) - p;
    const double d = std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI);
    if (d <= 0) break;
    x -= f / d;
  }
  return x;
}
void nf4_codebook_compute(float out[16]) {
  const double delta = 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
  const double start = 1.0 - delta;
  std::vector<double> v;
  const double step_pos = (0.5 - start) / 8.0;  // linspace(start, 0.5, 9)[:8]
  for (int i = 0; i < 8; ++i) v.push_back(normal_quantile(static_cast<double>(i) * step_pos + start));
  const double step_neg = (0.5 - start) / 7.0;  // -(linspace(start, 0.5, 8)[:7])
  for (int i = 0; i < 7; ++i) v.push_back(-normal_quantile(static_cast<double>(i) * step_neg + start));
  v.push_back(0.0);
  std::sort(v.begin(), v.end());
  const double mx = v.back();
  for (int i = 0; i < 16; ++i) out[i] = static_cast<float>(v[i] / mx);
}
const LUT16& codebook() {
  static LUT16 lut = [] {
    LUT16 l;
    nf4_codebook_compute(l.v);
    return l;
  }();
  return lut;
}

// ------------------------------------------------------------------ shapes and blob layout
constexpr size_t ALIGN = 256;
size_t align_up(size_t x) { return (x + ALIGN - 1) / ALIGN * ALIGN; }

struct ProjShape {
  int out, in;
};
void proj_shapes(const soup_model_config& c, ProjShape s[7]) {
  const int qd = c.n_heads * c.head_dim, kvd = c.n_kv_heads * c.head_dim;
  s[0] = {qd, c.hidden};
  s[1] = {kvd, c.hidden};
  s[2] = {kvd, c.hidden};
  s[3] = {c.hidden, qd};
  s[4] = {c.intermediate, c.hidden};
  s[5] = {c.intermediate, c.hidden};
  s[6] = {c.hidden, c.intermediate};
}

struct BlobLayout {
  size_t off[9][4];
  size_t sz[9][4];
  size_t total;
};
BlobLayout blob_layout(const soup_model_config& c) {
  BlobLayout L{};
  ProjShape s[7];
  proj_shapes(c, s);
  size_t o = 0;
  for (int p = 0; p < 7; ++p) {
    const long long n = static_cast<long long>(s[p].out) * s[p].in;
    const long long nb = (n + 63) / 64, ng = (nb + 255) / 256;
    const size_t sz[4] = {static_cast<size_t>((n + 1) / 2), static_cast<size_t>(nb), static_cast<size_t>(4 * ng), 4};
    for (int q = 0; q < 4; ++q) {
      L.off[p][q] = o;
      L.sz[p][q] = sz[q];
      o += align_up(sz[q]);
    }
  }
  for (int g = 0; g < 2; ++g) {
    L.off[7 + g][0] = o;
    L.sz[7 + g][0] = static_cast<size_t>(c.hidden) * 2;
    o += align_up(L.sz[7 + g][0]);
  }
  L.total = o;
  return L;
}

soup_status validate_cfg(const soup_model_config& c, std::string& why) {
  if (c.n_layers < 1 || c.hidden < 8 || c.n_heads < 1 || c.n_kv_heads < 1 || c.head_dim < 1 || c.intermediate < 8 ||
      c.vocab < 4 || c.lora_r < 1 || c.max_tokens < 1) {
    why = "config: sizes must be positive";
    return SOUP_ERR_INVALID_ARG;
  }
  if (!(c.rms_eps > 0.f) || !(c.rope_theta > 0.f) || !(c.lora_alpha == c.lora_alpha)) {
    why = "config: rms_eps and rope_theta must be > 0";
    return SOUP_ERR_INVALID_ARG;
  }
  if (c.mode != SOUP_RESIDENT && c.mode != SOUP_STREAMED) {
    why = "config: mode must be SOUP_RESIDENT or SOUP_STREAMED";
    return SOUP_ERR_INVALID_ARG;
  }
  if (c.mode == SOUP_STREAMED && c.n_layer_buffers < 2) {
    why = "config: streamed mode needs n_layer_buffers >= 2";
    return SOUP_ERR_INVALID_ARG;
  }
  if (c.n_heads % c.n_kv_heads != 0) {
    why = "config: n_heads must be a multiple of n_kv_heads";
    return SOUP_ERR_INVALID_ARG;
  }
  if (c.stream_source < SOUP_SOURCE_RAM || c.stream_source > SOUP_SOURCE_AUTO) {
    why = "config: stream_source must be SOUP_SOURCE_RAM, _FILE or _AUTO";
    return SOUP_ERR_INVALID_ARG;
  }
  if (c.stream_source == SOUP_SOURCE_FILE && (!c.stack_path || !c.stack_path[0])) {
    why = "config: the file source needs stack_path";
    return SOUP_ERR_INVALID_ARG;
  }
  if (c.head_dim != 64 && c.head_dim != 128) {
    why = "config: head_dim must be 64 or 128";
    return SOUP_ERR_UNSUPPORTED;
  }
  if (c.hidden % 8 || c.intermediate % 8 || c.lora_r % 8 || c.vocab % 4) {
    why = "config: hidden, intermediate, lora_r must be multiples of 8 and vocab of 4";
    return SOUP_ERR_UNSUPPORTED;
  }
  return SOUP_OK;
}

size_t lora_numel_of(const soup_model_config& c) {
  ProjShape s[7];
  proj_shapes(c, s);
  size_t per = 0;
  for (int p = 0; p < 7; ++p) per += static_cast<size_t>(c.lora_r) * (s[p].in + s[p].out);
  return per * c.n_layers;
}
// LoRA parameters of one layer (a contiguous slice of the flat buffer, starting at lora_off(c, l, 0, 0))
size_t lora_layer_numel(const soup_model_config& c) { return lora_numel_of(c) / c.n_layers; }
// offset of A_p (which=0) or B_p (which=1) of a layer in the flat LoRA buffer
size_t lora_off(const soup_model_config& c, int layer, int proj, int which) {
  ProjShape s[7];
  proj_shapes(c, s);
  size_t per = 0;
  for (int p = 0; p < 7; ++p) per += static_cast<size_t>(c.lora_r) * (s[p].in + s[p].out);
  size_t o = per * layer;
  if (which == 0) {
    for (int p = 0; p < proj; ++p) o += static_cast<size_t>(c.lora_r) * s[p].in;
  } else {
    for (int p = 0; p < 7; ++p) o += static_cast<size_t>(c.lora_r) * s[p].in;
    for (int p = 0; p < proj; ++p) o += static_cast<size_t>(c.lora_r) * s[p].out;
  }
  return o;
}

// ------------------------------------------------------------------ model
struct Saved {  // per-layer activations kept for the backward
  uint16_t *x, *n1, *qkv, *uqkv, *o, *uo, *x1, *n2, *gu, *ugu, *m, *ud;
  float *rstd1, *rstd2, *lse;
  int B = 0, S = 0, lora = 0, valid = 0;
};

struct LayerView {
  NF4Seg seg[7];
  const uint16_t* gamma[2];
};

}  // namespace
}  // namespace soup

struct soup_model {
  soup_model_config cfg{};
  soup_allocator alloc{};
  bool has_alloc = false;
  std::string err;
  soup::BlobLayout layout{};
  int qkv_cols = 0;
  float s_lora = 0.f;

  // host NF4 stack: page-locked RAM (one blob per layer), or a file streamed through
  // page-locked staging slots
  std::vector<uint8_t*> host_blob;
  std::vector<int> host_loaded;
  soup::LayerFile file;
  int use_file = 0;
  long long file_bytes0 = 0;  // file counters at the last soup_reset_stats
  double file_ms0 = 0.0;
  // device layer buffers
  std::vector<uint8_t*> dev_buf;   // resident: n_layers buffers; streamed: n_layer_buffers
  std::vector<int> buf_layer;      // which layer each buffer holds (-1: none / stale)
  std::vector<long long> buf_last; // last use tick
  std::vector<int> buf_inuse;
  std::vector<cudaEvent_t> copy_done, buf_free;
  cudaStream_t copy_stream = nullptr;
  long long tick = 0;

  // head
  const uint16_t* embed = nullptr;
  const uint16_t* final_gamma = nullptr;
  const uint16_t* lm_head = nullptr;
  // LoRA storage
  float *lora_p = nullptr, *lora_g = nullptr, *lora_m = nullptr, *lora_v = nullptr;
  uint16_t* lora_bf16 = nullptr;  // bf16 copy of the parameters: the GEMM operands
  size_t lora_n = 0;
  int lora_enabled = 1;
  int adam_t = 0;
  // Set while soup_step's backward pass runs with the optimizer on: the backward call of layer
  // i then also applies AdamW to layer i+1's LoRA slice (its gradients are complete and nothing
  // reads its parameters again this step), on the gradient side stream; lr and the bias
  // corrections come from device memory (scal + ADAM_HP_WORD) so that captured graphs replay
  // each step's values.
  int adam_in_bwd = 0;

  // activations
  std::vector<soup::Saved> saved;
  // work buffers
  uint16_t *xra = nullptr, *xrb = nullptr;  // reference-pass hidden states (DPO shared-load schedule)
  uint16_t *xa = nullptr, *xb = nullptr, *dqkv = nullptr, *dgu = nullptr, *dm = nullptr, *da = nullptr,
           *dn = nullptr, *dx1 = nullptr, *vqkv = nullptr, *vo = nullptr, *vgu = nullptr, *vd = nullptr,
           *hf = nullptr, *dh = nullptr, *dlogits = nullptr;
  float *delta = nullptr, *logits = nullptr, *rowlse = nullptr, *rowtgt = nullptr, *roww = nullptr,
        *rstdf = nullptr, *pi = nullptr, *ref = nullptr;
  int32_t* ids_dev = nullptr;
  uint8_t* mask_dev = nullptr;
  uint8_t* labels_dev = nullptr;  // KTO labels [B]
  // shared-prefix pair blocks (preference steps with share_prefix): packed ids, the targets of
  // each packed row (the last prefix row has two), their logits and row weights
  int pack_pl = 0, pack_rl = 0;  // non-zero while a packed step runs
  int32_t *pids = nullptr, *tgt1 = nullptr, *tgt2 = nullptr;
  float *rowtgt2 = nullptr, *roww2 = nullptr, *seqw = nullptr;
  // scalars: [0] loss (f32), [1] device error word (int)
  int* scal = nullptr;
  float* quant_scratch = nullptr;  // absmax scratch for the quantiser
  float* gemm_ws = nullptr;        // split-K partial tiles
  float *rope_cos = nullptr, *rope_sin = nullptr;  // [max_tokens, head_dim/2]
  size_t gemm_ws_bytes = 0;
  float* host_scal = nullptr;      // pinned staging: words 0-1 loss + error readback, 4-6 AdamW lr + bias corrections

  std::vector<void*> dev_allocs;
  // per-layer CUDA graphs of the step's layer calls (key: direction, layer, weight buffer,
  // activation buffers, shapes, LoRA flag)
  // one launch bracketed by CUDA events, and per-category totals of such launches
  struct ProfRec {
    int cat;
    cudaEvent_t a, b;
    double flops, bytes;
  };
  struct ProfCat {
    long long launches = 0;
    double ms = 0, flops = 0, bytes = 0;
  };
  struct GraphKey {
    int dir, layer, B, S, lora, pack;  // pack: shared-prefix length of a packed pair step (0: none)
    int tcat;                          // mask of the categories whose launches carry event nodes
    int adam;                          // backward call that also updates layer + 1's LoRA slice
    const void *base, *in, *out;
    bool operator==(const GraphKey& o) const { return std::memcmp(this, &o, sizeof(GraphKey)) == 0; }
  };
  struct GraphKeyHash {
    size_t operator()(const GraphKey& k) const {
      const unsigned long long* w = reinterpret_cast<const unsigned long long*>(&k);
      unsigned long long h = 1469598103934665603ull;
      for (size_t i = 0; i < sizeof(GraphKey) / 8; ++i) h = (h ^ w[i]) * 1099511628211ull;
      return static_cast<size_t>(h);
    }
  };
  struct GraphEntry {
    cudaGraphExec_t exec = nullptr;
    int seen = 0;
    long long launches = 0;
    std::vector<ProfRec> recs;  // event-record node pairs of the timed category (graph-owned events)
    int armed = 0;              // replayed since its events were last read
  };
  std::unordered_map<GraphKey, GraphEntry, GraphKeyHash> graphs;
  cudaStream_t cap_stream = nullptr;
  int use_graphs = 1;
  // low-priority stream for the LoRA weight-gradient GEMMs of a layer backward (they run
  // beside the dX GEMMs), its fork / join events and its own split-K workspace
  cudaStream_t grad_stream = nullptr;
  cudaEvent_t fork_ev = nullptr, join_ev = nullptr;
  float* gemm_ws2 = nullptr;
  size_t gemm_ws2_bytes = 0;
  int* gemm_cnt = nullptr;   // split-K tile counters of gemm_ws (zero between launches)
  int* gemm_cnt2 = nullptr;  // ... of gemm_ws2
  int concurrent_grads = 1;
  int grads_forked = 0;
  // live profile: event pairs per launch, resolved into per-category totals
  int prof = 0;
  std::vector<ProfRec> prof_pending;
  std::vector<cudaEvent_t> prof_pool;
  std::vector<ProfCat> prof_cats;
  // timed categories: event pairs around their launches in ordinary (graph-replayed) calls
  int tcat = 0;                              // bit c set: category c is timed (0: none)
  std::string tname;                         // the setting as given
  std::vector<ProfRec>* cap_recs = nullptr;  // the graph being captured collects its pairs here
  std::vector<ProfRec> tpending;             // pairs of eager launches and layer copies
  std::vector<ProfCat> taccs;                // per category
  soup_stats stats{};
  long long launches_at_reset = 0;
};

namespace soup {
namespace {

#define SOUP_CK(call)                                                                \
  do {                                                                               \
    cudaError_t e_ = (call);                                                         \
    if (e_ != cudaSuccess) {                                                         \
      m->err = std::string(#call) + ": " + cudaGetErrorString(e_);                   \
      return SOUP_ERR_CUDA;                                                          \
    }                                                                                \
  } while (0)

#define SOUP_TRY(st)                       \
  do {                                     \
    soup_status s_ = (st);                 \
    if (s_ != SOUP_OK) return s_;          \
  } while (0)

void* dev_alloc(soup_model* m, size_t bytes) {
  bytes = align_up(bytes ? bytes : ALIGN);
  void* p = nullptr;
  if (m->has_alloc) {
    p = m->alloc.alloc(bytes, m->alloc.user);
  } else if (cudaMalloc(&p, bytes) != cudaSuccess) {
    p = nullptr;
  }
  if (p) {
    m->dev_allocs.push_back(p);
    m->stats.device_bytes += static_cast<long long>(bytes);
  }
  return p;
}

template <class T>
soup_status alloc_into(soup_model* m, T*& out, size_t count) {
  out = static_cast<T*>(dev_alloc(m, count * sizeof(T)));
  if (!out) {
    m->err = "device allocation failed";
    return SOUP_ERR_OOM;
  }
  return SOUP_OK;
}

unsigned long long wait_limit_ms() {
  const char* e = std::getenv("SOUP_WAIT_TIMEOUT_MS");
  if (e) {
    const long long v = std::atoll(e);
    if (v > 0) return static_cast<unsigned long long>(v);
  }
  return 600000ull;
}

// Bounded host wait on all work queued on `st` so far.
soup_status wait_stream(soup_model* m, cudaStream_t st) {
  cudaEvent_t ev;
  SOUP_CK(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
  cudaError_t e = cudaEventRecord(ev, st);
  if (e != cudaSuccess) {
    cudaEventDestroy(ev);
    m->err = std::string("cudaEventRecord: ") + cudaGetErrorString(e);
    return SOUP_ERR_CUDA;
  }
  const auto t0 = std::chrono::steady_clock::now();
  const unsigned long long lim = wait_limit_ms();
  for (;;) {
    e = cudaEventQuery(ev);
    if (e == cudaSuccess) break;
    if (e != cudaErrorNotReady) {
      cudaEventDestroy(ev);
      m->err = std::string("stream error: ") + cudaGetErrorString(e);
      return SOUP_ERR_CUDA;
    }
    const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0).count();
    if (static_cast<unsigned long long>(ms) > lim) {
      cudaEventDestroy(ev);
      m->err = "timed out waiting for the GPU";
      return SOUP_ERR_TIMEOUT;
    }
    if (ms > 2) {
      struct timespec ts = {0, 200000};
      nanosleep(&ts, nullptr);
    }
  }
  cudaEventDestroy(ev);
  return SOUP_OK;
}

soup_status check_launch(soup_model* m, cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SOUP_OK;
  m->err = std::string(what) + ": " + cudaGetErrorString(e);
  return e == cudaErrorInvalidValue ? SOUP_ERR_UNSUPPORTED : SOUP_ERR_CUDA;
}

// ------------------------------------------------------------------ tracing
// NVTX ranges on the host thread around each layer call, layer copy, head pass and step, for a
// timeline tool (no cost when none is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  NvtxRange(const char* what, int i) {
    char b[48];
    std::snprintf(b, sizeof(b), "%s %d", what, i);
    nvtxRangePushA(b);
  }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// ------------------------------------------------------------------ live profile
enum ProfCatId : int {
  CAT_H2D = 0, CAT_NF4_FWD, CAT_NF4_DX, CAT_LORA, CAT_LORA_GRAD, CAT_LMHEAD_FWD, CAT_LMHEAD_DX, CAT_ATTN_FWD,
  CAT_ATTN_BWD, CAT_RMSNORM, CAT_ROPE, CAT_SWIGLU, CAT_CE, CAT_ADAMW, CAT_EMBED, CAT_D2D, CAT_QUANT, CAT_NULL,
  CAT_COUNT
};
const char* const kCatNames[CAT_COUNT] = {
    "h2d_layer_copy", "gemm_nf4_fwd", "gemm_nf4_dx", "gemm_lora", "gemm_lora_grad", "gemm_lm_head_fwd",
    "gemm_lm_head_dx", "attention_fwd", "attention_bwd", "rmsnorm", "rope", "swiglu", "cross_entropy", "adamw",
    "embed", "d2d_copy", "nf4_quantize", "event_overhead"};

cudaEvent_t prof_event(soup_model* m) {
  if (!m->prof_pool.empty()) {
    cudaEvent_t e = m->prof_pool.back();
    m->prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
int prof_begin(soup_model* m, cudaStream_t st) {
  if (!m->prof) return -1;
  soup_model::ProfRec r{};
  r.a = prof_event(m);
  r.b = prof_event(m);
  if (!r.a || !r.b) return -1;
  cudaEventRecord(r.a, st);
  m->prof_pending.push_back(r);
  return static_cast<int>(m->prof_pending.size()) - 1;
}
void prof_end(soup_model* m, cudaStream_t st, int idx, int cat, double flops, double bytes) {
  if (idx < 0) return;
  soup_model::ProfRec& r = m->prof_pending[idx];
  r.cat = cat;
  r.flops = flops;
  r.bytes = bytes;
  cudaEventRecord(r.b, st);
}
void prof_resolve(soup_model* m) {
  if (m->prof_cats.size() != CAT_COUNT) m->prof_cats.assign(CAT_COUNT, soup_model::ProfCat{});
  for (auto& r : m->prof_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      auto& c = m->prof_cats[r.cat];
      c.launches += 1;
      c.ms += ms;
      c.flops += r.flops;
      c.bytes += r.bytes;
    }
    m->prof_pool.push_back(r.a);
    m->prof_pool.push_back(r.b);
  }
  m->prof_pending.clear();
}
// ~30 us at the B200's 1.965 GHz: longer than the host takes to prepare and submit a launch
constexpr long long PROF_LEAD_CYCLES = 60000;
// Timed category: while a model call is captured into a graph the pair becomes two external
// event-record nodes of that graph (recorded on every replay); otherwise plain records.
bool timed_begin(soup_model* m, cudaStream_t st, int cat, soup_model::ProfRec* r) {
  // empty calibration launches are timed whenever any category is
  const bool want = ((m->tcat >> cat) & 1) != 0 || (cat == CAT_NULL && m->tcat != 0);
  if (m->prof || !want) return false;
  r->a = r->b = nullptr;
  if (cudaEventCreate(&r->a) != cudaSuccess || cudaEventCreate(&r->b) != cudaSuccess) {
    if (r->a) cudaEventDestroy(r->a);
    cudaGetLastError();
    return false;
  }
  if ((m->cap_recs ? cudaEventRecordWithFlags(r->a, st, cudaEventRecordExternal) : cudaEventRecord(r->a, st)) !=
      cudaSuccess) {
    cudaEventDestroy(r->a);
    cudaEventDestroy(r->b);
    cudaGetLastError();
    return false;
  }
  return true;
}
void timed_end(soup_model* m, cudaStream_t st, soup_model::ProfRec& r, int cat, double flops, double bytes) {
  r.cat = cat;
  r.flops = flops;
  r.bytes = bytes;
  if (m->cap_recs)
    cudaEventRecordWithFlags(r.b, st, cudaEventRecordExternal);
  else
    cudaEventRecord(r.b, st);
  (m->cap_recs ? *m->cap_recs : m->tpending).push_back(r);
}
// Adds the recorded durations of `recs` to the timed totals (waits for their end events);
// destroys the events when `drop`.
void timed_harvest(soup_model* m, std::vector<soup_model::ProfRec>& recs, bool drop) {
  if (m->taccs.size() != CAT_COUNT) m->taccs.assign(CAT_COUNT, soup_model::ProfCat{});
  for (auto& r : recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      auto& c = m->taccs[r.cat];
      c.launches += 1;
      c.ms += ms;
      c.flops += r.flops;
      c.bytes += r.bytes;
    } else {
      cudaGetLastError();  // not sticky: keep it from surfacing at the next launch check
    }
    if (drop) {
      cudaEventDestroy(r.a);
      cudaEventDestroy(r.b);
    }
  }
  if (drop) recs.clear();
}
void timed_harvest_all(soup_model* m) {
  for (auto& kv : m->graphs)
    if (kv.second.armed) {
      timed_harvest(m, kv.second.recs, false);
      kv.second.armed = 0;
    }
  timed_harvest(m, m->tpending, true);
}

template <class F>
soup_status launch(soup_model* m, cudaStream_t st, int cat, double flops, double bytes, const char* what, F&& f) {
  if (m->prof) busy_wait_launch(PROF_LEAD_CYCLES, st);
  const int idx = prof_begin(m, st);
  soup_model::ProfRec tr{};
  const bool timed = timed_begin(m, st, cat, &tr);
  const cudaError_t e = f();
  if (timed) timed_end(m, st, tr, cat, flops, bytes);
  prof_end(m, st, idx, cat, flops, bytes);
  return check_launch(m, e, what);
}

// While a category is timed, each layer call starts with one empty launch bracketed like the
// timed ones (inside the layer's graph): the event pairs' own cost per launch.
soup_status timed_calibration(soup_model* m, cudaStream_t st) {
  if (m->tcat == 0 || m->prof) return SOUP_OK;
  return launch(m, st, CAT_NULL, 0.0, 0.0, "empty launch", [&] { return null_launch(st); });
}

LayerView view_of(const soup_model* m, const uint8_t* base) {
  LayerView v{};
  for (int p = 0; p < 7; ++p) {
    v.seg[p].codes = base + m->layout.off[p][0];
    v.seg[p].q8 = reinterpret_cast<const int8_t*>(base + m->layout.off[p][1]);
    v.seg[p].scales = reinterpret_cast<const float*>(base + m->layout.off[p][2]);
    v.seg[p].mean = reinterpret_cast<const float*>(base + m->layout.off[p][3]);
  }
  v.gamma[0] = reinterpret_cast<const uint16_t*>(base + m->layout.off[7][0]);
  v.gamma[1] = reinterpret_cast<const uint16_t*>(base + m->layout.off[8][0]);
  return v;
}

NF4Group group_of(const soup_model* m, const LayerView& v, std::initializer_list<int> projs) {
  ProjShape s[7];
  proj_shapes(m->cfg, s);
  NF4Group g{};
  int row = 0, k = 0;
  for (int p : projs) {
    g.seg[k] = v.seg[p];
    g.seg[k].row_begin = row;
    g.seg[k].rows = s[p].out;
    g.cols = s[p].in;
    row += s[p].out;
    ++k;
  }
  g.nseg = k;
  g.total_rows = row;
  return g;
}

// ------------------------------------------------------------------ GEMM helpers
Operand opnd(int kind, const void* ptr, long long ld, float scale = 1.f, int lo = 0, int hi = INT_MAX) {
  Operand o;
  o.kind = kind;
  o.ptr = ptr;
  o.ld = ld;
  o.scale = scale;
  o.row_lo = lo;
  o.row_hi = hi;
  return o;
}
GemmParams gemm_base(soup_model* m, int M, int N, void* out, long long ldo, int out_f32, float alpha) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.out = out;
  p.ldo = ldo;
  p.out_f32 = out_f32;
  p.alpha = alpha;
  p.err = m->scal + 1;
  p.workspace = m->gemm_ws;
  p.ws_bytes = m->gemm_ws_bytes;
  p.tile_counters = m->gemm_cnt;
  p.n_counters = GEMM_COUNTERS;
  std::memcpy(p.lut, codebook().v, sizeof(p.lut));
  return p;
}
void add_seg(GemmParams& p, int K, const Operand& A, const Operand& B) {
  GemmSeg& s = p.seg[p.nseg++];
  s.K = K;
  s.A = A;
  s.B = B;
}
double operand_bytes_per_elem(int kind) {
  switch (kind) {
    case OP_BF16_K:
    case OP_BF16_MN:
      return 2.0;
    case OP_F32_K:
    case OP_F32_MN:
      return 4.0;
    default:  // NF4: code nibble + q8 absmax per 64 + fp32 scale per 16384
      return 0.5 + 1.0 / 64.0 + 4.0 / 16384.0;
  }
}
soup_status run_gemm(soup_model* m, const GemmParams& p, cudaStream_t st, const char* what) {
  double flops = 0, bytes = 0;
  for (int i = 0; i < p.nseg; ++i) {
    const GemmSeg& g = p.seg[i];
    if (g.K <= 0) continue;
    const int lo = std::max(0, g.B.row_lo), hi = std::min(p.N, g.B.row_hi);
    const double rows_b = hi > lo ? hi - lo : 0;
    flops += 2.0 * p.M * rows_b * g.K;
    bytes += operand_bytes_per_elem(g.A.kind) * p.M * g.K + operand_bytes_per_elem(g.B.kind) * rows_b * g.K;
  }
  bytes += static_cast<double>(p.M) * p.N * (p.out_f32 ? 4.0 : 2.0) * (p.accumulate ? 2.0 : 1.0);
  if (p.residual) bytes += 2.0 * p.M * p.N;
  int cat = CAT_LORA;
  const Operand& b0 = p.seg[0].B;
  if (b0.kind == OP_NF4_K) cat = CAT_NF4_FWD;
  else if (b0.kind == OP_NF4_MN) cat = CAT_NF4_DX;
  else if (b0.ptr == m->lm_head) cat = (b0.kind == OP_BF16_K) ? CAT_LMHEAD_FWD : CAT_LMHEAD_DX;
  else if (p.seg[0].A.kind == OP_BF16_MN) cat = CAT_LORA_GRAD;
  return launch(m, st, cat, flops, bytes, what, [&] { return gemm_launch(p, st); });
}

// ------------------------------------------------------------------ streamer
soup_status streamer_ensure(soup_model* m, int layer, int protect_lo, int protect_hi) {
  if (m->cfg.mode == SOUP_RESIDENT) return SOUP_OK;
  const NvtxRange trace("layer copy", layer);
  const int nb = static_cast<int>(m->dev_buf.size());
  for (int b = 0; b < nb; ++b)
    if (m->buf_layer[b] == layer) return SOUP_OK;
  if (!m->host_loaded[layer]) {
    m->err = "layer " + std::to_string(layer) + " has no weights loaded";
    return SOUP_ERR_STATE;
  }
  int victim = -1;
  for (int b = 0; b < nb; ++b) {
    if (m->buf_inuse[b]) continue;
    const int L = m->buf_layer[b];
    if (L >= protect_lo && L <= protect_hi && L >= 0) continue;
    if (victim < 0 || m->buf_last[b] < m->buf_last[victim]) victim = b;
  }
  if (victim < 0) {
    for (int b = 0; b < nb; ++b)
      if (!m->buf_inuse[b] && (victim < 0 || m->buf_last[b] < m->buf_last[victim])) victim = b;
  }
  if (victim < 0) {
    m->err = "streamer: every layer buffer is in use";
    return SOUP_ERR_STATE;
  }
  SOUP_CK(cudaStreamWaitEvent(m->copy_stream, m->buf_free[victim], 0));
  const int pidx = prof_begin(m, m->copy_stream);
  soup_model::ProfRec tr{};
  const bool timed = timed_begin(m, m->copy_stream, CAT_H2D, &tr);
  if (m->use_file) {
    SOUP_CK(m->file.stream_layer(layer, m->dev_buf[victim], m->copy_stream));
  } else {
    SOUP_CK(cudaMemcpyAsync(m->dev_buf[victim], m->host_blob[layer], m->layout.total, cudaMemcpyHostToDevice,
                            m->copy_stream));
  }
  if (timed) timed_end(m, m->copy_stream, tr, CAT_H2D, 0.0, static_cast<double>(m->layout.total));
  prof_end(m, m->copy_stream, pidx, CAT_H2D, 0.0, static_cast<double>(m->layout.total));
  SOUP_CK(cudaEventRecord(m->copy_done[victim], m->copy_stream));
  m->buf_layer[victim] = layer;
  m->buf_last[victim] = ++m->tick;
  m->stats.layer_loads += 1;
  m->stats.bytes_h2d += static_cast<long long>(m->layout.total);
  return SOUP_OK;
}

soup_status streamer_acquire(soup_model* m, int layer, cudaStream_t st, const uint8_t** base, int* buf) {
  if (m->cfg.mode == SOUP_RESIDENT) {
    if (!m->host_loaded[layer]) {
      m->err = "layer " + std::to_string(layer) + " has no weights loaded";
      return SOUP_ERR_STATE;
    }
    *base = m->dev_buf[layer];
    *buf = -1;
    return SOUP_OK;
  }
  const int nb = static_cast<int>(m->dev_buf.size());
  int b = -1;
  for (int i = 0; i < nb; ++i)
    if (m->buf_layer[i] == layer) b = i;
  if (b < 0) {
    SOUP_TRY(streamer_ensure(m, layer, layer, layer));
    for (int i = 0; i < nb; ++i)
      if (m->buf_layer[i] == layer) b = i;
  } else {
    m->stats.layer_reuses += 1;
  }
  SOUP_CK(cudaStreamWaitEvent(st, m->copy_done[b], 0));
  m->buf_inuse[b] = 1;
  m->buf_last[b] = ++m->tick;
  *base = m->dev_buf[b];
  *buf = b;
  return SOUP_OK;
}

soup_status streamer_release(soup_model* m, int buf, cudaStream_t st) {
  if (buf < 0) return SOUP_OK;
  SOUP_CK(cudaEventRecord(m->buf_free[buf], st));
  m->buf_inuse[buf] = 0;
  return SOUP_OK;
}

// Issue the copies of the first layers of a schedule (before compute that precedes them).
soup_status streamer_warm(soup_model* m, int first, int count) {
  if (m->cfg.mode == SOUP_RESIDENT) return SOUP_OK;
  const int n = std::min(count, static_cast<int>(m->dev_buf.size()));
  for (int k = 0; k < n && first + k < m->cfg.n_layers; ++k)
    SOUP_TRY(streamer_ensure(m, first + k, first, first + n - 1));
  return SOUP_OK;
}

// Prefetch the next layers of a schedule (as many as there are spare buffers).
soup_status streamer_prefetch(soup_model* m, const std::vector<int>& order, size_t pos) {
  if (m->cfg.mode == SOUP_RESIDENT) return SOUP_OK;
  const size_t depth = m->dev_buf.size() - 1;
  int lo = INT_MAX, hi = INT_MIN;
  for (size_t k = pos; k < order.size() && k <= pos + depth; ++k) {
    lo = std::min(lo, order[k]);
    hi = std::max(hi, order[k]);
  }
  for (size_t k = pos + 1; k < order.size() && k <= pos + depth; ++k) SOUP_TRY(streamer_ensure(m, order[k], lo, hi));
  return SOUP_OK;
}

// ------------------------------------------------------------------ layer forward / backward
soup_status layer_forward(soup_model* m, int i, const LayerView& L, const uint16_t* x_in, uint16_t* x_out, int B,
                          int S, cudaStream_t st) {
  const soup_model_config& c = m->cfg;
  const int T = B * S, h = c.hidden, r = c.lora_r, I = c.intermediate;
  const int qd = c.n_heads * c.head_dim, kvd = c.n_kv_heads * c.head_dim, QKV = m->qkv_cols;
  const float s = m->s_lora;
  const bool lora = m->lora_enabled && m->lora_p;
  Saved& A = m->saved[i];
  A.valid = 0;
  SOUP_TRY(timed_calibration(m, st));
  const double act = 2.0 * T * h;  // bytes of one [T, h] bf16 activation
  SOUP_TRY(launch(m, st, CAT_D2D, 0, 2 * act, "save x", [&] {
    return cudaMemcpyAsync(A.x, x_in, static_cast<size_t>(T) * h * 2, cudaMemcpyDeviceToDevice, st);
  }));
  SOUP_TRY(launch(m, st, CAT_RMSNORM, 0, 2 * act + 4.0 * T, "rmsnorm",
                  [&] { return rmsnorm_fwd_launch(A.x, L.gamma[0], T, h, c.rms_eps, A.n1, A.rstd1, st); }));
  const uint16_t* P = m->lora_bf16;
  // ---- q | k | v
  if (lora) {
    GemmParams p = gemm_base(m, T, 3 * r, A.uqkv, 3 * r, 0, s);
    add_seg(p, h, opnd(OP_BF16_K, A.n1, h), opnd(OP_BF16_K, P + lora_off(c, i, 0, 0), h));
    SOUP_TRY(run_gemm(m, p, st, "lora u qkv"));
  }
  {
    GemmParams p = gemm_base(m, T, QKV, A.qkv, QKV, 0, 1.f);
    p.nf4 = group_of(m, L, {0, 1, 2});
    add_seg(p, h, opnd(OP_BF16_K, A.n1, h), opnd(OP_NF4_K, nullptr, 0));
    if (lora) {
      const int lo[3] = {0, qd, qd + kvd}, hi[3] = {qd, qd + kvd, QKV};
      for (int q = 0; q < 3; ++q)
        add_seg(p, r, opnd(OP_BF16_K, A.uqkv + q * r, 3 * r), opnd(OP_BF16_K, P + lora_off(c, i, 0, 1), r, 1.f, lo[q], hi[q]));
    }
    // RoPE on the q and k columns, in the epilogue (rotate-half, the row's position)
    p.rope_cos = m->rope_cos;
    p.rope_sin = m->rope_sin;
    p.rope_cols = qd + kvd;
    p.rope_d = c.head_dim;
    p.rope_S = S;
    p.rope_rl = m->pack_rl;
    SOUP_TRY(run_gemm(m, p, st, "qkv gemm"));
  }
  AttnShape as{B, S, c.n_heads, c.n_kv_heads, c.head_dim, QKV, m->pack_pl, m->pack_rl, m->rope_cos, m->rope_sin};
  const double attn_flops = 2.0 * B * c.n_heads * c.head_dim * static_cast<double>(S) * (S + 1);
  SOUP_TRY(launch(m, st, CAT_ATTN_FWD, attn_flops, 2.0 * T * QKV + 2.0 * T * qd + 4.0 * T * c.n_heads, "attention fwd",
                  [&] {
                    return attn_fwd_launch(as, A.qkv, A.o, A.lse, m->scal + 1, st);
                  }));
  // ---- o + residual
  if (lora) {
    GemmParams p = gemm_base(m, T, r, A.uo, r, 0, s);
    add_seg(p, qd, opnd(OP_BF16_K, A.o, qd), opnd(OP_BF16_K, P + lora_off(c, i, 3, 0), qd));
    SOUP_TRY(run_gemm(m, p, st, "lora u o"));
  }
  {
    GemmParams p = gemm_base(m, T, h, A.x1, h, 0, 1.f);
    p.nf4 = group_of(m, L, {3});
    p.residual = A.x;
    p.ldr = h;
    add_seg(p, qd, opnd(OP_BF16_K, A.o, qd), opnd(OP_NF4_K, nullptr, 0));
    if (lora) add_seg(p, r, opnd(OP_BF16_K, A.uo, r), opnd(OP_BF16_K, P + lora_off(c, i, 3, 1), r));
    SOUP_TRY(run_gemm(m, p, st, "o gemm"));
  }
  SOUP_TRY(launch(m, st, CAT_RMSNORM, 0, 2 * act + 4.0 * T, "rmsnorm",
                  [&] { return rmsnorm_fwd_launch(A.x1, L.gamma[1], T, h, c.rms_eps, A.n2, A.rstd2, st); }));
  // ---- gate | up, SwiGLU
  if (lora) {
    GemmParams p = gemm_base(m, T, 2 * r, A.ugu, 2 * r, 0, s);
    add_seg(p, h, opnd(OP_BF16_K, A.n2, h), opnd(OP_BF16_K, P + lora_off(c, i, 4, 0), h));
    SOUP_TRY(run_gemm(m, p, st, "lora u gate/up"));
  }
  {
    GemmParams p = gemm_base(m, T, 2 * I, A.gu, 2 * I, 0, 1.f);
    p.nf4 = group_of(m, L, {4, 5});
    add_seg(p, h, opnd(OP_BF16_K, A.n2, h), opnd(OP_NF4_K, nullptr, 0));
    if (lora) {
      for (int q = 0; q < 2; ++q)
        add_seg(p, r, opnd(OP_BF16_K, A.ugu + q * r, 2 * r),
                opnd(OP_BF16_K, P + lora_off(c, i, 4, 1), r, 1.f, q * I, (q + 1) * I));
    }
    SOUP_TRY(run_gemm(m, p, st, "gate/up gemm"));
  }
  SOUP_TRY(launch(m, st, CAT_SWIGLU, 0, 6.0 * T * I, "swiglu", [&] { return swiglu_fwd_launch(A.gu, T, I, A.m, st); }));
  // ---- down + residual
  if (lora) {
    GemmParams p = gemm_base(m, T, r, A.ud, r, 0, s);
    add_seg(p, I, opnd(OP_BF16_K, A.m, I), opnd(OP_BF16_K, P + lora_off(c, i, 6, 0), I));
    SOUP_TRY(run_gemm(m, p, st, "lora u down"));
  }
  {
    GemmParams p = gemm_base(m, T, h, x_out, h, 0, 1.f);
    p.nf4 = group_of(m, L, {6});
    p.residual = A.x1;
    p.ldr = h;
    add_seg(p, I, opnd(OP_BF16_K, A.m, I), opnd(OP_NF4_K, nullptr, 0));
    if (lora) add_seg(p, r, opnd(OP_BF16_K, A.ud, r), opnd(OP_BF16_K, P + lora_off(c, i, 6, 1), r));
    SOUP_TRY(run_gemm(m, p, st, "down gemm"));
  }
  A.B = B;
  A.S = S;
  A.lora = lora ? 1 : 0;
  A.valid = 1;
  return SOUP_OK;
}

// LoRA gradient GEMMs for one projection: dB += g^T u_s, dA += v_s^T x  (both fp32, accumulate)
soup_status lora_grads(soup_model* m, int T, const uint16_t* g, long long ldg, int out, const uint16_t* us,
                       long long ldu, float* dB, const uint16_t* x, long long ldx, int in, const uint16_t* vs,
                       long long ldv, int nv, float* dA, cudaStream_t st, bool do_dB, bool do_dA) {
  const int r = m->cfg.lora_r;
  float* ws = (st == m->grad_stream) ? m->gemm_ws2 : m->gemm_ws;
  const size_t ws_bytes = (st == m->grad_stream) ? m->gemm_ws2_bytes : m->gemm_ws_bytes;
  int* cnt = (st == m->grad_stream) ? m->gemm_cnt2 : m->gemm_cnt;
  if (do_dB) {
    GemmParams p = gemm_base(m, out, r, dB, r, 1, 1.f);
    p.workspace = ws;
    p.ws_bytes = ws_bytes;
    p.tile_counters = cnt;
    p.accumulate = 1;
    add_seg(p, T, opnd(OP_BF16_MN, g, ldg), opnd(OP_BF16_MN, us, ldu));
    SOUP_TRY(run_gemm(m, p, st, "lora dB"));
  }
  if (do_dA) {
    // dA^T [in, nv] = x^T v_s, written transposed into dA [nv, in]
    GemmParams p = gemm_base(m, in, nv, dA, in, 1, 1.f);
    p.workspace = ws;
    p.ws_bytes = ws_bytes;
    p.tile_counters = cnt;
    p.accumulate = 1;
    p.out_trans = 1;
    add_seg(p, T, opnd(OP_BF16_MN, x, ldx), opnd(OP_BF16_MN, vs, ldv));
    SOUP_TRY(run_gemm(m, p, st, "lora dA"));
  }
  return SOUP_OK;
}

// The LoRA weight-gradient GEMMs (dA, dB) of a layer backward read only the main stream's
// v = g B, g and saved activations, and write grad regions nothing reads before the step
// ends: they run on a low-priority side stream beside the dX GEMMs, on SMs those leave idle.
// Each group forks as soon as its v GEMM is done, before the projection's dX GEMM, so that the
// last group of a layer (q|k|v) overlaps that GEMM instead of the layer's end.
// The side stream forks after each v and joins before the layer call returns (the g buffers
// are reused by the next layer).  Same kernels, same order per region: same bits.
soup_status grads_fork(soup_model* m, cudaStream_t st, cudaStream_t* gs) {
  *gs = st;
  // (not while profiling: per-launch event times of overlapping kernels would count each
  // other's time)
  if (!m->concurrent_grads || m->prof) return SOUP_OK;
  SOUP_CK(cudaEventRecord(m->fork_ev, st));
  SOUP_CK(cudaStreamWaitEvent(m->grad_stream, m->fork_ev, 0));
  m->grads_forked = 1;
  *gs = m->grad_stream;
  return SOUP_OK;
}
soup_status grads_join(soup_model* m, cudaStream_t st) {
  if (!m->grads_forked) return SOUP_OK;
  m->grads_forked = 0;
  SOUP_CK(cudaEventRecord(m->join_ev, m->grad_stream));
  SOUP_CK(cudaStreamWaitEvent(st, m->join_ev, 0));
  return SOUP_OK;
}

// Word offset in `scal` of the AdamW hyper-parameters of the running step (lr, 1/(1-b1^t),
// 1/(1-b2^t)).
constexpr int ADAM_HP_WORD = 8;
constexpr float ADAM_B1 = 0.9f, ADAM_B2 = 0.999f, ADAM_EPS = 1e-8f, ADAM_WD = 0.f;

bool adam_after(const soup_model* m, int i) { return m->adam_in_bwd && m->lora_p && i + 1 < m->cfg.n_layers; }

// AdamW on layer l's LoRA slice with the step's hyper-parameters from device memory.
soup_status adamw_layer(soup_model* m, int l, cudaStream_t st) {
  const size_t off = lora_off(m->cfg, l, 0, 0), n = lora_layer_numel(m->cfg);
  const float* hp = reinterpret_cast<const float*>(m->scal + ADAM_HP_WORD);
  return launch(m, st, CAT_ADAMW, 0, 28.0 * static_cast<double>(n), "adamw", [&] {
    return adamw_hp_launch(m->lora_p + off, m->lora_g + off, m->lora_m + off, m->lora_v + off,
                           m->lora_bf16 ? m->lora_bf16 + off : nullptr, static_cast<long long>(n), ADAM_B1, ADAM_B2,
                           ADAM_EPS, ADAM_WD, hp, st);
  });
}

soup_status layer_backward_body(soup_model* m, int i, const LayerView& L, const uint16_t* dy, uint16_t* dx, int B,
                                int S, cudaStream_t st);
soup_status layer_backward(soup_model* m, int i, const LayerView& L, const uint16_t* dy, uint16_t* dx, int B, int S,
                           cudaStream_t st) {
  const soup_status s1 = layer_backward_body(m, i, L, dy, dx, B, S, st);
  const soup_status s2 = grads_join(m, st);  // also on errors: a capture must end joined
  return s1 != SOUP_OK ? s1 : s2;
}

soup_status layer_backward_body(soup_model* m, int i, const LayerView& L, const uint16_t* dy, uint16_t* dx, int B,
                                int S, cudaStream_t st) {
  const soup_model_config& c = m->cfg;
  Saved& A = m->saved[i];
  if (!A.valid || A.B != B || A.S != S) {
    m->err = "layer_bwd: no matching forward for layer " + std::to_string(i);
    return SOUP_ERR_STATE;
  }
  SOUP_TRY(timed_calibration(m, st));
  if (adam_after(m, i)) {
    // layer i+1's update, beside this layer's backward: its last readers (the backward call of
    // layer i+1, joined at that call's end) are done
    cudaStream_t gs;
    SOUP_TRY(grads_fork(m, st, &gs));
    SOUP_TRY(adamw_layer(m, i + 1, gs));
  }
  const int T = B * S, h = c.hidden, r = c.lora_r, I = c.intermediate;
  const int qd = c.n_heads * c.head_dim, kvd = c.n_kv_heads * c.head_dim, QKV = m->qkv_cols;
  const float s = m->s_lora;
  const bool lora = A.lora && m->lora_p;
  const uint16_t* P = m->lora_bf16;
  float* G = m->lora_g;
  // ---- down
  if (lora) {
    GemmParams p = gemm_base(m, T, r, m->vd, r, 0, s);
    add_seg(p, h, opnd(OP_BF16_K, dy, h), opnd(OP_BF16_MN, P + lora_off(c, i, 6, 1), r));
    SOUP_TRY(run_gemm(m, p, st, "lora v down"));
  }
  cudaStream_t gs = st;
  if (lora) {
    SOUP_TRY(grads_fork(m, st, &gs));
    SOUP_TRY(lora_grads(m, T, dy, h, h, A.ud, r, G + lora_off(c, i, 6, 1), A.m, I, I, m->vd, r, r,
                        G + lora_off(c, i, 6, 0), gs, true, true));
  }
  {
    GemmParams p = gemm_base(m, T, I, m->dm, I, 0, 1.f);
    p.nf4 = group_of(m, L, {6});
    add_seg(p, h, opnd(OP_BF16_K, dy, h), opnd(OP_NF4_MN, nullptr, 0));
    if (lora) add_seg(p, r, opnd(OP_BF16_K, m->vd, r), opnd(OP_BF16_MN, P + lora_off(c, i, 6, 0), I));
    SOUP_TRY(run_gemm(m, p, st, "down dX"));
  }
  SOUP_TRY(launch(m, st, CAT_SWIGLU, 0, 10.0 * T * I, "swiglu bwd",
                  [&] { return swiglu_bwd_launch(m->dm, A.gu, T, I, m->dgu, st); }));
  // ---- gate | up
  if (lora) {
    // v_gate | v_up = [dgate | dup] . blockdiag(B_gate, B_up): one GEMM, each output block
    // reading its own projection's B through a row window (zero elsewhere); the operand is
    // indexed by the output column n, so B_p is addressed from q r columns before its start
    GemmParams p = gemm_base(m, T, 2 * r, m->vgu, 2 * r, 0, s);
    for (int q = 0; q < 2; ++q)
      add_seg(p, I, opnd(OP_BF16_K, m->dgu + q * I, 2 * I),
              opnd(OP_BF16_MN, P + lora_off(c, i, 4 + q, 1) - q * r, r, 1.f, q * r, (q + 1) * r));
    SOUP_TRY(run_gemm(m, p, st, "lora v gate/up"));
  }
  if (lora) {
    SOUP_TRY(grads_fork(m, st, &gs));
    for (int q = 0; q < 2; ++q)
      SOUP_TRY(lora_grads(m, T, m->dgu + q * I, 2 * I, I, A.ugu + q * r, 2 * r, G + lora_off(c, i, 4 + q, 1), nullptr,
                          0, 0, nullptr, 0, 0, nullptr, gs, true, false));
    SOUP_TRY(lora_grads(m, T, nullptr, 0, 0, nullptr, 0, nullptr, A.n2, h, h, m->vgu, 2 * r, 2 * r,
                        G + lora_off(c, i, 4, 0), gs, false, true));
  }
  {
    GemmParams p = gemm_base(m, T, h, m->dn, h, 0, 1.f);
    p.nf4 = group_of(m, L, {4, 5});
    add_seg(p, 2 * I, opnd(OP_BF16_K, m->dgu, 2 * I), opnd(OP_NF4_MN, nullptr, 0));
    if (lora)
      for (int q = 0; q < 2; ++q)
        add_seg(p, r, opnd(OP_BF16_K, m->vgu + q * r, 2 * r), opnd(OP_BF16_MN, P + lora_off(c, i, 4 + q, 0), h));
    SOUP_TRY(run_gemm(m, p, st, "gate/up dX"));
  }
  const double act = 2.0 * T * h;
  SOUP_TRY(launch(m, st, CAT_RMSNORM, 0, 4 * act + 4.0 * T, "rmsnorm bwd",
                  [&] { return rmsnorm_bwd_launch(m->dn, A.x1, A.rstd2, L.gamma[1], dy, T, h, m->dx1, st); }));
  // ---- o
  if (lora) {
    GemmParams p = gemm_base(m, T, r, m->vo, r, 0, s);
    add_seg(p, h, opnd(OP_BF16_K, m->dx1, h), opnd(OP_BF16_MN, P + lora_off(c, i, 3, 1), r));
    SOUP_TRY(run_gemm(m, p, st, "lora v o"));
  }
  if (lora) {
    SOUP_TRY(grads_fork(m, st, &gs));
    SOUP_TRY(lora_grads(m, T, m->dx1, h, h, A.uo, r, G + lora_off(c, i, 3, 1), A.o, qd, qd, m->vo, r, r,
                        G + lora_off(c, i, 3, 0), gs, true, true));
  }
  {
    GemmParams p = gemm_base(m, T, qd, m->da, qd, 0, 1.f);
    p.nf4 = group_of(m, L, {3});
    add_seg(p, h, opnd(OP_BF16_K, m->dx1, h), opnd(OP_NF4_MN, nullptr, 0));
    if (lora) add_seg(p, r, opnd(OP_BF16_K, m->vo, r), opnd(OP_BF16_MN, P + lora_off(c, i, 3, 0), qd));
    SOUP_TRY(run_gemm(m, p, st, "o dX"));
  }
  // ---- attention, RoPE
  AttnShape as{B, S, c.n_heads, c.n_kv_heads, c.head_dim, QKV, m->pack_pl, m->pack_rl, m->rope_cos, m->rope_sin};
  const double attn_flops = 4.0 * B * c.n_heads * c.head_dim * static_cast<double>(S) * (S + 1);
  SOUP_TRY(launch(m, st, CAT_ATTN_BWD, attn_flops, 4.0 * T * QKV + 4.0 * T * qd + 8.0 * T * c.n_heads, "attention bwd",
                  [&] {
                    return attn_bwd_launch(as, A.qkv, A.o, m->da, A.lse, m->delta, m->dqkv, m->gemm_ws,
                                              m->gemm_ws_bytes, m->scal + 1, st);
                  }));
  // ---- q | k | v
  const int off[3] = {0, qd, qd + kvd}, outs[3] = {qd, kvd, kvd};
  if (lora) {
    // v_q | v_k | v_v in one GEMM (block-diagonal B through row windows, as for gate | up)
    GemmParams p = gemm_base(m, T, 3 * r, m->vqkv, 3 * r, 0, s);
    for (int q = 0; q < 3; ++q)
      add_seg(p, outs[q], opnd(OP_BF16_K, m->dqkv + off[q], QKV),
              opnd(OP_BF16_MN, P + lora_off(c, i, q, 1) - q * r, r, 1.f, q * r, (q + 1) * r));
    SOUP_TRY(run_gemm(m, p, st, "lora v qkv"));
  }
  if (lora) {
    SOUP_TRY(grads_fork(m, st, &gs));
    for (int q = 0; q < 3; ++q)
      SOUP_TRY(lora_grads(m, T, m->dqkv + off[q], QKV, outs[q], A.uqkv + q * r, 3 * r, G + lora_off(c, i, q, 1),
                          nullptr, 0, 0, nullptr, 0, 0, nullptr, gs, true, false));
    SOUP_TRY(lora_grads(m, T, nullptr, 0, 0, nullptr, 0, nullptr, A.n1, h, h, m->vqkv, 3 * r, 3 * r,
                        G + lora_off(c, i, 0, 0), gs, false, true));
  }
  {
    GemmParams p = gemm_base(m, T, h, m->dn, h, 0, 1.f);
    p.nf4 = group_of(m, L, {0, 1, 2});
    add_seg(p, QKV, opnd(OP_BF16_K, m->dqkv, QKV), opnd(OP_NF4_MN, nullptr, 0));
    if (lora)
      for (int q = 0; q < 3; ++q)
        add_seg(p, r, opnd(OP_BF16_K, m->vqkv + q * r, 3 * r), opnd(OP_BF16_MN, P + lora_off(c, i, q, 0), h));
    SOUP_TRY(run_gemm(m, p, st, "qkv dX"));
  }
  SOUP_TRY(launch(m, st, CAT_RMSNORM, 0, 4 * act + 4.0 * T, "rmsnorm bwd",
                  [&] { return rmsnorm_bwd_launch(m->dn, A.x, A.rstd1, L.gamma[0], m->dx1, T, h, dx, st); }));
  return SOUP_OK;
}

// ------------------------------------------------------------------ head
// logits = RMSNorm(x) W_lm^T (fp32), per-row LSE and target logit.
soup_status head_forward(soup_model* m, const uint16_t* x, int B, int S, cudaStream_t st) {
  const NvtxRange trace("head fwd");
  const soup_model_config& c = m->cfg;
  const int T = B * S, h = c.hidden, V = c.vocab;
  SOUP_TRY(launch(m, st, CAT_RMSNORM, 0, 4.0 * T * h + 4.0 * T, "final norm",
                  [&] { return rmsnorm_fwd_launch(x, m->final_gamma, T, h, c.rms_eps, m->hf, m->rstdf, st); }));
  GemmParams p = gemm_base(m, T, V, m->logits, V, 1, 1.f);
  add_seg(p, h, opnd(OP_BF16_K, m->hf, h), opnd(OP_BF16_K, m->lm_head, h));
  SOUP_TRY(run_gemm(m, p, st, "lm_head"));
  if (m->pack_pl > 0) {
    SOUP_TRY(launch(m, st, CAT_CE, 0, 4.0 * T * V, "ce rows", [&] {
      return ce_rows_t_launch(m->logits, T, V, m->tgt1, m->tgt2, m->rowlse, m->rowtgt, m->rowtgt2, st);
    }));
    return SOUP_OK;
  }
  SOUP_TRY(launch(m, st, CAT_CE, 0, 4.0 * T * V, "ce rows", [&] {
    return ce_rows_launch(m->logits, T, V, m->ids_dev, B, S, nullptr, 0, m->rowlse, m->rowtgt, m->scal + 1, st);
  }));
  return SOUP_OK;
}
// dlogits = w_t (softmax - onehot) -> dh = dlogits W_lm -> final-norm backward into dx.
soup_status head_backward(soup_model* m, const uint16_t* x, int B, int S, uint16_t* dx, cudaStream_t st) {
  const NvtxRange trace("head bwd");
  const soup_model_config& c = m->cfg;
  const int T = B * S, h = c.hidden, V = c.vocab;
  SOUP_TRY(launch(m, st, CAT_CE, 0, 6.0 * T * V, "ce grad", [&] {
    return m->pack_pl > 0
               ? ce_grad_t_launch(m->logits, m->rowlse, m->tgt1, m->roww, m->tgt2, m->roww2, T, V, m->dlogits, st)
               : ce_grad_launch(m->logits, m->rowlse, m->ids_dev, m->roww, B, S, V, m->dlogits, st);
  }));
  GemmParams p = gemm_base(m, T, h, m->dh, h, 0, 1.f);
  add_seg(p, V, opnd(OP_BF16_K, m->dlogits, V), opnd(OP_BF16_MN, m->lm_head, h));
  SOUP_TRY(run_gemm(m, p, st, "lm_head dX"));
  SOUP_TRY(launch(m, st, CAT_RMSNORM, 0, 6.0 * T * h + 4.0 * T, "final norm bwd",
                  [&] { return rmsnorm_bwd_launch(m->dh, x, m->rstdf, m->final_gamma, nullptr, T, h, dx, st); }));
  return SOUP_OK;
}

// One layer call of a step, replayed from a CUDA graph once its key has been seen twice (the
// first run is eager so every kernel attribute and TMA descriptor exists before capture).
soup_status run_layer(soup_model* m, int dir, int i, const uint8_t* base, const uint16_t* in, uint16_t* out, int B,
                      int S, cudaStream_t st) {
  const NvtxRange trace(dir == 0 ? "layer fwd" : "layer bwd", i);
  const LayerView v = view_of(m, base);
  if (!m->use_graphs || m->prof) {
    return dir == 0 ? layer_forward(m, i, v, in, out, B, S, st) : layer_backward(m, i, v, in, out, B, S, st);
  }
  Saved& A = m->saved[i];
  const int lora = (dir == 0) ? ((m->lora_enabled && m->lora_p) ? 1 : 0) : A.lora;
  if (dir == 1 && (!A.valid || A.B != B || A.S != S)) {
    m->err = "layer_bwd: no matching forward for layer " + std::to_string(i);
    return SOUP_ERR_STATE;
  }
  soup_model::GraphKey key;
  std::memset(&key, 0, sizeof(key));
  key.dir = dir;
  key.layer = i;
  key.B = B;
  key.S = S;
  key.lora = lora;
  key.pack = m->pack_pl;
  key.tcat = m->tcat;
  key.adam = (dir == 1 && adam_after(m, i)) ? 1 : 0;
  key.base = base;
  key.in = in;
  key.out = out;
  soup_model::GraphEntry& e = m->graphs[key];
  if (!e.exec && e.seen == 0) {
    e.seen = 1;
    return dir == 0 ? layer_forward(m, i, v, in, out, B, S, st) : layer_backward(m, i, v, in, out, B, S, st);
  }
  if (!e.exec) {
    const long long l0 = g_kernel_launches.load();
    timed_harvest(m, e.recs, true);
    m->cap_recs = &e.recs;
    SOUP_CK(cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal));
    soup_status s = dir == 0 ? layer_forward(m, i, v, in, out, B, S, m->cap_stream)
                             : layer_backward(m, i, v, in, out, B, S, m->cap_stream);
    cudaGraph_t g = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(m->cap_stream, &g);
    m->cap_recs = nullptr;
    e.launches = g_kernel_launches.load() - l0;
    g_kernel_launches -= e.launches;  // captured, not run
    if (s != SOUP_OK || ce != cudaSuccess) {
      for (auto& r : e.recs) {
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
      }
      e.recs.clear();
    }
    if (s != SOUP_OK) {
      if (g) cudaGraphDestroy(g);
      return s;
    }
    if (ce != cudaSuccess) {
      m->err = std::string("graph capture: ") + cudaGetErrorString(ce);
      return SOUP_ERR_CUDA;
    }
    const cudaError_t ie = cudaGraphInstantiate(&e.exec, g, 0);
    cudaGraphDestroy(g);
    if (ie != cudaSuccess) {
      e.exec = nullptr;
      m->err = std::string("graph instantiate: ") + cudaGetErrorString(ie);
      return SOUP_ERR_CUDA;
    }
  }
  // a graph's event nodes hold its last replay: read them before they are recorded again
  if (e.armed) timed_harvest(m, e.recs, false);
  SOUP_CK(cudaGraphLaunch(e.exec, st));
  e.armed = e.recs.empty() ? 0 : 1;
  g_kernel_launches += e.launches;
  if (dir == 0) {
    A.B = B;
    A.S = S;
    A.lora = lora;
    A.valid = 1;
  }
  return SOUP_OK;
}

soup_status stream_forward_pass(soup_model* m, int B, int S, cudaStream_t st, uint16_t** x_final) {
  const int L = m->cfg.n_layers;
  std::vector<int> order(L);
  for (int i = 0; i < L; ++i) order[i] = i;
  uint16_t* cur = m->xa;
  uint16_t* nxt = m->xb;
  for (int i = 0; i < L; ++i) {
    const uint8_t* base;
    int buf;
    SOUP_TRY(streamer_acquire(m, i, st, &base, &buf));
    SOUP_TRY(streamer_prefetch(m, order, i));
    SOUP_TRY(run_layer(m, 0, i, base, cur, nxt, B, S, st));
    SOUP_TRY(streamer_release(m, buf, st));
    std::swap(cur, nxt);
  }
  *x_final = cur;
  return SOUP_OK;
}

// DPO with one load per layer: LoRA-off (reference) and LoRA-on (policy) forward of layer i
// back to back.  The reference pass runs first and its saved activations are overwritten by
// the policy pass, which is the one the backward uses.
soup_status stream_forward_pass_shared(soup_model* m, int B, int S, cudaStream_t st, uint16_t** x_ref,
                                       uint16_t** x_pol) {
  const int L = m->cfg.n_layers;
  std::vector<int> order(L);
  for (int i = 0; i < L; ++i) order[i] = i;
  uint16_t *pc = m->xa, *pn = m->xb, *rc = m->xra, *rn = m->xrb;
  const int saved_enabled = m->lora_enabled;
  for (int i = 0; i < L; ++i) {
    const uint8_t* base;
    int buf;
    SOUP_TRY(streamer_acquire(m, i, st, &base, &buf));
    SOUP_TRY(streamer_prefetch(m, order, i));
    m->lora_enabled = 0;
    soup_status s = run_layer(m, 0, i, base, rc, rn, B, S, st);
    m->lora_enabled = 1;
    if (s == SOUP_OK) s = run_layer(m, 0, i, base, pc, pn, B, S, st);
    m->lora_enabled = saved_enabled;
    SOUP_TRY(s);
    SOUP_TRY(streamer_release(m, buf, st));
    std::swap(pc, pn);
    std::swap(rc, rn);
  }
  *x_ref = rc;
  *x_pol = pc;
  return SOUP_OK;
}

soup_status stream_backward_pass(soup_model* m, int B, int S, uint16_t* dcur, uint16_t* dnxt, cudaStream_t st) {
  const int L = m->cfg.n_layers;
  std::vector<int> order(L);
  for (int i = 0; i < L; ++i) order[i] = L - 1 - i;
  for (int k = 0; k < L; ++k) {
    const int i = order[k];
    const uint8_t* base;
    int buf;
    SOUP_TRY(streamer_acquire(m, i, st, &base, &buf));
    SOUP_TRY(streamer_prefetch(m, order, k));
    SOUP_TRY(run_layer(m, 1, i, base, dcur, dnxt, B, S, st));
    SOUP_TRY(streamer_release(m, buf, st));
    std::swap(dcur, dnxt);
  }
  return SOUP_OK;
}

soup_status read_scalars(soup_model* m, cudaStream_t st, float* loss_out) {
  SOUP_CK(cudaMemcpyAsync(m->host_scal, m->scal, 8, cudaMemcpyDeviceToHost, st));
  SOUP_TRY(wait_stream(m, st));
  int errw;
  std::memcpy(&errw, m->host_scal + 1, 4);
  if (errw != 0) {
    SOUP_CK(cudaMemsetAsync(m->scal + 1, 0, 4, st));
    m->err = errw == DEVERR_TIMEOUT ? "a kernel's bounded wait timed out" : "a kernel bounds check fired";
    return errw == DEVERR_TIMEOUT ? SOUP_ERR_TIMEOUT : SOUP_ERR_DEVICE_CHECK;
  }
  if (m->use_file) {
    const std::string fe = m->file.take_error();
    if (!fe.empty()) {
      m->err = fe;
      return SOUP_ERR_IO;
    }
  }
  if (loss_out) *loss_out = m->host_scal[0];
  return SOUP_OK;
}

soup_status do_step_body(soup_model* m, soup_loss kind, const soup_batch* bt, float* loss_out, cudaStream_t st);
soup_status do_step(soup_model* m, soup_loss kind, const soup_batch* bt, float* loss_out, cudaStream_t st) {
  const NvtxRange trace("step");
  if (m->prof) {
    // the profile's own per-launch overhead: empty launches bracketed like every other one
    for (int k = 0; k < 8; ++k) SOUP_TRY(launch(m, st, CAT_NULL, 0.0, 0.0, "empty launch", [&] { return null_launch(st); }));
  }
  const soup_status s = do_step_body(m, kind, bt, loss_out, st);
  m->pack_pl = m->pack_rl = 0;
  return s;
}

soup_status do_step_body(soup_model* m, soup_loss kind, const soup_batch* bt, float* loss_out, cudaStream_t st) {
  const soup_model_config& c = m->cfg;
  if (!m->embed || !m->lm_head || !m->final_gamma) {
    m->err = "head weights not set";
    return SOUP_ERR_STATE;
  }
  if (!m->lora_p) {
    m->err = "LoRA storage not set";
    return SOUP_ERR_STATE;
  }
  const int B = bt->B, S = bt->S, T = B * S;
  if (B < 1 || S < 2 || T > c.max_tokens || !bt->ids) {
    m->err = "batch: need B >= 1, S >= 2, B*S <= max_tokens and ids";
    return SOUP_ERR_INVALID_ARG;
  }
  const bool paired = kind == SOUP_LOSS_DPO || kind == SOUP_LOSS_SIMPO || kind == SOUP_LOSS_ORPO;
  const bool needs_ref = kind == SOUP_LOSS_DPO || kind == SOUP_LOSS_KTO;
  if (paired && (bt->n_pairs < 1 || 2 * bt->n_pairs != B || B > 256 || bt->prefix_len < 0 || bt->prefix_len >= S)) {
    m->err = "preference batch: B must be 2*n_pairs <= 256 and 0 <= prefix_len < S";
    return SOUP_ERR_INVALID_ARG;
  }
  if (kind == SOUP_LOSS_KTO && (!bt->labels || B > 256 || bt->prefix_len < 0 || bt->prefix_len >= S)) {
    m->err = "KTO batch: labels[B] required, B <= 256 and 0 <= prefix_len < S";
    return SOUP_ERR_INVALID_ARG;
  }
  for (int i = 0; i < c.n_layers; ++i)
    if (!m->host_loaded[i]) {
      m->err = "layer " + std::to_string(i) + " has no weights loaded";
      return SOUP_ERR_STATE;
    }
  const long long launches0 = g_kernel_launches.load();
  // inputs
  SOUP_CK(cudaMemcpyAsync(m->ids_dev, bt->ids, static_cast<size_t>(T) * 4,
                          bt->ids_on_host ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice, st));
  const uint8_t* mask = nullptr;
  if (bt->loss_mask) {
    SOUP_CK(cudaMemcpyAsync(m->mask_dev, bt->loss_mask, static_cast<size_t>(T),
                            bt->ids_on_host ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice, st));
    mask = m->mask_dev;
  }
  if (kind == SOUP_LOSS_KTO)
    SOUP_CK(cudaMemcpyAsync(m->labels_dev, bt->labels, static_cast<size_t>(B),
                            bt->ids_on_host ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToDevice, st));
  // Shared-prefix pair blocks: each pair's common prefix runs once, [prefix | chosen |
  // rejected] (when the prefix and response lengths are multiples of the 64-row attention tile;
  // otherwise the plain layout).  Bx x Sx are the rows the layers see.
  const int pl = bt->prefix_len, rl = S - bt->prefix_len;
  const bool share = bt->share_prefix && paired && pl >= 64 && pl % 64 == 0 && rl % 64 == 0;
  const int Bx = share ? bt->n_pairs : B, Sx = share ? pl + 2 * rl : S, Tx = Bx * Sx;
  const int32_t* ids_x = m->ids_dev;
  if (share) {
    SOUP_TRY(check_launch(m, pair_pack_launch(m->ids_dev, bt->n_pairs, S, pl, c.vocab, m->pids, m->tgt1, m->tgt2,
                                              m->scal + 1, st),
                          "pair pack"));
    m->pack_pl = pl;
    m->pack_rl = rl;
    ids_x = m->pids;
  }
  SOUP_CK(cudaMemsetAsync(m->lora_g, 0, m->lora_n * sizeof(float), st));
  const int saved_enabled = m->lora_enabled;
  uint16_t* xL = nullptr;
  if (needs_ref && bt->dpo_shared_load) {
    SOUP_TRY(streamer_warm(m, 0, 2));
    SOUP_TRY(launch(m, st, CAT_EMBED, 0, 4.0 * Tx * c.hidden, "embed", [&] {
      return embed_launch(ids_x, m->embed, Tx, c.hidden, c.vocab, m->xa, m->scal + 1, st);
    }));
    SOUP_TRY(launch(m, st, CAT_D2D, 0, 4.0 * Tx * c.hidden, "embed copy", [&] {
      return cudaMemcpyAsync(m->xra, m->xa, static_cast<size_t>(Tx) * c.hidden * 2, cudaMemcpyDeviceToDevice, st);
    }));
    uint16_t* xR = nullptr;
    SOUP_TRY(stream_forward_pass_shared(m, Bx, Sx, st, &xR, &xL));
    SOUP_TRY(head_forward(m, xR, Bx, Sx, st));
    SOUP_TRY(check_launch(m,
                          share ? pair_logp_launch(m->rowlse, m->rowtgt, m->rowtgt2, Bx, pl, rl, m->ref, st)
                                : seq_logp_launch(m->rowlse, m->rowtgt, B, S, bt->prefix_len, m->ref, st),
                          "ref logp"));
    SOUP_TRY(head_forward(m, xL, Bx, Sx, st));
  } else {
  if (needs_ref) {
    // reference: same streamed base, LoRA off
    m->lora_enabled = 0;
    SOUP_TRY(streamer_warm(m, 0, 2));
    SOUP_TRY(launch(m, st, CAT_EMBED, 0, 4.0 * Tx * c.hidden, "embed", [&] {
      return embed_launch(ids_x, m->embed, Tx, c.hidden, c.vocab, m->xa, m->scal + 1, st);
    }));
    soup_status s1 = stream_forward_pass(m, Bx, Sx, st, &xL);
    if (s1 != SOUP_OK) {
      m->lora_enabled = saved_enabled;
      return s1;
    }
    SOUP_TRY(head_forward(m, xL, Bx, Sx, st));
    SOUP_TRY(check_launch(m,
                          share ? pair_logp_launch(m->rowlse, m->rowtgt, m->rowtgt2, Bx, pl, rl, m->ref, st)
                                : seq_logp_launch(m->rowlse, m->rowtgt, B, S, bt->prefix_len, m->ref, st),
                          "ref logp"));
    m->lora_enabled = 1;
  }
  SOUP_TRY(streamer_warm(m, 0, 2));
  SOUP_TRY(launch(m, st, CAT_EMBED, 0, 4.0 * Tx * c.hidden, "embed", [&] {
    return embed_launch(ids_x, m->embed, Tx, c.hidden, c.vocab, m->xa, m->scal + 1, st);
  }));
  soup_status s2 = stream_forward_pass(m, Bx, Sx, st, &xL);
  m->lora_enabled = saved_enabled;
  if (s2 != SOUP_OK) return s2;
  SOUP_TRY(head_forward(m, xL, Bx, Sx, st));
  }
  float* loss_dev = reinterpret_cast<float*>(m->scal);
  if (share) {
    SOUP_TRY(check_launch(m, pair_logp_launch(m->rowlse, m->rowtgt, m->rowtgt2, Bx, pl, rl, m->pi, st), "pair logp"));
    if (kind == SOUP_LOSS_DPO)
      SOUP_TRY(check_launch(m, dpo_loss_seqw_launch(m->pi, m->ref, bt->n_pairs, bt->beta, loss_dev, m->seqw, st),
                            "dpo loss"));
    else
      SOUP_TRY(check_launch(m, pref_loss_seqw_launch(static_cast<int>(kind), m->pi, m->ref, m->labels_dev, B, rl,
                                                     bt->beta, bt->gamma, bt->lambda_or, bt->lambda_d, bt->lambda_u,
                                                     loss_dev, m->seqw, st),
                            "preference loss"));
    SOUP_TRY(check_launch(m, pair_rowweight_launch(m->seqw, Bx, pl, rl, m->roww, m->roww2, st), "pair weights"));
  } else if (kind == SOUP_LOSS_SFT) {
    SOUP_TRY(check_launch(m, sft_finish_launch(m->rowlse, m->rowtgt, m->ids_dev, B, S, mask, loss_dev, m->roww, st),
                          "sft loss"));
  } else if (kind == SOUP_LOSS_DPO) {
    SOUP_TRY(check_launch(m, dpo_finish_launch(m->rowlse, m->rowtgt, B, S, bt->prefix_len, bt->n_pairs, bt->beta,
                                               m->ref, m->pi, loss_dev, m->roww, st),
                          "dpo loss"));
  } else {
    SOUP_TRY(check_launch(m, pref_finish_launch(static_cast<int>(kind), m->rowlse, m->rowtgt, B, S, bt->prefix_len,
                                                m->ref, m->labels_dev, bt->beta, bt->gamma, bt->lambda_or,
                                                bt->lambda_d, bt->lambda_u, m->pi, loss_dev, m->roww, st),
                          "preference loss"));
  }
  uint16_t* other = (xL == m->xa) ? m->xb : m->xa;
  SOUP_TRY(head_backward(m, xL, Bx, Sx, other, st));
  if (bt->apply_optimizer) {
    // this step's lr and bias corrections, for the AdamW launches inside the backward pass
    // (the pinned staging words are free: the previous step's read-back has completed)
    m->adam_t += 1;
    float* hp = m->host_scal + 4;
    hp[0] = bt->lr;
    adamw_bias_corrections(ADAM_B1, ADAM_B2, m->adam_t, &hp[1], &hp[2]);
    SOUP_CK(cudaMemcpyAsync(m->scal + ADAM_HP_WORD, hp, 3 * sizeof(float), cudaMemcpyHostToDevice, st));
    m->adam_in_bwd = 1;
  }
  // backward ping-pongs between `other` and the buffer that held x_L (no longer needed); with
  // the optimizer on, layer i's call also updates layer i+1's LoRA slice
  const soup_status sb = stream_backward_pass(m, Bx, Sx, other, xL, st);
  m->adam_in_bwd = 0;
  SOUP_TRY(sb);
  if (bt->apply_optimizer) SOUP_TRY(adamw_layer(m, 0, st));  // the last slice
  m->stats.kernel_launches += g_kernel_launches.load() - launches0;
  SOUP_TRY(read_scalars(m, st, loss_out));
  m->stats.steps += 1;
  return SOUP_OK;
}

void clear_graphs(soup_model* m) {
  for (auto& kv : m->graphs) {
    if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
    for (auto& r : kv.second.recs) {
      cudaEventDestroy(r.a);
      cudaEventDestroy(r.b);
    }
  }
  m->graphs.clear();
}

soup_status destroy_model(soup_model* m) {
  if (m->copy_stream) cudaStreamSynchronize(m->copy_stream);
  cudaDeviceSynchronize();
  for (void* p : m->dev_allocs) {
    if (m->has_alloc)
      m->alloc.free(p, m->alloc.user);
    else
      cudaFree(p);
  }
  for (uint8_t* h : m->host_blob)
    if (h) cudaFreeHost(h);
  m->file.close();
  if (m->host_scal) cudaFreeHost(m->host_scal);
  clear_graphs(m);
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  if (m->grad_stream) cudaStreamDestroy(m->grad_stream);
  if (m->fork_ev) cudaEventDestroy(m->fork_ev);
  if (m->join_ev) cudaEventDestroy(m->join_ev);
  for (auto& r : m->prof_pending) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : m->prof_pool) cudaEventDestroy(e);
  for (auto& r : m->tpending) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : m->copy_done) cudaEventDestroy(e);
  for (auto e : m->buf_free) cudaEventDestroy(e);
  if (m->copy_stream) cudaStreamDestroy(m->copy_stream);
  delete m;
  return SOUP_OK;
}

soup_status create_model(const soup_model_config* cfg, const soup_allocator* alloc, soup_model** out) {
  soup_model* m = new soup_model();
  m->cfg = *cfg;
  std::string why;
  soup_status vs = validate_cfg(*cfg, why);
  if (vs != SOUP_OK) {
    delete m;
    return vs;
  }
  if (alloc && alloc->alloc && alloc->free) {
    m->alloc = *alloc;
    m->has_alloc = true;
  }
  auto fail = [&](soup_status s) {
    destroy_model(m);
    return s;
  };
  if (cudaSetDevice(cfg->device) != cudaSuccess) return fail(SOUP_ERR_CUDA);
  const soup_model_config& c = m->cfg;
  m->layout = blob_layout(c);
  m->qkv_cols = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim;
  m->s_lora = c.lora_alpha / static_cast<float>(c.lora_r);
  (void)codebook();
  const int L = c.n_layers;
  m->host_blob.assign(L, nullptr);
  m->host_loaded.assign(L, 0);
  m->use_file = c.stream_source == SOUP_SOURCE_FILE;
  if (c.stream_source == SOUP_SOURCE_AUTO && c.stack_path && c.stack_path[0]) {
    // RAM when the stack fits in half of the free physical memory, else the file
    const double free_bytes = static_cast<double>(sysconf(_SC_AVPHYS_PAGES)) * static_cast<double>(sysconf(_SC_PAGESIZE));
    m->use_file = static_cast<double>(m->layout.total) * L > 0.5 * free_bytes;
  }
  if (m->use_file) {
    const int slots = std::max(2, c.n_layer_buffers);
    if (!m->file.open(c.stack_path, L, m->layout.total, slots, static_cast<long long>(wait_limit_ms()), m->err)) {
      std::fprintf(stderr, "libsoup: %s\n", m->err.c_str());
      return fail(SOUP_ERR_IO);
    }
    m->stats.pinned_bytes += static_cast<long long>(m->layout.total) * slots;
  } else {
    for (int i = 0; i < L; ++i) {
      if (cudaHostAlloc(reinterpret_cast<void**>(&m->host_blob[i]), m->layout.total, cudaHostAllocDefault) !=
          cudaSuccess)
        return fail(SOUP_ERR_OOM);
      m->stats.pinned_bytes += static_cast<long long>(m->layout.total);
    }
  }
  if (cudaHostAlloc(reinterpret_cast<void**>(&m->host_scal), 64, cudaHostAllocDefault) != cudaSuccess)
    return fail(SOUP_ERR_OOM);
  const int nbuf = (c.mode == SOUP_RESIDENT) ? L : c.n_layer_buffers;
  for (int b = 0; b < nbuf; ++b) {
    uint8_t* p = static_cast<uint8_t*>(dev_alloc(m, m->layout.total));
    if (!p) return fail(SOUP_ERR_OOM);
    m->dev_buf.push_back(p);
  }
  m->buf_layer.assign(nbuf, -1);
  m->buf_last.assign(nbuf, 0);
  m->buf_inuse.assign(nbuf, 0);
  if (cudaStreamCreateWithFlags(&m->copy_stream, cudaStreamNonBlocking) != cudaSuccess) return fail(SOUP_ERR_CUDA);
  if (cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking) != cudaSuccess) return fail(SOUP_ERR_CUDA);
  {
    const char* e = std::getenv("SOUP_GRAPHS");
    m->use_graphs = (e && e[0] == '0') ? 0 : 1;
    const char* g = std::getenv("SOUP_CONCURRENT_GRADS");
    m->concurrent_grads = (g && g[0] == '0') ? 0 : 1;
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return fail(SOUP_ERR_CUDA);
    if (cudaStreamCreateWithPriority(&m->grad_stream, cudaStreamNonBlocking, least) != cudaSuccess ||
        cudaEventCreateWithFlags(&m->fork_ev, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&m->join_ev, cudaEventDisableTiming) != cudaSuccess)
      return fail(SOUP_ERR_CUDA);
  }
  m->copy_done.resize(nbuf);
  m->buf_free.resize(nbuf);
  for (int b = 0; b < nbuf; ++b) {
    if (cudaEventCreateWithFlags(&m->copy_done[b], cudaEventDisableTiming) != cudaSuccess) return fail(SOUP_ERR_CUDA);
    if (cudaEventCreateWithFlags(&m->buf_free[b], cudaEventDisableTiming) != cudaSuccess) return fail(SOUP_ERR_CUDA);
  }
  // activations
  const size_t T = static_cast<size_t>(c.max_tokens), h = c.hidden, r = c.lora_r, I = c.intermediate;
  const size_t qd = static_cast<size_t>(c.n_heads) * c.head_dim, QKV = m->qkv_cols;
  m->saved.resize(L);
  for (int i = 0; i < L; ++i) {
    Saved& A = m->saved[i];
    if (alloc_into(m, A.x, T * h) || alloc_into(m, A.n1, T * h) || alloc_into(m, A.qkv, T * QKV) ||
        alloc_into(m, A.uqkv, T * 3 * r) || alloc_into(m, A.o, T * qd) || alloc_into(m, A.uo, T * r) ||
        alloc_into(m, A.x1, T * h) || alloc_into(m, A.n2, T * h) || alloc_into(m, A.gu, T * 2 * I) ||
        alloc_into(m, A.ugu, T * 2 * r) || alloc_into(m, A.m, T * I) || alloc_into(m, A.ud, T * r) ||
        alloc_into(m, A.rstd1, T) || alloc_into(m, A.rstd2, T) || alloc_into(m, A.lse, T * c.n_heads))
      return fail(SOUP_ERR_OOM);
  }
  const size_t V = c.vocab;
  if (alloc_into(m, m->xa, T * h) || alloc_into(m, m->xb, T * h) || alloc_into(m, m->xra, T * h) ||
      alloc_into(m, m->xrb, T * h) || alloc_into(m, m->dqkv, T * QKV) ||
      alloc_into(m, m->dgu, T * 2 * I) || alloc_into(m, m->dm, T * I) || alloc_into(m, m->da, T * qd) ||
      alloc_into(m, m->dn, T * h) || alloc_into(m, m->dx1, T * h) || alloc_into(m, m->vqkv, T * 3 * r) ||
      alloc_into(m, m->vo, T * r) || alloc_into(m, m->vgu, T * 2 * r) || alloc_into(m, m->vd, T * r) ||
      alloc_into(m, m->hf, T * h) || alloc_into(m, m->dh, T * h) || alloc_into(m, m->dlogits, T * V) ||
      alloc_into(m, m->delta, T * c.n_heads) || alloc_into(m, m->logits, T * V) || alloc_into(m, m->rowlse, T) ||
      alloc_into(m, m->rowtgt, T) || alloc_into(m, m->roww, T) || alloc_into(m, m->rstdf, T) ||
      alloc_into(m, m->pi, T) || alloc_into(m, m->ref, T) || alloc_into(m, m->ids_dev, T) ||
      alloc_into(m, m->mask_dev, T) || alloc_into(m, m->labels_dev, T) || alloc_into(m, m->pids, T) ||
      alloc_into(m, m->tgt1, T) || alloc_into(m, m->tgt2, T) || alloc_into(m, m->rowtgt2, T) ||
      alloc_into(m, m->roww2, T) || alloc_into(m, m->seqw, 256) || alloc_into(m, m->scal, 64))
    return fail(SOUP_ERR_OOM);
  {  // RoPE tables: angle = pos * theta^(-2i/d), computed in float64, stored as float32
    const int half = c.head_dim / 2;
    std::vector<float> hc(static_cast<size_t>(T) * half), hs(hc.size());
    for (size_t pos = 0; pos < T; ++pos)
      for (int i = 0; i < half; ++i) {
        const double ang = static_cast<double>(pos) * std::pow(static_cast<double>(c.rope_theta), -2.0 * i / c.head_dim);
        hc[pos * half + i] = static_cast<float>(std::cos(ang));
        hs[pos * half + i] = static_cast<float>(std::sin(ang));
      }
    if (alloc_into(m, m->rope_cos, hc.size()) || alloc_into(m, m->rope_sin, hs.size())) return fail(SOUP_ERR_OOM);
    if (cudaMemcpy(m->rope_cos, hc.data(), hc.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(m->rope_sin, hs.data(), hs.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
      return fail(SOUP_ERR_CUDA);
  }
  m->gemm_ws_bytes = static_cast<size_t>(64) << 20;
  if (alloc_into(m, m->gemm_ws, m->gemm_ws_bytes / sizeof(float))) return fail(SOUP_ERR_OOM);
  m->gemm_ws2_bytes = m->gemm_ws_bytes;
  if (alloc_into(m, m->gemm_ws2, m->gemm_ws2_bytes / sizeof(float))) return fail(SOUP_ERR_OOM);
  if (alloc_into(m, m->gemm_cnt, GEMM_COUNTERS) || alloc_into(m, m->gemm_cnt2, GEMM_COUNTERS)) return fail(SOUP_ERR_OOM);
  if (cudaMemset(m->gemm_cnt, 0, GEMM_COUNTERS * sizeof(int)) != cudaSuccess ||
      cudaMemset(m->gemm_cnt2, 0, GEMM_COUNTERS * sizeof(int)) != cudaSuccess)
    return fail(SOUP_ERR_CUDA);
  if (cudaMemset(m->scal, 0, 64 * sizeof(int)) != cudaSuccess) return fail(SOUP_ERR_CUDA);
  m->lora_n = lora_numel_of(c);
  if (alloc_into(m, m->lora_bf16, m->lora_n)) return fail(SOUP_ERR_OOM);
  *out = m;
  return SOUP_OK;
}

soup_status quantize_layer(soup_model* m, int layer, const float* const w[7], const uint16_t* ga, const uint16_t* gm,
                           cudaStream_t st) {
  const soup_model_config& c = m->cfg;
  ProjShape s[7];
  proj_shapes(c, s);
  if (!m->quant_scratch) {
    long long mx = 0;
    for (int p = 0; p < 7; ++p) mx = std::max(mx, (static_cast<long long>(s[p].out) * s[p].in + 63) / 64);
    if (alloc_into(m, m->quant_scratch, static_cast<size_t>(mx))) return SOUP_ERR_OOM;
  }
  // quantise into a device buffer (the layer's resident buffer, or a streamer buffer that is
  // then marked stale), then copy the blob to page-locked host memory
  uint8_t* dst;
  int stale_buf = -1;
  if (c.mode == SOUP_RESIDENT) {
    dst = m->dev_buf[layer];
  } else {
    int b = -1;
    for (int i = 0; i < static_cast<int>(m->dev_buf.size()); ++i)
      if (!m->buf_inuse[i] && (b < 0 || m->buf_last[i] < m->buf_last[b])) b = i;
    if (b < 0) {
      m->err = "no free layer buffer to quantise into";
      return SOUP_ERR_STATE;
    }
    SOUP_CK(cudaStreamWaitEvent(st, m->buf_free[b], 0));
    SOUP_CK(cudaStreamWaitEvent(st, m->copy_done[b], 0));
    dst = m->dev_buf[b];
    stale_buf = b;
  }
  for (int p = 0; p < 7; ++p) {
    const long long n = static_cast<long long>(s[p].out) * s[p].in;
    SOUP_TRY(check_launch(m,
                          nf4_quantize_launch(w[p], n, dst + m->layout.off[p][0],
                                              reinterpret_cast<int8_t*>(dst + m->layout.off[p][1]),
                                              reinterpret_cast<float*>(dst + m->layout.off[p][2]),
                                              reinterpret_cast<float*>(dst + m->layout.off[p][3]), m->quant_scratch,
                                              codebook(), st),
                          "nf4 quantize"));
  }
  SOUP_CK(cudaMemcpyAsync(dst + m->layout.off[7][0], ga, static_cast<size_t>(c.hidden) * 2, cudaMemcpyDeviceToDevice, st));
  SOUP_CK(cudaMemcpyAsync(dst + m->layout.off[8][0], gm, static_cast<size_t>(c.hidden) * 2, cudaMemcpyDeviceToDevice, st));
  std::vector<uint8_t> staged;
  if (m->use_file) {
    staged.resize(m->layout.total);
    SOUP_CK(cudaMemcpyAsync(staged.data(), dst, m->layout.total, cudaMemcpyDeviceToHost, st));
  } else {
    SOUP_CK(cudaMemcpyAsync(m->host_blob[layer], dst, m->layout.total, cudaMemcpyDeviceToHost, st));
  }
  SOUP_TRY(wait_stream(m, st));
  if (m->use_file && !m->file.write(layer, staged.data(), m->err)) return SOUP_ERR_IO;
  if (stale_buf >= 0) {
    m->buf_layer[stale_buf] = -1;
    SOUP_CK(cudaEventRecord(m->buf_free[stale_buf], st));
  }
  // any streamer buffer holding an older copy of this layer is now stale
  if (c.mode == SOUP_STREAMED)
    for (size_t b = 0; b < m->buf_layer.size(); ++b)
      if (m->buf_layer[b] == layer) m->buf_layer[b] = -1;
  m->host_loaded[layer] = 1;
  return SOUP_OK;
}

}  // namespace
}  // namespace soup

// ====================================================================== C-ABI
using namespace soup;

#define SOUP_GUARD(body)                                          \
  try {                                                           \
    body                                                          \
  } catch (const std::exception& ex) {                            \
    if (m) m->err = ex.what();                                    \
    return SOUP_ERR_INVALID_ARG;                                  \
  } catch (...) {                                                 \
    return SOUP_ERR_INVALID_ARG;                                  \
  }

extern "C" {

const char* soup_status_string(soup_status s) {
  switch (s) {
    case SOUP_OK: return "ok";
    case SOUP_ERR_INVALID_ARG: return "invalid argument";
    case SOUP_ERR_STATE: return "invalid call order or state";
    case SOUP_ERR_OOM: return "out of memory";
    case SOUP_ERR_CUDA: return "CUDA error";
    case SOUP_ERR_TIMEOUT: return "timed out";
    case SOUP_ERR_DEVICE_CHECK: return "device bounds check fired";
    case SOUP_ERR_UNSUPPORTED: return "unsupported shape";
    case SOUP_ERR_IO: return "layer stack file I/O failed";
    default: return "unknown status";
  }
}

const char* soup_last_error(const soup_model* m) { return m ? m->err.c_str() : ""; }

soup_status soup_layer_blob_bytes(const soup_model_config* cfg, size_t* bytes) {
  if (!cfg || !bytes) return SOUP_ERR_INVALID_ARG;
  std::string why;
  soup_status s = validate_cfg(*cfg, why);
  if (s != SOUP_OK) return s;
  *bytes = blob_layout(*cfg).total;
  return SOUP_OK;
}

soup_status soup_layer_blob_part(const soup_model_config* cfg, int proj, int part, size_t* offset, size_t* bytes) {
  if (!cfg || !offset || !bytes || proj < 0 || proj > 8 || part < 0 || part > 3) return SOUP_ERR_INVALID_ARG;
  if (proj >= 7 && part != 0) return SOUP_ERR_INVALID_ARG;
  std::string why;
  soup_status s = validate_cfg(*cfg, why);
  if (s != SOUP_OK) return s;
  const BlobLayout L = blob_layout(*cfg);
  *offset = L.off[proj][part];
  *bytes = L.sz[proj][part];
  return SOUP_OK;
}

soup_status soup_lora_numel(const soup_model_config* cfg, size_t* numel) {
  if (!cfg || !numel) return SOUP_ERR_INVALID_ARG;
  std::string why;
  soup_status s = validate_cfg(*cfg, why);
  if (s != SOUP_OK) return s;
  *numel = lora_numel_of(*cfg);
  return SOUP_OK;
}

soup_status soup_lora_offset(const soup_model_config* cfg, int layer, int proj, int which_b, size_t* offset, int* rows,
                             int* cols) {
  if (!cfg || !offset || layer < 0 || layer >= cfg->n_layers || proj < 0 || proj >= 7 || which_b < 0 || which_b > 1)
    return SOUP_ERR_INVALID_ARG;
  std::string why;
  soup_status s = validate_cfg(*cfg, why);
  if (s != SOUP_OK) return s;
  ProjShape sh[7];
  proj_shapes(*cfg, sh);
  *offset = lora_off(*cfg, layer, proj, which_b);
  if (rows) *rows = which_b ? sh[proj].out : cfg->lora_r;
  if (cols) *cols = which_b ? cfg->lora_r : sh[proj].in;
  return SOUP_OK;
}

soup_status soup_model_create(const soup_model_config* cfg, const soup_allocator* alloc, soup_model** out) {
  soup_model* m = nullptr;
  if (!cfg || !out) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD(return create_model(cfg, alloc, out);)
}

soup_status soup_model_destroy(soup_model* m) {
  if (!m) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD(return destroy_model(m);)
}

soup_status soup_model_quantize_layer(soup_model* m, int layer, const float* const w[7], const uint16_t* gamma_attn,
                                      const uint16_t* gamma_mlp, void* stream) {
  if (!m || !w || !gamma_attn || !gamma_mlp || layer < 0 || layer >= m->cfg.n_layers) return SOUP_ERR_INVALID_ARG;
  for (int p = 0; p < 7; ++p)
    if (!w[p]) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD(return quantize_layer(m, layer, w, gamma_attn, gamma_mlp, static_cast<cudaStream_t>(stream));)
}

soup_status soup_model_load_layer_nf4(soup_model* m, int layer, const void* blob, size_t bytes) {
  if (!m || !blob || layer < 0 || layer >= m->cfg.n_layers) return SOUP_ERR_INVALID_ARG;
  if (bytes != m->layout.total) {
    m->err = "blob size mismatch";
    return SOUP_ERR_INVALID_ARG;
  }
  SOUP_GUARD({
    if (m->use_file) {
      if (!m->file.write(layer, blob, m->err)) return SOUP_ERR_IO;
    } else {
      std::memcpy(m->host_blob[layer], blob, bytes);
    }
    if (m->cfg.mode == SOUP_RESIDENT) {
      SOUP_CK(cudaMemcpy(m->dev_buf[layer], blob, bytes, cudaMemcpyHostToDevice));
    } else {
      for (size_t b = 0; b < m->buf_layer.size(); ++b)
        if (m->buf_layer[b] == layer) m->buf_layer[b] = -1;
    }
    m->host_loaded[layer] = 1;
    return SOUP_OK;
  })
}

soup_status soup_model_load_layer(soup_model* m, int layer, const float* const w[7], const uint16_t* gamma_attn,
                                  const uint16_t* gamma_mlp) {
  if (!m || !w || !gamma_attn || !gamma_mlp || layer < 0 || layer >= m->cfg.n_layers) return SOUP_ERR_INVALID_ARG;
  for (int p = 0; p < 7; ++p)
    if (!w[p]) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD({
    // the streamer may still be copying an older blob of this layer out of page-locked memory
    if (m->copy_stream) SOUP_TRY(wait_stream(m, m->copy_stream));
    std::vector<uint8_t> staged;
    uint8_t* dst;
    if (m->use_file) {
      staged.assign(m->layout.total, 0);
      dst = staged.data();
    } else {
      dst = m->host_blob[layer];
      std::memset(dst, 0, m->layout.total);
    }
    ProjShape s[7];
    proj_shapes(m->cfg, s);
    for (int p = 0; p < 7; ++p) {
      const long long n = static_cast<long long>(s[p].out) * s[p].in;
      const int st = host_nf4_quantize(w[p], n, dst + m->layout.off[p][0],
                                       reinterpret_cast<int8_t*>(dst + m->layout.off[p][1]),
                                       reinterpret_cast<float*>(dst + m->layout.off[p][2]),
                                       reinterpret_cast<float*>(dst + m->layout.off[p][3]), 0);
      if (st != SOUP_OK) {
        m->host_loaded[layer] = 0;
        m->err = "host NF4 quantiser failed";
        return st;
      }
    }
    std::memcpy(dst + m->layout.off[7][0], gamma_attn, static_cast<size_t>(m->cfg.hidden) * 2);
    std::memcpy(dst + m->layout.off[8][0], gamma_mlp, static_cast<size_t>(m->cfg.hidden) * 2);
    if (m->use_file && !m->file.write(layer, dst, m->err)) return SOUP_ERR_IO;
    if (m->cfg.mode == SOUP_RESIDENT) {
      SOUP_CK(cudaMemcpy(m->dev_buf[layer], dst, m->layout.total, cudaMemcpyHostToDevice));
    } else {
      for (size_t b = 0; b < m->buf_layer.size(); ++b)
        if (m->buf_layer[b] == layer) m->buf_layer[b] = -1;
    }
    m->host_loaded[layer] = 1;
    return SOUP_OK;
  })
}

soup_status soup_model_read_layer_nf4(soup_model* m, int layer, void* blob, size_t bytes) {
  if (!m || !blob || layer < 0 || layer >= m->cfg.n_layers || bytes != m->layout.total) return SOUP_ERR_INVALID_ARG;
  if (!m->host_loaded[layer]) return SOUP_ERR_STATE;
  if (m->use_file) return m->file.read(layer, blob, m->err) ? SOUP_OK : SOUP_ERR_IO;
  std::memcpy(blob, m->host_blob[layer], bytes);
  return SOUP_OK;
}

soup_status soup_model_set_head(soup_model* m, const void* embed, const void* final_gamma, const void* lm_head) {
  if (!m || !embed || !final_gamma || !lm_head) return SOUP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(embed) | reinterpret_cast<uintptr_t>(lm_head) |
       reinterpret_cast<uintptr_t>(final_gamma)) & 15u) {
    m->err = "head weights must be 16-byte aligned";
    return SOUP_ERR_INVALID_ARG;
  }
  m->embed = static_cast<const uint16_t*>(embed);
  m->final_gamma = static_cast<const uint16_t*>(final_gamma);
  m->lm_head = static_cast<const uint16_t*>(lm_head);
  return SOUP_OK;
}

soup_status soup_model_set_lora(soup_model* m, float* params, float* grads, float* adam_m, float* adam_v) {
  if (!m || !params || !grads || !adam_m || !adam_v) return SOUP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(params) | reinterpret_cast<uintptr_t>(grads) | reinterpret_cast<uintptr_t>(adam_m) |
       reinterpret_cast<uintptr_t>(adam_v)) & 15u) {
    m->err = "LoRA buffers must be 16-byte aligned";
    return SOUP_ERR_INVALID_ARG;
  }
  clear_graphs(m);
  m->lora_p = params;
  m->lora_g = grads;
  m->lora_m = adam_m;
  m->lora_v = adam_v;
  m->adam_t = 0;
  for (auto& a : m->saved) a.valid = 0;
  SOUP_GUARD({
    SOUP_TRY(check_launch(m, f32_to_bf16_launch(params, m->lora_bf16, static_cast<long long>(m->lora_n), nullptr),
                          "lora copy"));
    SOUP_CK(cudaDeviceSynchronize());
    return SOUP_OK;
  })
}

soup_status soup_model_set_lora_proj(soup_model* m, int layer, int proj, const float* A, const float* B,
                                     void* stream) {
  if (!m || !A || !B || layer < 0 || layer >= m->cfg.n_layers || proj < 0 || proj > 6) return SOUP_ERR_INVALID_ARG;
  if (!m->lora_p) {
    m->err = "soup_model_set_lora first";
    return SOUP_ERR_STATE;
  }
  SOUP_GUARD({
    ProjShape s[7];
    proj_shapes(m->cfg, s);
    const int r = m->cfg.lora_r;
    const size_t na = static_cast<size_t>(r) * s[proj].in;
    const size_t nbb = static_cast<size_t>(s[proj].out) * r;
    const size_t oa = lora_off(m->cfg, layer, proj, 0);
    const size_t ob = lora_off(m->cfg, layer, proj, 1);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    SOUP_CK(cudaMemcpyAsync(m->lora_p + oa, A, na * sizeof(float), cudaMemcpyDefault, st));
    SOUP_CK(cudaMemcpyAsync(m->lora_p + ob, B, nbb * sizeof(float), cudaMemcpyDefault, st));
    SOUP_TRY(check_launch(m, f32_to_bf16_launch(m->lora_p + oa, m->lora_bf16 + oa, static_cast<long long>(na), st),
                          "lora copy"));
    SOUP_TRY(check_launch(m, f32_to_bf16_launch(m->lora_p + ob, m->lora_bf16 + ob, static_cast<long long>(nbb), st),
                          "lora copy"));
    for (auto& a : m->saved) a.valid = 0;
    return SOUP_OK;
  })
}

soup_status soup_model_refresh_lora(soup_model* m, void* stream) {
  if (!m) return SOUP_ERR_INVALID_ARG;
  if (!m->lora_p) return SOUP_ERR_STATE;
  SOUP_GUARD(return check_launch(m, f32_to_bf16_launch(m->lora_p, m->lora_bf16, static_cast<long long>(m->lora_n),
                                                       static_cast<cudaStream_t>(stream)),
                                 "lora copy");)
}

soup_status soup_set_lora_enabled(soup_model* m, int enabled) {
  if (!m) return SOUP_ERR_INVALID_ARG;
  m->lora_enabled = enabled ? 1 : 0;
  return SOUP_OK;
}

soup_status soup_model_merge_lora(soup_model* m, int layer, int proj, void* out, void* stream) {
  if (!m || !out || layer < 0 || layer >= m->cfg.n_layers || proj < 0 || proj > 6) return SOUP_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(out) & 15u) return SOUP_ERR_INVALID_ARG;
  if (!m->lora_p || !m->host_loaded[layer]) return SOUP_ERR_STATE;
  SOUP_GUARD({
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long l0 = g_kernel_launches.load();
    const uint8_t* base;
    int buf;
    SOUP_TRY(streamer_acquire(m, layer, st, &base, &buf));
    const LayerView v = view_of(m, base);
    ProjShape sh[7];
    proj_shapes(m->cfg, sh);
    const int rows = sh[proj].out;
    const int cols = sh[proj].in;
    const int r = m->cfg.lora_r;
    const NF4Seg& w = v.seg[proj];
    soup_status s = check_launch(m,
                                 nf4_dequant_launch(w.codes, w.q8, w.scales, w.mean,
                                                    static_cast<long long>(rows) * cols, static_cast<uint16_t*>(out),
                                                    codebook(), st),
                                 "merge dequant");
    if (s == SOUP_OK) {
      // out[rows, cols] += s * B[rows, r] . A[r, cols]: A operand B K-major (ld r), B operand
      // A^T read MN-major (element (n, k) at A[k * cols + n])
      const uint16_t* P = m->lora_bf16;
      GemmParams p = gemm_base(m, rows, cols, out, cols, 0, m->s_lora);
      p.residual = out;
      p.ldr = cols;
      add_seg(p, r, opnd(OP_BF16_K, P + lora_off(m->cfg, layer, proj, 1), r),
              opnd(OP_BF16_MN, P + lora_off(m->cfg, layer, proj, 0), cols));
      s = run_gemm(m, p, st, "merge lora");
    }
    soup_status s2 = streamer_release(m, buf, st);
    m->stats.kernel_launches += g_kernel_launches.load() - l0;
    return s != SOUP_OK ? s : s2;
  })
}

soup_status soup_layer_fwd(soup_model* m, int layer, const void* x_in, void* x_out, int B, int S, void* stream) {
  if (!m || !x_in || !x_out || layer < 0 || layer >= m->cfg.n_layers || B < 1 || S < 1 ||
      static_cast<long long>(B) * S > m->cfg.max_tokens)
    return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD({
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long l0 = g_kernel_launches.load();
    const uint8_t* base;
    int buf;
    SOUP_TRY(streamer_acquire(m, layer, st, &base, &buf));
    soup_status s = layer_forward(m, layer, view_of(m, base), static_cast<const uint16_t*>(x_in),
                                  static_cast<uint16_t*>(x_out), B, S, st);
    soup_status s2 = streamer_release(m, buf, st);
    m->stats.kernel_launches += g_kernel_launches.load() - l0;
    return s != SOUP_OK ? s : s2;
  })
}

soup_status soup_layer_bwd(soup_model* m, int layer, const void* dy, void* dx, int B, int S, void* stream) {
  if (!m || !dy || !dx || layer < 0 || layer >= m->cfg.n_layers || B < 1 || S < 1) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD({
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!m->saved[layer].valid) {
      m->err = "layer_bwd before layer_fwd";
      return SOUP_ERR_STATE;
    }
    if (m->saved[layer].lora && !m->lora_g) return SOUP_ERR_STATE;
    const long long l0 = g_kernel_launches.load();
    const uint8_t* base;
    int buf;
    SOUP_TRY(streamer_acquire(m, layer, st, &base, &buf));
    soup_status s = layer_backward(m, layer, view_of(m, base), static_cast<const uint16_t*>(dy),
                                   static_cast<uint16_t*>(dx), B, S, st);
    soup_status s2 = streamer_release(m, buf, st);
    m->stats.kernel_launches += g_kernel_launches.load() - l0;
    return s != SOUP_OK ? s : s2;
  })
}

soup_status soup_step(soup_model* m, soup_loss loss, const soup_batch* batch, float* loss_out, void* stream) {
  if (!m || !batch || loss < SOUP_LOSS_SFT || loss > SOUP_LOSS_SIMPO) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD(return do_step(m, loss, batch, loss_out, static_cast<cudaStream_t>(stream));)
}

soup_status soup_optimizer_step(soup_model* m, float lr, void* stream) {
  if (!m) return SOUP_ERR_INVALID_ARG;
  if (!m->lora_p) return SOUP_ERR_STATE;
  SOUP_GUARD({
    m->adam_t += 1;
    const long long l0 = g_kernel_launches.load();
    soup_status s = check_launch(m, adamw_launch(m->lora_p, m->lora_g, m->lora_m, m->lora_v, m->lora_bf16,
                                                 static_cast<long long>(m->lora_n), lr, ADAM_B1, ADAM_B2, ADAM_EPS,
                                                 ADAM_WD, m->adam_t, static_cast<cudaStream_t>(stream)),
                                 "adamw");
    m->stats.kernel_launches += g_kernel_launches.load() - l0;
    return s;
  })
}

soup_status soup_last_logps(soup_model* m, float* pi, float* ref, int n) {
  if (!m || !pi || !ref || n < 1 || n > m->cfg.max_tokens) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD({
    SOUP_CK(cudaMemcpy(pi, m->pi, static_cast<size_t>(n) * 4, cudaMemcpyDeviceToHost));
    SOUP_CK(cudaMemcpy(ref, m->ref, static_cast<size_t>(n) * 4, cudaMemcpyDeviceToHost));
    return SOUP_OK;
  })
}

soup_status soup_nf4_quantize(const float* w, long long n, uint8_t* codes, int8_t* q8, float* scales, float* mean,
                              float* scratch, void* stream) {
  if (!w || n <= 0 || !codes || !q8 || !scales || !mean || !scratch) return SOUP_ERR_INVALID_ARG;
  cudaError_t e = nf4_quantize_launch(w, n, codes, q8, scales, mean, scratch, codebook(), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SOUP_OK : SOUP_ERR_CUDA;
}

soup_status soup_nf4_dequantize(const uint8_t* codes, const int8_t* q8, const float* scales, const float* mean,
                                long long n, uint16_t* out, void* stream) {
  if (!codes || !q8 || !scales || !mean || !out || n < 0) return SOUP_ERR_INVALID_ARG;
  cudaError_t e = nf4_dequant_launch(codes, q8, scales, mean, n, out, codebook(), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SOUP_OK : SOUP_ERR_CUDA;
}

soup_status soup_nf4_matmul(const void* x, int M, int N, int K, const uint8_t* codes, const int8_t* q8,
                            const float* scales, const float* mean, int transpose_w, const void* residual, void* y,
                            void* stream) {
  if (!x || !codes || !q8 || !scales || !mean || !y || M < 0 || N <= 0 || K <= 0) return SOUP_ERR_INVALID_ARG;
  if (N % 8 || K % 8) return SOUP_ERR_UNSUPPORTED;
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  NF4Group g{};
  g.nseg = 1;
  g.seg[0] = NF4Seg{codes, q8, scales, mean, 0, N};
  g.cols = K;
  g.total_rows = N;
  p.nf4 = g;
  std::memcpy(p.lut, codebook().v, sizeof(p.lut));
  p.alpha = 1.f;
  p.out = y;
  p.nseg = 1;
  if (!transpose_w) {  // y[M,N] = x[M,K] W^T
    p.M = M;
    p.N = N;
    p.ldo = N;
    p.seg[0].K = K;
    p.seg[0].A = Operand{OP_BF16_K, x, K, 1.f, 0, INT_MAX};
    p.seg[0].B = Operand{OP_NF4_K, nullptr, 0, 1.f, 0, INT_MAX};
    if (residual) {
      p.residual = residual;
      p.ldr = N;
    }
  } else {  // y[M,K] = x[M,N] W
    p.M = M;
    p.N = K;
    p.ldo = K;
    p.seg[0].K = N;
    p.seg[0].A = Operand{OP_BF16_K, x, N, 1.f, 0, INT_MAX};
    p.seg[0].B = Operand{OP_NF4_MN, nullptr, 0, 1.f, 0, INT_MAX};
    if (residual) {
      p.residual = residual;
      p.ldr = K;
    }
  }
  // the stream-K schedule needs a workspace and tile counters: one pair per device, made on
  // first use and shared by every call on that device
  static std::mutex ws_mu;
  static float* ws[64] = {};
  static int* cnt[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
    std::lock_guard<std::mutex> lk(ws_mu);
    if (!ws[dev]) {
      void* a = nullptr;
      void* b = nullptr;
      if (cudaMalloc(&a, static_cast<size_t>(64) << 20) == cudaSuccess &&
          cudaMalloc(&b, GEMM_COUNTERS * sizeof(int)) == cudaSuccess &&
          cudaMemset(b, 0, GEMM_COUNTERS * sizeof(int)) == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess) {
        ws[dev] = static_cast<float*>(a);
        cnt[dev] = static_cast<int*>(b);
      } else {
        if (a) cudaFree(a);
        if (b) cudaFree(b);
        cudaGetLastError();
      }
    }
    p.workspace = ws[dev];
    p.ws_bytes = ws[dev] ? static_cast<size_t>(64) << 20 : 0;
    p.tile_counters = cnt[dev];
    p.n_counters = cnt[dev] ? GEMM_COUNTERS : 0;
  }
  cudaError_t e = gemm_launch(p, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorInvalidValue) return SOUP_ERR_UNSUPPORTED;
  return e == cudaSuccess ? SOUP_OK : SOUP_ERR_CUDA;
}

}  // extern "C"

// The library's NF4 levels for other translation units.
const soup::LUT16& soup_codebook_lut() { return soup::codebook(); }

extern "C" {

soup_status soup_gemm_plan(int M, int N, int K, int nf4, int transposed, int sms, soup_gemm_plan_info* out) {
  if (!out || M <= 0 || N <= 0 || K <= 0 || N % 8 || K % 8 || sms < 1) return SOUP_ERR_INVALID_ARG;
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.nseg = 1;
  p.seg[0].K = K;
  p.seg[0].A = Operand{OP_BF16_K, nullptr, K, 1.f, 0, INT_MAX};
  p.seg[0].B = Operand{nf4 ? (transposed ? OP_NF4_MN : OP_NF4_K) : OP_BF16_K, nullptr, K, 1.f, 0, INT_MAX};
  // the workspace the model and soup_nf4_matmul hand to their GEMMs (only its presence and
  // size count here)
  static float ws_tag;
  static int cnt_tag;
  p.workspace = &ws_tag;
  p.ws_bytes = static_cast<size_t>(64) << 20;
  p.tile_counters = &cnt_tag;
  p.n_counters = GEMM_COUNTERS;
  const GemmPlan pl = gemm_plan(p, sms, true);
  out->mt = pl.mt;
  out->bn = pl.bn;
  out->splits = pl.splits;
  out->fused_reduce = pl.fused_reduce;
  out->stream_k_ctas = pl.sk_ctas;
  out->stream_k_tiles = pl.sk_tiles;
  out->stream_k_tiles_m = pl.sk_tiles_m;
  out->stream_k_kblocks = pl.sk_nkt;
  return SOUP_OK;
}

soup_status soup_gemm_stream_k_pieces(long long tiles, int nkt, int ctas, int cta, int max_pieces, int* tile,
                                      int* kb_lo, int* kb_hi, int* slot, int* n_pieces) {
  if (tiles < 1 || nkt < 1 || ctas < 1 || cta < 0 || cta >= ctas || max_pieces < 0 || !n_pieces ||
      (max_pieces > 0 && (!tile || !kb_lo || !kb_hi || !slot)))
    return SOUP_ERR_INVALID_ARG;
  const int n = sk_piece_count(tiles, nkt, ctas, cta);
  for (int pc = 0; pc < n && pc < max_pieces; ++pc) {
    sk_piece(tiles, nkt, ctas, cta, pc, &tile[pc], &kb_lo[pc], &kb_hi[pc]);
    slot[pc] = (kb_lo[pc] == 0 && kb_hi[pc] == nkt) ? -1 : sk_slot(cta, pc);
  }
  *n_pieces = n;
  return SOUP_OK;
}

soup_status soup_gemm_stream_k_shares(long long tiles, int nkt, int ctas, int tile, int max_shares, int* cta,
                                      int* slot, int* n_shares) {
  if (tiles < 1 || nkt < 1 || ctas < 1 || tile < 0 || tile >= tiles || max_shares < 0 || !n_shares ||
      (max_shares > 0 && (!cta || !slot)))
    return SOUP_ERR_INVALID_ARG;
  const long long x0 = static_cast<long long>(tile) * nkt;
  const int n = sk_owner(tiles, nkt, ctas, x0 + nkt - 1) - sk_owner(tiles, nkt, ctas, x0) + 1;
  for (int k = 0; k < n && k < max_shares; ++k) {
    sk_share(tiles, nkt, ctas, tile, k, &cta[k], &slot[k]);
    if (n == 1) slot[k] = -1;
  }
  *n_shares = n;
  return SOUP_OK;
}

soup_status soup_nf4_codebook(float* out16) {
  if (!out16) return SOUP_ERR_INVALID_ARG;
  std::memcpy(out16, codebook().v, 16 * sizeof(float));
  return SOUP_OK;
}

soup_status soup_get_stats(soup_model* m, soup_stats* out) {
  if (!m || !out) return SOUP_ERR_INVALID_ARG;
  *out = m->stats;
  out->stream_source = m->use_file ? SOUP_SOURCE_FILE : SOUP_SOURCE_RAM;
  if (m->use_file) {
    out->file_bytes_read = m->file.bytes_read() - m->file_bytes0;
    out->file_read_ms = m->file.read_ms() - m->file_ms0;
  }
  return SOUP_OK;
}

soup_status soup_reset_stats(soup_model* m) {
  if (!m) return SOUP_ERR_INVALID_ARG;
  const long long dev = m->stats.device_bytes, pin = m->stats.pinned_bytes;
  m->stats = soup_stats{};
  m->stats.device_bytes = dev;
  m->stats.pinned_bytes = pin;
  if (m->use_file) {
    m->file_bytes0 = m->file.bytes_read();
    m->file_ms0 = m->file.read_ms();
  }
  return SOUP_OK;
}

soup_status soup_set_profiling(soup_model* m, int enabled) {
  if (!m) return SOUP_ERR_INVALID_ARG;
  m->prof = enabled ? 1 : 0;
  return SOUP_OK;
}

soup_status soup_get_profile(soup_model* m, soup_profile_entry* out, int max_entries, int* n_entries, int reset) {
  if (!m || !n_entries || (max_entries > 0 && !out)) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD({
    prof_resolve(m);
    int n = 0;
    for (int c = 0; c < CAT_COUNT; ++c) {
      const auto& pc = m->prof_cats[c];
      if (pc.launches == 0) continue;
      if (n < max_entries) {
        soup_profile_entry& e = out[n];
        std::memset(&e, 0, sizeof(e));
        std::strncpy(e.name, kCatNames[c], sizeof(e.name) - 1);
        e.launches = pc.launches;
        e.total_ms = pc.ms;
        e.flops = pc.flops;
        e.bytes = pc.bytes;
      }
      ++n;
    }
    *n_entries = std::min(n, std::max(max_entries, 0));
    if (reset) m->prof_cats.assign(CAT_COUNT, soup_model::ProfCat{});
    return SOUP_OK;
  })
}

soup_status soup_set_timed_category(soup_model* m, const char* category) {
  if (!m) return SOUP_ERR_INVALID_ARG;
  static_assert(CAT_COUNT <= 31, "category mask");
  int mask = 0;
  const std::string spec = category ? category : "";
  size_t pos = 0;
  while (pos < spec.size()) {  // comma-separated names, or "all"
    const size_t end = std::min(spec.find(',', pos), spec.size());
    const std::string name = spec.substr(pos, end - pos);
    pos = end + 1;
    int c = -1;
    if (name == "all") mask |= ((1 << CAT_COUNT) - 1) & ~(1 << CAT_NULL);
    for (int k = 0; k < CAT_COUNT; ++k)
      if (k != CAT_NULL && name == kCatNames[k]) c = k;
    if (c >= 0) mask |= 1 << c;
    if (c < 0 && name != "all") {
      m->err = "unknown kernel category: " + name;
      return SOUP_ERR_INVALID_ARG;
    }
  }
  SOUP_GUARD({
    timed_harvest_all(m);
    m->tcat = mask;
    m->tname = mask ? spec : std::string();
    m->taccs.assign(CAT_COUNT, soup_model::ProfCat{});
    return SOUP_OK;
  })
}

soup_status soup_get_timed_category(soup_model* m, soup_profile_entry* out, int reset) {
  if (!m || !out) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD({
    timed_harvest_all(m);
    std::memset(out, 0, sizeof(*out));
    std::strncpy(out->name, m->tname.c_str(), sizeof(out->name) - 1);
    for (int k = 0; k < static_cast<int>(m->taccs.size()); ++k) {
      if (k == CAT_NULL) continue;
      const auto& c = m->taccs[k];
      out->launches += c.launches;
      out->total_ms += c.ms;
      out->flops += c.flops;
      out->bytes += c.bytes;
    }
    if (reset) m->taccs.assign(CAT_COUNT, soup_model::ProfCat{});
    return SOUP_OK;
  })
}

soup_status soup_get_timed_profile(soup_model* m, soup_profile_entry* out, int max_entries, int* n_entries,
                                   int reset) {
  if (!m || !n_entries || (max_entries > 0 && !out)) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD({
    timed_harvest_all(m);
    int n = 0;
    for (int c = 0; c < CAT_COUNT; ++c) {
      const auto& pc = m->taccs[c];
      if (pc.launches == 0) continue;
      if (n < max_entries) {
        soup_profile_entry& e = out[n];
        std::memset(&e, 0, sizeof(e));
        std::strncpy(e.name, kCatNames[c], sizeof(e.name) - 1);
        e.launches = pc.launches;
        e.total_ms = pc.ms;
        e.flops = pc.flops;
        e.bytes = pc.bytes;
      }
      ++n;
    }
    *n_entries = std::min(n, std::max(max_entries, 0));
    if (reset) m->taccs.assign(CAT_COUNT, soup_model::ProfCat{});
    return SOUP_OK;
  })
}

soup_status soup_h2d_probe(soup_model* m, int reps, double* gbs) {
  if (!m || !gbs || reps < 1) return SOUP_ERR_INVALID_ARG;
  if (!m->host_loaded[0]) return SOUP_ERR_STATE;
  SOUP_GUARD({
    const int b = 0;
    const uint8_t* src = m->use_file ? m->file.probe_buffer() : m->host_blob[0];
    SOUP_CK(cudaStreamWaitEvent(m->copy_stream, m->buf_free[b], 0));
    cudaEvent_t e0 = nullptr;
    cudaEvent_t e1 = nullptr;
    SOUP_CK(cudaEventCreate(&e0));
    SOUP_CK(cudaEventCreate(&e1));
    SOUP_CK(cudaMemcpyAsync(m->dev_buf[b], src, m->layout.total, cudaMemcpyHostToDevice, m->copy_stream));
    SOUP_CK(cudaEventRecord(e0, m->copy_stream));
    for (int i = 0; i < reps; ++i)
      SOUP_CK(cudaMemcpyAsync(m->dev_buf[b], src, m->layout.total, cudaMemcpyHostToDevice, m->copy_stream));
    SOUP_CK(cudaEventRecord(e1, m->copy_stream));
    SOUP_CK(cudaEventRecord(m->copy_done[b], m->copy_stream));
    soup_status st = wait_stream(m, m->copy_stream);
    float ms = 0.f;
    if (st == SOUP_OK) SOUP_CK(cudaEventElapsedTime(&ms, e0, e1));
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (st != SOUP_OK) return st;
    if (m->cfg.mode == SOUP_STREAMED) m->buf_layer[b] = -1;
    *gbs = static_cast<double>(reps) * m->layout.total / (ms * 1e-3) / 1e9;
    return SOUP_OK;
  })
}

soup_status soup_selftest_bounded_wait(soup_model* m, int limit_us, void* stream) {
  if (!m || limit_us < 1 || limit_us > 1000000) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD(return check_launch(m,
                                 bounded_wait_selftest_launch(m->scal + 1, 1000ull * static_cast<unsigned>(limit_us),
                                                              static_cast<cudaStream_t>(stream)),
                                 "bounded wait self-test");)
}

soup_status soup_check_device(soup_model* m, void* stream) {
  if (!m) return SOUP_ERR_INVALID_ARG;
  SOUP_GUARD(return read_scalars(m, static_cast<cudaStream_t>(stream), nullptr);)
}

}  // extern "C"
