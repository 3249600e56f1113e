// Host runtime behind the C ABI: model / KV cache / active set / sampler
// objects, workspace ownership, GEMM tile planning and launch sequencing.
//
// The step follows the A_t / L_t / C formulation of SureLock ("Stopping
// Computation for Converged Tokens in Masked Diffusion-LM Decoding"):
// computation runs on the active rows only, locked rows are served from the
// cache C, and the active list is compacted after every sure test
// (Paper-Notes, "Method: overall framework" and "Key design").
#include <limits.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <array>
#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"

// ------------------------------------------------------------------ errors --
static thread_local std::string g_last_error;

namespace sl {

sl_status fail(sl_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

sl_status cuda_fail(cudaError_t e, const char *what) {
  if (e == cudaErrorMemoryAllocation)
    return fail(SL_ERR_OOM, "%s: %s", what, cudaGetErrorString(e));
  return fail(SL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int *device_error_word() {
  static int *words[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!words[dev]) {
    int *p = nullptr;
    if (cudaMalloc(&p, sizeof(int)) != cudaSuccess) return nullptr;
    if (cudaMemset(p, 0, sizeof(int)) != cudaSuccess) return nullptr;
    words[dev] = p;
  }
  return words[dev];
}

static std::atomic<long long> g_launches{0};
void note_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
long long launches_total() { return g_launches.load(std::memory_order_relaxed); }

static int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

static size_t dsize(int dtype) { return dtype == SL_BF16 ? 2 : 4; }

}  // namespace sl

using namespace sl;

// ---------------------------------------------------------------- objects --
// Weight descriptors for the tensor-core path: one TMA map per box height
// (32, 64, 96, 128, 192, 256 rows: whole, half and pair-half tiles of every
// tile width) so any tiling can be launched.
constexpr int kBoxRows[6] = {32, 64, 96, 128, 192, 256};
struct WMaps {
  TmaMat m[6];
  const TmaMat *box(int rows) const {
    for (int i = 0; i < 5; ++i)
      if (kBoxRows[i] == rows) return &m[i];
    return &m[5];
  }
};

enum { W_Q = 0, W_K, W_V, W_O, W_G, W_U, W_D, W_COUNT };

struct TimingRec {
  int cls;
  double bytes, flops;
  cudaEvent_t e0, e1;
};

struct sl_model {
  sl_config cfg;
  const void *tok_emb, *final_norm, *lm_head;
  std::vector<sl_layer_weights> layers;
  std::vector<std::array<WMaps, W_COUNT>> maps;
  int attn_q = 0, attn_splits = 0, attn_bn = 0;   // pinned attention layout (0 = cost model)
  bool head_fusion = true;           // samplers take the sure-test statistics from the
                                     // LM head's epilogue (bf16 models)
  int ablation = 0;                  // SL_ABLATE_* bits (0: the method itself)
  WMaps head_map;
  int num_sms;
  int *err;
  bool timing = false;
  std::vector<cudaEvent_t> ev_free;
  std::vector<TimingRec> recs;
  sl_timing acc{};
  long long launch_base = 0;
  // autotuned GEMM tilings: [kind][row-count bucket] = {bn, splits, variant} (bn 0 = untuned)
  std::vector<std::array<int, 3>> tuned[5];
};

struct sl_kv_cache {
  const sl_model *m;
  int batch, n_ctx, max_rows;
  std::vector<void *> k, v;
  float2 *rope = nullptr;
  float *h = nullptr;      // [max_rows][d] fp32 residual stream
  void *a = nullptr;       // [max_rows][d] normed activations
  void *qkv = nullptr;     // [max_rows][3d]
  void *q = nullptr;       // [max_rows][d]
  void *o = nullptr;       // [max_rows][d]
  void *act = nullptr;     // [max_rows][f]
  float *ws = nullptr;     // [max_rows][max(3d, 2f)] fp32 split-K workspace, kept zero
  float *attn_ws = nullptr;
  int attn_max_splits = 16;
  unsigned int *attn_tickets = nullptr;   // [max_rows][H] per-row split tickets, kept zero
  std::vector<TmaMat> k_maps, v_maps;     // per layer, 128-row boxes (tensor-core attention)
  std::vector<TmaMat> k_maps64, v_maps64; // per layer, 64-row boxes (two query tiles per CTA)
  TmaMat map_q;                           // q workspace [M][d], 128-row boxes
  TmaMat map_qx{};                        // a caller's q (sl_attention), by pointer and M
  unsigned int *fix_ctr = nullptr;        // split-K fix-up tickets [max_rows/32 + 8][384]
  float4 *head_stat = nullptr;            // [max_rows][V / 64] LM-head tile records (bf16)
  int *head_stat_idx = nullptr;
  int32_t *key_stamp = nullptr;   // [max_rows] visible-key stamps (no-KV-cache ablation)
  int key_gen = 0;                // the current stamp generation
  TmaMat map_a, map_o, map_act;
  // epilogue destinations at the current M: residual h (fp32), split-K
  // workspace as [M][3d] and [M][2f] (fp32), gate/up product act (bf16)
  TmaMat out_h, out_ws3, out_ws2, out_act;
  TmaMat out_hx{};            // a caller's hidden states (sl_layer_forward), by pointer
  int map_rows = -1;
};

struct sl_active {
  int batch, n_ctx;
  int32_t *rows = nullptr, *seq_off = nullptr;
  int32_t *h_off = nullptr;          // pinned mirror of seq_off
  cudaEvent_t ev = nullptr;
  bool pending = false;
  float4 *part = nullptr;            // lock-stats partial records
  unsigned int *counters = nullptr;  // per row, zero between calls
  int max_splits = 64;
  int num_sms;
};

struct sl_sampler {
  sl_model *m;
  sl_sampler_params p;
  int batch, n_ctx;
  sl_kv_cache *cache = nullptr;
  sl_active *act = nullptr;
  int32_t *tokens = nullptr;
  uint8_t *masked = nullptr, *locked = nullptr, *lock = nullptr;
  int32_t *lock_t = nullptr, *argmax = nullptr, *d_prompts = nullptr;
  void *logits[2] = {nullptr, nullptr};
  float *lse[2] = {nullptr, nullptr};
  float *kl = nullptr, *unc = nullptr, *conf = nullptr;
  int t = 0;
  bool started = false;
  // K/V reuse for active rows (refresh interval kv_reuse, 1 = off): the rows a
  // step between refreshes computes, the mask flags at the start of the
  // previous step, a per-position lock byte array (zero between steps) and the
  // lock flags mapped onto the active list
  int kv_reuse = 1;
  sl_active *comp = nullptr;
  uint8_t *masked_before = nullptr, *lock_by_pos = nullptr, *lock_act = nullptr;
};

// ----------------------------------------------------------------- timing --
namespace {

struct Timed {
  sl_model *m;
  TimingRec rec;
  bool on;
  Timed(sl_model *m_, int cls, double bytes, double flops, cudaStream_t s) : m(m_), on(false) {
    if (!m || !m->timing) return;
    rec.cls = cls;
    rec.bytes = bytes;
    rec.flops = flops;
    for (int i = 0; i < 2; ++i) {
      cudaEvent_t e;
      if (!m->ev_free.empty()) {
        e = m->ev_free.back();
        m->ev_free.pop_back();
      } else if (cudaEventCreate(&e) != cudaSuccess) {
        return;
      }
      (i == 0 ? rec.e0 : rec.e1) = e;
    }
    cudaEventRecord(rec.e0, s);
    on = true;
    stream = s;
  }
  cudaStream_t stream = nullptr;
  ~Timed() {
    if (!on) return;
    cudaEventRecord(rec.e1, stream);
    m->recs.push_back(rec);
  }
};

}  // namespace

// ------------------------------------------------------------------ version --
extern "C" const char *sl_last_error(void) { return g_last_error.c_str(); }
extern "C" const char *sl_version(void) { return "surelock-b200 0.1 (sm_100a)"; }

// ------------------------------------------------------------------- model --
extern "C" sl_status sl_model_create(const sl_config *cfg, const sl_weights *w, sl_model **out) {
  if (!cfg || !w || !out) return fail(SL_ERR_INVALID, "sl_model_create: null argument");
  *out = nullptr;
  const sl_config &c = *cfg;
  if (c.n_layers <= 0 || c.d_model <= 0 || c.n_heads <= 0 || c.head_dim <= 0 || c.d_ffn <= 0 ||
      c.vocab <= 0)
    return fail(SL_ERR_INVALID, "sl_model_create: non-positive dimension");
  if (c.n_heads * c.head_dim != c.d_model)
    return fail(SL_ERR_INVALID, "sl_model_create: n_heads * head_dim != d_model");
  if (c.mask_id < 0 || c.mask_id >= c.vocab)
    return fail(SL_ERR_INVALID, "sl_model_create: mask_id out of range");
  if (c.head_dim % 2 != 0) return fail(SL_ERR_INVALID, "sl_model_create: odd head_dim");
  if (c.vocab % 8 != 0) return fail(SL_ERR_INVALID, "sl_model_create: vocab must be a multiple of 8");
  if (c.dtype == SL_BF16) {
    if (c.head_dim != 128)
      return fail(SL_ERR_UNSUPPORTED, "sl_model_create: bf16 path needs head_dim 128");
    if (c.d_model % 256 != 0 || c.d_ffn % 256 != 0 || c.vocab % 128 != 0)
      return fail(SL_ERR_UNSUPPORTED,
                  "sl_model_create: bf16 path needs d_model, d_ffn multiples of 256, vocab of 128");
  } else if (c.dtype == SL_F32) {
    if (c.head_dim != 8 && c.head_dim != 16 && c.head_dim != 32 && c.head_dim != 64)
      return fail(SL_ERR_UNSUPPORTED, "sl_model_create: fp32 path needs head_dim in {8,16,32,64}");
  } else {
    return fail(SL_ERR_INVALID, "sl_model_create: unknown dtype %d", c.dtype);
  }
  if (!w->tok_emb || !w->final_norm || !w->lm_head || !w->layers)
    return fail(SL_ERR_INVALID, "sl_model_create: null weight pointer");
  for (int l = 0; l < c.n_layers; ++l) {
    const sl_layer_weights &lw = w->layers[l];
    const void *ps[9] = {lw.attn_norm, lw.wq, lw.wk, lw.wv, lw.wo, lw.ffn_norm, lw.w_gate,
                         lw.w_up, lw.w_down};
    for (int i = 0; i < 9; ++i)
      if (!ps[i]) return fail(SL_ERR_INVALID, "sl_model_create: layer %d weight %d is null", l, i);
  }
  sl_model *m = new sl_model();
  m->cfg = c;
  m->tok_emb = w->tok_emb;
  m->final_norm = w->final_norm;
  m->lm_head = w->lm_head;
  m->layers.assign(w->layers, w->layers + c.n_layers);
  m->num_sms = sm_count();
  m->err = device_error_word();
  if (!m->err) {
    delete m;
    return fail(SL_ERR_CUDA, "sl_model_create: cannot allocate the device error word");
  }
  if (c.dtype == SL_BF16) {
    const int *boxes = kBoxRows;
    m->maps.resize(c.n_layers);
    for (int l = 0; l < c.n_layers; ++l) {
      const sl_layer_weights &lw = m->layers[l];
      const void *ptr[W_COUNT] = {lw.wq, lw.wk, lw.wv, lw.wo, lw.w_gate, lw.w_up, lw.w_down};
      const int rows[W_COUNT] = {c.d_model, c.d_model, c.d_model, c.d_model, c.d_ffn, c.d_ffn,
                                 c.d_model};
      const int cols[W_COUNT] = {c.d_model, c.d_model, c.d_model, c.d_model, c.d_model,
                                 c.d_model, c.d_ffn};
      for (int i = 0; i < W_COUNT; ++i)
        for (int b = 0; b < 6; ++b)
          if (!tma_encode(&m->maps[l][i].m[b], ptr[i], rows[i], cols[i], boxes[b])) {
            delete m;
            return fail(SL_ERR_INVALID,
                        "sl_model_create: TMA descriptor for layer %d weight %d failed "
                        "(pointer must be 16-byte aligned)", l, i);
          }
    }
    for (int b = 0; b < 6; ++b)
      if (!tma_encode(&m->head_map.m[b], m->lm_head, c.vocab, c.d_model, boxes[b])) {
        delete m;
        return fail(SL_ERR_INVALID, "sl_model_create: TMA descriptor for lm_head failed");
      }
  }
  *out = m;
  return SL_OK;
}

extern "C" void sl_model_destroy(sl_model *m) {
  if (!m) return;
  for (auto &r : m->recs) {
    cudaEventDestroy(r.e0);
    cudaEventDestroy(r.e1);
  }
  for (auto e : m->ev_free) cudaEventDestroy(e);
  delete m;
}

extern "C" sl_status sl_timing_enable(sl_model *m, int enable) {
  if (!m) return fail(SL_ERR_INVALID, "sl_timing_enable: null model");
  m->timing = enable != 0;
  return SL_OK;
}

// Fold completed timing records into the totals and recycle their events.
// With `wait`, block until every record has completed.
static sl_status timing_harvest(sl_model *m, bool wait) {
  size_t i = 0;
  for (; i < m->recs.size(); ++i) {
    TimingRec &r = m->recs[i];
    if (wait) {
      if (cudaEventSynchronize(r.e1) != cudaSuccess) return cuda_fail(cudaGetLastError(), "event sync");
    } else if (cudaEventQuery(r.e1) != cudaSuccess) {
      break;
    }
    float ms = 0.f;
    cudaEventElapsedTime(&ms, r.e0, r.e1);
    m->acc.ms[r.cls] += ms;
    m->acc.bytes[r.cls] += r.bytes;
    m->acc.flops[r.cls] += r.flops;
    m->acc.launches[r.cls] += 1;
    m->ev_free.push_back(r.e0);
    m->ev_free.push_back(r.e1);
  }
  m->recs.erase(m->recs.begin(), m->recs.begin() + i);
  cudaGetLastError();   // clear cudaErrorNotReady left by the query
  return SL_OK;
}

extern "C" sl_status sl_timing_read(sl_model *m, sl_timing *out, int reset) {
  if (!m || !out) return fail(SL_ERR_INVALID, "sl_timing_read: null argument");
  sl_status st = timing_harvest(m, true);
  if (st != SL_OK) return st;
  m->acc.kernels = launches_total() - m->launch_base;
  *out = m->acc;
  if (reset) {
    memset(&m->acc, 0, sizeof(m->acc));
    m->launch_base = launches_total();
  }
  return SL_OK;
}

extern "C" sl_status sl_device_check(int clear) {
  int *w = device_error_word();
  if (!w) return fail(SL_ERR_CUDA, "sl_device_check: no device error word");
  SL_CUDA(cudaDeviceSynchronize());
  int v = 0;
  SL_CUDA(cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost));
  if (v != 0) {
    if (clear) SL_CUDA(cudaMemset(w, 0, sizeof(int)));
    if (v >= 1 && v <= 3) return fail(SL_ERR_TIMEOUT, "a kernel gave up a bounded wait (code %d)", v);
    if (v == DEV_BAD_INDEX)
      return fail(SL_ERR_STATE, "a kernel met a token id outside [0, vocab) and skipped it");
    return fail(SL_ERR_CUDA, "a kernel reported device error %d", v);
  }
  return SL_OK;
}

// ---------------------------------------------------------------- KV cache --
extern "C" void sl_kv_cache_destroy(sl_kv_cache *c) {
  if (!c) return;
  for (void *p : c->k) cudaFree(p);
  for (void *p : c->v) cudaFree(p);
  void *ps[] = {c->rope,         c->h,         c->a,          c->qkv,
                c->q,            c->o,         c->act,        c->ws,
                c->attn_ws,      c->key_stamp, c->attn_tickets, c->head_stat,
                c->head_stat_idx, c->fix_ctr};
  for (void *p : ps)
    if (p) cudaFree(p);
  delete c;
}

// Split-K fix-up tickets: one per (32-row group, column tile) of the widest
// split projection at the narrowest tile (64 columns).
static size_t fix_ctr_bytes(int max_rows, const sl_config &cfg) {
  const size_t cols = std::max((size_t)3 * cfg.d_model, (size_t)2 * cfg.d_ffn);
  return ((size_t)max_rows / 32 + 8) * (cols / 64) * sizeof(unsigned int);
}

extern "C" sl_status sl_kv_cache_create(const sl_model *m, int batch, int n_ctx,
                                        sl_kv_cache **out) {
  if (!m || !out) return fail(SL_ERR_INVALID, "sl_kv_cache_create: null argument");
  *out = nullptr;
  if (batch <= 0 || batch > SL_MAX_BATCH || n_ctx <= 0)
    return fail(SL_ERR_INVALID, "sl_kv_cache_create: batch in [1, %d] and n_ctx > 0 required",
                SL_MAX_BATCH);
  const sl_config &cfg = m->cfg;
  const size_t es = dsize(cfg.dtype);
  const int d = cfg.d_model, f = cfg.d_ffn;
  sl_kv_cache *c = new sl_kv_cache();
  c->m = m;
  c->batch = batch;
  c->n_ctx = n_ctx;
  c->max_rows = batch * n_ctx;
  const size_t rows = (size_t)c->max_rows;
  const size_t layer_bytes = rows * d * es;
  auto alloc = [&](void **p, size_t bytes) -> bool {
    if (cudaMalloc(p, bytes) != cudaSuccess) return false;
    return cudaMemset(*p, 0, bytes) == cudaSuccess;
  };
  bool ok = true;
  c->k.assign(cfg.n_layers, nullptr);
  c->v.assign(cfg.n_layers, nullptr);
  for (int l = 0; l < cfg.n_layers && ok; ++l)
    ok = alloc(&c->k[l], layer_bytes) && alloc(&c->v[l], layer_bytes);
  const size_t wsc = std::max((size_t)3 * d, (size_t)2 * f);
  ok = ok && alloc((void **)&c->h, rows * d * 4) && alloc(&c->a, rows * d * es) &&
       alloc(&c->qkv, rows * 3 * d * es) && alloc(&c->q, rows * d * es) &&
       alloc(&c->o, rows * d * es) && alloc(&c->act, rows * f * es) &&
       alloc((void **)&c->ws, rows * wsc * 4) && alloc((void **)&c->key_stamp, rows * 4);
  if (ok && cfg.dtype == SL_BF16) {
    ok = alloc((void **)&c->attn_ws, attn_bf16_workspace_bytes(c->max_rows, cfg.n_heads,
                                                               c->attn_max_splits)) &&
         alloc((void **)&c->attn_tickets, attn_tc_tickets_bytes(c->max_rows, cfg.n_heads)) &&
         alloc((void **)&c->head_stat, rows * (cfg.vocab / 64) * sizeof(float4)) &&
         alloc((void **)&c->head_stat_idx, rows * (cfg.vocab / 64) * sizeof(int)) &&
         alloc((void **)&c->fix_ctr, fix_ctr_bytes(c->max_rows, cfg));
    c->k_maps.resize(cfg.n_layers);
    c->v_maps.resize(cfg.n_layers);
    c->k_maps64.resize(cfg.n_layers);
    c->v_maps64.resize(cfg.n_layers);
    for (int l = 0; l < cfg.n_layers && ok; ++l)
      ok = tma_encode(&c->k_maps[l], c->k[l], c->max_rows, d, 128) &&
           tma_encode(&c->v_maps[l], c->v[l], c->max_rows, d, 128) &&
           tma_encode(&c->k_maps64[l], c->k[l], c->max_rows, d, 64) &&
           tma_encode(&c->v_maps64[l], c->v[l], c->max_rows, d, 64);
  }
  if (ok) {
    // rotary table in double precision: angle = pos * theta^(-2i/dh)
    const int half = cfg.head_dim / 2;
    std::vector<float2> tab((size_t)n_ctx * half);
    for (int pos = 0; pos < n_ctx; ++pos)
      for (int i = 0; i < half; ++i) {
        double inv = pow((double)cfg.rope_theta, -2.0 * i / cfg.head_dim);
        double ang = (double)pos * inv;
        tab[(size_t)pos * half + i] = make_float2((float)cos(ang), (float)sin(ang));
      }
    ok = alloc((void **)&c->rope, tab.size() * sizeof(float2)) &&
         cudaMemcpy(c->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) ==
             cudaSuccess;
  }
  if (!ok) {
    sl_kv_cache_destroy(c);
    return fail(SL_ERR_OOM, "sl_kv_cache_create: device allocation failed");
  }
  *out = c;
  return SL_OK;
}

extern "C" sl_status sl_kv_cache_reset(sl_kv_cache *c, void *stream) {
  if (!c) return fail(SL_ERR_INVALID, "sl_kv_cache_reset: null cache");
  const size_t bytes = (size_t)c->max_rows * c->m->cfg.d_model * dsize(c->m->cfg.dtype);
  for (size_t l = 0; l < c->k.size(); ++l) {
    SL_CUDA(cudaMemsetAsync(c->k[l], 0, bytes, (cudaStream_t)stream));
    SL_CUDA(cudaMemsetAsync(c->v[l], 0, bytes, (cudaStream_t)stream));
  }
  return SL_OK;
}

extern "C" sl_status sl_kv_cache_view(const sl_kv_cache *c, int layer, void **k, void **v) {
  if (!c || !k || !v) return fail(SL_ERR_INVALID, "sl_kv_cache_view: null argument");
  if (layer < 0 || layer >= (int)c->k.size())
    return fail(SL_ERR_INVALID, "sl_kv_cache_view: layer %d out of range", layer);
  *k = c->k[layer];
  *v = c->v[layer];
  return SL_OK;
}

// -------------------------------------------------------------- active set --
extern "C" void sl_active_destroy(sl_active *a) {
  if (!a) return;
  if (a->rows) cudaFree(a->rows);
  if (a->seq_off) cudaFree(a->seq_off);
  if (a->part) cudaFree(a->part);
  if (a->counters) cudaFree(a->counters);
  if (a->h_off) cudaFreeHost(a->h_off);
  if (a->ev) cudaEventDestroy(a->ev);
  delete a;
}

extern "C" sl_status sl_active_create(int batch, int n_ctx, sl_active **out) {
  if (!out) return fail(SL_ERR_INVALID, "sl_active_create: null out");
  *out = nullptr;
  if (batch <= 0 || batch > SL_MAX_BATCH || n_ctx <= 0)
    return fail(SL_ERR_INVALID, "sl_active_create: batch in [1, %d] and n_ctx > 0 required",
                SL_MAX_BATCH);
  sl_active *a = new sl_active();
  a->batch = batch;
  a->n_ctx = n_ctx;
  a->num_sms = sm_count();
  const size_t rows = (size_t)batch * n_ctx;
  bool ok = cudaMalloc(&a->rows, rows * 4) == cudaSuccess &&
            cudaMalloc(&a->seq_off, (batch + 1) * 4) == cudaSuccess &&
            cudaMalloc(&a->part, rows * a->max_splits * 2 * sizeof(float4)) == cudaSuccess &&
            cudaMalloc(&a->counters, rows * sizeof(unsigned)) == cudaSuccess &&
            cudaMemset(a->counters, 0, rows * sizeof(unsigned)) == cudaSuccess &&
            cudaMallocHost(&a->h_off, (batch + 1) * 4) == cudaSuccess &&
            cudaEventCreateWithFlags(&a->ev, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    sl_active_destroy(a);
    return fail(SL_ERR_OOM, "sl_active_create: allocation failed");
  }
  for (int b = 0; b <= batch; ++b) a->h_off[b] = b * n_ctx;
  *out = a;
  return SL_OK;
}

static sl_status active_mirror(sl_active *a, cudaStream_t s) {
  SL_CUDA(cudaMemcpyAsync(a->h_off, a->seq_off, (a->batch + 1) * 4, cudaMemcpyDeviceToHost, s));
  SL_CUDA(cudaEventRecord(a->ev, s));
  a->pending = true;
  return SL_OK;
}

extern "C" sl_status sl_active_reset(sl_active *a, void *stream) {
  if (!a) return fail(SL_ERR_INVALID, "sl_active_reset: null");
  SL_CUDA(launch_active_fill(a->rows, a->seq_off, a->batch, a->n_ctx, (cudaStream_t)stream));
  return active_mirror(a, (cudaStream_t)stream);
}

extern "C" sl_status sl_active_load(sl_active *a, const int32_t *h_counts, const int32_t *h_pos,
                                    void *stream) {
  if (!a || !h_counts || (!h_pos)) return fail(SL_ERR_INVALID, "sl_active_load: null argument");
  std::vector<int32_t> rows, off(a->batch + 1, 0);
  int k = 0;
  for (int b = 0; b < a->batch; ++b) {
    if (h_counts[b] < 0 || h_counts[b] > a->n_ctx)
      return fail(SL_ERR_INVALID, "sl_active_load: count %d of sequence %d out of range",
                  h_counts[b], b);
    off[b] = (int)rows.size();
    int prev = -1;
    for (int i = 0; i < h_counts[b]; ++i, ++k) {
      int p = h_pos[k];
      if (p <= prev || p >= a->n_ctx)
        return fail(SL_ERR_INVALID, "sl_active_load: positions of sequence %d not strictly "
                                    "ascending in [0, n_ctx)", b);
      prev = p;
      rows.push_back(b * a->n_ctx + p);
    }
  }
  off[a->batch] = (int)rows.size();
  cudaStream_t s = (cudaStream_t)stream;
  // synchronous copies from pageable memory: the host vectors die on return
  SL_CUDA(cudaStreamSynchronize(s));
  if (!rows.empty()) SL_CUDA(cudaMemcpy(a->rows, rows.data(), rows.size() * 4, cudaMemcpyHostToDevice));
  SL_CUDA(cudaMemcpy(a->seq_off, off.data(), off.size() * 4, cudaMemcpyHostToDevice));
  return active_mirror(a, s);
}

extern "C" sl_status sl_active_counts(sl_active *a, int32_t *h_counts) {
  if (!a || !h_counts) return fail(SL_ERR_INVALID, "sl_active_counts: null argument");
  if (a->pending) {
    SL_CUDA(cudaEventSynchronize(a->ev));
    a->pending = false;
  }
  for (int b = 0; b < a->batch; ++b) h_counts[b] = a->h_off[b + 1] - a->h_off[b];
  return SL_OK;
}

extern "C" sl_status sl_active_view(const sl_active *a, int32_t **d_rows, int32_t **d_seq_off) {
  if (!a || !d_rows || !d_seq_off) return fail(SL_ERR_INVALID, "sl_active_view: null argument");
  *d_rows = a->rows;
  *d_seq_off = a->seq_off;
  return SL_OK;
}

// --------------------------------------------------------- GEMM planning ---
namespace {

struct Plan {
  int bn, splits, msub;
  double cost;
  int pair = 0;     // 1: CTA-pair kernel (2-SM MMA)
  int swap = 0;     // 1: swapped operands (weights as the 128-row MMA operand, M <= 256)
};

// Kernel variant codes (sl_gemm_bf16, tuning tables): 0 = 1-SM 128-row units,
// 1 = 1-SM 256-row units, 2 = CTA pair, 3 = swapped operands (bn 128, at most
// 256 rows, fp32 reduce epilogues).
static int plan_variant(const Plan &p) {
  return p.swap ? 3 : p.pair ? 2 : (p.msub == 2 ? 1 : 0);
}
static void plan_set_variant(Plan &p, int v) {
  p.msub = v >= 1 ? 2 : 1;
  p.pair = v == 2 ? 1 : 0;
  p.swap = v == 3 ? 1 : 0;
}

// Choose the tile shape (BN, 128 or 256 rows per unit) and K split of one
// GEMM by a small cost model: the kernel time is the largest of the weight
// stream from HBM (read once), the operand traffic from L2 into the SMs (every
// unit re-reads its A and B tiles), and the tensor-core time of the padded
// tiles, stretched by wave quantisation over the SMs, plus a fixed cost per
// wave and, for split-K, the fp32 partial-sum traffic (atomics, and for
// SPLIT_ACCUM the finalize pass).
enum SplitKind { SPLIT_NONE = 0, SPLIT_RESID = 1, SPLIT_ACCUM = 2 };

// heads: the unsplit QKV epilogue rotates whole 128-column heads, so unsplit
// plans keep bn a multiple of 128.  seg: the weight is several matrices of
// `seg` rows stacked (Q|K|V); a tile takes its rows from one of them, so bn
// must divide seg.
Plan plan_gemm(int M, int N, int K, int split_kind, int num_sms, bool swiglu, int min_bn = 64,
               bool heads = false, int seg = 0) {
  const double bw_hbm = 6.5e12, bw_l2 = 9.0e12, peak = 1.6e15;
  const int kblocks = K / 64;
  Plan best{0, 1, 1, 1e30};
  for (int msub = 1; msub <= 2; ++msub) {
    if (msub == 2 && M <= 128) continue;
    const int rows_unit = 128 * msub;
    const int mt = (M + rows_unit - 1) / rows_unit;
    const double rows_live = std::min(M, rows_unit);
    const int bns[4] = {256, 192, 128, 64};
    for (int bi = 0; bi < 4; ++bi) {
      const int bn = bns[bi];
      if (N % bn || bn < min_bn || (seg && seg % bn)) continue;
      if (swiglu && (N / 2) % (bn / 2)) continue;
      const bool single_acc = 2 * msub * bn > 512;
      const double mma_eff = bn >= 192 ? 1.0 : (bn == 128 ? 0.8 : 0.5);
      const int max_s = split_kind != SPLIT_NONE ? std::min(32, std::max(1, kblocks / 4)) : 1;
      for (int sp = 1; sp <= max_s; ++sp) {
        const int kbp = (kblocks + sp - 1) / sp;
        const int ss = (kblocks + kbp - 1) / kbp;
        const long units = (long)mt * (N / bn) * ss;
        const long waves = (units + num_sms - 1) / num_sms;
        const double quant = (double)(waves * num_sms) / units;
        const double t_hbm = 2.0 * ((double)N * K + (double)M * K) / bw_hbm;
        const double t_l2 = (double)units * kbp * (bn * 128.0 + rows_live * 128.0) / bw_l2;
        const double t_mma = (double)units * kbp * 2.0 * rows_unit * bn * 64 / (peak * mma_eff);
        double t = std::max(t_hbm, std::max(t_l2, t_mma)) * std::min(quant, 2.0) + waves * 1.0e-6;
        if (single_acc && waves > 1) t += waves * 2.0e-6;     // epilogue not overlapped
        if (heads && bn % 128 != 0 && ss == 1) continue;
        if (ss > 1) {
          t += (double)M * N * 4.0 * ss / bw_l2;                               // fp32 atomics
          if (split_kind == SPLIT_ACCUM) t += (double)M * N * 8.0 / bw_hbm + 3.0e-6;   // finalize
        }
        if (t < best.cost - 1e-9) best = Plan{bn, ss, msub, t};
      }
    }
  }
  // CTA pairs: 256 x BN tiles on two SMs, each SM staging 128 rows of A and
  // BN/2 rows of B per K-block
  if (M > 128) {
    const int pairs = num_sms / 2;
    const int mt = (M + 255) / 256;
    const double rows_live = std::min(M, 256);
    for (int bn : {256, 192, 128}) {
      if (N % bn || bn < min_bn || (seg && seg % bn)) continue;
      if (swiglu && (N / 2) % (bn / 2)) continue;
      const int max_s = split_kind != SPLIT_NONE ? std::min(32, std::max(1, kblocks / 4)) : 1;
      for (int sp = 1; sp <= max_s; ++sp) {
        const int kbp = (kblocks + sp - 1) / sp;
        const int ss = (kblocks + kbp - 1) / kbp;
        const long units = (long)mt * (N / bn) * ss;
        const long waves = (units + pairs - 1) / pairs;
        const double quant = (double)(waves * pairs) / units;
        const double t_hbm = 2.0 * ((double)N * K + (double)M * K) / bw_hbm;
        const double t_l2 = (double)units * kbp * (bn * 128.0 + rows_live * 128.0) / bw_l2;
        const double t_mma = (double)units * kbp * 2.0 * 256 * bn * 64 / peak;
        double t = std::max(t_hbm, std::max(t_l2, t_mma)) * std::min(quant, 2.0) + waves * 1.0e-6;
        if (heads && bn % 128 != 0 && ss == 1) continue;
        if (ss > 1) {
          t += (double)M * N * 4.0 * ss / bw_l2;
          if (split_kind == SPLIT_ACCUM) t += (double)M * N * 8.0 / bw_hbm + 3.0e-6;
        }
        if (t < best.cost - 1e-9) {
          best = Plan{bn, ss, 2, t};
          best.pair = 1;
        }
      }
    }
  }
  // stream-K (splits = -1): every worker (SM, or CTA pair) runs an equal share
  // of the tiles x K-blocks; each flushes about (tiles + workers) / workers
  // partial tiles with fp32 atomics
  if (split_kind != SPLIT_NONE) {
    for (int variant = 0; variant <= 2; ++variant) {
      if (variant > 0 && M <= 128) continue;
      const int rows_unit = variant == 0 ? 128 : 256;
      const int workers = variant == 2 ? num_sms / 2 : num_sms;
      const double rate = variant == 2 ? 2.0 * peak / num_sms : peak / num_sms;
      const int mt = (M + rows_unit - 1) / rows_unit;
      const double rows_live = std::min(M, rows_unit);
      for (int bn : {256, 192, 128}) {
        if (N % bn || bn < min_bn || (seg && seg % bn)) continue;
        if (swiglu && (N / 2) % (bn / 2)) continue;
        if (variant == 1 && 4 * bn > 512) continue;      // keep double-buffered accumulators
        const long tiles = (long)mt * (N / bn);
        const long iters = tiles * kblocks;
        const double per_worker = std::ceil((double)iters / workers);
        const double t_hbm = 2.0 * ((double)N * K + (double)M * K) / bw_hbm;
        const double t_l2 = (double)iters * (bn * 128.0 + rows_live * 128.0) / bw_l2;
        const double t_mma = per_worker * 2.0 * rows_unit * bn * 64 / rate;
        double t = std::max(t_hbm, std::max(t_l2, t_mma)) + 1.0e-6;
        t += (double)M * N * 4.0 * (1.0 + (double)workers / tiles) / bw_l2;
        if (split_kind == SPLIT_ACCUM) t += (double)M * N * 8.0 / bw_hbm + 3.0e-6;
        if (t < best.cost - 1e-9) {
          best = Plan{bn, -1, variant == 0 ? 1 : 2, t};
          best.pair = variant == 2 ? 1 : 0;
        }
      }
    }
  }
  return best;
}

}  // namespace

// ------------------------------------------------------------------- step --
// Algorithmic bytes of a GEMM: weights + activations in + results out, bf16
// (fp32 for fp32 models), each counted once.
static double gemm_bytes(double M, double N, double K, double es) {
  return es * (N * K + M * K + M * N);
}

// The keys this step's queries may attend to.  The method: every cached key
// (stamp null).  The no-KV-cache ablation: the active rows' own keys, marked
// with a fresh stamp generation once per call (the stamps start at zero, so
// generation 1 onwards never matches a row that was not stamped).
struct KeySet {
  const int32_t *stamp = nullptr;
  int gen = 0;
};

static sl_status visible_keys(const sl_model *m, sl_kv_cache *c, const sl_active *a, int M,
                              cudaStream_t s, KeySet *ks) {
  *ks = KeySet{};
  if (!(m->ablation & SL_ABLATE_NO_KV_CACHE)) return SL_OK;
  if (c->key_gen == INT_MAX) {
    SL_CUDA(cudaMemsetAsync(c->key_stamp, 0, (size_t)c->max_rows * 4, s));
    c->key_gen = 0;
  }
  ++c->key_gen;
  SL_CUDA(launch_key_stamp(a->rows, M, c->key_gen, c->key_stamp, s));
  ks->stamp = c->key_stamp;
  ks->gen = c->key_gen;
  return SL_OK;
}

static sl_status layer_f32(sl_model *m, sl_kv_cache *c, sl_active *a, int l, float *h, int M,
                           const KeySet &ks, cudaStream_t s) {
  const sl_config &cfg = m->cfg;
  const int d = cfg.d_model, f = cfg.d_ffn;
  float *an = (float *)c->a, *qkv = (float *)c->qkv, *q = (float *)c->q;
  float *o = (float *)c->o, *ws = c->ws, *act = (float *)c->act;
  const sl_layer_weights &lw = m->layers[l];
  SL_CUDA(launch_rmsnorm(SL_F32, h, lw.attn_norm, d, cfg.rms_eps, M, an, s));
  {
    Timed t(m, SL_K_GEMM, gemm_bytes(M, 3.0 * d, d, 4), 6.0 * M * d * d, s);
    SL_CUDA(launch_gemm_f32(EPI_STORE, an, M, d, (const float *)lw.wq, d, qkv, 3 * d, 0, nullptr, s));
    SL_CUDA(launch_gemm_f32(EPI_STORE, an, M, d, (const float *)lw.wk, d, qkv, 3 * d, d, nullptr, s));
    SL_CUDA(launch_gemm_f32(EPI_STORE, an, M, d, (const float *)lw.wv, d, qkv, 3 * d, 2 * d, nullptr, s));
  }
  SL_CUDA(launch_rope_scatter(SL_F32, qkv, true, false, M, a->rows, c->n_ctx, cfg.n_heads,
                              cfg.head_dim, c->rope, q, c->k[l], c->v[l], s));
  {
    Timed t(m, SL_K_ATTN, 4.0 * (2.0 * M * d + 2.0 * c->batch * c->n_ctx * d),
            4.0 * M * c->n_ctx * d, s);
    SL_CUDA(launch_attn_f32(q, (const float *)c->k[l], (const float *)c->v[l], a->rows, M,
                            c->n_ctx, cfg.n_heads, cfg.head_dim, o, s, ks.stamp, ks.gen));
  }
  {
    Timed t(m, SL_K_GEMM, gemm_bytes(M, d, d, 4), 2.0 * M * d * d, s);
    SL_CUDA(launch_gemm_f32(EPI_RESID, o, M, d, (const float *)lw.wo, d, h, d, 0, nullptr, s));
  }
  SL_CUDA(launch_rmsnorm(SL_F32, h, lw.ffn_norm, d, cfg.rms_eps, M, an, s));
  {
    Timed t(m, SL_K_GEMM, gemm_bytes(M, 2.0 * f, d, 4), 4.0 * M * d * f, s);
    SL_CUDA(launch_gemm_f32(EPI_STORE, an, M, d, (const float *)lw.w_gate, f, ws, 2 * f, 0, nullptr, s));
    SL_CUDA(launch_gemm_f32(EPI_STORE, an, M, d, (const float *)lw.w_up, f, ws, 2 * f, f, nullptr, s));
  }
  SL_CUDA(launch_swiglu(SL_F32, ws, true, false, M, f, act, s));
  {
    Timed t(m, SL_K_GEMM, gemm_bytes(M, d, f, 4), 2.0 * M * d * f, s);
    SL_CUDA(launch_gemm_f32(EPI_RESID, act, M, f, (const float *)lw.w_down, d, h, d, 0, nullptr, s));
  }
  return SL_OK;
}

// Failure-detection test hooks (sl_debug_*): the wait limit of later GEMM
// launches, and a one-shot lost operand copy in the next one.
static std::atomic<unsigned long long> g_wait_limit_ns{0};
static std::atomic<int> g_lost_load{0};

// Split-K tile fix-up in the GEMM epilogue instead of a finalize kernel
// (SL_GEMM_FIXUP=0 turns it off; read once).
static bool gemm_fixup_enabled() {
  static int v = -1;
  if (v < 0) {
    const char *e = getenv("SL_GEMM_FIXUP");
    v = (e && atoi(e) == 0) ? 0 : 1;
  }
  return v == 1;
}

static cudaError_t launch_gemm_hooked(TcGemmArgs g, int num_sms, int *err, cudaStream_t s) {
  g.wait_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  g.lost_load = g_lost_load.exchange(0, std::memory_order_relaxed);
  return launch_gemm_tc(g, num_sms, err, s);
}

static sl_status tc_gemm(sl_model *m, const TcGemmArgs &g, cudaStream_t s) {
  cudaError_t e = launch_gemm_hooked(g, m->num_sms, m->err, s);
  if (e != cudaSuccess) return cuda_fail(e, "tcgen05 GEMM launch");
  return SL_OK;
}

extern "C" sl_status sl_debug_set_wait_limit(unsigned long long ns) {
  if (ns != 0 && (ns < 1000000ull || ns > WAIT_LIMIT_NS))
    return fail(SL_ERR_INVALID, "sl_debug_set_wait_limit: %llu ns outside [1 ms, %llu ns]", ns,
                WAIT_LIMIT_NS);
  g_wait_limit_ns.store(ns, std::memory_order_relaxed);
  return SL_OK;
}

extern "C" sl_status sl_debug_inject_lost_load(void) {
  g_lost_load.store(1, std::memory_order_relaxed);
  return SL_OK;
}

struct BfPlans {
  Plan qkv, o, gu, dn, hd;
};

enum GemmKind { G_QKV = 0, G_O = 1, G_GU = 2, G_DN = 3, G_HD = 4, G_KINDS = 5 };

// Row-count buckets of the GEMM autotuner: a step with M active rows uses the
// tiling tuned at the smallest bound >= M.
static const int kTuneBounds[] = {16,   32,   64,   96,   128,  160,  192,  224,  256,
                                  320,  384,  512,  768,  1024, 1536, 2048, 3072, 4096,
                                  6144, 8192, 12288, 16384, 24576, 32768, 65536, 131072};
static const int kTuneCount = sizeof(kTuneBounds) / sizeof(kTuneBounds[0]);
static int tune_bucket(int M) {
  for (int i = 0; i < kTuneCount; ++i)
    if (M <= kTuneBounds[i]) return i;
  return -1;
}

static Plan plan_kind(const sl_model *m, int kind, int M, int ns) {
  const int bkt = tune_bucket(M);
  if (bkt >= 0 && bkt < (int)m->tuned[kind].size() && m->tuned[kind][bkt][0] > 0) {
    const auto &t = m->tuned[kind][bkt];
    Plan pl{t[0], t[1], 1, 0.0};
    plan_set_variant(pl, t[2]);
    return pl;
  }
  const sl_config &cfg = m->cfg;
  const int d = cfg.d_model, f = cfg.d_ffn;
  switch (kind) {
    case G_QKV: return plan_gemm(M, 3 * d, d, SPLIT_ACCUM, ns, false, 128, true, d);
    case G_O: return plan_gemm(M, d, d, SPLIT_RESID, ns, false);
    case G_GU: return plan_gemm(M, 2 * f, d, SPLIT_ACCUM, ns, true);
    case G_DN: return plan_gemm(M, d, f, SPLIT_RESID, ns, false);
    default: return plan_gemm(M, cfg.vocab, d, SPLIT_NONE, ns, false);
  }
}

static BfPlans plans_for(const sl_model *m, int M, int ns) {
  BfPlans p;
  p.qkv = plan_kind(m, G_QKV, M, ns);
  p.o = plan_kind(m, G_O, M, ns);
  p.gu = plan_kind(m, G_GU, M, ns);
  p.dn = plan_kind(m, G_DN, M, ns);
  p.hd = plan_kind(m, G_HD, M, ns);
  return p;
}

static sl_status ensure_maps(sl_kv_cache *c, int M) {
  if (c->map_rows == M) return SL_OK;
  const sl_config &cfg = c->m->cfg;
  const int d = cfg.d_model, f = cfg.d_ffn;
  if (!tma_encode(&c->map_a, c->a, M, d, 128) || !tma_encode(&c->map_o, c->o, M, d, 128) ||
      !tma_encode(&c->map_q, c->q, M, d, 128) ||
      !tma_encode(&c->map_act, c->act, M, f, 128) ||
      !tma_encode_out(&c->out_h, c->h, M, d, d, true) ||
      !tma_encode_out(&c->out_ws3, c->ws, M, 3 * d, 3 * d, true) ||
      !tma_encode_out(&c->out_ws2, c->ws, M, 2 * f, 2 * f, true) ||
      !tma_encode_out(&c->out_act, c->act, M, f, f, false))
    return fail(SL_ERR_CUDA, "activation TMA descriptor encoding failed");
  c->map_rows = M;
  return SL_OK;
}

static void fill_seqs(AttnSeqs &seqs, const sl_active *a, const int32_t *counts) {
  seqs.batch = a->batch;
  int off = 0;
  for (int b = 0; b < a->batch; ++b) {
    seqs.seq_start[b] = off;
    seqs.seq_count[b] = counts[b];
    off += counts[b];
  }
}

// q_map: a TMA map over q with 128-row boxes (the tensor-core kernel reads q by
// TMA).  queries_per_cta 128 (or 0, the default) selects the tensor-core
// kernel; 16, 32 or 64 the mma.sync kernel with that layout.
static sl_status attn_bf16(sl_model *m, sl_kv_cache *c, const AttnSeqs &seqs, int l, int M,
                           const void *q, const TmaMat &q_map, void *o, const KeySet &ks,
                           cudaStream_t s) {
  const int d = m->cfg.d_model;
  Timed t(m, SL_K_ATTN, 2.0 * (2.0 * M * d + 2.0 * seqs.batch * c->n_ctx * d),
          4.0 * (double)M * c->n_ctx * d, s);
  // the output projection's weights follow; the attention leaves HBM idle
  if (m->attn_q == 0 || m->attn_q >= 128) {
    SL_CUDA(launch_attn_tc(q_map, c->k_maps[l], c->v_maps[l], c->k_maps64[l], c->v_maps64[l],
                           seqs, M, c->n_ctx, m->cfg.n_heads, o, c->attn_ws, c->attn_tickets,
                           c->attn_max_splits, m->num_sms, m->err,
                           g_wait_limit_ns.load(std::memory_order_relaxed), s, m->attn_q,
                           m->attn_splits, m->attn_bn, m->layers[l].wo, (size_t)d * d * 2,
                           ks.stamp, ks.gen));
    return SL_OK;
  }
  SL_CUDA(launch_attn_bf16(q, c->k[l], c->v[l], seqs, M, c->n_ctx, m->cfg.n_heads, o,
                           c->attn_ws, c->attn_max_splits, m->num_sms, s, m->attn_q,
                           m->attn_splits, m->layers[l].wo, (size_t)d * d * 2, ks.stamp,
                           ks.gen));
  return SL_OK;
}

// The sure test's statistics requested from the LM head's epilogue
// (sl_step_stats): previous logits and lse (null when there is no previous
// posterior) and the per-row outputs.
struct HeadStats {
  const void *prev = nullptr;
  const float *lse_prev = nullptr;
  float *lse_cur = nullptr, *kl = nullptr, *unc = nullptr, *conf = nullptr;
  int32_t *argmax = nullptr;
};

// One of the step's projection GEMMs on the current activation descriptors,
// with the split-K finalize pass when the plan splits K:
//   G_QKV  a (normed h) x [Wq|Wk|Wv]^T -> RoPE(q) -> q, RoPE(k), v -> C.k/C.v[rows]
//   G_O    o x Wo^T, added to the residual h
//   G_GU   b x [Wg|Wu]^T -> silu(gate) * up -> act
//   G_DN   act x Wd^T, added to the residual h
//   G_HD   RMSNorm(h) x W_out^T -> logits[rows]
static sl_status run_gemm(sl_model *m, sl_kv_cache *c, const int32_t *rows, int l, int kind,
                          const Plan &pl, int M, float *h, void *logits, cudaStream_t s,
                          const HeadStats *hs = nullptr) {
  const sl_config &cfg = m->cfg;
  const int d = cfg.d_model, f = cfg.d_ffn, V = cfg.vocab, H = cfg.n_heads;
  const double Md = (double)M;
  // split K, stream-K or swapped operands: fp32 partial sums (the swapped
  // kernel always leaves its tiles by reduce-add)
  const bool split = pl.splits != 1 || pl.swap;
  if (pl.swap && (kind == G_HD || M > 256 || pl.bn != 128))
    return fail(SL_ERR_INVALID, "swapped-operand GEMM: projections of at most 256 rows, bn 128");
  TcGemmArgs g{};
  g.M = M;
  g.bn = pl.bn;
  g.splits = pl.splits;
  g.msub = pl.msub;
  g.pair = pl.pair;
  g.swap = pl.swap;
  const int bbox = pl.pair ? pl.bn / 2 : pl.bn;    // weight rows per TMA box
  double bytes = 0, flops = 0;
  switch (kind) {
    case G_QKV: {
      // a tile's weight rows come from one of Wq, Wk, Wv
      if (d % pl.bn) return fail(SL_ERR_INVALID, "QKV tile width %d does not divide d_model", pl.bn);
      const auto &mp = m->maps[l];
      g.A = &c->map_a;
      g.B[0] = mp[W_Q].box(bbox);
      g.B[1] = mp[W_K].box(bbox);
      g.B[2] = mp[W_V].box(bbox);
      g.n_seg[0] = g.n_seg[1] = g.n_seg[2] = d;
      g.N = 3 * d;
      g.K = d;
      if (split) {
        // K split across CTAs: fp32 partial sums, then RoPE + scatter from them,
        // by the tile fix-up in the GEMM's epilogue when tiles hold whole heads
        g.epi = EPI_ACCUM;
        g.out = c->ws;
        g.ldo = 3 * d;
        g.OUT = &c->out_ws3;
        if (gemm_fixup_enabled() && pl.bn % 128 == 0 && !pl.swap) {
          g.fix_ctr = c->fix_ctr;
          g.row_map = rows;
          g.rope = c->rope;
          g.n_ctx = c->n_ctx;
          g.q_out = c->q;
          g.ck = c->k[l];
          g.cv = c->v[l];
        }
      } else {
        g.epi = EPI_QKV;
        g.row_map = rows;
        g.rope = c->rope;
        g.n_ctx = c->n_ctx;
        g.q_out = c->q;
        g.ck = c->k[l];
        g.cv = c->v[l];
      }
      bytes = gemm_bytes(Md, 3.0 * d, d, 2);
      flops = 6.0 * Md * d * d;
      break;
    }
    case G_O:
    case G_DN: {
      const auto &mp = m->maps[l];
      const int K = kind == G_O ? d : f;
      g.A = kind == G_O ? &c->map_o : &c->map_act;
      g.B[0] = mp[kind == G_O ? W_O : W_D].box(bbox);
      g.n_seg[0] = d;
      g.N = d;
      g.K = K;
      g.epi = EPI_RESID;
      g.out = h;
      g.ldo = d;
      if (h == c->h) {
        g.OUT = &c->out_h;
      } else {   // a caller's hidden states (sl_layer_forward)
        if (c->out_hx.ptr != h || c->out_hx.rows != M) {
          if (!tma_encode_out(&c->out_hx, h, M, d, d, true))
            return fail(SL_ERR_INVALID, "hidden-state TMA descriptor encoding failed");
        }
        g.OUT = &c->out_hx;
      }
      bytes = gemm_bytes(Md, d, K, 2);
      flops = 2.0 * Md * d * K;
      break;
    }
    case G_GU: {
      const auto &mp = m->maps[l];
      g.A = &c->map_a;
      g.B[0] = mp[W_G].box(pl.bn / 2);
      g.B[1] = mp[W_U].box(pl.bn / 2);
      g.b_swiglu = 1;
      g.N = 2 * f;
      g.K = d;
      g.epi = split ? EPI_ACCUM : EPI_SWIGLU;
      g.out = split ? (void *)c->ws : c->act;
      g.ldo = split ? 2 * f : f;
      g.OUT = split ? &c->out_ws2 : &c->out_act;
      if (split && gemm_fixup_enabled() && !pl.swap) {
        g.fix_ctr = c->fix_ctr;
        g.fix_act = c->act;
      }
      bytes = gemm_bytes(Md, 2.0 * f, d, 2) - 2.0 * Md * f;
      flops = 4.0 * Md * d * f;
      break;
    }
    default: {   // G_HD
      g.A = &c->map_a;
      g.B[0] = m->head_map.box(bbox);
      g.n_seg[0] = V;
      g.N = V;
      g.K = d;
      g.splits = 1;
      g.epi = EPI_STORE;
      g.out = logits;
      g.ldo = V;
      g.row_map = rows;
      bytes = gemm_bytes(Md, V, d, 2);
      flops = 2.0 * Md * d * V;
      if (hs) {
        g.epi = EPI_HEAD;
        g.prev = hs->prev;
        g.stat = c->head_stat;
        g.stat_idx = c->head_stat_idx;
        g.mask_id = cfg.mask_id;
        if (hs->prev) bytes += 2.0 * Md * V;       // the previous logits, read once
      }
      break;
    }
  }
  {
    Timed t(m, SL_K_GEMM, bytes, flops, s);
    sl_status st = tc_gemm(m, g, s);
    if (st != SL_OK) return st;
  }
  if (split && kind == G_QKV && !g.fix_ctr)
    SL_CUDA(launch_rope_scatter(SL_BF16, c->ws, true, true, M, rows, c->n_ctx, H, cfg.head_dim,
                                c->rope, c->q, c->k[l], c->v[l], s));
  if (split && kind == G_GU && !g.fix_ctr)
    SL_CUDA(launch_swiglu(SL_BF16, c->ws, true, true, M, f, c->act, s));
  return SL_OK;
}

static sl_status layer_bf16(sl_model *m, sl_kv_cache *c, sl_active *a, int l, float *h, int M,
                            const AttnSeqs &seqs, const BfPlans &pl, const KeySet &ks,
                            cudaStream_t s) {
  const sl_config &cfg = m->cfg;
  const int d = cfg.d_model;
  const sl_layer_weights &lw = m->layers[l];
  sl_status st;
  SL_CUDA(launch_rmsnorm(SL_BF16, h, lw.attn_norm, d, cfg.rms_eps, M, c->a, s));
  if ((st = run_gemm(m, c, a->rows, l, G_QKV, pl.qkv, M, h, nullptr, s)) != SL_OK) return st;
  if ((st = attn_bf16(m, c, seqs, l, M, c->q, c->map_q, c->o, ks, s)) != SL_OK) return st;
  if ((st = run_gemm(m, c, a->rows, l, G_O, pl.o, M, h, nullptr, s)) != SL_OK) return st;
  SL_CUDA(launch_rmsnorm(SL_BF16, h, lw.ffn_norm, d, cfg.rms_eps, M, c->a, s));
  if ((st = run_gemm(m, c, a->rows, l, G_GU, pl.gu, M, h, nullptr, s)) != SL_OK) return st;
  return run_gemm(m, c, a->rows, l, G_DN, pl.dn, M, h, nullptr, s);
}

static sl_status check_pair(sl_model *m, sl_kv_cache *c, sl_active *a, const char *who) {
  if (!m || !c || !a) return fail(SL_ERR_INVALID, "%s: null argument", who);
  if (c->m != m) return fail(SL_ERR_INVALID, "%s: cache belongs to another model", who);
  if (c->batch != a->batch || c->n_ctx != a->n_ctx)
    return fail(SL_ERR_INVALID, "%s: cache (%d x %d) and active set (%d x %d) differ", who,
                c->batch, c->n_ctx, a->batch, a->n_ctx);
  return SL_OK;
}

static sl_status kl_stats_unfused(sl_model *timing_model, sl_active *a, int M, int vocab,
                                  int mask_id, int dtype, const void *cur, const HeadStats &hs,
                                  cudaStream_t s);

static sl_status step_impl(sl_model *m, sl_kv_cache *c, sl_active *a, const int32_t *d_tokens,
                           void *d_logits, const HeadStats *hs, void *stream) {
  sl_status st = check_pair(m, c, a, "sl_step");
  if (st != SL_OK) return st;
  if (!d_tokens || !d_logits) return fail(SL_ERR_INVALID, "sl_step: null argument");
  if (m->cfg.dtype == SL_BF16 && ((uintptr_t)d_logits & 15))
    return fail(SL_ERR_INVALID, "sl_step: logits must be 16-byte aligned");
  if (hs && (!hs->lse_cur || !hs->kl || !hs->unc || !hs->conf || !hs->argmax ||
             (hs->prev && !hs->lse_prev)))
    return fail(SL_ERR_INVALID, "sl_step_stats: null statistics argument");
  if (hs && m->cfg.dtype == SL_BF16 && hs->prev && ((uintptr_t)hs->prev & 15))
    return fail(SL_ERR_INVALID, "sl_step_stats: previous logits must be 16-byte aligned");
  int32_t counts[SL_MAX_BATCH];
  if ((st = sl_active_counts(a, counts)) != SL_OK) return st;
  int M = 0;
  for (int b = 0; b < a->batch; ++b) M += counts[b];
  if (M == 0) return SL_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const sl_config &cfg = m->cfg;
  const int d = cfg.d_model, V = cfg.vocab;
  KeySet ks;
  if ((st = visible_keys(m, c, a, M, s, &ks)) != SL_OK) return st;
  SL_CUDA(launch_gather_embed(cfg.dtype, d_tokens, a->rows, M, m->tok_emb, d, V, c->h, m->err,
                              s));
  if (cfg.dtype == SL_F32) {
    for (int l = 0; l < cfg.n_layers; ++l)
      if ((st = layer_f32(m, c, a, l, c->h, M, ks, s)) != SL_OK) return st;
    SL_CUDA(launch_rmsnorm(SL_F32, c->h, m->final_norm, d, cfg.rms_eps, M, c->a, s));
    {
      Timed t(m, SL_K_GEMM, gemm_bytes(M, V, d, 4), 2.0 * M * d * V, s);
      SL_CUDA(launch_gemm_f32(EPI_STORE, (const float *)c->a, M, d, (const float *)m->lm_head,
                              V, (float *)d_logits, V, 0, a->rows, s));
    }
    // the fp32 path has no tensor-core epilogue: a separate pass over the logits
    if (hs) return kl_stats_unfused(m, a, M, V, cfg.mask_id, SL_F32, d_logits, *hs, s);
    return SL_OK;
  }
  if ((st = ensure_maps(c, M)) != SL_OK) return st;
  AttnSeqs seqs;
  fill_seqs(seqs, a, counts);
  const BfPlans pl = plans_for(m, M, m->num_sms);
  for (int l = 0; l < cfg.n_layers; ++l)
    if ((st = layer_bf16(m, c, a, l, c->h, M, seqs, pl, ks, s)) != SL_OK) return st;
  SL_CUDA(launch_rmsnorm(SL_BF16, c->h, m->final_norm, d, cfg.rms_eps, M, c->a, s));
  if ((st = run_gemm(m, c, a->rows, 0, G_HD, pl.hd, M, c->h, d_logits, s, hs)) != SL_OK)
    return st;
  if (hs) {
    Timed t(m, SL_K_LOCK, (double)M * (V / pl.hd.bn) * 20.0 + 24.0 * M, 0.0, s);
    SL_CUDA(launch_head_stats_merge(c->head_stat, c->head_stat_idx, V / pl.hd.bn, a->rows, M,
                                    hs->prev ? 1 : 0, hs->lse_prev, hs->lse_cur, hs->kl, hs->unc,
                                    hs->conf, hs->argmax, s));
  }
  // the previous step's timing events completed before this step was planned
  if (m->timing) timing_harvest(m, false);
  return SL_OK;
}

extern "C" sl_status sl_step(sl_model *m, sl_kv_cache *c, sl_active *a, const int32_t *d_tokens,
                             void *d_logits, void *stream) {
  return step_impl(m, c, a, d_tokens, d_logits, nullptr, stream);
}

extern "C" sl_status sl_step_stats(sl_model *m, sl_kv_cache *c, sl_active *a,
                                   const int32_t *d_tokens, void *d_logits,
                                   const void *d_logits_prev, const float *d_lse_prev,
                                   int has_prev, float *d_lse_cur, float *d_kl, float *d_unc,
                                   float *d_conf, int32_t *d_argmax, void *stream) {
  HeadStats hs;
  hs.prev = has_prev ? d_logits_prev : nullptr;
  hs.lse_prev = has_prev ? d_lse_prev : nullptr;
  if (has_prev && (!d_logits_prev || !d_lse_prev))
    return fail(SL_ERR_INVALID, "sl_step_stats: has_prev needs previous logits and lse");
  hs.lse_cur = d_lse_cur;
  hs.kl = d_kl;
  hs.unc = d_unc;
  hs.conf = d_conf;
  hs.argmax = d_argmax;
  return step_impl(m, c, a, d_tokens, d_logits, &hs, stream);
}

extern "C" sl_status sl_layer_forward(sl_model *m, sl_kv_cache *c, sl_active *a, int layer,
                                      float *d_h, void *stream) {
  sl_status st = check_pair(m, c, a, "sl_layer_forward");
  if (st != SL_OK) return st;
  if (!d_h) return fail(SL_ERR_INVALID, "sl_layer_forward: null hidden states");
  if (layer < 0 || layer >= m->cfg.n_layers)
    return fail(SL_ERR_INVALID, "sl_layer_forward: layer %d out of range", layer);
  if ((uintptr_t)d_h & 15) return fail(SL_ERR_INVALID, "sl_layer_forward: d_h must be 16-byte aligned");
  int32_t counts[SL_MAX_BATCH];
  if ((st = sl_active_counts(a, counts)) != SL_OK) return st;
  int M = 0;
  for (int b = 0; b < a->batch; ++b) M += counts[b];
  if (M == 0) return SL_OK;
  cudaStream_t s = (cudaStream_t)stream;
  KeySet ks;
  if ((st = visible_keys(m, c, a, M, s, &ks)) != SL_OK) return st;
  if (m->cfg.dtype == SL_F32) return layer_f32(m, c, a, layer, d_h, M, ks, s);
  if ((st = ensure_maps(c, M)) != SL_OK) return st;
  AttnSeqs seqs;
  fill_seqs(seqs, a, counts);
  return layer_bf16(m, c, a, layer, d_h, M, seqs, plans_for(m, M, m->num_sms), ks, s);
}

extern "C" sl_status sl_attention(sl_model *m, sl_kv_cache *c, sl_active *a, int layer,
                                  const void *d_q, void *d_o, void *stream) {
  sl_status st = check_pair(m, c, a, "sl_attention");
  if (st != SL_OK) return st;
  if (!d_q || !d_o) return fail(SL_ERR_INVALID, "sl_attention: null argument");
  if (layer < 0 || layer >= m->cfg.n_layers)
    return fail(SL_ERR_INVALID, "sl_attention: layer %d out of range", layer);
  int32_t counts[SL_MAX_BATCH];
  if ((st = sl_active_counts(a, counts)) != SL_OK) return st;
  int M = 0;
  for (int b = 0; b < a->batch; ++b) M += counts[b];
  if (M == 0) return SL_OK;
  cudaStream_t s = (cudaStream_t)stream;
  KeySet ks;
  if ((st = visible_keys(m, c, a, M, s, &ks)) != SL_OK) return st;
  if (m->cfg.dtype == SL_F32) {
    Timed t(m, SL_K_ATTN, 4.0 * (2.0 * M * m->cfg.d_model + 2.0 * c->batch * c->n_ctx * m->cfg.d_model),
            4.0 * M * c->n_ctx * m->cfg.d_model, s);
    SL_CUDA(launch_attn_f32((const float *)d_q, (const float *)c->k[layer],
                            (const float *)c->v[layer], a->rows, M, c->n_ctx, m->cfg.n_heads,
                            m->cfg.head_dim, (float *)d_o, s, ks.stamp, ks.gen));
    return SL_OK;
  }
  if (((uintptr_t)d_q & 15) || ((uintptr_t)d_o & 15))
    return fail(SL_ERR_INVALID, "sl_attention: q and o must be 16-byte aligned");
  if (c->map_qx.ptr != d_q || c->map_qx.rows != M) {
    if (!tma_encode(&c->map_qx, d_q, M, m->cfg.d_model, 128))
      return fail(SL_ERR_INVALID, "sl_attention: q TMA descriptor encoding failed");
  }
  AttnSeqs seqs;
  fill_seqs(seqs, a, counts);
  return attn_bf16(m, c, seqs, layer, M, d_q, c->map_qx, d_o, ks, s);
}

extern "C" sl_status sl_gemm_bf16(int epi, const void *d_a, int M, int K, const void *d_b,
                                  const void *d_b2, int N, void *d_out, int ldo,
                                  const int32_t *d_row_map, int bn, int splits, int variant,
                                  void *stream) {
  if (!d_a || !d_b || !d_out) return fail(SL_ERR_INVALID, "sl_gemm_bf16: null argument");
  if (epi < SL_GEMM_STORE || epi > SL_GEMM_ACCUM) return fail(SL_ERR_INVALID, "sl_gemm_bf16: bad epi");
  if (M < 0 || K <= 0 || N <= 0 || K % 64 != 0)
    return fail(SL_ERR_INVALID, "sl_gemm_bf16: need M >= 0, K > 0 with K %% 64 == 0, N > 0");
  const bool swiglu = epi == SL_GEMM_SWIGLU || (epi == SL_GEMM_ACCUM && d_b2);
  if (epi == SL_GEMM_SWIGLU && !d_b2) return fail(SL_ERR_INVALID, "sl_gemm_bf16: SWIGLU needs d_b2");
  if (swiglu && N % 2) return fail(SL_ERR_INVALID, "sl_gemm_bf16: gate/up needs even N");
  if (((uintptr_t)d_a | (uintptr_t)d_b | (uintptr_t)(d_b2 ? d_b2 : d_b) | (uintptr_t)d_out) & 15)
    return fail(SL_ERR_INVALID, "sl_gemm_bf16: pointers must be 16-byte aligned");
  {
    // output rows: fp32 (RESID/ACCUM) or bf16 (STORE/SWIGLU), 16-byte row pitch
    const bool f32_out = epi == SL_GEMM_RESID || epi == SL_GEMM_ACCUM;
    const int out_cols = epi == SL_GEMM_SWIGLU ? N / 2 : N;
    if (ldo < out_cols || ldo % (f32_out ? 4 : 8) != 0)
      return fail(SL_ERR_INVALID, "sl_gemm_bf16: ldo must cover the output columns and give "
                                  "16-byte aligned rows");
  }
  if (M == 0) return SL_OK;
  const int ns = sm_count();
  if (variant < 0 || variant > 3)
    return fail(SL_ERR_INVALID, "sl_gemm_bf16: variant must be 0, 1, 2 or 3");
  int msub = variant >= 1 ? 2 : 1;
  int pair = variant == 2 ? 1 : 0;
  const int swap = variant == 3 ? 1 : 0;
  if (swap && (M > 256 || bn != 128 || splits < 1 ||
               (epi != SL_GEMM_RESID && epi != SL_GEMM_ACCUM)))
    return fail(SL_ERR_INVALID, "sl_gemm_bf16: the swapped-operand kernel takes M <= 256, bn 128, "
                                "splits >= 1 and the RESID or ACCUM epilogue");
  if (bn == 0) {
    Plan p = plan_gemm(M, N, K, epi == SL_GEMM_RESID ? SPLIT_RESID
                                : epi == SL_GEMM_ACCUM ? SPLIT_ACCUM : SPLIT_NONE, ns, swiglu);
    bn = p.bn;
    msub = p.msub;
    pair = p.pair;
    if (splits == 0) splits = p.splits;
  }
  if (pair && bn < 128)
    return fail(SL_ERR_INVALID, "sl_gemm_bf16: the CTA-pair kernel needs bn 128, 192 or 256");
  if (bn != 64 && bn != 128 && bn != 192 && bn != 256)
    return fail(SL_ERR_INVALID, "sl_gemm_bf16: bn must be 64/128/192/256");
  if (N % bn || (swiglu && (N / 2) % (bn / 2)))
    return fail(SL_ERR_INVALID, "sl_gemm_bf16: N must be a multiple of bn");
  if (splits < 1 && splits != -1) splits = 1;
  if (splits == -1 && epi != SL_GEMM_RESID && epi != SL_GEMM_ACCUM)
    return fail(SL_ERR_INVALID, "sl_gemm_bf16: stream-K (splits -1) needs RESID or ACCUM");
  const int epi_k = epi == SL_GEMM_STORE ? EPI_STORE : epi == SL_GEMM_RESID ? EPI_RESID
                    : epi == SL_GEMM_SWIGLU ? EPI_SWIGLU : EPI_ACCUM;
  const int brows = (swiglu || pair) ? bn / 2 : bn;
  TmaMat ma, mb, mb2;
  if (!tma_encode(&ma, d_a, M, K, 128) || !tma_encode(&mb, d_b, swiglu ? N / 2 : N, K, brows) ||
      (swiglu && !tma_encode(&mb2, d_b2, N / 2, K, brows)))
    return fail(SL_ERR_INVALID, "sl_gemm_bf16: TMA descriptor encoding failed");
  TcGemmArgs g{};
  g.epi = epi_k;
  g.A = &ma;
  g.B[0] = &mb;
  g.B[1] = swiglu ? &mb2 : nullptr;
  g.b_swiglu = swiglu ? 1 : 0;
  g.n_seg[0] = swiglu ? 0 : N;
  g.M = M;
  g.N = N;
  g.K = K;
  g.bn = bn;
  g.splits = splits;
  g.out = d_out;
  g.ldo = ldo;
  g.row_map = d_row_map;
  g.msub = msub;
  g.pair = pair;
  g.swap = swap;
  // TMA epilogue when the output rows qualify (16-byte row pitch)
  TmaMat mo;
  if (epi == SL_GEMM_RESID || epi == SL_GEMM_ACCUM) {
    if (!tma_encode_out(&mo, d_out, M, N, ldo, true))
      return fail(SL_ERR_INVALID, "sl_gemm_bf16: output TMA descriptor encoding failed");
    g.OUT = &mo;
  } else if (epi == SL_GEMM_SWIGLU && (bn / 2) % 64 == 0) {
    if (tma_encode_out(&mo, d_out, M, N / 2, ldo, false)) g.OUT = &mo;
  }
  int *err = device_error_word();
  if (!err) return fail(SL_ERR_CUDA, "sl_gemm_bf16: no device error word");
  cudaError_t e = launch_gemm_hooked(g, ns, err, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sl_gemm_bf16 launch");
  return SL_OK;
}

// --------------------------------------------------------------- autotune --
// Time every valid tiling of the five projection GEMMs at each row-count bucket
// up to max_rows on this device, keep the fastest.  Uses layer 0's weights
// and the cache's workspaces (their contents are overwritten).
extern "C" sl_status sl_model_autotune(sl_model *m, sl_kv_cache *c, int max_rows, void *stream) {
  if (!m || !c) return fail(SL_ERR_INVALID, "sl_model_autotune: null argument");
  if (c->m != m) return fail(SL_ERR_INVALID, "sl_model_autotune: cache belongs to another model");
  if (m->cfg.dtype != SL_BF16) return SL_OK;            // the fp32 path has one tiling
  if (max_rows <= 0) return fail(SL_ERR_INVALID, "sl_model_autotune: max_rows must be positive");
  max_rows = std::min(max_rows, c->max_rows);
  cudaStream_t s = (cudaStream_t)stream;
  const sl_config &cfg = m->cfg;
  const int d = cfg.d_model, f = cfg.d_ffn, V = cfg.vocab;
  const int head_rows = std::min(max_rows, 8192);
  int32_t *rows = nullptr;
  void *logits = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  std::vector<int32_t> h_rows(max_rows);
  for (int i = 0; i < max_rows; ++i) h_rows[i] = i;
  sl_status st = SL_OK;
  const bool was_timing = m->timing;
  m->timing = false;
  auto cleanup = [&]() {
    if (rows) cudaFree(rows);
    if (logits) cudaFree(logits);
    if (e0) cudaEventDestroy(e0);
    if (e1) cudaEventDestroy(e1);
    m->timing = was_timing;
    c->map_rows = -1;
  };
  if (cudaMalloc(&rows, max_rows * sizeof(int32_t)) != cudaSuccess ||
      cudaMalloc(&logits, (size_t)head_rows * V * 2) != cudaSuccess ||
      cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) {
    cleanup();
    return fail(SL_ERR_OOM, "sl_model_autotune: scratch allocation failed");
  }
  if (cudaMemcpy(rows, h_rows.data(), max_rows * sizeof(int32_t), cudaMemcpyHostToDevice) !=
      cudaSuccess) {
    cleanup();
    return fail(SL_ERR_CUDA, "sl_model_autotune: copy failed");
  }
  for (int k = 0; k < G_KINDS; ++k) m->tuned[k].assign(kTuneCount, {0, 1, 1});
  const int Ns[G_KINDS] = {3 * d, d, 2 * f, d, V};
  const int Ks[G_KINDS] = {d, d, d, f, d};
  const int split_opts[] = {1, 2, 3, 4, 6, 8, 9, 12, 16, -1};   // -1: stream-K
  // one candidate's time at M rows: three blocks of three back-to-back
  // repetitions, the median block (a stray slow block does not decide); each
  // repetition is followed by a small kernel (an RMSNorm, as in the layer) so
  // that successive GEMMs cannot overlap each other through programmatic launch
  // and flatter tilings with few CTAs
  auto time_plan = [&](int kind, const Plan &pl, int M, float *ms_out) -> sl_status {
    auto launch = [&]() {
      sl_status r = run_gemm(m, c, rows, 0, kind, pl, M, c->h, logits, s);
      if (r != SL_OK) return r;
      cudaError_t e = launch_rmsnorm(SL_BF16, c->h, m->final_norm, d, cfg.rms_eps, M, c->a, s);
      return e == cudaSuccess ? SL_OK : cuda_fail(e, "sl_model_autotune: spacer");
    };
    sl_status r = launch();
    if (r != SL_OK) return r;
    float blocks[3] = {0.f, 0.f, 0.f};
    for (int blk = 0; blk < 3; ++blk) {
      cudaEventRecord(e0, s);
      for (int it = 0; it < 3; ++it)
        if ((r = launch()) != SL_OK) return r;
      cudaEventRecord(e1, s);
      if (cudaEventSynchronize(e1) != cudaSuccess)
        return cuda_fail(cudaGetLastError(), "sl_model_autotune: timing");
      cudaEventElapsedTime(&blocks[blk], e0, e1);
    }
    std::sort(blocks, blocks + 3);
    *ms_out = blocks[1];
    return SL_OK;
  };
  for (int b = 0; b < kTuneCount && st == SL_OK; ++b) {
    if (b > 0 && kTuneBounds[b - 1] >= max_rows) break;
    const int Mb = std::min(kTuneBounds[b], max_rows);
    // a bucket's tiling serves every row count in it: from 1024 rows up (where
    // a 256-row tile more or less is a large share of the work) it is timed at
    // both ends of the bucket and the tiling with the least summed slowdown
    // against each end's fastest is kept; below, at the bucket's upper end
    std::vector<int> pts = {Mb};
    if (b > 0 && Mb >= 1024 && kTuneBounds[b - 1] + 1 < Mb) pts.push_back(kTuneBounds[b - 1] + 1);
    // candidates of every GEMM kind, filtered at the upper end
    std::vector<std::array<int, 3>> cands[G_KINDS];
    for (int kind = 0; kind < G_KINDS; ++kind) {
      if (kind == G_HD && Mb > head_rows) continue;
      const int N = Ns[kind], K = Ks[kind], kblocks = K / 64;
      for (int variant = 0; variant <= 2; ++variant) {
        const int msub = variant >= 1 ? 2 : 1;
        if (variant >= 1 && Mb <= 128) continue;
        for (int bn : {256, 192, 128, 64}) {
          if (N % bn || (kind == G_QKV && (bn < 128 || d % bn))) continue;
          if (variant == 2 && bn < 128) continue;
          if (kind == G_GU && (N / 2) % (bn / 2)) continue;
          int last_ss = 0;
          for (int sp : split_opts) {
            if (kind == G_HD && sp != 1) break;
            if (kind == G_QKV && sp == 1 && bn % 128 != 0) continue;   // whole heads unsplit
            int ss = -1;
            if (sp > 0) {
              if (sp > std::max(1, kblocks / 2)) continue;
              const int kbp = (kblocks + sp - 1) / sp;
              ss = (kblocks + kbp - 1) / kbp;
              if (ss == last_ss) continue;
              last_ss = ss;
              const long units = (long)((Mb + 128 * msub - 1) / (128 * msub)) * (N / bn) * ss;
              if (units > 24L * m->num_sms) continue;
            }
            cands[kind].push_back({bn, ss, variant});
          }
        }
      }
      // swapped operands for buckets of at most 256 rows, for the projections
      // that add into the residual stream (output, down): Q|K|V and gate/up
      // would need their finishing pass as a kernel of its own, whose launch
      // boundary costs more in the decode than the swap saves (sl_gemm_bf16
      // and sl_model_set_tuning still take them)
      if ((kind == G_O || kind == G_DN) && Mb <= 256 && N % 128 == 0) {
        int last_ss = 0;
        for (int sp : split_opts) {
          if (sp < 1 || sp > std::max(1, kblocks / 2)) continue;
          const int kbp = (kblocks + sp - 1) / sp;
          const int ss = (kblocks + kbp - 1) / kbp;
          if (ss == last_ss) continue;
          last_ss = ss;
          if ((long)(N / 128) * ss > 24L * m->num_sms) continue;
          cands[kind].push_back({128, ss, 3});
        }
      }
    }
    std::vector<std::vector<float>> times[G_KINDS];
    for (int kind = 0; kind < G_KINDS; ++kind)
      times[kind].assign(cands[kind].size(), std::vector<float>(pts.size(), 0.f));
    for (size_t pi = 0; pi < pts.size() && st == SL_OK; ++pi) {
      if ((st = ensure_maps(c, pts[pi])) != SL_OK) break;
      for (int kind = 0; kind < G_KINDS && st == SL_OK; ++kind)
        for (size_t ci = 0; ci < cands[kind].size() && st == SL_OK; ++ci) {
          Plan pl{cands[kind][ci][0], cands[kind][ci][1], 1, 0.0};
          plan_set_variant(pl, cands[kind][ci][2]);
          st = time_plan(kind, pl, pts[pi], &times[kind][ci][pi]);
        }
    }
    if (st != SL_OK) break;
    for (int kind = 0; kind < G_KINDS; ++kind) {
      if (cands[kind].empty()) continue;
      std::vector<float> fastest(pts.size(), 1e30f);
      for (const auto &tc : times[kind])
        for (size_t pi = 0; pi < pts.size(); ++pi) fastest[pi] = std::min(fastest[pi], tc[pi]);
      double best_score = 1e30;
      std::array<int, 3> best = {0, 1, 1};
      for (size_t ci = 0; ci < cands[kind].size(); ++ci) {
        double score = 0.0;
        for (size_t pi = 0; pi < pts.size(); ++pi)
          score += times[kind][ci][pi] / std::max(fastest[pi], 1e-6f);
        if (score < best_score) {
          best_score = score;
          best = cands[kind][ci];
        }
      }
      m->tuned[kind][b] = best;
    }
  }
  cleanup();
  if (st != SL_OK) {
    for (int k = 0; k < G_KINDS; ++k) m->tuned[k].clear();
    return st;
  }
  return SL_OK;
}

extern "C" sl_status sl_model_tuning(const sl_model *m, int kind, int M, int *bn, int *splits,
                                     int *variant) {
  if (!m || !bn || !splits || !variant || kind < 0 || kind >= G_KINDS || M <= 0)
    return fail(SL_ERR_INVALID, "sl_model_tuning: bad argument");
  const Plan p = plan_kind(m, kind, M, m->num_sms);
  *bn = p.bn;
  *splits = p.splits;
  *variant = plan_variant(p);
  return SL_OK;
}

extern "C" sl_status sl_model_set_ablation(sl_model *m, int flags) {
  if (!m) return fail(SL_ERR_INVALID, "sl_model_set_ablation: null model");
  if (flags & ~(SL_ABLATE_NO_KV_CACHE | SL_ABLATE_GATE_ONLY))
    return fail(SL_ERR_INVALID, "sl_model_set_ablation: unknown flags 0x%x", flags);
  m->ablation = flags;
  return SL_OK;
}

extern "C" sl_status sl_model_set_attention(sl_model *m, int queries_per_cta, int splits) {
  if (!m || (queries_per_cta != 0 && queries_per_cta != 16 && queries_per_cta != 32 &&
             queries_per_cta != 64 && queries_per_cta != 128 && queries_per_cta != 256) ||
      splits < 0 || splits > 16)
    return fail(SL_ERR_INVALID,
                "sl_model_set_attention: queries_per_cta 0/16/32/64/128/256, splits 0..16");
  m->attn_q = queries_per_cta;
  m->attn_splits = splits;
  return SL_OK;
}

extern "C" sl_status sl_model_set_attention_keys(sl_model *m, int key_tile) {
  if (!m || (key_tile != 0 && key_tile != 64 && key_tile != 128))
    return fail(SL_ERR_INVALID, "sl_model_set_attention_keys: key_tile 0, 64 or 128");
  m->attn_bn = key_tile;
  return SL_OK;
}

extern "C" sl_status sl_model_set_tuning(sl_model *m, int kind, int M, int bn, int splits,
                                         int variant) {
  if (!m || kind < 0 || kind >= G_KINDS || M <= 0 || tune_bucket(M) < 0)
    return fail(SL_ERR_INVALID, "sl_model_set_tuning: bad argument");
  if (m->cfg.dtype != SL_BF16) return fail(SL_ERR_INVALID, "sl_model_set_tuning: bf16 models only");
  const int d = m->cfg.d_model, f = m->cfg.d_ffn, V = m->cfg.vocab;
  const int Ns[G_KINDS] = {3 * d, d, 2 * f, d, V};
  const int N = Ns[kind];
  if ((bn != 64 && bn != 128 && bn != 192 && bn != 256) || N % bn || (kind == G_GU && f % (bn / 2)) ||
      (kind == G_QKV && (bn < 128 || d % bn || (bn % 128 != 0 && splits == 1))) || variant < 0 ||
      variant > 3 || (variant == 2 && bn < 128) ||
      (variant == 3 && (bn != 128 || kind == G_HD || splits < 1 ||
                        kTuneBounds[tune_bucket(M)] > 256)) ||
      (splits < 1 && splits != -1) || (kind == G_HD && splits != 1))
    return fail(SL_ERR_INVALID, "sl_model_set_tuning: tiling not valid for this GEMM");
  if (m->tuned[kind].empty())
    for (int k = 0; k < G_KINDS; ++k) m->tuned[k].assign(kTuneCount, {0, 1, 1});
  m->tuned[kind][tune_bucket(M)] = {bn, splits, variant};
  return SL_OK;
}

// -------------------------------------------------------------- lock test --
// The statistics half of the sure test as its own pass over the stored logits
// (lock_stats): the path of sl_kl_lock, and of sl_step_stats on fp32 models.
static sl_status kl_stats_unfused(sl_model *timing_model, sl_active *a, int M, int vocab,
                                  int mask_id, int dtype, const void *cur, const HeadStats &hs,
                                  cudaStream_t s) {
  if (M == 0) return SL_OK;
  LockStatsArgs la;
  la.dtype = dtype;
  la.cur = cur;
  la.prev = hs.prev;
  la.lse_prev = hs.lse_prev;
  la.lse_cur = hs.lse_cur;
  la.rows = a->rows;
  la.M = M;
  la.V = vocab;
  la.mask_id = mask_id;
  la.has_prev = hs.prev ? 1 : 0;
  la.kl = hs.kl;
  la.unc = hs.unc;
  la.conf = hs.conf;
  la.argmax = hs.argmax;
  la.part = a->part;
  la.counters = a->counters;
  la.splits = std::min(a->max_splits, lock_stats_splits(M, vocab, a->num_sms));
  const double bytes = (double)M * vocab * dsize(dtype) * (hs.prev ? 2 : 1) + 24.0 * M;
  Timed t(timing_model, SL_K_LOCK, bytes, 6.0 * M * vocab, s);
  SL_CUDA(launch_lock_stats(la, s));
  return SL_OK;
}

// The decision half: gate threshold per sequence and the lock flags.
static sl_status lock_decide_impl(sl_active *a, const uint8_t *masked, const sl_lock_params *p,
                                  const float *kl, const float *unc, uint8_t *lock,
                                  cudaStream_t s) {
  const bool gate_only = p->gate_only && p->scripted_target < 0;
  // gate only: the same decision with the KL bound at +inf, where D <= eps
  // always holds, so the gate alone decides among the eligible rows
  const float eps = gate_only ? INFINITY : p->eps;
  SL_CUDA(launch_lock_decide(a->seq_off, a->batch, a->rows, kl, unc, masked, eps, p->gate_q,
                             p->has_prev, p->scripted_target, lock, s));
  return SL_OK;
}

static sl_status check_lock_params(const sl_lock_params *p, const char *who) {
  if (p->gate_q > 1.f) return fail(SL_ERR_INVALID, "%s: gate_q must be <= 1", who);
  const bool gate_only = p->gate_only && p->scripted_target < 0;
  if (gate_only && !(p->gate_q >= 0.f))
    return fail(SL_ERR_INVALID, "%s: the gate-only criterion needs gate_q >= 0", who);
  return SL_OK;
}

static sl_status kl_lock_impl(sl_model *timing_model, sl_active *a, int vocab, int mask_id,
                              int dtype, const void *cur, const void *prev, const float *lse_prev,
                              float *lse_cur, const uint8_t *masked, const sl_lock_params *p,
                              float *kl, float *unc, float *conf, int32_t *argmax,
                              uint8_t *lock, cudaStream_t s) {
  if (!a || !cur || !lse_cur || !masked || !p || !kl || !unc || !conf || !argmax || !lock)
    return fail(SL_ERR_INVALID, "sl_kl_lock: null argument");
  if (p->has_prev && (!prev || !lse_prev))
    return fail(SL_ERR_INVALID, "sl_kl_lock: has_prev needs previous logits and lse");
  if (vocab <= 0 || vocab % 8 != 0)
    return fail(SL_ERR_INVALID, "sl_kl_lock: vocab must be a positive multiple of 8");
  if (mask_id < -1 || mask_id >= vocab) return fail(SL_ERR_INVALID, "sl_kl_lock: bad mask_id");
  if (dtype != SL_F32 && dtype != SL_BF16) return fail(SL_ERR_INVALID, "sl_kl_lock: bad dtype");
  sl_status st = check_lock_params(p, "sl_kl_lock");
  if (st != SL_OK) return st;
  if (((uintptr_t)cur & 15) || (prev && ((uintptr_t)prev & 15)))
    return fail(SL_ERR_INVALID, "sl_kl_lock: logits must be 16-byte aligned");
  int32_t counts[SL_MAX_BATCH];
  st = sl_active_counts(a, counts);
  if (st != SL_OK) return st;
  int M = 0;
  for (int b = 0; b < a->batch; ++b) M += counts[b];
  if (M == 0) return SL_OK;
  HeadStats hs;
  hs.prev = p->has_prev ? prev : nullptr;
  hs.lse_prev = p->has_prev ? lse_prev : nullptr;
  hs.lse_cur = lse_cur;
  hs.kl = kl;
  hs.unc = unc;
  hs.conf = conf;
  hs.argmax = argmax;
  if ((st = kl_stats_unfused(timing_model, a, M, vocab, mask_id, dtype, cur, hs, s)) != SL_OK)
    return st;
  return lock_decide_impl(a, masked, p, kl, unc, lock, s);
}

extern "C" sl_status sl_lock_decide(sl_active *a, const uint8_t *d_masked,
                                    const sl_lock_params *p, const float *d_kl,
                                    const float *d_unc, uint8_t *d_lock, void *stream) {
  if (!a || !d_masked || !p || !d_kl || !d_unc || !d_lock)
    return fail(SL_ERR_INVALID, "sl_lock_decide: null argument");
  sl_status st = check_lock_params(p, "sl_lock_decide");
  if (st != SL_OK) return st;
  return lock_decide_impl(a, d_masked, p, d_kl, d_unc, d_lock, (cudaStream_t)stream);
}

extern "C" sl_status sl_model_set_head_fusion(sl_model *m, int enable) {
  if (!m) return fail(SL_ERR_INVALID, "sl_model_set_head_fusion: null model");
  m->head_fusion = enable != 0;
  return SL_OK;
}

extern "C" sl_status sl_kl_lock(sl_active *a, int vocab, int mask_id, int logits_dtype,
                                const void *d_logits_cur, const void *d_logits_prev,
                                const float *d_lse_prev, float *d_lse_cur,
                                const uint8_t *d_masked, const sl_lock_params *p, float *d_kl,
                                float *d_unc, float *d_conf, int32_t *d_argmax, uint8_t *d_lock,
                                void *stream) {
  return kl_lock_impl(nullptr, a, vocab, mask_id, logits_dtype, d_logits_cur, d_logits_prev,
                      d_lse_prev, d_lse_cur, d_masked, p, d_kl, d_unc, d_conf, d_argmax, d_lock,
                      (cudaStream_t)stream);
}

extern "C" sl_status sl_unmask_topk(sl_active *a, const float *d_conf, const int32_t *d_argmax,
                                    int block_lo, int block_hi, int k, int32_t *d_tokens,
                                    uint8_t *d_masked, void *stream) {
  if (!a || !d_conf || !d_argmax || !d_tokens || !d_masked)
    return fail(SL_ERR_INVALID, "sl_unmask_topk: null argument");
  if (block_lo < 0 || block_hi > a->n_ctx || block_lo > block_hi || k < 0)
    return fail(SL_ERR_INVALID, "sl_unmask_topk: bad block [%d, %d) or k %d", block_lo,
                block_hi, k);
  if (block_hi - block_lo > 2048)
    return fail(SL_ERR_UNSUPPORTED, "sl_unmask_topk: blocks longer than 2048");
  if (k == 0 || block_hi == block_lo) return SL_OK;
  SL_CUDA(launch_unmask(a->seq_off, a->batch, a->rows, a->n_ctx, d_conf, d_argmax, block_lo,
                        block_hi, k, d_tokens, d_masked, (cudaStream_t)stream));
  return SL_OK;
}

extern "C" sl_status sl_compact_active(sl_active *a, const uint8_t *d_lock, uint8_t *d_locked,
                                       int32_t *d_lock_t, int step, void *stream) {
  if (!a || !d_lock || !d_locked || !d_lock_t)
    return fail(SL_ERR_INVALID, "sl_compact_active: null argument");
  cudaStream_t s = (cudaStream_t)stream;
  SL_CUDA(launch_compact(a->rows, a->seq_off, a->batch, d_lock, d_locked, d_lock_t, step, s));
  return active_mirror(a, s);
}

// ----------------------------------------------------------------- sampler --
extern "C" void sl_sampler_destroy(sl_sampler *s) {
  if (!s) return;
  sl_kv_cache_destroy(s->cache);
  sl_active_destroy(s->act);
  sl_active_destroy(s->comp);
  void *ps[] = {s->tokens, s->masked, s->locked, s->lock, s->lock_t, s->argmax, s->d_prompts,
                s->logits[0], s->logits[1], s->lse[0], s->lse[1], s->kl, s->unc, s->conf,
                s->masked_before, s->lock_by_pos, s->lock_act};
  for (void *p : ps)
    if (p) cudaFree(p);
  delete s;
}

extern "C" sl_status sl_sampler_create(sl_model *m, int batch, const sl_sampler_params *p,
                                       sl_sampler **out) {
  if (!m || !p || !out) return fail(SL_ERR_INVALID, "sl_sampler_create: null argument");
  *out = nullptr;
  const sl_sampler_params &q = *p;
  if (q.prompt_len < 0 || q.gen_len <= 0 || q.steps <= 0 || q.block_len <= 0 ||
      q.tokens_per_step <= 0)
    return fail(SL_ERR_INVALID, "sl_sampler_create: non-positive sizes");
  if (q.gen_len % q.block_len != 0 || q.steps % (q.gen_len / q.block_len) != 0)
    return fail(SL_ERR_INVALID,
                "sl_sampler_create: gen_len must split into blocks and steps into blocks");
  if (q.block_len > 2048) return fail(SL_ERR_UNSUPPORTED, "sl_sampler_create: block_len > 2048");
  if (q.gate_q > 1.f) return fail(SL_ERR_INVALID, "sl_sampler_create: gate_q must be <= 1");
  sl_sampler *s = new sl_sampler();
  s->m = m;
  s->p = q;
  s->batch = batch;
  s->n_ctx = q.prompt_len + q.gen_len;
  sl_status st = sl_kv_cache_create(m, batch, s->n_ctx, &s->cache);
  if (st == SL_OK) st = sl_active_create(batch, s->n_ctx, &s->act);
  if (st != SL_OK) {
    sl_sampler_destroy(s);
    return st;
  }
  const size_t rows = (size_t)batch * s->n_ctx;
  const size_t es = dsize(m->cfg.dtype);
  bool ok = cudaMalloc(&s->tokens, rows * 4) == cudaSuccess &&
            cudaMalloc(&s->masked, rows) == cudaSuccess &&
            cudaMalloc(&s->locked, rows) == cudaSuccess &&
            cudaMalloc(&s->lock, rows) == cudaSuccess &&
            cudaMalloc(&s->lock_t, rows * 4) == cudaSuccess &&
            cudaMalloc(&s->argmax, rows * 4) == cudaSuccess &&
            cudaMalloc(&s->d_prompts, std::max<size_t>(1, (size_t)batch * q.prompt_len) * 4) ==
                cudaSuccess &&
            cudaMalloc(&s->logits[0], rows * m->cfg.vocab * es) == cudaSuccess &&
            cudaMalloc(&s->logits[1], rows * m->cfg.vocab * es) == cudaSuccess &&
            cudaMalloc(&s->lse[0], rows * 4) == cudaSuccess &&
            cudaMalloc(&s->lse[1], rows * 4) == cudaSuccess &&
            cudaMalloc(&s->kl, rows * 4) == cudaSuccess &&
            cudaMalloc(&s->unc, rows * 4) == cudaSuccess &&
            cudaMalloc(&s->conf, rows * 4) == cudaSuccess;
  if (!ok) {
    sl_sampler_destroy(s);
    return fail(SL_ERR_OOM, "sl_sampler_create: device allocation failed");
  }
  *out = s;
  return SL_OK;
}

namespace {
__global__ void sampler_init_kernel(const int32_t *prompts, int batch, int prompt_len, int n_ctx,
                                    int mask_id, int32_t *tokens, uint8_t *masked,
                                    uint8_t *locked, int32_t *lock_t) {
  pdl_wait();
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= batch * n_ctx) return;
  int b = i / n_ctx, pos = i - b * n_ctx;
  bool prompt = pos < prompt_len;
  tokens[i] = prompt ? prompts[b * prompt_len + pos] : mask_id;
  masked[i] = prompt ? 0 : 1;
  locked[i] = 0;
  lock_t[i] = -1;
}
}  // namespace

extern "C" sl_status sl_sampler_start(sl_sampler *s, const int32_t *d_prompts, void *stream) {
  if (!s || (!d_prompts && s->p.prompt_len > 0))
    return fail(SL_ERR_INVALID, "sl_sampler_start: null argument");
  cudaStream_t st = (cudaStream_t)stream;
  const int rows = s->batch * s->n_ctx;
  SL_CUDA(launch_k(sampler_init_kernel, (rows + 255) / 256, 256, 0, st, d_prompts, s->batch,
                   s->p.prompt_len, s->n_ctx, s->m->cfg.mask_id, s->tokens, s->masked, s->locked,
                   s->lock_t));
  sl_status r = sl_kv_cache_reset(s->cache, stream);
  if (r != SL_OK) return r;
  r = sl_active_reset(s->act, stream);
  if (r != SL_OK) return r;
  if (s->lock_by_pos)
    SL_CUDA(cudaMemsetAsync(s->lock_by_pos, 0, (size_t)rows, st));
  s->t = 0;
  s->started = true;
  return SL_OK;
}

extern "C" sl_status sl_sampler_set_kv_reuse(sl_sampler *s, int period) {
  if (!s) return fail(SL_ERR_INVALID, "sl_sampler_set_kv_reuse: null sampler");
  if (period < 1) return fail(SL_ERR_INVALID, "sl_sampler_set_kv_reuse: period %d < 1", period);
  if (period > 1 && s->p.scripted)
    return fail(SL_ERR_INVALID, "sl_sampler_set_kv_reuse: the scripted schedule counts its "
                                "locks over the whole active set");
  if (s->started && s->t < s->p.steps)
    return fail(SL_ERR_STATE, "sl_sampler_set_kv_reuse: a decode is in progress");
  if (period > 1 && !s->comp) {
    const size_t rows = (size_t)s->batch * s->n_ctx;
    sl_status st = sl_active_create(s->batch, s->n_ctx, &s->comp);
    if (st != SL_OK) return st;
    bool ok = cudaMalloc(&s->masked_before, rows) == cudaSuccess &&
              cudaMalloc(&s->lock_by_pos, rows) == cudaSuccess &&
              cudaMalloc(&s->lock_act, rows) == cudaSuccess &&
              cudaMemset(s->lock_by_pos, 0, rows) == cudaSuccess;
    if (!ok) {
      sl_active_destroy(s->comp);
      for (uint8_t **q : {&s->masked_before, &s->lock_by_pos, &s->lock_act}) {
        if (*q) cudaFree(*q);
        *q = nullptr;
      }
      s->comp = nullptr;
      return fail(SL_ERR_OOM, "sl_sampler_set_kv_reuse: device allocation failed");
    }
  }
  s->kv_reuse = period;
  return SL_OK;
}

extern "C" sl_status sl_sampler_step(sl_sampler *s, void *stream) {
  if (!s) return fail(SL_ERR_INVALID, "sl_sampler_step: null sampler");
  if (!s->started) return fail(SL_ERR_STATE, "sl_sampler_step: call sl_sampler_start first");
  if (s->t >= s->p.steps) return fail(SL_ERR_STATE, "sl_sampler_step: decode already finished");
  if ((s->m->ablation & SL_ABLATE_GATE_ONLY) && !s->p.scripted && !(s->p.gate_q >= 0.f))
    return fail(SL_ERR_INVALID, "sl_sampler_step: the gate-only ablation needs gate_q >= 0");
  const bool reuse = s->kv_reuse > 1;
  if (reuse && (s->m->ablation & SL_ABLATE_NO_KV_CACHE))
    return fail(SL_ERR_INVALID, "sl_sampler_step: K/V reuse needs the cache of every row (the "
                                "no-KV-cache ablation is on)");
  const int t = s->t;
  const int cur = t & 1, prv = cur ^ 1;
  const sl_config &cfg = s->m->cfg;
  sl_status st = SL_OK;
  cudaStream_t cs = (cudaStream_t)stream;
  // K/V reuse: all active rows at a refresh step (t mod R = 0), else the rows
  // that are masked or were masked at the start of the previous step; the
  // others carry their logits and lse into this step's buffers
  const bool refresh = !reuse || t % s->kv_reuse == 0;
  sl_active *run = refresh ? s->act : s->comp;
  if (!refresh) {
    SL_CUDA(launch_reuse_select(s->act->rows, s->act->seq_off, s->batch, s->masked,
                                s->masked_before, s->comp->rows, s->comp->seq_off, cs));
    if ((st = active_mirror(s->comp, cs)) != SL_OK) return st;
    int32_t ca[SL_MAX_BATCH], cc[SL_MAX_BATCH];
    if ((st = sl_active_counts(s->act, ca)) != SL_OK) return st;
    if ((st = sl_active_counts(s->comp, cc)) != SL_OK) return st;
    int ma = 0, mc = 0;
    for (int b = 0; b < s->batch; ++b) {
      ma += ca[b];
      mc += cc[b];
    }
    const size_t row_bytes = (size_t)cfg.vocab * dsize(cfg.dtype);
    Timed tm(s->m, SL_K_OTHER, 2.0 * (ma - mc) * ((double)row_bytes + 4.0), 0.0, cs);
    SL_CUDA(launch_reuse_carry(s->act->rows, s->act->seq_off, s->batch, ma, s->masked,
                               s->masked_before, s->logits[prv], s->logits[cur], s->lse[prv],
                               s->lse[cur], row_bytes, cs));
  }
  if (reuse)
    SL_CUDA(cudaMemcpyAsync(s->masked_before, s->masked, (size_t)s->batch * s->n_ctx,
                            cudaMemcpyDeviceToDevice, cs));
  sl_lock_params lp;
  lp.eps = s->p.eps;
  lp.gate_q = s->p.gate_q;
  lp.has_prev = t > 0 ? 1 : 0;
  lp.scripted_target = -1;
  lp.gate_only = (s->m->ablation & SL_ABLATE_GATE_ONLY) ? 1 : 0;
  if (s->p.scripted) {
    // M_{t+1} = round-half-up(N - 0.9 N (t+1)/(T-1))
    const double n = s->n_ctx;
    const double x = s->p.steps > 1 ? n - 0.9 * n * (t + 1) / (s->p.steps - 1) : n;
    lp.scripted_target = (int)floor(x + 0.5);
    if (lp.scripted_target < 0) lp.scripted_target = 0;
  }
  if (s->m->head_fusion && cfg.dtype == SL_BF16) {
    // the sure test's statistics come out of the LM head's epilogue
    st = sl_step_stats(s->m, s->cache, run, s->tokens, s->logits[cur], s->logits[prv],
                       s->lse[prv], lp.has_prev, s->lse[cur], s->kl, s->unc, s->conf, s->argmax,
                       stream);
    if (st != SL_OK) return st;
    st = lock_decide_impl(run, s->masked, &lp, s->kl, s->unc, s->lock, cs);
  } else {
    st = sl_step(s->m, s->cache, run, s->tokens, s->logits[cur], stream);
    if (st != SL_OK) return st;
    st = kl_lock_impl(s->m, run, cfg.vocab, cfg.mask_id, cfg.dtype, s->logits[cur],
                      s->logits[prv], s->lse[prv], s->lse[cur], s->masked, &lp, s->kl, s->unc,
                      s->conf, s->argmax, s->lock, (cudaStream_t)stream);
  }
  if (st != SL_OK) return st;
  const int spb = s->p.steps / (s->p.gen_len / s->p.block_len);
  const int lo = s->p.prompt_len + (t / spb) * s->p.block_len;
  st = sl_unmask_topk(run, s->conf, s->argmax, lo, lo + s->p.block_len, s->p.tokens_per_step,
                      s->tokens, s->masked, stream);
  if (st != SL_OK) return st;
  const uint8_t *lock_act = s->lock;
  if (!refresh) {
    SL_CUDA(launch_reuse_lock_map(s->comp->rows, s->comp->seq_off, s->lock, s->act->rows,
                                  s->act->seq_off, s->batch, s->lock_by_pos, s->lock_act, cs));
    lock_act = s->lock_act;
  }
  st = sl_compact_active(s->act, lock_act, s->locked, s->lock_t, t, stream);
  if (st != SL_OK) return st;
  s->t = t + 1;
  return SL_OK;
}

extern "C" sl_status sl_sampler_generate(sl_sampler *s, const int32_t *h_prompts,
                                         int32_t *h_tokens, void *stream) {
  if (!s || !h_tokens || (!h_prompts && s->p.prompt_len > 0))
    return fail(SL_ERR_INVALID, "sl_sampler_generate: null argument");
  const size_t n_prompt = (size_t)s->batch * s->p.prompt_len;
  for (size_t i = 0; i < n_prompt; ++i)
    if (h_prompts[i] < 0 || h_prompts[i] >= s->m->cfg.vocab)
      return fail(SL_ERR_INVALID, "sl_sampler_generate: prompt id %d at %zu outside [0, %d)",
                  (int)h_prompts[i], i, s->m->cfg.vocab);
  cudaStream_t st = (cudaStream_t)stream;
  if (s->p.prompt_len > 0)
    SL_CUDA(cudaMemcpyAsync(s->d_prompts, h_prompts, (size_t)s->batch * s->p.prompt_len * 4,
                            cudaMemcpyHostToDevice, st));
  sl_status r = sl_sampler_start(s, s->d_prompts, stream);
  if (r != SL_OK) return r;
  while (s->t < s->p.steps) {
    r = sl_sampler_step(s, stream);
    if (r != SL_OK) return r;
  }
  SL_CUDA(cudaMemcpyAsync(h_tokens, s->tokens, (size_t)s->batch * s->n_ctx * 4,
                          cudaMemcpyDeviceToHost, st));
  SL_CUDA(cudaStreamSynchronize(st));
  return SL_OK;
}

extern "C" sl_status sl_sampler_get_state(const sl_sampler *s, sl_sampler_state *o) {
  if (!s || !o) return fail(SL_ERR_INVALID, "sl_sampler_get_state: null argument");
  o->tokens = s->tokens;
  o->masked = s->masked;
  o->locked = s->locked;
  o->lock_t = s->lock_t;
  o->logits[0] = s->logits[0];
  o->logits[1] = s->logits[1];
  o->lse[0] = s->lse[0];
  o->lse[1] = s->lse[1];
  o->kl = s->kl;
  o->unc = s->unc;
  o->conf = s->conf;
  o->argmax = s->argmax;
  o->lock = s->lock;
  o->cache = s->cache;
  o->active = s->act;
  o->computed = s->comp;
  o->t = s->t;
  o->batch = s->batch;
  o->n_ctx = s->n_ctx;
  return SL_OK;
}
