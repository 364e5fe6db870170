// C ABI of the CCGQA hot path: host-side validation, workspace layout and
// kernel dispatch.  Every entry point validates all arguments before the first
// launch and returns a status; the kernels themselves never trap.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <map>
#include <mutex>
#include <new>
#include <utility>

#include "kernels.h"

namespace ccgqa {

static std::atomic<uint64_t> g_launches{0};

// Graph capture of the calling thread (ccgqa_graph_begin .. ccgqa_graph_end):
// the stream being captured and the library kernels recorded so far.  Kernels
// recorded into a graph count when a launch of the graph runs them.
struct Capture {
  cudaStream_t stream = nullptr;
  int64_t kernels = 0;
  bool active = false;
};
static thread_local Capture t_capture;

void count_launches(int n) {
  if (t_capture.active)
    t_capture.kernels += n;
  else
    g_launches.fetch_add(static_cast<uint64_t>(n));
}
// While this thread captures, every launching call must use the captured stream.
bool stream_allowed(cudaStream_t st) { return !t_capture.active || st == t_capture.stream; }

cudaError_t allow_smem(const void* func, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, int> allowed;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  int& have = allowed[{dev, func}];
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

int sm_count() {
  static std::mutex mu;
  static std::map<int, int> counts;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lock(mu);
  auto it = counts.find(dev);
  if (it != counts.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  counts[dev] = n;
  return n;
}

// Last CUDA error met by an entry point on this thread.
static thread_local char t_last_error[256] = "no error";
static ccgqa_status cuda_fail(cudaError_t e) {
  snprintf(t_last_error, sizeof(t_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return CCGQA_ERR_CUDA;
}

// Whether ccgqa_prefill may fuse the projection with the pre-attention
// (ccgqa_set_fused_projection; on unless switched off).
static std::atomic<int> g_fuse_proj{1};

// Optional phase events of the calling thread (ccgqa_set_phase_events).
static thread_local void* const* t_phase_events = nullptr;
static void phase_mark(int i, cudaStream_t st) {
  if (t_phase_events && !t_capture.active)
    cudaEventRecord(static_cast<cudaEvent_t>(t_phase_events[i]), st);
}

namespace {

struct Geo {
  int E, C, Hq, Hkv, d, G, N, K;
  int qk_mean, value_shift, causal, rope_on, channel_conv;
  double rope_log2_base;
  int dtype;
  size_t es;  // element size
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// theta_i / (2 pi) * 2^64 with theta_i = base^(-2i/d) (RoPE, "Compressed
// Convolutional Attention", Methodologie item 4), rounded to an integer in
// extended precision; below 2^62 since theta_i <= 1.
uint64_t rope_turn_fraction(double log2_base, int i, int d) {
  const long double th = exp2l(-(2.0L * i / d) * static_cast<long double>(log2_base));
  const long double two_pi = 6.283185307179586476925286766559005768L;
  return static_cast<uint64_t>(llroundl(th / two_pi * 18446744073709551616.0L));
}
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

ccgqa_status derive(const ccgqa_config* cfg, Geo* g) {
  if (!cfg) return CCGQA_ERR_INVALID_ARG;
  if (cfg->E <= 0 || cfg->C <= 0 || cfg->n_q_heads <= 0 || cfg->n_kv_heads <= 0)
    return CCGQA_ERR_INVALID_ARG;
  if (cfg->n_q_heads % cfg->n_kv_heads != 0) return CCGQA_ERR_INVALID_ARG;
  if (cfg->E % (cfg->C * cfg->n_q_heads) != 0) return CCGQA_ERR_INVALID_ARG;
  if (cfg->conv_width < 0 || cfg->conv_width > 4) return CCGQA_ERR_INVALID_ARG;
  if (cfg->qk_mean < 0 || cfg->qk_mean > 2 || cfg->value_shift < 0 || cfg->value_shift > 2 ||
      (cfg->causal & ~1) || (cfg->channel_conv & ~1))
    return CCGQA_ERR_INVALID_ARG;
  if (cfg->channel_conv && cfg->conv_width == 0) return CCGQA_ERR_INVALID_ARG;
  if (!(cfg->rope_base >= 0.0) || std::isinf(cfg->rope_base)) return CCGQA_ERR_INVALID_ARG;
  if (cfg->dtype != CCGQA_F32 && cfg->dtype != CCGQA_BF16) return CCGQA_ERR_INVALID_ARG;
  g->E = cfg->E;
  g->C = cfg->C;
  g->Hq = cfg->n_q_heads;
  g->Hkv = cfg->n_kv_heads;
  g->d = cfg->E / (cfg->C * cfg->n_q_heads);
  g->G = g->Hq / g->Hkv;
  g->N = (g->Hq + 2 * g->Hkv) * g->d;
  g->K = cfg->conv_width;
  g->qk_mean = cfg->qk_mean;
  g->value_shift = cfg->value_shift;
  g->causal = cfg->causal;
  g->channel_conv = cfg->channel_conv;
  g->rope_on = cfg->rope_base > 0.0;
  g->rope_log2_base = g->rope_on ? std::log2(cfg->rope_base) : 0.0;
  g->dtype = cfg->dtype;
  g->es = cfg->dtype == CCGQA_F32 ? 4 : 2;
  if (g->d != 16 && g->d != 32 && g->d != 64 && g->d != 128) return CCGQA_ERR_UNSUPPORTED;
  // the per-sequence decode pre-step stages (G + 2) d channels in shared memory
  if (!decode_pre_fits(g->G, g->d, g->K, static_cast<int>(g->es))) return CCGQA_ERR_UNSUPPORTED;
  return CCGQA_OK;
}

ccgqa_status check_weights(const Geo& g, const ccgqa_weights* w) {
  if (!w) return CCGQA_ERR_INVALID_ARG;
  if (w->W_qkv && !aligned16(w->W_qkv)) return CCGQA_ERR_INVALID_ARG;
  if (g.K > 0 && g.channel_conv) {
    // per-tap matrices only: [Hq, K, d, d] and [Hkv, K, d, d]
    if (!w->conv_q_chan || !w->conv_k_chan) return CCGQA_ERR_INVALID_ARG;
    if (!aligned16(w->conv_q_chan) || !aligned16(w->conv_k_chan)) return CCGQA_ERR_INVALID_ARG;
  } else if (g.K > 0) {
    if (!w->conv_q_seq || !w->conv_k_seq) return CCGQA_ERR_INVALID_ARG;
    if (!aligned16(w->conv_q_seq) || !aligned16(w->conv_k_seq)) return CCGQA_ERR_INVALID_ARG;
    if ((w->conv_q_chan && !aligned16(w->conv_q_chan)) ||
        (w->conv_k_chan && !aligned16(w->conv_k_chan)))
      return CCGQA_ERR_INVALID_ARG;
  }
  return CCGQA_OK;
}

ccgqa_status check_cache(const Geo& g, const ccgqa_kvcache* c, bool need_state) {
  if (!c) return CCGQA_ERR_INVALID_ARG;
  if (c->batch <= 0 || c->cap <= 0) return CCGQA_ERR_INVALID_ARG;
  if (!c->k || !c->v || !c->len || !aligned16(c->k) || !aligned16(c->v))
    return CCGQA_ERR_INVALID_ARG;
  if (need_state) {
    if (g.K > 1 && (!c->conv_hist_q || !c->conv_hist_k)) return CCGQA_ERR_INVALID_ARG;
    if (g.value_shift && !c->v_prev) return CCGQA_ERR_INVALID_ARG;
  }
  if (c->block_table) {
    // pages of a power-of-two size from 16 to 4096 tokens that divides cap;
    // the pool's page planes (n_pages * Hkv) index a TMA coordinate (int32)
    const int ps = c->page_size;
    if (ps < 16 || ps > 4096 || (ps & (ps - 1)) || c->cap % ps) return CCGQA_ERR_INVALID_ARG;
    if (c->n_pages <= 0 || static_cast<int64_t>(c->n_pages) * g.Hkv >= (int64_t(1) << 31))
      return CCGQA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(c->block_table) & 3) return CCGQA_ERR_INVALID_ARG;
  }
  return CCGQA_OK;
}

PageMap page_map(const ccgqa_kvcache* c) {
  PageMap pm{};
  if (c && c->block_table) {
    pm.table = c->block_table;
    int sh = 0;
    while ((1 << sh) < c->page_size) ++sh;
    pm.shift = sh;
    pm.per_seq = c->cap >> sh;
    pm.n_pages = c->n_pages;
  }
  return pm;
}

struct PrefillWs {
  size_t proj, q, k, v, total;
};
PrefillWs prefill_ws(const Geo& g, int64_t B, int64_t S) {
  PrefillWs w;
  size_t off = 0;
  w.proj = off;
  off += up256(static_cast<size_t>(B * S) * g.N * g.es);
  w.q = off;
  off += up256(static_cast<size_t>(B * S) * g.Hq * g.d * g.es);
  w.k = off;
  off += up256(static_cast<size_t>(B * S) * g.Hkv * g.d * g.es);
  w.v = off;
  off += up256(static_cast<size_t>(B * S) * g.Hkv * g.d * g.es);
  w.total = off;
  return w;
}

struct DecodeWs {
  size_t proj, q, po, pml, tick, total;
  int e_splits, splits, chunk;
};
DecodeWs decode_ws(const Geo& g, int64_t B, int64_t cap, bool has_proj) {
  DecodeWs w;
  decode_plan(static_cast<int>(B), g.Hkv, g.E, g.N, cap, has_proj, g.es, &w.e_splits, &w.splits,
              &w.chunk);
  size_t off = 0;
  w.tick = off;  // tickets first: the part a fresh zero-fill must cover
  off += up256(static_cast<size_t>(B * g.Hkv + B) * 4);
  w.proj = off;
  off += up256(static_cast<size_t>(w.e_splits) * B * g.N * 4);
  w.q = off;
  off += up256(static_cast<size_t>(B) * g.Hq * g.d * 4);
  w.po = off;
  off += up256(static_cast<size_t>(B) * g.Hkv * w.splits * g.G * g.d * 4);
  w.pml = off;
  off += up256(static_cast<size_t>(B) * g.Hkv * w.splits * g.G * 2 * 4);
  w.total = off;
  return w;
}

// The tensor-core attention covers d >= 32 and groups of at most 128 heads (a
// query tile packs floor(128 / G) positions of the G heads); d = 16 and larger
// groups run on the CUDA-core kernel.
bool attn_tc_applies(const Geo& g) { return g.d >= 32 && g.G <= 128; }

template <typename T>
ccgqa_status run_prefill(const Geo& g, const ccgqa_weights* w, const void* x, int B, int S,
                         void* out, const ccgqa_kvcache* cache, uint8_t* ws, int32_t* dev_err,
                         cudaStream_t st) {
  const PrefillWs L = prefill_ws(g, B, S);
  T* proj = reinterpret_cast<T*>(ws + L.proj);
  const T* src = w->W_qkv ? proj : static_cast<const T*>(x);
  cudaError_t e = cudaSuccess;
  phase_mark(0, st);
  PreAttnArgs<T> a{};
  a.src = src;
  a.src_ld = g.N;
  a.B = B;
  a.S = S;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.d = g.d;
  a.G = g.G;
  a.K = g.K;
  a.qk_mean = g.qk_mean;
  a.value_shift = g.value_shift;
  a.channel_conv = g.channel_conv;
  a.rope_on = g.rope_on;
  a.rope_log2_base = g.rope_log2_base;
  if (g.rope_on)
    for (int i = 0; i < g.d / 2; ++i) a.rope_frac[i] = rope_turn_fraction(g.rope_log2_base, i, g.d);
  a.wq_seq = static_cast<const T*>(w->conv_q_seq);
  a.wq_chan = static_cast<const T*>(w->conv_q_chan);
  a.wk_seq = static_cast<const T*>(w->conv_k_seq);
  a.wk_chan = static_cast<const T*>(w->conv_k_chan);
  a.q_out = reinterpret_cast<T*>(ws + L.q);
  // a paged cache takes k / v from the workspace after the attention
  const bool paged = cache && cache->block_table;
  if (cache && !paged) {
    a.k_out = static_cast<T*>(cache->k);
    a.v_out = static_cast<T*>(cache->v);
    a.kv_cap = cache->cap;
  } else {
    a.k_out = reinterpret_cast<T*>(ws + L.k);
    a.v_out = reinterpret_cast<T*>(ws + L.v);
    a.kv_cap = S;
  }
  if (cache) {
    a.hist_q = static_cast<T*>(cache->conv_hist_q);
    a.hist_k = static_cast<T*>(cache->conv_hist_k);
    a.v_prev = static_cast<T*>(cache->v_prev);
    a.len = cache->len;
  }
  a.dev_err = dev_err;
  bool fused = false;
  if constexpr (sizeof(T) == 2)
    fused = w->W_qkv && g_fuse_proj.load() &&
            proj_pre_tc_supported(a, static_cast<const bf16*>(x),
                                  static_cast<const bf16*>(w->W_qkv), g.E);
  if (fused) {
    // projection and pre-attention in one kernel (no q~ | k~ | v~ in HBM)
    if constexpr (sizeof(T) == 2)
      e = launch_proj_pre_tc(static_cast<const bf16*>(x), static_cast<const bf16*>(w->W_qkv), g.E,
                             a, st);
    if (e != cudaSuccess) return cuda_fail(e);
    phase_mark(1, st);
  } else {
    if (w->W_qkv) {
      if constexpr (sizeof(T) == 2)
        e = launch_proj_gemm_bf16(static_cast<const bf16*>(x),
                                  static_cast<const bf16*>(w->W_qkv), proj, B * S, g.N, g.E,
                                  dev_err, st);
      else
        e = launch_proj_gemm_f32(static_cast<const float*>(x),
                                 static_cast<const float*>(w->W_qkv), proj, B * S, g.N, g.E, st);
      if (e != cudaSuccess) return cuda_fail(e);
    }
    phase_mark(1, st);
    if ((e = launch_pre_attn<T>(a, st)) != cudaSuccess) return cuda_fail(e);
  }
  phase_mark(2, st);
  AttnArgs at{};
  at.q = a.q_out;
  at.k = a.k_out;
  at.v = a.v_out;
  at.out = out;
  at.B = B;
  at.S = S;
  at.Hq = g.Hq;
  at.Hkv = g.Hkv;
  at.d = g.d;
  at.G = g.G;
  at.kv_cap = a.kv_cap;
  at.causal = g.causal;
  at.dev_err = dev_err;
  if constexpr (sizeof(T) == 2) {
    if (attn_tc_applies(g))
      e = launch_attn_prefill_tc(at, st);
    else
      e = launch_attn_prefill_simt<T>(at, st);
  } else {
    e = launch_attn_prefill_simt<T>(at, st);
  }
  if (e == cudaSuccess && paged)
    e = launch_kv_scatter<T>(static_cast<T*>(cache->k), static_cast<T*>(cache->v),
                             page_map(cache), a.k_out, a.v_out, B, g.Hkv, g.d, cache->cap, S,
                             dev_err, st);
  phase_mark(3, st);
  return e == cudaSuccess ? CCGQA_OK : cuda_fail(e);
}

struct BwdWs {
  size_t z, q, k, v, o, dq, dk, dv, lse, dsum, dy, dzm, du, u, dz, dz_b, wt, dzt, xt, total;
  int64_t ldr;      // rows of the transposed gradient-GEMM operands (B S rounded up to 8)
  int64_t lse_ld;   // packed log-sum-exp rows per (sequence, kv group), tensor-core path
};
BwdWs backward_ws(const Geo& g, int64_t B, int64_t S, bool has_proj) {
  BwdWs w;
  const size_t rows = static_cast<size_t>(B * S);
  const size_t qn = rows * g.Hq * g.d, kvn = rows * g.Hkv * g.d;
  const size_t cqk = rows * (g.Hq + g.Hkv) * g.d;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += up256(bytes);
    return at;
  };
  w.z = take(has_proj ? rows * g.N * g.es : 0);
  w.q = take(qn * g.es);
  w.k = take(kvn * g.es);
  w.v = take(kvn * g.es);
  w.o = take(g.dtype == CCGQA_BF16 ? qn * g.es : 0);
  w.dq = take(qn * 4);
  w.dk = take(kvn * 4);
  w.dv = take(kvn * 4);
  // [B, Hq, S] for the CUDA-core kernels; [B Hkv, lse_ld] packed rows (S G
  // rounded up to 64) for the tensor-core ones
  w.lse_ld = (S * g.G + 63) / 64 * 64;
  const size_t n_lse = std::max(static_cast<size_t>(B) * g.Hq * S,
                                static_cast<size_t>(B) * g.Hkv * static_cast<size_t>(w.lse_ld));
  w.lse = take(n_lse * 4);
  w.dsum = take(n_lse * 4);
  w.dy = take(cqk * 4);
  w.dzm = take(cqk * 4);
  w.du = take(cqk * 4);
  w.u = take(cqk * 4);
  w.dz = take(rows * g.N * 4);
  // bf16 with a projection: operands of the tensor-core gradient GEMMs
  const bool tc_gemm = g.dtype == CCGQA_BF16 && has_proj;
  w.ldr = (static_cast<int64_t>(rows) + 7) / 8 * 8;
  w.dz_b = take(tc_gemm ? rows * g.N * 2 : 0);
  w.wt = take(tc_gemm ? static_cast<size_t>(g.E) * g.N * 2 : 0);
  w.dzt = take(tc_gemm ? static_cast<size_t>(g.N) * w.ldr * 2 : 0);
  w.xt = take(tc_gemm ? static_cast<size_t>(g.E) * w.ldr * 2 : 0);
  w.total = off;
  return w;
}

// Elements of each weight gradient (the shapes of the weights).
size_t grad_elems(const Geo& g, int which) {
  const size_t d = g.d, K = g.K;
  switch (which) {
    case 0: return static_cast<size_t>(g.N) * g.E;                       // W_qkv
    case 1: return g.channel_conv ? 0 : static_cast<size_t>(g.Hq) * d * K;   // conv_q_seq
    case 2: return static_cast<size_t>(g.Hq) * d * d * (g.channel_conv ? K : 1);
    case 3: return g.channel_conv ? 0 : static_cast<size_t>(g.Hkv) * d * K;
    default: return static_cast<size_t>(g.Hkv) * d * d * (g.channel_conv ? K : 1);
  }
}

template <typename T>
ccgqa_status run_backward(const Geo& g, const ccgqa_weights* w, const void* x, int B, int S,
                          const void* dout, void* dx, const ccgqa_weight_grads* dw, uint8_t* ws,
                          int32_t* dev_err, cudaStream_t st) {
  const BwdWs L = backward_ws(g, B, S, w->W_qkv != nullptr);
  cudaError_t e = cudaSuccess;
  // forward values the backward needs: z = q~ | k~ | v~, then q, k, v
  const T* z = static_cast<const T*>(x);
  if (w->W_qkv) {
    T* zw = reinterpret_cast<T*>(ws + L.z);
    if constexpr (sizeof(T) == 2)
      e = launch_proj_gemm_bf16(static_cast<const bf16*>(x), static_cast<const bf16*>(w->W_qkv),
                                zw, B * S, g.N, g.E, dev_err, st);
    else
      e = launch_proj_gemm_f32(static_cast<const float*>(x), static_cast<const float*>(w->W_qkv),
                               zw, B * S, g.N, g.E, st);
    if (e != cudaSuccess) return cuda_fail(e);
    z = zw;
  }
  PreAttnArgs<T> p{};
  p.src = z;
  p.src_ld = g.N;
  p.B = B;
  p.S = S;
  p.Hq = g.Hq;
  p.Hkv = g.Hkv;
  p.d = g.d;
  p.G = g.G;
  p.K = g.K;
  p.qk_mean = g.qk_mean;
  p.value_shift = g.value_shift;
  p.channel_conv = g.channel_conv;
  p.rope_on = g.rope_on;
  p.rope_log2_base = g.rope_log2_base;
  if (g.rope_on)
    for (int i = 0; i < g.d / 2; ++i) p.rope_frac[i] = rope_turn_fraction(g.rope_log2_base, i, g.d);
  p.wq_seq = static_cast<const T*>(w->conv_q_seq);
  p.wq_chan = static_cast<const T*>(w->conv_q_chan);
  p.wk_seq = static_cast<const T*>(w->conv_k_seq);
  p.wk_chan = static_cast<const T*>(w->conv_k_chan);
  p.q_out = reinterpret_cast<T*>(ws + L.q);
  p.k_out = reinterpret_cast<T*>(ws + L.k);
  p.v_out = reinterpret_cast<T*>(ws + L.v);
  p.kv_cap = S;
  p.dev_err = dev_err;
  if ((e = launch_pre_attn<T>(p, st)) != cudaSuccess) return cuda_fail(e);
  BwdArgs<T> a{};
  a.B = B;
  a.S = S;
  a.E = g.E;
  a.N = g.N;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.d = g.d;
  a.G = g.G;
  a.K = g.K;
  a.qk_mean = g.qk_mean;
  a.value_shift = g.value_shift;
  a.causal = g.causal;
  a.rope_on = g.rope_on;
  a.channel_conv = g.channel_conv;
  for (int i = 0; i < 64; ++i) a.rope_frac[i] = p.rope_frac[i];
  a.x = static_cast<const T*>(x);
  a.W = static_cast<const T*>(w->W_qkv);
  a.wq_seq = p.wq_seq;
  a.wq_chan = p.wq_chan;
  a.wk_seq = p.wk_seq;
  a.wk_chan = p.wk_chan;
  a.z = z;
  a.q = p.q_out;
  a.k = p.k_out;
  a.v = p.v_out;
  a.dout = static_cast<const T*>(dout);
  a.dq = reinterpret_cast<float*>(ws + L.dq);
  a.dk = reinterpret_cast<float*>(ws + L.dk);
  a.dv = reinterpret_cast<float*>(ws + L.dv);
  a.lse = reinterpret_cast<float*>(ws + L.lse);
  a.dsum = reinterpret_cast<float*>(ws + L.dsum);
  a.lse_ld = L.lse_ld;
  a.o = g.dtype == CCGQA_BF16 ? reinterpret_cast<T*>(ws + L.o) : nullptr;
  a.dev_err = dev_err;
  if (g.dtype == CCGQA_BF16 && w->W_qkv) {
    a.dz_b = reinterpret_cast<T*>(ws + L.dz_b);
    a.WT = reinterpret_cast<T*>(ws + L.wt);
    a.dzT = reinterpret_cast<T*>(ws + L.dzt);
    a.xT = reinterpret_cast<T*>(ws + L.xt);
    a.ldr = L.ldr;
  }
  a.dy = reinterpret_cast<float*>(ws + L.dy);
  a.dzm = reinterpret_cast<float*>(ws + L.dzm);
  a.du = reinterpret_cast<float*>(ws + L.du);
  a.u = reinterpret_cast<float*>(ws + L.u);
  a.dz = reinterpret_cast<float*>(ws + L.dz);
  a.dx = static_cast<T*>(dx);
  if (dw) {
    float* outs[5] = {dw->W_qkv, dw->conv_q_seq, dw->conv_q_chan, dw->conv_k_seq, dw->conv_k_chan};
    for (int i = 0; i < 5; ++i) {
      const size_t n = grad_elems(g, i);
      if (outs[i] && n > 0 && (e = cudaMemsetAsync(outs[i], 0, n * 4, st)) != cudaSuccess)
        return cuda_fail(e);
    }
    a.g_W = dw->W_qkv;
    a.g_q_seq = dw->conv_q_seq;
    a.g_q_chan = dw->conv_q_chan;
    a.g_k_seq = dw->conv_k_seq;
    a.g_k_chan = dw->conv_k_chan;
  }
  e = launch_backward<T>(a, st);
  return e == cudaSuccess ? CCGQA_OK : cuda_fail(e);
}

template <typename T>
ccgqa_status run_decode(const Geo& g, const ccgqa_weights* w, const void* x_t,
                        const ccgqa_kvcache* c, void* out, uint8_t* ws, int32_t* dev_err,
                        cudaStream_t st) {
  const DecodeWs L = decode_ws(g, c->batch, c->cap, w->W_qkv != nullptr);
  DecodeArgs<T> a{};
  a.x_t = static_cast<const T*>(x_t);
  a.W = static_cast<const T*>(w->W_qkv);
  a.B = c->batch;
  a.E = g.E;
  a.N = g.N;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.d = g.d;
  a.G = g.G;
  a.K = g.K;
  a.qk_mean = g.qk_mean;
  a.value_shift = g.value_shift;
  a.channel_conv = g.channel_conv;
  a.causal = g.causal;
  a.rope_on = g.rope_on;
  a.rope_log2_base = g.rope_log2_base;
  if (g.rope_on)
    for (int i = 0; i < g.d / 2; ++i) a.rope_frac[i] = rope_turn_fraction(g.rope_log2_base, i, g.d);
  a.wq_seq = static_cast<const T*>(w->conv_q_seq);
  a.wq_chan = static_cast<const T*>(w->conv_q_chan);
  a.wk_seq = static_cast<const T*>(w->conv_k_seq);
  a.wk_chan = static_cast<const T*>(w->conv_k_chan);
  a.cache_k = static_cast<T*>(c->k);
  a.cache_v = static_cast<T*>(c->v);
  a.pages = page_map(c);
  a.len = c->len;
  a.cap = c->cap;
  a.hist_q = static_cast<T*>(c->conv_hist_q);
  a.hist_k = static_cast<T*>(c->conv_hist_k);
  a.v_prev = static_cast<T*>(c->v_prev);
  a.out = static_cast<T*>(out);
  a.proj_part = reinterpret_cast<float*>(ws + L.proj);
  a.e_splits = L.e_splits;
  a.q_ws = reinterpret_cast<float*>(ws + L.q);
  a.part_o = reinterpret_cast<float*>(ws + L.po);
  a.part_ml = reinterpret_cast<float*>(ws + L.pml);
  a.tickets = reinterpret_cast<int32_t*>(ws + L.tick);
  a.splits = L.splits;
  a.chunk = L.chunk;
  a.dev_err = dev_err;
  a.phase_events = t_capture.active ? nullptr : t_phase_events;
  const cudaError_t e = launch_decode_step<T>(a, st);
  return e == cudaSuccess ? CCGQA_OK : cuda_fail(e);
}

}  // namespace

// ----------------------------------------------------------------------------
// Scratch of ccgqa_decode_step_noalloc: a fixed array in device global memory
// that exists on every GPU that loads the library, from load until exit.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
struct ScratchSlot {
  std::once_flag once;
  void* ptr = nullptr;
  cudaError_t err = cudaSuccess;
};
ScratchSlot g_scratch_slots[kMaxDevices];

// In host code g_noalloc_scratch only names a host-side stand-in, so the device
// address is looked up once per device, with that device current.
cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  ScratchSlot& slot = g_scratch_slots[dev];
  std::call_once(slot.once, [&] {
    slot.err = cudaGetSymbolAddress(&slot.ptr, g_noalloc_scratch);
  });
  *ptr = slot.ptr;
  return slot.err;
}
}  // namespace
}  // namespace ccgqa

using namespace ccgqa;

extern "C" {

CCGQA_API size_t ccgqa_prefill_workspace_size(const ccgqa_config* cfg, int32_t batch,
                                              int32_t seq_len) {
  Geo g;
  if (derive(cfg, &g) != CCGQA_OK || batch <= 0 || seq_len <= 0) return 0;
  return prefill_ws(g, batch, seq_len).total;
}

CCGQA_API size_t ccgqa_decode_workspace_size(const ccgqa_config* cfg, int32_t batch,
                                             int32_t cap) {
  Geo g;
  if (derive(cfg, &g) != CCGQA_OK || batch <= 0 || cap <= 0) return 0;
  return decode_ws(g, batch, cap, true).total;
}

CCGQA_API ccgqa_status ccgqa_prefill(const ccgqa_config* cfg, const ccgqa_weights* w,
                                     const void* x, int32_t batch, int32_t seq_len, void* out,
                                     const ccgqa_kvcache* cache, void* workspace,
                                     size_t workspace_bytes, int32_t* dev_err, void* stream) {
  Geo g;
  ccgqa_status s = derive(cfg, &g);
  if (s != CCGQA_OK) return s;
  if ((s = check_weights(g, w)) != CCGQA_OK) return s;
  if (batch <= 0 || seq_len <= 0) return CCGQA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(batch) * seq_len > (int64_t(1) << 30)) return CCGQA_ERR_UNSUPPORTED;
  if (!x || !out || !aligned16(x) || !aligned16(out)) return CCGQA_ERR_INVALID_ARG;
  if (cache) {
    if ((s = check_cache(g, cache, true)) != CCGQA_OK) return s;
    if (cache->batch != batch) return CCGQA_ERR_INVALID_ARG;
    if (seq_len > cache->cap) return CCGQA_ERR_CAPACITY;
  }
  // the CUDA-core pre-attention kernel must fit its smallest staging layout
  // (the tensor-core one checks its own layout and otherwise falls back here)
  if (!pre_attn_fits(g.K, g.G, g.d, static_cast<int>(g.es),
                     g.K > 0 && !g.channel_conv && (w->conv_q_chan || w->conv_k_chan)))
    return CCGQA_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      workspace_bytes < prefill_ws(g, batch, seq_len).total)
    return CCGQA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!stream_allowed(st)) return CCGQA_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (g.dtype == CCGQA_BF16)
    return run_prefill<bf16>(g, w, x, batch, seq_len, out, cache, ws, dev_err, st);
  return run_prefill<float>(g, w, x, batch, seq_len, out, cache, ws, dev_err, st);
}

CCGQA_API ccgqa_status ccgqa_decode_step(const ccgqa_config* cfg, const ccgqa_weights* w,
                                         const void* x_t, const ccgqa_kvcache* cache, void* out,
                                         void* workspace, size_t workspace_bytes,
                                         int32_t* dev_err, void* stream) {
  Geo g;
  ccgqa_status s = derive(cfg, &g);
  if (s != CCGQA_OK) return s;
  if ((s = check_weights(g, w)) != CCGQA_OK) return s;
  if ((s = check_cache(g, cache, true)) != CCGQA_OK) return s;
  if (!x_t || !out || !aligned16(x_t) || !aligned16(out)) return CCGQA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      workspace_bytes < decode_ws(g, cache->batch, cache->cap, w->W_qkv != nullptr).total)
    return CCGQA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!stream_allowed(st)) return CCGQA_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (g.dtype == CCGQA_BF16) return run_decode<bf16>(g, w, x_t, cache, out, ws, dev_err, st);
  return run_decode<float>(g, w, x_t, cache, out, ws, dev_err, st);
}

CCGQA_API ccgqa_status ccgqa_decode_step_noalloc(const ccgqa_config* cfg,
                                                 const ccgqa_weights* w, const void* x_t,
                                                 const ccgqa_kvcache* cache, void* out,
                                                 int32_t* dev_err, void* stream) {
  Geo g;
  ccgqa_status s = derive(cfg, &g);
  if (s != CCGQA_OK) return s;
  if ((s = check_weights(g, w)) != CCGQA_OK) return s;
  if ((s = check_cache(g, cache, true)) != CCGQA_OK) return s;
  if (!x_t || !out || !aligned16(x_t) || !aligned16(out)) return CCGQA_ERR_INVALID_ARG;
  const DecodeWs L = decode_ws(g, cache->batch, cache->cap, w->W_qkv != nullptr);
  if (L.total > kNoAllocScratchBytes) return CCGQA_ERR_WORKSPACE;
  if (!stream_allowed(static_cast<cudaStream_t>(stream))) return CCGQA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The merge tickets must start at zero; the array keeps whatever the last
  // call left, so clear them on every call (the other regions are written
  // before they are read).
  e = cudaMemsetAsync(static_cast<uint8_t*>(scratch) + L.tick, 0,
                      static_cast<size_t>(cache->batch) * (g.Hkv + 1) * sizeof(int32_t), st);
  if (e != cudaSuccess) return cuda_fail(e);
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  if (g.dtype == CCGQA_BF16) return run_decode<bf16>(g, w, x_t, cache, out, ws, dev_err, st);
  return run_decode<float>(g, w, x_t, cache, out, ws, dev_err, st);
}

CCGQA_API size_t ccgqa_decode_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

CCGQA_API ccgqa_status ccgqa_kvcache_append(const ccgqa_config* cfg, const ccgqa_kvcache* cache,
                                            const void* k_new, const void* v_new, int32_t n_new,
                                            int32_t* dev_err, void* stream) {
  Geo g;
  ccgqa_status s = derive(cfg, &g);
  if (s != CCGQA_OK) return s;
  if ((s = check_cache(g, cache, false)) != CCGQA_OK) return s;
  if (n_new < 0) return CCGQA_ERR_INVALID_ARG;
  if (n_new > cache->cap) return CCGQA_ERR_CAPACITY;
  if (n_new == 0) return CCGQA_OK;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return CCGQA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!stream_allowed(st)) return CCGQA_ERR_INVALID_ARG;
  cudaError_t e;
  if (g.dtype == CCGQA_BF16)
    e = launch_kv_append<bf16>(static_cast<bf16*>(cache->k), static_cast<bf16*>(cache->v),
                               page_map(cache), cache->len, static_cast<const bf16*>(k_new),
                               static_cast<const bf16*>(v_new), cache->batch, g.Hkv, g.d,
                               cache->cap, n_new, dev_err, st);
  else
    e = launch_kv_append<float>(static_cast<float*>(cache->k), static_cast<float*>(cache->v),
                                page_map(cache), cache->len, static_cast<const float*>(k_new),
                                static_cast<const float*>(v_new), cache->batch, g.Hkv, g.d,
                                cache->cap, n_new, dev_err, st);
  return e == cudaSuccess ? CCGQA_OK : cuda_fail(e);
}

CCGQA_API ccgqa_status ccgqa_output_projection(const ccgqa_config* cfg, const void* W_o,
                                               const void* o, int64_t M, void* y,
                                               int32_t* dev_err, void* stream) {
  Geo g;
  ccgqa_status s = derive(cfg, &g);
  if (s != CCGQA_OK) return s;
  if (M <= 0 || !W_o || !o || !y) return CCGQA_ERR_INVALID_ARG;
  if (!aligned16(W_o) || !aligned16(o) || !aligned16(y)) return CCGQA_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 30)) return CCGQA_ERR_UNSUPPORTED;
  const int K = g.Hq * g.d, N = g.E;   // y [M, E] = o [M, Hq d] W_o^T
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!stream_allowed(st)) return CCGQA_ERR_INVALID_ARG;
  cudaError_t e;
  if (g.dtype == CCGQA_BF16) {
    if (K % 8 != 0) return CCGQA_ERR_UNSUPPORTED;   // 16-byte TMA row pitch
    e = launch_proj_gemm_bf16(static_cast<const bf16*>(o), static_cast<const bf16*>(W_o),
                              static_cast<bf16*>(y), static_cast<int>(M), N, K, dev_err, st);
  } else {
    e = launch_proj_gemm_f32(static_cast<const float*>(o), static_cast<const float*>(W_o),
                             static_cast<float*>(y), static_cast<int>(M), N, K, st);
  }
  return e == cudaSuccess ? CCGQA_OK : cuda_fail(e);
}

CCGQA_API size_t ccgqa_prefill_backward_workspace_size(const ccgqa_config* cfg, int32_t batch,
                                                       int32_t seq_len) {
  Geo g;
  if (derive(cfg, &g) != CCGQA_OK || batch <= 0 || seq_len <= 0) return 0;
  return backward_ws(g, batch, seq_len, true).total;
}

CCGQA_API ccgqa_status ccgqa_prefill_backward(const ccgqa_config* cfg, const ccgqa_weights* w,
                                              const void* x, int32_t batch, int32_t seq_len,
                                              const void* dout, void* dx,
                                              const ccgqa_weight_grads* dw, void* workspace,
                                              size_t workspace_bytes, int32_t* dev_err,
                                              void* stream) {
  Geo g;
  ccgqa_status s = derive(cfg, &g);
  if (s != CCGQA_OK) return s;
  if ((s = check_weights(g, w)) != CCGQA_OK) return s;
  if (batch <= 0 || seq_len <= 0) return CCGQA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(batch) * seq_len > (int64_t(1) << 30)) return CCGQA_ERR_UNSUPPORTED;
  if (!x || !dout || !dx || !aligned16(x) || !aligned16(dout) || !aligned16(dx))
    return CCGQA_ERR_INVALID_ARG;
  if (!pre_attn_fits(g.K, g.G, g.d, static_cast<int>(g.es),
                     g.K > 0 && !g.channel_conv && (w->conv_q_chan || w->conv_k_chan)))
    return CCGQA_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      workspace_bytes < backward_ws(g, batch, seq_len, w->W_qkv != nullptr).total)
    return CCGQA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!stream_allowed(st)) return CCGQA_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (g.dtype == CCGQA_BF16)
    return run_backward<bf16>(g, w, x, batch, seq_len, dout, dx, dw, ws, dev_err, st);
  return run_backward<float>(g, w, x, batch, seq_len, dout, dx, dw, ws, dev_err, st);
}

CCGQA_API const char* ccgqa_status_string(ccgqa_status s) {
  switch (s) {
    case CCGQA_OK: return "ok";
    case CCGQA_ERR_INVALID_ARG: return "invalid argument";
    case CCGQA_ERR_UNSUPPORTED: return "unsupported configuration";
    case CCGQA_ERR_CAPACITY: return "tokens exceed the cache capacity";
    case CCGQA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case CCGQA_ERR_CUDA: return "CUDA launch or runtime error";
  }
  return "unknown status";
}

CCGQA_API uint64_t ccgqa_launch_count(void) { return g_launches.load(); }

CCGQA_API const char* ccgqa_last_error_string(void) { return t_last_error; }

CCGQA_API void ccgqa_set_fused_projection(int32_t enable) { g_fuse_proj.store(enable ? 1 : 0); }

CCGQA_API void ccgqa_set_phase_events(void* const* events, int32_t n) {
  t_phase_events = (events != nullptr && n >= 4) ? events : nullptr;
}

// ----------------------------------------------------------------------------
// CUDA graphs of library calls: the calls a thread makes on one stream between
// ccgqa_graph_begin and ccgqa_graph_end are recorded (not run) and become one
// executable graph, replayed with all its arguments fixed.
}  // extern "C"

struct ccgqa_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  int64_t kernels = 0;     // library kernels one launch runs
};

extern "C" {

CCGQA_API ccgqa_status ccgqa_graph_begin(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the legacy default stream cannot be captured
  if (st == nullptr || st == cudaStreamLegacy || st == cudaStreamPerThread)
    return CCGQA_ERR_INVALID_ARG;
  if (t_capture.active) return CCGQA_ERR_INVALID_ARG;
  const cudaError_t e = cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal);
  if (e != cudaSuccess) return cuda_fail(e);
  t_capture.stream = st;
  t_capture.kernels = 0;
  t_capture.active = true;
  return CCGQA_OK;
}

CCGQA_API ccgqa_status ccgqa_graph_end(void* stream, ccgqa_graph** graph) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (graph == nullptr || !t_capture.active || st != t_capture.stream)
    return CCGQA_ERR_INVALID_ARG;
  *graph = nullptr;
  t_capture.active = false;
  cudaGraph_t g = nullptr;
  cudaError_t e = cudaStreamEndCapture(st, &g);
  if (e != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    return cuda_fail(e);
  }
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, g, 0);
  if (e != cudaSuccess) {
    cudaGraphDestroy(g);
    return cuda_fail(e);
  }
  ccgqa_graph* h = new (std::nothrow) ccgqa_graph;
  if (h == nullptr) {
    cudaGraphExecDestroy(exec);
    cudaGraphDestroy(g);
    return CCGQA_ERR_WORKSPACE;
  }
  h->graph = g;
  h->exec = exec;
  h->kernels = t_capture.kernels;
  *graph = h;
  return CCGQA_OK;
}

CCGQA_API ccgqa_status ccgqa_graph_launch(const ccgqa_graph* graph, void* stream) {
  if (graph == nullptr) return CCGQA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!stream_allowed(st)) return CCGQA_ERR_INVALID_ARG;
  const cudaError_t e = cudaGraphLaunch(graph->exec, st);
  if (e != cudaSuccess) return cuda_fail(e);
  count_launches(static_cast<int>(graph->kernels));
  return CCGQA_OK;
}

CCGQA_API int64_t ccgqa_graph_kernel_count(const ccgqa_graph* graph) {
  return graph == nullptr ? -1 : graph->kernels;
}

CCGQA_API ccgqa_status ccgqa_graph_destroy(ccgqa_graph* graph) {
  if (graph == nullptr) return CCGQA_OK;
  cudaError_t e = cudaGraphExecDestroy(graph->exec);
  const cudaError_t e2 = cudaGraphDestroy(graph->graph);
  delete graph;
  if (e == cudaSuccess) e = e2;
  return e == cudaSuccess ? CCGQA_OK : cuda_fail(e);
}

}  // extern "C"
