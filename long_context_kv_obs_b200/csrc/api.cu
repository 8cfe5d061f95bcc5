// C ABI of libkvc: argument validation, workspace planning and the launch
// sequence of every call.  All work is enqueued on the caller's stream; no
// call allocates, frees or synchronises (except kvc_check_status, which is a
// host query by definition).
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <mutex>

#include "kernels.cuh"

namespace kvc {

// ----------------------------------------------------------------- state
__device__ unsigned g_status_word;

static thread_local char g_err[512];
static std::atomic<uint64_t> g_launches{0};

void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static kvc_status fail(kvc_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

kvc_status report(kvc_status s, const char* msg) { return fail(s, "%s", msg); }

static kvc_status cuda_fail(cudaError_t e, const char* where) {
  return fail(KVC_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

unsigned* status_ptr() {
  static unsigned* cache[64] = {nullptr};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return nullptr;
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) == cudaSuccess) cache[dev] = (unsigned*)p;
  }
  return cache[dev];
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = v > 0 ? v : 148;
  }
  return cache[dev];
}

// ----------------------------------------------------------------- helpers
static inline size_t esize(kvc_dtype t) { return t == KVC_BF16 ? 2 : 4; }
static inline bool dtype_ok(kvc_dtype t) { return t == KVC_F32 || t == KVC_BF16; }
static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base((char*)b) {}
  template <typename T> T* take(size_t count) {
    T* p = base ? (T*)(base + off) : nullptr;
    off += align256(count * sizeof(T));
    return p;
  }
};

static kvc_status check_model(const kvc_model* m) {
  if (!m) return fail(KVC_ERR_ARG, "model is NULL");
  if (m->n_layers <= 0 || m->n_q_heads <= 0 || m->n_kv_heads <= 0)
    return fail(KVC_ERR_ARG, "model sizes must be positive");
  if (m->n_q_heads % m->n_kv_heads) return fail(KVC_ERR_ARG, "n_q_heads must be a multiple of n_kv_heads");
  if (m->head_dim != 64 && m->head_dim != 128)
    return fail(KVC_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", m->head_dim);
  return KVC_OK;
}

static kvc_status check_kv(const kvc_kv& t, const char* name, int d, bool need) {
  if (!t.ptr) return need ? fail(KVC_ERR_ARG, "%s.ptr is NULL", name) : KVC_OK;
  if (!dtype_ok(t.dtype)) return fail(KVC_ERR_ARG, "%s.dtype invalid", name);
  const size_t es = esize(t.dtype);
  if ((uintptr_t)t.ptr % 16) return fail(KVC_ERR_ARG, "%s.ptr not 16-byte aligned", name);
  if ((t.s_tok * es) % 16 || (t.s_head * es) % 16 || (t.s_layer * es) % 16 || (t.s_batch * es) % 16)
    return fail(KVC_ERR_ARG, "%s strides must be multiples of 16 bytes", name);
  if (t.s_tok < d) return fail(KVC_ERR_ARG, "%s.s_tok smaller than head_dim", name);
  return KVC_OK;
}

static inline int64_t b2(const kvc_kv& t, int64_t s) { return s * (int64_t)esize(t.dtype); }

// ----------------------------------------------------------------- score
struct ScorePlan {
  bool compute_H, compute_D, infokv, overlap;
  int window_sms;
  float* Atmp;
  int R, nchunk, chunk;
  size_t bytes;
  float *H, *D, *estats, *part, *rowst, *vnorm;
  double* estats_part;
  float* ecand;      // candidates of the split-row entropy (few rows)
  float2* fpart;
  float* frowc;
  int* fsync;
};

static const int WIN_CHUNK = 1024;     // keys per item of the two-launch window path: 8 tiles keep the CTAs level
// The window pass beside the signal scans, by default: a quarter of the SMs, for rows of up
// to 32768 tokens.  Measured: at the 3B 16k shape the score stage takes 1.50 ms so against
// 1.98 ms in sequence; at the 8B 64k shape no split gained (the window pass on fewer SMs takes
// about as long as the scans it hides behind), so longer rows run the stages in sequence.
static const int WINDOW_SMS_NUM = 1, WINDOW_SMS_DEN = 4;
static const int OVERLAP_MAX_N = 32768;

// The library's second stream and its fork / join events, one set per device, created
// on first use with that device current and kept until exit.
struct AuxStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

static kvc_status aux_stream(AuxStream** out) {
  static std::mutex mu;
  static AuxStream cache[64];
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(KVC_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(mu);
  AuxStream& a = cache[dev];
  if (!a.s) {
    AuxStream n;
    if ((e = cudaStreamCreateWithFlags(&n.s, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "creating the library stream");
    if ((e = cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming)) != cudaSuccess)
      return cuda_fail(e, "creating the library events");
    a = n;
  }
  *out = &a;
  return KVC_OK;
}

static ScorePlan plan_score(const kvc_model* m, const kvc_score_args* a, void* ws) {
  ScorePlan p{};
  const int L = m->n_layers, Hkv = m->n_kv_heads, G = m->n_q_heads / m->n_kv_heads;
  p.infokv = a->mode == KVC_SCORE_INFOKV;
  p.compute_H = p.infokv && a->logits;
  p.compute_D = p.infokv && a->hidden;
  p.R = G * a->W;
  // the window pass beside the signal scans (see kvc_score_args.window_sms)
  p.overlap = p.infokv && a->S && (p.compute_H || p.compute_D) && a->window_sms >= 0 &&
              a->K.dtype == KVC_BF16 && m->head_dim == 128 && G * a->W <= 128 && !a->qpos;
  if (p.overlap && a->window_sms == 0 && a->n > OVERLAP_MAX_N) p.overlap = false;
  if (p.overlap) {
    const int sms = num_sms();
    int w = a->window_sms > 0 ? a->window_sms : (sms * WINDOW_SMS_NUM) / WINDOW_SMS_DEN;
    if (w < 8) w = 8;
    if (w > sms - 8) w = sms - 8;
    p.window_sms = w;
    p.overlap = w >= 8;
  }
  p.chunk = WIN_CHUNK;
  p.nchunk = (a->n + WIN_CHUNK - 1) / WIN_CHUNK;
  Carver c(ws);
  p.H = (p.compute_H && !a->H_out) ? c.take<float>((size_t)a->n) : nullptr;
  p.D = (p.compute_D && !a->D_out) ? c.take<float>((size_t)L * a->n) : nullptr;
  const size_t ecb = p.compute_H ? entropy_split_ws(a->n, a->vocab, a->logits_dtype, a->topk) : 0;
  p.ecand = ecb ? c.take<float>(ecb / sizeof(float)) : nullptr;
  p.estats = (p.infokv && a->S) ? c.take<float>((size_t)L * Hkv * 3) : nullptr;
  p.estats_part = (p.infokv && a->S) ? c.take<double>(estats_ws(a->n, L, Hkv) / sizeof(double)) : nullptr;
  if (a->S) {
    p.part = c.take<float>((size_t)L * Hkv * p.nchunk * p.R * 2);
    p.rowst = c.take<float>((size_t)L * Hkv * p.R * 2);
    if (a->mode == KVC_SCORE_VATP) p.vnorm = c.take<float>((size_t)L * Hkv * a->n);
    const size_t fchunks = (size_t)(a->n + WIN_FUSED_CHUNK - 1) / WIN_FUSED_CHUNK;
    const size_t fgroups = (fchunks + WIN_FUSED_GROUP - 1) / WIN_FUSED_GROUP;
    p.fpart = c.take<float2>((size_t)L * Hkv * (fchunks + fgroups) * 128);
    p.frowc = c.take<float>((size_t)L * Hkv * 128);
    p.fsync = c.take<int>((size_t)L * Hkv * (2 + fgroups));
  }
  if (p.overlap && !a->A) p.Atmp = c.take<float>((size_t)L * Hkv * a->n);
  p.bytes = c.off;
  return p;
}

static kvc_status check_score(const kvc_model* m, const kvc_score_args* a) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  const int d = m->head_dim, G = m->n_q_heads / m->n_kv_heads;
  if (a->mode < KVC_SCORE_INFOKV || a->mode > KVC_SCORE_ATTN) return fail(KVC_ERR_ARG, "mode invalid");
  if (a->n < 1) return fail(KVC_ERR_ARG, "n must be >= 1");
  if (!a->S) {
    // signals only: H from logits and / or D from hidden, no window attention
    if (a->mode != KVC_SCORE_INFOKV || a->A) return fail(KVC_ERR_ARG, "S is NULL");
    if (!a->logits && !a->hidden) return fail(KVC_ERR_ARG, "signals-only call without logits or hidden");
    if ((a->logits && !a->H_out) || (a->hidden && !a->D_out))
      return fail(KVC_ERR_ARG, "signals-only call needs H_out / D_out");
  } else {
    if (a->W < 1 || a->W > a->n) return fail(KVC_ERR_ARG, "W must be in [1, n]");
    if (G * a->W > 256) return fail(KVC_ERR_UNSUPPORTED, "G*W = %d window rows (max 256)", G * a->W);
    if (!a->Qw) return fail(KVC_ERR_ARG, "Qw is NULL");
    if ((s = check_kv(a->K, "K", d, true))) return s;
    if (a->mode == KVC_SCORE_VATP) {
      if ((s = check_kv(a->V, "V", d, true))) return s;
    }
    if (window_ffma_smem_max(G * a->W, d) > 227 * 1024) return fail(KVC_ERR_UNSUPPORTED, "window too large");
  }
  if (a->mode == KVC_SCORE_INFOKV) {
    if (!(a->alpha >= 0.f && a->alpha <= 1.f)) return fail(KVC_ERR_ARG, "alpha must be in [0, 1]");
    if (a->logits) {
      if (!dtype_ok(a->logits_dtype)) return fail(KVC_ERR_ARG, "logits_dtype invalid");
      if (a->vocab < 1 || a->logits_row_stride < a->vocab)
        return fail(KVC_ERR_ARG, "vocab / logits_row_stride invalid");
      if (a->topk < 1 || a->topk > 1024) return fail(KVC_ERR_ARG, "topk must be in [1, 1024]");
    } else if (!a->H_in && a->S) {
      return fail(KVC_ERR_ARG, "InfoKV mode needs logits or H_in");
    }
    if (a->hidden) {
      if (!dtype_ok(a->hidden_dtype)) return fail(KVC_ERR_ARG, "hidden_dtype invalid");
      const int per = a->hidden_dtype == KVC_BF16 ? 256 : 128;
      if (a->hidden_size < per || a->hidden_size % per || a->hidden_size > 16 * per)
        return fail(KVC_ERR_UNSUPPORTED, "hidden_size %d must be a multiple of %d up to %d",
                    a->hidden_size, per, 16 * per);
      if ((uintptr_t)a->hidden % 16) return fail(KVC_ERR_ARG, "hidden not 16-byte aligned");
    } else if (!a->D_in && a->S) {
      return fail(KVC_ERR_ARG, "InfoKV mode needs hidden or D_in");
    }
  }
  return KVC_OK;
}

// qlpb: layers per row of a->qpos (0: one row of W positions for every layer).
// qlpb: layers per row of the window-query positions (0: one row for every layer); wlse:
// the window rows' log-sum-exp recorded by their decode steps (kvc_recompress's win_lse)
static kvc_status run_score(const kvc_model* m, const kvc_score_args* a, void* ws, size_t ws_bytes,
                            cudaStream_t st, int qlpb = 0, const float* wlse = nullptr) {
  kvc_status s = check_score(m, a);
  if (s) return s;
  ScorePlan pl = plan_score(m, a, nullptr);
  if (pl.bytes && (!ws || ws_bytes < pl.bytes))
    return fail(KVC_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, pl.bytes);
  pl = plan_score(m, a, ws);
  const int L = m->n_layers, Hkv = m->n_kv_heads, G = m->n_q_heads / m->n_kv_heads, d = m->head_dim;
  cudaError_t e;
  WinParams p{};
  p.L = L; p.Hq = m->n_q_heads; p.Hkv = Hkv; p.G = G; p.d = d; p.n = a->n; p.W = a->W; p.R = G * a->W;
  p.Qw = a->Qw;
  p.K = a->K.ptr; p.Ksl = a->K.s_layer; p.Ksh = a->K.s_head; p.Kst = a->K.s_tok;
  p.V = a->V.ptr; p.Vsl = a->V.s_layer; p.Vsh = a->V.s_head; p.Vst = a->V.s_tok;
  p.kpos = a->kpos; p.kpsl = a->kpos_s_layer; p.kpsh = a->kpos_s_head;
  p.qpos = a->qpos;
  p.qlpb = a->qpos ? qlpb : 0;
  p.wlse = wlse;
  p.scale = a->scale > 0.f ? a->scale : 1.f / sqrtf((float)d);
  p.mode = a->mode; p.alpha = a->alpha;
  p.A = a->A; p.S = a->S;
  p.part = pl.part; p.rowst = pl.rowst; p.vnorm = pl.vnorm; p.nchunk = pl.nchunk; p.chunk = pl.chunk;
  p.fpart = pl.fpart; p.frowc = pl.frowc; p.fsync = pl.fsync; p.fchunk = WIN_FUSED_CHUNK;
  p.flag_wait_ns = a->wait_limit_ns;
  // InfoKV with the signals computed here: the window attention (A only) runs on the
  // library's stream beside the entropy and representation scans, which keep the
  // other SMs; S is formed after both (kvc_score_args.window_sms)
  AuxStream* aux = nullptr;
  bool overlap = pl.overlap && window_fused_supported(p, a->K.dtype);
  const float* Aw = a->A ? a->A : pl.Atmp;
  if (overlap) {
    if ((s = aux_stream(&aux))) return s;
    WinParams pa = p;
    pa.S = nullptr;
    pa.A = const_cast<float*>(Aw);
    if ((e = cudaEventRecord(aux->fork, st)) || (e = cudaStreamWaitEvent(aux->s, aux->fork, 0)))
      return cuda_fail(e, "fork");
    e = launch_window_fused(pa, aux->s, pl.window_sms);
    const cudaError_t ej = cudaEventRecord(aux->join, aux->s);
    if (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorNotSupported) {
      // the single launch cannot have all its CTAs resident: the stages run in sequence
      cudaGetLastError();
      cudaStreamWaitEvent(st, aux->join, 0);
      overlap = false;
    } else if (e) {
      cudaStreamWaitEvent(st, aux->join, 0);
      return cuda_fail(e, "window");
    } else if (ej) {
      return cuda_fail(ej, "join");
    }
  }
  const int sig_sms = overlap ? num_sms() - pl.window_sms : 0;
  // every return below, once the window pass is on the library stream, first makes the
  // caller's stream wait for it
  auto joined = [&](kvc_status r) {
    if (overlap) cudaStreamWaitEvent(st, aux->join, 0);
    return r;
  };
  const float* H = nullptr;
  int64_t Hsl = 0, Hsh = 0;
  const float* D = nullptr;
  int64_t Dsl = 0, Dsh = 0;
  if (pl.infokv) {
    if (pl.compute_H) {
      float* Hw = a->H_out ? a->H_out : pl.H;
      const size_t es = a->logits_dtype == KVC_BF16 ? 2 : 4;
      if (pl.ecand && (uintptr_t)a->logits % 16 == 0 && (a->logits_row_stride * es) % 16 == 0)
        e = launch_entropy_split(a->logits, a->logits_dtype, a->n, a->vocab, a->logits_row_stride, a->topk,
                                 pl.ecand, Hw, st);
      else
        e = launch_entropy(a->logits, a->logits_dtype, a->n, a->vocab, a->logits_row_stride, a->topk, Hw, st,
                           sig_sms);
      if (e) return joined(cuda_fail(e, "entropy"));
      H = Hw;
    } else {
      H = a->H_in; Hsl = a->H_s_layer; Hsh = a->H_s_head;
    }
    if (pl.compute_D) {
      float* Dw = a->D_out ? a->D_out : pl.D;
      e = launch_repr(a->hidden, a->hidden_dtype, L, a->n, a->hidden_size, a->tau, Dw, st, sig_sms);
      if (e) return joined(cuda_fail(e, "repr"));
      D = Dw; Dsl = a->n;
    } else {
      D = a->D_in; Dsl = a->D_s_layer; Dsh = a->D_s_head;
    }
    if (!a->S) return KVC_OK;   // signals only
    e = launch_estats(H, Hsl, Hsh, D, Dsl, Dsh, a->n, L, Hkv, pl.estats, a->Ebar, pl.estats_part, st);
    if (e) return joined(cuda_fail(e, "estats"));
  }
  if (overlap) {
    if ((e = cudaStreamWaitEvent(st, aux->join, 0))) return cuda_fail(e, "join");
    e = launch_combine(Aw, H, Hsl, Hsh, D, Dsl, Dsh, pl.estats, a->n, L, Hkv, a->alpha, a->S, st);
    if (e) return cuda_fail(e, "combine");
    return KVC_OK;
  }
  p.H = H; p.Hsl = Hsl; p.Hsh = Hsh; p.D = D; p.Dsl = Dsl; p.Dsh = Dsh;
  p.estats = pl.estats;
  if (window_fused_supported(p, a->K.dtype)) {
    e = launch_window_fused(p, st);
    if (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorNotSupported) {
      // every CTA of the single-launch kernel must be resident: two launches instead
      cudaGetLastError();
      e = launch_window_tc(p, st);
    }
  } else if (window_tc_supported(p, a->K.dtype)) {
    e = launch_window_tc(p, st);
  } else {
    e = launch_window_ffma(p, a->K.dtype, st);
  }
  if (e) return cuda_fail(e, "window");
  return KVC_OK;
}

// ----------------------------------------------------------------- select
static kvc_status check_select(const kvc_model* m, const kvc_select_args* a) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  if (a->n < 1) return fail(KVC_ERR_ARG, "n must be >= 1");
  if (a->w < 0) return fail(KVC_ERR_ARG, "w must be >= 0");
  if (!a->S || !a->k_out || !a->idx) return fail(KVC_ERR_ARG, "S, k_out and idx are required");
  if (a->sel_mode != KVC_SEL_PER_KV_HEAD && a->sel_mode != KVC_SEL_GQA_UNION)
    return fail(KVC_ERR_ARG, "sel_mode invalid");
  if (a->k_cap < 1) return fail(KVC_ERR_ARG, "k_cap must be >= 1");
  const int L = m->n_layers, lo = a->w < a->n ? a->w : a->n;
  switch (a->budget_mode) {
    case KVC_BUDGET_UNIFORM: {
      if (!(a->rho >= 0.0 && a->rho <= 1.0)) return fail(KVC_ERR_ARG, "rho must be in [0, 1]");
      long long k = (long long)floor(a->rho * a->n);
      if (k < lo) k = lo;
      if (k > a->k_cap) return fail(KVC_ERR_ARG, "k_cap %d < budget %lld", a->k_cap, k);
      break;
    }
    case KVC_BUDGET_EXPLICIT:
      if (!a->k_in) return fail(KVC_ERR_ARG, "k_in is NULL");
      break;
    case KVC_BUDGET_ADAPTIVE:
      if (!a->Ebar) return fail(KVC_ERR_ARG, "Ebar is NULL");
      if (a->B_total < (long long)L * lo || a->B_total > (long long)L * a->n)
        return fail(KVC_ERR_ARG, "B_total outside [L*min(w,n), L*n]");
      break;
    default:
      return fail(KVC_ERR_ARG, "budget_mode invalid");
  }
  return KVC_OK;
}

static size_t select_ws(const kvc_model* m, const kvc_select_args* a) {
  const int rows = a->sel_mode == KVC_SEL_GQA_UNION ? m->n_layers : m->n_layers * m->n_kv_heads;
  return align256((size_t)rows * a->n * sizeof(uint32_t));
}

static kvc_status run_select(const kvc_model* m, const kvc_select_args* a, void* ws, size_t ws_bytes,
                             cudaStream_t st) {
  kvc_status s = check_select(m, a);
  if (s) return s;
  const size_t need = select_ws(m, a);
  if (!ws || ws_bytes < need) return fail(KVC_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  cudaError_t e = launch_budget(a->budget_mode, m->n_layers, a->n, a->w, a->rho, a->k_in, a->B_total,
                                a->Ebar, a->k_out, st);
  if (e) return cuda_fail(e, "budget");
  e = launch_select(a->S, a->S_s_layer, a->S_s_head, m->n_layers, m->n_kv_heads, a->n, a->w,
                    a->sel_mode == KVC_SEL_GQA_UNION, a->k_out, a->idx, a->k_cap, (uint32_t*)ws, st);
  if (e) return cuda_fail(e, "select");
  return KVC_OK;
}

// ----------------------------------------------------------------- compact
static kvc_status compact_impl(const kvc_model* m, const kvc_compact_args* a, int64_t dside_row,
                               cudaStream_t st) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  const int d = m->head_dim;
  if (!a->idx || !a->k) return fail(KVC_ERR_ARG, "idx and k are required");
  if (a->n < 1 || a->k_cap < 1) return fail(KVC_ERR_ARG, "n and k_cap must be >= 1");
  if (!a->src_K.ptr && !a->src_V.ptr) return fail(KVC_ERR_ARG, "nothing to compact");
  if ((!a->src_K.ptr) != (!a->dst_K.ptr) || (!a->src_V.ptr) != (!a->dst_V.ptr))
    return fail(KVC_ERR_ARG, "src/dst pointers must be given in pairs");
  if ((s = check_kv(a->src_K, "src_K", d, false)) || (s = check_kv(a->dst_K, "dst_K", d, false)) ||
      (s = check_kv(a->src_V, "src_V", d, false)) || (s = check_kv(a->dst_V, "dst_V", d, false)))
    return s;
  const kvc_kv& ref = a->src_K.ptr ? a->src_K : a->src_V;
  if ((a->src_K.ptr && (a->src_K.dtype != ref.dtype || a->dst_K.dtype != ref.dtype)) ||
      (a->src_V.ptr && (a->src_V.dtype != ref.dtype || a->dst_V.dtype != ref.dtype)))
    return fail(KVC_ERR_ARG, "K/V src and dst must share one dtype");
  if ((a->src_K.ptr && a->src_K.ptr == a->dst_K.ptr) || (a->src_V.ptr && a->src_V.ptr == a->dst_V.ptr))
    return fail(KVC_ERR_ARG, "src and dst must not alias");
  if ((!a->src_H) != (!a->dst_H) || (!a->src_D) != (!a->dst_D) || (!a->src_U) != (!a->dst_U))
    return fail(KVC_ERR_ARG, "side arrays H, D and U go with both a source and a destination");
  CompactParams p{};
  p.L = m->n_layers; p.Hkv = m->n_kv_heads; p.n = a->n; p.k_cap = a->k_cap;
  p.vr = (int)(d * esize(ref.dtype) / 16);
  if (a->src_K.ptr) {
    p.sK = (const char*)a->src_K.ptr; p.sKl = b2(a->src_K, a->src_K.s_layer); p.sKh = b2(a->src_K, a->src_K.s_head); p.sKt = b2(a->src_K, a->src_K.s_tok);
    p.dK = (char*)a->dst_K.ptr; p.dKl = b2(a->dst_K, a->dst_K.s_layer); p.dKh = b2(a->dst_K, a->dst_K.s_head); p.dKt = b2(a->dst_K, a->dst_K.s_tok);
  }
  if (a->src_V.ptr) {
    p.sV = (const char*)a->src_V.ptr; p.sVl = b2(a->src_V, a->src_V.s_layer); p.sVh = b2(a->src_V, a->src_V.s_head); p.sVt = b2(a->src_V, a->src_V.s_tok);
    p.dV = (char*)a->dst_V.ptr; p.dVl = b2(a->dst_V, a->dst_V.s_layer); p.dVh = b2(a->dst_V, a->dst_V.s_head); p.dVt = b2(a->dst_V, a->dst_V.s_tok);
  }
  p.idx = a->idx; p.k = a->k;
  p.spos = a->src_pos; p.psl = a->pos_s_layer; p.psh = a->pos_s_head; p.dpos = a->dst_pos;
  p.sH = a->src_H; p.Hsl = a->H_s_layer; p.Hsh = a->H_s_head; p.dH = a->dst_H;
  p.sD = a->src_D; p.Dsl = a->D_s_layer; p.Dsh = a->D_s_head; p.dD = a->dst_D;
  p.sU = a->src_U; p.Usl = a->U_s_layer; p.Ush = a->U_s_head; p.dU = a->dst_U;
  p.dside_row = dside_row > 0 ? dside_row : a->k_cap;
  p.status = status_ptr();
  cudaError_t e = launch_compact(p, st);
  if (e) return cuda_fail(e, "compact");
  return KVC_OK;
}

static kvc_status run_compact(const kvc_model* m, const kvc_compact_args* a, cudaStream_t st) {
  return compact_impl(m, a, 0, st);
}

// ----------------------------------------------------------------- RoPE re-positioning
static kvc_status run_rope(const kvc_model* m, const kvc_rope_args* a, cudaStream_t st) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  const int d = m->head_dim;
  if ((s = check_kv(a->K, "K", d, true))) return s;
  const bool in_place = !a->K_dst.ptr || a->K_dst.ptr == a->K.ptr;
  const kvc_kv& dst = in_place ? a->K : a->K_dst;
  if (!in_place) {
    if ((s = check_kv(a->K_dst, "K_dst", d, true))) return s;
    if (a->K_dst.dtype != a->K.dtype) return fail(KVC_ERR_ARG, "K and K_dst must share one dtype");
  }
  if (!a->pos || !a->k) return fail(KVC_ERR_ARG, "pos and k are required");
  if (a->k_cap < 1) return fail(KVC_ERR_ARG, "k_cap must be >= 1");
  if (a->pos_s_row < a->k_cap) return fail(KVC_ERR_ARG, "pos_s_row smaller than k_cap");
  if (!(a->base > 1.0) || !std::isfinite(a->base)) return fail(KVC_ERR_ARG, "base must be finite and > 1");
  if (a->new0 < INT32_MIN || a->new0 + a->k_cap - 1 > INT32_MAX)
    return fail(KVC_ERR_ARG, "new0 .. new0 + k_cap - 1 must fit in int32");
  RopeParams p{};
  p.L = m->n_layers; p.Hkv = m->n_kv_heads; p.d = d; p.k_cap = a->k_cap;
  p.bf16 = a->K.dtype == KVC_BF16;
  p.src = (const char*)a->K.ptr; p.sl = b2(a->K, a->K.s_layer); p.sh = b2(a->K, a->K.s_head); p.st = b2(a->K, a->K.s_tok);
  p.dst = (char*)dst.ptr; p.dl = b2(dst, dst.s_layer); p.dh = b2(dst, dst.s_head); p.dt = b2(dst, dst.s_tok);
  p.pos = a->pos; p.pos_row = a->pos_s_row; p.pos_dst = a->pos_dst;
  p.k = a->k;
  p.new0 = a->new0;
  for (int i = 0; i < d / 2; ++i) p.theta[i] = std::pow(a->base, -2.0 * i / d);
  p.status = status_ptr();
  cudaError_t e = launch_rope(p, st);
  if (e) return cuda_fail(e, "rope_reposition");
  return KVC_OK;
}

// ----------------------------------------------------------------- merge
static kvc_status run_merge(const kvc_model* m, const kvc_merge_args* a, cudaStream_t st) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  const int d = m->head_dim;
  if (a->n < 1 || a->k_cap < 1) return fail(KVC_ERR_ARG, "n and k_cap must be >= 1");
  if (a->bucket < 1 || a->bucket > 4096) return fail(KVC_ERR_UNSUPPORTED, "bucket must be in [1, 4096]");
  if (!a->A || !a->idx || !a->k || !a->R) return fail(KVC_ERR_ARG, "A, idx, k and R are required");
  if ((s = check_kv(a->V, "V", d, true)) || (s = check_kv(a->dst_V, "dst_V", d, true))) return s;
  if (a->V.ptr == a->dst_V.ptr) return fail(KVC_ERR_ARG, "V and dst_V must not alias");
  MergeParams p{};
  p.L = m->n_layers; p.Hkv = m->n_kv_heads; p.n = a->n; p.d = d; p.bucket = a->bucket;
  p.nbuckets = (a->n + a->bucket - 1) / a->bucket; p.k_cap = a->k_cap;
  p.V = a->V.ptr; p.Vsl = a->V.s_layer; p.Vsh = a->V.s_head; p.Vst = a->V.s_tok; p.bf16 = a->V.dtype == KVC_BF16;
  p.A = a->A; p.Asl = a->A_s_layer; p.Ash = a->A_s_head;
  p.idx = a->idx; p.k = a->k;
  p.dV = a->dst_V.ptr; p.dVl = a->dst_V.s_layer; p.dVh = a->dst_V.s_head; p.dVt = a->dst_V.s_tok;
  p.dbf16 = a->dst_V.dtype == KVC_BF16;
  p.R = a->R; p.dVf = a->dst_V_f32; p.status = status_ptr();
  cudaError_t e = launch_merge(p, st);
  if (e) return cuda_fail(e, "merge");
  return KVC_OK;
}

// ----------------------------------------------------------------- decode
struct DecodePlan {
  int nsplit, split_len;
  size_t bytes;
};

static DecodePlan plan_decode_dims(const kvc_model* m, int batch, int max_len, bool probe,
                                   bool persistent = false) {
  DecodePlan pl{};
  const int rows = batch * m->n_layers * m->n_kv_heads;
  const int G = m->n_q_heads / m->n_kv_heads;
  // one CTA per split: enough CTAs for several waves on a full B200, splits of at least
  // 256 keys; persistent kernel (two CTAs per SM): about 12 items per CTA, so the
  // static round-robin split of items leaves little imbalance, items of at least 128 keys
  const int target = persistent ? 148 * 2 * 12 : 148 * 8;
  int ns = (target + rows - 1) / rows;
  const int maxns = (max_len + (persistent ? 127 : 255)) / (persistent ? 128 : 256);
  if (ns > maxns) ns = maxns;
  if (ns < 1) ns = 1;
  pl.split_len = (max_len + ns - 1) / ns;
  if (pl.split_len < 1) pl.split_len = 1;
  pl.nsplit = (max_len + pl.split_len - 1) / pl.split_len;
  if (pl.nsplit < 1) pl.nsplit = 1;
  pl.bytes = align256((size_t)rows * pl.nsplit * G * decode_rec_len(probe, m->head_dim) * sizeof(float));
  return pl;
}

static size_t decode_ws(const kvc_model* m, const kvc_decode_args* a) {
  size_t b = plan_decode_dims(m, a->batch, a->max_len, false).bytes;
  const size_t bp = plan_decode_dims(m, a->batch, a->max_len, false, true).bytes;
  if (bp > b) b = bp;
  if (a->K_full.ptr) {
    size_t b2v = plan_decode_dims(m, a->batch, a->max_len_full, true).bytes;
    if (b2v > b) b = b2v;
    b2v = plan_decode_dims(m, a->batch, a->max_len_full, true, true).bytes;
    if (b2v > b) b = b2v;
  }
  return b;
}

static kvc_status check_decode(const kvc_model* m, const kvc_decode_args* a) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  const int d = m->head_dim, G = m->n_q_heads / m->n_kv_heads;
  if (G > 8) return fail(KVC_ERR_UNSUPPORTED, "more than 8 query heads per KV head");
  if (a->batch < 1) return fail(KVC_ERR_ARG, "batch must be >= 1");
  if (!a->q || !a->len || !a->o) return fail(KVC_ERR_ARG, "q, len and o are required");
  if (!dtype_ok(a->q_dtype)) return fail(KVC_ERR_ARG, "q_dtype invalid");
  if (a->max_len < 1) return fail(KVC_ERR_ARG, "max_len must be >= 1");
  if (a->lse_stride < 0) return fail(KVC_ERR_ARG, "lse_stride must be >= 0");
  if ((s = check_kv(a->K, "K", d, true)) || (s = check_kv(a->V, "V", d, true))) return s;
  if (a->K.dtype != a->V.dtype) return fail(KVC_ERR_ARG, "K and V dtypes differ");
  if (a->K_full.ptr) {
    if ((s = check_kv(a->K_full, "K_full", d, true)) || (s = check_kv(a->V_full, "V_full", d, true))) return s;
    if (a->K_full.dtype != a->V_full.dtype) return fail(KVC_ERR_ARG, "K_full and V_full dtypes differ");
    if (!a->len_full || !a->kept_bits) return fail(KVC_ERR_ARG, "probe needs len_full and kept_bits");
    if (a->max_len_full < 1) return fail(KVC_ERR_ARG, "max_len_full must be >= 1");
  }
  return KVC_OK;
}

static kvc_status run_decode(const kvc_model* m, const kvc_decode_args* a, void* ws, size_t ws_bytes,
                             cudaStream_t st) {
  kvc_status s = check_decode(m, a);
  if (s) return s;
  const size_t need = decode_ws(m, a);
  if (!ws || ws_bytes < need) return fail(KVC_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  const int G = m->n_q_heads / m->n_kv_heads, d = m->head_dim;
  const float scale = a->scale > 0.f ? a->scale : 1.f / sqrtf((float)d);
  const int rows = a->batch * m->n_layers * m->n_kv_heads;
  for (int pass = 0; pass < (a->K_full.ptr ? 2 : 1); ++pass) {
    const bool probe = pass == 1;
    const kvc_kv& K = probe ? a->K_full : a->K;
    const kvc_kv& V = probe ? a->V_full : a->V;
    DecodeParams p{};
    p.B = a->batch; p.L = m->n_layers; p.Hq = m->n_q_heads; p.Hkv = m->n_kv_heads; p.G = G; p.d = d;
    p.q = a->q; p.qbf16 = a->q_dtype == KVC_BF16;
    p.K = (const char*)K.ptr; p.Ksb = b2(K, K.s_batch); p.Ksl = b2(K, K.s_layer); p.Ksh = b2(K, K.s_head); p.Kst = b2(K, K.s_tok);
    p.V = (const char*)V.ptr; p.Vsb = b2(V, V.s_batch); p.Vsl = b2(V, V.s_layer); p.Vsh = b2(V, V.s_head); p.Vst = b2(V, V.s_tok);
    p.len = probe ? a->len_full : a->len;
    p.max_len = probe ? a->max_len_full : a->max_len;
    p.status = status_ptr();
    p.R = probe ? nullptr : a->R; p.Rsb = a->R_s_batch; p.Rsl = a->R_s_layer; p.Rsh = a->R_s_head;
    p.alpha_c = a->alpha_c;
    p.qscale = scale * 1.4426950408889634f;
    p.bits = a->kept_bits; p.bsb = a->bits_s_batch; p.bsl = a->bits_s_layer; p.bsh = a->bits_s_head;
    const bool persistent = decode_mma_supported(p, K.dtype == KVC_BF16, probe) ||
                            decode_tma_supported(p, K.dtype == KVC_BF16, probe);
    DecodePlan pl = plan_decode_dims(m, a->batch, probe ? a->max_len_full : a->max_len, probe, persistent);
    p.nsplit = pl.nsplit; p.split_len = pl.split_len;
    p.part = (float*)ws;
    CombineParams c{};
    c.rows = rows; c.nsplit = pl.nsplit; c.G = G; c.d = d; c.Hkv = m->n_kv_heads; c.L = m->n_layers;
    c.Hq = m->n_q_heads; c.part = (float*)ws;
    if (!probe) {
      c.o = a->o; c.lse = a->lse; c.lse_stride = a->lse_stride > 0 ? a->lse_stride : 1;
    } else {
      c.delta = a->delta; c.vmax = a->vmax; c.err = a->err; c.bound = a->bound;
      c.o_full = a->o_full; c.o_kept = a->o_kept;
    }
    cudaError_t e = launch_decode(p, K.dtype == KVC_BF16, probe, c, st);
    if (e) return cuda_fail(e, "decode");
  }
  return KVC_OK;
}

// ----------------------------------------------------------------- recompress
static const int RECAS_MAX_N = 16384;   // rows the controller sorts in shared memory
static bool recompress_batchable(const kvc_model* m, const kvc_recompress_args* a);

static kvc_status check_recompress(const kvc_model* m, const kvc_recompress_args* a) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  const int d = m->head_dim;
  if (a->batch < 1 || a->len < 1 || a->t < a->len) return fail(KVC_ERR_ARG, "batch/len/t invalid");
  if (a->W < 1 || a->W > a->len) return fail(KVC_ERR_ARG, "W must be in [1, len]");
  if (!a->Qring || !a->qpos || !a->pos || !a->H || !a->D || !a->pos_dst || !a->H_dst || !a->D_dst)
    return fail(KVC_ERR_ARG, "Qring, qpos and the side arrays are required");
  if ((s = check_kv(a->K, "K", d, true)) || (s = check_kv(a->V, "V", d, true)) ||
      (s = check_kv(a->K_dst, "K_dst", d, true)) || (s = check_kv(a->V_dst, "V_dst", d, true)))
    return s;
  if (a->K.ptr == a->K_dst.ptr || a->V.ptr == a->V_dst.ptr) return fail(KVC_ERR_ARG, "src and dst alias");
  if (a->side_s_row < a->len || a->side_dst_s_row < a->cap_dst) return fail(KVC_ERR_ARG, "side row strides too small");
  const long long k = (long long)floor(a->rho * (double)a->t);
  const int lo = a->w < a->len ? a->w : a->len;
  long long kk = k < lo ? lo : (k > a->len ? a->len : k);
  if (kk > a->cap_dst) return fail(KVC_ERR_ARG, "cap_dst %d < kept %lld", a->cap_dst, kk);
  if (a->kept_bits_dst) {
    if (a->bits_words < 1) return fail(KVC_ERR_ARG, "bits_words must be >= 1");
    if ((uintptr_t)a->kept_bits_dst % 4) return fail(KVC_ERR_ARG, "kept_bits_dst not 4-byte aligned");
  }
  if ((!a->U) != (!a->U_dst)) return fail(KVC_ERR_ARG, "U and U_dst go together");
  if (a->recas_state) {
    if (!a->k_out) return fail(KVC_ERR_ARG, "the RECAS budget needs k_out");
    if (a->cap_dst < a->len) return fail(KVC_ERR_ARG, "the RECAS budget needs cap_dst >= len");
    if (a->len > RECAS_MAX_N) return fail(KVC_ERR_UNSUPPORTED, "RECAS budget: len %d > %d", a->len, RECAS_MAX_N);
    if (!recompress_batchable(m, a))
      return fail(KVC_ERR_UNSUPPORTED, "RECAS budget needs caches whose sequences are L layers apart");
  }
  return KVC_OK;
}

static int recompress_kept(const kvc_recompress_args* a) {
  const long long k = (long long)floor(a->rho * (double)a->t);
  const int lo = a->w < a->len ? a->w : a->len;
  return (int)(k < lo ? lo : (k > a->len ? a->len : k));
}

static void recompress_sub_args(const kvc_model* m, const kvc_recompress_args* a, int b,
                                kvc_score_args* sa, kvc_select_args* se, int* kk_out) {
  const int L = m->n_layers, Hkv = m->n_kv_heads, Hq = m->n_q_heads, d = m->head_dim;
  const size_t es = esize(a->K.dtype);
  memset(sa, 0, sizeof(*sa));
  sa->mode = KVC_SCORE_INFOKV;
  sa->n = a->len; sa->W = a->W; sa->alpha = a->alpha; sa->tau = a->tau; sa->scale = a->scale; sa->topk = 256;
  sa->Qw = (const char*)a->Qring + (size_t)b * L * Hq * a->W * d * es;
  sa->qpos = a->qpos + (size_t)b * a->W;
  sa->K = a->K; sa->K.ptr = (char*)a->K.ptr + (size_t)b * a->K.s_batch * es;
  const int64_t row = a->side_s_row;
  sa->kpos = a->pos + (size_t)b * L * Hkv * row; sa->kpos_s_layer = Hkv * row; sa->kpos_s_head = row;
  sa->H_in = a->H + (size_t)b * L * Hkv * row; sa->H_s_layer = Hkv * row; sa->H_s_head = row;
  sa->D_in = a->D + (size_t)b * L * Hkv * row; sa->D_s_layer = Hkv * row; sa->D_s_head = row;
  memset(se, 0, sizeof(*se));
  se->sel_mode = a->sel_mode; se->n = a->len; se->w = a->w;
  se->budget_mode = KVC_BUDGET_EXPLICIT;
  const long long k = (long long)floor(a->rho * (double)a->t);
  const int lo = a->w < a->len ? a->w : a->len;
  *kk_out = (int)(k < lo ? lo : (k > a->len ? a->len : k));
  se->k_cap = *kk_out;
}

struct RecompressPlan {
  size_t score_bytes, sel_bytes, bytes;
  float *S, *A;
  int32_t *idx, *kl, *need;
  int kcap;
  void *score_ws, *sel_ws;
};

// The batch folded into the layer dimension: sequence b's layer l is layer b * L + l.
static kvc_model batched_model(const kvc_model* m, int batch) {
  kvc_model mb = *m;
  mb.n_layers = m->n_layers * batch;
  return mb;
}

// Every per-sequence array steps from sequence b to b + 1 by exactly L layers, so the
// batch can run as one model of B * L layers.
static bool recompress_batchable(const kvc_model* m, const kvc_recompress_args* a) {
  const int64_t L = m->n_layers;
  auto flat = [&](const kvc_kv& t) { return a->batch == 1 || t.s_batch == L * t.s_layer; };
  return flat(a->K) && flat(a->V) && flat(a->K_dst) && flat(a->V_dst);
}

static RecompressPlan plan_recompress(const kvc_model* m0, const kvc_recompress_args* a, void* ws) {
  RecompressPlan p{};
  kvc_score_args sa;
  kvc_select_args se;
  int kk = 0;
  // sized for the whole batch at once (also enough for one sequence at a time)
  const kvc_model mb = batched_model(m0, a->batch);
  const kvc_model* m = &mb;
  recompress_sub_args(m0, a, 0, &sa, &se, &kk);
  const int L = m->n_layers, Hkv = m->n_kv_heads;
  Carver c(ws);
  p.kcap = a->recas_state ? a->len : (kk > 0 ? kk : 1);
  p.S = c.take<float>((size_t)L * Hkv * a->len);
  p.idx = c.take<int32_t>((size_t)L * Hkv * p.kcap);
  p.kl = c.take<int32_t>((size_t)L);
  if (a->recas_state) {
    p.A = c.take<float>((size_t)L * Hkv * a->len);
    p.need = c.take<int32_t>((size_t)L * Hkv);
  }
  sa.S = p.S;
  sa.A = p.A;
  p.score_bytes = plan_score(m, &sa, nullptr).bytes;
  p.score_ws = c.take<char>(p.score_bytes);
  p.sel_bytes = select_ws(m, &se);
  p.sel_ws = c.take<char>(p.sel_bytes);
  p.bytes = c.off;
  return p;
}

static kvc_status run_recompress(const kvc_model* m, const kvc_recompress_args* a, void* ws,
                                 size_t ws_bytes, cudaStream_t st) {
  kvc_status s = check_recompress(m, a);
  if (s) return s;
  RecompressPlan pl = plan_recompress(m, a, nullptr);
  if (!ws || ws_bytes < pl.bytes) return fail(KVC_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, pl.bytes);
  pl = plan_recompress(m, a, ws);
  const size_t es = esize(a->K.dtype);
  if (recompress_batchable(m, a)) {
    // one score / select / compact over all B * L layers; the window-query position rows
    // of the batch are told apart per layer (L layers per row)
    const kvc_model mb = batched_model(m, a->batch);
    const int LB = mb.n_layers, Hkv = mb.n_kv_heads;
    kvc_score_args sa;
    kvc_select_args se;
    int kk = 0;
    recompress_sub_args(m, a, 0, &sa, &se, &kk);   // sequence 0's bases, layer strides as given
    sa.S = pl.S;
    sa.A = pl.A;
    if ((s = run_score(&mb, &sa, pl.score_ws, pl.score_bytes, st, m->n_layers, a->win_lse))) return s;
    cudaError_t e;
    if (a->recas_state) {
      // [RECAS] 2.B adaptive budget: each row's need from the calibrated bound, the batch
      // keeps the largest (also the k_out every (sequence, layer) reports)
      RecasCtlParams cp{};
      cp.rows = LB * Hkv; cp.Hkv = Hkv; cp.n = a->len; cp.w = a->w; cp.k0 = kk;
      cp.np2 = 1;
      while (cp.np2 < a->len) cp.np2 <<= 1;
      cp.union_mode = a->sel_mode == KVC_SEL_GQA_UNION;
      cp.S = pl.S; cp.A = pl.A; cp.s_row = a->len;
      cp.state = a->recas_state; cp.eps = a->recas_eps; cp.need = pl.need;
      if ((e = launch_recas_control(cp, st))) return cuda_fail(e, "recas_control");
      const int kmax = a->recas_k_max > 0 && a->recas_k_max < a->len ? a->recas_k_max : a->len;
      if ((e = launch_recas_budget(pl.need, LB * Hkv, kmax < kk ? kk : kmax, nullptr, pl.kl, LB, a->k_out, LB, st)))
        return cuda_fail(e, "recas_budget");
    } else {
      e = launch_budget(KVC_BUDGET_UNIFORM, LB, kk, 0, 1.0, nullptr, 0, nullptr, pl.kl, st);
      if (e) return cuda_fail(e, "budget");
    }
    e = launch_select(pl.S, (int64_t)Hkv * a->len, a->len, LB, Hkv, a->len, a->w,
                      a->sel_mode == KVC_SEL_GQA_UNION, pl.kl, pl.idx, pl.kcap, (uint32_t*)pl.sel_ws, st);
    if (e) return cuda_fail(e, "select");
    kvc_compact_args ca;
    memset(&ca, 0, sizeof(ca));
    ca.n = a->len;
    ca.src_K = a->K; ca.src_V = a->V; ca.dst_K = a->K_dst; ca.dst_V = a->V_dst;
    ca.idx = pl.idx; ca.k_cap = pl.kcap; ca.k = pl.kl;
    const int64_t sr = a->side_s_row;
    ca.src_pos = a->pos; ca.pos_s_layer = Hkv * sr; ca.pos_s_head = sr;
    ca.src_H = a->H; ca.H_s_layer = Hkv * sr; ca.H_s_head = sr;
    ca.src_D = a->D; ca.D_s_layer = Hkv * sr; ca.D_s_head = sr;
    ca.dst_pos = a->pos_dst; ca.dst_H = a->H_dst; ca.dst_D = a->D_dst;
    ca.src_U = a->U; ca.U_s_layer = Hkv * sr; ca.U_s_head = sr; ca.dst_U = a->U_dst;
    if ((s = compact_impl(&mb, &ca, a->side_dst_s_row, st))) return s;
    if (a->kept_bits_dst) {
      e = launch_kept_bits(a->pos_dst, a->side_dst_s_row, pl.kl, pl.kcap, a->batch, m->n_layers, Hkv,
                           a->kept_bits_dst, a->bits_s_batch, a->bits_s_layer, a->bits_s_head, a->bits_words, st);
      if (e) return cuda_fail(e, "kept_bits");
    }
    if (a->recas_state) {
      if (a->recas_x &&
          (e = launch_recas_predictor(pl.A, a->len, a->len, pl.idx, pl.kcap, pl.kl, LB * Hkv, Hkv, a->recas_x, st)))
        return cuda_fail(e, "recas_predictor");
      if (a->host_kept) *a->host_kept = -1;
      return KVC_OK;
    }
    if (a->k_out) {
      e = launch_budget(KVC_BUDGET_UNIFORM, LB, kk, 0, 1.0, nullptr, 0, nullptr, a->k_out, st);
      if (e) return cuda_fail(e, "k_out");
    }
    if (a->host_kept) *a->host_kept = kk;
    return KVC_OK;
  }
  const int L = m->n_layers, Hkv = m->n_kv_heads;
  for (int b = 0; b < a->batch; ++b) {
    kvc_score_args sa;
    kvc_select_args se;
    int kk = 0;
    recompress_sub_args(m, a, b, &sa, &se, &kk);
    sa.S = pl.S;
    const float* wl = a->win_lse ? a->win_lse + (size_t)b * L * m->n_q_heads * a->W : nullptr;
    if ((s = run_score(m, &sa, pl.score_ws, pl.score_bytes, st, 0, wl))) return s;
    // every layer keeps kk: explicit budgets written by the budget kernel in uniform mode
    cudaError_t e = launch_budget(KVC_BUDGET_UNIFORM, L, kk, 0, 1.0, nullptr, 0, nullptr, pl.kl, st);
    if (e) return cuda_fail(e, "budget");
    e = launch_select(pl.S, (int64_t)Hkv * a->len, a->len, L, Hkv, a->len, a->w,
                      a->sel_mode == KVC_SEL_GQA_UNION, pl.kl, pl.idx, kk, (uint32_t*)pl.sel_ws, st);
    if (e) return cuda_fail(e, "select");
    kvc_compact_args ca;
    memset(&ca, 0, sizeof(ca));
    ca.n = a->len;
    ca.src_K = a->K; ca.src_K.ptr = (char*)a->K.ptr + (size_t)b * a->K.s_batch * es;
    ca.src_V = a->V; ca.src_V.ptr = (char*)a->V.ptr + (size_t)b * a->V.s_batch * es;
    ca.dst_K = a->K_dst; ca.dst_K.ptr = (char*)a->K_dst.ptr + (size_t)b * a->K_dst.s_batch * es;
    ca.dst_V = a->V_dst; ca.dst_V.ptr = (char*)a->V_dst.ptr + (size_t)b * a->V_dst.s_batch * es;
    ca.idx = pl.idx; ca.k_cap = kk; ca.k = pl.kl;
    // side arrays: source rows of side_s_row, destination rows of side_dst_s_row
    const int64_t sr = a->side_s_row;
    ca.src_pos = a->pos + (size_t)b * L * Hkv * sr; ca.pos_s_layer = Hkv * sr; ca.pos_s_head = sr;
    ca.src_H = a->H + (size_t)b * L * Hkv * sr; ca.H_s_layer = Hkv * sr; ca.H_s_head = sr;
    ca.src_D = a->D + (size_t)b * L * Hkv * sr; ca.D_s_layer = Hkv * sr; ca.D_s_head = sr;
    ca.dst_pos = a->pos_dst + (size_t)b * L * Hkv * a->side_dst_s_row;
    ca.dst_H = a->H_dst + (size_t)b * L * Hkv * a->side_dst_s_row;
    ca.dst_D = a->D_dst + (size_t)b * L * Hkv * a->side_dst_s_row;
    if (a->U) {
      ca.src_U = a->U + (size_t)b * L * Hkv * sr; ca.U_s_layer = Hkv * sr; ca.U_s_head = sr;
      ca.dst_U = a->U_dst + (size_t)b * L * Hkv * a->side_dst_s_row;
    }
    if ((s = compact_impl(m, &ca, a->side_dst_s_row, st))) return s;
    if (a->kept_bits_dst) {
      e = launch_kept_bits(ca.dst_pos, a->side_dst_s_row, pl.kl, kk, 1, L, Hkv,
                           a->kept_bits_dst + (size_t)b * a->bits_s_batch, 0, a->bits_s_layer, a->bits_s_head,
                           a->bits_words, st);
      if (e) return cuda_fail(e, "kept_bits");
    }
    if (a->k_out) {
      e = launch_budget(KVC_BUDGET_UNIFORM, L, kk, 0, 1.0, nullptr, 0, nullptr, a->k_out + (size_t)b * L, st);
      if (e) return cuda_fail(e, "k_out");
    }
  }
  if (a->host_kept) *a->host_kept = recompress_kept(a);
  return KVC_OK;
}

// ----------------------------------------------------------------- RECAS estimator and controller
static kvc_status run_recas_calibrate(const kvc_model* m, const kvc_recas_calibrate_args* a, cudaStream_t st) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  if (a->batch < 1) return fail(KVC_ERR_ARG, "batch must be >= 1");
  if (!a->delta || !a->x || !a->state) return fail(KVC_ERR_ARG, "delta, x and state are required");
  if (!(a->alpha > 0.f && a->alpha < 1.f)) return fail(KVC_ERR_ARG, "alpha must be in (0, 1)");
  if ((uintptr_t)a->state % 8) return fail(KVC_ERR_ARG, "state not 8-byte aligned");
  if (m->n_q_heads > KVC_RECAS_RING) return fail(KVC_ERR_UNSUPPORTED, "more query heads than ring slots");
  RecasCalParams p{};
  p.BL = a->batch * m->n_layers; p.Hq = m->n_q_heads; p.Hkv = m->n_kv_heads; p.G = m->n_q_heads / m->n_kv_heads;
  p.delta = a->delta; p.x = a->x; p.alpha = a->alpha; p.state = a->state;
  p.delta_hat = a->delta_hat; p.delta_bar = a->delta_bar;
  cudaError_t e = launch_recas_calibrate(p, st);
  if (e) return cuda_fail(e, "recas_calibrate");
  return KVC_OK;
}

static kvc_status run_recas_control(const kvc_model* m, const kvc_recas_control_args* a, cudaStream_t st) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  if (a->batch < 1 || a->n < 1 || a->w < 0) return fail(KVC_ERR_ARG, "batch, n and w invalid");
  if (a->n > RECAS_MAX_N) return fail(KVC_ERR_UNSUPPORTED, "n %d > %d", a->n, RECAS_MAX_N);
  if (a->k0 < 0 || a->k0 > a->n) return fail(KVC_ERR_ARG, "k0 must be in [0, n]");
  if (!a->S || !a->A || !a->state || !a->need) return fail(KVC_ERR_ARG, "S, A, state and need are required");
  if (a->s_row < a->n) return fail(KVC_ERR_ARG, "s_row smaller than n");
  if (a->sel_mode != KVC_SEL_PER_KV_HEAD && a->sel_mode != KVC_SEL_GQA_UNION)
    return fail(KVC_ERR_ARG, "sel_mode invalid");
  RecasCtlParams p{};
  p.rows = a->batch * m->n_layers * m->n_kv_heads; p.Hkv = m->n_kv_heads; p.n = a->n; p.w = a->w; p.k0 = a->k0;
  p.np2 = 1;
  while (p.np2 < a->n) p.np2 <<= 1;
  p.union_mode = a->sel_mode == KVC_SEL_GQA_UNION;
  p.S = a->S; p.A = a->A; p.s_row = a->s_row; p.state = a->state; p.eps = a->eps; p.need = a->need;
  cudaError_t e = launch_recas_control(p, st);
  if (e) return cuda_fail(e, "recas_control");
  const int kmax = a->k_max > 0 && a->k_max < a->n ? a->k_max : a->n;
  if (a->budget && (e = launch_recas_budget(a->need, p.rows, kmax, a->budget, nullptr, 0, nullptr, 0, st)))
    return cuda_fail(e, "recas_budget");
  return KVC_OK;
}

// ----------------------------------------------------------------- dynamic sparse decode
struct SparsePlan {
  size_t bytes;
  float *s, *hstat;
  int32_t* kt;
};

static SparsePlan plan_sparse(const kvc_model* m, const kvc_sparse_decode_args* a, void* ws) {
  SparsePlan p{};
  const size_t rows = (size_t)a->batch * m->n_layers * m->n_kv_heads;
  const int G = m->n_q_heads / m->n_kv_heads;
  Carver c(ws);
  p.s = c.take<float>(rows * G * a->max_len);
  p.hstat = c.take<float>(rows * ((a->max_len + SPARSE_CHUNK - 1) / SPARSE_CHUNK) * 16);
  p.kt = c.take<int32_t>((size_t)a->batch * m->n_layers);
  p.bytes = c.off;
  return p;
}

static kvc_status check_sparse(const kvc_model* m, const kvc_sparse_decode_args* a) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  const int G = m->n_q_heads / m->n_kv_heads;
  if (m->head_dim != 128 || G > 8) return fail(KVC_ERR_UNSUPPORTED, "sparse decode: head_dim 128, G <= 8");
  if (a->batch < 1 || a->max_len < 1) return fail(KVC_ERR_ARG, "batch and max_len must be >= 1");
  if (a->max_len > RECAS_MAX_N) return fail(KVC_ERR_UNSUPPORTED, "max_len %d > %d", a->max_len, RECAS_MAX_N);
  if (!a->q || !a->len || !a->pos || !a->acc || !a->o) return fail(KVC_ERR_ARG, "q, len, pos, acc and o are required");
  if (a->q_dtype != KVC_BF16) return fail(KVC_ERR_UNSUPPORTED, "sparse decode: bf16 queries");
  if ((uintptr_t)a->q % 4) return fail(KVC_ERR_ARG, "q not 4-byte aligned");
  if ((s = check_kv(a->K, "K", 128, true)) || (s = check_kv(a->V, "V", 128, true))) return s;
  if (a->K.dtype != KVC_BF16 || a->V.dtype != KVC_BF16) return fail(KVC_ERR_UNSUPPORTED, "sparse decode: bf16 caches");
  if (a->side_s_row < a->max_len) return fail(KVC_ERR_ARG, "side_s_row smaller than max_len");
  if (a->lse_stride < 0) return fail(KVC_ERR_ARG, "lse_stride must be >= 0");
  if (!(a->kappa > 0.0 && a->kappa <= 1.0)) return fail(KVC_ERR_ARG, "kappa must be in (0, 1]");
  if (a->n_prompt < 0 || a->t_cur <= a->n_prompt - 1) return fail(KVC_ERR_ARG, "t_cur / n_prompt invalid");
  return KVC_OK;
}

static kvc_status run_sparse(const kvc_model* m, const kvc_sparse_decode_args* a, void* ws, size_t ws_bytes,
                             cudaStream_t st) {
  kvc_status s = check_sparse(m, a);
  if (s) return s;
  SparsePlan pl = plan_sparse(m, a, nullptr);
  if (!ws || ws_bytes < pl.bytes) return fail(KVC_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, pl.bytes);
  pl = plan_sparse(m, a, ws);
  SparseParams p{};
  p.B = a->batch; p.L = m->n_layers; p.Hq = m->n_q_heads; p.Hkv = m->n_kv_heads; p.G = m->n_q_heads / m->n_kv_heads;
  p.max_len = a->max_len;
  p.q = a->q; p.qbf16 = a->q_dtype == KVC_BF16;
  p.K = (const char*)a->K.ptr; p.Ksb = b2(a->K, a->K.s_batch); p.Ksl = b2(a->K, a->K.s_layer); p.Ksh = b2(a->K, a->K.s_head); p.Kst = b2(a->K, a->K.s_tok);
  p.V = (const char*)a->V.ptr; p.Vsb = b2(a->V, a->V.s_batch); p.Vsl = b2(a->V, a->V.s_layer); p.Vsh = b2(a->V, a->V.s_head); p.Vst = b2(a->V, a->V.s_tok);
  p.len = a->len; p.pos = a->pos; p.acc = a->acc; p.side_row = a->side_s_row;
  p.t_cur = a->t_cur; p.n_prompt = a->n_prompt;
  p.kappa = a->kappa; p.a_tr = a->a_tr; p.b_hi = a->b_hi;
  p.scale = a->scale > 0.f ? a->scale : 1.f / sqrtf(128.f);
  p.s = pl.s; p.hstat = pl.hstat; p.kt = pl.kt; p.active = a->active;
  p.n_active = a->n_active; p.o = a->o;
  p.lse = a->lse; p.lse_stride = a->lse_stride > 0 ? a->lse_stride : 1;
  cudaError_t e = launch_sparse_decode(p, st);
  if (e) return cuda_fail(e, "sparse_decode");
  return KVC_OK;
}

// ----------------------------------------------------------------- LM-head entropy
static kvc_status check_lmhead(const kvc_lmhead_entropy_args* a) {
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  if (a->n < 1 || a->Dh < 1 || a->V < 1) return fail(KVC_ERR_ARG, "n, Dh and V must be >= 1");
  if (a->k < 1 || a->k > 256) return fail(KVC_ERR_UNSUPPORTED, "k must be in [1, 256]");
  if (a->dtype != KVC_BF16) return fail(KVC_ERR_UNSUPPORTED, "lmhead entropy: bf16 x and W");
  if (!a->x || !a->W || !a->H) return fail(KVC_ERR_ARG, "x, W and H are required");
  if ((uintptr_t)a->x % 16 || (uintptr_t)a->W % 16) return fail(KVC_ERR_ARG, "x / W not 16-byte aligned");
  if (a->x_stride < a->Dh || a->W_stride < a->Dh || a->x_stride % 8 || a->W_stride % 8)
    return fail(KVC_ERR_ARG, "strides must be >= Dh and multiples of 8 elements");
  return KVC_OK;
}

static kvc_status run_lmhead(const kvc_lmhead_entropy_args* a, void* ws, size_t ws_bytes, cudaStream_t st) {
  kvc_status s = check_lmhead(a);
  if (s) return s;
  const LmPlan pl = plan_lmhead(a->n, a->Dh, a->V, a->k, num_sms());
  if (!ws || ws_bytes < pl.bytes) return fail(KVC_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, pl.bytes);
  if ((uintptr_t)ws % 256) return fail(KVC_ERR_ARG, "workspace not 256-byte aligned");
  LmheadParams p{};
  p.n = a->n; p.Dh = a->Dh; p.V = a->V; p.k = a->k;
  p.x = a->x; p.x_stride = a->x_stride; p.W = a->W; p.W_stride = a->W_stride; p.H = a->H;
  cudaError_t e = launch_lmhead_entropy(p, ws, st);
  if (e) return cuda_fail(e, "lmhead_entropy");
  return KVC_OK;
}

// ----------------------------------------------------------------- append
static kvc_status check_append(const kvc_model* m, const kvc_append_args* a) {
  kvc_status s = check_model(m);
  if (s) return s;
  if (!a) return fail(KVC_ERR_ARG, "args is NULL");
  const int d = m->head_dim;
  if (a->batch < 1 || a->cap < 1) return fail(KVC_ERR_ARG, "batch and cap must be >= 1");
  if (!a->k || !a->v || !a->len) return fail(KVC_ERR_ARG, "k, v and len are required");
  if ((s = check_kv(a->K, "K", d, true)) || (s = check_kv(a->V, "V", d, true))) return s;
  if (a->K.dtype != a->V.dtype) return fail(KVC_ERR_ARG, "K and V dtypes differ");
  if ((uintptr_t)a->k % 16 || (uintptr_t)a->v % 16) return fail(KVC_ERR_ARG, "k / v not 16-byte aligned");
  if (a->pos < 0) return fail(KVC_ERR_ARG, "pos must be >= 0");
  if ((a->side_pos || a->side_H || a->side_D || a->side_R || a->side_U) && a->side_s_row < a->cap)
    return fail(KVC_ERR_ARG, "side_s_row smaller than cap");
  if (a->side_H && !a->H_new) return fail(KVC_ERR_ARG, "side_H needs H_new");
  if (a->side_D && !a->D_new) return fail(KVC_ERR_ARG, "side_D needs D_new");
  if (a->kept_bits) {
    if ((uintptr_t)a->kept_bits % 4) return fail(KVC_ERR_ARG, "kept_bits not 4-byte aligned");
    if (a->pos / 32 >= a->bits_words) return fail(KVC_ERR_ARG, "pos %d past the %d bit words", a->pos, a->bits_words);
  }
  if (a->K2.ptr || a->V2.ptr || a->len2) {
    if (!a->K2.ptr || !a->V2.ptr || !a->len2) return fail(KVC_ERR_ARG, "K2, V2 and len2 go together");
    if ((s = check_kv(a->K2, "K2", d, true)) || (s = check_kv(a->V2, "V2", d, true))) return s;
    if (a->K2.dtype != a->K.dtype || a->V2.dtype != a->K.dtype)
      return fail(KVC_ERR_ARG, "K2 / V2 dtype differs from K");
    if (a->cap2 < 1) return fail(KVC_ERR_ARG, "cap2 must be >= 1");
  }
  if (a->q || a->Qring || a->qpos) {
    if (!a->q || !a->Qring || !a->qpos) return fail(KVC_ERR_ARG, "q, Qring and qpos go together");
    if ((uintptr_t)a->q % 16 || (uintptr_t)a->Qring % 16) return fail(KVC_ERR_ARG, "q / Qring not 16-byte aligned");
    if (a->W < 1 || a->slot < 0 || a->slot >= a->W) return fail(KVC_ERR_ARG, "slot must be in [0, W)");
  }
  return KVC_OK;
}

static kvc_status run_append(const kvc_model* m, const kvc_append_args* a, cudaStream_t st) {
  kvc_status s = check_append(m, a);
  if (s) return s;
  const size_t es = esize(a->K.dtype);
  AppendParams p{};
  p.B = a->batch; p.L = m->n_layers; p.Hq = m->n_q_heads; p.Hkv = m->n_kv_heads; p.cap = a->cap;
  p.row_bytes = (int64_t)m->head_dim * (int64_t)es;
  p.vr = (int)(p.row_bytes / 16);
  p.k = (const char*)a->k; p.v = (const char*)a->v;
  p.K = (char*)a->K.ptr; p.Ksb = b2(a->K, a->K.s_batch); p.Ksl = b2(a->K, a->K.s_layer); p.Ksh = b2(a->K, a->K.s_head); p.Kst = b2(a->K, a->K.s_tok);
  p.V = (char*)a->V.ptr; p.Vsb = b2(a->V, a->V.s_batch); p.Vsl = b2(a->V, a->V.s_layer); p.Vsh = b2(a->V, a->V.s_head); p.Vst = b2(a->V, a->V.s_tok);
  p.len = a->len; p.pos = a->pos;
  p.spos = a->side_pos; p.sH = a->side_H; p.sD = a->side_D; p.sR = a->side_R; p.sU = a->side_U;
  p.side_row = a->side_s_row;
  p.H_new = a->H_new; p.D_new = a->D_new; p.Dnb = a->D_new_s_batch; p.Dnl = a->D_new_s_layer;
  p.bits = a->kept_bits; p.bsb = a->bits_s_batch; p.bsl = a->bits_s_layer; p.bsh = a->bits_s_head;
  p.q = (const char*)a->q; p.Qring = (char*)a->Qring; p.qpos = a->qpos; p.W = a->W; p.slot = a->slot;
  if (a->K2.ptr) {
    p.K2 = (char*)a->K2.ptr; p.K2sb = b2(a->K2, a->K2.s_batch); p.K2sl = b2(a->K2, a->K2.s_layer);
    p.K2sh = b2(a->K2, a->K2.s_head); p.K2st = b2(a->K2, a->K2.s_tok);
    p.V2 = (char*)a->V2.ptr; p.V2sb = b2(a->V2, a->V2.s_batch); p.V2sl = b2(a->V2, a->V2.s_layer);
    p.V2sh = b2(a->V2, a->V2.s_head); p.V2st = b2(a->V2, a->V2.s_tok);
    p.len2 = a->len2; p.cap2 = a->cap2;
  }
  p.status = status_ptr();
  cudaError_t e = launch_append(p, st);
  if (e) return cuda_fail(e, "append");
  return KVC_OK;
}

}  // namespace kvc

// ===================================================================== C ABI
using namespace kvc;

extern "C" {

kvc_status kvc_workspace_size(int op, const kvc_model* m, const void* args, size_t* bytes) {
  if (!bytes) return fail(KVC_ERR_ARG, "bytes is NULL");
  *bytes = 0;
  kvc_status s;
  switch (op) {
    case KVC_OP_SCORE: {
      auto a = (const kvc_score_args*)args;
      if ((s = check_score(m, a))) return s;
      *bytes = plan_score(m, a, nullptr).bytes;
      return KVC_OK;
    }
    case KVC_OP_SELECT: {
      auto a = (const kvc_select_args*)args;
      if ((s = check_select(m, a))) return s;
      *bytes = select_ws(m, a);
      return KVC_OK;
    }
    case KVC_OP_COMPACT:
    case KVC_OP_MERGE:
      if ((s = check_model(m))) return s;
      return KVC_OK;
    case KVC_OP_DECODE: {
      auto a = (const kvc_decode_args*)args;
      if ((s = check_decode(m, a))) return s;
      *bytes = decode_ws(m, a);
      return KVC_OK;
    }
    case KVC_OP_RECOMPRESS: {
      auto a = (const kvc_recompress_args*)args;
      if ((s = check_recompress(m, a))) return s;
      *bytes = plan_recompress(m, a, nullptr).bytes;
      return KVC_OK;
    }
    case KVC_OP_SPARSE_DECODE: {
      auto a = (const kvc_sparse_decode_args*)args;
      if ((s = check_sparse(m, a))) return s;
      *bytes = plan_sparse(m, a, nullptr).bytes;
      return KVC_OK;
    }
    case KVC_OP_LMHEAD_ENTROPY: {
      auto a = (const kvc_lmhead_entropy_args*)args;
      if ((s = check_lmhead(a))) return s;
      *bytes = plan_lmhead(a->n, a->Dh, a->V, a->k, num_sms()).bytes;
      return KVC_OK;
    }
  }
  return fail(KVC_ERR_ARG, "unknown op %d", op);
}

kvc_status kvc_score(const kvc_model* m, const kvc_score_args* a, void* ws, size_t ws_bytes,
                     kvc_stream_t stream) {
  return run_score(m, a, ws, ws_bytes, (cudaStream_t)stream);
}

kvc_status kvc_select(const kvc_model* m, const kvc_select_args* a, void* ws, size_t ws_bytes,
                      kvc_stream_t stream) {
  return run_select(m, a, ws, ws_bytes, (cudaStream_t)stream);
}

kvc_status kvc_compact(const kvc_model* m, const kvc_compact_args* a, kvc_stream_t stream) {
  return run_compact(m, a, (cudaStream_t)stream);
}

kvc_status kvc_merge(const kvc_model* m, const kvc_merge_args* a, void* ws, size_t ws_bytes,
                     kvc_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  return run_merge(m, a, (cudaStream_t)stream);
}

kvc_status kvc_rope_reposition(const kvc_model* m, const kvc_rope_args* a, kvc_stream_t stream) {
  return run_rope(m, a, (cudaStream_t)stream);
}

kvc_status kvc_decode_attn(const kvc_model* m, const kvc_decode_args* a, void* ws, size_t ws_bytes,
                           kvc_stream_t stream) {
  return run_decode(m, a, ws, ws_bytes, (cudaStream_t)stream);
}

kvc_status kvc_recompress(const kvc_model* m, const kvc_recompress_args* a, void* ws,
                          size_t ws_bytes, kvc_stream_t stream) {
  return run_recompress(m, a, ws, ws_bytes, (cudaStream_t)stream);
}

kvc_status kvc_append(const kvc_model* m, const kvc_append_args* a, kvc_stream_t stream) {
  return run_append(m, a, (cudaStream_t)stream);
}

kvc_status kvc_recas_calibrate(const kvc_model* m, const kvc_recas_calibrate_args* a, kvc_stream_t stream) {
  return run_recas_calibrate(m, a, (cudaStream_t)stream);
}

kvc_status kvc_recas_control(const kvc_model* m, const kvc_recas_control_args* a, kvc_stream_t stream) {
  return run_recas_control(m, a, (cudaStream_t)stream);
}

kvc_status kvc_sparse_decode(const kvc_model* m, const kvc_sparse_decode_args* a, void* ws, size_t ws_bytes,
                             kvc_stream_t stream) {
  return run_sparse(m, a, ws, ws_bytes, (cudaStream_t)stream);
}

kvc_status kvc_lmhead_entropy(const kvc_lmhead_entropy_args* a, void* ws, size_t ws_bytes, kvc_stream_t stream) {
  return run_lmhead(a, ws, ws_bytes, (cudaStream_t)stream);
}

kvc_status kvc_check_status(kvc_stream_t stream, uint32_t* host_code) {
  unsigned* p = status_ptr();
  if (!p) return fail(KVC_ERR_CUDA, "status word unavailable");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e) return cuda_fail(e, "check_status");
  unsigned v = 0;
  e = cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost);
  if (e) return cuda_fail(e, "check_status read");
  unsigned zero = 0;
  cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (host_code) *host_code = v;
  if (v & ST_TIMEOUT) return fail(KVC_ERR_TIMEOUT, "a bounded device wait ran out (status 0x%x)", v);
  if (v & ST_BOUNDS) return fail(KVC_ERR_DEVICE, "a device-side index check failed (status 0x%x)", v);
  return KVC_OK;
}

const char* kvc_last_error(void) { return g_err; }

int kvc_version(void) { return 100; }

uint64_t kvc_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
