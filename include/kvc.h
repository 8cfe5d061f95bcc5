/*
 * kvc.h - C ABI of libkvc: KV-cache scoring, selection, compaction, merging
 * and compressed decode attention for long-context decoding on NVIDIA B200
 * (sm_100a).
 *
 * Pages the operations restate (cited by title and section):
 *   [InfoKV] "긴 추론을 위한 정보 인지형 KV 캐시 압축(InfoKV)" (aitrends.kr):
 *            Methodology, Technical details, Glossary.
 *   [SelKV]  "SelKV: Selective KV Cache Merging with Per-Token Merge-or-Drop
 *            and Attention Compensation" (gist.science): Methodology / Core
 *            components, Pipeline overview.
 *   [RECAS]  "기술 요약: 긴 문맥 LLM을 위한 추론 인지적 오차 경계 KV-캐시 압축 및
 *            희소 어텐션" (gist.science): section 2.B.
 *
 * Conventions shared by every call
 *   - Every pointer is a DEVICE pointer unless its name starts with host_.
 *   - The caller owns every buffer (inputs, outputs, workspace).  The library
 *     never allocates, frees or synchronises; every call only enqueues
 *     kernels on the given stream and returns.
 *   - Arguments are validated before anything is launched: a bad argument
 *     returns KVC_ERR_ARG / KVC_ERR_UNSUPPORTED / KVC_ERR_WORKSPACE and
 *     launches nothing.  A launch failure returns KVC_ERR_CUDA.  The message
 *     of the last failure on the calling thread is kvc_last_error().
 *   - Faults detected on the device (a bounded wait that ran out, an index
 *     outside its row) set a per-device status word that kvc_check_status()
 *     reads; no kernel traps or spins without a limit.
 *   - Tensors of cached rows are described by kvc_kv: rows of head_dim
 *     contiguous elements, element (b, l, h, t, j) at
 *     ptr + b*s_batch + l*s_layer + h*s_head + t*s_tok + j (strides in
 *     elements).  Rows must start on 16-byte boundaries.
 *   - Supported: head_dim 64 or 128; K/V/Q/logits/hidden in fp32 or bf16.
 *     Scores, signals and outputs are fp32.
 */
#ifndef KVC_H
#define KVC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* kvc_stream_t; /* a cudaStream_t; NULL is the legacy default stream */

typedef enum {
  KVC_OK = 0,
  KVC_ERR_ARG = 1,          /* invalid argument (null pointer, size, stride, alignment) */
  KVC_ERR_UNSUPPORTED = 2,  /* valid but not implemented (head_dim, dtype, shape) */
  KVC_ERR_WORKSPACE = 3,    /* workspace smaller than kvc_workspace_size() */
  KVC_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
  KVC_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out (kvc_check_status) */
  KVC_ERR_DEVICE = 6        /* a device-side check failed (kvc_check_status) */
} kvc_status;

typedef enum { KVC_F32 = 0, KVC_BF16 = 1 } kvc_dtype;

/* Model shape.  Query head h belongs to KV head h / (n_q_heads / n_kv_heads). */
typedef struct {
  int n_layers;
  int n_q_heads;
  int n_kv_heads;
  int head_dim;
} kvc_model;

/* Strided cache tensor [B][L][Hkv][T][head_dim] (strides in elements). */
typedef struct {
  void* ptr;
  kvc_dtype dtype;
  int64_t s_batch;
  int64_t s_layer;
  int64_t s_head;
  int64_t s_tok;
} kvc_kv;

/* ------------------------------------------------------------------------
 * kvc_score: per-token importance of every (layer, KV head) row.
 *
 * [InfoKV] Methodology / Technical details:
 *   H_i   = entropy of token i's final-layer predictive distribution over its
 *           top-k entries (renormalised, natural log)              (topk = 256)
 *   D_i^l = 1 - cos(h_i^l, h_i^L) + tau                             (tau = 1)
 *   E_i^l = D_i^l * H_i,  P^l = Softmax over the row's tokens of E^l
 *   A_i^l = mean over the G*W window rows (the W window queries of the G query
 *           heads sharing the KV head) of softmax_causal(q k^T * scale)_i
 *   S_i^l = alpha * A_i^l + (1 - alpha) * P_i^l                     (alpha = 0.9)
 * [SelKV] Pipeline overview step 1 (VATP): S_i = A_i * ||v_i||_2.
 * KVC_SCORE_ATTN: S_i = A_i.
 *
 * Causality: key i is visible to window row r iff kpos(i) <= qpos(r).
 * ---------------------------------------------------------------------- */
typedef enum { KVC_SCORE_INFOKV = 0, KVC_SCORE_VATP = 1, KVC_SCORE_ATTN = 2 } kvc_score_mode;

typedef struct {
  kvc_score_mode mode;
  int n;                 /* cached tokens per (layer, KV head) row, >= 1 */
  int W;                 /* window queries, 1 <= W <= n */
  float alpha;           /* InfoKV mix */
  float tau;             /* representation-change bias */
  float scale;           /* logit scale; 0 selects 1/sqrt(head_dim) */
  int topk;              /* entropy top-k, 1..1024 */

  const void* Qw;        /* window queries [L][Hq][W][head_dim], contiguous, dtype of K */
  const int32_t* qpos;   /* [W] positions of the window queries; NULL: n - W + r */
  kvc_kv K;              /* keys [L][Hkv][n][d] (s_batch ignored) */
  kvc_kv V;              /* values, read in VATP mode only */
  const int32_t* kpos;   /* key positions kpos[l*kpos_s_layer + g*kpos_s_head + i]; NULL: i */
  int64_t kpos_s_layer, kpos_s_head;

  /* InfoKV signals: either raw inputs (logits / hidden) or precomputed H / D. */
  const void* logits;    /* [n][vocab] rows, row stride logits_row_stride elements; or NULL */
  kvc_dtype logits_dtype;
  int64_t vocab;
  int64_t logits_row_stride;
  const void* hidden;    /* [L][n][hidden_size] contiguous; layer L-1 is h^L; or NULL */
  kvc_dtype hidden_dtype;
  int hidden_size;       /* multiple of 256 (bf16) or 128 (fp32) */
  const float* H_in;     /* used when logits == NULL: H(l,g,i) = H_in[l*H_s_layer + g*H_s_head + i] */
  int64_t H_s_layer, H_s_head;
  const float* D_in;     /* used when hidden == NULL: D(l,g,i) = D_in[l*D_s_layer + g*D_s_head + i] */
  int64_t D_s_layer, D_s_head;

  /* Outputs (fp32, device); A, H_out, D_out and Ebar may be NULL.
   * S == NULL selects the signals-only form (InfoKV mode, A == NULL): only H_out
   * from logits and / or D_out from hidden are computed, W / Qw / K are not
   * read - used for the per-step signals of newly generated tokens. */
  float* S;              /* [L][Hkv][n] */
  float* A;              /* [L][Hkv][n] window attention */
  float* H_out;          /* [n]      when computed from logits */
  float* D_out;          /* [L][n]   when computed from hidden */
  float* Ebar;           /* [L]      mean of E over the layer's rows and tokens (InfoKV mode) */

  /* InfoKV mode with the entropy and / or representation change computed in this call:
   * the window attention does not depend on them, so it runs beside them on a second
   * stream owned by the library, on window_sms SMs, while they stream their inputs on the
   * others; S is then formed from A, D and H.  0: the library's choice (a quarter of the
   * SMs for rows of up to 32768 tokens, the stages in sequence for longer rows); > 0: that
   * many SMs for the window (clamped to [8, SMs - 8]); < 0: the stages run one after another.
   * The first such call on a device creates the library's stream and two events for that
   * device (kept until exit): make it before any stream capture. */
  int window_sms;
  /* Limit, in ns, of the single-launch window kernel's wait for the row constants another
   * CTA publishes (0: 2 s).  The wait is bounded like every device-side wait: when it runs
   * out the kernel drains its in-flight copies and MMAs, frees its tensor memory, and
   * kvc_check_status reports KVC_ERR_TIMEOUT.  A limit of microseconds makes it run out on
   * purpose (testing the timeout path); S is then not valid. */
  uint64_t wait_limit_ns;
} kvc_score_args;

/* ------------------------------------------------------------------------
 * kvc_select: per-layer budgets and kept positions.
 *
 * [InfoKV] Technical details: keep the top k_l tokens of each layer; uniform
 * budgets by default, optionally k_l = (Ebar^l / sum_m Ebar^m) * B.
 * [SelKV] Pipeline overview step 2: top tokens plus a recent window, per KV
 * head or through the GQA union (a token is ranked by max over KV heads).
 *
 * Per row: the last min(w, n) positions are always kept; the other
 * k_l - min(w, n) are the highest scores among positions < n - w, ties to the
 * lower position; idx lists ascend.  Budgets are clamped to [min(w, n), n];
 * adaptive budgets use the clamped proportional share whose sum is B, rounded
 * by largest remainder (ties to the lower layer).
 * ---------------------------------------------------------------------- */
typedef enum { KVC_SEL_PER_KV_HEAD = 0, KVC_SEL_GQA_UNION = 1 } kvc_sel_mode;
typedef enum { KVC_BUDGET_UNIFORM = 0, KVC_BUDGET_EXPLICIT = 1, KVC_BUDGET_ADAPTIVE = 2 } kvc_budget_mode;

typedef struct {
  kvc_sel_mode sel_mode;
  int n;                 /* tokens per row */
  int w;                 /* recent window */
  const float* S;        /* S(l,g,i) = S[l*S_s_layer + g*S_s_head + i] */
  int64_t S_s_layer, S_s_head;
  kvc_budget_mode budget_mode;
  double rho;            /* UNIFORM: k_l = floor(rho * n) */
  const int32_t* k_in;   /* EXPLICIT: [L] device budgets */
  int64_t B_total;       /* ADAPTIVE: total budget B, L*min(w,n) <= B <= L*n */
  const float* Ebar;     /* ADAPTIVE: [L] device */
  int32_t* k_out;        /* [L] device budgets actually used (required) */
  int32_t* idx;          /* [L][Hkv][k_cap] kept positions, ascending (required) */
  int k_cap;             /* row capacity of idx; must be >= every k_l (n is always safe) */
} kvc_select_args;

/* ------------------------------------------------------------------------
 * kvc_compact: gather the kept rows.  dst(l,g,j) = src(l,g,idx(l,g,j)) for
 * j < k_l, bit-exact, for K, V and the optional per-token side arrays.
 * [InfoKV] Technical details (keep the top k_l tokens of each layer).
 * src and dst must not overlap.
 * ---------------------------------------------------------------------- */
typedef struct {
  int n;                 /* source rows per (l, g) */
  kvc_kv src_K, src_V;   /* [L][Hkv][n][d] */
  kvc_kv dst_K, dst_V;   /* [L][Hkv][k_cap][d]; same dtype as src */
  const int32_t* idx;    /* [L][Hkv][k_cap] */
  int k_cap;
  const int32_t* k;      /* [L] device */
  /* Optional side arrays; destinations are [L][Hkv][k_cap] contiguous.
   * src(l,g,i) = src_x[l*x_s_layer + g*x_s_head + i]; src_pos NULL means pos = i. */
  const int32_t* src_pos; int64_t pos_s_layer, pos_s_head; int32_t* dst_pos;
  const float* src_H;     int64_t H_s_layer, H_s_head;     float* dst_H;
  const float* src_D;     int64_t D_s_layer, D_s_head;     float* dst_D;
  /* the RECAS attention history of kvc_sparse_decode (acc), same form as H and D */
  const float* src_U;     int64_t U_s_layer, U_s_head;     float* dst_U;
} kvc_compact_args;

/* ------------------------------------------------------------------------
 * kvc_merge: SelKV routing, soft-cosine-gated value merge and attention ratio.
 *
 * [SelKV] Methodology / Core components 1-2 and Pipeline overview steps 3-5.
 * Per (l, g) and positional bucket b = floor(i / bucket): the target t_b is
 * the kept position of the bucket with the highest A (ties: lower position);
 * every evicted j of the bucket gets g_j = max(cos(v_j, v_t), 0) and
 *   V'_t = (A_t v_t + sum_j g_j A_j v_j) / (A_t + sum_j g_j A_j),
 *   R_t  = (A_t + sum_j g_j A_j) / A_t.
 * Other kept slots: V' = v, R = 1.  A bucket with no kept token drops its
 * evicted tokens; a target whose gated mass sum_j g_j A_j is 0 (every gate 0)
 * keeps v bit for bit and R = 1.  A target with A_t = 0 merges nothing (V' = v,
 * R = 1) and ors the value 4 into the status word: kvc_check_status returns
 * KVC_OK for it (a defined outcome, not a fault) and passes it in host_code.
 * Keys are not touched (compact them with kvc_compact).
 * Deterministic: no atomics, fixed summation order.
 * ---------------------------------------------------------------------- */
typedef struct {
  int n;
  int bucket;            /* > 0 */
  kvc_kv V;              /* full values [L][Hkv][n][d] */
  const float* A;        /* A(l,g,i) = A[l*A_s_layer + g*A_s_head + i] */
  int64_t A_s_layer, A_s_head;
  const int32_t* idx;    /* [L][Hkv][k_cap] ascending kept positions */
  int k_cap;
  const int32_t* k;      /* [L] device */
  kvc_kv dst_V;          /* [L][Hkv][k_cap][d]; bf16 stores round to nearest even */
  float* R;              /* [L][Hkv][k_cap] */
  float* dst_V_f32;      /* optional [L][Hkv][k_cap][d] fp32 copy of V' before rounding */
} kvc_merge_args;

/* ------------------------------------------------------------------------
 * kvc_rope_reposition: re-embed the kept keys at contiguous positions.
 *
 * [SelKV] Pipeline overview, step 6 (RoPE re-positioning; the pages switch it
 * off for long-context evaluation).  Key row j < k_l of (l, g) carries the
 * rotary embedding of position pos(l, g, j) and is turned to position
 * new0 + j: with a = (new0 + j - pos) * base^(-2i/d), every dimension pair
 * (x_i, x_{i+d/2}), i < d/2, becomes
 *   x_i' = x_i cos a - x_{i+d/2} sin a,   x_{i+d/2}' = x_{i+d/2} cos a + x_i sin a
 * (half-split pairing as in the Llama / Qwen layouts; no frequency scaling).
 * Angles are formed in fp64 and reduced modulo pi/2 (two-constant Cody-Waite
 * step; the quadrant comes from the rounding); sine and cosine of the reduced
 * fp32 angle come from their Taylor series, the turn is fp32, bf16 stores round
 * to nearest even.  Rows j >= k_l are not touched.
 * ---------------------------------------------------------------------- */
typedef struct {
  kvc_kv K;              /* [L][Hkv][>= k_cap][d] keys */
  kvc_kv K_dst;          /* same dtype; ptr NULL or == K.ptr: in place.  Otherwise it must not
                            overlap K. */
  const int32_t* pos;    /* pos(l,g,j) = pos[(l*Hkv + g)*pos_s_row + j]: positions the keys carry */
  int64_t pos_s_row;     /* >= k_cap */
  int32_t* pos_dst;      /* optional: receives new0 + j (same layout; may be pos itself) */
  const int32_t* k;      /* [L] device: rows of every (l, g) to re-embed (clamped to k_cap) */
  int k_cap;
  int64_t new0;          /* position given to row 0; new0 + k_cap - 1 must fit in int32 */
  double base;           /* rotary base (theta), finite and > 1 */
} kvc_rope_args;

/* ------------------------------------------------------------------------
 * kvc_decode_attn: decode attention over a (compressed) cache.
 *
 * [SelKV] Methodology / Core component 2: logit bias alpha_c * log(R_i).
 *   o(b,l,h) = sum_i softmax_i(q k_i * scale + alpha_c * log R_i) v_i
 * over the first len[b][l] rows of KV head h / G of layer l.
 * Optional RECAS probe ([RECAS] 2.B) over the full history with a kept bit
 * per position: delta = attention mass (no bias) on evicted positions,
 * V_max = max ||v_i|| of the full history, o_full, o' = attention over the
 * kept positions only, err = ||o_full - o'||_2 and bound = 2 * V_max * delta.
 * ---------------------------------------------------------------------- */
typedef struct {
  int batch;
  const void* q;         /* [B][L][Hq][d] contiguous */
  kvc_dtype q_dtype;
  kvc_kv K, V;           /* [B][L][Hkv][cap][d] */
  const int32_t* len;    /* [B][L] device: valid rows of every (sequence, layer) */
  int max_len;           /* host upper bound on every len[b][l] */
  const float* R;        /* NULL: no bias; else R(b,l,g,i) = R[b*R_s_batch + l*R_s_layer + g*R_s_head + i] */
  int64_t R_s_batch, R_s_layer, R_s_head;
  float alpha_c;
  float scale;           /* 0 selects 1/sqrt(head_dim) */
  float* o;              /* [B][L][Hq][d] fp32 (required) */
  float* lse;            /* optional: natural-log sum-exp of the biased logits of (b, l, h) at
                            lse[((b*L + l)*Hq + h) * lse_stride] (see lse_stride, last field) */

  /* RECAS probe: enabled when K_full.ptr != NULL. */
  kvc_kv K_full, V_full; /* [B][L][Hkv][cap_full][d] */
  const int32_t* len_full; /* [B][L] device */
  int max_len_full;
  const uint32_t* kept_bits; /* bit i of word i/32 set if position i is kept */
  int64_t bits_s_batch, bits_s_layer, bits_s_head; /* strides in 32-bit words */
  float* delta;          /* [B][L][Hq] */
  float* vmax;           /* [B][L][Hkv] */
  float* err;            /* [B][L][Hq] */
  float* bound;          /* [B][L][Hq] */
  float* o_full;         /* optional [B][L][Hq][d] */
  float* o_kept;         /* optional [B][L][Hq][d] */
  int64_t lse_stride;    /* elements between consecutive (b, l, h) entries of lse; 0 or 1: a
                            contiguous [B][L][Hq] array; W: one slot of a [B][L][Hq][W] ring,
                            as kvc_recompress's win_lse reads it */
} kvc_decode_args;

/* ------------------------------------------------------------------------
 * kvc_recompress: decode-time periodic compression of a batch of caches.
 *
 * [InfoKV] Technical details: compression is also applied during decoding,
 * e.g. every 1024 generated tokens.  For every sequence, rescore the len
 * cached tokens with the last W generated queries (Qring, positions qpos) and
 * the stored per-token H and D (InfoKV score), keep floor(rho * t) of them
 * (t = prompt + generated length) with the recent window, and gather K, V,
 * pos, H and D into the destination buffers.  All rows of every sequence
 * hold the same count (len before, k after).
 * ---------------------------------------------------------------------- */
typedef struct {
  int batch;
  int len;               /* cached rows per (b, l, g) now */
  int t;                 /* current total length of every sequence */
  double rho;
  int w;
  float alpha, tau, scale;
  kvc_sel_mode sel_mode;
  int W;
  const void* Qring;     /* [B][L][Hq][W][d], dtype of K */
  const int32_t* qpos;   /* [B][W] positions of those queries */
  kvc_kv K, V;           /* source caches [B][L][Hkv][*][d] */
  const int32_t* pos;    /* [B][L][Hkv] rows of side_s_row elements */
  const float* H;
  const float* D;
  int64_t side_s_row;
  kvc_kv K_dst, V_dst;   /* destination caches (must not overlap the sources) */
  int32_t* pos_dst;
  float* H_dst;
  float* D_dst;
  int64_t side_dst_s_row;
  const float* U;        /* optional RECAS attention history (kvc_sparse_decode's acc), a side */
  float* U_dst;          /* array like H and D: given together, compacted with the rows */
  int cap_dst;           /* destination capacity per row, >= floor(rho * t) */
  int32_t* k_out;        /* optional [B][L] */
  /* Optional RECAS kept-position mask of the full history ([RECAS] 2.B), rebuilt from
   * pos_dst: row (b, l, g) of kept_bits_dst (word strides below, bits_words words per
   * row) is cleared, then bit p of word p/32 is set for every kept position p.  A kept
   * position at or past 32 * bits_words sets the status word (KVC_ERR_DEVICE). */
  uint32_t* kept_bits_dst;
  int64_t bits_s_batch, bits_s_layer, bits_s_head;
  int bits_words;
  int* host_kept;        /* optional HOST pointer: receives the rows every cache row holds
                            after the call (written before the call returns); -1 when the
                            RECAS controller below sets the budget on the device */
  /* Optional RECAS adaptive budget ([RECAS] 2.B), when recas_state != NULL: every row keeps
   * B_t = the largest need kvc_recas_control finds with k0 = floor(rho * t) (clamped as
   * above) and eps = recas_eps, instead of k0.  The budget is known on the device only:
   * k_out is required (it receives B_t), cap_dst must be >= len.  recas_x (optional,
   * [B][L][Hkv]) receives the predictor x of every row's new kept set. */
  const struct kvc_recas_cal_s* recas_state;   /* [B][L] */
  float recas_eps;
  float* recas_x;
  int recas_k_max;       /* largest budget the controller may choose (memory limit); <= 0: len.
                            Never below floor(rho * t). */
  /* Optional [B][L][Hq][W], slot-aligned with Qring: the natural-log sum-exp that each window
   * query's own decode step computed over this cache (kvc_decode_attn with lse at that slot,
   * lse_stride = W, no bias).  A window row's softmax runs over the keys at or before its
   * position; none of them has left the cache since its decode step (recompression is
   * periodic and the window is shorter than the period) and the keys appended after it are
   * masked, so its max and sum over the cache are the ones that step found.  When given, the
   * first pass of the window attention (those statistics) is not recomputed: A_i is formed
   * in one pass from exp(q k_i * scale - lse).  NULL: both passes run. */
  const float* win_lse;
} kvc_recompress_args;

/* ------------------------------------------------------------------------
 * RECAS calibrated dropped-mass estimator and adaptive budget ([RECAS] 2.B).
 *
 * The page: after eviction the exact full-cache attention is unavailable, so the
 * dropped attention mass delta is estimated from a normalised predictor that is
 * recalibrated at periodic full-attention probe steps, with a conservative upper
 * estimate from the empirical (1 - alpha)-quantile of the residuals; when that upper
 * estimate threatens the error target eps, the cache budget grows, keeping tokens in
 * utility order, until the bound holds.  Readings:
 *   predictor  x = share of the compression's window attention A on the tokens it
 *              drops: x = 1 - sum_kept A / sum_all A, per (sequence, layer, KV head);
 *   calibrate  per (sequence, layer) at a probe step (delta of every query head from
 *              kvc_decode_attn's probe): residuals r_h = delta_h - c x_{h/G}, c the
 *              ratio sum delta / sum x of the earlier probes (1 before any), kept in a
 *              ring of the last KVC_RECAS_RING; then c is updated and
 *              q = the ceil((m + 1)(1 - alpha))-th smallest of the m ring residuals
 *              (+inf while that rank exceeds m).  delta_hat = c x, delta_bar = c x + q;
 *   control    a row needs the smallest k >= k0 whose kept set (recent window plus the
 *              top k - w by the utility S, ties to the lower position; the union score
 *              max over KV heads in GQA-union mode) leaves c x(k) + q <= eps, the
 *              whole row if none; the budget B_t is the largest need of all rows.
 * ---------------------------------------------------------------------- */
/* ------------------------------------------------------------------------
 * kvc_sparse_decode: RECAS dynamic sparse decoding attention ([RECAS] 2.C, with the
 * utility of 2.A and the cost model of 2.D).  Inside the retained cache a query-aware
 * selector keeps the top K_t of a sparse score; only they take part in the step's
 * attention, the others stay cached.  Readings, per (sequence, layer, KV head) row of
 * n = len[b][l] cached tokens:
 *   tr_i    = attention of token i under the current query, averaged over the G query
 *             heads of the KV head (softmax over the row, scale 1/sqrt(d));
 *   hi_i    = acc_i / cnt_i: acc_i the attention the token received at the steps it has
 *             been cached (mean over the heads; 0 where it was inactive), cnt_i =
 *             t_cur - max(pos_i, n_prompt) those steps, this one included;
 *   sigma_i = a_tr tr_i + b_hi hi_i (the stage term gi is out of scope);
 *   active  = the top K_t = ceil(kappa n) (clamped to [1, n]) by sigma, ties to the lower
 *             position;
 *   o       = attention renormalised over the active set (each head), and
 *             acc_i += its mean over the heads, for the active i.
 * bf16 queries and caches, head_dim 128, G <= 8, max_len <= 16384.
 * ---------------------------------------------------------------------- */
typedef struct {
  int batch;
  const void* q;         /* [B][L][Hq][128] contiguous */
  kvc_dtype q_dtype;
  kvc_kv K, V;           /* retained caches [B][L][Hkv][cap][128] bf16 */
  const int32_t* len;    /* [B][L] device */
  int max_len;           /* host bound on every len */
  const int32_t* pos;    /* original positions, [B][L][Hkv] rows of side_s_row */
  float* acc;            /* accumulated attention, same layout; updated */
  int64_t side_s_row;
  int t_cur;             /* sequence length after this step's token was appended */
  int n_prompt;          /* prompt length (tokens below it count their steps from decode start) */
  double kappa;          /* active share, 0 < kappa <= 1 (double: ceil(kappa n) must be exact) */
  float a_tr, b_hi;
  float scale;           /* 0 selects 1/sqrt(head_dim) */
  float* o;              /* [B][L][Hq][128] fp32 out */
  int32_t* active;       /* optional [B][L][Hkv][max_len]: the active positions, ascending */
  int32_t* n_active;     /* optional [B][L][Hkv]: K_t */
  float* lse;            /* optional: natural-log sum-exp of q k * scale of (b, l, h) over the
                            whole retained cache (not only the active set) at
                            lse[((b*L + l)*Hq + h) * lse_stride], as kvc_decode_attn writes it */
  int64_t lse_stride;    /* 0 or 1: contiguous [B][L][Hq]; W: one slot of kvc_recompress's win_lse ring */
} kvc_sparse_decode_args;

#define KVC_RECAS_RING 256

/* Calibration state of one (sequence, layer).  Zeroed memory is the initial state
 * (c = 1, q = +inf).  c and q are derived fields, kept for readers. */
typedef struct kvc_recas_cal_s {
  double sum_delta, sum_x;   /* over every probe so far */
  double c, q;
  int32_t count;             /* residuals pushed so far */
  int32_t head;              /* next ring slot */
  double ring[KVC_RECAS_RING];
} kvc_recas_cal;

typedef struct {
  int batch;
  const float* delta;        /* [B][L][Hq] exact dropped mass of this probe step */
  const float* x;            /* [B][L][Hkv] predictors of the current kept sets */
  float alpha;               /* the bound aims to cover 1 - alpha; 0 < alpha < 1 */
  kvc_recas_cal* state;      /* [B][L], updated */
  float* delta_hat;          /* optional [B][L][Hkv]: c x after the update */
  float* delta_bar;          /* optional [B][L][Hkv]: c x + q after the update */
} kvc_recas_calibrate_args;

typedef struct {
  kvc_sel_mode sel_mode;     /* per KV head, or the GQA union score */
  int batch;
  int n;                     /* tokens per row, 1 .. 16384 */
  int w;                     /* recent window */
  int k0;                    /* base budget */
  const float* S;            /* utility: S(b,l,g,i) = S[((b*L + l)*Hkv + g)*s_row + i] */
  const float* A;            /* window attention, same layout (A >= 0) */
  int64_t s_row;             /* >= n */
  const kvc_recas_cal* state;  /* [B][L] */
  float eps;                 /* target on the dropped mass */
  int32_t* need;             /* [B][L][Hkv] out: each row's need */
  int32_t* budget;           /* optional, one int32 out: the largest need, at most k_max */
  int k_max;                 /* memory limit of the budget; <= 0: n */
} kvc_recas_control_args;

/* ------------------------------------------------------------------------
 * kvc_append: one generated token enters every (sequence, layer, KV head) cache row.
 *
 * [InfoKV] Technical details (decode-time compression): the token is cached with
 * the signals it is rescored with at the next compression (its position, H and D)
 * and its query joins the window of the last W generated queries.  [SelKV]
 * Methodology / Core component 2: an appended token is not merged, R = 1.
 * [RECAS] 2.B: its position is marked kept in the probe's bit mask.
 *
 * Row (b, l, g) receives k(b,l,g,:) and v(b,l,g,:) at row index len[b][l] of K and V;
 * then len[b][l] is incremented on the device.  A row already holding cap rows is
 * not written; the status word records it (KVC_ERR_DEVICE from kvc_check_status).
 * ---------------------------------------------------------------------- */
typedef struct {
  int batch;
  int cap;               /* rows each cache row can hold */
  const void* k;         /* [B][L][Hkv][d] contiguous, dtype of K */
  const void* v;         /* [B][L][Hkv][d] contiguous, dtype of K */
  kvc_kv K, V;           /* caches [B][L][Hkv][cap][d], one dtype */
  int32_t* len;          /* [B][L] device: rows in use, incremented */
  int pos;               /* original position of the appended token (every sequence) */
  /* optional side arrays, [B][L][Hkv] rows of side_s_row elements (NULL: skipped) */
  int32_t* side_pos;     /* receives pos */
  float* side_H;         /* receives H_new[b] */
  float* side_D;         /* receives D_new[b*D_new_s_batch + l*D_new_s_layer] */
  float* side_R;         /* receives 1 */
  float* side_U;         /* receives 0: the RECAS attention history of a new token */
  int64_t side_s_row;
  const float* H_new;    /* [B] device (with side_H) */
  const float* D_new;    /* device (with side_D) */
  int64_t D_new_s_batch, D_new_s_layer;
  uint32_t* kept_bits;   /* optional: bit pos of word pos/32 of every row is set */
  int64_t bits_s_batch, bits_s_layer, bits_s_head;   /* word strides */
  int bits_words;        /* words per row; pos / 32 must be below it */
  /* optional window-query ring: Qring[b][l][h][slot][:] = q[b][l][h][:], qpos[b][slot] = pos */
  const void* q;         /* [B][L][Hq][d] contiguous, dtype of K */
  void* Qring;           /* [B][L][Hq][W][d] contiguous */
  int32_t* qpos;         /* [B][W] */
  int W, slot;
  /* optional second cache that receives the same k and v rows (e.g. the full history the
   * RECAS probe reads), in the same launch: row (b, l, g) of K2 / V2 at row len2[b][l], then
   * len2[b][l] is incremented.  No side arrays, bits or ring go with it.  K2, V2 and len2
   * go together (NULL K2.ptr: no second cache); K2 / V2 have K's dtype and head_dim and
   * hold cap2 rows.  A row at capacity in either cache leaves both caches of that
   * (sequence, layer) unwritten and the status word records it. */
  kvc_kv K2, V2;         /* [B][L][Hkv][cap2][d] */
  int32_t* len2;         /* [B][L] device */
  int cap2;
} kvc_append_args;

/* ------------------------------------------------------------------------
 * kvc_lmhead_entropy: the entropy signal H_i of [InfoKV] Methodology (the top-k
 * restricted entropy of the final layer's predictive distribution, k = 256 there)
 * computed from the LM head's input, without writing the logits:
 *   z_i = W x_i                 logits of position i (bf16 products, fp32 sums)
 *   H_i = -sum_j p_j log p_j    p = softmax over the k largest entries of z_i
 * Where the logits are already in memory, kvc_score's entropy pass computes the same
 * H_i from them.
 *   x  [n][Dh] bf16, rows x_stride elements apart: the LM head's input at every
 *      position (the final hidden state after the model's last normalisation)
 *   W  [V][Dh] bf16, rows W_stride elements apart: the output projection
 *   H  [n] fp32 out
 * Requirements: 1 <= k <= 256; x and W 16-byte aligned; strides >= Dh and multiples
 * of 8 elements; finite inputs.  The workspace (kvc_workspace_size with
 * KVC_OP_LMHEAD_ENTROPY; the model argument may be NULL) holds per-row candidate
 * lists, about n * 2 * S * k * 4 bytes for S (<= 1024 / k) vocabulary segments plus
 * 512 KB per SM.  Errors: KVC_ERR_ARG / KVC_ERR_UNSUPPORTED for arguments outside
 * these limits, KVC_ERR_WORKSPACE for a short workspace (nothing is launched);
 * a bounded device wait that runs out sets KVC_ERR_TIMEOUT in the status word.
 * ---------------------------------------------------------------------- */
typedef struct {
  int n, Dh, V, k;
  kvc_dtype dtype;       /* KVC_BF16 */
  const void* x;
  int64_t x_stride;
  const void* W;
  int64_t W_stride;
  float* H;
} kvc_lmhead_entropy_args;

/* Operation ids for kvc_workspace_size. */
enum { KVC_OP_SCORE = 0, KVC_OP_SELECT = 1, KVC_OP_COMPACT = 2, KVC_OP_MERGE = 3,
       KVC_OP_DECODE = 4, KVC_OP_RECOMPRESS = 5, KVC_OP_SPARSE_DECODE = 6, KVC_OP_LMHEAD_ENTROPY = 7 };

/* Bytes of workspace the operation needs for these arguments (args points to
 * the operation's argument struct).  0 is a valid answer. */
kvc_status kvc_workspace_size(int op, const kvc_model* m, const void* args, size_t* bytes);

kvc_status kvc_score(const kvc_model* m, const kvc_score_args* a, void* ws, size_t ws_bytes,
                     kvc_stream_t stream);
kvc_status kvc_select(const kvc_model* m, const kvc_select_args* a, void* ws, size_t ws_bytes,
                      kvc_stream_t stream);
kvc_status kvc_compact(const kvc_model* m, const kvc_compact_args* a, kvc_stream_t stream);
kvc_status kvc_merge(const kvc_model* m, const kvc_merge_args* a, void* ws, size_t ws_bytes,
                     kvc_stream_t stream);
kvc_status kvc_rope_reposition(const kvc_model* m, const kvc_rope_args* a, kvc_stream_t stream);
kvc_status kvc_decode_attn(const kvc_model* m, const kvc_decode_args* a, void* ws, size_t ws_bytes,
                           kvc_stream_t stream);
kvc_status kvc_recompress(const kvc_model* m, const kvc_recompress_args* a, void* ws,
                          size_t ws_bytes, kvc_stream_t stream);
kvc_status kvc_append(const kvc_model* m, const kvc_append_args* a, kvc_stream_t stream);
kvc_status kvc_recas_calibrate(const kvc_model* m, const kvc_recas_calibrate_args* a, kvc_stream_t stream);
kvc_status kvc_recas_control(const kvc_model* m, const kvc_recas_control_args* a, kvc_stream_t stream);
kvc_status kvc_sparse_decode(const kvc_model* m, const kvc_sparse_decode_args* a, void* ws, size_t ws_bytes,
                             kvc_stream_t stream);
kvc_status kvc_lmhead_entropy(const kvc_lmhead_entropy_args* a, void* ws, size_t ws_bytes, kvc_stream_t stream);

/* ------------------------------------------------------------------------
 * kvc_decode_attn_noalloc: kvc_decode_attn for callers that cannot allocate.
 * The pages have no counterpart: this is an interface addition of the
 * library, not a step of the method.
 *
 * Some callers cannot call cudaMalloc and cannot pass a workspace - e.g. a
 * runtime that reserved all device memory up front for its own pool, or code
 * that must avoid the device-wide synchronisation cudaMalloc / cudaFree may
 * cause.  Same arguments and results as kvc_decode_attn, no workspace: the
 * split-K partial results live in a fixed 8 MiB array of this library's
 * device memory, held by every GPU that loads the library until exit.
 *   - The first call on a device looks up that array's device address (once
 *     per device, with the device current); make that first call before any
 *     stream capture.  Under CUDA's lazy module loading that lookup is also when
 *     the runtime first places the array in device memory: later calls take no
 *     device memory at all.
 *   - A call needing more scratch than 8 MiB (kvc_workspace_size with
 *     KVC_OP_DECODE reports the need) returns KVC_ERR_WORKSPACE and launches
 *     nothing.
 *   - All calls share the one array and it keeps the last call's contents;
 *     every value a call reads from it is written by that call first.  Calls
 *     that overlap on the GPU (unordered streams or threads) race on it.
 *   - Allocates nothing (no cudaMalloc / cudaFree, no allocating library call).
 * ---------------------------------------------------------------------- */
kvc_status kvc_decode_attn_noalloc(const kvc_model* m, const kvc_decode_args* a, kvc_stream_t stream);

/* Reads and clears the device status word of the current device after
 * synchronising `stream`.  Returns KVC_OK, KVC_ERR_TIMEOUT or KVC_ERR_DEVICE;
 * host_code (may be NULL) receives the raw word, an OR of: 1 = a bounded wait
 * ran out (KVC_ERR_TIMEOUT), 2 = an index or row count outside its bounds
 * (KVC_ERR_DEVICE), 4 = a merge target with zero attention (KVC_OK).
 *
 * The device addresses of the status word and of the no-alloc scratch are looked
 * up once per device ordinal and kept for the life of the process: after a
 * cudaDeviceReset of a device, unload and reload the library before using it on
 * that device again. */
kvc_status kvc_check_status(kvc_stream_t stream, uint32_t* host_code);

/* Message of the last failed call on this thread ("" if none). */
const char* kvc_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int kvc_version(void);

/* Number of GPU kernels this library has launched in this process, all
 * devices and threads together (a host-side counter incremented at every
 * launch the library issues; monotonic, never reset). */
uint64_t kvc_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* KVC_H */
