// Parameter blocks and launcher entry points shared by the C ABI (api.cu)
// and the kernel translation units.
#pragma once
#include "common.cuh"
#include "window.cuh"

namespace kvc {

// Host-side tally of the kernels the library launches (kvc_launch_count).
void count_launch(int n = 1);

struct CompactParams {
  int L, Hkv, n, k_cap, vr;                 // vr = 16-byte vectors per row
  const char* sK; int64_t sKl, sKh, sKt;    // byte strides
  const char* sV; int64_t sVl, sVh, sVt;
  char* dK; int64_t dKl, dKh, dKt;
  char* dV; int64_t dVl, dVh, dVt;
  const int32_t* idx;
  const int32_t* k;
  const int32_t* spos; int64_t psl, psh; int32_t* dpos;
  const float* sH; int64_t Hsl, Hsh; float* dH;
  const float* sD; int64_t Dsl, Dsh; float* dD;
  const float* sU; int64_t Usl, Ush; float* dU;   // RECAS attention history
  int64_t dside_row;                        // elements between (l, g) rows of dpos/dH/dD/dU
  unsigned* status;
};

struct MergeParams {
  int L, Hkv, n, d, bucket, nbuckets, k_cap;
  const void* V; int64_t Vsl, Vsh, Vst;     // element strides
  int bf16;
  const float* A; int64_t Asl, Ash;
  const int32_t* idx;
  const int32_t* k;
  void* dV; int64_t dVl, dVh, dVt; int dbf16;
  float* R;
  float* dVf;                               // optional fp32 copy [L][Hkv][k_cap][d]
  unsigned* status;
};

// RoPE re-positioning: row j of (l, g), j < k_l, turned from position pos(l,g,j) to
// new0 + j.  theta holds the d/2 rotary frequencies in fp64.
struct RopeParams {
  int L, Hkv, d, k_cap, bf16;
  const char* src; int64_t sl, sh, st;      // byte strides
  char* dst; int64_t dl, dh, dt;
  const int32_t* pos; int64_t pos_row;      // elements between (l, g) rows of pos / pos_dst
  int32_t* pos_dst;
  const int32_t* k;
  int64_t new0;
  double theta[64];
  unsigned* status;
};

struct DecodeParams {
  int B, L, Hq, Hkv, G, d;
  const void* q; int qbf16;
  const char* K; int64_t Ksb, Ksl, Ksh, Kst;  // byte strides
  const char* V; int64_t Vsb, Vsl, Vsh, Vst;
  const int32_t* len;
  int max_len;                  // host bound: rows past it are never read
  unsigned* status;
  const float* R; int64_t Rsb, Rsl, Rsh;
  float alpha_c;
  float qscale;                 // scale * log2(e)
  const uint32_t* bits; int64_t bsb, bsl, bsh;   // probe only
  int nsplit, split_len;
  float* part;                  // [rows][nsplit][G][rec]
};

struct CombineParams {
  int rows, nsplit, G, d, Hkv, L, Hq;
  const float* part;
  float* o; float* lse; int64_t lse_stride;
  float* delta; float* vmax; float* err; float* bound; float* o_full; float* o_kept;
};

// One decode step's append: row len[b][l] of every (b, l, g) cache row, byte strides.
struct AppendParams {
  int B, L, Hq, Hkv, cap, vr;               // vr = 16-byte vectors per row
  int64_t row_bytes;                        // bytes of one head_dim row
  const char* k; const char* v;             // [B][L][Hkv][d]
  char* K; int64_t Ksb, Ksl, Ksh, Kst;
  char* V; int64_t Vsb, Vsl, Vsh, Vst;
  int32_t* len;                             // [B][L]
  int pos;
  int32_t* spos; float* sH; float* sD; float* sR; float* sU; int64_t side_row;
  const float* H_new;                       // [B]
  const float* D_new; int64_t Dnb, Dnl;
  uint32_t* bits; int64_t bsb, bsl, bsh;    // word strides
  const char* q; char* Qring; int32_t* qpos; int W, slot;
  char* K2; int64_t K2sb, K2sl, K2sh, K2st;  // optional second cache (nullptr: none)
  char* V2; int64_t V2sb, V2sl, V2sh, V2st;
  int32_t* len2; int cap2;
  unsigned* status;
};

cudaError_t launch_append(const AppendParams& p, cudaStream_t st);

// RECAS dynamic sparse decode (bf16 caches, head_dim 128, G <= 8); byte strides.
constexpr int SPARSE_CHUNK = 256;           // keys per score block (one head-statistics partial each)
struct SparseParams {
  int B, L, Hq, Hkv, G, max_len;
  const void* q; int qbf16;                 // [B][L][Hq][128]
  const char* K; int64_t Ksb, Ksl, Ksh, Kst;
  const char* V; int64_t Vsb, Vsl, Vsh, Vst;
  const int32_t* len;                       // [B][L]
  const int32_t* pos; float* acc; int64_t side_row;   // [B][L][Hkv] rows
  int t_cur, n_prompt;
  double kappa;
  float a_tr, b_hi, scale;
  float* s;                                 // [rows][G][max_len]
  float* hstat;                             // [rows][key chunks][8 heads][2]: max, sum exp
  int32_t* kt;                              // [B * L]
  int32_t* active;                          // [rows][max_len] or NULL: the active positions
  int32_t* n_active;                        // [rows] or NULL
  float* o;                                 // [B][L][Hq][128]
  float* lse; int64_t lse_stride;           // or NULL: each head's log-sum-exp over the whole row
};

cudaError_t launch_sparse_decode(const SparseParams& p, cudaStream_t st);

// Top-k entropy from the LM head's input (bf16 x [n][Dh], W [V][Dh]; element strides).
struct LmheadParams {
  int n, Dh, V, k;
  const void* x;
  int64_t x_stride;
  const void* W;
  int64_t W_stride;
  float* H;
};
struct LmPlan {
  int S, tps, ntn, grid;
  int64_t total;
  size_t scratch_bytes, lists_bytes, counts_bytes, bytes;
};
LmPlan plan_lmhead(int n, int Dh, int V, int k, int sms);
cudaError_t launch_lmhead_entropy(const LmheadParams& p, void* ws, cudaStream_t st);

struct RecasCalParams {
  int BL, Hq, Hkv, G;
  const float* delta;                       // [BL][Hq]
  const float* x;                           // [BL][Hkv]
  double alpha;
  kvc_recas_cal* state;                     // [BL]
  float* delta_hat; float* delta_bar;       // [BL][Hkv] or NULL
};

struct RecasCtlParams {
  int rows, Hkv, n, w, k0, np2, union_mode;
  const float* S; const float* A; int64_t s_row;
  const kvc_recas_cal* state;               // [rows / Hkv]
  float eps;
  int32_t* need;                            // [rows]
};

cudaError_t launch_recas_calibrate(const RecasCalParams& p, cudaStream_t st);
cudaError_t launch_recas_control(const RecasCtlParams& p, cudaStream_t st);
cudaError_t launch_recas_budget(const int32_t* need, int rows, int k_max, int32_t* budget, int32_t* k, int nk,
                                int32_t* k2, int nk2, cudaStream_t st);
cudaError_t launch_recas_predictor(const float* A, int64_t s_row, int n, const int32_t* idx, int k_cap,
                                   const int32_t* k, int rows, int Hkv, float* x, cudaStream_t st);
cudaError_t launch_kept_bits(const int32_t* pos, int64_t pos_row, const int32_t* k, int k_cap, int B, int L,
                             int Hkv, uint32_t* bits, int64_t bsb, int64_t bsl, int64_t bsh, int words,
                             cudaStream_t st);
// sms: SMs the launch may fill (0: all of them), when another kernel runs beside it.
cudaError_t launch_entropy(const void* logits, kvc_dtype dt, int64_t rows, int64_t V,
                           int64_t row_stride, int k, float* H, cudaStream_t st, int sms = 0);
// The same entropy for a few long rows, each cut into chunks spread over the GPU: bytes
// of candidate workspace it needs (0: the row count or shape is not one it takes), and the
// launch, which needs 16-byte aligned rows.
size_t entropy_split_ws(int64_t rows, int64_t V, kvc_dtype dt, int k);
cudaError_t launch_entropy_split(const void* logits, kvc_dtype dt, int64_t rows, int64_t V,
                                 int64_t row_stride, int k, float* cand, float* H, cudaStream_t st);
cudaError_t launch_repr(const void* hidden, kvc_dtype dt, int L, int64_t n, int Dh, float tau,
                        float* D, cudaStream_t st, int sms = 0);
cudaError_t launch_combine(const float* A, const float* H, int64_t Hsl, int64_t Hsh, const float* D,
                           int64_t Dsl, int64_t Dsh, const float* stats, int n, int L, int Hkv, float alpha,
                           float* S, cudaStream_t st);
// E = D * H statistics of every (layer, KV head) row: [L*Hkv][3] max, sum exp(E - max), mean;
// part is a workspace of estats_ws(n, L, Hkv) bytes (per-chunk partials)
size_t estats_ws(int n, int L, int Hkv);
cudaError_t launch_estats(const float* H, int64_t Hsl, int64_t Hsh, const float* D, int64_t Dsl,
                          int64_t Dsh, int n, int L, int Hkv, float* stats, float* Ebar, double* part,
                          cudaStream_t st);
size_t window_ffma_smem_max(int R, int d);
bool window_tc_supported(const WinParams& p, kvc_dtype dt);
cudaError_t launch_window_tc(const WinParams& p, cudaStream_t st);
cudaError_t launch_budget(int mode, int L, int n, int w, double rho, const int32_t* k_in,
                          long long B, const float* Ebar, int32_t* k_out, cudaStream_t st);
// n_l (optional, [L]): each layer's rows hold only n_l[l] <= n tokens (row stride n)
cudaError_t launch_select(const float* S, int64_t Ssl, int64_t Ssh, int L, int Hkv, int n, int w,
                          int union_mode, const int32_t* k_l, int32_t* idx, int k_cap,
                          uint32_t* keys_ws, cudaStream_t st, const int32_t* n_l = nullptr);
cudaError_t launch_compact(const CompactParams& p, cudaStream_t st);
cudaError_t launch_merge(const MergeParams& p, cudaStream_t st);
cudaError_t launch_rope(const RopeParams& p, cudaStream_t st);
cudaError_t launch_decode(const DecodeParams& p, bool bf16, bool probe, const CombineParams& c,
                          cudaStream_t st);
int decode_rec_len(bool probe, int d);
// The persistent bulk-copy decode applies: bf16, head_dim 128, no probe, 16-byte
// aligned K / V bases and strides.
bool decode_tma_supported(const DecodeParams& p, bool bf16, bool probe);
// The tensor-core decode applies: bf16 K / V and q, head_dim 128, G <= 8, K / V
// layouts a 5-D TMA map can describe (16-byte multiple strides); for the probe, kept
// bits and no log R bias.
bool decode_mma_supported(const DecodeParams& p, bool bf16, bool probe);
cudaError_t launch_decode_mma(const DecodeParams& p, bool probe, cudaStream_t st);

}  // namespace kvc
