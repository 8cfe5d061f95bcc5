// Observation-window attention score A and the combined score S: shared
// parameters and epilogue for the FFMA and tensor-core implementations.
//
// [InfoKV] Methodology / Technical details:
//   A_i = mean over the G*W window rows of softmax_causal(q k^T * scale)_i
//   S_i = alpha * A_i + (1 - alpha) * Softmax(E)_i,   E_i = D_i * H_i
// [SelKV] Pipeline overview step 1 (VATP): S_i = A_i * ||v_i||_2.
//
// Two passes over the keys of each (layer, KV head): pass 1 gives every window
// row its max and sum-exp over all visible keys, pass 2 sums the normalised
// probabilities of each key over the rows.
#pragma once
#include "common.cuh"

struct CUtensorMap_st;   // cuda.h's tensor map

namespace kvc {

struct WinParams {
  int L, Hq, Hkv, G, d, n, W, R;  // R = G * W window rows per KV head
  const void* Qw;                 // [L][Hq][W][d]
  const void* K;
  int64_t Ksl, Ksh, Kst;
  const void* V;
  int64_t Vsl, Vsh, Vst;
  const int32_t* kpos;
  int64_t kpsl, kpsh;
  const int32_t* qpos;            // [W] (or [L / qlpb][W] rows) or NULL
  int qlpb;                       // layers per qpos row (0: one row for every layer)
  float scale;
  int mode;
  float alpha;
  const float* H;
  int64_t Hsl, Hsh;
  const float* D;
  int64_t Dsl, Dsh;
  const float* estats;            // [L*Hkv][3] max, sum-exp, mean of E
  float* A;                       // [L][Hkv][n] or NULL
  float* S;                       // [L][Hkv][n]
  float* part;                    // pass-1 partials [L*Hkv][nchunk][R][2]
  float* rowst;                   // [L*Hkv][R][2]: row max (scaled logit units), 1 / sum-exp
  const float* wlse;              // [L][Hq][W]: each window row's log-sum-exp, recorded by its decode
                                  // step; given, pass 1 is skipped and rowst = (lse, 1). NULL: computed
  float* vnorm;                   // [L][Hkv][n] value norms (VATP, tensor-core path)
  int nchunk, chunk;
  // single-launch tensor-core path
  float2* fpart;                  // pass-1 partials (log2 max, sum): [L*Hkv][nchunk][128] per chunk,
                                  // then [L*Hkv][ngroups][128] per group of 8 chunks
  float* frowc;                   // [L*Hkv][128] negated row constants -(log2 max + log2 sum)
  int* fsync;                     // ready flags [L*Hkv], finished groups [L*Hkv],
                                  // finished chunks [L*Hkv][ngroups]
  int fchunk;                     // keys per work item
  uint64_t flag_wait_ns;          // single launch: limit of the cross-CTA wait (0: the default)
};

constexpr int WIN_FUSED_NB = 4;       // epilogue warpgroups of the single-launch kernel
constexpr int WIN_FUSED_CHUNK = 1024; // keys per work item
#ifndef KVC_FU_LAG
#define KVC_FU_LAG 3
#endif
constexpr int WIN_FUSED_LAG = KVC_FU_LAG;   // slices between pass 1 and pass 2 of a slice
constexpr int WIN_FUSED_GROUP = 8;    // chunks per merge group

__device__ __forceinline__ int key_pos(const WinParams& p, int l, int g, int i) {
  return p.kpos ? p.kpos[l * p.kpsl + g * p.kpsh + i] : i;
}
// Position of window query w of layer l.
__device__ __forceinline__ int query_pos(const WinParams& p, int l, int w) {
  if (!p.qpos) return p.n - p.W + w;
  return p.qpos[(p.qlpb ? l / p.qlpb : 0) * p.W + w];
}
// Smallest window-query position over every layer (a lower bound for one layer's).
__device__ __forceinline__ int query_pos_min(const WinParams& p) {
  if (!p.qpos) return p.n - p.W;
  const int rows = p.qlpb ? (p.L + p.qlpb - 1) / p.qlpb : 1;
  int m = 0x7fffffff;
  for (int i = 0; i < rows * p.W; ++i) m = min(m, p.qpos[i]);
  return m;
}

template <typename T>
__device__ __forceinline__ float row_norm(const T* v, int d) {
  float s = 0.f;
  for (int e = 0; e < d; ++e) {
    const float x = to_f(v[e]);
    s = fmaf(x, x, s);
  }
  return sqrtf(s);
}

// S_i from A_i (mode-specific).  vnorm is only used in VATP mode.
__device__ __forceinline__ float score_from_A(const WinParams& p, int l, int g, int i, float A,
                                              float vnorm) {
  if (p.mode == KVC_SCORE_INFOKV) {
    const float* st = p.estats + 3 * (l * p.Hkv + g);
    const float E = p.D[l * p.Dsl + g * p.Dsh + i] * p.H[l * p.Hsl + g * p.Hsh + i];
    const float P = expf(E - st[0]) / st[1];
    return p.alpha * A + (1.f - p.alpha) * P;
  }
  if (p.mode == KVC_SCORE_VATP) return A * vnorm;
  return A;
}

cudaError_t launch_window_ffma(const WinParams& p, kvc_dtype dt, cudaStream_t st);

// Tensor-core paths (bf16 K, head_dim 128).  The K map is 4-D (dim, token, KV head,
// layer) with 64 x 128-token boxes, the Q map 2-D (dim, row) with 64 x QR boxes,
// both 128B-swizzled.
bool make_window_maps(const WinParams& p, int QR, ::CUtensorMap_st* mK, ::CUtensorMap_st* mQ);
cudaError_t launch_vnorm(const WinParams& p, cudaStream_t st);
bool window_fused_supported(const WinParams& p, kvc_dtype dt);
// grid: CTAs of the persistent launch (0: one per SM); S == NULL: A only.
cudaError_t launch_window_fused(const WinParams& p, cudaStream_t st, int grid = 0);
cudaError_t launch_window_combine(const WinParams& p, cudaStream_t st);

}  // namespace kvc
