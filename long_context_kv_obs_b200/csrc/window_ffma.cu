// Window attention score on the CUDA cores (any dtype, head_dim 64 or 128).
// Used for fp32 caches and for shapes the tensor-core path does not cover.
#include "kernels.cuh"

namespace kvc {

constexpr int WF1_THREADS = 256;  // pass 1: one thread per window row
constexpr int WF1_KT = 32;        // keys per shared tile
constexpr int WF2_THREADS = 128;  // pass 2: one thread per key

template <typename T>
__device__ __forceinline__ const T* qrow(const WinParams& p, int l, int g, int r) {
  const int h = g * p.G + r / p.W, w = r % p.W;
  return reinterpret_cast<const T*>(p.Qw) + (((int64_t)l * p.Hq + h) * p.W + w) * p.d;
}

// Pass 1: per window row, max and sum-exp of the scaled logits over one key chunk.
template <typename T>
__global__ void __launch_bounds__(WF1_THREADS) win_pass1_ffma(WinParams p) {
  extern __shared__ float wf_smem[];
  const int d = p.d, dp = d + 1;
  float* Qs = wf_smem;                    // [R][d+1]
  float* Ks = wf_smem + (size_t)p.R * dp; // [KT][d]
  const int lg = blockIdx.x, l = lg / p.Hkv, g = lg % p.Hkv;
  const int c = blockIdx.y;
  const int i0 = c * p.chunk, i1 = min(p.n, i0 + p.chunk);
  for (int t = threadIdx.x; t < p.R * d; t += blockDim.x) {
    const int r = t / d, e = t % d;
    Qs[r * dp + e] = to_f(qrow<T>(p, l, g, r)[e]);
  }
  const T* Kb = reinterpret_cast<const T*>(p.K) + l * p.Ksl + g * p.Ksh;
  for (int r0 = 0; r0 < p.R; r0 += blockDim.x) {
    const int r = r0 + threadIdx.x;
    const bool active = r < p.R;
    const int qp = active ? query_pos(p, l, r % p.W) : 0;
    float m = -INFINITY, s = 0.f;
    for (int k0 = i0; k0 < i1; k0 += WF1_KT) {
      const int nk = min(WF1_KT, i1 - k0);
      __syncthreads();
      for (int t = threadIdx.x; t < nk * d; t += blockDim.x) {
        const int j = t / d, e = t % d;
        Ks[j * d + e] = to_f(Kb[(int64_t)(k0 + j) * p.Kst + e]);
      }
      __syncthreads();
      if (active) {
        for (int j = 0; j < nk; ++j) {
          if (key_pos(p, l, g, k0 + j) > qp) continue;
          float acc = 0.f;
          for (int e = 0; e < d; ++e) acc = fmaf(Qs[r * dp + e], Ks[j * d + e], acc);
          const float x = acc * p.scale;
          if (x > m) {
            s = s * expf(m - x) + 1.f;
            m = x;
          } else {
            s += expf(x - m);
          }
        }
      }
    }
    if (active) {
      float* o = p.part + (((int64_t)lg * p.nchunk + c) * p.R + r) * 2;
      o[0] = m;
      o[1] = s;
    }
  }
}

// Merge the chunk partials of every row: rowst = (max, 1 / sum-exp).
__global__ void win_rowstats_combine(WinParams p) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)p.L * p.Hkv * p.R;
  if (t >= total) return;
  const int64_t lg = t / p.R;
  const int r = (int)(t % p.R);
  float M = -INFINITY;
  for (int c = 0; c < p.nchunk; ++c) M = fmaxf(M, p.part[((lg * p.nchunk + c) * p.R + r) * 2]);
  float s = 0.f;
  for (int c = 0; c < p.nchunk; ++c) {
    const float* q = p.part + ((lg * p.nchunk + c) * p.R + r) * 2;
    if (q[0] > -INFINITY) s += q[1] * expf(q[0] - M);
  }
  p.rowst[t * 2 + 0] = M;
  p.rowst[t * 2 + 1] = s > 0.f ? 1.f / s : 0.f;
}

// Pass 2: one thread per key, sum of normalised probabilities over the rows; epilogue to S.
template <typename T>
__global__ void __launch_bounds__(WF2_THREADS) win_pass2_ffma(WinParams p) {
  extern __shared__ float wf_smem[];
  const int d = p.d, dp = d + 1;
  float* Qs = wf_smem;                              // [R][d]
  float* Ks = wf_smem + (size_t)p.R * d;            // [128][d+1]
  float* RS = Ks + (size_t)WF2_THREADS * dp;        // [R][2]
  int* QP = reinterpret_cast<int*>(RS + 2 * p.R);   // [R]
  const int lg = blockIdx.x, l = lg / p.Hkv, g = lg % p.Hkv;
  const int i0 = blockIdx.y * WF2_THREADS;
  for (int t = threadIdx.x; t < p.R * d; t += blockDim.x) {
    const int r = t / d, e = t % d;
    Qs[r * d + e] = to_f(qrow<T>(p, l, g, r)[e]);
  }
  for (int t = threadIdx.x; t < p.R; t += blockDim.x) {
    RS[2 * t] = p.rowst[((int64_t)lg * p.R + t) * 2];
    RS[2 * t + 1] = p.rowst[((int64_t)lg * p.R + t) * 2 + 1];
    QP[t] = query_pos(p, l, t % p.W);
  }
  const T* Kb = reinterpret_cast<const T*>(p.K) + l * p.Ksl + g * p.Ksh;
  const int nk = min(WF2_THREADS, p.n - i0);
  for (int t = threadIdx.x; t < nk * d; t += blockDim.x) {
    const int j = t / d, e = t % d;
    Ks[j * dp + e] = to_f(Kb[(int64_t)(i0 + j) * p.Kst + e]);
  }
  __syncthreads();
  const int j = threadIdx.x;
  if (j >= nk) return;
  const int i = i0 + j;
  const int kp = key_pos(p, l, g, i);
  float acc = 0.f;
  for (int r = 0; r < p.R; ++r) {
    if (kp > QP[r]) continue;
    float s = 0.f;
    for (int e = 0; e < d; ++e) s = fmaf(Qs[r * d + e], Ks[j * dp + e], s);
    acc += expf(s * p.scale - RS[2 * r]) * RS[2 * r + 1];
  }
  const float A = acc / (float)p.R;
  float vn = 0.f;
  if (p.mode == KVC_SCORE_VATP) {
    const T* v = reinterpret_cast<const T*>(p.V) + l * p.Vsl + g * p.Vsh + (int64_t)i * p.Vst;
    vn = row_norm(v, d);
  }
  const int64_t o = ((int64_t)l * p.Hkv + g) * p.n + i;
  if (p.A) p.A[o] = A;
  p.S[o] = score_from_A(p, l, g, i, A, vn);
}

// The row statistics from the log-sum-exp each window row's own decode step recorded over
// the same keys: max = lse, 1 / sum = 1, so pass 2's exp(s * scale - max) / sum is
// exp(s * scale - lse).  Row r of group g is query head g G + r / W at window slot r % W.
__global__ void win_rowstats_from_lse(const WinParams p) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)p.L * p.Hkv * p.R) return;
  const int64_t lg = idx / p.R;
  const int r = (int)(idx - lg * p.R);
  const int l = (int)(lg / p.Hkv), g = (int)(lg - (int64_t)l * p.Hkv);
  p.rowst[idx * 2] = p.wlse[((int64_t)l * p.Hq + g * p.G + r / p.W) * p.W + r % p.W];
  p.rowst[idx * 2 + 1] = 1.f;
}

cudaError_t launch_window_combine(const WinParams& p, cudaStream_t st) {
  const int64_t total = (int64_t)p.L * p.Hkv * p.R;
  if (p.wlse) win_rowstats_from_lse<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(p);
  else win_rowstats_combine<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_window_ffma(const WinParams& p, kvc_dtype dt, cudaStream_t st) {
  const size_t s1 = ((size_t)p.R * (p.d + 1) + (size_t)WF1_KT * p.d) * sizeof(float);
  const size_t s2 = ((size_t)p.R * p.d + (size_t)WF2_THREADS * (p.d + 1) + 3 * (size_t)p.R) * sizeof(float);
  dim3 g1(p.L * p.Hkv, p.nchunk), g2(p.L * p.Hkv, (p.n + WF2_THREADS - 1) / WF2_THREADS);
  if (dt == KVC_BF16) {
    cudaFuncSetAttribute(win_pass1_ffma<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
    cudaFuncSetAttribute(win_pass2_ffma<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
    if (!p.wlse) {
      win_pass1_ffma<__nv_bfloat16><<<g1, WF1_THREADS, s1, st>>>(p);
      count_launch();
    }
    launch_window_combine(p, st);
    win_pass2_ffma<__nv_bfloat16><<<g2, WF2_THREADS, s2, st>>>(p);
    count_launch();
  } else {
    cudaFuncSetAttribute(win_pass1_ffma<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
    cudaFuncSetAttribute(win_pass2_ffma<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
    if (!p.wlse) {
      win_pass1_ffma<float><<<g1, WF1_THREADS, s1, st>>>(p);
      count_launch();
    }
    launch_window_combine(p, st);
    win_pass2_ffma<float><<<g2, WF2_THREADS, s2, st>>>(p);
    count_launch();
  }
  return cudaGetLastError();
}

size_t window_ffma_smem_max(int R, int d) {
  const size_t s1 = ((size_t)R * (d + 1) + (size_t)WF1_KT * d) * sizeof(float);
  const size_t s2 = ((size_t)R * d + (size_t)WF2_THREADS * (d + 1) + 3 * (size_t)R) * sizeof(float);
  return s1 > s2 ? s1 : s2;
}

}  // namespace kvc
