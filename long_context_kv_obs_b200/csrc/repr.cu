// Layer-wise representation change and entropy-score statistics.
//
// [InfoKV] Methodology: D_i^(l) = 1 - cos(h_i^(l), h_i^(L)) (+ tau, Technical
// details), E_i^(l) = D_i^(l) * H_i, Softmax over the layer's tokens; the
// adaptive budget uses E-bar^(l), the layer's mean entropy score.
//
// repr: one warp per token stages h^(L) in shared memory (each lane reads back the
// 16-byte vectors it wrote) and streams the other layers' hidden rows of that token,
// one dot product and one norm per layer.  Keeping h^(L) out of registers fits two
// CTAs per SM, twice the rows in flight.  The hidden tensor is read exactly once.
// estats: one CTA per (layer, KV head) row reduces max, sum-exp and mean of E
// in double precision with a fixed tree (deterministic).
#include "kernels.cuh"

namespace kvc {

constexpr int REPR_WARPS = 8;
constexpr int REPR_MAXV = 16;   // 16-byte vectors per lane: Dh <= 4096 bf16 / 2048 fp32

template <typename T>
__global__ void __launch_bounds__(REPR_WARPS * 32, 2)
repr_kernel(const T* __restrict__ hidden, int L, int64_t n, int Dh, int vpl, float tau,
            float* __restrict__ D) {
  constexpr int EPV = Vec<T>::N;
  extern __shared__ uint4 repr_hl[];                 // h^(L) of each warp's token: [warps][vpl * 32]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4* hls = repr_hl + (size_t)warp * vpl * 32;
  const int64_t layer_stride = n * (int64_t)Dh;
  const int64_t nw = (int64_t)gridDim.x * REPR_WARPS;
  for (int64_t i = (int64_t)blockIdx.x * REPR_WARPS + warp; i < n; i += nw) {
    const T* hL = hidden + (int64_t)(L - 1) * layer_stride + i * Dh;
    float nL = 0.f;
#pragma unroll 4
    for (int v = 0; v < vpl; ++v) {
      const uint4 x = ld_stream16(hL + (v * 32 + lane) * EPV);
      hls[v * 32 + lane] = x;
      float f[EPV];
      Vec<T>::unpack(x, f);
#pragma unroll
      for (int e = 0; e < EPV; ++e) nL = fmaf(f[e], f[e], nL);
    }
    nL = warp_sum(nL);
    const float sL = sqrtf(nL);
    for (int l = 0; l < L - 1; ++l) {
      const T* hl = hidden + (int64_t)l * layer_stride + i * Dh;
      uint4 r[REPR_MAXV];
#pragma unroll
      for (int v = 0; v < REPR_MAXV; ++v)
        if (v < vpl) r[v] = ld_stream16(hl + (v * 32 + lane) * EPV);
      float dot = 0.f, nl = 0.f;
#pragma unroll
      for (int v = 0; v < REPR_MAXV; ++v) {
        if (v < vpl) {
          float a[EPV], b[EPV];
          Vec<T>::unpack(r[v], a);
          Vec<T>::unpack(hls[v * 32 + lane], b);   // each lane reads back what it wrote
#pragma unroll
          for (int e = 0; e < EPV; ++e) {
            dot = fmaf(a[e], b[e], dot);
            nl = fmaf(a[e], a[e], nl);
          }
        }
      }
      dot = warp_sum(dot);
      nl = warp_sum(nl);
      if (lane == 0) {
        const float den = sqrtf(nl) * sL;
        const float c = den > 0.f ? dot / den : 0.f;
        D[(int64_t)l * n + i] = 1.f - c + tau;
      }
    }
    if (lane == 0) {
      const float den = sL * sL;
      const float c = den > 0.f ? nL / den : 0.f;
      D[(int64_t)(L - 1) * n + i] = 1.f - c + tau;
    }
  }
}

// Few tokens (a decode step's batch), where a warp per token would leave most SMs idle:
// one warp per (token, layer) pair, every layer of a token read at once.  Each warp also
// reads h^(L) (from L2 after the first).  Every product is taken in repr_kernel's per-lane
// order and reduced by the same warp tree, so D is bit-identical to it.
// It is launched as a programmatic dependent of the kernel before it (it reads only the
// hidden states, which no library kernel writes), so it can run beside that kernel; every
// thread waits for that kernel's grid before exiting, so its own completion still implies
// that grid's, and a kernel after it sees both.
template <typename T>
__global__ void __launch_bounds__(REPR_WARPS * 32)
repr_pair_kernel(const T* __restrict__ hidden, int L, int64_t n, int Dh, int vpl, float tau,
                 float* __restrict__ D) {
  constexpr int EPV = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * REPR_WARPS + warp;
  if (w < n * L) {
    const int64_t i = w / L;
    const int l = (int)(w - i * L);
    const bool last = l == L - 1;
    const int64_t layer_stride = n * (int64_t)Dh;
    const T* hL = hidden + (int64_t)(L - 1) * layer_stride + i * Dh;
    const T* hl = hidden + (int64_t)l * layer_stride + i * Dh;
    uint4 b[REPR_MAXV], a[REPR_MAXV];
#pragma unroll
    for (int v = 0; v < REPR_MAXV; ++v) {
      if (v < vpl) {
        b[v] = ld_stream16(hL + (v * 32 + lane) * EPV);
        if (!last) a[v] = ld_stream16(hl + (v * 32 + lane) * EPV);
      }
    }
    float nL = 0.f;
#pragma unroll
    for (int v = 0; v < REPR_MAXV; ++v) {
      if (v < vpl) {
        float f[EPV];
        Vec<T>::unpack(b[v], f);
#pragma unroll
        for (int e = 0; e < EPV; ++e) nL = fmaf(f[e], f[e], nL);
      }
    }
    nL = warp_sum(nL);
    const float sL = sqrtf(nL);
    float c = 0.f;
    if (last) {
      const float den = sL * sL;
      c = den > 0.f ? nL / den : 0.f;
    } else {
      float dot = 0.f, nl = 0.f;
#pragma unroll
      for (int v = 0; v < REPR_MAXV; ++v) {
        if (v < vpl) {
          float x[EPV], y[EPV];
          Vec<T>::unpack(a[v], x);
          Vec<T>::unpack(b[v], y);
#pragma unroll
          for (int e = 0; e < EPV; ++e) {
            dot = fmaf(x[e], y[e], dot);
            nl = fmaf(x[e], x[e], nl);
          }
        }
      }
      dot = warp_sum(dot);
      nl = warp_sum(nl);
      const float den = sqrtf(nl) * sL;
      c = den > 0.f ? dot / den : 0.f;
    }
    if (lane == 0) D[(int64_t)l * n + i] = 1.f - c + tau;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

cudaError_t launch_repr(const void* hidden, kvc_dtype dt, int L, int64_t n, int Dh, float tau,
                        float* D, cudaStream_t st, int sms) {
  if (n <= 0) return cudaSuccess;
  const int epv = dt == KVC_BF16 ? 8 : 4;
  const int vpl = Dh / (32 * epv);
  const size_t smem = (size_t)REPR_WARPS * vpl * 32 * 16;
  int64_t want = (n + REPR_WARPS - 1) / REPR_WARPS;
  if (2 * want <= num_sms()) {   // fewer CTAs than half the SMs: spread the layers too
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((n * L + REPR_WARPS - 1) / REPR_WARPS));
    cfg.blockDim = dim3(REPR_WARPS * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    const cudaError_t e =
        dt == KVC_BF16
            ? cudaLaunchKernelEx(&cfg, repr_pair_kernel<__nv_bfloat16>, (const __nv_bfloat16*)hidden, L, n, Dh,
                                 vpl, tau, D)
            : cudaLaunchKernelEx(&cfg, repr_pair_kernel<float>, (const float*)hidden, L, n, Dh, vpl, tau, D);
    count_launch();
    return e;
  }
  int64_t maxb = (int64_t)(sms > 0 ? sms : num_sms()) * 8;
  const int grid = (int)(want < maxb ? want : maxb);
  if (dt == KVC_BF16) {
    cudaFuncSetAttribute(repr_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    repr_kernel<__nv_bfloat16><<<grid, REPR_WARPS * 32, smem, st>>>((const __nv_bfloat16*)hidden, L, n, Dh, vpl,
                                                                    tau, D);
  } else {
    cudaFuncSetAttribute(repr_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    repr_kernel<float><<<grid, REPR_WARPS * 32, smem, st>>>((const float*)hidden, L, n, Dh, vpl, tau, D);
  }
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// E = D * H statistics per (layer, KV head) row: max, sum exp(E - max), mean.
// ---------------------------------------------------------------------------
constexpr int EST_THREADS = 256;
constexpr int EST_PER = 16;                    // tokens per thread
constexpr int EST_CHUNK = EST_THREADS * EST_PER;   // tokens per CTA

__device__ __forceinline__ double block_reduce_sum_d(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_d(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double r = 0.0;
  if (warp == 0) {
    r = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0;
    r = warp_sum_d(r);
    if (lane == 0) red[0] = r;
  }
  __syncthreads();
  return red[0];
}

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float r = lane < (int)(blockDim.x >> 5) ? red[lane] : -INFINITY;
    r = warp_max(r);
    if (lane == 0) red[0] = r;
  }
  __syncthreads();
  return red[0];
}

// One chunk of EST_CHUNK tokens of a row per CTA, in one pass: the chunk's max, the sum of
// exp(e - that max) (fp32 terms, summed in fp64) and the sum of e (fp64).
__global__ void __launch_bounds__(EST_THREADS)
estats_part_kernel(const float* __restrict__ H, int64_t Hsl, int64_t Hsh, const float* __restrict__ D,
                   int64_t Dsl, int64_t Dsh, int n, int Hkv, double* __restrict__ part) {
  __shared__ double redd[32];
  __shared__ float redf[32];
  const int row = blockIdx.y, ch = blockIdx.x;
  const int l = row / Hkv, g = row % Hkv;
  const float* h = H + l * Hsl + g * Hsh;
  const float* dd = D + l * Dsl + g * Dsh;
  const int i0 = ch * EST_CHUNK, i1 = min(n, i0 + EST_CHUNK);
  float ev[EST_PER];
  float mx = -INFINITY;
  double sum = 0.0;
#pragma unroll
  for (int k = 0; k < EST_PER; ++k) {
    const int i = i0 + k * EST_THREADS + (int)threadIdx.x;
    ev[k] = i < i1 ? __ldg(dd + i) * __ldg(h + i) : -INFINITY;
    if (i < i1) {
      mx = fmaxf(mx, ev[k]);
      sum += (double)ev[k];
    }
  }
  mx = block_reduce_max(mx, redf);
  double se = 0.0;
#pragma unroll
  for (int k = 0; k < EST_PER; ++k)
    if (i0 + k * EST_THREADS + (int)threadIdx.x < i1) se += (double)expf(ev[k] - mx);
  se = block_reduce_sum_d(se, redd);
  sum = block_reduce_sum_d(sum, redd);
  if (threadIdx.x == 0) {
    double* o = part + ((int64_t)row * gridDim.x + ch) * 3;
    o[0] = mx;
    o[1] = se;
    o[2] = sum;
  }
}

// A row's statistics from its chunks, merged in chunk order: max, sum exp(E - max), mean.
// Partial row row / share (share rows read the same D and H: one partial row each).
__global__ void estats_merge_kernel(const double* __restrict__ part, int rows, int share, int nch, int n,
                                    float* __restrict__ stats) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= rows) return;
  const double* p = part + (int64_t)(row / share) * nch * 3;
  double M = -INFINITY;
  for (int c = 0; c < nch; ++c) M = fmax(M, p[3 * c]);
  double se = 0.0, sum = 0.0;
  for (int c = 0; c < nch; ++c) {
    se += p[3 * c + 1] * exp(p[3 * c] - M);
    sum += p[3 * c + 2];
  }
  stats[3 * row + 0] = (float)M;
  stats[3 * row + 1] = (float)se;
  stats[3 * row + 2] = (float)(sum / n);
}

// Ebar[l] = mean over KV heads of the rows' mean E.
__global__ void ebar_kernel(const float* __restrict__ stats, int L, int Hkv, float* __restrict__ Ebar) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l >= L) return;
  double s = 0.0;
  for (int g = 0; g < Hkv; ++g) s += stats[3 * (l * Hkv + g) + 2];
  Ebar[l] = (float)(s / Hkv);
}

// S = alpha * A + (1 - alpha) * Softmax(E), E = D * H, from the window attention A and the
// row statistics of E: the InfoKV combination when A was computed beside the signals
// rather than after them.  Same expression as the fused window epilogue.
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ A, const float* __restrict__ H, int64_t Hsl, int64_t Hsh,
               const float* __restrict__ D, int64_t Dsl, int64_t Dsh, const float* __restrict__ stats,
               int n, int Hkv, float alpha, float* __restrict__ S) {
  const int row = blockIdx.y;
  const int l = row / Hkv, g = row % Hkv;
  const float* h = H + l * Hsl + g * Hsh;
  const float* dd = D + l * Dsl + g * Dsh;
  const float mx = stats[3 * row + 0], se = stats[3 * row + 1];
  const int64_t o = (int64_t)row * n;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float pre = __ldg(dd + i) * __ldg(h + i);
    S[o + i] = alpha * __ldg(A + o + i) + (1.f - alpha) * (expf(pre - mx) / se);
  }
}

cudaError_t launch_combine(const float* A, const float* H, int64_t Hsl, int64_t Hsh, const float* D,
                           int64_t Dsl, int64_t Dsh, const float* stats, int n, int L, int Hkv, float alpha,
                           float* S, cudaStream_t st) {
  const int bx = (int)((n + 1023) / 1024);
  combine_kernel<<<dim3(bx, L * Hkv), 256, 0, st>>>(A, H, Hsl, Hsh, D, Dsl, Dsh, stats, n, Hkv, alpha, S);
  count_launch();
  return cudaGetLastError();
}

size_t estats_ws(int n, int L, int Hkv) {
  return (size_t)L * Hkv * ((n + EST_CHUNK - 1) / EST_CHUNK) * 3 * sizeof(double);
}

cudaError_t launch_estats(const float* H, int64_t Hsl, int64_t Hsh, const float* D, int64_t Dsl,
                          int64_t Dsh, int n, int L, int Hkv, float* stats, float* Ebar, double* part,
                          cudaStream_t st) {
  const int nch = (n + EST_CHUNK - 1) / EST_CHUNK, rows = L * Hkv;
  // D and H without a KV-head stride (prefill: D per layer, H per token): E is the same in
  // every KV head of a layer, so each layer's statistics are taken once
  const bool per_layer = Hsh == 0 && Dsh == 0;
  const int prow = per_layer ? L : rows;
  estats_part_kernel<<<dim3(nch, prow), EST_THREADS, 0, st>>>(H, Hsl, Hsh, D, Dsl, Dsh, n, per_layer ? 1 : Hkv,
                                                              part);
  count_launch();
  estats_merge_kernel<<<(rows + 127) / 128, 128, 0, st>>>(part, rows, per_layer ? Hkv : 1, nch, n, stats);
  count_launch();
  if (Ebar) {
    ebar_kernel<<<(L + 127) / 128, 128, 0, st>>>(stats, L, Hkv, Ebar);
    count_launch();
  }
  return cudaGetLastError();
}

}  // namespace kvc
