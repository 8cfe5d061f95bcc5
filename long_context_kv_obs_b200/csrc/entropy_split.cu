// Top-k restricted entropy of a few long logits rows (a decode step's batch).
//
// [InfoKV] Methodology (second signal H_i) and Glossary "Top-k restricted
// entropy": the entropy of the renormalised distribution over a row's k largest
// logits.  Only the multiset of the k largest values matters.
//
// The row-per-warp kernel leaves most of the GPU idle when there are only a
// handful of rows (one decoded token per sequence), so here every row is cut
// into chunks of 16 KB, one CTA each:
//   chunk: the chunk's k-th largest value v_c by bisection over order-preserving
//          keys (block-wide counts of values >= the probe), then the chunk's top-k
//          multiset -- its values > v_c and enough copies of v_c to make k -- is
//          written out (padding is -inf).
//   merge: one CTA per row takes the k-th largest T of the chunks' candidates, the
//          same way (starting from the largest v_c: T >= every v_c), and the entropy
//          of {candidates > T} plus (k - their count) copies of T.  It is launched as
//          a programmatic dependent of the chunk grid, so its launch overlaps the
//          chunks' tail.
// The union of the chunks' top-k multisets holds the row's top-k multiset: a
// value above the row's k-th largest T is above its chunk's k-th largest, and a
// chunk that drops copies of T keeps at least as many as the row needs.  So the
// merge sees exactly the row's top-k values, ties included.
#include "kernels.cuh"

namespace kvc {

constexpr int ES_THREADS = 256;                 // chunk CTA
constexpr int ES_VPT = 4;                       // 16-byte vectors per thread
constexpr int ES_VEC = ES_THREADS * ES_VPT;     // vectors per chunk (16 KB)
constexpr int EM_THREADS = 1024;                // merge CTA
constexpr int EM_PER = 16;                      // candidates per merge thread
constexpr int ES_MAX_ROWS = 512;                // more rows keep every SM busy row by row

// Keys: bf16 rows compare on the upper 16 bits of the fp32 key (their values are
// bf16-exact), fp32 rows on all 32.
template <bool B16>
__device__ __forceinline__ uint32_t es_key(float x) {
  return B16 ? f2key(x) >> 16 : f2key(x);
}
template <bool B16>
__device__ __forceinline__ float es_value(uint32_t key) {
  if (B16) {
    const uint32_t b = (key & 0x8000u) ? (key & 0x7fffu) : (~key & 0xffffu);
    return __uint_as_float(b << 16);
  }
  return key2f(key);
}

// Block-wide sum of one int per thread (WARPS <= 32): the warps' totals go through
// shared memory and lane j of every warp adds total j.  `red` has 2 x warps slots and
// `par` alternates between calls, so one barrier per call suffices.
template <int WARPS>
__device__ __forceinline__ int es_sum(int v, int* red, int par) {
  v = __reduce_add_sync(FULL, v);
  const int lane = threadIdx.x & 31;
  if (lane == 0) red[par * WARPS + (threadIdx.x >> 5)] = v;
  __syncthreads();
  return __reduce_add_sync(FULL, lane < WARPS ? red[par * WARPS + lane] : 0);
}

// Block-wide reduction of two keys, once per kernel: the minimum of `a` (MIN_A) or its
// maximum, and the maximum of `b`.
template <int WARPS, bool MIN_A>
__device__ __forceinline__ void es_keys(uint32_t& a, uint32_t& b, uint32_t* red) {
  a = MIN_A ? __reduce_min_sync(FULL, a) : __reduce_max_sync(FULL, a);
  b = __reduce_max_sync(FULL, b);
  const int lane = threadIdx.x & 31;
  if (lane == 0) {
    red[threadIdx.x >> 5] = a;
    red[WARPS + (threadIdx.x >> 5)] = b;
  }
  __syncthreads();
  const uint32_t ra = lane < WARPS ? red[lane] : (MIN_A ? 0xffffffffu : 0u);
  const uint32_t rb = lane < WARPS ? red[WARPS + lane] : 0u;
  a = MIN_A ? __reduce_min_sync(FULL, ra) : __reduce_max_sync(FULL, ra);
  b = __reduce_max_sync(FULL, rb);
}

// The largest key t in [lo, hi] with count(values >= value(t)) >= k; count(lo) >= k
// on entry.  `count` returns this thread's share of the count.
template <bool B16, int WARPS, typename F>
__device__ __forceinline__ float es_kth(uint32_t lo, uint32_t hi, int k, int* red, int& par, F count) {
  while (lo < hi) {
    const uint32_t mid = lo + ((hi - lo + 1) >> 1);
    const int c = es_sum<WARPS>(count(es_value<B16>(mid)), red, par);
    par ^= 1;
    if (c >= k) lo = mid; else hi = mid - 1;
  }
  return es_value<B16>(lo);
}

__device__ __forceinline__ __nv_bfloat162 es_b2(uint32_t w) { return *reinterpret_cast<__nv_bfloat162*>(&w); }

// The chunk's values as kept in registers: bf16 pairs (packed compares count two values
// per instruction) or fp32.
template <typename T> struct EsHeld;
template <> struct EsHeld<__nv_bfloat16> {
  static constexpr int W = ES_VPT * 4;          // 32-bit words per thread
  uint32_t w[W];
  __device__ __forceinline__ void set(int j, const uint4& u) {
    w[4 * j] = u.x; w[4 * j + 1] = u.y; w[4 * j + 2] = u.z; w[4 * j + 3] = u.w;
  }
  __device__ __forceinline__ void set_ragged(int j, const __nv_bfloat16* z, int64_t e0, int64_t V, bool tail) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t word = 0xff80ff80u;              // -inf pair
      if (tail) {
        const int64_t a = e0 + 2 * q, b = a + 1;
        const uint32_t lo16 = a < V ? (uint32_t)__bfloat16_as_ushort(z[a]) : 0xff80u;
        const uint32_t hi16 = b < V ? (uint32_t)__bfloat16_as_ushort(z[b]) : 0xff80u;
        word = lo16 | (hi16 << 16);
      }
      w[4 * j + q] = word;
    }
  }
  __device__ __forceinline__ float val(int e) const { return (e & 1) ? bf_hi(w[e >> 1]) : bf_lo(w[e >> 1]); }
  static constexpr int N = 2 * W;
  __device__ __forceinline__ int count_ge(float t) const {
    const __nv_bfloat162 t2 = __float2bfloat162_rn(t);   // t is bf16-exact
    int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
#pragma unroll
    for (int i = 0; i < W; i += 4) {
      c0 += __popc(__hge2_mask(es_b2(w[i]), t2));
      c1 += __popc(__hge2_mask(es_b2(w[i + 1]), t2));
      c2 += __popc(__hge2_mask(es_b2(w[i + 2]), t2));
      c3 += __popc(__hge2_mask(es_b2(w[i + 3]), t2));
    }
    return (c0 + c1 + c2 + c3) >> 4;
  }
};
template <> struct EsHeld<float> {
  static constexpr int N = ES_VPT * 4;
  float x[N];
  __device__ __forceinline__ void set(int j, const uint4& u) {
    x[4 * j] = __uint_as_float(u.x); x[4 * j + 1] = __uint_as_float(u.y);
    x[4 * j + 2] = __uint_as_float(u.z); x[4 * j + 3] = __uint_as_float(u.w);
  }
  __device__ __forceinline__ void set_ragged(int j, const float* z, int64_t e0, int64_t V, bool tail) {
#pragma unroll
    for (int q = 0; q < 4; ++q) x[4 * j + q] = (tail && e0 + q < V) ? z[e0 + q] : -INFINITY;
  }
  __device__ __forceinline__ float val(int e) const { return x[e]; }
  __device__ __forceinline__ int count_ge(float t) const {
    int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      c0 += x[i] >= t; c1 += x[i + 1] >= t; c2 += x[i + 2] >= t; c3 += x[i + 3] >= t;
    }
    return c0 + c1 + c2 + c3;
  }
};

template <typename T>
__global__ void __launch_bounds__(ES_THREADS)
entropy_chunk_kernel(const T* __restrict__ logits, int64_t V, int64_t row_stride, int k,
                     float* __restrict__ cand, float* __restrict__ vthr) {
  constexpr bool B16 = sizeof(T) == 2;
  constexpr int EPV = Vec<T>::N;
  constexpr int WARPS = ES_THREADS / 32;
  __shared__ int red[2 * WARPS];
  __shared__ uint32_t kred[2 * WARPS];
  const int c = blockIdx.x, nchunk = gridDim.x;
  const int64_t row = blockIdx.y;
  const T* z = logits + row * row_stride;
  const int64_t nvec = V / EPV;                  // whole vectors of the row
  EsHeld<T> h;
#pragma unroll
  for (int j = 0; j < ES_VPT; ++j) {
    const int64_t vi = (int64_t)c * ES_VEC + j * ES_THREADS + threadIdx.x;
    if (vi < nvec) h.set(j, ld_stream16(z + vi * EPV));
    else h.set_ragged(j, z, vi * EPV, V, vi == nvec);   // the row's ragged end sits in slot nvec
  }
  // the merge may be scheduled now; it waits for this grid before reading its output
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // bracket: every thread holds a value >= the least of the threads' maxima, so at
  // least ES_THREADS values are >= it; else the chunk's minimum
  uint32_t tmin = 0xffffffffu, tmax = 0u;
#pragma unroll
  for (int e = 0; e < EsHeld<T>::N; ++e) {
    const uint32_t kk = es_key<B16>(h.val(e));
    tmin = min(tmin, kk);
    tmax = max(tmax, kk);
  }
  uint32_t lo = k <= ES_THREADS ? tmax : tmin, hi = tmax;
  es_keys<WARPS, true>(lo, hi, kred);
  int par = 0;
  const float v = es_kth<B16, WARPS>(lo, hi, k, red, par, [&](float t) { return h.count_ge(t); });
  // values > v, compacted in thread order, then copies of v up to k
  int mine = 0;
#pragma unroll
  for (int e = 0; e < EsHeld<T>::N; ++e) mine += h.val(e) > v;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) red[par * WARPS + warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < WARPS; ++w) {
    const int s = red[par * WARPS + w];
    before += w < warp ? s : 0;
    total += s;
  }
  float* out = cand + (row * nchunk + c) * (int64_t)k;
  int pos = before + incl - mine;
#pragma unroll
  for (int e = 0; e < EsHeld<T>::N; ++e) {
    const float x = h.val(e);
    if (x > v) out[pos++] = x;
  }
  for (int i = total + threadIdx.x; i < k; i += ES_THREADS) out[i] = v;
  if (threadIdx.x == 0) vthr[row * nchunk + c] = v;
}

template <bool B16>
__global__ void __launch_bounds__(EM_THREADS)
entropy_merge_kernel(const float* __restrict__ cand, const float* __restrict__ vthr, int nchunk, int k,
                     float* __restrict__ H) {
  constexpr int WARPS = EM_THREADS / 32;
  __shared__ int red[2 * WARPS];
  __shared__ uint32_t kred[2 * WARPS];
  __shared__ float fred[2 * WARPS];
  // a dependent launched after this grid (the representation-change pass) reads nothing
  // it writes and may start now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the chunk grid's output is complete
  const int64_t row = blockIdx.x;
  const int ncand = nchunk * k;
  const float* src = cand + row * (int64_t)ncand;
  float x[EM_PER];
  uint32_t hi = 0u;
#pragma unroll
  for (int j = 0; j < EM_PER; ++j) {
    const int i = j * EM_THREADS + threadIdx.x;
    x[j] = i < ncand ? src[i] : -INFINITY;
    hi = max(hi, es_key<B16>(x[j]));
  }
  // the row's k-th largest is at least every chunk's k-th largest
  uint32_t lo = (int)threadIdx.x < nchunk ? es_key<B16>(vthr[row * nchunk + threadIdx.x]) : 0u;
  es_keys<WARPS, false>(lo, hi, kred);
  int par = 0;
  const float T = es_kth<B16, WARPS>(lo, hi, k, red, par, [&](float t) {
    int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
#pragma unroll
    for (int j = 0; j < EM_PER; j += 4) {
      c0 += x[j] >= t; c1 += x[j + 1] >= t; c2 += x[j + 2] >= t; c3 += x[j + 3] >= t;
    }
    return c0 + c1 + c2 + c3;
  });
  const float m = es_value<B16>(hi);
  int gt = 0;
  float s = 0.f, u = 0.f;
#pragma unroll
  for (int j = 0; j < EM_PER; ++j) {
    if (x[j] > T) {
      const float d = x[j] - m;
      const float ex = expf(d);
      s += ex;
      u += ex * d;
      ++gt;
    }
  }
  gt = es_sum<WARPS>(gt, red, par);
  s = warp_sum(s);
  u = warp_sum(u);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    fred[warp] = s;
    fred[WARPS + warp] = u;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float ss = 0.f, uu = 0.f;
    for (int w = 0; w < WARPS; ++w) {
      ss += fred[w];
      uu += fred[WARPS + w];
    }
    const int fillc = T == -INFINITY ? 0 : k - gt;   // fewer than k finite logits: no fill
    if (fillc > 0) {
      const float d = T - m;
      const float ex = expf(d);
      ss += fillc * ex;
      uu += fillc * ex * d;
    }
    H[row] = (m == -INFINITY || ss <= 0.f) ? 0.f : logf(ss) - uu / ss;
  }
}

static int64_t es_chunks(int64_t V, kvc_dtype dt) {
  const int64_t epv = dt == KVC_BF16 ? 8 : 4;
  return ((V + epv - 1) / epv + ES_VEC - 1) / ES_VEC;
}

size_t entropy_split_ws(int64_t rows, int64_t V, kvc_dtype dt, int k) {
  const int64_t kk = k < V ? k : V;
  const int64_t nc = es_chunks(V, dt);
  if (rows < 1 || rows > ES_MAX_ROWS || nc < 2 || nc > EM_THREADS || kk < 1 || nc * kk > EM_PER * EM_THREADS)
    return 0;
  return (size_t)(rows * nc * (kk + 1)) * sizeof(float);
}

cudaError_t launch_entropy_split(const void* logits, kvc_dtype dt, int64_t rows, int64_t V,
                                 int64_t row_stride, int k, float* cand, float* H, cudaStream_t st) {
  const int kk = (int)(k < V ? k : V);
  const int nc = (int)es_chunks(V, dt);
  float* vthr = cand + rows * nc * (int64_t)kk;
  const dim3 grid((unsigned)nc, (unsigned)rows);
  if (dt == KVC_BF16)
    entropy_chunk_kernel<__nv_bfloat16><<<grid, ES_THREADS, 0, st>>>((const __nv_bfloat16*)logits, V, row_stride,
                                                                      kk, cand, vthr);
  else
    entropy_chunk_kernel<float><<<grid, ES_THREADS, 0, st>>>((const float*)logits, V, row_stride, kk, cand, vthr);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e) return e;
  // the merge is launched as a programmatic dependent of the chunk grid: its CTAs may
  // be scheduled early and wait on the chunk grid's completion in the kernel
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(EM_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const float* cc = cand;
  const float* vt = vthr;
  e = dt == KVC_BF16 ? cudaLaunchKernelEx(&cfg, entropy_merge_kernel<true>, cc, vt, nc, kk, H)
                     : cudaLaunchKernelEx(&cfg, entropy_merge_kernel<false>, cc, vt, nc, kk, H);
  count_launch();
  return e;
}

}  // namespace kvc
