// Top-k restricted entropy of logits rows.
//
// [InfoKV] Methodology (second signal H_i) and Glossary "Top-k restricted
// entropy": the entropy of token i's final-layer predictive distribution
// restricted to its k most probable entries (k = 256), renormalised, natural
// log.  Only the multiset of the k largest logits matters.
//
// One warp streams one row with 16-byte coalesced loads.  Values above the
// running threshold go to a per-warp candidate buffer in shared memory; when
// the buffer fills, a warp radix select finds the k-th largest candidate,
// which becomes the new threshold, and only strictly larger candidates are
// kept (plus a count of threshold copies that complete the top-k multiset).
// On random-order rows the threshold climbs fast and almost every vector is
// rejected by one max + compare, so the kernel runs at HBM speed.
#include "kernels.cuh"

namespace kvc {

constexpr int ENT_WARPS = 16;
constexpr int ENT_UNROLL = 4;

// k-th largest (1-based) value among buf[0..cnt), cnt >= k.  Radix select on
// order-preserving keys, 8 bits per pass from the top; `passes` = 2 suffices
// for bf16-valued data (16 significant key bits), 4 for fp32.
__device__ float warp_kth_largest(const float* buf, int cnt, int k, uint32_t* hist, int lane,
                                  int passes) {
  uint32_t prefix = 0, mask = 0;
  uint32_t krem = (uint32_t)k;
  for (int p = 0; p < passes; ++p) {
    const int shift = 24 - 8 * p;
    for (int b = lane; b < 256; b += 32) hist[b] = 0u;
    __syncwarp();
    for (int i = lane; i < cnt; i += 32) {
      uint32_t key = f2key(buf[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xffu], 1u);
    }
    __syncwarp();
    // lane j owns bins 255-8j .. 248-8j, scanned from the top
    uint32_t c[8], s = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) { c[t] = hist[255 - 8 * lane - t]; s += c[t]; }
    uint32_t incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t excl = incl - s;
    const unsigned own = __ballot_sync(FULL, excl < krem && krem <= incl);
    const int owner = __ffs(own) - 1;
    uint32_t digit = 0, above = 0;
    if (lane == owner) {
      uint32_t run = excl;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (run + c[t] >= krem) { digit = 255u - 8u * lane - t; above = run; break; }
        run += c[t];
      }
    }
    digit = __shfl_sync(FULL, digit, owner);
    above = __shfl_sync(FULL, above, owner);
    krem -= above;
    prefix |= digit << shift;
    mask |= 0xffu << shift;
    __syncwarp();
  }
  // any candidate whose key matches the prefix has the k-th largest value
  float v = -INFINITY;
  bool found = false;
  for (int base = 0; base < cnt && !found; base += 32) {
    int i = base + lane;
    bool hit = i < cnt && (f2key(buf[i]) & mask) == prefix;
    unsigned m = __ballot_sync(FULL, hit);
    if (m) {
      v = __shfl_sync(FULL, i < cnt ? buf[i] : 0.f, __ffs(m) - 1);
      found = true;
    }
  }
  return v;
}

// Keep only candidates > new threshold; nfill copies of the threshold complete the top-k.
__device__ void warp_prune(float* buf, int& cnt, int k, uint32_t* hist, int lane, int passes,
                           float& thr, int& nfill) {
  const float v = warp_kth_largest(buf, cnt, k, hist, lane, passes);
  int out = 0;
  for (int base = 0; base < cnt; base += 32) {
    const int i = base + lane;
    const float x = i < cnt ? buf[i] : -INFINITY;
    const bool keep = i < cnt && x > v;
    const unsigned m = __ballot_sync(FULL, keep);
    __syncwarp();
    if (keep) buf[out + __popc(m & ((1u << lane) - 1u))] = x;
    out += __popc(m);
    __syncwarp();
  }
  cnt = out;
  thr = v;
  nfill = k - out;
}

// Offer NV values per lane to the warp's candidate set.
template <int NV>
__device__ __forceinline__ void offer(const float* f, float* buf, int& cnt, int cap, int k,
                                      uint32_t* hist, int lane, int passes, float& thr, int& nfill) {
  float mx = f[0];
#pragma unroll
  for (int e = 1; e < NV; ++e) mx = fmaxf(mx, f[e]);
  if (!__any_sync(FULL, mx > thr)) return;
  int c = 0;
#pragma unroll
  for (int e = 0; e < NV; ++e) c += f[e] > thr ? 1 : 0;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += y;
  }
  int total = __shfl_sync(FULL, incl, 31);
  if (cnt + total > cap) {
    warp_prune(buf, cnt, k, hist, lane, passes, thr, nfill);
    c = 0;
#pragma unroll
    for (int e = 0; e < NV; ++e) c += f[e] > thr ? 1 : 0;
    incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += y;
    }
    total = __shfl_sync(FULL, incl, 31);
  }
  int pos = cnt + incl - c;
#pragma unroll
  for (int e = 0; e < NV; ++e)
    if (f[e] > thr) buf[pos++] = f[e];
  cnt += total;
  __syncwarp();
}

template <typename T>
__global__ void __launch_bounds__(ENT_WARPS * 32)
entropy_topk_kernel(const T* __restrict__ logits, int64_t rows, int64_t V, int64_t row_stride,
                    int k, int cap, bool vec_ok, float* __restrict__ H) {
  extern __shared__ float ent_smem[];
  constexpr int EPV = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* buf = ent_smem + (size_t)warp * (cap + 256);
  uint32_t* hist = reinterpret_cast<uint32_t*>(buf + cap);
  const int passes = sizeof(T) == 2 ? 2 : 4;
  const int64_t nw = (int64_t)gridDim.x * ENT_WARPS;
  for (int64_t row = (int64_t)blockIdx.x * ENT_WARPS + warp; row < rows; row += nw) {
    const T* z = logits + row * row_stride;
    float thr = -INFINITY;
    int cnt = 0, nfill = 0;
    const int64_t nvec = vec_ok ? V / EPV : 0;
    for (int64_t v0 = 0; v0 < nvec; v0 += 32 * ENT_UNROLL) {
      uint4 u[ENT_UNROLL];
#pragma unroll
      for (int t = 0; t < ENT_UNROLL; ++t) {
        const int64_t vi = v0 + t * 32 + lane;
        u[t] = vi < nvec ? ld_stream16(z + vi * EPV) : make_uint4(0xff80ff80u, 0xff80ff80u,
                                                                  0xff80ff80u, 0xff80ff80u);
      }
#pragma unroll
      for (int t = 0; t < ENT_UNROLL; ++t) {
        float f[EPV];
        Vec<T>::unpack(u[t], f);
        if (v0 + t * 32 + lane >= nvec) {
#pragma unroll
          for (int e = 0; e < EPV; ++e) f[e] = -INFINITY;
        }
        offer<EPV>(f, buf, cnt, cap, k, hist, lane, passes, thr, nfill);
      }
    }
    for (int64_t e0 = nvec * EPV; e0 < V; e0 += 32) {
      const int64_t e = e0 + lane;
      float f[1] = {e < V ? to_f(z[e]) : -INFINITY};
      offer<1>(f, buf, cnt, cap, k, hist, lane, passes, thr, nfill);
    }
    // final top-k multiset: {x > v} plus copies of v (or of the threshold)
    float fillv = thr;
    int fillc = 0;
    if (cnt >= k) {
      warp_prune(buf, cnt, k, hist, lane, passes, thr, nfill);
      fillv = thr;
      fillc = nfill;
    } else {
      fillc = k - cnt;
    }
    if (fillv == -INFINITY) fillc = 0;  // fewer than k finite logits
    float m = fillc > 0 ? fillv : -INFINITY;
    for (int i = lane; i < cnt; i += 32) m = fmaxf(m, buf[i]);
    m = warp_max(m);
    float s = 0.f, t = 0.f;
    for (int i = lane; i < cnt; i += 32) {
      const float x = buf[i] - m;
      const float ex = expf(x);
      s += ex;
      t += ex * x;
    }
    s = warp_sum(s);
    t = warp_sum(t);
    if (lane == 0) {
      if (fillc > 0) {
        const float x = fillv - m;
        const float ex = expf(x);
        s += fillc * ex;
        t += fillc * ex * x;
      }
      H[row] = (m == -INFINITY || s <= 0.f) ? 0.f : logf(s) - t / s;
    }
    __syncwarp();
  }
}

size_t entropy_smem_bytes(int k) { return (size_t)ENT_WARPS * ((k + 512) + 256) * sizeof(float); }

cudaError_t launch_entropy(const void* logits, kvc_dtype dt, int64_t rows, int64_t V,
                           int64_t row_stride, int k, float* H, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const int kk = (int)(k < V ? k : V);
  const int cap = kk + 512;
  const size_t smem = entropy_smem_bytes(kk);
  const size_t es = dt == KVC_BF16 ? 2 : 4;
  const bool vec_ok = ((uintptr_t)logits % 16 == 0) && ((row_stride * es) % 16 == 0);
  int64_t want = (rows + ENT_WARPS - 1) / ENT_WARPS;
  int64_t maxb = (int64_t)num_sms() * 2;
  const int grid = (int)(want < maxb ? want : maxb);
  if (dt == KVC_BF16) {
    auto kern = entropy_topk_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, ENT_WARPS * 32, smem, st>>>((const __nv_bfloat16*)logits, rows, V, row_stride,
                                              kk, cap, vec_ok, H);
  } else {
    auto kern = entropy_topk_kernel<float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, ENT_WARPS * 32, smem, st>>>((const float*)logits, rows, V, row_stride, kk, cap,
                                              vec_ok, H);
  }
  return cudaGetLastError();
}

}  // namespace kvc
