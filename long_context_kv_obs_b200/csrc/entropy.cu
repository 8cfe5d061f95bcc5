// Top-k restricted entropy of logits rows.
//
// [InfoKV] Methodology (second signal H_i) and Glossary "Top-k restricted
// entropy": the entropy of token i's final-layer predictive distribution
// restricted to its k most probable entries (k = 256), renormalised, natural
// log.  Only the multiset of the k largest logits matters.
//
// One warp owns one row; the row is split into groups of ENT_U 16-byte vectors
// (the 64 bf16 / 32 fp32 values one lane loads per step).
//   streaming pass (HBM): keep every group's two largest values (packed
//        min/max, three instructions per 32-bit word) in shared memory.
//   t  = the k-th largest of those ~2 x groups values.  They are elements of
//        the row, so the row's k-th largest value T is >= t.
//   A group whose second value is < t holds at most one element >= t (its
//   maximum); only groups whose second value is >= t (~1 % of them) can hold
//   more and are re-read.  The maxima >= t of the other groups plus every
//   element >= t of the re-read groups are exactly the row's elements >= t,
//   a superset of the top-k (~k candidates); a warp radix select over them
//   gives the exact top-k multiset.
// Rows whose candidate set would overflow the buffer (adversarial orders,
// huge ties) fall back to a streaming pass with a running threshold: values
// above it are appended to the buffer and pruned to the k largest by the same
// radix select when it fills.
#include "kernels.cuh"

namespace kvc {

constexpr int ENT_WARPS = 12;
constexpr int ENT_U = 8;   // 16-byte vectors per lane per step
constexpr int ENT_PD = 2;  // steps prefetched into L2 ahead of the register loads

// k-th largest (1-based) value among buf[0..cnt), cnt >= k.  Radix select on
// order-preserving keys, 8 bits per pass from the top with warp-aggregated
// shared-memory histograms; `passes` = 2 suffices for bf16-valued data (16
// significant key bits), 4 for fp32.
__device__ float warp_kth_largest(const float* buf, int cnt, int k, uint32_t* hist, int lane,
                                  int passes) {
  uint32_t prefix = 0, mask = 0;
  uint32_t krem = (uint32_t)k;
  for (int p = 0; p < passes; ++p) {
    const int shift = 24 - 8 * p;
    for (int b = lane; b < 256; b += 32) hist[b] = 0u;
    __syncwarp();
    for (int base = 0; base < cnt; base += 32) {
      const int i = base + lane;
      const uint32_t key = i < cnt ? f2key(buf[i]) : 0u;
      const bool valid = i < cnt && (key & mask) == prefix;
      const uint32_t digit = (key >> shift) & 0xffu;
      const unsigned act = __ballot_sync(FULL, valid);
      if (valid) {
        const unsigned peers = __match_any_sync(act, digit);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (uint32_t)__popc(peers));
      }
    }
    __syncwarp();
    // lane j owns bins 255-8j .. 248-8j, scanned from the top
    uint32_t c[8], s = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) { c[t] = hist[255 - 8 * lane - t]; s += c[t]; }
    uint32_t incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t excl = incl - s;
    const unsigned own = __ballot_sync(FULL, excl < krem && krem <= incl);
    const int owner = own ? __ffs(own) - 1 : 0;
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
  for (int base = 0; base < cnt; base += 32) {
    const int i = base + lane;
    const bool hit = i < cnt && (f2key(buf[i]) & mask) == prefix;
    const unsigned m = __ballot_sync(FULL, hit);
    if (m) {
      v = __shfl_sync(FULL, i < cnt ? buf[i] : 0.f, __ffs(m) - 1);
      break;
    }
  }
  return v;
}

// Keep only candidates > the new threshold; nfill copies of it complete the top-k.
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

// Per-type vector helpers: packed "any element > thr" test, survivor count and extraction.
template <typename T> struct EntVec;
template <> struct EntVec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static uint4 sentinel() {
    return make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);  // bf16 -inf
  }
  __device__ __forceinline__ static __nv_bfloat162 b2(uint32_t w) {
    return *reinterpret_cast<__nv_bfloat162*>(&w);
  }
  __device__ __forceinline__ static bool any_gt(const uint4& u, __nv_bfloat162 t2, float) {
    const __nv_bfloat162 m = __hmax2(__hmax2(b2(u.x), b2(u.y)), __hmax2(b2(u.z), b2(u.w)));
    return __hgt2_mask(m, t2) != 0u;
  }
  __device__ __forceinline__ static int count_gt(const uint4& u, __nv_bfloat162 t2, float) {
    return (__popc(__hgt2_mask(b2(u.x), t2)) + __popc(__hgt2_mask(b2(u.y), t2)) +
            __popc(__hgt2_mask(b2(u.z), t2)) + __popc(__hgt2_mask(b2(u.w), t2))) >> 4;
  }
};
template <> struct EntVec<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static uint4 sentinel() {
    return make_uint4(0xff800000u, 0xff800000u, 0xff800000u, 0xff800000u);  // fp32 -inf
  }
  __device__ __forceinline__ static bool any_gt(const uint4& u, __nv_bfloat162, float t) {
    return fmaxf(fmaxf(__uint_as_float(u.x), __uint_as_float(u.y)),
                 fmaxf(__uint_as_float(u.z), __uint_as_float(u.w))) > t;
  }
  __device__ __forceinline__ static int count_gt(const uint4& u, __nv_bfloat162, float t) {
    return (__uint_as_float(u.x) > t) + (__uint_as_float(u.y) > t) + (__uint_as_float(u.z) > t) +
           (__uint_as_float(u.w) > t);
  }
};

template <typename T>
struct EntRow {
  float* buf;
  uint32_t* hist;
  int cap, k, passes, lane;
  float thr;
  int cnt, nfill;

  __device__ __forceinline__ __nv_bfloat162 thr2() const { return __float2bfloat162_rn(thr); }

  // Offer one step: ENT_U vectors per lane.
  __device__ __forceinline__ void step(const uint4 (&u)[ENT_U]) {
    unsigned hm = 0;
    {
      const __nv_bfloat162 t2 = thr2();
#pragma unroll
      for (int v = 0; v < ENT_U; ++v) hm |= (EntVec<T>::any_gt(u[v], t2, thr) ? 1u : 0u) << v;
    }
    if (!__any_sync(FULL, hm != 0u)) return;
    int c = 0;
    {
      const __nv_bfloat162 t2 = thr2();
#pragma unroll
      for (int v = 0; v < ENT_U; ++v)
        if (hm & (1u << v)) c += EntVec<T>::count_gt(u[v], t2, thr);
    }
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += y;
    }
    int total = __shfl_sync(FULL, incl, 31);
    if (cnt + total > cap) {
      warp_prune(buf, cnt, k, hist, lane, passes, thr, nfill);
      const __nv_bfloat162 t2 = thr2();
      hm = 0;
      c = 0;
#pragma unroll
      for (int v = 0; v < ENT_U; ++v) {
        if (EntVec<T>::any_gt(u[v], t2, thr)) {
          hm |= 1u << v;
          c += EntVec<T>::count_gt(u[v], t2, thr);
        }
      }
      incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += y;
      }
      total = __shfl_sync(FULL, incl, 31);
    }
    int pos = cnt + incl - c;
#pragma unroll
    for (int v = 0; v < ENT_U; ++v) {
      if (hm & (1u << v)) {
        float f[Vec<T>::N];
        Vec<T>::unpack(u[v], f);
#pragma unroll
        for (int e = 0; e < Vec<T>::N; ++e)
          if (f[e] > thr) buf[pos++] = f[e];
      }
    }
    cnt += total;
    __syncwarp();
  }

  // Offer one value per lane (ragged tail / unaligned rows).
  __device__ __forceinline__ void scalar(float x) {
    const bool h = x > thr;
    if (!__any_sync(FULL, h)) return;
    const unsigned b = __ballot_sync(FULL, h);
    int total = __popc(b);
    if (cnt + total > cap) {
      warp_prune(buf, cnt, k, hist, lane, passes, thr, nfill);
      total = __popc(__ballot_sync(FULL, x > thr));
    }
    const unsigned bb = __ballot_sync(FULL, x > thr);
    if (x > thr) buf[cnt + __popc(bb & ((1u << lane) - 1u))] = x;
    cnt += total;
    __syncwarp();
  }
};

// ---------------------------------------------------------------- two-pass kernel

constexpr int ENT_CAND = 1024;   // candidate buffer (values)
constexpr int ENT_LIST = 512;    // qualifying groups

template <typename T> struct GTop2;
template <> struct GTop2<__nv_bfloat16> {
  using S = unsigned short;                // stored as bf16 bits
  // two largest of the lane's ENT_U x 8 values
  __device__ __forceinline__ static void of(const uint4 (&u)[ENT_U], S& s1, S& s2) {
    const __nv_bfloat162 ninf = EntVec<__nv_bfloat16>::b2(0xff80ff80u);
    __nv_bfloat162 m1 = ninf, m2 = ninf;
#pragma unroll
    for (int v = 0; v < ENT_U; ++v) {
      const uint32_t w4[4] = {u[v].x, u[v].y, u[v].z, u[v].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 w = EntVec<__nv_bfloat16>::b2(w4[j]);
        m2 = __hmax2(m2, __hmin2(m1, w));
        m1 = __hmax2(m1, w);
      }
    }
    const __nv_bfloat16 a1 = __low2bfloat16(m1), b1 = __high2bfloat16(m1);
    const __nv_bfloat16 top = __hmax(a1, b1);
    const __nv_bfloat16 sec = __hmax(__hmin(a1, b1), __hmax(__low2bfloat16(m2), __high2bfloat16(m2)));
    s1 = *reinterpret_cast<const unsigned short*>(&top);
    s2 = *reinterpret_cast<const unsigned short*>(&sec);
  }
  __device__ __forceinline__ static float val(S s) { return __uint_as_float((uint32_t)s << 16); }
};
template <> struct GTop2<float> {
  using S = float;
  __device__ __forceinline__ static void of(const uint4 (&u)[ENT_U], S& s1, S& s2) {
    float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
    for (int v = 0; v < ENT_U; ++v) {
      const float w4[4] = {__uint_as_float(u[v].x), __uint_as_float(u[v].y), __uint_as_float(u[v].z),
                           __uint_as_float(u[v].w)};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        m2 = fmaxf(m2, fminf(m1, w4[j]));
        m1 = fmaxf(m1, w4[j]);
      }
    }
    s1 = m1;
    s2 = m2;
  }
  __device__ __forceinline__ static float val(S s) { return s; }
};

// count of stored values >= t (bf16 summaries: eight per 16-byte shared load, packed compares)
template <typename T>
__device__ __forceinline__ int count_ge(const typename GTop2<T>::S* g, int n, float t, int lane) {
  int c = 0;
  if constexpr (sizeof(typename GTop2<T>::S) == 2) {
    const __nv_bfloat162 t2 = __float2bfloat162_rn(t);
    const uint4* g4 = reinterpret_cast<const uint4*>(g);
    const int n8 = n >> 3;
    for (int i = lane; i < n8; i += 32) {
      const uint4 u = g4[i];
      c += __popc(__hge2_mask(EntVec<__nv_bfloat16>::b2(u.x), t2)) +
           __popc(__hge2_mask(EntVec<__nv_bfloat16>::b2(u.y), t2)) +
           __popc(__hge2_mask(EntVec<__nv_bfloat16>::b2(u.z), t2)) +
           __popc(__hge2_mask(EntVec<__nv_bfloat16>::b2(u.w), t2));
    }
    c >>= 4;
    for (int i = (n8 << 3) + lane; i < n; i += 32) c += GTop2<T>::val(g[i]) >= t ? 1 : 0;
  } else {
    for (int i = lane; i < n; i += 32) c += GTop2<T>::val(g[i]) >= t ? 1 : 0;
  }
  return __reduce_add_sync(FULL, c);
}

// Largest value t with count(g >= t) >= k among the n stored values (n > k):
// bisection over the order-preserving key of the value (t is exact: a stored value).
// k-th largest (1-based, k <= n) of the n stored group maxima, found by bisection over
// order-preserving keys between the keys of their minimum and maximum (bf16 keys in
// that bracket take a few hundred values, so about 9 passes instead of 16).  It is a
// lower bound of the row's k-th largest value: the maxima are k of its elements or more.
template <typename T>
__device__ float kth_maxima(const typename GTop2<T>::S* g, int n, int k, int lane) {
  float mn = INFINITY, mx = -INFINITY;
  for (int i = lane; i < n; i += 32) {
    const float v = GTop2<T>::val(g[i]);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
  }
  if (sizeof(typename GTop2<T>::S) == 2) {
    // keys of bf16 values: the upper half of the fp32 key, decoded exactly
    uint32_t lo = f2key(mn) >> 16, hi = f2key(mx) >> 16;
    auto value = [&](uint32_t key) -> float {
      const uint32_t b16 = (key & 0x8000u) ? (key & 0x7fffu) : (~key & 0xffffu);
      return __uint_as_float(b16 << 16);
    };
    while (lo < hi) {   // invariant: count(>= value(lo)) >= k
      const uint32_t mid = lo + ((hi - lo + 1) >> 1);
      if (count_ge<T>(g, n, value(mid), lane) >= k) lo = mid; else hi = mid - 1;
    }
    return value(lo);
  }
  uint32_t lo = f2key(mn), hi = f2key(mx);
  while (lo < hi) {
    const uint32_t mid = lo + ((hi - lo + 1) >> 1);
    if (count_ge<T>(g, n, key2f(mid), lane) >= k) lo = mid; else hi = mid - 1;
  }
  return key2f(lo);
}

template <typename T>
__device__ float kth_stored(const typename GTop2<T>::S* g, int n, int k, int lane) {
  const int bits = sizeof(typename GTop2<T>::S) * 8;
  // keys below the key of -inf decode to NaNs; count(g >= -inf) = n > k holds at lo
  uint32_t lo = bits == 16 ? 0x007fu : 0x007fffffu, hi = bits == 16 ? 0xffffu : 0xffffffffu;
  auto value = [&](uint32_t key) -> float {
    if (bits == 16) {
      const uint32_t b16 = (key & 0x8000u) ? (key & 0x7fffu) : (~key & 0xffffu);
      return __uint_as_float(b16 << 16);
    }
    return key2f(key);
  };
  while (lo < hi) {
    const uint32_t mid = lo + ((hi - lo + 1) >> 1);
    if (count_ge<T>(g, n, value(mid), lane) >= k) lo = mid; else hi = mid - 1;
  }
  return value(lo);
}

template <typename T>
__global__ void __launch_bounds__(ENT_WARPS * 32, 1)
entropy_twopass_kernel(const T* __restrict__ logits, int64_t rows, int64_t V, int64_t row_stride,
                       int k, int cap, bool vec_ok, int nwarps, int gcap, size_t warp_bytes,
                       float* __restrict__ H) {
  using GS = typename GTop2<T>::S;
  extern __shared__ __align__(16) unsigned char ent2_smem[];
  constexpr int EPV = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= nwarps) return;
  unsigned char* wbase = ent2_smem + (size_t)warp * warp_bytes;
  uint32_t* hist = reinterpret_cast<uint32_t*>(wbase);                 // 256 words
  float* region = reinterpret_cast<float*>(wbase + 1024);              // reused by the fallback
  GS* gtop = reinterpret_cast<GS*>(region);                            // [0, gcap): maxima, [gcap, 2 gcap): seconds
  float* cand = reinterpret_cast<float*>(wbase + 1024 + ((2 * (size_t)gcap * sizeof(GS) + 15) / 16) * 16);
  int* list = reinterpret_cast<int*>(cand + ENT_CAND);
  const int passes = sizeof(T) == 2 ? 2 : 4;
  const int64_t per_step = 32 * ENT_U;
  const int64_t nw = (int64_t)gridDim.x * nwarps;
  const int64_t nvec = vec_ok ? V / EPV : 0;
  const int64_t nsteps = (nvec + per_step - 1) / per_step;
  const int64_t full = nvec / per_step;                            // steps with no ragged end
  const bool stream_ok = vec_ok && (int)(nsteps * 32) <= gcap;
  // the summary area can take the packed candidates
  const bool pack_ok = 2 * (size_t)gcap * sizeof(GS) >= (size_t)ENT_CAND * sizeof(float);
  // The first two steps of a row are loaded before the row is reached: while a warp
  // works on the selection tail of row r, the head of its next row is in flight.
  // Streamed lines are demoted to evict-first once read, so that the lines prefetched
  // ahead of them are the last to leave L2.
  const uint64_t evict_first = l2_evict_first_policy();
  uint4 pa[ENT_U], pb[ENT_U];
  auto load_full = [&](uint4 (&dst)[ENT_U], const T* zz, int64_t s) {
    const uint4* q = reinterpret_cast<const uint4*>(zz) + lane + s * per_step;
#pragma unroll
    for (int v = 0; v < ENT_U; ++v) dst[v] = ld_stream16_policy(q + v * 32, evict_first);
  };
  {
    const int64_t r0 = (int64_t)blockIdx.x * nwarps + warp;
    if (stream_ok && r0 < rows) {
      if (full > 0) load_full(pa, logits + r0 * row_stride, 0);
      if (full > 1) load_full(pb, logits + r0 * row_stride, 1);
    }
  }
  for (int64_t row = (int64_t)blockIdx.x * nwarps + warp; row < rows; row += nw) {
    const T* z = logits + row * row_stride;
    const int ngroups = (int)(nsteps * 32);
    const int64_t tail0 = nvec * EPV;
    bool fast = stream_ok;
    float t0 = -INFINITY;
    int ncand = 0;
    float* cbuf = cand;   // where the candidates end up
    if (fast) {
      // ---- streaming pass: the two largest values of every group
      GS* g1 = gtop;
      GS* g2 = gtop + gcap;
      // pa / pb hold steps 0 / 1 on entry; each is reloaded two steps ahead after use.
      // A step is one contiguous 4 KB range; lane 0 prefetches step s + ENT_PD into L2.
      const uint32_t step_bytes = (uint32_t)(per_step * 16);
      for (int64_t s = 0; s < full; s += 2) {
        if (lane == 0) {
          if (s + ENT_PD < full) prefetch_l2(reinterpret_cast<const uint4*>(z) + (s + ENT_PD) * per_step, step_bytes);
          if (s + 1 + ENT_PD < full)
            prefetch_l2(reinterpret_cast<const uint4*>(z) + (s + 1 + ENT_PD) * per_step, step_bytes);
        }
        GTop2<T>::of(pa, g1[s * 32 + lane], g2[s * 32 + lane]);
        if (s + 2 < full) load_full(pa, z, s + 2);
        if (s + 1 < full) {
          GTop2<T>::of(pb, g1[(s + 1) * 32 + lane], g2[(s + 1) * 32 + lane]);
          if (s + 3 < full) load_full(pb, z, s + 3);
        }
      }
      if (full < nsteps) {                                          // the ragged last step
        uint4 r[ENT_U];
#pragma unroll
        for (int v = 0; v < ENT_U; ++v) {
          const int64_t vi = full * per_step + v * 32 + lane;
          r[v] = vi < nvec ? ld_stream16(z + vi * EPV) : EntVec<T>::sentinel();
        }
        GTop2<T>::of(r, g1[full * 32 + lane], g2[full * 32 + lane]);
      }
      if (row + nw < rows) {                                        // head of the next row
        const T* zn = logits + (row + nw) * row_stride;
        if (full > 0) load_full(pa, zn, 0);
        if (full > 1) load_full(pb, zn, 1);
        if (lane == 0)
          for (int64_t s = 2; s < 2 + ENT_PD && s < full; ++s)
            prefetch_l2(reinterpret_cast<const uint4*>(zn) + s * per_step, step_bytes);
      }
      __syncwarp();
      // the summaries of all groups are contiguous: maxima then seconds, 2 * ngroups values
      if (ngroups >= k) {
        t0 = kth_maxima<T>(g1, ngroups, k, lane);
      } else if (2 * ngroups > k) {
        if (ngroups < gcap) {   // close the gap between the two halves
          for (int i = lane; i < ngroups; i += 32) g1[ngroups + i] = g2[i];
          __syncwarp();
        }
        t0 = kth_stored<T>(gtop, 2 * ngroups, k, lane);
      }
      const GS* sec = ngroups < gcap ? g1 + ngroups : g2;
      // ---- groups to re-read: second value >= t0
      int nq = 0;
      for (int g0 = 0; g0 < ngroups; g0 += 32) {
        const int g = g0 + lane;
        const bool q = g < ngroups && GTop2<T>::val(sec[g]) >= t0;
        const unsigned bq = __ballot_sync(FULL, q);
        const int pos = nq + __popc(bq & ((1u << lane) - 1u));
        if (q && pos < ENT_LIST) list[pos] = g;
        nq += __popc(bq);
      }
      __syncwarp();
      if (nq > ENT_LIST) fast = false;
      if (fast) {
        // ---- candidates: maxima >= t0 of groups not re-read, elements >= t0 of re-read
        // groups, the tail.  One pass writes each lane's into its own segment of `cand`;
        // they are then packed lane-major into the summary area (no longer needed), the
        // order a counted two-pass gather gives.  A lane whose segment overflows sends the
        // row to that two-pass gather.
        constexpr int SEG = ENT_CAND / 32;
        float* seg = cand + lane * SEG;
        int c = 0;
        for (int g = lane; g < ngroups; g += 32) {
          const float mx = GTop2<T>::val(g1[g]);
          if (GTop2<T>::val(sec[g]) < t0 && mx >= t0) {
            if (c < SEG) seg[c] = mx;
            ++c;
          }
        }
        for (int j = lane; j < nq; j += 32) {
          const int g = list[j];
          const int64_t s = g >> 5, ln = g & 31;
#pragma unroll
          for (int v = 0; v < ENT_U; ++v) {
            const int64_t vi = s * per_step + v * 32 + ln;
            if (vi < nvec) {
              float f[EPV];
              Vec<T>::unpack(ldg16(z + vi * EPV), f);
#pragma unroll
              for (int e = 0; e < EPV; ++e) {
                if (f[e] >= t0) {
                  if (c < SEG) seg[c] = f[e];
                  ++c;
                }
              }
            }
          }
        }
        const int64_t te = tail0 + lane;
        const float tv = te < V ? to_f(z[te]) : -INFINITY;
        if (te < V && tv >= t0) {
          if (c < SEG) seg[c] = tv;
          ++c;
        }
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(FULL, incl, o);
          if (lane >= o) incl += y;
        }
        ncand = __shfl_sync(FULL, incl, 31);
        const bool over = __any_sync(FULL, c > SEG);
        if (ncand > ENT_CAND) {
          fast = false;
        } else if (!over && pack_ok) {
          __syncwarp();
          float* dst = reinterpret_cast<float*>(gtop);
          for (int i = 0; i < c; ++i) dst[incl - c + i] = seg[i];
          __syncwarp();
          cbuf = dst;
        } else {
          // ---- gather again (same traversal, same per-lane order)
          __syncwarp();
          int pos = incl - c;
          for (int g = lane; g < ngroups; g += 32)
            if (GTop2<T>::val(sec[g]) < t0 && GTop2<T>::val(g1[g]) >= t0) cand[pos++] = GTop2<T>::val(g1[g]);
          for (int j = lane; j < nq; j += 32) {
            const int g = list[j];
            const int64_t s = g >> 5, ln = g & 31;
#pragma unroll
            for (int v = 0; v < ENT_U; ++v) {
              const int64_t vi = s * per_step + v * 32 + ln;
              if (vi < nvec) {
                float f[EPV];
                Vec<T>::unpack(ldg16(z + vi * EPV), f);
#pragma unroll
                for (int e = 0; e < EPV; ++e)
                  if (f[e] >= t0) cand[pos++] = f[e];
              }
            }
          }
          if (te < V && tv >= t0) cand[pos++] = tv;
          __syncwarp();
        }
      }
    }
    float fillv = -INFINITY;
    int fillc = 0;
    const float* buf;
    int cnt;
    if (fast) {
      buf = cbuf;
      cnt = ncand;
      if (cnt >= k) {
        // exact k-th largest of the candidates; top-k = {x > v} plus copies of v
        const float v = warp_kth_largest(cbuf, cnt, k, hist, lane, passes);
        int out = 0;
        for (int base = 0; base < cnt; base += 32) {
          const int i = base + lane;
          const float x = i < cnt ? cbuf[i] : -INFINITY;
          const bool keep = i < cnt && x > v;
          const unsigned m = __ballot_sync(FULL, keep);
          __syncwarp();
          if (keep) cbuf[out + __popc(m & ((1u << lane) - 1u))] = x;
          out += __popc(m);
          __syncwarp();
        }
        cnt = out;
        fillv = v;
        fillc = k - out;
      }
    } else {
      // ---- fallback: streaming pass with a running threshold
      EntRow<T> st;
      st.buf = region;
      st.hist = hist;
      st.cap = cap;
      st.k = k;
      st.passes = passes;
      st.lane = lane;
      st.thr = -INFINITY;
      st.cnt = 0;
      st.nfill = 0;
      uint4 a[ENT_U];
      for (int64_t s = 0; s < nsteps; ++s) {
#pragma unroll
        for (int v = 0; v < ENT_U; ++v) {
          const int64_t vi = s * per_step + v * 32 + lane;
          a[v] = vi < nvec ? ldg16(z + vi * EPV) : EntVec<T>::sentinel();
        }
        st.step(a);
      }
      for (int64_t e0 = tail0; e0 < V; e0 += 32) {
        const int64_t e = e0 + lane;
        st.scalar(e < V ? to_f(z[e]) : -INFINITY);
      }
      if (st.cnt >= k) {
        warp_prune(st.buf, st.cnt, k, st.hist, lane, st.passes, st.thr, st.nfill);
        fillv = st.thr;
        fillc = st.nfill;
      } else {
        fillv = st.thr;
        fillc = k - st.cnt;
      }
      buf = st.buf;
      cnt = st.cnt;
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

static int ent_cap(int k, size_t es) { return k + 32 * ENT_U * (16 / (int)es); }

cudaError_t launch_entropy(const void* logits, kvc_dtype dt, int64_t rows, int64_t V,
                           int64_t row_stride, int k, float* H, cudaStream_t st, int sms) {
  if (rows <= 0) return cudaSuccess;
  const int kk = (int)(k < V ? k : V);
  const size_t es = dt == KVC_BF16 ? 2 : 4;
  const int cap = ent_cap(kk, es);
  const bool vec_ok = ((uintptr_t)logits % 16 == 0) && ((row_stride * es) % 16 == 0);
  // per-warp shared memory: histogram + [group top-2 | candidates | group list], the
  // bracketed region doubling as the fallback's candidate buffer of `cap` values
  const int64_t epv = 16 / (int64_t)es;
  const int64_t nsteps = (V / epv + 32 * ENT_U - 1) / (32 * ENT_U);
  int gcap = (int)(nsteps * 32);
  const size_t gbytes = (2 * (size_t)gcap * es + 15) / 16 * 16;
  size_t region = gbytes + ENT_CAND * 4 + ENT_LIST * 4;
  const size_t fb = (size_t)cap * 4;
  if (region < fb) region = fb;
  size_t warp_bytes = 1024 + region;
  warp_bytes = (warp_bytes + 127) / 128 * 128;
  const size_t budget = 220 * 1024;
  int nwarps = (int)(budget / warp_bytes);
  if (nwarps > ENT_WARPS) nwarps = ENT_WARPS;
  if (nwarps < 1) {            // enormous vocabularies: no group maxima, streaming path only
    gcap = 0;
    warp_bytes = (1024 + fb + 127) / 128 * 128;
    nwarps = (int)(budget / warp_bytes);
    if (nwarps < 1) return cudaErrorInvalidValue;
    if (nwarps > ENT_WARPS) nwarps = ENT_WARPS;
  }
  const size_t smem = (size_t)nwarps * warp_bytes;
  const int64_t want = (rows + nwarps - 1) / nwarps;
  const int64_t maxb = (int64_t)(sms > 0 ? sms : num_sms()) * (smem <= 110 * 1024 ? 2 : 1);
  const int grid = (int)(want < maxb ? want : maxb);
  if (dt == KVC_BF16) {
    auto kern = entropy_twopass_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, nwarps * 32, smem, st>>>((const __nv_bfloat16*)logits, rows, V, row_stride, kk, cap,
                                           vec_ok, nwarps, gcap, warp_bytes, H);
    count_launch();
  } else {
    auto kern = entropy_twopass_kernel<float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, nwarps * 32, smem, st>>>((const float*)logits, rows, V, row_stride, kk, cap, vec_ok,
                                           nwarps, gcap, warp_bytes, H);
    count_launch();
  }
  return cudaGetLastError();
}

}  // namespace kvc
