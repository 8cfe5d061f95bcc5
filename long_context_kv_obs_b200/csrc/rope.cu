// RoPE re-positioning of the kept keys.
//
// [SelKV] Pipeline overview, step 6 "RoPE re-positioning": after selection
// and merging, the kept keys are re-embedded at contiguous positions (the
// pages switch the step off for long-context evaluation).  A key carrying the
// rotary embedding of position p has every dimension pair (x_i, x_{i+d/2})
// turned by p * theta_i, theta_i = base^(-2i/d); moving it to p' is one more
// turn by (p' - p) * theta_i.  Row j of (l, g) moves from pos(l, g, j) to
// new0 + j.
//
// HBM-bound: each row is read once and written once (in place or to another
// buffer).  A thread owns one 16-byte vector of each half of a row, i.e. 8
// (bf16) or 4 (fp32) pairs, and loads two rows before turning either.
// Angles reach 1e5 radians, beyond what an fp32 product can carry (its
// rounding alone is ~4e-3 rad there), so each angle is formed and reduced
// modulo pi/2 in fp64 (Cody-Waite: pi/2 split into a double and the double of
// its remainder).  The reduced angle r, |r| <= pi/4, is rounded to fp32 and
// its sine and cosine come from their Taylor series to degree 9 and 10
// (truncation below 2e-9 on that interval), two pairs' series at a time on packed
// fp32 pairs; the quadrant picks signs and swaps.  Sine and cosine are within 1e-7 of
// the exact values.
#include <type_traits>

#include "kernels.cuh"

namespace kvc {

constexpr int RP_THREADS = 256;
constexpr double RP_2_OVER_PI = 0.6366197723675814;         // 2 / pi
constexpr double RP_PIO2_HI = 1.5707963267948966;           // pi / 2 rounded to a double
constexpr double RP_PIO2_LO = 6.123233995736766e-17;        // pi / 2 - RP_PIO2_HI
// Rounding by the 1.5 * 2^52 shifter: for |x| < 2^51, x + 1.5 * 2^52 rounded to a double
// is 1.5 * 2^52 + rint(x), whose low mantissa bits hold rint(x) in two's complement.
constexpr double RP_SHIFTER = 6755399441055744.0;

// packed fp32 product of two pairs (each lane rounds as mul.rn.f32)
__device__ __forceinline__ uint64_t rp_mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// sin and cos of two angles phi0, phi1 (radians, fp64): each phi = q pi/2 + r, reduced in
// fp64, then the Taylor series at r for both angles at once on packed fp32 pairs (each lane
// rounds as the scalar instruction).  Also -sin, for the rotation's negated product.
__device__ __forceinline__ void rp_sincos2(double phi0, double phi1, float (&sn)[2], float (&nsn)[2],
                                           float (&cs)[2]) {
  const double sh[2] = {fma(phi0, RP_2_OVER_PI, RP_SHIFTER), fma(phi1, RP_2_OVER_PI, RP_SHIFTER)};
  const double ph[2] = {phi0, phi1};
  float rf[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const double q = sh[i] - RP_SHIFTER;
    double rr = fma(-q, RP_PIO2_HI, ph[i]);
    rr = fma(-q, RP_PIO2_LO, rr);
    rf[i] = (float)rr;
  }
  const uint64_t r = pk2(rf[0], rf[1]);
  const uint64_t t = rp_mul2(r, r);
  // sin r = r (1 - t/3! + t^2/5! - t^3/7! + t^4/9!),  cos r = 1 - t/2! + ... + t^5/10!
  uint64_t ps = fma2(t, pk2(1.f / 362880.f, 1.f / 362880.f), pk2(-1.f / 5040.f, -1.f / 5040.f));
  ps = fma2(t, ps, pk2(1.f / 120.f, 1.f / 120.f));
  ps = fma2(t, ps, pk2(-1.f / 6.f, -1.f / 6.f));
  const float2 s = upk2(fma2(rp_mul2(r, t), ps, r));
  uint64_t pc = fma2(t, pk2(-1.f / 3628800.f, -1.f / 3628800.f), pk2(1.f / 40320.f, 1.f / 40320.f));
  pc = fma2(t, pc, pk2(-1.f / 720.f, -1.f / 720.f));
  pc = fma2(t, pc, pk2(1.f / 24.f, 1.f / 24.f));
  pc = fma2(t, pc, pk2(-0.5f, -0.5f));
  const float2 c = upk2(fma2(t, pc, pk2(1.f, 1.f)));
  const float s2[2] = {s.x, s.y}, c2[2] = {c.x, c.y};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int quad = __double2loint(sh[i]) & 3;  // sin(r + k pi/2), cos(r + k pi/2)
    const float s_ = (quad & 1) ? c2[i] : s2[i], c_ = (quad & 1) ? s2[i] : c2[i];
    sn[i] = (quad & 2) ? -s_ : s_;
    nsn[i] = (quad & 2) ? s_ : -s_;
    cs[i] = ((quad + 1) & 2) ? -c_ : c_;
  }
}

// one 16-byte vector from 8 (bf16, rounded to nearest even) or 4 (fp32) floats
__device__ __forceinline__ uint4 rp_pack(const float* f, __nv_bfloat16*) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}
__device__ __forceinline__ uint4 rp_pack(const float* f, float*) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
}

template <bool BF16>
__global__ void __launch_bounds__(RP_THREADS, 4) rope_kernel(const RopeParams p) {
  constexpr int P = BF16 ? 8 : 4;                 // pairs per thread
  using T = typename std::conditional<BF16, __nv_bfloat16, float>::type;
  const int h = p.d / 2;
  const int tpr = h / P;                          // threads per row (4 .. 16, a power of two)
  const int rpb = RP_THREADS / tpr;               // rows per block step
  const int part = threadIdx.x % tpr;
  const int i0 = part * P;
  const int lane = threadIdx.x & 31;
  const unsigned rowmask = ((1u << tpr) - 1u) << (lane & ~(tpr - 1));   // this row's lanes
  // the frequencies go through shared memory: read from the parameter bank, each lane of a
  // row at its own index, every load would be serialised
  __shared__ double s_theta[64];
  if (threadIdx.x < h) s_theta[threadIdx.x] = p.theta[threadIdx.x];
  __syncthreads();
  const double* th = s_theta + i0;
  const int64_t rows = (int64_t)p.L * p.Hkv * p.k_cap;
  const int64_t step = (int64_t)gridDim.x * rpb;
  // two rows per trip (r and r + step), both loaded before either is turned
  for (int64_t r0 = (int64_t)blockIdx.x * rpb + threadIdx.x / tpr; r0 < rows; r0 += 2 * step) {
    uint4 ua[2], ub[2];
    int jj[2], ll[2], gg[2];
    int64_t lgg[2];
    double shift[2];
    bool act[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t r = r0 + u * step;
      act[u] = false;
      if (r >= rows) continue;
      const int64_t lg = r / p.k_cap;
      const int j = (int)(r - lg * p.k_cap);
      const int l = (int)(lg / p.Hkv), g = (int)(lg - (int64_t)l * p.Hkv);
      lgg[u] = lg; jj[u] = j; ll[u] = l; gg[u] = g;
      if (j >= min(p.k[l], p.k_cap)) continue;    // the whole row's lanes take the same branch
      act[u] = true;
      const int32_t old = p.pos[lg * p.pos_row + j];
      shift[u] = (double)(p.new0 + j - (int64_t)old);
      const char* srow = p.src + l * p.sl + g * p.sh + (int64_t)j * p.st;
      ua[u] = ldg16(srow + (size_t)i0 * sizeof(T));
      ub[u] = ldg16(srow + (size_t)(h + i0) * sizeof(T));
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (!act[u]) continue;
      float x1[P], x2[P];
      Vec<T>::unpack(ua[u], x1);
      Vec<T>::unpack(ub[u], x2);
      // pairs e, e + 1 together: x1 cos - x2 sin and x2 cos + x1 sin on packed fp32 pairs,
      // the first product taken with -sin (the same value as the negated product)
#pragma unroll
      for (int e = 0; e < P; e += 2) {
        float sn[2], nsn[2], cs[2];
        rp_sincos2(shift[u] * th[e], shift[u] * th[e + 1], sn, nsn, cs);
        const uint64_t a2 = pk2(x1[e], x1[e + 1]), b2 = pk2(x2[e], x2[e + 1]), cs2 = pk2(cs[0], cs[1]);
        const float2 y1 = upk2(fma2(a2, cs2, rp_mul2(b2, pk2(nsn[0], nsn[1]))));
        const float2 y2 = upk2(fma2(b2, cs2, rp_mul2(a2, pk2(sn[0], sn[1]))));
        x1[e] = y1.x;
        x1[e + 1] = y1.y;
        x2[e] = y2.x;
        x2[e + 1] = y2.y;
      }
      char* drow = p.dst + ll[u] * p.dl + gg[u] * p.dh + (int64_t)jj[u] * p.dt;
      *reinterpret_cast<uint4*>(drow + (size_t)i0 * sizeof(T)) = rp_pack(x1, (T*)nullptr);
      *reinterpret_cast<uint4*>(drow + (size_t)(h + i0) * sizeof(T)) = rp_pack(x2, (T*)nullptr);
      if (p.pos_dst) {
        __syncwarp(rowmask);                      // every lane of the row has read pos (it may be pos_dst)
        if (part == 0) p.pos_dst[lgg[u] * p.pos_row + jj[u]] = (int32_t)(p.new0 + jj[u]);
      }
    }
  }
}

cudaError_t launch_rope(const RopeParams& p, cudaStream_t st) {
  const int64_t rows = (int64_t)p.L * p.Hkv * p.k_cap;
  if (rows == 0) return cudaSuccess;
  const int P = p.bf16 ? 8 : 4;
  const int tpr = p.d / 2 / P;
  const int64_t rpb = RP_THREADS / tpr;
  int64_t grid = (rows + rpb - 1) / rpb;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (grid > cap) grid = cap;
  if (p.bf16) rope_kernel<true><<<(unsigned)grid, RP_THREADS, 0, st>>>(p);
  else rope_kernel<false><<<(unsigned)grid, RP_THREADS, 0, st>>>(p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace kvc
