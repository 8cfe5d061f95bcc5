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
// (bf16) or 4 (fp32) pairs.  Angles reach 1e5 radians, beyond what an fp32
// product can carry (its rounding alone is ~4e-3 rad there), so each angle is
// formed and reduced modulo 2 pi in fp64 (Cody-Waite: 2 pi split into a
// double and the double of its remainder), and only the reduced angle, in
// [-pi, pi], goes to sincosf.
#include <type_traits>

#include "kernels.cuh"

namespace kvc {

constexpr int RP_THREADS = 256;
constexpr double RP_INV_2PI = 0.15915494309189535;          // 1 / (2 pi)
constexpr double RP_2PI_HI = 6.283185307179586;             // 2 pi rounded to a double
constexpr double RP_2PI_LO = 2.4492935982947064e-16;        // 2 pi - RP_2PI_HI

// one 16-byte vector from 8 (bf16, rounded to nearest even) or 4 (fp32) floats
__device__ __forceinline__ uint4 rp_pack(const float* f, __nv_bfloat16*) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}
__device__ __forceinline__ uint4 rp_pack(const float* f, float*) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
}

template <bool BF16>
__global__ void __launch_bounds__(RP_THREADS) rope_kernel(const RopeParams p) {
  constexpr int P = BF16 ? 8 : 4;                 // pairs per thread
  using T = typename std::conditional<BF16, __nv_bfloat16, float>::type;
  const int h = p.d / 2;
  const int tpr = h / P;                          // threads per row (4 .. 16, a power of two)
  const int rpb = RP_THREADS / tpr;               // rows per block step
  const int part = threadIdx.x % tpr;
  const int i0 = part * P;
  const int lane = threadIdx.x & 31;
  const unsigned rowmask = ((1u << tpr) - 1u) << (lane & ~(tpr - 1));   // this row's lanes
  double th[P];
#pragma unroll
  for (int e = 0; e < P; ++e) th[e] = p.theta[i0 + e];
  const int64_t rows = (int64_t)p.L * p.Hkv * p.k_cap;
  for (int64_t r = (int64_t)blockIdx.x * rpb + threadIdx.x / tpr; r < rows; r += (int64_t)gridDim.x * rpb) {
    const int64_t lg = r / p.k_cap;
    const int j = (int)(r - lg * p.k_cap);
    const int l = (int)(lg / p.Hkv), g = (int)(lg - (int64_t)l * p.Hkv);
    if (j >= min(p.k[l], p.k_cap)) continue;      // the whole row's lanes take the same branch
    const int32_t old = p.pos[lg * p.pos_row + j];
    const double shift = (double)(p.new0 + j - (int64_t)old);
    const char* srow = p.src + l * p.sl + g * p.sh + (int64_t)j * p.st;
    const uint4 ua = ldg16(srow + (size_t)i0 * sizeof(T));
    const uint4 ub = ldg16(srow + (size_t)(h + i0) * sizeof(T));
    float x1[P], x2[P];
    Vec<T>::unpack(ua, x1);
    Vec<T>::unpack(ub, x2);
    float y1[P], y2[P];
#pragma unroll
    for (int e = 0; e < P; ++e) {
      const double ph = shift * th[e];
      const double q = rint(ph * RP_INV_2PI);
      double rr = fma(-q, RP_2PI_HI, ph);
      rr = fma(-q, RP_2PI_LO, rr);
      float sn, cs;
      sincosf((float)rr, &sn, &cs);
      y1[e] = fmaf(x1[e], cs, -x2[e] * sn);
      y2[e] = fmaf(x2[e], cs, x1[e] * sn);
    }
    char* drow = p.dst + l * p.dl + g * p.dh + (int64_t)j * p.dt;
    *reinterpret_cast<uint4*>(drow + (size_t)i0 * sizeof(T)) = rp_pack(y1, (T*)nullptr);
    *reinterpret_cast<uint4*>(drow + (size_t)(h + i0) * sizeof(T)) = rp_pack(y2, (T*)nullptr);
    if (p.pos_dst) {
      __syncwarp(rowmask);                        // every lane of the row has read pos (it may be pos_dst)
      if (part == 0) p.pos_dst[lg * p.pos_row + j] = (int32_t)(p.new0 + j);
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
