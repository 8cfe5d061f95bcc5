// Compaction of the kept rows.
//
// [InfoKV] Technical details: each layer keeps its top k_l tokens.  dst row j
// of (l, g) is a bit-exact copy of src row idx(l, g, j); the per-token side
// arrays (original position, H, D) travel with it so the token can be
// rescored at a later compression.
//
// Each thread moves one 16-byte vector of one row for both K and V; a row of
// 128 bf16 is 16 threads, so a 256-thread CTA moves 16 rows per step with
// fully coalesced 256-byte row reads and writes.
#include "kernels.cuh"

namespace kvc {



constexpr int CP_THREADS = 256;
constexpr int CP_ROWS_PER_THREAD = 4;

// SIDE: the per-token side arrays (position, H, D) travel too.
template <bool SIDE>
__global__ void __launch_bounds__(CP_THREADS) compact_kernel(CompactParams p) {
  const int lg = blockIdx.x, l = lg / p.Hkv, g = lg % p.Hkv;
  const int kl = min(p.k[l], p.k_cap);
  const int rpb = CP_THREADS / p.vr;                       // rows per step
  const int r_in = threadIdx.x / p.vr, v = threadIdx.x % p.vr;
  if (r_in >= rpb) return;
  const int j0 = blockIdx.y * rpb * CP_ROWS_PER_THREAD;
  int src[CP_ROWS_PER_THREAD], spv[SIDE ? CP_ROWS_PER_THREAD : 1];
  float shv[SIDE ? CP_ROWS_PER_THREAD : 1], sdv[SIDE ? CP_ROWS_PER_THREAD : 1];
  uint4 kv[CP_ROWS_PER_THREAD], vv[CP_ROWS_PER_THREAD];
#pragma unroll
  for (int t = 0; t < CP_ROWS_PER_THREAD; ++t) {
    const int j = j0 + t * rpb + r_in;
    src[t] = -1;
    if (j < kl) {
      int s = p.idx[(int64_t)lg * p.k_cap + j];
      if (s < 0 || s >= p.n) {
        flag(p.status, ST_BOUNDS);
        s = -1;
      }
      src[t] = s;
    }
    if (src[t] >= 0) {
      if (p.sK) kv[t] = ldg16(p.sK + l * p.sKl + g * p.sKh + (int64_t)src[t] * p.sKt + v * 16);
      if (p.sV) vv[t] = ldg16(p.sV + l * p.sVl + g * p.sVh + (int64_t)src[t] * p.sVt + v * 16);
      // side arrays: issued with the row loads, so all of them are in flight together
      if (SIDE && v == 0) {
        spv[t] = p.spos ? __ldg(p.spos + l * p.psl + g * p.psh + src[t]) : src[t];
        if (p.dH) shv[t] = __ldg(p.sH + l * p.Hsl + g * p.Hsh + src[t]);
        if (p.dD) sdv[t] = __ldg(p.sD + l * p.Dsl + g * p.Dsh + src[t]);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < CP_ROWS_PER_THREAD; ++t) {
    const int j = j0 + t * rpb + r_in;
    if (src[t] < 0) continue;
    if (p.dK) *reinterpret_cast<uint4*>(p.dK + l * p.dKl + g * p.dKh + (int64_t)j * p.dKt + v * 16) = kv[t];
    if (p.dV) *reinterpret_cast<uint4*>(p.dV + l * p.dVl + g * p.dVh + (int64_t)j * p.dVt + v * 16) = vv[t];
    if (SIDE && v == 0) {
      const int64_t o = (int64_t)lg * p.dside_row + j;
      if (p.dpos) p.dpos[o] = spv[t];
      if (p.dH) p.dH[o] = shv[t];
      if (p.dD) p.dD[o] = sdv[t];
    }
  }
}

cudaError_t launch_compact(const CompactParams& p, cudaStream_t st) {
  const int rpb = CP_THREADS / p.vr;
  const int per_block = rpb * CP_ROWS_PER_THREAD;
  dim3 grid(p.L * p.Hkv, (p.k_cap + per_block - 1) / per_block);
  if (grid.y == 0) return cudaSuccess;
  if (p.dpos || p.dH || p.dD) compact_kernel<true><<<grid, CP_THREADS, 0, st>>>(p);
  else compact_kernel<false><<<grid, CP_THREADS, 0, st>>>(p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace kvc
