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

// SIDE: the per-token side arrays (position, H, D, and the RECAS attention history U)
// travel too; lane v < 4 of a row's threads carries side array v (a row has at least 8
// vectors: head_dim 64 or 128).
template <bool SIDE>
__global__ void __launch_bounds__(CP_THREADS, 4) compact_kernel(CompactParams p) {
  const int lg = blockIdx.x, l = lg / p.Hkv, g = lg % p.Hkv;
  const int kl = min(p.k[l], p.k_cap);
  const int rpb = CP_THREADS / p.vr;                       // rows per step
  const int r_in = threadIdx.x / p.vr, v = threadIdx.x % p.vr;
  if (r_in >= rpb) return;
  const int j0 = blockIdx.y * rpb * CP_ROWS_PER_THREAD;
  // this lane's side array: source row (null: the position is the source index itself)
  // and destination row (null: not wanted)
  const uint32_t* s_src = nullptr;
  uint32_t* s_dst = nullptr;
  if (SIDE && v < 4) {
    const int64_t o = (int64_t)lg * p.dside_row;
    if (v == 0) {
      s_src = reinterpret_cast<const uint32_t*>(p.spos ? p.spos + l * p.psl + g * p.psh : nullptr);
      s_dst = reinterpret_cast<uint32_t*>(p.dpos ? p.dpos + o : nullptr);
    } else if (v == 1) {
      s_src = reinterpret_cast<const uint32_t*>(p.sH + l * p.Hsl + g * p.Hsh);
      s_dst = reinterpret_cast<uint32_t*>(p.dH ? p.dH + o : nullptr);
    } else if (v == 2) {
      s_src = reinterpret_cast<const uint32_t*>(p.sD + l * p.Dsl + g * p.Dsh);
      s_dst = reinterpret_cast<uint32_t*>(p.dD ? p.dD + o : nullptr);
    } else if (p.sU) {
      s_src = reinterpret_cast<const uint32_t*>(p.sU + l * p.Usl + g * p.Ush);
      s_dst = reinterpret_cast<uint32_t*>(p.dU ? p.dU + o : nullptr);
    }
  }
  // this thread's 16-byte column of the (l, g) source and destination rows
  const char* kb = p.sK ? p.sK + l * p.sKl + g * p.sKh + v * 16 : nullptr;
  const char* vb = p.sV ? p.sV + l * p.sVl + g * p.sVh + v * 16 : nullptr;
  int src[CP_ROWS_PER_THREAD];
  uint32_t sv[SIDE ? CP_ROWS_PER_THREAD : 1];
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
      if (kb) kv[t] = ldg16(kb + (int64_t)src[t] * p.sKt);
      if (vb) vv[t] = ldg16(vb + (int64_t)src[t] * p.sVt);
      // side arrays: issued with the row loads, so all of them are in flight together
      if (SIDE && s_dst) sv[t] = s_src ? __ldg(s_src + src[t]) : (uint32_t)src[t];
    }
  }
  char* dkb = p.dK ? p.dK + l * p.dKl + g * p.dKh + v * 16 : nullptr;
  char* dvb = p.dV ? p.dV + l * p.dVl + g * p.dVh + v * 16 : nullptr;
#pragma unroll
  for (int t = 0; t < CP_ROWS_PER_THREAD; ++t) {
    const int j = j0 + t * rpb + r_in;
    if (src[t] < 0) continue;
    if (dkb) *reinterpret_cast<uint4*>(dkb + (int64_t)j * p.dKt) = kv[t];
    if (dvb) *reinterpret_cast<uint4*>(dvb + (int64_t)j * p.dVt) = vv[t];
    if (SIDE && s_dst) s_dst[j] = sv[t];
  }
}

cudaError_t launch_compact(const CompactParams& p, cudaStream_t st) {
  const int rpb = CP_THREADS / p.vr;
  const int per_block = rpb * CP_ROWS_PER_THREAD;
  dim3 grid(p.L * p.Hkv, (p.k_cap + per_block - 1) / per_block);
  if (grid.y == 0) return cudaSuccess;
  if (p.dpos || p.dH || p.dD || p.dU) compact_kernel<true><<<grid, CP_THREADS, 0, st>>>(p);
  else compact_kernel<false><<<grid, CP_THREADS, 0, st>>>(p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace kvc
