// Per-step cache bookkeeping of decode-time compression, on the device.
//
// [InfoKV] Technical details: under decode-time compression every generated
// token enters the cache with the signals it will be rescored with at the next
// compression (its position, its entropy H and its representation change D per
// layer), and the last W generated queries form the observation window of that
// compression.  [SelKV] Methodology / Core component 2: a token that was not
// merged carries the attention ratio R = 1.  [RECAS] 2.B: the dropped-mass probe
// needs to know which positions of the full history are still cached.
//
// append_kernel: one CTA per (sequence, layer).  Row len[b][l] of every KV head
// receives the token's key and value rows (16-byte vectors), its side-array
// entries and its kept bit; the window-query ring slot receives the query of every
// query head; len[b][l] is then incremented.  An optional second cache (the full
// history) receives the same key and value rows at its own row len2[b][l], from the
// same loads.  kept_bits_kernel: one CTA per
// (sequence, layer, KV head) row rebuilds the kept-position bit mask of a row from
// the positions its cache holds after a compression.
#include "kernels.cuh"

namespace kvc {

constexpr int AP_THREADS = 256;

__global__ void __launch_bounds__(AP_THREADS) append_kernel(AppendParams p) {
  const int bl = blockIdx.x, b = bl / p.L, l = bl % p.L;
  const int len = p.len[bl];
  const int len2 = p.K2 ? p.len2[bl] : 0;
  __syncthreads();                               // every thread has read len before it moves
  if (len < 0 || len >= p.cap || (p.K2 && (len2 < 0 || len2 >= p.cap2))) {
    if (threadIdx.x == 0) flag(p.status, ST_BOUNDS);
    return;
  }
  // key and value rows: Hkv rows of vr 16-byte vectors each, into one or two caches
  const int nv = p.Hkv * p.vr;
  for (int i = threadIdx.x; i < nv; i += AP_THREADS) {
    const int g = i / p.vr, v = i % p.vr;
    const int64_t src = ((int64_t)bl * p.Hkv + g) * p.row_bytes + v * 16;
    const uint4 kk = ldg16(p.k + src);
    const uint4 vv = ldg16(p.v + src);
    *reinterpret_cast<uint4*>(p.K + b * p.Ksb + l * p.Ksl + g * p.Ksh + len * p.Kst + v * 16) = kk;
    *reinterpret_cast<uint4*>(p.V + b * p.Vsb + l * p.Vsl + g * p.Vsh + len * p.Vst + v * 16) = vv;
    if (p.K2) {
      *reinterpret_cast<uint4*>(p.K2 + b * p.K2sb + l * p.K2sl + g * p.K2sh + len2 * p.K2st + v * 16) = kk;
      *reinterpret_cast<uint4*>(p.V2 + b * p.V2sb + l * p.V2sl + g * p.V2sh + len2 * p.V2st + v * 16) = vv;
    }
  }
  // side arrays and the kept bit, one KV head per thread
  for (int g = threadIdx.x; g < p.Hkv; g += AP_THREADS) {
    const int64_t o = ((int64_t)bl * p.Hkv + g) * p.side_row + len;
    if (p.spos) p.spos[o] = p.pos;
    if (p.sH) p.sH[o] = p.H_new[b];
    if (p.sD) p.sD[o] = p.D_new[b * p.Dnb + l * p.Dnl];
    if (p.sR) p.sR[o] = 1.f;
    if (p.sU) p.sU[o] = 0.f;
    if (p.bits) atomicOr(p.bits + b * p.bsb + l * p.bsl + g * p.bsh + (p.pos >> 5), 1u << (p.pos & 31));
  }
  // window-query ring: slot `slot` of every query head
  if (p.q) {
    const int nq = p.Hq * p.vr;
    for (int i = threadIdx.x; i < nq; i += AP_THREADS) {
      const int h = i / p.vr, v = i % p.vr;
      const int64_t qh = (int64_t)bl * p.Hq + h;
      const uint4 qq = ldg16(p.q + qh * p.row_bytes + v * 16);
      *reinterpret_cast<uint4*>(p.Qring + (qh * p.W + p.slot) * p.row_bytes + v * 16) = qq;
    }
    if (l == 0 && threadIdx.x == 0) p.qpos[(int64_t)b * p.W + p.slot] = p.pos;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    p.len[bl] = len + 1;
    if (p.K2) p.len2[bl] = len2 + 1;
  }
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t st) {
  append_kernel<<<p.B * p.L, AP_THREADS, 0, st>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

constexpr int KB_THREADS = 256;

// Row r of `rows` (folded sequence-layer index lb = r / Hkv, KV head g = r % Hkv): clear
// the row's words, then set the bit of every kept position pos[r][j], j < k[lb].
__global__ void __launch_bounds__(KB_THREADS) kept_bits_kernel(const int32_t* pos, int64_t pos_row,
                                                               const int32_t* k, int k_cap, int Hkv, int L,
                                                               uint32_t* bits, int64_t bsb, int64_t bsl,
                                                               int64_t bsh, int words, unsigned* status) {
  const int r = blockIdx.x, lb = r / Hkv, g = r % Hkv, b = lb / L, l = lb % L;
  uint32_t* row = bits + b * bsb + l * bsl + g * bsh;
  for (int w = threadIdx.x; w < words; w += KB_THREADS) row[w] = 0u;
  __syncthreads();
  const int kl = min(k[lb], k_cap);
  const int32_t* pr = pos + (int64_t)r * pos_row;
  for (int j = threadIdx.x; j < kl; j += KB_THREADS) {
    const int x = pr[j];
    if (x < 0 || (x >> 5) >= words) {
      flag(status, ST_BOUNDS);
      continue;
    }
    atomicOr(row + (x >> 5), 1u << (x & 31));
  }
}

cudaError_t launch_kept_bits(const int32_t* pos, int64_t pos_row, const int32_t* k, int k_cap, int B, int L,
                             int Hkv, uint32_t* bits, int64_t bsb, int64_t bsl, int64_t bsh, int words,
                             cudaStream_t st) {
  kept_bits_kernel<<<B * L * Hkv, KB_THREADS, 0, st>>>(pos, pos_row, k, k_cap, Hkv, L, bits, bsb, bsl, bsh,
                                                       words, status_ptr());
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

}  // namespace kvc
