// Decode attention on the tensor cores: o = softmax(q K^T * scale + alpha_c log R) V.
//
// [SelKV] Methodology, core component 2 (attention compensation at decode).
// [RECAS] dropped-mass probe (PROBE = true): over the full history with a bit per
// position saying whether the compressed cache kept it, the same pass gives the
// kept and evicted softmax mass, the output over all keys and over kept keys only,
// and the largest value norm (delta, o, o', V_max of the probe).
//
// Decode attention streams K and V once and does 2 x 128 multiply-adds per
// key and query head, so it is bound by HBM, but on CUDA cores the per-key
// instruction count (bf16 unpacking, dot-product reductions, the weighted V
// sum) caps it well below the bandwidth.  Here both contractions run as
// mma.sync m16n8k16 (bf16 operands, fp32 accumulation), the G <= 8 query heads
// of a KV head padded to the 16 rows of the A operand:
//   S = Q K^T   A = q rows (exact bf16), B = K rows read by ldmatrix
//   O += P V    A = P as bf16 hi + lo parts (two MMAs: P is carried to about
//               16 bits, so O keeps fp32-level accuracy), B = V rows read by
//               ldmatrix.trans
// The softmax runs online per head in the accumulator layout (log2 units,
// rescaled only when the running max grows by more than 2^8).
//
// Memory: a producer warp loads 64-key chunks of K and V with TMA (128B
// swizzle, so ldmatrix reads are bank-conflict free) into a ring of stages;
// each of the four consumer warps takes 16 keys of every chunk with its own
// online state (every warp waits on every stage in order, so a stage's phase
// parity is never ambiguous), and releases the stage when done.  At the end of
// a (row, split) item the warps are merged in shared memory and the item's
// partial goes to the split combine.  Persistent CTAs, two per SM, take items
// c, c + grid, ...; the producer runs ahead across items.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "tc_sm100.cuh"

namespace kvc {
using namespace tc;

constexpr int DM_KEYS = 64;                  // keys per chunk (stage), 16 per consumer warp
constexpr int DM_CW = 4;                     // consumer warps
constexpr int DM_THREADS = 32 * (1 + DM_CW);
constexpr int DM_ATOM = DM_KEYS * 128;       // 64 rows x 64 bf16, 128B-swizzled (8 KB)
constexpr int DM_STAGE = 4 * DM_ATOM;        // K dims 0-63, 64-127, then V likewise (32 KB)
#ifndef KVC_DM_PER_SM
#define KVC_DM_PER_SM 2
#endif
constexpr int DM_PER_SM = KVC_DM_PER_SM;     // CTAs per SM
template <bool PROBE>
constexpr int dm_rec() { return PROBE ? 4 + 2 * 128 : 2 + 128; }   // split-combine record

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// C (16 x 8, fp32) += A (16 x 16, bf16, row) * B (16 x 8, bf16, col); rows 8-15 of A are zero.
__device__ __forceinline__ void mma_rows8(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
// The same with all 16 rows of A: rows 8-15 carry a second set of query rows.
__device__ __forceinline__ void mma_rows16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// Byte offset of 16-byte chunk ch (0-7) of row r inside a 128B-swizzled atom.
__device__ __forceinline__ uint32_t sw_off(int r, int ch) { return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4)); }

struct DmArgs {
  DecodeParams p;
  int nitems, nst;
};

// Partial record of one (row, split, head): [max, sum] then o[128] (plain);
// [max, kept sum, evicted sum, max |v|^2] then o_all[128], o_kept[128] (probe).
template <bool PROBE>
__global__ void __launch_bounds__(DM_THREADS, DM_PER_SM)
decode_mma_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                  const DmArgs a) {
  constexpr int DM_REC = dm_rec<PROBE>();
  const DecodeParams& p = a.p;
  const int NST = a.nst;
  extern __shared__ uint8_t dm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + (size_t)NST * DM_STAGE);
  uint64_t* empty = full + NST;
  int* abort_flag = reinterpret_cast<int*>(empty + NST);
  float* dsm = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(abort_flag) + 16);   // [CW][G][REC]
  volatile int* abort = abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], DM_CW);        // every consumer warp
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_map(&mapK);
    prefetch_map(&mapV);
  }
  __syncthreads();
  auto item_range = [&](int item, int& row, int& split, int& s0, int& s1) {
    row = item / p.nsplit;
    split = item % p.nsplit;
    const int b = row / (p.Hkv * p.L), l = (row / p.Hkv) % p.L;
    int n = p.len[b * p.L + l];
    if (n > p.max_len || n < 0) n = n < 0 ? 0 : p.max_len;   // flagged by the consumers
    s0 = split * p.split_len;
    s1 = min(n, s0 + p.split_len);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t chunk = 0;
      for (int item = blockIdx.x; item < a.nitems; item += gridDim.x) {
        int row, split, s0, s1;
        item_range(item, row, split, s0, s1);
        const int g = row % p.Hkv, l = (row / p.Hkv) % p.L, b = row / (p.Hkv * p.L);
        for (int i0 = s0; i0 < s1; i0 += DM_KEYS, ++chunk) {
          const int s = chunk % NST;
          if (!mbar_wait(&empty[s], ((chunk / NST) & 1) ^ 1, abort, p.status)) goto producer_done;
          mbar_expect_tx(&full[s], DM_STAGE);   // whole boxes, rows past the tensor read as 0
          uint8_t* st = ring + (size_t)s * DM_STAGE;
          tma_load_5d(st, &mapK, 0, i0, g, l, b, &full[s]);
          tma_load_5d(st + DM_ATOM, &mapK, 64, i0, g, l, b, &full[s]);
          tma_load_5d(st + 2 * DM_ATOM, &mapV, 0, i0, g, l, b, &full[s]);
          tma_load_5d(st + 3 * DM_ATOM, &mapV, 64, i0, g, l, b, &full[s]);
        }
      }
    producer_done:;
    }
    return;
  }
  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;
  const int gid = lane >> 2, tig = lane & 3;  // accumulator row (query head) and column pair
  const int G = p.G;
  uint32_t chunk = 0;
  for (int item = blockIdx.x; item < a.nitems; item += gridDim.x) {
    int row, split, s0, s1;
    item_range(item, row, split, s0, s1);
    const int g = row % p.Hkv, l = (row / p.Hkv) % p.L, b = row / (p.Hkv * p.L);
    if (cw == 0 && lane == 0 && split == 0) {
      const int n = p.len[b * p.L + l];
      if (n > p.max_len || n < 0) flag(p.status, ST_BOUNDS);
    }
    // A fragments of q (exact bf16): head gid, dims 16 kc + 2 tig (+1) and 16 kc + 8 + 2 tig (+1)
    uint32_t qa[8][2];
    {
      const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p.q) +
                               (((int64_t)b * p.L + l) * p.Hq + g * G + gid) * 128;
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {
        qa[kc][0] = gid < G ? __ldg(reinterpret_cast<const uint32_t*>(q + kc * 16 + 2 * tig)) : 0u;
        qa[kc][1] = gid < G ? __ldg(reinterpret_cast<const uint32_t*>(q + kc * 16 + 8 + 2 * tig)) : 0u;
      }
    }
    // accumulator rows 0-7: o of head gid; probe rows 8-15: o' of head gid (kept keys only)
    float O[16][4];
#pragma unroll
    for (int t = 0; t < 16; ++t) O[t][0] = O[t][1] = O[t][2] = O[t][3] = 0.f;
    float m = -INFINITY, lsum = 0.f;           // head gid, this lane's share of the (kept) sum
    float lev = 0.f, vmax2 = 0.f;              // probe: evicted sum share, max |v|^2 seen
    const float* Rr = p.R ? p.R + b * p.Rsb + l * p.Rsl + g * p.Rsh : nullptr;
    const uint32_t* Br = PROBE ? p.bits + b * p.bsb + l * p.bsl + g * p.bsh : nullptr;
    for (int i0 = s0; i0 < s1; i0 += DM_KEYS, ++chunk) {
      const int s = chunk % NST;
      bool ok = !*abort && mbar_wait(&full[s], (chunk / NST) & 1, abort, p.status);
      if (!__all_sync(FULL, ok)) continue;
      const int r0 = cw * 16;                  // this warp's keys of the chunk: r0 .. r0 + 15
      const int nk = min(DM_KEYS, s1 - i0) - r0;   // of them valid (may be <= 0)
      uint8_t* st = ring + (size_t)s * DM_STAGE;
      const uint32_t kb = smem_u32(st), vb = kb + 2 * DM_ATOM;
      if (nk < 16) {
        // rows past the item may hold anything: zero this warp's V rows there (P is 0
        // for them, but 0 * NaN is not)
        for (int i = max(nk, 0) * 16 + lane; i < 16 * 16; i += 32) {
          const int r = r0 + (i >> 4), c = i & 15;
          *reinterpret_cast<uint4*>(st + 2 * DM_ATOM + (c >> 3) * DM_ATOM + r * 128 + (c & 7) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
      }
      if (PROBE) {
        // |v|^2 of the warp's keys: lane pair (2 r, 2 r + 1) takes key r0 + r, 64 dims each
        const int r = r0 + (lane >> 1);
        const uint8_t* va = st + 2 * DM_ATOM + (lane & 1) * DM_ATOM;
        float vv = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(va + sw_off(r, c));
          float f[8];
          Vec<__nv_bfloat16>::unpack(u, f);
#pragma unroll
          for (int e = 0; e < 8; ++e) vv = fmaf(f[e], f[e], vv);
        }
        vv += __shfl_xor_sync(FULL, vv, 1);
        if ((lane >> 1) < nk) vmax2 = fmaxf(vmax2, vv);
      }
      // S = Q K^T for the warp's 16 keys: two 8-key tiles
      float S[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        S[nt][0] = S[nt][1] = S[nt][2] = S[nt][3] = 0.f;
        const int r = r0 + nt * 8 + (lane & 7);
#pragma unroll
        for (int kc2 = 0; kc2 < 4; ++kc2) {
          const int d0 = kc2 * 32 + (lane >> 3) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + (d0 >> 6) * DM_ATOM + sw_off(r, (d0 & 63) >> 3), b0, b1, b2, b3);
          mma_rows8(S[nt], qa[2 * kc2][0], qa[2 * kc2][1], b0, b1);
          mma_rows8(S[nt], qa[2 * kc2 + 1][0], qa[2 * kc2 + 1][1], b2, b3);
        }
      }
      // online softmax of head gid over keys 8 nt + 2 tig + j
      float x[2][2];
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int key = nt * 8 + 2 * tig + j;   // relative to r0
          float v = S[nt][j] * p.qscale;
          // the hardware log2 (absolute error ~2^-22, below 1e-6 in the logit): every lane
          // sharing a key computes it, and the accurate log2f doubled the instructions a key.
          // (The probe form never has a bias: a probe with R takes the general kernel.)
          if (Rr && key < nk) {
            const float rv = __ldg(Rr + i0 + r0 + key);
            v += p.alpha_c * (PROBE ? log2f(rv) : __log2f(rv));
          }
          v = key < nk ? v : -INFINITY;
          x[nt][j] = v;
          mx = fmaxf(mx, v);
        }
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
      if (mx > m + 8.f) {
        const float corr = ex2(m - mx);        // 0 while nothing was seen
        lsum *= corr;
        lev *= corr;
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          O[t][0] *= corr;
          O[t][1] *= corr;
          if (PROBE) {
            O[t][2] *= corr;
            O[t][3] *= corr;
          }
        }
        m = mx;
      }
      float pr[2][2], pk[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          pr[nt][j] = x[nt][j] == -INFINITY ? 0.f : ex2(x[nt][j] - m);
          if (PROBE) {
            const int key = nt * 8 + 2 * tig + j;
            const int i = i0 + r0 + key;
            const bool kept = key < nk && ((__ldg(Br + (i >> 5)) >> (i & 31)) & 1u);
            pk[nt][j] = kept ? pr[nt][j] : 0.f;
            if (kept) lsum += pr[nt][j];
            else lev += pr[nt][j];
          } else {
            lsum += pr[nt][j];
          }
        }
      // O += P V over the warp's 16 keys, P as bf16 hi + lo
      {
        const uint32_t h0 = pack_bf16(pr[0][0], pr[0][1]);
        const uint32_t h2 = pack_bf16(pr[1][0], pr[1][1]);
        const __nv_bfloat162 hb0 = *reinterpret_cast<const __nv_bfloat162*>(&h0);
        const __nv_bfloat162 hb2 = *reinterpret_cast<const __nv_bfloat162*>(&h2);
        const uint32_t l0 = pack_bf16(pr[0][0] - __low2float(hb0), pr[0][1] - __high2float(hb0));
        const uint32_t l2 = pack_bf16(pr[1][0] - __low2float(hb2), pr[1][1] - __high2float(hb2));
        uint32_t kh0 = 0, kh2 = 0, kl0 = 0, kl2 = 0;
        if (PROBE) {
          kh0 = pack_bf16(pk[0][0], pk[0][1]);
          kh2 = pack_bf16(pk[1][0], pk[1][1]);
          const __nv_bfloat162 kb0 = *reinterpret_cast<const __nv_bfloat162*>(&kh0);
          const __nv_bfloat162 kb2 = *reinterpret_cast<const __nv_bfloat162*>(&kh2);
          kl0 = pack_bf16(pk[0][0] - __low2float(kb0), pk[0][1] - __high2float(kb0));
          kl2 = pack_bf16(pk[1][0] - __low2float(kb2), pk[1][1] - __high2float(kb2));
        }
        const int r = r0 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
        for (int dt2 = 0; dt2 < 8; ++dt2) {
          const int d0 = dt2 * 16 + (lane >> 4) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vb + (d0 >> 6) * DM_ATOM + sw_off(r, (d0 & 63) >> 3), b0, b1, b2, b3);
          if (PROBE) {
            // A rows 0-7: P of the head; rows 8-15: P masked to the kept keys
            mma_rows16(O[2 * dt2], h0, kh0, h2, kh2, b0, b1);
            mma_rows16(O[2 * dt2], l0, kl0, l2, kl2, b0, b1);
            mma_rows16(O[2 * dt2 + 1], h0, kh0, h2, kh2, b2, b3);
            mma_rows16(O[2 * dt2 + 1], l0, kl0, l2, kl2, b2, b3);
          } else {
            mma_rows8(O[2 * dt2], h0, h2, b0, b1);
            mma_rows8(O[2 * dt2], l0, l2, b0, b1);
            mma_rows8(O[2 * dt2 + 1], h0, h2, b2, b3);
            mma_rows8(O[2 * dt2 + 1], l0, l2, b2, b3);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // this warp's record: head gid, o[8 t + 2 tig + j] = O[t][j]
    lsum += __shfl_xor_sync(FULL, lsum, 1);
    lsum += __shfl_xor_sync(FULL, lsum, 2);
    if (PROBE) {
      lev += __shfl_xor_sync(FULL, lev, 1);
      lev += __shfl_xor_sync(FULL, lev, 2);
#pragma unroll
      for (int o = 2; o < 32; o <<= 1) vmax2 = fmaxf(vmax2, __shfl_xor_sync(FULL, vmax2, o));
    }
    constexpr int base = PROBE ? 4 : 2;
    if (gid < G) {
      float* r = dsm + ((size_t)cw * G + gid) * DM_REC;
      if (tig == 0) {
        r[0] = m;
        r[1] = lsum;
        if (PROBE) {
          r[2] = lev;
          r[3] = vmax2;
        }
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        r[base + t * 8 + 2 * tig] = O[t][0];
        r[base + t * 8 + 2 * tig + 1] = O[t][1];
        if (PROBE) {
          r[base + 128 + t * 8 + 2 * tig] = O[t][2];
          r[base + 128 + t * 8 + 2 * tig + 1] = O[t][3];
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(DM_CW * 32) : "memory");
    float* out = p.part + (((int64_t)row * p.nsplit + split) * G) * DM_REC;
    for (int t = threadIdx.x - 32; t < G * DM_REC; t += DM_CW * 32) {
      const int gg = t / DM_REC, c = t % DM_REC;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < DM_CW; ++w) M = fmaxf(M, dsm[((size_t)w * G + gg) * DM_REC]);
      float v = 0.f;
      if (c == 0) {
        v = M;
      } else if (PROBE && c == 3) {
#pragma unroll
        for (int w = 0; w < DM_CW; ++w) v = fmaxf(v, dsm[((size_t)w * G + gg) * DM_REC + 3]);
      } else {
#pragma unroll
        for (int w = 0; w < DM_CW; ++w) {
          const float* r = dsm + ((size_t)w * G + gg) * DM_REC;
          const float sc = (M == -INFINITY) ? 0.f : ex2(r[0] - M);
          v += r[c] * sc;
        }
      }
      out[t] = v;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(DM_CW * 32) : "memory");
  }
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 dm_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 5-D map (dim, token, KV head, layer, batch) with 64 x 32-token boxes, 128B swizzle.
// A dimension of extent 1 gets the stride its inner neighbour implies (any legal value works).
static bool dm_map(CUtensorMap* m, const char* base, int64_t sb, int64_t sl, int64_t sh, int64_t st,
                   const DecodeParams& p) {
  auto enc = dm_encode();
  if (!enc) return false;
  cuuint64_t dims[5] = {128, (cuuint64_t)p.max_len, (cuuint64_t)p.Hkv, (cuuint64_t)p.L, (cuuint64_t)p.B};
  int64_t s[4] = {st, sh, sl, sb};
  for (int i = 1; i < 4; ++i)
    if (dims[i + 1] == 1) s[i] = s[i - 1] * (int64_t)dims[i];
  for (int i = 0; i < 4; ++i)
    if (s[i] <= 0 || s[i] % 16) return false;
  cuuint64_t strides[4] = {(cuuint64_t)s[0], (cuuint64_t)s[1], (cuuint64_t)s[2], (cuuint64_t)s[3]};
  cuuint32_t box[5] = {64, DM_KEYS, 1, 1, 1};
  cuuint32_t el[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<char*>(base), dims, strides, box, el,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool decode_mma_supported(const DecodeParams& p, bool bf16, bool probe) {
  if (!bf16 || !p.qbf16 || p.d != 128 || p.G > 8) return false;
  if (probe && (p.R || !p.bits)) return false;
  if (((uintptr_t)p.K | (uintptr_t)p.V | (uintptr_t)p.q) % 16) return false;
  CUtensorMap mk, mv;
  return dm_map(&mk, p.K, p.Ksb, p.Ksl, p.Ksh, p.Kst, p) && dm_map(&mv, p.V, p.Vsb, p.Vsl, p.Vsh, p.Vst, p);
}

template <bool PROBE>
static cudaError_t launch_decode_mma_t(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                                       cudaStream_t st) {
  DmArgs a{};
  a.p = p;
  a.nitems = p.B * p.L * p.Hkv * p.nsplit;
  // DM_PER_SM CTAs per SM, as many ring stages (at most 6) as the SM's shared memory
  // holds for them after the merge records (the runtime reserves 1 KB per CTA)
  int dev = 0, smem_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  const size_t fixed = 1024 + 16 + (size_t)DM_CW * p.G * dm_rec<PROBE>() * 4;
  const int per_sm = DM_PER_SM;
  const long long room = (long long)smem_sm / per_sm - 1024 - (long long)fixed;
  a.nst = (int)(room / (DM_STAGE + 16));
  if (a.nst > 6) a.nst = 6;
  if (a.nst < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = fixed + (size_t)a.nst * (DM_STAGE + 16);
  auto kern = decode_mma_kernel<PROBE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = per_sm * num_sms();
  if (grid > a.nitems) grid = a.nitems;
  kern<<<grid, DM_THREADS, smem, st>>>(mk, mv, a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_decode_mma(const DecodeParams& p, bool probe, cudaStream_t st) {
  CUtensorMap mk, mv;
  if (!dm_map(&mk, p.K, p.Ksb, p.Ksl, p.Ksh, p.Kst, p) || !dm_map(&mv, p.V, p.Vsb, p.Vsl, p.Vsh, p.Vst, p))
    return cudaErrorInvalidValue;
  return probe ? launch_decode_mma_t<true>(p, mk, mv, st) : launch_decode_mma_t<false>(p, mk, mv, st);
}

}  // namespace kvc
