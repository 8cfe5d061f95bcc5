// Observation-window attention score on the 5th-generation tensor cores.
//
// [InfoKV] Methodology / Technical details: A_i is the window attention of
// key i - the softmax of every window query (the W window queries of each of
// the G query heads sharing the KV head) against all keys, averaged over the
// G*W rows - and S_i = alpha * A_i + (1 - alpha) * Softmax(D * H)_i.
// [SelKV] Pipeline overview step 1: S_i = A_i * ||v_i|| (VATP).
//
// Two passes, each a persistent warp-specialised kernel (one CTA per SM):
//   warp 0     TMA producer: 128-key K tiles (two 64-element 128B-swizzled
//              atoms, 32 KB) into a 4-stage ring; the group's Q rows once per head
//   warp 1     TMEM owner and MMA issuer (one thread): tcgen05.mma kind::f16,
//              bf16 operands from shared memory, fp32 accumulators in TMEM,
//              double-buffered so the epilogue of tile t overlaps MMA t+1
//   warps 2-   epilogue: NB * SPL warpgroups; tiles go round-robin to the NB
//              TMEM accumulator buffers, and SPL warpgroups share a buffer
//              (tcgen05.ld, exp2 on the MUFU pipe); NB = 3 where three
//              accumulators fit in TMEM.  With 256 window rows only two fit, so
//              two warpgroups split each: pass 1 one M tile each, pass 2 half of
//              the row columns each, their partial sums added in a fixed order
// Pass 1 computes S1 = Q K^T (M = 128 window rows, N = 128 keys): every thread
// owns one window row and keeps its running max and sum of exp over the keys.
// Pass 2 computes S2 = K Q^T (M = 128 keys, N = G*W rows): every thread owns
// one key and sums its normalised probabilities over the rows, so A needs no
// cross-thread reduction; the S epilogue is fused.
#include <cudaTypedefs.h>

#include <cstddef>

#include "kernels.cuh"
#include "tc_sm100.cuh"

namespace kvc {
using namespace tc;

constexpr int TC_MAXNB = 3;                    // epilogue warpgroups = TMEM accumulator buffers
constexpr int TC_KT = 128;                        // keys per tile
constexpr int TC_NST = 4;                         // K pipeline stages
constexpr int TC_ATOM_BYTES = TC_KT * 128;        // 128 rows x 64 bf16
constexpr int TC_TILE_BYTES = 2 * TC_ATOM_BYTES;  // head_dim 128 = two atoms
constexpr float TC_LOG2E = 1.4426950408889634f;
constexpr float TC_LN2 = 0.6931471805599453f;

struct TcArgs {
  WinParams p;
  int QR;            // staged Q rows (128 or 256)
  int MT;            // pass-1 M tiles (QR / 128)
  int NC;            // pass-2 accumulator columns per buffer (R rounded up to 32)
  int total, per;    // work items (layer, KV head, key chunk) and items per CTA
  float c2;          // scale * log2(e)
  const float* vnorm;
  uint32_t tmem_cols;
  unsigned* status;
};

struct TcSmem {
  uint64_t full[TC_NST], empty[TC_NST], tfull[TC_MAXNB], tempty[TC_MAXNB], qfull, qempty;
  uint32_t tmem_base;
  int abort;
  int qmin;
  alignas(16) float rowc[256];   // pass 2: row max * log2 e + log2(row sum); read as float4
  int qp[256];       // pass 2: position of every window row
  float2 pm[TC_MAXNB - 1][2][128]; // pass 1: other buffers' (max, sum) per row, merged by buffer 0's warpgroups
  float xa[2][2][128];             // pass 2, split buffers: the second half's sum per key [buffer][parity][key]
};

static_assert(offsetof(TcSmem, rowc) % 16 == 0, "rowc is read with 16-byte loads");
static_assert(offsetof(TcSmem, pm) % 8 == 0, "pm holds float2");

struct Item {
  int lg, l, g, c, key0, key1, ntile;
};

__device__ __forceinline__ Item get_item(const WinParams& p, int it) {
  Item x;
  x.lg = it / p.nchunk;
  x.c = it % p.nchunk;
  x.l = x.lg / p.Hkv;
  x.g = x.lg % p.Hkv;
  x.key0 = x.c * p.chunk;
  x.key1 = min(p.n, x.key0 + p.chunk);
  x.ntile = (x.key1 - x.key0 + TC_KT - 1) / TC_KT;
  return x;
}

template <int NWG>
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NWG * 128) : "memory"); }

// the two warpgroups sharing accumulator buffer b (named barriers 2 and 3)
__device__ __forceinline__ void pair_sync(int b) { asm volatile("bar.sync %0, 256;" ::"r"(2 + b) : "memory"); }

__device__ __forceinline__ float tree_max32(const float* v) {
  float a[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) a[j] = fmaxf(v[j], v[j + 16]);
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int j = 0; j < w; ++j) a[j] = fmaxf(a[j], a[j + w]);
  return a[0];
}

template <int PASS, int MT, int NB, int SPL>
__global__ void __launch_bounds__(64 + NB * SPL * 128, 1)
win_tc_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapQ,
              const TcArgs a) {
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Qs = base;
  uint8_t* Ks = base + a.QR * 256;
  TcSmem* sm = reinterpret_cast<TcSmem*>(Ks + TC_NST * TC_TILE_BYTES);
  const WinParams& p = a.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sm->abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_NST; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&sm->tfull[b], 1);
      mbar_init(&sm->tempty[b], 4 * SPL);   // every warp of the warpgroups sharing buffer b
    }
    mbar_init(&sm->qfull, 1);
    mbar_init(&sm->qempty, 1);
    sm->abort = 0;
    sm->qmin = query_pos_min(p);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&sm->tmem_base, a.tmem_cols);
  if (warp == 0 && lane == 0) {
    prefetch_map(&mapK);
    prefetch_map(&mapQ);
  }
  __syncthreads();
  fence_after();
  const uint32_t tmem = sm->tmem_base;
  const int item0 = blockIdx.x * a.per;
  const int item1 = min(a.total, item0 + a.per);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t tile = 0, qcount = 0;
      int prev = -1;
      for (int it = item0; it < item1; ++it) {
        const Item x = get_item(p, it);
        if (x.lg != prev) {
          if (qcount > 0 && !mbar_wait(&sm->qempty, (qcount - 1) & 1, abort, a.status)) goto producer_done;
          mbar_expect_tx(&sm->qfull, a.QR * 256);
          const int row0 = (x.l * p.Hq + x.g * p.G) * p.W;
          tma_load_2d(Qs, &mapQ, 0, row0, &sm->qfull);
          tma_load_2d(Qs + a.QR * 128, &mapQ, 64, row0, &sm->qfull);
          ++qcount;
          prev = x.lg;
        }
        for (int t = 0; t < x.ntile; ++t, ++tile) {
          const int s = tile % TC_NST;
          const uint32_t ph = (tile / TC_NST) & 1;
          if (!mbar_wait(&sm->empty[s], ph ^ 1, abort, a.status)) goto producer_done;
          mbar_expect_tx(&sm->full[s], TC_TILE_BYTES);
          uint8_t* dst = Ks + s * TC_TILE_BYTES;
          const int key = x.key0 + t * TC_KT;
          tma_load_4d(dst, &mapK, 0, key, x.g, x.l, &sm->full[s]);
          tma_load_4d(dst + TC_ATOM_BYTES, &mapK, 64, key, x.g, x.l, &sm->full[s]);
        }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = PASS == 1 ? idesc_bf16(128, 128) : idesc_bf16(128, p.R);
      // stage s lies s * TC_TILE_BYTES past the first: that many 16-byte descriptor units
      const uint64_t kd0 = sw128_desc(Ks), qd0 = sw128_desc(Qs);
      const uint32_t qatom = (uint32_t)(a.QR * 128 / 16);
      uint32_t tile = 0, qcount = 0;
      int prev = -1;
      for (int it = item0; it < item1; ++it) {
        const Item x = get_item(p, it);
        if (x.lg != prev) {
          if (!mbar_wait(&sm->qfull, qcount & 1, abort, a.status)) goto mma_done;
          ++qcount;
          prev = x.lg;
        }
        for (int t = 0; t < x.ntile; ++t, ++tile) {
          const int s = tile % TC_NST;
          const uint32_t ph = (tile / TC_NST) & 1;
          const int b = tile % NB;
          const uint32_t tph = (tile / NB) & 1;
          if (!mbar_wait(&sm->full[s], ph, abort, a.status)) goto mma_done;
          if (!mbar_wait(&sm->tempty[b], tph ^ 1, abort, a.status)) goto mma_done;
          fence_after();
          const uint64_t kd = kd0 + (uint64_t)s * (TC_TILE_BYTES / 16);
          if (PASS == 1) {
            for (int mt = 0; mt < MT; ++mt) {
              // M tile mt: window rows 128 mt.., 128 x 128 B into each Q atom
              const uint32_t d = tmem + (uint32_t)((b * MT + mt) * 128);
              mma_bf16_k128(d, qd0 + (uint64_t)mt * 1024, kd, qatom, TC_ATOM_BYTES / 16, idesc);
            }
          } else {
            const uint32_t d = tmem + (uint32_t)(b * a.NC);
            mma_bf16_k128(d, kd, qd0, TC_ATOM_BYTES / 16, qatom, idesc);
          }
          mma_commit(&sm->empty[s]);
          mma_commit(&sm->tfull[b]);
        }
        const bool head_ends = (it + 1 >= item1) || get_item(p, it + 1).lg != x.lg;
        if (head_ends) mma_commit(&sm->qempty);
      }
    mma_done:;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    static_assert(SPL == 1 || (SPL == 2 && NB == 2), "a split buffer pairs two warpgroups");
    static_assert(PASS == 2 || SPL == 1 || MT == 2, "pass 1 splits by M tile");
    constexpr int NWG = NB * SPL;
    const int wg = (warp - 2) >> 2;          // warpgroup
    const int bw = wg / SPL;                 // its accumulator buffer: the tiles with tile % NB == bw
    const int h = wg % SPL;                  // its half of a shared buffer
    const int q4 = warp & 3;                 // TMEM lane quarter this warp may access
    const int rowl = q4 * 32 + lane;         // accumulator row (TMEM lane) of this thread
    const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
    const int qmin = sm->qmin;
    const int et = threadIdx.x - 64;         // 0 .. NWG*128-1 over the epilogue warpgroups
    uint32_t tile = 0;
    int prev = -1;
    for (int it = item0; it < item1; ++it) {
      const Item x = get_item(p, it);
      if (PASS == 2 && x.lg != prev) {
        epi_sync<NWG>();
        for (int r = et; r < p.R; r += NWG * 128) {
          const float M = p.rowst[((int64_t)x.lg * p.R + r) * 2];
          const float inv = p.rowst[((int64_t)x.lg * p.R + r) * 2 + 1];
          // p_ri = 2^(s c2 - (M log2e + log2 L)); a row with no visible key contributes 0
          // stored negated, -(M log2e + log2 L), the addend of the exponent's FMA
          sm->rowc[r] = (M == -INFINITY || !(inv > 0.f)) ? -INFINITY : log2f(inv) - M * TC_LOG2E;
          sm->qp[r] = query_pos(p, x.l, r % p.W);
        }
        epi_sync<NWG>();
        prev = x.lg;
      }
      // row statistics of this thread's rows: M tile i, or the warpgroup's own M tile h when split
      constexpr int NM = SPL == 2 ? 1 : MT;
      float m2[NM], s1[NM];
      int qrow[NM];
#pragma unroll
      for (int i = 0; i < NM; ++i) {
        m2[i] = -INFINITY;
        s1[i] = 0.f;
        const int r = (SPL == 2 ? h : i) * 128 + rowl;
        qrow[i] = (PASS == 1 && r < p.R) ? query_pos(p, x.l, r % p.W) : -0x7fffffff;
      }
      for (int t = 0; t < x.ntile; ++t, ++tile) {
        if ((int)(tile % NB) != bw) continue;
        const int b = bw;
        const uint32_t tph = (tile / NB) & 1;
        // after an abort the tile is skipped but every named barrier is still reached
        bool ok = !*abort && mbar_wait(&sm->tfull[b], tph, abort, a.status);
        ok = __all_sync(FULL, ok);
        if (!ok) {
          if (PASS == 2 && SPL == 2) pair_sync(b);
          continue;
        }
        fence_after();
        const int key0 = x.key0 + t * TC_KT;
        const bool need_mask = key0 + TC_KT > x.key1 || key_pos(p, x.l, x.g, key0 + TC_KT - 1) > qmin;
        if (PASS == 1) {
#pragma unroll
          for (int i = 0; i < NM; ++i) {
            const int mt = SPL == 2 ? h : i;
            if (mt * 128 + q4 * 32 >= p.R) continue;   // the warp's rows are all padding
#pragma unroll 1
            for (int c = 0; c < 4; c += 2) {
              float v[64];
              __syncwarp();
              tmem_ld32(lane_addr + (uint32_t)((b * MT + mt) * 128 + c * 32), v);
              tmem_ld32(lane_addr + (uint32_t)((b * MT + mt) * 128 + c * 32 + 32), v + 32);
              tmem_wait_ld();
              if (need_mask) {
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                  const int key = key0 + c * 32 + j;
                  if (key >= x.key1 || key_pos(p, x.l, x.g, key) > qrow[i]) v[j] = -INFINITY;
                }
              }
              const float mx = fmaxf(tree_max32(v), tree_max32(v + 32));
              const float mn = fmaxf(m2[i], mx * a.c2);
              if (mn > -INFINITY) {
                // column pairs through packed FMAs and adds (each lane rounds as the scalar
                // instruction): s01 sums columns = 0, 1 (mod 4), s23 columns 2, 3
                uint64_t s01 = pk2(0.f, 0.f), s23 = pk2(0.f, 0.f);
                const uint64_t c2x2 = pk2(a.c2, a.c2), nmn = pk2(-mn, -mn);
#pragma unroll
                for (int j = 0; j < 64; j += 4) {
                  const float2 x01 = upk2(fma2(pk2(v[j], v[j + 1]), c2x2, nmn));
                  const float2 x23 = upk2(fma2(pk2(v[j + 2], v[j + 3]), c2x2, nmn));
                  s01 = add2(s01, pk2(ex2(x01.x), ex2(x01.y)));
                  s23 = add2(s23, pk2(ex2(x23.x), ex2(x23.y)));
                }
                const float2 a01 = upk2(s01), a23 = upk2(s23);
                s1[i] = s1[i] * ex2(m2[i] - mn) + ((a01.x + a01.y) + (a23.x + a23.y));
                m2[i] = mn;
              }
            }
          }
        } else {
          const int key = key0 + rowl;
          const bool kvalid = key < x.key1;
          const int kp = kvalid ? key_pos(p, x.l, x.g, key) : 0x7fffffff;
          // inputs of the score epilogue, loaded before the accumulator so their latency
          // overlaps the exponentials
          float pre = 0.f, st0 = 0.f, st1 = 1.f;
          if (kvalid && (SPL == 1 || h == 0)) {
            if (p.mode == KVC_SCORE_INFOKV) {
              pre = __ldg(p.D + x.l * p.Dsl + x.g * p.Dsh + key) * __ldg(p.H + x.l * p.Hsl + x.g * p.Hsh + key);
              st0 = __ldg(p.estats + 3 * x.lg);
              st1 = __ldg(p.estats + 3 * x.lg + 1);
            } else if (p.mode == KVC_SCORE_VATP) {
              pre = __ldg(a.vnorm + (int64_t)x.lg * p.n + key);
            }
          }
          uint64_t acc01 = pk2(0.f, 0.f), acc23 = pk2(0.f, 0.f);
          const uint64_t c2x2 = pk2(a.c2, a.c2);
          const int nc16 = p.R >> 4;
          // a split buffer: the first warpgroup takes the first ceil(nc16 / 2) 16-column chunks
          const int c0 = SPL == 2 && h == 1 ? (nc16 + 1) >> 1 : 0;
          const int c1 = SPL == 2 && h == 0 ? (nc16 + 1) >> 1 : nc16;
          const float4* rc4 = reinterpret_cast<const float4*>(sm->rowc);
#pragma unroll 1
          for (int c = c0; c < c1; ++c) {
            // the chunk's row constants first: the wait below orders memory, so shared loads
            // issued after it would add their latency to every chunk
            float4 r4c[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) r4c[q] = rc4[c * 4 + q];
            float v[16];
            __syncwarp();
            tmem_ld16(lane_addr + (uint32_t)(b * a.NC + c * 16), v);
            tmem_wait_ld();
            // column pairs through packed FMAs and adds: acc01 sums columns = 0, 1 (mod 4),
            // acc23 columns 2, 3; the row constants are stored negated
            if (!need_mask) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float4 r4 = r4c[q];
                const float2 x01 = upk2(fma2(pk2(v[q * 4 + 0], v[q * 4 + 1]), c2x2, pk2(r4.x, r4.y)));
                const float2 x23 = upk2(fma2(pk2(v[q * 4 + 2], v[q * 4 + 3]), c2x2, pk2(r4.z, r4.w)));
                acc01 = add2(acc01, pk2(ex2(x01.x), ex2(x01.y)));
                acc23 = add2(acc23, pk2(ex2(x23.x), ex2(x23.y)));
              }
            } else {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float e[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const int r = c * 16 + q * 4 + u;
                  const float x = ex2(fmaf(v[q * 4 + u], a.c2, sm->rowc[r]));
                  e[u] = kp > sm->qp[r] ? 0.f : x;
                }
                acc01 = add2(acc01, pk2(e[0], e[1]));
                acc23 = add2(acc23, pk2(e[2], e[3]));
              }
            }
          }
          const float2 a01 = upk2(acc01), a23 = upk2(acc23);
          float asum = (a01.x + a01.y) + (a23.x + a23.y);
          if (SPL == 2) {
            // the accumulator is read out: free it before the exchange
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->tempty[b]);
            float* xa = sm->xa[b][tph];
            if (h == 1) xa[rowl] = asum;
            pair_sync(b);
            if (h == 1) continue;
            asum += xa[rowl];
          }
          if (kvalid) {
            const float A = asum / (float)p.R;
            const int64_t o = (int64_t)x.lg * p.n + key;
            float S = A;
            if (p.mode == KVC_SCORE_INFOKV) {
              S = p.alpha * A + (1.f - p.alpha) * (expf(pre - st0) / st1);
            } else if (p.mode == KVC_SCORE_VATP) {
              S = A * pre;
            }
            if (p.A) p.A[o] = A;
            p.S[o] = S;
          }
        }
        if (PASS == 2 && SPL == 2) continue;   // released before the exchange
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->tempty[b]);
      }
      if (PASS == 1) {
        // merge the buffers' partial row statistics of this item (per M tile when split)
        if (bw > 0) {
#pragma unroll
          for (int i = 0; i < NM; ++i) sm->pm[bw - 1][SPL == 2 ? h : i][rowl] = make_float2(m2[i], s1[i]);
        }
        epi_sync<NWG>();
        if (bw == 0) {
#pragma unroll
          for (int i = 0; i < NM; ++i) {
            const int mt = SPL == 2 ? h : i;
            const int r = mt * 128 + rowl;
            float mn = m2[i];
#pragma unroll
            for (int o = 0; o < NB - 1; ++o) mn = fmaxf(mn, sm->pm[o][mt][rowl].x);
            float sum = 0.f;
            if (mn > -INFINITY) {
              sum = s1[i] * ex2(m2[i] - mn);
#pragma unroll
              for (int o = 0; o < NB - 1; ++o) {
                const float2 o2 = sm->pm[o][mt][rowl];
                sum += o2.y * ex2(o2.x - mn);
              }
            }
            if (r < p.R) {
              float* op = p.part + (((int64_t)x.lg * p.nchunk + x.c) * p.R + r) * 2;
              op[0] = mn == -INFINITY ? -INFINITY : mn * TC_LN2;
              op[1] = sum;
            }
          }
        }
        epi_sync<NWG>();
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem, a.tmem_cols);
  }
}

// ||v_i|| for the VATP score (bf16, head_dim 128): a half-warp per row, each lane one
// 16-byte vector, four rows per half-warp in flight.
__global__ void __launch_bounds__(256) vnorm_kernel(const __nv_bfloat16* __restrict__ V, int64_t Vsl, int64_t Vsh,
                                                    int64_t Vst, int L, int Hkv, int n, float* __restrict__ out) {
  constexpr int U = 4;
  const int64_t rows = (int64_t)L * Hkv * n;
  const int part = threadIdx.x & 15;
  const int64_t hw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;    // half-warp index
  const int64_t nhw = ((int64_t)gridDim.x * blockDim.x) >> 4;
  // the warp's two halves take rows 2 w and 2 w + 1 of a block of rows; trip count is warp-uniform
  for (int64_t r0 = (hw & ~int64_t(1)) * U; r0 < rows; r0 += nhw * U) {
    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t r = r0 + 2 * u + (hw & 1);
      if (r < rows) {
        const int i = (int)(r % n);
        const int64_t lg = r / n;
        const int l = (int)(lg / Hkv), g = (int)(lg % Hkv);
        raw[u] = ldg16(V + l * Vsl + g * Vsh + (int64_t)i * Vst + part * 8);
      } else {
        raw[u] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float f[8];
      Vec<__nv_bfloat16>::unpack(raw[u], f);
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(f[e], f[e], s);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
      const int64_t r = r0 + 2 * u + (hw & 1);
      if (part == 0 && r < rows) out[r] = sqrtf(s);
    }
  }
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool make_window_maps(const WinParams& p, int QR, CUtensorMap* mK, CUtensorMap* mQ) {
  auto enc = encode_fn();
  if (!enc) return false;
  const uint64_t es = 2;
  int64_t sl = p.Ksl, sh = p.Ksh, st = p.Kst;
  if (p.Hkv == 1) sh = st * p.n;          // unused coordinate: any legal stride
  if (p.L == 1) sl = sh * p.Hkv;
  cuuint64_t dK[4] = {128, (cuuint64_t)p.n, (cuuint64_t)p.Hkv, (cuuint64_t)p.L};
  cuuint64_t sK[3] = {(cuuint64_t)(st * es), (cuuint64_t)(sh * es), (cuuint64_t)(sl * es)};
  cuuint32_t bK[4] = {64, TC_KT, 1, 1};
  cuuint32_t e4[4] = {1, 1, 1, 1};
  CUresult r = enc(mK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.K), dK, sK, bK, e4,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  cuuint64_t dQ[2] = {128, (cuuint64_t)p.L * p.Hq * p.W};
  cuuint64_t sQ[1] = {128 * es};
  cuuint32_t bQ[2] = {64, (cuuint32_t)QR};
  r = enc(mQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p.Qw), dQ, sQ, bQ, e4,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_vnorm(const WinParams& p, cudaStream_t st) {
  vnorm_kernel<<<num_sms() * 16, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(p.V), p.Vsl, p.Vsh, p.Vst,
                                               p.L, p.Hkv, p.n, p.vnorm);
  count_launch();
  return cudaGetLastError();
}

static int tc_qr(int R) { return R <= 128 ? 128 : 256; }

bool window_tc_supported(const WinParams& p, kvc_dtype dt) {
  if (dt != KVC_BF16 || p.d != 128) return false;
  if (p.R % 16 != 0 || p.R > 256 || p.R < 16) return false;
  if (p.chunk % TC_KT != 0) return false;
  if ((uintptr_t)p.Qw % 16 || (uintptr_t)p.K % 16) return false;
  if (p.mode == KVC_SCORE_VATP && ((uintptr_t)p.V % 16 || (p.Vst * 2) % 16)) return false;
  CUtensorMap a, b;
  return make_window_maps(p, tc_qr(p.R), &a, &b);
}

static size_t tc_smem(int QR) { return (size_t)QR * 256 + (size_t)TC_NST * TC_TILE_BYTES + sizeof(TcSmem) + 1024; }

cudaError_t launch_window_tc(const WinParams& p, cudaStream_t st) {
  CUtensorMap mK, mQ;
  const int QR = tc_qr(p.R);
  if (!make_window_maps(p, QR, &mK, &mQ)) return cudaErrorInvalidValue;
  TcArgs a{};
  a.p = p;
  a.QR = QR;
  a.MT = QR / 128;
  a.NC = (p.R + 31) / 32 * 32;
  a.total = p.L * p.Hkv * p.nchunk;
  const int grid = a.total < num_sms() ? a.total : num_sms();
  a.per = (a.total + grid - 1) / grid;
  a.c2 = p.scale * TC_LOG2E;
  a.status = status_ptr();
  a.vnorm = p.vnorm;
  const size_t smem = tc_smem(QR);
  if (p.mode == KVC_SCORE_VATP) {
    const cudaError_t ev = launch_vnorm(p, st);
    if (ev != cudaSuccess) return ev;
  }
  // pass 1: row statistics (not when the decode steps recorded them)
  cudaError_t e;
  if (p.wlse) {
  } else if (a.MT == 1) {
    a.tmem_cols = 512;                       // three 128-column accumulators
    auto k1 = win_tc_kernel<1, 1, 3, 1>;
    cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k1<<<grid, 64 + 3 * 128, smem, st>>>(mK, mQ, a);
    count_launch();
  } else {
    a.tmem_cols = 512;                       // two 256-column accumulators, a warpgroup per M tile
    auto k1 = win_tc_kernel<1, 2, 2, 2>;
    cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k1<<<grid, 64 + 4 * 128, smem, st>>>(mK, mQ, a);
    count_launch();
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_window_combine(p, st);
  if (e != cudaSuccess) return e;
  // pass 2: probabilities summed per key, fused score epilogue
  a.tmem_cols = 512;
  if (3 * a.NC <= 512) {
    auto k2 = win_tc_kernel<2, 1, 3, 1>;
    cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k2<<<grid, 64 + 3 * 128, smem, st>>>(mK, mQ, a);
    count_launch();
  } else {
    auto k2 = win_tc_kernel<2, 1, 2, 2>;     // two warpgroups split each buffer's columns
    cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k2<<<grid, 64 + 4 * 128, smem, st>>>(mK, mQ, a);
    count_launch();
  }
  return cudaGetLastError();
}

}  // namespace kvc
