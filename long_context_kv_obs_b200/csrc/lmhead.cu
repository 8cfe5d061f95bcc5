// Top-k restricted entropy H_i from the LM head's input, the logits never written.
//
// [InfoKV] Methodology: H_i is the entropy of the final layer's predictive distribution
// restricted to its k largest entries.  The distribution of position i is softmax(W x_i),
// W the [V][Dh] output projection and x_i the LM head's input.  Only the k largest
// logits of a row matter, so they are picked out while the logits leave the tensor-core
// accumulator, and the [n][V] logits matrix never exists in HBM.
//
// lmh_topk_kernel: persistent, one CTA per SM.  Work item (m, s) is the 256 rows of row
// tile m against vocabulary segment s, a run of 256-column N tiles.
//   warp 0      TMA producer: 64-wide K slices of x (256 x 64) and W (256 x 64), 128B
//               swizzled, into a 3-stage ring
//   warp 1      TMEM owner and tcgen05.mma issuer: per N tile, two 128 x 256 products
//               (the two row halves against the same W slice) accumulated over Dh in
//               the two halves of TMEM
//   warps 2-9   two epilogue warpgroups; warpgroup b drains the accumulator of row half
//               b, one row per thread
// Each W slice staged in shared memory feeds both row halves, so a CTA moves 64 KB per
// 8.4 MFLOP of MMA work; with every 512 TMEM columns in use, the accumulators are not
// double-buffered and the epilogue of one N tile runs before the next tile's MMAs.
//
// Per row, the epilogue keeps a candidate list in global scratch and a threshold T: a
// logit above T is appended.  A full list is trimmed: four rounds of quaternary search
// between the list's least and greatest value find a value lo with at least k entries
// >= lo; the entries >= lo stay and T becomes lo.  A logit at or below T cannot change
// the multiset of the k largest (k list entries are >= T), so dropping it is exact.
// When a trim would free too little (many equal values), the exact cut runs instead:
// the k largest by bisection on order-preserving keys, copies of the k-th value filling
// a tie.  At the end of the item each row's list is cut to k and stored: the k largest
// logits of the segment.  One list per row and segment.
//
// lmh_entropy_kernel: a warp per row takes the k largest of the row's lists and their
// entropy, in the same arithmetic as the logits-row entropy kernel.
//
// The segment count bounds the x tiles live in L2 at once: with S segments about SMs / S
// row tiles run together, each re-reading its 256 x Dh slice of x for every N tile,
// while the CTAs sweeping one segment read the same W tiles at about the same time.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "tc_sm100.cuh"

namespace kvc {
using namespace tc;

constexpr int LM_BM = 256;                      // rows per CTA tile: two 128-row halves
constexpr int LM_BN = 256;                      // vocabulary columns per N tile
constexpr int LM_BK = 64;                       // Dh per stage: one 128-byte swizzle atom
constexpr int LM_NST = 3;                       // ring stages
constexpr int LM_ABYTES = LM_BM * LM_BK * 2;
constexpr int LM_BBYTES = LM_BN * LM_BK * 2;
constexpr int LM_STAGE = LM_ABYTES + LM_BBYTES;
constexpr int LM_EPI0 = 2;                      // first epilogue warp
constexpr int LM_THREADS = (LM_EPI0 + 8) * 32;
constexpr int LM_CAP = 512;                     // candidate list capacity per row
constexpr int LM_NI = LM_CAP / 32;
constexpr int LE_WARPS = 8;                     // rows per entropy block
constexpr int LE_NK = 64;                       // keys per lane: lists x k <= 2048

struct LmArgs {
  int n, V, k;
  int S, tps, ntn, nk;
  int64_t total;           // work items: M tiles x segments
  float* scratch;          // [grid][2][128][LM_CAP]
  float* lists;            // [n][S][k]
  int32_t* counts;         // [n][S]
  unsigned* status;
};

struct LmSmem {
  uint64_t full[LM_NST], empty[LM_NST], tfull[1], tempty[1], mdrain;
  uint32_t tmem_base;
  int abort;
};

// Bounded wait that ignores the abort flag: lets the copies and MMAs a CTA already
// issued land before it frees its memory.
__device__ __forceinline__ void lm_drain_wait(uint64_t* bar, uint32_t parity, unsigned* status) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = gtimer();
  while (!mbar_try_wait(bar, parity)) {
    if (gtimer() - t0 > WAIT_NS) {
      flag(status, ST_TIMEOUT);
      return;
    }
  }
}

// D[tmem] (+)= A B^T over one 64-wide K slice: four K = 16 steps, 32 bytes apart inside
// the swizzle atom (2 in the descriptor's 16-byte address units).  `acc` = 0 makes the
// first step overwrite D.
__device__ __forceinline__ void mma_bf16_k64(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                             uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p0, p1;\n setp.ne.b32 p0, %9, 0;\n setp.eq.b32 p1, %8, %8;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %8, p0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %8, p1;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %8, p1;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %10, %8, p1;\n}\n" ::"r"(d_tmem),
      "l"(a0), "l"(a0 + 2), "l"(a0 + 4), "l"(a0 + 6), "l"(b0), "l"(b0 + 2), "l"(b0 + 4), "r"(idesc),
      "r"(acc), "l"(b0 + 6)
      : "memory");
}

// The k largest of the c values src[0, c) (k < c <= LM_CAP), written in index order to
// dst[0, k): the values above the k-th largest, then copies of it.  Returns the k-th
// largest.  Warp-wide; src and dst may be the same list.  The k-th largest key t is found
// bit by bit from the top: the largest t with at least k keys >= t.
__device__ float lm_cut(const float* src, int c, int k, float* dst, int lane) {
  __syncwarp();                                     // the list's appends by its lane are visible
  uint32_t key[LM_NI];
#pragma unroll
  for (int i = 0; i < LM_NI; ++i) {
    const int idx = lane + 32 * i;
    key[i] = idx < c ? f2key(src[idx]) : 0u;      // key 0 is below every float's key
  }
  uint32_t t = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = t | (1u << bit);
    int m = 0;
#pragma unroll
    for (int i = 0; i < LM_NI; ++i) m += key[i] >= cand;
    if (__reduce_add_sync(FULL, m) >= k) t = cand;
  }
  __syncwarp();                                     // every lane has read src
  const unsigned below = (1u << lane) - 1u;
  int w = 0;
#pragma unroll
  for (int i = 0; i < LM_NI; ++i) {
    const bool keep = key[i] > t;
    const unsigned bal = __ballot_sync(FULL, keep);
    if (keep) dst[w + __popc(bal & below)] = key2f(key[i]);
    w += __popc(bal);
  }
  const float tv = key2f(t);
  for (int i = w + lane; i < k; i += 32) dst[i] = tv;
  __syncwarp();
  return tv;
}

// Frees room in a row's list of c entries: finds, by four rounds of quaternary search
// between the list's least and greatest value, a value lo with at least k entries >= lo,
// and keeps those entries in place.  Dropping values below lo is exact (k values >= lo
// remain), and lo becomes the row's threshold.  When that keeps more than half the
// room past k (many equal values), the exact cut runs instead.  Warp-wide.
__device__ float lm_trim(float* l, int c, int k, int lane, int& newc) {
  __syncwarp();
  float val[LM_NI];
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll
  for (int i = 0; i < LM_NI; ++i) {
    const int idx = lane + 32 * i;
    val[i] = idx < c ? l[idx] : -INFINITY;
    if (idx < c) {
      mx = fmaxf(mx, val[i]);
      mn = fminf(mn, val[i]);
    }
  }
  mx = warp_max(mx);
  mn = -warp_max(-mn);
  float lo = mn, hi = mx;                          // at least k entries >= lo
#pragma unroll 1
  for (int r = 0; r < 4; ++r) {
    const float w = (hi - lo) * 0.25f;
    const float t1 = lo + w, t2 = lo + 2.f * w, t3 = lo + 3.f * w;
    int m1 = 0, m2 = 0, m3 = 0;
#pragma unroll
    for (int i = 0; i < LM_NI; ++i) {
      m1 += val[i] >= t1;
      m2 += val[i] >= t2;
      m3 += val[i] >= t3;
    }
    m1 = __reduce_add_sync(FULL, m1);
    m2 = __reduce_add_sync(FULL, m2);
    m3 = __reduce_add_sync(FULL, m3);
    if (m3 >= k) {
      lo = t3;
    } else if (m2 >= k) {
      lo = t2;
      hi = t3;
    } else if (m1 >= k) {
      lo = t1;
      hi = t2;
    } else {
      hi = t1;
    }
  }
  int kept = 0;
#pragma unroll
  for (int i = 0; i < LM_NI; ++i) kept += val[i] >= lo;
  kept = __reduce_add_sync(FULL, kept);
  if (kept > (LM_CAP + k) / 2) {
    newc = k;
    return lm_cut(l, c, k, l, lane);
  }
  const unsigned below = (1u << lane) - 1u;
  int w = 0;
#pragma unroll
  for (int i = 0; i < LM_NI; ++i) {
    const bool keep = val[i] >= lo;
    const unsigned bal = __ballot_sync(FULL, keep);
    if (keep) l[w + __popc(bal & below)] = val[i];
    w += __popc(bal);
  }
  __syncwarp();
  newc = w;
  return lo;
}

__global__ void __launch_bounds__(LM_THREADS, 1)
lmh_topk_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW,
                const LmArgs a) {
  extern __shared__ uint8_t lm_smem_raw[];
  uint8_t* stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(lm_smem_raw) + 1023) & ~uintptr_t(1023));
  LmSmem* sm = reinterpret_cast<LmSmem*>(stages + LM_NST * LM_STAGE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sm->abort;
  const int64_t stride = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < LM_NST; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    mbar_init(&sm->tfull[0], 1);
    mbar_init(&sm->tempty[0], 8);                 // every epilogue warp
    mbar_init(&sm->mdrain, 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&sm->tmem_base, 512);
  if (warp == 0 && lane == 0) {
    prefetch_map(&mapX);
    prefetch_map(&mapW);
  }
  __syncthreads();
  fence_after();
  const uint32_t tmem = sm->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kt = 0;
      for (int64_t o = blockIdx.x; o < a.total; o += stride) {
        const int m = (int)(o / a.S), s = (int)(o % a.S);
        const int t1 = min(a.ntn, (s + 1) * a.tps);
        for (int t = s * a.tps; t < t1; ++t) {
          for (int kb = 0; kb < a.nk; ++kb, ++kt) {
            const int st = kt % LM_NST;
            if (!mbar_wait(&sm->empty[st], ((kt / LM_NST) & 1) ^ 1, abort, a.status)) goto producer_done;
            mbar_expect_tx(&sm->full[st], LM_STAGE);
            uint8_t* dst = stages + st * LM_STAGE;
            tma_load_2d(dst, &mapX, kb * LM_BK, m * LM_BM, &sm->full[st]);
            tma_load_2d(dst + LM_ABYTES, &mapW, kb * LM_BK, t * LM_BN, &sm->full[st]);
          }
        }
      }
    producer_done:
      // the copies of the last LM_NST stages land before the CTA moves on
      for (uint32_t j = kt > LM_NST ? kt - LM_NST : 0; j < kt; ++j)
        lm_drain_wait(&sm->full[j % LM_NST], (j / LM_NST) & 1, a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, LM_BN);
      const uint64_t d0 = sw128_desc(stages);
      uint32_t kt = 0, gt = 0;
      for (int64_t o = blockIdx.x; o < a.total; o += stride) {
        const int s = (int)(o % a.S);
        const int t1 = min(a.ntn, (s + 1) * a.tps);
        for (int t = s * a.tps; t < t1; ++t, ++gt) {
          if (!mbar_wait(&sm->tempty[0], (gt & 1) ^ 1, abort, a.status)) goto mma_done;
          fence_after();
          for (int kb = 0; kb < a.nk; ++kb, ++kt) {
            const int st = kt % LM_NST;
            if (!mbar_wait(&sm->full[st], (kt / LM_NST) & 1, abort, a.status)) goto mma_done;
            fence_after();
            const uint64_t ad = d0 + (uint64_t)(st * (LM_STAGE / 16));
            const uint64_t bd = ad + (uint64_t)(LM_ABYTES / 16);
            mma_bf16_k64(tmem, ad, bd, idesc, kb > 0);
            mma_bf16_k64(tmem + (uint32_t)LM_BN, ad + (uint64_t)(LM_ABYTES / 32), bd, idesc, kb > 0);
            mma_commit(&sm->empty[st]);
          }
          mma_commit(&sm->tfull[0]);
        }
      }
    mma_done:
      // every MMA issued so far completes before TMEM is freed
      mma_commit(&sm->mdrain);
      lm_drain_wait(&sm->mdrain, 0, a.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int wg = (warp - LM_EPI0) >> 2;          // accumulator = row half
    const int q = warp & 3;                        // TMEM lane quarter this warp may read
    const int rl = wg * 128 + q * 32 + lane;       // row within the CTA tile
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(wg * LM_BN);
    float* const qlists = a.scratch + (((int64_t)blockIdx.x * 2 + wg) * 128 + q * 32) * LM_CAP;
    float* const mine = qlists + (int64_t)lane * LM_CAP;
    float T = -INFINITY;
    int cnt = 0;
    uint32_t gt = 0, got = 0;
    for (int64_t o = blockIdx.x; o < a.total; o += stride) {
      const int m = (int)(o / a.S), s = (int)(o % a.S);
      const int t1 = min(a.ntn, (s + 1) * a.tps);
      const bool rvalid = m * LM_BM + rl < a.n;
      for (int t = s * a.tps; t < t1; ++t, ++gt) {
        const bool ok = mbar_wait(&sm->tfull[0], got & 1, abort, a.status);
        ++got;
        if (!__all_sync(FULL, ok)) goto epilogue_done;
        fence_after();
        const int col0 = t * LM_BN;
#pragma unroll 1
        for (int c = 0; c < LM_BN / 32; ++c) {
          float v[32];
          __syncwarp();
          tmem_ld32(lane_addr + (uint32_t)(c * 32), v);
          tmem_wait_ld();
          // room for 32 more in every list of the warp: full lists are cut to k first
          for (unsigned need = __ballot_sync(FULL, cnt + 32 > LM_CAP); need; need &= need - 1) {
            const int src = __ffs(need) - 1;
            float* l = qlists + (int64_t)src * LM_CAP;
            int nc;
            const float tv = lm_trim(l, __shfl_sync(FULL, cnt, src), a.k, lane, nc);
            if (lane == src) {
              T = tv;
              cnt = nc;
            }
          }
          if (rvalid) {
            const int cb = col0 + c * 32;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (cb + j < a.V && v[j] > T) mine[cnt++] = v[j];
          }
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->tempty[0]);
      }
      // end of the item: each row's list, cut to k, is list s of the row
      __syncwarp();
      for (int src = 0; src < 32; ++src) {
        const int row = m * LM_BM + wg * 128 + q * 32 + src;
        if (row >= a.n) break;
        const int cs = __shfl_sync(FULL, cnt, src);
        const float* l = qlists + (int64_t)src * LM_CAP;
        const int64_t li = (int64_t)row * a.S + s;
        float* dst = a.lists + li * a.k;
        if (cs > a.k) {
          lm_cut(l, cs, a.k, dst, lane);
        } else {
          for (int i = lane; i < cs; i += 32) dst[i] = l[i];
        }
        if (lane == 0) a.counts[li] = cs < a.k ? cs : a.k;
      }
      __syncwarp();
      T = -INFINITY;
      cnt = 0;
    }
  epilogue_done:;
  }
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// H of one row per warp from its nl lists of at most k values each (nl * k <= 32 LE_NK):
// the kk = min(k, values) largest, found by bisection on their keys, then
// H = log(sum e) - sum(e (z - max)) / sum e with e = exp(z - max).
__global__ void __launch_bounds__(LE_WARPS * 32)
lmh_entropy_kernel(const float* __restrict__ lists, const int32_t* __restrict__ counts, int n, int nl, int k,
                   float* __restrict__ H) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * LE_WARPS + (threadIdx.x >> 5);
  if (row >= n) return;
  const float* L = lists + (int64_t)row * nl * k;
  const int32_t* C = counts + (int64_t)row * nl;
  const int tot = nl * k;
  uint32_t key[LE_NK];
  int have = 0;
#pragma unroll
  for (int i = 0; i < LE_NK; ++i) {
    const int f = lane + 32 * i;
    uint32_t kv = 0;
    if (f < tot) {
      const int j = f / k;
      if (f - j * k < __ldg(C + j)) kv = f2key(__ldg(L + f));
    }
    key[i] = kv;
    have += kv != 0u;
  }
  const int total = __reduce_add_sync(FULL, have);
  const int kk = total < k ? total : k;
  uint32_t t = 0, top = 0;
  int ngt = 0;
  if (kk > 0) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = t | (1u << bit);
      int c = 0;
#pragma unroll
      for (int i = 0; i < LE_NK; ++i) c += key[i] >= cand;
      if (__reduce_add_sync(FULL, c) >= kk) t = cand;
    }
#pragma unroll
    for (int i = 0; i < LE_NK; ++i) {
      ngt += key[i] > t;
      top = key[i] > top ? key[i] : top;
    }
    ngt = __reduce_add_sync(FULL, ngt);
    top = __reduce_max_sync(FULL, top);
  }
  const float m = key2f(top), tv = key2f(t);
  float s = 0.f, u = 0.f;
#pragma unroll
  for (int i = 0; i < LE_NK; ++i) {
    if (key[i] > t) {
      const float x = key2f(key[i]) - m;
      const float ex = expf(x);
      s += ex;
      u += ex * x;
    }
  }
  s = warp_sum(s);
  u = warp_sum(u);
  if (lane == 0) {
    const int fill = kk - ngt;                      // copies of the kk-th value
    if (fill > 0) {
      const float x = tv - m;
      const float ex = expf(x);
      s += fill * ex;
      u += fill * ex * x;
    }
    H[row] = (kk == 0 || s <= 0.f) ? 0.f : logf(s) - u / s;
  }
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 lm_encode() {
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

// [rows][Dh] bf16, rows `stride` elements apart, boxes of 64 x box_rows, 128B swizzle;
// rows and columns past the ends read as zero.
static bool lm_map(CUtensorMap* map, const void* base, int64_t rows, int Dh, int64_t stride, int box_rows) {
  auto enc = lm_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)Dh, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)stride * 2};
  cuuint32_t box[2] = {(cuuint32_t)LM_BK, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

LmPlan plan_lmhead(int n, int Dh, int V, int k, int sms) {
  LmPlan p{};
  const int nmt = (n + LM_BM - 1) / LM_BM;
  const int ntn = (V + LM_BN - 1) / LM_BN;
  // x tiles live at once (about sms / S of them) stay within 64 MB of L2; enough items
  // for two per SM; at most 32 LE_NK / k segments, so a row's lists fit one warp
  const int64_t xtile = (int64_t)LM_BM * Dh * 2;
  int S = (int)(((int64_t)sms * xtile + (64ll << 20) - 1) / (64ll << 20));
  const int s_par = (2 * sms + nmt - 1) / nmt;
  if (s_par > S) S = s_par;
  const int s_max = 32 * LE_NK / k;
  if (S > s_max) S = s_max;
  if (S > ntn) S = ntn;
  if (S < 1) S = 1;
  p.tps = (ntn + S - 1) / S;
  p.S = (ntn + p.tps - 1) / p.tps;
  p.ntn = ntn;
  p.total = (int64_t)nmt * p.S;
  p.grid = (int)(p.total < sms ? p.total : sms);
  p.scratch_bytes = (size_t)p.grid * LM_BM * LM_CAP * sizeof(float);   // [grid][2][128][LM_CAP]
  p.lists_bytes = (size_t)n * p.S * k * sizeof(float);
  p.counts_bytes = (size_t)n * p.S * sizeof(int32_t);
  auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
  p.bytes = al(p.scratch_bytes) + al(p.lists_bytes) + al(p.counts_bytes);
  return p;
}

static size_t lm_smem() { return (size_t)LM_NST * LM_STAGE + sizeof(LmSmem) + 1024; }

cudaError_t launch_lmhead_entropy(const LmheadParams& q, void* ws, cudaStream_t st) {
  const LmPlan p = plan_lmhead(q.n, q.Dh, q.V, q.k, num_sms());
  CUtensorMap mX, mW;
  if (!lm_map(&mX, q.x, q.n, q.Dh, q.x_stride, LM_BM) || !lm_map(&mW, q.W, q.V, q.Dh, q.W_stride, LM_BN))
    return cudaErrorInvalidValue;
  auto al = [](size_t b) { return (b + 255) & ~size_t(255); };
  uint8_t* w = static_cast<uint8_t*>(ws);
  LmArgs a{};
  a.n = q.n;
  a.V = q.V;
  a.k = q.k;
  a.S = p.S;
  a.tps = p.tps;
  a.ntn = p.ntn;
  a.nk = (q.Dh + LM_BK - 1) / LM_BK;
  a.total = p.total;
  a.scratch = reinterpret_cast<float*>(w);
  a.lists = reinterpret_cast<float*>(w + al(p.scratch_bytes));
  a.counts = reinterpret_cast<int32_t*>(w + al(p.scratch_bytes) + al(p.lists_bytes));
  a.status = status_ptr();
  const size_t smem = lm_smem();
  cudaError_t e = cudaFuncSetAttribute(lmh_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  lmh_topk_kernel<<<p.grid, LM_THREADS, smem, st>>>(mX, mW, a);
  if ((e = cudaGetLastError())) return e;
  count_launch();
  lmh_entropy_kernel<<<(q.n + LE_WARPS - 1) / LE_WARPS, LE_WARPS * 32, 0, st>>>(a.lists, a.counts, q.n, p.S,
                                                                                 q.k, q.H);
  if ((e = cudaGetLastError())) return e;
  count_launch();
  return cudaSuccess;
}

}  // namespace kvc
