// Observation-window attention score, both passes in one persistent launch.
//
// [InfoKV] Methodology / Technical details: A_i is the mean over the G*W
// window rows of softmax(q k^T * scale)_i, S_i = alpha * A_i + (1 - alpha) *
// Softmax(D * H)_i; [SelKV] Pipeline overview step 1 (VATP): S_i = A_i ||v_i||.
//
// The two-pass method needs every key twice: pass 1 gives each window row its
// max and sum of exp over all keys, pass 2 sums each key's normalised
// probabilities over the rows.  Run as two launches, each pass streams all of
// K from HBM.  Here the passes are interleaved per (layer, KV head) slice in
// one launch, so the pass-2 reads of a slice come from L2:
//
//   work order  step k = pass-1 chunks of slice k, then pass-2 chunks of
//               slice k - lag; CTA c takes items c, c + grid, c + 2 grid, ...
//   pass 1      each epilogue warpgroup leaves its (max, sum) partial of the
//               chunk in shared memory; a helper warp merges them into the
//               chunk's partial and stores it.  Chunks form groups of 8: the
//               helper that completes a group (acq_rel counter) merges its
//               partials, the one that completes the last group of the slice
//               merges the group partials into the slice's row constants and
//               publishes a ready flag (release).  The merge order is fixed,
//               so the result does not depend on timing.
//   pass 2      the producer waits for the slice's ready flag (acquire,
//               bounded), then bulk-copies the row constants into a ring that
//               the epilogue reads
//
// Every item a CTA waits on comes earlier in the order than the waiting item
// and depends only on still earlier items, and the grid is launched
// cooperatively (all CTAs resident), so the waits always end; each is still
// bounded in time and reports ST_TIMEOUT.
//
// Roles per CTA (one per SM): warp 0 TMA producer (K tiles of 128 keys in a
// 4-stage ring, Q rows double-buffered per item, row constants in a 4-deep
// ring), warp 1 TMEM owner and tcgen05.mma issuer, warp 2 helper (partials,
// counts, merges), warps 3.. four epilogue warpgroups (WIN_FUSED_NB) that take tiles
// round-robin, each owning one 128-column TMEM accumulator.
#include <cudaTypedefs.h>

#include <cstddef>

#include "exp2_poly.cuh"
#include "kernels.cuh"
#include "tc_sm100.cuh"

namespace kvc {
using namespace tc;

constexpr int FU_NB = WIN_FUSED_NB;          // epilogue warpgroups = TMEM accumulators
constexpr int FU_KT = 128;                   // keys per tile
constexpr int FU_NST = 4;                    // K ring stages
constexpr int FU_QR = 128;                   // staged Q rows (R <= 128)
constexpr int FU_ATOM = FU_KT * 128;         // 128 rows x 64 bf16, 128B-swizzled
constexpr int FU_TILE = 2 * FU_ATOM;         // head_dim 128
constexpr int FU_QBYTES = FU_QR * 256;
constexpr int FU_RCN = 4;                    // row-constant ring depth (pass-2 items)
constexpr int FU_PBN = 4;                    // partial buffers (pass-1 items)
constexpr int FU_EPI0 = 3;                   // first epilogue warp
constexpr int FU_GRP = WIN_FUSED_GROUP;      // chunks per merge group
constexpr float FU_LOG2E = 1.4426950408889634f;
#ifndef KVC_FU_POLY
#define KVC_FU_POLY 0
#endif
constexpr int FU_POLY = KVC_FU_POLY;         // every FU_POLY-th exponential on the FMA pipe (0: none)

// 2^x for element j of an unrolled loop (j a compile-time constant there): the MUFU
// exp2, or the FMA-pipe polynomial for one element in FU_POLY.
__device__ __forceinline__ float fu_exp2(float x, int j) {
  return (FU_POLY > 0 && (j % (FU_POLY > 0 ? FU_POLY : 1)) == FU_POLY - 1) ? exp2_poly(x) : ex2(x);
}

struct FuArgs {
  WinParams p;
  int nslices, nchunk, chunk, lag;
  int64_t total;     // items: 2 * nslices * nchunk
  float c2;          // scale * log2(e)
  uint64_t flag_wait_ns;   // limit of the wait for another CTA's row constants
  unsigned* status;
};

struct FuSmem {
  uint64_t full[FU_NST], empty[FU_NST], tfull[FU_NB], tempty[FU_NB], qfull[2], qempty[2];
  uint64_t rcfull[FU_RCN], rcempty[FU_RCN], pfull[FU_PBN], pempty[FU_PBN];
  uint64_t mdrain;                            // the MMA issuer's final commit
  uint32_t tmem_base;
  int abort;
  int qmin;
  alignas(16) float rowc[FU_RCN][FU_QR];      // pass 2: negated row constant -(log2 max + log2 sum)
  float2 pbuf[FU_PBN][FU_NB * FU_QR];         // pass 1: the warpgroups' (log2 max, sum) per row
  int qp[FU_QR];                              // position of every window row
};
static_assert(offsetof(FuSmem, rowc) % 16 == 0, "rowc is filled by a bulk copy and read as float4");

struct FuItem {
  int pass, slice, l, g, chunk, key0, key1, ntile;
};

// Bounded wait that ignores the abort flag: used after an abort to let the asynchronous
// copies and MMAs this CTA already issued land before it frees its memory.
__device__ __forceinline__ void fu_drain_wait(uint64_t* bar, uint32_t parity, unsigned* status) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = gtimer();
  while (!mbar_try_wait(bar, parity)) {
    if (gtimer() - t0 > WAIT_NS) {
      flag(status, ST_TIMEOUT);
      return;
    }
  }
}

// Item o of the work order (see the file comment).
__device__ __forceinline__ FuItem fu_item(const FuArgs& a, int64_t o) {
  const int ns = a.nslices, lag = a.lag;
  const int u = (int)(o / a.nchunk);
  FuItem x;
  x.chunk = (int)(o % a.nchunk);
  if (u < lag) {
    x.pass = 1; x.slice = u;
  } else if (u < 2 * ns - lag) {
    const int v = u + lag;
    x.pass = (v & 1) ? 2 : 1;
    x.slice = (v & 1) ? (v >> 1) - lag : (v >> 1);
  } else {
    x.pass = 2; x.slice = u - ns;
  }
  x.l = x.slice / a.p.Hkv;
  x.g = x.slice % a.p.Hkv;
  x.key0 = x.chunk * a.chunk;
  x.key1 = min(a.p.n, x.key0 + a.chunk);
  x.ntile = (x.key1 - x.key0 + FU_KT - 1) / FU_KT;
  return x;
}

// (max, sum) of `count` partials src[i * 128 + r] for the rows r = lane + 32 j,
// j < 4: max in log2 units, sum relative to it; merged in index order.
__device__ __forceinline__ void fu_merge_rows(const float2* src, int count, int lane, float (&M)[4],
                                              float (&S)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) { M[j] = -INFINITY; S[j] = 0.f; }
  for (int i0 = 0; i0 < count; i0 += 8) {
    float2 v[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        v[i][j] = i0 + i < count ? __ldcg(src + (int64_t)(i0 + i) * FU_QR + lane + 32 * j)
                                 : make_float2(-INFINITY, 0.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float mx = M[j];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx = fmaxf(mx, v[i][j].x);
      if (mx > -INFINITY) {
        float acc = S[j] * ex2(M[j] - mx);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc += v[i][j].y * ex2(v[i][j].x - mx);
        S[j] = acc;
        M[j] = mx;
      }
    }
  }
}

// Pass 2, 16 window rows (columns c*16 .. c*16+15) of one key: acc += their probabilities
// 2^(s c2 + nrc), nrc the row's negated constant; masked rows (the key after the row's query)
// contribute nothing.  r4 holds the 16 negated constants, loaded by the caller before the
// accumulator columns.  Column pairs go through packed FMAs and adds (each lane rounds as
// the scalar instruction): acc01 holds the sums of columns = 0, 1 (mod 4), acc23 of 2, 3.
__device__ __forceinline__ void fu_pass2_cols(const float* v, const float4 (&r4)[4], int c, const float* rc,
                                              const int* qp, int kp, bool need_mask, uint64_t c2x2,
                                              uint64_t& acc01, uint64_t& acc23) {
  if (!need_mask) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 x01 = upk2(fma2(pk2(v[q * 4 + 0], v[q * 4 + 1]), c2x2, pk2(r4[q].x, r4[q].y)));
      const float2 x23 = upk2(fma2(pk2(v[q * 4 + 2], v[q * 4 + 3]), c2x2, pk2(r4[q].z, r4[q].w)));
      acc01 = add2(acc01, pk2(ex2(x01.x), ex2(x01.y)));
      acc23 = add2(acc23, pk2(ex2(x23.x), ex2(x23.y)));
    }
  } else {
    const float c2 = upk2(c2x2).x;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float e[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = c * 16 + q * 4 + u;
        e[u] = kp > qp[r] ? 0.f : ex2(fmaf(v[q * 4 + u], c2, rc[r]));
      }
      acc01 = add2(acc01, pk2(e[0], e[1]));
      acc23 = add2(acc23, pk2(e[2], e[3]));
    }
  }
}

__device__ __forceinline__ float fu_tree_max32(const float* v) {
  float t[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) t[j] = fmaxf(v[j], v[j + 16]);
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
  return t[0];
}

__global__ void __launch_bounds__(FU_EPI0 * 32 + FU_NB * 128, 1)
win_fused_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapQ,
                 const FuArgs a) {
  extern __shared__ uint8_t fu_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fu_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Qs = base;                          // [2][FU_QBYTES]
  uint8_t* Ks = base + 2 * FU_QBYTES;          // [FU_NST][FU_TILE]
  FuSmem* sm = reinterpret_cast<FuSmem*>(Ks + FU_NST * FU_TILE);
  const WinParams& p = a.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &sm->abort;
  const int64_t stride = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < FU_NST; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int b = 0; b < FU_NB; ++b) {
      mbar_init(&sm->tfull[b], 1);
      mbar_init(&sm->tempty[b], 4);            // the four warps of warpgroup b
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&sm->qfull[q], 1);
      mbar_init(&sm->qempty[q], 1);            // MMA commit
    }
    for (int q = 0; q < FU_RCN; ++q) {
      mbar_init(&sm->rcfull[q], 1);
      mbar_init(&sm->rcempty[q], 4 * FU_NB);   // every epilogue warp
    }
    for (int q = 0; q < FU_PBN; ++q) {
      mbar_init(&sm->pfull[q], 4 * FU_NB);     // every epilogue warp
      mbar_init(&sm->pempty[q], 1);            // helper
    }
    mbar_init(&sm->mdrain, 1);
    sm->abort = 0;
    sm->qmin = query_pos_min(p);
    fence_mbar_init();
  }
  for (int r = threadIdx.x; r < FU_QR; r += blockDim.x) sm->qp[r] = r < p.R ? query_pos(p, 0, r % p.W) : -0x7fffffff;
  if (warp == 1) tmem_alloc(&sm->tmem_base, 512);
  if (warp == 0 && lane == 0) {
    prefetch_map(&mapK);
    prefetch_map(&mapQ);
  }
  __syncthreads();
  fence_after();
  const uint32_t tmem = sm->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();    // pass-1 tiles are read again by pass 2
      const uint64_t done = l2_policy_evict_first();   // pass-2 tiles are not
      uint32_t tile = 0, qi = 0, p2i = 0, qissued = 0;
      for (int64_t o = blockIdx.x; o < a.total; o += stride, ++qi) {
        const FuItem x = fu_item(a, o);
        const int qb = qi & 1;
        if (x.pass == 2) {
          const int rs = p2i % FU_RCN;
          if (!mbar_wait(&sm->rcempty[rs], ((p2i / FU_RCN) & 1) ^ 1, abort, a.status)) goto producer_done;
          // the slice's row constants: published by the warpgroup that merged its partials
          const int* rdy = a.p.fsync + x.slice;
          if (ld_acquire_gpu(rdy) == 0) {
            const uint64_t t0 = gtimer();
            while (ld_acquire_gpu(rdy) == 0) {
              if (*abort) goto producer_done;
              if (gtimer() - t0 > a.flag_wait_ns) {
                flag(a.status, ST_TIMEOUT);
                *abort = 1;
                goto producer_done;
              }
              __nanosleep(256);
            }
          }
          fence_proxy_async_global();
          mbar_expect_tx(&sm->rcfull[rs], FU_QR * 4);
          bulk_load(sm->rowc[rs], a.p.frowc + (int64_t)x.slice * FU_QR, FU_QR * 4, &sm->rcfull[rs]);
          ++p2i;
        }
        if (!mbar_wait(&sm->qempty[qb], ((qi >> 1) & 1) ^ 1, abort, a.status)) goto producer_done;
        mbar_expect_tx(&sm->qfull[qb], FU_QBYTES);
        {
          const int row0 = (x.l * p.Hq + x.g * p.G) * p.W;
          uint8_t* q = Qs + qb * FU_QBYTES;
          tma_load_2d(q, &mapQ, 0, row0, &sm->qfull[qb]);
          tma_load_2d(q + FU_QR * 128, &mapQ, 64, row0, &sm->qfull[qb]);
          ++qissued;
        }
        const uint64_t pol = x.pass == 1 ? keep : done;
        for (int t = 0; t < x.ntile; ++t, ++tile) {
          const int s = tile % FU_NST;
          if (!mbar_wait(&sm->empty[s], ((tile / FU_NST) & 1) ^ 1, abort, a.status)) goto producer_done;
          mbar_expect_tx(&sm->full[s], FU_TILE);
          uint8_t* dst = Ks + s * FU_TILE;
          const int key = x.key0 + t * FU_KT;
          tma_load_4d_policy(dst, &mapK, 0, key, x.g, x.l, &sm->full[s], pol);
          tma_load_4d_policy(dst + FU_ATOM, &mapK, 64, key, x.g, x.l, &sm->full[s], pol);
        }
      }
    producer_done:
      // every copy issued so far lands before the CTA moves on (after an abort, some were
      // never consumed): the last FU_NST K tiles, the last two Q loads, the last FU_RCN
      // row-constant copies, each on the phase its arming started
      for (uint32_t t = tile > FU_NST ? tile - FU_NST : 0; t < tile; ++t)
        fu_drain_wait(&sm->full[t % FU_NST], (t / FU_NST) & 1, a.status);
      for (uint32_t j = qissued > 2 ? qissued - 2 : 0; j < qissued; ++j)
        fu_drain_wait(&sm->qfull[j & 1], (j >> 1) & 1, a.status);
      for (uint32_t j = p2i > FU_RCN ? p2i - FU_RCN : 0; j < p2i; ++j)
        fu_drain_wait(&sm->rcfull[j % FU_RCN], (j / FU_RCN) & 1, a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id1 = idesc_bf16(128, 128);   // S1 = Q K^T: window rows x keys
      const uint32_t id2 = idesc_bf16(128, p.R);   // S2 = K Q^T: keys x window rows
      uint32_t tile = 0, qi = 0;
      // operand descriptors: stage s / Q buffer qb lie s * FU_TILE / qb * FU_QBYTES bytes
      // past the first, i.e. that many 16-byte units in the descriptor's address field
      const uint64_t kd0 = sw128_desc(Ks), qd0 = sw128_desc(Qs);
      for (int64_t o = blockIdx.x; o < a.total; o += stride, ++qi) {
        const FuItem x = fu_item(a, o);
        const int qb = qi & 1;
        if (!mbar_wait(&sm->qfull[qb], (qi >> 1) & 1, abort, a.status)) goto mma_done;
        for (int t = 0; t < x.ntile; ++t, ++tile) {
          const int s = tile % FU_NST;
          const int b = tile % FU_NB;
          if (!mbar_wait(&sm->full[s], (tile / FU_NST) & 1, abort, a.status)) goto mma_done;
          if (!mbar_wait(&sm->tempty[b], ((tile / FU_NB) & 1) ^ 1, abort, a.status)) goto mma_done;
          fence_after();
          const uint32_t d = tmem + (uint32_t)(b * 128);
          if (x.pass == 1) mma_bf16_k128(d, qd0 + qb * (FU_QBYTES / 16), kd0 + s * (FU_TILE / 16), FU_QR * 8, FU_ATOM / 16, id1);
          else mma_bf16_k128(d, kd0 + s * (FU_TILE / 16), qd0 + qb * (FU_QBYTES / 16), FU_ATOM / 16, FU_QR * 8, id2);
          mma_commit(&sm->empty[s]);
          mma_commit(&sm->tfull[b]);
        }
        mma_commit(&sm->qempty[qb]);
      }
    mma_done:
      // every MMA issued so far completes before TMEM is freed
      mma_commit(&sm->mdrain);
      fu_drain_wait(&sm->mdrain, 0, a.status);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ helper: pass-1 partials
    const int ngroups = (a.nchunk + FU_GRP - 1) / FU_GRP;
    int* ready = p.fsync;                          // [nslices]
    int* scount = p.fsync + a.nslices;             // [nslices] finished groups
    int* gcount = p.fsync + 2 * a.nslices;         // [nslices][ngroups] finished chunks
    float2* gpart = p.fpart + (int64_t)a.nslices * a.nchunk * FU_QR;   // [nslices][ngroups][128]
    uint32_t pi = 0;
    for (int64_t o = blockIdx.x; o < a.total; o += stride) {
      const FuItem x = fu_item(a, o);
      if (x.pass != 1) continue;
      const int ps = pi % FU_PBN;
      const bool ok = mbar_wait(&sm->pfull[ps], (pi / FU_PBN) & 1, abort, a.status);
      if (!__all_sync(FULL, ok)) break;
      // the chunk's partial: the warpgroups' partials merged, 4 rows per lane
      float2* cp = p.fpart + ((int64_t)x.slice * a.nchunk + x.chunk) * FU_QR;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = lane + 32 * j;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < FU_NB; ++w) mx = fmaxf(mx, sm->pbuf[ps][w * FU_QR + r].x);
        float sum = 0.f;
        if (mx > -INFINITY) {
#pragma unroll
          for (int w = 0; w < FU_NB; ++w) {
            const float2 q = sm->pbuf[ps][w * FU_QR + r];
            sum += q.y * ex2(q.x - mx);
          }
        }
        cp[r] = make_float2(mx, sum);
      }
      // The warp barrier orders every lane's stores before lane 0's release-add; the
      // add's acquire side (for the last of a group) covers the other CTAs' partials.
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm->pempty[ps]);
      ++pi;
      const int grp = x.chunk / FU_GRP;
      const int gsize = min(FU_GRP, a.nchunk - grp * FU_GRP);
      int old = 0;
      if (lane == 0) old = atom_add_acq_rel_gpu(gcount + x.slice * ngroups + grp, 1);
      old = __shfl_sync(FULL, old, 0);
      if (old != gsize - 1) continue;
      float M[4], S[4];
      fu_merge_rows(p.fpart + ((int64_t)x.slice * a.nchunk + grp * FU_GRP) * FU_QR, gsize, lane, M, S);
      float2* gp = gpart + ((int64_t)x.slice * ngroups + grp) * FU_QR;
#pragma unroll
      for (int j = 0; j < 4; ++j) gp[lane + 32 * j] = make_float2(M[j], S[j]);
      __syncwarp();
      if (lane == 0) old = atom_add_acq_rel_gpu(scount + x.slice, 1);
      old = __shfl_sync(FULL, old, 0);
      if (old != ngroups - 1) continue;
      // every group of the slice is in: the row constants
      fu_merge_rows(gpart + (int64_t)x.slice * ngroups * FU_QR, ngroups, lane, M, S);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = lane + 32 * j;
        // p_ri = 2^(s c2 - rowc); a row with no visible key contributes nothing
        p.frowc[(int64_t)x.slice * FU_QR + r] =
            (r < p.R && M[j] > -INFINITY && S[j] > 0.f) ? -(M[j] + log2f(S[j])) : -INFINITY;
      }
      __syncwarp();
      if (lane == 0) st_release_gpu(ready + x.slice, 1);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int wg = (warp - FU_EPI0) >> 2;    // takes the tiles with tile % FU_NB == wg
    const int q4 = warp & 3;                 // TMEM lane quarter of this warp
    const int rowl = q4 * 32 + lane;         // accumulator row (TMEM lane) of this thread
    const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(wg * 128);
    const int qmin = sm->qmin;
    const int qrow = sm->qp[rowl];
    uint32_t tile = 0, pi = 0, p2i = 0;
    for (int64_t o = blockIdx.x; o < a.total; o += stride) {
      const FuItem x = fu_item(a, o);
      const int rs = p2i % FU_RCN;
      const uint32_t tile0 = tile;
      const uint32_t first = tile0 + (uint32_t)((wg - (int)(tile0 % FU_NB) + FU_NB) % FU_NB);
      const bool mine = first < tile0 + (uint32_t)x.ntile;
      if (x.pass == 2 && mine && !*abort) mbar_wait(&sm->rcfull[rs], (p2i / FU_RCN) & 1, abort, a.status);
      float m2 = -INFINITY, s1 = 0.f;
      for (int t = 0; t < x.ntile; ++t, ++tile) {
        if ((int)(tile % FU_NB) != wg) continue;
        bool ok = !*abort && mbar_wait(&sm->tfull[wg], (tile / FU_NB) & 1, abort, a.status);
        ok = __all_sync(FULL, ok);
        if (!ok) continue;
        fence_after();
        const int key0 = x.key0 + t * FU_KT;
        const bool need_mask = key0 + FU_KT > x.key1 || key_pos(p, x.l, x.g, key0 + FU_KT - 1) > qmin;
        if (x.pass == 1) {
#pragma unroll 1
          for (int c = 0; c < 4; c += 2) {
            float v[64];
            __syncwarp();
            tmem_ld32(lane_addr + (uint32_t)(c * 32), v);
            tmem_ld32(lane_addr + (uint32_t)(c * 32 + 32), v + 32);
            tmem_wait_ld();
            if (need_mask) {
#pragma unroll
              for (int j = 0; j < 64; ++j) {
                const int key = key0 + c * 32 + j;
                if (key >= x.key1 || key_pos(p, x.l, x.g, key) > qrow) v[j] = -INFINITY;
              }
            }
            const float mx = fmaxf(fu_tree_max32(v), fu_tree_max32(v + 32));
            const float mn = fmaxf(m2, mx * a.c2);
            if (mn > -INFINITY) {
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
              s1 = s1 * ex2(m2 - mn) + ((a01.x + a01.y) + (a23.x + a23.y));
              m2 = mn;
            }
          }
        } else {
          const int key = key0 + rowl;
          const bool kvalid = key < x.key1;
          const int kp = kvalid ? key_pos(p, x.l, x.g, key) : 0x7fffffff;
          // inputs of the score epilogue, loaded before the accumulator so their latency
          // overlaps the exponentials
          float pre = 0.f, st0 = 0.f, st1 = 1.f;
          if (kvalid && p.S) {
            if (p.mode == KVC_SCORE_INFOKV) {
              pre = __ldg(p.D + x.l * p.Dsl + x.g * p.Dsh + key) * __ldg(p.H + x.l * p.Hsl + x.g * p.Hsh + key);
              st0 = __ldg(p.estats + 3 * x.slice);
              st1 = __ldg(p.estats + 3 * x.slice + 1);
            } else if (p.mode == KVC_SCORE_VATP) {
              pre = __ldg(p.vnorm + (int64_t)x.slice * p.n + key);
            }
          }
          const float* rc = sm->rowc[rs];
          uint64_t acc01 = pk2(0.f, 0.f), acc23 = pk2(0.f, 0.f);
          const uint64_t c2x2 = pk2(a.c2, a.c2);
          const int nc16 = p.R >> 4;
#pragma unroll 1
          for (int c = 0; c < nc16; ++c) {
            // the chunk's row constants first: the wait below orders memory, so shared loads
            // issued after it would add their latency to every chunk
            float4 r4[4];
            const float4* rc4 = reinterpret_cast<const float4*>(rc) + c * 4;
#pragma unroll
            for (int q = 0; q < 4; ++q) r4[q] = rc4[q];
            float v[16];
            __syncwarp();
            tmem_ld16(lane_addr + (uint32_t)(c * 16), v);
            tmem_wait_ld();
            fu_pass2_cols(v, r4, c, rc, sm->qp, kp, need_mask, c2x2, acc01, acc23);
          }
          if (kvalid) {
            const float2 a01 = upk2(acc01), a23 = upk2(acc23);
            const float A = ((a01.x + a01.y) + (a23.x + a23.y)) / (float)p.R;
            const int64_t oo = (int64_t)x.slice * p.n + key;
            float S = A;
            if (!p.S) {
            } else if (p.mode == KVC_SCORE_INFOKV) {
              S = p.alpha * A + (1.f - p.alpha) * (expf(pre - st0) / st1);
            } else if (p.mode == KVC_SCORE_VATP) {
              S = A * pre;
            }
            if (p.A) p.A[oo] = A;
            if (p.S) p.S[oo] = S;
          }
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->tempty[wg]);
      }
      if (x.pass == 1) {
        // this warpgroup's partial of the chunk, handed to the helper warp
        const int ps = pi % FU_PBN;
        if (!*abort) mbar_wait(&sm->pempty[ps], ((pi / FU_PBN) & 1) ^ 1, abort, a.status);
        sm->pbuf[ps][wg * FU_QR + rowl] = make_float2(m2, s1);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->pfull[ps]);
        ++pi;
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->rcempty[rs]);
        ++p2i;
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
static size_t fu_smem() { return (size_t)2 * FU_QBYTES + (size_t)FU_NST * FU_TILE + sizeof(FuSmem) + 1024; }

bool window_fused_supported(const WinParams& p, kvc_dtype dt) {
  // the query positions are staged once per CTA: one row for every layer
  return window_tc_supported(p, dt) && p.R <= FU_QR && p.qlpb == 0 && !p.wlse && p.fpart && p.frowc && p.fsync &&
         p.fchunk % FU_KT == 0 && p.fchunk > 0;
}

cudaError_t launch_window_fused(const WinParams& p, cudaStream_t st, int grid_ctas) {
  CUtensorMap mK, mQ;
  if (!make_window_maps(p, FU_QR, &mK, &mQ)) return cudaErrorInvalidValue;
  FuArgs a{};
  a.p = p;
  a.nslices = p.L * p.Hkv;
  a.chunk = p.fchunk;
  a.nchunk = (p.n + p.fchunk - 1) / p.fchunk;
  a.lag = a.nslices < WIN_FUSED_LAG ? a.nslices : WIN_FUSED_LAG;
  a.total = (int64_t)2 * a.nslices * a.nchunk;
  a.c2 = p.scale * FU_LOG2E;
  a.flag_wait_ns = p.flag_wait_ns > 0 ? p.flag_wait_ns : WAIT_NS;
  a.status = status_ptr();
  const int ngroups = (a.nchunk + FU_GRP - 1) / FU_GRP;
  cudaError_t e = cudaMemsetAsync(p.fsync, 0, sizeof(int) * (size_t)a.nslices * (2 + ngroups), st);
  if (e != cudaSuccess) return e;
  if (p.mode == KVC_SCORE_VATP) {
    e = launch_vnorm(p, st);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = fu_smem();
  auto kern = win_fused_kernel;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = grid_ctas > 0 && grid_ctas < num_sms() ? grid_ctas : num_sms();
  if ((int64_t)grid > a.total) grid = (int)a.total;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(FU_EPI0 * 32 + FU_NB * 128);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the cross-CTA waits can end
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, mK, mQ, a);
  if (e == cudaSuccess) count_launch();
  return e;
}

}  // namespace kvc
