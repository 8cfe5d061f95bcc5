// RECAS dynamic sparse decoding attention.
//
// [RECAS] 2.C: inside the retained cache a query-aware selector limits each decode
// step's interactions: a sparse score combining the immediate query-key compatibility
// with the utility score picks the top K_t tokens (the active set); the others stay
// cached for later steps.  2.A: the utility is alpha tr + beta hi (+ the stage term gi,
// out of scope), hi the normalised attention accumulated over earlier steps.  2.D: the
// active attention costs O(kappa rho N d).
//
// Readings: per (sequence, layer, KV head) row of n cached tokens,
//   tr_i    = attention of token i under the current query, averaged over the G query
//             heads of the KV head (softmax over the row, scale 1/sqrt(d));
//   hi_i    = acc_i / cnt_i, acc_i the attention the token received at the steps it has
//             been cached (head mean, 0 when inactive), cnt_i = t_cur - max(pos_i, n0);
//   sigma_i = a_tr tr_i + b_hi hi_i; the active set is the top K_t = ceil(kappa n) by
//             sigma, ties to the lower position;
//   o       = attention renormalised over the active set; acc_i += its head mean there.
//
// Launches: sparse_scores_kernel streams the row's keys once on mma.sync (the G queries
// as register fragments, the keys straight from global memory in 16-byte loads) and
// stores s = q k scale for the G heads, with each 256-key chunk's per-head max and sum of
// exponentials; sparse_row_kernel (one CTA per row, seven per SM, templated on G) merges
// those partials into the head softmax statistics, forms sigma, selects the active set
// (a radix select over sigma's keys in shared memory, ties to the lower position, as
// kvc_select) and compacts it in place, then takes the softmax statistics over the active
// set, gathers the active value rows (eight in flight per warp), renormalises over the
// active set, writes o and updates acc.
#include "kernels.cuh"

namespace kvc {

constexpr int SP_D = 128;
constexpr int SP_SC_THREADS = 128;            // scores: 4 warps, 64 keys each per block
constexpr int SP_SC_KEYS = SPARSE_CHUNK;
constexpr int SP_MAXG = 8;

// s = scale * q k for the G heads and 8 keys per mma.sync m16n8k16 (bf16 in, fp32
// accumulate): A = the G queries padded to 16 rows (fragments kept in registers for the
// whole row), B = 8 key rows read straight from global memory.  A dot product does not
// depend on the order of the dimensions, so the fragments take the dimensions in the
// order 16-byte loads deliver them, the same order for the queries and the keys: thread
// (gq, cq) loads bytes 64 j + 16 cq .. + 15 of key gq's row (j = 0..3), and MMA step
// 2 j + t uses its 4-byte pieces 2 t and 2 t + 1 as the k-rows (2 cq, 2 cq + 1) and
// (2 cq + 8, 2 cq + 9).
__device__ __forceinline__ void sp_mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Also writes, per head, the max and the sum of exp(s - max) over the block's keys (one
// partial per 256-key chunk), which the row kernel merges in chunk order.
__global__ void __launch_bounds__(SP_SC_THREADS) sparse_scores_kernel(SparseParams p) {
  __shared__ float hs[SP_SC_THREADS / 32][SP_MAXG][2];
  const int row = blockIdx.y, bl = row / p.Hkv, g = row % p.Hkv;
  const int b = bl / p.L, l = bl % p.L;
  const int n = min(p.len[bl], p.max_len);
  const int key0 = blockIdx.x * SP_SC_KEYS;
  if (key0 >= n) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, cq = lane & 3;          // mma fragment row / column pair
  // query fragments in the dimension order of the key loads (rows >= G and 8..15 zero)
  uint32_t qa[8][2];
  const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
      reinterpret_cast<const __nv_bfloat16*>(p.q) + ((int64_t)bl * p.Hq + g * p.G + gq) * SP_D);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int w = (ks >> 1) * 16 + cq * 4 + (ks & 1) * 2;
    qa[ks][0] = gq < p.G ? __ldg(qrow + w) : 0u;
    qa[ks][1] = gq < p.G ? __ldg(qrow + w + 1) : 0u;
  }
  const char* Kb = p.K + b * p.Ksb + l * p.Ksl + g * p.Ksh + cq * 16;
  float* srow = p.s + (int64_t)row * p.G * p.max_len;
  const int wkey0 = key0 + warp * (SP_SC_KEYS / (SP_SC_THREADS / 32));
  float hm = -INFINITY, hz = 0.f;                   // head gq, over this thread's keys
#pragma unroll 1
  for (int t = 0; t < SP_SC_KEYS / (SP_SC_THREADS / 32); t += 16) {
    // two 8-key tiles in flight
    uint4 kb[2][4];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int key = wkey0 + t + u * 8 + gq;
      const char* kr = Kb + (int64_t)(key < n ? key : 0) * p.Kst;
#pragma unroll
      for (int j = 0; j < 4; ++j) kb[u][j] = __ldg(reinterpret_cast<const uint4*>(kr + j * 64));
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t a0[4] = {qa[2 * j][0], 0u, qa[2 * j][1], 0u};
        sp_mma(c, a0, kb[u][j].x, kb[u][j].y);
        const uint32_t a1[4] = {qa[2 * j + 1][0], 0u, qa[2 * j + 1][1], 0u};
        sp_mma(c, a1, kb[u][j].z, kb[u][j].w);
      }
      // c[0], c[1]: head gq, keys 2 cq, 2 cq + 1 of the tile
      const int k2 = wkey0 + t + u * 8 + 2 * cq;
      if (gq < p.G) {
        float* dst = srow + (int64_t)gq * p.max_len + k2;
        const float s0 = c[0] * p.scale, s1 = c[1] * p.scale;
        const bool v0 = k2 < n, v1 = k2 + 1 < n;
        if (v0) dst[0] = s0;
        if (v1) dst[1] = s1;
        const float mx = fmaxf(v0 ? s0 : -INFINITY, v1 ? s1 : -INFINITY);
        if (mx > -INFINITY) {
          const float mn = fmaxf(hm, mx);
          hz = hz * expf(hm - mn) + (v0 ? expf(s0 - mn) : 0.f) + (v1 ? expf(s1 - mn) : 0.f);
          hm = mn;
        }
      }
    }
  }
  // the four lanes of a head, then the warps, in a fixed order
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    const float mo = __shfl_xor_sync(FULL, hm, o), zo = __shfl_xor_sync(FULL, hz, o);
    const float mn = fmaxf(hm, mo);
    hz = mn == -INFINITY ? 0.f : hz * expf(hm - mn) + zo * expf(mo - mn);
    hm = mn;
  }
  if (cq == 0 && gq < SP_MAXG) {
    hs[warp][gq][0] = hm;
    hs[warp][gq][1] = hz;
  }
  __syncthreads();
  if (threadIdx.x < p.G) {
    float m = -INFINITY;
    for (int w = 0; w < SP_SC_THREADS / 32; ++w) m = fmaxf(m, hs[w][threadIdx.x][0]);
    float z = 0.f;
    for (int w = 0; w < SP_SC_THREADS / 32; ++w)
      if (hs[w][threadIdx.x][0] > -INFINITY) z += hs[w][threadIdx.x][1] * expf(hs[w][threadIdx.x][0] - m);
    float* hp = p.hstat + (((int64_t)row * gridDim.x + blockIdx.x) * SP_MAXG + threadIdx.x) * 2;
    hp[0] = m;
    hp[1] = z;
  }
}

// ---------------------------------------------------------------------------
// sigma, the active set and the attention of one row in one CTA (after the score kernel).
// The row's sigma keys (order-preserving images of sigma) sit in shared memory; a radix
// select (three passes of 11, 11 and 10 bits) finds the K_t-th largest key T and how many
// keys equal to T to take (the lowest positions first, as kvc_select); an ordered block
// compaction writes the active positions, ascending, over the keys they came from (each
// chunk's keys are read before any of its writes, and a write never passes the chunk it
// came from); then the attention over the active set.
constexpr int SPR_THREADS = 128;
constexpr int SPR_WARPS = SPR_THREADS / 32;
constexpr int SPR_BINS = 2048;
constexpr int SPR_ITEMS = 8;                   // keys per thread per compaction chunk
constexpr int SPR_SU = 4;                      // sigma keys per thread with their loads in flight

// The two bf16 of a 32-bit word as an fp32 pair (low half first), exact.
__device__ __forceinline__ uint64_t bf2pair(uint32_t w) {
  uint64_t r;
  asm("{\n .reg .b32 lo, hi;\n shl.b32 lo, %1, 16;\n and.b32 hi, %1, 0xffff0000;\n mov.b64 %0, {lo, hi};\n}"
      : "=l"(r)
      : "r"(w));
  return r;
}

__device__ __forceinline__ int spr_excl_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < SPR_WARPS; ++w) {
    const int x = wsum[w];
    before += w < warp ? x : 0;
    all += x;
  }
  *total = all;
  return before + incl - v;
}

template <int G>
__global__ void __launch_bounds__(SPR_THREADS, 7) sparse_row_kernel(SparseParams p) {
  extern __shared__ uint32_t keys[];              // [max_len]: sigma keys, then the active list
  // the selection's histogram and the warps' partial outputs are never live together
  __shared__ __align__(16) union {
    uint32_t hist[SPR_BINS];
    float part[SPR_WARPS][G][SP_D];                // one partial o per warp (first the warp's staged probabilities)
  } u;
  uint32_t* hist = u.hist;
  auto& part = u.part;
  __shared__ float mh[G], zh[G], ma[G], la[G];
  __shared__ float red[2][SPR_WARPS * G];
  __shared__ int wsum[SPR_WARPS];
  __shared__ uint32_t sh_digit, sh_above;
  const int row = blockIdx.x, bl = row / p.Hkv, g = row % p.Hkv;
  const int b = bl / p.L, l = bl % p.L;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = min(p.len[bl], p.max_len);
  int kt = (int)ceil(p.kappa * (double)n - 1e-12);
  kt = min(n, max(1, kt));
  const float* srow = p.s + (int64_t)row * G * p.max_len;
  const int64_t so = (int64_t)row * p.side_row;
  // ---- head statistics over the row from the score blocks' partials, chunk order
  for (int h = warp; h < G; h += SPR_WARPS) {
    const int nch = (n + SP_SC_KEYS - 1) / SP_SC_KEYS, stride = (p.max_len + SP_SC_KEYS - 1) / SP_SC_KEYS;
    const float* hp = p.hstat + ((int64_t)row * stride * SP_MAXG + h) * 2;
    float m = -INFINITY;
    for (int c = lane; c < nch; c += 32) m = fmaxf(m, hp[(int64_t)c * SP_MAXG * 2]);
    m = warp_max(m);
    float z = 0.f;
    for (int c = lane; c < nch; c += 32) {
      const float mc = hp[(int64_t)c * SP_MAXG * 2];
      if (mc > -INFINITY) z += hp[(int64_t)c * SP_MAXG * 2 + 1] * expf(mc - m);
    }
    z = warp_sum(z);
    if (lane == 0) {
      mh[h] = m;
      zh[h] = 1.f / z;
      if (p.lse)   // over every cached key, as the dense decode step's
        p.lse[((int64_t)bl * p.Hq + g * G + h) * p.lse_stride] = z > 0.f ? m + logf(z) : -INFINITY;
    }
  }
  __syncthreads();
  // ---- sigma keys: SPR_SU keys per thread, every load issued before the first use
  for (int i0 = threadIdx.x; i0 < n; i0 += SPR_THREADS * SPR_SU) {
    float sv[SPR_SU][G], av[SPR_SU];
    int pv[SPR_SU];
#pragma unroll
    for (int su = 0; su < SPR_SU; ++su) {
      const int i = i0 + su * SPR_THREADS;
      const bool ok = i < n;
#pragma unroll
      for (int h = 0; h < G; ++h) sv[su][h] = ok ? srow[(int64_t)h * p.max_len + i] : 0.f;
      pv[su] = ok ? p.pos[so + i] : 0;
      av[su] = ok ? p.acc[so + i] : 0.f;
    }
#pragma unroll
    for (int su = 0; su < SPR_SU; ++su) {
      const int i = i0 + su * SPR_THREADS;
      if (i >= n) break;
      float tr = 0.f;
#pragma unroll
      for (int h = 0; h < G; ++h) tr += expf(sv[su][h] - mh[h]) * zh[h];
      const int cnt = p.t_cur - max(pv[su], p.n_prompt);
      const float hi = cnt > 0 ? av[su] / (float)cnt : 0.f;
      keys[i] = f2key(p.a_tr * (tr / (float)G) + p.b_hi * hi);
    }
  }
  __syncthreads();
  // ---- the kt-th largest key T and the number of keys equal to T to take
  uint32_t T = 0;
  int need_eq = 0;
  const bool take_all = kt >= n;
  if (!take_all) {
    uint32_t prefix = 0, mask = 0, krem = (uint32_t)kt;
    for (int ps = 0; ps < 3; ++ps) {
      const int shift = ps == 0 ? 21 : ps == 1 ? 10 : 0;
      const uint32_t dmask = ps == 2 ? 0x3ffu : 0x7ffu;
      for (int bn = threadIdx.x; bn < SPR_BINS; bn += SPR_THREADS) hist[bn] = 0u;
      __syncthreads();
      for (int i = threadIdx.x; i < n; i += SPR_THREADS) {
        const uint32_t kk = keys[i];
        if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & dmask], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        // lane j owns bins 2047-64j .. 1984-64j, scanned from the top; the sum starts at a
        // lane-dependent offset so the lanes hit different banks
        uint32_t sm = 0;
        for (int t = 0; t < 64; ++t) sm += hist[SPR_BINS - 1 - 64 * lane - ((t + lane) & 63)];
        uint32_t incl = sm;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(FULL, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - sm;
        if (excl < krem && krem <= incl) {
          uint32_t run = excl;
          for (int t = 0; t < 64; ++t) {
            const uint32_t c = hist[SPR_BINS - 1 - 64 * lane - t];
            if (run + c >= krem) {
              sh_digit = (uint32_t)(SPR_BINS - 1 - 64 * lane - t);
              sh_above = run;
              break;
            }
            run += c;
          }
        }
      }
      __syncthreads();
      krem -= sh_above;
      prefix |= sh_digit << shift;
      mask |= dmask << shift;
      __syncthreads();
    }
    T = prefix;
    need_eq = (int)krem;
  }
  // ---- ordered compaction of the active positions over the keys
  int out_base = 0, eq_base = 0;
  for (int c0 = 0; c0 < n; c0 += SPR_THREADS * SPR_ITEMS) {
    const int i0 = c0 + threadIdx.x * SPR_ITEMS;
    uint32_t kv[SPR_ITEMS];
    int neq = 0;
#pragma unroll
    for (int t = 0; t < SPR_ITEMS; ++t) {
      const int i = i0 + t;
      kv[t] = i < n ? keys[i] : 0u;
      neq += (!take_all && i < n && kv[t] == T) ? 1 : 0;
    }
    int eq_tot;
    int eq_rank = eq_base + spr_excl_scan(neq, wsum, &eq_tot);
    bool keep[SPR_ITEMS];
    int nkeep = 0;
#pragma unroll
    for (int t = 0; t < SPR_ITEMS; ++t) {
      const int i = i0 + t;
      bool kp = false;
      if (i < n) {
        if (take_all || kv[t] > T) {
          kp = true;
        } else if (kv[t] == T) {
          kp = eq_rank < need_eq;
          ++eq_rank;
        }
      }
      keep[t] = kp;
      nkeep += kp ? 1 : 0;
    }
    int keep_tot;
    int pos = out_base + spr_excl_scan(nkeep, wsum, &keep_tot);
    __syncthreads();                               // the chunk's keys are all read
#pragma unroll
    for (int t = 0; t < SPR_ITEMS; ++t)
      if (keep[t]) keys[pos++] = (uint32_t)(i0 + t);
    out_base += keep_tot;
    eq_base += eq_tot;
    __syncthreads();
  }
  const int kl = min(out_base, kt);                // == kt
  const int* act = reinterpret_cast<const int*>(keys);
  if (p.active)
    for (int j = threadIdx.x; j < kl; j += SPR_THREADS) p.active[(int64_t)row * p.max_len + j] = act[j];
  if (p.n_active && threadIdx.x == 0) p.n_active[row] = kl;
  if (g == 0 && threadIdx.x == 0) p.kt[bl] = kt;
  // ---- attention over the active set: per head max and sum of exp(s - max)
  float m[G], z[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    z[h] = 0.f;
  }
  for (int j = threadIdx.x; j < kl; j += SPR_THREADS) {
    const int i = act[j];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float x = srow[(int64_t)h * p.max_len + i];
      const float mn = fmaxf(m[h], x);
      z[h] = z[h] * expf(m[h] - mn) + expf(x - mn);
      m[h] = mn;
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float mo = __shfl_xor_sync(FULL, m[h], o), zo = __shfl_xor_sync(FULL, z[h], o);
      const float mn = fmaxf(m[h], mo);
      z[h] = (mn == -INFINITY) ? 0.f : z[h] * expf(m[h] - mn) + zo * expf(mo - mn);
      m[h] = mn;
    }
  }
  if (lane == 0)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      red[0][warp * G + h] = m[h];
      red[1][warp * G + h] = z[h];
    }
  __syncthreads();
  if (threadIdx.x < G) {
    float mm = -INFINITY;
    for (int w = 0; w < SPR_WARPS; ++w) mm = fmaxf(mm, red[0][w * G + threadIdx.x]);
    float zz = 0.f;
    for (int w = 0; w < SPR_WARPS; ++w) {
      const float mw = red[0][w * G + threadIdx.x];
      if (mw > -INFINITY) zz += red[1][w * G + threadIdx.x] * expf(mw - mm);
    }
    ma[threadIdx.x] = mm;
    la[threadIdx.x] = 1.f / zz;
  }
  __syncthreads();
  // o = sum over the active rows of p v: warps take 32-row chunks; lane j forms row j's
  // probabilities and history update and leaves them in shared memory as duplicated pairs
  // (p_h, p_h), then the warp streams the 32 value rows: a broadcast 16-byte load gives two
  // heads' pairs, each multiplied into a lane's two pairs of value dimensions by packed FMAs
  constexpr int GP = (G + 1) / 2;
  float4* stg = reinterpret_cast<float4*>(&part[warp][0][0]);   // [32][GP]; part[warp] after the loop
  const char* Vb = p.V + b * p.Vsb + l * p.Vsl + g * p.Vsh + lane * 8;
  const float invG = 1.f / (float)G;
  uint64_t acc[G][2];                              // dimensions (4 lane, 4 lane + 1), (4 lane + 2, 4 lane + 3)
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h][0] = acc[h][1] = pk2(0.f, 0.f);
  for (int c0 = warp * 32; c0 < kl; c0 += SPR_THREADS) {
    const int j = c0 + lane;
    const bool has = j < kl;
    const int i = has ? act[j] : 0;
    float pr[G];
    float pm = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      pr[h] = has ? expf(srow[(int64_t)h * p.max_len + i] - ma[h]) * la[h] : 0.f;
      pm += pr[h];
    }
    if (has) p.acc[so + i] += pm * invG;            // each active row belongs to one lane
    __syncwarp();                                   // the previous chunk's pairs are consumed
#pragma unroll
    for (int hp = 0; hp < GP; ++hp) {
      const float a = pr[2 * hp], c = 2 * hp + 1 < G ? pr[2 * hp + 1] : 0.f;
      stg[lane * GP + hp] = make_float4(a, a, c, c);
    }
    __syncwarp();
    const int nr = min(32, kl - c0);
#pragma unroll 1
    for (int r0 = 0; r0 < nr; r0 += 8) {
      uint2 vv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int iu = __shfl_sync(FULL, i, r0 + u);
        vv[u] = r0 + u < nr ? __ldg(reinterpret_cast<const uint2*>(Vb + (int64_t)iu * p.Vst)) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint64_t v01 = bf2pair(vv[u].x), v23 = bf2pair(vv[u].y);
        const float4* q = stg + (r0 + u) * GP;
#pragma unroll
        for (int hp = 0; hp < GP; ++hp) {
          const float4 pp = q[hp];
          const uint64_t pa = pk2(pp.x, pp.y);
          acc[2 * hp][0] = fma2(pa, v01, acc[2 * hp][0]);
          acc[2 * hp][1] = fma2(pa, v23, acc[2 * hp][1]);
          if (2 * hp + 1 < G) {
            const uint64_t pb = pk2(pp.z, pp.w);
            acc[2 * hp + 1][0] = fma2(pb, v01, acc[2 * hp + 1][0]);
            acc[2 * hp + 1][1] = fma2(pb, v23, acc[2 * hp + 1][1]);
          }
        }
      }
    }
  }
  __syncwarp();                                     // the staged pairs are consumed before part[warp] is written
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float2 lo = upk2(acc[h][0]), hi = upk2(acc[h][1]);
    *reinterpret_cast<float4*>(&part[warp][h][lane * 4]) = make_float4(lo.x, lo.y, hi.x, hi.y);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * SP_D; e += SPR_THREADS) {
    const int h = e / SP_D, c = e % SP_D;
    float sum = 0.f;
    for (int w = 0; w < SPR_WARPS; ++w) sum += part[w][h][c];
    p.o[(((int64_t)bl * p.Hq) + g * G + h) * SP_D + c] = sum;
  }
}

template <int G>
static cudaError_t launch_sparse_row(const SparseParams& p, int rows, cudaStream_t st) {
  const size_t smem = (size_t)p.max_len * sizeof(uint32_t);
  auto kern = sparse_row_kernel<G>;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e) return e;
  }
  kern<<<rows, SPR_THREADS, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_sparse_decode(const SparseParams& p, cudaStream_t st) {
  const int rows = p.B * p.L * p.Hkv;
  const dim3 g1((p.max_len + SP_SC_KEYS - 1) / SP_SC_KEYS, rows);
  sparse_scores_kernel<<<g1, SP_SC_THREADS, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e) return e;
  count_launch();
  switch (p.G) {
    case 1: e = launch_sparse_row<1>(p, rows, st); break;
    case 2: e = launch_sparse_row<2>(p, rows, st); break;
    case 3: e = launch_sparse_row<3>(p, rows, st); break;
    case 4: e = launch_sparse_row<4>(p, rows, st); break;
    case 5: e = launch_sparse_row<5>(p, rows, st); break;
    case 6: e = launch_sparse_row<6>(p, rows, st); break;
    case 7: e = launch_sparse_row<7>(p, rows, st); break;
    default: e = launch_sparse_row<8>(p, rows, st); break;
  }
  if (e) return e;
  count_launch();
  return cudaSuccess;
}

}  // namespace kvc
