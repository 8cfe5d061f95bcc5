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
// as register fragments, the keys straight from global memory) and stores s = q k scale
// for the G heads; sparse_sigma_kernel forms
// the head softmax statistics and sigma (fp32, fixed-order reductions) and K_t; the
// selection kernel of kvc_select picks the active positions in ascending order;
// sparse_attend_kernel gathers the active value rows (half a warp per row, 16-byte loads),
// renormalises over the active set, writes o and updates acc.
#include "kernels.cuh"

namespace kvc {

constexpr int SP_D = 128;
constexpr int SP_SC_THREADS = 128;            // scores: 4 warps, 64 keys each per block
constexpr int SP_SC_KEYS = 256;
constexpr int SP_SIG_THREADS = 512;
constexpr int SP_AT_THREADS = 256;
constexpr int SP_MAXG = 8;

// s = scale * q k for the G heads and 8 keys per mma.sync m16n8k16 (bf16 in, fp32
// accumulate): A = the G queries padded to 16 rows (fragments kept in registers for the
// whole row), B = 8 key rows read straight from global memory (each thread two 4-byte
// pieces per 16-dim step, 32 contiguous bytes per key per step across the quad).
__device__ __forceinline__ void sp_mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(SP_SC_THREADS) sparse_scores_kernel(SparseParams p) {
  const int row = blockIdx.y, bl = row / p.Hkv, g = row % p.Hkv;
  const int b = bl / p.L, l = bl % p.L;
  const int n = min(p.len[bl], p.max_len);
  const int key0 = blockIdx.x * SP_SC_KEYS;
  if (key0 >= n) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, cq = lane & 3;          // mma fragment row / column pair
  // query fragments: row gq is head gq (rows >= G and 8..15 are zero), columns of the
  // 16-dim step ks: 2 cq, 2 cq + 1 and 2 cq + 8, 2 cq + 9
  uint32_t qa[8][2];
  const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
      reinterpret_cast<const __nv_bfloat16*>(p.q) + ((int64_t)bl * p.Hq + g * p.G + gq) * SP_D);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    qa[ks][0] = gq < p.G ? __ldg(qrow + ks * 8 + cq) : 0u;
    qa[ks][1] = gq < p.G ? __ldg(qrow + ks * 8 + cq + 4) : 0u;
  }
  const char* Kb = p.K + b * p.Ksb + l * p.Ksl + g * p.Ksh + cq * 4;
  float* srow = p.s + (int64_t)row * p.G * p.max_len;
  const int wkey0 = key0 + warp * (SP_SC_KEYS / (SP_SC_THREADS / 32));
#pragma unroll 1
  for (int t = 0; t < SP_SC_KEYS / (SP_SC_THREADS / 32); t += 16) {
    // two 8-key tiles in flight
    uint32_t kb[2][8][2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int key = wkey0 + t + u * 8 + gq;
      const char* kr = Kb + (int64_t)(key < n ? key : 0) * p.Kst;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        kb[u][ks][0] = __ldg(reinterpret_cast<const uint32_t*>(kr + ks * 32));
        kb[u][ks][1] = __ldg(reinterpret_cast<const uint32_t*>(kr + ks * 32 + 16));
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t a[4] = {qa[ks][0], 0u, qa[ks][1], 0u};
        sp_mma(c, a, kb[u][ks][0], kb[u][ks][1]);
      }
      // c[0], c[1]: head gq, keys 2 cq, 2 cq + 1 of the tile
      const int k2 = wkey0 + t + u * 8 + 2 * cq;
      if (gq < p.G) {
        float* dst = srow + (int64_t)gq * p.max_len + k2;
        if (k2 < n) dst[0] = c[0] * p.scale;
        if (k2 + 1 < n) dst[1] = c[1] * p.scale;
      }
    }
  }
}

// Max and sum over a block of one value per head and thread, all heads at once; fixed order.
template <int NT>
__device__ __forceinline__ void sp_block_reduce_heads(float (&v)[SP_MAXG], int G, bool is_max, float* red,
                                                      float* out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int h = 0; h < SP_MAXG; ++h) v[h] = is_max ? warp_max(v[h]) : warp_sum(v[h]);
  __syncthreads();
  if (lane == 0)
#pragma unroll
    for (int h = 0; h < SP_MAXG; ++h) red[warp * SP_MAXG + h] = v[h];
  __syncthreads();
  if (threadIdx.x < G) {
    float r = is_max ? -INFINITY : 0.f;
    for (int w = 0; w < NT / 32; ++w) {
      const float x = red[w * SP_MAXG + threadIdx.x];
      r = is_max ? fmaxf(r, x) : r + x;
    }
    out[threadIdx.x] = r;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(SP_SIG_THREADS) sparse_sigma_kernel(SparseParams p) {
  __shared__ float red[(SP_SIG_THREADS / 32) * SP_MAXG];
  __shared__ float mh[SP_MAXG], zh[SP_MAXG];
  const int row = blockIdx.x, bl = row / p.Hkv, g = row % p.Hkv;
  const int n = min(p.len[bl], p.max_len);
  const float* srow = p.s + (int64_t)row * p.G * p.max_len;
  float v[SP_MAXG];
#pragma unroll
  for (int h = 0; h < SP_MAXG; ++h) v[h] = -INFINITY;
  for (int i = threadIdx.x; i < n; i += SP_SIG_THREADS)
#pragma unroll
    for (int h = 0; h < SP_MAXG; ++h)
      if (h < p.G) v[h] = fmaxf(v[h], srow[(int64_t)h * p.max_len + i]);
  sp_block_reduce_heads<SP_SIG_THREADS>(v, p.G, true, red, mh);
#pragma unroll
  for (int h = 0; h < SP_MAXG; ++h) v[h] = 0.f;
  for (int i = threadIdx.x; i < n; i += SP_SIG_THREADS)
#pragma unroll
    for (int h = 0; h < SP_MAXG; ++h)
      if (h < p.G) v[h] += expf(srow[(int64_t)h * p.max_len + i] - mh[h]);
  sp_block_reduce_heads<SP_SIG_THREADS>(v, p.G, false, red, zh);
  const int64_t so = (int64_t)row * p.side_row;
  const float invG = 1.f / (float)p.G;
  float* sig = p.sigma + (int64_t)row * p.max_len;
  for (int i = threadIdx.x; i < p.max_len; i += SP_SIG_THREADS) {
    float val = -INFINITY;
    if (i < n) {
      float tr = 0.f;
      for (int h = 0; h < p.G; ++h) tr += expf(srow[(int64_t)h * p.max_len + i] - mh[h]) / zh[h];
      const int cnt = p.t_cur - max(p.pos[so + i], p.n_prompt);
      const float hi = cnt > 0 ? p.acc[so + i] / (float)cnt : 0.f;
      val = p.a_tr * (tr * invG) + p.b_hi * hi;
    }
    sig[i] = val;
  }
  if (g == 0 && threadIdx.x == 0) {
    int k = (int)ceil(p.kappa * (double)n - 1e-12);
    p.kt[bl] = min(n, max(1, k));
  }
}

// One CTA per row.  Pass A: softmax statistics of every head over the active set (online
// max and sum per thread, then a fixed-order block reduction).  Pass B: warps take 32-row
// chunks of the active list; lane j fetches row j's position and G scores and forms its G
// normalised probabilities (and the row's history update), then the warp streams the 32
// value rows, 8 loads in flight, each lane 4 dimensions, the probabilities broadcast by
// shuffle.  The warps' partial outputs are summed in a fixed order.
__global__ void __launch_bounds__(SP_AT_THREADS, 3) sparse_attend_kernel(SparseParams p) {
  __shared__ float red[2][(SP_AT_THREADS / 32) * SP_MAXG];
  __shared__ float mh[SP_MAXG], lh[SP_MAXG];
  __shared__ float part[SP_AT_THREADS / 32][SP_MAXG][SP_D];   // one partial o per warp
  const int row = blockIdx.x, bl = row / p.Hkv, g = row % p.Hkv;
  const int b = bl / p.L, l = bl % p.L;
  const int kl = p.kt[bl];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int32_t* act = p.active + (int64_t)row * p.max_len;
  const float* srow = p.s + (int64_t)row * p.G * p.max_len;
  // ---- pass A: per head, max m and sum l of exp(s - m) over the active rows
  float m[SP_MAXG], z[SP_MAXG];
#pragma unroll
  for (int h = 0; h < SP_MAXG; ++h) {
    m[h] = -INFINITY;
    z[h] = 0.f;
  }
  for (int j = threadIdx.x; j < kl; j += SP_AT_THREADS) {
    const int i = __ldg(act + j);
#pragma unroll
    for (int h = 0; h < SP_MAXG; ++h) {
      if (h < p.G) {
        const float x = srow[(int64_t)h * p.max_len + i];
        const float mn = fmaxf(m[h], x);
        z[h] = z[h] * expf(m[h] - mn) + expf(x - mn);
        m[h] = mn;
      }
    }
  }
#pragma unroll
  for (int h = 0; h < SP_MAXG; ++h) {
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
    for (int h = 0; h < SP_MAXG; ++h) {
      red[0][warp * SP_MAXG + h] = m[h];
      red[1][warp * SP_MAXG + h] = z[h];
    }
  __syncthreads();
  if (threadIdx.x < p.G) {
    float mm = -INFINITY;
    for (int w = 0; w < SP_AT_THREADS / 32; ++w) mm = fmaxf(mm, red[0][w * SP_MAXG + threadIdx.x]);
    float zz = 0.f;
    for (int w = 0; w < SP_AT_THREADS / 32; ++w) {
      const float mw = red[0][w * SP_MAXG + threadIdx.x];
      if (mw > -INFINITY) zz += red[1][w * SP_MAXG + threadIdx.x] * expf(mw - mm);
    }
    mh[threadIdx.x] = mm;
    lh[threadIdx.x] = 1.f / zz;
  }
  __syncthreads();
  // ---- pass B
  const char* Vb = p.V + b * p.Vsb + l * p.Vsl + g * p.Vsh + lane * 8;
  const int64_t so = (int64_t)row * p.side_row;
  const float invG = 1.f / (float)p.G;
  float acc[SP_MAXG][4];
#pragma unroll
  for (int h = 0; h < SP_MAXG; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
  for (int c0 = warp * 32; c0 < kl; c0 += SP_AT_THREADS) {
    const int j = c0 + lane;
    const bool has = j < kl;
    const int i = has ? __ldg(act + j) : 0;
    float pr[SP_MAXG];
    float pm = 0.f;
#pragma unroll
    for (int h = 0; h < SP_MAXG; ++h) {
      pr[h] = (has && h < p.G) ? expf(srow[(int64_t)h * p.max_len + i] - mh[h]) * lh[h] : 0.f;
      pm += pr[h];
    }
    if (has) p.acc[so + i] += pm * invG;            // each active row belongs to one lane
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
        const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv[u].x));
        const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vv[u].y));
#pragma unroll
        for (int h = 0; h < SP_MAXG; ++h) {
          const float ph = __shfl_sync(FULL, pr[h], r0 + u);
          acc[h][0] = fmaf(ph, v01.x, acc[h][0]);
          acc[h][1] = fmaf(ph, v01.y, acc[h][1]);
          acc[h][2] = fmaf(ph, v23.x, acc[h][2]);
          acc[h][3] = fmaf(ph, v23.y, acc[h][3]);
        }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < SP_MAXG; ++h)
#pragma unroll
    for (int e = 0; e < 4; ++e) part[warp][h][lane * 4 + e] = acc[h][e];
  __syncthreads();
  for (int e = threadIdx.x; e < p.G * SP_D; e += SP_AT_THREADS) {
    const int h = e / SP_D, c = e % SP_D;
    float sum = 0.f;
    for (int w = 0; w < SP_AT_THREADS / 32; ++w) sum += part[w][h][c];
    p.o[(((int64_t)bl * p.Hq) + g * p.G + h) * SP_D + c] = sum;
  }
  if (p.n_active && threadIdx.x == 0) p.n_active[row] = kl;
}

cudaError_t launch_sparse_decode(const SparseParams& p, cudaStream_t st) {
  const int rows = p.B * p.L * p.Hkv;
  const dim3 g1((p.max_len + SP_SC_KEYS - 1) / SP_SC_KEYS, rows);
  sparse_scores_kernel<<<g1, SP_SC_THREADS, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e) return e;
  count_launch();
  sparse_sigma_kernel<<<rows, SP_SIG_THREADS, 0, st>>>(p);
  if ((e = cudaGetLastError())) return e;
  count_launch();
  e = launch_select(p.sigma, (int64_t)p.Hkv * p.max_len, p.max_len, p.B * p.L, p.Hkv, p.max_len, 0, 0, p.kt,
                    p.active, p.max_len, nullptr, st, p.len);
  if (e) return e;
  sparse_attend_kernel<<<rows, SP_AT_THREADS, 0, st>>>(p);
  if ((e = cudaGetLastError())) return e;
  count_launch();
  return cudaSuccess;
}

}  // namespace kvc
