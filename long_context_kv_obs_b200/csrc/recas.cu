// RECAS calibrated dropped-mass estimator and adaptive budget controller.
//
// [RECAS] 2.B: after eviction the exact full-cache attention is gone, so the dropped
// attention mass is estimated from a normalised predictor and recalibrated at periodic
// full-attention probe steps, with a conservative upper estimate from the empirical
// (1 - alpha)-quantile of the residuals; when that upper estimate threatens the error
// target eps, the controller grows the cache budget, keeping tokens in utility order,
// until the bound holds.
//
// The readings these kernels implement:
//   predictor  x = share of the compression's window attention A on the dropped tokens,
//              x = 1 - sum_kept A / sum_all A, per (sequence, layer, KV head) row;
//   calibrate  per (sequence, layer), at a probe step: residuals r_h = delta_h - c x_{h/G}
//              with the ratio c = sum delta / sum x of the earlier probes (1 before any),
//              kept in a ring of the last KVC_RECAS_RING; then c is updated and q is the
//              ceil((m + 1)(1 - alpha))-th smallest of the m ring residuals (+inf if that
//              rank exceeds m);
//   control    a row needs the smallest k >= k0 whose kept set (recent window plus the
//              top k - w by utility S, ties to the lower position) leaves x(k) with
//              c x(k) + q <= eps, the whole row if none; the budget is the largest need.
//
// recas_calibrate_kernel: one CTA per (sequence, layer); the quantile is an order
// statistic found by rank counting over the ring (fp64, deterministic).
// recas_control_kernel: one CTA per row; the row's candidates are sorted by (utility
// descending, position ascending) with a bitonic sort of 64-bit keys in shared memory,
// the attention of that order is prefix-summed in fp64, and the first budget meeting the
// bound is found with a block-wide minimum.  recas_budget_kernel: the largest need,
// broadcast as the budget of every (sequence, layer).  recas_predictor_kernel: x of the
// kept sets a selection produced.
#include <cfloat>
#include <cstddef>

#include "kernels.cuh"

namespace kvc {

static_assert(sizeof(kvc_recas_cal) == 8 * (5 + KVC_RECAS_RING), "kvc_recas_cal layout: 5 words + ring");
static_assert(offsetof(kvc_recas_cal, count) == 32 && offsetof(kvc_recas_cal, ring) == 40,
              "kvc_recas_cal layout");

constexpr int RC_THREADS = 1024;
constexpr int CAL_THREADS = KVC_RECAS_RING;

__device__ __forceinline__ double cal_c(const kvc_recas_cal& s) {
  return s.sum_x > 0.0 ? s.sum_delta / s.sum_x : 1.0;
}
__device__ __forceinline__ double cal_q(const kvc_recas_cal& s) {
  return s.count > 0 ? s.q : (double)INFINITY;
}

// Rank of the split-conformal quantile among m residuals (1-based; > m means +inf).  The
// product is taken 1e-12 low so that an integer product (e.g. 10 * 0.9) is not pushed up
// by the binary rounding of 1 - alpha.
__device__ __forceinline__ int conformal_rank(int m, double alpha) {
  int r = (int)ceil((double)(m + 1) * (1.0 - alpha) - 1e-12);
  return r < 1 ? 1 : r;
}

__global__ void __launch_bounds__(CAL_THREADS) recas_calibrate_kernel(RecasCalParams p) {
  __shared__ double ring[KVC_RECAS_RING];
  __shared__ double sh_q;
  const int bl = blockIdx.x, t = threadIdx.x;
  kvc_recas_cal& st = p.state[bl];
  const float* delta = p.delta + (int64_t)bl * p.Hq;
  const float* x = p.x + (int64_t)bl * p.Hkv;
  const double c_old = cal_c(st);
  const int head = st.head;
  __syncthreads();                                   // every thread read the old state
  for (int h = t; h < p.Hq; h += CAL_THREADS)
    st.ring[(head + h) % KVC_RECAS_RING] = (double)delta[h] - c_old * (double)x[h / p.G];
  __syncthreads();
  if (t == 0) {
    double sd = 0.0, sx = 0.0;
    for (int h = 0; h < p.Hq; ++h) {                 // fixed order
      sd += (double)delta[h];
      sx += (double)x[h / p.G];
    }
    st.sum_delta += sd;
    st.sum_x += sx;
    st.count += p.Hq;
    st.head = (head + p.Hq) % KVC_RECAS_RING;
    sh_q = INFINITY;
  }
  __syncthreads();
  const int m = min(st.count, KVC_RECAS_RING);
  const int rank = conformal_rank(m, p.alpha);
  for (int i = t; i < m; i += CAL_THREADS) ring[i] = st.ring[i];
  __syncthreads();
  if (rank <= m) {
    for (int i = t; i < m; i += CAL_THREADS) {
      const double ri = ring[i];
      int below = 0;
      for (int j = 0; j < m; ++j) {
        const double rj = ring[j];
        below += (rj < ri) || (rj == ri && j < i);
      }
      if (below == rank - 1) sh_q = ri;              // exactly one thread
    }
  }
  __syncthreads();
  if (t == 0) {
    st.q = sh_q;
    st.c = cal_c(st);
  }
  __syncthreads();
  const double c = cal_c(st), q = sh_q;
  for (int g = t; g < p.Hkv; g += CAL_THREADS) {
    const double xg = (double)x[g];
    if (p.delta_hat) p.delta_hat[(int64_t)bl * p.Hkv + g] = (float)(c * xg);
    if (p.delta_bar) p.delta_bar[(int64_t)bl * p.Hkv + g] = (float)(c * xg + q);
  }
}

cudaError_t launch_recas_calibrate(const RecasCalParams& p, cudaStream_t st) {
  recas_calibrate_kernel<<<p.BL, CAL_THREADS, 0, st>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

// Block-wide reductions of the control kernel (RC_THREADS threads, fixed order).
__device__ __forceinline__ double block_sum_d(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_d(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double s = 0.0;
  if (warp == 0) {
    s = lane < RC_THREADS / 32 ? red[lane] : 0.0;
    s = warp_sum_d(s);
    if (lane == 0) red[0] = s;
  }
  __syncthreads();
  return red[0];
}

__global__ void __launch_bounds__(RC_THREADS) recas_control_kernel(RecasCtlParams p) {
  extern __shared__ uint64_t rc_keys[];                 // [np2]
  __shared__ double red[RC_THREADS / 32];
  __shared__ double seg_base[RC_THREADS];
  __shared__ int sh_first;
  const int row = blockIdx.x, t = threadIdx.x;
  const int bl = row / p.Hkv;
  const int n = p.n, w = min(p.w, n), nc = n - w;
  const float* A = p.A + (int64_t)row * p.s_row;
  const float* S = p.S + (int64_t)row * p.s_row;
  const float* S0 = p.S + (int64_t)bl * p.Hkv * p.s_row;   // the layer's first head (union)
  // candidates: positions below n - w, ordered by utility descending, position ascending
  for (int i = t; i < p.np2; i += RC_THREADS) {
    uint64_t k = ~0ull;
    if (i < nc) {
      float s = S[i];
      if (p.union_mode) {
        s = S0[i];
        for (int g = 1; g < p.Hkv; ++g) s = fmaxf(s, S0[(int64_t)g * p.s_row + i]);
      }
      k = ((uint64_t)(~f2key(s)) << 32) | (uint32_t)i;
    }
    rc_keys[i] = k;
  }
  __syncthreads();
  for (int kk = 2; kk <= p.np2; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = t; i < p.np2; i += RC_THREADS) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = rc_keys[i], b = rc_keys[ixj];
          const bool up = (i & kk) == 0;
          if ((a > b) == up) {
            rc_keys[i] = b;
            rc_keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // the row's attention mass and the recent window's share (fp64, fixed order)
  double tot = 0.0, win = 0.0;
  for (int i = t; i < n; i += RC_THREADS) {
    const double a = (double)A[i];
    tot += a;
    if (i >= nc) win += a;
  }
  tot = block_sum_d(tot, red);
  win = block_sum_d(win, red);
  const kvc_recas_cal& st = p.state[bl];
  const double c = cal_c(st), q = cal_q(st), eps = (double)p.eps;
  // thread t owns sorted entries [t*seg, (t+1)*seg): prefix of its segment's attention
  const int seg = (nc + RC_THREADS - 1) / RC_THREADS;
  const int s0 = min(nc, t * seg), s1 = min(nc, s0 + seg);
  double local = 0.0;
  for (int j = s0; j < s1; ++j) local += (double)A[(uint32_t)rc_keys[j]];
  seg_base[t] = local;
  if (t == 0) sh_first = nc + 1;
  __syncthreads();
  // exclusive prefix of the segment totals, one serial pass (fixed order)
  if (t == 0) {
    double run = 0.0;
    for (int u = 0; u < RC_THREADS; ++u) {
      const double v = seg_base[u];
      seg_base[u] = run;
      run += v;
    }
  }
  __syncthreads();
  // j re-admitted candidates keep mass win + P_j; the budget is w + j
  const int jmin = max(0, p.k0 - w);
  double P = seg_base[t];
  int first = nc + 1;
  for (int j = s0; j <= s1; ++j) {
    if (j >= jmin) {
      const double xj = tot > 0.0 ? 1.0 - (win + P) / tot : 0.0;
      if (c * xj + q <= eps) {
        first = j;
        break;
      }
    }
    if (j < s1) P += (double)A[(uint32_t)rc_keys[j]];
  }
  if (first <= nc) atomicMin(&sh_first, first);
  __syncthreads();
  if (t == 0) {
    const int need = sh_first <= nc ? w + sh_first : n;
    if (p.need) p.need[row] = need;
  }
}

cudaError_t launch_recas_control(const RecasCtlParams& p, cudaStream_t st) {
  const size_t smem = (size_t)p.np2 * sizeof(uint64_t);
  cudaError_t e = cudaFuncSetAttribute(recas_control_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  recas_control_kernel<<<p.rows, RC_THREADS, smem, st>>>(p);
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

// The largest need over `rows`, at most k_max, written to budget[0] and to every entry of
// k[0 .. nk) and k2[0 .. nk2).
__global__ void __launch_bounds__(256) recas_budget_kernel(const int32_t* need, int rows, int k_max, int32_t* budget,
                                                           int32_t* k, int nk, int32_t* k2, int nk2) {
  __shared__ int sh;
  if (threadIdx.x == 0) sh = 0;
  __syncthreads();
  int mx = 0;
  for (int r = threadIdx.x; r < rows; r += blockDim.x) mx = max(mx, need[r]);
  atomicMax(&sh, mx);
  __syncthreads();
  const int b = min(sh, k_max);
  if (threadIdx.x == 0 && budget) budget[0] = b;
  for (int i = threadIdx.x; i < nk; i += blockDim.x) k[i] = b;
  for (int i = threadIdx.x; i < nk2; i += blockDim.x) k2[i] = b;
}

cudaError_t launch_recas_budget(const int32_t* need, int rows, int k_max, int32_t* budget, int32_t* k, int nk,
                                int32_t* k2, int nk2, cudaStream_t st) {
  recas_budget_kernel<<<1, 256, 0, st>>>(need, rows, k_max, budget, k, nk, k2, nk2);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

// x of row r: 1 - sum_{j < k} A[idx[j]] / sum_i A[i] (fp64, fixed order).
__global__ void __launch_bounds__(256) recas_predictor_kernel(const float* A, int64_t s_row, int n,
                                                              const int32_t* idx, int k_cap, const int32_t* k,
                                                              int Hkv, float* x) {
  __shared__ double red[2][8];
  const int r = blockIdx.x, lb = r / Hkv, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const float* Ar = A + (int64_t)r * s_row;
  const int32_t* id = idx + (int64_t)r * k_cap;
  const int kl = min(k[lb], k_cap);
  double tot = 0.0, kept = 0.0;
  for (int i = t; i < n; i += 256) tot += (double)Ar[i];
  for (int j = t; j < kl; j += 256) {
    const int i = id[j];
    if (i >= 0 && i < n) kept += (double)Ar[i];
  }
  tot = warp_sum_d(tot);
  kept = warp_sum_d(kept);
  if (lane == 0) {
    red[0][warp] = tot;
    red[1][warp] = kept;
  }
  __syncthreads();
  if (t == 0) {
    double a = 0.0, b = 0.0;
    for (int u = 0; u < 8; ++u) {
      a += red[0][u];
      b += red[1][u];
    }
    x[r] = a > 0.0 ? (float)(1.0 - b / a) : 0.f;
  }
}

cudaError_t launch_recas_predictor(const float* A, int64_t s_row, int n, const int32_t* idx, int k_cap,
                                   const int32_t* k, int rows, int Hkv, float* x, cudaStream_t st) {
  recas_predictor_kernel<<<rows, 256, 0, st>>>(A, s_row, n, idx, k_cap, k, Hkv, x);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

}  // namespace kvc
