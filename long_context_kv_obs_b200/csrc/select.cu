// Per-layer budgets and top-k selection of kept positions.
//
// [InfoKV] Technical details: keep the top k_l tokens of every layer, uniform
// budgets by default or adaptive k_l = (E-bar^(l) / sum_m E-bar^(m)) * B
// (Methodology, Glossary "Adaptive budget allocation").
// [SelKV] Pipeline overview step 2: top tokens per KV head, or through the
// GQA union, together with a recent window.
//
// budget_kernel: one thread, fp64, clamped proportional share (the scale
// lambda with sum_l clamp(lambda * E-bar_l, w, n) = B, found from the
// breakpoints of that piecewise-linear sum) then largest remainder.
// keys_kernel: scores -> order-preserving uint32 keys (max over KV heads for
// the union).  select_kernel: one CTA per row, four 8-bit radix passes from
// the top with warp-aggregated shared-memory histograms find the k-th key and
// how many of its equal keys to take (lowest positions first), then an
// ordered block-wide stream compaction writes the ascending index list.
#include "kernels.cuh"

namespace kvc {

__global__ void budget_kernel(int mode, int L, int n, int w, double rho, const int32_t* k_in,
                              long long B, const float* Ebar, int32_t* k_out) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const int lo = w < n ? w : n, hi = n;
  if (mode == KVC_BUDGET_UNIFORM) {
    long long k = (long long)floor(rho * (double)n);
    if (k < lo) k = lo;
    if (k > hi) k = hi;
    for (int l = 0; l < L; ++l) k_out[l] = (int32_t)k;
    return;
  }
  if (mode == KVC_BUDGET_EXPLICIT) {
    for (int l = 0; l < L; ++l) {
      int k = k_in[l];
      k_out[l] = k < lo ? lo : (k > hi ? hi : k);
    }
    return;
  }
  // adaptive
  bool any = false;
  for (int l = 0; l < L; ++l) any |= Ebar[l] > 0.f;
  auto E = [&](int l) -> double { return any ? (double)Ebar[l] : 1.0; };
  auto f = [&](double lam) -> double {
    double s = 0.0;
    for (int l = 0; l < L; ++l) {
      double x = lam * E(l);
      s += x < lo ? (double)lo : (x > hi ? (double)hi : x);
    }
    return s;
  };
  const double Bd = (double)B;
  double b0 = 0.0;
  // candidate breakpoints: 0, lo / E_l, hi / E_l
  for (int c = 0; c < 2 * L; ++c) {
    const int l = c % L;
    const double e = E(l);
    if (!(e > 0.0)) continue;
    const double b = (c < L ? (double)lo : (double)hi) / e;
    if (b > b0 && f(b) <= Bd) b0 = b;
  }
  double above = INFINITY;
  for (int c = 0; c < 2 * L; ++c) {
    const int l = c % L;
    const double e = E(l);
    if (!(e > 0.0)) continue;
    const double b = (c < L ? (double)lo : (double)hi) / e;
    if (b > b0 && b < above) above = b;
  }
  const double mid = above < INFINITY ? 0.5 * (b0 + above) : 2.0 * b0 + 1.0;
  double slope = 0.0;
  for (int l = 0; l < L; ++l) {
    const double x = mid * E(l);
    if (x > lo && x < hi) slope += E(l);
  }
  const double lam = slope == 0.0 ? b0 : b0 + (Bd - f(b0)) / slope;
  long long sum = 0;
  for (int l = 0; l < L; ++l) {
    double x = lam * E(l);
    x = x < lo ? (double)lo : (x > hi ? (double)hi : x);
    k_out[l] = (int32_t)floor(x);
    sum += k_out[l];
  }
  long long extra = B - sum;
  // one extra token to the layers with the largest fractional parts, ties to
  // the lower layer, never past n; a layer already raised has k != floor(x)
  for (long long e = 0; e < extra; ++e) {
    int best = -1;
    double bf = -1.0;
    for (int l = 0; l < L; ++l) {
      if (k_out[l] >= hi) continue;
      double x = lam * E(l);
      x = x < lo ? (double)lo : (x > hi ? (double)hi : x);
      const double fl = floor(x);
      if ((double)k_out[l] != fl) continue;
      const double fr = x - fl;
      if (fr > bf) { bf = fr; best = l; }
    }
    if (best < 0) break;
    k_out[best] += 1;
  }
}

__global__ void keys_kernel(const float* __restrict__ S, int64_t Ssl, int64_t Ssh, int L, int Hkv,
                            int n, int union_mode, uint32_t* __restrict__ keys) {
  const int rows = union_mode ? L : L * Hkv;
  const int64_t total = (int64_t)rows * n;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int row = (int)(t / n), i = (int)(t % n);
    float s;
    if (union_mode) {
      s = -INFINITY;
      for (int g = 0; g < Hkv; ++g) s = fmaxf(s, S[row * Ssl + g * Ssh + i]);
    } else {
      s = S[(row / Hkv) * Ssl + (row % Hkv) * Ssh + i];
    }
    keys[t] = f2key(s);
  }
}

constexpr int SEL_THREADS = 512;
constexpr int SEL_ITEMS = 4;
constexpr int SEL_BITS = 11;                 // digit width: passes on bits 31-21, 20-10, 9-0
constexpr int SEL_BINS = 1 << SEL_BITS;

// Block-wide exclusive scan of one int per thread; returns the block total in *total.
__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int x = lane < (SEL_THREADS / 32) ? wsum[lane] : 0;
    int xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(FULL, xi, o);
      if (lane >= o) xi += y;
    }
    wsum[lane] = xi - x;
    if (lane == 31) wsum[32] = xi;
  }
  __syncthreads();
  *total = wsum[32];
  return wsum[warp] + incl - v;
}

// Key of element i of the row: the order-preserving image of S (per KV head) or
// the precomputed max-over-heads key (GQA union).
struct RowKeys {
  const float* S;        // per-head mode
  const uint32_t* keys;  // union mode
  __device__ __forceinline__ uint32_t operator[](int i) const {
    return keys ? keys[i] : f2key(S[i]);
  }
};

__global__ void __launch_bounds__(SEL_THREADS, 2)
select_kernel(const float* __restrict__ S, int64_t Ssl, int64_t Ssh, const uint32_t* __restrict__ keys,
              int n, int w, const int32_t* __restrict__ k_l, int Hkv, int union_mode,
              int32_t* __restrict__ idx, int k_cap, unsigned* status, const int32_t* __restrict__ n_l) {
  __shared__ uint32_t hist[SEL_BINS];
  __shared__ int wsum[33];
  __shared__ uint32_t sh_digit, sh_above;
  const int row = blockIdx.x;
  const int l = union_mode ? row : row / Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nstride = n;                      // keys rows keep the full stride
  if (n_l) n = min(n, max(n_l[l], 0));        // rows of their own length
  RowKeys key;
  key.S = union_mode ? nullptr : S + (int64_t)l * Ssl + (int64_t)(row % Hkv) * Ssh;
  key.keys = union_mode ? keys + (int64_t)row * nstride : nullptr;
  const int w_ = w < n ? w : n;
  const int ncand = n - w_;
  int k = k_l[l];
  if (k > k_cap) {
    if (threadIdx.x == 0) flag(status, ST_BOUNDS);
    k = k_cap;
  }
  int m = k - w_;
  if (m < 0) m = 0;
  // threshold key T and the number of keys equal to T to take (lowest positions first)
  uint32_t T = 0;
  int need_eq = 0;
  const bool take_all = m >= ncand, take_none = m == 0;
  if (!take_all && !take_none) {
    uint32_t prefix = 0, mask = 0, krem = (uint32_t)m;
    for (int p = 0; p < 3; ++p) {
      const int shift = p == 0 ? 21 : p == 1 ? 10 : 0;
      const uint32_t dmask = p == 2 ? 0x3ffu : 0x7ffu;
      for (int b = threadIdx.x; b < SEL_BINS; b += SEL_THREADS) hist[b] = 0u;
      __syncthreads();
      for (int i = threadIdx.x; i < ncand; i += SEL_THREADS) {
        const uint32_t kk = key[i];
        if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & dmask], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        // lane j owns bins 2047-64j .. 1984-64j, scanned from the top; its sum reads them
        // starting at a lane-dependent offset, so the 32 lanes hit 32 different banks
        uint32_t s = 0;
        for (int t = 0; t < 64; ++t) s += hist[SEL_BINS - 1 - 64 * lane - ((t + lane) & 63)];
        uint32_t incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(FULL, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - s;
        if (excl < krem && krem <= incl) {
          uint32_t run = excl;
          for (int t = 0; t < 64; ++t) {
            const uint32_t c = hist[SEL_BINS - 1 - 64 * lane - t];
            if (run + c >= krem) {
              sh_digit = (uint32_t)(SEL_BINS - 1 - 64 * lane - t);
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
  // ordered emit: kept positions in ascending order
  const int chunk = SEL_THREADS * SEL_ITEMS;
  int out_base = 0, eq_base = 0;
  for (int c0 = 0; c0 < n; c0 += chunk) {
    const int i0 = c0 + threadIdx.x * SEL_ITEMS;
    uint32_t kv[SEL_ITEMS];
    int neq = 0;
#pragma unroll
    for (int t = 0; t < SEL_ITEMS; ++t) {
      const int i = i0 + t;
      kv[t] = (i < ncand) ? key[i] : 0u;
      neq += (!take_all && !take_none && i < ncand && kv[t] == T) ? 1 : 0;
    }
    int eq_tot;
    int eq_rank = eq_base + block_excl_scan(neq, wsum, &eq_tot);
    bool keep[SEL_ITEMS];
    int nkeep = 0;
#pragma unroll
    for (int t = 0; t < SEL_ITEMS; ++t) {
      const int i = i0 + t;
      bool kp = false;
      if (i < n) {
        if (i >= ncand || take_all) kp = true;
        else if (!take_none) {
          if (kv[t] > T) kp = true;
          else if (kv[t] == T) { kp = eq_rank < need_eq; ++eq_rank; }
        }
      }
      keep[t] = kp;
      nkeep += kp ? 1 : 0;
    }
    int keep_tot;
    int pos = out_base + block_excl_scan(nkeep, wsum, &keep_tot);
#pragma unroll
    for (int t = 0; t < SEL_ITEMS; ++t) {
      if (keep[t]) {
        if (pos < k_cap) {
          if (union_mode) {
            for (int g = 0; g < Hkv; ++g) idx[((int64_t)row * Hkv + g) * k_cap + pos] = i0 + t;
          } else {
            idx[(int64_t)row * k_cap + pos] = i0 + t;
          }
        } else {
          flag(status, ST_BOUNDS);
        }
        ++pos;
      }
    }
    out_base += keep_tot;
    eq_base += eq_tot;
  }
}

cudaError_t launch_budget(int mode, int L, int n, int w, double rho, const int32_t* k_in,
                          long long B, const float* Ebar, int32_t* k_out, cudaStream_t st) {
  budget_kernel<<<1, 1, 0, st>>>(mode, L, n, w, rho, k_in, B, Ebar, k_out);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_select(const float* S, int64_t Ssl, int64_t Ssh, int L, int Hkv, int n, int w,
                          int union_mode, const int32_t* k_l, int32_t* idx, int k_cap,
                          uint32_t* keys_ws, cudaStream_t st, const int32_t* n_l) {
  const int rows = union_mode ? L : L * Hkv;
  if (union_mode) {
    const int64_t total = (int64_t)rows * n;
    int grid = (int)((total + 255) / 256);
    if (grid > num_sms() * 16) grid = num_sms() * 16;
    keys_kernel<<<grid, 256, 0, st>>>(S, Ssl, Ssh, L, Hkv, n, union_mode, keys_ws);
    count_launch();
  }
  select_kernel<<<rows, SEL_THREADS, 0, st>>>(S, Ssl, Ssh, union_mode ? keys_ws : nullptr, n, w, k_l, Hkv,
                                              union_mode, idx, k_cap, status_ptr(), n_l);
  count_launch();
  return cudaGetLastError();
}

}  // namespace kvc
