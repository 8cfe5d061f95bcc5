// Decode attention over a (compressed) cache, with the SelKV logit bias and
// the RECAS dropped-mass probe.
//
// [SelKV] Methodology / Core component 2 "attention compensation": add
// alpha_c * log(R_i) to the attention logit of every cached slot.
// [RECAS] 2.B: delta_t = attention mass on evicted tokens; with
// ||v_i|| <= V_max the output deviation obeys ||o - o'||_2 <= 2 V_max delta_t.
//
// Split-K ("flash decoding"): each CTA streams a contiguous range of one
// (sequence, layer, KV head) row and keeps, for each of the G query heads of
// the group, an online max / sum / weighted value sum; a second kernel merges
// the splits.  A group of LPK = head_dim / EPL lanes owns one key (EPL
// elements per lane, 16-byte loads for bf16 at EPL = 8), so a warp covers
// 32 / LPK keys per step with fully coalesced row reads.  Logits are kept in
// log2 units (scale * log2(e) folded into q) and exponentiated with exp2f.
#include "kernels.cuh"
#include "tc_sm100.cuh"

namespace kvc {

constexpr int DC_THREADS = 128;
constexpr float LN2 = 0.6931471805599453f;



template <typename T> struct Ld;
template <> struct Ld<__nv_bfloat16> {
  template <int EPL>
  __device__ __forceinline__ static void row(const char* p, float* f) {
    if constexpr (EPL == 8) {
      uint4 u = ldg16(p);
      Vec<__nv_bfloat16>::unpack(u, f);
    } else {
      uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
      f[0] = bf_lo(u.x); f[1] = bf_hi(u.x); f[2] = bf_lo(u.y); f[3] = bf_hi(u.y);
    }
  }
};
template <> struct Ld<float> {
  template <int EPL>
  __device__ __forceinline__ static void row(const char* p, float* f) {
    uint4 u = ldg16(p);
    Vec<float>::unpack(u, f);
    if constexpr (EPL == 8) {
      uint4 u2 = ldg16(p + 16);
      Vec<float>::unpack(u2, f + 4);
    }
  }
};

// Record per (split, query head): [m, l, acc[d]] (decode) or
// [m, l_kept, l_ev, vmax2, acc_all[d], acc_kept[d]] (probe); m in log2 units.
template <bool PROBE> __host__ __device__ constexpr int rec_len(int d) { return PROBE ? 4 + 2 * d : 2 + d; }

template <typename T, int EPL, int GM, bool PROBE>
__global__ void __launch_bounds__(DC_THREADS) decode_split_kernel(DecodeParams p) {
  constexpr int ES = sizeof(T);
  const int row = blockIdx.x;                  // (b, l, g)
  const int g = row % p.Hkv, l = (row / p.Hkv) % p.L, b = row / (p.Hkv * p.L);
  const int split = blockIdx.y;
  const int lpk = p.d / EPL;                   // lanes per key
  const int kpw = 32 / lpk;                    // keys per warp step
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / lpk, part = lane % lpk;
  int n = p.len[b * p.L + l];
  if (n > p.max_len || n < 0) {
    if (threadIdx.x == 0 && split == 0) flag(p.status, ST_BOUNDS);
    n = n < 0 ? 0 : p.max_len;
  }
  const int s0 = split * p.split_len, s1 = min(n, s0 + p.split_len);
  const int G = p.G;
  // query slices (scale * log2e folded in)
  float qr[GM][EPL];
#pragma unroll
  for (int gg = 0; gg < GM; ++gg) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      float x = 0.f;
      if (gg < G) {
        const int64_t off = (((int64_t)b * p.L + l) * p.Hq + g * G + gg) * p.d + part * EPL + e;
        x = p.qbf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.q)[off])
                    : reinterpret_cast<const float*>(p.q)[off];
      }
      qr[gg][e] = x * p.qscale;
    }
  }
  float m[GM], ls[GM], lev[GM], acc[GM][EPL], acck[GM][PROBE ? EPL : 1];
  float vmax2 = 0.f;
#pragma unroll
  for (int gg = 0; gg < GM; ++gg) {
    m[gg] = -INFINITY; ls[gg] = 0.f; lev[gg] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[gg][e] = 0.f;
#pragma unroll
    for (int e = 0; e < (PROBE ? EPL : 1); ++e) acck[gg][e] = 0.f;
  }
  const char* Kr = p.K + b * p.Ksb + l * p.Ksl + g * p.Ksh + part * EPL * ES;
  const char* Vr = p.V + b * p.Vsb + l * p.Vsl + g * p.Vsh + part * EPL * ES;
  const float* Rr = p.R ? p.R + b * p.Rsb + l * p.Rsl + g * p.Rsh : nullptr;
  const uint32_t* Br = PROBE ? p.bits + b * p.bsb + l * p.bsl + g * p.bsh : nullptr;
  const int step = kpw * (DC_THREADS / 32);
  // U key-steps per iteration: every load of the iteration is issued before any math.
  // The running max m is a lazy reference: it only moves (with a rescale) when a
  // logit exceeds it by more than 2^8, so p = 2^(s - m) <= 256 and no per-key
  // rescale is needed.
  constexpr int U = 4;
  for (int ib = s0 + warp * kpw; ib < s1; ib += U * step) {
    float kf[U][EPL], vf[U][EPL];
    bool val[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = ib + u * step + sub;
      val[u] = i < s1;
      if (val[u]) {
        Ld<T>::template row<EPL>(Kr + (int64_t)i * p.Kst, kf[u]);
        Ld<T>::template row<EPL>(Vr + (int64_t)i * p.Vst, vf[u]);
      } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) { kf[u][e] = 0.f; vf[u][e] = 0.f; }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = ib + u * step + sub;
      const bool valid = val[u];
      float bias = 0.f;
      if (Rr && valid) bias = p.alpha_c * log2f(Rr[i]);
      bool kept = true;
      if (PROBE && valid) kept = (Br[i >> 5] >> (i & 31)) & 1u;
      if (PROBE) {
        float vv = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) vv = fmaf(vf[u][e], vf[u][e], vv);
        for (int o = lpk >> 1; o > 0; o >>= 1) vv += __shfl_xor_sync(FULL, vv, o);
        if (valid) vmax2 = fmaxf(vmax2, vv);
      }
#pragma unroll
      for (int gg = 0; gg < GM; ++gg) {
        if (gg >= G) break;
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) s = fmaf(qr[gg][e], kf[u][e], s);
        for (int o = lpk >> 1; o > 0; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
        if (!valid) continue;
        s += bias;
        if (s > m[gg] + 8.f) {            // new reference (first key, or a much larger logit)
          const float corr = exp2f(m[gg] - s);
          m[gg] = s;
          ls[gg] *= corr;
          lev[gg] *= corr;
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            acc[gg][e] *= corr;
            if (PROBE) acck[gg][e] *= corr;
          }
        }
        const float pr = exp2f(s - m[gg]);
        if (PROBE) {
          if (kept) ls[gg] += pr; else lev[gg] += pr;
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            acc[gg][e] = fmaf(pr, vf[u][e], acc[gg][e]);
            if (kept) acck[gg][e] = fmaf(pr, vf[u][e], acck[gg][e]);
          }
        } else {
          ls[gg] += pr;
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[gg][e] = fmaf(pr, vf[u][e], acc[gg][e]);
        }
      }
    }
  }
  // merge the key sub-groups of the warp (lanes with equal `part`)
  for (int o = lpk; o < 32; o <<= 1) {
    vmax2 = fmaxf(vmax2, __shfl_xor_sync(FULL, vmax2, o));
#pragma unroll
    for (int gg = 0; gg < GM; ++gg) {
      const float om = __shfl_xor_sync(FULL, m[gg], o);
      const float ol = __shfl_xor_sync(FULL, ls[gg], o);
      const float oe = __shfl_xor_sync(FULL, lev[gg], o);
      const float mn = fmaxf(m[gg], om);
      const float c1 = mn == -INFINITY ? 0.f : exp2f(m[gg] - mn);
      const float c2 = mn == -INFINITY ? 0.f : exp2f(om - mn);
      m[gg] = mn;
      ls[gg] = ls[gg] * c1 + ol * c2;
      lev[gg] = lev[gg] * c1 + oe * c2;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const float oa = __shfl_xor_sync(FULL, acc[gg][e], o);
        acc[gg][e] = acc[gg][e] * c1 + oa * c2;
        if (PROBE) {
          const float ok = __shfl_xor_sync(FULL, acck[gg][e], o);
          acck[gg][e] = acck[gg][e] * c1 + ok * c2;
        }
      }
    }
  }
  // merge the warps through shared memory, in warp order
  extern __shared__ float dsm[];
  const int rec = rec_len<PROBE>(p.d);
  float* wrec = dsm + (size_t)warp * GM * rec;
  if (sub == 0) {
#pragma unroll
    for (int gg = 0; gg < GM; ++gg) {
      if (gg >= G) break;
      float* r = wrec + gg * rec;
      if (part == 0) {
        r[0] = m[gg];
        r[1] = ls[gg];
        if (PROBE) { r[2] = lev[gg]; r[3] = vmax2; }
      }
      const int base = PROBE ? 4 : 2;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        r[base + part * EPL + e] = acc[gg][e];
        if (PROBE) r[base + p.d + part * EPL + e] = acck[gg][e];
      }
    }
  }
  __syncthreads();
  const int nw = DC_THREADS / 32;
  float* out = p.part + (((int64_t)row * p.nsplit + split) * G) * rec;
  for (int t = threadIdx.x; t < G * rec; t += DC_THREADS) {
    const int gg = t / rec, c = t % rec;
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, dsm[((size_t)w * GM + gg) * rec]);
    float v = 0.f;
    if (c == 0) v = M;
    else if (PROBE && c == 3) {
      for (int w = 0; w < nw; ++w) v = fmaxf(v, dsm[((size_t)w * GM + gg) * rec + 3]);
    } else {
      for (int w = 0; w < nw; ++w) {
        const float* r = dsm + ((size_t)w * GM + gg) * rec;
        const float sc = (M == -INFINITY) ? 0.f : exp2f(r[0] - M);
        v += r[c] * sc;
      }
    }
    out[t] = v;
  }
}



// ---------------------------------------------------------------------------
// bf16, head_dim 128, no probe: the production decode path.
//
// A group of 16 lanes owns one key (8 elements = one 16-byte load per lane for
// K and for V); a warp covers 2 keys per step and U steps per batch, and the
// next batch's raw loads are issued before the current batch is computed, so
// every warp keeps 2 batches of K/V rows in flight.  The G partial dot products
// of a 16-lane group are folded with a transpose-reduce: after log2(GM)
// exchange rounds every lane holds the full score of one query head
// g = (part >> (4 - log2 GM)) & (GM - 1), so the online-softmax update (and its
// exp) runs once per lane instead of G times; the probabilities are then
// broadcast back for the P·V FMAs.
// ---------------------------------------------------------------------------
template <int GM>
__device__ __forceinline__ float transpose_reduce(const float (&ps)[GM], int part) {
  float v[GM];
#pragma unroll
  for (int j = 0; j < GM; ++j) v[j] = ps[j];
  int o = 8;
#pragma unroll
  for (int w = GM; w > 1; w >>= 1, o >>= 1) {
    const bool hi = (part & o) != 0;
#pragma unroll
    for (int j = 0; j < w / 2; ++j) {
      const float send = hi ? v[j] : v[j + w / 2];
      const float keep = hi ? v[j + w / 2] : v[j];
      v[j] = keep + __shfl_xor_sync(FULL, send, o);
    }
  }
#pragma unroll
  for (; o >= 1; o >>= 1) v[0] += __shfl_xor_sync(FULL, v[0], o);
  return v[0];
}

// ---------------------------------------------------------------------------
// Persistent decode for bf16 K/V with head_dim 128, no probe, when the
// tensor-core kernel (decode_mma.cu) does not apply (fp32 q): a producer warp
// streams 32-key chunks of K and V into a shared-memory ring with bulk copies
// (cp.async.bulk, mbarrier completion); each of four consumer warps takes 8 keys
// of every chunk, two at a time, 16 lanes per key (8 dims per lane), with the G
// partial dot products of a lane reduced by a transposing butterfly and an
// online softmax in log2 units.  With two CTAs per SM about 190 KB per SM are
// in flight.  CTA c takes the (row, split) items c, c + grid, ...; the producer
// runs ahead across item boundaries.
constexpr int DT_KEYS = 32;                      // keys per stage
constexpr int DT_CW = 4;                         // consumer warps
constexpr int DT_THREADS = 32 * (1 + DT_CW);
constexpr int DT_ROW = 256;                      // bytes of one bf16 row of 128
constexpr int DT_STAGE = 2 * DT_KEYS * DT_ROW;   // K rows, then V rows

template <int GM> constexpr int dt_stages() { return GM == 8 ? 5 : 6; }

template <int GM>
__host__ __device__ constexpr size_t dt_smem() {
  return (size_t)dt_stages<GM>() * DT_STAGE + 2 * dt_stages<GM>() * 8 + 16 +
         (size_t)DT_CW * GM * rec_len<false>(128) * sizeof(float);
}

template <int GM>
__global__ void __launch_bounds__(DT_THREADS, 2) decode_tma_kernel(DecodeParams p, int nitems) {
  using namespace tc;
  constexpr int NST = dt_stages<GM>();
  constexpr int SH = GM == 8 ? 1 : GM == 4 ? 2 : 3;   // score of head (part >> SH) & (GM-1)
  extern __shared__ __align__(128) uint8_t dt_raw[];
  uint8_t* ring = dt_raw;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + NST * DT_STAGE);
  uint64_t* empty = full + NST;
  int* abort_flag = reinterpret_cast<int*>(empty + NST);
  float* dsm = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(abort_flag) + 16);
  volatile int* abort = abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], DT_CW);
    }
    *abort_flag = 0;
    fence_mbar_init();
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
      for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
        int row, split, s0, s1;
        item_range(item, row, split, s0, s1);
        const int g = row % p.Hkv, l = (row / p.Hkv) % p.L, b = row / (p.Hkv * p.L);
        const char* Kb = p.K + b * p.Ksb + l * p.Ksl + g * p.Ksh;
        const char* Vb = p.V + b * p.Vsb + l * p.Vsl + g * p.Vsh;
        for (int i0 = s0; i0 < s1; i0 += DT_KEYS, ++chunk) {
          const int s = chunk % NST;
          if (!mbar_wait(&empty[s], ((chunk / NST) & 1) ^ 1, abort, p.status)) goto producer_done;
          const int nk = min(DT_KEYS, s1 - i0);
          mbar_expect_tx(&full[s], 2u * nk * DT_ROW);
          uint8_t* dk = ring + s * DT_STAGE;
          uint8_t* dv = dk + DT_KEYS * DT_ROW;
          if (p.Kst == DT_ROW) {
            bulk_load(dk, Kb + (int64_t)i0 * DT_ROW, nk * DT_ROW, &full[s]);
          } else {
            for (int j = 0; j < nk; ++j) bulk_load(dk + j * DT_ROW, Kb + (int64_t)(i0 + j) * p.Kst, DT_ROW, &full[s]);
          }
          if (p.Vst == DT_ROW) {
            bulk_load(dv, Vb + (int64_t)i0 * DT_ROW, nk * DT_ROW, &full[s]);
          } else {
            for (int j = 0; j < nk; ++j) bulk_load(dv + j * DT_ROW, Vb + (int64_t)(i0 + j) * p.Vst, DT_ROW, &full[s]);
          }
        }
      }
    producer_done:;
    }
    return;
  }
  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;
  const int sub = lane >> 4, part = lane & 15;
  const int myg = (part >> SH) & (GM - 1);
  const int gbase = lane & 16;
  const int G = p.G;
  constexpr int rec = rec_len<false>(128);
  uint32_t chunk = 0;
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    int row, split, s0, s1;
    item_range(item, row, split, s0, s1);
    const int g = row % p.Hkv, l = (row / p.Hkv) % p.L, b = row / (p.Hkv * p.L);
    if (cw == 0 && lane == 0 && split == 0) {
      const int n = p.len[b * p.L + l];
      if (n > p.max_len || n < 0) flag(p.status, ST_BOUNDS);
    }
    float qr[GM][8];
#pragma unroll
    for (int gg = 0; gg < GM; ++gg) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float x = 0.f;
        if (gg < G) {
          const int64_t off = (((int64_t)b * p.L + l) * p.Hq + g * G + gg) * 128 + part * 8 + e;
          x = p.qbf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.q)[off])
                      : reinterpret_cast<const float*>(p.q)[off];
        }
        qr[gg][e] = x * p.qscale;
      }
    }
    float acc[GM][8];
#pragma unroll
    for (int gg = 0; gg < GM; ++gg)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[gg][e] = 0.f;
    float m = -INFINITY, lsum = 0.f;            // online state of head myg
    const float* Rr = p.R ? p.R + b * p.Rsb + l * p.Rsl + g * p.Rsh : nullptr;
    for (int i0 = s0; i0 < s1; i0 += DT_KEYS, ++chunk) {
      const int s = chunk % NST;
      bool ok = !*abort && mbar_wait(&full[s], (chunk / NST) & 1, abort, p.status);
      ok = __all_sync(FULL, ok);
      const int nk = min(DT_KEYS, s1 - i0);
      const uint8_t* sk = ring + s * DT_STAGE;
      const uint8_t* sv = sk + DT_KEYS * DT_ROW;
      // this warp's keys of the chunk: 8 of them, two at a time (one per half-warp)
#pragma unroll 2
      for (int t = 0; t < 4 && ok; ++t) {
        const int j = cw * 8 + t * 2 + sub;
        const bool valid = j < nk;
        uint4 kk = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
        if (valid) {
          kk = *reinterpret_cast<const uint4*>(sk + j * DT_ROW + part * 16);
          vv = *reinterpret_cast<const uint4*>(sv + j * DT_ROW + part * 16);
        }
        float kf[8], vf[8];
        Vec<__nv_bfloat16>::unpack(kk, kf);
        float ps[GM];
#pragma unroll
        for (int gg = 0; gg < GM; ++gg) {
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) a = fmaf(qr[gg][e], kf[e], a);
          ps[gg] = a;
        }
        float sc = transpose_reduce<GM>(ps, part);
        if (Rr && valid) sc += p.alpha_c * log2f(Rr[i0 + j]);
        if (!valid || myg >= G) sc = -INFINITY;
        const bool resc = sc > m + 8.f;
        float corr = 1.f;
        if (resc) {
          corr = exp2f(m - sc);
          m = sc;
          lsum *= corr;
        }
        const float pr = sc == -INFINITY ? 0.f : exp2f(sc - m);
        lsum += pr;
        if (__any_sync(FULL, resc)) {
#pragma unroll
          for (int gg = 0; gg < GM; ++gg) {
            const float cg = __shfl_sync(FULL, corr, gbase | (gg << SH));
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[gg][e] *= cg;
          }
        }
        Vec<__nv_bfloat16>::unpack(vv, vf);
#pragma unroll
        for (int gg = 0; gg < GM; ++gg) {
          const float pg = __shfl_sync(FULL, pr, gbase | (gg << SH));
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[gg][e] = fmaf(pg, vf[e], acc[gg][e]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // merge the warp's two key groups, then the four warps through shared memory
    float mg[GM], lg[GM];
#pragma unroll
    for (int gg = 0; gg < GM; ++gg) {
      mg[gg] = __shfl_sync(FULL, m, gbase | (gg << SH));
      lg[gg] = __shfl_sync(FULL, lsum, gbase | (gg << SH));
    }
#pragma unroll
    for (int gg = 0; gg < GM; ++gg) {
      const float om = __shfl_xor_sync(FULL, mg[gg], 16);
      const float ol = __shfl_xor_sync(FULL, lg[gg], 16);
      const float mn = fmaxf(mg[gg], om);
      const float c1 = mn == -INFINITY ? 0.f : exp2f(mg[gg] - mn);
      const float c2 = mn == -INFINITY ? 0.f : exp2f(om - mn);
      mg[gg] = mn;
      lg[gg] = lg[gg] * c1 + ol * c2;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float oa = __shfl_xor_sync(FULL, acc[gg][e], 16);
        acc[gg][e] = acc[gg][e] * c1 + oa * c2;
      }
    }
    float* wrec = dsm + (size_t)cw * GM * rec;
    if (sub == 0) {
#pragma unroll
      for (int gg = 0; gg < GM; ++gg) {
        if (gg >= G) break;
        float* r = wrec + gg * rec;
        if (part == 0) {
          r[0] = mg[gg];
          r[1] = lg[gg];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) r[2 + part * 8 + e] = acc[gg][e];
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(DT_CW * 32) : "memory");
    float* out = p.part + (((int64_t)row * p.nsplit + split) * G) * rec;
    for (int t = threadIdx.x - 32; t < G * rec; t += DT_CW * 32) {
      const int gg = t / rec, c = t % rec;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < DT_CW; ++w) M = fmaxf(M, dsm[((size_t)w * GM + gg) * rec]);
      float v = 0.f;
      if (c == 0) {
        v = M;
      } else {
#pragma unroll
        for (int w = 0; w < DT_CW; ++w) {
          const float* r = dsm + ((size_t)w * GM + gg) * rec;
          const float sc = (M == -INFINITY) ? 0.f : exp2f(r[0] - M);
          v += r[c] * sc;
        }
      }
      out[t] = v;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(DT_CW * 32) : "memory");
  }
}

bool decode_tma_supported(const DecodeParams& p, bool bf16, bool probe) {
  if (probe || !bf16 || p.d != 128 || p.G > 8) return false;
  const uintptr_t a = (uintptr_t)p.K | (uintptr_t)p.V;
  const int64_t st = p.Ksb | p.Ksl | p.Ksh | p.Kst | p.Vsb | p.Vsl | p.Vsh | p.Vst;
  return (a % 16) == 0 && (st % 16) == 0;
}

template <int GM>
static void launch_decode_tma_t(const DecodeParams& p, int grid, int nitems, cudaStream_t st) {
  auto kern = decode_tma_kernel<GM>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dt_smem<GM>());
  kern<<<grid, DT_THREADS, dt_smem<GM>(), st>>>(p, nitems);
  count_launch();
}

static cudaError_t launch_decode_tma(const DecodeParams& p, cudaStream_t st) {
  const int nitems = p.B * p.L * p.Hkv * p.nsplit;
  int grid = 2 * num_sms();
  if (grid > nitems) grid = nitems;
  if (p.G <= 2) launch_decode_tma_t<2>(p, grid, nitems, st);
  else if (p.G <= 4) launch_decode_tma_t<4>(p, grid, nitems, st);
  else launch_decode_tma_t<8>(p, grid, nitems, st);
  return cudaGetLastError();
}

constexpr int DC_MAXQ = 4;                       // dimensions per lane: head_dim 64 or 128

// One warp per (row, query head): merge splits.
template <bool PROBE>
__global__ void decode_combine_kernel(CombineParams c) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (wid >= c.rows * c.G) return;
  const int row = wid / c.G, gg = wid % c.G;
  const int g = row % c.Hkv, bl = row / c.Hkv;
  const int h = g * c.G + gg;
  const int64_t oidx = ((int64_t)bl * c.Hq + h);
  const int rec = rec_len<PROBE>(c.d);
  float M = -INFINITY;
  for (int s = 0; s < c.nsplit; ++s) M = fmaxf(M, c.part[(((int64_t)row * c.nsplit + s) * c.G + gg) * rec]);
  float l = 0.f, lev = 0.f, vm = 0.f;
  for (int s = 0; s < c.nsplit; ++s) {
    const float* r = c.part + (((int64_t)row * c.nsplit + s) * c.G + gg) * rec;
    const float sc = M == -INFINITY ? 0.f : exp2f(r[0] - M);
    l += r[1] * sc;
    if (PROBE) { lev += r[2] * sc; vm = fmaxf(vm, r[3]); }
  }
  // o = sum over the splits, in split order, of each split's partial times 2^(m_s - M): the
  // weights once per warp (lane j of a 32-split group holds split s0 + j's), then every lane
  // sums its dimensions e = lane + 32 q with all of a split's loads independent
  float acc[DC_MAXQ], acck[DC_MAXQ];
#pragma unroll
  for (int q = 0; q < DC_MAXQ; ++q) acc[q] = acck[q] = 0.f;
  for (int s0 = 0; s0 < c.nsplit; s0 += 32) {
    const int sj = s0 + lane;
    const float mj = sj < c.nsplit ? c.part[(((int64_t)row * c.nsplit + sj) * c.G + gg) * rec] : -INFINITY;
    const float wj = (M == -INFINITY || sj >= c.nsplit) ? 0.f : exp2f(mj - M);
    const int ns = min(32, c.nsplit - s0);
    for (int j = 0; j < ns; ++j) {
      const float w = __shfl_sync(FULL, wj, j);
      const float* r = c.part + (((int64_t)row * c.nsplit + s0 + j) * c.G + gg) * rec;
#pragma unroll
      for (int q = 0; q < DC_MAXQ; ++q) {
        const int e = lane + 32 * q;
        if (e < c.d) {
          acc[q] += r[(PROBE ? 4 : 2) + e] * w;
          if (PROBE) acck[q] += r[4 + c.d + e] * w;
        }
      }
    }
  }
  if (!PROBE) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int q = 0; q < DC_MAXQ; ++q) {
      const int e = lane + 32 * q;
      if (e < c.d) c.o[oidx * c.d + e] = acc[q] * inv;
    }
    if (c.lse && lane == 0) c.lse[oidx * c.lse_stride] = l > 0.f ? (M + log2f(l)) * LN2 : -INFINITY;
  } else {
    const float lall = l + lev;
    const float inv_all = lall > 0.f ? 1.f / lall : 0.f;
    const float inv_k = l > 0.f ? 1.f / l : 0.f;
    float e2 = 0.f;
#pragma unroll
    for (int q = 0; q < DC_MAXQ; ++q) {
      const int e = lane + 32 * q;
      if (e >= c.d) continue;
      const float va = acc[q] * inv_all, vk = acck[q] * inv_k;
      if (c.o_full) c.o_full[oidx * c.d + e] = va;
      if (c.o_kept) c.o_kept[oidx * c.d + e] = vk;
      e2 += (va - vk) * (va - vk);
    }
    e2 = warp_sum(e2);
    if (lane == 0) {
      const float dl = lall > 0.f ? lev / lall : 0.f;
      const float vmx = sqrtf(vm);
      if (c.delta) c.delta[oidx] = dl;
      if (c.err) c.err[oidx] = sqrtf(e2);
      if (c.bound) c.bound[oidx] = 2.f * vmx * dl;
      if (c.vmax && gg == 0) c.vmax[row] = vmx;
    }
  }
}

int decode_rec_len(bool probe, int d) { return probe ? rec_len<true>(d) : rec_len<false>(d); }

template <typename T, int EPL, bool PROBE>
static cudaError_t launch_split_t(const DecodeParams& p, cudaStream_t st) {
  dim3 grid(p.B * p.L * p.Hkv, p.nsplit);
  const int rec = rec_len<PROBE>(p.d);
#define KVC_DEC_CASE(GMV)                                                                       \
  {                                                                                             \
    const size_t sm = (size_t)(DC_THREADS / 32) * GMV * rec * sizeof(float);                    \
    auto kern = decode_split_kernel<T, EPL, GMV, PROBE>;                                        \
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);           \
    kern<<<grid, DC_THREADS, sm, st>>>(p);                                                      \
    count_launch();                                                                             \
    return cudaGetLastError();                                                                  \
  }
  if (p.G <= 2) KVC_DEC_CASE(2)
  if (p.G <= 4) KVC_DEC_CASE(4)
  KVC_DEC_CASE(8)
#undef KVC_DEC_CASE
}

cudaError_t launch_decode(const DecodeParams& p, bool bf16, bool probe, const CombineParams& c,
                          cudaStream_t st) {
  cudaError_t e;
  if (decode_mma_supported(p, bf16, probe)) {
    e = launch_decode_mma(p, probe, st);
  } else if (decode_tma_supported(p, bf16, probe)) {
    e = launch_decode_tma(p, st);
  } else if (!probe) {
    e = bf16 ? launch_split_t<__nv_bfloat16, 8, false>(p, st) : launch_split_t<float, 8, false>(p, st);
  } else {
    e = bf16 ? launch_split_t<__nv_bfloat16, 4, true>(p, st) : launch_split_t<float, 4, true>(p, st);
  }
  if (e != cudaSuccess) return e;
  const int warps = c.rows * c.G;
  const int blocks = (warps * 32 + 255) / 256;
  if (probe) decode_combine_kernel<true><<<blocks, 256, 0, st>>>(c);
  else decode_combine_kernel<false><<<blocks, 256, 0, st>>>(c);
  count_launch();
  return cudaGetLastError();
}

}  // namespace kvc
