// SelKV routing, soft-cosine-gated value merge and attention ratio.
//
// [SelKV] Methodology / Core components: soft cosine gate
// g = max(cos(v_evicted, v_kept), 0) sets how strongly an evicted token is
// merged (1: full merge, 0: drop); the kept slot's value becomes the gated,
// attention-weighted average of its own and the evicted contributions; the
// attention ratio R (mass the merged slot should receive relative to its
// original) feeds the decode-time logit bias.  Pipeline overview steps 3-5:
// evicted tokens are routed inside fixed positional buckets to the kept token
// with the highest prefill attention.
//
// One CTA per (layer, KV head, bucket).  Each warp owns a fixed subset of
// the bucket's evicted tokens (lane = d/32 slice of the value) and
// accumulates its gated sums; warp partials are added in warp order, so the
// result is deterministic (no atomics).
#include "kernels.cuh"

namespace kvc {

constexpr int MG_WARPS = 8;
constexpr int MG_MAXB = 4096;   // largest bucket
constexpr int MG_MAXE = 4;      // value elements per lane (head_dim <= 128)



__device__ __forceinline__ float ld_elem(const void* base, int bf16, int64_t off) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[off])
              : reinterpret_cast<const float*>(base)[off];
}

__global__ void __launch_bounds__(MG_WARPS * 32) merge_kernel(MergeParams p) {
  __shared__ uint32_t keptbits[MG_MAXB / 32];
  __shared__ float part[MG_WARPS][MG_MAXE * 32];
  __shared__ float partden[MG_WARPS];
  __shared__ int sh_j0, sh_j1, sh_t;
  __shared__ float sh_At;
  const int lg = blockIdx.x / p.nbuckets, b = blockIdx.x % p.nbuckets;
  const int l = lg / p.Hkv, g = lg % p.Hkv;
  const int lo = b * p.bucket, hi = min(p.n, lo + p.bucket);
  const int kl = min(p.k[l], p.k_cap);
  const int32_t* id = p.idx + (int64_t)lg * p.k_cap;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    // kept slots of this bucket: [j0, j1) of the ascending index list
    int a = 0, c = kl;
    while (a < c) { int mid = (a + c) >> 1; if (id[mid] < lo) a = mid + 1; else c = mid; }
    sh_j0 = a;
    c = kl;
    while (a < c) { int mid = (a + c) >> 1; if (id[mid] < hi) a = mid + 1; else c = mid; }
    sh_j1 = a;
  }
  for (int w = threadIdx.x; w < MG_MAXB / 32; w += blockDim.x) keptbits[w] = 0u;
  __syncthreads();
  const int j0 = sh_j0, j1 = sh_j1;
  if (j0 == j1) return;   // no kept token: the bucket's evicted tokens are dropped
  const float* Ar = p.A + l * p.Asl + g * p.Ash;
  // target: highest A among the kept slots (ties: lower position = lower slot)
  if (warp == 0) {
    float best = -INFINITY;
    int bj = 0x7fffffff;
    for (int j = j0 + lane; j < j1; j += 32) {
      const float a = Ar[id[j]];
      if (a > best || (a == best && j < bj)) { best = a; bj = j; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(FULL, best, o);
      const int oj = __shfl_xor_sync(FULL, bj, o);
      if (ob > best || (ob == best && oj < bj)) { best = ob; bj = oj; }
    }
    if (lane == 0) {
      if (bj < j0 || bj >= j1) { bj = j0; best = -INFINITY; }   // no finite attention: no merge
      sh_t = bj;
      sh_At = best;
    }
  }
  for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
    const int pos = id[j] - lo;
    atomicOr(&keptbits[pos >> 5], 1u << (pos & 31));
  }
  __syncthreads();
  const int tj = sh_t;
  const int tpos = id[tj];
  const float At = sh_At;
  const int d = p.d;
  const int epl = d / 32;
  const char* Vb = reinterpret_cast<const char*>(p.V);
  const int64_t vrow0 = l * p.Vsl + g * p.Vsh;
  float vt[MG_MAXE];
  float nt = 0.f;
#pragma unroll
  for (int e = 0; e < MG_MAXE; ++e) {
    vt[e] = e < epl ? ld_elem(Vb, p.bf16, vrow0 + (int64_t)tpos * p.Vst + lane * epl + e) : 0.f;
    nt = fmaf(vt[e], vt[e], nt);
  }
  nt = warp_sum(nt);
  float acc[MG_MAXE] = {0.f, 0.f, 0.f, 0.f};
  float den = 0.f;
  const bool do_merge = At > 0.f;
  if (!do_merge && threadIdx.x == 0) flag(p.status, ST_ZERO_ATTN);
  if (do_merge) {
    // evicted positions of the bucket, warp w takes the w-th, (w+8)-th, ... in position order
    int ord = 0;
    for (int pos = lo; pos < hi; ++pos) {
      const int rel = pos - lo;
      if (keptbits[rel >> 5] & (1u << (rel & 31))) continue;
      if ((ord++ % MG_WARPS) != warp) continue;
      float vj[MG_MAXE];
      float dot = 0.f, nj = 0.f;
#pragma unroll
      for (int e = 0; e < MG_MAXE; ++e) {
        vj[e] = e < epl ? ld_elem(Vb, p.bf16, vrow0 + (int64_t)pos * p.Vst + lane * epl + e) : 0.f;
        dot = fmaf(vj[e], vt[e], dot);
        nj = fmaf(vj[e], vj[e], nj);
      }
      dot = warp_sum(dot);
      nj = warp_sum(nj);
      const float dn = sqrtf(nj) * sqrtf(nt);
      const float cs = dn > 0.f ? dot / dn : 0.f;
      const float gate = fmaxf(cs, 0.f);
      const float wgt = gate * Ar[pos];
#pragma unroll
      for (int e = 0; e < MG_MAXE; ++e) acc[e] = fmaf(wgt, vj[e], acc[e]);
      den += wgt;
    }
  }
#pragma unroll
  for (int e = 0; e < MG_MAXE; ++e) part[warp][lane * MG_MAXE + e] = acc[e];
  if (lane == 0) partden[warp] = den;
  __syncthreads();
  // slots of the bucket: the target gets the merge, the others a copy and R = 1
  for (int j = j0 + warp; j < j1; j += MG_WARPS) {
    const int pos = id[j];
    float out[MG_MAXE];
    float r = 1.f;
    // a zero gated mass (every gate 0, or no evicted token) is a drop: the slot keeps v
    // bit for bit and R = 1, rather than (A_t v_t) / A_t rounded
    float gsum = 0.f;
    for (int w = 0; w < MG_WARPS; ++w) gsum += partden[w];
    if (j == tj && do_merge && gsum > 0.f) {
      float num[MG_MAXE], dsum = At;
#pragma unroll
      for (int e = 0; e < MG_MAXE; ++e) num[e] = At * vt[e];
      for (int w = 0; w < MG_WARPS; ++w) {
#pragma unroll
        for (int e = 0; e < MG_MAXE; ++e) num[e] += part[w][lane * MG_MAXE + e];
        dsum += partden[w];
      }
#pragma unroll
      for (int e = 0; e < MG_MAXE; ++e) out[e] = num[e] / dsum;
      r = dsum / At;
    } else {
#pragma unroll
      for (int e = 0; e < MG_MAXE; ++e)
        out[e] = e < epl ? ld_elem(Vb, p.bf16, vrow0 + (int64_t)pos * p.Vst + lane * epl + e) : 0.f;
    }
    const int64_t drow = l * p.dVl + g * p.dVh + (int64_t)j * p.dVt + lane * epl;
#pragma unroll
    for (int e = 0; e < MG_MAXE; ++e) {
      if (e >= epl) break;
      if (p.dbf16)
        reinterpret_cast<__nv_bfloat16*>(p.dV)[drow + e] = __float2bfloat16_rn(out[e]);
      else
        reinterpret_cast<float*>(p.dV)[drow + e] = out[e];
      if (p.dVf) p.dVf[((int64_t)lg * p.k_cap + j) * d + lane * epl + e] = out[e];
    }
    if (lane == 0) p.R[(int64_t)lg * p.k_cap + j] = r;
  }
}

// ---------------------------------------------------------------------------
// bf16 values, head_dim 128: the same merge with 16-byte loads.  As soon as the bucket's
// kept slots are known, warps 1.. copy every kept row (R = 1), eight rows in flight per
// half-warp, while warp 0 finds the merge target; only the target is rewritten at the
// end.  The bucket's evicted positions are listed once (block scan, position order);
// half-warp h of warp w takes list entries 2 w + h, 2 w + h + 16, ... and keeps four rows
// in flight; lanes of a half-warp hold 8 dims each.  Sums run in a fixed order (half-warp
// rows in list order, the two halves, then the warps), so the result does not depend on
// timing.
constexpr int MF_U = 4;   // evicted rows in flight per half-warp
constexpr int MG_CU = 8;  // kept rows in flight per half-warp in the early copy

// First j in [0, n) with id[j] >= key (n if none), for ascending id; called by a whole
// warp, every lane gets the answer.  Each round probes 32 evenly spaced entries, so the
// range shrinks 32-fold per dependent load.
__device__ __forceinline__ int warp_lower_bound(const int32_t* __restrict__ id, int n, int key, int lane) {
  int a = 0, c = n;   // the answer is in [a, c]
  while (a < c) {
    const int step = (c - a + 31) >> 5;
    const int probe = a + lane * step;
    const bool lt = probe < c && __ldg(id + probe) < key;
    const int t = __popc(__ballot_sync(FULL, lt));   // the probes below key are a prefix
    if (t == 0) return a;
    const int na = a + (t - 1) * step + 1;
    const int nc = min(c, a + t * step);
    a = na;
    c = nc;
  }
  return a;
}

__global__ void __launch_bounds__(MG_WARPS * 32, 4) merge_fast_kernel(MergeParams p) {
  __shared__ uint32_t keptbits[MG_MAXB / 32];
  __shared__ int ev[MG_MAXB];
  __shared__ int wsum[MG_WARPS];
  __shared__ float part[MG_WARPS][128];
  __shared__ float partden[MG_WARPS];
  __shared__ int sh_j0, sh_j1, sh_t, sh_ne;
  __shared__ float sh_At;
  const int lg = blockIdx.x / p.nbuckets, b = blockIdx.x % p.nbuckets;
  const int l = lg / p.Hkv, g = lg % p.Hkv;
  const int lo = b * p.bucket, hi = min(p.n, lo + p.bucket);
  const int kl = min(p.k[l], p.k_cap);
  const int32_t* id = p.idx + (int64_t)lg * p.k_cap;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane >> 4, part16 = lane & 15;
  if (threadIdx.x == 64 && p.Vst == p.d) {
    // contiguous rows: the bucket's values start on their way to L2 while the slots are found
    const char* vb0 = reinterpret_cast<const char*>(p.V) + ((l * p.Vsl + g * p.Vsh) + (int64_t)lo * p.d) * 2;
    const uint32_t nbytes = (uint32_t)(hi - lo) * (uint32_t)p.d * 2u;
    for (uint32_t o = 0; o < nbytes; o += 32768u) prefetch_l2(vb0 + o, min(32768u, nbytes - o));
  }
  // kept slots of this bucket: [j0, j1) of the ascending index list
  if (warp == 0) {
    const int a = warp_lower_bound(id, kl, lo, lane);
    if (lane == 0) sh_j0 = a;
  } else if (warp == 1) {
    const int c = warp_lower_bound(id, kl, hi, lane);
    if (lane == 0) sh_j1 = c;
  }
  for (int w = threadIdx.x; w < MG_MAXB / 32; w += blockDim.x) keptbits[w] = 0u;
  __syncthreads();
  const int j0 = sh_j0, j1 = sh_j1;
  if (j0 == j1) return;   // no kept token: the bucket's evicted tokens are dropped
  const float* Ar = p.A + l * p.Asl + g * p.Ash;
  const char* Vb = reinterpret_cast<const char*>(p.V) + (l * p.Vsl + g * p.Vsh) * 2;
  const int64_t vst = p.Vst * 2;                   // bytes between rows
  if (warp != 0) {
    // every kept slot starts as a bit-exact copy of its row with R = 1, while warp 0 looks
    // for the merge target; the target is rewritten at the end if it takes a merge
    const int hwi = (warp - 1) * 2 + sub, nhw = (MG_WARPS - 1) * 2;
    for (int jb = j0 + hwi; jb < j1; jb += nhw * MG_CU) {
      uint4 cv[MG_CU];
#pragma unroll
      for (int u = 0; u < MG_CU; ++u) {
        const int j = jb + u * nhw;
        if (j < j1) cv[u] = ldg16(Vb + (int64_t)id[j] * vst + part16 * 16);
      }
#pragma unroll
      for (int u = 0; u < MG_CU; ++u) {
        const int j = jb + u * nhw;
        if (j >= j1) break;
        const int64_t drow = l * p.dVl + g * p.dVh + (int64_t)j * p.dVt + part16 * 8;
        float f[8];
        Vec<__nv_bfloat16>::unpack(cv[u], f);
        if (p.dbf16) {
          *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.dV) + drow) = cv[u];
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) reinterpret_cast<float*>(p.dV)[drow + e] = f[e];
        }
        if (p.dVf) {
#pragma unroll
          for (int e = 0; e < 8; ++e) p.dVf[((int64_t)lg * p.k_cap + j) * 128 + part16 * 8 + e] = f[e];
        }
        if (part16 == 0) p.R[(int64_t)lg * p.k_cap + j] = 1.f;
      }
    }
  }
  if (warp == 0) {
    float best = -INFINITY;
    int bj = 0x7fffffff;
    for (int j = j0 + lane; j < j1; j += 32) {
      const float a = Ar[id[j]];
      if (a > best || (a == best && j < bj)) { best = a; bj = j; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(FULL, best, o);
      const int oj = __shfl_xor_sync(FULL, bj, o);
      if (ob > best || (ob == best && oj < bj)) { best = ob; bj = oj; }
    }
    if (lane == 0) {
      if (bj < j0 || bj >= j1) { bj = j0; best = -INFINITY; }   // no finite attention: no merge
      sh_t = bj;
      sh_At = best;
    }
  }
  for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
    const int pos = id[j] - lo;
    atomicOr(&keptbits[pos >> 5], 1u << (pos & 31));
  }
  __syncthreads();
  // evicted positions of the bucket in position order (block-wide exclusive scan)
  const int nb = hi - lo;
  for (int base = 0; base < nb; base += blockDim.x) {
    const int rel = base + threadIdx.x;
    const bool e = rel < nb && !((keptbits[rel >> 5] >> (rel & 31)) & 1u);
    const unsigned bal = __ballot_sync(FULL, e);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int off = base == 0 ? 0 : sh_ne;
    for (int w = 0; w < warp; ++w) off += wsum[w];
    if (e) ev[off + __popc(bal & ((1u << lane) - 1u))] = lo + rel;
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = base == 0 ? 0 : sh_ne;
      for (int w = 0; w < MG_WARPS; ++w) t += wsum[w];
      sh_ne = t;
    }
    __syncthreads();
  }
  const int ne = sh_ne;
  const int tj = sh_t;
  const int tpos = id[tj];
  const float At = sh_At;
  float vt[8];
  Vec<__nv_bfloat16>::unpack(ldg16(Vb + (int64_t)tpos * vst + part16 * 16), vt);
  float nt = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) nt = fmaf(vt[e], vt[e], nt);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) nt += __shfl_xor_sync(FULL, nt, o);
  const float snt = sqrtf(nt);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float den = 0.f;
  const bool do_merge = At > 0.f;
  if (!do_merge && threadIdx.x == 0) flag(p.status, ST_ZERO_ATTN);
  if (do_merge) {
    const int stride = 2 * MG_WARPS;
    // warp-uniform trip count (the shuffles below need both halves of the warp)
    for (int ew = 2 * warp; ew < ne; ew += stride * MF_U) {
      const int e0 = ew + sub;
      uint4 raw[MF_U];
      float av[MF_U];
#pragma unroll
      for (int u = 0; u < MF_U; ++u) {
        const int e = e0 + u * stride;
        if (e < ne) {
          const int pos = ev[e];
          raw[u] = ldg16(Vb + (int64_t)pos * vst + part16 * 16);
          av[u] = __ldg(Ar + pos);
        } else {
          raw[u] = make_uint4(0, 0, 0, 0);
          av[u] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < MF_U; ++u) {
        float vj[8];
        Vec<__nv_bfloat16>::unpack(raw[u], vj);
        float dot = 0.f, nj = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          dot = fmaf(vj[e], vt[e], dot);
          nj = fmaf(vj[e], vj[e], nj);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          dot += __shfl_xor_sync(FULL, dot, o);
          nj += __shfl_xor_sync(FULL, nj, o);
        }
        if (e0 + u * stride < ne) {
          const float dn = sqrtf(nj) * snt;
          const float cs = dn > 0.f ? dot / dn : 0.f;
          const float wgt = fmaxf(cs, 0.f) * av[u];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fmaf(wgt, vj[e], acc[e]);
          den += wgt;
        }
      }
    }
  }
  // the warp's two halves, then the warps in order
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(FULL, acc[e], 16);
  den += __shfl_xor_sync(FULL, den, 16);
  if (sub == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) part[warp][part16 * 8 + e] = acc[e];
    if (part16 == 0) partden[warp] = den;
  }
  __syncthreads();
  // the merge target gets the merged value and its R (every kept slot was copied at the start)
  for (int j = (warp == 0 && sub == 0) ? tj : j1; j < j1; j = j1) {
    const int pos = id[j];
    float out[8];
    float r = 1.f;
    // a zero gated mass (every gate 0, or no evicted token) is a drop: the slot keeps v
    // bit for bit and R = 1, rather than (A_t v_t) / A_t rounded
    float gsum = 0.f;
    for (int w = 0; w < MG_WARPS; ++w) gsum += partden[w];
    if (j == tj && do_merge && gsum > 0.f) {
      float dsum = At;
#pragma unroll
      for (int e = 0; e < 8; ++e) out[e] = At * vt[e];
      for (int w = 0; w < MG_WARPS; ++w) {
#pragma unroll
        for (int e = 0; e < 8; ++e) out[e] += part[w][part16 * 8 + e];
        dsum += partden[w];
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) out[e] /= dsum;
      r = dsum / At;
    } else {
      Vec<__nv_bfloat16>::unpack(ldg16(Vb + (int64_t)pos * vst + part16 * 16), out);
    }
    const int64_t drow = l * p.dVl + g * p.dVh + (int64_t)j * p.dVt + part16 * 8;
    if (p.dbf16) {
      uint4 o;
      o.x = pack_bf16x2(out[0], out[1]);
      o.y = pack_bf16x2(out[2], out[3]);
      o.z = pack_bf16x2(out[4], out[5]);
      o.w = pack_bf16x2(out[6], out[7]);
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.dV) + drow) = o;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) reinterpret_cast<float*>(p.dV)[drow + e] = out[e];
    }
    if (p.dVf) {
#pragma unroll
      for (int e = 0; e < 8; ++e) p.dVf[((int64_t)lg * p.k_cap + j) * 128 + part16 * 8 + e] = out[e];
    }
    if (part16 == 0) p.R[(int64_t)lg * p.k_cap + j] = r;
  }
}

cudaError_t launch_merge(const MergeParams& p, cudaStream_t st) {
  const unsigned grid = (unsigned)((int64_t)p.L * p.Hkv * p.nbuckets);
  if (grid == 0) return cudaSuccess;
  const bool fast = p.bf16 && p.d == 128 && ((uintptr_t)p.V % 16 == 0) && ((p.Vst * 2) % 16 == 0) &&
                    ((p.Vsl * 2) % 16 == 0) && ((p.Vsh * 2) % 16 == 0) &&
                    (!p.dbf16 || (((uintptr_t)p.dV % 16 == 0) && (p.dVt * 2) % 16 == 0 &&
                                  (p.dVl * 2) % 16 == 0 && (p.dVh * 2) % 16 == 0));
  if (fast) merge_fast_kernel<<<grid, MG_WARPS * 32, 0, st>>>(p);
  else merge_kernel<<<grid, MG_WARPS * 32, 0, st>>>(p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace kvc
