// losa.cu -- the two steps of a LoSA denoising step around the block-query attention:
// sorting the block's tokens into active and stable by how much their queries changed,
// and the attention inside the block, joined with the prefix result.
//
// What is computed (LoSA, "2. 방법론"):
//   * activity: every denoising step measures the change of each token's query vectors
//     since the previous step by their mean squared difference (over all query heads and
//     dims); tokens that changed much are active, the others stable.  Active iff the
//     change exceeds tau, or (n_top > 0) iff it is among the n_top largest (equal changes:
//     the lower token index first).  The changes are summed and compared in fp64, so the
//     decision does not depend on the summation order except at exact ties.
//   * intra-block attention + merge: every token of the block (active or stable) attends
//     bidirectionally over the block's own Tq keys, which sit at cache rows
//     T_prefix .. T_prefix + Tq - 1, and the result is joined with the token's prefix
//     result (o_pre, lse_pre) -- computed this step for active tokens, reused for stable
//     ones -- by log-sum-exp: the softmax over the union of both token sets.
//
// How (B200): both are small, latency-bound kernels (a block of 32 tokens moves well
// under 1 MB), so the design keeps every load in flight at once and avoids block-wide
// round trips: the change of a token is a 16-byte-vectorised sum over a cluster of 8 CTAs
// whose partial results meet in rank 0's shared memory (one DSMEM store per token); the
// intra-block attention maps one query row to one warp (lane = key for the logits, lane =
// 4 output dims for P.V) with the block's keys in padded shared-memory rows.
#include <math.h>

#include "cluster.cuh"
#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {
namespace {

// ---- activity ---------------------------------------------------------------------------
constexpr int kClsThreads = 512;
constexpr int kClsCluster = 8;
constexpr int kClsTok = 8;  // tokens per CTA: Tq <= 64 over a cluster of 8
constexpr int kMaxTq = 64;

__device__ __forceinline__ void st_cluster_f64(uint32_t addr, double v) {
  asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(addr), "d"(v) : "memory");
}

// Sum of the squared differences of 8 bf16 pairs, in fp64 (bf16 -> fp32 -> fp64 widening
// is exact; a bf16 pair sits in one 32-bit word, element 2e in the low half).
__device__ __forceinline__ double sqdiff8(const uint4& a, const uint4& b) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w};
  const uint32_t wb[4] = {b.x, b.y, b.z, b.w};
  double s = 0.0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const double lo = (double)__uint_as_float(wa[e] << 16) - (double)__uint_as_float(wb[e] << 16);
    const double hi = (double)__uint_as_float(wa[e] & 0xffff0000u) -
                      (double)__uint_as_float(wb[e] & 0xffff0000u);
    s = fma(lo, lo, s);
    s = fma(hi, hi, s);
  }
  return s;
}

// Grid (8, B), clusters of 8: CTA `rank` of sequence b owns tokens
// [rank * per, min(Tq, rank * per + per)), per = ceil(Tq / 8).
__global__ void __cluster_dims__(kClsCluster, 1, 1) __launch_bounds__(kClsThreads)
    losa_classify_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ qp,
                         int Hq, int Tq, int d8_log2, double tau, int n_top,
                         double* __restrict__ mse_out, uint8_t* __restrict__ active) {
  const int rank = cluster_rank();
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kClsThreads / 32;
  __shared__ double all_mse[kMaxTq];  // rank 0: the change of every token of the block
  __shared__ double red[kWarps][kClsTok];
  pdl_trigger();  // the next kernel (the block-query step) may start its prologue now
  cluster_arrive_relaxed();  // rank 0's shared memory is written only after all have started

  const int per = (Tq + kClsCluster - 1) / kClsCluster;
  const int t0 = rank * per;
  const int nt = max(0, min(Tq, t0 + per) - t0);
  const int D = 8 << d8_log2;
  const int nch = Hq << d8_log2;  // 16-byte chunks of one token (all heads)
  double acc[kClsTok];
#pragma unroll
  for (int t = 0; t < kClsTok; ++t) acc[t] = 0.0;
  for (int c = tid; c < nch; c += kClsThreads) {
    const int h = c >> d8_log2, cc = c & ((1 << d8_log2) - 1);
    const size_t base = (((size_t)b * Hq + h) * Tq + t0) * D + (size_t)cc * 8;
    uint4 va[kClsTok], vb[kClsTok];
#pragma unroll
    for (int t = 0; t < kClsTok; ++t) {  // every load of the iteration first
      va[t] = make_uint4(0u, 0u, 0u, 0u);
      vb[t] = va[t];
      if (t < nt) {
        va[t] = __ldg(reinterpret_cast<const uint4*>(q + base + (size_t)t * D));
        vb[t] = __ldg(reinterpret_cast<const uint4*>(qp + base + (size_t)t * D));
      }
    }
#pragma unroll
    for (int t = 0; t < kClsTok; ++t)
      if (t < nt) acc[t] += sqdiff8(va[t], vb[t]);
  }
#pragma unroll
  for (int t = 0; t < kClsTok; ++t) {
    double v = acc[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][t] = v;
  }
  __syncthreads();
  cluster_wait();
  if (warp == 0 && lane < nt) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[w][lane];
    const double m = s / (double)(Hq * D);
    if (mse_out) mse_out[(size_t)b * Tq + t0 + lane] = m;
    st_cluster_f64(map_rank(&all_mse[t0 + lane], 0), m);
  }
  cluster_arrive_release();
  cluster_wait();
  if (rank == 0 && tid < Tq) {
    const double mi = all_mse[tid];
    bool on;
    if (n_top > 0) {
      int r = 0;  // tokens ranked before this one
      for (int j = 0; j < Tq; ++j) {
        const double mj = all_mse[j];
        r += (mj > mi || (mj == mi && j < tid)) ? 1 : 0;
      }
      on = r < n_top;
    } else {
      on = mi > tau;
    }
    active[(size_t)b * Tq + tid] = on ? 1 : 0;
  }
}

// ---- attention inside the block, merged with the prefix part ----------------------------
constexpr int kIntraRows = 8;  // query rows (tokens) per CTA, one per warp
constexpr int kIntraThreads = kIntraRows * 32;

// Grid (ceil(Tq / 8), Hq, B).  Warp w takes token i = 8 * blockIdx.x + w of head h.
template <int D>
__global__ void __launch_bounds__(kIntraThreads) intra_merge_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, int Hkv, int G, int Tq, int T_prefix, int T_cap,
    float scale2, const __nv_bfloat16* o_pre, const float* lse_pre, __nv_bfloat16* o, float* lse) {
  constexpr int kKS = D + 8;       // padded key row (bf16): 16-byte reads of 8 rows hit 8 bank groups
  constexpr int kC = D / 8;        // 16-byte chunks per row
  constexpr int kDL = D / 32;      // output dims per lane (4 or 2)
  __shared__ __align__(16) __nv_bfloat16 Ks[kMaxTq * kKS];
  __shared__ __align__(16) __nv_bfloat16 Vs[kMaxTq * D];
  __shared__ __align__(16) __nv_bfloat16 Qs[kIntraRows * D];
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / G, Hq = Hkv * G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i0 = blockIdx.x * kIntraRows;
  const int nq = min(kIntraRows, Tq - i0);

  // the block's keys and values (cache rows T_prefix ..) and this CTA's query rows
  const size_t kvrow0 = ((size_t)b * Hkv + g) * T_cap + T_prefix;
  for (int id = tid; id < Tq * kC; id += kIntraThreads) {
    const int r = id / kC, c = id - r * kC;
    const uint4 kk = __ldg(reinterpret_cast<const uint4*>(k + (kvrow0 + r) * D) + c);
    const uint4 vv = __ldg(reinterpret_cast<const uint4*>(v + (kvrow0 + r) * D) + c);
    *reinterpret_cast<uint4*>(Ks + r * kKS + c * 8) = kk;
    *reinterpret_cast<uint4*>(Vs + r * D + c * 8) = vv;
  }
  const size_t qrow0 = ((size_t)b * Hq + h) * Tq + i0;
  for (int id = tid; id < nq * kC; id += kIntraThreads) {
    const int r = id / kC, c = id - r * kC;
    *reinterpret_cast<uint4*>(Qs + r * D + c * 8) =
        __ldg(reinterpret_cast<const uint4*>(q + (qrow0 + r) * D) + c);
  }
  __syncthreads();
  if (warp >= nq) return;  // (no block barrier below)

  // logits of the row against keys lane and lane + 32 (base-2 units)
  float s0 = 0.f, s1 = 0.f;
  const bool has0 = lane < Tq, has1 = lane + 32 < Tq;
  const __nv_bfloat16* qr = Qs + warp * D;
#pragma unroll 4
  for (int c = 0; c < kC; ++c) {
    const uint4 qv = *reinterpret_cast<const uint4*>(qr + c * 8);
    const uint4 k0 = has0 ? *reinterpret_cast<const uint4*>(Ks + lane * kKS + c * 8) : make_uint4(0u, 0u, 0u, 0u);
    const uint4 k1 = has1 ? *reinterpret_cast<const uint4*>(Ks + (lane + 32) * kKS + c * 8) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t wq[4] = {qv.x, qv.y, qv.z, qv.w};
    const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w};
    const uint32_t w1[4] = {k1.x, k1.y, k1.z, k1.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float qlo = __uint_as_float(wq[e] << 16), qhi = __uint_as_float(wq[e] & 0xffff0000u);
      s0 = fmaf(qlo, __uint_as_float(w0[e] << 16), s0);
      s0 = fmaf(qhi, __uint_as_float(w0[e] & 0xffff0000u), s0);
      s1 = fmaf(qlo, __uint_as_float(w1[e] << 16), s1);
      s1 = fmaf(qhi, __uint_as_float(w1[e] & 0xffff0000u), s1);
    }
  }
  s0 = has0 ? s0 * scale2 : -INFINITY;
  s1 = has1 ? s1 * scale2 : -INFINITY;
  float mx = fmaxf(s0, s1);
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
  const float p0 = has0 ? ex2(s0 - mx) : 0.f;
  const float p1 = has1 ? ex2(s1 - mx) : 0.f;
  const float l = warp_sum(p0 + p1);

  // P.V: lane owns dims kDL * lane .. kDL * lane + kDL - 1
  float acc[kDL];
#pragma unroll
  for (int e = 0; e < kDL; ++e) acc[e] = 0.f;
  for (int j = 0; j < Tq; ++j) {
    const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
    const __nv_bfloat16* vr = Vs + j * D + kDL * lane;
    if constexpr (kDL == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(vr);
      acc[0] = fmaf(pj, __uint_as_float(w.x << 16), acc[0]);
      acc[1] = fmaf(pj, __uint_as_float(w.x & 0xffff0000u), acc[1]);
      acc[2] = fmaf(pj, __uint_as_float(w.y << 16), acc[2]);
      acc[3] = fmaf(pj, __uint_as_float(w.y & 0xffff0000u), acc[3]);
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(vr);
      acc[0] = fmaf(pj, __uint_as_float(w << 16), acc[0]);
      acc[1] = fmaf(pj, __uint_as_float(w & 0xffff0000u), acc[1]);
    }
  }
  const float lse_in = (mx + log2f(l)) * kLn2;
  const float inv_l = 1.f / l;

  // merge with the prefix part (read after the previous kernel of the stream completed)
  pdl_wait();
  const size_t row = qrow0 + warp;
  const float lp = lse_pre[row];
  float pre[kDL];
  if constexpr (kDL == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(o_pre + row * D + kDL * lane);
    pre[0] = __uint_as_float(w.x << 16); pre[1] = __uint_as_float(w.x & 0xffff0000u);
    pre[2] = __uint_as_float(w.y << 16); pre[3] = __uint_as_float(w.y & 0xffff0000u);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(o_pre + row * D + kDL * lane);
    pre[0] = __uint_as_float(w << 16); pre[1] = __uint_as_float(w & 0xffff0000u);
  }
  __syncwarp();  // every lane has read o_pre / lse_pre before any write (o, lse may alias them)
  float wp = 0.f, wi = inv_l, tot_lse = lse_in;
  if (lp != -INFINITY) {
    const float m2 = fmaxf(lp, lse_in);
    const float ep = expf(lp - m2), ei = expf(lse_in - m2);
    const float inv = 1.f / (ep + ei);
    wp = ep * inv;
    wi = ei * inv * inv_l;
    tot_lse = m2 + logf(ep + ei);
  }
  float out[kDL];
#pragma unroll
  for (int e = 0; e < kDL; ++e) out[e] = fmaf(wp, pre[e], wi * acc[e]);
  if constexpr (kDL == 4) {
    *reinterpret_cast<uint2*>(o + row * D + kDL * lane) =
        make_uint2(pack_bf16x2(out[0], out[1]), pack_bf16x2(out[2], out[3]));
  } else {
    *reinterpret_cast<uint32_t*>(o + row * D + kDL * lane) = pack_bf16x2(out[0], out[1]);
  }
  if (lane == 0) lse[row] = tot_lse;
}

}  // namespace

cudaError_t launch_losa_classify(const void* q, const void* q_prev, int B, int Hq, int Tq, int D,
                                 double tau, int n_top, uint8_t* active, double* mse,
                                 cudaStream_t stream) {
  const int d8_log2 = D == 128 ? 4 : 3;
  losa_classify_kernel<<<dim3(kClsCluster, B, 1), kClsThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(q_prev), Hq, Tq,
      d8_log2, tau, n_top, mse, active);
  return cudaGetLastError();
}

cudaError_t launch_intra_merge(const IntraMergeArgs& a, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.Tq + kIntraRows - 1) / kIntraRows, a.Hkv * a.G, a.B);
  cfg.blockDim = dim3(kIntraThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  const float scale2 = a.scale * kLog2e;
  const auto* q = static_cast<const __nv_bfloat16*>(a.q);
  const auto* k = static_cast<const __nv_bfloat16*>(a.k);
  const auto* v = static_cast<const __nv_bfloat16*>(a.v);
  const auto* op = static_cast<const __nv_bfloat16*>(a.o_pre);
  auto* o = static_cast<__nv_bfloat16*>(a.o);
  if (a.D == 128)
    return cudaLaunchKernelEx(&cfg, intra_merge_kernel<128>, q, k, v, a.Hkv, a.G, a.Tq, a.T_prefix,
                              a.T_cap, scale2, op, a.lse_pre, o, a.lse);
  return cudaLaunchKernelEx(&cfg, intra_merge_kernel<64>, q, k, v, a.Hkv, a.G, a.Tq, a.T_prefix,
                            a.T_cap, scale2, op, a.lse_pre, o, a.lse);
}

}  // namespace lsa
