// nsa.cu -- NSA's two other parallel branches for a decode step, with fixed parts in place
// of the learned ones: the compressed branch (attention over mean-pooled tokens, block
// length l at stride d) and the sliding window (attention over the last w tokens), joined
// with the selected branch (the sparse decode of decode.cu) by constant gates.
//
// What is computed (NSA news article, "NSA 구조": three parallel attention paths --
// compressed coarse tokens, selected fine tokens, a sliding window -- with l = 32,
// d = 16, l' = 64, n = 16, w = 512):
//   kc[b, g, i] = mean of k[b, g, t] over the valid t in [i*d, i*d + l), i < ceil(T_b / d)
//                 (vc likewise), stored in bf16;
//   o_cmp = softmax attention of q over kc/vc rows [0, ceil(T_b / d));
//   o_win = softmax attention of q over k/v rows [max(0, T_b - w), T_b);
//   o     = g_cmp * o_cmp + g_slc * o_slc + g_win * o_win.
//
// How (B200): the pool is a coalesced streaming kernel (a thread per 16-byte column of a
// compressed token, all its row loads in flight), which a decode loop runs over the last
// two compressed tokens only (the ones a new token changes).  The two branches are one
// launch: a cluster of 16 CTAs per (sequence, KV head) splits the concatenated rows
// [window | compressed] evenly, so a CTA may hold rows of both; each CTA runs an online
// softmax over 64-row tiles (K and V by cp.async into padded rows, logits and P.V on the
// FMA pipes: G <= 16 query rows are too few for a tensor-core tile), then stores each
// branch's partial (m, l, acc) into the shared memory of the CTA that owns that part of
// the output.  After one cluster barrier each CTA merges its slice from its own shared
// memory, adds the gated selected-branch output and writes o.  The only waits are
// hardware cluster barriers that every thread reaches.
#include <math.h>

#include "cluster.cuh"
#include "launch_cache.h"
#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {
namespace {

// ---- the pool ---------------------------------------------------------------------------
constexpr int kPoolThreads = 256;

// Grid (ceil(range_max / tokens per CTA), Hkv, 2 * B): z = 2b (k -> kc) or 2b + 1 (v -> vc).
// Thread: token tl = tid / kC of the CTA, 16-byte column c = tid % kC.
template <int D>
__global__ void __launch_bounds__(kPoolThreads) nsa_compress_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, int Hkv, int T_cap,
    const int32_t* __restrict__ seqlens, int len, int stride, int nc_begin, int nc_end,
    __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc) {
  constexpr int kC = D / 8;
  constexpr int kTok = kPoolThreads / kC;
  const int b = blockIdx.z >> 1, which = blockIdx.z & 1, g = blockIdx.y;
  const int tl = threadIdx.x / kC, c = threadIdx.x % kC;
  const int T = checked_range(seqlens[b], 0, T_cap, kBoundsSeqlen, kSiteNsaCompress);
  const int NC = (T + stride - 1) / stride;
  const int NC_cap = (T_cap + stride - 1) / stride;
  // the range of compressed tokens: [nc_begin, min(nc_end, NC)) or, for nc_begin < 0, the
  // last -nc_begin of this sequence
  int lo, hi;
  if (nc_begin >= 0) {
    lo = nc_begin;
    hi = min(nc_end >= 0 ? nc_end : NC_cap, NC_cap);
  } else {
    lo = max(0, NC + nc_begin);
    hi = NC;
  }
  const int i = lo + blockIdx.x * kTok + tl;
  if (i >= hi) return;
  const size_t unit = (size_t)b * Hkv + g;
  const __nv_bfloat16* src = (which ? v : k) + unit * (size_t)T_cap * D + (size_t)c * 8;
  __nv_bfloat16* dst = (which ? vc : kc) + (unit * NC_cap + i) * D + (size_t)c * 8;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const int t0 = i * stride;
  const int t1 = i < NC ? min(t0 + len, T) : t0;  // rows past the sequence: a zero row
#pragma unroll 8
  for (int t = t0; t < t1; ++t) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + (size_t)t * D));
    const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += __uint_as_float(wd[e] << 16);
      acc[2 * e + 1] += __uint_as_float(wd[e] & 0xffff0000u);
    }
  }
  const float inv = t1 > t0 ? 1.f / (float)(t1 - t0) : 0.f;
  *reinterpret_cast<uint4*>(dst) =
      make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                 pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
}

// ---- the window and compressed branches, merged and gated ------------------------------
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCL = 16;
constexpr int kMaxG = 16;
constexpr int kTile = 64;

template <int D>
struct BranchSmem {
  static constexpr int kKS = D + 8;  // padded bf16 rows: conflict-free 16-byte reads
  __nv_bfloat16 kt[kTile * kKS];
  __nv_bfloat16 vt[kTile * kKS];
  __nv_bfloat16 q[kMaxG * D];
  float s[kMaxG][kTile];              // logits (base 2), then probabilities
  float m_run[kMaxG], l_run[kMaxG], alpha[kMaxG];
  float2 recv_ml[2][kCL][kMaxG];      // [branch][source CTA][head] (m, l)
  float recv_acc[2][kCL][kMaxG * D / kCL];  // [branch][source CTA][element of my slice]
};

struct BranchParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* kc;
  const __nv_bfloat16* vc;
  const int32_t* seqlens;
  const __nv_bfloat16* o_slc;
  __nv_bfloat16* o;
  float* lse_win;
  float* lse_cmp;
  int Hkv, G, T_cap, NC_cap, window, stride;
  float scale2, g_cmp, g_slc, g_win;
};

// Launched with clusters of kCL CTAs along x (grid (kCL, Hkv, B)), dynamic shared memory
// sizeof(BranchSmem<D>).
template <int D>
__global__ void __launch_bounds__(kThreads) nsa_branches_kernel(const BranchParams p) {
  using S = BranchSmem<D>;
  constexpr int kKS = S::kKS;
  constexpr int kC = D / 8;
  constexpr int kHS = kThreads / D;     // heads interleaved per output column: 2 or 4
  constexpr int kPH = kMaxG / kHS;      // heads per thread in P.V
  extern __shared__ __align__(16) unsigned char smem_raw[];
  S& sm = *reinterpret_cast<S*>(smem_raw);
  const int rank = cluster_rank();
  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G, Hq = p.Hkv * G;
  const size_t unit = (size_t)b * p.Hkv + g;
  cluster_arrive_relaxed();  // peers' shared memory is written only after all have started

  for (int id = tid; id < G * kC; id += kThreads) {
    const int h = id / kC, c = id - h * kC;
    cp_async16(sm.q + h * D + c * 8, p.q + ((size_t)b * Hq + (size_t)g * G + h) * D + c * 8, true);
  }
  cp_async_commit();
  const int T = checked_range(p.seqlens[b], 0, p.T_cap, kBoundsSeqlen, kSiteNsaBranches);
  const int nw = min(p.window, T);                  // window rows
  const int nc = (T + p.stride - 1) / p.stride;     // compressed rows
  const int R = nw + nc;
  const int per = (R + kCL - 1) / kCL;
  const int r0 = min(R, rank * per), r1 = min(R, r0 + per);
  const int d = tid % D, h0 = tid / D;              // P.V mapping: column d, heads h0 + i*kHS
  const int per_out = G * D / kCL;                  // output elements each CTA merges
  cp_async_wait<0>();  // (q; also when this CTA gets no rows)
  cluster_wait();      // (matches the arrive at the start) DSMEM is live from here on

  for (int part = 0; part < 2; ++part) {  // 0: window rows [0, nw), 1: compressed [nw, R)
    const int lo = part == 0 ? max(r0, 0) : max(r0, nw);
    const int hi = part == 0 ? min(r1, nw) : min(r1, R);
    // concatenated row r of this part is row r - roff of its source: the window starts at
    // token T - nw of k / v, the compressed rows at index 0 of kc / vc
    const int roff = part == 0 ? 0 : nw;
    const __nv_bfloat16* ksrc = part == 0 ? p.k + (unit * p.T_cap + (size_t)(T - nw)) * D
                                          : p.kc + unit * p.NC_cap * D;
    const __nv_bfloat16* vsrc = part == 0 ? p.v + (unit * p.T_cap + (size_t)(T - nw)) * D
                                          : p.vc + unit * p.NC_cap * D;
    __syncthreads();  // (the previous part's statistics have been pushed)
    for (int h = tid; h < G; h += kThreads) {
      sm.m_run[h] = -INFINITY;
      sm.l_run[h] = 0.f;
    }
    float acc[kPH];
#pragma unroll
    for (int i = 0; i < kPH; ++i) acc[i] = 0.f;
    for (int t0 = lo; t0 < hi; t0 += kTile) {
      const int nt = min(kTile, hi - t0);
      __syncthreads();  // (the previous tile's K/V/P are no longer read)
      for (int id = tid; id < nt * kC; id += kThreads) {
        const int r = id / kC, c = id - r * kC;
        const size_t src = (size_t)(t0 + r - roff) * D + c * 8;
        cp_async16(sm.kt + r * kKS + c * 8, ksrc + src, true);
        cp_async16(sm.vt + r * kKS + c * 8, vsrc + src, true);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      // logits: pair (h, t) = (pp >> 6, pp & 63), a warp shares h
      for (int pp = tid; pp < G * kTile; pp += kThreads) {
        const int h = pp >> 6, t = pp & (kTile - 1);
        float sv = -INFINITY;
        if (t < nt) {
          float a0 = 0.f, a1 = 0.f;
          const __nv_bfloat16* kr = sm.kt + t * kKS;
          const __nv_bfloat16* qr = sm.q + h * D;
#pragma unroll 4
          for (int c = 0; c < kC; ++c) {
            const uint4 kk = *reinterpret_cast<const uint4*>(kr + c * 8);
            const uint4 qq = *reinterpret_cast<const uint4*>(qr + c * 8);
            const uint32_t wk[4] = {kk.x, kk.y, kk.z, kk.w};
            const uint32_t wq[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              a0 = fmaf(__uint_as_float(wq[e] << 16), __uint_as_float(wk[e] << 16), a0);
              a1 = fmaf(__uint_as_float(wq[e] & 0xffff0000u), __uint_as_float(wk[e] & 0xffff0000u), a1);
            }
          }
          sv = (a0 + a1) * p.scale2;
        }
        sm.s[h][t] = sv;
      }
      __syncthreads();
      // online softmax per head (warp per head): new max, rescale factor, probabilities
      for (int h = warp; h < G; h += kWarps) {
        const float x0 = sm.s[h][lane], x1 = sm.s[h][lane + 32];
        float mx = fmaxf(x0, x1);
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
        const float m_old = sm.m_run[h];
        const float m_new = fmaxf(m_old, mx);  // finite: the tile has at least one row
        const float p0 = lane < nt ? ex2(x0 - m_new) : 0.f;
        const float p1 = lane + 32 < nt ? ex2(x1 - m_new) : 0.f;
        sm.s[h][lane] = p0;
        sm.s[h][lane + 32] = p1;
        const float ps = warp_sum(p0 + p1);
        if (lane == 0) {
          const float a = m_old == -INFINITY ? 0.f : ex2(m_old - m_new);
          sm.alpha[h] = a;
          sm.l_run[h] = sm.l_run[h] * a + ps;
          sm.m_run[h] = m_new;
        }
      }
      __syncthreads();
      // acc = alpha * acc + P.V, 4 rows at a time (one 16-byte read of each head's P)
#pragma unroll
      for (int i = 0; i < kPH; ++i) {
        const int h = h0 + i * kHS;
        if (h < G) acc[i] *= sm.alpha[h];
      }
      const int nt4 = nt & ~3;
      for (int t = 0; t < nt4; t += 4) {
        float vv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) vv[u] = __bfloat162float(sm.vt[(t + u) * kKS + d]);
#pragma unroll
        for (int i = 0; i < kPH; ++i) {
          const int h = h0 + i * kHS;
          if (h < G) {
            const float4 p4 = *reinterpret_cast<const float4*>(&sm.s[h][t]);
            acc[i] = fmaf(p4.x, vv[0], acc[i]);
            acc[i] = fmaf(p4.y, vv[1], acc[i]);
            acc[i] = fmaf(p4.z, vv[2], acc[i]);
            acc[i] = fmaf(p4.w, vv[3], acc[i]);
          }
        }
      }
      for (int t = nt4; t < nt; ++t) {
        const float vv = __bfloat162float(sm.vt[t * kKS + d]);
#pragma unroll
        for (int i = 0; i < kPH; ++i) {
          const int h = h0 + i * kHS;
          if (h < G) acc[i] = fmaf(sm.s[h][t], vv, acc[i]);
        }
      }
    }
    __syncthreads();  // (m_run / l_run final)
    // this part's partial into the owners' tables (an empty range gives m = -inf, l = 0)
    for (int i = tid; i < kCL * G; i += kThreads) {
      const int peer = i / G, h = i - peer * G;
      st_cluster(map_rank(&sm.recv_ml[part][rank][h], peer), make_float2(sm.m_run[h], sm.l_run[h]));
    }
#pragma unroll
    for (int i = 0; i < kPH; ++i) {
      const int h = h0 + i * kHS;
      if (h < G) {
        const int e = h * D + d, owner = e / per_out;
        st_cluster(map_rank(&sm.recv_acc[part][rank][e - owner * per_out], owner), acc[i]);
      }
    }
  }
  cluster_arrive_release();  // every partial is in its owner's shared memory ...
  cluster_wait();            // ... and no CTA touches another's shared memory after this

  // merge my slice of the outputs: both branches, then the gated sum with the selection
  for (int le = tid; le < per_out; le += kThreads) {
    const int e = rank * per_out + le;
    const int h = e / D, dd = e - h * D;
    float ob[2], lb[2];
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      float M = -INFINITY;
#pragma unroll
      for (int c = 0; c < kCL; ++c) M = fmaxf(M, sm.recv_ml[part][c][h].x);
      float L = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int c = 0; c < kCL; ++c) {
          const float2 ml = sm.recv_ml[part][c][h];
          const float w = ml.x == -INFINITY ? 0.f : ex2(ml.x - M);
          L = fmaf(ml.y, w, L);
          O = fmaf(sm.recv_acc[part][c][le], w, O);
        }
      }
      ob[part] = L > 0.f ? O / L : 0.f;
      lb[part] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
    const size_t row = (size_t)b * Hq + (size_t)g * G + h;
    float out = p.g_win * ob[0] + p.g_cmp * ob[1];
    if (p.o_slc) out = fmaf(p.g_slc, __bfloat162float(p.o_slc[row * D + dd]), out);
    p.o[row * D + dd] = __float2bfloat16_rn(out);
    if (dd == 0) {
      if (p.lse_win) p.lse_win[row] = lb[0];
      if (p.lse_cmp) p.lse_cmp[row] = lb[1];
    }
  }
}

template <int D>
cudaError_t launch_branches(const NsaBranchArgs& a, cudaStream_t stream) {
  auto kernel = nsa_branches_kernel<D>;
  const int smem = (int)sizeof(BranchSmem<D>);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kCL, a.Hkv, a.B);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // the attributes and the occupancy check depend only on the kernel and its fixed block
  // shape: done once per device (the first launch on a device runs it, racing host threads
  // wait for it)
  static DeviceOnce check_once;
  const cudaError_t check_err = check_once.run([&]() {
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err == cudaSuccess) err = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    int nclusters = 0;
    if (err == cudaSuccess) err = cudaOccupancyMaxActiveClusters(&nclusters, kernel, &cfg);
    if (err == cudaSuccess && nclusters == 0) err = cudaErrorInvalidConfiguration;
    return err;
  });
  if (check_err != cudaSuccess) return check_err;
  BranchParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.kc = static_cast<const __nv_bfloat16*>(a.kc);
  p.vc = static_cast<const __nv_bfloat16*>(a.vc);
  p.seqlens = a.seqlens;
  p.o_slc = static_cast<const __nv_bfloat16*>(a.o_slc);
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse_win = a.lse_win;
  p.lse_cmp = a.lse_cmp;
  p.Hkv = a.Hkv; p.G = a.G; p.T_cap = a.T_cap;
  p.NC_cap = (a.T_cap + a.stride - 1) / a.stride;
  p.window = a.window; p.stride = a.stride;
  p.scale2 = a.scale * kLog2e;
  p.g_cmp = a.g_cmp; p.g_slc = a.g_slc; p.g_win = a.g_win;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

}  // namespace

cudaError_t launch_nsa_compress(const void* k, const void* v, int B, int Hkv, int T_cap, int D,
                                const int32_t* seqlens, int len, int stride, int nc_begin,
                                int nc_end, int range_max, void* kc, void* vc, cudaStream_t stream) {
  const int tok = kPoolThreads / (D / 8);
  const dim3 grid((range_max + tok - 1) / tok, Hkv, 2 * B);
  const auto* kk = static_cast<const __nv_bfloat16*>(k);
  const auto* vv = static_cast<const __nv_bfloat16*>(v);
  auto* kco = static_cast<__nv_bfloat16*>(kc);
  auto* vco = static_cast<__nv_bfloat16*>(vc);
  if (D == 128)
    nsa_compress_kernel<128><<<grid, kPoolThreads, 0, stream>>>(kk, vv, Hkv, T_cap, seqlens, len, stride,
                                                                nc_begin, nc_end, kco, vco);
  else
    nsa_compress_kernel<64><<<grid, kPoolThreads, 0, stream>>>(kk, vv, Hkv, T_cap, seqlens, len, stride,
                                                               nc_begin, nc_end, kco, vco);
  return cudaGetLastError();
}

cudaError_t launch_nsa_branches(const NsaBranchArgs& a, cudaStream_t stream) {
  return a.D == 128 ? launch_branches<128>(a, stream) : launch_branches<64>(a, stream);
}

LSA_BOUNDS_READER(nsa)

}  // namespace lsa
