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
// softmax over 64-row tiles (K and V by cp.async into a two-stage ring, the next tile in
// flight while the current one is used; logits and P.V on mma.sync m16n8k16 with the
// G <= 16 query heads as the 16 rows, zero-padded), then stores each branch's partial
// (m, l, acc) into the shared memory of the CTA that owns that part of the output.  After one cluster barrier each CTA merges its slice from its own shared
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
constexpr int kCL = 16;
constexpr int kMaxG = 16;
constexpr int kTile = 64;

constexpr int kSStride = 68;  // fp32 row stride of the logits tile

template <int D>
struct BranchSmem {
  static constexpr int kTileBytes = kTile * D * 2;
  // [stage][K, V]: 64 rows in the 128-byte-swizzled box layout of kv_off (ldmatrix over 8
  // consecutive rows is conflict-free)
  alignas(128) unsigned char kv[2][2][kTileBytes];
  alignas(128) unsigned char q[16 * D * 2];   // [16 rows][D], chunk-swizzled; rows >= G zero
  alignas(128) unsigned char pb[16 * kTile * 2];  // P (bf16) [16][64], chunk-swizzled
  float s[16][kSStride];                      // logits (base 2)
  float m_run[kMaxG], l_run[kMaxG], alpha[16];
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
  constexpr int kC = D / 8;               // 16-byte chunks per row
  constexpr int kRowBytes = D * 2;
  constexpr int NT = D / 64;              // n8 tiles of the output per warp
  extern __shared__ __align__(128) unsigned char smem_raw[];
  S& sm = *reinterpret_cast<S*>(smem_raw);
  const int rank = cluster_rank();
  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G, Hq = p.Hkv * G;
  const size_t unit = (size_t)b * p.Hkv + g;
  cluster_arrive_relaxed();  // peers' shared memory is written only after all have started

  for (int id = tid; id < 16 * kC; id += kThreads) {
    const int h = id / kC, c = id - h * kC;
    unsigned char* dst = sm.q + swz(h, c, kRowBytes);
    if (h < G)
      cp_async16(dst, p.q + ((size_t)b * Hq + (size_t)g * G + h) * D + c * 8, true);
    else
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
  cp_async_commit();
  const int T = checked_range(p.seqlens[b], 0, p.T_cap, kBoundsSeqlen, kSiteNsaBranches);
  const int nw = min(p.window, T);                  // window rows
  const int nc = (T + p.stride - 1) / p.stride;     // compressed rows
  const int R = nw + nc;
  const int per = (R + kCL - 1) / kCL;
  const int r0 = min(R, rank * per), r1 = min(R, r0 + per);
  const int per_out = G * D / kCL;                  // output elements each CTA merges
  const int srow = tid >> 4, ssub = tid & 15;       // softmax: row srow, keys 4 ssub .. + 3
  cluster_wait();  // (matches the arrive at the start) DSMEM is live from here on

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
    // rows t0 .. t0 + 63 of this part into stage st; rows past hi: K and V zero (P is 0
    // there, V must be finite)
    auto load_tile = [&](int t0, int st) {
      const int nt = min(kTile, hi - t0);
      for (int id = tid; id < kTile * kC; id += kThreads) {
        const int r = id / kC, c = id - r * kC;
        const int off = kv_off(r, c);
        if (r < nt) {
          const size_t src = (size_t)(t0 + r - roff) * D + c * 8;
          cp_async16(sm.kv[st][0] + off, ksrc + src, true);
          cp_async16(sm.kv[st][1] + off, vsrc + src, true);
        } else {
          *reinterpret_cast<uint4*>(sm.kv[st][0] + off) = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(sm.kv[st][1] + off) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      cp_async_commit();
    };
    __syncthreads();  // (the previous part's statistics have been pushed, its stages are free)
    if (lo < hi) load_tile(lo, 0);
    float m_run = -INFINITY, l_run = 0.f;  // (row srow; every thread of the row keeps them)
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
    int st = 0;
    for (int t0 = lo; t0 < hi; t0 += kTile, st ^= 1) {
      const int nt = min(kTile, hi - t0);
      __syncthreads();  // (the other stage, P and the logits of the previous tile are free)
      if (t0 + kTile < hi) {
        load_tile(t0 + kTile, st ^ 1);
        cp_async_wait<1>();  // this tile (and q) landed; the next one stays in flight
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const unsigned char* Ks = sm.kv[st][0];
      const unsigned char* Vs = sm.kv[st][1];
      // logits S = q K^T (base 2): warp w -> keys 8w .. 8w + 7
      {
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < D / 16; ks += 2) {
          uint32_t kb[4], qa0[4], qa1[4];
          ldsm_x4(kb, Ks + kv_off(8 * warp + (lane & 7), 2 * ks + (lane >> 3)));
          const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
          ldsm_x4(qa0, sm.q + swz(row, 2 * ks + (lane >> 4), kRowBytes));
          ldsm_x4(qa1, sm.q + swz(row, 2 * ks + 2 + (lane >> 4), kRowBytes));
          mma_bf16(sc, qa0, kb[0], kb[1]);
          mma_bf16(sc, qa1, kb[2], kb[3]);
        }
        const int col = 8 * warp + 2 * (lane & 3);
        const bool v0 = col < nt, v1 = col + 1 < nt;
        const int rr = lane >> 2;
        *reinterpret_cast<float2*>(&sm.s[rr][col]) =
            make_float2(v0 ? sc[0] * p.scale2 : -INFINITY, v1 ? sc[1] * p.scale2 : -INFINITY);
        *reinterpret_cast<float2*>(&sm.s[rr + 8][col]) =
            make_float2(v0 ? sc[2] * p.scale2 : -INFINITY, v1 ? sc[3] * p.scale2 : -INFINITY);
      }
      __syncthreads();
      // online softmax: 16 threads per row (a half warp), 4 keys each; rows >= G get P = 0
      {
        const float4 x = *reinterpret_cast<const float4*>(&sm.s[srow][4 * ssub]);
        float mx = fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w));
#pragma unroll
        for (int o2 = 8; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
        const float m_new = fmaxf(m_run, mx);  // finite: the tile has at least one row
        float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f, alpha = 1.f;
        if (srow < G) {
          p0 = ex2(x.x - m_new);
          p1 = ex2(x.y - m_new);
          p2 = ex2(x.z - m_new);
          p3 = ex2(x.w - m_new);
          alpha = m_run == -INFINITY ? 0.f : ex2(m_run - m_new);
        }
        float ps = (p0 + p1) + (p2 + p3);
#pragma unroll
        for (int o2 = 8; o2 > 0; o2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
        l_run = l_run * alpha + ps;
        m_run = m_new;
        *reinterpret_cast<uint2*>(sm.pb + swz(srow, ssub >> 1, kTile * 2) + 8 * (ssub & 1)) =
            make_uint2(pack_bf16x2(p0, p1), pack_bf16x2(p2, p3));
        if (ssub == 0) sm.alpha[srow] = alpha;
      }
      __syncthreads();
      // acc = alpha * acc + P V: warp w -> output dims 8 NT w .. 8 NT w + 8 NT - 1
      {
        const float a_lo = sm.alpha[lane >> 2], a_hi = sm.alpha[(lane >> 2) + 8];
#pragma unroll
        for (int n2 = 0; n2 < NT; ++n2) {
          acc[n2][0] *= a_lo; acc[n2][1] *= a_lo;
          acc[n2][2] *= a_hi; acc[n2][3] *= a_hi;
        }
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks) {
          const int vrow = 16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1);
          uint32_t vb[4], pa[4];
          if constexpr (NT == 2) {
            ldsm_x4_t(vb, Vs + kv_off(vrow, 2 * warp + (lane >> 4)));
          } else {
            uint32_t v2[2];
            ldsm_x2_t(v2, Vs + kv_off(vrow, warp));
            vb[0] = v2[0]; vb[1] = v2[1]; vb[2] = 0u; vb[3] = 0u;
          }
          const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
          ldsm_x4(pa, sm.pb + swz(row, 2 * ks + (lane >> 4), kTile * 2));
          mma_bf16(acc[0], pa, vb[0], vb[1]);
          if constexpr (NT == 2) mma_bf16(acc[1], pa, vb[2], vb[3]);
        }
      }
    }
    if (ssub == 0 && srow < G) {
      sm.m_run[srow] = m_run;
      sm.l_run[srow] = l_run;
    }
    __syncthreads();  // (m_run / l_run final)
    // this part's partial into the owners' tables (an empty range gives m = -inf, l = 0)
    for (int i = tid; i < kCL * G; i += kThreads) {
      const int peer = i / G, h = i - peer * G;
      st_cluster(map_rank(&sm.recv_ml[part][rank][h], peer), make_float2(sm.m_run[h], sm.l_run[h]));
    }
#pragma unroll
    for (int n2 = 0; n2 < NT; ++n2) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int h = (lane >> 2) + 8 * half;
        if (h < G) {
          const int e = h * D + 8 * NT * warp + 8 * n2 + 2 * (lane & 3), owner = e / per_out;
          st_cluster(map_rank(&sm.recv_acc[part][rank][e - owner * per_out], owner),
                     make_float2(acc[n2][2 * half], acc[n2][2 * half + 1]));
        }
      }
    }
  }
  cp_async_wait<0>();        // (q, when this CTA had no rows)
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
