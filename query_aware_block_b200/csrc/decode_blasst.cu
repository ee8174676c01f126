// decode_blasst.cu -- sparse decode attention over a given block selection with BLASST's
// softmax-threshold skip: a selected block whose scores trail the running maximum by more
// than -ln(lambda) for every query head of the GQA group is dropped before its V block is
// read (the decode kernel of BLASST, "2. 방법론" / "알고리즘 및 커널 설계", saves exactly
// those V loads, the memory traffic being what bounds decode).
//
// What is computed, for each (sequence b, KV head g): the selected blocks idx[b, g, :nsel]
// (ascending) are the KV blocks of a blockwise online softmax visited in that order.  For
// block s, r_h = the block's maximum logit of query head h and m_h = the maximum over the
// blocks visited before it (equal to the running maximum: a skipped block never raises
// it); the block is skipped iff it is not the first and max_h (r_h - m_h) < ln(lambda).
// The output is softmax attention over the tokens of the kept blocks.
//
// How (B200): one thread-block cluster of 16 CTAs per (b, g), CTA r owning selection slot
// r.  Each CTA loads q and its K block, computes the G x 64 logits and the G block maxima,
// and stores the maxima into every peer's shared memory (DSMEM); after one cluster barrier
// every CTA knows every block's maxima and evaluates its own block's test (the maximum
// over the earlier slots is the running maximum, so the sequential rule is decided in
// parallel).  Only kept blocks load V.  Each CTA stores its partial (m, l, acc) into the
// shared memory of the CTAs that own each slice of the outputs (DSMEM stores), and after
// one more cluster barrier every CTA merges its 1/16 of the outputs by log-sum-exp from its
// own shared memory.  The only waits are hardware cluster barriers that every thread of
// every CTA reaches.
#include <math.h>

#include "cluster.cuh"
#include "launch_cache.h"
#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCL = 16;      // CTAs per cluster = maximum selection slots
constexpr int kMaxG = 16;


template <int D>
struct Smem {
  static constexpr int kKS = D + 8;  // padded K/V row (bf16): conflict-free 16-byte reads
  __nv_bfloat16 kv[kBlk * kKS];      // the K block, then (if kept) the V block
  __nv_bfloat16 q[kMaxG * D];
  float s[kMaxG][kBlk];              // logits (base 2), then probabilities
  float rmax[kCL][kMaxG];            // every slot's block maxima (written by the peers)
  float rloc[kMaxG];                 // this CTA's block maxima
  float2 recv_ml[kCL][kMaxG];            // (m, l) of every CTA's partial, every head
  float recv_acc[kCL][kMaxG * D / kCL];  // every CTA's partial of this CTA's output slice
  int slot_block[kCL];               // the block of every slot, -1 if none
  uint32_t valid;                    // bit s: slot s holds a block
};

// Launched with clusters of kCL CTAs along x (grid (kCL, Hkv, B)).
template <int D>
__global__ void __launch_bounds__(kThreads)
    decode_blasst_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                         const __nv_bfloat16* __restrict__ v, int Hkv, int G, int T_cap,
                         const int32_t* __restrict__ seqlens, const int32_t* __restrict__ idx,
                         const int32_t* __restrict__ nsel, int topk, float scale2, float log2_lambda,
                         __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                         uint32_t* __restrict__ skip_bits) {
  using S = Smem<D>;
  constexpr int kKS = S::kKS;
  constexpr int kC = D / 8;  // 16-byte chunks per row
  __shared__ __align__(16) S sm;
  const int rank = cluster_rank();
  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hq = Hkv * G;
  const size_t unit = (size_t)b * Hkv + g;
  cluster_arrive_relaxed();  // peers' shared memory is written only after all have started

  // which slots hold a block (the same on every CTA): one load per lane of warp 0, all in
  // flight together; the q rows of the group start copying meanwhile
  for (int id = tid; id < G * kC; id += kThreads) {
    const int h = id / kC, c = id - h * kC;
    cp_async16(sm.q + h * D + c * 8, q + ((size_t)b * Hq + (size_t)g * G + h) * D + c * 8, true);
  }
  cp_async_commit();
  const int T = seqlens[b];
  if (warp == 0) {
    const int ns = nsel[unit];
    const int jj = lane < topk && lane < kCL ? idx[unit * topk + lane] : -1;
    const bool on = lane < ns && jj >= 0;
    const uint32_t bits = __ballot_sync(0xffffffffu, on);
    if (lane < kCL) sm.slot_block[lane] = on ? jj : -1;
    if (lane == 0) sm.valid = bits;
  }
  __syncthreads();
  const uint32_t valid = sm.valid;
  const bool has = (valid >> rank) & 1u;
  const int j = has ? sm.slot_block[rank] : 0;
  const int nv = has ? max(0, min(kBlk, T - j * kBlk)) : 0;  // valid rows of the block
  const size_t kvrow0 = unit * (size_t)T_cap + (size_t)j * kBlk;

  // the K block (rows past the sequence are not read), every copy in flight at once
  for (int id = tid; id < nv * kC; id += kThreads) {
    const int r = id / kC, c = id - r * kC;
    cp_async16(sm.kv + r * kKS + c * 8, k + (kvrow0 + r) * D + c * 8, true);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  // logits in base 2: pair (h, t) = (p >> 6, p & 63); a warp shares h (q reads broadcast)
  for (int p = tid; p < G * kBlk; p += kThreads) {
    const int h = p >> 6, t = p & (kBlk - 1);
    float acc = -INFINITY;
    if (t < nv) {
      float a0 = 0.f, a1 = 0.f;
      const __nv_bfloat16* kr = sm.kv + t * kKS;
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
      acc = (a0 + a1) * scale2;
    }
    sm.s[h][t] = acc;
  }
  __syncthreads();
  // block maxima (warp per head)
  for (int h = warp; h < G; h += kWarps) {
    float mx = fmaxf(sm.s[h][lane], sm.s[h][lane + 32]);
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
    if (lane == 0) sm.rloc[h] = mx;
  }
  __syncthreads();
  cluster_wait();  // (matches the arrive at the start) every CTA has started: DSMEM is live
  if (has) {       // this block's maxima into every CTA's table, row `rank`
    for (int i = tid; i < kCL * G; i += kThreads) {
      const int peer = i / G, h = i - peer * G;
      st_cluster(map_rank(&sm.rmax[rank][h], peer), sm.rloc[h]);
    }
  }
  cluster_arrive_release();  // the stores above are visible to every peer ...
  cluster_wait();            // ... once every CTA has passed here

  // the test for every slot (each CTA decides all of them; it acts on its own)
  uint32_t skipped = 0u;
  {
    float m_run[kMaxG];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) m_run[h] = -INFINITY;
    bool first = true;
    for (int s = 0; s < kCL; ++s) {
      if (!((valid >> s) & 1u)) continue;
      float gap = -INFINITY;
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) {
        if (h < G) {
          const float r = sm.rmax[s][h];
          const float gi = r == -INFINITY ? -INFINITY : (m_run[h] == -INFINITY ? INFINITY : r - m_run[h]);
          gap = fmaxf(gap, gi);
        }
      }
      if (!first && gap < log2_lambda) skipped |= 1u << s;
      first = false;
#pragma unroll
      for (int h = 0; h < kMaxG; ++h)
        if (h < G) m_run[h] = fmaxf(m_run[h], sm.rmax[s][h]);
    }
  }
  const bool keep = has && !((skipped >> rank) & 1u) && nv > 0;

  // V of a kept block (into the K buffer: the logits are done), softmax, P.V
  __syncthreads();
  if (keep) {
    for (int id = tid; id < nv * kC; id += kThreads) {
      const int r = id / kC, c = id - r * kC;
      cp_async16(sm.kv + r * kKS + c * 8, v + (kvrow0 + r) * D + c * 8, true);
    }
  }
  cp_async_commit();
  for (int h = warp; h < G; h += kWarps) {  // probabilities and row sums (warp per head)
    const float r = sm.rmax[rank][h];
    float p0 = 0.f, p1 = 0.f;
    if (keep) {
      p0 = lane < nv ? ex2(sm.s[h][lane] - r) : 0.f;
      p1 = lane + 32 < nv ? ex2(sm.s[h][lane + 32] - r) : 0.f;
    }
    sm.s[h][lane] = p0;
    sm.s[h][lane + 32] = p1;
    const float l = warp_sum(p0 + p1);
    if (lane < kCL)  // (m, l) of head h into every CTA's table, row `rank`
      st_cluster(map_rank(&sm.recv_ml[rank][h], lane), make_float2(keep ? r : -INFINITY, l));
  }
  cp_async_wait<0>();  // (the V copies overlapped the softmax above)
  __syncthreads();
  {
    // output element (h, d): thread takes d = tid % D and heads tid / D + k * (256 / D)
    constexpr int kHS = kThreads / D;  // 2 (D 128) or 4 (D 64)
    const int d = tid % D, h0 = tid / D;
    float acc[kMaxG / kHS];
#pragma unroll
    for (int i = 0; i < kMaxG / kHS; ++i) acc[i] = 0.f;
    if (keep) {
      // 4 keys at a time: one 16-byte read of each head's probabilities (a broadcast) per
      // 4 value reads; rows at or past nv hold no loaded value and are never read
      const int nv4 = nv & ~3;
      for (int t = 0; t < nv4; t += 4) {
        float vv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) vv[u] = __bfloat162float(sm.kv[(t + u) * kKS + d]);
#pragma unroll
        for (int i = 0; i < kMaxG / kHS; ++i) {
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
      for (int t = nv4; t < nv; ++t) {
        const float vv = __bfloat162float(sm.kv[t * kKS + d]);
#pragma unroll
        for (int i = 0; i < kMaxG / kHS; ++i) {
          const int h = h0 + i * kHS;
          if (h < G) acc[i] = fmaf(sm.s[h][t], vv, acc[i]);
        }
      }
    }
    // each output element's partial goes to the CTA that owns its slice of the outputs
    const int per = G * D / kCL;  // (G * D is a multiple of 16: D is 64 or 128)
#pragma unroll
    for (int i = 0; i < kMaxG / kHS; ++i) {
      const int h = h0 + i * kHS;
      if (h < G) {
        const int e = h * D + d, owner = e / per;
        st_cluster(map_rank(&sm.recv_acc[rank][e - owner * per], owner), acc[i]);
      }
    }
  }
  cluster_arrive_release();  // every partial has been stored into its owner ...
  cluster_wait();            // ... and after this no CTA touches another's shared memory

  // merge: this CTA's 1/16 of the G x D outputs, from its own shared memory
  const int per = G * D / kCL;
  for (int le = tid; le < per; le += kThreads) {
    const int e = rank * per + le;
    const int h = e / D, d = e - h * D;
    float pm[kCL], pl[kCL], pa[kCL];
#pragma unroll
    for (int c = 0; c < kCL; ++c) {
      const float2 ml = sm.recv_ml[c][h];
      pm[c] = ml.x;
      pl[c] = ml.y;
      pa[c] = sm.recv_acc[c][le];
    }
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kCL; ++c) M = fmaxf(M, pm[c]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int c = 0; c < kCL; ++c) {
        const float w = pm[c] == -INFINITY ? 0.f : ex2(pm[c] - M);
        L = fmaf(pl[c], w, L);
        O = fmaf(pa[c], w, O);
      }
    }
    const size_t row = (size_t)b * Hq + (size_t)g * G + h;
    o[row * D + d] = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
    if (d == 0 && lse) lse[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
  }
  if (rank == 0 && tid == 0 && skip_bits) skip_bits[unit] = skipped;
}

template <int D>
cudaError_t launch_d(const DecodeBlasstArgs& a, cudaStream_t stream) {
  auto kernel = decode_blasst_kernel<D>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kCL, a.Hkv, a.B);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // the cluster attribute and the occupancy check depend only on the kernel and its fixed
  // block shape: done once per device (the first launch on a device runs it, racing host
  // threads wait for it), so that a launch costs only the launch
  static DeviceOnce check_once;
  const cudaError_t check_err = check_once.run([&]() {
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    int nclusters = 0;
    if (err == cudaSuccess) err = cudaOccupancyMaxActiveClusters(&nclusters, kernel, &cfg);
    if (err == cudaSuccess && nclusters == 0) err = cudaErrorInvalidConfiguration;
    return err;
  });
  if (check_err != cudaSuccess) return check_err;
  const float scale2 = a.scale * kLog2e;
  const float log2_lambda = a.lambda > 0.f ? log2f(a.lambda) : -INFINITY;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<const __nv_bfloat16*>(a.q),
                            static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v),
                            a.Hkv, a.G, a.T_cap, a.seqlens, a.idx, a.nsel, a.topk, scale2, log2_lambda,
                            static_cast<__nv_bfloat16*>(a.o), a.lse, a.skip_bits);
}

}  // namespace

cudaError_t launch_decode_blasst(const DecodeBlasstArgs& a, cudaStream_t stream) {
  return a.D == 128 ? launch_d<128>(a, stream) : launch_d<64>(a, stream);
}

}  // namespace lsa
