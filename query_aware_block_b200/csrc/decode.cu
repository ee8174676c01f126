// decode.cu -- block selection and sparse decode attention, one thread-block cluster per
// (sequence b, KV head g).
//
// What is computed (NSA news article, "NSA 구조"; FASA "2. 방법론", FAC):
//   score_j   = scale * sum_{h in g} q_h . summ_j           (one selection per KV head,
//               shared by its G query heads)
//   selected  = forced {0..n_sink-1} U {NB-n_local..NB-1} plus the topk-|F| best others
//               (ties to the lower block index); all blocks when NB <= topk
//   o_h, lse_h = softmax attention of q_h over the tokens of the selected blocks
//
// How (B200):
//   * A cluster of CL CTAs (16, 8 or 4) owns one (b, g).  Each CTA scores a contiguous
//     slice of the NB block summaries with coalesced float4 loads (a warp per summary
//     row), keeps its local top-m (m = topk - |F|) as 64-bit keys, and the CTAs exchange
//     their sorted lists through distributed shared memory (DSMEM).  Every CTA derives the
//     same global top-m from the gathered lists by binary-search ranking.
//   * The selected blocks are dealt round-robin to the CTAs.  Forced blocks are known
//     before any score is read, so in fused mode their K/V copies are issued before the
//     summary scan and overlap it.
//   * A 64-token block of K and V (16 KB each at D = 128, bf16) is staged with 16-byte
//     cp.async into XOR-swizzled shared memory (2-stage pipeline).  For bf16 the G <= 16
//     query heads form the M = 16 rows of mma.sync m16n8k16 for S = Q K^T and O += P V;
//     the fp32 path uses CUDA-core FMA.  Online softmax in base 2, fp32 statistics.
//   * The per-CTA partial (m, l, acc) is merged across the cluster by log-sum-exp over
//     DSMEM; each CTA merges a 1/CL slice of the G x D outputs.
// No global scratch memory, no spin-waits: cross-CTA ordering uses cluster barriers only.
#include <cooperative_groups.h>

#include <math.h>

#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace cg = cooperative_groups;

namespace lsa {
namespace {

typedef unsigned long long u64;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 16;      // query-head rows per group (G <= 16): the mma M dimension
constexpr int kMaxTopk = 64;
constexpr int kMaxCluster = 16;
constexpr int kStages = 2;
constexpr int kSStride = 72;   // fp32 row stride of the score tile (bank spread)

struct Params {
  const void* q;
  const void* k;
  const void* v;
  int Hkv, G, T_cap, NB_cap;
  const int32_t* seqlens;
  const float* summ;
  const int32_t* idx_in;
  const int32_t* nsel_in;
  int topk, n_sink, n_local;
  float scale;       // natural-log softmax scale
  int32_t* idx_out;
  int32_t* nsel_out;
  float* scores_out;
  void* o;
  float* lse;
  int per_max;       // max summary rows scored by one CTA
  int m_pad;         // power of two >= topk
};

__host__ __device__ inline size_t align128(size_t x) { return (x + 127) & ~(size_t)127; }

// Shared-memory carve-up (byte offsets), identical on host and device.
struct Layout {
  size_t qs, qsum, keys, top, work, all, gtop, order, kv, ss, ps, alpha, pm, pl, pacc, total;
  size_t kv_row, kv_tile;  // bytes per K/V row in smem, bytes per 64-row tile
};

__host__ __device__ inline Layout make_layout(int elem_bytes, int D, int per_max, int m_pad) {
  Layout L;
  size_t off = 0;
  const bool f32 = elem_bytes == 4;
  L.kv_row = f32 ? (size_t)(D + 4) * 4 : (size_t)D * 2;
  L.kv_tile = L.kv_row * kBlk;
  L.qs = off;    off = align128(off + (size_t)kRows * D * elem_bytes);
  L.qsum = off;  off = align128(off + (size_t)D * 4);
  L.keys = off;  off = align128(off + (size_t)per_max * 8);
  L.top = off;   off = align128(off + (size_t)m_pad * 8);
  L.work = off;  off = align128(off + (size_t)(m_pad + kThreads) * 8);
  L.all = off;   off = align128(off + (size_t)kMaxCluster * m_pad * 8);
  L.gtop = off;  off = align128(off + (size_t)m_pad * 8);
  L.order = off; off = align128(off + (size_t)kMaxTopk * 4);
  L.kv = off;    off = align128(off + (size_t)kStages * 2 * L.kv_tile);
  L.ss = off;    off = align128(off + (size_t)kRows * kSStride * 4);
  L.ps = off;    off = align128(off + (size_t)kRows * kBlk * 4);
  L.alpha = off; off = align128(off + (size_t)kRows * 4);
  L.pm = off;    off = align128(off + (size_t)kRows * 4);
  L.pl = off;    off = align128(off + (size_t)kRows * 4);
  L.pacc = off;  off = align128(off + (size_t)kRows * D * 4);
  L.total = off;
  return L;
}

// ---- selection helpers ------------------------------------------------------------------

// Top-m of n keys (0 = not a candidate) into top[0..min(m, #valid)), descending.
// top[] must be zero on entry.  Candidates are taken kThreads at a time together with the
// current top list; each candidate's rank is the count of larger keys (keys are unique).
__device__ void block_topm(const u64* keys, int n, int m, u64* top, u64* work) {
  int cur = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int cn = min(kThreads, n - base);
    const int w = cur + cn;
    for (int i = threadIdx.x; i < w; i += kThreads) work[i] = i < cur ? top[i] : keys[base + i - cur];
    __syncthreads();
    int nvalid = 0;
    for (int i0 = 0; i0 < w; i0 += kThreads) {
      const int i = i0 + threadIdx.x;
      const u64 x = (i < w) ? work[i] : 0ull;
      if (x != 0ull) {
        int r = 0;
        for (int u = 0; u < w; ++u) r += work[u] > x;
        if (r < m) top[r] = x;
      }
      nvalid += __syncthreads_count(x != 0ull);
    }
    cur = min(m, nvalid);
  }
  __syncthreads();
}

// Number of entries greater than x in a descending, zero-padded list of n (power of 2).
__device__ __forceinline__ int count_greater(const u64* L, int n, u64 x) {
  int lo = 0;
  for (int step = n >> 1; step > 0; step >>= 1)
    if (L[lo + step - 1] > x) lo += step;
  if (L[lo] > x) ++lo;
  return lo;
}

// ---- K/V block staging ----------------------------------------------------------------

// Copy the K and V rows of block j into a stage (rows >= Tb are zero-filled and never
// read from global memory).  bf16 rows are chunk-swizzled; fp32 rows are padded.
template <typename T, int D>
__device__ __forceinline__ void stage_block(unsigned char* dst_k, unsigned char* dst_v,
                                            const T* kbase, const T* vbase, int j, int Tb,
                                            int kv_row) {
  constexpr int kChunks = D * (int)sizeof(T) / 16;  // 16-byte chunks per row
  constexpr int kTotal = 2 * kBlk * kChunks;
  constexpr bool kF32 = sizeof(T) == 4;
#pragma unroll
  for (int it = 0; it < kTotal / kThreads; ++it) {
    const int id = threadIdx.x + it * kThreads;
    const int tensor = id / (kBlk * kChunks);
    const int rem = id % (kBlk * kChunks);
    const int row = rem / kChunks, c = rem % kChunks;
    const int t = j * kBlk + row;
    const bool valid = j >= 0 && t < Tb;
    const T* src = (tensor ? vbase : kbase) + (size_t)(valid ? t : 0) * D + c * (16 / sizeof(T));
    unsigned char* dst = (tensor ? dst_v : dst_k) + (kF32 ? row * kv_row + c * 16 : swz(row, c, kv_row));
    cp_async16(dst, src, valid);
  }
}

// ---- the kernel ---------------------------------------------------------------------

template <typename T, int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1) decode_cluster_kernel(const Params p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  const int Tb = p.seqlens[b];
  const int NB = (Tb + kBlk - 1) / kBlk;
  constexpr bool kF32 = sizeof(T) == 4;
  constexpr int kRowBytesQ = D * (int)sizeof(T);

  extern __shared__ __align__(1024) unsigned char smem[];
  const Layout Lo = make_layout((int)sizeof(T), D, p.per_max, p.m_pad);
  unsigned char* Qs = smem + Lo.qs;
  float* qsum = reinterpret_cast<float*>(smem + Lo.qsum);
  u64* keys = reinterpret_cast<u64*>(smem + Lo.keys);
  u64* top = reinterpret_cast<u64*>(smem + Lo.top);
  u64* work = reinterpret_cast<u64*>(smem + Lo.work);
  u64* all = reinterpret_cast<u64*>(smem + Lo.all);
  u64* gtop = reinterpret_cast<u64*>(smem + Lo.gtop);
  int* order = reinterpret_cast<int*>(smem + Lo.order);
  unsigned char* kv = smem + Lo.kv;
  float* Ss = reinterpret_cast<float*>(smem + Lo.ss);
  unsigned char* Ps = smem + Lo.ps;
  float* alpha_s = reinterpret_cast<float*>(smem + Lo.alpha);
  float* pm = reinterpret_cast<float*>(smem + Lo.pm);
  float* pl = reinterpret_cast<float*>(smem + Lo.pl);
  float* pacc = reinterpret_cast<float*>(smem + Lo.pacc);
  const int kv_row = (int)Lo.kv_row;
  const int kv_tile = (int)Lo.kv_tile;

  const size_t unit = (size_t)b * p.Hkv + g;
  const T* qg = static_cast<const T*>(p.q) + ((size_t)b * p.Hkv * G + (size_t)g * G) * D;
  const T* kbase = static_cast<const T*>(p.k) + unit * (size_t)p.T_cap * D;
  const T* vbase = static_cast<const T*>(p.v) + unit * (size_t)p.T_cap * D;

  // ---- the forced set and the block order ------------------------------------------------
  // order[0..n_order) lists the blocks to attend; order[i] is handled by CTA i % CL.
  const bool select = MODE != MODE_ATTEND;
  const bool all_blocks = select && NB <= p.topk;
  int nf = 0, n_order = 0;
  if (select) {
    if (all_blocks) {
      for (int i = tid; i < NB; i += kThreads) order[i] = i;
      n_order = NB;
    } else {
      // NB > topk >= n_sink + n_local: the two forced ranges are disjoint
      nf = p.n_sink + p.n_local;
      for (int i = tid; i < nf; i += kThreads) order[i] = i < p.n_sink ? i : NB - p.n_local + (i - p.n_sink);
      n_order = p.topk;
    }
  } else {
    const int ns = max(0, min(p.nsel_in[unit], p.topk));  // never past order[kMaxTopk]
    for (int i = tid; i < ns; i += kThreads) order[i] = p.idx_in[unit * p.topk + i];
    n_order = ns;
  }
  // query rows (zero rows beyond G): bf16 swizzled for ldmatrix, fp32 plain
  if (MODE != MODE_SELECT) {
    constexpr int kQChunks = kRows * kRowBytesQ / 16;
    for (int id = tid; id < kQChunks; id += kThreads) {
      const int row = id / (kRowBytesQ / 16), c = id % (kRowBytesQ / 16);
      const bool valid = row < G;
      const T* src = qg + (size_t)(valid ? row : 0) * D + c * (16 / sizeof(T));
      unsigned char* dst = Qs + (kF32 ? row * kRowBytesQ + c * 16 : swz(row, c, kRowBytesQ));
      cp_async16(dst, src, valid);
    }
    cp_async_commit();
  }
  __syncthreads();

  // ---- prefetch the blocks already known (forced, or all) ------------------------------
  int issued = 0;  // number of my blocks whose copies were committed
  auto my_block = [&](int i) { return order[rank + i * CL]; };
  int n_my_known = 0;
  if (MODE == MODE_FUSED) {
    const int known = all_blocks ? n_order : nf;
    n_my_known = known > rank ? (known - rank + CL - 1) / CL : 0;
    while (issued < kStages && issued < n_my_known) {
      const int j = my_block(issued);
      unsigned char* st = kv + (size_t)(issued % kStages) * 2 * kv_tile;
      stage_block<T, D>(st, st + kv_tile, kbase, vbase, j, Tb, kv_row);
      cp_async_commit();
      ++issued;
    }
  }

  // ---- selection ----------------------------------------------------------------------
  if (select && !all_blocks) {
    const int m = p.topk - nf;
    // summed, scaled query of the group
    for (int d = tid; d < D; d += kThreads) {
      float s = 0.f;
      for (int h = 0; h < G; ++h) s += to_f32(qg[(size_t)h * D + d]);
      qsum[d] = s * p.scale;
    }
    for (int i = tid; i < p.m_pad; i += kThreads) top[i] = 0ull;
    __syncthreads();
    constexpr int VEC = D / 32;  // floats per lane per summary row
    float qv[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) qv[e] = qsum[lane * VEC + e];
    const int per = (NB + CL - 1) / CL;
    const int j0 = rank * per;
    const int nloc = max(0, min(NB, j0 + per) - j0);
    const float* sb = p.summ + unit * (size_t)p.NB_cap * D + lane * VEC;
    constexpr int kUnroll = 8;
    for (int o0 = warp; o0 < nloc; o0 += kWarps * kUnroll) {
      float vals[kUnroll][VEC];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int oo = o0 + u * kWarps;
        if (oo < nloc) {
          const float* src = sb + (size_t)(j0 + oo) * D;
          if constexpr (VEC == 4) {
            const float4 t4 = __ldg(reinterpret_cast<const float4*>(src));
            vals[u][0] = t4.x; vals[u][1] = t4.y; vals[u][2] = t4.z; vals[u][3] = t4.w;
          } else {
            const float2 t2 = __ldg(reinterpret_cast<const float2*>(src));
            vals[u][0] = t2.x; vals[u][1] = t2.y;
          }
        } else {
#pragma unroll
          for (int e = 0; e < VEC; ++e) vals[u][e] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int oo = o0 + u * kWarps;
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) dot = fmaf(vals[u][e], qv[e], dot);
        dot = warp_sum(dot);
        if (oo < nloc && lane == 0) {
          const int j = j0 + oo;
          const bool forced = j < p.n_sink || j >= NB - p.n_local;
          keys[oo] = forced ? 0ull : make_key(dot, j);
          if (p.scores_out) p.scores_out[unit * p.NB_cap + j] = dot;
        }
      }
    }
    __syncthreads();
    block_topm(keys, nloc, m, top, work);
    cluster.sync();  // every CTA's local list is complete
    // gather all lists and rank every candidate among them
    const int nall = CL * p.m_pad;
    for (int t = tid; t < nall; t += kThreads) {
      const u64* peer = cluster.map_shared_rank(top, t / p.m_pad);
      all[t] = peer[t % p.m_pad];
    }
    __syncthreads();
    for (int t = tid; t < nall; t += kThreads) {
      const u64 x = all[t];
      if (x == 0ull) continue;
      const int c = t / p.m_pad;
      int r = t % p.m_pad;
      for (int l = 0; l < CL; ++l)
        if (l != c) r += count_greater(all + l * p.m_pad, p.m_pad, x);
      if (r < m) gtop[r] = x;
    }
    __syncthreads();
    for (int r = tid; r < m; r += kThreads) order[nf + r] = key_block(gtop[r]);
    __syncthreads();
  }

  // selected indices, ascending (written by rank 0)
  if (select && rank == 0) {
    int32_t* out = p.idx_out ? p.idx_out + unit * p.topk : nullptr;
    if (out) {
      for (int i = tid; i < p.topk; i += kThreads) {
        if (i < n_order) {
          const int v = order[i];
          int pos = 0;
          for (int u = 0; u < n_order; ++u) pos += order[u] < v;
          out[pos] = v;
        } else {
          out[i] = -1;
        }
      }
    }
    if (MODE == MODE_SELECT && tid == 0) p.nsel_out[unit] = n_order;
  }
  if (MODE == MODE_SELECT) {
    cluster.sync();  // peers may still be reading this CTA's list
    return;
  }

  // ---- attention over my share of the blocks ------------------------------------------
  const int n_my = n_order > rank ? (n_order - rank + CL - 1) / CL : 0;
  while (issued < kStages && issued < n_my) {
    const int j = my_block(issued);
    unsigned char* st = kv + (size_t)(issued % kStages) * 2 * kv_tile;
    stage_block<T, D>(st, st + kv_tile, kbase, vbase, j, Tb, kv_row);
    cp_async_commit();
    ++issued;
  }
  // the query copy was committed before every K/V copy: wait for it alone
  if (issued >= 2) cp_async_wait<2>();
  else if (issued == 1) cp_async_wait<1>();
  else cp_async_wait<0>();
  __syncthreads();

  const float scale2 = p.scale * kLog2e;
  float m_run = -INFINITY, l_run = 0.f;  // softmax row state (row = tid >> 4)
  const int srow = tid >> 4, ssub = tid & 15;
  // bf16 path: query A fragments and output accumulators in registers
  constexpr int NT = kF32 ? 1 : D / 64;  // n8 tiles of the output per warp
  uint32_t qa[kF32 ? 1 : D / 16][4];
  float acc[kF32 ? D / 16 : NT][kF32 ? 1 : 4];
  if constexpr (kF32) {
#pragma unroll
    for (int i = 0; i < D / 16; ++i) acc[i][0] = 0.f;
  } else {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
    if (n_my > 0) {
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
        ldsm_x4(qa[ks], Qs + swz(row, 2 * ks + (lane >> 4), kRowBytesQ));
      }
    }
  }

  for (int i = 0; i < n_my; ++i) {
    if (issued > i + 1) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncthreads();
    const int j = my_block(i);
    const unsigned char* Ks = kv + (size_t)(i % kStages) * 2 * kv_tile;
    const unsigned char* Vs = Ks + kv_tile;

    // S = scale2 * Q K^T (masked past Tb) -> Ss
    if constexpr (kF32) {
      const int tok = tid & 63, rg = tid >> 6;  // 4 rows per thread
      const float* Kr = reinterpret_cast<const float*>(Ks + tok * kv_row);
      const float* Qf = reinterpret_cast<const float*>(Qs);
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int d = 0; d < D; d += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(Kr + d);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 q4 = *reinterpret_cast<const float4*>(Qf + (rg * 4 + r) * D + d);
          s[r] = fmaf(q4.x, k4.x, fmaf(q4.y, k4.y, fmaf(q4.z, k4.z, fmaf(q4.w, k4.w, s[r]))));
        }
      }
      const bool valid = j >= 0 && j * kBlk + tok < Tb;
#pragma unroll
      for (int r = 0; r < 4; ++r) Ss[(rg * 4 + r) * kSStride + tok] = valid ? s[r] * scale2 : -INFINITY;
    } else {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < D / 16; ks += 2) {
        uint32_t kb[4];
        ldsm_x4(kb, Ks + swz(8 * warp + (lane & 7), 2 * ks + (lane >> 3), kv_row));
        mma_bf16(s, qa[ks], kb[0], kb[1]);
        mma_bf16(s, qa[ks + 1], kb[2], kb[3]);
      }
      const int col = 8 * warp + 2 * (lane & 3);
      const int r0 = lane >> 2;
      const bool v0 = j >= 0 && j * kBlk + col < Tb, v1 = j >= 0 && j * kBlk + col + 1 < Tb;
      *reinterpret_cast<float2*>(Ss + r0 * kSStride + col) =
          make_float2(v0 ? s[0] * scale2 : -INFINITY, v1 ? s[1] * scale2 : -INFINITY);
      *reinterpret_cast<float2*>(Ss + (r0 + 8) * kSStride + col) =
          make_float2(v0 ? s[2] * scale2 : -INFINITY, v1 ? s[3] * scale2 : -INFINITY);
    }
    __syncthreads();

    // online softmax, row srow, columns 4*ssub .. 4*ssub+3
    {
      const float4 s4 = *reinterpret_cast<const float4*>(Ss + srow * kSStride + 4 * ssub);
      float mx = fmaxf(fmaxf(s4.x, s4.y), fmaxf(s4.z, s4.w));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m_run, mx);
      float alpha = 1.f, p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
      if (m_new != -INFINITY) {
        alpha = ex2(m_run - m_new);
        p0 = ex2(s4.x - m_new); p1 = ex2(s4.y - m_new);
        p2 = ex2(s4.z - m_new); p3 = ex2(s4.w - m_new);
      }
      float ps = (p0 + p1) + (p2 + p3);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      l_run = l_run * alpha + ps;
      m_run = m_new;
      if constexpr (kF32) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(Ps) + srow * kBlk + 4 * ssub) =
            make_float4(p0, p1, p2, p3);
      } else {
        *reinterpret_cast<uint2*>(Ps + swz(srow, ssub >> 1, kBlk * 2) + (ssub & 1) * 8) =
            make_uint2(pack_bf16x2(p0, p1), pack_bf16x2(p2, p3));
      }
      if (ssub == 0) alpha_s[srow] = alpha;
    }
    __syncthreads();

    // O = alpha * O + P V
    if constexpr (kF32) {
      const float a = alpha_s[srow];
      const float* Pf = reinterpret_cast<const float*>(Ps) + srow * kBlk;
#pragma unroll
      for (int e = 0; e < D / 16; ++e) acc[e][0] *= a;
      for (int t = 0; t < kBlk; ++t) {
        const float pt = Pf[t];
        const float* Vr = reinterpret_cast<const float*>(Vs + t * kv_row);
#pragma unroll
        for (int e = 0; e < D / 16; ++e) acc[e][0] = fmaf(pt, Vr[ssub + 16 * e], acc[e][0]);
      }
    } else {
      const float a_lo = alpha_s[lane >> 2], a_hi = alpha_s[(lane >> 2) + 8];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[nt][0] *= a_lo; acc[nt][1] *= a_lo;
        acc[nt][2] *= a_hi; acc[nt][3] *= a_hi;
      }
#pragma unroll
      for (int ks = 0; ks < kBlk / 16; ++ks) {
        uint32_t pa[4];
        const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
        ldsm_x4(pa, Ps + swz(row, 2 * ks + (lane >> 4), kBlk * 2));
        const int vrow = 16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1);
        if constexpr (D == 128) {
          uint32_t vb[4];
          ldsm_x4_t(vb, Vs + swz(vrow, 2 * warp + (lane >> 4), kv_row));
          mma_bf16(acc[0], pa, vb[0], vb[1]);
          mma_bf16(acc[1], pa, vb[2], vb[3]);
        } else {
          uint32_t vb[2];
          ldsm_x2_t(vb, Vs + swz(vrow, warp, kv_row));
          mma_bf16(acc[0], pa, vb[0], vb[1]);
        }
      }
    }
    __syncthreads();  // the stage may now be refilled
    if (issued < n_my) {
      const int jn = my_block(issued);
      unsigned char* st = kv + (size_t)(issued % kStages) * 2 * kv_tile;
      stage_block<T, D>(st, st + kv_tile, kbase, vbase, jn, Tb, kv_row);
      cp_async_commit();
      ++issued;
    }
  }

  // ---- partial (m, l, acc) of this CTA -> shared memory ---------------------------------
  if (ssub == 0) {
    pm[srow] = m_run;
    pl[srow] = l_run;
  }
  if constexpr (kF32) {
#pragma unroll
    for (int e = 0; e < D / 16; ++e) pacc[srow * D + ssub + 16 * e] = acc[e][0];
  } else {
    const int r0 = lane >> 2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int d = (D == 128 ? 16 * warp : 8 * warp) + 8 * nt + 2 * (lane & 3);
      *reinterpret_cast<float2*>(pacc + r0 * D + d) = make_float2(acc[nt][0], acc[nt][1]);
      *reinterpret_cast<float2*>(pacc + (r0 + 8) * D + d) = make_float2(acc[nt][2], acc[nt][3]);
    }
  }
  cluster.sync();

  // ---- log-sum-exp merge of the CL partials; this CTA writes a 1/CL slice -----------
  {
    const int E = G * D;
    const int chunk = (E + CL - 1) / CL;
    const int e_end = min(E, (rank + 1) * chunk);
    T* og = static_cast<T*>(p.o) + ((size_t)b * p.Hkv * G + (size_t)g * G) * D;
    for (int e = rank * chunk + tid; e < e_end; e += kThreads) {
      const int h = e / D, d = e % D;
      float mp[kMaxCluster];
      float M = -INFINITY;
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) {
        mp[r] = -INFINITY;
        if (r < CL) {
          mp[r] = *cluster.map_shared_rank(pm + h, r);
          M = fmaxf(M, mp[r]);
        }
      }
      float Lsum = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
          if (r < CL) {
            const float w = ex2(mp[r] - M);
            Lsum = fmaf(*cluster.map_shared_rank(pl + h, r), w, Lsum);
            O = fmaf(*cluster.map_shared_rank(pacc + h * D + d, r), w, O);
          }
        }
      }
      og[(size_t)h * D + d] = from_f32<T>(M == -INFINITY ? 0.f : O / Lsum);
      if (d == 0 && p.lse)
        p.lse[(size_t)b * p.Hkv * G + (size_t)g * G + h] =
            M == -INFINITY ? -INFINITY : (M + log2f(Lsum)) * kLn2;
    }
  }
  cluster.sync();  // keep this CTA's shared memory alive until every peer has read it
}

// ---- host side --------------------------------------------------------------------------

int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

template <typename T, int D, int MODE>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t stream) {
  auto kernel = decode_cluster_kernel<T, D, MODE>;
  // cluster size: many CTAs per unit when there are few units
  const int units = a.B * a.Hkv;
  int CL = units <= 18 ? 16 : (units <= 74 ? 8 : 4);
  Params p;
  p.q = a.q; p.k = a.k; p.v = a.v;
  p.Hkv = a.Hkv; p.G = a.G; p.T_cap = a.T_cap; p.NB_cap = a.NB_cap;
  p.seqlens = a.seqlens; p.summ = a.summ; p.idx_in = a.idx_in; p.nsel_in = a.nsel_in;
  p.topk = a.topk; p.n_sink = a.n_sink; p.n_local = a.n_local; p.scale = a.scale;
  p.idx_out = a.idx_out; p.nsel_out = a.nsel_out; p.scores_out = a.scores_out;
  p.o = a.o; p.lse = a.lse;
  p.m_pad = next_pow2(a.topk < 2 ? 2 : a.topk);
  // per template instance: the largest dynamic smem size set so far, and the last
  // (cluster size, smem) pair whose occupancy was checked
  static int smem_set = 0;
  static int last_cl = 0, last_smem = -1;
  cudaError_t err;
  for (;;) {
    p.per_max = (a.NB_cap + CL - 1) / CL;
    const Layout Lo = make_layout((int)sizeof(T), D, p.per_max, p.m_pad);
    const int smem = (int)Lo.total;
    if (smem > smem_set) {
      err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (err != cudaSuccess) return err;
      err = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (err != cudaSuccess) return err;
      smem_set = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL, a.Hkv, a.B);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (!(CL == last_cl && smem == last_smem)) {
      int nclusters = 0;
      err = cudaOccupancyMaxActiveClusters(&nclusters, kernel, &cfg);
      if (err != cudaSuccess || nclusters == 0) {
        (void)cudaGetLastError();
        if (CL > 2) {
          CL >>= 1;
          continue;
        }
        return err != cudaSuccess ? err : cudaErrorInvalidConfiguration;
      }
      last_cl = CL;
      last_smem = smem;
    }
    return cudaLaunchKernelEx(&cfg, kernel, p);
  }
}

template <typename T, int D>
cudaError_t launch_mode(const DecodeArgs& a, cudaStream_t s) {
  switch (a.mode) {
    case MODE_SELECT: return launch_t<T, D, MODE_SELECT>(a, s);
    case MODE_ATTEND: return launch_t<T, D, MODE_ATTEND>(a, s);
    default: return launch_t<T, D, MODE_FUSED>(a, s);
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.B == 0 || a.Hkv == 0) return cudaSuccess;
  if (a.dtype == DT_BF16) {
    if (a.D == 128) return launch_mode<__nv_bfloat16, 128>(a, stream);
    return launch_mode<__nv_bfloat16, 64>(a, stream);
  }
  if (a.D == 128) return launch_mode<float, 128>(a, stream);
  return launch_mode<float, 64>(a, stream);
}

}  // namespace lsa
