// blockquery.cu -- one denoising step of a block of Tq query tokens against a cached
// prefix (block-wise diffusion LM), one thread-block cluster per (sequence b, KV head g).
//
// What is computed (LoSA, "1. 문제 정의" and "2. 방법론"):
//   active token i (active[b, i] != 0) selects, per KV group g, its top-k prefix blocks by
//     s_i(j) = scale * sum_{h in g} q[b, h, i, :] . summ[b, g, j, :]   (forced blocks kept);
//   U(b, g) = the union of those selections over the active tokens (deduplicated);
//   every active row (i, h in g) attends over all prefix tokens of the blocks in U(b, g);
//   stable rows (active == 0) keep the cached output and log-sum-exp, bit-exactly.
//
// How (B200):
//   * Each CTA of the cluster owns a contiguous slice of the prefix blocks.  It scores its
//     slice for every active token (a warp per summary row, coalesced float4), keeps each
//     token's local top-k as 64-bit keys, and pushes the lists to every peer through
//     distributed shared memory.  After one cluster barrier a batched tree of warp-wide
//     bitonic merges yields every token's global k-th best key: the token's threshold.
//   * A block of this CTA's slice is in the union iff some active token's key for it
//     clears that token's threshold, so every CTA decides its own part of the union from
//     the scores it already holds and attends exactly those blocks: the union is loaded
//     from HBM once, spread over the cluster, with no redistribution.
//   * Attention rows (active token x head) are processed 32 at a time (two mma m-tiles):
//     K/V blocks are staged with cp.async into swizzled shared memory (2 stages, prefetch
//     across row chunks; later chunks re-read the blocks from L2), S = Q K^T and O += P V
//     on mma.sync m16n8k16 bf16, online softmax in base 2.
//   * Each CTA writes its per-row partial (acc, m, l) to the caller's workspace; after a
//     second cluster barrier every CTA merges a 1/CL slice of the outputs by log-sum-exp.
//     Stable rows are copied from the cache, the union list is written by offsets that the
//     CTAs exchange over DSMEM.
#include <math.h>

#include <mutex>

#include "cluster.cuh"
#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {
namespace {

typedef unsigned long long u64;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTokChunk = 8;    // active tokens per selection exchange
constexpr int kRowChunk = 32;   // attention rows per pass (two mma m-tiles)
constexpr int kLP = 16;         // length of an exchanged list (topk_per_query <= 16)
constexpr int kMaxCluster = 16;
constexpr int kMaxTq = 64;
constexpr int kStages = 2;
constexpr int kSStride = 68;    // fp32 row stride of the score tile

struct BQParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  int Hkv, G, Tq, T_prefix, T_cap, NB_cap;
  const float* summ;
  int topk, n_sink, n_local;
  float scale;
  const uint8_t* active;
  const __nv_bfloat16* o_cache;
  const float* lse_cache;
  __nv_bfloat16* o;
  float* lse;
  int32_t* union_idx;
  int32_t* union_cnt;
  float* ws;       // [B][Hkv][kMaxCluster][rows_max][D + 2]
  int rows_max;    // Tq * G
  int per_max;     // max prefix blocks in one CTA's slice
};

__host__ __device__ inline size_t al128(size_t x) { return (x + 127) & ~(size_t)127; }

struct BQLayout {
  size_t act, stab, ulist, cnt_in, thr, qs, ss, ps, alpha, region, total;
  // selection buffers, inside `region` (dead once the attention starts)
  size_t qsum, keys, top, recv, work, inu;
  size_t kv_tile;
};

__host__ __device__ inline BQLayout bq_layout(int D, int per_max) {
  BQLayout L;
  size_t off = 0;
  L.act = off;    off = al128(off + kMaxTq * 4);
  L.stab = off;   off = al128(off + kMaxTq * 4);
  L.ulist = off;  off = al128(off + (size_t)per_max * 4);
  L.cnt_in = off; off = al128(off + kMaxCluster * 4);
  L.thr = off;    off = al128(off + kTokChunk * 8);
  L.qs = off;     off = al128(off + (size_t)kRowChunk * D * 2);
  L.ss = off;     off = al128(off + (size_t)kRowChunk * kSStride * 4);
  L.ps = off;     off = al128(off + (size_t)kRowChunk * kBlk * 2);
  L.alpha = off;  off = al128(off + kRowChunk * 4);
  L.region = off;
  L.kv_tile = (size_t)kBlk * D * 2;
  const size_t kv_bytes = kStages * 2 * L.kv_tile;
  size_t r = 0;
  L.qsum = r; r = al128(r + (size_t)kTokChunk * D * 4);
  L.keys = r; r = al128(r + (size_t)kTokChunk * per_max * 8);
  L.top = r;  r = al128(r + (size_t)kTokChunk * kLP * 8);
  L.recv = r; r = al128(r + (size_t)kMaxCluster * kTokChunk * kLP * 8);
  L.work = r; r = al128(r + (size_t)kTokChunk * (kMaxCluster / 2) * kLP * 8);
  L.inu = r;  r = al128(r + (size_t)per_max);
  L.total = off + (r > kv_bytes ? r : kv_bytes);
  return L;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2) blockquery_kernel(const BQParams p) {
  const int CL = cluster_size();
  const int rank = cluster_rank();
  cluster_arrive_relaxed();  // DSMEM is written only after every CTA has started
  bool started = false;

  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G, Tq = p.Tq, Hq = p.Hkv * G;
  const size_t unit = (size_t)b * p.Hkv + g;

  extern __shared__ __align__(1024) unsigned char smem[];
  const BQLayout Lo = bq_layout(D, p.per_max);
  int* act = reinterpret_cast<int*>(smem + Lo.act);
  int* stab = reinterpret_cast<int*>(smem + Lo.stab);
  int* ulist = reinterpret_cast<int*>(smem + Lo.ulist);
  int* cnt_in = reinterpret_cast<int*>(smem + Lo.cnt_in);
  u64* thr = reinterpret_cast<u64*>(smem + Lo.thr);
  unsigned char* Qs = smem + Lo.qs;
  float* Ss = reinterpret_cast<float*>(smem + Lo.ss);
  unsigned char* Ps = smem + Lo.ps;
  float* alpha_s = reinterpret_cast<float*>(smem + Lo.alpha);
  unsigned char* region = smem + Lo.region;
  float* qsum = reinterpret_cast<float*>(region + Lo.qsum);
  u64* keys = reinterpret_cast<u64*>(region + Lo.keys);
  u64* top = reinterpret_cast<u64*>(region + Lo.top);
  u64* recv = reinterpret_cast<u64*>(region + Lo.recv);
  u64* work = reinterpret_cast<u64*>(region + Lo.work);
  unsigned char* inu = region + Lo.inu;
  unsigned char* kv = region;
  const int kv_tile = (int)Lo.kv_tile;
  constexpr int kRowBytes = D * 2;

  // ---- active / stable token lists (ascending) ----------------------------------------
  __shared__ int counts[2];
  if (warp == 0) {
    int na = 0, ns = 0;
    for (int base = 0; base < Tq; base += 32) {
      const int t = base + lane;
      const bool on = t < Tq && p.active[(size_t)b * Tq + t] != 0;
      const bool off = t < Tq && !on;
      const unsigned m_on = __ballot_sync(0xffffffffu, on), m_off = __ballot_sync(0xffffffffu, off);
      const unsigned below = (1u << lane) - 1u;
      if (on) act[na + __popc(m_on & below)] = t;
      if (off) stab[ns + __popc(m_off & below)] = t;
      na += __popc(m_on);
      ns += __popc(m_off);
    }
    if (lane == 0) {
      counts[0] = na;
      counts[1] = ns;
    }
  }
  __syncthreads();
  const int A = counts[0], S = counts[1];

  const int NBp = (p.T_prefix + kBlk - 1) / kBlk;
  const int per = (NBp + CL - 1) / CL;
  const int j0 = rank * per;
  const int nloc = max(0, min(NBp, j0 + per) - j0);
  const bool all_blocks = NBp <= p.topk;
  const int nf = all_blocks ? 0 : p.n_sink + p.n_local;  // disjoint when NBp > topk
  const int m = p.topk - nf;
  auto forced = [&](int j) { return j < p.n_sink || j >= NBp - p.n_local; };

  // ---- the union over this CTA's slice --------------------------------------------------
  for (int i = tid; i < nloc; i += kThreads) inu[i] = (A > 0 && (all_blocks || forced(j0 + i))) ? 1 : 0;
  __syncthreads();
  if (A > 0 && !all_blocks && m > 0) {  // (m == 0: every slot is a forced block)
    constexpr int VEC = D / 32;
    const float* sb = p.summ + unit * (size_t)p.NB_cap * D + lane * VEC;
    for (int tc0 = 0; tc0 < A; tc0 += kTokChunk) {
      const int na = min(kTokChunk, A - tc0);
      // summed, scaled queries of the chunk's tokens
      for (int i = tid; i < na * D; i += kThreads) {
        const int a = i / D, d = i - a * D;
        const __nv_bfloat16* qrow = p.q + (((size_t)b * Hq + (size_t)g * G) * Tq + act[tc0 + a]) * D + d;
        float s = 0.f;
        for (int h = 0; h < G; ++h) s += __bfloat162float(qrow[(size_t)h * Tq * D]);
        qsum[a * D + d] = s * p.scale;
      }
      for (int i = tid; i < kTokChunk * kLP; i += kThreads) top[i] = 0ull;
      __syncthreads();
      // scores of the slice for every token: a warp per summary row, 8 rows in flight
      constexpr int kRowsPerWarp = 8;
      for (int o0 = warp; o0 < nloc; o0 += kWarps * kRowsPerWarp) {
        float vals[kRowsPerWarp][VEC];
#pragma unroll
        for (int u = 0; u < kRowsPerWarp; ++u) {
          const int oo = o0 + u * kWarps;
          const float* src = sb + (size_t)(j0 + (oo < nloc ? oo : 0)) * D;
          if constexpr (VEC == 4) {
            const float4 t4 = __ldg(reinterpret_cast<const float4*>(src));
            vals[u][0] = t4.x; vals[u][1] = t4.y; vals[u][2] = t4.z; vals[u][3] = t4.w;
          } else {
            const float2 t2 = __ldg(reinterpret_cast<const float2*>(src));
            vals[u][0] = t2.x; vals[u][1] = t2.y;
          }
        }
#pragma unroll
        for (int u = 0; u < kRowsPerWarp; ++u) {
          const int oo = o0 + u * kWarps;
          if (oo >= nloc) break;
          const int j = j0 + oo;
          const bool fj = forced(j);
          for (int a = 0; a < na; ++a) {
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) dot = fmaf(vals[u][e], qsum[a * D + lane * VEC + e], dot);
            dot = warp_sum(dot);
            if (lane == 0) keys[a * p.per_max + oo] = fj ? 0ull : make_key(dot, j);
          }
        }
      }
      __syncthreads();
      // local top-m of every token (rank = number of larger keys; keys are unique)
      for (int i = tid; i < na * nloc; i += kThreads) {
        const int a = i / nloc, jj = i - a * nloc;
        const u64* ka = keys + a * p.per_max;
        const u64 x = ka[jj];
        if (x == 0ull) continue;
        int r = 0;
        for (int u = 0; u < nloc; ++u) r += ka[u] > x;
        if (r < m) top[a * kLP + r] = x;
      }
      __syncthreads();
      // push the lists: recv[rank][a][*] on every CTA
      if (!started) {
        cluster_wait();
        started = true;
      }
      for (int i = tid; i < CL * kTokChunk * kLP; i += kThreads) {
        const int peer = i / (kTokChunk * kLP), rem = i - peer * (kTokChunk * kLP);
        st_cluster(map_rank(recv + (size_t)rank * kTokChunk * kLP + rem, peer), top[rem]);
      }
      cluster_arrive_release();
      cluster_wait();
      // batched merge trees: token a's lists are recv[c][a][*], c < CL
      {
        u64* src = recv;
        u64* dst = work;
        int cs = kTokChunk * kLP, as = kLP;
        for (int n = CL; n > 1; n >>= 1) {
          const int pairs = n >> 1;
          for (int t = warp; t < na * pairs; t += kWarps) {
            const int a = t / pairs, pr = t - a * pairs;
            const u64* LA = src + (size_t)(2 * pr) * cs + a * as;
            const u64* LB = src + (size_t)(2 * pr + 1) * cs + a * as;
            u64 x[1];
            x[0] = lane < kLP ? LA[lane] : LB[2 * kLP - 1 - lane];
            warp_merge_desc<1>(x);
            if (lane < kLP) dst[(size_t)a * (kMaxCluster / 2) * kLP + pr * kLP + lane] = x[0];
          }
          __syncthreads();
          u64* t2 = src;
          src = dst;
          dst = t2;
          cs = kLP;
          as = (kMaxCluster / 2) * kLP;
        }
        if (tid < na) thr[tid] = src[(size_t)tid * as + (m - 1)];  // the token's m-th best key
      }
      __syncthreads();
      for (int i = tid; i < nloc; i += kThreads) {
        bool in = false;
        for (int a = 0; a < na; ++a) {
          const u64 x = keys[a * p.per_max + i];
          in |= (x != 0ull && x >= thr[a]);
        }
        if (in) inu[i] = 1;
      }
      if (tc0 + kTokChunk < A) {  // peers must finish reading recv before the next push
        cluster_arrive_release();
        cluster_wait();
      }
      __syncthreads();
    }
  }
  // compact this slice's union flags into an ascending list (block-wide ballot scan)
  __shared__ int warp_tot[kWarps];
  int n_my = 0;
  for (int base = 0; base < nloc; base += kThreads) {
    const int i = base + tid;
    const bool on = i < nloc && inu[i];
    const unsigned mk = __ballot_sync(0xffffffffu, on);
    if (lane == 0) warp_tot[warp] = __popc(mk);
    __syncthreads();
    int off = n_my;
    for (int w = 0; w < warp; ++w) off += warp_tot[w];
    if (on) ulist[off + __popc(mk & ((1u << lane) - 1u))] = j0 + i;
    int tot = 0;
    for (int w = 0; w < kWarps; ++w) tot += warp_tot[w];
    n_my += tot;
    __syncthreads();
  }

  // ---- attention: rows (active token x head) in chunks of 32, my union blocks -----------
  const int rows = A * G;
  const int nchunks = (rows + kRowChunk - 1) / kRowChunk;
  const int total = nchunks * n_my;
  const __nv_bfloat16* kbase = p.k + unit * (size_t)p.T_cap * D;
  const __nv_bfloat16* vbase = p.v + unit * (size_t)p.T_cap * D;
  float* wsu = p.ws + (unit * kMaxCluster + rank) * (size_t)p.rows_max * (D + 2);
  int issued = 0;
  auto issue = [&]() {
    unsigned char* st = kv + (size_t)(issued % kStages) * 2 * kv_tile;
    stage_block<__nv_bfloat16, D, kThreads>(st, st + kv_tile, kbase, vbase, ulist[issued % n_my],
                                            p.T_prefix, kRowBytes);
    cp_async_commit();
    ++issued;
  };
  while (issued < kStages && issued < total) issue();

  constexpr int NT = D / 64;  // n8 tiles of the output per warp
  const float scale2 = p.scale * kLog2e;
  const int srow = tid >> 3, ssub = tid & 7;  // softmax mapping: 32 rows x 8 threads
  float m_run = -INFINITY, l_run = 0.f;
  float acc[2][NT][4];

  for (int c = 0; c < nchunks; ++c) {
    const int c0 = c * kRowChunk;
    const int nr = min(kRowChunk, rows - c0);
    // query rows of the chunk (row r: token act[r / G], head r % G), zero beyond nr
    for (int id = tid; id < kRowChunk * (kRowBytes / 16); id += kThreads) {
      const int r = id / (kRowBytes / 16), cc = id - r * (kRowBytes / 16);
      uint4 v4 = make_uint4(0u, 0u, 0u, 0u);
      if (r < nr) {
        const int rr = c0 + r, a = rr / G, hh = rr - a * G;
        v4 = __ldg(reinterpret_cast<const uint4*>(p.q + (((size_t)b * Hq + (size_t)g * G + hh) * Tq + act[a]) * D) + cc);
      }
      *reinterpret_cast<uint4*>(Qs + swz(r, cc, kRowBytes)) = v4;
    }
    m_run = -INFINITY;
    l_run = 0.f;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
    __syncthreads();

    for (int i = 0; i < n_my; ++i) {
      const int it = c * n_my + i;
      if (issued > it + 1) cp_async_wait<1>(); else cp_async_wait<0>();
      __syncthreads();
      const int j = ulist[i];
      const unsigned char* Ks = kv + (size_t)(it % kStages) * 2 * kv_tile;
      const unsigned char* Vs = Ks + kv_tile;
      // S = Q K^T: warp w -> tokens 8w .. 8w+7, both m-tiles
      {
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < D / 16; ks += 2) {
          uint32_t kb[4];
          ldsm_x4(kb, Ks + swz(8 * warp + (lane & 7), 2 * ks + (lane >> 3), kRowBytes));
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const int row = 16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1);
            uint32_t qa0[4], qa1[4];
            ldsm_x4(qa0, Qs + swz(row, 2 * ks + (lane >> 4), kRowBytes));
            ldsm_x4(qa1, Qs + swz(row, 2 * ks + 2 + (lane >> 4), kRowBytes));
            mma_bf16(s[mt], qa0, kb[0], kb[1]);
            mma_bf16(s[mt], qa1, kb[2], kb[3]);
          }
        }
        const int col = 8 * warp + 2 * (lane & 3);
        const bool v0 = j * kBlk + col < p.T_prefix, v1 = j * kBlk + col + 1 < p.T_prefix;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const int r0 = 16 * mt + (lane >> 2);
          *reinterpret_cast<float2*>(Ss + r0 * kSStride + col) =
              make_float2(v0 ? s[mt][0] * scale2 : -INFINITY, v1 ? s[mt][1] * scale2 : -INFINITY);
          *reinterpret_cast<float2*>(Ss + (r0 + 8) * kSStride + col) =
              make_float2(v0 ? s[mt][2] * scale2 : -INFINITY, v1 ? s[mt][3] * scale2 : -INFINITY);
        }
      }
      __syncthreads();
      // online softmax: row srow, columns 8*ssub .. 8*ssub+7
      {
        const float4 sa = *reinterpret_cast<const float4*>(Ss + srow * kSStride + 8 * ssub);
        const float4 sb4 = *reinterpret_cast<const float4*>(Ss + srow * kSStride + 8 * ssub + 4);
        float mx = fmaxf(fmaxf(fmaxf(sa.x, sa.y), fmaxf(sa.z, sa.w)), fmaxf(fmaxf(sb4.x, sb4.y), fmaxf(sb4.z, sb4.w)));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_new = fmaxf(m_run, mx);
        float pv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float alpha = 1.f;
        if (m_new != -INFINITY) {
          alpha = ex2(m_run - m_new);
          pv[0] = ex2(sa.x - m_new); pv[1] = ex2(sa.y - m_new);
          pv[2] = ex2(sa.z - m_new); pv[3] = ex2(sa.w - m_new);
          pv[4] = ex2(sb4.x - m_new); pv[5] = ex2(sb4.y - m_new);
          pv[6] = ex2(sb4.z - m_new); pv[7] = ex2(sb4.w - m_new);
        }
        float ps = ((pv[0] + pv[1]) + (pv[2] + pv[3])) + ((pv[4] + pv[5]) + (pv[6] + pv[7]));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        l_run = l_run * alpha + ps;
        m_run = m_new;
        *reinterpret_cast<uint4*>(Ps + swz(srow, ssub, kBlk * 2)) =
            make_uint4(pack_bf16x2(pv[0], pv[1]), pack_bf16x2(pv[2], pv[3]),
                       pack_bf16x2(pv[4], pv[5]), pack_bf16x2(pv[6], pv[7]));
        if (ssub == 0) alpha_s[srow] = alpha;
      }
      __syncthreads();
      // O = alpha * O + P V: warp w -> output dims of its n-tiles, both m-tiles
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const float a_lo = alpha_s[16 * mt + (lane >> 2)], a_hi = alpha_s[16 * mt + (lane >> 2) + 8];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[mt][nt][0] *= a_lo; acc[mt][nt][1] *= a_lo;
          acc[mt][nt][2] *= a_hi; acc[mt][nt][3] *= a_hi;
        }
      }
#pragma unroll
      for (int ks = 0; ks < kBlk / 16; ++ks) {
        const int vrow = 16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1);
        uint32_t vb[4];
        if constexpr (D == 128) {
          ldsm_x4_t(vb, Vs + swz(vrow, 2 * warp + (lane >> 4), kRowBytes));
        } else {
          uint32_t v2[2];
          ldsm_x2_t(v2, Vs + swz(vrow, warp, kRowBytes));
          vb[0] = v2[0]; vb[1] = v2[1]; vb[2] = 0u; vb[3] = 0u;
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          uint32_t pa[4];
          const int row = 16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1);
          ldsm_x4(pa, Ps + swz(row, 2 * ks + (lane >> 4), kBlk * 2));
          mma_bf16(acc[mt][0], pa, vb[0], vb[1]);
          if constexpr (NT == 2) mma_bf16(acc[mt][1], pa, vb[2], vb[3]);
        }
      }
      __syncthreads();  // the stage may now be refilled
      if (issued < total) issue();
    }
    // partial of this chunk -> workspace: acc rows, then (m, l)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int d = (D == 128 ? 16 * warp : 8 * warp) + 8 * nt + 2 * (lane & 3);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int r = 16 * mt + (lane >> 2) + 8 * half;
          if (r < nr)
            *reinterpret_cast<float2*>(wsu + (size_t)(c0 + r) * (D + 2) + d) =
                make_float2(acc[mt][nt][2 * half], acc[mt][nt][2 * half + 1]);
        }
      }
    }
    if (ssub == 0 && srow < nr)
      *reinterpret_cast<float2*>(wsu + (size_t)(c0 + srow) * (D + 2) + D) = make_float2(m_run, l_run);
    __syncthreads();  // Qs / stats are rewritten by the next chunk
  }

  // ---- exchange union counts, barrier, then merge my output slice ------------------------
  if (!started) {
    cluster_wait();
    started = true;
  }
  if (tid < CL) st_cluster_u32(map_rank(cnt_in + rank, tid), (uint32_t)n_my);
  cluster_arrive_release();
  cluster_wait();

  const int E = rows * D;
  const int chunk = (E + CL - 1) / CL;
  const float* wsg = p.ws + unit * kMaxCluster * (size_t)p.rows_max * (D + 2);
  for (int e = rank * chunk + tid; e < min(E, (rank + 1) * chunk); e += kThreads) {
    const int r = e / D, d = e - r * D;
    float M = -INFINITY;
    float mm[kMaxCluster], ll[kMaxCluster];
#pragma unroll
    for (int c2 = 0; c2 < kMaxCluster; ++c2) {
      mm[c2] = -INFINITY;
      ll[c2] = 0.f;
      if (c2 < CL) {
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(wsg + ((size_t)c2 * p.rows_max + r) * (D + 2) + D));
        mm[c2] = ml.x;
        ll[c2] = ml.y;
        M = fmaxf(M, ml.x);
      }
    }
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int c2 = 0; c2 < kMaxCluster; ++c2) {
        if (c2 < CL && mm[c2] != -INFINITY) {
          const float w = ex2(mm[c2] - M);
          Lsum = fmaf(ll[c2], w, Lsum);
          O = fmaf(__ldcg(wsg + ((size_t)c2 * p.rows_max + r) * (D + 2) + d), w, O);
        }
      }
    }
    const int a = r / G, hh = r - a * G;
    const size_t orow = ((size_t)b * Hq + (size_t)g * G + hh) * Tq + act[a];
    p.o[orow * D + d] = __float2bfloat16_rn(M == -INFINITY ? 0.f : O / Lsum);
    if (d == 0) p.lse[orow] = M == -INFINITY ? -INFINITY : (M + log2f(Lsum)) * kLn2;
  }

  // ---- stable rows: the cached output and log-sum-exp, unchanged --------------------------
  const int srows = S * G;
  if (p.o_cache != p.o && srows > 0) {
    const int per_row = kRowBytes / 16;
    const int n16 = srows * per_row;
    const int c16 = (n16 + CL - 1) / CL;
    for (int i = rank * c16 + tid; i < min(n16, (rank + 1) * c16); i += kThreads) {
      const int r = i / per_row, cc = i - r * per_row;
      const int s_i = r / G, hh = r - s_i * G;
      const size_t orow = ((size_t)b * Hq + (size_t)g * G + hh) * Tq + stab[s_i];
      reinterpret_cast<uint4*>(p.o + orow * D)[cc] = reinterpret_cast<const uint4*>(p.o_cache + orow * D)[cc];
    }
  }
  if (p.lse_cache != p.lse && srows > 0) {
    const int c1 = (srows + CL - 1) / CL;
    for (int r = rank * c1 + tid; r < min(srows, (rank + 1) * c1); r += kThreads) {
      const int s_i = r / G, hh = r - s_i * G;
      const size_t orow = ((size_t)b * Hq + (size_t)g * G + hh) * Tq + stab[s_i];
      p.lse[orow] = p.lse_cache[orow];
    }
  }

  // ---- the union list, by the offsets of the slices -------------------------------------
  int off = 0, tot = 0;
  for (int c2 = 0; c2 < CL; ++c2) {
    const int cnt = cnt_in[c2];
    if (c2 < rank) off += cnt;
    tot += cnt;
  }
  if (p.union_idx) {
    int32_t* ui = p.union_idx + unit * (size_t)NBp;
    for (int i = tid; i < n_my; i += kThreads) ui[off + i] = ulist[i];
    if (rank == CL - 1)
      for (int i = tot + tid; i < NBp; i += kThreads) ui[i] = -1;
  }
  if (p.union_cnt && rank == 0 && tid == 0) p.union_cnt[unit] = tot;
}

}  // namespace

size_t blockquery_workspace_bytes(int B, int Hkv, int G, int D, int Tq) {
  return (size_t)B * Hkv * kMaxCluster * (size_t)Tq * G * (D + 2) * sizeof(float);
}

cudaError_t launch_blockquery(const BlockQueryArgs& a, cudaStream_t stream) {
  const int units = a.B * a.Hkv;
  int CL = units <= 14 ? 16 : (units <= 37 ? 8 : 4);
  const int NBp = (a.T_prefix + kBlk - 1) / kBlk;
  BQParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v);
  p.Hkv = a.Hkv; p.G = a.G; p.Tq = a.Tq; p.T_prefix = a.T_prefix; p.T_cap = a.T_cap;
  p.NB_cap = (a.T_cap + kBlk - 1) / kBlk;
  p.summ = a.summ; p.topk = a.topk; p.n_sink = a.n_sink; p.n_local = a.n_local;
  p.scale = a.scale; p.active = a.active;
  p.o_cache = static_cast<const __nv_bfloat16*>(a.o_cache); p.lse_cache = a.lse_cache;
  p.o = static_cast<__nv_bfloat16*>(a.o); p.lse = a.lse;
  p.union_idx = a.union_idx; p.union_cnt = a.union_cnt;
  p.ws = static_cast<float*>(a.workspace);
  p.rows_max = a.Tq * a.G;
  auto kernel = a.D == 128 ? blockquery_kernel<128> : blockquery_kernel<64>;
  static int smem_set128 = 0, smem_set64 = 0;
  int& smem_set = a.D == 128 ? smem_set128 : smem_set64;
  for (;;) {
    p.per_max = (NBp + CL - 1) / CL;
    if (p.per_max < 1) p.per_max = 1;
    const BQLayout Lo = bq_layout(a.D, p.per_max);
    const int smem = (int)Lo.total;
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t err;
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
    return cudaLaunchKernelEx(&cfg, kernel, p);
  }
}


// ---- fixed scratch for callers that cannot allocate device memory -----------------------
// Some callers may not allocate device memory at all (for instance code that runs where
// allocation is forbidden or must not change the memory footprint).  For them the
// block-query partials live in one statically sized device array instead of a caller
// workspace.  The array exists once per GPU that loads this library and stays allocated
// until the process exits; every call shares it, so calls that overlap on the GPU (other
// streams, or other host threads) race on its contents.  Nothing in it has to start at
// zero: each call writes every partial it reads back.
constexpr size_t kStaticWorkspaceBytes = (size_t)16 << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_blockquery_scratch[kStaticWorkspaceBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
}  // namespace

size_t blockquery_static_workspace_bytes() { return kStaticWorkspaceBytes; }

// Device address of the fixed scratch on the current device.  The first call on a device
// looks it up with cudaGetSymbolAddress (the host-side name of the array is not a device
// address); later calls reuse the cached pointer.
cudaError_t blockquery_static_workspace(void** ptr) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_blockquery_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace lsa
