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
//   * Each CTA of the cluster owns a contiguous slice of the prefix blocks, copied into
//     shared memory by one bulk copy at launch.  It scores its slice for 8 active tokens
//     at a time (lane = token x quarter of a summary row, the summed queries in registers,
//     4 rows in flight per warp), keeps each token's local top-m as 64-bit keys, and
//     pushes the lists to every peer with st.async into a double-buffered receive area
//     whose bytes complete on an mbarrier (no cluster-wide barrier).
//   * A warp per token runs a tournament over the token's CL sorted lists (the warp
//     maximum of the list heads, m rounds): its selected blocks go into a bitmap of the
//     union, so every CTA holds the same union U(b, g) and attends entries rank, rank + CL,
//     ... of its ascending list (balanced over the cluster).
//   * Attention rows (active token x head) are processed 32 at a time: K/V blocks arrive
//     as TMA boxes (128-byte swizzle) on a 2-stage ring with per-stage mbarriers; warp w
//     owns 16 rows and a quarter (16 keys) of every block, computes S = Q K^T and
//     O += P V on mma.sync m16n8k16 bf16 with the logits kept in registers (online softmax
//     in base 2), and the last warp done with a stage refills it.  The four key quarters
//     are merged by log-sum-exp once per row chunk, through the ring.
//   * When the rows fit one chunk, each CTA pushes its per-row partial (acc, m, l) into the
//     shared memory of the CTA that merges that slice of the outputs (st.async on the
//     owner's mbarrier) and the owners merge by log-sum-exp; more rows go through the
//     caller's workspace and one cluster barrier (all loads of a merge issued before use).
//     Stable rows are copied from the cache; rank 0 writes the union list.
//   Every mbarrier wait is bounded (about 2 s); after a timeout the CTA waits (bounded) for
//   its copies and its peers' list bytes still in flight before it exits, and a device status
//   word records the failure.
#include <math.h>

#include <mutex>

#include "cluster.cuh"
#include "launch_cache.h"
#include "lsa_common.cuh"
#include "lsa_internal.h"
#include "tcgen05.cuh"

namespace lsa {
namespace {

typedef unsigned long long u64;

// Set when a bounded wait on a cross-CTA exchange or a bulk copy runs out (the launch's
// outputs are then undefined); read and cleared by the host.
__device__ int g_blockquery_status = 0;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTokChunk = 8;    // active tokens per selection exchange
constexpr int kRowChunk = 32;   // attention rows per pass (two mma m-tiles)
constexpr int kLP = 16;         // length of an exchanged list (topk_per_query <= 16)
constexpr int kMaxCluster = 16;
constexpr int kMaxTq = 64;
constexpr int kStages = 2;
constexpr int kQStride = 132;   // fp32 row stride of the summed queries (bank spread)
constexpr int kStageRows = 64;  // summary rows of a CTA's slice staged by one bulk copy
constexpr int kMaxUnion = kMaxTq * kLP;  // a union holds at most Tq * topk blocks
static_assert(kTokChunk == 8, "the scoring maps lane l to token l & 7");
static_assert(kThreads == 256 && kRowChunk == 32, "attention: 8 warps = 2 row tiles x 4 key quarters");
// the key quarters' partials of a row chunk (fp32) are merged in the K/V ring
static_assert(kStages * 2 * kBlk * 2 >= (kWarps / 2) * kRowChunk * 4, "merge buffer exceeds the ring");

struct alignas(64) BQParams {
  // K and V as [B * Hkv][T_cap][D], box {64, 64, 1}, 128-byte swizzle
  CUtensorMap tmk;
  CUtensorMap tmv;
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
  int NBp;         // prefix blocks
  FastDiv g_div;   // division by G
  FastDiv per_div; // division by per_max
  long long budget;  // clock-cycle limit of every bounded wait
};

// st.async of four floats into a peer CTA's shared memory, counted on its mbarrier
__device__ __forceinline__ void st_async4(uint32_t addr, float4 v, uint32_t mbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   addr),
               "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(mbar)
               : "memory");
}

__host__ __device__ inline size_t al128(size_t x) { return (x + 127) & ~(size_t)127; }

struct BQLayout {
  size_t act, stab, ulist, ubits, qs, pml, pacc, region, total;
  // selection buffers, inside `region` (dead once the attention starts)
  size_t qsum, keys, top, recv, sumbuf, qrows;
  size_t kv_tile;
};

// dense: every prefix block is selected (topk_per_query >= NBp), the selection buffers are
// not used and the union holds all NBp blocks
__host__ __device__ inline BQLayout bq_layout(int D, int per_max, int NBp, int G, bool dense) {
  BQLayout L;
  size_t off = 0;
  const int ucap = (dense || NBp < kMaxUnion) ? NBp : kMaxUnion;
  const int stage_rows = dense ? 0 : (per_max < kStageRows ? per_max : kStageRows);
  const int per_sel = dense ? 0 : per_max;
  const int tok_sel = dense ? 0 : kTokChunk;
  L.act = off;    off = al128(off + kMaxTq * 4);
  L.stab = off;   off = al128(off + kMaxTq * 4);
  L.ulist = off;  off = al128(off + (size_t)(ucap > 0 ? ucap : 1) * 4);
  L.ubits = off;  off = al128(off + (size_t)((NBp + 31) / 32 + 1) * 4);
  L.qs = off;     off = al128(off + (size_t)kRowChunk * D * 2);
  // the partials pushed by the cluster's CTAs when the rows fit one chunk: every CTA's
  // (m, l) of every row and its part of this CTA's slice of the outputs
  L.pml = off;    off = al128(off + (size_t)kMaxCluster * kRowChunk * 8);
  L.pacc = off;   off = al128(off + (size_t)kRowChunk * D * 4 + kMaxCluster * 16);
  L.region = off;
  L.kv_tile = (size_t)kBlk * D * 2;
  // the K/V ring starts at the first 1024-byte boundary of the region (TMA 128-byte swizzle)
  const size_t kv_bytes = kStages * 2 * L.kv_tile + 1024;
  size_t r = 0;
  L.qsum = r; r = al128(r + (size_t)tok_sel * kQStride * 4);
  L.keys = r; r = al128(r + (size_t)tok_sel * per_sel * 8);
  L.top = r;  r = al128(r + (size_t)tok_sel * kLP * 8);
  L.recv = r; r = al128(r + (size_t)2 * kMaxCluster * tok_sel * kLP * 8);  // two buffers
  L.sumbuf = r; r = al128(r + (size_t)stage_rows * D * 4);
  L.qrows = r; r = al128(r + (size_t)tok_sel * G * D * 2);  // a token chunk's query rows
  L.total = off + (r > kv_bytes ? r : kv_bytes);
  return L;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2) blockquery_kernel(const __grid_constant__ BQParams p) {
  const int CL = cluster_size();
  const int rank = cluster_rank();
  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G, Tq = p.Tq, Hq = p.Hkv * G;
  const size_t unit = (size_t)b * p.Hkv + g;

  extern __shared__ __align__(1024) unsigned char smem[];
  const BQLayout Lo = bq_layout(D, p.per_max, p.NBp, p.G, p.NBp <= p.topk);
  int* act = reinterpret_cast<int*>(smem + Lo.act);
  int* stab = reinterpret_cast<int*>(smem + Lo.stab);
  int* ulist = reinterpret_cast<int*>(smem + Lo.ulist);
  uint32_t* ubits = reinterpret_cast<uint32_t*>(smem + Lo.ubits);
  unsigned char* Qs = smem + Lo.qs;
  float2* pml = reinterpret_cast<float2*>(smem + Lo.pml);
  float* pacc = reinterpret_cast<float*>(smem + Lo.pacc);
  unsigned char* region = smem + Lo.region;
  float* qsum = reinterpret_cast<float*>(region + Lo.qsum);
  u64* keys = reinterpret_cast<u64*>(region + Lo.keys);
  u64* top = reinterpret_cast<u64*>(region + Lo.top);
  u64* recv = reinterpret_cast<u64*>(region + Lo.recv);
  float* sumbuf = reinterpret_cast<float*>(region + Lo.sumbuf);
  unsigned char* qrows = region + Lo.qrows;
  unsigned char* kv = region + ((1024u - (tc::smem_u32(region) & 1023u)) & 1023u);
  const int kv_tile = (int)Lo.kv_tile;
  constexpr int kRowBytes = D * 2;

  const int NBp = p.NBp;
  const int per = p.per_max;
  const int j0 = rank * per;
  const int nloc = max(0, min(NBp, j0 + per) - j0);
  const bool all_blocks = NBp <= p.topk;
  // mbarriers: [0], [1] count the bytes of the candidate-list exchange (two buffers, one
  // phase per token chunk that uses the buffer); [2] the bulk copy of the summary slice;
  // [3 + s] the TMA loads into K/V stage s (one phase per use of the stage); [3 + kStages]
  // the partials pushed into this CTA (one phase)
  __shared__ __align__(8) uint64_t xbar[4 + kStages];
  __shared__ int xabort;
  const int staged_rows = all_blocks ? 0 : min(nloc, kStageRows);
  if (tid == 0) {
    for (int i = 0; i < 4 + kStages; ++i) tc::mbar_init(&xbar[i], 1);
    xabort = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&p.tmk);
    tc::prefetch_tmap(&p.tmv);
  }
  // The launch is a programmatic dependent one: nothing above reads an input, and every
  // input may come from the previous kernel of the stream, which is complete (and its
  // memory visible) once this wait returns.  The trigger then lets the next kernel start
  // its own prologue; one that reads this grid's outputs waits for its completion first.
  pdl_wait();
  if (tid == 0 && staged_rows > 0) {  // the slice's first summary rows, one bulk copy
    const uint32_t bytes = (uint32_t)(staged_rows * D * 4);
    tc::mbar_arrive_expect_tx(&xbar[2], bytes);
    tc::bulk_load(sumbuf, p.summ + (unit * (size_t)p.NB_cap + j0) * D, bytes, &xbar[2]);
  }
  pdl_trigger();
  cluster_arrive_relaxed();  // DSMEM is written only after every CTA has started
  bool started = false;

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
  const int nf = all_blocks ? 0 : p.n_sink + p.n_local;  // disjoint when NBp > topk
  const int m = p.topk - nf;
  const bool selecting = A > 0 && !all_blocks && m > 0;  // (m == 0: every slot is forced)
  const int rows = A * G;

  // ---- query rows by cp.async, requested as soon as the active tokens are known: those of
  // a token chunk (scoring) into qrows, those of an attention row chunk into Qs (row r is
  // token act[r / G], head r % G; rows past the end are zero)
  auto load_token_rows = [&](int tc0) {
    const int na = min(kTokChunk, A - tc0);
    constexpr int kC = kRowBytes / 16;
    for (int id = tid; id < na * G * kC; id += kThreads) {
      const int rr = id / kC, cc = id - rr * kC, a2 = fdiv(rr, p.g_div), hh = rr - a2 * G;
      cp_async16(qrows + (size_t)rr * kRowBytes + cc * 16,
                 p.q + (((size_t)b * Hq + (size_t)g * G + hh) * Tq + act[tc0 + a2]) * D + cc * 8, true);
    }
  };
  auto load_attn_rows = [&](int c0) {
    constexpr int kC = kRowBytes / 16;
    for (int id = tid; id < kRowChunk * kC; id += kThreads) {
      const int r = id / kC, cc = id - r * kC, rr = c0 + r;
      const bool ok = rr < rows;
      const int a2 = ok ? fdiv(rr, p.g_div) : 0, hh = ok ? rr - a2 * G : 0;
      cp_async16(Qs + swz(r, cc, kRowBytes),
                 p.q + (((size_t)b * Hq + (size_t)g * G + hh) * Tq + act[ok ? a2 : 0]) * D + cc * 8, ok);
    }
  };
  if (A > 0) {
    if (selecting) load_token_rows(0);
    load_attn_rows(0);
    cp_async_commit();
  }

  auto forced = [&](int j) { return j < p.n_sink || j >= NBp - p.n_local; };
  const int nwords = (NBp + 31) / 32;

  // ---- the union U(b, g) as a bitmap over the prefix blocks, the same on every CTA --------
  for (int w = tid; w < nwords; w += kThreads) ubits[w] = 0u;
  __syncthreads();
  if (A > 0) {
    for (int j = tid; j < NBp; j += kThreads)
      if (all_blocks || forced(j)) atomicOr(&ubits[j >> 5], 1u << (j & 31));
  }
  if (selecting) {
    if (staged_rows > 0) tc::mbar_wait(&xbar[2], 0, &xabort, p.budget);
    constexpr int kSeg = D / 4;  // summary floats per lane: lane l takes quarter l >> 3
    const int ta = lane & 7, q4 = lane >> 3;
    const float* grow = p.summ + (unit * (size_t)p.NB_cap + j0) * D + q4 * kSeg;
    for (int tc0 = 0; tc0 < A; tc0 += kTokChunk) {
      const int chunk_id = tc0 / kTokChunk, buf = chunk_id & 1;
      const int na = min(kTokChunk, A - tc0);
      if (tc0 > 0) {
        load_token_rows(tc0);
        cp_async_commit();
      }
      cp_async_wait<0>();
      __syncthreads();
      // summed, scaled queries of the chunk's tokens (rows past na are zero)
      for (int i = tid; i < kTokChunk * D; i += kThreads) {
        const int a2 = i / D, d = i - a2 * D;
        float sum = 0.f;
        if (a2 < na) {
          const __nv_bfloat16* qr = reinterpret_cast<const __nv_bfloat16*>(qrows) + (size_t)a2 * G * D + d;
          for (int h = 0; h < G; ++h) sum += __bfloat162float(qr[(size_t)h * D]);
        }
        qsum[a2 * kQStride + d] = sum * p.scale;
      }
      for (int i = tid; i < kTokChunk * kLP; i += kThreads) top[i] = 0ull;
      __syncthreads();
      // scores of the slice: lane (token ta, quarter q4) keeps its token's quarter of the
      // summed query in registers; a quarter-warp reads one 16-byte chunk of a summary
      // row (a broadcast), and the 4 quarters are summed with two shuffles
      float qv[kSeg];
#pragma unroll
      for (int k4 = 0; k4 < kSeg / 4; ++k4) {
        const float4 v = *reinterpret_cast<const float4*>(qsum + ta * kQStride + q4 * kSeg + 4 * k4);
        qv[4 * k4] = v.x; qv[4 * k4 + 1] = v.y; qv[4 * k4 + 2] = v.z; qv[4 * k4 + 3] = v.w;
      }
      constexpr int kRU = 4;  // rows per warp at a time (independent chains)
      for (int r0 = warp; r0 < nloc; r0 += kWarps * kRU) {  // warp-uniform
        float dot[kRU];
#pragma unroll
        for (int u = 0; u < kRU; ++u) {
          const int r = r0 + u * kWarps;
          float a0 = 0.f, a1 = 0.f;
          if (r < nloc) {
            const float* row = r < staged_rows ? sumbuf + r * D + q4 * kSeg : grow + (size_t)r * D;
#pragma unroll
            for (int k4 = 0; k4 < kSeg / 4; ++k4) {
              const float4 v = r < staged_rows ? reinterpret_cast<const float4*>(row)[k4]
                                               : __ldg(reinterpret_cast<const float4*>(row) + k4);
              a0 = fmaf(v.x, qv[4 * k4], a0);
              a1 = fmaf(v.y, qv[4 * k4 + 1], a1);
              a0 = fmaf(v.z, qv[4 * k4 + 2], a0);
              a1 = fmaf(v.w, qv[4 * k4 + 3], a1);
            }
          }
          dot[u] = a0 + a1;
        }
#pragma unroll
        for (int u = 0; u < kRU; ++u) dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], 8);
#pragma unroll
        for (int u = 0; u < kRU; ++u) dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], 16);
        if (q4 == 0 && ta < na) {
#pragma unroll
          for (int u = 0; u < kRU; ++u) {
            const int r = r0 + u * kWarps;
            if (r < nloc) {
              const int j = j0 + r;
              keys[ta * per + r] = forced(j) ? 0ull : make_key(dot[u], j);
            }
          }
        }
      }
      __syncthreads();
      // local top-m of every token (rank = number of larger keys; keys are unique)
      for (int i = tid; i < na * per; i += kThreads) {
        const int a2 = fdiv(i, p.per_div), jj = i - a2 * per;
        if (jj >= nloc) continue;
        const u64* ka = keys + a2 * per;
        const u64 x = ka[jj];
        if (x == 0ull) continue;
        int r = 0;
        for (int u = 0; u < nloc; ++u) r += ka[u] > x;
        if (r < m) top[a2 * kLP + r] = x;
      }
      __syncthreads();
      // push the lists into every peer's buffer `buf` (recv[buf][rank][a][*]); each CTA
      // waits only until the CL lists of the chunk have landed on its own mbarrier
      if (!started) {
        cluster_wait();
        started = true;
      }
      u64* rb = recv + (size_t)buf * kMaxCluster * kTokChunk * kLP;
      if (tid == 0) tc::mbar_arrive_expect_tx(&xbar[buf], (uint32_t)(CL * kTokChunk * kLP * 8));
      for (int i = tid; i < CL * kTokChunk * kLP; i += kThreads) {
        const int peer = i / (kTokChunk * kLP), rem = i - peer * (kTokChunk * kLP);
        st_async(map_rank(rb + (size_t)rank * kTokChunk * kLP + rem, peer), top[rem], map_rank(&xbar[buf], peer));
      }
      tc::mbar_wait(&xbar[buf], (uint32_t)((chunk_id >> 1) & 1), &xabort, p.budget);
      // every token's m best keys by a tournament over its CL sorted lists rb[c][a][*]: a
      // warp per token, lane l (and l + 16) holds the head of list l & 15; each round the
      // warp's maximum is a selected block and its list advances (keys are unique, so
      // exactly one list holds it).  m rounds of 4 shuffle steps, no block barrier.
      for (int a2 = warp; a2 < na; a2 += kWarps) {
        const int c = lane & 15;
        const u64* L = rb + (size_t)c * kTokChunk * kLP + a2 * kLP;
        int ptr = 0;
        u64 head = c < CL ? L[0] : 0ull;
        for (int r = 0; r < m; ++r) {
          u64 best = head;
#pragma unroll
          for (int o = 8; o >= 1; o >>= 1) {
            const u64 y = __shfl_xor_sync(0xffffffffu, best, o);
            best = y > best ? y : best;
          }
          if (best == 0ull) break;  // (uniform: both half-warps hold the same heads)
          if (head == best) {
            ++ptr;
            head = ptr < kLP ? L[ptr] : 0ull;
          }
          if (lane == 0) {
            const int j = key_block(best);
            // (a key is always a prefix block; the check keeps even a corrupted list -- after
            // a timed-out exchange -- inside the bitmap)
            if (j >= 0 && j < NBp) atomicOr(&ubits[j >> 5], 1u << (j & 31));
          }
        }
      }
      __syncthreads();  // (qsum, top and keys are rewritten by the next chunk)
    }
  } else if (staged_rows > 0) {
    __syncthreads();  // (thread 0's mbarrier initialisation first)
    tc::mbar_wait(&xbar[2], 0, &xabort, p.budget);  // no copy outlives its buffer's reuse
  }
  __syncthreads();
  // the union as an ascending list (block-wide scan of the bitmap's popcounts)
  __shared__ int warp_tot[kWarps];
  int U = 0;
  for (int base = 0; base < nwords; base += kThreads) {
    const int w = base + tid;
    const uint32_t bits = w < nwords ? ubits[w] : 0u;
    const int cnt = __popc(bits);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int off = U + incl - cnt;
    for (int w2 = 0; w2 < warp; ++w2) off += warp_tot[w2];
    uint32_t rest = bits;
    while (rest) {
      const int bit = __ffs(rest) - 1;
      ulist[off++] = w * 32 + bit;
      rest &= rest - 1u;
    }
    for (int w2 = 0; w2 < kWarps; ++w2) U += warp_tot[w2];
    __syncthreads();
  }
  // this CTA attends union entries rank, rank + CL, ... (balanced over the cluster)
  const int cl_log2 = __ffs(CL) - 1;  // CL is a power of two
  const int n_my = U > rank ? (U - rank + CL - 1) >> cl_log2 : 0;

  // ---- attention: rows (active token x head) in chunks of 32, my union blocks -----------
  // Warp w owns rows 16 (w & 1) .. + 15 of the chunk and keys 16 (w >> 1) .. + 15 of every
  // block: its logits stay in registers and become the A operand of P V directly, so a block
  // costs no block-wide barrier.  The four key quarters of a row are merged once per chunk,
  // by log-sum-exp, through the K/V ring (free once the chunk's blocks are done).
  const int nchunks = (rows + kRowChunk - 1) / kRowChunk;
  // one chunk of rows: the partials go straight into the shared memory of the CTAs that
  // merge them (st.async, counted on the owner's mbarrier), with no workspace round trip and
  // no cluster barrier; more rows go through the caller's workspace
  const bool dsm = nchunks == 1;
  float* wsu = p.ws + (unit * kMaxCluster + rank) * (size_t)p.rows_max * (D + 2);
  __shared__ int stage_rel[kStages];  // warps done with the stage's current block (mod 8)
  __shared__ int n_issued;             // block loads issued so far
  // block `it` of the processing order (row chunk it / n_my, union entry it % n_my): K and V
  // as TMA boxes (128-byte swizzled tiles) into stage it % kStages, landing on the stage's
  // mbarrier; called by one thread
  auto issue = [&](int it) {
    unsigned char* st = kv + (size_t)(it % kStages) * 2 * kv_tile;
    const int j = ulist[rank + (it % n_my) * CL];
    tc::fence_proxy_async();  // earlier generic accesses to this stage come first
    tc::mbar_arrive_expect_tx(&xbar[3 + it % kStages], (uint32_t)(2 * kv_tile));
#pragma unroll
    for (int h = 0; h < D / 64; ++h) {
      tc::tma_load_3d(st + h * 8192, &p.tmk, h * 64, j * kBlk, (int)unit, &xbar[3 + it % kStages]);
      tc::tma_load_3d(st + kv_tile + h * 8192, &p.tmv, h * 64, j * kBlk, (int)unit, &xbar[3 + it % kStages]);
    }
    atomicMax(&n_issued, it + 1);
  };
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) stage_rel[s] = 0;
    n_issued = 0;
  }
  __syncthreads();  // (the selection buffers that share the ring are dead)
  if (tid == 0 && rows > 0)
    for (int it = 0; it < kStages && it < n_my; ++it) issue(it);

  constexpr int NA = D / 8;   // n8 tiles of the output: all of D in every warp
  constexpr int KS = D / 16;  // k16 steps of Q K^T
  const int mt = warp & 1, kq = warp >> 1;
  const float scale2 = p.scale * kLog2e;
  // (m, l) of every row per key quarter, posted for the merge at the end of a chunk
  __shared__ float2 qml[kWarps / 2][kRowChunk];
  // the merge buffer over the ring: [key quarter][row][D] fp32, 32-byte granules of a row
  // XOR-swizzled by (row & 3) (the fragment stores and the float4 reads are conflict-free)
  float* mb = reinterpret_cast<float*>(kv);
  const int r_lo = 16 * mt + (lane >> 2), r_hi = r_lo + 8;  // this lane's rows in the chunk
  const int mr = tid >> 3, mc = tid & 7;  // merge mapping: row mr, columns 32 i + 4 mc .. + 3
  float M_row = -INFINITY, L_row = 0.f;
  float4 o_row[D / 32];

  for (int c = 0; c < nchunks; ++c) {
    const int c0 = c * kRowChunk;
    const int nr = min(kRowChunk, rows - c0);
    // query rows of the chunk (chunk 0 was requested at the start)
    if (c > 0) {
      load_attn_rows(c0);
      cp_async_commit();
    }
    cp_async_wait<0>();
    __syncthreads();
    const bool live = 16 * mt < nr;  // (a warp of padding rows only waits and releases)
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
    float acc[NA][4];
#pragma unroll
    for (int n = 0; n < NA; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
    const int q_row = 16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1);  // ldmatrix row of the A tile

    for (int i = 0; i < n_my; ++i) {
      const int it = c * n_my + i;
      tc::mbar_wait(&xbar[3 + it % kStages], (uint32_t)((it / kStages) & 1), &xabort, p.budget);
      const int j = ulist[rank + i * CL];
      const unsigned char* Ks = kv + (size_t)(it % kStages) * 2 * kv_tile;
      const unsigned char* Vs = Ks + kv_tile;
      if (live) {
        // S = Q K^T for my 16 rows x 16 keys: s[nt] = keys 8 nt .. 8 nt + 7 of my quarter
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t qa[4], kb[4];
          ldsm_x4(qa, Qs + swz(q_row, 2 * ks + (lane >> 4), kRowBytes));
          ldsm_x4(kb, Ks + kv_off(16 * kq + (lane & 7) + 8 * (lane >> 4), 2 * ks + ((lane >> 3) & 1)));
          mma_bf16(s[0], qa, kb[0], kb[1]);
          mma_bf16(s[1], qa, kb[2], kb[3]);
        }
        // online softmax in base 2 over my quarter (row maxima over the lane quad); keys
        // past the prefix are -inf
        const int key0 = j * kBlk + 16 * kq + 2 * (lane & 3);
        float x[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            x[nt][e] = key0 + 8 * nt + (e & 1) < p.T_prefix ? s[nt][e] * scale2 : -INFINITY;
        float mx_lo = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
        float mx_hi = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, o));
          mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, o));
        }
        const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
        // a row with no valid key so far subtracts 0: its P is 0 and its (zero) state stays
        const float base_lo = mn_lo == -INFINITY ? 0.f : mn_lo;
        const float base_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
        const float a_lo = ex2(m_lo - base_lo), a_hi = ex2(m_hi - base_hi);
        float pr[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          pr[nt][0] = ex2(x[nt][0] - base_lo); pr[nt][1] = ex2(x[nt][1] - base_lo);
          pr[nt][2] = ex2(x[nt][2] - base_hi); pr[nt][3] = ex2(x[nt][3] - base_hi);
        }
        l_lo = fmaf(l_lo, a_lo, (pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]));
        l_hi = fmaf(l_hi, a_hi, (pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]));
        m_lo = mn_lo;
        m_hi = mn_hi;
        // the S fragments are the A fragments of P (16 rows x 16 keys)
        const uint32_t pa[4] = {pack_bf16x2(pr[0][0], pr[0][1]), pack_bf16x2(pr[0][2], pr[0][3]),
                                pack_bf16x2(pr[1][0], pr[1][1]), pack_bf16x2(pr[1][2], pr[1][3])};
        // V rows past the prefix hold other tokens: P is 0 there, and V is masked to 0 in
        // the B fragments (lane: keys 2 (lane & 3) + {0, 1} in the low / high halves, + 8 in
        // the second register) so that no NaN reaches the sum
        const int nvk = p.T_prefix - (j * kBlk + 16 * kq);
        uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
        if (nvk < 16) {
          const int k0 = 2 * (lane & 3);
          vm0 = (k0 < nvk ? 0x0000ffffu : 0u) | (k0 + 1 < nvk ? 0xffff0000u : 0u);
          vm1 = (k0 + 8 < nvk ? 0x0000ffffu : 0u) | (k0 + 9 < nvk ? 0xffff0000u : 0u);
        }
        // O = alpha O + P V over all of D
#pragma unroll
        for (int n = 0; n < NA; ++n) {
          acc[n][0] *= a_lo; acc[n][1] *= a_lo;
          acc[n][2] *= a_hi; acc[n][3] *= a_hi;
        }
#pragma unroll
        for (int np = 0; np < NA / 2; ++np) {
          uint32_t vb[4];
          ldsm_x4_t(vb, Vs + kv_off(16 * kq + (lane & 7) + 8 * ((lane >> 3) & 1), 2 * np + (lane >> 4)));
          mma_bf16(acc[2 * np], pa, vb[0] & vm0, vb[1] & vm1);
          mma_bf16(acc[2 * np + 1], pa, vb[2] & vm0, vb[3] & vm1);
        }
      }
      // release the stage: the last of the eight warps refills it with the block kStages
      // later in this chunk (after a timeout nothing more is loaded)
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        const int old = atomicAdd(&stage_rel[it % kStages], 1);
        if ((old & (kWarps - 1)) == kWarps - 1 && i + kStages < n_my) {
          __threadfence_block();
          if (!*reinterpret_cast<volatile int*>(&xabort)) issue(it + kStages);
        }
      }
    }

    // ---- merge the four key quarters of every row by log-sum-exp ------------------------
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
    if ((lane & 3) == 0) {
      qml[kq][r_lo] = make_float2(m_lo, l_lo);
      qml[kq][r_hi] = make_float2(m_hi, l_hi);
    }
    __syncthreads();  // (every warp is past the chunk's last block: the ring is free)
    {
      float Ml = -INFINITY, Mh = -INFINITY;
#pragma unroll
      for (int q2 = 0; q2 < kWarps / 2; ++q2) {
        Ml = fmaxf(Ml, qml[q2][r_lo].x);
        Mh = fmaxf(Mh, qml[q2][r_hi].x);
      }
      const float f_lo = Ml == -INFINITY ? 0.f : ex2(m_lo - Ml);
      const float f_hi = Mh == -INFINITY ? 0.f : ex2(m_hi - Mh);
      float* mrow = mb + (size_t)(kq * kRowChunk + r_lo) * D + 2 * (lane & 3);
#pragma unroll
      for (int n = 0; n < NA; ++n) {  // (rows r_lo and r_hi share r & 3)
        const int gcol = (n ^ (r_lo & 3)) << 3;
        *reinterpret_cast<float2*>(mrow + gcol) = make_float2(acc[n][0] * f_lo, acc[n][1] * f_lo);
        *reinterpret_cast<float2*>(mrow + 8 * D + gcol) = make_float2(acc[n][2] * f_hi, acc[n][3] * f_hi);
      }
    }
    __syncthreads();
    M_row = -INFINITY;
    L_row = 0.f;
#pragma unroll
    for (int q2 = 0; q2 < kWarps / 2; ++q2) M_row = fmaxf(M_row, qml[q2][mr].x);
    if (M_row != -INFINITY) {
#pragma unroll
      for (int q2 = 0; q2 < kWarps / 2; ++q2) L_row = fmaf(qml[q2][mr].y, ex2(qml[q2][mr].x - M_row), L_row);
    }
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const int off = (((4 * i + (mc >> 1)) ^ (mr & 3)) << 3) + 4 * (mc & 1);
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q2 = 0; q2 < kWarps / 2; ++q2) {
        const float4 u = *reinterpret_cast<const float4*>(mb + (size_t)(q2 * kRowChunk + mr) * D + off);
        t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
      }
      o_row[i] = t;
    }
    // partial of this chunk -> workspace: row values, then (m, l) (rows that fit one chunk
    // are pushed to the owners' shared memory instead, below)
    if (!dsm && mr < nr) {
      float* wrow = wsu + (size_t)(c0 + mr) * (D + 2);
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        *reinterpret_cast<float2*>(wrow + 32 * i + 4 * mc) = make_float2(o_row[i].x, o_row[i].y);
        *reinterpret_cast<float2*>(wrow + 32 * i + 4 * mc + 2) = make_float2(o_row[i].z, o_row[i].w);
      }
      if (mc == 0) *reinterpret_cast<float2*>(wrow + D) = make_float2(M_row, L_row);
    }
    // every thread's generic accesses to the ring (the merge buffer) before the next chunk's
    // TMA writes into it
    tc::fence_proxy_async();
    __syncthreads();  // (the merge buffer is read; Qs and qml are rewritten by the next chunk)
    if (c + 1 < nchunks && tid == 0 && !*reinterpret_cast<volatile int*>(&xabort))
      for (int it = (c + 1) * n_my; it < (c + 1) * n_my + min(kStages, n_my); ++it) issue(it);
  }

  // ---- barrier (the partials are in the workspace), then merge my output slice ----------
  // Stable rows: the cached output and log-sum-exp, unchanged.  Each thread loads its first
  // chunk here, before the cluster barrier, and stores it after the merge, so that round
  // trip overlaps the barrier and the merge's own loads; any further chunks (more stable
  // rows than threads) are copied after the merge.
  const int srows = S * G;
  const bool copy_o = p.o_cache != p.o && srows > 0;
  const bool copy_l = p.lse_cache != p.lse && srows > 0;
  constexpr int kPerRow = kRowBytes / 16;  // 16-byte chunks of an output row
  const int n16 = srows * kPerRow;
  const int c16 = (n16 + CL - 1) >> cl_log2;
  const int i16 = rank * c16 + tid, i16_end = min(n16, (rank + 1) * c16);
  const int c1 = (srows + CL - 1) >> cl_log2;
  const int li = rank * c1 + tid, l_end = min(srows, (rank + 1) * c1);
  auto stable_row = [&](int r) {  // row r of the stable rows: token stab[r / G], head r % G
    const int s_i = fdiv(r, p.g_div), hh = r - s_i * G;
    return ((size_t)b * Hq + (size_t)g * G + hh) * Tq + stab[s_i];
  };
  const bool have_o = copy_o && i16 < i16_end;
  const bool have_l = copy_l && li < l_end;
  uint4 o_keep = make_uint4(0u, 0u, 0u, 0u);
  size_t o_at = 0, l_at = 0;
  float l_keep = 0.f;
  if (have_o) {
    const int r = i16 / kPerRow;
    o_at = stable_row(r) * kPerRow + (i16 - r * kPerRow);
    o_keep = reinterpret_cast<const uint4*>(p.o_cache)[o_at];
  }
  if (have_l) {
    l_at = stable_row(li);
    l_keep = p.lse_cache[l_at];
  }

  if (!started) {
    cluster_wait();
    started = true;
  }
  const int E = rows * D;
  // an output row's (m, l) and values from the CL partials: the log-sum-exp merge
  auto merge_out = [&](int e, const float2 (&ml)[kMaxCluster], const float (&ov)[kMaxCluster]) {
    const int r = e / D, d = e - r * D;
    float M = -INFINITY;
#pragma unroll
    for (int c2 = 0; c2 < kMaxCluster; ++c2) M = fmaxf(M, ml[c2].x);
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int c2 = 0; c2 < kMaxCluster; ++c2) {
        const float w = ml[c2].x == -INFINITY ? 0.f : ex2(ml[c2].x - M);
        Lsum = fmaf(ml[c2].y, w, Lsum);
        O = fmaf(ov[c2], w, O);
      }
    }
    const int a = fdiv(r, p.g_div), hh = r - a * G;
    const size_t orow = ((size_t)b * Hq + (size_t)g * G + hh) * Tq + act[a];
    p.o[orow * D + d] = __float2bfloat16_rn(M == -INFINITY ? 0.f : O / Lsum);
    if (d == 0) p.lse[orow] = M == -INFINITY ? -INFINITY : (M + log2f(Lsum)) * kLn2;
  };
  if (dsm) {
    // slice of the outputs each CTA merges (a multiple of 4, so a pushed float4 never
    // straddles two)
    const int chunk = ((E + CL - 1) / CL + 3) & ~3;
    if (tid == 0) {
      const int own = max(0, min(E, (rank + 1) * chunk) - rank * chunk);
      tc::mbar_arrive_expect_tx(&xbar[3 + kStages], (uint32_t)(CL * (rows * 8 + own * 4)));
    }
    if (mr < rows) {
      for (int peer = mc; peer < CL; peer += 8)
        st_async(map_rank(pml + rank * kRowChunk + mr, peer), make_float2(M_row, L_row),
                 map_rank(&xbar[3 + kStages], peer));
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        const int e = mr * D + 32 * i + 4 * mc, owner = e / chunk;
        st_async4(map_rank(pacc + rank * chunk + (e - owner * chunk), owner), o_row[i],
                 map_rank(&xbar[3 + kStages], owner));
      }
    }
    tc::mbar_wait(&xbar[3 + kStages], 0, &xabort, p.budget);
    for (int e = rank * chunk + tid; e < min(E, (rank + 1) * chunk); e += kThreads) {
      const int r = e / D;
      float2 ml[kMaxCluster];
      float ov[kMaxCluster];
#pragma unroll
      for (int c2 = 0; c2 < kMaxCluster; ++c2) {
        ml[c2] = c2 < CL ? pml[c2 * kRowChunk + r] : make_float2(-INFINITY, 0.f);
        ov[c2] = c2 < CL ? pacc[c2 * chunk + (e - rank * chunk)] : 0.f;
      }
      merge_out(e, ml, ov);
    }
  } else {
    cluster_arrive_release();  // every partial is in the workspace ...
    cluster_wait();            // ... for every CTA of the cluster
    const int chunk = (E + CL - 1) >> cl_log2;
    const float* wsg = p.ws + unit * kMaxCluster * (size_t)p.rows_max * (D + 2);
    for (int e = rank * chunk + tid; e < min(E, (rank + 1) * chunk); e += kThreads) {
      const int r = e / D, d = e - r * D;
      // every partial's (m, l) and value first (independent loads, one round trip)
      float2 ml[kMaxCluster];
      float ov[kMaxCluster];
#pragma unroll
      for (int c2 = 0; c2 < kMaxCluster; ++c2) {
        ml[c2] = make_float2(-INFINITY, 0.f);
        ov[c2] = 0.f;
        if (c2 < CL) {
          const float* part = wsg + ((size_t)c2 * p.rows_max + r) * (D + 2);
          ml[c2] = __ldcg(reinterpret_cast<const float2*>(part + D));
          ov[c2] = __ldcg(part + d);
        }
      }
      merge_out(e, ml, ov);
    }
  }

  // ---- stable rows: the chunks loaded before the barrier, then any further ones -----------
  if (have_o) reinterpret_cast<uint4*>(p.o)[o_at] = o_keep;
  if (copy_o) {
    for (int i = i16 + kThreads; i < i16_end; i += kThreads) {
      const int r = i / kPerRow;
      const size_t at = stable_row(r) * kPerRow + (i - r * kPerRow);
      reinterpret_cast<uint4*>(p.o)[at] = reinterpret_cast<const uint4*>(p.o_cache)[at];
    }
  }
  if (have_l) p.lse[l_at] = l_keep;
  if (copy_l) {
    for (int r = li + kThreads; r < l_end; r += kThreads) {
      const size_t at = stable_row(r);
      p.lse[at] = p.lse_cache[at];
    }
  }

  // ---- the union list (every CTA holds it; rank 0 writes it) ----------------------------
  if (rank == 0) {
    if (p.union_idx) {
      int32_t* ui = p.union_idx + unit * (size_t)NBp;
      for (int i = tid; i < NBp; i += kThreads) ui[i] = i < U ? ulist[i] : -1;
    }
    if (p.union_cnt && tid == 0) p.union_cnt[unit] = U;
  }
  // after a timeout (the outputs are then undefined) the CTA must not exit while its own
  // copies, or list bytes its peers owe it, are in flight: wait for each (bounded, ignoring
  // the abort) and record the failure
  if (*reinterpret_cast<volatile int*>(&xabort)) {
    if (staged_rows > 0) tc::mbar_drain(&xbar[2], 0, kDrainBudget);
    if (selecting) {
      const int nsel_chunks = (A + kTokChunk - 1) / kTokChunk;
      for (int c = nsel_chunks - 2 < 0 ? 0 : nsel_chunks - 2; c < nsel_chunks; ++c)
        tc::mbar_drain(&xbar[c & 1], (uint32_t)((c >> 1) & 1), kDrainBudget);
    }
    const int n_iss = *reinterpret_cast<volatile int*>(&n_issued);
    for (int i = n_iss - kStages < 0 ? 0 : n_iss - kStages; i < n_iss; ++i)
      tc::mbar_drain(&xbar[3 + i % kStages], (uint32_t)((i / kStages) & 1), kDrainBudget);
    if (dsm) tc::mbar_drain(&xbar[3 + kStages], 0, kDrainBudget);  // (the partials peers owe)
    g_blockquery_status = 1;
  }
}

}  // namespace

cudaError_t read_blockquery_status(int* status, bool reset) {
  cudaError_t err = cudaMemcpyFromSymbol(status, g_blockquery_status, sizeof(int));
  if (err == cudaSuccess && reset) {
    const int zero = 0;
    err = cudaMemcpyToSymbol(g_blockquery_status, &zero, sizeof(int));
  }
  return err;
}

size_t blockquery_workspace_bytes(int B, int Hkv, int G, int D, int Tq) {
  return (size_t)B * Hkv * kMaxCluster * (size_t)Tq * G * (D + 2) * sizeof(float);
}

cudaError_t launch_blockquery(const BlockQueryArgs& a, cudaStream_t stream) {
  const int units = a.B * a.Hkv;
  int CL = units <= 14 ? 16 : (units <= 37 ? 8 : 4);
  const int NBp = (a.T_prefix + kBlk - 1) / kBlk;
  BQParams p{};
  if (!kv_tensor_maps(a.k, a.v, a.D, a.T_cap, a.B * a.Hkv, &p.tmk, &p.tmv)) return cudaErrorInvalidValue;
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
  p.NBp = NBp;
  p.g_div = make_fastdiv((uint32_t)a.G);
  p.budget = wait_budget();
  auto kernel = a.D == 128 ? blockquery_kernel<128> : blockquery_kernel<64>;
  // per head dim and device: the largest dynamic smem size set so far and the (cluster
  // size, smem) pairs found schedulable (thread-safe; see launch_cache.h)
  static LaunchRecord rec128, rec64;
  LaunchRecord& rec = a.D == 128 ? rec128 : rec64;
  int dev = 0;
  {
    const cudaError_t derr = current_device(&dev);
    if (derr != cudaSuccess) return derr;
  }
  for (;;) {
    p.per_max = (NBp + CL - 1) / CL;
    if (p.per_max < 1) p.per_max = 1;
    p.per_div = make_fastdiv((uint32_t)p.per_max);
    const BQLayout Lo = bq_layout(a.D, p.per_max, NBp, a.G, NBp <= a.topk);
    const int smem = (int)Lo.total;
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL, a.Hkv, a.B);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    {
      std::lock_guard<std::mutex> lock(rec.mu);
      err = rec.ensure_smem(dev, kernel, smem, true);
      if (err != cudaSuccess) return err;
      if (!rec.shape_ok(dev, CL, smem)) {
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
        rec.remember_shape(dev, CL, smem);
      }
    }
    cfg.numAttrs = 2;  // launched as a programmatic dependent of the previous kernel
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
// per device: the scratch's device address and the id of the context it was looked up in
struct ScratchSlot {
  void* ptr = nullptr;
  unsigned long long ctx = 0;
};
std::mutex g_scratch_mutex;
ScratchSlot g_scratch[kMaxDevices];
}  // namespace

size_t blockquery_static_workspace_bytes() { return kStaticWorkspaceBytes; }

// Device address of the fixed scratch on the current device.  The first call on a device
// looks it up with cudaGetSymbolAddress (the host-side name of the array is not a device
// address); later calls reuse it while the device's context is the same one.  A device
// reset (cudaDeviceReset) destroys the context and reloads the module, so a call after it
// sees a new context id and looks the address up again.
cudaError_t blockquery_static_workspace(void** ptr) {
  int dev = 0;
  cudaError_t err = current_device(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchSlot& slot = g_scratch[dev];
  unsigned long long ctx = 0;
  const bool known_ctx = current_context_id(&ctx);
  if (slot.ptr == nullptr || !known_ctx || ctx != slot.ctx) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_blockquery_scratch);
    if (err != cudaSuccess) return err;
    // (the lookup made the device's primary context current on this thread)
    unsigned long long now = 0;
    slot.ctx = current_context_id(&now) ? now : 0;
    slot.ptr = p;
  }
  *ptr = slot.ptr;
  return cudaSuccess;
}

}  // namespace lsa
