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
//   * Attention rows (active token x head) are processed 32 at a time (two mma m-tiles):
//     K/V blocks arrive as TMA boxes (128-byte swizzle) on a 2-stage ring with per-stage
//     mbarriers, S = Q K^T and O += P V on mma.sync m16n8k16 bf16, online softmax in base 2.
//   * Each CTA writes its per-row partial (acc, m, l) to the caller's workspace; after a
//     cluster barrier every CTA merges a 1/CL slice of the outputs by log-sum-exp (all
//     loads issued before use).  Stable rows are copied from the cache; rank 0 writes the
//     union list.
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
constexpr int kSStride = 68;    // fp32 row stride of the score tile
constexpr int kQStride = 132;   // fp32 row stride of the summed queries (bank spread)
constexpr int kStageRows = 64;  // summary rows of a CTA's slice staged by one bulk copy
constexpr int kMaxUnion = kMaxTq * kLP;  // a union holds at most Tq * topk blocks
static_assert(kTokChunk == 8, "the scoring maps lane l to token l & 7");

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

__host__ __device__ inline size_t al128(size_t x) { return (x + 127) & ~(size_t)127; }

struct BQLayout {
  size_t act, stab, ulist, ubits, qs, ss, ps, alpha, pml, pacc, region, total;
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
  L.ss = off;     off = al128(off + (size_t)kRowChunk * kSStride * 4);
  L.ps = off;     off = al128(off + (size_t)kRowChunk * kBlk * 2);
  L.alpha = off;  off = al128(off + kRowChunk * 4);
  // the partials pushed by the cluster's CTAs when the rows fit one chunk: every CTA's
  // (m, l) of every row and its part of this CTA's slice of the outputs
  L.pml = off;    off = al128(off + (size_t)kMaxCluster * kRowChunk * 8);
  L.pacc = off;   off = al128(off + (size_t)kRowChunk * D * 4 + kMaxCluster * 8);
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
  float* Ss = reinterpret_cast<float*>(smem + Lo.ss);
  unsigned char* Ps = smem + Lo.ps;
  float* alpha_s = reinterpret_cast<float*>(smem + Lo.alpha);
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
  const int nchunks = (rows + kRowChunk - 1) / kRowChunk;
  // one chunk of rows: the partials go straight into the shared memory of the CTAs that
  // merge them (st.async, counted on the owner's mbarrier), with no workspace round trip and
  // no cluster barrier; more rows go through the caller's workspace
  const bool dsm = nchunks == 1;
  const int total = nchunks * n_my;
  float* wsu = p.ws + (unit * kMaxCluster + rank) * (size_t)p.rows_max * (D + 2);
  int issued = 0;
  // the next block in processing order: K and V as TMA boxes (128-byte swizzled tiles)
  // issued by thread 0, landing on the stage's mbarrier
  auto issue = [&]() {
    const int stg = issued % kStages;
    if (tid == 0) {
      unsigned char* st = kv + (size_t)stg * 2 * kv_tile;
      const int j = ulist[rank + (issued % n_my) * CL];
      tc::fence_proxy_async();  // earlier generic accesses to this stage come first
      tc::mbar_arrive_expect_tx(&xbar[3 + stg], (uint32_t)(2 * kv_tile));
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        tc::tma_load_3d(st + h * 8192, &p.tmk, h * 64, j * kBlk, (int)unit, &xbar[3 + stg]);
        tc::tma_load_3d(st + kv_tile + h * 8192, &p.tmv, h * 64, j * kBlk, (int)unit, &xbar[3 + stg]);
      }
    }
    ++issued;
  };
  __syncthreads();  // (the selection buffers that share the ring are dead)
  while (issued < kStages && issued < total) issue();

  constexpr int NT = D / 64;  // n8 tiles of the output per warp
  const float scale2 = p.scale * kLog2e;
  const int srow = tid >> 3, ssub = tid & 7;  // softmax mapping: 32 rows x 8 threads
  float m_run = -INFINITY, l_run = 0.f;
  float acc[2][NT][4];

  for (int c = 0; c < nchunks; ++c) {
    const int c0 = c * kRowChunk;
    const int nr = min(kRowChunk, rows - c0);
    // query rows of the chunk (chunk 0 was requested at the start)
    if (c > 0) {
      load_attn_rows(c0);
      cp_async_commit();
    }
    cp_async_wait<0>();
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
      tc::mbar_wait(&xbar[3 + it % kStages], (uint32_t)((it / kStages) & 1), &xabort, p.budget);
      __syncthreads();
      const int j = ulist[rank + i * CL];
      const unsigned char* Ks = kv + (size_t)(it % kStages) * 2 * kv_tile;
      const unsigned char* Vs = Ks + kv_tile;
      {  // V rows past the prefix hold other tokens: zero them (P is 0 there, V must be finite)
        const int nv = min(kBlk, p.T_prefix - j * kBlk);
        for (int id = tid; id < (kBlk - nv) * (D / 8); id += kThreads) {
          const int r = nv + id / (D / 8), cc = id % (D / 8);
          *reinterpret_cast<uint4*>(const_cast<unsigned char*>(Vs) + kv_off(r, cc)) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      // S = Q K^T: warp w -> tokens 8w .. 8w+7, both m-tiles
      {
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < D / 16; ks += 2) {
          uint32_t kb[4];
          ldsm_x4(kb, Ks + kv_off(8 * warp + (lane & 7), 2 * ks + (lane >> 3)));
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
          ldsm_x4_t(vb, Vs + kv_off(vrow, 2 * warp + (lane >> 4)));
        } else {
          uint32_t v2[2];
          ldsm_x2_t(v2, Vs + kv_off(vrow, warp));
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
    // partial of this chunk -> workspace: acc rows, then (m, l) (rows that fit one chunk are
    // pushed to the owners' shared memory instead, below)
#pragma unroll
    for (int mt = 0; mt < 2 && !dsm; ++mt) {
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
    if (!dsm && ssub == 0 && srow < nr)
      *reinterpret_cast<float2*>(wsu + (size_t)(c0 + srow) * (D + 2) + D) = make_float2(m_run, l_run);
    __syncthreads();  // Qs / stats are rewritten by the next chunk
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
    // slice of the outputs each CTA merges (even, so a pushed pair never straddles two)
    const int chunk = ((E + CL - 1) / CL + 1) & ~1;
    if (tid == 0) {
      const int own = max(0, min(E, (rank + 1) * chunk) - rank * chunk);
      tc::mbar_arrive_expect_tx(&xbar[3 + kStages], (uint32_t)(CL * (rows * 8 + own * 4)));
    }
    if (srow < rows)
      for (int peer = ssub; peer < CL; peer += 8)
        st_async(map_rank(pml + rank * kRowChunk + srow, peer), make_float2(m_run, l_run),
                 map_rank(&xbar[3 + kStages], peer));
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int d = (D == 128 ? 16 * warp : 8 * warp) + 8 * nt + 2 * (lane & 3);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int r = 16 * mt + (lane >> 2) + 8 * half;
          if (r < rows) {
            const int e = r * D + d, owner = e / chunk;
            st_async(map_rank(pacc + rank * chunk + (e - owner * chunk), owner),
                     make_float2(acc[mt][nt][2 * half], acc[mt][nt][2 * half + 1]),
                     map_rank(&xbar[3 + kStages], owner));
          }
        }
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
    for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
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
