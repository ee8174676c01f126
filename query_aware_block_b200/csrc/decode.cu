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
// How (B200).  A decode step moves only a few MB, so the kernel is built for latency:
//   * A cluster of CL CTAs (16, 8 or 4) owns one (b, g); 2 CTAs fit per SM, so a 16-CTA
//     cluster per KV head fits in one wave.  At launch thread 0 of every CTA starts one bulk
//     copy (cp.async.bulk, the copy engine) of its slice of the summary rows into shared
//     memory (the slice is fixed by the capacity, so the copy does not wait for the sequence
//     length); CTAs that own a forced block also start its K/V as TMA boxes, so that copy
//     overlaps the scan.  The group's query rows follow (16-byte cp.async).
//   * Scoring: 4 threads per summary row (quarter-warp-uniform lane mapping: conflict-free
//     128-bit shared loads) against the summed query in shared memory.
//   * Each CTA ranks its candidates (64-bit keys: score, then lower index) and PUSHES its
//     sorted local top-m list into every peer's shared memory with st.async, whose bytes
//     count toward an mbarrier in the receiving CTA: each CTA waits only until the CL lists
//     have landed (no cluster-wide barrier), then merges them with a tree of warp-wide
//     bitonic merges (shuffles only; levels hand over through pairwise named barriers) and
//     derives the same global top-m as its peers; warp 0 ends the tree holding the list and
//     starts the TMA copy of this CTA's first scored block at once.
//     DSMEM is touched only after a split arrive(relaxed)/wait barrier that proves every
//     CTA of the cluster has started and initialised its mbarriers.
//   * Overlapped launch (optional, programmatic dependent launch): the summary rows and the
//     K/V of the forced blocks other than the newest one are requested before the kernel
//     waits for the previous kernel of the stream; q and the newest block after it.
//   * The selected blocks are dealt round-robin.  bf16: a 64-token block of K and V (16 KB
//     each at D = 128) arrives as TMA boxes (128-byte swizzle) on a per-stage mbarrier
//     (2-stage ring); the G <= 16 query heads are the M = 16 rows of mma.sync m16n8k16 for
//     S = Q K^T and O += P V.  fp32: 16-byte cp.async into padded rows and CUDA-core FMA.
//     Online softmax in base 2 with fp32 statistics.
//   * Each CTA pushes its partial (m, l) and the slices of its accumulator to the CTAs
//     that own those output elements (st.async again, second mbarrier); each CTA waits for
//     its CL partials and merges its 1/CL slice by log-sum-exp from its own shared memory.
//     Every byte a CTA receives is counted by its own mbarriers and waited for before it
//     ends, so no CTA leaves while a peer may still write into it; no trailing barrier.
//   * Optionally the CTA that attends the sequence's last block (always a forced local
//     block) also refreshes that block's summary from the keys it staged: the summary
//     update of a decode step costs no extra launch and no extra HBM read.
// No global scratch memory.  The mbarrier waits are bounded (about 2 s of clock); if one
// runs out the launch's outputs are undefined and a device status word records it.
#include <math.h>

#include <type_traits>

#include "cluster.cuh"
#include "lsa_common.cuh"
#include "launch_cache.h"
#include "lsa_internal.h"
#include "tcgen05.cuh"

namespace lsa {
namespace {

typedef unsigned long long u64;

// Set when a bounded wait on a cross-CTA exchange runs out (the outputs of that launch are
// then undefined); read and cleared by the host.
__device__ int g_decode_status = 0;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 16;       // query-head rows per group (G <= 16): the mma M dimension
constexpr int kMaxTopk = 64;
constexpr int kMaxCluster = 16;
constexpr int kStages = 2;
constexpr int kSStride = 72;    // fp32 row stride of the score tile (bank spread)
// A scoring pass covers kPassRows summary rows, 8 per warp; the local rank count after it
// gives each key 4 threads (lane l of warp w: key 8w + (l & 7), quarter l >> 3 of the keys).
constexpr int kPassRows = kWarps * 8;

struct alignas(64) Params {
  // bf16 K and V as [B * Hkv][T_cap][D], box {64, 64, 1}, 128-byte swizzle (unused for fp32)
  CUtensorMap tmk;
  CUtensorMap tmv;
  const void* q;
  const void* k;
  const void* v;
  int Hkv, G, T_cap, NB_cap;
  const int32_t* seqlens;
  const float* summ;
  float* summ_w;          // refresh target (fused mode), or null
  const int32_t* idx_in;
  const int32_t* nsel_in;
  int topk, n_sink, n_local;
  float scale;            // natural-log softmax scale
  int32_t* idx_out;
  int32_t* nsel_out;
  float* scores_out;
  void* o;
  float* lse;
  int per_max;            // max summary rows scored by one CTA
  int m_pad;              // power of two >= topk
  int lp;                 // length of an exchanged candidate list: max(16, m_pad)
  int chunk;              // output elements merged by one CTA (even)
  int pdl;                // launched as a programmatic dependent of the previous kernel
  long long budget;       // clock-cycle limit of every bounded wait
  FastDiv chunk_div;      // division by chunk
};

__host__ __device__ inline size_t align128(size_t x) { return (x + 127) & ~(size_t)127; }


// Shared-memory carve-up (byte offsets), identical on host and device.
struct Layout {
  size_t qs, qsum, keys, top, work, all, order, kv, ss, ps, alpha, ml_in, pacc_in, total;
  size_t kv_row, kv_tile;  // bytes per K/V row in smem, bytes per 64-row tile
};

__host__ __device__ inline Layout make_layout(int elem_bytes, int D, int per_max, int m_pad) {
  Layout L;
  size_t off = 0;
  const int lp = m_pad < 16 ? 16 : m_pad;
  const int nwork = (m_pad + kThreads) > (kMaxCluster / 2) * lp ? (m_pad + kThreads) : (kMaxCluster / 2) * lp;
  const bool f32 = elem_bytes == 4;
  L.kv_row = f32 ? (size_t)(D + 4) * 4 : (size_t)D * 2;
  L.kv_tile = L.kv_row * kBlk;
  L.qs = off;      off = align128(off + (size_t)kRows * D * elem_bytes);
  L.qsum = off;    off = align128(off + (size_t)D * 4);
  L.keys = off;    off = align128(off + (size_t)per_max * 8);
  L.top = off;     off = align128(off + (size_t)lp * 8);
  L.work = off;    off = align128(off + (size_t)nwork * 8);
  L.all = off;     off = align128(off + (size_t)kMaxCluster * lp * 8);
  L.order = off;   off = align128(off + (size_t)kMaxTopk * 4);
  // (the K/V ring is placed at the first 1024-byte boundary inside this range: a 128-byte
  // swizzled TMA box must land 1024-byte aligned)
  L.kv = off;      off = align128(off + (size_t)kStages * 2 * L.kv_tile + 1024);
  L.ss = off;      off = align128(off + (size_t)kRows * kSStride * 4);
  L.ps = off;      off = align128(off + (size_t)kRows * kBlk * 4);
  L.alpha = off;   off = align128(off + (size_t)kRows * 4);
  L.ml_in = off;   off = align128(off + (size_t)kMaxCluster * kRows * 8);
  L.pacc_in = off; off = align128(off + (size_t)(kRows * D + 2 * kMaxCluster) * 4);
  L.total = off;
  return L;
}

// ---- selection helpers ------------------------------------------------------------------

// Top-m of n keys (0 = not a candidate) into top[0..min(m, #valid)), descending; top[]
// must be zero on entry.  Candidates are taken kThreads at a time together with the
// current list; a candidate's rank is the number of larger keys (keys are unique).
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
        int u = 0;
        for (; u + 8 <= w; u += 8) {
#pragma unroll
          for (int k2 = 0; k2 < 8; ++k2) r += work[u + k2] > x;
        }
        for (; u < w; ++u) r += work[u] > x;
        if (r < m) top[r] = x;
      }
      nvalid += __syncthreads_count(x != 0ull);
    }
    cur = min(m, nvalid);
  }
  __syncthreads();
}

// Top list of the union of CL descending lists of 16E keys (zero padded) stored at
// lists[c * 16E]: pairs are merged one warp each, level by level, ping-ponging between
// `lists` and `work`.  Returns the buffer that holds the final list.
template <int E>
__device__ const u64* merge_lists(u64* lists, u64* work, int CL) {
  constexpr int LP = 16 * E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  u64* src = lists;
  u64* dst = work;
  for (int n = CL; n > 1; n >>= 1) {
    for (int pr = warp; pr < (n >> 1); pr += kWarps) {
      const u64* A = src + (2 * pr) * LP;
      const u64* Bl = src + (2 * pr + 1) * LP;
      u64 x[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int pos = lane * E + e;
        x[e] = pos < LP ? A[pos] : Bl[2 * LP - 1 - pos];
      }
      warp_merge_desc<E>(x);
      if (lane < 16) {
#pragma unroll
        for (int e = 0; e < E; ++e) dst[pr * LP + lane * E + e] = x[e];
      }
    }
    __syncthreads();
    u64* t = src;
    src = dst;
    dst = t;
  }
  return src;
}

// Global top list of the union of CL (a power of two, 2..16) descending lists of 16 keys
// at lists[c * 16] (zero padded), as a tree of warp-wide bitonic merges: warp w first
// merges lists 2w and 2w + 1; at each later level a warp keeps its result in registers and
// takes its partner warp's from shared memory after a pairwise named barrier (ids 1..7, one
// per producing warp), so no level waits for the whole block.  Writes order[nf + r] for
// r < m (m <= 16) from warp 0; the caller synchronises the block afterwards.
__device__ __forceinline__ void merge_tree16(const u64* lists, u64* work, int CL, int m, int nf, int* order) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int npairs = CL >> 1;
  if (warp >= npairs) return;
  u64 x[1];
  x[0] = lane < 16 ? lists[(2 * warp) * 16 + lane] : lists[(2 * warp + 1) * 16 + 31 - lane];
  warp_merge_desc<1>(x);
  for (int s = 1; s < npairs; s <<= 1) {
    if (warp & s) {  // producer at this level: hand the top 16 to warp - s and leave
      if (lane < 16) work[warp * 16 + lane] = x[0];
      asm volatile("bar.arrive %0, 64;" ::"r"(warp) : "memory");
      return;
    }
    if (warp + s >= npairs) continue;  // no partner at this level
    asm volatile("bar.sync %0, 64;" ::"r"(warp + s) : "memory");
    if (lane >= 16) x[0] = work[(warp + s) * 16 + 31 - lane];
    warp_merge_desc<1>(x);
  }
  if (lane < m) order[nf + lane] = key_block(x[0]);
}

// ---- the kernel ---------------------------------------------------------------------

template <typename T, int D, int MODE>
__global__ void __launch_bounds__(kThreads, 2) decode_cluster_kernel(const __grid_constant__ Params p) {
  // the parameter block is fetched all at once here (fields spaced < 32 bytes apart), not
  // one constant-cache miss after another on first use
  asm volatile("" ::"l"(p.q), "r"(p.T_cap), "l"(p.summ_w), "r"(p.topk), "l"(p.nsel_out), "l"(p.lse),
               "r"(p.chunk));
  const int CL = cluster_size();
  const int rank = cluster_rank();
  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  const int Tb = checked_range(p.seqlens[b], 0, p.T_cap, kBoundsSeqlen, kSiteDecode);
  const int NB = (Tb + kBlk - 1) / kBlk;
  constexpr bool kF32 = sizeof(T) == 4;
  constexpr int kRowBytesQ = D * (int)sizeof(T);

  // mbarriers: [0] and [1] count the bytes of the two cross-CTA exchanges and [2] the bulk
  // copy of this CTA's summary rows (one phase each); [3 + s] the TMA loads into K/V stage s
  // (bf16; one phase per use of the stage)
  __shared__ __align__(8) uint64_t xbar[3 + kStages];
  __shared__ int xabort;
  extern __shared__ __align__(1024) unsigned char smem[];
  const Layout Lo = make_layout((int)sizeof(T), D, p.per_max, p.m_pad);
  unsigned char* Qs = smem + Lo.qs;
  u64* keys = reinterpret_cast<u64*>(smem + Lo.keys);
  u64* top = reinterpret_cast<u64*>(smem + Lo.top);
  u64* work = reinterpret_cast<u64*>(smem + Lo.work);
  u64* all = reinterpret_cast<u64*>(smem + Lo.all);
  int* order = reinterpret_cast<int*>(smem + Lo.order);
  unsigned char* kv = smem + Lo.kv + ((1024u - ((tc::smem_u32(smem) + (uint32_t)Lo.kv) & 1023u)) & 1023u);
  float* Ss = reinterpret_cast<float*>(smem + Lo.ss);
  unsigned char* Ps = smem + Lo.ps;
  float* alpha_s = reinterpret_cast<float*>(smem + Lo.alpha);
  float2* ml_in = reinterpret_cast<float2*>(smem + Lo.ml_in);
  float* pacc_in = reinterpret_cast<float*>(smem + Lo.pacc_in);
  const int kv_row = (int)Lo.kv_row;
  const int kv_tile = (int)Lo.kv_tile;

  const size_t unit = (size_t)b * p.Hkv + g;
  const T* qg = static_cast<const T*>(p.q) + ((size_t)b * p.Hkv * G + (size_t)g * G) * D;
  const T* kbase = static_cast<const T*>(p.k) + unit * (size_t)p.T_cap * D;
  const T* vbase = static_cast<const T*>(p.v) + unit * (size_t)p.T_cap * D;
  const bool select = MODE != MODE_ATTEND;

  // ---- the first pass of this CTA's summary rows, requested before anything else with one
  // bulk copy (the copy engine, not the load/store unit): the slice [j0, j0 + per) depends
  // on the capacity only, so it need not wait for the sequence length, and the previous
  // kernel of the stream cannot write it.  Stage 1 of the K/V ring holds it while scanning.
  const int per = p.per_max;
  const int j0 = rank * per;
  float* sumbuf = reinterpret_cast<float*>(kv + 2 * (size_t)kv_tile);
  const bool may_scan = select && p.NB_cap > p.topk;
  const int staged_rows = may_scan ? max(0, min(min(per, p.NB_cap - j0), kPassRows)) : 0;
  if (tid == 0) {
    tc::mbar_init(&xbar[0], 1);
    tc::mbar_init(&xbar[1], 1);
    tc::mbar_init(&xbar[2], 1);
    for (int st = 0; st < kStages; ++st) tc::mbar_init(&xbar[3 + st], 1);
    xabort = 0;
    tc::fence_mbar_init();
    if constexpr (!kF32) {
      tc::prefetch_tmap(&p.tmk);
      tc::prefetch_tmap(&p.tmv);
    }
    if (staged_rows > 0) {
      const uint32_t bytes = (uint32_t)(staged_rows * D * 4);
      tc::mbar_arrive_expect_tx(&xbar[2], bytes);
      tc::bulk_load(sumbuf, p.summ + (unit * (size_t)p.NB_cap + j0) * D, bytes, &xbar[2]);
    }
  }
  // DSMEM may be written only once every CTA of the cluster runs (and has initialised its
  // barriers): arrive now, wait late
  cluster_arrive_relaxed();
  bool started = false;  // uniform: the start barrier has been waited on

  // The query rows (the mma's A tile; rows >= G zero) by 16-byte cp.async, one commit
  // group.  Without overlapped launch (nothing to wait for) and with the K/V on TMA (bf16:
  // no other cp.async group), they are requested here, before anything waits for the
  // sequence length; otherwise after the wait for the previous kernel, which may write q.
  auto stage_q = [&]() {
    constexpr int kQChunks = kRows * kRowBytesQ / 16;
    for (int id = tid; id < kQChunks; id += kThreads) {
      const int row = id / (kRowBytesQ / 16), c = id % (kRowBytesQ / 16);
      cp_async16(Qs + (kF32 ? row * kRowBytesQ + c * 16 : swz(row, c, kRowBytesQ)),
                 qg + (size_t)(row < G ? row : 0) * D + c * (16 / (int)sizeof(T)), row < G);
    }
    cp_async_commit();
  };
  const bool q_early = !kF32 && !p.pdl;
  if (q_early) stage_q();

  // ---- which blocks: forced / all known up front; order[i] is handled by CTA i % CL ----
  const bool all_blocks = select && NB <= p.topk;
  const int nf = (select && !all_blocks) ? p.n_sink + p.n_local : 0;  // disjoint: NB > topk
  int n_order;
  if (select) {
    n_order = all_blocks ? NB : p.topk;
    const int known = all_blocks ? NB : nf;
    for (int i = tid; i < known; i += kThreads)
      order[i] = all_blocks ? i : (i < p.n_sink ? i : NB - p.n_local + (i - p.n_sink));
  } else {
    n_order = max(0, min(checked_range(__ldcg(p.nsel_in + unit), 0, p.topk, kBoundsCount, kSiteDecode), p.topk));
    for (int i = tid; i < n_order; i += kThreads)
      order[i] = checked_range(__ldcg(p.idx_in + unit * p.topk + i), -1, NB - 1, kBoundsIndex, kSiteDecode);
  }
  auto known_block = [&](int i) {
    const int o = rank + i * CL;
    return all_blocks ? o : (o < p.n_sink ? o : NB - p.n_local + (o - p.n_sink));
  };
  for (int i = tid; i < p.lp; i += kThreads) top[i] = 0ull;

  // ---- before waiting on the previous kernel of the stream: copies of data that kernel
  // cannot have written (the K/V of the known blocks except the sequence's newest one, and
  // the summary rows above).  With overlapped launch the caller vouches for this.
  int issued = 0;  // my blocks whose copies were started, in processing order
  // Start the copy of block j's K and V into stage issued % kStages (every thread calls
  // this).  bf16: TMA boxes issued by thread 0 that land on the stage's mbarrier; fp32:
  // 16-byte cp.async by every thread, one commit group per block.
  auto issue_block = [&](int j) {
    const int stg = issued % kStages;
    unsigned char* st = kv + (size_t)stg * 2 * kv_tile;
    if constexpr (kF32) {
      stage_block<T, D, kThreads>(st, st + kv_tile, kbase, vbase, j, Tb, kv_row);
      cp_async_commit();
    } else {
      if (tid == 0) {
        tc::fence_proxy_async();  // earlier generic accesses to this stage come first
        uint64_t* bar = &xbar[3 + stg];
        if (j >= 0) {
          tc::mbar_arrive_expect_tx(bar, (uint32_t)(2 * kv_tile));
#pragma unroll
          for (int h = 0; h < D / 64; ++h) {
            tc::tma_load_3d(st + h * 8192, &p.tmk, h * 64, j * kBlk, (int)unit, bar);
            tc::tma_load_3d(st + kv_tile + h * 8192, &p.tmv, h * 64, j * kBlk, (int)unit, bar);
          }
        } else {
          tc::mbar_arrive(bar);  // nothing to copy: the phase completes empty
        }
      }
    }
    ++issued;
  };
  const int known = all_blocks ? NB : nf;
  const int n_known = (MODE == MODE_FUSED && known > rank) ? (known - rank + CL - 1) >> (__ffs(CL) - 1) : 0;
  const bool scan = select && !all_blocks;
  const int nloc = scan ? max(0, min(NB, j0 + per) - j0) : 0;
  // while scanning, stage 1 holds the first pass of this CTA's summary rows
  const int early_stages = scan ? 1 : kStages;
  // a short sequence that scans nothing reuses stage 1 once the summary copy has landed
  // (the barrier makes thread 0's mbarrier initialisation visible first)
  if (!scan && staged_rows > 0) {
    __syncthreads();
    tc::mbar_wait(&xbar[2], 0, &xabort, p.budget);
  }
  if (MODE == MODE_FUSED) {
    while (issued < early_stages && issued < n_known && known_block(issued) != NB - 1) {
      issue_block(known_block(issued));
    }
  }
  // After a timeout (the launch's outputs are then undefined) the CTA must not exit while
  // copies it issued, or bytes its cluster peers owe it, are still in flight: every thread
  // that sees the abort waits for each of them (bounded, ignoring the abort) and records
  // the failure in the status word.
  auto drain_on_abort = [&](bool lists, bool partials) {
    if (!*reinterpret_cast<volatile int*>(&xabort)) return;
    if (staged_rows > 0) tc::mbar_drain(&xbar[2], 0, kDrainBudget);
    if (lists) tc::mbar_drain(&xbar[0], 0, kDrainBudget);
    if (partials) tc::mbar_drain(&xbar[1], 0, kDrainBudget);
    if constexpr (!kF32) {
      for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
        tc::mbar_drain(&xbar[3 + i % kStages], (uint32_t)((i / kStages) & 1), kDrainBudget);
    }
    g_decode_status = 1;
  };
  pdl_trigger();
  pdl_wait();

  // ---- query rows (the mma's A tile; rows >= G zero), then the remaining known blocks ----
  if (!q_early) stage_q();
  const int issued_before_q = issued;
  bool newest_issued = false;
  if (MODE == MODE_FUSED && scan && issued == 0 && n_known > 0) {  // the newest block, now
    issue_block(known_block(0));
    newest_issued = true;
  }
  if (MODE == MODE_FUSED && !scan) {
    while (issued < kStages && issued < n_known) {
      issue_block(known_block(issued));
    }
  }

  // ---- selection --------------------------------------------------------------------
  bool early = false;  // (uniform) the first block's copy was started by warp 0 after the merge
  if (scan) {
    // the staged query rows: only the newest block's copy may be in flight after them
    if (kF32 && newest_issued) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncthreads();
    const int m = p.topk - nf;
    // summed, scaled query row of the group (fp32, shared), from the staged query rows
    float* qsum = reinterpret_cast<float*>(smem + Lo.qsum);
    for (int d = tid; d < D; d += kThreads) {
      float acc = 0.f;
      for (int h = 0; h < G; ++h) {
        if constexpr (kF32)
          acc += reinterpret_cast<const float*>(Qs + h * kRowBytesQ)[d];
        else
          acc += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
              Qs + swz(h, (2 * d) >> 4, kRowBytesQ) + ((2 * d) & 15)));
      }
      qsum[d] = acc * p.scale;
    }
    __syncthreads();
    // the summary rows (the barriers above ordered thread 0's mbarrier initialisation first)
    if (staged_rows > 0) tc::mbar_wait(&xbar[2], 0, &xabort, p.budget);
    // lane l of warp w scores rows 8w + (l >> 3) and 8w + 4 + (l >> 3) of a pass, taking
    // 16-byte chunks cs, cs + 8, ... (cs = l & 7): a quarter-warp reads 128 contiguous bytes
    // of one row (conflict-free), and every lane needs the same D / 8 summed-query values
    // for both of its rows
    constexpr int kCPL = D / 32;  // chunks of a row per lane
    const int cs = lane & 7;
    float qv[4 * kCPL];
#pragma unroll
    for (int m = 0; m < kCPL; ++m) {
      const float4 v = reinterpret_cast<const float4*>(qsum)[cs + 8 * m];
      qv[4 * m] = v.x; qv[4 * m + 1] = v.y; qv[4 * m + 2] = v.z; qv[4 * m + 3] = v.w;
    }
    const float* grow = p.summ + (unit * (size_t)p.NB_cap + j0) * D;
    // one pass: rows base .. base + kPassRows - 1 of this CTA's slice, from the rows staged
    // in shared memory (the first pass) or from global memory (any later one); the two
    // sources are separate instantiations so that the staged rows are read with shared loads
    auto score_pass = [&](int base, auto staged) {
      float dot[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int oo = base + warp * 8 + (lane >> 3) + 4 * i;
        float a0 = 0.f, a1 = 0.f;
        if (oo < nloc) {
#pragma unroll
          for (int m = 0; m < kCPL; ++m) {
            float4 v;
            if constexpr (decltype(staged)::value)
              v = reinterpret_cast<const float4*>(sumbuf + oo * D)[cs + 8 * m];
            else
              v = __ldg(reinterpret_cast<const float4*>(grow + (size_t)oo * D) + cs + 8 * m);
            a0 = fmaf(v.x, qv[4 * m], a0);
            a1 = fmaf(v.y, qv[4 * m + 1], a1);
            a0 = fmaf(v.z, qv[4 * m + 2], a0);
            a1 = fmaf(v.w, qv[4 * m + 3], a1);
          }
        }
        dot[i] = a0 + a1;
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        dot[0] += __shfl_xor_sync(0xffffffffu, dot[0], o);
        dot[1] += __shfl_xor_sync(0xffffffffu, dot[1], o);
      }
      if (cs == 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int oo = base + warp * 8 + (lane >> 3) + 4 * i;
          if (oo < nloc) {
            const int j = j0 + oo;
            const bool forced = j < p.n_sink || j >= NB - p.n_local;
            keys[oo] = forced ? 0ull : make_key(dot[i], j);
            if (p.scores_out) p.scores_out[unit * p.NB_cap + j] = dot[i];
          } else if (oo < kPassRows && oo < per) {
            keys[oo] = 0ull;  // the rank count below reads a full pass
          }
        }
      }
    };
    if (nloc > 0) score_pass(0, std::true_type{});
    for (int base = kPassRows; base < nloc; base += kPassRows) score_pass(base, std::false_type{});
    if (nloc == 0) {  // no pass ran: the rank count below still reads a full pass
      for (int i = tid; i < min(kPassRows, per); i += kThreads) keys[i] = 0ull;
    }
    __syncthreads();
    // local top-m, sorted, zero padded to lp
    if (nloc <= kPassRows && per >= kPassRows) {
      // 4 threads per key (the lane mapping of the scoring), each counting the larger keys
      // in a quarter of the pass
      const int i = warp * 8 + (lane & 7), part = lane >> 3;
      const u64 x = keys[i];
      const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(keys + part * (kPassRows / 4));
      int r = 0;
#pragma unroll
      for (int q4 = 0; q4 < kPassRows / 8; ++q4) {
        const ulonglong2 kk = k2[q4];
        r += (kk.x > x) + (kk.y > x);
      }
      r += __shfl_xor_sync(0xffffffffu, r, 8);
      r += __shfl_xor_sync(0xffffffffu, r, 16);
      if (part == 0 && x != 0ull && r < m) top[r] = x;
      __syncthreads();
    } else if (nloc <= kThreads) {
      const u64 x = tid < nloc ? keys[tid] : 0ull;
      if (x != 0ull) {
        int r = 0, u = 0;
        for (; u + 8 <= nloc; u += 8) {
          const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(keys + u);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const ulonglong2 kk = k2[q4];
            r += (kk.x > x) + (kk.y > x);
          }
        }
        for (; u < nloc; ++u) r += keys[u] > x;
        if (r < m) top[r] = x;
      }
      __syncthreads();
    } else {
      block_topm(keys, nloc, m, top, work);
    }
    // push the list into every peer (all[rank][*] on each CTA), wait until all CL lists
    // have landed here, then merge them
    cluster_wait();
    started = true;
    if (tid == 0) tc::mbar_arrive_expect_tx(&xbar[0], (uint32_t)(CL * p.lp * 8));
    const int lp_log2 = __ffs(p.lp) - 1;  // lp is a power of two
    for (int t = tid; t < CL * p.lp; t += kThreads) {
      const int peer = t >> lp_log2, pos = t & (p.lp - 1);
      st_async(map_rank(all + rank * p.lp + pos, peer), top[pos], map_rank(&xbar[0], peer));
    }
    tc::mbar_wait(&xbar[0], 0, &xabort, p.budget);
    if (p.lp == 16 && CL >= 2) {
      merge_tree16(all, work, CL, m, nf, order);
      // warp 0 ends the tree holding the final list: when this CTA's first block is a scored
      // one (bf16, nothing staged yet), its TMA starts here, before the block barrier
      early = !kF32 && MODE == MODE_FUSED && rank >= nf && rank - nf < m && issued == 0;
      if (early && warp == 0) {
        __syncwarp();  // (order[] was written by warp 0's lanes)
        if (lane == 0) {
          const int jb = order[rank];
          tc::fence_proxy_async();
          tc::mbar_arrive_expect_tx(&xbar[3], (uint32_t)(2 * kv_tile));
#pragma unroll
          for (int h = 0; h < D / 64; ++h) {
            tc::tma_load_3d(kv + h * 8192, &p.tmk, h * 64, jb * kBlk, (int)unit, &xbar[3]);
            tc::tma_load_3d(kv + kv_tile + h * 8192, &p.tmv, h * 64, jb * kBlk, (int)unit, &xbar[3]);
          }
        }
      }
    } else {
      const u64* fin = p.lp == 16 ? merge_lists<1>(all, work, CL)
                     : (p.lp == 32 ? merge_lists<2>(all, work, CL) : merge_lists<4>(all, work, CL));
      for (int r = tid; r < m; r += kThreads) order[nf + r] = key_block(fin[r]);
    }
  }
  __syncthreads();
  if (early) ++issued;

  // selected indices, ascending (written by rank 0; in fused mode after its attention
  // copies have been started)
  auto write_indices = [&]() {
    if (!(select && rank == 0)) return;
    int32_t* out = p.idx_out ? p.idx_out + unit * p.topk : nullptr;
    if (out) {
      for (int i = tid; i < p.topk; i += kThreads) {
        if (i < n_order) {
          const int v = order[i];
          int pos = 0;
#pragma unroll 8
          for (int u = 0; u < n_order; ++u) pos += order[u] < v;
          out[pos] = v;
        } else {
          out[i] = -1;
        }
      }
    }
    if (MODE == MODE_SELECT && tid == 0) p.nsel_out[unit] = n_order;
  };
  if (MODE == MODE_SELECT) write_indices();
  if (MODE == MODE_SELECT) {
    cp_async_wait<0>();  // no copy into shared memory outlives the CTA
    if (!started) cluster_wait();
    drain_on_abort(scan, false);
    return;  // every byte this CTA receives has landed: no trailing barrier
  }

  // ---- attention over my share of the blocks ------------------------------------------
  const int n_my = n_order > rank ? (n_order - rank + CL - 1) >> (__ffs(CL) - 1) : 0;  // CL: power of two
  while (issued < kStages && issued < n_my) issue_block(order[rank + issued * CL]);
  if (MODE == MODE_FUSED) write_indices();
  if (!scan) {  // the query rows' copy, followed (fp32) by at most kStages block copies
    const int after_q = kF32 ? issued - issued_before_q : 0;
    if (after_q >= 2) cp_async_wait<2>(); else if (after_q == 1) cp_async_wait<1>(); else cp_async_wait<0>();
  }
  __syncthreads();  // (the staged query rows are visible)

  const float scale2 = p.scale * kLog2e;
  float m_run = -INFINITY, l_run = 0.f;  // softmax row state (row = tid >> 4)
  const int srow = tid >> 4, ssub = tid & 15;
  constexpr int NT = kF32 ? 1 : D / 64;  // n8 tiles of the output per warp (bf16)
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
    if constexpr (kF32) {
      if (issued > i + 1) cp_async_wait<1>(); else cp_async_wait<0>();
    } else {
      tc::mbar_wait(&xbar[3 + i % kStages], (uint32_t)((i / kStages) & 1), &xabort, p.budget);
    }
    __syncthreads();
    const int j = order[rank + i * CL];
    const unsigned char* Ks = kv + (size_t)(i % kStages) * 2 * kv_tile;
    const unsigned char* Vs = Ks + kv_tile;
    if constexpr (!kF32) {
      // V rows past the sequence (or all rows of an invalid j) hold whatever the cache
      // holds there: zero them, so that P = 0 never meets a NaN (ordered before P V by the
      // barrier after S)
      const int nv = (j < 0 || j >= NB) ? 0 : min(kBlk, Tb - j * kBlk);
      for (int id = tid; id < (kBlk - nv) * (D / 8); id += kThreads) {
        const int r = nv + id / (D / 8), c = id % (D / 8);
        *reinterpret_cast<uint4*>(const_cast<unsigned char*>(Vs) + kv_off(r, c)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }

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
      const bool valid = j >= 0 && j < NB && j * kBlk + tok < Tb;
#pragma unroll
      for (int r = 0; r < 4; ++r) Ss[(rg * 4 + r) * kSStride + tok] = valid ? s[r] * scale2 : -INFINITY;
    } else {
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < D / 16; ks += 2) {
        uint32_t kb[4];
        ldsm_x4(kb, Ks + kv_off(8 * warp + (lane & 7), 2 * ks + (lane >> 3)));
        mma_bf16(s, qa[ks], kb[0], kb[1]);
        mma_bf16(s, qa[ks + 1], kb[2], kb[3]);
      }
      const int col = 8 * warp + 2 * (lane & 3);
      const int r0 = lane >> 2;
      const bool jin = j >= 0 && j < NB;
      const bool v0 = jin && j * kBlk + col < Tb, v1 = jin && j * kBlk + col + 1 < Tb;
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
          ldsm_x4_t(vb, Vs + kv_off(vrow, 2 * warp + (lane >> 4)));
          mma_bf16(acc[0], pa, vb[0], vb[1]);
          mma_bf16(acc[1], pa, vb[2], vb[3]);
        } else {
          uint32_t vb[2];
          ldsm_x2_t(vb, Vs + kv_off(vrow, warp));
          mma_bf16(acc[0], pa, vb[0], vb[1]);
        }
      }
    }
    // the summary of the sequence's last block, from the keys staged here
    if (p.summ_w != nullptr && j == NB - 1) {
      const int n = Tb - j * kBlk;
      if constexpr (kF32) {
        for (int d = tid; d < D; d += kThreads) {
          float s = 0.f;
#pragma unroll 8
          for (int t = 0; t < n; ++t) s += reinterpret_cast<const float*>(Ks + t * kv_row)[d];
          p.summ_w[(unit * p.NB_cap + j) * D + d] = s / (float)n;
        }
      } else {
        // every thread: one column pair over a slice of the rows, then the slices are
        // added through the score tile (free after the softmax)
        constexpr int kPairs = D / 2, kSlices = kThreads / kPairs, kRowsPer = kBlk / kSlices;
        float* red = Ss;
        const int cp = tid % kPairs, sl = tid / kPairs;
        const int c = (2 * cp) >> 3, wd = (2 * cp) & 7;
        const int t_end = min(n, (sl + 1) * kRowsPer);
        float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
        int t = sl * kRowsPer;
        for (; t + 1 < t_end; t += 2) {
          const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(Ks + kv_off(t, c) + 2 * wd);
          const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162*>(Ks + kv_off(t + 1, c) + 2 * wd);
          a0 += __low2float(x); a1 += __high2float(x);
          b0 += __low2float(y); b1 += __high2float(y);
        }
        if (t < t_end) {
          const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(Ks + kv_off(t, c) + 2 * wd);
          a0 += __low2float(x); a1 += __high2float(x);
        }
        red[sl * D + 2 * cp] = a0 + b0;
        red[sl * D + 2 * cp + 1] = a1 + b1;
        __syncthreads();
        for (int d = tid; d < D; d += kThreads) {
          float s = 0.f;
#pragma unroll
          for (int q = 0; q < kSlices; ++q) s += red[q * D + d];
          p.summ_w[(unit * p.NB_cap + j) * D + d] = s / (float)n;
        }
      }
    }
    if (issued < n_my) {
      __syncthreads();  // the stage may now be refilled
      issue_block(order[rank + issued * CL]);
    }
  }

  cp_async_wait<0>();  // (a CTA with no block may still have its query copy in flight)
  // ---- push the partial (m, l, acc) to the CTAs that merge each output slice -----------
  if (!started) {
    cluster_wait();
    started = true;
  }
  const int E = G * D;
  const int chunk = p.chunk;
  if (tid == 0) {  // from every CTA: kRows (m, l) pairs and this CTA's slice of the accumulator
    const int own = max(0, min(E, (rank + 1) * chunk) - rank * chunk);
    tc::mbar_arrive_expect_tx(&xbar[1], (uint32_t)(CL * (kRows * 8 + own * 4)));
  }
  if (ssub < CL)
    st_async(map_rank(ml_in + rank * kRows + srow, ssub), make_float2(m_run, l_run), map_rank(&xbar[1], ssub));
  if constexpr (kF32) {
    if (srow < G) {
#pragma unroll
      for (int e2 = 0; e2 < D / 16; ++e2) {
        const int e = srow * D + ssub + 16 * e2;
        const int owner = fdiv(e, p.chunk_div);
        st_async(map_rank(pacc_in + rank * chunk + (e - owner * chunk), owner), acc[e2][0],
                 map_rank(&xbar[1], owner));
      }
    }
  } else {
    const int r0 = lane >> 2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int d = (D == 128 ? 16 * warp : 8 * warp) + 8 * nt + 2 * (lane & 3);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int row = r0 + 8 * half;
        if (row < G) {
          const int e = row * D + d;
          const int owner = fdiv(e, p.chunk_div);
          st_async(map_rank(pacc_in + rank * chunk + (e - owner * chunk), owner),
                   make_float2(acc[nt][2 * half], acc[nt][2 * half + 1]), map_rank(&xbar[1], owner));
        }
      }
    }
  }
  tc::mbar_wait(&xbar[1], 0, &xabort, p.budget);

  // ---- log-sum-exp merge of this CTA's slice, from its own shared memory ---------------
  {
    T* og = static_cast<T*>(p.o) + ((size_t)b * p.Hkv * G + (size_t)g * G) * D;
    const int e0 = rank * chunk;
    const int e_end = min(E, e0 + chunk);
    for (int e = e0 + tid; e < e_end; e += kThreads) {
      const int h = e / D, d = e - h * D;
      float2 ml[kMaxCluster];
      float M = -INFINITY;
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) {
        if (r < CL) {
          ml[r] = ml_in[r * kRows + h];
          M = fmaxf(M, ml[r].x);
        }
      }
      float Lsum = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
          if (r < CL) {
            const float w = ex2(ml[r].x - M);
            Lsum = fmaf(ml[r].y, w, Lsum);
            O = fmaf(pacc_in[r * chunk + (e - e0)], w, O);
          }
        }
      }
      og[(size_t)h * D + d] = from_f32<T>(M == -INFINITY ? 0.f : O / Lsum);
      if (d == 0 && p.lse)
        p.lse[(size_t)b * p.Hkv * G + (size_t)g * G + h] =
            M == -INFINITY ? -INFINITY : (M + log2f(Lsum)) * kLn2;
    }
  }
  drain_on_abort(scan, true);
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
  // per template instance and device: the largest dynamic smem size set so far, the
  // (cluster size, smem) pairs found schedulable and the SM count (thread-safe; see
  // launch_cache.h)
  static LaunchRecord rec;
  int dev = 0;
  cudaError_t err = current_device(&dev);
  if (err != cudaSuccess) return err;
  int sms = 0;
  {
    std::lock_guard<std::mutex> lock(rec.mu);
    err = rec.sm_count(dev, &sms);
    if (err != cudaSuccess) return err;
  }
  // cluster size: as many CTAs per unit (2 to 16) as fit in one wave of two CTAs per SM
  // (measured on the batched workload, 128 units: 2 per unit 23.7 us, 4 26.4 us, 8 34.4 us)
  const int units = a.B * a.Hkv;
  int CL = 16;
  while (CL > 2 && (long long)units * CL > 2LL * sms) CL >>= 1;
  Params p{};
  if (sizeof(T) == 2 && MODE != MODE_SELECT &&
      !kv_tensor_maps(a.k, a.v, a.D, a.T_cap, a.B * a.Hkv, &p.tmk, &p.tmv))
    return cudaErrorInvalidValue;
  p.q = a.q; p.k = a.k; p.v = a.v;
  p.Hkv = a.Hkv; p.G = a.G; p.T_cap = a.T_cap; p.NB_cap = a.NB_cap;
  p.seqlens = a.seqlens; p.summ = a.summ; p.summ_w = a.summ_w;
  p.idx_in = a.idx_in; p.nsel_in = a.nsel_in;
  p.topk = a.topk; p.n_sink = a.n_sink; p.n_local = a.n_local; p.scale = a.scale;
  p.idx_out = a.idx_out; p.nsel_out = a.nsel_out; p.scores_out = a.scores_out;
  p.o = a.o; p.lse = a.lse;
  p.m_pad = next_pow2(a.topk < 2 ? 2 : a.topk);
  p.lp = p.m_pad < 16 ? 16 : p.m_pad;
  for (;;) {
    p.per_max = (a.NB_cap + CL - 1) / CL;
    const int E = a.G * D;
    p.chunk = ((E + CL - 1) / CL + 1) & ~1;
    p.chunk_div = make_fastdiv((uint32_t)p.chunk);
    const Layout Lo = make_layout((int)sizeof(T), D, p.per_max, p.m_pad);
    const int smem = (int)Lo.total;
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
    cfg.numAttrs = (MODE == MODE_FUSED && a.pdl) ? 2 : 1;
    p.pdl = cfg.numAttrs == 2;
    p.budget = wait_budget();
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

cudaError_t read_decode_status(int* status, bool reset) {
  cudaError_t err = cudaMemcpyFromSymbol(status, g_decode_status, sizeof(int));
  if (err == cudaSuccess && reset) {
    const int zero = 0;
    err = cudaMemcpyToSymbol(g_decode_status, &zero, sizeof(int));
  }
  return err;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.B == 0 || a.Hkv == 0) return cudaSuccess;
  if (a.dtype == DT_BF16) {
    if (a.D == 128) return launch_mode<__nv_bfloat16, 128>(a, stream);
    return launch_mode<__nv_bfloat16, 64>(a, stream);
  }
  if (a.D == 128) return launch_mode<float, 128>(a, stream);
  return launch_mode<float, 64>(a, stream);
}

LSA_BOUNDS_READER(decode)

}  // namespace lsa
