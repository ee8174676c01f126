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
// r (topk <= 16).  Thread 0 reads the slot's block index and starts the K block as TMA
// boxes (128-byte swizzle) on one mbarrier; q arrives by cp.async meanwhile.  S = Q K^T
// runs on mma.sync m16n8k16 (the G <= 16 query heads are the 16 rows), the block maxima are
// reduced across the warps, and each CTA stores its G maxima into every peer's shared
// memory with st.async, completed on the receiver's mbarrier (no cluster barrier).  Every
// CTA then evaluates the test for every slot (the maximum over the earlier slots is the
// running maximum, so the sequential rule is decided in parallel); a kept block's CTA
// starts its V block by TMA (second mbarrier), forms P = 2^(S - r) in bf16 and computes
// P V on mma.sync.  Each CTA pushes its partial (m, l) and the slices of its accumulator
// to the CTAs that own those output elements (st.async, third mbarrier), and every CTA
// merges its 1/16 of the outputs by log-sum-exp from its own shared memory.  Every byte a
// CTA receives is counted by its own mbarriers and waited for before it ends, so no CTA
// leaves while a peer may still write into it.  Waits are bounded (about 2 s of clock); if
// one runs out the launch's outputs are undefined, the CTA waits (bounded) for what is still
// in flight before it exits, and a status word records the failure.
// With many (b, g) units (64 and up) one CTA per unit does the same in phases instead
// (decode_blasst_unit_kernel below): every block's S, every slot's test at once, then the
// kept blocks' V and P V spread over its warps.
#include <math.h>

#include "cluster.cuh"
#include "launch_cache.h"
#include "lsa_common.cuh"
#include "lsa_internal.h"
#include "tcgen05.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCL = 16;      // CTAs per cluster = maximum selection slots
constexpr int kRows = 16;    // query-head rows (G <= 16): the mma M dimension

// Set when a bounded wait runs out (the outputs of that launch are then undefined); read
// and cleared by the host.
__device__ int g_blasst_decode_status = 0;

struct Params {
  CUtensorMap tmk;  // bf16 K and V as [B * Hkv][T_cap][D], box {64, 64, 1}, 128-byte swizzle
  CUtensorMap tmv;
  const __nv_bfloat16* q;
  int Hkv, G, T_cap;
  const int32_t* seqlens;
  const int32_t* idx;
  const int32_t* nsel;
  int topk;
  float scale2;       // softmax scale times log2(e)
  float log2_lambda;  // log2(lambda), -inf for lambda = 0
  __nv_bfloat16* o;
  float* lse;
  uint32_t* skip_bits;
  long long budget;  // clock-cycle limit of every bounded wait
};

// Shared-memory carve-up (byte offsets from the first 1024-byte boundary of the dynamic buffer).
template <int D>
struct Lay {
  static constexpr int kTile = kBlk * D * 2;            // one K or V block (bf16)
  static constexpr int kK = 0;                          // TMA boxes: 1024-byte aligned
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;                 // [16][D] bf16, chunk-swizzled
  static constexpr int kP = kQ + kRows * D * 2;         // [16][64] bf16, chunk-swizzled
  static constexpr int kRed = kP + kRows * kBlk * 2;    // [8 warps][16] float
  static constexpr int kRmax = kRed + kWarps * kRows * 4;        // [16 slots][16 heads] float
  static constexpr int kMl = kRmax + kCL * kRows * 4;            // [16 CTAs][16 heads] float2
  static constexpr int kAcc = kMl + kCL * kRows * 8;             // [16 CTAs][16 D / 16] float
  static constexpr int kTotal = kAcc + kCL * (kRows * D / kCL) * 4;
};

template <int D>
__global__ void __launch_bounds__(kThreads) decode_blasst_kernel(const __grid_constant__ Params p) {
  using L = Lay<D>;
  constexpr int kRowBytes = D * 2;
  constexpr int NT = D / 64;  // n8 tiles of the output per warp
  extern __shared__ __align__(1024) unsigned char smem[];
  // mbarriers: [0] the K block, [1] the V block, [2] the block maxima of every slot, [3] the
  // partials of every CTA (one phase each)
  __shared__ __align__(8) uint64_t bar[4];
  __shared__ int slot_block[kCL];
  __shared__ uint32_t valid_bits, skip_word;
  __shared__ float rloc[kRows], lloc[kRows];
  __shared__ int xabort;
  // the K/V boxes land 1024-byte aligned (128-byte swizzle): the layout starts at the first
  // 1024-byte boundary of the dynamic buffer (1 KB of slack is allocated for it)
  unsigned char* base = smem + ((1024u - (tc::smem_u32(smem) & 1023u)) & 1023u);
  unsigned char* Ks = base + L::kK;
  unsigned char* Vs = base + L::kV;
  unsigned char* Qs = base + L::kQ;
  unsigned char* Ps = base + L::kP;
  float* red = reinterpret_cast<float*>(base + L::kRed);
  float* rmax = reinterpret_cast<float*>(base + L::kRmax);
  float2* ml_in = reinterpret_cast<float2*>(base + L::kMl);
  float* acc_in = reinterpret_cast<float*>(base + L::kAcc);

  const int rank = cluster_rank();
  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  const int Hq = p.Hkv * G;
  const int unit = b * p.Hkv + g;
  const int per = G * D / kCL;  // output elements merged by one CTA (G * D is a multiple of 16)

  // the slot's block and the sequence length first (the K copy waits only for them)
  const int T = checked_range(__ldg(p.seqlens + b), 0, p.T_cap, kBoundsSeqlen, kSiteDecodeBlasst);
  const int NBq = (T + kBlk - 1) / kBlk;
  const int ns = checked_range(__ldg(p.nsel + unit), 0, p.topk, kBoundsCount, kSiteDecodeBlasst);
  const int jj = rank < p.topk ? checked_range(__ldg(p.idx + unit * p.topk + rank), -1, NBq - 1, kBoundsIndex, kSiteDecodeBlasst) : -1;
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) tc::mbar_init(&bar[i], 1);
    xabort = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&p.tmk);
    tc::prefetch_tmap(&p.tmv);
    const bool has0 = rank < ns && jj >= 0;
    if (has0 && jj * kBlk < T) {
      tc::mbar_arrive_expect_tx(&bar[0], (uint32_t)L::kTile);
#pragma unroll
      for (int h = 0; h < D / 64; ++h) tc::tma_load_3d(Ks + h * 8192, &p.tmk, h * 64, jj * kBlk, unit, &bar[0]);
    }
  }
  cluster_arrive_relaxed();  // DSMEM is written only after every CTA has started
  // the query rows (rows >= G zero) by 16-byte cp.async
  {
    const __nv_bfloat16* qg = p.q + ((size_t)b * Hq + (size_t)g * G) * D;
    constexpr int kQChunks = kRows * kRowBytes / 16;
    for (int id = tid; id < kQChunks; id += kThreads) {
      const int row = id / (kRowBytes / 16), c = id % (kRowBytes / 16);
      cp_async16(Qs + swz(row, c, kRowBytes), qg + (size_t)(row < G ? row : 0) * D + c * 8, row < G);
    }
    cp_async_commit();
  }
  // which slots hold a block (the same on every CTA)
  if (warp == 0) {
    const int j2 = lane < p.topk && lane < kCL
        ? checked_range(__ldg(p.idx + unit * p.topk + lane), -1, NBq - 1, kBoundsIndex, kSiteDecodeBlasst) : -1;
    const bool on = lane < ns && lane < kCL && j2 >= 0;
    const uint32_t bits = __ballot_sync(0xffffffffu, on);
    if (lane < kCL) slot_block[lane] = on ? j2 : -1;
    if (lane == 0) valid_bits = bits;
  }
  cp_async_wait<0>();
  __syncthreads();
  const uint32_t valid = valid_bits;
  const int nvalid = __popc(valid);
  const bool has = (valid >> rank) & 1u;
  const int j = has ? slot_block[rank] : 0;
  const int nv = has ? max(0, min(kBlk, T - j * kBlk)) : 0;  // valid rows of the block
  const bool loaded = nv > 0;

  // ---- S = Q K^T (base-2 logits), the block maxima --------------------------------------
  float s[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  uint32_t qa[D / 16][4];
  const int r0 = lane >> 2;
  const int col = 8 * warp + 2 * (lane & 3);
  if (loaded) {
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
      ldsm_x4(qa[ks], Qs + swz(row, 2 * ks + (lane >> 4), kRowBytes));
    }
    tc::mbar_wait(&bar[0], 0, &xabort, p.budget);
    float c4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < D / 16; ks += 2) {
      uint32_t kb[4];
      ldsm_x4(kb, Ks + kv_off(8 * warp + (lane & 7), 2 * ks + (lane >> 3)));
      mma_bf16(c4, qa[ks], kb[0], kb[1]);
      mma_bf16(c4, qa[ks + 1], kb[2], kb[3]);
    }
    const bool v0 = col < nv, v1 = col + 1 < nv;
    s[0] = v0 && r0 < G ? c4[0] * p.scale2 : -INFINITY;
    s[1] = v1 && r0 < G ? c4[1] * p.scale2 : -INFINITY;
    s[2] = v0 && r0 + 8 < G ? c4[2] * p.scale2 : -INFINITY;
    s[3] = v1 && r0 + 8 < G ? c4[3] * p.scale2 : -INFINITY;
  }
  {
    float m_lo = fmaxf(s[0], s[1]), m_hi = fmaxf(s[2], s[3]);
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      m_lo = fmaxf(m_lo, __shfl_xor_sync(0xffffffffu, m_lo, o2));
      m_hi = fmaxf(m_hi, __shfl_xor_sync(0xffffffffu, m_hi, o2));
    }
    if ((lane & 3) == 0) {
      red[warp * kRows + r0] = m_lo;
      red[warp * kRows + r0 + 8] = m_hi;
    }
  }
  __syncthreads();
  if (tid < kRows) {
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, red[w * kRows + tid]);
    rloc[tid] = mx;
  }
  cluster_wait();  // (matches the arrive at the start) every CTA runs: DSMEM is live
  if (tid == 0) tc::mbar_arrive_expect_tx(&bar[2], (uint32_t)(nvalid * G * 4));
  __syncthreads();  // (rloc is complete)
  // this slot's maxima into every CTA's table, row `rank`
  if (has && tid < kCL * G) {
    const int peer = tid / G, h = tid - peer * G;
    st_async(map_rank(rmax + rank * kRows + h, peer), rloc[h], map_rank(&bar[2], peer));
  }
  if (nvalid > 0) tc::mbar_wait(&bar[2], 0, &xabort, p.budget);

  // ---- the test for every slot (each CTA decides all of them; it acts on its own) ----------
  // Warp 0, lane s = slot s: per head, the running maximum before slot s is an exclusive
  // prefix maximum over the lanes (slots without a block contribute -inf); the slot's gap is
  // the maximum over the heads of (r_h - m_h).  The first slot holding a block is never
  // skipped.  The decision reaches the other warps through shared memory.
  if (warp == 0) {
    const bool vs = lane < kCL && ((valid >> lane) & 1u);
    float gap = -INFINITY;
#pragma unroll
    for (int h = 0; h < kRows; ++h) {
      if (h < G) {
        const float r = vs ? rmax[lane * kRows + h] : -INFINITY;
        float m = r;  // inclusive prefix maximum over lanes 0 .. lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float t = __shfl_up_sync(0xffffffffu, m, o);
          if (lane >= o) m = fmaxf(m, t);
        }
        float before = __shfl_up_sync(0xffffffffu, m, 1);
        if (lane == 0) before = -INFINITY;
        const float gi = r == -INFINITY ? -INFINITY : (before == -INFINITY ? INFINITY : r - before);
        gap = fmaxf(gap, gi);
      }
    }
    const int first = valid ? __ffs(valid) - 1 : -1;
    const uint32_t bits = __ballot_sync(0xffffffffu, vs && lane != first && gap < p.log2_lambda);
    if (lane == 0) skip_word = bits;
  }
  __syncthreads();
  const uint32_t skipped = skip_word;
  const bool keep = loaded && !((skipped >> rank) & 1u);
  if (keep && tid == 0) {
    tc::mbar_arrive_expect_tx(&bar[1], (uint32_t)L::kTile);
#pragma unroll
    for (int h = 0; h < D / 64; ++h) tc::tma_load_3d(Vs + h * 8192, &p.tmv, h * 64, j * kBlk, unit, &bar[1]);
  }

  // ---- P = 2^(S - r) (bf16, into shared memory), the row sums, O = P V ---------------------
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  if (keep) {  // (uniform)
    const float rl = rloc[r0], rh = rloc[r0 + 8];
    const float p0 = s[0] == -INFINITY ? 0.f : ex2(s[0] - rl);
    const float p1 = s[1] == -INFINITY ? 0.f : ex2(s[1] - rl);
    const float p2 = s[2] == -INFINITY ? 0.f : ex2(s[2] - rh);
    const float p3 = s[3] == -INFINITY ? 0.f : ex2(s[3] - rh);
    *reinterpret_cast<uint32_t*>(Ps + swz(r0, col >> 3, kBlk * 2) + (col & 7) * 2) = pack_bf16x2(p0, p1);
    *reinterpret_cast<uint32_t*>(Ps + swz(r0 + 8, col >> 3, kBlk * 2) + (col & 7) * 2) = pack_bf16x2(p2, p3);
    float l_lo = p0 + p1, l_hi = p2 + p3;
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      l_lo += __shfl_xor_sync(0xffffffffu, l_lo, o2);
      l_hi += __shfl_xor_sync(0xffffffffu, l_hi, o2);
    }
    // (red held the maxima, all read before the barrier after the rloc reduction)
    if ((lane & 3) == 0) {
      red[warp * kRows + r0] = l_lo;
      red[warp * kRows + r0 + 8] = l_hi;
    }
    // V rows past the sequence hold whatever the cache holds there: zero them once they
    // have landed, so that P = 0 never meets a NaN
    tc::mbar_wait(&bar[1], 0, &xabort, p.budget);
    for (int id = tid; id < (kBlk - nv) * (D / 8); id += kThreads) {
      const int r = nv + id / (D / 8), c = id % (D / 8);
      *reinterpret_cast<uint4*>(Vs + kv_off(r, c)) = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    if (tid < kRows) {
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) l += red[w * kRows + tid];
      lloc[tid] = l;
    }
    // warp w takes output columns [w * D / 8, (w + 1) * D / 8)
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
  __syncthreads();  // (lloc is complete)

  // ---- partials to the CTAs that own each output slice -------------------------------------
  if (tid == 0) tc::mbar_arrive_expect_tx(&bar[3], (uint32_t)(kCL * (G * 8 + per * 4)));
  if (tid < kCL * G) {  // (m, l) of every head into every CTA, row `rank`
    const int peer = tid / G, h = tid - peer * G;
    const float2 ml = keep ? make_float2(rloc[h], lloc[h]) : make_float2(-INFINITY, 0.f);
    st_async(map_rank(ml_in + rank * kRows + h, peer), ml, map_rank(&bar[3], peer));
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int d = (D == 128 ? 16 * warp : 8 * warp) + 8 * nt + 2 * (lane & 3);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = r0 + 8 * half;
      if (row < G) {
        const int e = row * D + d;
        const int owner = e / per;  // (per is even, so both elements share the owner)
        st_async(map_rank(acc_in + rank * per + (e - owner * per), owner),
                 make_float2(acc[nt][2 * half], acc[nt][2 * half + 1]), map_rank(&bar[3], owner));
      }
    }
  }
  tc::mbar_wait(&bar[3], 0, &xabort, p.budget);

  // ---- merge this CTA's slice by log-sum-exp ------------------------------------------------
  for (int le = tid; le < per; le += kThreads) {
    const int e = rank * per + le;
    const int h = e / D, d = e - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kCL; ++c) M = fmaxf(M, ml_in[c * kRows + h].x);
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int c = 0; c < kCL; ++c) {
        const float2 ml = ml_in[c * kRows + h];
        const float w = ml.x == -INFINITY ? 0.f : ex2(ml.x - M);
        Lsum = fmaf(ml.y, w, Lsum);
        O = fmaf(acc_in[c * per + le], w, O);
      }
    }
    const size_t row = (size_t)b * Hq + (size_t)g * G + h;
    p.o[row * D + d] = __float2bfloat16_rn(Lsum > 0.f ? O / Lsum : 0.f);
    if (d == 0 && p.lse) p.lse[row] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
  }
  if (rank == 0 && tid == 0 && p.skip_bits) p.skip_bits[unit] = skipped;
  // after a timeout (the outputs are then undefined) the CTA must not exit while its own
  // copies, or bytes its peers owe it, are in flight: wait for each (bounded, ignoring the
  // abort) and record the failure
  if (*reinterpret_cast<volatile int*>(&xabort)) {
    if (loaded) tc::mbar_drain(&bar[0], 0, kDrainBudget);
    if (keep) tc::mbar_drain(&bar[1], 0, kDrainBudget);
    if (nvalid > 0) tc::mbar_drain(&bar[2], 0, kDrainBudget);
    tc::mbar_drain(&bar[3], 0, kDrainBudget);
    g_blasst_decode_status = 1;
  }
}

// ---- many (b, g) units: one CTA per unit, the test taken in two halves --------------------
// The sequential rule needs, for each selected block, only the maximum of the earlier
// blocks' maxima (a skipped block never raises it), so nothing has to run block by block,
// and the first eight slots can be decided before the last eight are scored:
//   1. warp w computes S of slot w on its own TMA stage, keeps the logits in registers and
//      posts the block's per-head maxima, then requests slot w + 8's K into the same stage;
//   2. slots 0..7 are tested (a thread per (slot, head): the exclusive prefix maximum over
//      the earlier slots, then the maximum over the heads) and the V of up to four kept
//      ones starts at once into four extra stages, while warp w computes S of slot w + 8;
//   3. slots 8..15 are tested; each warp then loads the V of its kept slots that have no
//      stage yet into its own stage (free again) and folds its kept slots into an online
//      softmax of its own, P built from the logits in registers straight into the mma A
//      operand;
//   4. the eight warps' (m, l, O) merged by log-sum-exp.
// One CTA per unit (128 CTAs for 16 sequences x 8 KV heads: one wave, one per SM), no
// cluster, no cross-CTA exchange.
template <int D>
struct UnitLay {
  static constexpr int kTile = kBlk * D * 2;                 // one K or V block (bf16)
  static constexpr int kXS = 4;                              // extra V stages
  static constexpr int kRing = 0;                            // kWarps stages, 1024-byte aligned
  static constexpr int kX = kRing + kWarps * kTile;          // kXS extra V stages
  static constexpr int kQ = kX + kXS * kTile;                // [16][D] bf16, chunk-swizzled
  static constexpr int kRmax = kQ + kRows * D * 2;           // [16 slots][16 heads] fp32
  static constexpr int kTotal = kRmax + kCL * kRows * 4;
  static_assert(kWarps * kRows * D * 4 <= kWarps * kTile, "the warps' partials fit the ring");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) decode_blasst_unit_kernel(const __grid_constant__ Params p) {
  using L = UnitLay<D>;
  constexpr int kRowBytes = D * 2;
  constexpr int NO = D / 8;  // n8 tiles of a warp's output (all D columns)
  constexpr int NS = kBlk / 8;  // n8 tiles of a block's logits
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t kbar[kWarps], vbar[kWarps], xbar[L::kXS];
  __shared__ int slot_block[kCL], slot_id[kCL], nslots;
  __shared__ int skipf[kCL], xstage[kCL];
  __shared__ float2 ml_w[kWarps][kRows];
  __shared__ int xabort;
  unsigned char* base = smem + ((1024u - (tc::smem_u32(smem) & 1023u)) & 1023u);
  unsigned char* ring = base + L::kRing;
  unsigned char* xring = base + L::kX;
  unsigned char* Qs = base + L::kQ;
  float* rmax = reinterpret_cast<float*>(base + L::kRmax);

  const int g = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  const int Hq = p.Hkv * G;
  const int unit = b * p.Hkv + g;
  const int T = checked_range(__ldg(p.seqlens + b), 0, p.T_cap, kBoundsSeqlen, kSiteDecodeBlasst);
  const int NBq = (T + kBlk - 1) / kBlk;
  if (tid == 0) {
    for (int i = 0; i < kWarps; ++i) {
      tc::mbar_init(&kbar[i], 1);
      tc::mbar_init(&vbar[i], 1);
    }
    for (int i = 0; i < L::kXS; ++i) tc::mbar_init(&xbar[i], 1);
    xabort = 0;
    tc::fence_mbar_init();
    tc::prefetch_tmap(&p.tmk);
    tc::prefetch_tmap(&p.tmv);
  }
  // the slots holding a block, compacted in ascending slot order
  if (warp == 0) {
    const int ns = checked_range(__ldg(p.nsel + unit), 0, p.topk, kBoundsCount, kSiteDecodeBlasst);
    const int j2 = lane < p.topk && lane < kCL
        ? checked_range(__ldg(p.idx + unit * p.topk + lane), -1, NBq - 1, kBoundsIndex, kSiteDecodeBlasst) : -1;
    const bool on = lane < ns && lane < kCL && j2 >= 0;
    const uint32_t bits = __ballot_sync(0xffffffffu, on);
    const int pos = __popc(bits & ((1u << lane) - 1u));
    if (on) {
      slot_block[pos] = j2;
      slot_id[pos] = lane;
    }
    if (lane == 0) nslots = __popc(bits);
    if (lane < kCL) {
      skipf[lane] = 0;
      xstage[lane] = -1;
    }
  }
  {
    const __nv_bfloat16* qg = p.q + ((size_t)b * Hq + (size_t)g * G) * D;
    constexpr int kQChunks = kRows * kRowBytes / 16;
    for (int id = tid; id < kQChunks; id += kThreads) {
      const int row = id / (kRowBytes / 16), c = id % (kRowBytes / 16);
      cp_async16(Qs + swz(row, c, kRowBytes), qg + (size_t)(row < G ? row : 0) * D + c * 8, row < G);
    }
    cp_async_commit();
  }
  __syncthreads();  // (the slot list and the barriers are set up)
  const int n = nslots;
  unsigned char* stage = ring + warp * L::kTile;  // this warp's TMA stage
  // lane 0 of the warp: block j of `map` into `dst`, completing on `bar`
  auto load_block = [&](const CUtensorMap* map, int j, unsigned char* dst, uint64_t* bar) {
    tc::fence_proxy_async();  // this warp's earlier reads of the stage come first
    tc::mbar_arrive_expect_tx(bar, (uint32_t)L::kTile);
#pragma unroll
    for (int h = 0; h < D / 64; ++h) tc::tma_load_3d(dst + h * 8192, map, h * 64, j * kBlk, unit, bar);
  };
  auto prefetch_block = [&](const CUtensorMap* map, int j) {
#pragma unroll
    for (int h = 0; h < D / 64; ++h) tc::tma_prefetch_l2_3d(map, h * 64, j * kBlk, unit);
  };
  // loads issued on this warp's barriers and seen complete: a load into a stage is issued
  // only after the previous one on the same barrier was seen complete, so at most one is in
  // flight per barrier
  int k_issued = 0, k_seen = 0, v_issued = 0, v_seen = 0, x_issued = 0, x_seen = 0, my_x = -1;
  if (lane == 0 && warp < n) {
    load_block(&p.tmk, slot_block[warp], stage, &kbar[warp]);
    k_issued = 1;
    // the second slot's K waits for this stage: bring it into L2 meanwhile
    if (warp + kWarps < n) prefetch_block(&p.tmk, slot_block[warp + kWarps]);
  }
  cp_async_wait<0>();
  __syncthreads();  // (q)
  uint32_t qa[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
    ldsm_x4(qa[ks], Qs + swz(row, 2 * ks + (lane >> 4), kRowBytes));
  }
  const int r0 = lane >> 2, q2 = 2 * (lane & 3);

  // logits of slot i (base 2, -inf where masked) from the stage into registers, and the
  // block's per-head maxima into rmax[i][*]
  auto logits = [&](int i, bool ok, float (&S)[NS][4]) {
    const int nv = max(0, min(kBlk, T - slot_block[i] * kBlk));
    float mlo = -INFINITY, mhi = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NS; ++nt) {
      float c4[4] = {0.f, 0.f, 0.f, 0.f};
      if (ok) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ks += 2) {
          uint32_t kb[4];
          ldsm_x4(kb, stage + kv_off(8 * nt + (lane & 7), 2 * ks + (lane >> 3)));
          mma_bf16(c4, qa[ks], kb[0], kb[1]);
          mma_bf16(c4, qa[ks + 1], kb[2], kb[3]);
        }
      }
      const int col = 8 * nt + q2;
      const bool v0 = col < nv, v1 = col + 1 < nv;
      S[nt][0] = v0 && r0 < G ? c4[0] * p.scale2 : -INFINITY;
      S[nt][1] = v1 && r0 < G ? c4[1] * p.scale2 : -INFINITY;
      S[nt][2] = v0 && r0 + 8 < G ? c4[2] * p.scale2 : -INFINITY;
      S[nt][3] = v1 && r0 + 8 < G ? c4[3] * p.scale2 : -INFINITY;
      mlo = fmaxf(mlo, fmaxf(S[nt][0], S[nt][1]));
      mhi = fmaxf(mhi, fmaxf(S[nt][2], S[nt][3]));
    }
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, o2));
      mhi = fmaxf(mhi, __shfl_xor_sync(0xffffffffu, mhi, o2));
    }
    if ((lane & 3) == 0) {
      rmax[i * kRows + r0] = mlo;
      rmax[i * kRows + r0 + 8] = mhi;
    }
  };
  // the test of slots [lo, hi): a thread per (slot, head); skipf[slot] = skipped
  auto test_slots = [&](int lo, int hi) {
    const int sl = tid >> 4, h = tid & 15;  // (kThreads = 16 slots x 16 heads)
    float gi = -INFINITY;
    if (sl >= lo && sl < hi && sl < n && h < G) {
      const float r = rmax[sl * kRows + h];
      float m = -INFINITY;  // the maximum over the earlier slots = the running maximum
      for (int e = 0; e < sl; ++e) m = fmaxf(m, rmax[e * kRows + h]);
      gi = r == -INFINITY ? -INFINITY : (m == -INFINITY ? INFINITY : r - m);
    }
#pragma unroll
    for (int o2 = 8; o2 > 0; o2 >>= 1) gi = fmaxf(gi, __shfl_xor_sync(0xffffffffu, gi, o2));
    if (h == 0 && sl >= lo && sl < hi) skipf[sl] = sl > 0 && sl < n && gi < p.log2_lambda;
  };

  // ---- 1. slot w's logits; slot w + 8's K requested into the same stage ----------------------
  float S0[NS][4], S1[NS][4];
  bool ok0 = false, ok1 = false;
  if (warp < n) {
    ok0 = __all_sync(0xffffffffu, tc::mbar_wait(&kbar[warp], 0, &xabort, p.budget));
    k_seen += ok0 ? 1 : 0;
    logits(warp, ok0, S0);
    __syncwarp();  // (every lane has read the stage)
    if (ok0 && lane == 0 && warp + kWarps < n) {
      load_block(&p.tmk, slot_block[warp + kWarps], stage, &kbar[warp]);
      k_issued = 2;
    }
  }
  __syncthreads();
  // ---- 2. slots 0..7 decided; up to kXS of the kept ones get an extra stage, V at once -------
  test_slots(0, kWarps);
  __syncthreads();
  if (warp == 0) {
    const bool keep = lane < kWarps && lane < n && !skipf[lane];
    const uint32_t kb2 = __ballot_sync(0xffffffffu, keep);
    const int rank = __popc(kb2 & ((1u << lane) - 1u));
    if (keep && rank < L::kXS) xstage[lane] = rank;
  }
  __syncthreads();
  if (warp < n && !skipf[warp] && xstage[warp] >= 0) {
    my_x = xstage[warp];
    if (lane == 0 && *reinterpret_cast<volatile int*>(&xabort) == 0) {
      load_block(&p.tmv, slot_block[warp], xring + my_x * L::kTile, &xbar[my_x]);
      x_issued = 1;
    }
  }
  if (warp + kWarps < n) {
    ok1 = __all_sync(0xffffffffu, tc::mbar_wait(&kbar[warp], 1, &xabort, p.budget));
    k_seen += ok1 ? 1 : 0;
    logits(warp + kWarps, ok1, S1);
  }
  __syncthreads();
  // ---- 3. slots 8..15 decided; each warp folds in its kept slots ---------------------------
  test_slots(kWarps, kCL);
  __syncthreads();
  if (warp == 0) {  // the skip bits by selection slot
    const uint32_t sb = __ballot_sync(0xffffffffu, lane < n && skipf[lane & (kCL - 1)]);
    uint32_t bits = 0u;
    for (int e = 0; e < kCL; ++e)
      if ((sb >> e) & 1u) bits |= 1u << slot_id[e];
    if (lane == 0 && p.skip_bits) p.skip_bits[unit] = bits;
  }
  const bool keep0 = warp < n && !skipf[warp];
  const bool keep1 = warp + kWarps < n && !skipf[warp + kWarps];
  float acc[NO][4];
#pragma unroll
  for (int nt = 0; nt < NO; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  // one kept slot folded in: O = alpha O + P V, P from the logits S, V at `vs`
  auto fold = [&](int i, const float (&S)[NS][4], const unsigned char* vs, bool ok) {
    const int nv = max(0, min(kBlk, T - slot_block[i] * kBlk));
    // V rows past the sequence hold whatever the cache holds there: zero them (P is 0 there)
    for (int id = lane; id < (kBlk - nv) * (D / 8); id += 32) {
      const int r = nv + id / (D / 8), c = id % (D / 8);
      *reinterpret_cast<uint4*>(const_cast<unsigned char*>(vs) + kv_off(r, c)) = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncwarp();
    const float rlo = rmax[i * kRows + r0], rhi = rmax[i * kRows + r0 + 8];
    const float nlo = fmaxf(m_lo, rlo), nhi = fmaxf(m_hi, rhi);
    const float alo = m_lo == -INFINITY ? 0.f : ex2(m_lo - nlo);
    const float ahi = m_hi == -INFINITY ? 0.f : ex2(m_hi - nhi);
    m_lo = nlo;
    m_hi = nhi;
#pragma unroll
    for (int nt = 0; nt < NO; ++nt) {
      acc[nt][0] *= alo; acc[nt][1] *= alo;
      acc[nt][2] *= ahi; acc[nt][3] *= ahi;
    }
    float slo = 0.f, shi = 0.f;
#pragma unroll
    for (int kk = 0; kk < kBlk / 16; ++kk) {
      uint32_t pa[4];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float* x = S[2 * kk + hf];
        const float p0 = x[0] == -INFINITY ? 0.f : ex2(x[0] - nlo);
        const float p1 = x[1] == -INFINITY ? 0.f : ex2(x[1] - nlo);
        const float p2 = x[2] == -INFINITY ? 0.f : ex2(x[2] - nhi);
        const float p3 = x[3] == -INFINITY ? 0.f : ex2(x[3] - nhi);
        slo += p0 + p1;
        shi += p2 + p3;
        pa[2 * hf] = pack_bf16x2(p0, p1);
        pa[2 * hf + 1] = pack_bf16x2(p2, p3);
      }
      if (ok) {
        const int vrow = 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int np = 0; np < D / 16; ++np) {
          uint32_t vb[4];
          ldsm_x4_t(vb, vs + kv_off(vrow, 2 * np + (lane >> 4)));
          mma_bf16(acc[2 * np], pa, vb[0], vb[1]);
          mma_bf16(acc[2 * np + 1], pa, vb[2], vb[3]);
        }
      }
    }
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      slo += __shfl_xor_sync(0xffffffffu, slo, o2);
      shi += __shfl_xor_sync(0xffffffffu, shi, o2);
    }
    l_lo = l_lo * alo + slo;
    l_hi = l_hi * ahi + shi;
  };
  // the stage's V loads: slot w's when it has no extra stage, then slot w + 8's
  const bool w_in_stage = keep0 && my_x < 0;
  if (lane == 0 && *reinterpret_cast<volatile int*>(&xabort) == 0) {
    if (w_in_stage) {
      load_block(&p.tmv, slot_block[warp], stage, &vbar[warp]);
      v_issued = 1;
    } else if (keep1) {
      load_block(&p.tmv, slot_block[warp + kWarps], stage, &vbar[warp]);
      v_issued = 1;
    }
  }
  v_issued = __shfl_sync(0xffffffffu, v_issued, 0);
  if (keep0) {
    bool ok;
    const unsigned char* vs;
    if (my_x >= 0) {
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&xbar[my_x], 0, &xabort, p.budget));
      x_seen += ok ? 1 : 0;
      vs = xring + my_x * L::kTile;
    } else {
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&vbar[warp], 0, &xabort, p.budget));
      v_seen += ok ? 1 : 0;
      vs = stage;
    }
    fold(warp, S0, vs, ok && ok0);
  }
  if (keep1) {
    if (w_in_stage) {  // the stage held slot w's V: slot w + 8's now
      __syncwarp();  // (every lane has read the stage)
      if (lane == 0 && v_seen == 1 && *reinterpret_cast<volatile int*>(&xabort) == 0) {
        load_block(&p.tmv, slot_block[warp + kWarps], stage, &vbar[warp]);
        v_issued = 2;
      }
      v_issued = __shfl_sync(0xffffffffu, v_issued, 0);
    }
    const int ph = v_issued - 1;
    bool ok = ph >= 0 && __all_sync(0xffffffffu, tc::mbar_wait(&vbar[warp], (uint32_t)(ph & 1), &xabort, p.budget));
    v_seen += ok ? 1 : 0;
    fold(warp + kWarps, S1, stage, ok && ok1);
  }
  __syncthreads();  // (every stage has been read: the ring holds the partials now)

  // ---- 4. the warps' partials, merged by log-sum-exp ---------------------------------------
  float* part = reinterpret_cast<float*>(ring);  // [warp][16 rows][D]
#pragma unroll
  for (int nt = 0; nt < NO; ++nt) {
    const int d = 8 * nt + q2;
    *reinterpret_cast<float2*>(part + (warp * kRows + r0) * D + d) = make_float2(acc[nt][0], acc[nt][1]);
    *reinterpret_cast<float2*>(part + (warp * kRows + r0 + 8) * D + d) = make_float2(acc[nt][2], acc[nt][3]);
  }
  if ((lane & 3) == 0) {
    ml_w[warp][r0] = make_float2(m_lo, l_lo);
    ml_w[warp][r0 + 8] = make_float2(m_hi, l_hi);
  }
  __syncthreads();
  const size_t orow = (size_t)b * Hq + (size_t)g * G;
  for (int e = tid; e < G * D; e += kThreads) {
    const int h = e / D, d = e - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, ml_w[w][h].x);
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float2 ml = ml_w[w][h];
        const float wt = ml.x == -INFINITY ? 0.f : ex2(ml.x - M);
        Lsum = fmaf(ml.y, wt, Lsum);
        O = fmaf(part[(w * kRows + h) * D + d], wt, O);
      }
    }
    p.o[(orow + h) * D + d] = __float2bfloat16_rn(Lsum > 0.f ? O / Lsum : 0.f);
    if (d == 0 && p.lse) p.lse[orow + h] = Lsum > 0.f ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
  }
  // after a timeout (the outputs are then undefined): this warp's copies still in flight
  // land before the CTA exits
  if (*reinterpret_cast<volatile int*>(&xabort)) {
    if (lane == 0) {
      if (k_issued > k_seen) tc::mbar_drain(&kbar[warp], (uint32_t)((k_issued - 1) & 1), kDrainBudget);
      if (v_issued > v_seen) tc::mbar_drain(&vbar[warp], (uint32_t)((v_issued - 1) & 1), kDrainBudget);
      if (x_issued > x_seen) tc::mbar_drain(&xbar[my_x], 0, kDrainBudget);
    }
    if (tid == 0) g_blasst_decode_status = 1;
  }
}

// Units from which one CTA per unit fills the GPU better than a 16-CTA cluster per unit.
constexpr int kUnitKernelUnits = 64;

template <int D>
cudaError_t launch_unit(const DecodeBlasstArgs& a, const Params& p, cudaStream_t stream) {
  auto kernel = decode_blasst_unit_kernel<D>;
  const int smem = UnitLay<D>::kTotal + 1024;
  static DeviceOnce attr_once;
  const cudaError_t err = attr_once.run([&]() {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (err != cudaSuccess) return err;
  kernel<<<dim3(a.Hkv, a.B, 1), kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const DecodeBlasstArgs& a, cudaStream_t stream) {
  auto kernel = decode_blasst_kernel<D>;
  Params p{};
  if (!kv_tensor_maps(a.k, a.v, D, a.T_cap, a.B * a.Hkv, &p.tmk, &p.tmv)) return cudaErrorInvalidValue;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.Hkv = a.Hkv;
  p.G = a.G;
  p.T_cap = a.T_cap;
  p.seqlens = a.seqlens;
  p.idx = a.idx;
  p.nsel = a.nsel;
  p.topk = a.topk;
  p.scale2 = a.scale * kLog2e;
  p.log2_lambda = a.lambda > 0.f ? log2f(a.lambda) : -INFINITY;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.skip_bits = a.skip_bits;
  p.budget = wait_budget();
  if (a.B * a.Hkv >= kUnitKernelUnits) return launch_unit<D>(a, p, stream);
  const int smem = Lay<D>::kTotal + 1024;
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
  // shape: done once per device (the first launch on a device runs it, racing host
  // threads wait for it), so that a launch costs only the launch
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
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

}  // namespace

cudaError_t launch_decode_blasst(const DecodeBlasstArgs& a, cudaStream_t stream) {
  return a.D == 128 ? launch_d<128>(a, stream) : launch_d<64>(a, stream);
}

cudaError_t read_decode_blasst_status(int* status, bool reset) {
  cudaError_t err = cudaMemcpyFromSymbol(status, g_blasst_decode_status, sizeof(int));
  if (err == cudaSuccess && reset) {
    const int zero = 0;
    err = cudaMemcpyToSymbol(g_blasst_decode_status, &zero, sizeof(int));
  }
  return err;
}

LSA_BOUNDS_READER(decode_blasst)

}  // namespace lsa
