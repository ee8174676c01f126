// blasst_prefill.cu -- causal prefill that skips whole KV tiles by a softmax threshold
// (BLASST), on the sm_100a tensor cores (tcgen05, accumulators in tensor memory).
//
// What is computed (BLASST, "2. 방법론": "핵심 아이디어: 온라인 Softmax 통계 활용",
// "알고리즘 및 커널 설계"): for each query head and 128-row query tile, the 64-key KV tiles
// up to the causal diagonal are visited in ascending order with an online softmax; a tile
// is skipped -- no exponentials, no P.V product -- when every row's tile maximum trails its
// running maximum by more than -ln(lambda):  max_i (r_i - m_i) < ln(lambda).
//
// How (B200): one CTA per (b, h, query tile), heaviest tiles first, the query tiles of one
// head launched together (their KV group stays in L2); 8 warps, 2 CTAs per SM so that one
// CTA's softmax overlaps the other's tensor-core work (each holds 256 of the 512 TMEM
// columns).
//   warp 0    TMA producers: lane 0 loads Q once (2 boxes of 128 x 64 bf16, 128-byte
//             swizzle) and then the K tiles, lane 1 the V tiles, each into its own 2-stage
//             ring (3-D tensor maps, no multicast): K_j is released when S_j is done, V_j
//             when P_j V_j is, so the next K tiles arrive while P V is still pending.
//   warp 1    MMA issuer (one thread): S_j = Q K_j^T (M 128, N 64, K 128) into a
//             double-buffered TMEM tile; O += P_j V_j (M 128, N 128, K 64) with P read from
//             tensor memory; tcgen05.commit signals S ready, O updated, stage free.
//   warp 2    allocates / frees 256 TMEM columns: S0 [0,64), S1 [64,128), O [128,256).
//   warps 4-7 softmax: thread = query row = TMEM lane.  Loads its S row, masks, takes the
//             row max, votes on the skip (a warp with a non-negligible row marks the tile
//             kept and goes on; only an all-negligible warp waits on the vote mbarrier), writes
//             P (bf16) back over its S columns, rescales its O row only when its running
//             max grew by more than 2^8 since the exponent base was last set (exact: the
//             final normalisation uses the same base), and stores o and lse at the end.
// The MMA for S_{j+2} is issued as soon as P_j is consumed, so Q K^T of the next tiles
// overlaps the softmax of the current one.  Every mbarrier wait is clock-bounded; a
// timeout raises a CTA-wide abort and every role leaves its loop; the TMA producers then wait
// (with a second bound) for the loads they issued, the MMA thread for the tensor-core work
// it issued, so nothing lands in shared or tensor memory after the TMEM is freed, and the
// device status word records the failure.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include "launch_cache.h"
#include "lsa_common.cuh"
#include "lsa_internal.h"
#include "tcgen05.cuh"

namespace lsa {

// 0 = no error; LSA_DEVICE_TIMEOUT when a bounded wait of a kernel ran out.
__device__ int g_device_status = 0;

namespace {

constexpr int kThreads = 256;
constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 64;           // keys per KV tile
constexpr int kD = 128;           // head dim
constexpr int kStages = 2;       // (2 CTAs per SM: their softmax and MMA phases interleave)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 128;
constexpr int kQBytes = kBM * kD * 2;        // 32 KB
constexpr int kKVTileBytes = kBN * kD * 2;   // 16 KB per tensor
constexpr int kStageBytes = 2 * kKVTileBytes;
constexpr float kRescaleLog2 = 8.0f;             // rescale O when the max grew by > 2^8
constexpr int kDeviceTimeout = 1;

struct alignas(64) PrefillParams {
  CUtensorMap tq;  // [B*Hq][L][D]
  CUtensorMap tk;  // [B*Hkv][L][D]
  CUtensorMap tv;
  __nv_bfloat16* o;
  float* lse;
  uint32_t* skip_bits;
  unsigned long long* skipped;
  int Hq, Hkv, L, nqt, words;
  float scale2;    // softmax scale * log2(e)
  float log2lam;   // log2(lambda), -inf for lambda = 0
  long long budget;  // clock-cycle limit of every bounded wait
  int drop_s;        // test injection: the first S tile is never signalled
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[kStages];   // K and V have separate rings: K_j is free once S_j is done,
  uint64_t k_empty[kStages];  // long before P_j V_j frees V_j
  uint64_t v_full[kStages];
  uint64_t v_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t vote[2];           // one arrival per softmax warp and tile: the skip vote is in
  uint64_t o_done[2];         // P.V number n completes on o_done[n & 1]
  uint64_t drain;             // after a timeout: every tcgen05 operation issued has completed
  uint32_t tmem;
  int nonneg[2];              // the last tile (of this buffer) some softmax warp kept
  int abort;
};

constexpr size_t kSmemBytes = 1024 /*alignment slack*/ + kQBytes + kStages * kStageBytes + 256;

__global__ void __launch_bounds__(kThreads, 2) blasst_prefill_kernel(const __grid_constant__ PrefillParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* Qs = smem;
  unsigned char* Kring = smem + kQBytes;                        // kStages K tiles
  unsigned char* Vring = Kring + kStages * kKVTileBytes;        // kStages V tiles
  Bars* bars = reinterpret_cast<Bars*>(smem + kQBytes + kStages * kStageBytes);
  volatile int* abort = &bars->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid x: query tiles, heaviest first; y: b * Hq + h, so that the CTAs running together
  // share one KV group's K/V in L2
  const int bh = blockIdx.y;
  const int a = p.nqt - 1 - (int)blockIdx.x;
  const int G = p.Hq / p.Hkv;
  const int b = bh / p.Hq, h = bh - b * p.Hq;
  const int bg = b * p.Hkv + h / G;
  const int i0 = a * kBM;
  const int i1 = min(i0 + kBM, p.L);
  const int n_visit = (i1 - 1) / kBN + 1;

  if (tid == 0) {
    tc::mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->k_full[s], 1);
      tc::mbar_init(&bars->k_empty[s], 1);
      tc::mbar_init(&bars->v_full[s], 1);
      tc::mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->p_full[s], 128);
      tc::mbar_init(&bars->vote[s], 4);
      bars->nonneg[s] = -1;
    }
    tc::mbar_init(&bars->o_done[0], 1);
    tc::mbar_init(&bars->o_done[1], 1);
    tc::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 2) {
    tc::tmem_alloc(&bars->tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem;

  int kv_issued = 0;  // (TMA producer lanes) loads issued into the ring
  if (warp == 0 && lane < 2) {
    // --------------------------------------------------------------- TMA producers ----
    // lane 0: Q, then the K tiles; lane 1: the V tiles (each ring on its own barriers)
    if (lane == 0) {
      tc::prefetch_tmap(&p.tq);
      tc::prefetch_tmap(&p.tk);
      tc::mbar_arrive_expect_tx(&bars->q_full, kQBytes);
      tc::tma_load_3d(Qs, &p.tq, 0, i0, bh, &bars->q_full);
      tc::tma_load_3d(Qs + kQBytes / 2, &p.tq, 64, i0, bh, &bars->q_full);
    } else {
      tc::prefetch_tmap(&p.tv);
    }
    const CUtensorMap* map = lane == 0 ? &p.tk : &p.tv;
    unsigned char* ring = lane == 0 ? Kring : Vring;
    uint64_t* full = lane == 0 ? bars->k_full : bars->v_full;
    uint64_t* empty = lane == 0 ? bars->k_empty : bars->v_empty;
    for (int j = 0; j < n_visit; ++j) {
      const int s = j % kStages;
      if (j >= kStages && !tc::mbar_wait(&empty[s], ((j / kStages) - 1) & 1, abort, p.budget)) break;
      unsigned char* dst = ring + s * kKVTileBytes;
      tc::mbar_arrive_expect_tx(&full[s], kKVTileBytes);
      tc::tma_load_3d(dst, map, 0, j * kBN, bg, &full[s]);
      tc::tma_load_3d(dst + kKVTileBytes / 2, map, 64, j * kBN, bg, &full[s]);
      ++kv_issued;
    }
  } else if (warp == 1 && lane == 0) {
    // ----------------------------------------------------------------- MMA issuer ----
    constexpr uint32_t idesc_qk = tc::idesc_bf16_f32(kBM, kBN, false);
    constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(kBM, kD, true);
    const uint32_t q_addr = tc::smem_u32(Qs);
    const uint32_t kring_addr = tc::smem_u32(Kring);
    const uint32_t vring_addr = tc::smem_u32(Vring);
    auto issue_s = [&](int j) -> bool {
      const int s = j % kStages;
      if (!tc::mbar_wait(&bars->k_full[s], (j / kStages) & 1, abort, p.budget)) return false;
      const uint32_t k_addr = kring_addr + s * kKVTileBytes;
      const uint32_t d = tmem + (uint32_t)(j & 1) * 64u;
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        // K-major, 128-byte swizzle: 64-element boxes; a K step of 16 is 32 bytes in a box
        const uint64_t ad = tc::smem_desc_sw128(q_addr + (ks >> 2) * (kQBytes / 2) + (ks & 3) * 32, 16, 1024);
        const uint64_t bd = tc::smem_desc_sw128(k_addr + (ks >> 2) * (kKVTileBytes / 2) + (ks & 3) * 32, 16, 1024);
        tc::mma_ss(d, ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
      }
      if (!(p.drop_s && j == 0)) tc::mma_commit(&bars->s_full[j & 1]);
      tc::mma_commit(&bars->k_empty[s]);  // K_j is no longer needed once S_j is done
      return true;
    };
    bool ok = tc::mbar_wait(&bars->q_full, 0, abort, p.budget);
    if (ok) ok = issue_s(0);
    if (ok && n_visit > 1) ok = issue_s(1);
    int pv_count = 0;
    for (int j = 0; ok && j < n_visit; ++j) {
      const int buf = j & 1, s = j % kStages;
      if (!tc::mbar_wait(&bars->p_full[buf], (j >> 1) & 1, abort, p.budget)) break;
      tc::fence_after_sync();
      const bool kept = reinterpret_cast<volatile int*>(bars->nonneg)[buf] == j;
      if (kept) {
        if (!tc::mbar_wait(&bars->v_full[s], (j / kStages) & 1, abort, p.budget)) break;
        const uint32_t v_addr = vring_addr + s * kKVTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // V as B (K = keys, N = dims): MN-major, 128-byte swizzle; the two 64-dim boxes are
          // LBO = 8 KB apart, 8-key groups SBO = 1 KB apart; P from TMEM (8 columns per K 16)
          const uint64_t bd = tc::smem_desc_sw128(v_addr + kk * 16 * 128, kKVTileBytes / 2, 1024);
          tc::mma_ts(tmem + kColO, tmem + (uint32_t)buf * 64u + (uint32_t)kk * 8u, bd, idesc_pv,
                     (pv_count > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(&bars->o_done[pv_count & 1]);
        ++pv_count;
      } else if (!tc::mbar_wait(&bars->v_full[s], (j / kStages) & 1, abort, p.budget)) {
        break;
      }
      tc::mma_commit(&bars->v_empty[s]);  // (a skipped tile's V is released unread)
      if (j + 2 < n_visit && !issue_s(j + 2)) break;
    }

  } else if (warp >= 4) {
    // ------------------------------------------------------------------- softmax ----
    const int row = tid - 128;
    const int i = i0 + row;
    const bool row_ok = i < p.L;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp - 4)) << 16);
    float m_run = -INFINITY, m_used = -INFINITY, l = 0.f;
    int pv_issued = 0;
    uint32_t skipmask = 0;
    int nskipped = 0;
    bool failed = false;
    uint32_t* bits_row = p.skip_bits ? p.skip_bits + ((size_t)bh * p.nqt + a) * p.words : nullptr;
    // No block-wide barrier inside the loop: every wait is a bounded mbarrier wait whose
    // outcome is made warp-uniform, so a failure lets each warp leave on its own.
    for (int j = 0; j < n_visit; ++j) {
      const int buf = j & 1;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->s_full[buf], (j >> 1) & 1, abort, p.budget))) {
        failed = true;
        break;
      }
      tc::fence_after_sync();
      uint32_t sr[64];
      {
        uint32_t lo[32], hi[32];
        tc::tmem_ld32(lane_addr + (uint32_t)buf * 64u, lo);
        tc::tmem_ld32(lane_addr + (uint32_t)buf * 64u + 32u, hi);
        tc::tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          sr[c] = lo[c];
          sr[32 + c] = hi[c];
        }
      }
      // the row max of the raw logits, masking (-inf) only where the causal / length mask
      // cuts this tile; scaled to log2 units after the max (scale2 > 0 commutes with it)
      const int t0 = j * kBN;
      const int lim = min(i, p.L - 1) - t0;  // keys t0 + c with c <= lim are visible
      // (8 independent chains of three-input maxima: a single chain of 64 dependent max
      // operations would dominate the softmax latency)
      if (!(row_ok && lim >= kBN - 1)) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          sr[c] = (row_ok && c <= lim) ? sr[c] : __float_as_uint(-INFINITY);
      }
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float mk = fmax3f(__uint_as_float(sr[e]), __uint_as_float(sr[e + 8]), __uint_as_float(sr[e + 16]));
        mk = fmax3f(mk, __uint_as_float(sr[e + 24]), __uint_as_float(sr[e + 32]));
        mk = fmax3f(mk, __uint_as_float(sr[e + 40]), __uint_as_float(sr[e + 48]));
        mx8[e] = fmaxf(mk, __uint_as_float(sr[e + 56]));
      }
      const float rmax = fmaxf(fmax3f(mx8[0], mx8[1], mx8[2]), fmax3f(fmax3f(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
      const float r = rmax * p.scale2;
      // the skip vote: every row negligible (absent rows and rows without a visible key agree)
      const bool negligible = !row_ok || r == -INFINITY || (m_run != -INFINITY && (r - m_run) < p.log2lam);
      // The vote, without a block barrier: a warp holding a non-negligible row marks the
      // tile kept and goes on (the tile cannot be skipped any more); a warp whose rows are
      // all negligible waits for the four warps' votes.  The MMA thread reads the mark after
      // all 128 rows have released the tile.
      const bool warp_neg = __all_sync(0xffffffffu, negligible);
      if (!warp_neg && lane == 0) reinterpret_cast<volatile int*>(bars->nonneg)[buf] = j;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->vote[buf]);
      bool skip = false;
      if (warp_neg) {
        if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->vote[buf], (j >> 1) & 1, abort, p.budget))) {
          failed = true;
          break;
        }
        skip = reinterpret_cast<volatile int*>(bars->nonneg)[buf] != j;
      }
      if (skip) {
        if (row == 0) {
          skipmask |= 1u << (j & 31);
          ++nskipped;
        }
        tc::mbar_arrive(&bars->p_full[buf]);
      } else {
        m_run = fmaxf(m_run, r);
        float base = m_used;
        bool resc = false;
        if (m_used == -INFINITY) {
          base = m_run;
        } else if (m_run > m_used + kRescaleLog2) {
          base = m_run;
          resc = true;
        }
        const float alpha = resc ? ex2(m_used - base) : 1.f;
        m_used = base;
        uint32_t pk[32];
        float rs = 0.f;
        if (base == -INFINITY) {  // no visible key so far: P = 0
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = 0u;
        } else {
          // p = 2^(scale2 * s - base): the scale folded into one two-wide FMA per pair of
          // elements; the row sum in 4 independent two-wide partial sums
          const unsigned long long sc2 = f2_pack(p.scale2, p.scale2), nb2 = f2_pack(-base, -base);
          unsigned long long rs2[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) rs2[e] = 0ull;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sc2, nb2), x0, x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            rs2[c & 3] = f2_add(rs2[c & 3], f2_pack(p0, p1));
            pk[c] = pack_bf16x2(p0, p1);
          }
          float a0, a1;
          f2_unpack(f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3])), a0, a1);
          rs = a0 + a1;
        }
        l = l * alpha + rs;
        tc::tmem_st32(lane_addr + (uint32_t)buf * 64u, pk);
        tc::tmem_st_wait();
        const bool warp_resc = __any_sync(0xffffffffu, resc);
        if (warp_resc && pv_issued > 0) {
          // O is rescaled in place, so the last P.V issued (number pv_issued - 1) must be
          // complete (tcgen05 work completes in issue order: so are all earlier ones).  It
          // is the ((pv_issued - 1) >> 1)-th completion of o_done[(pv_issued - 1) & 1], and
          // that barrier cannot complete again before this warp releases a later tile, so
          // the parity wait is unambiguous.  Without a rescale nothing waits for O.
          const int n = pv_issued - 1;
          if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->o_done[n & 1], (uint32_t)((n >> 1) & 1), abort,
                                                     p.budget))) {
            failed = true;
            break;
          }
          tc::fence_after_sync();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t ov[32];
            tc::tmem_ld32(lane_addr + kColO + 32u * q4, ov);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tc::tmem_st32(lane_addr + kColO + 32u * q4, ov);
          }
          tc::tmem_st_wait();
        }
        tc::fence_before_sync();
        tc::mbar_arrive(&bars->p_full[buf]);
        ++pv_issued;
      }
      if (row == 0 && bits_row && ((j & 31) == 31 || j == n_visit - 1)) {
        bits_row[j >> 5] = skipmask;
        skipmask = 0;
      }
    }
    if (!failed && pv_issued > 0) {  // the last P.V (and with it every earlier one) is complete
      const int n = pv_issued - 1;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&bars->o_done[n & 1], (uint32_t)((n >> 1) & 1), abort,
                                                 p.budget)))
        failed = true;
    }
    if (!failed) {
      tc::fence_after_sync();
      const float inv_l = (pv_issued > 0 && l > 0.f) ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.o + ((size_t)bh * p.L + (row_ok ? i : 0)) * kD;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t ov[32];
        tc::tmem_ld32(lane_addr + kColO + 32u * q4, ov);
        tc::tmem_ld_wait();
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q4);
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ov[8 * c8 + 0]) * inv_l, __uint_as_float(ov[8 * c8 + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(ov[8 * c8 + 2]) * inv_l, __uint_as_float(ov[8 * c8 + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(ov[8 * c8 + 4]) * inv_l, __uint_as_float(ov[8 * c8 + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(ov[8 * c8 + 6]) * inv_l, __uint_as_float(ov[8 * c8 + 7]) * inv_l);
            dst[c8] = w;
          }
        }
      }
      if (row_ok && p.lse) p.lse[(size_t)bh * p.L + i] = (m_used + log2f(l)) * kLn2;
      if (row == 0 && bits_row)
        for (int w = (n_visit + 31) >> 5; w < p.words; ++w) bits_row[w] = 0u;
      if (row == 0 && p.skipped && nskipped) atomicAdd(p.skipped, (unsigned long long)nskipped);
    }
    tc::fence_before_sync();
  }

  __syncthreads();
  // every role has left its loop: after a timeout, nothing may land in shared or tensor
  // memory once the CTA has gone, so the producers wait (bounded) for the last load issued
  // into every stage of their ring (earlier ones into a stage completed before it was
  // reused) and the MMA thread for all the tensor-core work it issued
  const bool aborted = bars->abort != 0;
  if (aborted) {
    if (warp == 0 && lane < 2) {
      uint64_t* full = lane == 0 ? bars->k_full : bars->v_full;
      for (int j = kv_issued - kStages < 0 ? 0 : kv_issued - kStages; j < kv_issued; ++j)
        tc::mbar_drain(&full[j % kStages], (uint32_t)((j / kStages) & 1), kDrainBudget);
      if (lane == 0) tc::mbar_drain(&bars->q_full, 0, kDrainBudget);
    } else if (warp == 1 && lane == 0) {
      tc::mma_commit(&bars->drain);
      tc::mbar_drain(&bars->drain, 0, kDrainBudget);
    }
    __syncthreads();
  }
  if (tid == 0 && aborted) g_device_status = kDeviceTimeout;
  if (warp == 2) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host ---------------------------------------------------------------------------------
// 3-D map over [planes][rows][D] bf16, box {64, box_rows, 1}, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* map, const void* base, int planes, int rows, int box_rows) {
  return encode_rows_bf16(map, base, kD, rows, planes, box_rows);
}

}  // namespace

cudaError_t launch_blasst_prefill(const PrefillArgs& a, cudaStream_t stream) {
  PrefillParams p;
  memset(&p, 0, sizeof(p));
  if (!make_map(&p.tq, a.q, a.B * a.Hq, a.L, kBM) || !make_map(&p.tk, a.k, a.B * a.Hkv, a.L, kBN) ||
      !make_map(&p.tv, a.v, a.B * a.Hkv, a.L, kBN))
    return cudaErrorInvalidValue;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.skip_bits = a.skip_bits;
  p.skipped = a.skipped_tiles;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.L = a.L;
  p.nqt = (a.L + kBM - 1) / kBM;
  p.words = ((a.L + kBN - 1) / kBN + 31) / 32;
  p.scale2 = a.scale * kLog2e;
  p.log2lam = a.lambda > 0.f ? log2f(a.lambda) : -INFINITY;
  p.budget = wait_budget();
  p.drop_s = debug_inject() == 1 ? 1 : 0;
  // the shared memory attribute applies to the current device: set once per device
  static DeviceOnce attr_once;
  const cudaError_t err = attr_once.run([] {
    return cudaFuncSetAttribute(blasst_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  });
  if (err != cudaSuccess) return err;
  dim3 grid(p.nqt, a.B * a.Hq, 1);
  blasst_prefill_kernel<<<grid, kThreads, kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t read_device_status(int* status, bool reset) {
  cudaError_t err = cudaMemcpyFromSymbol(status, g_device_status, sizeof(int));
  if (err == cudaSuccess && reset) {
    const int zero = 0;
    err = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  }
  return err;
}

}  // namespace lsa
