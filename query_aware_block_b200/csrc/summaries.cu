// summaries.cu -- mean-pooled key summary of each 64-token KV block.
//
// Prism, "1. 문제 정의" / "2. 핵심 이론적 발견": training-free block importance is estimated
// from the mean of the block's keys.  summ[b,g,j,:] = mean of the valid keys of block j
// (a partial last block is averaged over its valid tokens), accumulated in fp32.
//
// HBM-bound streaming read: each CTA owns kBPC consecutive blocks of one (b, g); every
// thread issues all of its 16-byte loads for those blocks before it accumulates, so a
// CTA keeps kBPC * 64 rows in flight.  Row groups are then reduced through shared memory.
#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {
namespace {

constexpr int kThreads = 256;
constexpr int kBPC = 4;  // blocks per CTA

template <typename T, int D>
struct SummaryGeom {
  static constexpr int kElemsPerChunk = 16 / sizeof(T);
  static constexpr int kChunksPerRow = D / kElemsPerChunk;
  static constexpr int kRowGroups = kThreads / kChunksPerRow;
  static constexpr int kRowsPerThread = kBlk / kRowGroups;
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
build_summaries_kernel(const T* __restrict__ k, int Hkv, int T_cap, const int32_t* __restrict__ seqlens,
                       int nb_begin, int nb_end, float* __restrict__ summ) {
  using Geo = SummaryGeom<T, D>;
  constexpr int EPC = Geo::kElemsPerChunk;
  constexpr int RPT = Geo::kRowsPerThread;
  __shared__ float red[Geo::kRowGroups][D];

  const int g = blockIdx.y, b = blockIdx.z;
  const int Tb = checked_range(seqlens[b], 0, T_cap, kBoundsSeqlen, kSiteSummaries);
  const int NB = (Tb + kBlk - 1) / kBlk;
  const int lo = nb_begin >= 0 ? nb_begin : max(0, NB + nb_begin);
  const int hi = nb_end >= 0 ? min(nb_end, NB) : NB;
  const int j0 = lo + blockIdx.x * kBPC;
  if (j0 >= hi) return;
  const int NB_cap = (T_cap + kBlk - 1) / kBlk;

  const int chunk = threadIdx.x % Geo::kChunksPerRow;
  const int rg = threadIdx.x / Geo::kChunksPerRow;
  const T* base = k + ((size_t)b * Hkv + g) * (size_t)T_cap * D + chunk * EPC;

  // issue every load first
  uint4 raw[kBPC][RPT];
#pragma unroll
  for (int bb = 0; bb < kBPC; ++bb) {
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int t = (j0 + bb) * kBlk + rg + r * Geo::kRowGroups;
      if (j0 + bb < hi && t < Tb)
        raw[bb][r] = __ldg(reinterpret_cast<const uint4*>(base + (size_t)t * D));
      else
        raw[bb][r] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

#pragma unroll
  for (int bb = 0; bb < kBPC; ++bb) {
    const int j = j0 + bb;
    if (j >= hi) break;  // uniform across the CTA
    float acc[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const T* v = reinterpret_cast<const T*>(&raw[bb][r]);
#pragma unroll
      for (int e = 0; e < EPC; ++e) acc[e] += to_f32(v[e]);
    }
#pragma unroll
    for (int e = 0; e < EPC; ++e) red[rg][chunk * EPC + e] = acc[e];
    __syncthreads();
    if (threadIdx.x < D) {
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < Geo::kRowGroups; ++q) s += red[q][threadIdx.x];
      const int n = min(kBlk, Tb - j * kBlk);
      summ[(((size_t)b * Hkv + g) * NB_cap + j) * D + threadIdx.x] = s / (float)n;
    }
    __syncthreads();
  }
}

template <typename T, int D>
cudaError_t launch_t(const void* k, int B, int Hkv, int T_cap, const int32_t* seqlens,
                     int nb_begin, int nb_end, int range_max, float* summ, cudaStream_t st) {
  if (range_max <= 0 || B <= 0 || Hkv <= 0) return cudaSuccess;
  dim3 grid((range_max + kBPC - 1) / kBPC, Hkv, B);
  build_summaries_kernel<T, D><<<grid, kThreads, 0, st>>>(
      static_cast<const T*>(k), Hkv, T_cap, seqlens, nb_begin, nb_end, summ);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_build_summaries(const void* k, int dtype, int B, int Hkv, int T_cap, int D,
                                   const int32_t* seqlens, int nb_begin, int nb_end,
                                   int range_max, float* summ, cudaStream_t stream) {
  if (dtype == DT_BF16) {
    if (D == 128)
      return launch_t<__nv_bfloat16, 128>(k, B, Hkv, T_cap, seqlens, nb_begin, nb_end, range_max, summ, stream);
    return launch_t<__nv_bfloat16, 64>(k, B, Hkv, T_cap, seqlens, nb_begin, nb_end, range_max, summ, stream);
  }
  if (D == 128)
    return launch_t<float, 128>(k, B, Hkv, T_cap, seqlens, nb_begin, nb_end, range_max, summ, stream);
  return launch_t<float, 64>(k, B, Hkv, T_cap, seqlens, nb_begin, nb_end, range_max, summ, stream);
}

LSA_BOUNDS_READER(summaries)

}  // namespace lsa
