// weighted.cu -- block selection with a weight per head dimension (FASA- and Prism-style
// scorers): the group score becomes scale * sum_h sum_d w_d q_{h,d} kbar_{j,d}, which is the
// plain score of the reweighted queries q'_{h,d} = w_d q_{h,d}.  One small kernel forms q'
// in fp32 (no rounding that could move a near-tie), then the selection kernel of decode.cu
// runs on q' unchanged (its fp32 path).
//
// FASA, "2. 방법론" (token importance from the dominant rotary frequency chunks only) and
// Prism, "3. 제안 방법론" (dual-band block importance with a temperature per band).
#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {
namespace {

template <typename T>
__global__ void weight_queries_kernel(const T* q, const float* __restrict__ w, int D, size_t n,
                                      float* out) {  // (out may be q: element i read, then written)
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    out[i] = to_f32(q[i]) * w[i % D];
}

}  // namespace

cudaError_t launch_weight_queries(const void* q, int dtype, const float* w, int B, int Hq, int D,
                                  float* out, cudaStream_t stream) {
  const size_t n = (size_t)B * Hq * D;
  const int threads = 256;
  const int blocks = (int)((n + threads - 1) / threads < 4096 ? (n + threads - 1) / threads : 4096);
  if (dtype == DT_BF16)
    weight_queries_kernel<__nv_bfloat16><<<blocks, threads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), w, D, n, out);
  else
    weight_queries_kernel<float><<<blocks, threads, 0, stream>>>(static_cast<const float*>(q), w, D, n, out);
  return cudaGetLastError();
}

}  // namespace lsa
