// kv_append.cu -- writes a decode step's new key and value rows into the KV cache; and a
// plain kernel copy for a step's small inputs and outputs.
//
// A decode step appends the newest token's key and value at cache row seqlens[b] - 1 (the
// sequence length already counts it) before attending: NSA news article, "NSA 구조" (the
// cache keeps every token; the selected, compressed and window branches read from it).
// One thread moves 16 bytes; the launch is tiny and latency-bound, so it lets the next
// kernel of the stream start at once (programmatic dependent launch): a decode step launched
// with LSA_FLAG_PDL overlaps its prologue with this copy and waits for it before it reads
// the newest block.  Launched itself with LSA_FLAG_PDL, it reads k_new / v_new only after
// the previous kernel of the stream (the one that produced them) has completed -- unless
// LSA_FLAG_INPUTS_READY says they were complete when the call was enqueued (written by the
// host): then it reads them at once, over PCIe when they are in pinned host memory, and waits
// only before writing.  The same launch may also copy the step's query rows.
#include "cluster.cuh"
#include "lsa_common.cuh"
#include "lsa_internal.h"

namespace lsa {
namespace {

constexpr int kThreads = 128;

// chunks [0, nq): the step's query rows, q_dst[c] = q_src[c]; then chunk c of the
// n = B * Hkv * rows16 16-byte chunks of k_new (then of v_new): unit u = c / rows16 =
// b * Hkv + g, column part c % rows16
__global__ void __launch_bounds__(kThreads)
    kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, int Hkv, int T_cap,
                     int rows16, int n, const int32_t* __restrict__ seqlens, uint4* __restrict__ k,
                     uint4* __restrict__ v, const uint4* __restrict__ q_src, uint4* __restrict__ q_dst, int nq,
                     int inputs_ready) {
  pdl_trigger();  // the next kernel may start its prologue now ...
  // ... while this one waits for the kernel that produced its inputs (or, when they are
  // ready at enqueue, reads them first and waits only before writing)
  if (!inputs_ready) pdl_wait();
  int c = blockIdx.x * kThreads + threadIdx.x;
  if (c < nq) {
    const uint4 x = q_src[c];
    if (inputs_ready) pdl_wait();
    q_dst[c] = x;
    return;
  }
  c -= nq;
  if (c >= 2 * n) return;
  const bool is_v = c >= n;
  const int cc = is_v ? c - n : c;
  const int u = cc / rows16, part = cc - u * rows16;
  const int b = u / Hkv;
  const int t = checked_range(seqlens[b], 0, T_cap, kBoundsSeqlen, kSiteKvAppend) - 1;
  if (t < 0 || t >= T_cap) return;  // an empty sequence has no newest token
  const uint4 x = is_v ? v_new[cc] : k_new[cc];
  uint4* dst = (is_v ? v : k) + ((size_t)u * T_cap + t) * rows16 + part;
  if (inputs_ready) pdl_wait();
  *dst = x;
}

// A copy by a kernel, 16 bytes per thread and iteration: either side may be pinned host
// memory (every pinned allocation is mapped under unified addressing, and plain loads and
// stores reach it over PCIe), so a decode step's small inputs and outputs need no copy-engine
// round trip.  It lets the next kernel start at once and touches memory only after the
// previous kernel of the stream has completed (programmatic dependent launch), or, with
// inputs ready at enqueue, reads its first chunk at once and waits only before writing.
__global__ void __launch_bounds__(kThreads) copy16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          size_t n16, int inputs_ready) {
  pdl_trigger();
  if (!inputs_ready) pdl_wait();
  const size_t i0 = blockIdx.x * (size_t)kThreads + threadIdx.x, step = (size_t)gridDim.x * kThreads;
  if (inputs_ready && i0 < n16) {  // the first chunk read before the wait
    const uint4 x = src[i0];
    pdl_wait();
    dst[i0] = x;
    for (size_t i = i0 + step; i < n16; i += step) dst[i] = src[i];
  } else {
    for (size_t i = i0; i < n16; i += step) dst[i] = src[i];
  }
}

}  // namespace

cudaError_t launch_copy16(void* dst, const void* src, size_t bytes, int pdl, cudaStream_t stream,
                          int inputs_ready) {
  const size_t n16 = bytes / 16;
  size_t blocks = (n16 + kThreads - 1) / kThreads;
  if (blocks > 1184) blocks = 1184;  // (8 per SM on 148 SMs; the loop strides over the rest)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, copy16_kernel, static_cast<const uint4*>(src), static_cast<uint4*>(dst), n16,
                            pdl && inputs_ready ? 1 : 0);
}

cudaError_t launch_kv_append(const void* k_new, const void* v_new, int elem_bytes, int B, int Hkv,
                             int T_cap, int D, const int32_t* seqlens, void* k, void* v, int pdl,
                             cudaStream_t stream, const void* q_src, void* q_dst, size_t q_bytes,
                             int inputs_ready) {
  const int rows16 = D * elem_bytes / 16;
  const int n = B * Hkv * rows16;
  const int nq = (int)(q_bytes / 16);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((nq + 2 * n + kThreads - 1) / kThreads, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kv_append_kernel, static_cast<const uint4*>(k_new),
                            static_cast<const uint4*>(v_new), Hkv, T_cap, rows16, n, seqlens,
                            static_cast<uint4*>(k), static_cast<uint4*>(v), static_cast<const uint4*>(q_src),
                            static_cast<uint4*>(q_dst), nq, pdl && inputs_ready ? 1 : 0);
}

LSA_BOUNDS_READER(kv_append)

}  // namespace lsa
