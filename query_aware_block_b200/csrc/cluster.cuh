// cluster.cuh -- thread-block-cluster and launch primitives shared by the kernels
// (PTX ISA: barrier.cluster, mapa, st.shared::cluster, st.async, griddepcontrol), and the warp-wide
// bitonic merge used to combine sorted candidate lists.
#pragma once

#include <stdint.h>

namespace lsa {

// ---- cluster primitives (PTX ISA: barrier.cluster, mapa, st.shared::cluster) ----------
__device__ __forceinline__ int cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return (int)r;
}
__device__ __forceinline__ int cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return (int)r;
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_rank(const void* p, int r) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(a), "r"(r));
  return out;
}
__device__ __forceinline__ void st_cluster(uint32_t addr, unsigned long long v) {
  asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}
__device__ __forceinline__ void st_cluster(uint32_t addr, float2 v) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(v.x), "f"(v.y)
               : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// st.async: a store into a peer CTA's shared memory whose bytes count toward the
// transaction count of an mbarrier in that CTA (both addresses from mapa).  The receiver
// learns that the data has landed by waiting on its own mbarrier; no cluster barrier.
__device__ __forceinline__ void st_async(uint32_t addr, unsigned long long v, uint32_t mbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];" ::"r"(addr),
               "l"(v), "r"(mbar)
               : "memory");
}
__device__ __forceinline__ void st_async(uint32_t addr, float2 v, uint32_t mbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(
                   addr),
               "f"(v.x), "f"(v.y), "r"(mbar)
               : "memory");
}
__device__ __forceinline__ void st_async(uint32_t addr, float v, uint32_t mbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];" ::"r"(addr),
               "f"(v), "r"(mbar)
               : "memory");
}

// Programmatic dependent launch (PTX griddepcontrol): with the launch attribute set, the
// grid may start while the previous kernel of the stream still runs; `wait` blocks until
// that kernel has completed and its memory is visible.  Without the attribute both are
// no-ops in effect.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Bitonic merge, descending, of the 32E-long sequence held by a warp (lane l holds
// positions l*E .. l*E+E-1): positions [0, 16E) are a descending list and [16E, 32E) a
// list in ascending order, so the whole is bitonic.  Afterwards the sequence is sorted
// descending; the top 16E keys sit in lanes 0..15.
template <int E>
__device__ __forceinline__ void warp_merge_desc(unsigned long long (&x)[E]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int dist = 16 * E; dist >= 1; dist >>= 1) {
    if (dist >= E) {
      const int ld = dist / E;
      const bool lower = (lane & ld) == 0;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, x[e], ld);
        x[e] = lower ? (x[e] > y ? x[e] : y) : (x[e] < y ? x[e] : y);
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        if ((e & dist) == 0) {
          const unsigned long long a = x[e], b = x[e ^ dist];
          x[e] = a > b ? a : b;
          x[e ^ dist] = a > b ? b : a;
        }
      }
    }
  }
}

}  // namespace lsa
