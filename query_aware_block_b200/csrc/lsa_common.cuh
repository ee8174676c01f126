// lsa_common.cuh -- device helpers shared by the liblsa kernels (sm_100a).
//
// Small wrappers over PTX instructions documented in the PTX ISA: cp.async (16-byte
// global->shared copies with zero fill), ldmatrix, mma.sync m16n8k16 bf16, ex2.approx,
// plus warp reductions and the 64-bit selection key.  No math-library code is
// reproduced here.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lsa {

constexpr int kBlk = 64;            // KV block (selection unit) in tokens
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---- division by a divisor known only at launch -----------------------------------------
// floor(n / d) for 0 <= n < 2^31 as one 32x32->64 multiply and a shift: m = ceil(2^(31+l)/d)
// with l = ceil(log2 d) (the round-up method of Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994).  An integer division by a run-time
// value costs tens of instructions on the GPU; the constants are computed on the host.
struct FastDiv {
  uint32_t m;
  uint32_t sh;
};
inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  const unsigned long long num = 1ull << (31 + l);
  FastDiv f;
  f.m = (uint32_t)((num + d - 1) / d);
  f.sh = 31 + l;
  return f;
}
__device__ __forceinline__ int fdiv(int n, FastDiv f) {
  return (int)(((unsigned long long)(uint32_t)n * f.m) >> f.sh);
}

// ---- debug bounds checks (a build with LSA_DEBUG_BOUNDS) -------------------------------
// A value read from device memory that decides where a kernel reads or writes (a sequence
// length, a selection index, a selection count) is trusted by the release build.  A build
// with LSA_DEBUG_BOUNDS checks it instead: the first value out of its documented range is
// recorded in this translation unit's status word as (kind << 8) | site, the value is
// clamped into range so that every access stays in bounds, and nothing traps.
enum { kBoundsSeqlen = 1, kBoundsIndex = 2, kBoundsCount = 3 };
enum { kSiteSummaries = 1, kSiteDecode = 2, kSiteDecodeBlasst = 3, kSiteNsaCompress = 4,
       kSiteNsaBranches = 5, kSiteKvAppend = 6 };
#ifdef LSA_DEBUG_BOUNDS
namespace {
__device__ int g_bounds_word = 0;
}
__device__ __forceinline__ int checked_range(int v, int lo, int hi, int kind, int site) {
  if (v < lo || v > hi) {
    atomicCAS(&g_bounds_word, 0, (kind << 8) | site);
    return v < lo ? lo : hi;
  }
  return v;
}
#define LSA_BOUNDS_READER(name)                                                   \
  cudaError_t read_bounds_##name(int* word, bool reset) {                         \
    cudaError_t err = cudaMemcpyFromSymbol(word, g_bounds_word, sizeof(int));     \
    if (err == cudaSuccess && reset) {                                            \
      const int zero = 0;                                                         \
      err = cudaMemcpyToSymbol(g_bounds_word, &zero, sizeof(int));                \
    }                                                                             \
    return err;                                                                   \
  }
#else
__device__ __forceinline__ int checked_range(int v, int, int, int, int) { return v; }
#define LSA_BOUNDS_READER(name)                              \
  cudaError_t read_bounds_##name(int* word, bool) {          \
    *word = 0;                                               \
    return cudaSuccess;                                      \
  }
#endif

// ---- element conversion ------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low 16 bits)
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---- fast base-2 exponential: the hardware MUFU instruction -------------------------
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- sm_100 three-input max and packed two-wide fp32 arithmetic (PTX ISA: max with three
// inputs; fma / add .rn.f32x2): one instruction for two lanes of work ---------------------
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
// a * b + c, element-wise on pairs, rounded to nearest
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// ---- warp reductions -----------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---- selection key: larger key = higher score, ties to the lower block index --------
__device__ __forceinline__ uint32_t orderable(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ unsigned long long make_key(float score, int j) {
  return ((unsigned long long)orderable(score) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)j);
}
__device__ __forceinline__ int key_block(unsigned long long key) {
  return (int)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
}

// ---- cp.async (Ampere-style async copies, 16 bytes, zero fill when !valid) -----------
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ---- ldmatrix / mma.sync ---------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(s));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(s));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], const void* p) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(s));
}
// D(16x8 f32) += A(16x16 bf16, row) * B(16x8 bf16, col)
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk c of row r in a [rows][row_bytes] shared tile whose chunks
// are XOR-swizzled by (r & 7): conflict-free for ldmatrix and for row-wise cp.async.
__device__ __forceinline__ int swz(int r, int c, int row_bytes) {
  return r * row_bytes + ((c ^ (r & 7)) << 4);
}

// Byte offset of 16-byte chunk c of row r in a bf16 K/V tile of 64 rows: [c / 8][r][128 B]
// with the chunk index XOR-swizzled by (r & 7), i.e. where 128-byte-swizzled TMA boxes of
// 64 elements x 64 rows land; ldmatrix over 8 consecutive rows is conflict-free.
__device__ __forceinline__ int kv_off(int r, int c) {
  return ((c >> 3) << 13) + (r << 7) + ((((c & 7) ^ (r & 7))) << 4);
}

// ---- K/V block staging ----------------------------------------------------------------

// Copy the K and V rows of block j (64 tokens) into a stage with 16-byte cp.async: rows
// >= Tb, and every row of an invalid j < 0, are zero-filled and never read from global
// memory.  bf16 rows are chunk-swizzled; fp32 rows are padded by 16 bytes.
template <typename T, int D, int kThreads>
__device__ __forceinline__ void stage_block(unsigned char* dst_k, unsigned char* dst_v,
                                            const T* kbase, const T* vbase, int j, int Tb,
                                            int kv_row) {
  constexpr int kChunks = D * (int)sizeof(T) / 16;  // 16-byte chunks per row
  constexpr int kTotal = 2 * kBlk * kChunks;
  constexpr bool kF32 = sizeof(T) == 4;
#pragma unroll
  for (int it = 0; it < kTotal / kThreads; ++it) {
    const int id = threadIdx.x + it * kThreads;
    const int tensor = id / (kBlk * kChunks);
    const int rem = id % (kBlk * kChunks);
    const int row = rem / kChunks, c = rem % kChunks;
    const int t = j * kBlk + row;
    const bool valid = j >= 0 && j < (Tb + kBlk - 1) / kBlk && t < Tb;
    const T* src = (tensor ? vbase : kbase) + (size_t)(valid ? t : 0) * D + c * (16 / sizeof(T));
    unsigned char* dst = (tensor ? dst_v : dst_k) + (kF32 ? row * kv_row + c * 16 : swz(row, c, kv_row));
    cp_async16(dst, src, valid);
  }
}

}  // namespace lsa
