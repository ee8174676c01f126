// tensor_map.cu -- host-side encoding of TMA tensor maps, through the driver entry point
// cuTensorMapEncodeTiled (so the library does not link against libcuda).
#include <cuda.h>
#include <cuda_runtime.h>

#include "lsa_internal.h"

namespace lsa {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

void* driver_entry(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
    return ptr;
  return nullptr;
}

// (function-local statics: initialised once, also when host threads race)
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(driver_entry("cuTensorMapEncodeTiled"));
  return fn;
}

}  // namespace

bool current_context_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_current = reinterpret_cast<CtxGetCurrentFn>(driver_entry("cuCtxGetCurrent"));
  static const CtxGetIdFn get_id = reinterpret_cast<CtxGetIdFn>(driver_entry("cuCtxGetId"));
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}


bool encode_rows_bf16(CUtensorMap* map, const void* base, int D, int rows, int planes, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)planes};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  const cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
// The K and V maps of the last call on this host thread: decode and block-query loops call
// with the same cache tensors every step, so the maps are encoded once.
struct KVMapCache {
  const void* k = nullptr;
  const void* v = nullptr;
  int D = 0, T_cap = 0, planes = 0;
  CUtensorMap mk, mv;
};
}  // namespace

bool kv_tensor_maps(const void* k, const void* v, int D, int T_cap, int planes, CUtensorMap* mk,
                    CUtensorMap* mv) {
  static thread_local KVMapCache c;
  if (!(c.k == k && c.v == v && c.D == D && c.T_cap == T_cap && c.planes == planes)) {
    c.k = nullptr;
    if (!encode_rows_bf16(&c.mk, k, D, T_cap, planes, 64) || !encode_rows_bf16(&c.mv, v, D, T_cap, planes, 64))
      return false;
    c.k = k; c.v = v; c.D = D; c.T_cap = T_cap; c.planes = planes;
  }
  *mk = c.mk;
  *mv = c.mv;
  return true;
}

}  // namespace lsa
