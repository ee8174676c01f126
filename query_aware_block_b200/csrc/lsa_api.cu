// lsa_api.cu -- the exported C ABI (include/lsa.h): host-side validation, then launch.
// Nothing is launched when an argument is invalid; the library allocates nothing.
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "../../include/lsa.h"
#include "lsa_internal.h"

namespace lsa {
namespace {
std::atomic<long long> g_wait_budget{kDefaultWaitBudget};
std::atomic<int> g_inject{0};
}  // namespace
long long wait_budget() { return g_wait_budget.load(std::memory_order_relaxed); }
int debug_inject() { return g_inject.load(std::memory_order_relaxed); }
}  // namespace lsa

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return LSA_OK;
  g_last_cuda_error = (int)e;
  return LSA_ERR_CUDA;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int ceil_div(int a, int b) { return (a + b - 1) / b; }

float resolve_scale(float scale, int D) { return scale > 0.f ? scale : 1.0f / sqrtf((float)D); }

// Shape checks shared by the attention entry points.
int check_common(int dtype, int B, int Hkv, int G, int D, int blk) {
  if (B < 0 || Hkv < 0 || G < 1) return LSA_ERR_INVALID_ARG;
  if (dtype != LSA_F32 && dtype != LSA_BF16) return LSA_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return LSA_ERR_UNSUPPORTED;
  if (blk != 64) return LSA_ERR_UNSUPPORTED;
  if (G > 16) return LSA_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return LSA_ERR_UNSUPPORTED;  // (grid y and z of the launches)
  return LSA_OK;
}

constexpr int kMaxTcap = 1 << 21;  // 2M tokens: 32768 blocks per sequence

}  // namespace

extern "C" {

const char* lsa_status_string(int status) {
  switch (status) {
    case LSA_OK: return "LSA_OK";
    case LSA_ERR_INVALID_ARG: return "LSA_ERR_INVALID_ARG: an argument is out of range or a required pointer is NULL/misaligned";
    case LSA_ERR_UNSUPPORTED: return "LSA_ERR_UNSUPPORTED: dtype, head dim, block size or size not supported";
    case LSA_ERR_CUDA: return "LSA_ERR_CUDA: a kernel launch failed (see lsa_last_cuda_error)";
    case LSA_ERR_DEVICE_STATUS: return "LSA_ERR_DEVICE_STATUS: a kernel reported an error status";
    default: return "unknown lsa status";
  }
}

int lsa_last_cuda_error(void) { return g_last_cuda_error; }

int lsa_version(void) { return 100; }

int lsa_build_summaries(const void* k, int dtype, int B, int Hkv, int T_cap, int D,
                        const int32_t* seqlens, int blk, int nb_begin, int nb_end,
                        float* summ, cudaStream_t stream) {
  int st = check_common(dtype, B, Hkv, 1, D, blk);
  if (st != LSA_OK) return st;
  if (T_cap < 0 || T_cap > kMaxTcap) return T_cap < 0 ? LSA_ERR_INVALID_ARG : LSA_ERR_UNSUPPORTED;
  if (B == 0 || Hkv == 0 || T_cap == 0) return LSA_OK;
  if (!k || !seqlens || !summ) return LSA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(summ)) return LSA_ERR_INVALID_ARG;
  const int NB_cap = ceil_div(T_cap, blk);
  // the widest block range any sequence can have
  int range_max;
  if (nb_begin >= 0) {
    const int hi = nb_end >= 0 ? (nb_end < NB_cap ? nb_end : NB_cap) : NB_cap;
    range_max = hi - nb_begin;
  } else {
    range_max = -nb_begin < NB_cap ? -nb_begin : NB_cap;
  }
  if (range_max <= 0) return LSA_OK;
  return cuda_status(lsa::launch_build_summaries(k, dtype, B, Hkv, T_cap, D, seqlens, nb_begin,
                                                 nb_end, range_max, summ, stream));
}

int lsa_select_blocks(const void* q, int dtype, const float* summ, int B, int Hkv, int G,
                      int D, int NB_cap, const int32_t* seqlens, int blk, int topk,
                      int n_sink, int n_local, float scale, int32_t* idx, int32_t* nsel,
                      float* scores_out, cudaStream_t stream) {
  int st = check_common(dtype, B, Hkv, G, D, blk);
  if (st != LSA_OK) return st;
  if (topk < 1 || topk > 64 || n_sink < 0 || n_local < 0 || n_sink + n_local > topk)
    return LSA_ERR_INVALID_ARG;
  if (NB_cap < 0) return LSA_ERR_INVALID_ARG;
  if (NB_cap > kMaxTcap / 64) return LSA_ERR_UNSUPPORTED;
  if (B == 0 || Hkv == 0) return LSA_OK;
  if (!q || !summ || !seqlens || !idx || !nsel) return LSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(summ)) return LSA_ERR_INVALID_ARG;
  lsa::DecodeArgs a = {};
  a.q = q; a.dtype = dtype; a.summ = summ;
  a.B = B; a.Hkv = Hkv; a.G = G; a.D = D; a.T_cap = NB_cap * blk; a.NB_cap = NB_cap;
  a.seqlens = seqlens; a.topk = topk; a.n_sink = n_sink; a.n_local = n_local;
  a.scale = resolve_scale(scale, D);
  a.idx_out = idx; a.nsel_out = nsel; a.scores_out = scores_out;
  a.mode = lsa::MODE_SELECT;
  return cuda_status(lsa::launch_decode(a, stream));
}

int lsa_select_blocks_weighted(const void* q, int dtype, const float* summ,
                               const float* dim_weights, int B, int Hkv, int G, int D, int NB_cap,
                               const int32_t* seqlens, int blk, int topk, int n_sink,
                               int n_local, float scale, float* q_weighted, int32_t* idx,
                               int32_t* nsel, float* scores_out, cudaStream_t stream) {
  int st = check_common(dtype, B, Hkv, G, D, blk);
  if (st != LSA_OK) return st;
  if (topk < 1 || topk > 64 || n_sink < 0 || n_local < 0 || n_sink + n_local > topk)
    return LSA_ERR_INVALID_ARG;
  if (NB_cap < 0) return LSA_ERR_INVALID_ARG;
  if (NB_cap > kMaxTcap / 64) return LSA_ERR_UNSUPPORTED;
  if (B == 0 || Hkv == 0) return LSA_OK;
  if (!q || !summ || !dim_weights || !seqlens || !q_weighted || !idx || !nsel)
    return LSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(summ) || !aligned16(q_weighted)) return LSA_ERR_INVALID_ARG;
  // q_weighted may be q itself only for float32 q (the same element is read, then written, by
  // one thread); any other overlap would let a thread overwrite query elements that others
  // have not read yet
  {
    const size_t n = (size_t)B * Hkv * G * D;
    const uintptr_t w0 = (uintptr_t)q_weighted, q0 = (uintptr_t)q;
    const size_t wbytes = n * 4, qbytes = n * (dtype == LSA_F32 ? 4 : 2);
    const bool same = dtype == LSA_F32 && w0 == q0;
    if (!same && w0 < q0 + qbytes && q0 < w0 + wbytes) return LSA_ERR_INVALID_ARG;
    const uintptr_t d0 = (uintptr_t)dim_weights;
    if (w0 < d0 + (size_t)D * 4 && d0 < w0 + wbytes) return LSA_ERR_INVALID_ARG;
  }
  cudaError_t err = lsa::launch_weight_queries(q, dtype, dim_weights, B, Hkv * G, D, q_weighted, stream);
  if (err != cudaSuccess) return cuda_status(err);
  lsa::DecodeArgs a = {};
  a.q = q_weighted; a.dtype = LSA_F32; a.summ = summ;
  a.B = B; a.Hkv = Hkv; a.G = G; a.D = D; a.T_cap = NB_cap * blk; a.NB_cap = NB_cap;
  a.seqlens = seqlens; a.topk = topk; a.n_sink = n_sink; a.n_local = n_local;
  a.scale = resolve_scale(scale, D);
  a.idx_out = idx; a.nsel_out = nsel; a.scores_out = scores_out;
  a.mode = lsa::MODE_SELECT;
  return cuda_status(lsa::launch_decode(a, stream));
}

int lsa_sparse_attn_decode(const void* q, const void* k, const void* v, int dtype, int B,
                           int Hkv, int G, int D, int T_cap, const int32_t* seqlens,
                           int blk, const int32_t* idx, const int32_t* nsel, int topk,
                           float scale, float* summ, int n_sink, int n_local,
                           int refresh_last_summary, int32_t* idx_out, void* o, float* lse,
                           int flags, cudaStream_t stream) {
  int st = check_common(dtype, B, Hkv, G, D, blk);
  if (st != LSA_OK) return st;
  if (topk < 1 || topk > 64) return LSA_ERR_INVALID_ARG;
  if (T_cap < 0 || (flags & ~LSA_FLAG_PDL) != 0) return LSA_ERR_INVALID_ARG;
  if (T_cap > kMaxTcap) return LSA_ERR_UNSUPPORTED;
  if (B == 0 || Hkv == 0) return LSA_OK;
  if (!q || !k || !v || !seqlens || !o) return LSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LSA_ERR_INVALID_ARG;
  const bool fused = idx == nullptr;
  if (fused) {
    if (!summ || !aligned16(summ)) return LSA_ERR_INVALID_ARG;
    if (n_sink < 0 || n_local < 0 || n_sink + n_local > topk) return LSA_ERR_INVALID_ARG;
    // the refreshed block must be a forced one, so that no CTA scores it meanwhile
    if (refresh_last_summary && n_local < 1) return LSA_ERR_INVALID_ARG;
  } else if (!nsel || refresh_last_summary || (flags & LSA_FLAG_PDL)) {
    return LSA_ERR_INVALID_ARG;
  }
  lsa::DecodeArgs a = {};
  a.q = q; a.k = k; a.v = v; a.dtype = dtype;
  a.B = B; a.Hkv = Hkv; a.G = G; a.D = D; a.T_cap = T_cap; a.NB_cap = ceil_div(T_cap, blk);
  a.seqlens = seqlens; a.summ = summ; a.summ_w = refresh_last_summary ? summ : nullptr;
  a.idx_in = idx; a.nsel_in = nsel;
  a.topk = topk; a.n_sink = n_sink; a.n_local = n_local;
  a.scale = resolve_scale(scale, D);
  a.idx_out = fused ? idx_out : nullptr;
  a.o = o; a.lse = lse;
  a.mode = fused ? lsa::MODE_FUSED : lsa::MODE_ATTEND;
  a.pdl = (flags & LSA_FLAG_PDL) != 0;
  return cuda_status(lsa::launch_decode(a, stream));
}

int lsa_append_kv(const void* k_new, const void* v_new, int dtype, int B, int Hkv, int T_cap,
                  int D, const int32_t* seqlens, void* k, void* v, int flags, cudaStream_t stream) {
  return lsa_append_kv_stage_q(nullptr, nullptr, 0, k_new, v_new, dtype, B, Hkv, T_cap, D, seqlens, k, v,
                               flags, stream);
}

int lsa_append_kv_stage_q(const void* q_src, void* q_dst, size_t q_bytes, const void* k_new,
                          const void* v_new, int dtype, int B, int Hkv, int T_cap, int D,
                          const int32_t* seqlens, void* k, void* v, int flags, cudaStream_t stream) {
  int st = check_common(dtype, B, Hkv, 1, D, 64);
  if (st != LSA_OK) return st;
  if (T_cap < 0 || (flags & ~(LSA_FLAG_PDL | LSA_FLAG_INPUTS_READY)) != 0 || q_bytes % 16 != 0)
    return LSA_ERR_INVALID_ARG;
  if (T_cap > kMaxTcap || (long long)B * Hkv * D > (1 << 24) || q_bytes > ((size_t)1 << 28))
    return LSA_ERR_UNSUPPORTED;
  if (q_bytes > 0) {
    if (!q_src || !q_dst || !aligned16(q_src) || !aligned16(q_dst)) return LSA_ERR_INVALID_ARG;
    const char* s = static_cast<const char*>(q_src);
    const char* d = static_cast<const char*>(q_dst);
    if (s < d + q_bytes && d < s + q_bytes) return LSA_ERR_INVALID_ARG;  // overlapping ranges
  }
  const bool kv = B > 0 && Hkv > 0 && T_cap > 0;
  if (kv) {
    if (!k_new || !v_new || !seqlens || !k || !v) return LSA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k) || !aligned16(v)) return LSA_ERR_INVALID_ARG;
  }
  if (!kv && q_bytes == 0) return LSA_OK;
  return cuda_status(lsa::launch_kv_append(k_new, v_new, dtype == LSA_BF16 ? 2 : 4, kv ? B : 0, Hkv, T_cap, D,
                                           seqlens, k, v, (flags & LSA_FLAG_PDL) != 0, stream, q_src, q_dst,
                                           q_bytes, (flags & LSA_FLAG_INPUTS_READY) != 0));
}

int lsa_copy_async(void* dst, const void* src, size_t bytes, int flags, cudaStream_t stream) {
  if ((flags & ~(LSA_FLAG_PDL | LSA_FLAG_INPUTS_READY)) != 0 || bytes % 16 != 0) return LSA_ERR_INVALID_ARG;
  if (bytes == 0) return LSA_OK;
  if (!dst || !src || !aligned16(dst) || !aligned16(src)) return LSA_ERR_INVALID_ARG;
  const char* s = static_cast<const char*>(src);
  const char* d = static_cast<const char*>(dst);
  if (s < d + bytes && d < s + bytes) return LSA_ERR_INVALID_ARG;  // overlapping ranges
  return cuda_status(lsa::launch_copy16(dst, src, bytes, (flags & LSA_FLAG_PDL) != 0, stream,
                                        (flags & LSA_FLAG_INPUTS_READY) != 0));
}

int lsa_sparse_attn_decode_blasst(const void* q, const void* k, const void* v, int dtype, int B,
                                  int Hkv, int G, int D, int T_cap, const int32_t* seqlens,
                                  int blk, const int32_t* idx, const int32_t* nsel, int topk,
                                  float scale, float lambda, void* o, float* lse,
                                  uint32_t* skip_bits, cudaStream_t stream) {
  int st = check_common(dtype, B, Hkv, G, D, blk);
  if (st != LSA_OK) return st;
  if (dtype != LSA_BF16) return LSA_ERR_UNSUPPORTED;
  if (T_cap < 0 || topk < 1 || topk > 16 || !(lambda >= 0.f) || !(lambda < 1.f))
    return LSA_ERR_INVALID_ARG;
  if (T_cap > kMaxTcap || B > 65535 || Hkv > 65535) return LSA_ERR_UNSUPPORTED;
  if (B == 0 || Hkv == 0) return LSA_OK;
  if (!q || !k || !v || !seqlens || !idx || !nsel || !o) return LSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LSA_ERR_INVALID_ARG;
  lsa::DecodeBlasstArgs a = {};
  a.q = q; a.k = k; a.v = v;
  a.B = B; a.Hkv = Hkv; a.G = G; a.D = D; a.T_cap = T_cap;
  a.seqlens = seqlens; a.idx = idx; a.nsel = nsel; a.topk = topk;
  a.scale = resolve_scale(scale, D);
  a.lambda = lambda;
  a.o = o; a.lse = lse; a.skip_bits = skip_bits;
  return cuda_status(lsa::launch_decode_blasst(a, stream));
}

int lsa_nsa_compress(const void* k, const void* v, int dtype, int B, int Hkv, int T_cap, int D,
                     const int32_t* seqlens, int len, int stride, int nc_begin, int nc_end,
                     void* kc, void* vc, cudaStream_t stream) {
  int st = check_common(dtype, B, Hkv, 1, D, 64);
  if (st != LSA_OK) return st;
  if (dtype != LSA_BF16) return LSA_ERR_UNSUPPORTED;
  if (T_cap < 0 || len < 1 || stride < 1) return LSA_ERR_INVALID_ARG;
  if (T_cap > kMaxTcap || len > 4096 || B > 32767 || Hkv > 65535) return LSA_ERR_UNSUPPORTED;
  if (B == 0 || Hkv == 0 || T_cap == 0) return LSA_OK;
  if (!k || !v || !seqlens || !kc || !vc) return LSA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(kc) || !aligned16(vc)) return LSA_ERR_INVALID_ARG;
  const int NC_cap = ceil_div(T_cap, stride);
  int range_max;
  if (nc_begin >= 0) {
    const int hi = nc_end >= 0 ? (nc_end < NC_cap ? nc_end : NC_cap) : NC_cap;
    range_max = hi - nc_begin;
  } else {
    range_max = -nc_begin < NC_cap ? -nc_begin : NC_cap;
  }
  if (range_max <= 0) return LSA_OK;
  return cuda_status(lsa::launch_nsa_compress(k, v, B, Hkv, T_cap, D, seqlens, len, stride,
                                              nc_begin, nc_end, range_max, kc, vc, stream));
}

int lsa_nsa_branches(const void* q, const void* k, const void* v, const void* kc, const void* vc,
                     int dtype, int B, int Hkv, int G, int D, int T_cap, const int32_t* seqlens,
                     int window, int stride, float scale, float g_cmp, float g_slc, float g_win,
                     const void* o_slc, void* o, float* lse_win, float* lse_cmp,
                     cudaStream_t stream) {
  int st = check_common(dtype, B, Hkv, G, D, 64);
  if (st != LSA_OK) return st;
  if (dtype != LSA_BF16) return LSA_ERR_UNSUPPORTED;
  if (T_cap < 0 || window < 0 || stride < 1) return LSA_ERR_INVALID_ARG;
  if (!(g_cmp == g_cmp) || !(g_slc == g_slc) || !(g_win == g_win)) return LSA_ERR_INVALID_ARG;
  if (T_cap > kMaxTcap || B > 65535 || Hkv > 65535) return LSA_ERR_UNSUPPORTED;
  if (B == 0 || Hkv == 0) return LSA_OK;
  if (!q || !k || !v || !kc || !vc || !seqlens || !o) return LSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kc) || !aligned16(vc) ||
      !aligned16(o))
    return LSA_ERR_INVALID_ARG;
  lsa::NsaBranchArgs a = {};
  a.q = q; a.k = k; a.v = v; a.kc = kc; a.vc = vc;
  a.B = B; a.Hkv = Hkv; a.G = G; a.D = D; a.T_cap = T_cap;
  a.seqlens = seqlens; a.window = window; a.stride = stride;
  a.scale = resolve_scale(scale, D);
  a.g_cmp = g_cmp; a.g_slc = g_slc; a.g_win = g_win;
  a.o_slc = o_slc; a.o = o; a.lse_win = lse_win; a.lse_cmp = lse_cmp;
  return cuda_status(lsa::launch_nsa_branches(a, stream));
}

size_t lsa_blockquery_workspace_size(int B, int Hkv, int G, int D, int Tq) {
  if (B <= 0 || Hkv <= 0 || G <= 0 || D <= 0 || Tq <= 0) return 0;
  return lsa::blockquery_workspace_bytes(B, Hkv, G, D, Tq);
}

int lsa_sparse_attn_blockquery(const void* q, const void* k, const void* v, int dtype,
                               int B, int Hkv, int G, int D, int Tq, int T_prefix,
                               int T_cap, const float* summ, int blk, int topk_per_query,
                               int n_sink, int n_local, float scale, const uint8_t* active,
                               const void* o_cache, const float* lse_cache, void* o,
                               float* lse, int32_t* union_idx, int32_t* union_cnt,
                               void* workspace, size_t ws_bytes, cudaStream_t stream) {
  int st = check_common(dtype, B, Hkv, G, D, blk);
  if (st != LSA_OK) return st;
  if (dtype != LSA_BF16) return LSA_ERR_UNSUPPORTED;
  if (Tq < 1 || Tq > 64 || T_prefix < 0 || T_cap < T_prefix) return LSA_ERR_INVALID_ARG;
  if (T_cap > kMaxTcap) return LSA_ERR_UNSUPPORTED;
  // topk_per_query <= 16 selects; topk_per_query >= ceil(T_prefix / blk) takes every prefix
  // block (the dense first step of a block)
  if (topk_per_query < 1 || (topk_per_query > 16 && topk_per_query < ceil_div(T_prefix, blk)) ||
      n_sink < 0 || n_local < 0 || n_sink + n_local > topk_per_query)
    return LSA_ERR_INVALID_ARG;
  if (B == 0 || Hkv == 0) return LSA_OK;
  if (!q || !k || !v || !summ || !active || !o_cache || !lse_cache || !o || !lse || !workspace)
    return LSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(summ) || !aligned16(o) ||
      !aligned16(o_cache) || !aligned16(workspace))
    return LSA_ERR_INVALID_ARG;
  if (ws_bytes < lsa::blockquery_workspace_bytes(B, Hkv, G, D, Tq)) return LSA_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535) return LSA_ERR_UNSUPPORTED;  // (grid y, z)
  // o may be o_cache and lse may be lse_cache (stable rows are then left as they are); a
  // partial overlap would let the copy of one stable row overwrite another's cached value
  {
    const size_t obytes = (size_t)B * Hkv * G * Tq * D * 2, lbytes = (size_t)B * Hkv * G * Tq * 4;
    const uintptr_t o0 = (uintptr_t)o, c0 = (uintptr_t)o_cache, l0 = (uintptr_t)lse,
                    lc0 = (uintptr_t)lse_cache;
    if (o0 != c0 && o0 < c0 + obytes && c0 < o0 + obytes) return LSA_ERR_INVALID_ARG;
    if (l0 != lc0 && l0 < lc0 + lbytes && lc0 < l0 + lbytes) return LSA_ERR_INVALID_ARG;
  }
  lsa::BlockQueryArgs a = {};
  a.q = q; a.k = k; a.v = v;
  a.B = B; a.Hkv = Hkv; a.G = G; a.D = D; a.Tq = Tq; a.T_prefix = T_prefix; a.T_cap = T_cap;
  a.summ = summ; a.topk = topk_per_query; a.n_sink = n_sink; a.n_local = n_local;
  a.scale = resolve_scale(scale, D);
  a.active = active; a.o_cache = o_cache; a.lse_cache = lse_cache; a.o = o; a.lse = lse;
  a.union_idx = union_idx; a.union_cnt = union_cnt; a.workspace = workspace;
  return cuda_status(lsa::launch_blockquery(a, stream));
}

int lsa_sparse_attn_blockquery_noalloc(const void* q, const void* k, const void* v, int dtype,
                                       int B, int Hkv, int G, int D, int Tq, int T_prefix,
                                       int T_cap, const float* summ, int blk,
                                       int topk_per_query, int n_sink, int n_local,
                                       float scale, const uint8_t* active,
                                       const void* o_cache, const float* lse_cache, void* o,
                                       float* lse, int32_t* union_idx, int32_t* union_cnt,
                                       cudaStream_t stream) {
  if (B > 0 && Hkv > 0 && G > 0 && D > 0 && Tq > 0 &&
      lsa::blockquery_workspace_bytes(B, Hkv, G, D, Tq) > lsa::blockquery_static_workspace_bytes())
    return LSA_ERR_UNSUPPORTED;  // larger than the fixed scratch: use the workspace variant
  void* ws = nullptr;
  const cudaError_t err = lsa::blockquery_static_workspace(&ws);
  if (err != cudaSuccess) return cuda_status(err);
  return lsa_sparse_attn_blockquery(q, k, v, dtype, B, Hkv, G, D, Tq, T_prefix, T_cap, summ,
                                    blk, topk_per_query, n_sink, n_local, scale, active,
                                    o_cache, lse_cache, o, lse, union_idx, union_cnt, ws,
                                    lsa::blockquery_static_workspace_bytes(), stream);
}

int lsa_losa_classify(const void* q, const void* q_prev, int dtype, int B, int Hq, int Tq, int D,
                      double tau, int n_top, uint8_t* active, double* mse, cudaStream_t stream) {
  if (B < 0 || Hq < 1 || Tq < 1 || n_top < 0) return LSA_ERR_INVALID_ARG;
  if (dtype != LSA_BF16 || (D != 64 && D != 128)) return LSA_ERR_UNSUPPORTED;
  if (Tq > 64 || B > 65535 || !(tau == tau)) return Tq > 64 || B > 65535 ? LSA_ERR_UNSUPPORTED
                                                                         : LSA_ERR_INVALID_ARG;
  if (B == 0) return LSA_OK;
  if (!q || !q_prev || !active) return LSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(q_prev) || (mse && ((uintptr_t)mse & 7u) != 0))
    return LSA_ERR_INVALID_ARG;
  return cuda_status(lsa::launch_losa_classify(q, q_prev, B, Hq, Tq, D, tau, n_top, active, mse,
                                               stream));
}

int lsa_blockquery_intra_merge(const void* q, const void* k, const void* v, int dtype, int B,
                               int Hkv, int G, int D, int Tq, int T_prefix, int T_cap,
                               float scale, const void* o_pre, const float* lse_pre, void* o,
                               float* lse, int flags, cudaStream_t stream) {
  int st = check_common(dtype, B, Hkv, G, D, 64);
  if (st != LSA_OK) return st;
  if (dtype != LSA_BF16) return LSA_ERR_UNSUPPORTED;
  if (Tq < 1 || Tq > 64 || T_prefix < 0 || T_cap < T_prefix + Tq) return LSA_ERR_INVALID_ARG;
  if (T_cap > kMaxTcap || B > 65535 || (long long)Hkv * G > 65535) return LSA_ERR_UNSUPPORTED;
  if ((flags & ~LSA_FLAG_PDL) != 0) return LSA_ERR_INVALID_ARG;
  if (B == 0 || Hkv == 0) return LSA_OK;
  if (!q || !k || !v || !o_pre || !lse_pre || !o || !lse) return LSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_pre) || !aligned16(o))
    return LSA_ERR_INVALID_ARG;
  // o may be o_pre and lse may be lse_pre; a partial overlap is rejected
  const size_t obytes = (size_t)B * Hkv * G * Tq * D * 2, lbytes = (size_t)B * Hkv * G * Tq * 4;
  const uintptr_t o0 = (uintptr_t)o, p0 = (uintptr_t)o_pre, l0 = (uintptr_t)lse, lp0 = (uintptr_t)lse_pre;
  if (o0 != p0 && o0 < p0 + obytes && p0 < o0 + obytes) return LSA_ERR_INVALID_ARG;
  if (l0 != lp0 && l0 < lp0 + lbytes && lp0 < l0 + lbytes) return LSA_ERR_INVALID_ARG;
  lsa::IntraMergeArgs a = {};
  a.q = q; a.k = k; a.v = v;
  a.B = B; a.Hkv = Hkv; a.G = G; a.D = D; a.Tq = Tq; a.T_prefix = T_prefix; a.T_cap = T_cap;
  a.scale = resolve_scale(scale, D);
  a.o_pre = o_pre; a.lse_pre = lse_pre; a.o = o; a.lse = lse;
  a.pdl = (flags & LSA_FLAG_PDL) != 0;
  return cuda_status(lsa::launch_intra_merge(a, stream));
}

int lsa_blasst_prefill(const void* q, const void* k, const void* v, int dtype, int B, int Hq,
                       int Hkv, int L, int D, float scale, float lambda, void* o, float* lse,
                       uint32_t* skip_bits, unsigned long long* skipped_tiles,
                       cudaStream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || L < 0) return LSA_ERR_INVALID_ARG;
  if (dtype != LSA_BF16 || D != 128) return LSA_ERR_UNSUPPORTED;
  if (Hq % Hkv != 0 || !(lambda >= 0.f) || !(lambda < 1.f)) return LSA_ERR_INVALID_ARG;
  if (L > kMaxTcap || (long long)B * Hq > 65535LL * 65535LL) return LSA_ERR_UNSUPPORTED;
  if (B == 0 || L == 0) return LSA_OK;
  if (!q || !k || !v || !o) return LSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LSA_ERR_INVALID_ARG;
  if ((long long)B * Hq > 65535) return LSA_ERR_UNSUPPORTED;
  lsa::PrefillArgs a = {};
  a.q = q; a.k = k; a.v = v;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.L = L;
  a.scale = resolve_scale(scale, D);
  a.lambda = lambda;
  a.o = o; a.lse = lse; a.skip_bits = skip_bits; a.skipped_tiles = skipped_tiles;
  return cuda_status(lsa::launch_blasst_prefill(a, stream));
}

int lsa_debug_set_wait_budget(long long cycles) {
  lsa::g_wait_budget.store(cycles > 0 ? cycles : lsa::kDefaultWaitBudget, std::memory_order_relaxed);
  return LSA_OK;
}

int lsa_debug_inject(int kind) {
  if (kind != 0 && kind != LSA_DEBUG_PREFILL_DROP_S) return LSA_ERR_INVALID_ARG;
  lsa::g_inject.store(kind, std::memory_order_relaxed);
  return LSA_OK;
}

#ifdef LSA_DEBUG_BOUNDS
// The first recorded bounds violation over the translation units (0 if none).
static int bounds_code(bool reset, cudaError_t* err) {
  cudaError_t (*readers[])(int*, bool) = {lsa::read_bounds_summaries, lsa::read_bounds_decode,
                                          lsa::read_bounds_decode_blasst, lsa::read_bounds_nsa,
                                          lsa::read_bounds_kv_append};
  int first = 0;
  *err = cudaSuccess;
  for (auto rd : readers) {
    int w = 0;
    const cudaError_t e = rd(&w, reset);
    if (e != cudaSuccess) {
      *err = e;
      return 0;
    }
    if (first == 0) first = w;
  }
  return first;
}
#endif

int lsa_debug_bounds_code(int* code, int reset) {
  if (!code) return LSA_ERR_INVALID_ARG;
#ifdef LSA_DEBUG_BOUNDS
  cudaError_t err;
  *code = bounds_code(reset != 0, &err);
  return cuda_status(err);
#else
  (void)reset;
  *code = 0;
  return LSA_ERR_UNSUPPORTED;
#endif
}

int lsa_device_status(int* status, int reset) {
  if (!status) return LSA_ERR_INVALID_ARG;
  int prefill = 0, decode = 0;
  int st = cuda_status(lsa::read_device_status(&prefill, reset != 0));
  if (st != LSA_OK) return st;
  st = cuda_status(lsa::read_decode_status(&decode, reset != 0));
  if (st != LSA_OK) return st;
  int bq = 0;
  st = cuda_status(lsa::read_blockquery_status(&bq, reset != 0));
  if (st != LSA_OK) return st;
  int dbl = 0;
  st = cuda_status(lsa::read_decode_blasst_status(&dbl, reset != 0));
  if (st != LSA_OK) return st;
  int bounds = 0;
#ifdef LSA_DEBUG_BOUNDS
  {
    cudaError_t err;
    bounds = bounds_code(reset != 0, &err) != 0 ? LSA_DEVICE_BOUNDS : 0;
    if (err != cudaSuccess) return cuda_status(err);
  }
#endif
  *status = prefill | decode | bq | dbl | bounds;
  return LSA_OK;
}

}  // extern "C"
