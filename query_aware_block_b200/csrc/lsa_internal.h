// lsa_internal.h -- launchers behind the C ABI (host side, not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lsa {

enum { DT_F32 = 0, DT_BF16 = 1 };

cudaError_t launch_build_summaries(const void* k, int dtype, int B, int Hkv, int T_cap, int D,
                                   const int32_t* seqlens, int nb_begin, int nb_end,
                                   int range_max, float* summ, cudaStream_t stream);

// The decode family: one thread-block cluster per (sequence, KV head).
enum DecodeMode { MODE_SELECT = 0, MODE_ATTEND = 1, MODE_FUSED = 2 };

struct DecodeArgs {
  const void* q;
  const void* k;
  const void* v;
  int dtype;
  int B, Hkv, G, D, T_cap;
  const int32_t* seqlens;
  const float* summ;
  float* summ_w;           // MODE_FUSED: refresh the last block's summary here, or NULL
  int NB_cap;
  const int32_t* idx_in;   // MODE_ATTEND
  const int32_t* nsel_in;  // MODE_ATTEND
  int topk, n_sink, n_local;
  float scale;
  int32_t* idx_out;        // MODE_SELECT / MODE_FUSED (may be NULL in fused mode)
  int32_t* nsel_out;       // MODE_SELECT
  float* scores_out;       // MODE_SELECT, optional
  void* o;                 // MODE_ATTEND / MODE_FUSED
  float* lse;              // optional
  int mode;
  int pdl;                 // MODE_FUSED: launch with programmatic stream serialization
};

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

// The block-query step: one cluster per (sequence, KV head); partials in a workspace.
struct BlockQueryArgs {
  const void* q;
  const void* k;
  const void* v;
  int B, Hkv, G, D, Tq, T_prefix, T_cap;
  const float* summ;
  int topk, n_sink, n_local;
  float scale;
  const uint8_t* active;
  const void* o_cache;
  const float* lse_cache;
  void* o;
  float* lse;
  int32_t* union_idx;
  int32_t* union_cnt;
  void* workspace;
};

size_t blockquery_workspace_bytes(int B, int Hkv, int G, int D, int Tq);
cudaError_t launch_blockquery(const BlockQueryArgs& a, cudaStream_t stream);

// Queries reweighted per head dimension (fp32 out) for the weighted block selection.
cudaError_t launch_weight_queries(const void* q, int dtype, const float* w, int B, int Hq, int D,
                                  float* out, cudaStream_t stream);

// Sparse decode over a given selection with BLASST's skip (V not read for negligible blocks).
struct DecodeBlasstArgs {
  const void* q;
  const void* k;
  const void* v;
  int B, Hkv, G, D, T_cap;
  const int32_t* seqlens;
  const int32_t* idx;
  const int32_t* nsel;
  int topk;
  float scale, lambda;
  void* o;
  float* lse;
  uint32_t* skip_bits;
};
cudaError_t launch_decode_blasst(const DecodeBlasstArgs& a, cudaStream_t stream);
cudaError_t read_decode_blasst_status(int* status, bool reset);

// NSA's compressed and sliding-window branches (fixed pool, constant gates).
cudaError_t launch_nsa_compress(const void* k, const void* v, int B, int Hkv, int T_cap, int D,
                                const int32_t* seqlens, int len, int stride, int nc_begin,
                                int nc_end, int range_max, void* kc, void* vc, cudaStream_t stream);
struct NsaBranchArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* kc;
  const void* vc;
  int B, Hkv, G, D, T_cap;
  const int32_t* seqlens;
  int window, stride;
  float scale, g_cmp, g_slc, g_win;
  const void* o_slc;
  void* o;
  float* lse_win;
  float* lse_cmp;
};
cudaError_t launch_nsa_branches(const NsaBranchArgs& a, cudaStream_t stream);

// LoSA: token activity and the attention inside the query block merged with the prefix.
cudaError_t launch_losa_classify(const void* q, const void* q_prev, int B, int Hq, int Tq, int D,
                                 double tau, int n_top, uint8_t* active, double* mse,
                                 cudaStream_t stream);
struct IntraMergeArgs {
  const void* q;
  const void* k;
  const void* v;
  int B, Hkv, G, D, Tq, T_prefix, T_cap;
  float scale;
  const void* o_pre;
  const float* lse_pre;
  void* o;
  float* lse;
  int pdl;
};
cudaError_t launch_intra_merge(const IntraMergeArgs& a, cudaStream_t stream);

// BLASST causal prefill on tcgen05.
struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  int B, Hq, Hkv, L;
  float scale, lambda;
  void* o;
  float* lse;
  uint32_t* skip_bits;
  unsigned long long* skipped_tiles;
};
cudaError_t launch_blasst_prefill(const PrefillArgs& a, cudaStream_t stream);
cudaError_t read_device_status(int* status, bool reset);
cudaError_t read_decode_status(int* status, bool reset);
cudaError_t read_blockquery_status(int* status, bool reset);

// 3-D TMA map over a row-major bf16 tensor [planes][rows][D]: box {64, box_rows, 1} (one
// 128-byte swizzled row segment per box row), rows past `rows` read as zero.  False when
// the driver entry point is missing or rejects the map.
bool encode_rows_bf16(CUtensorMap* map, const void* base, int D, int rows, int planes, int box_rows);
// Maps of a bf16 K/V cache pair [planes][T_cap][D] with 64-row boxes, cached per host
// thread for the last (k, v, D, T_cap, planes).
bool kv_tensor_maps(const void* k, const void* v, int D, int T_cap, int planes, CUtensorMap* mk,
                    CUtensorMap* mv);

// The new token's key and value rows into the cache at row seqlens[b] - 1.
cudaError_t launch_copy16(void* dst, const void* src, size_t bytes, int pdl, cudaStream_t stream,
                          int inputs_ready = 0);
cudaError_t launch_kv_append(const void* k_new, const void* v_new, int elem_bytes, int B, int Hkv,
                             int T_cap, int D, const int32_t* seqlens, void* k, void* v, int pdl,
                             cudaStream_t stream,
                             const void* q_src = nullptr, void* q_dst = nullptr, size_t q_bytes = 0,
                             int inputs_ready = 0);

// The debug bounds-check status word of each translation unit (always 0 in the release
// build, which compiles no checks).
cudaError_t read_bounds_summaries(int* word, bool reset);
cudaError_t read_bounds_decode(int* word, bool reset);
cudaError_t read_bounds_decode_blasst(int* word, bool reset);
cudaError_t read_bounds_nsa(int* word, bool reset);
cudaError_t read_bounds_kv_append(int* word, bool reset);

// Bounded waits: the clock-cycle limit of the first wait (settable for tests) and of the
// drain that follows a timeout; the fault injected for tests (0 = none).
constexpr long long kDefaultWaitBudget = 4000000000LL;  // about 2 s of clock
constexpr long long kDrainBudget = 4000000000LL;
long long wait_budget();
int debug_inject();

// Unique id of the context current on this host thread (false when none is current or the
// driver lacks the entry points).
bool current_context_id(unsigned long long* id);

// The fixed device scratch used by lsa_sparse_attn_blockquery_noalloc.
size_t blockquery_static_workspace_bytes();
cudaError_t blockquery_static_workspace(void** ptr);

}  // namespace lsa
