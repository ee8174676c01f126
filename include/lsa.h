/*
 * lsa.h -- C ABI of liblsa.so: query-aware block-sparse softmax attention over a long KV
 * cache, for NVIDIA B200 (sm_100a).
 *
 * The hot path: per-block key summaries -> block scoring shared by a GQA group and top-n
 * selection with forced initial/local blocks (or, for a block of queries, the union of
 * the tokens' selections) -> online-softmax attention over only the selected KV blocks;
 * plus a causal prefill that skips whole KV tiles by a softmax threshold (BLASST).
 *
 * One LoSA denoising step of a block of Tq query tokens is three calls on one stream:
 *   lsa_losa_classify           (queries now vs the previous step -> active mask)
 *   lsa_sparse_attn_blockquery  (prefix part: active tokens select and attend, stable
 *                                tokens keep it; o_cache/lse_cache = o/lse = the prefix
 *                                cache, updated in place)
 *   lsa_blockquery_intra_merge  (the block's own tokens, merged with the prefix cache into
 *                                the step's output)
 * The first step of a block passes topk_per_query >= ceil(T_prefix / blk) and an all-ones
 * mask (dense prefix attention, which fills the cache).
 *
 * One decode step with the host on both ends (inputs in, outputs out through pinned host
 * memory) is two calls on one stream, the second a programmatic dependent of the first:
 *   lsa_append_kv_stage_q       (q to the device and k_new, v_new into the cache, all read
 *                                from pinned host memory)
 *   lsa_sparse_attn_decode      (o, lse, idx_out written straight into pinned host memory)
 *
 * One NSA decode step with fixed parts is three calls on one stream:
 *   lsa_sparse_attn_decode      (the selected branch, fused selection)
 *   lsa_nsa_compress            (nc_begin = -2: the compressed tokens the new token changes)
 *   lsa_nsa_branches            (compressed and window branches, gated sum with the above)
 * Variants: lsa_select_blocks_weighted scores with a weight per head dimension (FASA /
 * Prism-style scorers); lsa_sparse_attn_decode_blasst drops, before reading their V, the
 * selected blocks whose softmax weight is negligible (BLASST inside sparse decode).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every tensor argument is a raw DEVICE pointer to a contiguous row-major array
 *           in the stated layout, aligned to 16 bytes (except where a call states that
 *           pinned host memory is accepted: lsa_copy_async, q_src / q_dst / k_new / v_new
 *           of lsa_append_kv and lsa_append_kv_stage_q, o / lse / idx_out of
 *           lsa_sparse_attn_decode).  The caller owns all memory; the library allocates
 *           nothing, keeps no per-call state and never frees.
 * Streams.  All work is enqueued on `stream` (a cudaStream_t; 0 = legacy default
 *           stream).  Calls return as soon as the work is enqueued; nothing synchronises
 *           the host.  Calls are thread-safe.
 * Shapes.   B = batch, Hkv = KV heads, G = query heads per KV head (query head h belongs
 *           to KV group h / G), Hq = Hkv * G, D = head dim, blk = KV block size.
 *           KV cache k, v: [B, Hkv, T_cap, D].  seqlens[b] = valid tokens of sequence b
 *           (0 <= seqlens[b] <= T_cap), a device int32 array.  A sequence has
 *           NB_b = ceil(seqlens[b] / blk) blocks; NB_cap = ceil(T_cap / blk).
 *           Summaries summ: [B, Hkv, NB_cap, D] float32.
 * Types.    dtype = LSA_F32 or LSA_BF16 for q, k, v and o.  lse, summaries and scores are
 *           always float32; indices int32.
 * Support.  D in {64, 128}; blk == 64; G <= 16; B and Hkv <= 65535 (grid dimensions).
 *           bf16 everywhere; fp32 in summaries, selection and decode.  Anything else
 *           returns LSA_ERR_UNSUPPORTED.
 * Scale.    scale <= 0 means 1/sqrt(D).
 * Errors.   Every argument is validated on the host before anything is launched; on
 *           error nothing is enqueued and the status is returned.  LSA_ERR_CUDA means a
 *           launch failed; lsa_last_cuda_error() returns that cudaError_t for the
 *           calling thread.  Device-side values (seqlens, idx) are trusted: they must obey
 *           the documented ranges.  Waits between the CTAs of one launch are bounded in
 *           time (about 2 s); should one ever run out, the launch's outputs are undefined
 *           and lsa_device_status() reports LSA_DEVICE_TIMEOUT.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LSA_API __attribute__((visibility("default")))
#else
#define LSA_API
#endif

#define LSA_OK 0
#define LSA_ERR_INVALID_ARG 1
#define LSA_ERR_UNSUPPORTED 2
#define LSA_ERR_CUDA 3
#define LSA_ERR_DEVICE_STATUS 4

#define LSA_F32 0
#define LSA_BF16 1

/* lsa_sparse_attn_decode / lsa_blockquery_intra_merge / lsa_append_kv / lsa_append_kv_stage_q /
 * lsa_copy_async flags */
#define LSA_FLAG_PDL 1
/* lsa_append_kv / lsa_append_kv_stage_q / lsa_copy_async, with LSA_FLAG_PDL: the call's
 * inputs (q_src, k_new, v_new, seqlens; src) are complete when the call is enqueued (written
 * by the host, say), so they are read at once; only the writes wait for the previous
 * kernel. */
#define LSA_FLAG_INPUTS_READY 2

/* Human-readable name of a status code (static storage). */
LSA_API const char* lsa_status_string(int status);

/* cudaError_t of the last failed launch on the calling thread (0 if none). */
LSA_API int lsa_last_cuda_error(void);

/* Library version: major * 10000 + minor * 100 + patch. */
LSA_API int lsa_version(void);

/*
 * lsa_build_summaries -- mean-pooled key summary of each KV block.
 *
 * Defined by: Prism, "1. 문제 정의" (training-free block importance uses mean pooling of
 * the keys of a block) and "2. 핵심 이론적 발견" (mean pooling acts as a low-pass filter).
 *
 *   summ[b, g, j, :] = (1 / n_j) * sum_{t = j*blk}^{min(j*blk + blk, seqlens[b]) - 1} k[b, g, t, :]
 *
 * with n_j the number of valid tokens of block j (a partial last block is averaged over
 * its valid tokens only).  Accumulation is float32.
 *
 * k        [B, Hkv, T_cap, D] (dtype), read only.
 * summ     [B, Hkv, NB_cap, D] float32, written for the blocks in range only.
 * nb_begin, nb_end: block range per sequence, clipped to [0, NB_b).  nb_begin < 0 means
 *          NB_b + nb_begin (the last -nb_begin blocks); nb_end < 0 means NB_b.  (0, -1)
 *          rebuilds every block; (-1, -1) refreshes only the last block after a token
 *          was appended.  Blocks outside the range are not touched.
 */
LSA_API int lsa_build_summaries(const void* k, int dtype, int B, int Hkv, int T_cap, int D,
                        const int32_t* seqlens, int blk, int nb_begin, int nb_end,
                        float* summ, cudaStream_t stream);

/*
 * lsa_select_blocks -- query-aware block scores and top-n selection, one selection per
 * KV head shared by its G query heads.
 *
 * Defined by: NSA news article, "NSA 구조" (selection blocks of l' = 64 tokens; n = 16
 * blocks selected, the initial block and 2 local blocks included) and "기존 스파스 어텐션
 * 접근법의 한계 분석" / "기술 구현의 실제적 도전과 해결" (query-aware chunk scoring;
 * GQA-compatible selection decides memory-access efficiency).
 *
 *   score[b, g, j] = scale * sum_{h in group g} q[b, h, :] . summ[b, g, j, :]    (j < NB_b)
 *   F = {0 .. n_sink-1} U {NB_b - n_local .. NB_b - 1}  (clipped, deduplicated)
 *   selected = F U (the topk - |F| highest-scoring blocks outside F; ties -> lower j)
 *   if NB_b <= topk, every block is selected.
 *
 * q          [B, Hq, D] (dtype).  summ [B, Hkv, NB_cap, D] float32.
 * idx        [B, Hkv, topk] int32 out: selected block indices ascending, padded with -1.
 * nsel       [B, Hkv] int32 out: number of selected blocks (min(topk, NB_b)).
 * scores_out [B, Hkv, NB_cap] float32 out, or NULL: the block scores, written only for
 *            sequences with NB_b > topk and only for j < NB_b (other entries untouched).
 * Requires 1 <= topk <= 64, n_sink >= 0, n_local >= 0, n_sink + n_local <= topk.
 */
LSA_API int lsa_select_blocks(const void* q, int dtype, const float* summ, int B, int Hkv, int G,
                      int D, int NB_cap, const int32_t* seqlens, int blk, int topk,
                      int n_sink, int n_local, float scale, int32_t* idx, int32_t* nsel,
                      float* scores_out, cudaStream_t stream);

/*
 * lsa_sparse_attn_decode -- softmax attention of one query token per head over only the
 * tokens of the selected KV blocks (original positions kept), split over the selected
 * blocks with a log-sum-exp merge.
 *
 * Defined by: NSA news article, "NSA 구조" and "처리 속도" (decoding touches only the
 * selected blocks' tokens); FASA, "2. 방법론", Focused Attention Computation (exact
 * full-dimension attention over the selected tokens, positions preserved).
 *
 *   tokens(b, g) = { t : floor(t / blk) in selected(b, g), t < seqlens[b] }
 *   o[b, h, :]   = sum_t softmax_t(scale * q[b,h,:] . k[b,g,t,:]) v[b,g,t,:]
 *   lse[b, h]    = log sum_t exp(scale * q[b,h,:] . k[b,g,t,:])        (g = h / G)
 * An empty token set gives o = 0 and lse = -inf.
 *
 * Two modes:
 *   given selection (idx != NULL): idx [B, Hkv, topk] and nsel [B, Hkv] as written by
 *       lsa_select_blocks (entries in [0, NB_b), the first nsel valid; -1 ignored).
 *   fused selection (idx == NULL): selection as in lsa_select_blocks is computed inside
 *       the same launch from summ (required) with n_sink / n_local; the selected indices
 *       are written to idx_out [B, Hkv, topk] (ascending, -1 padded) when it is non-NULL.
 *       With refresh_last_summary != 0 (requires n_local >= 1) the launch also rewrites
 *       summ[b, g, NB_b - 1, :] as the mean of that block's valid keys, i.e. the summary
 *       update a decode step owes after appending a token, from the keys it loads anyway.
 * q [B, Hq, D]; k, v [B, Hkv, T_cap, D]; o [B, Hq, D] (dtype); lse [B, Hq] float32 or NULL.
 * o, lse and idx_out may be pinned host memory (written with plain stores, over PCIe).
 * summ [B, Hkv, NB_cap, D] float32 (fused mode; written only by the refresh).
 * K/V rows at or beyond seqlens[b] are never used (they may hold any bits, NaN included).
 * refresh_last_summary must be 0 in given-selection mode.
 * flags: 0, or LSA_FLAG_PDL (fused mode only): launch with programmatic dependent launch,
 *     so the kernel may start while the previous kernel of the stream still runs.  It then
 *     reads seqlens, the summaries and the K/V of the forced blocks other than each
 *     sequence's last block BEFORE that kernel completes; q and the last block's K/V are
 *     read after it.  The caller guarantees the previous kernel writes none of the former
 *     (true for a decode loop, where the previous kernel produces q and appends the newest
 *     token; the summary a previous decode step refreshed is forced when n_local >= 2).
 */
LSA_API int lsa_sparse_attn_decode(const void* q, const void* k, const void* v, int dtype, int B,
                           int Hkv, int G, int D, int T_cap, const int32_t* seqlens,
                           int blk, const int32_t* idx, const int32_t* nsel, int topk,
                           float scale, float* summ, int n_sink, int n_local,
                           int refresh_last_summary, int32_t* idx_out, void* o, float* lse,
                           int flags, cudaStream_t stream);

/*
 * lsa_append_kv -- writes the newest token's key and value into the KV cache, the first
 * part of a decode step (the cache keeps every token; NSA news article, "NSA 구조": the
 * selected, compressed and window branches all read the cache).
 *
 *   k[b, g, seqlens[b] - 1, :] = k_new[b, g, :]     v[b, g, seqlens[b] - 1, :] = v_new[b, g, :]
 * seqlens[b] already counts the new token; a sequence with seqlens[b] == 0 is left alone.
 * k_new, v_new [B, Hkv, D] (dtype; device or pinned host memory, read with plain loads);
 * k, v [B, Hkv, T_cap, D] (dtype), written in place.
 * flags: 0, or LSA_FLAG_PDL: launched as a programmatic dependent of the previous kernel of
 *     the stream; it reads k_new, v_new and seqlens only after that kernel completes, and
 *     lets the next kernel start at once (a decode call with LSA_FLAG_PDL then overlaps its
 *     prologue with this copy; it reads the newest block only after this call completes).
 *     LSA_FLAG_PDL | LSA_FLAG_INPUTS_READY: the inputs are read at once (they do not depend
 *     on the previous kernel), and only the writes into the cache wait for it.
 * Support: D in {64, 128}; B * Hkv * D <= 2^24.
 */
LSA_API int lsa_append_kv(const void* k_new, const void* v_new, int dtype, int B, int Hkv,
                          int T_cap, int D, const int32_t* seqlens, void* k, void* v, int flags,
                          cudaStream_t stream);

/*
 * lsa_append_kv_stage_q -- lsa_append_kv, and in the same launch the step's query rows:
 * q_bytes (a multiple of 16) copied from q_src to q_dst with 16-byte loads and stores.  With
 * q_src, k_new and v_new in pinned host memory, the inputs of a decode step reach the device
 * in one launch, their PCIe round trips overlapping.  Arguments and flags as lsa_append_kv;
 * q_src, q_dst 16-byte aligned and not overlapping (either may be pinned host memory);
 * q_bytes == 0 appends only.  Support: q_bytes <= 2^28.
 */
LSA_API int lsa_append_kv_stage_q(const void* q_src, void* q_dst, size_t q_bytes, const void* k_new,
                                  const void* v_new, int dtype, int B, int Hkv, int T_cap, int D,
                                  const int32_t* seqlens, void* k, void* v, int flags,
                                  cudaStream_t stream);

/*
 * lsa_copy_async -- copies `bytes` from src to dst with a kernel (16-byte loads and stores),
 * enqueued on `stream`.  Either side may be pinned host memory (cudaHostAlloc / a pinned
 * tensor: under unified addressing its pointer is valid in kernels, and the kernel's loads or
 * stores cross PCIe), which moves a decode step's small inputs to the device without a
 * copy-engine round trip.  The other library calls accept pinned host memory in the same
 * way for k_new / v_new of lsa_append_kv and for the outputs o, lse and idx_out of
 * lsa_sparse_attn_decode (plain loads and stores); every other pointer must be device memory.
 * flags: 0, or LSA_FLAG_PDL: launched as a programmatic dependent of the previous kernel of
 *     the stream; it touches src and dst only after that kernel completes, and lets the next
 *     kernel start at once; with LSA_FLAG_INPUTS_READY as well, src is read at once and only
 *     the writes wait.
 * Errors: LSA_ERR_INVALID_ARG for bytes not a multiple of 16, a pointer not 16-byte aligned,
 * overlapping ranges, or unknown flags; bytes == 0 enqueues nothing.
 */
LSA_API int lsa_copy_async(void* dst, const void* src, size_t bytes, int flags, cudaStream_t stream);

/*
 * lsa_sparse_attn_blockquery -- one denoising step of a block of Tq query tokens
 * (block-wise diffusion LM) against a cached prefix of T_prefix tokens.
 *
 * Defined by: LoSA, "1. 문제 정의" (the union of the KV positions selected by the
 * queries of a block sets memory traffic and latency) and "2. 방법론" (only active tokens
 * select and attend, sparsely; stable tokens reuse the previous step's prefix-attention
 * output and statistics; the union is taken over active tokens only).
 *
 * For every active token i (active[b, i] != 0) and KV group g:
 *   s_i(j)    = scale * sum_{h in g} q[b, h, i, :] . summ[b, g, j, :]   over prefix blocks
 *               j < NBp = ceil(T_prefix / blk)
 *   S(i, g)   = top-`topk_per_query` of s_i with forced blocks as in lsa_select_blocks
 *   U(b, g)   = union over active i of S(i, g), deduplicated, ascending
 *   every active row (b, h in g, i) attends over all tokens t < T_prefix of the blocks in
 *   U(b, g) (no mask inside the prefix): o = softmax-weighted v, lse = log-sum-exp.
 * Stable rows (active == 0): o[b,h,i,:] = o_cache[b,h,i,:] and lse = lse_cache, bit-exact
 * (o_cache / lse_cache may alias o / lse, in which case stable rows are left as they are;
 * a partial overlap of o with o_cache, or of lse with lse_cache, is LSA_ERR_INVALID_ARG).
 *
 * q [B, Hq, Tq, D] bf16; k, v [B, Hkv, T_cap, D] bf16 (T_prefix <= T_cap);
 * summ [B, Hkv, NB_cap, D] float32; active [B, Tq] uint8;
 * o_cache [B, Hq, Tq, D] bf16; lse_cache [B, Hq, Tq] float32; o, lse: same shapes, out.
 * union_idx [B, Hkv, NBp] int32 out or NULL (ascending, -1 padded);
 * union_cnt [B, Hkv] int32 out or NULL.
 * workspace: device scratch of at least lsa_blockquery_workspace_size(B, Hkv, G, D, Tq)
 *     bytes (16-byte aligned, contents need no initialisation), for the per-CTA partial
 *     results of the split over the union; calls that overlap on the GPU need their own.
 * Launch: programmatic dependent launch.  The kernel may start while the previous kernel
 * of the stream still runs, but reads no input before that kernel has completed (so any
 * previous kernel may produce any input), and it lets the next kernel of the stream start
 * early; a next kernel launched with programmatic dependent launch must wait for this
 * one's completion before reading its outputs (lsa_blockquery_intra_merge with
 * LSA_FLAG_PDL does).
 * Requires bf16, 1 <= Tq <= 64, B and Hkv <= 65535, n_sink + n_local <= topk_per_query, and either
 * 1 <= topk_per_query <= 16 or topk_per_query >= NBp.  The latter selects every prefix
 * block: with every token active this is the dense first denoising step of a block
 * (LoSA, "2. 방법론": the first step attends densely to build the cache, later steps
 * are sparse).
 */
LSA_API size_t lsa_blockquery_workspace_size(int B, int Hkv, int G, int D, int Tq);

LSA_API int lsa_sparse_attn_blockquery(const void* q, const void* k, const void* v, int dtype,
                               int B, int Hkv, int G, int D, int Tq, int T_prefix,
                               int T_cap, const float* summ, int blk, int topk_per_query,
                               int n_sink, int n_local, float scale, const uint8_t* active,
                               const void* o_cache, const float* lse_cache, void* o,
                               float* lse, int32_t* union_idx, int32_t* union_cnt,
                               void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * lsa_sparse_attn_blockquery_noalloc -- lsa_sparse_attn_blockquery for callers that may
 * not allocate device memory at all (nothing of theirs may call cudaMalloc, for example
 * code that runs where allocation is not allowed or must keep a fixed memory footprint).
 *
 * The pages have no counterpart of this entry point: it only changes where the scratch
 * of the block-query split lives.  Arguments, outputs and errors are those of
 * lsa_sparse_attn_blockquery without the workspace: the library uses one fixed device
 * array of 16 MiB instead, which every GPU that loads the library holds until the
 * process exits.  It allocates nothing and calls no allocating routine.
 *   - Shapes whose lsa_blockquery_workspace_size(B, Hkv, G, D, Tq) exceeds 16 MiB are
 *     rejected with LSA_ERR_UNSUPPORTED.
 *   - All calls share the array: calls that overlap on the GPU (different streams or host
 *     threads) race and must be serialised by the caller.  Its contents are left from the
 *     previous call; none of them needs to start at zero.
 *   - The first call on each device looks the array's device address up (the host-side
 *     name of a __device__ array is not a device address) and caches it; make that first
 *     call before any stream capture.
 */
LSA_API int lsa_sparse_attn_blockquery_noalloc(const void* q, const void* k, const void* v,
                                               int dtype, int B, int Hkv, int G, int D,
                                               int Tq, int T_prefix, int T_cap,
                                               const float* summ, int blk, int topk_per_query,
                                               int n_sink, int n_local, float scale,
                                               const uint8_t* active, const void* o_cache,
                                               const float* lse_cache, void* o, float* lse,
                                               int32_t* union_idx, int32_t* union_cnt,
                                               cudaStream_t stream);

/*
 * lsa_select_blocks_weighted -- lsa_select_blocks with a weight per head dimension in the
 * group score (FASA- and Prism-style scorers).
 *
 * Defined by: FASA, "2. 방법론" (token importance estimated from the dominant rotary
 * frequency chunks only) and Prism, "3. 제안 방법론" (block importance per frequency band,
 * each band with its own temperature that restores what mean pooling attenuates).
 *
 *   s[b, g, j] = scale * sum_{h in g} sum_d dim_weights[d] * q[b, h, d] * summ[b, g, j, d]
 * then the selection of lsa_select_blocks.  A 0/1 weight keeps a subset of the rotary
 * chunks (dims j and j + D/2 form chunk j under rotate-half pairing); one weight per band,
 * 1 / temperature, gives the dual-band score.  Choosing the chunks or temperatures is the
 * caller's.  The reweighted queries w * q are formed in fp32 in q_weighted (scratch,
 * [B, Hq, D] float32, 16-byte aligned; it may be q itself when q is float32, and any other
 * overlap with q or dim_weights returns LSA_ERR_INVALID_ARG) and scored by the selection
 * kernel.  dim_weights: [D] float32, device.  Other arguments and outputs as
 * lsa_select_blocks (scores_out holds the weighted scores).
 */
LSA_API int lsa_select_blocks_weighted(const void* q, int dtype, const float* summ,
                                       const float* dim_weights, int B, int Hkv, int G, int D,
                                       int NB_cap, const int32_t* seqlens, int blk, int topk,
                                       int n_sink, int n_local, float scale, float* q_weighted,
                                       int32_t* idx, int32_t* nsel, float* scores_out,
                                       cudaStream_t stream);

/*
 * lsa_sparse_attn_decode_blasst -- sparse decode attention over a given block selection
 * that drops, before reading their V, the selected blocks whose softmax weight is
 * negligible (BLASST inside sparse decode).
 *
 * Defined by: BLASST, "2. 방법론" -- "핵심 아이디어: 온라인 Softmax 통계 활용" (a block whose
 * local maximum trails the running maximum by more than the threshold contributes
 * nothing after the softmax) and "알고리즘 및 커널 설계" (block_max - running_max < ln(lambda);
 * the decode kernel, bound by memory, saves the V-block loads).
 *
 * For each (b, g) the selected blocks idx[b, g, :nsel] (ascending) are visited in order as
 * the blocks of an online softmax.  For block s and query head h of the group:
 *   r_h = max over the block's tokens t < seqlens[b] of scale * q_h . k_t
 *   m_h = the running maximum over the blocks visited before s
 *   skip block s  iff  s is not the first visited and max over h of (r_h - m_h) < ln(lambda)
 * (the group's heads share the block's V, so it is dropped only when every head finds it
 * negligible).  The output is softmax attention over the tokens of the kept blocks:
 * o [B, Hq, D] bf16, lse [B, Hq] float32 or NULL.  lambda = 0 never skips (and equals
 * lsa_sparse_attn_decode with the same selection).
 * skip_bits [B, Hkv] uint32 out or NULL: bit s set iff slot s was skipped.
 * q [B, Hq, D] bf16; k, v [B, Hkv, T_cap, D] bf16; seqlens [B]; idx [B, Hkv, topk]
 * ascending, -1 padded; nsel [B, Hkv].
 * Requires bf16, 1 <= topk <= 16, 0 <= lambda < 1.
 */
LSA_API int lsa_sparse_attn_decode_blasst(const void* q, const void* k, const void* v, int dtype,
                                          int B, int Hkv, int G, int D, int T_cap,
                                          const int32_t* seqlens, int blk, const int32_t* idx,
                                          const int32_t* nsel, int topk, float scale,
                                          float lambda, void* o, float* lse,
                                          uint32_t* skip_bits, cudaStream_t stream);

/*
 * lsa_nsa_compress -- NSA's compressed tokens with a fixed compression: the mean pool of
 * every `len` keys (and values) at stride `stride`.
 *
 * Defined by: NSA news article, "NSA 구조" (a compressed path of coarse tokens beside the
 * selected path and the sliding window; compression block l = 32, stride d = 16).  The
 * learned compression of the model is replaced by its plainest fixed form, the mean.
 *
 *   kc[b, g, i, :] = mean of k[b, g, t, :] over t in [i*stride, i*stride + len), t < T_b,
 *                    for i < NC_b = ceil(T_b / stride); rows i >= NC_b in the range are 0
 * (vc likewise from v), accumulated in fp32 and stored in bf16 (round to nearest even).
 * Range: nc_begin >= 0 -> compressed tokens [nc_begin, nc_end) (nc_end = -1: all);
 *        nc_begin < 0  -> the last -nc_begin compressed tokens of each sequence (a decode
 *        step that appended one token changes only the last ceil(len / stride) of them).
 * k, v [B, Hkv, T_cap, D] bf16; kc, vc [B, Hkv, ceil(T_cap / stride), D] bf16 out.
 * Requires bf16, D in {64, 128}, len, stride >= 1.
 */
LSA_API int lsa_nsa_compress(const void* k, const void* v, int dtype, int B, int Hkv, int T_cap,
                             int D, const int32_t* seqlens, int len, int stride, int nc_begin,
                             int nc_end, void* kc, void* vc, cudaStream_t stream);

/*
 * lsa_nsa_branches -- NSA's compressed and sliding-window branches for a decode step,
 * combined with the selected branch by constant gates.
 *
 * Defined by: NSA news article, "NSA 구조" (three parallel attention paths -- compressed
 * coarse tokens, selected fine tokens, a sliding window of w = 512 -- joined by gates; the
 * model's gates are learned, here they are constants chosen by the caller).
 *
 *   o_cmp = softmax attention of q over kc / vc rows [0, ceil(T_b / stride))
 *   o_win = softmax attention of q over k / v rows [max(0, T_b - window), T_b)
 *   o     = g_cmp * o_cmp + g_slc * o_slc + g_win * o_win      (logits scale * q . k)
 * o_slc is the selected branch's output (lsa_sparse_attn_decode), or NULL for none.
 * q [B, Hq, D] bf16; k, v [B, Hkv, T_cap, D] bf16; kc, vc [B, Hkv, ceil(T_cap / stride), D]
 * bf16 (lsa_nsa_compress); o [B, Hq, D] bf16 out (may be o_slc); lse_win, lse_cmp
 * [B, Hq] float32 out or NULL (-inf for an empty branch).
 * Requires bf16, D in {64, 128}, G <= 16, stride >= 1, window >= 0.
 */
LSA_API int lsa_nsa_branches(const void* q, const void* k, const void* v, const void* kc,
                             const void* vc, int dtype, int B, int Hkv, int G, int D, int T_cap,
                             const int32_t* seqlens, int window, int stride, float scale,
                             float g_cmp, float g_slc, float g_win, const void* o_slc, void* o,
                             float* lse_win, float* lse_cmp, cudaStream_t stream);

/*
 * lsa_losa_classify -- active and stable tokens of a query block between two denoising
 * steps.
 *
 * Defined by: LoSA, "2. 방법론" (each denoising step measures how much every token's query
 * vector changed, by its mean squared error, and calls the tokens that changed much
 * active and the others stable).
 *
 *   mse[b, i] = (1 / (Hq * D)) * sum over query heads h and dims d of
 *               (q[b, h, i, d] - q_prev[b, h, i, d])^2          (fp64)
 *   n_top > 0:  active[b, i] = 1 for the n_top tokens of largest mse (equal mse: the
 *               lower token index first), 0 for the others;
 *   n_top == 0: active[b, i] = (mse[b, i] > tau).
 * The sums and the comparison are carried out in double precision.  The kernel lets the
 * next kernel of the stream start early (the block-query step, which waits for it before
 * reading the mask).
 *
 * q, q_prev [B, Hq, Tq, D] bf16 (the block's queries this step and the previous one);
 * active [B, Tq] uint8 out (the mask lsa_sparse_attn_blockquery reads);
 * mse [B, Tq] double out, or NULL (8-byte aligned).
 * Requires bf16, D in {64, 128}, 1 <= Tq <= 64, n_top >= 0, B <= 65535, tau not NaN.
 */
LSA_API int lsa_losa_classify(const void* q, const void* q_prev, int dtype, int B, int Hq,
                              int Tq, int D, double tau, int n_top, uint8_t* active,
                              double* mse, cudaStream_t stream);

/*
 * lsa_blockquery_intra_merge -- attention of a query block over its own tokens, joined
 * with the prefix result: the last step of a LoSA denoising step.
 *
 * Defined by: LoSA, "2. 방법론" (active tokens attend sparsely to the prefix, stable tokens
 * reuse their prefix result -- output and statistics -- from the previous step; the block's
 * own tokens change every step and are attended every step).
 *
 * For query row (b, h, i), KV group g = h / G: the block's tokens are rows
 * T_prefix .. T_prefix + Tq - 1 of k[b, g] and v[b, g] (the caller writes this step's keys
 * and values of the block there).  The row attends over all Tq of them, with no mask
 * (attention inside the block is bidirectional):
 *   (o_in, lse_in) = softmax attention with logits scale * q . k_t
 * and the result is merged with the prefix part (o_pre, lse_pre) -- the softmax attention
 * of the same row over its prefix tokens, as lsa_sparse_attn_blockquery returns it -- by
 * log-sum-exp, i.e. the softmax over the union of both token sets:
 *   lse = log(exp(lse_pre) + exp(lse_in))
 *   o   = exp(lse_pre - lse) * o_pre + exp(lse_in - lse) * o_in
 * lse_pre = -inf means an empty prefix part (o = o_in).
 *
 * q [B, Hq, Tq, D] bf16; k, v [B, Hkv, T_cap, D] bf16 with T_prefix + Tq <= T_cap;
 * o_pre [B, Hq, Tq, D] bf16, lse_pre [B, Hq, Tq] float32; o, lse: same shapes, out.
 * o may be o_pre and lse may be lse_pre (updated in place); other overlaps are rejected.
 * flags: 0, or LSA_FLAG_PDL: launch with programmatic dependent launch; the kernel reads
 *     q, k and v at once and o_pre, lse_pre only after the previous kernel of the stream
 *     has completed, so the previous kernel may produce o_pre / lse_pre (the block-query
 *     step) but must not write q, k or v.
 * Requires bf16, D in {64, 128}, 1 <= Tq <= 64, G <= 16.
 */
LSA_API int lsa_blockquery_intra_merge(const void* q, const void* k, const void* v, int dtype,
                                       int B, int Hkv, int G, int D, int Tq, int T_prefix,
                                       int T_cap, float scale, const void* o_pre,
                                       const float* lse_pre, void* o, float* lse, int flags,
                                       cudaStream_t stream);

/*
 * lsa_blasst_prefill -- causal softmax attention that skips whole KV tiles whose
 * softmax weight is negligible (BLASST).
 *
 * Defined by: BLASST, "2. 방법론" -- "핵심 아이디어: 온라인 Softmax 통계 활용" (compare each
 * block's local maximum with the running maximum of the blockwise online softmax; skip
 * the exponentials, the V-block load and the P.V product of a block that trails by more
 * than the threshold) and "알고리즘 및 커널 설계" (the test block_max - running_max < ln(lambda)).
 *
 * For query head h (KV head h / (Hq / Hkv)) and query tile a (rows [128a, 128a + 128)),
 * KV tiles c = 0, 1, ... of 64 keys are visited in ascending order up to the diagonal:
 *   S = scale * Q K_c^T with the causal mask; r_i = max_t S_it; m_i = running row max
 *   skip tile c  iff  max over the tile's rows of (r_i - m_i) < ln(lambda)
 *   otherwise the usual online-softmax update of (m, l, acc) with tile c.
 * lambda = 0 never skips (plain causal attention).  The first tile is never skipped.
 * Outputs o = acc / l, lse = m + ln l.
 *
 * q [B, Hq, L, D] bf16; k, v [B, Hkv, L, D] bf16; o [B, Hq, L, D] bf16 out;
 * lse [B, Hq, L] float32 out or NULL;
 * skip_bits [B, Hq, ceil(L/128), ceil(ceil(L/64)/32)] uint32 out or NULL: bit c of a
 *     (b, h, a) row is set iff tile c was skipped;
 * skipped_tiles: one uint64 counter or NULL, incremented by the number of skipped tiles
 *     (the caller zeroes it).
 * Requires bf16, D == 128, Hq % Hkv == 0, B * Hq <= 65535, 0 <= lambda < 1.
 * Every wait of the kernel on its own pipeline is bounded in time; should one ever run
 * out, the kernel stops cleanly and lsa_device_status() reports LSA_DEVICE_TIMEOUT.
 */
LSA_API int lsa_blasst_prefill(const void* q, const void* k, const void* v, int dtype, int B, int Hq,
                       int Hkv, int L, int D, float scale, float lambda, void* o, float* lse,
                       uint32_t* skip_bits, unsigned long long* skipped_tiles,
                       cudaStream_t stream);

/*
 * lsa_device_status -- the device-side status word the kernels set when a bounded wait
 * runs out (LSA_DEVICE_TIMEOUT; a debug-bounds build also ORs in LSA_DEVICE_BOUNDS), 0
 * otherwise.  Synchronises with the device (it is a
 * debugging and failure-detection aid, not for the hot loop).  reset != 0 clears it.
 */
#define LSA_DEVICE_TIMEOUT 1
#define LSA_DEVICE_BOUNDS 2
LSA_API int lsa_device_status(int* status, int reset);

/*
 * lsa_debug_bounds_code -- the first out-of-range device-side value found by a library built
 * with LSA_DEBUG_BOUNDS (liblsa_debug.so), as (kind << 8) | site, 0 if none; reset != 0
 * clears it.  Kinds: 1 a sequence length outside [0, T_cap], 2 a selection index outside
 * [-1, NB_b), 3 a selection count outside [0, topk].  Sites: 1 summaries, 2 decode /
 * selection, 3 BLASST decode, 4 NSA pool, 5 NSA branches, 6 KV append.  The debug build
 * clamps such a value into range (every access stays in bounds, nothing traps) and also
 * reports LSA_DEVICE_BOUNDS in lsa_device_status().  The release build checks nothing,
 * sets *code = 0 and returns LSA_ERR_UNSUPPORTED.  Synchronises with the device.
 */
LSA_API int lsa_debug_bounds_code(int* code, int reset);

/*
 * Failure-handling controls, for tests of the bounded waits (no counterpart on the pages;
 * they exist so that the timeout path can be exercised without faulting a GPU).
 *
 * lsa_debug_set_wait_budget -- the clock-cycle limit of every bounded wait inside the
 *     kernels launched from now on (process-wide); cycles <= 0 restores the default
 *     (4e9 cycles, about 2 s).  After a wait runs out a kernel leaves its loops, waits (with
 *     a second, fixed 4e9-cycle limit) for its own copies and tensor-core work in flight and
 *     for the bytes its cluster peers still owe it, frees its tensor memory, and sets the
 *     status word; the launch's outputs are then undefined.
 * lsa_debug_inject -- kind 0: normal operation (the default).  LSA_DEBUG_PREFILL_DROP_S:
 *     the next lsa_blasst_prefill launches never signal their first S tile, so the softmax
 *     warps' wait for it runs out and the timeout path above runs.  Process-wide.
 * Both return LSA_OK, or LSA_ERR_INVALID_ARG for an unknown kind.
 */
#define LSA_DEBUG_PREFILL_DROP_S 1
LSA_API int lsa_debug_set_wait_budget(long long cycles);
LSA_API int lsa_debug_inject(int kind);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
