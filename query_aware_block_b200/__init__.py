"""Thin Python binding of liblsa.so (query-aware block-sparse attention for B200).

The functions carry the names of the C ABI in include/lsa.h and only marshal arguments:
shapes are read from the torch tensors, pointers and the current CUDA stream are passed
through ctypes, and a non-zero status raises LsaError.  Every step of the computation runs
in the library's CUDA kernels; there is no fallback of any kind.  If liblsa.so has not been
built (``python query_aware_block_b200/_build.py``), importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# LSA_LIBRARY=debug loads the bounds-checking build (liblsa_debug.so, see _build.py)
LIB_PATH = os.path.join(_HERE, "liblsa_debug.so" if os.environ.get("LSA_LIBRARY") == "debug" else "liblsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python query_aware_block_b200/_build.py`"
                      + (" --debug-bounds" if LIB_PATH.endswith("_debug.so") else ""))

_lib = ctypes.CDLL(LIB_PATH)

LSA_OK, LSA_ERR_INVALID_ARG, LSA_ERR_UNSUPPORTED, LSA_ERR_CUDA, LSA_ERR_DEVICE_STATUS = 0, 1, 2, 3, 4
LSA_F32, LSA_BF16 = 0, 1
LSA_FLAG_PDL = 1
LSA_FLAG_INPUTS_READY = 2
LSA_DEBUG_PREFILL_DROP_S = 1
BLK = 64

EXPORTED = ("lsa_status_string", "lsa_last_cuda_error", "lsa_version", "lsa_build_summaries",
            "lsa_select_blocks", "lsa_sparse_attn_decode", "lsa_blockquery_workspace_size",
            "lsa_sparse_attn_blockquery", "lsa_sparse_attn_blockquery_noalloc",
            "lsa_blasst_prefill", "lsa_device_status", "lsa_losa_classify",
            "lsa_blockquery_intra_merge", "lsa_sparse_attn_decode_blasst", "lsa_nsa_compress",
            "lsa_nsa_branches", "lsa_select_blocks_weighted", "lsa_append_kv", "lsa_append_kv_stage_q", "lsa_copy_async",
            "lsa_debug_set_wait_budget", "lsa_debug_inject", "lsa_debug_bounds_code")

_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_lib.lsa_status_string.restype = ctypes.c_char_p
_lib.lsa_status_string.argtypes = [_i]
_lib.lsa_last_cuda_error.restype = _i
_lib.lsa_last_cuda_error.argtypes = []
_lib.lsa_version.restype = _i
_lib.lsa_version.argtypes = []
_lib.lsa_build_summaries.argtypes = [_vp, _i, _i, _i, _i, _i, _vp, _i, _i, _i, _vp, _vp]
_lib.lsa_select_blocks.argtypes = [_vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _i, _i, _i, _i, _f,
                                   _vp, _vp, _vp, _vp]
_lib.lsa_sparse_attn_decode.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp,
                                        _i, _f, _vp, _i, _i, _i, _vp, _vp, _vp, _i, _vp]
_lib.lsa_debug_set_wait_budget.argtypes = [ctypes.c_longlong]
_lib.lsa_debug_inject.argtypes = [_i]
_lib.lsa_debug_bounds_code.argtypes = [_vp, _i]
_lib.lsa_append_kv.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _i, _vp]
_lib.lsa_copy_async.argtypes = [_vp, _vp, ctypes.c_size_t, _i, _vp]
_lib.lsa_append_kv_stage_q.argtypes = [_vp, _vp, ctypes.c_size_t, _vp, _vp, _i, _i, _i, _i, _i, _vp,
                                       _vp, _vp, _i, _vp]
_lib.lsa_blockquery_workspace_size.argtypes = [_i, _i, _i, _i, _i]
_lib.lsa_blockquery_workspace_size.restype = ctypes.c_size_t
_lib.lsa_sparse_attn_blockquery.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp,
                                            _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _vp, _vp,
                                            _vp, _vp, ctypes.c_size_t, _vp]
_lib.lsa_sparse_attn_blockquery_noalloc.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                                    _i, _vp, _i, _i, _i, _i, _f, _vp, _vp, _vp,
                                                    _vp, _vp, _vp, _vp, _vp]
_lib.lsa_blasst_prefill.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _f, _vp, _vp, _vp,
                                    _vp, _vp]
_lib.lsa_device_status.argtypes = [_vp, _i]
_lib.lsa_sparse_attn_decode_blasst.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _i,
                                               _vp, _vp, _i, _f, _f, _vp, _vp, _vp, _vp]
_lib.lsa_select_blocks_weighted.argtypes = [_vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _i, _i,
                                            _i, _f, _vp, _vp, _vp, _vp, _vp]
_lib.lsa_nsa_compress.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _i, _i, _i, _vp, _vp, _vp]
_lib.lsa_nsa_branches.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _i, _i, _f,
                                  _f, _f, _f, _vp, _vp, _vp, _vp, _vp]
_lib.lsa_losa_classify.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, ctypes.c_double, _i, _vp, _vp,
                                   _vp]
_lib.lsa_blockquery_intra_merge.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                                            _vp, _vp, _vp, _vp, _i, _vp]
for _n in EXPORTED[3:]:
    if _n != "lsa_blockquery_workspace_size":
        getattr(_lib, _n).restype = _i


class LsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.lsa_status_string(status).decode()
        if status == LSA_ERR_CUDA:
            msg += f" (cudaError {_lib.lsa_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")
        self.status = status


def library():
    """The loaded ctypes library (for tests of the raw ABI)."""
    return _lib


def lsa_version() -> int:
    return int(_lib.lsa_version())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LSA_BF16
    if t.dtype == torch.float32:
        return LSA_F32
    return -1  # rejected by the library as unsupported


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(status: int, where: str):
    if status != LSA_OK:
        raise LsaError(status, where)


def lsa_build_summaries(k, seqlens, summ, nb_begin=0, nb_end=-1, blk=BLK, stream=None):
    """k [B,Hkv,T_cap,D] -> summ [B,Hkv,ceil(T_cap/blk),D] float32 (in place)."""
    B, Hkv, T_cap, D = k.shape
    _check(_lib.lsa_build_summaries(_ptr(k), _dtype(k), B, Hkv, T_cap, D, _ptr(seqlens), blk,
                                    nb_begin, nb_end, _ptr(summ), _stream(stream)),
           "lsa_build_summaries")
    return summ


def lsa_select_blocks(q, summ, seqlens, topk, n_sink, n_local, idx, nsel, scale=0.0,
                      scores_out=None, blk=BLK, stream=None):
    """q [B,Hq,D], summ [B,Hkv,NB_cap,D] -> idx [B,Hkv,topk], nsel [B,Hkv] (in place)."""
    B, Hq, D = q.shape
    _, Hkv, NB_cap, _ = summ.shape
    _check(_lib.lsa_select_blocks(_ptr(q), _dtype(q), _ptr(summ), B, Hkv, Hq // Hkv, D, NB_cap,
                                  _ptr(seqlens), blk, topk, n_sink, n_local, float(scale),
                                  _ptr(idx), _ptr(nsel), _ptr(scores_out), _stream(stream)),
           "lsa_select_blocks")
    return idx, nsel


def lsa_append_kv(k_new, v_new, seqlens, k, v, flags=0, stream=None):
    """k_new, v_new [B,Hkv,D] -> k, v [B,Hkv,T_cap,D] at row seqlens[b] - 1 (in place)."""
    B, Hkv, T_cap, D = k.shape
    _check(_lib.lsa_append_kv(_ptr(k_new), _ptr(v_new), _dtype(k), B, Hkv, T_cap, D, _ptr(seqlens),
                              _ptr(k), _ptr(v), flags, _stream(stream)), "lsa_append_kv")
    return k, v


def lsa_append_kv_stage_q(q_src, q_dst, k_new, v_new, seqlens, k, v, flags=0, stream=None):
    """lsa_append_kv and q_dst <- q_src in one launch; q_src, k_new, v_new may be pinned host."""
    B, Hkv, T_cap, D = k.shape
    n = q_src.numel() * q_src.element_size()
    assert q_dst.numel() * q_dst.element_size() == n, "lsa_append_kv_stage_q: q sizes differ"
    _check(_lib.lsa_append_kv_stage_q(_ptr(q_src), _ptr(q_dst), n, _ptr(k_new), _ptr(v_new), _dtype(k), B,
                                      Hkv, T_cap, D, _ptr(seqlens), _ptr(k), _ptr(v), int(flags),
                                      _stream(stream)), "lsa_append_kv_stage_q")
    return k, v


def lsa_copy_async(dst, src, flags=0, stream=None):
    """dst <- src (same number of bytes) by a kernel; either may be a pinned host tensor."""
    n = src.numel() * src.element_size()
    assert dst.numel() * dst.element_size() == n, "lsa_copy_async: sizes differ"
    _check(_lib.lsa_copy_async(_ptr(dst), _ptr(src), n, int(flags), _stream(stream)), "lsa_copy_async")
    return dst


def lsa_sparse_attn_decode(q, k, v, seqlens, o, topk, idx=None, nsel=None, summ=None,
                           n_sink=0, n_local=0, refresh_last_summary=False, idx_out=None,
                           lse=None, scale=0.0, blk=BLK, flags=0, stream=None):
    """Sparse decode attention.  Given selection: idx, nsel.  Fused selection: summ (and,
    with refresh_last_summary, the last block's summary is rewritten in the same launch)."""
    B, Hq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    _check(_lib.lsa_sparse_attn_decode(_ptr(q), _ptr(k), _ptr(v), _dtype(q), B, Hkv, Hq // Hkv,
                                       D, T_cap, _ptr(seqlens), blk, _ptr(idx), _ptr(nsel),
                                       topk, float(scale), _ptr(summ), n_sink, n_local,
                                       int(bool(refresh_last_summary)), _ptr(idx_out), _ptr(o),
                                       _ptr(lse), int(flags), _stream(stream)),
           "lsa_sparse_attn_decode")
    return o


def lsa_blockquery_workspace_size(B, Hkv, G, D, Tq) -> int:
    return int(_lib.lsa_blockquery_workspace_size(B, Hkv, G, D, Tq))


def lsa_sparse_attn_blockquery(q, k, v, summ, T_prefix, topk_per_query, active, o_cache,
                               lse_cache, o, lse, workspace, n_sink=0, n_local=0,
                               union_idx=None, union_cnt=None, scale=0.0, blk=BLK,
                               stream=None):
    """Block-query step: q [B,Hq,Tq,D] against the prefix of k, v [B,Hkv,T_cap,D].
    workspace: a device buffer of at least lsa_blockquery_workspace_size(...) bytes."""
    B, Hq, Tq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    _check(_lib.lsa_sparse_attn_blockquery(_ptr(q), _ptr(k), _ptr(v), _dtype(q), B, Hkv,
                                           Hq // Hkv, D, Tq, T_prefix, T_cap, _ptr(summ), blk,
                                           topk_per_query, n_sink, n_local, float(scale),
                                           _ptr(active), _ptr(o_cache), _ptr(lse_cache),
                                           _ptr(o), _ptr(lse), _ptr(union_idx), _ptr(union_cnt),
                                           _ptr(workspace),
                                           workspace.numel() * workspace.element_size(),
                                           _stream(stream)),
           "lsa_sparse_attn_blockquery")
    return o, lse


def lsa_blasst_prefill(q, k, v, o, lam, lse=None, skip_bits=None, skipped_tiles=None,
                       scale=0.0, stream=None):
    """BLASST causal prefill: q [B,Hq,L,D], k, v [B,Hkv,L,D] -> o (in place)."""
    B, Hq, L, D = q.shape
    Hkv = k.shape[1]
    _check(_lib.lsa_blasst_prefill(_ptr(q), _ptr(k), _ptr(v), _dtype(q), B, Hq, Hkv, L, D,
                                   float(scale), float(lam), _ptr(o), _ptr(lse), _ptr(skip_bits),
                                   _ptr(skipped_tiles), _stream(stream)),
           "lsa_blasst_prefill")
    return o


def lsa_select_blocks_weighted(q, summ, seqlens, dim_weights, topk, n_sink, n_local, idx, nsel,
                               q_weighted=None, scale=0.0, scores_out=None, blk=BLK, stream=None):
    """Block selection with a weight per head dimension (FASA / Prism-style scorers):
    dim_weights [D] float32 on the device; q_weighted: float32 [B,Hq,D] scratch (allocated
    here when not given)."""
    B, Hq, D = q.shape
    _, Hkv, NB_cap, _ = summ.shape
    if q_weighted is None:
        q_weighted = torch.empty(B, Hq, D, dtype=torch.float32, device=q.device)
    _check(_lib.lsa_select_blocks_weighted(_ptr(q), _dtype(q), _ptr(summ), _ptr(dim_weights), B, Hkv,
                                           Hq // Hkv, D, NB_cap, _ptr(seqlens), blk, topk, n_sink,
                                           n_local, float(scale), _ptr(q_weighted), _ptr(idx),
                                           _ptr(nsel), _ptr(scores_out), _stream(stream)),
           "lsa_select_blocks_weighted")
    return idx, nsel


def lsa_sparse_attn_decode_blasst(q, k, v, seqlens, idx, nsel, o, lam, lse=None, skip_bits=None,
                                  scale=0.0, blk=BLK, stream=None):
    """Sparse decode over the given selection idx [B,Hkv,topk] with BLASST's skip: blocks
    every head of the group finds negligible (below the running max by -ln(lam)) are not
    read.  skip_bits: optional int32 [B,Hkv] out (bit s = slot s skipped)."""
    B, Hq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    _check(_lib.lsa_sparse_attn_decode_blasst(_ptr(q), _ptr(k), _ptr(v), _dtype(q), B, Hkv,
                                              Hq // Hkv, D, T_cap, _ptr(seqlens), blk, _ptr(idx),
                                              _ptr(nsel), idx.shape[-1], float(scale), float(lam),
                                              _ptr(o), _ptr(lse), _ptr(skip_bits), _stream(stream)),
           "lsa_sparse_attn_decode_blasst")
    return o


def lsa_nsa_compress(k, v, seqlens, kc, vc, length=32, stride=16, nc_begin=0, nc_end=-1,
                     stream=None):
    """Mean-pooled compressed keys and values: kc, vc [B,Hkv,ceil(T_cap/stride),D] bf16 (in
    place); nc_begin < 0 refreshes the last -nc_begin compressed tokens of each sequence."""
    B, Hkv, T_cap, D = k.shape
    _check(_lib.lsa_nsa_compress(_ptr(k), _ptr(v), _dtype(k), B, Hkv, T_cap, D, _ptr(seqlens),
                                 int(length), int(stride), int(nc_begin), int(nc_end), _ptr(kc),
                                 _ptr(vc), _stream(stream)),
           "lsa_nsa_compress")
    return kc, vc


def lsa_nsa_branches(q, k, v, kc, vc, seqlens, o, gates=(1 / 3, 1 / 3, 1 / 3), o_slc=None,
                     window=512, stride=16, lse_win=None, lse_cmp=None, scale=0.0, stream=None):
    """NSA's compressed and window branches of a decode step, combined with the selected
    branch output o_slc: o = gates[0] * o_cmp + gates[1] * o_slc + gates[2] * o_win."""
    B, Hq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    g = [float(x) for x in gates]
    _check(_lib.lsa_nsa_branches(_ptr(q), _ptr(k), _ptr(v), _ptr(kc), _ptr(vc), _dtype(q), B, Hkv,
                                 Hq // Hkv, D, T_cap, _ptr(seqlens), int(window), int(stride),
                                 float(scale), g[0], g[1], g[2], _ptr(o_slc), _ptr(o),
                                 _ptr(lse_win), _ptr(lse_cmp), _stream(stream)),
           "lsa_nsa_branches")
    return o


def lsa_losa_classify(q, q_prev, active, tau=0.0, n_top=0, mse=None, stream=None):
    """Active mask [B,Tq] uint8 (in place) from the change of q [B,Hq,Tq,D] since q_prev:
    the n_top largest mean squared changes, or (n_top == 0) those above tau.
    mse: optional float64 [B,Tq] out."""
    B, Hq, Tq, D = q.shape
    _check(_lib.lsa_losa_classify(_ptr(q), _ptr(q_prev), _dtype(q), B, Hq, Tq, D, float(tau),
                                  int(n_top), _ptr(active), _ptr(mse), _stream(stream)),
           "lsa_losa_classify")
    return active


def lsa_blockquery_intra_merge(q, k, v, T_prefix, o_pre, lse_pre, o, lse, scale=0.0, flags=0,
                               stream=None):
    """Bidirectional attention of q [B,Hq,Tq,D] over the block's own keys (rows
    T_prefix .. T_prefix+Tq-1 of k, v [B,Hkv,T_cap,D]), merged with the prefix result
    (o_pre, lse_pre) by log-sum-exp into o, lse (in place; o may be o_pre)."""
    B, Hq, Tq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    _check(_lib.lsa_blockquery_intra_merge(_ptr(q), _ptr(k), _ptr(v), _dtype(q), B, Hkv,
                                           Hq // Hkv, D, Tq, T_prefix, T_cap, float(scale),
                                           _ptr(o_pre), _ptr(lse_pre), _ptr(o), _ptr(lse),
                                           int(flags), _stream(stream)),
           "lsa_blockquery_intra_merge")
    return o, lse


def lsa_device_status(reset=False) -> int:
    """The device status word (0, or LSA_DEVICE_TIMEOUT after a bounded wait ran out)."""
    out = ctypes.c_int(0)
    _check(_lib.lsa_device_status(ctypes.byref(out), int(bool(reset))), "lsa_device_status")
    return out.value


LSA_DEVICE_TIMEOUT = 1


def lsa_debug_set_wait_budget(cycles: int) -> None:
    """Clock-cycle limit of the kernels' bounded waits (tests only; <= 0 restores 4e9)."""
    _check(_lib.lsa_debug_set_wait_budget(int(cycles)), "lsa_debug_set_wait_budget")


def lsa_debug_bounds_code(reset=False) -> int:
    """The first out-of-range device-side value a bounds-checking build found, as
    (kind << 8) | site (0 if none); raises LsaError (LSA_ERR_UNSUPPORTED) in the release build."""
    out = ctypes.c_int(0)
    _check(_lib.lsa_debug_bounds_code(ctypes.byref(out), int(bool(reset))), "lsa_debug_bounds_code")
    return out.value


def lsa_debug_inject(kind: int) -> None:
    """Fault injected into later launches (tests only; 0 = none)."""
    _check(_lib.lsa_debug_inject(int(kind)), "lsa_debug_inject")
