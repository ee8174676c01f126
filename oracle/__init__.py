"""fp64 CPU oracle for query-aware block-sparse attention.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The arithmetic lives in
``lsa_oracle.c`` (plain C, double precision, one loop nest per definition); this module
only compiles it with gcc and marshals torch CPU tensors into it.  It shares nothing with
the CUDA library in ``query_aware_block_b200``.

Parity status of each function (what pins it is in tests/test_oracle_pins.py):
  summaries, block_scores, select, decode_attn, blockquery_select, blockquery_attn,
  blasst_prefill, decode_blasst, losa_classify, blockquery_intra_merge (and the losa_step
  composition), nsa_compress, range_attn_f64, window_attn (and the nsa_decode composition),
  block_scores_weighted with the FASA / Prism weight builders
  -- all pinned (textbook special cases, brute force, library routines, closed forms and
  invariants).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblsa_oracle.so")
_lib = None
_lock = threading.Lock()

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile lsa_oracle.c into liblsa_oracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = ctypes.CDLL(_LIB_PATH)
            _lib.oracle_num_threads.restype = ctypes.c_int
    return _lib


def _p(t: torch.Tensor | None):
    if t is None:
        return ctypes.c_void_p(0)
    assert t.device.type == "cpu" and t.is_contiguous(), "oracle takes contiguous CPU tensors"
    return ctypes.c_void_p(t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"oracle inputs are float32 or bfloat16, got {t.dtype}")


def _i32(t):
    return t.to(torch.int32).contiguous()


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(ctypes.c_int(n))


def _scale(scale, D):
    return 1.0 / math.sqrt(D) if (scale is None or scale <= 0) else float(scale)


def summaries(k, seqlens, blk=64):
    """k [B,Hkv,T_cap,D] -> fp64 summaries [B,Hkv,ceil(T_cap/blk),D] (zeros past each T_b)."""
    k = k.contiguous()
    B, Hkv, T_cap, D = k.shape
    NB_cap = -(-T_cap // blk)
    out = torch.zeros(B, Hkv, NB_cap, D, dtype=torch.float64)
    sl = _i32(seqlens)
    _load().oracle_summaries(_p(k), _dt(k), B, Hkv, T_cap, D, _p(sl), blk, _p(out))
    return out


def block_scores(q, summ, seqlens, blk=64, scale=None):
    """q [B,Hq,D], fp64 summ [B,Hkv,NB_cap,D] -> fp64 group scores [B,Hkv,NB_cap]."""
    q = q.contiguous()
    summ = summ.to(torch.float64).contiguous()
    B, Hq, D = q.shape
    _, Hkv, NB_cap, _ = summ.shape
    G = Hq // Hkv
    out = torch.empty(B, Hkv, NB_cap, dtype=torch.float64)
    sl = _i32(seqlens)
    _load().oracle_block_scores(_p(q), _dt(q), _p(summ), B, Hkv, G, D, NB_cap, _p(sl), blk,
                                ctypes.c_double(_scale(scale, D)), _p(out))
    return out


def select(scores, seqlens, topk, n_sink, n_local, blk=64):
    """fp64 scores [B,Hkv,NB_cap] -> (idx [B,Hkv,topk] ascending, -1 pad; nsel [B,Hkv])."""
    scores = scores.to(torch.float64).contiguous()
    B, Hkv, NB_cap = scores.shape
    idx = torch.empty(B, Hkv, topk, dtype=torch.int32)
    nsel = torch.empty(B, Hkv, dtype=torch.int32)
    sl = _i32(seqlens)
    _load().oracle_select(_p(scores), B, Hkv, NB_cap, _p(sl), blk, topk, n_sink, n_local,
                          _p(idx), _p(nsel))
    return idx, nsel


def decode_attn(q, k, v, seqlens, idx, nsel, blk=64, scale=None):
    """Sparse decode attention over the listed blocks -> (o fp64 [B,Hq,D], lse fp64 [B,Hq])."""
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    assert q.dtype == k.dtype == v.dtype
    B, Hq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    G = Hq // Hkv
    idx = _i32(idx)
    nsel = _i32(nsel)
    topk = idx.shape[-1]
    o = torch.empty(B, Hq, D, dtype=torch.float64)
    lse = torch.empty(B, Hq, dtype=torch.float64)
    sl = _i32(seqlens)
    _load().oracle_decode_attn(_p(q), _p(k), _p(v), _dt(q), B, Hkv, G, D, T_cap, _p(sl), blk,
                               _p(idx), _p(nsel), topk, ctypes.c_double(_scale(scale, D)),
                               _p(o), _p(lse))
    return o, lse


def decode(q, k, v, seqlens, topk, n_sink, n_local, blk=64, scale=None):
    """The whole decode path in the oracle: summaries -> scores -> select -> attention."""
    summ = summaries(k, seqlens, blk)
    s = block_scores(q, summ, seqlens, blk, scale)
    idx, nsel = select(s, seqlens, topk, n_sink, n_local, blk)
    o, lse = decode_attn(q, k, v, seqlens, idx, nsel, blk, scale)
    return dict(summ=summ, scores=s, idx=idx, nsel=nsel, o=o, lse=lse)


def blockquery_select(q, summ, active, T_prefix, topk, n_sink=0, n_local=0, blk=64,
                      scale=None, return_sel=False):
    """Per-active-token top-k and the union per (b, kv group).

    q [B,Hq,Tq,D]; fp64 summ [B,Hkv,NB_cap,D]; active [B,Tq] (uint8/bool).
    Returns union_idx [B,Hkv,NBp] (ascending, -1 pad), union_cnt [B,Hkv] and, if asked,
    each token's own selection [B,Tq,Hkv,topk]."""
    q = q.contiguous()
    summ = summ.to(torch.float64).contiguous()
    B, Hq, Tq, D = q.shape
    _, Hkv, NB_cap, _ = summ.shape
    G = Hq // Hkv
    NBp = -(-T_prefix // blk)
    act = active.to(torch.uint8).contiguous()
    uidx = torch.empty(B, Hkv, NBp, dtype=torch.int32)
    ucnt = torch.empty(B, Hkv, dtype=torch.int32)
    sel = torch.empty(B, Tq, Hkv, topk, dtype=torch.int32) if return_sel else None
    _load().oracle_blockquery_select(_p(q), _dt(q), _p(summ), B, Hkv, G, D, Tq, T_prefix,
                                     NB_cap, blk, topk, n_sink, n_local,
                                     ctypes.c_double(_scale(scale, D)), _p(act), _p(uidx),
                                     _p(ucnt), _p(sel))
    return (uidx, ucnt, sel) if return_sel else (uidx, ucnt)


def blockquery_attn(q, k, v, active, o_cache, lse_cache, union_idx, union_cnt, T_prefix,
                    blk=64, scale=None):
    """Active rows attend over the union blocks; stable rows copy the cache.

    -> (o fp64 [B,Hq,Tq,D], lse fp64 [B,Hq,Tq])."""
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    B, Hq, Tq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    G = Hq // Hkv
    act = active.to(torch.uint8).contiguous()
    oc = o_cache.to(q.dtype).contiguous()
    lc = lse_cache.to(torch.float32).contiguous()
    ui = _i32(union_idx)
    uc = _i32(union_cnt)
    NBp = -(-T_prefix // blk)
    assert ui.shape[-1] == NBp
    o = torch.empty(B, Hq, Tq, D, dtype=torch.float64)
    lse = torch.empty(B, Hq, Tq, dtype=torch.float64)
    _load().oracle_blockquery_attn(_p(q), _p(k), _p(v), _dt(q), B, Hkv, G, D, Tq, T_prefix,
                                   T_cap, blk, ctypes.c_double(_scale(scale, D)), _p(act),
                                   _p(oc), _p(lc), _p(ui), _p(uc), _p(o), _p(lse))
    return o, lse


def blasst_prefill(q, k, v, units, lam, tq=128, tk=64, scale=None, forced_bits=None):
    """BLASST causal prefill on a list of (b, h, a) work units.

    q [B,Hq,L,D]; k, v [B,Hkv,L,D]; units int [n,3].
    Returns dict(o [n,tq,D] fp64, lse [n,tq] fp64, bits [n,words] uint32 as int64,
    gap [n,nkv] fp64) where words = ceil(ceil(L/tk)/32)."""
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    B, Hq, L, D = q.shape
    Hkv = k.shape[1]
    units = _i32(torch.as_tensor(units).reshape(-1, 3))
    n = units.shape[0]
    nkv = -(-L // tk)
    words = -(-nkv // 32)
    o = torch.empty(n, tq, D, dtype=torch.float64)
    lse = torch.empty(n, tq, dtype=torch.float64)
    bits = torch.empty(n, words, dtype=torch.int32)
    gap = torch.empty(n, nkv, dtype=torch.float64)
    fb = None
    if forced_bits is not None:
        fb = np.asarray(torch.as_tensor(forced_bits).to(torch.int64).reshape(n, words))
        fb = torch.from_numpy((fb & 0xFFFFFFFF).astype(np.uint32).view(np.int32).copy())
    _load().oracle_blasst_prefill(_p(q), _p(k), _p(v), _dt(q), B, Hq, Hkv, L, D,
                                  ctypes.c_double(_scale(scale, D)), ctypes.c_double(float(lam)),
                                  tq, tk, n, _p(units), _p(fb), words, _p(o), _p(lse),
                                  _p(bits), _p(gap))
    return dict(o=o, lse=lse, bits=bits.to(torch.int64) & 0xFFFFFFFF, gap=gap)


def losa_classify(q, q_prev, tau=0.0, n_top=0):
    """Active / stable tokens from the mean squared change of their queries.

    q, q_prev [B,Hq,Tq,D] (same dtype).  Returns (mse fp64 [B,Tq], active uint8 [B,Tq]):
    n_top > 0 marks the n_top largest changes (ties: lower index), else mse > tau."""
    q, q_prev = q.contiguous(), q_prev.contiguous()
    assert q.dtype == q_prev.dtype and q.shape == q_prev.shape
    B, Hq, Tq, D = q.shape
    mse = torch.empty(B, Tq, dtype=torch.float64)
    act = torch.empty(B, Tq, dtype=torch.uint8)
    _load().oracle_losa_classify(_p(q), _p(q_prev), _dt(q), B, Hq, Tq, D,
                                 ctypes.c_double(float(tau)), int(n_top), _p(mse), _p(act))
    return mse, act


def blockquery_intra_merge(q, k, v, T_prefix, o_pre, lse_pre, scale=None):
    """Bidirectional attention over the block's own tokens (rows T_prefix .. T_prefix+Tq-1
    of k and v), merged with the prefix result (o_pre, lse_pre) by log-sum-exp.

    The prefix result is widened exactly to fp64.  -> (o fp64 [B,Hq,Tq,D], lse fp64 [B,Hq,Tq])."""
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    assert q.dtype == k.dtype == v.dtype
    B, Hq, Tq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    assert T_prefix + Tq <= T_cap
    G = Hq // Hkv
    op = o_pre.to(torch.float64).contiguous()
    lp = lse_pre.to(torch.float64).contiguous()
    o = torch.empty(B, Hq, Tq, D, dtype=torch.float64)
    lse = torch.empty(B, Hq, Tq, dtype=torch.float64)
    _load().oracle_blockquery_intra_merge(_p(q), _p(k), _p(v), _dt(q), B, Hkv, G, D, Tq,
                                          T_prefix, T_cap, ctypes.c_double(_scale(scale, D)),
                                          _p(op), _p(lp), _p(o), _p(lse))
    return o, lse


def losa_step(q, q_prev, k, v, summ, T_prefix, o_cache, lse_cache, topk, tau=0.0, n_top=0,
              n_sink=0, n_local=0, blk=64, scale=None, union=None):
    """One LoSA denoising step in the oracle, in the pages' order: classify the tokens,
    select and attend the prefix for the active ones (stable ones keep the cache), attend
    inside the block and merge.  `union` = (union_idx, union_cnt) replaces the oracle's own
    union (to evaluate another implementation's choice among tied scores).

    Returns dict(mse, active, union_idx, union_cnt, o_prefix, lse_prefix, o, lse); the
    prefix part is fp64 (not rounded)."""
    mse, active = losa_classify(q, q_prev, tau, n_top)
    if union is None:
        uidx, ucnt = blockquery_select(q, summ, active, T_prefix, topk, n_sink, n_local, blk, scale)
    else:
        uidx, ucnt = union
    o_p, lse_p = blockquery_attn(q, k, v, active, o_cache, lse_cache, uidx, ucnt, T_prefix,
                                 blk, scale)
    o, lse = blockquery_intra_merge(q, k, v, T_prefix, o_p, lse_p, scale)
    return dict(mse=mse, active=active, union_idx=uidx, union_cnt=ucnt, o_prefix=o_p,
                lse_prefix=lse_p, o=o, lse=lse)


def decode_blasst(q, k, v, seqlens, idx, nsel, lam, blk=64, scale=None, forced_bits=None):
    """Sparse decode attention over the listed blocks (visited in ascending order) with
    BLASST's skip test over the group's heads.

    Returns dict(o fp64 [B,Hq,D], lse fp64 [B,Hq], bits [B,Hkv] (int64, bit r = slot r
    skipped), gap fp64 [B,Hkv,topk]); forced_bits [B,Hkv] replaces the decisions."""
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    assert q.dtype == k.dtype == v.dtype
    B, Hq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    G = Hq // Hkv
    idx = _i32(idx)
    nsel = _i32(nsel)
    topk = idx.shape[-1]
    assert topk <= 32
    o = torch.empty(B, Hq, D, dtype=torch.float64)
    lse = torch.empty(B, Hq, dtype=torch.float64)
    bits = torch.empty(B, Hkv, dtype=torch.int32)
    gap = torch.empty(B, Hkv, topk, dtype=torch.float64)
    fb = None
    if forced_bits is not None:
        fb = np.asarray(torch.as_tensor(forced_bits).to(torch.int64).reshape(B, Hkv))
        fb = torch.from_numpy((fb & 0xFFFFFFFF).astype(np.uint32).view(np.int32).copy())
    sl = _i32(seqlens)
    _load().oracle_decode_blasst(_p(q), _p(k), _p(v), _dt(q), B, Hkv, G, D, T_cap, _p(sl), blk,
                                 _p(idx), _p(nsel), topk, ctypes.c_double(_scale(scale, D)),
                                 ctypes.c_double(float(lam)), _p(fb), _p(o), _p(lse), _p(bits),
                                 _p(gap))
    return dict(o=o, lse=lse, bits=bits.to(torch.int64) & 0xFFFFFFFF, gap=gap)


def nsa_compress(x, seqlens, length=32, stride=16):
    """Mean-pooled compressed tokens: x [B,Hkv,T_cap,D] -> fp64 [B,Hkv,ceil(T_cap/stride),D],
    row i the mean of the valid tokens of [i*stride, i*stride + length) (zeros past
    ceil(T_b/stride))."""
    x = x.contiguous()
    B, Hkv, T_cap, D = x.shape
    out = torch.empty(B, Hkv, -(-T_cap // stride), D, dtype=torch.float64)
    sl = _i32(seqlens)
    _load().oracle_nsa_compress(_p(x), _dt(x), B, Hkv, T_cap, D, _p(sl), int(length), int(stride),
                                _p(out))
    return out


def range_attn_f64(q, kc, vc, t0, t1, scale=None):
    """Attention of q [B,Hq,D] over tokens [t0_b, t1_b) of fp64 kc, vc [B,Hkv,N_cap,D]."""
    q = q.contiguous()
    kc = kc.to(torch.float64).contiguous()
    vc = vc.to(torch.float64).contiguous()
    B, Hq, D = q.shape
    _, Hkv, N_cap, _ = kc.shape
    o = torch.empty(B, Hq, D, dtype=torch.float64)
    lse = torch.empty(B, Hq, dtype=torch.float64)
    _load().oracle_range_attn_f64(_p(q), _dt(q), _p(kc), _p(vc), B, Hkv, Hq // Hkv, D, N_cap,
                                  _p(_i32(t0)), _p(_i32(t1)), ctypes.c_double(_scale(scale, D)),
                                  _p(o), _p(lse))
    return o, lse


def window_attn(q, k, v, seqlens, w=512, scale=None):
    """Attention of the decode query over the last w tokens of each sequence."""
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    B, Hq, D = q.shape
    _, Hkv, T_cap, _ = k.shape
    o = torch.empty(B, Hq, D, dtype=torch.float64)
    lse = torch.empty(B, Hq, dtype=torch.float64)
    _load().oracle_window_attn(_p(q), _p(k), _p(v), _dt(q), B, Hkv, Hq // Hkv, D, T_cap,
                               _p(_i32(seqlens)), int(w), ctypes.c_double(_scale(scale, D)),
                               _p(o), _p(lse))
    return o, lse


def nsa_decode(q, k, v, seqlens, topk=16, n_sink=1, n_local=2, gates=(1 / 3, 1 / 3, 1 / 3),
               length=32, stride=16, window=512, blk=64, scale=None, idx=None):
    """NSA's three parallel branches for one decode step, with fixed parts in place of the
    learned ones: the compressed branch (attention over mean-pooled tokens of `length`
    keys at `stride`), the selected branch (the query-aware block selection and sparse
    attention of this oracle; `idx` replaces the oracle's own selection) and the sliding
    window (the last `window` tokens), combined as
        o = gates[0] * o_cmp + gates[1] * o_slc + gates[2] * o_win.
    Returns the branches, the combined o and the tokens each branch reads."""
    B = q.shape[0]
    sl = _i32(seqlens)
    kc = nsa_compress(k, sl, length, stride)
    vc = nsa_compress(v, sl, length, stride)
    nc = torch.tensor([-(-int(t) // stride) for t in sl], dtype=torch.int32)
    o_cmp, lse_cmp = range_attn_f64(q, kc, vc, torch.zeros(B, dtype=torch.int32), nc, scale)
    if idx is None:
        r = decode(q, k, v, sl, topk, n_sink, n_local, blk, scale)
        idx, nsel = r["idx"], r["nsel"]
        o_slc, lse_slc = r["o"], r["lse"]
    else:
        idx = _i32(idx)
        nsel = (idx >= 0).sum(-1).to(torch.int32)
        o_slc, lse_slc = decode_attn(q, k, v, sl, idx, nsel, blk, scale)
    o_win, lse_win = window_attn(q, k, v, sl, window, scale)
    g = [float(x) for x in gates]
    o = g[0] * o_cmp + g[1] * o_slc + g[2] * o_win
    tokens = dict(compressed=[int(x) for x in nc],
                  selected=[[min(blk, int(t) - int(j) * blk) if j >= 0 else 0 for j in row]
                            for row, t in zip(idx[:, 0].tolist(), sl.tolist())],
                  window=[min(window, int(t)) for t in sl])
    return dict(o=o, o_cmp=o_cmp, lse_cmp=lse_cmp, o_slc=o_slc, lse_slc=lse_slc, o_win=o_win,
                lse_win=lse_win, idx=idx, nsel=nsel, kc=kc, vc=vc, tokens=tokens)


def block_scores_weighted(q, summ, seqlens, w, blk=64, scale=None):
    """Group block scores with per-dimension weights w [D]:
    s[b,g,j] = scale * sum_{h in g} sum_d w_d q[b,h,d] summ[b,g,j,d]."""
    q = q.contiguous()
    summ = summ.to(torch.float64).contiguous()
    w = torch.as_tensor(w, dtype=torch.float64).contiguous()
    B, Hq, D = q.shape
    _, Hkv, NB_cap, _ = summ.shape
    assert w.shape == (D,)
    out = torch.empty(B, Hkv, NB_cap, dtype=torch.float64)
    _load().oracle_block_scores_weighted(_p(q), _dt(q), _p(summ), _p(w), B, Hkv, Hq // Hkv, D,
                                         NB_cap, _p(_i32(seqlens)), blk,
                                         ctypes.c_double(_scale(scale, D)), _p(out))
    return out


def rope_chunk_of_dim(D):
    """Rotary frequency chunk of every head dimension under rotate-half pairing: dims j and
    j + D/2 form chunk j, rotated at frequency theta^(-2j/D)."""
    return torch.cat([torch.arange(D // 2), torch.arange(D // 2)])


def rope_block_attenuation(D, theta=1e4, blk=64):
    """Magnitude left of a unit vector of rotary chunk j after mean pooling over blk
    consecutive positions: |sin(blk * w_j / 2) / (blk * sin(w_j / 2))|, w_j = theta^(-2j/D)
    (the Dirichlet kernel: a constant vector rotating at w_j averaged over blk positions).
    Returns a [D/2] fp64 tensor (1 for a chunk that does not rotate)."""
    j = torch.arange(D // 2, dtype=torch.float64)
    wj = theta ** (-2.0 * j / D)
    half = torch.sin(wj / 2)
    a = torch.abs(torch.sin(blk * wj / 2) / (blk * half))
    return torch.where(half.abs() < 1e-300, torch.ones_like(a), a)


def fasa_weights(D, chunks):
    """0/1 weight per dimension keeping the given rotary chunks (both dims of each)."""
    keep = set(int(c) for c in chunks)
    return torch.tensor([1.0 if int(c) in keep else 0.0 for c in rope_chunk_of_dim(D)],
                        dtype=torch.float64)


def prism_weights(D, theta=1e4, blk=64):
    """Dual-band weights: the high band holds the chunks that turn by more than a full
    period inside one block (w_j > 2 pi / blk: mean pooling cancels them), the low band the
    rest; each band's temperature is the mean attenuation of its chunks under the pool
    (rope_block_attenuation), and every dim of a band is weighted by 1 / temperature, which
    restores the band's pooled magnitude.  Returns (w [D], high-band chunk mask [D/2],
    (tau_high, tau_low))."""
    j = torch.arange(D // 2, dtype=torch.float64)
    wj = theta ** (-2.0 * j / D)
    high = wj > 2 * math.pi / blk
    a = rope_block_attenuation(D, theta, blk)
    tau_hi = float(a[high].mean()) if bool(high.any()) else 1.0
    tau_lo = float(a[~high].mean()) if bool((~high).any()) else 1.0
    per_chunk = torch.where(high, torch.full_like(a, 1 / tau_hi), torch.full_like(a, 1 / tau_lo))
    return per_chunk[rope_chunk_of_dim(D)], high, (tau_hi, tau_lo)
