"""The C ABI boundary on the CPU: liblsa.so loads, exports every entry point that
include/lsa.h declares, and rejects bad arguments on the host before any launch (so these
calls are safe without a GPU: none of them reaches a CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsa.h")


def _declared():
    text = open(HEADER).read()
    return re.findall(r"LSA_API\s+[\w\s\*]+?\b(lsa_\w+)\s*\(", text)


def test_header_declares_the_five_entry_points():
    names = _declared()
    for n in ("lsa_build_summaries", "lsa_select_blocks", "lsa_sparse_attn_decode",
              "lsa_sparse_attn_blockquery", "lsa_blasst_prefill"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import query_aware_block_b200 as lsa
    lib = ctypes.CDLL(lsa.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(lsa.EXPORTED) == set(_declared())


def test_status_strings_and_version():
    import query_aware_block_b200 as lsa
    lib = lsa.library()
    assert lib.lsa_status_string(0) == b"LSA_OK"
    for s in (1, 2, 3, 4):
        assert lib.lsa_status_string(s).startswith(b"LSA_ERR")
    assert lib.lsa_status_string(99) == b"unknown lsa status"
    assert lsa.lsa_version() >= 100


NULL = None


def test_build_summaries_validation():
    import query_aware_block_b200 as lsa
    f = lsa.library().lsa_build_summaries
    good = ctypes.c_void_p(4096)
    # dtype, head dim, block size
    assert f(good, 7, 1, 1, 64, 128, good, 64, 0, -1, good, NULL) == lsa.LSA_ERR_UNSUPPORTED
    assert f(good, 1, 1, 1, 64, 96, good, 64, 0, -1, good, NULL) == lsa.LSA_ERR_UNSUPPORTED
    assert f(good, 1, 1, 1, 64, 128, good, 32, 0, -1, good, NULL) == lsa.LSA_ERR_UNSUPPORTED
    # null / misaligned pointers
    assert f(NULL, 1, 1, 1, 64, 128, good, 64, 0, -1, good, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(4098), 1, 1, 1, 64, 128, good, 64, 0, -1, good, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert f(good, 1, -1, 1, 64, 128, good, 64, 0, -1, good, NULL) == lsa.LSA_ERR_INVALID_ARG
    # empty problems are a successful no-op, nothing launched
    assert f(NULL, 1, 0, 1, 64, 128, NULL, 64, 0, -1, NULL, NULL) == lsa.LSA_OK
    assert f(good, 1, 1, 1, 64, 128, good, 64, 5, 3, good, NULL) == lsa.LSA_OK  # empty range


def test_select_and_decode_validation():
    import query_aware_block_b200 as lsa
    lib = lsa.library()
    g = ctypes.c_void_p(4096)
    sel = lib.lsa_select_blocks
    # topk range, forced count larger than topk, G > 16
    assert sel(g, 1, g, 1, 8, 8, 128, 1024, g, 64, 0, 1, 2, 0.0, g, g, NULL, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert sel(g, 1, g, 1, 8, 8, 128, 1024, g, 64, 65, 1, 2, 0.0, g, g, NULL, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert sel(g, 1, g, 1, 8, 8, 128, 1024, g, 64, 2, 1, 2, 0.0, g, g, NULL, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert sel(g, 1, g, 1, 8, 17, 128, 1024, g, 64, 16, 1, 2, 0.0, g, g, NULL, NULL) == lsa.LSA_ERR_UNSUPPORTED
    assert sel(g, 1, g, 1, 8, 8, 128, 1024, g, 64, 16, 1, 2, 0.0, NULL, g, NULL, 0, NULL) == lsa.LSA_ERR_INVALID_ARG
    dec = lib.lsa_sparse_attn_decode
    # fused mode (idx NULL) needs summaries; given mode needs nsel
    assert dec(g, g, g, 1, 1, 8, 8, 128, 65536, g, 64, NULL, NULL, 16, 0.0, NULL, 1, 2, 0, NULL, g, NULL, 0, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert dec(g, g, g, 1, 1, 8, 8, 128, 65536, g, 64, g, NULL, 16, 0.0, NULL, 1, 2, 0, NULL, g, NULL, 0, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert dec(g, g, g, 1, 1, 8, 8, 128, 1 << 22, g, 64, g, g, 16, 0.0, NULL, 1, 2, 0, NULL, g, NULL, 0, NULL) == lsa.LSA_ERR_UNSUPPORTED
    assert dec(g, g, NULL, 1, 1, 8, 8, 128, 65536, g, 64, g, g, 16, 0.0, NULL, 1, 2, 0, NULL, g, NULL, 0, NULL) == lsa.LSA_ERR_INVALID_ARG
    # the refreshed last block must be forced (n_local >= 1), and only in fused mode
    assert dec(g, g, g, 1, 1, 8, 8, 128, 65536, g, 64, NULL, NULL, 16, 0.0, g, 1, 0, 1, NULL, g, NULL, 0, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert dec(g, g, g, 1, 1, 8, 8, 128, 65536, g, 64, g, g, 16, 0.0, g, 1, 2, 1, NULL, g, NULL, 0, NULL) == lsa.LSA_ERR_INVALID_ARG
    # overlapped launch only in fused mode; unknown flags rejected
    assert dec(g, g, g, 1, 1, 8, 8, 128, 65536, g, 64, g, g, 16, 0.0, NULL, 1, 2, 0, NULL, g, NULL, 1, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert dec(g, g, g, 1, 1, 8, 8, 128, 65536, g, 64, NULL, NULL, 16, 0.0, g, 1, 2, 0, NULL, g, NULL, 2, NULL) == lsa.LSA_ERR_INVALID_ARG
    # B or Hkv past a grid dimension
    assert dec(g, g, g, 1, 65536, 1, 8, 128, 4096, g, 64, NULL, NULL, 16, 0.0, g, 1, 2, 0, NULL, g, NULL, 0, NULL) == lsa.LSA_ERR_UNSUPPORTED
    assert sel(g, 1, g, 1, 65536, 8, 128, 64, g, 64, 16, 1, 2, 0.0, g, g, NULL, NULL) == lsa.LSA_ERR_UNSUPPORTED
    assert lib.lsa_build_summaries(g, 1, 1, 65536, 4096, 128, g, 64, 0, -1, g, NULL) == lsa.LSA_ERR_UNSUPPORTED


def test_losa_entry_points_validation():
    import query_aware_block_b200 as lsa
    lib = lsa.library()
    g = ctypes.c_void_p(4096)
    cls = lib.lsa_losa_classify
    assert cls(g, g, 0, 1, 32, 32, 128, 0.1, 0, g, NULL, NULL) == lsa.LSA_ERR_UNSUPPORTED  # fp32
    assert cls(g, g, 1, 1, 32, 65, 128, 0.1, 0, g, NULL, NULL) == lsa.LSA_ERR_UNSUPPORTED  # Tq > 64
    assert cls(g, g, 1, 1, 32, 32, 96, 0.1, 0, g, NULL, NULL) == lsa.LSA_ERR_UNSUPPORTED   # D
    assert cls(g, g, 1, 1, 32, 32, 128, 0.1, -1, g, NULL, NULL) == lsa.LSA_ERR_INVALID_ARG  # n_top
    assert cls(g, g, 1, 1, 32, 32, 128, float("nan"), 0, g, NULL, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert cls(g, NULL, 1, 1, 32, 32, 128, 0.1, 0, g, NULL, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert cls(g, g, 1, 1, 32, 32, 128, 0.1, 0, g, ctypes.c_void_p(4100), NULL) == lsa.LSA_ERR_INVALID_ARG
    assert cls(NULL, NULL, 1, 0, 32, 32, 128, 0.1, 0, NULL, NULL, NULL) == lsa.LSA_OK  # empty batch
    im = lib.lsa_blockquery_intra_merge
    big = 1 << 30
    # the block must fit behind the prefix: T_prefix + Tq <= T_cap
    assert im(g, g, g, 1, 1, 8, 4, 128, 32, 100, 131, 0.0, g, g, ctypes.c_void_p(big), g, 0, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert im(g, g, g, 1, 1, 8, 4, 128, 65, 100, 1000, 0.0, g, g, ctypes.c_void_p(big), g, 0, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert im(g, g, g, 0, 1, 8, 4, 128, 32, 100, 1000, 0.0, g, g, ctypes.c_void_p(big), g, 0, NULL) == lsa.LSA_ERR_UNSUPPORTED
    assert im(g, g, g, 1, 1, 8, 4, 128, 32, 100, 1000, 0.0, g, g, ctypes.c_void_p(big), g, 2, NULL) == lsa.LSA_ERR_INVALID_ARG
    # o overlapping o_pre without being it
    assert im(g, g, g, 1, 1, 8, 4, 128, 32, 100, 1000, 0.0, g, g, ctypes.c_void_p(4096 + 256), g, 0, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert im(g, g, g, 1, 0, 8, 4, 128, 32, 100, 1000, 0.0, NULL, NULL, NULL, NULL, 0, NULL) == lsa.LSA_OK
    bq = lib.lsa_sparse_attn_blockquery
    # topk_per_query in (16, NBp) is rejected (>= NBp, every prefix block, is the dense step)
    args = lambda topk, T: (g, g, g, 1, 1, 8, 4, 128, 32, T, T + 32, g, 64, topk, 0, 0, 0.0, g, g, g, g, g, NULL, NULL, g, 0, NULL)
    assert bq(*args(17, 64 * 100)) == lsa.LSA_ERR_INVALID_ARG
    assert bq(*args(0, 64 * 100)) == lsa.LSA_ERR_INVALID_ARG
    # o / lse may be o_cache / lse_cache, but must not overlap them partially
    ws = 1 << 30
    over = lambda o, lse: (g, g, g, 1, 1, 8, 4, 128, 32, 6400, 6432, g, 64, 8, 1, 2, 0.0, g,
                           g, g, o, lse, NULL, NULL, g, ws, NULL)
    assert bq(*over(ctypes.c_void_p(4096 + 256), ctypes.c_void_p(big))) == lsa.LSA_ERR_INVALID_ARG
    assert bq(*over(ctypes.c_void_p(big), ctypes.c_void_p(4096 + 4))) == lsa.LSA_ERR_INVALID_ARG
    # more sequences than a grid dimension holds
    assert bq(g, g, g, 1, 65536, 1, 4, 128, 8, 6400, 6432, g, 64, 8, 1, 2, 0.0, g, g, g,
              ctypes.c_void_p(big), ctypes.c_void_p(big), NULL, NULL, g, 1 << 62, NULL) == lsa.LSA_ERR_UNSUPPORTED


def test_decode_blasst_validation():
    import query_aware_block_b200 as lsa
    f = lsa.library().lsa_sparse_attn_decode_blasst
    g = ctypes.c_void_p(4096)
    args = lambda dtype=1, D=128, topk=16, lam=1e-3, G=8: (g, g, g, dtype, 1, 8, G, D, 65536, g, 64, g, g, topk, 0.0, lam, g, NULL, NULL, NULL)
    assert f(*args(dtype=0)) == lsa.LSA_ERR_UNSUPPORTED      # fp32
    assert f(*args(D=96)) == lsa.LSA_ERR_UNSUPPORTED
    assert f(*args(G=17)) == lsa.LSA_ERR_UNSUPPORTED
    assert f(*args(topk=17)) == lsa.LSA_ERR_INVALID_ARG      # one cluster slot per block
    assert f(*args(topk=0)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(lam=1.0)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(lam=-0.1)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(lam=float("nan"))) == lsa.LSA_ERR_INVALID_ARG
    bad = list(args())
    bad[11] = NULL  # idx
    assert f(*bad) == lsa.LSA_ERR_INVALID_ARG
    assert f(g, g, g, 1, 0, 8, 8, 128, 65536, NULL, 64, NULL, NULL, 16, 0.0, 1e-3, NULL, NULL, NULL, NULL) == lsa.LSA_OK


def test_nsa_entry_points_validation():
    import query_aware_block_b200 as lsa
    lib = lsa.library()
    g = ctypes.c_void_p(4096)
    cmp_ = lib.lsa_nsa_compress
    assert cmp_(g, g, 0, 1, 8, 65536, 128, g, 32, 16, 0, -1, g, g, NULL) == lsa.LSA_ERR_UNSUPPORTED  # fp32
    assert cmp_(g, g, 1, 1, 8, 65536, 96, g, 32, 16, 0, -1, g, g, NULL) == lsa.LSA_ERR_UNSUPPORTED  # D
    assert cmp_(g, g, 1, 1, 8, 65536, 128, g, 0, 16, 0, -1, g, g, NULL) == lsa.LSA_ERR_INVALID_ARG  # len
    assert cmp_(g, g, 1, 1, 8, 65536, 128, g, 32, 0, 0, -1, g, g, NULL) == lsa.LSA_ERR_INVALID_ARG  # stride
    assert cmp_(g, g, 1, 1, 8, 65536, 128, g, 32, 16, 0, -1, NULL, g, NULL) == lsa.LSA_ERR_INVALID_ARG
    assert cmp_(g, g, 1, 1, 8, 65536, 128, g, 32, 16, 5000, 4000, g, g, NULL) == lsa.LSA_OK  # empty range
    assert cmp_(g, g, 1, 0, 8, 65536, 128, NULL, 32, 16, 0, -1, NULL, NULL, NULL) == lsa.LSA_OK
    br = lib.lsa_nsa_branches
    args = lambda **kw: [kw.get(n, d) for n, d in (
        ("q", g), ("k", g), ("v", g), ("kc", g), ("vc", g), ("dtype", 1), ("B", 1), ("Hkv", 8),
        ("G", 8), ("D", 128), ("T_cap", 65536), ("sl", g), ("window", 512), ("stride", 16),
        ("scale", 0.0), ("gc", 1 / 3), ("gs", 1 / 3), ("gw", 1 / 3), ("oslc", NULL), ("o", g),
        ("lw", NULL), ("lc", NULL), ("stream", NULL))]
    assert br(*args(dtype=0)) == lsa.LSA_ERR_UNSUPPORTED
    assert br(*args(G=17)) == lsa.LSA_ERR_UNSUPPORTED
    assert br(*args(window=-1)) == lsa.LSA_ERR_INVALID_ARG
    assert br(*args(stride=0)) == lsa.LSA_ERR_INVALID_ARG
    assert br(*args(gc=float("nan"))) == lsa.LSA_ERR_INVALID_ARG
    assert br(*args(kc=NULL)) == lsa.LSA_ERR_INVALID_ARG
    assert br(*args(o=ctypes.c_void_p(4100))) == lsa.LSA_ERR_INVALID_ARG
    assert br(*args(B=0, q=NULL, o=NULL)) == lsa.LSA_OK


def test_weighted_select_validation():
    import query_aware_block_b200 as lsa
    f = lsa.library().lsa_select_blocks_weighted
    g = ctypes.c_void_p(4096)
    args = lambda **kw: [kw.get(n, d) for n, d in (
        ("q", g), ("dtype", 1), ("summ", g), ("w", g), ("B", 1), ("Hkv", 8), ("G", 8), ("D", 128),
        ("NB", 1024), ("sl", g), ("blk", 64), ("topk", 16), ("ns", 1), ("nl", 2), ("scale", 0.0),
        ("qw", g), ("idx", g), ("nsel", g), ("sc", NULL), ("stream", NULL))]
    assert f(*args(w=NULL)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(qw=NULL)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(qw=ctypes.c_void_p(4100))) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(topk=0)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(ns=10, nl=10)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(D=96)) == lsa.LSA_ERR_UNSUPPORTED
    assert f(*args(blk=32)) == lsa.LSA_ERR_UNSUPPORTED
    assert f(*args(B=0, q=NULL, w=NULL, qw=NULL)) == lsa.LSA_OK
    # q_weighted (fp32, B*Hq*D*4 bytes) may not overlap a bf16 q, nor partly overlap an fp32
    # q, nor overlap the weights (q and w far apart here; each call stops at the overlap check)
    far = ctypes.c_void_p(1 << 30)
    assert f(*args(q=g, qw=g, w=far)) == lsa.LSA_ERR_INVALID_ARG                       # bf16 q
    assert f(*args(q=g, qw=ctypes.c_void_p(4096 + 4096), w=far)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(dtype=0, q=g, qw=ctypes.c_void_p(4096 + 256), w=far)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(q=far, qw=g, w=ctypes.c_void_p(4096 + 512))) == lsa.LSA_ERR_INVALID_ARG


def test_binding_raises_lsa_error_on_bad_arguments():
    import torch
    import query_aware_block_b200 as lsa
    k = torch.zeros(1, 1, 64, 96)  # D = 96 unsupported; rejected before any launch
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_build_summaries(k, torch.zeros(1, dtype=torch.int32), torch.zeros(1, 1, 1, 96), stream=0)
    assert e.value.status == lsa.LSA_ERR_UNSUPPORTED


def test_binding_argtypes_match_header_parameter_counts():
    # every ctypes prototype has exactly as many arguments as the C declaration
    import query_aware_block_b200 as lsa
    text = open(HEADER).read()
    lib = lsa.library()
    for name in _declared():
        m = re.search(r"LSA_API[^;]*?\b" + name + r"\s*\(([^)]*)\)", text)
        params = m.group(1).strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        argt = getattr(lib, name).argtypes
        assert argt is not None and len(argt) == n, (name, n, argt and len(argt))


def test_append_kv_validation():
    import query_aware_block_b200 as lsa
    f = lsa.library().lsa_append_kv
    g = ctypes.c_void_p(4096)
    args = lambda **kw: [kw.get(n, d) for n, d in (
        ("kn", g), ("vn", g), ("dtype", 1), ("B", 1), ("Hkv", 8), ("T", 65536), ("D", 128),
        ("sl", g), ("k", g), ("v", g), ("flags", 0), ("stream", NULL))]
    assert f(*args(kn=NULL)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(v=ctypes.c_void_p(4104))) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(flags=4)) == lsa.LSA_ERR_INVALID_ARG  # unknown flag
    assert f(*args(T=-1)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(D=96)) == lsa.LSA_ERR_UNSUPPORTED
    assert f(*args(dtype=5)) == lsa.LSA_ERR_UNSUPPORTED
    assert f(*args(B=0, kn=NULL, vn=NULL, k=NULL, v=NULL, sl=NULL)) == lsa.LSA_OK



def test_copy_async_validation():
    import query_aware_block_b200 as lsa
    f = lsa.library().lsa_copy_async
    a, b = ctypes.c_void_p(4096), ctypes.c_void_p(8192)
    assert f(a, b, 0, 0, NULL) == lsa.LSA_OK  # nothing to copy: nothing enqueued
    assert f(a, b, 24, 0, NULL) == lsa.LSA_ERR_INVALID_ARG  # not a multiple of 16 bytes
    assert f(ctypes.c_void_p(4104), b, 32, 0, NULL) == lsa.LSA_ERR_INVALID_ARG  # misaligned
    assert f(a, ctypes.c_void_p(4112), 32, 0, NULL) == lsa.LSA_ERR_INVALID_ARG  # overlapping
    assert f(a, b, 32, 4, NULL) == lsa.LSA_ERR_INVALID_ARG  # unknown flag
    assert f(NULL, b, 32, 0, NULL) == lsa.LSA_ERR_INVALID_ARG


def test_append_kv_stage_q_validation():
    import query_aware_block_b200 as lsa
    f = lsa.library().lsa_append_kv_stage_q
    g = ctypes.c_void_p(4096)
    args = lambda **kw: [kw.get(n, d) for n, d in (
        ("qs", ctypes.c_void_p(1 << 20)), ("qd", ctypes.c_void_p(2 << 20)), ("qb", 4096), ("kn", g),
        ("vn", g), ("dtype", 1), ("B", 1), ("Hkv", 8), ("T", 65536), ("D", 128), ("sl", g), ("k", g),
        ("v", g), ("flags", 0), ("stream", NULL))]
    assert f(*args(qb=24)) == lsa.LSA_ERR_INVALID_ARG           # not a multiple of 16 bytes
    assert f(*args(qs=NULL)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(qd=ctypes.c_void_p((1 << 20) + 16))) == lsa.LSA_ERR_INVALID_ARG  # overlapping
    assert f(*args(kn=NULL)) == lsa.LSA_ERR_INVALID_ARG
    assert f(*args(flags=4)) == lsa.LSA_ERR_INVALID_ARG  # unknown flag
    assert f(*args(D=96)) == lsa.LSA_ERR_UNSUPPORTED
    assert f(*args(qb=0, B=0, kn=NULL, vn=NULL, k=NULL, v=NULL, sl=NULL)) == lsa.LSA_OK


def test_debug_controls_validate_without_a_gpu():
    import query_aware_block_b200 as lsa
    lib = lsa.library()
    assert lib.lsa_debug_inject(7) == lsa.LSA_ERR_INVALID_ARG
    assert lib.lsa_debug_inject(0) == lsa.LSA_OK
    assert lib.lsa_debug_set_wait_budget(0) == lsa.LSA_OK  # restores the default
