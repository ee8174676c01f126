"""The bounds-checking build (liblsa_debug.so, built with LSA_DEBUG_BOUNDS): device-side
values that decide where a kernel reads or writes -- sequence lengths, selection indices and
counts -- are checked; the first one out of range is recorded as (kind << 8) | site, the
value is clamped into range, and nothing traps.  These inputs are given only to the debug
build, whose own checks turn them into an error code; the release build trusts them.

The decode and block-query parity suites were also run with LSA_LIBRARY=debug (the package
then loads this build)."""
import ctypes
import os

import pytest
import torch

import oracle
import synth
from tests.parity import LSE_TOL, TOL, max_abs, nsel_of

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEBUG_LIB = os.path.join(ROOT, "query_aware_block_b200", "liblsa_debug.so")
SEQLEN, INDEX, COUNT = 1, 2, 3
SITE_DECODE = 2


@pytest.fixture(scope="module")
def libs(cuda_device):
    import query_aware_block_b200 as lsa
    if not os.path.exists(DEBUG_LIB):
        pytest.skip("liblsa_debug.so not built (python query_aware_block_b200/_build.py --debug-bounds)")
    dbg = ctypes.CDLL(DEBUG_LIB)
    rel = lsa.library()
    for n in lsa.EXPORTED:
        f = getattr(dbg, n)
        f.argtypes = getattr(rel, n).argtypes
        f.restype = getattr(rel, n).restype
    return lsa, dbg


def _code(dbg, reset=True):
    c = ctypes.c_int(0)
    assert dbg.lsa_debug_bounds_code(ctypes.byref(c), int(reset)) == 0
    return c.value


def _decode(lsa, lib, q, k, v, sl, summ, topk, idx=None, nsel=None):
    B, Hq, D = q.shape
    Hkv, T_cap = k.shape[1], k.shape[2]
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, device=q.device)
    idx_out = torch.empty(B, Hkv, topk, dtype=torch.int32, device=q.device)
    st = lib.lsa_sparse_attn_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), lsa.LSA_BF16, B, Hkv, Hq // Hkv, D,
                                    T_cap, sl.data_ptr(), 64, None if idx is None else idx.data_ptr(),
                                    None if nsel is None else nsel.data_ptr(), topk, 0.0,
                                    None if idx is not None else summ.data_ptr(), 1, 2, 0,
                                    None if idx is not None else idx_out.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                    0, torch.cuda.current_stream().cuda_stream)
    assert st == 0, st
    torch.cuda.synchronize()
    return o, lse, idx_out


def test_release_build_reports_no_bounds_checks(libs):
    lsa, _ = libs
    # (the release library by its path: with LSA_LIBRARY=debug the package itself loads the
    # debug build)
    rel = ctypes.CDLL(os.path.join(ROOT, "query_aware_block_b200", "liblsa.so"))
    rel.lsa_debug_bounds_code.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_int]
    rel.lsa_debug_bounds_code.restype = ctypes.c_int
    c = ctypes.c_int(7)
    assert rel.lsa_debug_bounds_code(ctypes.byref(c), 0) == lsa.LSA_ERR_UNSUPPORTED
    assert c.value == 0


def test_sequence_length_past_capacity_is_recorded_and_clamped(libs):
    lsa, dbg = libs
    T_cap = 64 * 20
    case = synth.decode_case(B=2, Hkv=2, G=4, D=128, T_cap=T_cap, seqlens=[T_cap, 500], dtype=torch.bfloat16,
                             topk=8, n_sink=1, n_local=2, seed=301)
    d = torch.device("cuda:0")
    q, k, v, sl = case.q.to(d), case.k.to(d), case.v.to(d), case.seqlens.to(d)
    summ = torch.zeros(2, 2, 20, 128, device=d)
    lsa.lsa_build_summaries(k, sl, summ)
    _code(dbg)  # clear
    # valid lengths: no code, the oracle's answer
    o, lse, idx = _decode(lsa, dbg, q, k, v, sl, summ, 8)
    assert _code(dbg) == 0
    idx_c = idx.cpu()
    o_ref, lse_ref = oracle.decode_attn(case.q, case.k, case.v, case.seqlens, idx_c, nsel_of(idx_c))
    assert max_abs(o.float().cpu(), o_ref) <= TOL[torch.bfloat16]
    # a length past the capacity: recorded as (seqlen, decode) and clamped to T_cap
    bad = torch.tensor([T_cap + 100, 500], dtype=torch.int32, device=d)
    o2, lse2, idx2 = _decode(lsa, dbg, q, k, v, bad, summ, 8)
    assert _code(dbg) == (SEQLEN << 8) | SITE_DECODE
    assert torch.equal(idx2.cpu(), idx_c)
    assert max_abs(o2.float().cpu(), o_ref) <= TOL[torch.bfloat16]
    assert max_abs(lse2.cpu(), lse_ref) <= LSE_TOL[torch.bfloat16]


def test_selection_index_and_count_out_of_range_are_recorded(libs):
    lsa, dbg = libs
    T_cap = 64 * 20
    case = synth.decode_case(B=1, Hkv=2, G=4, D=128, T_cap=T_cap, seqlens=T_cap, dtype=torch.bfloat16,
                             topk=8, n_sink=1, n_local=2, seed=302)
    d = torch.device("cuda:0")
    q, k, v, sl = case.q.to(d), case.k.to(d), case.v.to(d), case.seqlens.to(d)
    r = oracle.decode(case.q, case.k, case.v, case.seqlens, 8, 1, 2)
    idx, nsel = r["idx"].clone(), r["nsel"].clone()
    _code(dbg)
    idx_bad = idx.clone()
    idx_bad[0, 1, 3] = 20 + 5  # past the sequence's 20 blocks
    _decode(lsa, dbg, q, k, v, sl, None, 8, idx=idx_bad.to(d), nsel=nsel.to(d))
    assert _code(dbg) == (INDEX << 8) | SITE_DECODE
    nsel_bad = nsel.clone()
    nsel_bad[0, 0] = 99  # more than topk
    _decode(lsa, dbg, q, k, v, sl, None, 8, idx=idx.to(d), nsel=nsel_bad.to(d))
    assert _code(dbg) == (COUNT << 8) | SITE_DECODE
    st = ctypes.c_int(0)
    assert dbg.lsa_device_status(ctypes.byref(st), 1) == 0
    assert st.value == 0  # no timeout; the bounds word was cleared above
