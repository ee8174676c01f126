"""The block-query entry point for callers that may not allocate device memory.

lsa_sparse_attn_blockquery_noalloc keeps the scratch of the block-query split in one fixed
device array inside the library instead of a caller workspace, for code that must not
call cudaMalloc (or anything that allocates).  These tests call it through the raw C ABI
and check it against lsa_sparse_attn_blockquery with a caller workspace, on two calls in a
row with different inputs (the fixed array keeps the previous call's contents, which must
not leak into the next result).  This file is collected last on purpose."""
import ctypes

import pytest
import torch

import synth
from tests.parity import LSE_TOL, TOL, max_abs


def _inputs(case, d):
    B, Hq, Tq, D = case.q.shape
    Hkv = case.k.shape[1]
    T_cap = case.k.shape[2]
    t = dict(q=case.q.to(d), k=case.k.to(d), v=case.v.to(d), active=case.active.to(d),
             oc=case.o_cache.to(d), lc=case.lse_cache.to(d))
    t["sl"] = torch.full((B,), T_cap, dtype=torch.int32, device=d)
    t["summ"] = torch.zeros(B, Hkv, -(-T_cap // 64), D, device=d)
    return t


def _call(lib, fn, case, t, ws=None):
    """One raw C-ABI call; returns (status, o, lse, union_idx, union_cnt)."""
    B, Hq, Tq, D = case.q.shape
    Hkv = case.k.shape[1]
    T_cap = case.k.shape[2]
    NBp = -(-case.T_prefix // 64)
    o = torch.full_like(t["oc"], 5.0)
    lse = torch.full_like(t["lc"], 5.0)
    ui = torch.full((B, Hkv, NBp), -9, dtype=torch.int32, device=o.device)
    uc = torch.full((B, Hkv), -9, dtype=torch.int32, device=o.device)
    args = [t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), 1, B, Hkv, Hq // Hkv, D, Tq,
            case.T_prefix, T_cap, t["summ"].data_ptr(), 64, case.topk, case.n_sink,
            case.n_local, ctypes.c_float(0.0), t["active"].data_ptr(), t["oc"].data_ptr(),
            t["lc"].data_ptr(), o.data_ptr(), lse.data_ptr(), ui.data_ptr(), uc.data_ptr()]
    if ws is not None:
        args += [ws.data_ptr(), ctypes.c_size_t(ws.numel())]
    args.append(torch.cuda.current_stream().cuda_stream)
    st = fn(*args)
    torch.cuda.synchronize()
    return st, o.cpu(), lse.cpu(), ui.cpu(), uc.cpu()


@pytest.mark.gpu
def test_noalloc_blockquery_matches_workspace_variant_twice(cuda_device):
    import query_aware_block_b200 as lsa
    lib = lsa.library()
    cases = [
        synth.blockquery_case(B=1, Hkv=8, G=4, D=128, Tq=32, T_prefix=32768, n_active=8, topk=8,
                              seed=61),
        synth.blockquery_case(B=2, Hkv=2, G=4, D=128, Tq=16, T_prefix=64 * 200 + 5,
                              T_cap=64 * 201, n_active=11, topk=6, n_sink=1, n_local=1, seed=62),
    ]
    for i, case in enumerate(cases):  # two calls in a row, different inputs and shapes
        t = _inputs(case, cuda_device)
        lsa.lsa_build_summaries(t["k"], t["sl"], t["summ"])
        B, Hq, Tq, D = case.q.shape
        Hkv = case.k.shape[1]
        ws = torch.empty(lsa.lsa_blockquery_workspace_size(B, Hkv, Hq // Hkv, D, Tq),
                         dtype=torch.uint8, device=cuda_device)
        st_ref, o_ref, lse_ref, ui_ref, uc_ref = _call(lib, lib.lsa_sparse_attn_blockquery, case,
                                                       t, ws)
        st, o, lse, ui, uc = _call(lib, lib.lsa_sparse_attn_blockquery_noalloc, case, t)
        assert st_ref == 0 and st == 0, (i, st_ref, st)
        assert torch.equal(ui, ui_ref) and torch.equal(uc, uc_ref), f"call {i}: union differs"
        assert max_abs(o.float(), o_ref.float()) <= TOL[torch.bfloat16], f"call {i}: o"
        assert max_abs(lse, lse_ref) <= LSE_TOL[torch.bfloat16], f"call {i}: lse"


def test_noalloc_blockquery_rejects_shapes_beyond_the_fixed_scratch():
    # 1 x 8 KV heads x 16 q heads x 64 tokens x D 128 needs about 68 MB of partials, more
    # than the fixed 16 MiB: rejected on the host before any device work
    import query_aware_block_b200 as lsa
    lib = lsa.library()
    g = ctypes.c_void_p(4096)
    st = lib.lsa_sparse_attn_blockquery_noalloc(g, g, g, 1, 1, 8, 16, 128, 64, 4096, 4096, g, 64,
                                                8, 0, 0, ctypes.c_float(0.0), g, g, g, g, g,
                                                None, None, None)
    assert st == lsa.LSA_ERR_UNSUPPORTED
    assert lsa.lsa_blockquery_workspace_size(1, 8, 16, 128, 64) > 16 * 2 ** 20
