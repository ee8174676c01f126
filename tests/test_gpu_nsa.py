"""GPU parity of NSA's compressed and sliding-window branches (fixed mean pool, constant
gates) against the fp64 oracle, through the C ABI: the pool (bf16 output: the bound is on
the error beyond its own rounding), the decode-time refresh of the last compressed tokens,
and the three-branch output of a decode step (the selected branch from the fused decode,
the oracle evaluated on the GPU's own selection) on the 64K decode workload, ragged
batches (sequences shorter than the window and than a compression block), D 64, and
gates that isolate one branch."""
import pytest
import torch

import oracle
import synth
from tests.parity import LSE_TOL, TOL, max_abs, max_abs_beyond_rounding

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def lsa(cuda_device):
    import query_aware_block_b200 as m
    return m


def _gpu_compress(lsa, k, v, sl, length=32, stride=16, nc_begin=0, kc=None, vc=None):
    B, Hkv, T_cap, D = k.shape
    NC_cap = -(-T_cap // stride)
    if kc is None:
        kc = torch.full((B, Hkv, NC_cap, D), 7.0, dtype=torch.bfloat16, device=DEV)
        vc = torch.full((B, Hkv, NC_cap, D), 7.0, dtype=torch.bfloat16, device=DEV)
    lsa.lsa_nsa_compress(k, v, sl, kc, vc, length=length, stride=stride, nc_begin=nc_begin)
    return kc, vc


@pytest.mark.parametrize("kw", [
    dict(B=2, Hkv=2, D=128, T_cap=1200, seqlens=[1200, 333], length=32, stride=16),
    dict(B=3, Hkv=1, D=64, T_cap=700, seqlens=[700, 20, 64], length=32, stride=16),
    dict(B=1, Hkv=2, D=128, T_cap=1000, seqlens=[1000], length=64, stride=64),   # = block summaries
    dict(B=1, Hkv=1, D=128, T_cap=500, seqlens=[500], length=48, stride=16),
])
def test_nsa_compress_matches_oracle(lsa, kw):
    kw = dict(kw)
    length, stride = kw.pop("length"), kw.pop("stride")
    case = synth.decode_case(dtype=torch.bfloat16, G=1, topk=4, n_sink=0, n_local=0, seed=101, **kw)
    k, v, sl = case.k.to(DEV), case.v.to(DEV), case.seqlens.to(DEV)
    kc, vc = _gpu_compress(lsa, k, v, sl, length, stride)
    torch.cuda.synchronize()
    kr = oracle.nsa_compress(case.k, case.seqlens, length, stride)
    vr = oracle.nsa_compress(case.v, case.seqlens, length, stride)
    assert max_abs_beyond_rounding(kc.cpu(), kr) <= 1e-5, kw
    assert max_abs_beyond_rounding(vc.cpu(), vr) <= 1e-5, kw


def test_nsa_compress_refresh_of_the_last_tokens(lsa):
    # a decode step appends token T: only the last 2 compressed tokens (l = 32, d = 16)
    # change, and refreshing them equals rebuilding everything
    case = synth.decode_case(B=2, Hkv=2, G=1, D=128, T_cap=1024, seqlens=[1000, 777],
                             dtype=torch.bfloat16, topk=4, n_sink=0, n_local=0, seed=102)
    k, v = case.k.to(DEV), case.v.to(DEV)
    sl = case.seqlens.to(DEV)
    kc, vc = _gpu_compress(lsa, k, v, sl)
    sl2 = sl + 1
    g = torch.Generator(device="cpu").manual_seed(5)
    for b in range(2):
        t = int(case.seqlens[b])
        k[b, :, t] = torch.randn(2, 128, generator=g).to(torch.bfloat16).to(DEV)
        v[b, :, t] = torch.randn(2, 128, generator=g).to(torch.bfloat16).to(DEV)
    _gpu_compress(lsa, k, v, sl2, nc_begin=-2, kc=kc, vc=vc)
    full_k, full_v = _gpu_compress(lsa, k, v, sl2)
    torch.cuda.synchronize()
    assert torch.equal(kc.cpu(), full_k.cpu()) and torch.equal(vc.cpu(), full_v.cpu())


def _nsa_gpu(lsa, case, topk, gates, window=512, stride=16, with_slc=True):
    q, k, v, sl = (t.to(DEV) for t in (case.q, case.k, case.v, case.seqlens))
    B, Hq, D = q.shape
    Hkv, T_cap = k.shape[1], k.shape[2]
    summ = torch.zeros(B, Hkv, -(-T_cap // 64), D, device=DEV)
    lsa.lsa_build_summaries(k, sl, summ)
    o_slc = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=DEV)
    idx = torch.empty(B, Hkv, topk, dtype=torch.int32, device=DEV)
    lsa.lsa_sparse_attn_decode(q, k, v, sl, o_slc, topk, summ=summ, n_sink=1, n_local=2, idx_out=idx)
    kc, vc = _gpu_compress(lsa, k, v, sl, 32, stride)
    o = torch.full((B, Hq, D), 7.0, dtype=torch.bfloat16, device=DEV)
    lw = torch.full((B, Hq), 7.0, device=DEV)
    lc = torch.full((B, Hq), 7.0, device=DEV)
    lsa.lsa_nsa_branches(q, k, v, kc, vc, sl, o, gates=gates, o_slc=o_slc if with_slc else None,
                         window=window, stride=stride, lse_win=lw, lse_cmp=lc)
    torch.cuda.synchronize()
    assert lsa.lsa_device_status() == 0
    return o.cpu(), lw.cpu(), lc.cpu(), idx.cpu(), o_slc.cpu()


def _check(case, gates, window, o, lw, lc, idx, o_slc, with_slc=True, where=""):
    # the oracle on the GPU's own selection (the index set the decode tests check)
    r = oracle.nsa_decode(case.q, case.k, case.v, case.seqlens, gates=gates, window=window,
                          idx=idx)
    ref = r["o"] if with_slc else gates[0] * r["o_cmp"] + gates[2] * r["o_win"]
    assert max_abs_beyond_rounding(o, ref) <= TOL[torch.bfloat16], where
    assert max_abs(lw, r["lse_win"]) <= LSE_TOL[torch.bfloat16], where
    assert max_abs(lc, r["lse_cmp"]) <= LSE_TOL[torch.bfloat16], where


@pytest.mark.parametrize("kw,gates,with_slc", [
    (dict(B=3, Hkv=2, G=4, D=128, T_cap=1500, seqlens=[1500, 700, 100]), (1 / 3, 1 / 3, 1 / 3), True),
    (dict(B=2, Hkv=2, G=8, D=64, T_cap=2000, seqlens=[2000, 20]), (1 / 3, 1 / 3, 1 / 3), True),
    (dict(B=1, Hkv=2, G=16, D=128, T_cap=3000, seqlens=[3000]), (1.0, 0.0, 0.0), True),
    (dict(B=1, Hkv=2, G=4, D=128, T_cap=3000, seqlens=[3000]), (0.0, 0.0, 1.0), False),
    (dict(B=1, Hkv=1, G=2, D=128, T_cap=64 * 40 + 9, seqlens=[64 * 40 + 9]), (0.5, 0.25, 0.25), False),
])
def test_nsa_branches_match_oracle(lsa, kw, gates, with_slc):
    case = synth.decode_case(dtype=torch.bfloat16, topk=8, n_sink=1, n_local=2, seed=103, **kw)
    o, lw, lc, idx, o_slc = _nsa_gpu(lsa, case, 8, gates, with_slc=with_slc)
    _check(case, gates, 512, o, lw, lc, idx, o_slc, with_slc, str(kw))


def test_nsa_decode_64k_workload(lsa):
    # the 64K GQA decode inputs: 4,096 compressed tokens, 16 selected blocks, a 512 window
    case = synth.gqa_decode_64k()
    gates = (1 / 3, 1 / 3, 1 / 3)
    o, lw, lc, idx, o_slc = _nsa_gpu(lsa, case, 16, gates)
    _check(case, gates, 512, o, lw, lc, idx, o_slc, True, "64k")
