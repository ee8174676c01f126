"""GPU parity of the weighted block selection (FASA- and Prism-style scorers,
lsa_select_blocks_weighted) against the fp64 oracle, through the C ABI: the chosen blocks
under the gap rule on the oracle's weighted scores, and the weighted scores themselves.
Cases: a FASA chunk subset and Prism's dual-band weights, bf16 and fp32 queries (fp32
reweighted in place), D 64 and 128, and the 64K decode inputs."""
import pytest
import torch

import oracle
import synth
from tests.parity import check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa(cuda_device):
    import query_aware_block_b200 as m
    return m


def _weights(kind, D):
    if kind == "fasa":
        return oracle.fasa_weights(D, [0, 3, 9, 17, D // 2 - 5, D // 2 - 1])
    return oracle.prism_weights(D)[0]


def _run(lsa, case, w, topk, ns, nl, in_place=False):
    d = torch.device("cuda:0")
    q, sl = case.q.to(d), case.seqlens.to(d)
    summ_ref = oracle.summaries(case.k, case.seqlens)
    summ = summ_ref.float().to(d)  # the same (rounded) summaries on both sides
    B, Hkv, NB_cap, D = summ.shape
    idx = torch.full((B, Hkv, topk), -7, dtype=torch.int32, device=d)
    nsel = torch.zeros(B, Hkv, dtype=torch.int32, device=d)
    sc = torch.zeros(B, Hkv, NB_cap, device=d)
    wd = w.float().to(d)
    qw = q if in_place else None
    lsa.lsa_select_blocks_weighted(q, summ, sl, wd, topk, ns, nl, idx, nsel, q_weighted=qw,
                                   scores_out=sc)
    torch.cuda.synchronize()
    ref = oracle.block_scores_weighted(case.q, summ_ref, case.seqlens, w)
    return idx.cpu(), nsel.cpu(), sc.cpu(), ref


@pytest.mark.parametrize("kind,B,Hkv,G,D,T,topk,ns,nl,dtype,in_place", [
    ("fasa", 2, 2, 4, 128, [64 * 300, 64 * 40 + 9], 16, 1, 2, torch.bfloat16, False),
    ("prism", 2, 2, 4, 128, [64 * 300, 64 * 40 + 9], 16, 1, 2, torch.bfloat16, False),
    ("prism", 1, 3, 8, 64, [5000], 8, 1, 2, torch.float32, True),
    ("fasa", 3, 1, 2, 64, [3000, 700, 64], 8, 0, 0, torch.float32, False),
])
def test_weighted_select_matches_oracle(lsa, kind, B, Hkv, G, D, T, topk, ns, nl, dtype, in_place):
    case = synth.decode_case(B, Hkv, G, D, max(T), T, dtype, topk, ns, nl, seed=111)
    w = _weights(kind, D)
    idx, nsel, sc, ref = _run(lsa, case, w, topk, ns, nl, in_place)
    for b in range(B):
        NB = -(-int(case.seqlens[b]) // 64)
        for g in range(Hkv):
            check_selection(idx[b, g], ref[b, g], NB, topk, ns, nl, f"{kind} b{b}g{g}")
            assert int(nsel[b, g]) == min(topk, NB)
            if NB > topk:
                err = (sc[b, g, :NB].double() - ref[b, g, :NB]).abs().max()
                assert float(err) < 1e-4 * (1 + float(ref[b, g, :NB].abs().max()))


def test_weighted_select_64k_workload(lsa):
    case = synth.gqa_decode_64k()
    for kind in ("fasa", "prism"):
        w = _weights(kind, 128)
        idx, nsel, sc, ref = _run(lsa, case, w, 16, 1, 2)
        for g in range(8):
            check_selection(idx[0, g], ref[0, g], 1024, 16, 1, 2, f"64k {kind} g{g}")
