"""GPU parity of the block-query step (per-token selection, union across the query block,
attention of active rows over the union, stable-row reuse) against the fp64 oracle,
through the C ABI: the diffusion-LM workload at full size, small shapes spanning several
cluster slices, token chunks and row chunks, and the edge cases (no active token, every
token active, a prefix shorter than top-k, ragged prefixes, forced blocks, an empty
prefix, the cache aliasing the output)."""
import pytest
import torch

import oracle
import synth
from tests.parity import GAP_REL, LSE_TOL, TOL, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa(cuda_device):
    import query_aware_block_b200 as m
    return m


def _run_gpu(lsa, case, alias=False):
    d = torch.device("cuda:0")
    q, k, v = case.q.to(d), case.k.to(d), case.v.to(d)
    B, Hq, Tq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    T_cap = k.shape[2]
    sl = torch.full((B,), T_cap, dtype=torch.int32, device=d)
    summ = torch.zeros(B, Hkv, -(-T_cap // 64), D, device=d)
    lsa.lsa_build_summaries(k, sl, summ)
    NBp = -(-case.T_prefix // 64)
    active = case.active.to(d)
    oc = case.o_cache.to(d)
    lc = case.lse_cache.to(d)
    if alias:
        o, lse = oc.clone(), lc.clone()
        oc_arg, lc_arg = o, lse
    else:
        o = torch.full_like(oc, 7.0)
        lse = torch.full_like(lc, 7.0)
        oc_arg, lc_arg = oc, lc
    ui = torch.full((B, Hkv, max(NBp, 1)), -7, dtype=torch.int32, device=d)
    uc = torch.full((B, Hkv), -7, dtype=torch.int32, device=d)
    ws = torch.empty(lsa.lsa_blockquery_workspace_size(B, Hkv, G, D, Tq), dtype=torch.uint8,
                     device=d)
    lsa.lsa_sparse_attn_blockquery(q, k, v, summ, case.T_prefix, case.topk, active, oc_arg,
                                   lc_arg, o, lse, ws, n_sink=case.n_sink, n_local=case.n_local,
                                   union_idx=ui, union_cnt=uc)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu(), ui[..., :NBp].cpu(), uc.cpu()


def _check_union(case, ui, uc, where, summ_len=None):
    """The GPU union against the per-token oracle selections under the gap rule
    (summaries over the first summ_len cache rows, by default all of them)."""
    B, Hq, Tq, D = case.q.shape
    Hkv = case.k.shape[1]
    NBp = -(-case.T_prefix // 64)
    sl = torch.full((B,), summ_len or case.k.shape[2], dtype=torch.int32)
    summ = oracle.summaries(case.k, sl)
    k = case.topk
    for b in range(B):
        act = [i for i in range(Tq) if case.active[b, i]]
        for g in range(Hkv):
            got = [int(j) for j in ui[b, g] if j >= 0]
            assert int(uc[b, g]) == len(got), f"{where}: count"
            assert got == sorted(got) and len(set(got)) == len(got), f"{where}: not ascending"
            if not act or NBp == 0:
                assert got == [], f"{where}: union must be empty"
                continue
            if NBp <= k:
                assert got == list(range(NBp)), f"{where}: all blocks"
                continue
            F = set(range(min(case.n_sink, NBp))) | set(range(max(0, NBp - case.n_local), NBp))
            m = k - len(F)
            must, may = set(F), set(F)
            for i in act:
                qi = case.q[b:b + 1, :, i].contiguous()
                s = oracle.block_scores(qi, summ[b:b + 1, :, :].contiguous(),
                                        torch.tensor([case.T_prefix]))[0, g, :NBp]
                cand = sorted(((float(s[j]), -j) for j in range(NBp) if j not in F), reverse=True)
                s_k, s_k1 = cand[m - 1][0], cand[m][0]
                band = GAP_REL * max(abs(s_k), abs(s_k1))
                for sc, nj in cand:
                    if sc > s_k + band:
                        must.add(-nj)
                    if sc >= s_k - band:
                        may.add(-nj)
                if s_k - s_k1 > band:
                    must |= {-c[1] for c in cand[:m]}
            assert must <= set(got), f"{where}: b{b} g{g} missing {sorted(must - set(got))}"
            assert set(got) <= may, f"{where}: b{b} g{g} extra {sorted(set(got) - may)}"


def _check_outputs(case, o, lse, ui, uc, where, alias=False):
    o_ref, lse_ref = oracle.blockquery_attn(case.q, case.k, case.v, case.active, case.o_cache,
                                            case.lse_cache, ui, uc, case.T_prefix)
    act = case.active.bool()
    B, Hq, Tq, D = case.q.shape
    am = act[:, None, :].expand(B, Hq, Tq)
    err = max_abs(o.float()[am], o_ref[am]) if am.any() else 0.0
    assert err <= TOL[torch.bfloat16], f"{where}: o err {err}"
    lerr = max_abs(lse[am], lse_ref[am]) if am.any() else 0.0
    assert lerr <= LSE_TOL[torch.bfloat16], f"{where}: lse err {lerr}"
    sm = ~am
    assert torch.equal(o[sm], case.o_cache[sm]), f"{where}: stable rows not bit-exact"
    assert torch.equal(lse[sm], case.lse_cache[sm]), f"{where}: stable lse not bit-exact"


@pytest.mark.parametrize("kw", [
    dict(B=1, Hkv=2, G=4, D=128, Tq=32, T_prefix=64 * 100, n_active=8, topk=8),
    dict(B=2, Hkv=2, G=2, D=64, Tq=8, T_prefix=1000, n_active=3, topk=4),        # ragged prefix
    dict(B=1, Hkv=1, G=4, D=128, Tq=32, T_prefix=64 * 300, n_active=20, topk=8),  # 3 token chunks, 3 row chunks
    dict(B=1, Hkv=2, G=16, D=128, Tq=8, T_prefix=64 * 80, n_active=8, topk=16),  # 128 rows, topk 16
    dict(B=1, Hkv=2, G=4, D=128, Tq=16, T_prefix=64 * 60, n_active=16, topk=8, n_sink=1, n_local=2),
    dict(B=1, Hkv=2, G=4, D=128, Tq=16, T_prefix=64 * 5 + 3, n_active=5, topk=8),  # NBp <= topk
    dict(B=1, Hkv=2, G=4, D=128, Tq=16, T_prefix=64 * 50, n_active=0, topk=8),    # nothing active
    dict(B=1, Hkv=2, G=4, D=128, Tq=16, T_prefix=64 * 50, n_active=9, topk=8),    # 36 rows: just past one chunk
    dict(B=4, Hkv=8, G=2, D=128, Tq=16, T_prefix=64 * 64, n_active=4, topk=8),    # 32 units: 8-CTA clusters
    dict(B=1, Hkv=2, G=4, D=128, Tq=64, T_prefix=64 * 40, n_active=64, topk=4),   # all 64 tokens active
    # 1,100 blocks: a CTA's slice (69 rows) exceeds the 64 staged rows (the rest from global)
    dict(B=1, Hkv=1, G=4, D=128, Tq=8, T_prefix=64 * 1100 + 17, n_active=5, topk=8, n_sink=1, n_local=1),
])
def test_blockquery_matches_oracle(lsa, kw):
    kw = dict(kw)
    T_cap = kw.pop("T_cap", None) or kw["T_prefix"] + 100
    case = synth.blockquery_case(T_cap=T_cap, seed=51, **kw)
    o, lse, ui, uc = _run_gpu(lsa, case)
    _check_union(case, ui, uc, str(kw))
    _check_outputs(case, o, lse, ui, uc, str(kw))


def test_blockquery_identical_queries_union_is_topk(lsa):
    case = synth.blockquery_case(B=1, Hkv=2, G=2, D=128, Tq=8, T_prefix=64 * 40, n_active=8,
                                 topk=5, seed=52, same_query=True)
    o, lse, ui, uc = _run_gpu(lsa, case)
    assert uc.tolist() == [[5, 5]]
    _check_outputs(case, o, lse, ui, uc, "same query")


def test_blockquery_cache_aliases_output(lsa):
    case = synth.blockquery_case(B=1, Hkv=2, G=4, D=128, Tq=16, T_prefix=64 * 30, n_active=4,
                                 topk=4, seed=53)
    o, lse, ui, uc = _run_gpu(lsa, case, alias=True)
    _check_outputs(case, o, lse, ui, uc, "alias")


def test_blockquery_empty_prefix(lsa):
    case = synth.blockquery_case(B=1, Hkv=1, G=2, D=128, Tq=8, T_prefix=0, T_cap=64, n_active=3,
                                 topk=4, seed=54)
    o, lse, ui, uc = _run_gpu(lsa, case)
    assert uc.tolist() == [[0]]
    act = case.active.bool()[:, None, :].expand(1, 2, 8)
    assert torch.count_nonzero(o[act]) == 0
    assert bool(torch.isinf(lse[act]).all()) and bool((lse[act] < 0).all())


def test_diffusion_blockquery_workload(lsa):
    case = synth.diffusion_blockquery()
    o, lse, ui, uc = _run_gpu(lsa, case)
    _check_union(case, ui, uc, "diffusion workload")
    _check_outputs(case, o, lse, ui, uc, "diffusion workload")
    # the union is far smaller than dense: KV density |U| / NB (expected ~60 of 512)
    assert 8 <= int(uc.max()) <= 64
