"""GPU parity of the LoSA denoising step around the block-query attention, through the
C ABI, against the fp64 oracle: the token classification by query change (mse in fp64
on both sides, so the masks must be equal; only exact ties could differ), the attention
inside the block merged with the prefix result, the dense first step (every prefix block),
and the three calls of a whole step on the diffusion workload at full size."""
import math

import pytest
import torch

import oracle
import synth
from tests.parity import LSE_TOL, TOL, max_abs, max_abs_beyond_rounding
from tests.test_gpu_blockquery import _check_union

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def lsa(cuda_device):
    import query_aware_block_b200 as m
    return m


def _gpu_classify(lsa, q, q_prev, tau=0.0, n_top=0):
    B, Hq, Tq, D = q.shape
    act = torch.full((B, Tq), 7, dtype=torch.uint8, device=DEV)
    mse = torch.full((B, Tq), -1.0, dtype=torch.float64, device=DEV)
    lsa.lsa_losa_classify(q.to(DEV), q_prev.to(DEV), act, tau=tau, n_top=n_top, mse=mse)
    torch.cuda.synchronize()
    return mse.cpu(), act.cpu()


def _assert_masks(act, ref_act, mse_ref, tau, n_top, where):
    """Equal masks, except where an exact tie in fp64 leaves the choice open."""
    if torch.equal(act, ref_act):
        return
    B, Tq = act.shape
    for b in range(B):
        m = mse_ref[b]
        for i in range(Tq):
            if act[b, i] == ref_act[b, i]:
                continue
            if n_top > 0:
                srt = torch.sort(m, descending=True).values
                edge = float(srt[n_top - 1])
                assert abs(float(m[i]) - edge) <= 1e-12 * max(abs(edge), 1e-300), f"{where}: b{b} i{i}"
            else:
                assert abs(float(m[i]) - tau) <= 1e-12 * max(abs(tau), 1e-300), f"{where}: b{b} i{i}"
    assert int(act.sum()) == int(ref_act.sum()) or n_top == 0, f"{where}: count"


@pytest.mark.parametrize("kw", [
    dict(B=2, Hkv=8, G=4, D=128, Tq=32, n_active=8),
    dict(B=1, Hkv=2, G=4, D=64, Tq=64, n_active=20),   # 8 tokens per CTA of the cluster
    dict(B=3, Hkv=1, G=2, D=128, Tq=5, n_active=2),    # ragged: CTAs without tokens
    dict(B=1, Hkv=2, G=2, D=128, Tq=1, n_active=1),
])
def test_losa_classify_matches_oracle(lsa, kw):
    kw = dict(kw)
    case = synth.losa_case(T_prefix=256, topk=4, seed=61, **kw)
    n = kw["n_active"]
    for tau, n_top in ((0.1, 0), (0.0, n), (1e-4, 0)):
        mse, act = _gpu_classify(lsa, case.q, case.q_prev, tau, n_top)
        mse_ref, act_ref = oracle.losa_classify(case.q, case.q_prev, tau, n_top)
        assert torch.allclose(mse, mse_ref, rtol=1e-12, atol=0), f"{kw} mse"
        _assert_masks(act, act_ref, mse_ref, tau, n_top, str(kw))
    # the planted active tokens are what both find
    _, act = _gpu_classify(lsa, case.q, case.q_prev, 0.1, 0)
    assert torch.equal(act, case.active)


def test_losa_classify_ties_and_no_change(lsa):
    case = synth.losa_case(B=2, Hkv=2, G=4, D=128, Tq=32, T_prefix=128, n_active=0, topk=2, seed=62)
    q = case.q
    mse, act = _gpu_classify(lsa, q, q.clone(), 0.0, 5)   # every change is 0: the first 5
    assert torch.count_nonzero(mse) == 0
    assert act.tolist() == [[1] * 5 + [0] * 27] * 2
    mse, act = _gpu_classify(lsa, q, q.clone(), 0.0, 0)   # strict: 0 > 0 is false
    assert torch.count_nonzero(act) == 0


def _intra_inputs(case, seed, empty_rows=()):
    g = torch.Generator().manual_seed(seed)
    B, Hq, Tq, D = case.q.shape
    o_pre = torch.randn(B, Hq, Tq, D, generator=g).to(torch.bfloat16)
    # prefix weights comparable to the block's own (log of ~32 keys) so both parts count
    lse_pre = torch.randn(B, Hq, Tq, generator=g) + 4.0
    for (b, h, i) in empty_rows:
        lse_pre[b, h, i] = -math.inf
    return o_pre, lse_pre


def _gpu_intra(lsa, case, o_pre, lse_pre, alias=False, flags=0):
    q, k, v = case.q.to(DEV), case.k.to(DEV), case.v.to(DEV)
    op, lp = o_pre.to(DEV), lse_pre.to(DEV)
    if alias:
        o, lse = op, lp
    else:
        o = torch.full_like(op, 7.0)
        lse = torch.full_like(lp, 7.0)
    lsa.lsa_blockquery_intra_merge(q, k, v, case.T_prefix, op, lp, o, lse, flags=flags)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("kw", [
    dict(B=1, Hkv=2, G=4, D=128, Tq=32),
    dict(B=2, Hkv=2, G=2, D=64, Tq=64),     # keys 32..63 in the second lane slot
    dict(B=1, Hkv=1, G=3, D=128, Tq=13),    # ragged: the last CTA holds 5 rows
    dict(B=1, Hkv=2, G=1, D=128, Tq=1),
])
def test_intra_merge_matches_oracle(lsa, kw):
    case = synth.losa_case(T_prefix=320, n_active=1, topk=4, seed=63, **kw)
    o_pre, lse_pre = _intra_inputs(case, 64, empty_rows=[(0, 0, 0)])
    o, lse = _gpu_intra(lsa, case, o_pre, lse_pre)
    o_ref, lse_ref = oracle.blockquery_intra_merge(case.q, case.k, case.v, case.T_prefix, o_pre, lse_pre)
    assert max_abs_beyond_rounding(o, o_ref) <= TOL[torch.bfloat16], kw
    assert max_abs(lse, lse_ref) <= LSE_TOL[torch.bfloat16], kw


def test_intra_merge_in_place_and_overlapped_launch(lsa):
    case = synth.losa_case(B=1, Hkv=2, G=4, D=128, Tq=32, T_prefix=640, n_active=4, topk=4, seed=65)
    o_pre, lse_pre = _intra_inputs(case, 66)
    o_ref, lse_ref = oracle.blockquery_intra_merge(case.q, case.k, case.v, case.T_prefix, o_pre, lse_pre)
    for alias, flags in ((True, 0), (False, 1), (True, 1)):
        o, lse = _gpu_intra(lsa, case, o_pre, lse_pre, alias=alias, flags=flags)
        assert max_abs_beyond_rounding(o, o_ref) <= TOL[torch.bfloat16], (alias, flags)
        assert max_abs(lse, lse_ref) <= LSE_TOL[torch.bfloat16], (alias, flags)


def _gpu_blockquery(lsa, case, active, topk, o_cache, lse_cache, o, lse, summ):
    B, Hq, Tq, D = case.q.shape
    Hkv = case.k.shape[1]
    NBp = -(-case.T_prefix // 64)
    ws = torch.empty(lsa.lsa_blockquery_workspace_size(B, Hkv, Hq // Hkv, D, Tq), dtype=torch.uint8,
                     device=DEV)
    ui = torch.full((B, Hkv, max(NBp, 1)), -7, dtype=torch.int32, device=DEV)
    uc = torch.full((B, Hkv), -7, dtype=torch.int32, device=DEV)
    lsa.lsa_sparse_attn_blockquery(case.q.to(DEV), case.k.to(DEV), case.v.to(DEV), summ,
                                   case.T_prefix, topk, active, o_cache, lse_cache, o, lse, ws,
                                   union_idx=ui, union_cnt=uc)
    return ui, uc


def _gpu_summ(lsa, case):
    B, Hkv, T_cap, D = case.k.shape
    sl = torch.full((B,), case.T_prefix, dtype=torch.int32, device=DEV)
    summ = torch.zeros(B, Hkv, -(-T_cap // 64), D, device=DEV)
    lsa.lsa_build_summaries(case.k.to(DEV), sl, summ)
    return summ


@pytest.mark.parametrize("T_prefix,Tq,sample", [
    (64 * 40, 16, None),                # 40 blocks: dense through the small-union path size
    (64 * 1100 + 17, 8, [0, 5, 7]),     # 1,101 blocks: more than any sparse union holds
    (32768, 32, [0, 13, 31]),           # the diffusion workload's prefix, every token
])
def test_dense_first_step_matches_oracle(lsa, T_prefix, Tq, sample):
    case = synth.losa_case(B=1, Hkv=2 if T_prefix < 32768 else 8, G=4, D=128, Tq=Tq,
                           T_prefix=T_prefix, n_active=Tq, topk=4, seed=67)
    NBp = -(-T_prefix // 64)
    summ = _gpu_summ(lsa, case)
    B, Hq, _, D = case.q.shape
    active = torch.ones(B, Tq, dtype=torch.uint8, device=DEV)
    o = torch.full((B, Hq, Tq, D), 7.0, dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, Hq, Tq), 7.0, device=DEV)
    ui, uc = _gpu_blockquery(lsa, case, active, NBp, case.o_cache.to(DEV), case.lse_cache.to(DEV),
                             o, lse, summ)
    torch.cuda.synchronize()
    Hkv = case.k.shape[1]
    assert uc.cpu().tolist() == [[NBp] * Hkv]
    assert torch.equal(ui.cpu()[0, :, :NBp], torch.arange(NBp, dtype=torch.int32).expand(Hkv, NBp))
    # rows are independent: the oracle attends the sampled tokens only
    toks = sample if sample is not None else list(range(Tq))
    qs = case.q[:, :, toks].contiguous()
    n = len(toks)
    all_on = torch.ones(B, n, dtype=torch.uint8)
    o_ref, lse_ref = oracle.blockquery_attn(qs, case.k, case.v, all_on, case.o_cache[:, :, toks].contiguous(),
                                            case.lse_cache[:, :, toks].contiguous(), ui.cpu()[..., :NBp],
                                            uc.cpu(), T_prefix)
    og, lg = o.cpu()[:, :, toks], lse.cpu()[:, :, toks]
    assert max_abs(og.float(), o_ref) <= TOL[torch.bfloat16]
    assert max_abs(lg, lse_ref) <= LSE_TOL[torch.bfloat16]


@pytest.mark.parametrize("kw", [
    dict(B=1, Hkv=2, G=4, D=128, Tq=32, T_prefix=64 * 100, n_active=8, topk=8),
    dict(B=2, Hkv=2, G=2, D=128, Tq=16, T_prefix=64 * 50 + 9, n_active=3, topk=4),
    None,  # the diffusion workload at full size: 8 KV heads x 4, prefix 32768, 8 of 32 active
])
def test_losa_step_matches_oracle(lsa, kw):
    case = synth.diffusion_losa_step() if kw is None else synth.losa_case(seed=68, **kw)
    B, Hq, Tq, D = case.q.shape
    n_top = int(case.active[0].sum())
    # 1. classify
    act = torch.empty(B, Tq, dtype=torch.uint8, device=DEV)
    lsa.lsa_losa_classify(case.q.to(DEV), case.q_prev.to(DEV), act, n_top=n_top)
    # 2. prefix part, the cache updated in place
    summ = _gpu_summ(lsa, case)
    cache_o, cache_l = case.o_cache.to(DEV).clone(), case.lse_cache.to(DEV).clone()
    ui, uc = _gpu_blockquery(lsa, case, act, case.topk, cache_o, cache_l, cache_o, cache_l, summ)
    # 3. the block itself, merged (overlapped launch)
    o = torch.empty_like(cache_o)
    lse = torch.empty_like(cache_l)
    lsa.lsa_blockquery_intra_merge(case.q.to(DEV), case.k.to(DEV), case.v.to(DEV), case.T_prefix,
                                   cache_o, cache_l, o, lse, flags=lsa.LSA_FLAG_PDL)
    torch.cuda.synchronize()
    assert lsa.lsa_device_status() == 0
    assert torch.equal(act.cpu(), case.active)
    NBp = -(-case.T_prefix // 64)
    ui_c, uc_c = ui.cpu()[..., :NBp], uc.cpu()
    _check_union(case, ui_c, uc_c, "losa step", summ_len=case.T_prefix)
    r = oracle.losa_step(case.q, case.q_prev, case.k, case.v, None, case.T_prefix, case.o_cache,
                         case.lse_cache, case.topk, n_top=n_top, union=(ui_c, uc_c))
    assert torch.equal(r["active"], case.active)
    stable = ~case.active.bool()[:, None, :].expand(B, Hq, Tq)
    # the cache: stable rows untouched, active rows the new prefix result
    assert torch.equal(cache_o.cpu()[stable], case.o_cache[stable])
    assert max_abs(cache_o.cpu().float()[~stable], r["o_prefix"][~stable]) <= TOL[torch.bfloat16]
    # the step's output
    # (stable rows keep cached N(0, 1) values up to ~5: the bound is on the error beyond
    # the output's own rounding to bf16)
    assert max_abs_beyond_rounding(o.cpu(), r["o"]) <= TOL[torch.bfloat16]
    assert max_abs(lse.cpu(), r["lse"]) <= LSE_TOL[torch.bfloat16]
