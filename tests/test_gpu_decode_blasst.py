"""GPU parity of BLASST inside sparse decode (lsa_sparse_attn_decode_blasst) against the
fp64 oracle, through the C ABI.  The skip decisions must equal the oracle's wherever the
oracle's gap max_h (r_h - m_h) is further than 1e-3 (logit units) from ln(lambda); the
outputs are compared with the oracle forced onto the GPU's own decisions.  Cases: the
64K decode workload (plain, where nothing is negligible, and with sharpened queries, where
blocks are skipped), ragged sequences, padded selections, D 64, a planted block that only
one head needs, and lambda = 0 against the plain sparse decode."""
import math

import pytest
import torch

import oracle
import synth
from tests.parity import LSE_TOL, TOL, max_abs, max_abs_beyond_rounding

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
BAND = 1e-3


@pytest.fixture(scope="module")
def lsa(cuda_device):
    import query_aware_block_b200 as m
    return m


def _gpu(lsa, q, k, v, sl, idx, nsel, lam):
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    o = torch.full((B, Hq, D), 7.0, dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, Hq), 7.0, device=DEV)
    bits = torch.full((B, Hkv), -1, dtype=torch.int32, device=DEV)
    lsa.lsa_sparse_attn_decode_blasst(q.to(DEV), k.to(DEV), v.to(DEV), sl.to(DEV), idx.to(DEV),
                                      nsel.to(DEV), o, lam, lse=lse, skip_bits=bits)
    torch.cuda.synchronize()
    assert lsa.lsa_device_status() == 0
    return o.cpu(), lse.cpu(), bits.cpu().to(torch.int64) & 0xFFFFFFFF


def _check(q, k, v, sl, idx, nsel, lam, o, lse, bits, where):
    ref = oracle.decode_blasst(q, k, v, sl, idx, nsel, lam)
    ln_l = math.log(lam) if lam > 0 else -math.inf
    B, Hkv, topk = idx.shape
    for b in range(B):
        for g in range(Hkv):
            for s in range(topk):
                gb = (int(bits[b, g]) >> s) & 1
                rb = (int(ref["bits"][b, g]) >> s) & 1
                if gb != rb:
                    gap = float(ref["gap"][b, g, s])
                    assert abs(gap - ln_l) <= BAND, f"{where}: b{b} g{g} slot {s} gap {gap}"
    forced = oracle.decode_blasst(q, k, v, sl, idx, nsel, lam, forced_bits=bits)
    assert max_abs_beyond_rounding(o, forced["o"]) <= TOL[torch.bfloat16], where
    assert max_abs(lse, forced["lse"]) <= LSE_TOL[torch.bfloat16], where
    return ref


def _selection(case, topk, n_sink, n_local):
    r = oracle.decode(case.q, case.k, case.v, case.seqlens, topk, n_sink, n_local)
    return r["idx"], r["nsel"]


@pytest.mark.parametrize("kw,qscale,lam,expect_skips", [
    (dict(B=1, Hkv=2, G=8, D=128, T_cap=64 * 100 + 7, seqlens=64 * 100 + 7, topk=16, n_needles=6), 1.0, 1e-3, False),
    (dict(B=1, Hkv=2, G=8, D=128, T_cap=64 * 100 + 7, seqlens=64 * 100 + 7, topk=16, n_needles=6), 4.0, 1e-3, True),
    (dict(B=3, Hkv=2, G=4, D=64, T_cap=3000, seqlens=[3000, 1500, 700], topk=8, n_needles=3), 4.0, 1e-2, True),
    (dict(B=2, Hkv=1, G=16, D=128, T_cap=2000, seqlens=[2000, 999], topk=12, n_needles=2), 2.0, 0.1, True),
    (dict(B=1, Hkv=2, G=8, D=128, T_cap=64 * 100, seqlens=64 * 100, topk=16, n_needles=6), 4.0, 0.0, False),
])
def test_decode_blasst_matches_oracle(lsa, kw, qscale, lam, expect_skips):
    kw = dict(kw)
    topk = kw.pop("topk")
    case = synth.decode_case(dtype=torch.bfloat16, topk=topk, n_sink=1, n_local=2, seed=91, **kw)
    q = (case.q.float() * qscale).to(torch.bfloat16)  # a power of two (or 1): exact
    idx, nsel = _selection(case, topk, 1, 2)
    o, lse, bits = _gpu(lsa, q, case.k, case.v, case.seqlens, idx, nsel, lam)
    _check(q, case.k, case.v, case.seqlens, idx, nsel, lam, o, lse, bits, str(kw))
    if expect_skips:
        assert int(sum(bin(int(x)).count("1") for x in bits.flatten())) > 0, "nothing skipped"
    if lam == 0.0:
        assert int(bits.sum()) == 0


def test_decode_blasst_padded_selection_and_first_block(lsa):
    # slots past nsel and -1 slots hold no block; the first listed block is never skipped
    case = synth.decode_case(B=2, Hkv=2, G=4, D=128, T_cap=64 * 30, seqlens=[64 * 30, 64 * 20 + 5],
                             dtype=torch.bfloat16, topk=6, n_sink=0, n_local=0, seed=92)
    idx = torch.tensor([[[3, 9, 17, -1, -1, -1], [0, 5, -1, -1, -1, -1]],
                        [[2, 20, -1, -1, -1, -1], [1, 4, 7, 11, -1, -1]]], dtype=torch.int32)
    nsel = torch.tensor([[3, 2], [2, 4]], dtype=torch.int32)
    q = (case.q.float() * 4).to(torch.bfloat16)
    o, lse, bits = _gpu(lsa, q, case.k, case.v, case.seqlens, idx, nsel, 0.5)
    assert all(int(bits[b, g]) & 1 == 0 for b in range(2) for g in range(2))
    assert all(int(bits[b, g]) >> int(nsel[b, g]) == 0 for b in range(2) for g in range(2))
    _check(q, case.k, case.v, case.seqlens, idx, nsel, 0.5, o, lse, bits, "padded")


def test_decode_blasst_block_needed_by_one_head_is_kept(lsa):
    # two heads with opposite directions u: block 1 is below the running max for both
    # (skipped), block 2 for head 0 only (kept), block 3 for neither
    D, G, T = 128, 2, 64 * 5
    g = torch.Generator().manual_seed(93)
    u = torch.randn(D, generator=g, dtype=torch.float64)
    u = u / u.norm()
    w = torch.randn(D, generator=g, dtype=torch.float64)
    w = w - (w @ u) * u
    w = w / w.norm()
    q = torch.stack([8 * u + 8 * w, -8 * u + 8 * w])[None].to(torch.bfloat16)
    k = 0.05 * torch.randn(1, 1, T, D, generator=g, dtype=torch.float64)
    k[0, 0, 0:64] += 8 * w
    k[0, 0, 64:128] -= 8 * w
    k[0, 0, 128:192] += -8 * u - 8 * w
    k = k.to(torch.bfloat16)
    v = torch.randn(1, 1, T, D, generator=g).to(torch.bfloat16)
    sl = torch.tensor([T], dtype=torch.int32)
    idx = torch.tensor([[[0, 1, 2, 3]]], dtype=torch.int32)
    nsel = torch.tensor([[4]], dtype=torch.int32)
    o, lse, bits = _gpu(lsa, q, k, v, sl, idx, nsel, 1e-4)
    ref = _check(q, k, v, sl, idx, nsel, 1e-4, o, lse, bits, "planted")
    assert int(ref["bits"][0, 0]) == 0b0010 and int(bits[0, 0]) == 0b0010


def test_decode_blasst_lambda_zero_equals_plain_sparse_decode(lsa):
    case = synth.decode_case(B=2, Hkv=2, G=8, D=128, T_cap=64 * 50, seqlens=[64 * 50, 64 * 33 + 9],
                             dtype=torch.bfloat16, topk=16, n_sink=1, n_local=2, n_needles=4, seed=94)
    idx, nsel = _selection(case, 16, 1, 2)
    o, lse, bits = _gpu(lsa, case.q, case.k, case.v, case.seqlens, idx, nsel, 0.0)
    o2 = torch.empty(2, 16, 128, dtype=torch.bfloat16, device=DEV)
    lse2 = torch.empty(2, 16, device=DEV)
    lsa.lsa_sparse_attn_decode(case.q.to(DEV), case.k.to(DEV), case.v.to(DEV), case.seqlens.to(DEV),
                               o2, 16, idx=idx.to(DEV), nsel=nsel.to(DEV), lse=lse2)
    torch.cuda.synchronize()
    assert max_abs(o.float(), o2.cpu().float()) <= TOL[torch.bfloat16]
    assert max_abs(lse, lse2.cpu()) <= LSE_TOL[torch.bfloat16]
    _check(case.q, case.k, case.v, case.seqlens, idx, nsel, 0.0, o, lse, bits, "lambda 0")


def test_decode_blasst_64k_workload(lsa):
    # the 64K GQA decode inputs, given the oracle's selection; sharpened queries (x4) make
    # the two local blocks negligible next to the needles
    case = synth.gqa_decode_64k()
    idx, nsel = _selection(case, 16, 1, 2)
    for qscale, lam in ((1.0, 1e-3), (4.0, 1e-3)):
        q = (case.q.float() * qscale).to(torch.bfloat16)
        o, lse, bits = _gpu(lsa, q, case.k, case.v, case.seqlens, idx, nsel, lam)
        _check(q, case.k, case.v, case.seqlens, idx, nsel, lam, o, lse, bits, f"64k x{qscale}")


# ---- many (b, g) units: one CTA per unit, in phases (64 units and up) ----

@pytest.mark.parametrize("kw,qscale,lam", [
    (dict(B=32, Hkv=2, G=4, D=128, T_cap=3000, seqlens=None, topk=8, n_needles=3), 4.0, 1e-2),
    (dict(B=16, Hkv=4, G=8, D=64, T_cap=2500, seqlens=None, topk=12, n_needles=2), 2.0, 1e-3),
    (dict(B=8, Hkv=8, G=16, D=128, T_cap=64 * 40, seqlens=64 * 40, topk=16, n_needles=4), 4.0, 0.0),
])
def test_decode_blasst_many_units_matches_oracle(lsa, kw, qscale, lam):
    kw = dict(kw)
    topk = kw.pop("topk")
    if kw["seqlens"] is None:  # ragged lengths, partial last blocks
        g = torch.Generator().manual_seed(95)
        kw["seqlens"] = torch.randint(kw["T_cap"] // 3, kw["T_cap"] + 1, (kw["B"],), generator=g).tolist()
    case = synth.decode_case(dtype=torch.bfloat16, topk=topk, n_sink=1, n_local=2, seed=96, **kw)
    q = (case.q.float() * qscale).to(torch.bfloat16)
    idx, nsel = _selection(case, topk, 1, 2)
    o, lse, bits = _gpu(lsa, q, case.k, case.v, case.seqlens, idx, nsel, lam)
    _check(q, case.k, case.v, case.seqlens, idx, nsel, lam, o, lse, bits, str(kw))
    if lam == 0.0:
        assert int(bits.sum()) == 0


def test_decode_blasst_many_units_padded_selection(lsa):
    # 64 units whose slots past nsel and -1 slots hold no block; first listed never skipped
    B, Hkv, topk = 32, 2, 6
    case = synth.decode_case(B=B, Hkv=Hkv, G=4, D=128, T_cap=64 * 30, seqlens=64 * 30,
                             dtype=torch.bfloat16, topk=topk, n_sink=0, n_local=0, seed=97)
    g = torch.Generator().manual_seed(98)
    idx = torch.full((B, Hkv, topk), -1, dtype=torch.int32)
    nsel = torch.randint(1, topk + 1, (B, Hkv), generator=g, dtype=torch.int32)
    for b in range(B):
        for h in range(Hkv):
            n = int(nsel[b, h])
            blocks = sorted(torch.randperm(30, generator=g)[:n].tolist())
            idx[b, h, :n] = torch.tensor(blocks, dtype=torch.int32)
            if n > 2:
                idx[b, h, 1] = -1  # an unused slot inside the list
    nsel[0, 0] = 0  # a unit with no block at all: o = 0, lse = -inf
    idx[0, 0] = -1
    q = (case.q.float() * 4).to(torch.bfloat16)
    o, lse, bits = _gpu(lsa, q, case.k, case.v, case.seqlens, idx, nsel, 0.5)
    assert float(o[0, :4].float().abs().max()) == 0.0 and bool(torch.isinf(lse[0, :4]).all())
    assert all(int(bits[b, h]) >> int(nsel[b, h]) == 0 for b in range(B) for h in range(Hkv))
    _check(q, case.k, case.v, case.seqlens, idx, nsel, 0.5, o, lse, bits, "padded, many units")


def test_decode_blasst_batched_workload(lsa):
    # the batched varlen decode inputs (16 x 8 units), queries x4: a quarter or more of the
    # V blocks are negligible
    case = synth.batched_decode()
    q = (case.q.float() * 4).to(torch.bfloat16)
    idx, nsel = _selection(case, 16, 1, 2)
    o, lse, bits = _gpu(lsa, q, case.k, case.v, case.seqlens, idx, nsel, 1e-3)
    _check(q, case.k, case.v, case.seqlens, idx, nsel, 1e-3, o, lse, bits, "batched")
    skipped = sum(bin(int(x) & 0xFFFFFFFF).count("1") for x in bits.flatten())
    assert skipped > 0.2 * int(nsel.sum())
