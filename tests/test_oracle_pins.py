"""Pins for the fp64 oracle: every check here ties the oracle to something other than
itself -- textbook special cases, closed forms, brute-force enumeration, library routines
(torch scaled_dot_product_attention / logsumexp / topk in fp64) and invariants of the
method -- so that a dropped term, a wrong sign or index, or a transposed operand in
oracle/lsa_oracle.c fails at least one of them.  CPU only."""
import itertools
import json
import math
import os

import pytest
import torch
import torch.nn.functional as F

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf(x):
    return x.to(torch.bfloat16)


# ---------------------------------------------------------------- rotary generator ----

def test_rope_preserves_norm_and_is_relative():
    g = torch.Generator().manual_seed(0)
    D = 64
    x = torch.randn(5, D, generator=g, dtype=torch.float64)
    pos = torch.tensor([0, 3, 17, 1000, 65535])
    y = synth.rope(x, pos, 1e4)
    assert torch.allclose(y.norm(dim=-1), x.norm(dim=-1), rtol=0, atol=1e-12)
    # R(m) q . R(n) k depends only on m - n
    q = torch.randn(D, generator=g, dtype=torch.float64)
    k = torch.randn(D, generator=g, dtype=torch.float64)
    d1 = (synth.rope(q[None], torch.tensor([10]), 1e4) * synth.rope(k[None], torch.tensor([4]), 1e4)).sum()
    d2 = (synth.rope(q[None], torch.tensor([106]), 1e4) * synth.rope(k[None], torch.tensor([100]), 1e4)).sum()
    assert abs(float(d1 - d2)) < 1e-10
    # position 0 is the identity
    assert torch.allclose(synth.rope(q[None], torch.tensor([0]), 1e4)[0], q, atol=0)


# ---------------------------------------------------------------------- summaries ----

def test_summary_of_constant_keys_is_exact():
    B, Hkv, T, D = 2, 3, 200, 16
    c = torch.randn(B, Hkv, 1, D).expand(B, Hkv, T, D).contiguous()
    s = oracle.summaries(c, torch.tensor([200, 77]))
    # NB_cap = 4; sequence 0 has 4 blocks (last one 8 tokens), sequence 1 has 2 blocks
    for j in range(4):
        assert torch.equal(s[0, :, j], c[0, :, 0].double())
    for j in range(2):
        assert torch.equal(s[1, :, j], c[1, :, 0].double())
    assert torch.count_nonzero(s[1, :, 2:]) == 0


def test_summary_partial_block_closed_form():
    # keys k_t = t in every dim: the mean of block j is (t0 + t1 - 1) / 2 over valid tokens
    T_cap, T = 256, 150
    k = torch.arange(T_cap, dtype=torch.float32).view(1, 1, T_cap, 1).expand(1, 1, T_cap, 4).contiguous()
    s = oracle.summaries(k, torch.tensor([T]))
    expect = [(0 + 63) / 2, (64 + 127) / 2, (128 + 149) / 2, 0.0]
    assert s[0, 0, :, 0].tolist() == expect


def test_summary_is_dirichlet_low_pass_of_rotated_constant():
    # Mean pooling of a rotated constant over n positions scales each rotary pair's
    # magnitude by |sin(n w / 2) / (n sin(w / 2))| (Dirichlet kernel) -- the low-pass
    # effect of mean pooling on RoPE dims [Prism, "2. 핵심 이론적 발견"].
    D, theta, T = 32, 1e4, 64 + 40
    c = torch.randn(D, dtype=torch.float64, generator=torch.Generator().manual_seed(3))
    keys = synth.rope(c.expand(T, D), torch.arange(T), theta).to(torch.float32)
    s = oracle.summaries(keys.view(1, 1, T, D).contiguous(), torch.tensor([T]))
    half = D // 2
    cf = c.to(torch.float32).double()
    for j, n in ((0, 64), (1, 40)):
        for p in range(half):
            w = theta ** (-2.0 * p / D)
            ratio = abs(math.sin(n * w / 2) / (n * math.sin(w / 2)))
            mag_c = math.hypot(cf[p], cf[p + half])
            mag_s = math.hypot(s[0, 0, j, p], s[0, 0, j, p + half])
            assert abs(mag_s - ratio * mag_c) < 2e-6 * (1 + mag_c), (j, p)
    # the highest-frequency pair is strongly attenuated, the lowest is not
    assert math.hypot(s[0, 0, 0, 0], s[0, 0, 0, half]) < 0.05 * math.hypot(cf[0], cf[half])
    assert math.hypot(s[0, 0, 0, half - 1], s[0, 0, 0, D - 1]) > 0.99 * math.hypot(cf[half - 1], cf[D - 1])


def test_summary_bf16_widening_is_exact():
    k = torch.randn(1, 1, 64, 8).to(torch.bfloat16)
    s = oracle.summaries(k, torch.tensor([64]))
    exact = k.double().sum(dim=2) / 64.0
    assert torch.allclose(s[0, :, 0], exact[0], rtol=0, atol=1e-15)


# ------------------------------------------------------------------------- scores ----

def test_group_score_is_sum_of_single_head_scores():
    # a group score with G heads equals the sum of the scores of each head on its own;
    # catches a dropped head or a wrong head -> group mapping (h belongs to group h // G)
    g = torch.Generator().manual_seed(5)
    B, Hkv, G, D, T = 2, 3, 4, 16, 320
    q = torch.randn(B, Hkv * G, D, generator=g)
    summ = torch.randn(B, Hkv, 5, D, generator=g, dtype=torch.float64)
    sl = torch.tensor([320, 130])
    full = oracle.block_scores(q, summ, sl, scale=0.25)
    acc = torch.zeros_like(full)
    for hh in range(G):
        qh = q.view(B, Hkv, G, D)[:, :, hh].contiguous()  # one head per group
        acc += oracle.block_scores(qh, summ, sl, scale=0.25)
    valid = torch.isfinite(full)
    assert torch.allclose(full[valid], acc[valid], rtol=1e-13, atol=1e-13)
    assert valid[1].sum() == Hkv * 3  # 130 tokens -> 3 blocks
    assert torch.isinf(full[1, :, 3:]).all() and (full[1, :, 3:] < 0).all()


def test_score_sign_and_scale():
    # a block whose summary points along the summed query scores highest (Cauchy-Schwarz);
    # the anti-aligned block scores lowest; the score scales linearly with `scale`
    D, G = 8, 2
    q = torch.tensor([[1.0, 2, 0, 0, 0, 0, 0, 1], [0.0, 1, 1, 0, 0, 0, 0, 0]]).view(1, G, D)
    u = q.sum(dim=1)[0].double()
    u = u / u.norm()
    summ = torch.randn(1, 1, 6, D, dtype=torch.float64, generator=torch.Generator().manual_seed(1))
    summ = summ / summ.norm(dim=-1, keepdim=True)
    summ[0, 0, 2] = u
    summ[0, 0, 4] = -u
    s1 = oracle.block_scores(q, summ, torch.tensor([6 * 64]), scale=1.0)[0, 0]
    s3 = oracle.block_scores(q, summ, torch.tensor([6 * 64]), scale=3.0)[0, 0]
    assert int(s1.argmax()) == 2 and int(s1.argmin()) == 4
    assert abs(float(s1[2]) - float(q.sum(dim=1)[0].double().norm())) < 1e-12
    assert torch.allclose(s3, 3 * s1, rtol=1e-14, atol=0)


# ----------------------------------------------------------------------- selection ----

def _brute_best_sum(s, NB, k, forced):
    free = [j for j in range(NB) if j not in forced]
    best = -math.inf
    for comb in itertools.combinations(free, k - len(forced)):
        best = max(best, sum(s[j] for j in comb))
    return best


@pytest.mark.parametrize("NB,k,ns,nl", [(10, 5, 1, 2), (12, 6, 0, 0), (9, 4, 2, 1), (11, 3, 1, 2)])
def test_select_matches_brute_force(NB, k, ns, nl):
    g = torch.Generator().manual_seed(NB * 100 + k)
    for trial in range(20):
        s = torch.randn(1, 1, NB, generator=g, dtype=torch.float64)
        idx, nsel = oracle.select(s, torch.tensor([NB * 64]), k, ns, nl)
        chosen = [int(j) for j in idx[0, 0] if j >= 0]
        assert int(nsel[0, 0]) == k == len(chosen)
        assert chosen == sorted(chosen)
        forced = set(range(ns)) | set(range(NB - nl, NB))
        assert forced <= set(chosen)
        got = sum(float(s[0, 0, j]) for j in chosen if j not in forced)
        assert abs(got - _brute_best_sum(s[0, 0].tolist(), NB, k, forced)) < 1e-12


def test_select_agrees_with_torch_topk():
    g = torch.Generator().manual_seed(9)
    NB, k = 1024, 16
    s = torch.randn(1, 1, NB, generator=g, dtype=torch.float64)
    idx, _ = oracle.select(s, torch.tensor([NB * 64]), k, 1, 2)
    masked = s[0, 0].clone()
    masked[[0, NB - 2, NB - 1]] = -math.inf
    top = torch.topk(masked, k - 3).indices.tolist()
    assert idx[0, 0].tolist() == sorted(top + [0, NB - 2, NB - 1])


def test_select_ties_go_to_lower_index_and_small_nb_takes_all():
    s = torch.zeros(1, 1, 8, dtype=torch.float64)
    s[0, 0, 5] = 1.0
    idx, nsel = oracle.select(s, torch.tensor([8 * 64]), 4, 0, 0)
    assert idx[0, 0].tolist() == [0, 1, 2, 5]
    idx, nsel = oracle.select(s, torch.tensor([3 * 64 + 1]), 6, 1, 2)  # NB = 4 <= 6
    assert idx[0, 0].tolist() == [0, 1, 2, 3, -1, -1] and int(nsel[0, 0]) == 4
    idx, nsel = oracle.select(s, torch.tensor([0]), 4, 1, 2)  # empty sequence
    assert idx[0, 0].tolist() == [-1] * 4 and int(nsel[0, 0]) == 0


def test_nsa_token_accounting_golden():
    # The NSA page gives, for 64K decoding, 5,632 tokens touched instead of 65,536 with
    # compression block 32 / stride 16, 16 selected blocks of 64 *including* the initial
    # block and 2 local blocks, and a 512-token window.  The selection count that makes
    # the total come out is 16 blocks (forced inside n), which is what the oracle keeps.
    with open(os.path.join(GOLDEN, "nsa_decode_token_accounting.json")) as f:
        gold = json.load(f)
    T = gold["context"]
    NB = T // gold["selection_block"]
    s = torch.randn(1, 1, NB, dtype=torch.float64, generator=torch.Generator().manual_seed(2))
    _, nsel = oracle.select(s, torch.tensor([T]), gold["selected_blocks"], 1, 2)
    compressed = T // gold["compression_stride"]
    total = compressed + int(nsel[0, 0]) * gold["selection_block"] + gold["window"]
    assert total == gold["tokens_accessed"]


# ------------------------------------------------------------------ decode attention ----

def _sdpa64(q, k, v, mask=None):
    """Library routine: fp64 scaled dot-product attention (default scale 1/sqrt(D))."""
    return F.scaled_dot_product_attention(q.double(), k.double(), v.double(), attn_mask=mask)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_with_all_blocks_equals_dense(dtype):
    B, Hkv, G, D = 2, 2, 3, 32
    case = synth.decode_case(B, Hkv, G, D, T_cap=300, seqlens=[300, 190], dtype=dtype,
                             topk=8, n_sink=1, n_local=2, seed=11, poison_tail=True)
    r = oracle.decode(case.q, case.k, case.v, case.seqlens, case.topk, 1, 2)
    assert r["nsel"].tolist() == [[5, 5], [3, 3]]
    for b in range(B):
        T = int(case.seqlens[b])
        for h in range(Hkv * G):
            g = h // G
            ref = _sdpa64(case.q[b, h][None, None], case.k[b, g, :T][None], case.v[b, g, :T][None])
            assert torch.allclose(r["o"][b, h], ref[0, 0], rtol=0, atol=1e-12)
            logits = case.q[b, h].double() @ case.k[b, g, :T].double().T / math.sqrt(D)
            assert abs(float(r["lse"][b, h] - torch.logsumexp(logits, 0))) < 1e-12


def test_decode_subset_equals_masked_dense_and_ignores_tail():
    B, Hkv, G, D, T = 1, 2, 2, 64, 1000  # last block partial (1000 = 15*64 + 40)
    case = synth.decode_case(B, Hkv, G, D, T_cap=1024, seqlens=T, dtype=torch.bfloat16,
                             topk=5, n_sink=1, n_local=2, seed=12, poison_tail=True)
    r = oracle.decode(case.q, case.k, case.v, case.seqlens, 5, 1, 2)
    assert torch.isfinite(r["o"]).all()
    for g in range(Hkv):
        blocks = [int(j) for j in r["idx"][0, g] if j >= 0]
        assert blocks[0] == 0 and blocks[-2:] == [14, 15]
        mask = torch.zeros(T, dtype=torch.bool)
        for j in blocks:
            mask[j * 64:min(j * 64 + 64, T)] = True
        for hh in range(G):
            h = g * G + hh
            ref = _sdpa64(case.q[0, h][None, None], case.k[0, g, :T][None], case.v[0, g, :T][None],
                          mask=mask[None, None])
            assert torch.allclose(r["o"][0, h], ref[0, 0], rtol=0, atol=1e-12)


def test_decode_uniform_keys_give_mean_of_values():
    D = 16
    k = torch.zeros(1, 1, 128, D)
    k[0, 0, 64:] = torch.randn(D)  # all keys of block 1 equal
    v = torch.randn(1, 1, 128, D)
    q = torch.randn(1, 1, D)
    o, lse = oracle.decode_attn(q, k, v, torch.tensor([128]), torch.tensor([[[1]]]),
                                torch.tensor([[1]]))
    assert torch.allclose(o[0, 0], v[0, 0, 64:].double().mean(0), rtol=0, atol=1e-14)
    logit = float(q[0, 0].double() @ k[0, 0, 64].double()) / 4.0
    assert abs(float(lse[0, 0]) - (logit + math.log(64))) < 1e-12


def test_decode_split_merge_associativity():
    # attention over blocks S = S1 U S2 equals the log-sum-exp merge of the two halves
    case = synth.decode_case(1, 1, 4, 32, 640, 640, torch.float32, 6, 0, 0, seed=13)
    idx = torch.tensor([[[0, 2, 3, 5, 7, 9]]])
    full_o, full_l = oracle.decode_attn(case.q, case.k, case.v, case.seqlens, idx, torch.tensor([[6]]))
    o1, l1 = oracle.decode_attn(case.q, case.k, case.v, case.seqlens, idx[..., :2].contiguous(), torch.tensor([[2]]))
    o2, l2 = oracle.decode_attn(case.q, case.k, case.v, case.seqlens, idx[..., 2:].contiguous(), torch.tensor([[4]]))
    lm = torch.logaddexp(l1, l2)
    om = o1 * torch.exp(l1 - lm)[..., None] + o2 * torch.exp(l2 - lm)[..., None]
    assert torch.allclose(lm, full_l, rtol=0, atol=1e-12)
    assert torch.allclose(om, full_o, rtol=0, atol=1e-12)


def test_decode_block_permutation_invariance_without_rope():
    # with no rotary embedding and no forced blocks, permuting the KV blocks permutes the
    # selection and leaves the output unchanged
    B, Hkv, G, D, NB = 1, 2, 2, 16, 12
    case = synth.decode_case(B, Hkv, G, D, NB * 64, NB * 64, torch.float32, 4, 0, 0,
                             theta=1e30, seed=14)  # theta -> inf: all angles ~ 0
    perm = torch.randperm(NB, generator=torch.Generator().manual_seed(4))
    kp = case.k.view(B, Hkv, NB, 64, D)[:, :, perm].reshape(case.k.shape).contiguous()
    vp = case.v.view(B, Hkv, NB, 64, D)[:, :, perm].reshape(case.v.shape).contiguous()
    r0 = oracle.decode(case.q, case.k, case.v, case.seqlens, 4, 0, 0)
    r1 = oracle.decode(case.q, kp, vp, case.seqlens, 4, 0, 0)
    inv = torch.argsort(perm)
    for g in range(Hkv):
        a = sorted(int(j) for j in r0["idx"][0, g])
        b = sorted(int(perm[int(j)]) for j in r1["idx"][0, g])
        assert a == b
        assert sorted(int(inv[j]) for j in a) == [int(j) for j in r1["idx"][0, g]]
    assert torch.allclose(r0["o"], r1["o"], rtol=0, atol=1e-12)


# --------------------------------------------------------------------- block-query ----

def _bq_run(case, topk=None):
    sl = torch.full((case.k.shape[0],), case.T_prefix, dtype=torch.int32)
    summ = oracle.summaries(case.k[:, :, :case.T_prefix].contiguous(), sl)
    ui, uc, sel = oracle.blockquery_select(case.q, summ, case.active, case.T_prefix,
                                           topk or case.topk, case.n_sink, case.n_local,
                                           return_sel=True)
    o, lse = oracle.blockquery_attn(case.q, case.k, case.v, case.active, case.o_cache,
                                    case.lse_cache, ui, uc, case.T_prefix)
    return summ, ui, uc, sel, o, lse


def test_blockquery_union_is_union_of_token_selections():
    case = synth.blockquery_case(B=2, Hkv=2, G=2, D=32, Tq=8, T_prefix=1024, n_active=3,
                                 topk=4, seed=21)
    summ, ui, uc, sel, o, lse = _bq_run(case)
    NB = 16
    for b in range(2):
        A = int(case.active[b].sum())
        for g in range(2):
            want = set()
            for i in range(8):
                row = [int(j) for j in sel[b, i, g] if j >= 0]
                if case.active[b, i]:
                    assert len(row) == 4
                    want |= set(row)
                else:
                    assert row == []
            got = [int(j) for j in ui[b, g] if j >= 0]
            assert got == sorted(want) and int(uc[b, g]) == len(got)
            assert len(got) <= min(NB, 4 * A)


def test_blockquery_token_selection_brute_force():
    # each active token's own selection maximises the summed block scores (tiny NB)
    case = synth.blockquery_case(B=1, Hkv=1, G=2, D=16, Tq=4, T_prefix=10 * 64, n_active=4,
                                 topk=3, seed=22)
    summ, ui, uc, sel, o, lse = _bq_run(case)
    for i in range(4):
        qi = case.q[:, :, i].contiguous()  # [1, G, D]
        s = oracle.block_scores(qi, summ, torch.tensor([640]))[0, 0].tolist()
        chosen = [int(j) for j in sel[0, i, 0]]
        assert abs(sum(s[j] for j in chosen) - _brute_best_sum(s, 10, 3, set())) < 1e-12


def test_blockquery_identical_queries_union_equals_topk():
    case = synth.blockquery_case(B=1, Hkv=2, G=2, D=32, Tq=8, T_prefix=2048, n_active=8,
                                 topk=5, seed=23, same_query=True)
    _, ui, uc, _, _, _ = _bq_run(case)
    assert uc.tolist() == [[5, 5]]


def test_blockquery_all_stable_is_cache_bit_exact():
    case = synth.blockquery_case(B=1, Hkv=2, G=2, D=32, Tq=8, T_prefix=1024, n_active=0,
                                 topk=4, seed=24)
    _, ui, uc, _, o, lse = _bq_run(case)
    assert uc.tolist() == [[0, 0]]
    assert torch.equal(o, case.o_cache.double()) and torch.equal(lse, case.lse_cache.double())


def test_blockquery_all_blocks_equals_dense_prefix_attention():
    case = synth.blockquery_case(B=1, Hkv=2, G=2, D=32, Tq=6, T_prefix=400, T_cap=512,
                                 n_active=4, topk=16, seed=25)
    _, ui, uc, _, o, lse = _bq_run(case)
    assert uc.tolist() == [[7, 7]]
    for h in range(4):
        g = h // 2
        ref = _sdpa64(case.q[0, h][None], case.k[0, g, :400][None], case.v[0, g, :400][None])[0]
        for i in range(6):
            if case.active[0, i]:
                assert torch.allclose(o[0, h, i], ref[i], rtol=0, atol=1e-12)
            else:
                assert torch.equal(o[0, h, i], case.o_cache[0, h, i].double())


# ------------------------------------------------------------------------- BLASST ----

def _dense_causal(q, k, v):
    return F.scaled_dot_product_attention(q.double(), k.double(), v.double(), is_causal=True)


def _all_units(B, Hq, L, tq=128):
    return [(b, h, a) for b in range(B) for h in range(Hq) for a in range(-(-L // tq))]


def _assemble(r, units, B, Hq, L, D, tq=128):
    out = torch.zeros(B, Hq, L, D, dtype=torch.float64)
    for u, (b, h, a) in enumerate(units):
        n = min(tq, L - a * tq)
        out[b, h, a * tq:a * tq + n] = r["o"][u, :n]
    return out


@pytest.mark.parametrize("L", [256, 300])
def test_blasst_lambda_zero_is_dense_causal(L):
    case = synth.prefill_case(B=1, Hq=4, Hkv=2, L=L, D=32, lam=0.0, seed=31)
    units = _all_units(1, 4, L)
    r = oracle.blasst_prefill(case.q, case.k, case.v, units, 0.0)
    assert int(r["bits"].sum()) == 0
    o = _assemble(r, units, 1, 4, L, 32)
    kx = case.k.repeat_interleave(2, dim=1)
    vx = case.v.repeat_interleave(2, dim=1)
    ref = _dense_causal(case.q, kx, vx)
    assert torch.allclose(o, ref, rtol=0, atol=1e-12)
    logits = case.q.double() @ kx.double().transpose(-1, -2) / math.sqrt(32)
    logits = logits.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), -math.inf)
    lse_ref = torch.logsumexp(logits, -1)
    for u, (b, h, a) in enumerate(units):
        n = min(128, L - a * 128)
        assert torch.allclose(r["lse"][u, :n], lse_ref[b, h, a * 128:a * 128 + n], rtol=0, atol=1e-12)


def _sharp_case(L=512, seed=32, sink=7.0):
    return synth.prefill_case(B=1, Hq=2, Hkv=1, L=L, D=32, lam=1e-3, sink=sink, seed=seed)


def test_blasst_skips_equal_masked_dense_and_respect_error_bound():
    case = _sharp_case()
    L, lam = 512, 0.05
    units = _all_units(1, 2, L)
    r = oracle.blasst_prefill(case.q, case.k, case.v, units, lam)
    nskip = int(sum(bin(int(w)).count("1") for w in r["bits"].flatten()))
    nvis = sum((min(a * 128 + 128, L) - 1) // 64 + 1 for (_, _, a) in units)
    assert 0 < nskip < nvis - len(units), "the sink case must skip some tiles, not all"
    ln_lam = math.log(lam)
    kx = case.k.repeat_interleave(2, dim=1).double()
    vx = case.v.repeat_interleave(2, dim=1).double()
    dense = _dense_causal(case.q, kx, vx)
    for u, (b, h, a) in enumerate(units):
        words = int(r["bits"][u, 0])
        nvisit = (min(a * 128 + 128, L) - 1) // 64 + 1
        assert words & 1 == 0  # the first visited tile is never skipped
        for c in range(nvisit):
            skipped = (words >> c) & 1
            assert skipped == (r["gap"][u, c] < ln_lam)
        # output = dense softmax restricted to the keys of the non-skipped tiles
        rows = torch.arange(a * 128, a * 128 + 128)
        keep = torch.zeros(128, L, dtype=torch.bool)
        for c in range(nvisit):
            if not (words >> c) & 1:
                keep[:, c * 64:(c + 1) * 64] = True
        keep &= rows[:, None] >= torch.arange(L)[None, :]
        ref = F.scaled_dot_product_attention(case.q[b, h, a * 128:a * 128 + 128].double()[None],
                                             kx[b, h][None], vx[b, h][None], attn_mask=keep[None])[0]
        assert torch.allclose(r["o"][u], ref, rtol=0, atol=1e-12)
        # error bound against dense: each dropped weight is < lambda relative to the
        # final row max, so |o - dense| <= 2 max|v| * n_dropped * lambda
        dropped = (~keep & (rows[:, None] >= torch.arange(L)[None, :])).sum(1).double()
        bound = 2 * vx[b, h].abs().max() * dropped * lam
        err = (r["o"][u] - dense[b, h, a * 128:a * 128 + 128]).abs().max(dim=1).values
        assert (err <= bound + 1e-12).all()


def test_blasst_constructed_negligible_tile_is_skipped():
    # keys of tile 1 have logits far below tile 0's for every row -> tile 1 (and only it)
    # is skipped, and the rows that see tile 1 attend to tile 0 only
    D, L = 16, 128
    q = torch.zeros(1, 1, L, D)
    q[..., 0] = 4.0
    k = torch.zeros(1, 1, L, D)
    k[0, 0, :64, 0] = 4.0     # logits 16/4 = 4 for tile 0
    k[0, 0, 64:, 0] = -4.0    # logits -4 for tile 1: gap -8 < ln(1e-3) = -6.9
    v = torch.randn(1, 1, L, D)
    r = oracle.blasst_prefill(q, k, v, [(0, 0, 0)], 1e-3, scale=0.25)
    assert int(r["bits"][0, 0]) == 0b10
    assert abs(float(r["gap"][0, 1]) + 8.0) < 1e-12
    assert torch.allclose(r["o"][0, 64:], v[0, 0, :64].double().mean(0).expand(64, D), atol=1e-12)
    r2 = oracle.blasst_prefill(q, k, v, [(0, 0, 0)], 1e-4, scale=0.25)  # ln 1e-4 = -9.2 < -8
    assert int(r2["bits"][0, 0]) == 0


def test_blasst_skip_needs_every_row_negligible():
    # the tile above, but row 100's query points the other way: tile 1 is that row's best
    # tile (gap +8), so the tile is kept although every other row finds it negligible
    D, L = 16, 128
    q = torch.zeros(1, 1, L, D)
    q[..., 0] = 4.0
    q[0, 0, 100, 0] = -4.0
    k = torch.zeros(1, 1, L, D)
    k[0, 0, :64, 0] = 4.0
    k[0, 0, 64:, 0] = -4.0
    v = torch.randn(1, 1, L, D)
    r = oracle.blasst_prefill(q, k, v, [(0, 0, 0)], 1e-3, scale=0.25)
    assert int(r["bits"][0, 0]) == 0
    assert abs(float(r["gap"][0, 1]) - 8.0) < 1e-12


def test_blasst_forced_bits_follow_the_given_decisions():
    case = _sharp_case(L=256, seed=33)
    units = _all_units(1, 2, 256)
    free = oracle.blasst_prefill(case.q, case.k, case.v, units, 0.0)
    forced = torch.zeros_like(free["bits"])
    forced[:, 0] = 0b0100  # skip tile 2 wherever it is visited
    r = oracle.blasst_prefill(case.q, case.k, case.v, units, 0.0, forced_bits=forced)
    for u, (b, h, a) in enumerate(units):
        nvisit = (min(a * 128 + 128, 256) - 1) // 64 + 1
        assert int(r["bits"][u, 0]) == (0b0100 if nvisit > 2 else 0)


# ------------------------------------------------------------- LoSA step (classify) ----

def _grid_bf16(shape, gen, lim=64):
    """Values k/8 with |k| <= lim: exact in bf16, and so are their sums with eighths."""
    return (torch.randint(-lim, lim + 1, shape, generator=gen).double() / 8).to(torch.bfloat16)


def test_losa_classify_unchanged_queries():
    gen = torch.Generator().manual_seed(40)
    q = torch.randn(2, 4, 6, 16, generator=gen).to(torch.bfloat16)
    mse, act = oracle.losa_classify(q, q.clone(), tau=0.0)
    assert torch.count_nonzero(mse) == 0 and torch.count_nonzero(act) == 0
    _, act = oracle.losa_classify(q, q.clone(), tau=-1.0)
    assert bool(act.all())
    # every change ties at 0: the n_top lowest token indices rank first
    _, act = oracle.losa_classify(q, q.clone(), n_top=3)
    assert act.tolist() == [[1, 1, 1, 0, 0, 0]] * 2


def test_losa_classify_constant_shift_closed_form():
    # token i of sequence b moves by c[b, i] in every head and dim: its MSE is c^2 exactly
    B, Hq, Tq, D = 2, 3, 7, 16
    gen = torch.Generator().manual_seed(41)
    q_prev = _grid_bf16((B, Hq, Tq, D), gen)
    c = torch.randint(0, 9, (B, Tq), generator=gen).double() / 8
    c[0, 0] = 0.5  # a token exactly at the threshold below
    q = (q_prev.double() + c[:, None, :, None]).to(torch.bfloat16)
    assert torch.equal(q.double() - q_prev.double(), c[:, None, :, None].expand(B, Hq, Tq, D))
    mse, act = oracle.losa_classify(q, q_prev, tau=0.25)
    assert torch.equal(mse, c * c)
    assert torch.equal(act.bool(), c * c > 0.25)
    assert int(act[0, 0]) == 0  # strict: a change equal to tau is stable


def test_losa_classify_single_element_change():
    # one element (head 3, token 2, dim 17) moves by 0.5: that token's MSE is
    # 0.25 / (Hq * D), every other token's is 0
    B, Hq, Tq, D = 1, 5, 4, 24
    q_prev = torch.zeros(B, Hq, Tq, D, dtype=torch.bfloat16)
    q = q_prev.clone()
    q[0, 3, 2, 17] = 0.5
    mse, act = oracle.losa_classify(q, q_prev, tau=0.0)
    expect = torch.zeros(B, Tq, dtype=torch.float64)
    expect[0, 2] = 0.25 / (Hq * D)
    assert torch.allclose(mse, expect, rtol=1e-15, atol=0)
    assert act.tolist() == [[0, 0, 1, 0]]


def test_losa_classify_top_n_is_a_stable_descending_sort():
    # library routine: a stable sort of the negated changes ranks the tokens (equal changes:
    # lower index first); duplicated shifts plant exact ties
    B, Hq, Tq, D = 3, 4, 16, 8
    gen = torch.Generator().manual_seed(42)
    q_prev = _grid_bf16((B, Hq, Tq, D), gen)
    c = torch.randint(0, 5, (B, Tq), generator=gen).double() / 8  # many equal shifts
    q = (q_prev.double() + c[:, None, :, None]).to(torch.bfloat16)
    for n in (1, 5, 16):
        mse, act = oracle.losa_classify(q, q_prev, n_top=n)
        for b in range(B):
            order = torch.sort(-c[b] * c[b], stable=True).indices
            expect = torch.zeros(Tq, dtype=torch.uint8)
            expect[order[:n]] = 1
            assert torch.equal(act[b], expect), (n, b)
        assert torch.equal(mse, c * c)


# ---------------------------------------------------- LoSA step (intra-block + merge) ----

def _dense_rows(q, k, v, scale):
    """Library routines: fp64 SDPA with no mask and the log-sum-exp of the logits."""
    o = F.scaled_dot_product_attention(q.double(), k.double(), v.double(), scale=scale)
    lse = torch.logsumexp(scale * q.double() @ k.double().transpose(-1, -2), dim=-1)
    return o, lse


def test_losa_step_all_blocks_equals_dense_attention_over_prefix_and_block():
    # every token active and every prefix block selected: the prefix part is dense, the
    # block part is bidirectional, so the merged row is plain softmax attention over all
    # T_prefix + Tq keys
    case = synth.losa_case(B=1, Hkv=2, G=2, D=32, Tq=6, T_prefix=320, n_active=6, topk=16,
                           dtype=torch.float32, seed=43)
    T, Tq, D = case.T_prefix, 6, 32
    sl = torch.full((1,), T, dtype=torch.int32)
    summ = oracle.summaries(case.k[:, :, :T].contiguous(), sl)
    r = oracle.losa_step(case.q, case.q_prev, case.k, case.v, summ, T, case.o_cache,
                         case.lse_cache, topk=16, tau=0.1)
    assert r["active"].tolist() == [[1] * 6]
    assert r["union_cnt"].tolist() == [[5, 5]]
    for h in range(4):
        g = h // 2
        o_ref, lse_ref = _dense_rows(case.q[0, h], case.k[0, g, :T + Tq], case.v[0, g, :T + Tq],
                                     1 / math.sqrt(D))
        assert torch.allclose(r["o"][0, h], o_ref, rtol=0, atol=1e-12)
        assert torch.allclose(r["lse"][0, h], lse_ref, rtol=0, atol=1e-12)
        # the prefix part alone is dense prefix attention
        o_p, lse_p = _dense_rows(case.q[0, h], case.k[0, g, :T], case.v[0, g, :T], 1 / math.sqrt(D))
        assert torch.allclose(r["o_prefix"][0, h], o_p, rtol=0, atol=1e-12)
        assert torch.allclose(r["lse_prefix"][0, h], lse_p, rtol=0, atol=1e-12)


def test_intra_merge_empty_prefix_and_single_token():
    case = synth.losa_case(B=2, Hkv=1, G=3, D=16, Tq=5, T_prefix=128, n_active=5, topk=2,
                           dtype=torch.float32, seed=44)
    T = case.T_prefix
    none_o = torch.zeros(2, 3, 5, 16, dtype=torch.float64)
    none_l = torch.full((2, 3, 5), -math.inf, dtype=torch.float64)
    o, lse = oracle.blockquery_intra_merge(case.q, case.k, case.v, T, none_o, none_l)
    for b in range(2):
        for h in range(3):
            o_ref, lse_ref = _dense_rows(case.q[b, h], case.k[b, 0, T:T + 5], case.v[b, 0, T:T + 5], 0.25)
            assert torch.allclose(o[b, h], o_ref, rtol=0, atol=1e-12)
            assert torch.allclose(lse[b, h], lse_ref, rtol=0, atol=1e-12)
    # one token in the block and no prefix: the row's output is that token's value
    q1 = case.q[:, :, :1].contiguous()
    o1, lse1 = oracle.blockquery_intra_merge(q1, case.k, case.v, T, none_o[:, :, :1], none_l[:, :, :1])
    for b in range(2):
        for h in range(3):
            assert torch.equal(o1[b, h, 0], case.v[b, 0, T].double())
            assert abs(float(lse1[b, h, 0]) - 0.25 * float(case.q[b, h, 0].double() @ case.k[b, 0, T].double())) < 1e-12


def test_losa_step_stable_rows_with_exact_cache_match_recomputation():
    # a stable token whose cache holds its exact prefix result ends where recomputing it
    # would: dense attention over prefix and block (fp32 cache: ~1e-7)
    case = synth.losa_case(B=1, Hkv=2, G=2, D=32, Tq=8, T_prefix=256, n_active=3, topk=16,
                           dtype=torch.float32, seed=45)
    T, Tq, D = case.T_prefix, 8, 32
    sc = 1 / math.sqrt(D)
    o_cache = torch.empty(1, 4, Tq, D)
    lse_cache = torch.empty(1, 4, Tq)
    for h in range(4):
        o_p, lse_p = _dense_rows(case.q[0, h], case.k[0, h // 2, :T], case.v[0, h // 2, :T], sc)
        o_cache[0, h], lse_cache[0, h] = o_p.float(), lse_p.float()
    sl = torch.full((1,), T, dtype=torch.int32)
    summ = oracle.summaries(case.k[:, :, :T].contiguous(), sl)
    r = oracle.losa_step(case.q, case.q_prev, case.k, case.v, summ, T, o_cache, lse_cache,
                         topk=16, n_top=3)
    assert torch.equal(r["active"], case.active)
    for h in range(4):
        o_ref, lse_ref = _dense_rows(case.q[0, h], case.k[0, h // 2, :T + Tq],
                                     case.v[0, h // 2, :T + Tq], sc)
        assert torch.allclose(r["o"][0, h], o_ref, rtol=0, atol=1e-6)
        assert torch.allclose(r["lse"][0, h], lse_ref, rtol=0, atol=1e-5)


# ------------------------------------------------------ BLASST inside sparse decode ----

def _masked_rows(q, k, v, T, blocks, scale):
    """Library routines: fp64 SDPA of the query rows over the tokens of `blocks` (t < T),
    and the log-sum-exp of those logits."""
    mask = torch.zeros(T, dtype=torch.bool)
    for j in blocks:
        mask[j * 64:min(j * 64 + 64, T)] = True
    kk, vv = k[:T][mask].double(), v[:T][mask].double()
    o = F.scaled_dot_product_attention(q.double()[None], kk[None], vv[None], scale=scale)[0]
    lse = torch.logsumexp(scale * q.double() @ kk.T, dim=-1)
    return o, lse


def _decode_sel(case, topk, n_sink=1, n_local=2):
    r = oracle.decode(case.q, case.k, case.v, case.seqlens, topk, n_sink, n_local)
    return r["idx"], r["nsel"]


def test_decode_blasst_lambda_zero_is_masked_dense():
    B, Hkv, G, D, T = 2, 2, 3, 32, 1000
    case = synth.decode_case(B, Hkv, G, D, T_cap=1024, seqlens=[T, 700], dtype=torch.float32,
                             topk=6, n_sink=1, n_local=2, seed=81)
    idx, nsel = _decode_sel(case, 6)
    r = oracle.decode_blasst(case.q, case.k, case.v, case.seqlens, idx, nsel, 0.0)
    assert int(r["bits"].sum()) == 0
    for b in range(B):
        Tb = int(case.seqlens[b])
        for g in range(Hkv):
            blocks = [int(j) for j in idx[b, g] if j >= 0]
            qh = case.q[b, g * G:(g + 1) * G]
            o_ref, lse_ref = _masked_rows(qh, case.k[b, g], case.v[b, g], Tb, blocks, 1 / math.sqrt(D))
            assert torch.allclose(r["o"][b, g * G:(g + 1) * G], o_ref, rtol=0, atol=1e-12)
            assert torch.allclose(r["lse"][b, g * G:(g + 1) * G], lse_ref, rtol=0, atol=1e-12)


def _planted_case(seed):
    """G = 2 heads with opposite queries; block 1 is negligible for both heads (keys
    orthogonal-ish and far below), block 2 is negligible for head 0 only, block 3 for
    neither; block 0 holds a key every head scores highly (it sets the running maxima)."""
    D, G, T = 32, 2, 64 * 5
    g = torch.Generator().manual_seed(seed)
    u = torch.randn(D, generator=g, dtype=torch.float64)
    u = u / u.norm()
    w = torch.randn(D, generator=g, dtype=torch.float64)
    w = w - (w @ u) * u
    w = w / w.norm()
    q = torch.stack([8 * u + 8 * w, -8 * u + 8 * w])[None].float()          # [1, 2, D]
    k = 0.05 * torch.randn(1, 1, T, D, generator=g, dtype=torch.float64)
    k[0, 0, 0:64] += 4 * w                  # block 0: logit ~ 8*4/sqrt(32) = 5.7 for both heads
    k[0, 0, 64:128] -= 4 * w                # block 1: ~ -5.7 for both: gap ~ -11.3
    k[0, 0, 128:192] += -4 * u - 4 * w      # block 2: head 0 ~ -11.3, head 1 ~ 0: gap ~ -5.7
    k[0, 0, 192:256] += 0.0                 # block 3: ~ 0 for both: gap ~ -5.7
    v = torch.randn(1, 1, T, D, generator=g)
    return q, k.float(), v, T


def test_decode_blasst_skips_only_blocks_every_head_finds_negligible():
    q, k, v, T = _planted_case(82)
    sl = torch.tensor([T], dtype=torch.int32)
    idx = torch.tensor([[[0, 1, 2, 3, -1]]], dtype=torch.int32)
    nsel = torch.tensor([[4]], dtype=torch.int32)
    # ln(1e-4) = -9.2: block 1 (gap -11.3) is skipped; blocks 2 and 3 (gap -5.7) are kept
    r = oracle.decode_blasst(q, k, v, sl, idx, nsel, 1e-4)
    assert int(r["bits"][0, 0]) == 0b0010
    gap = r["gap"][0, 0]
    assert math.isinf(float(gap[0])) and float(gap[1]) < math.log(1e-4) < float(gap[2])
    assert math.isnan(float(gap[4]))
    o_ref, lse_ref = _masked_rows(q[0], k[0, 0], v[0, 0], T, [0, 2, 3], 1 / math.sqrt(32))
    assert torch.allclose(r["o"][0], o_ref, rtol=0, atol=1e-12)
    assert torch.allclose(r["lse"][0], lse_ref, rtol=0, atol=1e-12)
    # ln(0.01) = -4.6: now blocks 2 and 3 are negligible for every head too
    r = oracle.decode_blasst(q, k, v, sl, idx, nsel, 1e-2)
    assert int(r["bits"][0, 0]) == 0b1110
    # the first visited block is never skipped, however small: with block 1 first, its gap
    # is +inf and block 0 (gap +11.3) is kept as well
    idx2 = torch.tensor([[[1, 0, 2, 3, -1]]], dtype=torch.int32)
    r = oracle.decode_blasst(q, k, v, sl, idx2, nsel, 1e-2)
    assert int(r["bits"][0, 0]) & 0b0011 == 0


def test_decode_blasst_output_is_dense_over_kept_blocks_within_the_error_bound():
    # a sharpened query (x3) makes some selected blocks negligible at lambda = 1e-3
    B, Hkv, G, D, T = 1, 2, 2, 64, 64 * 24
    case = synth.decode_case(B, Hkv, G, D, T_cap=T, seqlens=T, dtype=torch.float32, topk=12,
                             n_sink=1, n_local=2, n_needles=3, seed=83)
    q = (case.q * 3).contiguous()
    idx, nsel = _decode_sel(case, 12)
    lam = 1e-3
    r = oracle.decode_blasst(q, case.k, case.v, case.seqlens, idx, nsel, lam)
    full = oracle.decode_blasst(q, case.k, case.v, case.seqlens, idx, nsel, 0.0)
    assert int(r["bits"].sum()) > 0, "the case should skip something"
    sc = 1 / math.sqrt(D)
    for g in range(Hkv):
        kept = [int(idx[0, g, s]) for s in range(12) if not (int(r["bits"][0, g]) >> s) & 1]
        dropped = 64 * (12 - len(kept))
        qh = q[0, g * G:(g + 1) * G]
        o_ref, lse_ref = _masked_rows(qh, case.k[0, g], case.v[0, g], T, kept, sc)
        assert torch.allclose(r["o"][0, g * G:(g + 1) * G], o_ref, rtol=0, atol=1e-12)
        assert torch.allclose(r["lse"][0, g * G:(g + 1) * G], lse_ref, rtol=0, atol=1e-12)
        # each dropped weight is < lambda relative to the final max, whose weight is 1
        vmax = float(case.v[0, g].abs().max())
        err = float((r["o"][0, g * G:(g + 1) * G] - full["o"][0, g * G:(g + 1) * G]).abs().max())
        assert err <= 2 * vmax * dropped * lam
        # forcing the same decisions reproduces the output; forcing none gives lambda = 0
    forced = oracle.decode_blasst(q, case.k, case.v, case.seqlens, idx, nsel, 0.5,
                                  forced_bits=r["bits"])
    assert torch.equal(forced["o"], r["o"]) and torch.equal(forced["bits"], r["bits"])
    none = oracle.decode_blasst(q, case.k, case.v, case.seqlens, idx, nsel, 0.5,
                                forced_bits=torch.zeros(1, Hkv, dtype=torch.int64))
    assert torch.equal(none["o"], full["o"])


# ------------------------------------------ NSA's compressed and sliding-window branches ----

def test_nsa_compress_is_avg_pool_with_clipped_tail():
    # library routine: avg_pool1d (kernel 32, stride 16, ceil mode: a window that runs past
    # the end is divided by its valid count) gives every window that starts at least one
    # stride before the end; the last window (start 16 * (NC - 1)) has a closed form
    B, Hkv, T_cap, D = 2, 2, 700, 8
    g = torch.Generator().manual_seed(71)
    k = torch.randn(B, Hkv, T_cap, D, generator=g)
    sl = torch.tensor([700, 333], dtype=torch.int32)
    kc = oracle.nsa_compress(k, sl, 32, 16)
    assert kc.shape == (B, Hkv, 44, D)
    for b in range(B):
        T = int(sl[b])
        NC = -(-T // 16)
        x = k[b, :, :T].double().transpose(1, 2)  # [Hkv, D, T]
        ref = F.avg_pool1d(x, kernel_size=32, stride=16, ceil_mode=True).transpose(1, 2)
        n = ref.shape[1]
        assert n in (NC, NC - 1)
        assert torch.allclose(kc[b, :, :n], ref, rtol=0, atol=1e-12)
        t0 = 16 * (NC - 1)
        assert torch.allclose(kc[b, :, NC - 1], k[b, :, t0:T].double().mean(dim=1), rtol=0, atol=1e-12)
        assert torch.count_nonzero(kc[b, :, NC:]) == 0
    # a ramp k_t = t: window [16i, min(16i + 32, T)) has mean (t0 + t1 - 1) / 2
    ramp = torch.arange(T_cap, dtype=torch.float32)[None, None, :, None].expand(1, 1, T_cap, 4).contiguous()
    kr = oracle.nsa_compress(ramp, torch.tensor([T_cap]), 32, 16)
    for i in range(44):
        t0, t1 = 16 * i, min(16 * i + 32, T_cap)
        assert float(kr[0, 0, i, 0]) == (t0 + t1 - 1) / 2


def test_nsa_compress_with_block_length_equal_to_stride_is_the_block_summary():
    case = synth.decode_case(1, 2, 2, 32, T_cap=300, seqlens=300, dtype=torch.bfloat16, topk=4,
                             n_sink=1, n_local=2, seed=72)
    kc = oracle.nsa_compress(case.k, case.seqlens, 64, 64)
    assert torch.equal(kc, oracle.summaries(case.k, case.seqlens))


def test_nsa_window_and_compressed_branches_are_sdpa():
    B, Hkv, G, D = 2, 2, 2, 32
    case = synth.decode_case(B, Hkv, G, D, T_cap=1200, seqlens=[1200, 300], dtype=torch.float32,
                             topk=4, n_sink=1, n_local=2, seed=73)
    o_w, lse_w = oracle.window_attn(case.q, case.k, case.v, case.seqlens, 512)
    kc = oracle.nsa_compress(case.k, case.seqlens, 32, 16)
    vc = oracle.nsa_compress(case.v, case.seqlens, 32, 16)
    nc = torch.tensor([75, 19], dtype=torch.int32)
    o_c, lse_c = oracle.range_attn_f64(case.q, kc, vc, torch.zeros(2, dtype=torch.int32), nc)
    sc = 1 / math.sqrt(D)
    for b, T in ((0, 1200), (1, 300)):
        t0 = max(0, T - 512)  # sequence 1 is shorter than the window: all of it
        for g in range(Hkv):
            qh = case.q[b, g * G:(g + 1) * G]
            o_ref, lse_ref = _dense_rows(qh, case.k[b, g, t0:T], case.v[b, g, t0:T], sc)
            assert torch.allclose(o_w[b, g * G:(g + 1) * G], o_ref, rtol=0, atol=1e-12)
            assert torch.allclose(lse_w[b, g * G:(g + 1) * G], lse_ref, rtol=0, atol=1e-12)
            n = int(nc[b])
            o_ref, lse_ref = _dense_rows(qh, kc[b, g, :n], vc[b, g, :n], sc)
            assert torch.allclose(o_c[b, g * G:(g + 1) * G], o_ref, rtol=0, atol=1e-12)
            assert torch.allclose(lse_c[b, g * G:(g + 1) * G], lse_ref, rtol=0, atol=1e-12)


def test_nsa_decode_combines_the_three_branches_and_reproduces_the_64k_accounting():
    # the NSA page's 64K decoding count: 5,632 of 65,536 tokens read (4,096 compressed
    # tokens, 16 selected blocks of 64, a 512-token window)
    with open(os.path.join(GOLDEN, "nsa_decode_token_accounting.json")) as f:
        gold = json.load(f)
    T = gold["context"]
    case = synth.decode_case(1, 1, 2, 16, T_cap=T, seqlens=T, dtype=torch.bfloat16, topk=16,
                             n_sink=1, n_local=2, seed=74)
    r = oracle.nsa_decode(case.q, case.k, case.v, case.seqlens, topk=gold["selected_blocks"],
                          n_sink=gold["forced_initial_blocks"], n_local=gold["forced_local_blocks"],
                          length=gold["compression_block"], stride=gold["compression_stride"],
                          window=gold["window"])
    t = r["tokens"]
    assert t["compressed"] == [4096] and sum(t["selected"][0]) == 1024 and t["window"] == [512]
    assert t["compressed"][0] + sum(t["selected"][0]) + t["window"][0] == gold["tokens_accessed"]
    assert torch.allclose(r["o"], (r["o_cmp"] + r["o_slc"] + r["o_win"]) / 3, rtol=0, atol=1e-15)
    only = oracle.nsa_decode(case.q, case.k, case.v, case.seqlens, gates=(0.0, 1.0, 0.0), idx=r["idx"])
    assert torch.equal(only["o"], r["o_slc"])


# ------------------------------------- weighted block scores (FASA / Prism-style scorers) ----

def _scorer_case(seed=75):
    case = synth.decode_case(2, 2, 3, 64, T_cap=640, seqlens=[640, 400], dtype=torch.bfloat16,
                             topk=4, n_sink=1, n_local=2, seed=seed)
    summ = oracle.summaries(case.k, case.seqlens)
    return case, summ


def test_weighted_scores_reduce_to_the_plain_score_and_are_linear_in_the_weights():
    case, summ = _scorer_case()
    D = 64
    plain = oracle.block_scores(case.q, summ, case.seqlens)
    assert torch.equal(oracle.block_scores_weighted(case.q, summ, case.seqlens, torch.ones(D)), plain)
    g = torch.Generator().manual_seed(76)
    w1 = torch.rand(D, generator=g, dtype=torch.float64)
    w2 = torch.rand(D, generator=g, dtype=torch.float64)
    s1 = oracle.block_scores_weighted(case.q, summ, case.seqlens, w1)
    s2 = oracle.block_scores_weighted(case.q, summ, case.seqlens, w2)
    s12 = oracle.block_scores_weighted(case.q, summ, case.seqlens, w1 + 3 * w2)
    fin = torch.isfinite(s12)
    assert torch.allclose(s12[fin], (s1 + 3 * s2)[fin], rtol=1e-12, atol=1e-12)
    assert torch.equal(torch.isinf(s12), torch.isinf(plain))


def test_fasa_weights_score_with_the_kept_chunks_only():
    # library routine: einsum over the sliced dims of the kept rotary chunks
    case, summ = _scorer_case()
    D, G = 64, 3
    chunks = [2, 5, 17, 30]
    w = oracle.fasa_weights(D, chunks)
    dims = [d for d in range(D) if int(oracle.rope_chunk_of_dim(D)[d]) in chunks]
    assert dims == [2, 5, 17, 30, 34, 37, 49, 62] and int(w.sum()) == 8
    s = oracle.block_scores_weighted(case.q, summ, case.seqlens, w)
    for b, T in ((0, 640), (1, 400)):
        NB = -(-T // 64)
        for g in range(2):
            qs = case.q[b, g * G:(g + 1) * G][:, dims].double().sum(0)
            ref = (summ[b, g, :NB][:, dims] @ qs) / math.sqrt(D)
            assert torch.allclose(s[b, g, :NB], ref, rtol=1e-12, atol=1e-12)


def test_rope_attenuation_is_the_measured_magnitude_of_a_pooled_rotating_constant():
    # pool a constant unit vector of chunk j rotated over 64 positions (the generator's
    # rotary embedding, the oracle's block mean): what is left is the closed form
    D = 32
    a = oracle.rope_block_attenuation(D, 1e4, 64)
    for j in (0, 1, 3, 7, 15):
        c = torch.zeros(1, 1, 64, D, dtype=torch.float64)
        c[..., j] = 1.0
        k = synth.rope(c[0, 0], torch.arange(64), 1e4)[None, None].float()
        kbar = oracle.summaries(k, torch.tensor([64]))[0, 0, 0]
        mag = float(torch.hypot(kbar[j], kbar[j + D // 2]))
        assert abs(mag - float(a[j])) < 2e-6, (j, mag, float(a[j]))   # fp32 keys


def test_prism_weights_split_the_bands_at_one_rotation_per_block():
    D, blk = 128, 64
    w, high, (t_hi, t_lo) = oracle.prism_weights(D, 1e4, blk)
    j = torch.arange(D // 2, dtype=torch.float64)
    period = 2 * math.pi / (1e4 ** (-2 * j / D))
    assert torch.equal(high, period < blk)
    a = oracle.rope_block_attenuation(D, 1e4, blk)
    assert abs(t_hi - float(a[high].mean())) < 1e-15 and abs(t_lo - float(a[~high].mean())) < 1e-15
    chunk = oracle.rope_chunk_of_dim(D)
    for d in range(D):
        assert float(w[d]) == (1 / t_hi if bool(high[chunk[d]]) else 1 / t_lo)
    assert t_hi < 0.1 < 0.9 < t_lo  # pooling erases the fast chunks, keeps the slow ones


def test_fasa_weighted_selection_ignores_a_decoy_in_the_dropped_chunks():
    # block 5's summary matches the query strongly in chunk 0 only, block 9's moderately in
    # chunk 20 only: the plain score picks block 5, the score on chunk 20 picks block 9
    D, NB = 64, 16
    q = torch.zeros(1, 1, D)
    q[0, 0, 0] = 1.0
    q[0, 0, 20] = 1.0
    summ = torch.zeros(1, 1, NB, D, dtype=torch.float64)
    summ[0, 0, 5, 0] = 3.0
    summ[0, 0, 9, 20] = 1.0
    sl = torch.tensor([NB * 64])
    plain = oracle.block_scores(q, summ, sl)
    idx_plain, _ = oracle.select(plain, sl, 1, 0, 0)
    ws = oracle.block_scores_weighted(q, summ, sl, oracle.fasa_weights(D, [20]))
    idx_w, _ = oracle.select(ws, sl, 1, 0, 0)
    assert idx_plain.tolist() == [[[5]]] and idx_w.tolist() == [[[9]]]


def test_losa_generator_plants_what_the_classification_finds():
    # the synthetic previous queries separate the planted active tokens by a wide margin:
    # both rules of the oracle recover them (stable change ~4e-4, active ~2 per element)
    case = synth.losa_case(B=2, Hkv=2, G=4, D=64, Tq=32, T_prefix=128, n_active=8, topk=2, seed=46)
    mse, act = oracle.losa_classify(case.q, case.q_prev, tau=0.1)
    assert torch.equal(act, case.active)
    _, act = oracle.losa_classify(case.q, case.q_prev, n_top=8)
    assert torch.equal(act, case.active)
    on = case.active.bool()
    assert float(mse[~on].max()) < 1e-3 < 1.0 < float(mse[on].min())
