"""The seeded input recipes (synth/) on CPU, at reduced sizes: the properties the workload
descriptions state -- shapes, dtypes, seeds, planted needles, sequence-length ranges,
poisoned tails, active counts, the LoSA query change and the prefill's attention sink.
synth draws inputs only; nothing here computes the method."""
import math

import torch

import synth


def test_tiny_decode_recipe_and_seeding():
    a = synth.tiny_decode()
    assert a.q.shape == (1, 4, 64) and a.k.shape == (1, 1, 2048, 64) and a.v.shape == a.k.shape
    assert a.q.dtype == a.k.dtype == torch.float32
    assert a.seqlens.tolist() == [2048] and (a.topk, a.n_sink, a.n_local) == (8, 1, 2)
    b = synth.tiny_decode()
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    c = synth.tiny_decode(seed=1234)
    assert not torch.equal(a.k, c.k)


def test_needles_sit_in_free_full_blocks_along_the_group_query():
    B, Hkv, G, D, blk = 2, 2, 2, 32, 64
    case = synth.decode_case(B, Hkv, G, D, T_cap=1000, seqlens=[1000, 700], dtype=torch.float32,
                             topk=8, n_sink=1, n_local=2, n_needles=3, seed=81)
    assert len(case.needles) == B * Hkv
    for b, g, blocks in case.needles:
        T = int(case.seqlens[b])
        NB = -(-T // blk)
        assert len(blocks) == 3 and blocks == sorted(set(blocks))
        for j in blocks:
            assert 1 <= j < NB - 2 and (j + 1) * blk <= T  # not forced, full length
        u = case.q[b, g * G:(g + 1) * G].double().mean(0)
        u = u / u.norm()
        for j in range(NB):
            rows = case.k[b, g, j * blk:min(T, (j + 1) * blk)].double()
            cos = (rows @ u / rows.norm(dim=1)).mean()
            if j in blocks:  # key = sqrt(D) u + 0.5 N(0, I): cosine about 1 / sqrt(1.25)
                assert cos > 0.8, (b, g, j, float(cos))
            else:
                assert abs(cos) < 0.3, (b, g, j, float(cos))


def test_batched_decode_lengths_and_poisoned_tails():
    case = synth.batched_decode(B=6, T_lo=100, T_hi=300, poison_tail=True)
    sl = case.seqlens.tolist()
    assert case.k.shape == (6, 8, 300, 128) and case.k.dtype == torch.bfloat16
    assert all(100 <= t <= 300 for t in sl) and len(set(sl)) > 1
    for b, T in enumerate(sl):
        assert torch.isfinite(case.k[b, :, :T].float()).all() and torch.isfinite(case.v[b, :, :T].float()).all()
        assert torch.isnan(case.k[b, :, T:].float()).all() and torch.isnan(case.v[b, :, T:].float()).all()
    assert (case.topk, case.n_sink, case.n_local) == (16, 1, 2)


def test_blockquery_case_active_tokens_and_caches():
    case = synth.blockquery_case(B=3, Hkv=1, G=2, D=32, Tq=16, T_prefix=200, n_active=5, topk=4, seed=82)
    assert case.q.shape == (3, 2, 16, 32) and case.q.is_contiguous() and case.q.dtype == torch.bfloat16
    assert case.k.shape == (3, 1, 200, 32) and case.active.dtype == torch.uint8
    assert case.active.sum(1).tolist() == [5, 5, 5]
    assert case.o_cache.shape == case.q.shape and case.lse_cache.shape == (3, 2, 16)
    assert abs(float(case.lse_cache.mean()) - 10.0) < 0.5  # N(0, 1) + 10
    same = synth.blockquery_case(B=1, Hkv=1, G=2, D=32, Tq=8, T_prefix=128, same_query=True, seed=83)
    assert torch.equal(same.q[:, :, :1].expand_as(same.q), same.q)


def test_losa_case_query_change_separates_active_from_stable():
    case = synth.losa_case(B=2, Hkv=1, G=2, D=64, Tq=16, T_prefix=256, n_active=4, seed=84)
    assert case.k.shape[2] == 256 + 16  # the block's own rows follow the prefix
    change = (case.q.float() - case.q_prev.float()).pow(2).mean(dim=(1, 3))  # [B, Tq]
    on = case.active.bool()
    assert float(change[~on].max()) < 0.01       # stable: 0.02 * N(0, 1), about 4e-4
    assert float(change[on].min()) > 1.0         # active: a fresh draw, about 2
    assert on.sum(1).tolist() == [4, 4]


def test_prefill_sink_raises_the_first_keys_logits_by_about_its_height():
    L, D, sink = 256, 128, 10.5
    case = synth.prefill_case(B=1, Hq=2, Hkv=1, L=L, D=D, sink=sink, seed=85)
    plain = synth.prefill_case(B=1, Hq=2, Hkv=1, L=L, D=D, seed=85)
    assert case.q.shape == (1, 2, L, D) and case.k.shape == (1, 1, L, D)
    s = (case.q[0].float() @ case.k[0, 0].float().T) / math.sqrt(D)  # [Hq, L, L]
    gap = float(s[:, :, :64].mean() - s[:, :, 64:].mean())
    assert abs(gap - sink) < 1.0, gap
    s0 = (plain.q[0].float() @ plain.k[0, 0].float().T) / math.sqrt(D)
    assert abs(float(s0[:, :, :64].mean() - s0[:, :, 64:].mean())) < 0.3
