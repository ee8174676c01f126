"""GPU parity of the decode family (summaries, selection, sparse decode attention) against
the fp64 oracle, through the C ABI, on seeded synthetic inputs: small shapes that span
several cluster slices and ragged tails, the three decode workloads at full size, and the
edge cases (empty sequences, NB <= topk, partial last blocks with NaN-poisoned tails,
G = 1 / 16, D = 64 / 128, fp32 / bf16)."""
import math

import pytest
import torch

import oracle
import synth
from tests.parity import LSE_TOL, TOL, check_selection, max_abs, nsel_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa(cuda_device):
    import query_aware_block_b200 as m
    return m


def _dev(case):
    d = torch.device("cuda:0")
    return (case.q.to(d), case.k.to(d), case.v.to(d), case.seqlens.to(d))


def _gpu_summaries(lsa, k, sl, nb_begin=0, nb_end=-1, fill=0.0):
    B, Hkv, T_cap, D = k.shape
    summ = torch.full((B, Hkv, -(-T_cap // 64), D), fill, device=k.device, dtype=torch.float32)
    lsa.lsa_build_summaries(k, sl, summ, nb_begin, nb_end)
    return summ


# ------------------------------------------------------------------------ summaries ----

@pytest.mark.parametrize("dtype,D", [(torch.float32, 64), (torch.float32, 128),
                                     (torch.bfloat16, 64), (torch.bfloat16, 128)])
def test_summaries_match_oracle(lsa, dtype, D):
    case = synth.decode_case(B=3, Hkv=2, G=1, D=D, T_cap=1000, seqlens=[1000, 1, 640],
                             dtype=dtype, topk=4, n_sink=1, n_local=1, seed=41, poison_tail=True)
    q, k, v, sl = _dev(case)
    summ = _gpu_summaries(lsa, k, sl)
    ref = oracle.summaries(case.k, case.seqlens)
    torch.cuda.synchronize()
    for b, T in enumerate(case.seqlens.tolist()):
        NB = -(-T // 64)
        assert max_abs(summ[b, :, :NB], ref[b, :, :NB]) < 1e-5
        assert torch.count_nonzero(summ[b, :, NB:]) == 0  # untouched past NB_b


def test_summaries_ranges(lsa):
    case = synth.decode_case(B=2, Hkv=2, G=1, D=128, T_cap=700, seqlens=[700, 300],
                             dtype=torch.bfloat16, topk=4, n_sink=1, n_local=1, seed=42)
    q, k, v, sl = _dev(case)
    ref = oracle.summaries(case.k, case.seqlens)
    last = _gpu_summaries(lsa, k, sl, -1, -1, fill=7.0)  # last block of each sequence only
    mid = _gpu_summaries(lsa, k, sl, 2, 5, fill=7.0)     # blocks [2, 5) clipped to NB_b
    torch.cuda.synchronize()
    for b, NB in ((0, 11), (1, 5)):
        for j in range(11):
            want_last = j == NB - 1
            want_mid = 2 <= j < min(5, NB)
            for got, want in ((last, want_last), (mid, want_mid)):
                if want:
                    assert max_abs(got[b, :, j], ref[b, :, j]) < 1e-5
                else:
                    assert bool((got[b, :, j] == 7.0).all())


# ------------------------------------------------------------------------ selection ----

@pytest.mark.parametrize("B,Hkv,G,D,T,topk,ns,nl,dtype", [
    (1, 2, 4, 128, 64 * 300, 16, 1, 2, torch.bfloat16),     # 300 blocks over a 16-CTA cluster
    (2, 3, 8, 64, [5000, 2000], 8, 1, 2, torch.float32),
    (1, 1, 1, 128, 64 * 40 + 17, 13, 0, 0, torch.bfloat16),  # no forcing, ragged tail
    (3, 2, 16, 128, [64 * 1000, 640, 70], 64, 2, 3, torch.bfloat16),  # topk 64, NB <= topk rows
    (40, 2, 2, 64, 64 * 100, 16, 1, 2, torch.float32),      # many units: smaller clusters
])
def test_select_matches_oracle(lsa, B, Hkv, G, D, T, topk, ns, nl, dtype):
    T_cap = max(T) if isinstance(T, list) else T
    case = synth.decode_case(B, Hkv, G, D, T_cap, T, dtype, topk, ns, nl, seed=43)
    q, k, v, sl = _dev(case)
    summ_ref = oracle.summaries(case.k, case.seqlens)
    scores_ref = oracle.block_scores(case.q, summ_ref, case.seqlens)
    summ = summ_ref.float().cuda()  # selection on the same (rounded) summaries
    NB_cap = summ.shape[2]
    idx = torch.full((B, Hkv, topk), -7, device="cuda", dtype=torch.int32)
    nsel = torch.zeros(B, Hkv, device="cuda", dtype=torch.int32)
    sc = torch.zeros(B, Hkv, NB_cap, device="cuda")
    lsa.lsa_select_blocks(q, summ, sl, topk, ns, nl, idx, nsel, scores_out=sc)
    idx, nsel, sc = idx.cpu(), nsel.cpu(), sc.cpu()
    for b in range(B):
        NB = -(-int(case.seqlens[b]) // 64)
        for g in range(Hkv):
            check_selection(idx[b, g], scores_ref[b, g], NB, topk, ns, nl, f"b{b}g{g}")
            assert int(nsel[b, g]) == min(topk, NB)
            if NB > topk:
                rel = (sc[b, g, :NB].double() - scores_ref[b, g, :NB]).abs().max()
                assert float(rel) < 1e-4 * (1 + float(scores_ref[b, g, :NB].abs().max()))


def test_select_ties_go_to_lower_index(lsa):
    # identical summaries for every block: all scores tie, the lowest indices win
    B, Hkv, G, D, NB = 1, 1, 2, 64, 50
    summ = torch.ones(B, Hkv, NB, D, device="cuda")
    q = torch.randn(B, G, D, device="cuda")
    sl = torch.tensor([NB * 64], dtype=torch.int32, device="cuda")
    idx = torch.zeros(B, Hkv, 8, device="cuda", dtype=torch.int32)
    nsel = torch.zeros(B, Hkv, device="cuda", dtype=torch.int32)
    lsa.lsa_select_blocks(q, summ, sl, 8, 1, 2, idx, nsel)
    assert idx[0, 0].tolist() == [0, 1, 2, 3, 4, 5, 48, 49]


# ------------------------------------------------------------------ decode attention ----

def _check_attention(case, o, lse, idx_gpu, dtype, where):
    """Compare o / lse with the oracle evaluated on the GPU's own block choice."""
    idx_cpu = idx_gpu.cpu()
    o_ref, lse_ref = oracle.decode_attn(case.q, case.k, case.v, case.seqlens, idx_cpu,
                                        nsel_of(idx_cpu))
    err = max_abs(o.float().cpu(), o_ref)
    assert err <= TOL[dtype], f"{where}: o max abs err {err}"
    lerr = max_abs(lse.cpu(), lse_ref)
    assert lerr <= LSE_TOL[dtype], f"{where}: lse max abs err {lerr}"
    return err


def _run_both_modes(lsa, case, dtype, check_sel=True):
    q, k, v, sl = _dev(case)
    B, Hkv, G, D, T_cap = case.shape
    topk, ns, nl = case.topk, case.n_sink, case.n_local
    summ = _gpu_summaries(lsa, k, sl)
    # given selection: the oracle's own choice
    r = oracle.decode(case.q, case.k, case.v, case.seqlens, topk, ns, nl)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hkv * G, device="cuda")
    lsa.lsa_sparse_attn_decode(q, k, v, sl, o, topk, idx=r["idx"].cuda(), nsel=r["nsel"].cuda(),
                               lse=lse)
    _check_attention(case, o, lse, r["idx"], dtype, "given")
    # fused selection + attention; when the last block is forced, also refresh its summary
    # (poisoned first, so a refresh that did not happen or was read by the scan shows)
    refresh = nl >= 1
    summ_ref = oracle.summaries(case.k, case.seqlens)
    if refresh:
        for b in range(B):
            NB = -(-int(case.seqlens[b]) // 64)
            if NB:
                summ[b, :, NB - 1] = float("nan")
    o2 = torch.empty_like(q)
    lse2 = torch.empty(B, Hkv * G, device="cuda")
    idx2 = torch.full((B, Hkv, topk), -7, device="cuda", dtype=torch.int32)
    lsa.lsa_sparse_attn_decode(q, k, v, sl, o2, topk, summ=summ, n_sink=ns, n_local=nl,
                               refresh_last_summary=refresh, idx_out=idx2, lse=lse2)
    idx2c = idx2.cpu()
    if refresh:
        sc = summ.cpu()
        for b in range(B):
            NB = -(-int(case.seqlens[b]) // 64)
            if NB:
                assert max_abs(sc[b, :, NB - 1], summ_ref[b, :, NB - 1]) < 1e-5, "refresh"
                assert max_abs(sc[b, :, :NB - 1], summ_ref[b, :, :NB - 1]) < 1e-5
    if check_sel:
        for b in range(B):
            NB = -(-int(case.seqlens[b]) // 64)
            for g in range(Hkv):
                check_selection(idx2c[b, g], r["scores"][b, g], NB, topk, ns, nl, f"fused b{b}g{g}")
    _check_attention(case, o2, lse2, idx2c, dtype, "fused")
    assert lsa.lsa_device_status() == 0, "a bounded cross-CTA wait ran out"
    return r, idx2c


@pytest.mark.parametrize("B,Hkv,G,D,T,topk,ns,nl,dtype", [
    (1, 1, 4, 64, 2048, 8, 1, 2, torch.float32),
    (1, 2, 8, 128, 64 * 200 + 5, 16, 1, 2, torch.bfloat16),
    (2, 2, 1, 128, [3000, 64], 8, 1, 2, torch.bfloat16),
    (2, 1, 16, 64, [64 * 90, 1000], 12, 2, 1, torch.bfloat16),
    (1, 2, 3, 128, 64 * 50, 32, 0, 0, torch.float32),
    (3, 2, 4, 128, [0, 100, 64 * 70 + 1], 16, 1, 2, torch.bfloat16),  # empty sequence
    (20, 3, 2, 64, 64 * 40, 4, 1, 1, torch.bfloat16),  # 60 units -> 8-CTA clusters, 1 CTA of work
    (80, 1, 4, 128, 64 * 20, 6, 1, 2, torch.float32),  # 80 units -> 4-CTA clusters, 2 blocks each
    # 1,100 blocks: 69 summary rows per CTA, two scoring passes (the second from global memory)
    (1, 1, 8, 128, 64 * 1100 + 7, 16, 1, 2, torch.bfloat16),
])
def test_decode_matches_oracle(lsa, B, Hkv, G, D, T, topk, ns, nl, dtype):
    T_cap = max(T) if isinstance(T, list) else T
    T_cap = max(T_cap, 1)
    case = synth.decode_case(B, Hkv, G, D, T_cap, T, dtype, topk, ns, nl, seed=44,
                             poison_tail=True)
    _run_both_modes(lsa, case, dtype)


def test_decode_empty_sequence_outputs(lsa):
    case = synth.decode_case(2, 1, 2, 64, 128, [0, 128], torch.float32, 4, 1, 1, seed=45)
    q, k, v, sl = _dev(case)
    summ = _gpu_summaries(lsa, k, sl)
    o = torch.full_like(q, 3.0)
    lse = torch.zeros(2, 2, device="cuda")
    idx = torch.zeros(2, 1, 4, device="cuda", dtype=torch.int32)
    lsa.lsa_sparse_attn_decode(q, k, v, sl, o, 4, summ=summ, n_sink=1, n_local=1, idx_out=idx,
                               lse=lse)
    assert torch.count_nonzero(o[0]) == 0
    assert bool(torch.isinf(lse[0]).all()) and bool((lse[0] < 0).all())
    assert idx[0, 0].tolist() == [-1, -1, -1, -1] and idx[1, 0].tolist() == [0, 1, -1, -1]


# --------------------------------------------------------------- the three workloads ----

def test_tiny_fp32_decode(lsa):
    case = synth.tiny_decode()
    _run_both_modes(lsa, case, torch.float32)


def test_gqa_decode_64k(lsa):
    case = synth.gqa_decode_64k()
    r, idx = _run_both_modes(lsa, case, torch.bfloat16)
    # needle recall: 13 free slots, 16 planted needles per group -> 13 needles selected
    for (b, g, blocks) in case.needles:
        chosen = set(int(j) for j in idx[b, g] if j >= 0)
        assert len(chosen & set(blocks)) == 13


def test_batched_varlen_decode(lsa):
    case = synth.batched_decode(poison_tail=True)
    _run_both_modes(lsa, case, torch.bfloat16)


# ------------------------------------------------------------ append + decode step ----

@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_append_then_decode_step(lsa, dtype, D):
    """A decode step as a serving loop runs it: the newest token's k/v appended by
    lsa_append_kv (its cache row NaN before), then the fused decode launched with
    LSA_FLAG_PDL (its prologue overlaps the append).  The cache must equal the original bit
    for bit, and the outputs must match the oracle on the original inputs."""
    case = synth.decode_case(B=3, Hkv=2, G=4, D=D, T_cap=64 * 60, seqlens=[64 * 60, 64 * 31 + 1, 0],
                             dtype=dtype, topk=8, n_sink=1, n_local=2, seed=46, poison_tail=True)
    q, k, v, sl = _dev(case)
    B, Hkv, G, D, T_cap = case.shape
    last = [int(t) - 1 for t in case.seqlens.tolist()]
    k_new = torch.zeros(B, Hkv, D, device="cuda", dtype=dtype)
    v_new = torch.zeros_like(k_new)
    for b in range(B):
        if last[b] >= 0:
            k_new[b] = k[b, :, last[b]]
            v_new[b] = v[b, :, last[b]]
            k[b, :, last[b]] = float("nan")
            v[b, :, last[b]] = float("nan")
    summ = _gpu_summaries(lsa, case.k.cuda(), sl)  # the prefill's summaries of the true keys
    o = torch.empty_like(q)
    lse = torch.empty(B, Hkv * G, device="cuda")
    idx = torch.empty(B, Hkv, case.topk, device="cuda", dtype=torch.int32)
    lsa.lsa_append_kv(k_new, v_new, sl, k, v)
    lsa.lsa_sparse_attn_decode(q, k, v, sl, o, case.topk, summ=summ, n_sink=1, n_local=2,
                               refresh_last_summary=True, idx_out=idx, lse=lse,
                               flags=lsa.LSA_FLAG_PDL)
    torch.cuda.synchronize()
    kc, vc = k.cpu(), v.cpu()
    for b in range(B):
        T = int(case.seqlens[b])
        # bit-exact up to the sequence end (rows past it keep their poison)
        assert torch.equal(kc[b, :, :T].view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                           case.k[b, :, :T].view(torch.int16 if dtype == torch.bfloat16 else torch.int32))
        assert torch.equal(vc[b, :, :T].view(torch.int16 if dtype == torch.bfloat16 else torch.int32),
                           case.v[b, :, :T].view(torch.int16 if dtype == torch.bfloat16 else torch.int32))
    _check_attention(case, o, lse, idx, dtype, "append + decode")
    assert lsa.lsa_device_status() == 0
