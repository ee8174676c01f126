"""Launches from several host threads at once: every entry point keeps its one-time set-up
(shared-memory attribute, occupancy check) per device under a lock, so threads that launch
different shapes concurrently on their own streams must all get correct results.  Eight
threads each run fused decode (shapes that need different shared-memory sizes and cluster
sizes), block-query and the BLASST prefill on their own stream, and every result is checked
against the fp64 oracle."""
import threading

import pytest
import torch

import oracle
import synth
from tests.parity import LSE_TOL, TOL, max_abs, max_abs_beyond_rounding, nsel_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa(cuda_device):
    import query_aware_block_b200 as m
    return m


def _decode_job(lsa, i, stream):
    # per thread a different capacity (summary slice, hence shared memory) and unit count
    # (hence cluster size)
    B = [1, 2, 24, 3, 1, 40, 2, 5][i]
    T = [64 * 300, 64 * 700 + 9, 64 * 40, 5000, 64 * 1100 + 7, 64 * 30, 2048, 64 * 90][i]
    case = synth.decode_case(B=B, Hkv=2, G=4, D=128, T_cap=T, seqlens=T, dtype=torch.bfloat16,
                             topk=16, n_sink=1, n_local=2, seed=300 + i)
    with torch.cuda.stream(stream):
        q, k, v, sl = (t.cuda() for t in (case.q, case.k, case.v, case.seqlens))
        summ = torch.zeros(B, 2, -(-T // 64), 128, device="cuda")
        lsa.lsa_build_summaries(k, sl, summ)
        o = torch.empty_like(q)
        lse = torch.empty(B, 8, device="cuda")
        idx = torch.empty(B, 2, 16, device="cuda", dtype=torch.int32)
        for _ in range(3):
            lsa.lsa_sparse_attn_decode(q, k, v, sl, o, 16, summ=summ, n_sink=1, n_local=2,
                                       idx_out=idx, lse=lse)
        stream.synchronize()
    idx_c = idx.cpu()
    o_ref, lse_ref = oracle.decode_attn(case.q, case.k, case.v, case.seqlens, idx_c, nsel_of(idx_c))
    return max_abs(o.float().cpu(), o_ref), max_abs(lse.cpu(), lse_ref)


def _prefill_job(lsa, i, stream):
    L = [256, 300, 512, 640][i % 4]
    case = synth.prefill_case(B=1, Hq=4, Hkv=2, L=L, D=128, lam=0.0, seed=320 + i)
    with torch.cuda.stream(stream):
        q, k, v = case.q.cuda(), case.k.cuda(), case.v.cuda()
        o = torch.empty_like(q)
        lse = torch.empty(1, 4, L, device="cuda")
        lsa.lsa_blasst_prefill(q, k, v, o, 0.0, lse=lse)
        stream.synchronize()
    units = [(0, h, a) for h in range(4) for a in range(-(-L // 128))]
    r = oracle.blasst_prefill(case.q, case.k, case.v, units, 0.0)
    err = lerr = 0.0
    oc, lc = o.cpu(), lse.cpu()
    for u, (b, h, a) in enumerate(units):
        n = min(128, L - 128 * a)
        # early rows of a causal prefill keep |o| up to ~4 (row 0 is v_0), where the bf16
        # output's own rounding reaches 2^-8 |o|: the bound applies beyond that rounding
        err = max(err, max_abs_beyond_rounding(oc[b, h, 128 * a:128 * a + n].float(), r["o"][u, :n]))
        lerr = max(lerr, max_abs(lc[b, h, 128 * a:128 * a + n], r["lse"][u, :n]))
    return err, lerr


def test_concurrent_launches_from_eight_threads(lsa):
    results = {}
    errors = []
    streams = [torch.cuda.Stream() for _ in range(8)]
    barrier = threading.Barrier(8)

    def run(i):
        try:
            torch.cuda.set_device(0)
            barrier.wait()
            results[("decode", i)] = _decode_job(lsa, i, streams[i])
            results[("prefill", i)] = _prefill_job(lsa, i, streams[i])
        except Exception as e:  # noqa: BLE001 (re-raised below with the thread's index)
            errors.append((i, repr(e)))

    threads = [threading.Thread(target=run, args=(i,)) for i in range(8)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for (kind, i), (err, lerr) in results.items():
        assert err <= TOL[torch.bfloat16], f"{kind} thread {i}: o err {err}"
        assert lerr <= LSE_TOL[torch.bfloat16], f"{kind} thread {i}: lse err {lerr}"
    assert len(results) == 16
    assert lsa.lsa_device_status() == 0
