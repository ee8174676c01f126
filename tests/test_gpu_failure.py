"""Failure detection on the GPU without a fault: a bounded wait is made to run out, and the
kernel must stop cleanly, report LSA_DEVICE_TIMEOUT in the device status word, and leave
the context usable.

The wait limit is shortened to about a millisecond (lsa_debug_set_wait_budget) and the
prefill is told never to signal its first S tile (lsa_debug_inject), a flag nothing else
sets: its softmax warps' wait for that tile runs out, every role leaves its loop, the TMA
producers and the MMA thread wait for the copies and tensor-core work they issued, the
tensor memory is freed, and the status word is set.  No fault, trap or endless wait is
involved.  A normal launch afterwards must match the oracle."""
import pytest
import torch

import oracle
import synth
from tests.parity import LSE_TOL, TOL, max_abs, max_abs_beyond_rounding

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa(cuda_device):
    import query_aware_block_b200 as m
    return m


def _prefill(lsa, case):
    d = torch.device("cuda:0")
    q, k, v = case.q.to(d), case.k.to(d), case.v.to(d)
    o = torch.zeros_like(q)
    lse = torch.zeros(q.shape[0], q.shape[1], q.shape[2], device=d)
    lsa.lsa_blasst_prefill(q, k, v, o, case.lam, lse=lse)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def test_prefill_wait_runs_out_and_the_context_survives(lsa):
    case = synth.prefill_case(B=1, Hq=2, Hkv=1, L=256, D=128, lam=0.0, seed=81)
    lsa.lsa_device_status(reset=True)
    lsa.lsa_debug_set_wait_budget(2_000_000)  # about a millisecond of clock
    lsa.lsa_debug_inject(lsa.LSA_DEBUG_PREFILL_DROP_S)
    try:
        _prefill(lsa, case)
        assert lsa.lsa_device_status(reset=True) == lsa.LSA_DEVICE_TIMEOUT
    finally:
        lsa.lsa_debug_inject(0)
        lsa.lsa_debug_set_wait_budget(0)
    # the same launch without the injection: correct, and no timeout
    o, lse = _prefill(lsa, case)
    assert lsa.lsa_device_status() == 0
    units = [(0, h, a) for h in range(2) for a in range(2)]
    r = oracle.blasst_prefill(case.q, case.k, case.v, units, 0.0)
    for u, (b, h, a) in enumerate(units):
        rows = slice(128 * a, 128 * a + 128)
        assert max_abs_beyond_rounding(o[b, h, rows].float(), r["o"][u]) <= TOL[torch.bfloat16]
        assert max_abs(lse[b, h, rows], r["lse"][u]) <= LSE_TOL[torch.bfloat16]
