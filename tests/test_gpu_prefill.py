"""GPU parity of the BLASST causal prefill (tcgen05 kernel) against the fp64 oracle, through
the C ABI.  lambda = 0 must give plain causal attention; with lambda > 0 the GPU's skip
decisions must equal the oracle's wherever the oracle's gap is more than 1e-3 (in logit
units) away from ln(lambda), and the outputs must equal the oracle evaluated on the GPU's
own decisions.  Ragged lengths, GQA, several sequences, and the 32K workload on sampled
query tiles."""
import math

import pytest
import torch

import oracle
import synth
from tests.parity import LSE_TOL, TOL, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa(cuda_device):
    import query_aware_block_b200 as m
    return m


def _run(lsa, case):
    d = torch.device("cuda:0")
    q, k, v = case.q.to(d), case.k.to(d), case.v.to(d)
    B, Hq, L, D = q.shape
    nqt = -(-L // 128)
    words = -(-(-(-L // 64)) // 32)
    o = torch.full_like(q, 3.0)
    lse = torch.full((B, Hq, L), 3.0, device=d)
    bits = torch.full((B, Hq, nqt, words), 0x7fffffff, dtype=torch.int32, device=d)
    cnt = torch.zeros(1, dtype=torch.int64, device=d)
    lsa.lsa_blasst_prefill(q, k, v, o, case.lam, lse=lse, skip_bits=bits, skipped_tiles=cnt)
    torch.cuda.synchronize()
    assert lsa.lsa_device_status() == 0
    return o.cpu(), lse.cpu(), bits.cpu().to(torch.int64) & 0xFFFFFFFF, int(cnt.item())


def _check_units(case, o, lse, bits, units, where):
    B, Hq, L, D = case.q.shape
    ln_lam = math.log(case.lam) if case.lam > 0 else -math.inf
    gpu_bits = torch.stack([bits[b, h, a] for (b, h, a) in units])
    r = oracle.blasst_prefill(case.q, case.k, case.v, units, case.lam, forced_bits=gpu_bits)
    nskip = 0
    for u, (b, h, a) in enumerate(units):
        n = min(128, L - 128 * a)
        nvisit = (min(128 * a + 128, L) - 1) // 64 + 1
        for c in range(nvisit):
            gbit = (int(gpu_bits[u, c // 32]) >> (c % 32)) & 1
            nskip += gbit
            gap = float(r["gap"][u, c])
            if abs(gap - ln_lam) > 1e-3:
                assert gbit == (1 if gap < ln_lam else 0), f"{where}: unit {(b, h, a)} tile {c} gap {gap}"
        for c in range(nvisit, 32 * gpu_bits.shape[1]):
            assert (int(gpu_bits[u, c // 32]) >> (c % 32)) & 1 == 0
        rows = slice(128 * a, 128 * a + n)
        err = max_abs(o[b, h, rows].float(), r["o"][u, :n])
        assert err <= TOL[torch.bfloat16], f"{where}: unit {(b, h, a)} o err {err}"
        lerr = max_abs(lse[b, h, rows], r["lse"][u, :n])
        assert lerr <= LSE_TOL[torch.bfloat16], f"{where}: unit {(b, h, a)} lse err {lerr}"
    return nskip


@pytest.mark.parametrize("L", [50, 128, 256, 300, 1000])
def test_prefill_lambda_zero_is_causal_attention(lsa, L):
    case = synth.prefill_case(B=1, Hq=4, Hkv=2, L=L, D=128, lam=0.0, seed=71)
    o, lse, bits, cnt = _run(lsa, case)
    assert cnt == 0 and int(bits.sum()) == 0
    units = [(0, h, a) for h in range(4) for a in range(-(-L // 128))]
    _check_units(case, o, lse, bits, units, f"L={L}")


@pytest.mark.parametrize("B,Hq,Hkv,L,lam,sink", [
    (1, 2, 1, 512, 0.05, 7.0),
    (2, 8, 2, 640, 1e-3, 9.0),
    (1, 4, 4, 777, 1e-2, 8.0),
])
def test_prefill_skips_match_oracle(lsa, B, Hq, Hkv, L, lam, sink):
    case = synth.prefill_case(B=B, Hq=Hq, Hkv=Hkv, L=L, D=128, lam=lam, sink=sink, seed=72)
    o, lse, bits, cnt = _run(lsa, case)
    units = [(b, h, a) for b in range(B) for h in range(Hq) for a in range(-(-L // 128))]
    nskip = _check_units(case, o, lse, bits, units, f"{(B, Hq, Hkv, L, lam)}")
    assert nskip == cnt
    assert cnt > 0, "the sink inputs must make some tiles skippable"


def test_blasst_prefill_32k_workload_sampled(lsa):
    case = synth.blasst_prefill_32k()
    o, lse, bits, cnt = _run(lsa, case)
    # every KV group (4 query heads each): the first tiles, a mid-diagonal tile that moves
    # with the group, and the last (diagonal) tile; plus the heaviest tiles of three heads
    units = [(0, 4 * g + g % 4, a) for g in range(8) for a in (0, 1 + 3 * g, 64 + 17 * g, 255)]
    units += [(0, h, a) for h in (0, 13, 31) for a in (97, 254)]
    _check_units(case, o, lse, bits, units, "32K workload")
    total = sum(bin(int(w)).count("1") for w in bits.flatten())
    assert total == cnt
