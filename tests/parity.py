"""Shared parity rules for the GPU tests (compare the CUDA path with the fp64 oracle).

Tolerances (stated for the workloads): outputs within 1e-2 max-abs error for bf16 I/O and
1e-5 for fp32 I/O, against the oracle evaluated on the GPU's own selection.  Selection
indices must equal the oracle's wherever the gap between the k-th and (k+1)-th best
oracle scores exceeds 1e-3 * max(|s_k|, |s_k+1|); inside that band any set whose oracle
scores differ from the best only within the band is accepted."""
import math

import torch

TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-2}
LSE_TOL = {torch.float32: 1e-5, torch.bfloat16: 1e-3}
GAP_REL = 1e-3


def forced_set(NB, topk, n_sink, n_local):
    if NB <= topk:
        return set(range(NB))
    return set(range(min(n_sink, NB))) | set(range(max(0, NB - n_local), NB))


def check_selection(gpu_row, scores_row, NB, topk, n_sink, n_local, where=""):
    """gpu_row: the GPU's idx row (ascending, -1 padded); scores_row: oracle fp64 scores.

    Returns True when the oracle's choice is unique under the gap rule (and matched)."""
    gpu = [int(j) for j in gpu_row if int(j) >= 0]
    assert gpu == sorted(gpu) and len(gpu) == len(set(gpu)), f"{where}: not ascending/unique {gpu}"
    assert len(gpu) == min(topk, NB), f"{where}: {len(gpu)} selected, want {min(topk, NB)}"
    assert all(0 <= j < NB for j in gpu), f"{where}: index out of range"
    F = forced_set(NB, topk, n_sink, n_local)
    assert F <= set(gpu), f"{where}: forced blocks missing"
    if NB <= topk:
        return True
    m = topk - len(F)
    cand = sorted(((float(scores_row[j]), -j) for j in range(NB) if j not in F), reverse=True)
    s_k, s_k1 = cand[m - 1][0], cand[m][0]
    band = GAP_REL * max(abs(s_k), abs(s_k1))
    oracle_free = {-c[1] for c in cand[:m]}
    gpu_free = set(gpu) - F
    if s_k - s_k1 > band:
        assert gpu_free == oracle_free, f"{where}: selection differs outside the near-tie band"
        return True
    # near tie: every chosen block scores within the band of the k-th, every other below it
    for j in gpu_free:
        assert float(scores_row[j]) >= s_k - band, f"{where}: block {j} too low"
    for j in set(range(NB)) - F - gpu_free:
        assert float(scores_row[j]) <= s_k + band, f"{where}: block {j} wrongly dropped"
    return False


def max_abs(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    both_inf = torch.isinf(a) & torch.isinf(b) & (torch.sign(a) == torch.sign(b))
    d = (a - b).abs()
    d[both_inf] = 0.0
    return float(d.max()) if d.numel() else 0.0


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits): 2^(e - 8) for
    2^e <= |x| < 2^(e + 1) -- the most that rounding x to bf16 (nearest) moves it."""
    ax = x.abs().clamp_min(2.0 ** -126)
    return torch.exp2(torch.floor(torch.log2(ax)) - 8)


def max_abs_beyond_rounding(gpu, ref):
    """max over elements of |gpu - ref| - bf16_half_ulp(ref): the error of a bf16 output
    beyond the rounding of the exact value to bf16 (compare with TOL[torch.bfloat16]).
    A bf16 output cannot be closer to the exact value than that rounding: where |ref| >= 2
    its half-ulp (>= 2^-7) is a sizeable share of a 1e-2 bound, and where |ref| < 1 it is
    at most 2^-9."""
    a = gpu.double().cpu()
    b = ref.double().cpu()
    d = (a - b).abs() - bf16_half_ulp(b)
    return float(d.max()) if d.numel() else 0.0


def nsel_of(idx):
    return (idx >= 0).sum(-1).to(torch.int32)
