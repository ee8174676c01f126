#!/usr/bin/env python
"""Benchmark of the query-aware block-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gqa_decode_64k|batched_decode|tiny_decode|blockquery|
                                losa_step|decode_blasst|nsa_decode|blasst_prefill_32k]

Default workload: 64K-context GQA decode, bf16 (1 sequence, 8 KV heads x 8 query heads,
head dim 128, 65,536 cached tokens = 1,024 blocks of 64, top-16 blocks per KV head with
block 0 and the last 2 blocks forced, 16 planted needle blocks per group).

One step = one decode step of the whole hot path in one launch of lsa_sparse_attn_decode
(idx == NULL, refresh_last_summary = 1): refresh of the summary of the block that holds the
newest token, block scoring + top-k selection, and sparse attention over the selected
blocks.  Inputs are resident in HBM; R distinct input
copies are rotated so that R x (bytes a step touches) exceeds 4x the L2 size, i.e. every
step reads cold data.  The K timed steps are replayed from a CUDA graph of one rotation
cycle, bracketed by barrier + synchronize, timed with CUDA events (max over ranks).

Reported: value = tokens/s over all ranks (1 token per sequence per step), the effective
HBM GB/s of the algorithmic bytes, the roofline of the dominant kernel (fused decode) with
its own CUDA-event launch duration, e2e through the C ABI with pinned host buffers (q and
the new token's k, v copied in; o, lse, idx copied out every step), SM clocks sampled
during the timed region, and the fp64 CPU oracle on a bounded sample as the CPU baseline.
Multi-GPU (torchrun): every rank decodes its own independent sequence (the path shards by
sequence with no collective): weak scaling.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "64K-ctx sparse decode tokens/s and effective KV GB/s (% of B200 HBM roofline)"
UNIT = "tokens/s"
KERNEL_SOURCES = ["query_aware_block_b200/csrc/decode.cu", "query_aware_block_b200/csrc/lsa_common.cuh",
                  "query_aware_block_b200/csrc/cluster.cuh", "query_aware_block_b200/csrc/tcgen05.cuh"]
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "decode_fused_gqa_decode_64k.md")

WORKLOADS = {
    "gqa_decode_64k": dict(B=1, Hkv=8, G=8, D=128, T_cap=65536, T=65536, topk=16, n_sink=1,
                           n_local=2, n_needles=16, dtype="bf16"),
    "batched_decode": dict(B=16, Hkv=8, G=4, D=128, T_cap=32768, T=None, topk=16, n_sink=1,
                           n_local=2, n_needles=8, dtype="bf16"),
    "tiny_decode": dict(B=1, Hkv=1, G=4, D=64, T_cap=2048, T=2048, topk=8, n_sink=1,
                        n_local=2, n_needles=0, dtype="f32"),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 200000 decode steps; 20 prefills; 20000 block-query steps)")
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["blockquery", "blasst_prefill_32k", "losa_step",
                                                          "decode_blasst", "nsa_decode"],
                    default="gqa_decode_64k")
    ap.add_argument("--prefill-sink", type=float, default=0.0,
                    help="blasst_prefill_32k: plant an attention sink of this logit height")
    ap.add_argument("--prefill-qscale", type=float, default=1.0,
                    help="prefill: scale the queries (peakier softmax, more skippable tiles)")
    ap.add_argument("--decode-qscale", type=float, default=4.0,
                    help="decode_blasst: scale of the queries (1 = the plain 64K inputs)")
    ap.add_argument("--decode-lambda", type=float, default=1e-3, help="decode_blasst: threshold")
    ap.add_argument("--decode-batched", action="store_true",
                    help="decode_blasst: the batched varlen decode inputs (16 sequences) instead of 64K")
    ap.add_argument("--rotate", type=int, default=0, help="input copies (0 = auto, > 4x L2)")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-overlap", dest="overlap", action="store_false",
                    help="launch steps without programmatic dependent launch")
    ap.add_argument("--profile-small", action="store_true",
                    help="a few launches on 2 input copies, for ncu captures")
    a = ap.parse_args()
    defaults = {"blockquery": (20000, 200), "blasst_prefill_32k": (20, 3),
                "losa_step": (8000, 200), "decode_blasst": (80000, 600),
                "nsa_decode": (20000, 200)}.get(a.workload, (200000, 600))
    if a.steps is None:
        a.steps = defaults[0]
    if a.warmup is None:
        a.warmup = defaults[1]
    return a


# ---------------------------------------------------------------------------- helpers --

def _dtype(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


def make_case(wl, seed, device):
    import synth
    w = WORKLOADS[wl]
    if wl == "batched_decode":
        return synth.batched_decode(seed=seed, device=device)
    return synth.decode_case(B=w["B"], Hkv=w["Hkv"], G=w["G"], D=w["D"], T_cap=w["T_cap"],
                             seqlens=w["T"], dtype=_dtype(w["dtype"]), topk=w["topk"],
                             n_sink=w["n_sink"], n_local=w["n_local"], n_needles=w["n_needles"],
                             theta=1e4, seed=seed, device=device)


def algorithmic_bytes(case):
    """Bytes the method must move in one decode step, from the definitions: summaries of
    the candidate blocks + K and V of the selected blocks' valid tokens + q + o + lse + idx
    + the refreshed summary of the newest block (its keys are among the selected ones).
    Returns (bytes of the fused launch, bytes a separate summary refresh would add)."""
    B, Hkv, G, D, T_cap = case.shape
    esz = case.k.element_size()
    dec = 0
    ref = 0
    for b in range(B):
        T = int(case.seqlens[b])
        NB = -(-T // 64)
        if NB > case.topk:
            nf = case.n_sink + case.n_local
            dec += Hkv * (NB - nf) * D * 4                      # candidate summaries
            nsel = case.topk
            # selected tokens: all full blocks except possibly the (forced) partial last one
            toks = (nsel - 1) * 64 + (T - (NB - 1) * 64) if case.n_local > 0 else nsel * 64
        else:
            toks = T
        dec += Hkv * toks * D * esz * 2                            # K and V
        last = T - (NB - 1) * 64 if NB else 0
        dec += Hkv * D * 4 if NB else 0                            # refreshed summary
        ref += Hkv * last * D * esz
    Hq = Hkv * G
    dec += B * Hq * D * esz * 2 + B * Hq * 4 + B * Hkv * case.topk * 4  # q, o, lse, idx
    return dec, ref


def _nvtx_push(name):
    """An NVTX range around a timed region (seen by nsys or ncu --nvtx); no-op without NVTX."""
    try:
        torch.cuda.nvtx.range_push(name)
        return True
    except (RuntimeError, AttributeError):
        return False


def _nvtx_pop(pushed):
    if pushed:
        try:
            torch.cuda.nvtx.range_pop()
        except (RuntimeError, AttributeError):
            pass


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons during the timed region, which
    is also marked as an NVTX range ("timed region")."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        self.nvtx = _nvtx_push("timed region")
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        _nvtx_pop(self.nvtx)
        time.sleep(0.2)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the fused decode from the committed ncu summary, if it was
    taken on the current kernel source; else None."""
    try:
        text = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel source hash:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"dram bytes per launch \(read \+ write\):\s*([0-9]+)", text)
    if not (m_hash and m_tr) or m_hash.group(1) != source_hash():
        return None
    return int(m_tr.group(1))


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


# ----------------------------------------------------------------------- our arm ----

# ---- the job across ranks (one process per GPU; replicas on independent sequences) ------

def rank_seed(rank, r=0):
    """Seed of rank `rank`'s r-th input copy: every rank decodes its own sequences."""
    return 1000 + 2 + 7919 * rank + 101 * r


def max_over_ranks(x, world, device):
    """The slowest rank's value (step time of the whole job)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(rate, world, device):
    """A whole-job rate from per-rank rates: the slowest rank's rate times the rank count
    (every rank does the same work)."""
    if world == 1:
        return float(rate)
    t = torch.tensor([float(rate)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MIN)
    return float(t.item()) * world


def plan_rotation(K, step_bytes, l2, rotate=0):
    """Input copies and graph length for K timed steps that each read cold data.

    r_cold = the copies whose bytes exceed 4x the L2 size.  A step's copy must have seen at
    least that much other traffic since it was last touched.
      K <  r_cold: n = ceil(r_cold / K) + 1 graphs of K steps over distinct copies (R = n K);
                   warm-up replays all of them in order and the timed region replays graph 0,
                   whose copies were last touched (n - 1) K >= r_cold steps earlier.
      K >= r_cold: one graph of R = r_cold steps replayed K // R times plus a remainder graph
                   of K % R steps; warm-up replays the remainder, then the full graph, so the
                   timed region starts on copy 0, last touched R steps earlier.
    Returns (R, steps per graph)."""
    r_cold = rotate or max(4, min(128, math.ceil(4 * l2 / step_bytes)))
    if K < r_cold:
        n = math.ceil(r_cold / K) + 1
        return n * K, K
    return r_cold, r_cold


def blocking_sleep(stream):
    """A short device-side wait queued before a start event (as nvbench's blocking kernel):
    the host then enqueues the timed launches while the GPU is still busy, so the start
    event is not followed by an idle gap while the first launch is submitted."""
    with torch.cuda.stream(stream):
        torch.cuda._sleep(200_000)  # about 0.1 ms of clock cycles


def run_ours(args, rank, world, local_rank):
    import query_aware_block_b200 as lsa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = args.workload
    # one step's algorithmic bytes set the rotation depth
    base = make_case(wl, rank_seed(rank), "cpu" if wl == "tiny_decode" else dev)
    dec_bytes, _ = algorithmic_bytes(base)
    step_bytes = dec_bytes
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    K, W = args.steps, args.warmup
    if args.profile_small:
        K, W = 2, 2
        R, per_graph = 2, 2
    else:
        R, per_graph = plan_rotation(K, step_bytes, l2, args.rotate)
    B, Hkv, G, D, T_cap = base.shape
    copies = []
    for r in range(R):
        c = base if r == 0 else make_case(wl, rank_seed(rank, r), dev)
        q, k, v, sl = (t.to(dev) for t in (c.q, c.k, c.v, c.seqlens))
        summ = torch.zeros(B, Hkv, -(-T_cap // 64), D, device=dev)
        lsa.lsa_build_summaries(k, sl, summ)  # prefill-time summaries (not timed)
        o = torch.empty_like(q)
        lse = torch.empty(B, Hkv * G, device=dev)
        idx = torch.empty(B, Hkv, base.topk, device=dev, dtype=torch.int32)
        copies.append(dict(q=q, k=k, v=v, sl=sl, summ=summ, o=o, lse=lse, idx=idx))
        del c
    torch.cuda.synchronize()
    topk, ns, nl = base.topk, base.n_sink, base.n_local

    flags = lsa.LSA_FLAG_PDL if args.overlap else 0

    def step(c, stream=None, flags=flags):
        # one launch: refresh of the newest block's summary + scoring + selection + attention
        lsa.lsa_sparse_attn_decode(c["q"], c["k"], c["v"], c["sl"], c["o"], topk, summ=c["summ"],
                                   n_sink=ns, n_local=nl, refresh_last_summary=True,
                                   idx_out=c["idx"], lse=c["lse"], flags=flags, stream=stream)

    def decode_only(c, stream=None):
        step(c, stream, flags=0)  # timed alone: no overlap with a neighbour

    # eager warm-up (also sets kernel attributes before any capture)
    for i in range(max(3, min(W, 4 * R))):
        step(copies[i % R])
    torch.cuda.synchronize()

    def capture(fn, cs):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for c in cs:
                fn(c)
        return g

    # the timed graphs (see plan_rotation)
    if per_graph == K:  # graphs of K steps over distinct copies; graph 0 is timed
        graphs = [capture(step, copies[i:i + per_graph]) for i in range(0, R, per_graph)]
        timed = [0]
        rem_graph = None
        gap_steps = R - K if len(graphs) > 1 else R  # steps since the timed copies were last touched
    else:               # a full cycle of R steps replayed K // R times, then a remainder
        graphs = [capture(step, copies)]
        rem = K - (K // R) * R
        rem_graph = capture(step, copies[:rem]) if rem else None
        timed = [0] * (K // R)
        gap_steps = R
    # the dominant kernel alone: R back-to-back launches without overlap (the average launch
    # duration then includes the launch gap, which errs on the slow side)
    g_dec = capture(decode_only, copies)
    torch.cuda.synchronize()

    def make_cold():
        """Replays that leave the timed copies last touched gap_steps steps ago (and, the
        first time, run every timed graph once untimed).  Returns the steps replayed."""
        n = 0
        if rem_graph is not None:
            rem_graph.replay()
            n += K - (K // R) * R
        for g in (graphs[1:] + graphs[:1]) if len(graphs) > 1 else graphs:
            g.replay()
            n += per_graph if len(graphs) > 1 else R
        return n

    # warm-up replays (untimed): at least W steps, ending with the data of the timed region cold
    warm_steps = 0
    while True:
        warm_steps += make_cold()
        if warm_steps >= W:
            break
    if len(graphs) > 1:  # graph 0 ran last: replay the others once more so its copies are cold
        for g in graphs[1:]:
            g.replay()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    stream = torch.cuda.current_stream()

    def timed_region():
        """Exactly K steps between two events on the launching stream."""
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        blocking_sleep(stream)
        e0.record(stream)
        for i in timed:
            graphs[i].replay()
        if rem_graph is not None:
            rem_graph.replay()
        e1.record(stream)
        return e0, e1

    with ClockSampler(local_rank) as clocks:
        barrier()
        torch.cuda.synchronize()
        e_start, e_stop = timed_region()
        torch.cuda.synchronize()
        barrier()
    ms_total = max_over_ranks(e_start.elapsed_time(e_stop), world, dev)
    ms_step = ms_total / K
    tokens = world * B * K
    value = tokens / (ms_total / 1e3)

    # the same K-step region again, each repeat preceded by replays that make its data cold
    # again: the spread of the headline (rank-local)
    reps_ms = []
    n_rep = max(3, min(20, int(2000.0 / max(ms_total, 1e-3))))
    for _ in range(n_rep):
        if len(graphs) > 1:
            for g in graphs[1:]:
                g.replay()
        elif rem_graph is not None:
            rem_graph.replay()
            graphs[0].replay()
        r0, r1 = timed_region()
        torch.cuda.synchronize()
        reps_ms.append(r0.elapsed_time(r1) / K)
    reps_ms.sort()

    # dominant kernel alone: CUDA events around graph replays of R launches each
    durs = []
    k0 = torch.cuda.Event(enable_timing=True)
    k1 = torch.cuda.Event(enable_timing=True)
    g_dec.replay()
    for _ in range(max(3, min(64, 8192 // R))):
        blocking_sleep(stream)
        k0.record(stream)
        g_dec.replay()
        k1.record(stream)
        torch.cuda.synchronize()
        durs.append(k0.elapsed_time(k1) / R)
    durs.sort()
    dec_ms = sum(durs) / len(durs)
    dec_ms_med = durs[len(durs) // 2]
    peak, peak_kind = measured_peaks()
    achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": profiled_traffic(),
                "kernel": "decode_cluster_kernel<bf16,128,FUSED>" if base.k.dtype == torch.bfloat16
                else "decode_cluster_kernel<f32,FUSED>",
                "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({peak_kind}, of measured)",
                "algorithmic_bytes_per_launch": dec_bytes,
                "launch_us_mean": round(dec_ms * 1e3, 3), "launch_us_median": round(dec_ms_med * 1e3, 3),
                "launch_timing": "CUDA events around graph replays of back-to-back launches "
                                 "(no overlapped launch), divided by the launch count",
                "achieved_per_overlapped_step": round(dec_bytes / (ms_step * 1e-3) / 1e9, 1)}

    stages = stage_lines(args, lsa, copies, base, dev, peak) if wl != "tiny_decode" else None

    # end to end through the C ABI with pinned host buffers
    flags = lsa.LSA_FLAG_PDL if args.overlap else 0
    e2e = run_e2e(args, lsa, copies, base, dev, topk, ns, nl, flags)
    e2e["value"] = job_rate(e2e["value"], world, dev)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": round(ms_step, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if base.k.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded N(0,1) q/k/v with RoPE theta 1e4 and planted needle blocks)",
        "config": {"workload": wl, "batch": B, "kv_heads": Hkv, "q_heads_per_kv": G,
                   "head_dim": D, "context": T_cap, "block": 64, "topk": topk,
                   "forced": {"sink": ns, "local": nl},
                   "l2": (f"{R} input copies rotated; the {K} timed steps read {min(K, R)} distinct "
                          f"copies, each last touched {gap_steps} steps ({gap_steps * step_bytes / 1e6:.0f} MB "
                          f"of other traffic) earlier, against a {l2 / 1e6:.0f} MB L2"
                          + (": a profiling run, not a measurement" if args.profile_small else "")),
                   "timing": "every timed graph replayed once untimed first; a 0.1 ms device-side "
                             "wait queued before the start event; CUDA events on the launching stream",
                   "parallelism": f"replicas x{world} (independent sequences, no collective)",
                   "overlapped_launch": bool(args.overlap)},
        "effective_gbs": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
        "bytes_per_step": step_bytes,
        "repeats": {"n": len(reps_ms), "ms_per_step_median": round(reps_ms[len(reps_ms) // 2], 6),
                    "ms_per_step_min": round(reps_ms[0], 6), "ms_per_step_max": round(reps_ms[-1], 6),
                    "what": "the same K-step timed region repeated, each on cold copies"},
        "needle_recall": needle_recall(base, copies[0]["idx"]),
        "roofline": roofline,
        "stages": stages,
        "e2e": e2e,
        "gpu_launches": K,
        "clocks": clocks.summary(),
    }
    return result


def _time_graph_launches(g, n_launch, reps, stream):
    """Mean and median of the per-launch time of a graph of n_launch launches."""
    k0 = torch.cuda.Event(enable_timing=True)
    k1 = torch.cuda.Event(enable_timing=True)
    g.replay()
    torch.cuda.synchronize()
    durs = []
    for _ in range(reps):
        blocking_sleep(stream)
        k0.record(stream)
        g.replay()
        k1.record(stream)
        torch.cuda.synchronize()
        durs.append(k0.elapsed_time(k1) / n_launch)
    durs.sort()
    return sum(durs) / len(durs), durs[len(durs) // 2]


def stage_lines(args, lsa, copies, base, dev, peak):
    """The decode path's stages on their own, each against the HBM peak with its own
    algorithmic bytes: the whole-cache summary build (K1, once per prefill), the unfused
    selection (scores + top-k; lsa_select_blocks) and the attention over a given selection
    (lsa_sparse_attn_decode with idx).  Graphs of back-to-back launches over the rotated
    copies, CUDA events, mean per launch."""
    R = len(copies)
    B, Hkv, G, D, T_cap = base.shape
    esz = base.k.element_size()
    NB_cap = -(-T_cap // 64)
    stream = torch.cuda.current_stream()
    out = {}
    nsel = [torch.empty(B, Hkv, device=dev, dtype=torch.int32) for _ in range(R)]
    summ_scratch = [torch.empty_like(c["summ"]) for c in copies[:min(R, 8)]]

    def capture(fn, n):
        for i in range(n):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                fn(i)
        return g

    # K1: every key read once, every summary written once
    n_sum = len(summ_scratch)
    g = capture(lambda i: lsa.lsa_build_summaries(copies[i]["k"], copies[i]["sl"], summ_scratch[i]), n_sum)
    mean, med = _time_graph_launches(g, n_sum, 5, stream)
    toks = sum(int(x) for x in base.seqlens.tolist())
    nbs = sum(-(-int(x) // 64) for x in base.seqlens.tolist())
    by = Hkv * toks * D * esz + Hkv * nbs * D * 4
    out["summaries"] = {"kernel": "build_summaries_kernel", "bytes_per_launch": by,
                        "us_per_launch": round(mean * 1e3, 3), "us_median": round(med * 1e3, 3),
                        "gbs": round(by / (mean * 1e-3) / 1e9, 1),
                        "frac": round(by / (mean * 1e-3) / 1e9 / peak, 4),
                        "what": "whole-cache build: keys read + fp32 summaries written"}
    del g

    # unfused selection: candidate summaries + q read, idx / nsel written
    def sel(i):
        c = copies[i]
        lsa.lsa_select_blocks(c["q"], c["summ"], c["sl"], base.topk, base.n_sink, base.n_local,
                              c["idx"], nsel[i])
    g = capture(sel, R)
    mean, med = _time_graph_launches(g, R, 10, stream)
    nf = base.n_sink + base.n_local
    by = 0
    for T in base.seqlens.tolist():
        NB = -(-int(T) // 64)
        by += Hkv * (NB - nf) * D * 4 if NB > base.topk else 0
    by += base.q.numel() * esz + B * Hkv * (base.topk + 1) * 4
    out["select"] = {"kernel": "decode_cluster_kernel<SELECT>", "bytes_per_launch": by,
                     "us_per_launch": round(mean * 1e3, 3), "us_median": round(med * 1e3, 3),
                     "gbs": round(by / (mean * 1e-3) / 1e9, 1),
                     "frac": round(by / (mean * 1e-3) / 1e9 / peak, 4),
                     "what": "lsa_select_blocks: scores of every candidate block + top-k"}
    del g

    # attention over the selection just made
    def att(i):
        c = copies[i]
        lsa.lsa_sparse_attn_decode(c["q"], c["k"], c["v"], c["sl"], c["o"], base.topk, idx=c["idx"],
                                   nsel=nsel[i], lse=c["lse"])
    g = capture(att, R)
    mean, med = _time_graph_launches(g, R, 10, stream)
    dec, _ = algorithmic_bytes(base)
    by = dec - sum((Hkv * (-(-int(T) // 64) - nf) * D * 4 if -(-int(T) // 64) > base.topk else 0)
                   + Hkv * D * 4 for T in base.seqlens.tolist()) + B * Hkv * 4
    out["attend"] = {"kernel": "decode_cluster_kernel<ATTEND>", "bytes_per_launch": by,
                     "us_per_launch": round(mean * 1e3, 3), "us_median": round(med * 1e3, 3),
                     "gbs": round(by / (mean * 1e-3) / 1e9, 1),
                     "frac": round(by / (mean * 1e-3) / 1e9 / peak, 4),
                     "what": "lsa_sparse_attn_decode over a given selection: selected K/V + q, o, lse, idx"}
    del g
    torch.cuda.synchronize()
    return out


def _carve(buf, specs):
    """Views of one byte buffer: specs = [(dtype, shape), ...], each view 16-byte aligned."""
    out, off = [], 0
    for dt, shape in specs:
        n = math.prod(shape) * torch.tensor([], dtype=dt).element_size()
        out.append(buf[off:off + n].view(dt).view(shape))
        off += (n + 15) // 16 * 16
    return out, off


def needle_recall(case, idx):
    """Planted needle blocks (synth) found in the selected indices of the same inputs."""
    planted = sum(len(blocks) for _, _, blocks in case.needles)
    if planted == 0:
        return None
    sel = idx.cpu()
    found = sum(int(j) in set(sel[b, g].tolist()) for b, g, blocks in case.needles for j in blocks)
    return {"found": found, "planted": planted, "fraction": round(found / planted, 4)}


def run_e2e(args, lsa, copies, base, dev, topk, ns, nl, flags):
    """Same metric through the public API with pinned host buffers on both ends: every step
    moves q to the device and appends the newest token's k and v, all three read straight
    from pinned host memory by one kernel whose loads cross PCIe (lsa_append_kv_stage_q),
    then decodes (lsa_sparse_attn_decode, fused selection and summary refresh, a programmatic
    dependent of the staging) with o, lse and idx written straight into pinned host memory.  The steps of one rotation cycle are captured once in a
    CUDA graph and replayed, as a serving loop does; the same calls issued eagerly from
    Python are timed beside it."""
    R = len(copies)
    B, Hkv, G, D, T_cap = base.shape
    dt = copies[0]["q"].dtype
    n_cycles = max(1, math.ceil(min(args.e2e_steps, max(args.steps, R)) / R))
    n = n_cycles * R
    last = [int(x) - 1 for x in base.seqlens.tolist()]
    in_specs = [(dt, tuple(copies[0]["q"].shape)), (dt, (B, Hkv, D)), (dt, (B, Hkv, D))]
    out_specs = [(dt, tuple(copies[0]["o"].shape)), (torch.float32, tuple(copies[0]["lse"].shape)),
                 (torch.int32, tuple(copies[0]["idx"].shape))]
    _, in_bytes = _carve(torch.empty(1 << 20, dtype=torch.uint8), in_specs)
    _, out_bytes = _carve(torch.empty(1 << 20, dtype=torch.uint8), out_specs)
    in_host = []
    for r in range(R):
        hb = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
        (hq, hk, hv), _ = _carve(hb, in_specs)
        hq.copy_(copies[r]["q"].cpu())
        hk.copy_(torch.stack([copies[r]["k"][b, :, last[b]] for b in range(B)]).cpu())
        hv.copy_(torch.stack([copies[r]["v"][b, :, last[b]] for b in range(B)]).cpu())
        in_host.append(hb)
    in_views = [_carve(hb, in_specs)[0] for hb in in_host]
    q_dev = torch.empty(tuple(copies[0]["q"].shape), dtype=dt, device=dev)
    out_host = torch.empty(out_bytes, dtype=torch.uint8).pin_memory()
    (o_host, lse_host, idx_host), _ = _carve(out_host, out_specs)
    h2d = sum(math.prod(sh) * torch.tensor([], dtype=d).element_size() for d, sh in in_specs)
    d2h = sum(math.prod(sh) * torch.tensor([], dtype=d).element_size() for d, sh in out_specs)

    def one(i):
        c = copies[i % R]
        hq, hk, hv = in_views[i % R]
        # (the host wrote this step's inputs before enqueueing it: they are read at once)
        lsa.lsa_append_kv_stage_q(hq, q_dev, hk, hv, c["sl"], c["k"], c["v"],
                                  flags=flags | (lsa.LSA_FLAG_INPUTS_READY if flags else 0))
        lsa.lsa_sparse_attn_decode(q_dev, c["k"], c["v"], c["sl"], o_host, topk, summ=c["summ"],
                                   n_sink=ns, n_local=nl, refresh_last_summary=True,
                                   idx_out=idx_host, lse=lse_host, flags=flags)

    stream = torch.cuda.current_stream()

    def timed(fn):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        nv = _nvtx_push("e2e timed region")
        blocking_sleep(stream)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        _nvtx_pop(nv)
        return e0.elapsed_time(e1), time.perf_counter() - t0

    # eager: every call issued from Python each step
    for i in range(min(n, 3 * R)):
        one(i)
    torch.cuda.synchronize()
    ms_eager, wall_eager = timed(lambda: [one(i) for i in range(n)])

    # graph: one rotation cycle captured once, replayed
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(R):
            one(i)
    g.replay()
    torch.cuda.synchronize()
    ms_graph, wall_graph = timed(lambda: [g.replay() for _ in range(n_cycles)])
    # the last step's outputs arrived in host memory: a finite o and in-range indices
    ok = bool(torch.isfinite(o_host.float()).all()) and int(idx_host.max()) < -(-T_cap // 64)
    del g
    return {"value": round(B * n / (ms_graph / 1e3), 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n, "host_wall_s": round(wall_graph, 3),
            "us_per_step": round(ms_graph * 1e3 / n, 3),
            "eager": {"value": round(B * n / (ms_eager / 1e3), 1), "us_per_step": round(ms_eager * 1e3 / n, 3),
                      "host_wall_s": round(wall_eager, 3)},
            "outputs_checked": ok,
            "path": "python ctypes -> lsa_append_kv_stage_q (q, k, v read from pinned host memory by "
                    "one kernel) + lsa_sparse_attn_decode (fused selection, summary "
                    "refresh; o, lse, idx written into pinned host memory), every byte crossing PCIe "
                    "each step; value: the steps of a rotation cycle captured once in a CUDA graph "
                    "and replayed; eager: the same calls issued from Python every step"}


# ------------------------------------------------------------------ CPU (oracle) arm ----

def oracle_step_runner(wl, seed=1002):
    """The fp64 oracle's decode step on the same workload (inputs on the host): refresh the
    last block's summary, score every block, select, attend.  Returns (run(units), meta)."""
    import oracle
    case = make_case(wl, seed, "cpu")
    B, Hkv, G, D, T_cap = case.shape
    summ = oracle.summaries(case.k, case.seqlens)  # prefill-time, not timed

    kv_cache = {}  # the K/V of a head subset, made contiguous once (outside any timing)

    def run(heads=None):
        heads = heads or list(range(Hkv))
        for b in range(B):
            T = int(case.seqlens[b])
            if T == 0:
                continue
            j = (T - 1) // 64
            kb = case.k[b:b + 1, :, j * 64:T].contiguous()
            summ[b:b + 1, :, j] = oracle.summaries(kb, torch.tensor([T - j * 64]))[:, :, 0]
        hs = heads
        q = case.q.view(B, Hkv, G, D)[:, hs].reshape(B, len(hs) * G, D).contiguous()
        if len(hs) < Hkv:
            key = tuple(hs)
            if key not in kv_cache:
                kv_cache[key] = (case.k[:, hs].contiguous(), case.v[:, hs].contiguous())
            k, v = kv_cache[key]
        else:
            k, v = case.k, case.v
        s = oracle.block_scores(q, summ[:, hs].contiguous(), case.seqlens)
        idx, nsel = oracle.select(s, case.seqlens, case.topk, case.n_sink, case.n_local)
        return oracle.decode_attn(q, k, v, case.seqlens, idx, nsel)

    return run, dict(B=B, Hkv=Hkv)


def cpu_baseline(wl, seconds):
    import oracle
    run, meta = oracle_step_runner(wl)
    run()  # warm
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds or n < 3:
        run()
        n += 1
    dt = time.perf_counter() - t0
    return {"value": round(meta["B"] * n / dt, 2), "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{n} full decode steps of the {wl} workload (last-block summary refresh, "
                      f"scores of every block, selection, attention) in fp64 over {dt:.1f} s"}


def run_reference(args):
    import oracle
    wl = args.workload
    run, meta = oracle_step_runner(wl)
    Hkv = meta["Hkv"]
    t0 = time.perf_counter()
    run()
    t_full = time.perf_counter() - t0
    budget = 150.0
    K, W = args.steps, args.warmup
    heads = Hkv
    while heads > 1 and (K + W) * t_full * heads / Hkv > budget:
        heads -= 1
    hs = list(range(heads))
    run(hs)  # (makes the head subset's K/V contiguous before the timed steps)
    for _ in range(W):
        run(hs)
    timed = K
    t0 = time.perf_counter()
    done = 0
    for i in range(K):
        run(hs)
        done += 1
        if time.perf_counter() - t0 > budget:
            break
    dt = time.perf_counter() - t0
    timed = done
    frac = heads / Hkv
    value = meta["B"] * frac * timed / dt
    sample = (f"{timed} steps of the {wl} decode step restricted to {heads} of {Hkv} KV heads "
              f"(heads are independent; tokens counted as {frac:.3f} per sequence per step)")
    return {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 1, "steps": timed,
        "warmup": W, "ms_per_step": round(dt / timed * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl}, "impl": "reference",
        # (the oracle's OpenMP loops run over (sequence, KV head) units)
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT,
                         "cores": min(oracle.num_threads(), meta["B"] * heads),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------ other workloads (extra lines) --

def measured_tensor_peak():
    """The bf16 burst peak: the prefill line times its kernel alone (a run of back-to-back
    prefills, each a single launch), so the burst cuBLAS figure is the comparable one."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured, burst"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback, burst"


def prefill_tile_counts(L, tq=128, tk=64):
    """Visited KV tiles of one head (causal, ascending up to the diagonal)."""
    n = 0
    for a in range(-(-L // tq)):
        n += (min(a * tq + tq, L) - 1) // tk + 1
    return n


def run_prefill(args):
    """BLASST causal prefill, 32 q heads / 8 KV heads, D 128, L 32768, lambda 1e-3: a step is
    one whole prefill.  Inputs (q 256 MB, k/v 128 MB) exceed the L2, so every step reads
    them from HBM."""
    import query_aware_block_b200 as lsa
    import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    case = synth.prefill_case(B=1, Hq=32, Hkv=8, L=32768, D=128, lam=1e-3, sink=args.prefill_sink,
                              q_scale=args.prefill_qscale, seed=1005, device=dev)
    B, Hq, L, D = case.q.shape
    o = torch.empty_like(case.q)
    lse = torch.empty(B, Hq, L, device=dev)
    nqt, words = -(-L // 128), -(-(-(-L // 64)) // 32)
    bits = torch.zeros(B, Hq, nqt, words, dtype=torch.int32, device=dev)
    cnt = torch.zeros(1, dtype=torch.int64, device=dev)

    def step():
        lsa.lsa_blasst_prefill(case.q, case.k, case.v, o, case.lam, lse=lse, skip_bits=bits,
                               skipped_tiles=cnt)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    cnt.zero_()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    K = args.steps
    with ClockSampler(0) as clocks:
        torch.cuda.synchronize()
        e0.record()
        for _ in range(K):
            step()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / K
    visited = B * Hq * prefill_tile_counts(L)
    skipped = int(cnt.item()) / K
    tile_flop = 2 * 128 * 64 * D
    flops = visited * tile_flop + (visited - skipped) * tile_flop  # Q K^T always, P V if kept
    tflops = flops / (ms * 1e-3) / 1e12
    peak, kind = measured_tensor_peak()
    return {
        "metric": "BLASST causal prefill TFLOP/s (algorithmic: QK^T of every visited tile + PV of kept tiles)",
        "value": round(tflops, 1), "unit": "TFLOP/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) q/k/v with RoPE theta 1e4"
                                  + (f", attention sink {args.prefill_sink}" if args.prefill_sink else "")
                                  + (f", q scaled by {args.prefill_qscale}" if args.prefill_qscale != 1.0 else "")
                                  + ")",
        "config": {"workload": "blasst_prefill_32k", "batch": B, "q_heads": Hq, "kv_heads": case.k.shape[1],
                   "head_dim": D, "seq_len": L, "tiles": "128 x 64", "lambda": case.lam,
                   "l2": "inputs (512 MB) larger than L2"},
        "tokens_per_s": round(B * L / (ms * 1e-3), 1),
        "skip_fraction": round(skipped / visited, 4),
        "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(tflops / peak, 4), "traffic": None,
                     "kernel": "blasst_prefill_kernel (tcgen05)",
                     "peak_source": f"MEASURED_PEAKS.json bf16_tflops ({kind}, of measured)",
                     "algorithmic_flops_per_launch": flops},
        "gpu_launches": K,
        "clocks": clocks.summary(),
    }


def run_blockquery(args):
    """Diffusion-LM block-query step (32 query tokens, 8 active, prefix 32768, top-8 blocks
    per token and KV head).  A step is one call; R rotated input copies exceed 4x L2."""
    import query_aware_block_b200 as lsa
    import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    base = synth.diffusion_blockquery(device=dev)
    B, Hq, Tq, D = base.q.shape
    Hkv = base.k.shape[1]
    G = Hq // Hkv
    T_cap = base.k.shape[2]
    NBp = -(-base.T_prefix // 64)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    ws = torch.empty(lsa.lsa_blockquery_workspace_size(B, Hkv, G, D, Tq), dtype=torch.uint8, device=dev)
    copies = []
    R = 4
    for r in range(64):
        c = base if r == 0 else synth.blockquery_case(seed=1004 + 101 * r, device=dev)
        sl = torch.full((B,), T_cap, dtype=torch.int32, device=dev)
        summ = torch.zeros(B, Hkv, -(-T_cap // 64), D, device=dev)
        lsa.lsa_build_summaries(c.k, sl, summ)
        copies.append(dict(c=c, summ=summ, o=torch.empty_like(c.o_cache), lse=torch.empty_like(c.lse_cache),
                           ui=torch.empty(B, Hkv, NBp, dtype=torch.int32, device=dev),
                           uc=torch.empty(B, Hkv, dtype=torch.int32, device=dev)))
        if r == 0:
            def one(x):
                lsa.lsa_sparse_attn_blockquery(x["c"].q, x["c"].k, x["c"].v, x["summ"], x["c"].T_prefix,
                                               x["c"].topk, x["c"].active, x["c"].o_cache, x["c"].lse_cache,
                                               x["o"], x["lse"], ws, union_idx=x["ui"], union_cnt=x["uc"])
            one(copies[0])
            torch.cuda.synchronize()
            U = int(copies[0]["uc"].sum())
            A = int(base.active.sum())
            step_bytes = (Hkv * NBp * D * 4 + U * 64 * D * 2 * 2 + 2 * A * G * Hkv * D * 2
                          + (Tq - A) * G * Hkv * D * 2 * 2)
            R = max(4, min(64, math.ceil(4 * l2 / step_bytes)))
            if args.profile_small:
                R = 4
        if len(copies) >= R:
            break
    for x in copies:
        one(x)
    torch.cuda.synchronize()
    U_mean = sum(int(x["uc"].sum()) for x in copies) / len(copies)
    A = int(base.active.sum())
    step_bytes = (Hkv * NBp * D * 4 + U_mean * 64 * D * 2 * 2 + 2 * A * G * Hkv * D * 2
                  + (Tq - A) * G * Hkv * D * 2 * 2 + Hkv * NBp * 4)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for x in copies:
            one(x)
    K = args.steps
    reps = max(1, K // R)
    for _ in range(max(1, args.warmup // R)):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks:
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
    steps = reps * R
    ms = e0.elapsed_time(e1) / steps
    gbs = step_bytes / (ms * 1e-3) / 1e9
    peak, kind = measured_peaks()
    return {
        "metric": "block-query denoising step: query tokens/s and effective GB/s (% of HBM roofline)",
        "value": round(B * Tq / (ms * 1e-3), 1), "unit": "tokens/s", "n_gpus": 1, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 6), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1), RoPE theta 1e4)",
        "config": {"workload": "blockquery", "batch": B, "kv_heads": Hkv, "q_heads_per_kv": G,
                   "head_dim": D, "query_tokens": Tq, "active": A, "prefix": base.T_prefix,
                   "topk_per_token": base.topk,
                   "l2": f"rotating {R} input copies ({R * step_bytes / 1e6:.0f} MB per cycle)"},
        "mean_union_blocks_per_kv_head": round(U_mean / (B * Hkv), 2),
        "kv_density": round(U_mean / (B * Hkv) / NBp, 4),
        "effective_gbs": round(gbs, 1), "bytes_per_step": int(step_bytes),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": None, "kernel": "blockquery_kernel<128>",
                     "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({kind})"},
        "gpu_launches": steps,
        "clocks": clocks.summary(),
    }


def run_losa_step(args):
    """One LoSA denoising step of the diffusion workload (32 query tokens, prefix 32768,
    8 KV heads x 4 query heads, top-8 blocks per active token): the tokens are classified
    by the change of their queries (the 8 largest), the active ones select and attend the
    prefix (the prefix cache is updated in place, stable rows keep theirs), and every token
    attends the block itself, merged with its prefix result.  A step is three launches
    (the last one overlapped with PDL); R rotated input copies exceed 4x L2."""
    import query_aware_block_b200 as lsa
    import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    base = synth.diffusion_losa_step(device=dev)
    B, Hq, Tq, D = base.q.shape
    Hkv = base.k.shape[1]
    G = Hq // Hkv
    T_cap = base.k.shape[2]
    T = base.T_prefix
    NBp = -(-T // 64)
    n_top = int(base.active[0].sum())
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    ws = torch.empty(lsa.lsa_blockquery_workspace_size(B, Hkv, G, D, Tq), dtype=torch.uint8, device=dev)

    def make(r):
        c = base if r == 0 else synth.losa_case(seed=1006 + 101 * r, device=dev)
        sl = torch.full((B,), T, dtype=torch.int32, device=dev)
        summ = torch.zeros(B, Hkv, -(-T_cap // 64), D, device=dev)
        lsa.lsa_build_summaries(c.k, sl, summ)
        return dict(c=c, summ=summ, act=torch.empty(B, Tq, dtype=torch.uint8, device=dev),
                    co=c.o_cache.clone(), cl=c.lse_cache.clone(), o=torch.empty_like(c.o_cache),
                    lse=torch.empty_like(c.lse_cache),
                    ui=torch.empty(B, Hkv, NBp, dtype=torch.int32, device=dev),
                    uc=torch.empty(B, Hkv, dtype=torch.int32, device=dev))

    def classify(x):
        lsa.lsa_losa_classify(x["c"].q, x["c"].q_prev, x["act"], n_top=n_top)

    def prefix(x):
        c = x["c"]
        lsa.lsa_sparse_attn_blockquery(c.q, c.k, c.v, x["summ"], T, c.topk, x["act"], x["co"], x["cl"],
                                       x["co"], x["cl"], ws, union_idx=x["ui"], union_cnt=x["uc"])

    def intra(x, flags=lsa.LSA_FLAG_PDL):
        c = x["c"]
        lsa.lsa_blockquery_intra_merge(c.q, c.k, c.v, T, x["co"], x["cl"], x["o"], x["lse"], flags=flags)

    def one(x):
        classify(x)
        prefix(x)
        intra(x)

    copies = [make(0)]
    one(copies[0])
    torch.cuda.synchronize()
    A = int(copies[0]["act"].sum())
    U0 = int(copies[0]["uc"].sum())
    blk_bytes = lambda U: (Hkv * NBp * D * 4 + U * 64 * D * 2 * 2 + 2 * A * G * Hkv * D * 2 + Hkv * NBp * 4)
    other_bytes = (2 * Tq * Hq * D * 2 + Tq * B                      # classify: q, q_prev; mask
                   + Hkv * Tq * D * 2 * 2 + Tq * Hq * D * 2          # intra: block K/V, q
                   + 2 * Tq * Hq * D * 2 + 2 * Tq * Hq * 4 * 2)     # o_pre in, o out, lse in/out
    R = 4 if args.profile_small else max(4, min(64, math.ceil(4 * l2 / (blk_bytes(U0) + other_bytes))))
    while len(copies) < R:
        copies.append(make(len(copies)))
    for x in copies:
        one(x)
    torch.cuda.synchronize()
    U_mean = sum(int(x["uc"].sum()) for x in copies) / len(copies)
    step_bytes = blk_bytes(U_mean) + other_bytes

    def graph_of(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for x in copies:
                fn(x)
        return g

    def time_graph(g, reps, clocks=None):
        for _ in range(max(1, args.warmup // R)):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (reps * R)

    g_step = graph_of(one)
    reps = max(1, args.steps // R)
    with ClockSampler(0) as clocks:
        ms = time_graph(g_step, reps)
    # per-kernel breakdown (each alone, back to back)
    parts = {}
    for name, fn in (("classify", classify), ("blockquery", prefix), ("intra_merge", lambda x: intra(x, 0))):
        parts[name] = round(time_graph(graph_of(fn), max(1, reps // 4)) * 1e3, 2)
    # the dense first step of a block: every token, every prefix block
    x0 = copies[0]
    ones = torch.ones(B, Tq, dtype=torch.uint8, device=dev)
    c0 = x0["c"]
    dense = lambda: lsa.lsa_sparse_attn_blockquery(c0.q, c0.k, c0.v, x0["summ"], T, NBp, ones, x0["co"], x0["cl"],
                                                   x0["o"], x0["lse"], ws, union_idx=x0["ui"], union_cnt=x0["uc"])
    for _ in range(3):
        dense()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(10):
        dense()
    e1.record()
    torch.cuda.synchronize()
    dense_ms = e0.elapsed_time(e1) / 10
    dense_bytes = 2 * Hkv * T * D * 2 + Tq * Hq * D * 2 * 2
    gbs = step_bytes / (ms * 1e-3) / 1e9
    peak, kind = measured_peaks()
    return {
        "metric": "LoSA denoising step (classify + sparse prefix + intra-block merge): query tokens/s and "
                  "effective GB/s (% of HBM roofline)",
        "value": round(B * Tq / (ms * 1e-3), 1), "unit": "tokens/s", "n_gpus": 1, "steps": reps * R,
        "warmup": args.warmup, "ms_per_step": round(ms, 6), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1), RoPE theta 1e4; "
        "previous queries: +0.02 N(0,1) for stable tokens, fresh draws for the 8 changing ones)",
        "config": {"workload": "losa_step", "batch": B, "kv_heads": Hkv, "q_heads_per_kv": G,
                   "head_dim": D, "query_tokens": Tq, "active": A, "prefix": T, "topk_per_token": base.topk,
                   "l2": f"rotating {R} input copies ({R * step_bytes / 1e6:.0f} MB per cycle)"},
        "mean_union_blocks_per_kv_head": round(U_mean / (B * Hkv), 2),
        "effective_gbs": round(gbs, 1), "bytes_per_step": int(step_bytes),
        "kernel_us_alone": parts,
        "dense_first_step": {"us": round(dense_ms * 1e3, 1),
                             "effective_gbs": round(dense_bytes / (dense_ms * 1e-3) / 1e9, 1),
                             "bytes": int(dense_bytes),
                             "note": "every token over every prefix block (same K/V each call)"},
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": None, "kernel": "whole step (3 launches)",
                     "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({kind})"},
        "gpu_launches": 3 * reps * R,
        "clocks": clocks.summary(),
    }


def run_decode_blasst(args):
    """BLASST inside sparse decode on the 64K GQA decode inputs: the selection of the fused
    decode (16 blocks per KV head, its own kernels) is given to lsa_sparse_attn_decode_blasst,
    which reads K of every selected block and V only of the blocks some head still needs.
    The queries are scaled by --decode-qscale (a sharper softmax: 1 = the plain workload,
    where no block is negligible).  R input copies (distinct caches, queries and
    selections) are rotated so that a launch's data was last touched more than 4x the L2
    size of traffic earlier; back-to-back launches over one rotation are captured in a CUDA
    graph and timed with CUDA events, next to the plain given-selection decode on the same
    inputs timed the same way."""
    import query_aware_block_b200 as lsa
    import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    lam = args.decode_lambda
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    if args.decode_batched:
        B, Hkv, G, D, T_cap = 16, 8, 4, 128, 32768
        make = lambda seed: synth.batched_decode(seed=seed, device=dev)
        seed0, what = 1003, "batched varlen decode inputs (16 sequences, T ~ U[8K, 32K])"
    else:
        B, Hkv, G, D, T_cap = 1, 8, 8, 128, 65536
        make = lambda seed: synth.gqa_decode_64k(seed=seed, device=dev)
        seed0, what = 1002, "64K GQA decode inputs"
    Hq = Hkv * G
    approx_step = B * Hkv * 16 * 64 * D * 2 * 2
    R = 4 if args.profile_small else (args.rotate or max(8, min(160, math.ceil(4 * l2 / approx_step))))
    copies = []
    for r in range(R):
        c = make(seed0 + 7919 * r)
        q = (c.q.float() * args.decode_qscale).to(torch.bfloat16)
        summ = torch.zeros(B, Hkv, -(-T_cap // 64), D, device=dev)
        lsa.lsa_build_summaries(c.k, c.seqlens, summ)
        idx = torch.empty(B, Hkv, 16, dtype=torch.int32, device=dev)
        o = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(B, Hq, device=dev)
        lsa.lsa_sparse_attn_decode(c.q, c.k, c.v, c.seqlens, o, 16, summ=summ, n_sink=1, n_local=2,
                                   idx_out=idx, lse=lse)
        nsel = (idx >= 0).sum(-1).to(torch.int32)
        bits = torch.zeros(B, Hkv, dtype=torch.int32, device=dev)
        copies.append(dict(q=q, k=c.k, v=c.v, sl=c.seqlens, idx=idx, nsel=nsel, o=o, lse=lse, bits=bits))
        del summ, c
    torch.cuda.synchronize()

    def blasst(c):
        lsa.lsa_sparse_attn_decode_blasst(c["q"], c["k"], c["v"], c["sl"], c["idx"], c["nsel"], c["o"], lam,
                                          lse=c["lse"], skip_bits=c["bits"])

    def plain(c):
        lsa.lsa_sparse_attn_decode(c["q"], c["k"], c["v"], c["sl"], c["o"], 16, idx=c["idx"], nsel=c["nsel"],
                                   lse=c["lse"])

    def graph_of(fn):
        for c in copies:
            fn(c)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for c in copies:
                fn(c)
        g.replay()
        torch.cuda.synchronize()
        return g

    stream = torch.cuda.current_stream()
    g_b, g_p = graph_of(blasst), graph_of(plain)
    reps = 2 if args.profile_small else max(5, min(50, args.steps // R))
    with ClockSampler(0) as clocks:
        t_blasst, med_b = _time_graph_launches(g_b, R, reps, stream)
        t_plain, med_p = _time_graph_launches(g_p, R, reps, stream)
    del g_b, g_p
    torch.cuda.synchronize()
    # per launch: K rows of every selected block and V rows of the kept ones (valid tokens
    # only), q, o, lse, idx, nsel
    k_tok = v_tok = skipped = slots = 0
    for c in copies:
        idx_c, bits_c, sl_c = c["idx"].cpu(), c["bits"].cpu(), c["sl"].cpu()
        for b in range(B):
            T = int(sl_c[b])
            for g in range(Hkv):
                word = int(bits_c[b, g]) & 0xFFFFFFFF
                for s_, j in enumerate(idx_c[b, g].tolist()):
                    if j < 0:
                        continue
                    n = max(0, min(64, T - 64 * j))
                    slots += 1
                    k_tok += n
                    if (word >> s_) & 1:
                        skipped += 1
                    else:
                        v_tok += n
    row = D * 2
    small = 2 * B * Hq * D * 2 + B * Hq * 4 + B * Hkv * 17 * 4
    step_bytes = (k_tok + v_tok) * row / R + small
    plain_bytes = 2 * k_tok * row / R + small
    t_us, tp_us = t_blasst * 1e3, t_plain * 1e3
    gbs = step_bytes / (t_us * 1e-6) / 1e9
    peak, kind = measured_peaks()
    return {
        "metric": f"BLASST sparse decode over a given selection ({what}): tokens/s and effective GB/s",
        "value": round(B / (t_us * 1e-6), 1), "unit": "tokens/s", "n_gpus": 1, "steps": reps * R,
        "warmup": R, "ms_per_step": round(t_us * 1e-3, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": f"synthetic {what} (seeded), queries x{args.decode_qscale}",
        "config": {"workload": "decode_blasst" + ("_batched" if args.decode_batched else ""), "batch": B, "kv_heads": Hkv, "q_heads_per_kv": G,
                   "head_dim": D, "context": T_cap, "topk": 16, "lambda": lam,
                   "l2": f"{R} input copies rotated ({R * step_bytes / 1e6:.0f} MB touched per rotation, "
                         f"L2 {l2 / 1e6:.0f} MB); back-to-back launches of one rotation in a CUDA graph"},
        "skip_fraction": round(skipped / max(1, slots), 4), "skipped_v_blocks": skipped, "selected_blocks": slots,
        "blasst_decode_us": round(t_us, 3), "blasst_decode_us_median": round(med_b * 1e3, 3),
        "plain_given_selection_decode_us": round(tp_us, 3),
        "plain_given_selection_decode_us_median": round(med_p * 1e3, 3),
        "bytes_per_step": int(step_bytes), "plain_bytes_per_step": int(plain_bytes),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": None,
                     # (the library runs one CTA per (b, g) unit from 64 units up, else a cluster per unit)
                     "kernel": "decode_blasst_unit_kernel<128>" if B * Hkv >= 64 else "decode_blasst_kernel<128>",
                     "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({kind}, of measured)"},
        "gpu_launches": reps * R * 2,
        "clocks": clocks.summary(),
    }


def run_nsa_decode(args):
    """NSA's three branches for a 64K GQA decode step (the fixed-part variant): the fused
    selected-branch decode (summary refresh, selection, sparse attention), the refresh of
    the 2 compressed tokens the newest token changes (mean pool, block 32, stride 16) and
    one launch for the compressed (4,096 tokens) and window (512 tokens) branches joined
    with the selected one by gates of 1/3.  A step is three launches; R rotated input
    copies exceed 4x L2; graph replays timed with CUDA events."""
    import query_aware_block_b200 as lsa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = "gqa_decode_64k"
    base = make_case(wl, rank_seed(0), dev)
    B, Hkv, G, D, T_cap = base.shape
    Hq = Hkv * G
    stride, length, window = 16, 32, 512
    NC_cap = -(-T_cap // stride)
    dec_bytes, _ = algorithmic_bytes(base)
    T = int(base.seqlens[0])
    nc = -(-T // stride)
    nsa_bytes = (B * Hkv * (min(window, T) + nc) * D * 2 * 2             # window + compressed K/V
                 + B * Hkv * (length + stride) * D * 2 * 2                 # pool refresh reads
                 + B * Hkv * 2 * D * 2 * 2                                 # pool refresh writes
                 + B * Hq * D * 2 * 3)                                     # q, o_slc, o
    step_bytes = dec_bytes + nsa_bytes
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = 2 if args.profile_small else max(4, min(64, math.ceil(4 * l2 / step_bytes)))
    copies = []
    for r in range(R):
        c = base if r == 0 else make_case(wl, rank_seed(0, r), dev)
        q, k, v, sl = (t.to(dev) for t in (c.q, c.k, c.v, c.seqlens))
        summ = torch.zeros(B, Hkv, -(-T_cap // 64), D, device=dev)
        lsa.lsa_build_summaries(k, sl, summ)
        kc = torch.empty(B, Hkv, NC_cap, D, dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        lsa.lsa_nsa_compress(k, v, sl, kc, vc, length=length, stride=stride)
        copies.append(dict(q=q, k=k, v=v, sl=sl, summ=summ, kc=kc, vc=vc,
                           o_slc=torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev),
                           o=torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev),
                           idx=torch.empty(B, Hkv, base.topk, dtype=torch.int32, device=dev)))
        del c
    torch.cuda.synchronize()

    def selected(c):
        lsa.lsa_sparse_attn_decode(c["q"], c["k"], c["v"], c["sl"], c["o_slc"], base.topk, summ=c["summ"],
                                   n_sink=base.n_sink, n_local=base.n_local, refresh_last_summary=True,
                                   idx_out=c["idx"])

    def pool(c):
        lsa.lsa_nsa_compress(c["k"], c["v"], c["sl"], c["kc"], c["vc"], length=length, stride=stride,
                             nc_begin=-2)

    def branches(c):
        lsa.lsa_nsa_branches(c["q"], c["k"], c["v"], c["kc"], c["vc"], c["sl"], c["o"], o_slc=c["o_slc"],
                             window=window, stride=stride)

    def one(c):
        selected(c)
        pool(c)
        branches(c)

    for i in range(max(3, min(args.warmup, 2 * R))):
        one(copies[i % R])
    torch.cuda.synchronize()

    def graph_of(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for c in copies:
                fn(c)
        return g

    def time_graph(g, reps):
        for _ in range(max(1, args.warmup // R)):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (reps * R)

    reps = max(1, (args.steps or 20000) // R)
    g_step = graph_of(one)
    with ClockSampler(0) as clocks:
        ms = time_graph(g_step, reps)
    parts = {name: round(time_graph(graph_of(fn), max(1, reps // 4)) * 1e3, 2)
             for name, fn in (("selected_decode", selected), ("pool_refresh", pool), ("branches", branches))}
    gbs = step_bytes / (ms * 1e-3) / 1e9
    peak, kind = measured_peaks()
    return {
        "metric": "NSA decode step, fixed parts (selected + compressed + window branches): tokens/s and "
                  "effective GB/s",
        "value": round(B / (ms * 1e-3), 1), "unit": "tokens/s", "n_gpus": 1, "steps": reps * R,
        "warmup": args.warmup, "ms_per_step": round(ms, 6), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic 64K GQA decode inputs (seeded, needles)",
        "config": {"workload": "nsa_decode", "batch": B, "kv_heads": Hkv, "q_heads_per_kv": G,
                   "head_dim": D, "context": T_cap, "topk": base.topk, "compress": [length, stride],
                   "window": window, "gates": [1 / 3, 1 / 3, 1 / 3],
                   "l2": f"rotating {R} input copies ({R * step_bytes / 1e6:.0f} MB per cycle)"},
        "tokens_read_per_kv_head": nc + base.topk * 64 + min(window, T),
        "bytes_per_step": int(step_bytes), "effective_gbs": round(gbs, 1),
        "kernel_us_alone": parts,
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": None, "kernel": "whole step (3 launches)",
                     "peak_source": f"MEASURED_PEAKS.json hbm_gbs ({kind})"},
        "gpu_launches": 3 * reps * R,
        "clocks": clocks.summary(),
    }


def main():
    args = parse()
    if args.workload in ("blockquery", "blasst_prefill_32k", "losa_step", "decode_blasst", "nsa_decode"):
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the oracle arm covers the decode workloads"}))
            return
        res = {"blockquery": run_blockquery, "blasst_prefill_32k": run_prefill,
               "losa_step": run_losa_step, "decode_blasst": run_decode_blasst,
               "nsa_decode": run_nsa_decode}[args.workload](args)
        print(json.dumps(res), flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    res = run_ours(args, rank, world, local_rank)
    if rank == 0 and not args.no_cpu_baseline and not args.profile_small:
        res["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
