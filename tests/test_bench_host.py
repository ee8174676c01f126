"""The single-process host logic of bench.py on CPU: how the timed region is planned so
that every timed step reads cold data, and where the roofline line's denominators and DRAM
counters come from."""
import importlib.util
import json
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_host_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


L2 = 132_644_864  # the B200's L2 size as the CUDA runtime reports it


@pytest.mark.parametrize("step_bytes", [8_413_952, 88_000_000, 18_546_688, 1_000_000_000, 4096])
@pytest.mark.parametrize("K", [1, 2, 3, 5, 20, 63, 64, 65, 200, 200_000])
def test_rotation_keeps_every_timed_step_cold(bench, K, step_bytes):
    R, per_graph = bench.plan_rotation(K, step_bytes, L2)
    r_cold = max(4, min(128, math.ceil(4 * L2 / step_bytes)))
    if K < r_cold:
        # graphs of K steps over distinct copies; the timed graph's copies were last touched
        # by the other graphs' (R / K - 1) K steps, at least r_cold of them
        assert per_graph == K and R % K == 0
        assert R - K >= r_cold
    else:
        # one cycle of R = r_cold copies replayed (plus a remainder): a copy comes back after
        # R other steps
        assert (R, per_graph) == (r_cold, r_cold)
    # the copies' traffic between two uses of one copy is at least 4x the L2 size, unless the
    # 128-copy cap binds (steps of under 4 MiB)
    if 4 * L2 / step_bytes <= 128:
        gap = R - per_graph if K < r_cold else R
        assert gap * step_bytes >= 4 * L2


def test_rotation_respects_an_explicit_depth(bench):
    assert bench.plan_rotation(200, 8_000_000, L2, rotate=10) == (10, 10)
    R, per = bench.plan_rotation(4, 8_000_000, L2, rotate=10)
    assert per == 4 and R - 4 >= 10


def test_profiled_traffic_is_tied_to_the_kernel_source(bench, monkeypatch):
    text = open(bench.PROFILE_SUMMARY).read()
    hashes = set(re.findall(r"kernel source hash:\s*([0-9a-f]+)", text))
    assert len(hashes) == 1, "the decode summary names exactly one kernel source hash"
    if bench.source_hash() in hashes:
        traffic = bench.profiled_traffic()
        assert isinstance(traffic, int) and traffic > 0
    # another source (any edit of the hashed files) voids the committed counters
    monkeypatch.setattr(bench, "source_hash", lambda: "0" * 16)
    assert bench.profiled_traffic() is None


def test_source_hash_covers_the_decode_kernel_sources(bench):
    assert "query_aware_block_b200/csrc/decode.cu" in bench.KERNEL_SOURCES
    for rel in bench.KERNEL_SOURCES:
        assert os.path.isfile(os.path.join(bench.ROOT, rel)), rel
    h = bench.source_hash()
    assert len(h) == 16 and int(h, 16) >= 0


def test_measured_peaks_then_fallback(bench, monkeypatch, tmp_path):
    peak, kind = bench.measured_peaks()
    path = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if os.path.isfile(path):
        assert kind == "measured" and peak == float(json.load(open(path))["hbm_gbs"])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))  # no MEASURED_PEAKS.json there
    assert bench.measured_peaks() == (6650.0, "fallback")
