"""Host-side arithmetic of bench.py on the CPU: the derived peaks, the algorithmic
byte count of a decode step, and the guard that ties the captured DRAM traffic to
the kernel sources it was measured on."""
import json
import os

import numpy as np
import pytest

import bench


def test_alu_peaks_follow_unit_counts_and_clock():
    mhz = 1965.0
    path = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            mhz = float(json.load(f).get("sm_max_mhz", mhz))
    p32, src32 = bench.fp32_alu_peak()
    p64, src64 = bench.fp64_alu_peak()
    assert p32 == pytest.approx(148 * 128 * 2 * mhz * 1e6 / 1e12)
    assert p64 == pytest.approx(p32 / 2)          # 64 fp64 lanes per SM against 128 fp32
    assert f"{mhz:.0f} MHz" in src32 and f"{mhz:.0f} MHz" in src64


def test_step_bytes_counts_lists_by_hand():
    # one sequence, one KV head: a scored level with |A| = 600 (k = 256) and a level-0
    # list of 4096 tokens; s_vec = 256 bytes
    k, s_vec, d, esize = 256, 256, 128, 2
    counts = np.array([[[4096, 600, 0]]])
    tot, per = bench.step_bytes(counts, k, s_vec, B=1, Hkv=1, Hq=4, d=d, esize=esize)
    keys = (600 - 1) * s_vec             # every entry but the current node
    summaries = (600 - 256) * s_vec      # the unselected entries' values
    level0 = 2 * 4096 * s_vec            # K and V of every level-0 entry
    io = 1 * 4 * d * esize * 2 + 1 * 1 * 2 * d * esize   # q, out, the appended k and v
    assert per[1] == keys + summaries and per[0] == level0 and 2 not in per
    assert tot == keys + summaries + level0 + io


def test_captured_traffic_is_tied_to_the_sources(monkeypatch):
    import hashlib
    h = hashlib.sha256()
    for f in bench.TRAFFIC_PASS_B1["sources"]:
        with open(os.path.join(bench.ROOT, f), "rb") as fh:
            h.update(fh.read())
    # the sources as they are: the capture applies (scaled by the batch) only if it
    # was taken on them
    monkeypatch.setitem(bench.TRAFFIC_PASS_B1, "sha256", h.hexdigest())
    assert bench.captured_traffic("pass_kernel", 4) == 4 * bench.TRAFFIC_PASS_B1["bytes"]
    assert bench.captured_traffic("build_pass_kernel", 4) is None
    monkeypatch.setitem(bench.TRAFFIC_PASS_B1, "sha256", "0" * 64)
    assert bench.captured_traffic("pass_kernel", 4) is None   # sources changed since
