"""Host-side bookkeeping of bench.py (no GPU): the algorithmic bytes the
roofline divides by, and the ncu traffic record that is reported only while
the decode sources are the ones it was measured on."""
import os

import pytest

import bench
from rank_kv_cache_lrkv_b200 import workloads as wk

LLAMA = wk.LLAMA31_LAYER_32K_ANCHORS


def test_step_bytes_of_the_llama_layer_by_hand():
    # 32 units; at L = 32769: 1 sink + 128 window anchors, 32640 latent tokens;
    # codes 2 B x (64 + 32), anchors 2 x 128 x 2 B, q and o 32 heads x 128 x 2 B
    L = 32769
    lat = L - 1 - 128
    want = 4 * 8 * lat * 96 * 2 + 4 * 8 * 129 * 512 + 2 * 4 * 32 * 256
    assert bench.step_bytes(LLAMA, L) == want == 202_719_232


def test_step_bytes_short_sequences_are_all_anchors():
    # below sink + window every token is full-rank and nothing is latent
    assert bench.step_bytes(LLAMA, 50) == 4 * 8 * 50 * 512 + 2 * 4 * 32 * 256
    assert bench.step_bytes(LLAMA, 0) == 2 * 4 * 32 * 256


def _current_sources():
    import hashlib
    csrc = os.path.join(os.path.dirname(os.path.abspath(bench.__file__)),
                        "rank_kv_cache_lrkv_b200", "csrc")
    return {f: hashlib.sha256(open(os.path.join(csrc, f), "rb").read()).hexdigest()
            for f in ("decode.cu", "common.cuh")}


def test_traffic_record_scales_with_the_algorithmic_bytes(monkeypatch):
    ctx, nbytes = 32769, 205_418_240
    monkeypatch.setitem(bench.TRAFFIC, LLAMA.name,
                        {"bytes": nbytes, "context": ctx, "sources": _current_sources()})
    assert bench.measured_traffic(LLAMA, ctx) == nbytes
    L = ctx + 263
    ratio = nbytes / bench.step_bytes(LLAMA, ctx)
    assert bench.measured_traffic(LLAMA, L) == round(ratio * bench.step_bytes(LLAMA, L))


def test_committed_traffic_record_is_plausible():
    # whether or not it still matches the sources, the record holds one
    # call's DRAM bytes: the pages once plus small overheads
    rec = bench.TRAFFIC[LLAMA.name]
    assert 1.0 < rec["bytes"] / bench.step_bytes(LLAMA, rec["context"]) < 1.05


def test_traffic_record_is_dropped_when_the_sources_change(monkeypatch):
    rec = dict(bench.TRAFFIC[LLAMA.name])
    rec["sources"] = dict(rec["sources"], **{"decode.cu": "0" * 64})
    monkeypatch.setitem(bench.TRAFFIC, LLAMA.name, rec)
    assert bench.measured_traffic(LLAMA, rec["context"]) is None
    assert bench.measured_traffic(wk.TINY_SINGLE_HEAD, 512) is None  # no record at all


def test_config_names_the_workload_and_its_sizes():
    c = bench.config_of(LLAMA)
    assert c["workload"] == LLAMA.name
    assert (c["B"], c["H_q"], c["H_kv"], c["T"], c["r_k"], c["r_v"]) == (4, 32, 8, 32768, 64, 32)
    assert "model" not in c
