"""Host-side logic of bench.py, on the CPU: the algorithmic byte and FLOP
counts the roofline fractions divide by, the ncu-traffic lookup and its source
digest, the steady-round statistics, and the load-peaks fallback."""
import json
import os
import shutil

import pytest

import bench
import workloads as W


def test_algorithmic_bytes_of_the_headline_step():
    wl = W.BY_NAME[bench.HEADLINE]
    assert (wl.B, wl.T, wl.H, wl.d_k, wl.d_v, wl.io) == (8, 4096, 16, 128, 128, "bf16")
    # q, k, log_alpha, b (d_k each) and v, w, o (d_v each) in bf16, once; S_T in fp32, once
    tokens = 8 * 4096 * 16 * (4 * 128 + 3 * 128) * 2
    state = 8 * 16 * 128 * 128 * 4
    assert bench.chunk_bytes(wl, with_s0=False) == tokens + state == 947_912_704
    assert bench.chunk_bytes(wl, with_s0=True) == tokens + 2 * state
    assert bench.chunk_bytes(wl, with_s0=False, with_st=False) == tokens


def test_algorithmic_bytes_of_a_decode_step():
    wl = W.BY_NAME["decode_bf16"]
    # one token per (sequence, head) in bf16, the fp32 state read once and written once
    per_head = (4 * wl.d_k + 3 * wl.d_v) * 2 + 2 * wl.d_k * wl.d_v * 4
    assert bench.decode_bytes(wl) == wl.B * wl.H * per_head


def test_chunk_flops_counts():
    wl = W.BY_NAME[bench.HEADLINE]
    C = wl.chunk
    per = C * (3 * wl.d_k + 2 * wl.d_v) + C * C / 3 + 6 * wl.d_k * wl.d_v
    assert bench.chunk_flops(wl) == pytest.approx(per * wl.B * wl.T * wl.H)
    # dominated by the state terms: more than 6 d_k d_v per token-head
    assert bench.chunk_flops(wl) > 6 * wl.d_k * wl.d_v * wl.B * wl.T * wl.H


def _copy_tree(tmp_path):
    """The files measured_traffic reads, copied under a scratch root."""
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    os.makedirs(tmp_path / "profiles")
    shutil.copy(os.path.join(bench.ROOT, "profiles", "traffic.json"), tmp_path / "profiles" / "traffic.json")
    for k in rec.values():
        for src in k["sources"]:
            dst = tmp_path / src
            os.makedirs(dst.parent, exist_ok=True)
            shutil.copy(os.path.join(bench.ROOT, src), dst)
    return rec


def test_measured_traffic_scales_and_checks_the_source_digest(tmp_path, monkeypatch):
    rec = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    c = rec["chunk_fwd_tc"]
    per_case = c["dram_bytes_read"] + c["dram_bytes_write"]
    assert bench.measured_traffic("chunk_fwd_tc", c["case_batch"]) == pytest.approx(per_case)
    assert bench.measured_traffic("chunk_fwd_tc", 4 * c["case_batch"]) == pytest.approx(4 * per_case)
    assert bench.measured_traffic("no_such_kernel", 8) is None
    # any change to a source the capture covers makes the figure stale
    with open(tmp_path / c["sources"][0], "a") as f:
        f.write("\n")
    assert bench.measured_traffic("chunk_fwd_tc", 8) is None
    assert bench.measured_traffic("decode_step", 256) is not None or \
        c["sources"][0] in rec["decode_step"]["sources"]


def test_committed_traffic_matches_the_sources():
    # the committed capture was taken of the committed kernel sources
    assert bench.measured_traffic("chunk_fwd_tc", 8) is not None
    assert bench.measured_traffic("decode_step", 256) is not None


def test_steady_round_statistics(monkeypatch):
    times = iter([10.0, 30.0, 20.0, 40.0, 50.0])   # ms per round of `per_round` calls
    monkeypatch.setattr(bench, "device_time_ms", lambda fn, steps, stream: next(times))
    st = bench.steady_rounds(lambda: None, None, min_s=0.1, per_round=10)
    # rounds until 100 ms of device time: 10 + 30 + 20 + 40 = 100
    assert st["rounds"] == 4 and st["calls_per_round"] == 10
    assert st["ms_per_call_median"] == pytest.approx(2.5)
    assert st["ms_per_call_min"] == pytest.approx(1.0) and st["ms_per_call_max"] == pytest.approx(4.0)
    assert st["seconds"] == pytest.approx(0.1)


def test_load_peaks_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6538.3, "bf16_tflops": 1662.5}))
    p = bench.load_peaks()
    assert p == {"hbm_gbs": 6538.3, "bf16_tflops": 1662.5, "source": "measured"}
