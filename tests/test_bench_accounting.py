"""bench.py's roofline arithmetic on CPU, with made-up kernel times: the step's
algorithmic work of a kernel (both directions) divided evenly over its
launches, against the average launch time; the peak by bound; the traffic
record scaled to the tokens one launch processes."""
import json
import math

import pytest

import bench
from test_rnn_layer_b200 import synth as S

PEAKS = {"hbm_gbs": 6543.4, "bf16_tflops": 1637.0, "bf16_tflops_sustained": 1386.2, "sm_max_mhz": 1965.0,
         "_source": "measured"}
CLOCKS = {"sm_mhz": 1965.0}


def test_scan_flops_per_head_token_match_the_chunk_algebra():
    w = S.FULL63S
    per_dir = bench._algorithmic(w)["scan_chunk_tc2"][1]
    # 7 d-by-m products (A, Y, P, the two updates, Aq, Z1) + the two causal b-wide corrections
    assert per_dir == w.H * w.T * (7 * 2 * w.d * w.m + 2 * w.b * (w.d + w.m))
    assert per_dir / (w.H * w.T) == 270336


def test_scan_roofline_divides_two_directions_over_the_launches():
    w = S.FULL63S
    launches, ms_each = 50, 1.9
    roof = bench._roofline("scan_chunk_tc2", ms_each, launches, w, PEAKS, CLOCKS)
    per_dir = bench._algorithmic(w)["scan_chunk_tc2"][1]
    expect_work = 2 * per_dir / launches
    assert roof["work_per_launch"] == pytest.approx(expect_work)
    assert roof["achieved"] == pytest.approx(expect_work / (ms_each * 1e-3) / 1e12, rel=1e-3)
    tf32 = PEAKS["bf16_tflops_sustained"] * 1.1 / 2.25
    assert roof["peak"] == pytest.approx(tf32, rel=1e-3) and roof["bound"] == "tensor"
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"], rel=1e-3)
    # the same work done in one launch per direction gives the same fraction
    roof1 = bench._roofline("scan_chunk_tc2", ms_each * launches / 2, 2, w, PEAKS, CLOCKS)
    assert roof1["frac"] == pytest.approx(roof["frac"], rel=1e-3)


def test_gate_and_alu_bounds():
    w = S.FULL63S
    g = bench._roofline("gate", 2.0, 2, w, PEAKS, CLOCKS)
    assert g["bound"] == "hbm" and g["unit"] == "GB/s" and g["peak"] == PEAKS["hbm_gbs"]
    assert g["work_per_launch"] == w.T * w.model_dim * 11
    s = bench._roofline("scan_linear", 100.0, 2, w, PEAKS, CLOCKS)
    assert s["bound"] == "alu" and s["peak"] == pytest.approx(148 * 128 * 2 * 1965e6 / 1e12, rel=1e-3)
    # the scan backward's products: tf32 for a bf16 layer, three tf32 products each for an fp32 one
    tf32 = PEAKS["bf16_tflops_sustained"] * 1.1 / 2.25
    b16 = bench._roofline("scan_backward", 100.0, 2, w, PEAKS, CLOCKS)
    b32 = bench._roofline("scan_backward", 100.0, 2, w.with_(dtype="f32"), PEAKS, CLOCKS)
    assert b16["bound"] == b32["bound"] == "tensor"
    assert b16["peak"] == pytest.approx(tf32, rel=1e-3) and b32["peak"] == pytest.approx(tf32 / 3, rel=1e-3)


def test_traffic_record_scales_with_the_tokens_of_a_launch(tmp_path, monkeypatch):
    w = S.FULL63S
    src_hash = bench._src_hash(*bench.KERNEL_SRC["scan_chunk_tc2"])
    rec = {"scan_chunk_tc2": {"src_hash": src_hash, "bytes_per_launch_per_unit": 1000.0}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_PATH", str(path))
    roof = bench._roofline("scan_chunk_tc2", 1.0, 50, w, PEAKS, CLOCKS)
    assert roof["traffic"] == pytest.approx(1000.0 * w.T * 2 / 50 / 1024)
    rec["scan_chunk_tc2"]["src_hash"] = "stale"
    path.write_text(json.dumps(rec))
    assert bench._roofline("scan_chunk_tc2", 1.0, 50, w, PEAKS, CLOCKS)["traffic"] is None


def test_attention_flops_count_every_segment():
    """4 L_s^2 D per segment, the last segment ragged."""
    assert bench._attention_flops(10, 8, 4) == 4.0 * (16 + 16 + 4) * 8
    assert bench._attention_flops(313344, 3072, 14922) == 4.0 * 3072 * (20 * 14922 ** 2 + 14904 ** 2)
