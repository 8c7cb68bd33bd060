"""The benchmark's roofline arithmetic on the host: algorithmic work per stage, achieved rate
= work / measured stage time, fraction = achieved / peak, and which stages are listed."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from kv_cache_compression_group_b200 import jolt as J, synth  # noqa: E402

W = synth.WORKLOADS["llama31_8b_64k"]
OPTS = J.default_options(W.T, W.D, "randomized")
NU = 2 * W.n_layers // W.layers_per_group
PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
ALU = {"peak_tops": 40.0}


def test_table_op_count_by_hand():
    # 4 shared operations + 4 per bit-width b > 0 + 1 for b = 0, bits {0, 1, 2, 3, 4, 8}
    ops, per = bench.table_alu_ops(W, OPTS, NU)
    assert per == 4 + 5 * 4 + 1 == 25
    elements = 16 * (4 * 8 * 65536 * 128)   # 16 units of 4 layers x 8 heads x 64K tokens x 128
    assert ops == elements * 4 * 4 * 25 == 1_717_986_918_400


def _recs(pairs):
    return [dict(r_T=rt, r_D=128, bits=b) for rt, b in pairs]


def test_stage_rooflines_arithmetic():
    per_call = 400.0
    n_calls = 4
    # (total ms over the calls, launches, unused): table 130 ms per call, sketch 6 x 12.5 ms,
    # encode 24 ms, a latency-bound stage 60 ms, and one below 5 % of a call
    prof = {
        "table_kernel": (4 * 130.0, 4, None),
        "sketch_product": (4 * 75.0, 24, None),
        "encode": (4 * 24.0, 4, None),
        "sym_eig": (4 * 60.0, 4, None),
        "allocate": (4 * 0.3, 4, None),
    }
    chosen = [_recs([(960, 4), (512, 0)] * (NU // 2)), _recs([(256, 2)] * NU)]
    lines = bench.stage_rooflines(W, OPTS, NU, prof, n_calls, per_call, PEAKS, "measured", ALU, chosen)
    by = {l["kernel"]: l for l in lines}
    assert "allocate" not in by                       # 0.3 ms < 5 % of 400 ms
    assert [l["kernel"] for l in lines] == ["table_kernel", "sketch_product", "sym_eig", "encode"]
    assert by["sym_eig"]["bound"] == "latency" and "frac" not in by["sym_eig"]

    t = by["table_kernel"]
    assert t["bound"] == "alu" and t["ms_per_launch"] == pytest.approx(130.0)
    assert t["achieved"] == pytest.approx(1_717_986_918_400 / 0.130 / 1e12)
    assert t["frac"] == pytest.approx(t["achieved"] / 40.0)
    assert t["share_of_compress"] == pytest.approx(130.0 / 400.0)

    s = by["sketch_product"]
    k = max(OPTS.token_ranks) + OPTS.oversample   # 970
    flops = (2 + 2 * OPTS.power_iters) * 2.0 * W.T * (W.layers_per_group * W.n_heads * W.D) * k * NU
    assert s["work_per_launch"] == pytest.approx(flops)
    assert s["frac"] == pytest.approx(flops / 0.075 / 1e12 / 1400.0)   # the sustained peak

    # encode: the reconstruction of the units that store a residual, at their chosen ranks,
    # averaged over the step's budgets
    e = by["encode"]
    per_rank = 2.0 * W.T * (W.layers_per_group * W.n_heads) * W.D
    expect = (per_rank * 960 * (NU // 2) + per_rank * 256 * NU) / 2
    assert e["bound"] == "tensor" and e["work_per_launch"] == pytest.approx(expect)


def test_stage_rooflines_without_allocation_records():
    # no blobs (no chosen ranks): the encode stage has zero work rather than a made-up one
    prof = {"encode": (100.0, 1, None)}
    lines = bench.stage_rooflines(W, OPTS, NU, prof, 1, 100.0, PEAKS, "measured", ALU, [])
    assert lines[0]["work_per_launch"] == 0.0 and lines[0]["frac"] == 0.0
