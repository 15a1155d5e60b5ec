"""Host-side helpers of bench.py that the reported numbers depend on (no GPU needed)."""

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_interleave_rows_puts_gate_on_even_rows():
    a = np.arange(12).reshape(3, 4)
    b = -np.arange(12).reshape(3, 4) - 1
    out = bench.interleave_rows(a, b)
    assert out.shape == (6, 4)
    assert np.array_equal(out[0::2], a) and np.array_equal(out[1::2], b)


def test_fused_weights_interleaves_codes_scales_and_zeros():
    rng = np.random.default_rng(0)
    w = {nm: (rng.integers(0, 256, (8, 256), dtype=np.uint8), rng.random((8, 2)).astype(np.float16),
              rng.integers(0, 256, (8, 2), dtype=np.uint8)) for nm in ("gate", "up", "down")}
    f = bench.fused_weights(w)
    assert set(f) == {"gate_up", "down"}
    for i in range(3):
        assert np.array_equal(f["gate_up"][i][0::2], w["gate"][i])
        assert np.array_equal(f["gate_up"][i][1::2], w["up"][i])
        assert f["gate_up"][i].dtype == w["gate"][i].dtype
    assert f["down"] is w["down"]


def test_step_units_count_each_call_once():
    dec = bench.workload_spec("ffn8b_decode")
    pre = bench.workload_spec("ffn8b_prefill")
    F, D, G = bench.D_FF, bench.D_MODEL, bench.GROUP
    b, f = bench.step_units(dec)
    exp_b = exp_f = 0
    for r in dec["widths"]:
        for M in dec["batches"]:
            # gate+up: planes + scales/zeros of 2F rows, x once, gated output [M, F]
            exp_b += 2 * F * D * r // 8 + 2 * F * (D // G) * 3 + M * D * 2 + M * F * 2
            # down
            exp_b += D * F * r // 8 + D * (F // G) * 3 + M * F * 2 + M * D * 2
            exp_f += 2 * M * (2 * F) * D + 2 * M * D * F
    assert (b, f) == (exp_b, exp_f)
    # both workloads write the gated product of the gate+up call
    assert bench.out_cols(pre, "gate_up") == F and bench.out_cols(dec, "gate_up") == F
    _, fp = bench.step_units(pre)
    assert fp == sum(2 * 2048 * (2 * F) * D + 2 * 2048 * D * F for _ in pre["widths"])


def test_both_arms_report_the_same_workload_config():
    args = type("A", (), dict(workload="ffn8b_decode"))()
    spec = bench.workload_spec("ffn8b_decode")
    c = bench.workload_config(args, spec, 1)
    assert c["workload"] == "ffn8b_decode" and c["widths"] == [2, 3, 4, 6, 8] and c["batches"] == [1, 4, 16]
    assert "gated" in c["shapes"]
    assert "gated" in bench.workload_config(type("A", (), dict(workload="ffn8b_prefill"))(),
                                            bench.workload_spec("ffn8b_prefill"), 1)["shapes"]


def test_copy_groups_cover_every_call_once_in_order():
    # decode-sized inputs (M in {1, 4, 16} rows of 4096 bf16) at five widths: one run per step
    dec = [m * 4096 * 2 for m in (1, 4, 16)] * 5
    assert bench.copy_groups(dec) == [list(range(15))]
    # prefill-sized inputs (M = 2048): one run per call
    assert bench.copy_groups([2048 * 4096 * 2] * 3) == [[0], [1], [2]]
    # a run closes at the threshold; the remainder forms the last run
    assert bench.copy_groups([3, 1, 2, 2, 1], min_bytes=4) == [[0, 1], [2, 3], [4]]
    assert bench.copy_groups([], min_bytes=4) == []
    for sizes in ([5, 1, 1, 1, 9, 2], [1] * 7, [10]):
        flat = [i for g in bench.copy_groups(sizes, min_bytes=4) for i in g]
        assert flat == list(range(len(sizes)))


def test_choose_case_cpu_baseline_is_bounded_and_well_formed():
    t = bench.time.perf_counter()
    rec = bench.cpu_choose_rate(budget_s=0.05, rows=1)
    assert bench.time.perf_counter() - t < 30
    assert rec["kind"] == "oracle" and rec["unit"] == "Gweights/s"
    assert rec["value"] > 0 and rec["cores"] >= 1
    assert "1 rows" in rec["sample"] and "pass" in rec["sample"]
