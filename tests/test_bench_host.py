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


def test_stack_permutations_keep_gate_up_pairs_and_are_distinct():
    """The stack's layers are row-permuted copies of the seeded 8B layer: gate+up rows move in
    pairs (row 2i gate, 2i + 1 up of the same output channel), down rows singly; every layer's
    permutation is a bijection and layers differ."""
    perms = bench.stack_perms(layers=3)
    for pp, pd in perms:
        assert sorted(pp.tolist()) == list(range(bench.D_FF))
        assert sorted(pd.tolist()) == list(range(bench.D_MODEL))
        rows = bench.stack_rows(pp)
        assert np.array_equal(rows[0::2], 2 * pp) and np.array_equal(rows[1::2], 2 * pp + 1)
    assert not np.array_equal(perms[0][0], perms[1][0])
    assert np.array_equal(bench.stack_perms(layers=3)[2][1], perms[2][1])   # seeded


def test_stack_layer_host_moves_codes_scales_and_zeros_together():
    rng = np.random.default_rng(1)
    F, D, G = bench.D_FF, bench.D_MODEL, bench.GROUP
    fused = {"gate_up": (np.arange(2 * F, dtype=np.int64)[:, None] * np.ones((1, 2)), np.arange(2 * F)[:, None],
                         -np.arange(2 * F)[:, None]),
             "down": (np.arange(D)[:, None] * np.ones((1, 2)), np.arange(D)[:, None], -np.arange(D)[:, None])}
    perms = bench.stack_perms(layers=2)
    gu, dn = bench.stack_layer_host(fused, perms, 1)
    idx = bench.stack_rows(perms[1][0])
    assert np.array_equal(gu[0][:, 0], idx) and np.array_equal(gu[1][:, 0], idx) and np.array_equal(gu[2][:, 0], -idx)
    assert np.array_equal(dn[0][:, 0], perms[1][1]) and np.array_equal(dn[2][:, 0], -perms[1][1])
    del rng, G


def test_stack_units_count_each_layer_once():
    """One pass: per layer the gated gate+up call (bf16 out, N/2 columns) and the down call into
    the fp32 residual (read and written); flops 2 M (2F D + D F) per layer."""
    widths = [2, 3, 4]
    b, f = bench.stack_units(1, widths)
    D, F, G = bench.D_MODEL, bench.D_FF, bench.GROUP
    want = 0
    for r in widths:
        want += 2 * F * D * r // 8 + 2 * F * (D // G) * 3 + D * 2 + F * 2
        want += D * F * r // 8 + D * (F // G) * 3 + F * 2 + D * 8
    assert b == want
    assert f == len(widths) * 2 * (2 * F * D + D * F)


def test_sweep_shapes_and_configs():
    sw = bench.SWEEPS["ffn9b_sweep"]
    assert sw["group"] == 64 and sw["batches"] == (1, 8, 32, 128, 512, 2048) and tuple(sw["widths"]) == (2, 3, 4, 6, 8)
    one = bench.SWEEPS["linear1024"]
    assert (one["n"], one["k"], one["group"], one["batches"]) == (1024, 1024, 128, (1,))
    import argparse
    cfg = bench.sweep_config(argparse.Namespace(workload="ffn9b_sweep"), sw, {"gate_up": [28672, 3584]}, 1)
    assert cfg["workload"] == "ffn9b_sweep" and cfg["group"] == 64 and cfg["batches"][-1] == 2048


def test_linear_bytes_counts_exactly_r_bits_a_weight():
    for r in (2, 3, 4, 6, 8):
        b = bench.linear_bytes(1, 4096, 14336, r)
        assert b == 4096 * 14336 * r // 8 + 4096 * (14336 // 128) * 3 + 14336 * 2 + 4096 * 2
