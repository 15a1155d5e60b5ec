"""Pins for the fp64 oracle, against what the pages and the mathematics fix.

Each test is chosen so that a plausible mistake in the oracle (a wrong shift,
a dropped delta or zero point, a transposed operand or scale, a wrong tie or
clamp) fails at least one of them.  No expected value here comes from the
CUDA library.
"""

import itertools

import numpy as np
import pytest

import oracle as O
from nested_bit_weight_msb_b200 import synth

ALL_CODES = np.arange(256, dtype=np.uint8)


# --------------------------------------------------------------------------
# Worked examples printed on the pages (tests/golden)
# --------------------------------------------------------------------------

def test_errata_example_234(golden):
    rows = golden("matquant_errata_234.txt")
    assert len(rows) == 2
    for code, r, mode, expect in rows:
        got = O.reconstruct(np.array([int(code)], dtype=np.uint8), int(r), mode=mode)[0]
        assert got == float(expect)
    # the intermediate value the page prints: 234 / 64 rounds to 4
    assert np.floor(234 / 64 + 0.5) == 4


def test_int2_grid(golden):
    for r, mode, *vals in golden("int2_grid_from_int8.txt"):
        got = np.unique(O.reconstruct(ALL_CODES, int(r), mode=mode))
        assert got.tolist() == [float(v) for v in vals]
        assert np.all(np.diff(got) == 64.0)          # "constant spacing 64"


def test_true_prefix_hand_example(golden):
    rows = golden("true_prefix_234.txt")
    assert {int(r[1]) for r in rows} == set(O.WIDTHS)
    for code, r, p, qh in rows:
        q = np.array([int(code)], dtype=np.uint8)
        assert O.prefix(q, int(r))[0] == int(p)
        assert O.reconstruct(q, int(r))[0] == float(qh)


# --------------------------------------------------------------------------
# Exhaustive slicing invariants (256 codes x every width)
# --------------------------------------------------------------------------

def test_r8_is_identity():
    assert np.array_equal(O.prefix(ALL_CODES, 8), ALL_CODES.astype(np.int64))
    assert np.array_equal(O.reconstruct(ALL_CODES, 8), ALL_CODES.astype(np.float64))
    assert O.delta(8) == 0.0


@pytest.mark.parametrize("r", O.WIDTHS)
def test_prefix_range_and_bits(r):
    p = O.prefix(ALL_CODES, r)
    assert p.min() == 0 and p.max() == (1 << r) - 1
    # each prefix value is shared by exactly 2^(8-r) codes (a cell)
    counts = np.bincount(p, minlength=1 << r)
    assert np.all(counts == (1 << (8 - r)))
    # it is the top r bits, read bit by bit
    for q in (0, 1, 0x55, 0xAA, 0x80, 0x7F, 234, 255):
        bits = [(q >> (7 - i)) & 1 for i in range(r)]
        assert O.prefix(np.array([q], dtype=np.uint8), r)[0] == int("".join(map(str, bits)), 2)


@pytest.mark.parametrize("r_hi,r_lo", [(a, b) for a, b in itertools.product(O.WIDTHS, O.WIDTHS) if b < a])
def test_nesting(r_hi, r_lo):
    # slicing to r then to r' < r equals slicing directly to r'
    p_hi = O.prefix(ALL_CODES, r_hi)
    assert np.array_equal(p_hi >> (r_hi - r_lo), O.prefix(ALL_CODES, r_lo))
    trunc = O.reconstruct(ALL_CODES, r_hi, mode="truncate").astype(np.uint8)
    assert np.array_equal(O.prefix(trunc, r_lo), O.prefix(ALL_CODES, r_lo))
    # the centred code lies in the same r-cell, hence keeps every shorter prefix
    centred = O.reconstruct(ALL_CODES, r_hi)
    assert np.array_equal(np.floor(centred).astype(np.int64) >> (8 - r_lo), O.prefix(ALL_CODES, r_lo))


@pytest.mark.parametrize("r", O.WIDTHS)
def test_delta_centres_cell(r):
    width = 1 << (8 - r)
    assert 2 * O.delta(r) == width - 1
    p = O.prefix(ALL_CODES, r).astype(np.float64)
    qh = O.reconstruct(ALL_CODES, r)
    assert np.all(qh >= p * width) and np.all(qh <= (p + 1) * width - 1)
    # brute force: among offsets in steps of 1/4 across the cell, delta_r minimises
    # the squared error to the c-bit codes of each cell (App. A.1's claim)
    cand = np.arange(0, width * 4 + 1) / 4.0
    for cell in range(1 << r):
        codes = np.arange(cell * width, (cell + 1) * width, dtype=np.float64)
        err = [np.sum((codes - (cell * width + c)) ** 2) for c in cand]
        best = cand[int(np.argmin(err))]
        assert best == O.delta(r)


@pytest.mark.parametrize("r", [2, 3, 4, 6])
def test_centring_beats_truncation(r):
    rms_tp = np.sqrt(np.mean((O.reconstruct(ALL_CODES, r) - ALL_CODES) ** 2))
    rms_tr = np.sqrt(np.mean((O.reconstruct(ALL_CODES, r, mode="truncate") - ALL_CODES) ** 2))
    assert rms_tp < rms_tr
    # truncation sits at the lower edge of each cell
    assert np.all(O.reconstruct(ALL_CODES, r, mode="truncate") <= ALL_CODES)


def test_half_cell_reading_differs():
    assert O.delta(2, "half_cell") == 32.0 and O.delta(2) == 31.5


def test_matquant_rule_properties():
    # clamped rule stays on 2^r levels; the unclamped one has 2^r + 1
    for r in (2, 3, 4, 6):
        lv_c = np.unique(O.reconstruct(ALL_CODES, r, mode="matquant_round"))
        lv_e = np.unique(O.reconstruct(ALL_CODES, r, mode="extra_precision"))
        assert len(lv_c) == (1 << r)
        assert len(lv_e) == (1 << r) + 1 and lv_e.max() == 256.0
    # it reads r+1 bits, the true prefix exactly r (MatGPTQ §2.3, App. A.1)
    assert O.bits_read_per_weight(2, "matquant_round") == 3
    assert O.bits_read_per_weight(2, "true_prefix") == 2
    # rounding rule is not nested: 95 -> 4 bits -> 2 bits differs from 95 -> 2 bits
    q = np.array([95], dtype=np.uint8)
    via4 = O.reconstruct(O.reconstruct(q, 4, mode="matquant_round").astype(np.uint8), 2, mode="matquant_round")
    direct = O.reconstruct(q, 2, mode="matquant_round")
    assert via4[0] == 128.0 and direct[0] == 64.0
    # tie rules differ on an exact tie (96 / 64 = 1.5)
    t = np.array([96], dtype=np.uint8)
    assert O.reconstruct(t, 2, mode="matquant_round", tie="up")[0] == 128.0
    assert O.reconstruct(t, 2, mode="matquant_round", tie="even")[0] == 128.0
    t = np.array([160], dtype=np.uint8)               # 2.5 -> 3 (up) vs 2 (even)
    assert O.reconstruct(t, 2, mode="matquant_round", tie="up")[0] == 192.0
    assert O.reconstruct(t, 2, mode="matquant_round", tie="even")[0] == 128.0


def test_codes_are_validated():
    with pytest.raises(ValueError):
        O.prefix(np.array([256]), 2)
    with pytest.raises(TypeError):
        O.prefix(np.array([1.5]), 2)


# --------------------------------------------------------------------------
# Dequantisation and the product: closed forms
# --------------------------------------------------------------------------

def _rand_problem(M, N, K, group, seed):
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    s = rng.uniform(1e-3, 2e-2, size=(N, K // group)).astype(np.float16)
    z = rng.integers(0, 256, size=(N, K // group), dtype=np.uint8)
    x = rng.standard_normal((M, K))
    return x, q, s, z


@pytest.mark.parametrize("r", O.WIDTHS)
def test_zero_point_equal_codes_give_zero(r):
    # W = s * (q_hat - z) vanishes when every code equals its zero point at r = 8;
    # at r < 8 it equals s * (q_hat - q), which the cell pins bound by s * 2^(8-r) / 2
    x, q, s, z = _rand_problem(3, 5, 256, 128, 1)
    z = q[:, ::128].copy()
    q = np.repeat(z, 128, axis=1)
    w = O.dequant(q, s, z, r, 128)
    bound = np.repeat(s.astype(np.float64), 128, axis=1) * ((1 << (8 - r)) / 2.0)
    assert np.all(np.abs(w) <= bound)
    if r == 8:
        assert np.all(O.linear(x, q, s, z, 8, 128) == 0.0)


def test_one_hot_picks_a_column():
    # x = e_k returns W_hat[:, k]: pins the orientation (W stored [out, in]) and
    # the per-group indexing of scale and zero (non-square, several groups)
    x, q, s, z = _rand_problem(1, 7, 384, 128, 2)
    for r in O.WIDTHS:
        w = O.dequant(q, s, z, r, 128)
        for k in (0, 127, 128, 300, 383):
            e = np.zeros((1, 384))
            e[0, k] = 1.0
            y = O.linear(e, q, s, z, r, 128)
            g = k // 128
            expect = s[:, g].astype(np.float64) * (O.reconstruct(q[:, k], r) - z[:, g].astype(np.float64))
            assert np.array_equal(y[0], w[:, k])
            assert np.array_equal(y[0], expect)


def test_unit_scale_integer_product_is_exact():
    # s = 1, z = 0, r = 8: W_hat = q, so with integer x the product is an integer
    # matrix product, which int64 arithmetic gives exactly
    rng = np.random.default_rng(3)
    q = rng.integers(0, 256, size=(9, 512), dtype=np.uint8)
    x = rng.integers(-50, 51, size=(4, 512))
    s = np.ones((9, 4), dtype=np.float16)
    z = np.zeros((9, 4), dtype=np.uint8)
    y = O.linear(x.astype(np.float64), q, s, z, 8, 128)
    assert np.array_equal(y, (x.astype(np.int64) @ q.astype(np.int64).T).astype(np.float64))
    # r = 4: twice the reconstructed code is the integer 2*16*p + 15
    y4 = O.linear(x.astype(np.float64), q, s, z, 4, 128)
    two_qh = 32 * (q.astype(np.int64) >> 4) + 15
    assert np.array_equal(2 * y4, (x.astype(np.int64) @ two_qh.T).astype(np.float64))


def test_scale_is_per_row_and_group():
    # doubling the scale of one (row, group) doubles only that row's contribution
    x, q, s, z = _rand_problem(2, 4, 256, 64, 4)
    base = O.linear(x, q, s, z, 4, 64)
    s2 = s.copy()
    s2[1, 2] = s2[1, 2] * 2
    y2 = O.linear(x, q, s2, z, 4, 64)
    assert np.array_equal(np.delete(y2, 1, axis=1), np.delete(base, 1, axis=1))
    contrib = x[:, 128:192] @ (s[1, 2].astype(np.float64) * (O.reconstruct(q[1, 128:192], 4) - float(z[1, 2])))
    assert np.allclose(y2[:, 1] - base[:, 1], contrib, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", O.MODES)
def test_matmul_vs_scalar_loops(mode):
    x, q, s, z = _rand_problem(2, 3, 128, 64, 5)
    for r in (2, 3, 8):
        a = O.linear(x, q, s, z, r, 64, mode=mode)
        b = O.linear_loops(x, q, s, z, r, 64, mode=mode)
        assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("r", O.WIDTHS)
@pytest.mark.parametrize("group", [64, 128])
def test_group_sum_identity(r, group):
    x, q, s, z = _rand_problem(5, 6, 512, group, 6)
    a = O.linear(x, q, s, z, r, group)
    b = O.linear_group_sums(x, q, s, z, r, group)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def test_metadata_shape_checked():
    x, q, s, z = _rand_problem(1, 2, 256, 128, 7)
    with pytest.raises(ValueError):
        O.dequant(q, s[:, :1], z, 4, 128)


# --------------------------------------------------------------------------
# Mix'n'Match glue
# --------------------------------------------------------------------------

def test_rmsnorm_properties():
    rng = np.random.default_rng(8)
    h = rng.standard_normal((3, 257)) * 5
    n = O.rmsnorm(h, eps=0.0)
    assert np.allclose(np.mean(n * n, axis=-1), 1.0, rtol=1e-12)
    assert np.allclose(O.rmsnorm(7 * h, eps=0.0), n, rtol=1e-12)
    n_eps = O.rmsnorm(h, eps=1e-5)
    ms = np.mean(h * h, axis=-1)
    assert np.allclose(np.mean(n_eps * n_eps, axis=-1), ms / (ms + 1e-5), rtol=1e-12)


def test_silu_properties():
    t = np.linspace(-30, 30, 1201)
    # silu(t) - silu(-t) = t * (sigmoid(t) + sigmoid(-t)) = t
    assert np.allclose(O.silu(t) - O.silu(-t), t, rtol=1e-13, atol=1e-13)
    assert O.silu(np.array([0.0]))[0] == 0.0
    # slope 1/2 at the origin; silu(t) -> t for large t, -> 0 for very negative t
    hs = 1e-6
    assert abs((O.silu(np.array([hs]))[0] - O.silu(np.array([-hs]))[0]) / (2 * hs) - 0.5) < 1e-9
    assert abs(O.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(O.silu(np.array([-40.0]))[0]) < 1e-15
    # sigmoid(1) = e / (1 + e)
    assert abs(O.silu(np.array([1.0]))[0] - np.e / (1 + np.e)) < 1e-15


def test_ffn_block_zero_down_is_identity():
    rng = np.random.default_rng(9)
    K, F = 256, 128
    h = rng.standard_normal((2, K))
    qg = rng.integers(0, 256, (F, K), dtype=np.uint8)
    sg = np.full((F, K // 128), 0.01, dtype=np.float16)
    zg = rng.integers(0, 256, (F, K // 128), dtype=np.uint8)
    zd = rng.integers(0, 256, (K, F // 128), dtype=np.uint8)
    qd = np.repeat(zd, 128, axis=1)
    sd = np.full((K, F // 128), 0.01, dtype=np.float16)
    layer = {"gate": (qg, sg, zg), "up": (qg, sg, zg), "down": (qd, sd, zd)}
    assert np.array_equal(O.ffn_block(h, layer, 8, 128), h)


def _ffn_golden(golden):
    rows = golden("ffn_block_hand.txt")
    eps = [float(r[1]) for r in rows if r[0] == "eps"][0]
    h = np.array([[float(v) for v in r[1:]] for r in rows if r[0] == "h"])
    out = np.array([[float(v) for v in r[1:]] for r in rows if r[0] == "out"])
    layer = {}
    for r in rows:
        if r[0] == "codes":
            n, k = int(r[2]), int(r[3])
            q = np.array([int(v) for v in r[4:]], dtype=np.uint8).reshape(n, k)
            layer[r[1]] = (q, np.ones((n, k), dtype=np.float16), np.ones((n, k), dtype=np.uint8))
    return h, layer, eps, out


def test_ffn_block_hand_example(golden):
    """The block's result on a hand-worked two-row example (tests/golden/ffn_block_hand.txt)."""
    h, layer, eps, out = _ffn_golden(golden)
    got = O.ffn_block(h, layer, 8, 1, eps=eps)
    assert np.allclose(got, out, rtol=0, atol=1e-13)


def test_ffn_block_hand_example_catches_mutations(golden):
    """Each plausible mistake in the block glue moves the hand-worked answer: swapped gate and
    up, no RMSNorm, no residual, eps outside the square root, a transposed down projection."""
    h, layer, eps, out = _ffn_golden(golden)

    def lin(x, name, transpose=False):
        q, s, z = layer[name]
        if transpose:
            q, s, z = q.T.copy(), s.T.copy(), z.T.copy()
        return O.linear(x, q, s, z, 8, 1)

    def block(swap=False, norm=True, residual=True, eps_outside=False, transpose_down=False):
        if not norm:
            n = h
        elif eps_outside:
            n = h / (np.sqrt(np.mean(h * h, axis=-1, keepdims=True)) + eps)
        else:
            n = O.rmsnorm(h, eps)
        g, u = lin(n, "gate"), lin(n, "up")
        a = O.silu(u) * g if swap else O.silu(g) * u
        d = lin(a, "down", transpose=transpose_down)
        return h + d if residual else d

    assert np.allclose(block(), out, rtol=0, atol=1e-13)   # the reading itself matches
    for kw in ({"swap": True}, {"norm": False}, {"residual": False}, {"eps_outside": True},
               {"transpose_down": True}):
        assert np.max(np.abs(block(**kw) - out)) > 1e-2, kw


def test_mixnmatch_widths_recipe():
    w = synth.mixnmatch_widths(0)
    assert len(w) == 32 and sorted(w.tolist()) == [2] * 11 + [3] * 10 + [4] * 11
    assert O.mixnmatch_effective_bits(w) == 3.0
    assert not np.array_equal(w, synth.mixnmatch_widths(1))
    assert O.mixnmatch_effective_bits([2, 4], sizes=[3, 1]) == 2.5


# --------------------------------------------------------------------------
# Input generator sanity (inputs, not graded)
# --------------------------------------------------------------------------

def test_generator_sanity():
    q, s, z = synth.parent_weights(64, 1024, 128, seed=0)
    assert q.dtype == np.uint8 and s.dtype == np.float16 and z.dtype == np.uint8
    assert q.min() == 0 or q.max() == 255
    assert 100 < float(z.mean()) < 156
    q2, _, _ = synth.parent_weights(64, 1024, 128, seed=0)
    assert np.array_equal(q, q2)
    # dequantised r=8 weights reproduce the Gaussian draw to within half a step,
    # except where the fp16-rounded scale makes the group's extreme clip (rare)
    rng = np.random.default_rng(np.random.SeedSequence([0, 0, 0, 0]))
    w = 0.02 * rng.standard_normal((64, 1024), dtype=np.float32)
    w8 = O.dequant(q, s, z, 8, 128)
    step = np.repeat(s.astype(np.float64), 128, axis=1)
    err = np.abs(w8 - w) / step
    assert np.mean(err <= 0.5 + 1e-3) > 0.999 and err.max() < 2.0


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(10)
    a = (rng.standard_normal(10000) * np.exp(rng.uniform(-20, 20, 10000))).astype(np.float32)
    bits, vals = synth.bf16_round(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(vals, ref)
    xb, xv = synth.activations(4, 1000, outlier_frac=0.01)
    big = np.abs(xv).max(axis=0)
    assert (big > 10).sum() >= 5


# --------------------------------------------------------------------------
# Parent-code choice for several widths (MatGPTQ §3.2 item 2, App. A.2)
# --------------------------------------------------------------------------

def _one_weight(mode, s, z, widths, lams, w, group=64):
    wm = np.zeros((1, group), dtype=np.float32)
    wm[0, 0] = np.float32(w)
    return int(O.choose_codes(wm, np.array([[s]], np.float16), np.array([[z]], np.uint8), group,
                              widths, lams, mode)[0, 0])


def test_code_choice_hand_examples(golden):
    rows = golden("matgptq_code_choice.txt")
    assert len(rows) == 11
    for mode, s, z, widths, lams, w, want in rows:
        widths = tuple(int(v) for v in widths.split(","))
        lams = [float(v) for v in lams.split(",")]
        assert _one_weight(mode, float(s), int(z), widths, lams, float(w)) == int(want), (mode, widths, lams, w)


def _choice_problem(N=48, K=256, group=64, seed=5, spread=1.0):
    w, s, z = synth.float_weights(N, K, group, seed=seed)
    w = (w * np.float32(spread)).astype(np.float32)
    u = w.astype(np.float64) / np.repeat(s.astype(np.float64), group, axis=1) + np.repeat(z, group, axis=1)
    return w, s, z, u


@pytest.mark.parametrize("widths", [(8,), (2, 8), (3, 4, 8), (2, 3, 4, 6, 8), (4, 6, 8)])
def test_centred_choice_is_round_to_nearest(widths):
    # With the centred reconstruction the boundary between two cells of any width lies half
    # way between two 8-bit codes, so the nearest 8-bit code sits in the nearest cell of every
    # width and minimises every term at once: the choice is round-to-nearest whenever the
    # 8-bit term carries weight (ties at half-way excluded).  spread > 1 pushes weights past
    # the grid so the clamps at 0 and 255 are met too.
    rng = np.random.default_rng(len(widths))
    for spread in (1.0, 1.6):
        w, s, z, u = _choice_problem(spread=spread, seed=int(10 * spread))
        lams = rng.uniform(0.1, 2.0, len(widths)).astype(np.float32)
        got = O.choose_codes(w, s, z, 64, widths, lams, "true_prefix")
        want = np.clip(np.floor(u + 0.5), 0, 255)
        keep = np.abs(u - np.floor(u) - 0.5) > 1e-3
        assert keep.mean() > 0.99
        assert np.array_equal(got[keep], want[keep].astype(np.uint8))
        if spread > 1:
            assert (want == 0).any() and (want == 255).any()


@pytest.mark.parametrize("r", [2, 3, 4, 6])
@pytest.mark.parametrize("mode", ["true_prefix", "truncate"])
def test_single_width_choice_is_smallest_code_of_nearest_cell(r, mode):
    # one width below 8: every code of a cell scores the same, so the smallest code of the
    # cell whose reconstruction is nearest wins
    w, s, z, u = _choice_problem(seed=7, spread=1.3)
    got = O.choose_codes(w, s, z, 64, (r,), None, mode)
    step = 1 << (8 - r)
    off = (step - 1) / 2 if mode == "true_prefix" else 0.0
    v = (u - off) / step
    p = np.clip(np.floor(v + 0.5), 0, (1 << r) - 1)
    keep = np.abs(v - np.floor(v) - 0.5) > 1e-4
    assert np.array_equal(got[keep], (p[keep] * step).astype(np.uint8))
    assert np.all(got % step == 0)


@pytest.mark.parametrize("r", [2, 3, 4, 6])
def test_truncated_two_width_choice_by_cells(r):
    # Raw truncation, widths {r, 8}: a different algorithm in fp64 -- per cell of width r the
    # best code is the nearest code clamped into the cell, the cell's cost is
    # lam_r*(u - edge)^2 + lam_8*(u - code)^2, and the cheapest cell wins.  Near-ties between
    # cells and half-way codes are excluded.
    w, s, z, u = _choice_problem(N=32, seed=9, spread=1.2)
    lam = np.array([0.7, 1.3], dtype=np.float32)
    got = O.choose_codes(w, s, z, 64, (r, 8), lam, "truncate")
    step = 1 << (8 - r)
    edges = np.arange(1 << r, dtype=np.float64) * step
    uu = u[..., None]
    code = np.clip(np.floor(uu + 0.5), edges, edges + step - 1)
    cost = float(lam[0]) * (uu - edges) ** 2 + float(lam[1]) * (uu - code) ** 2
    order = np.sort(cost, axis=-1)
    best = np.argmin(cost, axis=-1)
    want = np.take_along_axis(code, best[..., None], axis=-1)[..., 0]
    keep = (order[..., 1] - order[..., 0] > 1e-6 * (1 + order[..., 0])) & (np.abs(u - np.floor(u) - 0.5) > 1e-4)
    assert keep.mean() > 0.95
    assert np.array_equal(got[keep], want[keep].astype(np.uint8))
    # the trade-off is real: some weights leave the nearest code
    assert (got != np.clip(np.floor(u + 0.5), 0, 255)).mean() > 0.05


def test_code_choice_lambda_properties():
    w, s, z, _ = _choice_problem(N=16, seed=11)
    base = O.choose_codes(w, s, z, 64, (2, 4, 8), [0.25, 0.5, 1.0], "truncate")
    # a power-of-two scale of every lambda scales every fp32 total exactly
    assert np.array_equal(base, O.choose_codes(w, s, z, 64, (2, 4, 8), [1.0, 2.0, 4.0], "truncate"))
    # zero weights drop their widths (0 + 0 + t == t exactly)
    only8 = O.choose_codes(w, s, z, 64, (8,), [1.0], "truncate")
    assert np.array_equal(only8, O.choose_codes(w, s, z, 64, (2, 4, 8), [0, 0, 1], "truncate"))
    only2 = O.choose_codes(w, s, z, 64, (2,), [1.0], "truncate")
    assert np.array_equal(only2, O.choose_codes(w, s, z, 64, (2, 4, 8), [1, 0, 0], "truncate"))
    assert not np.array_equal(only2, only8)
    # every lambda zero: all totals tie and the smallest code wins
    assert not O.choose_codes(w, s, z, 64, (3, 8), [0, 0], "truncate").any()


def test_code_choice_is_validated():
    w, s, z, _ = _choice_problem(N=2, K=64)
    for widths, lams in (((8, 4), None), ((4, 4), None), ((5,), None), ((), None), ((4, 8), [1, -1]),
                         ((4, 8), [1]), ((4, 8), [1, float("nan")])):
        with pytest.raises(ValueError):
            O.choose_codes(w, s, z, 64, widths, lams)
