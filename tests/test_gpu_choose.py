"""GPU parity of the parent-code choice (matq_choose_codes; "MatGPTQ: Efficient and Accurate
Inference over Nested Quantized Models", §3.2 item 2 and App. A.2) against the oracle's
brute force over all 256 codes: the codes must be identical, bit for bit.  Both sides make
the decision in fp32 with every operation rounded on its own, so equal inputs give equal
totals and the same first minimum."""

import itertools

import numpy as np
import pytest

import oracle as O
from nested_bit_weight_msb_b200 import synth

pytestmark = pytest.mark.gpu

SUBSETS = [c for n in range(1, 6) for c in itertools.combinations(O.WIDTHS, n)]
MODES = {"true_prefix": 0, "truncate": 1}


@pytest.fixture(scope="module")
def M():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nested_bit_weight_msb_b200 import matq
    return matq


def _device(w, s, z):
    import torch
    return (torch.from_numpy(np.ascontiguousarray(w, dtype=np.float32)).cuda(),
            torch.from_numpy(np.ascontiguousarray(s).view(np.int16)).cuda(),
            torch.from_numpy(np.ascontiguousarray(z)).cuda())


def _run(M, w, s, z, group, widths, lam, mode):
    dw, ds, dz = _device(w, s, z)
    return M.choose_codes(dw, ds, dz, group, widths, lam, MODES[mode]).cpu().numpy()


@pytest.mark.parametrize("mode", list(MODES))
def test_every_width_set(M, mode):
    """All 31 width sets, random lambdas (some zero), weights inside and beyond the grid, two
    group sizes, K a multiple of the group but not of 256, odd N."""
    rng = np.random.default_rng(3)
    for i, widths in enumerate(SUBSETS):
        N, K, group = (5, 192, 64) if i % 2 else (3, 384, 128)
        w, s, z = synth.float_weights(N, K, group, seed=i)
        w = (w * np.float32(rng.choice([0.4, 1.0, 1.7]))).astype(np.float32)
        lam = rng.uniform(0, 2, len(widths)).astype(np.float32)
        if i % 3 == 0:
            lam[rng.integers(0, len(widths))] = 0
        got = _run(M, w, s, z, group, widths, lam, mode)
        want = O.choose_codes(w, s, z, group, widths, lam, mode)
        assert np.array_equal(got, want), (widths, mode, int((got != want).sum()))


def _edge_problem(group=64):
    N, K = 6, 256
    w, s, z = synth.float_weights(N, K, group, seed=42)
    s = s.copy()
    z = z.copy()
    s[1, :] = np.float16(6e-8)     # smallest subnormal fp16 scale
    s[2, :] = np.float16(300.0)
    z[3, :] = 0
    z[4, :] = 255
    s32 = np.repeat(s.astype(np.float32), group, 1)
    z32 = np.repeat(z.astype(np.float32), group, 1)
    codes = np.arange(K, dtype=np.float32) % 256
    w[0, :64] = 0
    w[0, 64:128] = s32[0, 64:128] * (codes[64:128] - z32[0, 64:128])          # exact grid points
    w[0, 128:192] = s32[0, 128:192] * (codes[128:192] + 0.5 - z32[0, 128:192])  # half way
    w[0, 192:200] = [1e3, -1e3, 5e5, -5e5, 3e7, -3e7, 1e-30, -1e-30]
    w[5, :4] = [np.nan, np.inf, -np.inf, 0.0]
    return w.astype(np.float32), s, z


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("widths,lam", [((3, 4, 8), None), ((2, 8), (1.0, 1.0)), ((4,), (1.0,)),
                                        ((2, 3, 4, 6, 8), (0.1, 0.2, 0.3, 0.4, 0.5)),
                                        ((3, 8), (0.0, 0.0)), ((2, 4, 8), (1e25, 1.0, 1.0)),
                                        ((2, 4, 8), (1.0, 1.0, 0.0))])
def test_edge_inputs(M, mode, widths, lam):
    """Zero weights, exact grid points, half-way points, weights far outside the grid, NaN and
    infinities, subnormal and large scales, zero points 0 and 255, all-zero lambdas, lambdas
    past the range the cell search accepts, a zero weight on the finest width."""
    w, s, z = _edge_problem()
    got = _run(M, w, s, z, 64, widths, lam, mode)
    with np.errstate(invalid="ignore", over="ignore"):
        want = O.choose_codes(w, s, z, 64, widths, lam, mode)
    assert np.array_equal(got, want), int((got != want).sum())


@pytest.mark.parametrize("shape,group,widths,lam,mode", [
    ((14336, 4096), 128, (3, 4, 8), None, "true_prefix"),
    ((4096, 14336), 128, (2, 8), (1.0, 1.0), "truncate"),
    ((14336, 3584), 64, (2, 3, 4, 6, 8), (1.0, 0.5, 0.25, 0.125, 0.0625), "truncate"),
])
def test_full_size_sampled(M, shape, group, widths, lam, mode):
    """Benchmark FFN shapes in the launch configuration the bench times; 12 sampled rows are
    checked against the oracle in full."""
    N, K = shape
    w, s, z = synth.float_weights(N, K, group, seed=1)
    got = _run(M, w, s, z, group, widths, lam, mode)
    rows = np.random.default_rng(N).choice(N, 12, replace=False)
    rows[0], rows[1] = 0, N - 1
    want = O.choose_codes(w[rows], s[rows], z[rows], group, widths, lam, mode)
    assert np.array_equal(got[rows], want)


def test_output_stays_in_bounds_and_feeds_pack(M):
    """The call writes exactly N*K bytes (a canary after the output survives), and its codes
    are ordinary parent codes: packed and served at width r they give the oracle's product."""
    import torch
    from helpers import check_close
    N, K, group = 37, 512, 128
    w, s, z = synth.float_weights(N, K, group, seed=8)
    dw, ds, dz = _device(w, s, z)
    buf = torch.full((N * K + 64,), 0xA5, dtype=torch.uint8, device="cuda")
    out = buf[: N * K].view(N, K)
    M.choose_codes(dw, ds, dz, group, (3, 4, 8), None, M.MATQ_SLICE_TRUE_PREFIX, out=out)
    tail = buf[N * K:].cpu().numpy()
    assert np.all(tail == 0xA5)
    codes = O.choose_codes(w, s, z, group, (3, 4, 8))
    assert np.array_equal(out.cpu().numpy(), codes)
    planes = M.pack(out, r_keep=8)
    xb, xv = synth.activations(3, K, seed=8)
    dx = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    for r in (3, 4, 8):
        y = M.linear(dx, planes, 8, ds, dz, N, r, group, y_mode=M.MATQ_OUT_F32)
        check_close(y.cpu().numpy(), O.linear(xv, codes, s, z, r, group), what=f"r={r}")
