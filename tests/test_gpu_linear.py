"""GPU parity of matq_linear against the fp64 oracle.

Decode path (M <= 16) and prefill path (M > 16), all widths, both group sizes, every
output mode; small shapes that span several tiles with ragged tails compared element by
element; the benchmark shapes compared on sampled output rows (the oracle computes those
rows one by one).  Bar: |y - ref| <= 1e-2 (|ref| + 1) elementwise and relative Frobenius
error <= 2e-3 (tests/helpers.py).
"""

import numpy as np
import pytest

import oracle as O
from helpers import check_close, problem, to_device
from nested_bit_weight_msb_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nested_bit_weight_msb_b200 import matq
    return matq


def run(M, q, s, z, xb, r, group, r_keep=8, y_mode=0):
    import torch
    dq, ds, dz, dx = to_device(q, s, z, xb)
    planes = M.pack(dq, r_keep=r_keep)
    y = M.linear(dx, planes, r_keep, ds, dz, q.shape[0], r, group, y_mode=y_mode)
    torch.cuda.synchronize()
    return y.float().cpu().numpy()


# ---- decode path -------------------------------------------------------------------------

@pytest.mark.parametrize("r", O.WIDTHS)
def test_single_linear_1024(M, r):
    """K = N = 1024, group 128, M = 1, seed 0 (the single-linear-layer workload)."""
    q, s, z, xb, xv = problem(1, 1024, 1024, 128, seed=0)
    ref = O.linear(xv, q, s, z, r, 128)
    for mode in (M.MATQ_OUT_BF16, M.MATQ_OUT_F32):
        y = run(M, q, s, z, xb, r, 128, y_mode=mode)
        check_close(y, ref, what=f"r={r} mode={mode}")


@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("Mt", [1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16])
def test_decode_small_sweep(M, Mt, group):
    """Several row tiles with a ragged last tile, several chunks, every width."""
    N, K = 83, 768
    q, s, z, xb, xv = problem(Mt, N, K, group, seed=Mt + group)
    dq, ds, dz, dx = to_device(q, s, z, xb)
    planes = M.pack(dq, r_keep=8)
    for r in O.WIDTHS:
        ref = O.linear(xv, q, s, z, r, group)
        y = M.linear(dx, planes, 8, ds, dz, N, r, group, y_mode=M.MATQ_OUT_F32).cpu().numpy()
        check_close(y, ref, what=f"M={Mt} g={group} r={r}")


def test_decode_accumulate_mode(M):
    import torch
    N, K, Mt = 130, 512, 4
    q, s, z, xb, xv = problem(Mt, N, K, 64, seed=5)
    dq, ds, dz, dx = to_device(q, s, z, xb)
    planes = M.pack(dq, r_keep=8)
    base = np.random.default_rng(1).standard_normal((Mt, N)).astype(np.float32)
    y = torch.from_numpy(base.copy()).cuda()
    M.linear(dx, planes, 8, ds, dz, N, 3, 64, y=y, y_mode=M.MATQ_OUT_F32_ACCUM)
    check_close(y.cpu().numpy(), base + O.linear(xv, q, s, z, 3, 64), what="accumulate")


@pytest.mark.parametrize("r", O.WIDTHS)
def test_truncated_pack_gives_identical_output(M, r):
    """Mode A (only the r-bit prefix resident) and mode B (all 8 bits, r per call) read the
    same bits, so the outputs are bitwise equal."""
    import torch
    N, K, Mt = 64, 1024, 3
    q, s, z, xb, xv = problem(Mt, N, K, 128, seed=r)
    dq, ds, dz, dx = to_device(q, s, z, xb)
    full = M.pack(dq, r_keep=8)
    trunc = M.slice_copy(full, N, K, 8, r)
    a = M.linear(dx, full, 8, ds, dz, N, r, 128, y_mode=M.MATQ_OUT_F32)
    b = M.linear(dx, trunc, r, ds, dz, N, r, 128, y_mode=M.MATQ_OUT_F32)
    assert torch.equal(a, b)


def test_decode_closed_forms(M):
    import torch
    N, K = 32, 512
    # codes equal to their zero point at r = 8: W_hat = 0, so y = 0
    rng = np.random.default_rng(3)
    z = rng.integers(0, 256, (N, K // 128), dtype=np.uint8)
    q = np.repeat(z, 128, axis=1)
    s = rng.uniform(1e-3, 1e-2, (N, K // 128)).astype(np.float16)
    xb, xv = synth.bf16_round(rng.standard_normal((2, K)).astype(np.float32))
    y = run(M, q, s, z, xb, 8, 128, y_mode=M.MATQ_OUT_F32)
    # the exact result is 0; fp32 rounding of the cancelling terms s*z*sum(x) stays tiny
    scale = float((s.astype(np.float64) * z).max()) * float(np.abs(xv).sum())
    assert np.max(np.abs(y)) <= 1e-5 * scale
    # one-hot activations pick a column of W_hat
    q = rng.integers(0, 256, (N, K), dtype=np.uint8)
    for k in (0, 7, 8, 15, 200, 511):
        e = np.zeros((1, K), dtype=np.float32)
        e[0, k] = 1.0
        eb, ev = synth.bf16_round(e)
        for r in O.WIDTHS:
            y = run(M, q, s, z, eb, r, 128, y_mode=M.MATQ_OUT_F32)
            col = O.dequant(q, s, z, r, 128)[:, k]
            assert np.allclose(y[0], col, rtol=1e-5, atol=1e-6), (k, r)


def test_decode_outlier_activations(M):
    N, K = 256, 4096
    q, s, z, xb, xv = problem(16, N, K, 128, seed=9, outlier_frac=0.01)
    for r in O.WIDTHS:
        check_close(run(M, q, s, z, xb, r, 128), O.linear(xv, q, s, z, r, 128), what=f"r={r}")


@pytest.mark.parametrize("shape,group", [((14336, 4096), 128), ((4096, 14336), 128),
                                         ((14336, 3584), 64), ((3584, 14336), 64)])
def test_decode_full_size_sampled(M, shape, group):
    """Benchmark FFN shapes (8B gate/up and down, g=128; 9B gate/up and down, g=64) at the
    decode batch sizes, every width, in the same launch configuration the bench times;
    64 sampled output rows are checked against the oracle."""
    import torch
    N, K = shape
    q, s, z = synth.parent_weights(N, K, group, seed=0, proj="gate" if N > K else "down")
    dq = torch.from_numpy(q).cuda()
    ds = torch.from_numpy(s.view(np.int16)).cuda()
    dz = torch.from_numpy(z).cuda()
    planes = M.pack(dq, r_keep=8)
    rows = np.sort(np.random.default_rng(N).choice(N, 64, replace=False))
    for Mt in (1, 4, 8, 16):
        xb, xv = synth.activations(Mt, K, seed=0)
        dx = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
        for r in O.WIDTHS:
            y = M.linear(dx, planes, 8, ds, dz, N, r, group).float().cpu().numpy()
            ref = O.linear(xv, q[rows], s[rows], z[rows], r, group)
            check_close(y[:, rows], ref, what=f"{shape} M={Mt} r={r}")


# ---- prefill path ------------------------------------------------------------------------

def _device_status(M, ws, Mt, K, N, group):
    """Device-side status words in the workspace header (0 = every call completed normally)."""
    return M.workspace_status(ws)


@pytest.mark.parametrize("Mt,N,K,group", [(17, 128, 256, 128), (31, 300, 512, 128), (64, 200, 512, 64),
                                          (100, 384, 768, 128), (129, 130, 512, 64), (300, 256, 1024, 128)])
def test_prefill_small(M, Mt, N, K, group):
    """Tiles of every token-tile size (64, 128, 256), ragged tokens and rows, both groups."""
    import torch
    q, s, z, xb, xv = problem(Mt, N, K, group, seed=Mt * 7 + N)
    dq, ds, dz, dx = to_device(q, s, z, xb)
    planes = M.pack(dq, r_keep=8)
    ws = M.workspace(Mt, K, N, group)
    for r in O.WIDTHS:
        ref = O.linear(xv, q, s, z, r, group)
        for mode in (M.MATQ_OUT_BF16, M.MATQ_OUT_F32):
            y = M.linear(dx, planes, 8, ds, dz, N, r, group, y_mode=mode, workspace=ws).float().cpu().numpy()
            assert _device_status(M, ws, Mt, K, N, group) == 0
            check_close(y, ref, what=f"M={Mt} N={N} K={K} g={group} r={r} mode={mode}")


def test_prefill_accumulate_and_mode_a(M):
    import torch
    Mt, N, K = 40, 256, 512
    q, s, z, xb, xv = problem(Mt, N, K, 128, seed=21)
    dq, ds, dz, dx = to_device(q, s, z, xb)
    full = M.pack(dq, r_keep=8)
    base = np.random.default_rng(2).standard_normal((Mt, N)).astype(np.float32)
    y = torch.from_numpy(base.copy()).cuda()
    M.linear(dx, full, 8, ds, dz, N, 4, 128, y=y, y_mode=M.MATQ_OUT_F32_ACCUM)
    check_close(y.cpu().numpy(), base + O.linear(xv, q, s, z, 4, 128), what="accumulate")
    for r in O.WIDTHS:
        trunc = M.slice_copy(full, N, K, 8, r)
        a = M.linear(dx, full, 8, ds, dz, N, r, 128, y_mode=M.MATQ_OUT_F32)
        b = M.linear(dx, trunc, r, ds, dz, N, r, 128, y_mode=M.MATQ_OUT_F32)
        assert torch.equal(a, b)


def test_prefill_closed_forms(M):
    N, K, Mt = 128, 512, 32
    rng = np.random.default_rng(4)
    z = rng.integers(0, 256, (N, K // 128), dtype=np.uint8)
    q = np.repeat(z, 128, axis=1)
    s = rng.uniform(1e-3, 1e-2, (N, K // 128)).astype(np.float16)
    xb, xv = synth.bf16_round(rng.standard_normal((Mt, K)).astype(np.float32))
    y = run(M, q, s, z, xb, 8, 128, y_mode=M.MATQ_OUT_F32)
    assert np.all(y == 0.0)          # every weight dequantises to exactly 0 at r = 8


@pytest.mark.parametrize("shape,group,Ms,widths", [
    ((14336, 4096), 128, (2048,), (3, 4, 8)),
    ((4096, 14336), 128, (2048,), (3, 4, 8)),
    ((14336, 3584), 64, (32, 128, 512, 2048), (2, 3, 4, 6, 8)),
    ((3584, 14336), 64, (32, 128, 512, 2048), (2, 3, 4, 6, 8)),
])
def test_prefill_full_size_sampled(M, shape, group, Ms, widths):
    """Benchmark shapes at the prefill batch sizes (8B FFN at M = 2048 with 1% outlier
    channels x20; 9B FFN batch sweep at every width, the down projection through its K-split
    path at M <= 512), in the bench's launch configuration; 48 sampled output rows against the
    oracle."""
    import torch
    N, K = shape
    q, s, z = synth.parent_weights(N, K, group, seed=0, proj="gate" if N > K else "down")
    dq = torch.from_numpy(q).cuda()
    ds = torch.from_numpy(s.view(np.int16)).cuda()
    dz = torch.from_numpy(z).cuda()
    planes = M.pack(dq, r_keep=8)
    rows = np.sort(np.random.default_rng(N + 1).choice(N, 48, replace=False))
    for Mt in Ms:
        xb, xv = synth.activations(Mt, K, seed=0, outlier_frac=0.01 if K == 4096 else 0.0)
        dx = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
        for r in widths:
            y = M.linear(dx, planes, 8, ds, dz, N, r, group).float()[:, torch.from_numpy(rows).cuda()].cpu().numpy()
            ref = O.linear(xv, q[rows], s[rows], z[rows], r, group)
            check_close(y, ref, what=f"{shape} M={Mt} r={r}")


@pytest.mark.parametrize("N,K,Mt", [(4096, 256, 1), (4096, 256, 16), (25600, 512, 4), (25600, 512, 9),
                                    (51200, 256, 1)])
def test_decode_work_split_paths(M, N, K, Mt):
    """Shapes whose work items give every CTA whole row groups (direct stores), and a mix of
    whole and split row groups (split ones combined through the workspace)."""
    import torch
    q, s, z, xb, xv = problem(Mt, N, K, 128, seed=N + Mt)
    dq, ds, dz, dx = to_device(q, s, z, xb)
    planes = M.pack(dq, r_keep=8)
    ws = M.workspace(Mt, K, N, 128)
    rows = np.sort(np.random.default_rng(N).choice(N, 512, replace=False))
    for r in (2, 4, 8):
        ref = O.linear(xv, q[rows], s[rows], z[rows], r, 128)
        y1 = M.linear(dx, planes, 8, ds, dz, N, r, 128, y_mode=M.MATQ_OUT_F32, workspace=ws)
        y2 = M.linear(dx, planes, 8, ds, dz, N, r, 128, y_mode=M.MATQ_OUT_F32, workspace=ws)
        assert torch.equal(y1, y2)        # same workspace reused: counters reset, result bitwise stable
        assert M.workspace_status(ws) == 0
        check_close(y1.cpu().numpy()[:, rows], ref, what=f"N={N} K={K} M={Mt} r={r}")


def _wide_range_x(rng, Mt, K, lo_exp, hi_exp):
    """bf16 activations whose magnitudes are log-uniform over [2^lo_exp, 2^hi_exp], random
    signs, with the extremes present in every row."""
    e = rng.uniform(lo_exp, hi_exp, (Mt, K))
    x = np.sign(rng.standard_normal((Mt, K))) * np.exp2(e)
    x[:, 0] = 2.0 ** lo_exp
    x[:, 1] = -(2.0 ** hi_exp)
    return synth.bf16_round(x.astype(np.float32))


@pytest.mark.parametrize("r", [2, 8])
def test_prefill_serves_the_whole_bf16_range(M, r):
    """Activations from 2^-24 to 2^20 (beyond fp16's 65504): the prefill path divides each token by
    the power of two that keeps it finite in fp16 and multiplies its results back (exact)."""
    import torch
    Mt, N, K, G = 40, 256, 1024, 128
    q, s, z, _, _ = problem(1, N, K, G, seed=31)
    rng = np.random.default_rng(r)
    xb, xv = _wide_range_x(rng, Mt, K, -24, 20)
    xb[5], xv[5] = synth.bf16_round((rng.standard_normal(K) * 0.5).astype(np.float32))   # an ordinary token too
    dq, ds, dz, dx = to_device(q, s, z, xb)
    planes = M.pack(dq, r_keep=8)
    ws = M.workspace(Mt, K, N, G)
    # The prefill path multiplies fp16 weights s * (q_hat - z) (each within 2^-11 of the exact
    # value) by fp16 activations x * 2^-e (exact down to 2^-14, then on the subnormal grid of
    # spacing 2^-24) and accumulates K = 1024 products in fp32 (within 2^-14 of sum |x w|).  With
    # activations up to 2^20 and random signs, outputs that cancel to near zero sit far below the
    # products' magnitude, so the bar adds that arithmetic's own bound to the usual one:
    #   |y - ref| <= 1e-2 (|ref| + 1) + 2^-10 sum_k |x_k w_k| + 2^(e_t - 24) sum_k |w_k|.
    xf = xv.astype(np.float64)
    wd = O.dequant(q, s, z, r, G)
    mag = np.abs(xf) @ np.abs(wd).T
    e_t = np.maximum(0, np.floor(np.log2(np.max(np.abs(xf), axis=1))) - 15)
    arith = 2.0 ** -10 * mag + np.exp2(e_t - 24)[:, None] * np.abs(wd).sum(axis=1)[None, :]
    ref = O.linear(xf, q, s, z, r, G)
    for mode in (M.MATQ_OUT_F32, M.MATQ_OUT_BF16):
        y = M.linear(dx, planes, 8, ds, dz, N, r, G, y_mode=mode, workspace=ws)
        torch.cuda.synchronize()
        assert M.workspace_status(ws) == 0
        yh = y.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(yh))
        err = np.abs(yh - ref)
        bound = 1e-2 * (np.abs(ref) + 1.0) + arith
        assert np.all(err <= bound), f"prefill wide x r={r} mode={mode}: worst {np.max(err / bound):.3g}"
        rel = np.linalg.norm(yh - ref) / np.linalg.norm(ref)
        assert rel <= 2e-3, f"prefill wide x r={r} mode={mode}: relative Frobenius {rel:.3e}"
        # the rows whose activations needed no prescale keep the ordinary bar
        check_close(yh[5:6], ref[5:6], what=f"prefill wide x r={r} mode={mode} ordinary token")


@pytest.mark.parametrize("r", [2, 8])
@pytest.mark.parametrize("Mt", [1, 16])
def test_decode_input_range(M, r, Mt):
    """The decode path's fp16 operands: activations from 2^-24 to just below 2^16 match the oracle
    (values below 2^-14 land on fp16's subnormal grid, far inside the tolerance); one activation
    of magnitude 2^17 raises MATQ_STATUS_XRANGE in the workspace status."""
    import torch
    N, K, G = 4096, 4096, 128
    q, s, z, _, _ = problem(1, N, K, G, seed=32)
    rng = np.random.default_rng(10 * r + Mt)
    xb, xv = _wide_range_x(rng, Mt, K, -24, 15.9)
    dq, ds, dz, dx = to_device(q, s, z, xb)
    planes = M.pack(dq, r_keep=8)
    ws = M.workspace(Mt, K, N, G)
    y = M.linear(dx, planes, 8, ds, dz, N, r, G, y_mode=M.MATQ_OUT_F32, workspace=ws)
    torch.cuda.synchronize()
    assert M.workspace_status(ws) == 0
    rows = np.sort(np.random.default_rng(7).choice(N, 512, replace=False))
    # The decode path multiplies x (fp16, exact down to 2^-14) by the exact operands
    # 1024 + sigma * v, accumulates in fp32 and removes the 1024 bias afterwards, then scales by
    # s * 2^(8-r) / sigma (sigma >= 1).  The bias makes each term up to 1280 * 2^(8-r) * s * |x|
    # large, so an output that cancels to near zero under activations up to 2^16 carries fp32
    # rounding of that size: the bar adds 2^-22 * sum_k 1280 * 2^(8-r) * s_k * |x_k| (and the
    # fp16 subnormal grid, 2^-25 * sum_k |w_k|) to the usual 1e-2 (|ref| + 1).
    xf = xv.astype(np.float64)
    qs, ss, zs = q[rows], s[rows], z[rows]
    ref = O.linear(xf, qs, ss, zs, r, G)
    s_full = np.repeat(ss.astype(np.float64), G, axis=1)
    bias_mag = np.abs(xf) @ (1280.0 * 2 ** (8 - r) * s_full).T
    wd = O.dequant(qs, ss, zs, r, G)
    arith = 2.0 ** -22 * bias_mag + 2.0 ** -25 * np.abs(wd).sum(axis=1)[None, :]
    yh = y.cpu().numpy().astype(np.float64)[:, rows]
    err = np.abs(yh - ref)
    bound = 1e-2 * (np.abs(ref) + 1.0) + arith
    assert np.all(err <= bound), f"decode wide x r={r} M={Mt}: worst {np.max(err / bound):.3g}"
    rel = np.linalg.norm(yh - ref) / np.linalg.norm(ref)
    assert rel <= 2e-3, f"decode wide x r={r} M={Mt}: relative Frobenius {rel:.3e}"
    big = xb.copy()
    big[Mt - 1, K // 3] = synth.bf16_round(np.array([2.0 ** 17], dtype=np.float32))[0][0]
    dbig = torch.from_numpy(big.view(np.int16)).cuda().view(torch.bfloat16)
    M.linear(dbig, planes, 8, ds, dz, N, r, G, y_mode=M.MATQ_OUT_F32, workspace=ws)
    torch.cuda.synchronize()
    assert M.workspace_status(ws) & M.MATQ_STATUS_XRANGE


@pytest.mark.parametrize("Mt,N,K,group", [(40, 512, 4096, 128), (130, 264, 2048, 64), (512, 3584, 14336, 64)])
def test_prefill_k_split(M, Mt, N, K, group):
    """Small matrices leave most SMs without a (row block, token tile): these three shapes have
    4, 3 and 56 such tiles for 148 SMs, so the prefill path splits K (8, 8 and 2 ways) and sums
    the partial results in split order.  Every output mode against the oracle."""
    import torch
    q, s, z, xb, xv = problem(Mt, N, K, group, seed=41, outlier_frac=0.01)
    dq, ds, dz, dx = to_device(q, s, z, xb)
    planes = M.pack(dq, r_keep=8)
    rows = np.arange(N) if N <= 512 else np.sort(np.random.default_rng(3).choice(N, 512, replace=False))
    xf = xv.astype(np.float64)
    ws = M.workspace(Mt, K, N, group)
    for r in (2, 8):
        ref = O.linear(xf, q[rows], s[rows], z[rows], r, group)
        y32 = M.linear(dx, planes, 8, ds, dz, N, r, group, y_mode=M.MATQ_OUT_F32, workspace=ws)
        y32 = y32.cpu().numpy().astype(np.float64)
        check_close(y32[:, rows], ref, what=f"split r={r} M={Mt} N={N}")
        base = np.random.default_rng(r).standard_normal((Mt, N)).astype(np.float32)
        ya = torch.from_numpy(base.copy()).cuda()
        M.linear(dx, planes, 8, ds, dz, N, r, group, y=ya, y_mode=M.MATQ_OUT_F32_ACCUM, workspace=ws)
        check_close(ya.cpu().numpy()[:, rows] - base[:, rows], ref, what=f"split accum r={r}")
        yb = M.linear(dx, planes, 8, ds, dz, N, r, group, y_mode=M.MATQ_OUT_BF16, workspace=ws)
        check_close(yb.float().cpu().numpy()[:, rows], ref, what=f"split bf16 r={r}")
        ga = M.linear(dx, planes, 8, ds, dz, N, r, group, y_mode=M.MATQ_OUT_SILU_GATED, workspace=ws)
        gref = O.gated_product(y32[:, 0::2], y32[:, 1::2])
        err = np.abs(ga.float().cpu().numpy().astype(np.float64) - gref)
        assert np.all(err <= 2.0 ** -8 * np.abs(gref) + 1e-6), f"split gated r={r}"
        assert M.workspace_status(ws) == 0
