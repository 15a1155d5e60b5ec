"""GPU parity of rounded slicing: strict MatQuant and Extra-Precision MatQuant
("Matryoshka Quantization | Summary" §3.2 and §7 Errata).

The extraction (clamped-level pack + CSR list of the weights whose rounded level is 2^r) is
compared bit for bit with the fp64 oracle's `matquant_round` and `extra_precision`
reconstructions; the linear layer against `oracle.linear` in those modes, on the decode path
(M <= 16: dense call on the levels, then the list correction) and the prefill path (listed
weights patched into the fp16 tiles), every output mode, ragged rows, both group sizes.
"""

import numpy as np
import pytest

import oracle as O
from helpers import check_close, to_device
from nested_bit_weight_msb_b200 import synth

pytestmark = pytest.mark.gpu

ROUNDING_WIDTH = {2: 3, 3: 4, 4: 6, 6: 8, 8: 8}


@pytest.fixture(scope="module")
def M():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nested_bit_weight_msb_b200 import matq
    return matq


def expected_slice(q, r):
    """(clamped levels as bytes, row_ptr, cols) from the oracle's two rounding modes."""
    step = 2 ** (8 - r)
    lc = (O.reconstruct(q, r, mode="matquant_round") / step).astype(np.uint8)
    top = O.reconstruct(q, r, mode="extra_precision") == 256.0
    counts = top.sum(axis=1)
    row_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    cols = np.concatenate([np.nonzero(top[n])[0] for n in range(q.shape[0])]).astype(np.int64)
    return lc, row_ptr, cols


def extract(M, q, r, r_keep):
    import torch
    N, K = q.shape
    planes = M.pack(torch.from_numpy(q).cuda(), r_keep=r_keep)
    return M.round_extract(planes, N, K, r_keep, r)


def crafted_codes(N, K, seed):
    """Uniform codes plus rows built to stress the list: row 3 at 255 over inputs 0..511 (a whole
    slice of listed weights, many windows), row 5 alternating 224 / 223 (the rounding edge of
    width 2), row 7 at 0."""
    q = synth.random_codes((N, K), seed=seed)
    q[3, :512] = 255
    q[5, 0::2] = 224
    q[5, 1::2] = 223
    q[7, :] = 0
    return q


@pytest.mark.parametrize("r", [2, 3, 4, 6, 8])
@pytest.mark.parametrize("keep", ["minimal", "all"])
def test_round_extract_matches_oracle(M, r, keep):
    N, K = 40, 768
    q = crafted_codes(N, K, seed=r)
    r_keep = ROUNDING_WIDTH[r] if keep == "minimal" else 8
    levels, row_ptr, cols = extract(M, q, r, r_keep)
    lc, rp, cl = expected_slice(q, r)
    got_levels = M.slice_prefix(levels, N, K, r, r).cpu().numpy()
    assert np.array_equal(got_levels, lc)
    assert np.array_equal(row_ptr.cpu().numpy().astype(np.int64), rp)
    nnz = int(rp[-1])
    got_cols = cols.cpu().numpy().view(np.uint16)[:nnz].astype(np.int64)
    assert np.array_equal(got_cols, cl)
    if r == 8:
        assert nnz == 0
    else:
        assert np.all(row_ptr.cpu().numpy()[4] - row_ptr.cpu().numpy()[3] >= 512)


def test_round_extract_rejects_a_pack_without_the_rounding_bit(M):
    import torch
    q = synth.random_codes((16, 256), seed=1)
    planes = M.pack(torch.from_numpy(q).cuda(), r_keep=2)
    with pytest.raises(M.MatqError):
        M.round_extract(planes, 16, 256, 2, 2)


def _problem(N, K, G, seed, uniform):
    q, s, z = synth.parent_weights(N, K, G, seed=seed)
    if uniform:
        q = crafted_codes(N, K, seed)
    return q, s, z


@pytest.mark.parametrize("Mt", [1, 3, 8, 16, 40, 300])
@pytest.mark.parametrize("r", [2, 3, 4, 6])
def test_linear_extra_precision(M, Mt, r):
    """Extra-Precision (with the list) and strict MatQuant (without) against the oracle, bf16
    output; ragged rows (N = 264); the list from uniform codes (about 2^-(r+1) of the weights)."""
    import torch
    N, K, G = 264, 1024, 128
    q, s, z = _problem(N, K, G, seed=10 + r, uniform=True)
    levels, row_ptr, cols = extract(M, q, r, 8)
    xb, xv = synth.activations(Mt, K, seed=Mt, outlier_frac=0.01 if Mt > 16 else 0.0)
    _, ds, dz, dx = to_device(q, s, z, xb)
    xf = xv.astype(np.float64)
    y = M.linear_rounded(dx, levels, r, ds, dz, N, G, row_ptr=row_ptr, cols=cols)
    check_close(y.float().cpu().numpy(), O.linear(xf, q, s, z, r, G, mode="extra_precision"),
                what=f"extra precision M={Mt} r={r}")
    y = M.linear_rounded(dx, levels, r, ds, dz, N, G)
    check_close(y.float().cpu().numpy(), O.linear(xf, q, s, z, r, G, mode="matquant_round"),
                what=f"strict MatQuant M={Mt} r={r}")


@pytest.mark.parametrize("Mt", [1, 16, 40])
@pytest.mark.parametrize("mode", ["f32", "accum", "gated"])
@pytest.mark.parametrize("group", [64, 128])
def test_linear_extra_precision_output_modes(M, Mt, mode, group):
    import torch
    N, K, r = 256, 768, 2
    q, s, z = _problem(N, K, group, seed=20, uniform=True)
    levels, row_ptr, cols = extract(M, q, r, 3)
    xb, xv = synth.activations(Mt, K, seed=3)
    _, ds, dz, dx = to_device(q, s, z, xb)
    xf = xv.astype(np.float64)
    ref = O.linear(xf, q, s, z, r, group, mode="extra_precision")
    if mode == "f32":
        y = M.linear_rounded(dx, levels, r, ds, dz, N, group, row_ptr, cols, y_mode=M.MATQ_OUT_F32)
        check_close(y.cpu().numpy(), ref, what=f"f32 M={Mt} g={group}")
    elif mode == "accum":
        base = np.random.default_rng(5).standard_normal((Mt, N)).astype(np.float32)
        y = torch.from_numpy(base.copy()).cuda()
        M.linear_rounded(dx, levels, r, ds, dz, N, group, row_ptr, cols, y=y, y_mode=M.MATQ_OUT_F32_ACCUM)
        check_close(y.cpu().numpy() - base, ref, what=f"accum M={Mt} g={group}")
    else:
        a = M.linear_rounded(dx, levels, r, ds, dz, N, group, row_ptr, cols, y_mode=M.MATQ_OUT_SILU_GATED)
        check_close(a.float().cpu().numpy(), O.gated_product(ref[:, 0::2], ref[:, 1::2]),
                    what=f"gated M={Mt} g={group}")


@pytest.mark.parametrize("Mt", [1, 16, 512])
def test_extra_precision_8b_gate_up_sampled(M, Mt):
    """The 8B gate+up matrix (row-interleaved [28672, 4096], group 128) at r = 2 from the seeded
    weights, fp32 output, 512 sampled rows against the oracle; the gated output on every column
    equals the fp64 gated product of those fp32 results up to its bf16 rounding."""
    import torch
    D, F, G, r = 4096, 14336, 128, 2
    host = {nm: synth.parent_weights(F, D, G, seed=0, proj=nm) for nm in ("gate", "up")}
    q, s, z = (np.stack([host["gate"][i], host["up"][i]], axis=1).reshape((2 * F,) + host["gate"][i].shape[1:])
               for i in range(3))
    levels, row_ptr, cols = extract(M, q, r, 8)
    nnz = int(row_ptr[-1].item())
    assert 0 < nnz < q.size // 8
    xb, xv = synth.activations(Mt, D, seed=0, outlier_frac=0.01 if Mt > 16 else 0.0)
    _, ds, dz, dx = to_device(q, s, z, xb)
    y32 = M.linear_rounded(dx, levels, r, ds, dz, 2 * F, G, row_ptr, cols, y_mode=M.MATQ_OUT_F32)
    y32 = y32.cpu().numpy().astype(np.float64)
    rows = np.sort(np.random.default_rng(Mt).choice(2 * F, 512, replace=False))
    check_close(y32[:, rows], O.linear(xv.astype(np.float64), q[rows], s[rows], z[rows], r, G,
                                       mode="extra_precision"), what=f"8B gate+up M={Mt}")
    a = M.linear_rounded(dx, levels, r, ds, dz, 2 * F, G, row_ptr, cols, y_mode=M.MATQ_OUT_SILU_GATED)
    ref = O.gated_product(y32[:, 0::2], y32[:, 1::2])
    err = np.abs(a.float().cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-6)


def test_extra_precision_prefill_k_split(M):
    """A K-split prefill call (N = 264: three 128-row blocks, one token tile, so K = 4096 is
    split 8 ways) starts each split's list cursor past the split's first input (a binary search
    in the row's list)."""
    N, K, G, r, Mt = 264, 4096, 128, 2, 40
    q, s, z = _problem(N, K, G, seed=33, uniform=True)
    levels, row_ptr, cols = extract(M, q, r, 3)
    xb, xv = synth.activations(Mt, K, seed=2)
    _, ds, dz, dx = to_device(q, s, z, xb)
    y = M.linear_rounded(dx, levels, r, ds, dz, N, G, row_ptr, cols, y_mode=M.MATQ_OUT_F32)
    check_close(y.cpu().numpy(), O.linear(xv.astype(np.float64), q, s, z, r, G, mode="extra_precision"),
                what="extra precision K split")


@pytest.mark.parametrize("Mt", [8, 16])
@pytest.mark.parametrize("mode", ["bf16", "gated"])
def test_extra_precision_long_k_windows(M, Mt, mode):
    """A long input range (K = 14336, the 8B down projection's) at 8 and 16 tokens: the
    correction stages the activations in two and three windows of inputs and walks the list once
    per window; the decode path's dense part splits each row group across many CTAs."""
    N, K, G, r = 264, 14336, 128, 2
    q, s, z = _problem(N, K, G, seed=44, uniform=True)
    levels, row_ptr, cols = extract(M, q, r, 3)
    xb, xv = synth.activations(Mt, K, seed=6)
    _, ds, dz, dx = to_device(q, s, z, xb)
    ref = O.linear(xv.astype(np.float64), q, s, z, r, G, mode="extra_precision")
    if mode == "bf16":
        y = M.linear_rounded(dx, levels, r, ds, dz, N, G, row_ptr, cols)
        check_close(y.float().cpu().numpy(), ref, what=f"long K M={Mt}")
    else:
        a = M.linear_rounded(dx, levels, r, ds, dz, N, G, row_ptr, cols, y_mode=M.MATQ_OUT_SILU_GATED)
        check_close(a.float().cpu().numpy(), O.gated_product(ref[:, 0::2], ref[:, 1::2]),
                    what=f"long K gated M={Mt}")
