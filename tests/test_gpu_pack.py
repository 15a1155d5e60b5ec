"""GPU tests of the one-time pack and of slicing (bit-exact).

The expected prefixes come from the oracle (p = q >> (8 - r)); the expected pack bytes
come from a NumPy model of the plane layout written from its description in
include/matq.h (so the documentation is checked too).  Nothing expected is produced by
the CUDA library.
"""

import numpy as np
import pytest

import oracle as O
from nested_bit_weight_msb_b200 import synth

pytestmark = pytest.mark.gpu

SHAPES = [(16, 256), (1, 256), (17, 512), (100, 768), (1000, 1024), (64, 2304)]


@pytest.fixture(scope="module")
def M():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nested_bit_weight_msb_b200 import matq
    return matq


def edge_codes(N, K, seed):
    q = synth.random_codes((N, K), seed=seed)
    edges = np.array([0, 255, 0x55, 0xAA, 1, 2, 4, 8, 16, 32, 64, 128, 0x7F, 0x80, 234], dtype=np.uint8)
    flat = q.reshape(-1)
    flat[: min(flat.size, 4 * edges.size)] = np.resize(edges, min(flat.size, 4 * edges.size))
    return q


from layout_model import layout_model  # noqa: E402  (NumPy model of the documented layout)


# --- tests ----------------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", SHAPES)
def test_pack_matches_documented_layout(M, N, K):
    import torch
    q = edge_codes(N, K, seed=N + K)
    planes = M.pack(torch.from_numpy(q).cuda(), r_keep=8)
    assert planes.numel() == M.matq_packed_bytes(N, K, 8)
    assert np.array_equal(planes.cpu().numpy(), layout_model(q, 8))


@pytest.mark.parametrize("N,K", SHAPES)
def test_slice_roundtrip_is_exact(M, N, K):
    import torch
    q = edge_codes(N, K, seed=3 * N + K)
    dq = torch.from_numpy(q).cuda()
    for r_keep in (8, 4):
        planes = M.pack(dq, r_keep=r_keep)
        for r in O.WIDTHS:
            if r > r_keep:
                continue
            p = M.slice_prefix(planes, N, K, r_keep, r).cpu().numpy()
            assert np.array_equal(p.astype(np.int64), O.prefix(q, r)), (N, K, r_keep, r)


def test_exhaustive_codes_every_width(M):
    import torch
    # all 256 codes in every position class: 16 x 256 tile holding each code 16 times
    q = np.tile(np.arange(256, dtype=np.uint8), (16, 1))
    for i in range(16):
        q[i] = np.roll(q[i], 17 * i)
    planes = M.pack(torch.from_numpy(q).cuda(), r_keep=8)
    for r in O.WIDTHS:
        p = M.slice_prefix(planes, 16, 256, 8, r).cpu().numpy()
        assert np.array_equal(p.astype(np.int64), O.prefix(q, r))


@pytest.mark.parametrize("r", O.WIDTHS)
def test_mode_a_prefix_and_bytes(M, r):
    import torch
    N, K = 100, 1024
    q = edge_codes(N, K, seed=r)
    dq = torch.from_numpy(q).cuda()
    full = M.pack(dq, r_keep=8)
    own = M.pack(dq, r_keep=r)
    nbytes = M.matq_packed_bytes(N, K, r)
    assert own.numel() == nbytes == 112 * K * r // 8
    assert torch.equal(full[:nbytes], own)
    copy = M.slice_copy(full, N, K, 8, r)
    assert torch.equal(copy, own)
    p = M.slice_prefix(copy, N, K, r, r).cpu().numpy()
    assert np.array_equal(p.astype(np.int64), O.prefix(q, r))


@pytest.mark.parametrize("r", [2, 3, 4, 6])
def test_prefix_bytes_ignore_low_bits(M, r):
    """The width-r prefix of a pack depends only on the top r bits of each code."""
    import torch
    N, K = 48, 512
    q = edge_codes(N, K, seed=11)
    rng = np.random.default_rng(r)
    low = rng.integers(0, 1 << (8 - r), size=q.shape)
    q2 = ((q.astype(np.int64) >> (8 - r) << (8 - r)) | low).astype(np.uint8)
    nbytes = M.matq_packed_bytes(N, K, r)
    a = M.pack(torch.from_numpy(q).cuda(), r_keep=8)[:nbytes]
    b = M.pack(torch.from_numpy(q2).cuda(), r_keep=8)[:nbytes]
    assert torch.equal(a, b)
    c = M.pack(torch.from_numpy(q2).cuda(), r_keep=8)
    assert not torch.equal(M.pack(torch.from_numpy(q).cuda(), r_keep=8), c) or np.array_equal(q, q2)


def test_full_size_pack_sampled(M):
    """8B-FFN-shaped gate matrix: pack once, check sampled rows of every width's prefix."""
    import torch
    N, K = 14336, 4096
    q, _, _ = synth.parent_weights(N, K, 128, seed=0)
    planes = M.pack(torch.from_numpy(q).cuda(), r_keep=8)
    assert planes.numel() == N * K
    rows = np.random.default_rng(0).choice(N, 64, replace=False)
    for r in O.WIDTHS:
        p = M.slice_prefix(planes, N, K, 8, r)[torch.from_numpy(rows).cuda()].cpu().numpy()
        assert np.array_equal(p.astype(np.int64), O.prefix(q[rows], r))
