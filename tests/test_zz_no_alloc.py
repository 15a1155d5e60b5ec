"""matq_linear_noalloc: the sliced linear layer with libmatq's own fixed scratch.

Collected last (file name) so that it also runs after every other GPU test has used the
library in the same process.  The GPU cases call it twice in a row through the C ABI and
compare each output with matq_linear's (caller workspace) at the parity tolerance.
"""

import numpy as np
import pytest

from helpers import check_close, problem, to_device

FAKE = 1 << 20  # 16-byte aligned, never dereferenced: every call below is rejected first


@pytest.fixture(scope="module")
def M():
    from nested_bit_weight_msb_b200 import matq
    return matq


def _call(M, x=FAKE, Mt=1, K=1024, planes=FAKE, r_keep=8, s=FAKE, z=FAKE, N=64, r=4, group=128,
          y=FAKE, y_mode=0, status=None):
    return M.matq_linear_noalloc(x, Mt, K, planes, r_keep, s, z, N, r, group, y, y_mode, status, None)


def test_noalloc_rejects_before_any_launch(M):
    assert _call(M, r=5) == M.MATQ_EINVAL_R
    assert _call(M, r=8, r_keep=4) == M.MATQ_ETRUNC
    assert _call(M, K=1000) == M.MATQ_EINVAL_SHAPE
    assert _call(M, group=32) == M.MATQ_EINVAL_GROUP
    assert _call(M, y_mode=4) == M.MATQ_EDTYPE
    assert _call(M, y_mode=M.MATQ_OUT_SILU_GATED, N=63) == M.MATQ_EINVAL_SHAPE
    assert _call(M, x=None) == M.MATQ_ENULL
    assert _call(M, y=FAKE + 8) == M.MATQ_EALIGN
    assert _call(M, status=FAKE + 2) == M.MATQ_EALIGN
    # beyond the fixed scratch: the prefill path's fp16 copy of x does not fit
    cap = 8 << 20
    assert M.matq_linear_workspace(2048, 4096, 14336, 128) > cap
    assert _call(M, Mt=2048, K=4096, N=14336) == M.MATQ_ESCRATCH
    assert M.matq_linear_workspace(992, 4096, 64, 128) > cap
    assert _call(M, Mt=992, K=4096) == M.MATQ_ESCRATCH
    assert "matq_linear_noalloc" in M.matq_strerror(M.MATQ_ESCRATCH).decode()


CASES = [
    # (M, N, K, group, r, y_mode)
    (1, 1000, 1024, 128, 2, 0),       # decode, ragged row tile
    (5, 333, 2560, 64, 3, 1),         # decode, odd M, fp32 out
    (16, 4096, 4096, 128, 8, 0),      # decode, rows split between CTAs
    (64, 1000, 1024, 128, 4, 0),      # prefill path within the fixed scratch
    (991, 256, 4096, 128, 6, 1),      # largest M at K = 4096 that fits
]


@pytest.mark.gpu
@pytest.mark.parametrize("Mt,N,K,group,r,y_mode", CASES)
def test_noalloc_matches_linear_twice(M, Mt, N, K, group, r, y_mode):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    q, s, z, xb, _ = problem(Mt, N, K, group, seed=Mt + N)
    dq, ds, dz, dx = to_device(q, s, z, xb)
    planes = M.pack(dq, r_keep=8)
    ref = M.linear(dx, planes, 8, ds, dz, N, r, group, y_mode=y_mode)
    ref = ref.float().cpu().numpy().astype(np.float64)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):
        y = M.linear_noalloc(dx, planes, 8, ds, dz, N, r, group, y_mode=y_mode, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        check_close(y.float().cpu().numpy(), ref, what=f"noalloc call {call}")
        status.fill_(-1)


@pytest.mark.gpu
def test_noalloc_accumulate_and_oversize_on_device(M):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    Mt, N, K, group, r = 3, 700, 1536, 128, 4
    q, s, z, xb, _ = problem(Mt, N, K, group, seed=11)
    dq, ds, dz, dx = to_device(q, s, z, xb)
    planes = M.pack(dq, r_keep=4)
    base = torch.randn(Mt, N, device="cuda")
    ref = base.clone()
    M.linear(dx, planes, 4, ds, dz, N, r, group, y=ref, y_mode=M.MATQ_OUT_F32_ACCUM)
    ref2 = ref.clone()
    M.linear(dx, planes, 4, ds, dz, N, r, group, y=ref2, y_mode=M.MATQ_OUT_F32_ACCUM)
    y = base.clone()
    M.linear_noalloc(dx, planes, 4, ds, dz, N, r, group, y=y, y_mode=M.MATQ_OUT_F32_ACCUM)
    check_close(y.cpu().numpy(), ref.cpu().numpy(), what="accumulate call 0")
    M.linear_noalloc(dx, planes, 4, ds, dz, N, r, group, y=y, y_mode=M.MATQ_OUT_F32_ACCUM)
    check_close(y.cpu().numpy(), ref2.cpu().numpy(), what="accumulate call 1")
    # too large for the fixed scratch: rejected, nothing launched, y untouched
    Mb = 4096
    assert M.matq_linear_workspace(Mb, K, N, group) > (8 << 20)
    big = torch.zeros(Mb, K, dtype=torch.bfloat16, device="cuda")
    yb = torch.full((Mb, N), 7.0, device="cuda")
    st = M.matq_linear_noalloc(big.data_ptr(), Mb, K, planes.data_ptr(), 4, ds.data_ptr(), dz.data_ptr(),
                               N, r, group, yb.data_ptr(), M.MATQ_OUT_F32, None, None)
    assert st == M.MATQ_ESCRATCH
    torch.cuda.synchronize()
    assert bool((yb == 7.0).all())
