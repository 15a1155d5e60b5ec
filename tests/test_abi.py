"""Host-side checks of the C-ABI library: it loads, exports every entry point the header
declares, answers the layout queries, and rejects bad arguments with the documented
status before touching a GPU (every call here fails validation, so none launches)."""

import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "matq.h")


@pytest.fixture(scope="module")
def M():
    from nested_bit_weight_msb_b200 import build
    build.build()
    from nested_bit_weight_msb_b200 import matq
    return matq


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(matq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("matq_pack", "matq_slice", "matq_slice_copy", "matq_linear", "matq_linear_workspace",
              "matq_packed_bytes", "matq_strerror"):
        assert n in names


def test_every_declared_symbol_is_exported(M):
    import ctypes
    lib = ctypes.CDLL(M.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(declared_functions()) == set(M.EXPORTED)


def test_layout_queries(M):
    assert [M.matq_plane_count(r) for r in (2, 3, 4, 6, 8)] == [1, 2, 3, 4, 5]
    assert M.matq_plane_count(5) == 0 and M.matq_plane_count(1) == 0
    for N, K in [(1024, 1024), (14336, 4096), (4096, 14336), (3584, 14336), (17, 256), (1, 512)]:
        npad = (N + 15) // 16 * 16
        for r in (2, 3, 4, 6, 8):
            assert M.matq_packed_bytes(N, K, r) == npad * K * r // 8
    # exactly r bits per weight on the benchmark shapes
    assert M.matq_packed_bytes(14336, 4096, 2) == 14336 * 4096 * 2 // 8
    assert M.matq_packed_bytes(1024, 1000, 4) == 0          # K not a multiple of 256
    assert M.matq_packed_bytes(0, 1024, 4) == 0
    assert M.matq_packed_bytes(16, 1024, 5) == 0
    assert M.matq_version() >= 100
    assert M.matq_strerror(M.MATQ_ETRUNC).decode().startswith("pack holds")


def test_workspace_query(M):
    assert M.matq_linear_workspace(1, 4096, 14336, 128) > 0
    assert M.matq_linear_workspace(1, 4096, 14336, 128) % 256 == 0
    assert M.matq_linear_workspace(2048, 4096, 14336, 128) >= 2048 * 4096 * 2
    assert M.matq_linear_workspace(1, 4096, 14336, 96) == 0


FAKE = 1 << 20          # non-null, 16-byte aligned, never dereferenced (validation fails first)


def test_pack_rejects(M):
    assert M.matq_pack(FAKE, 16, 1024, 5, FAKE, 1 << 30, None) == M.MATQ_EINVAL_R
    assert M.matq_pack(FAKE, 16, 1000, 4, FAKE, 1 << 30, None) == M.MATQ_EINVAL_SHAPE
    assert M.matq_pack(FAKE, 0, 1024, 4, FAKE, 1 << 30, None) == M.MATQ_EINVAL_SHAPE
    assert M.matq_pack(None, 16, 1024, 4, FAKE, 1 << 30, None) == M.MATQ_ENULL
    assert M.matq_pack(FAKE + 8, 16, 1024, 4, FAKE, 1 << 30, None) == M.MATQ_EALIGN
    assert M.matq_pack(FAKE, 16, 1024, 4, FAKE, 16 * 1024 * 4 // 8 - 1, None) == M.MATQ_ESIZE


def test_slice_rejects(M):
    assert M.matq_slice(FAKE, 16, 1024, 4, 6, FAKE, None) == M.MATQ_ETRUNC
    assert M.matq_slice(FAKE, 16, 1024, 4, 5, FAKE, None) == M.MATQ_EINVAL_R
    assert M.matq_slice(FAKE, 16, 1024, 8, 4, None, None) == M.MATQ_ENULL
    assert M.matq_slice_copy(FAKE, 16, 1024, 8, 4, FAKE, 16 * 1024 * 4 // 8 - 16, None) == M.MATQ_ESIZE
    assert M.matq_slice_copy(FAKE, 16, 1024, 2, 4, FAKE, 1 << 20, None) == M.MATQ_ETRUNC


def test_linear_rejects(M):
    ws = 1 << 30

    def call(**kw):
        a = dict(x=FAKE, M=1, K=1024, planes=FAKE, r_keep=8, scales=FAKE, zeros=FAKE, N=64, r=4, group=128,
                 y=FAKE, y_mode=0, ws=FAKE, ws_bytes=ws)
        a.update(kw)
        return M.matq_linear(a["x"], a["M"], a["K"], a["planes"], a["r_keep"], a["scales"], a["zeros"], a["N"],
                             a["r"], a["group"], a["y"], a["y_mode"], a["ws"], a["ws_bytes"], None)

    assert call(r=5) == M.MATQ_EINVAL_R
    assert call(r=8, r_keep=4) == M.MATQ_ETRUNC
    assert call(M=0) == M.MATQ_EINVAL_SHAPE
    assert call(K=1000) == M.MATQ_EINVAL_SHAPE
    assert call(N=0) == M.MATQ_EINVAL_SHAPE
    assert call(group=32) == M.MATQ_EINVAL_GROUP
    assert call(y_mode=4) == M.MATQ_EDTYPE
    assert call(y_mode=-1) == M.MATQ_EDTYPE
    assert call(y_mode=M.MATQ_OUT_SILU_GATED, N=63) == M.MATQ_EINVAL_SHAPE
    assert call(x=None) == M.MATQ_ENULL
    assert call(zeros=FAKE + 4) == M.MATQ_EALIGN
    assert call(ws_bytes=16) == M.MATQ_ESIZE


def test_workspace_init_rejects(M):
    assert M.matq_workspace_init(None, 1 << 20, None) == M.MATQ_ENULL
    assert M.matq_workspace_init(FAKE + 4, 1 << 20, None) == M.MATQ_EALIGN
    assert M.matq_workspace_init(FAKE, 16, None) == M.MATQ_ESIZE
    import ctypes
    assert M.matq_workspace_status(None, ctypes.byref(ctypes.c_int(0))) == M.MATQ_ENULL


def test_glue_rejects(M):
    assert M.matq_rmsnorm(FAKE, 0, 16, 1e-5, FAKE, None) == M.MATQ_EINVAL_SHAPE
    assert M.matq_rmsnorm(None, 1, 16, 1e-5, FAKE, None) == M.MATQ_ENULL
    assert M.matq_silu_mul(FAKE, FAKE + 2, 1, 16, FAKE, None) == M.MATQ_EALIGN
    assert M.matq_silu_mul_gu(FAKE, 0, 16, FAKE, None) == M.MATQ_EINVAL_SHAPE
    assert M.matq_silu_mul_gu(FAKE, 1, 0, FAKE, None) == M.MATQ_EINVAL_SHAPE
    assert M.matq_silu_mul_gu(None, 1, 16, FAKE, None) == M.MATQ_ENULL
    assert M.matq_silu_mul_gu(FAKE + 2, 1, 16, FAKE, None) == M.MATQ_EALIGN


def test_binding_rejects_host_and_strided_tensors(M):
    """The tensor helpers refuse what the C ABI cannot detect itself (before any CUDA call):
    host memory, which a kernel would fault on, and wrong element types."""
    import torch
    x = torch.zeros((1, 256), dtype=torch.bfloat16)
    planes = torch.zeros(4096, dtype=torch.uint8)
    s = torch.zeros((16, 2), dtype=torch.int16)
    z = torch.zeros((16, 2), dtype=torch.uint8)
    y = torch.zeros((1, 16), dtype=torch.bfloat16)
    ws = torch.zeros(1 << 20, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        M.linear(x, planes, 8, s, z, 16, 4, 128, y=y, workspace=ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        M.pack(torch.zeros((16, 256), dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        M.silu_mul_gu(torch.zeros((1, 32), dtype=torch.bfloat16), out=torch.zeros((1, 16), dtype=torch.bfloat16))


def test_choose_codes_rejects(M):
    import ctypes

    def call(N=4, K=128, group=64, widths=(3, 4, 8), lams=(1, 1, 1), mode=0, w=FAKE, s=FAKE, z=FAKE, out=FAKE,
             n=None):
        rw = (ctypes.c_int * max(1, len(widths)))(*widths) if widths is not None else None
        lw = (ctypes.c_float * max(1, len(lams)))(*lams) if lams is not None else None
        nw = len(widths) if (n is None and widths is not None) else (n or 0)
        return M.matq_choose_codes(w, N, K, s, z, group, nw, rw, lw, mode, out, None)

    assert call(group=32) == M.MATQ_EINVAL_GROUP
    assert call(N=0) == M.MATQ_EINVAL_SHAPE
    assert call(K=96) == M.MATQ_EINVAL_SHAPE
    assert call(K=32) == M.MATQ_EINVAL_SHAPE
    assert call(widths=None) == M.MATQ_ENULL
    assert call(lams=None) == M.MATQ_ENULL
    assert call(widths=(), lams=(), n=0) == M.MATQ_EINVAL_R
    assert call(widths=(2, 3, 4, 6, 8, 8), lams=(1,) * 6) == M.MATQ_EINVAL_R
    assert call(widths=(8, 4), lams=(1, 1)) == M.MATQ_EINVAL_R
    assert call(widths=(4, 4), lams=(1, 1)) == M.MATQ_EINVAL_R
    assert call(widths=(5,), lams=(1,)) == M.MATQ_EINVAL_R
    assert call(lams=(1, -1, 1)) == M.MATQ_EINVAL_ARG
    assert call(lams=(1, float("nan"), 1)) == M.MATQ_EINVAL_ARG
    assert call(lams=(1, float("inf"), 1)) == M.MATQ_EINVAL_ARG
    assert call(mode=2) == M.MATQ_EINVAL_ARG
    assert call(w=None) == M.MATQ_ENULL
    assert call(out=None) == M.MATQ_ENULL
    assert call(w=FAKE + 4) == M.MATQ_EALIGN
    assert call(out=FAKE + 1) == M.MATQ_EALIGN
    assert call(z=FAKE + 8) == M.MATQ_EALIGN
    assert "lambda" in M.matq_strerror(M.MATQ_EINVAL_ARG).decode()
    import torch
    with pytest.raises(ValueError, match="CUDA tensor"):
        M.choose_codes(torch.zeros((4, 128)), torch.zeros((4, 2), dtype=torch.float16),
                       torch.zeros((4, 2), dtype=torch.uint8), 64)


def test_rounded_slicing_queries_and_rejects(M):
    """Strict / Extra-Precision MatQuant entry points: sizes, and every argument error caught on
    the host (nothing launches)."""
    assert M.matq_round_scratch_bytes(28672, 4096) == 28672 * 16 * 4
    assert M.matq_round_scratch_bytes(17, 512) == 256            # 17 * 2 * 4 bytes, rounded up to 256
    assert M.matq_round_scratch_bytes(16, 1000) == 0
    base = M.matq_linear_workspace(16, 4096, 28672, 128)
    assert M.matq_linear_rounded_workspace(16, 4096, 28672, 128) >= base + 16 * 28672 * 4
    assert M.matq_linear_rounded_workspace(64, 4096, 28672, 128) == M.matq_linear_workspace(64, 4096, 28672, 128)
    big = 1 << 30

    def ext(**kw):
        a = dict(planes=FAKE, N=16, K=1024, r_keep=8, r=2, levels=FAKE, lb=big, row_ptr=FAKE, cols=FAKE,
                 cap=big, scratch=FAKE, sb=big)
        a.update(kw)
        return M.matq_round_extract(a["planes"], a["N"], a["K"], a["r_keep"], a["r"], a["levels"], a["lb"],
                                    a["row_ptr"], a["cols"], a["cap"], a["scratch"], a["sb"], None)

    assert ext(r=5) == M.MATQ_EINVAL_R
    # rounding to width r reads code bit 7 - r: widths 3, 4, 6, 8 hold it for r = 2, 3, 4, 6
    for r, need in ((2, 3), (3, 4), (4, 6), (6, 8)):
        smaller = {3: 2, 4: 3, 6: 4, 8: 6}[need]
        assert ext(r=r, r_keep=smaller) == M.MATQ_ETRUNC
    assert ext(K=1000) == M.MATQ_EINVAL_SHAPE
    assert ext(K=65536 + 256) == M.MATQ_EINVAL_SHAPE             # inputs are listed as uint16
    assert ext(N=1 << 20, K=4096) == M.MATQ_EINVAL_SHAPE         # N * K >= 2^31
    assert ext(row_ptr=None) == M.MATQ_ENULL
    assert ext(scratch=None) == M.MATQ_ENULL
    assert ext(cols=FAKE + 2) == M.MATQ_EALIGN
    assert ext(lb=16 * 1024 * 2 // 8 - 1) == M.MATQ_ESIZE
    assert ext(sb=4) == M.MATQ_ESIZE

    def lin(**kw):
        a = dict(x=FAKE, M=1, K=1024, levels=FAKE, r=2, scales=FAKE, zeros=FAKE, N=64, group=128, row_ptr=FAKE,
                 cols=FAKE, y=FAKE, y_mode=0, ws=FAKE, wsb=big)
        a.update(kw)
        return M.matq_linear_rounded(a["x"], a["M"], a["K"], a["levels"], a["r"], a["scales"], a["zeros"], a["N"],
                                     a["group"], a["row_ptr"], a["cols"], a["y"], a["y_mode"], a["ws"], a["wsb"],
                                     None)

    assert lin(r=5) == M.MATQ_EINVAL_R
    assert lin(cols=None) == M.MATQ_ENULL
    assert lin(row_ptr=None) == M.MATQ_ENULL
    assert lin(K=1000) == M.MATQ_EINVAL_SHAPE
    assert lin(group=32) == M.MATQ_EINVAL_GROUP
    assert lin(y_mode=4) == M.MATQ_EDTYPE
    assert lin(y_mode=M.MATQ_OUT_SILU_GATED, N=63) == M.MATQ_EINVAL_SHAPE
    assert lin(row_ptr=FAKE + 4) == M.MATQ_EALIGN
    assert lin(wsb=M.matq_linear_workspace(1, 1024, 64, 128)) == M.MATQ_ESIZE  # no room for the fp32 copy
    # without a list (strict MatQuant) the plain linear's checks and workspace apply
    assert lin(row_ptr=None, cols=None, wsb=16) == M.MATQ_ESIZE
    assert lin(row_ptr=None, cols=None, x=None) == M.MATQ_ENULL
