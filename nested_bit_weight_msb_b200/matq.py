"""ctypes binding of libmatq (C ABI declared in include/matq.h).

Argument marshalling only: every step of the sliced linear layer runs in libmatq's CUDA
kernels.  The functions named like the C entry points take raw pointers (ints) and sizes;
the helpers below them take torch tensors (used for device memory and streams only) and
raise ``MatqError`` on a non-zero status.  There is no CPU fallback: importing this module
fails loudly when the shared library is missing.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmatq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libmatq.so not found at {LIB_PATH}; build it with "
        "`python -m nested_bit_weight_msb_b200.build` (needs nvcc)"
    )

_lib = ctypes.CDLL(LIB_PATH)

# status codes and output modes (mirror include/matq.h)
MATQ_OK = 0
MATQ_EINVAL_R = -1
MATQ_EINVAL_SHAPE = -2
MATQ_EINVAL_GROUP = -3
MATQ_EALIGN = -4
MATQ_ENULL = -5
MATQ_ETRUNC = -6
MATQ_ECUDA = -7
MATQ_ESIZE = -8
MATQ_EDTYPE = -9
MATQ_EDEVICE = -10
MATQ_ESCRATCH = -11
MATQ_EINVAL_ARG = -12
MATQ_OUT_BF16 = 0
MATQ_OUT_F32 = 1
MATQ_OUT_F32_ACCUM = 2
MATQ_OUT_SILU_GATED = 3
MATQ_SLICE_TRUE_PREFIX = 0
MATQ_SLICE_TRUNCATE = 1
MATQ_STATUS_SELFTEST = 0x100
MATQ_STATUS_XRANGE = 0x200

WIDTHS = (2, 3, 4, 6, 8)
DECODE_MAX_M = 16

_c_int, _c_size, _c_vp, _c_float = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float

_SIGNATURES = {
    "matq_version": (_c_int, []),
    "matq_strerror": (ctypes.c_char_p, [_c_int]),
    "matq_last_cuda_error": (_c_int, []),
    "matq_plane_count": (_c_int, [_c_int]),
    "matq_packed_bytes": (_c_size, [_c_int, _c_int, _c_int]),
    "matq_pack": (_c_int, [_c_vp, _c_int, _c_int, _c_int, _c_vp, _c_size, _c_vp]),
    "matq_slice": (_c_int, [_c_vp, _c_int, _c_int, _c_int, _c_int, _c_vp, _c_vp]),
    "matq_slice_copy": (_c_int, [_c_vp, _c_int, _c_int, _c_int, _c_int, _c_vp, _c_size, _c_vp]),
    "matq_linear_workspace": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "matq_workspace_init": (_c_int, [_c_vp, _c_size, _c_vp]),
    "matq_workspace_status": (_c_int, [_c_vp, ctypes.POINTER(_c_int)]),
    "matq_selftest_timeout": (_c_int, [_c_vp, _c_size, _c_vp]),
    "matq_linear": (_c_int, [_c_vp, _c_int, _c_int, _c_vp, _c_int, _c_vp, _c_vp, _c_int, _c_int, _c_int,
                             _c_vp, _c_int, _c_vp, _c_size, _c_vp]),
    "matq_round_scratch_bytes": (_c_size, [_c_int, _c_int]),
    "matq_round_extract": (_c_int, [_c_vp, _c_int, _c_int, _c_int, _c_int, _c_vp, _c_size, _c_vp, _c_vp, _c_size,
                                    _c_vp, _c_size, _c_vp]),
    "matq_linear_rounded_workspace": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "matq_linear_rounded": (_c_int, [_c_vp, _c_int, _c_int, _c_vp, _c_int, _c_vp, _c_vp, _c_int, _c_int, _c_vp,
                                     _c_vp, _c_vp, _c_int, _c_vp, _c_size, _c_vp]),
    "matq_linear_noalloc": (_c_int, [_c_vp, _c_int, _c_int, _c_vp, _c_int, _c_vp, _c_vp, _c_int, _c_int, _c_int,
                                     _c_vp, _c_int, _c_vp, _c_vp]),
    "matq_rmsnorm": (_c_int, [_c_vp, _c_int, _c_int, _c_float, _c_vp, _c_vp]),
    "matq_silu_mul": (_c_int, [_c_vp, _c_vp, _c_int, _c_int, _c_vp, _c_vp]),
    "matq_silu_mul_gu": (_c_int, [_c_vp, _c_int, _c_int, _c_vp, _c_vp]),
    "matq_choose_codes": (_c_int, [_c_vp, _c_int, _c_int, _c_vp, _c_vp, _c_int, _c_int, ctypes.POINTER(_c_int),
                                   ctypes.POINTER(_c_float), _c_int, _c_vp, _c_vp]),
}

for _name, (_res, _args) in _SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args
    globals()[_name] = _fn

EXPORTED = tuple(_SIGNATURES)


class MatqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = matq_strerror(status).decode()
        if status == MATQ_ECUDA:
            msg += f" (cudaError {matq_last_cuda_error()})"
        super().__init__(f"{what}: {msg} [status {status}]")


def check(status: int, what: str) -> None:
    if status != MATQ_OK:
        raise MatqError(status, what)


# ---------------------------------------------------------------------------------------
# torch-tensor helpers (memory and streams only)
# ---------------------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _stream_ptr(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _ptr(t) -> int:
    return int(t.data_ptr())


def _dev(t, name: str, dtypes, what: str):
    """Pointer of a CUDA tensor after the checks the C ABI cannot make itself: the memory is
    on the GPU, contiguous, of an accepted element type.  (A host pointer or a strided view
    would be read as garbage, or fault.)"""
    if not t.is_cuda:
        raise ValueError(f"{what}: {name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what}: {name} must be contiguous")
    if t.dtype not in dtypes:
        raise ValueError(f"{what}: {name} has dtype {t.dtype}, expected one of {dtypes}")
    return int(t.data_ptr())


def _dt(*names):
    torch = _torch()
    return tuple(getattr(torch, n) for n in names)


def pack(codes, r_keep: int = 8, stream=None):
    """Pack [N, K] uint8 codes (CUDA tensor) into a uint8 plane buffer (CUDA tensor)."""
    torch = _torch()
    N, K = codes.shape
    pc = _dev(codes, "codes", _dt("uint8"), "pack")
    nbytes = matq_packed_bytes(N, K, r_keep)
    if nbytes == 0:
        check(MATQ_EINVAL_SHAPE if r_keep in WIDTHS else MATQ_EINVAL_R, "matq_packed_bytes")
    planes = torch.empty(nbytes, dtype=torch.uint8, device=codes.device)
    check(matq_pack(pc, N, K, r_keep, _ptr(planes), nbytes, _stream_ptr(stream)), "matq_pack")
    return planes


def slice_prefix(planes, N: int, K: int, r_keep: int, r: int, stream=None):
    """Prefixes p = q >> (8 - r) as a [N, K] uint8 CUDA tensor."""
    torch = _torch()
    pp = _dev(planes, "planes", _dt("uint8"), "slice_prefix")
    out = torch.empty((N, K), dtype=torch.uint8, device=planes.device)
    check(matq_slice(pp, N, K, r_keep, r, _ptr(out), _stream_ptr(stream)), "matq_slice")
    return out


def slice_copy(planes, N: int, K: int, r_keep: int, r: int, stream=None):
    """Deployment mode A: a new plane buffer holding only the width-r prefix."""
    torch = _torch()
    pp = _dev(planes, "planes", _dt("uint8"), "slice_copy")
    nbytes = matq_packed_bytes(N, K, r)
    out = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=planes.device)
    check(matq_slice_copy(pp, N, K, r_keep, r, _ptr(out), out.numel(), _stream_ptr(stream)),
          "matq_slice_copy")
    return out[:nbytes]


def workspace_bytes(M: int, K: int, N: int, group: int) -> int:
    return int(matq_linear_workspace(M, K, N, group))


def workspace(M: int, K: int, N: int, group: int, device="cuda"):
    """A zero-filled workspace (uint8 CUDA tensor) for calls up to these sizes."""
    torch = _torch()
    return torch.zeros(max(workspace_bytes(M, K, N, group), 256), dtype=torch.uint8, device=device)


def workspace_status(ws) -> int:
    """Device status word of a workspace (0 = every call so far completed normally)."""
    out = _c_int(0)
    check(matq_workspace_status(_dev(ws, "workspace", _dt("uint8"), "workspace_status"), ctypes.byref(out)),
          "matq_workspace_status")
    return int(out.value)


def selftest_timeout(ws, stream=None) -> None:
    """Run the bounded-wait self-test on a workspace (its status then reports
    MATQ_STATUS_SELFTEST, after about a second on the device)."""
    check(matq_selftest_timeout(_dev(ws, "workspace", _dt("uint8"), "selftest_timeout"), ws.numel(),
                                _stream_ptr(stream)), "matq_selftest_timeout")


def linear(x, planes, r_keep: int, scales, zeros, N: int, r: int, group: int, y=None,
           y_mode: int = MATQ_OUT_BF16, workspace=None, stream=None):
    """y = x . W_hat_r^T.  x: [M, K] bf16 CUDA tensor; scales: [N, K/group] (fp16 or int16
    bits); zeros: [N, K/group] uint8.  Returns y ([M, N] bf16 or fp32)."""
    torch = _torch()
    M, K = x.shape
    if y is None:
        dt = torch.bfloat16 if y_mode in (MATQ_OUT_BF16, MATQ_OUT_SILU_GATED) else torch.float32
        cols = N // 2 if y_mode == MATQ_OUT_SILU_GATED else N
        y = (torch.zeros if y_mode == MATQ_OUT_F32_ACCUM else torch.empty)((M, cols), dtype=dt, device=x.device)
    if workspace is None:
        workspace = torch.zeros(max(workspace_bytes(M, K, N, group), 256), dtype=torch.uint8, device=x.device)
    w = "linear"
    ydt = _dt("bfloat16") if y_mode in (MATQ_OUT_BF16, MATQ_OUT_SILU_GATED) else _dt("float32")
    check(matq_linear(_dev(x, "x", _dt("bfloat16"), w), M, K, _dev(planes, "planes", _dt("uint8"), w), r_keep,
                      _dev(scales, "scales", _dt("float16", "int16"), w), _dev(zeros, "zeros", _dt("uint8"), w),
                      N, r, group, _dev(y, "y", ydt, w), y_mode, _dev(workspace, "workspace", _dt("uint8"), w),
                      workspace.numel(), _stream_ptr(stream)), "matq_linear")
    return y


def round_extract(planes, N: int, K: int, r_keep: int, r: int, stream=None):
    """The width-r rounded slice of a pack (strict / Extra-Precision MatQuant): returns
    (levels, row_ptr, cols) -- the clamped-level pack of width r, and the CSR list of the
    weights whose rounded level is 2^r (cols padded to a multiple of 8 entries).  Reads the
    list's length back to the host once (a synchronisation of `stream`)."""
    torch = _torch()
    w = "round_extract"
    pp = _dev(planes, "planes", _dt("uint8"), w)
    dev = planes.device
    levels = torch.empty(max(matq_packed_bytes(N, K, r), 16), dtype=torch.uint8, device=dev)
    row_ptr = torch.empty(N + 1, dtype=torch.int32, device=dev)
    scratch = torch.empty(max(matq_round_scratch_bytes(N, K), 256), dtype=torch.uint8, device=dev)
    sp = _stream_ptr(stream)
    check(matq_round_extract(pp, N, K, r_keep, r, _ptr(levels), levels.numel(), _ptr(row_ptr), None, 0,
                             _ptr(scratch), scratch.numel(), sp), "matq_round_extract")
    if stream is not None:
        stream.synchronize()
    else:
        torch.cuda.current_stream(dev).synchronize()
    nnz = int(row_ptr[N].item())
    cols = torch.zeros((((nnz + 7) // 8) * 8 + 8,), dtype=torch.int16, device=dev)
    check(matq_round_extract(pp, N, K, r_keep, r, _ptr(levels), levels.numel(), _ptr(row_ptr), _ptr(cols),
                             cols.numel(), _ptr(scratch), scratch.numel(), sp), "matq_round_extract")
    return levels, row_ptr, cols


def rounded_workspace(M: int, K: int, N: int, group: int, device="cuda"):
    torch = _torch()
    ws = torch.zeros(max(matq_linear_rounded_workspace(M, K, N, group), 256), dtype=torch.uint8, device=device)
    return ws


def linear_rounded(x, levels, r: int, scales, zeros, N: int, group: int, row_ptr=None, cols=None, y=None,
                   y_mode: int = MATQ_OUT_BF16, workspace=None, stream=None):
    """y = x . W_hat^T for a rounded slice: Extra-Precision MatQuant with the overflow list
    (row_ptr, cols from ``round_extract``), strict MatQuant without it."""
    torch = _torch()
    M, K = x.shape
    if y is None:
        dt = torch.bfloat16 if y_mode in (MATQ_OUT_BF16, MATQ_OUT_SILU_GATED) else torch.float32
        ncols = N // 2 if y_mode == MATQ_OUT_SILU_GATED else N
        y = (torch.zeros if y_mode == MATQ_OUT_F32_ACCUM else torch.empty)((M, ncols), dtype=dt, device=x.device)
    if workspace is None:
        workspace = rounded_workspace(M, K, N, group, device=x.device)
    w = "linear_rounded"
    ydt = _dt("bfloat16") if y_mode in (MATQ_OUT_BF16, MATQ_OUT_SILU_GATED) else _dt("float32")
    rp = None if row_ptr is None else _dev(row_ptr, "row_ptr", _dt("int32"), w)
    cp = None if cols is None else _dev(cols, "cols", _dt("int16", "uint16"), w)
    check(matq_linear_rounded(_dev(x, "x", _dt("bfloat16"), w), M, K, _dev(levels, "levels", _dt("uint8"), w), r,
                              _dev(scales, "scales", _dt("float16", "int16"), w), _dev(zeros, "zeros", _dt("uint8"), w),
                              N, group, rp, cp, _dev(y, "y", ydt, w), y_mode,
                              _dev(workspace, "workspace", _dt("uint8"), w), workspace.numel(), _stream_ptr(stream)),
          "matq_linear_rounded")
    return y


def linear_noalloc(x, planes, r_keep: int, scales, zeros, N: int, r: int, group: int, y=None,
                   y_mode: int = MATQ_OUT_BF16, status=None, stream=None):
    """Same as ``linear`` but with libmatq's own fixed scratch (no workspace argument).
    ``status``: optional int32 CUDA tensor of one element that receives the call's device
    status word.  Returns y."""
    torch = _torch()
    M, K = x.shape
    if y is None:
        dt = torch.bfloat16 if y_mode in (MATQ_OUT_BF16, MATQ_OUT_SILU_GATED) else torch.float32
        cols = N // 2 if y_mode == MATQ_OUT_SILU_GATED else N
        y = (torch.zeros if y_mode == MATQ_OUT_F32_ACCUM else torch.empty)((M, cols), dtype=dt, device=x.device)
    w = "linear_noalloc"
    sp = _dev(status, "status", _dt("int32"), w) if status is not None else None
    ydt = _dt("bfloat16") if y_mode in (MATQ_OUT_BF16, MATQ_OUT_SILU_GATED) else _dt("float32")
    check(matq_linear_noalloc(_dev(x, "x", _dt("bfloat16"), w), M, K, _dev(planes, "planes", _dt("uint8"), w),
                              r_keep, _dev(scales, "scales", _dt("float16", "int16"), w),
                              _dev(zeros, "zeros", _dt("uint8"), w), N, r, group, _dev(y, "y", ydt, w), y_mode, sp,
                              _stream_ptr(stream)), "matq_linear_noalloc")
    return y


def rmsnorm(h, eps: float = 1e-5, out=None, stream=None):
    torch = _torch()
    M, D = h.shape
    if out is None:
        out = torch.empty((M, D), dtype=torch.bfloat16, device=h.device)
    check(matq_rmsnorm(_dev(h, "h", _dt("float32"), "rmsnorm"), M, D, eps,
                       _dev(out, "out", _dt("bfloat16"), "rmsnorm"), _stream_ptr(stream)), "matq_rmsnorm")
    return out


def silu_mul(gate, up, out=None, stream=None):
    torch = _torch()
    M, F = gate.shape
    if out is None:
        out = torch.empty((M, F), dtype=torch.bfloat16, device=gate.device)
    if tuple(up.shape) != (M, F):
        raise ValueError("silu_mul: gate and up must have the same shape")
    b = _dt("bfloat16")
    check(matq_silu_mul(_dev(gate, "gate", b, "silu_mul"), _dev(up, "up", b, "silu_mul"), M, F,
                        _dev(out, "out", b, "silu_mul"), _stream_ptr(stream)), "matq_silu_mul")
    return out


def silu_mul_gu(gu, out=None, stream=None):
    """a = silu(gate) * up from one fused gate+up output gu [M, 2F] (gate = first F columns)."""
    torch = _torch()
    M, F2 = gu.shape
    F = F2 // 2
    if out is None:
        out = torch.empty((M, F), dtype=torch.bfloat16, device=gu.device)
    if F2 % 2:
        raise ValueError("silu_mul_gu: gu must have an even number of columns")
    b = _dt("bfloat16")
    check(matq_silu_mul_gu(_dev(gu, "gu", b, "silu_mul_gu"), M, F, _dev(out, "out", b, "silu_mul_gu"),
                           _stream_ptr(stream)), "matq_silu_mul_gu")
    return out


def choose_codes(w, scales, zeros, group: int, widths=(3, 4, 8), lambdas=None,
                 mode: int = MATQ_SLICE_TRUE_PREFIX, out=None, stream=None):
    """Parent codes [N, K] uint8 chosen for several widths at once (matq_choose_codes).

    w fp32 [N, K], scales fp16 [N, K/group] and zeros uint8 [N, K/group] are CUDA tensors;
    widths (ascending) and lambdas are host sequences, lambdas defaulting to equal weights
    that sum to one."""
    torch = _torch()
    N, K = w.shape
    widths = [int(r) for r in widths]
    if lambdas is None:
        lambdas = [1.0 / len(widths)] * len(widths)
    lambdas = [float(v) for v in lambdas]
    if len(lambdas) != len(widths):
        raise ValueError("choose_codes: one lambda per width")
    if out is None:
        out = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    what = "choose_codes"
    rw = (_c_int * len(widths))(*widths)
    lw = (_c_float * len(lambdas))(*lambdas)
    check(matq_choose_codes(_dev(w, "w", _dt("float32"), what), N, K,
                            _dev(scales, "scales", _dt("float16", "int16"), what),
                            _dev(zeros, "zeros", _dt("uint8"), what), group, len(widths), rw, lw, mode,
                            _dev(out, "out", _dt("uint8"), what), _stream_ptr(stream)), "matq_choose_codes")
    return out
