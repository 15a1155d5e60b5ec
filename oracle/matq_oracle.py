"""Plain, slow, fp64 CPU oracle for the sliced r-bit (Matryoshka) linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` use it.  It shares no code, tables or helpers with the CUDA
library; it works on plain NumPy arrays (codes, scales, zeros, activations)
that a separate seeded generator produces.

What it computes, and the passages it follows
---------------------------------------------
Pages are cited by title and section.

* ``prefix``      -- the r most significant bits of an unsigned c-bit code:
  a right shift by c-r.  "MatGPTQ: Efficient and Accurate Inference over
  Nested Quantized Models", App. A.1 (Improved nested representation).
* ``reconstruct`` -- the sliced code mapped back into c-bit code space.
  Primary rule ("true_prefix"): left shift back, then add delta_r, the offset
  that moves the value from the lower edge to the centre of its cell
  (same page, App. A.1; contribution 3 of its §1).  delta_r = (2^(c-r)-1)/2,
  the mean of the c-bit codes in a cell (reading stated below).
  Variant rules, kept for study and pins:
    "truncate"        -- raw MSB truncation, delta = 0 (App. A.1, first paragraph);
    "matquant_round"  -- clamp(round(q / 2^(c-r)), 0, 2^r - 1) * 2^(c-r)
                         ("Matryoshka Quantization | Summary", §3.2 MatQuant);
    "extra_precision" -- the same without the clamp, 2^r + 1 levels
                         (same page, §7 Errata).
* ``dequant``     -- w_hat = s * (q_hat - z), with one scale s and zero point z
  per group of ``group`` consecutive inputs of a row, shared by every width
  ("Matryoshka Quantization | Summary", §3.1 MinMax quantizer; the MatQuant
  rebuttal page, "Single Precision (S. P.) MatQuant vs Baseline", item 2:
  scale and zero come from the 8-bit model; MatGPTQ §1: single shared-scale
  representation).
* ``linear``      -- y = x . W_hat^T, the product the nested kernel computes
  (MatGPTQ §4, Fast Matryoshka Kernels: Y = X W_D with the torch.nn.Linear
  interface, so W is stored [out, in]).  NumPy fp64 matmul is the step.
* ``linear_loops``-- the same product as an explicit scalar triple loop, used
  to check ``linear`` on tiny shapes.
* ``linear_group_sums`` -- the same product regrouped per K-group with delta_r
  and the zero point applied to the per-group activation sums (App. A.1: delta
  can be absorbed into the zero point).  Exact algebra, checked against
  ``linear``.
* ``choose_codes`` -- the parent code of each weight chosen for several widths
  at once: every candidate code is dequantised at each target width with the
  shared scale and zero point, and the lambda-weighted sum of squared errors
  decides (MatGPTQ §3.2 item 2, App. A.2 Algorithm 2, brute force over all 2^c
  candidates, fp32 as the page keeps the candidate errors).  lambda is an
  input: the pages do not print the values they used.
* ``rmsnorm``, ``silu``, ``ffn_block`` -- the glue of the Mix'n'Match stack
  ("Matryoshka Quantization | Summary", §4.3 Layerwise Mix'n'Match; MatGPTQ
  §5.4).  The pages give no block formula; the reading taken is a Llama-style
  FFN block with a unit-gain RMSNorm and a residual:
  h <- h + down(silu(gate(n)) * up(n)), n = h / sqrt(mean(h^2) + eps).

Readings where the pages are silent or ambiguous
------------------------------------------------
* delta_r is the mean of the c-bit codes in the cell, (2^(c-r)-1)/2, not the
  continuous cell centre 2^(c-r-1): App. A.1 says the centred value balances
  the distances to the c-bit values and minimises the RMS reconstruction
  error, which is the discrete mean; it also makes r = c the identity.  The
  other reading is available as ``delta_rule="half_cell"``.
* "round" in the MatQuant rule has no stated tie rule: round half up is the
  default, round half to even is ``tie="even"``.
* Codes, zero points are unsigned in [0, 255] (the Errata's worked example
  uses "unsigned int8 value 234").
* Scales are fp16 values; the oracle takes them as exact fp64 numbers.

Parity status: every function here is pinned by tests under ``tests/``
(``test_oracle_pins.py``) against worked examples printed on the pages,
closed forms, invariants and brute force.  ``ffn_block`` is pinned by a
hand-worked two-row block (``tests/golden/ffn_block_hand.txt``) that a swapped
gate and up, a skipped RMSNorm, a dropped residual, eps outside the square
root or a transposed projection each fail.  Only the end-to-end Mix'n'Match
stack deviation over many layers is reported, not gated ("parity unpinned"
beyond the per-layer, teacher-forced checks).
"""

from __future__ import annotations

import numpy as np

C_BITS = 8
WIDTHS = (2, 3, 4, 6, 8)
MODES = ("true_prefix", "truncate", "matquant_round", "extra_precision")


def _as_codes(q):
    q = np.asarray(q)
    if q.dtype.kind not in "ui":
        raise TypeError("codes must be an integer array")
    if q.size and (q.min() < 0 or q.max() > (1 << C_BITS) - 1):
        raise ValueError("codes must lie in [0, 255]")
    return q.astype(np.int64)


def _check_width(r):
    if r not in range(1, C_BITS + 1):
        raise ValueError(f"width r={r} outside 1..{C_BITS}")


def prefix(q, r):
    """The r most significant bits of each c-bit code, as an integer in [0, 2^r).

    MatGPTQ App. A.1: a right shift by c - r keeps the r MSBs.
    """
    _check_width(r)
    q = _as_codes(q)
    return q >> (C_BITS - r)


def delta(r, rule="code_mean"):
    """Offset added to the shifted-back prefix so the value sits in its cell's centre.

    MatGPTQ App. A.1.  ``code_mean``: (2^(c-r) - 1) / 2, the mean of the c-bit codes
    that share the prefix (zero for r = c).  ``half_cell``: 2^(c-r-1), the centre of
    the continuous cell (alternative reading, zero only by convention at r = c).
    """
    _check_width(r)
    width = 1 << (C_BITS - r)
    if rule == "code_mean":
        return (width - 1) / 2.0
    if rule == "half_cell":
        return width / 2.0 if r < C_BITS else 0.0
    raise ValueError(f"unknown delta rule {rule!r}")


def _round_half(v, tie):
    if tie == "up":
        return np.floor(v + 0.5)
    if tie == "even":
        return np.rint(v)
    raise ValueError(f"unknown tie rule {tie!r}")


def reconstruct(q, r, mode="true_prefix", delta_rule="code_mean", tie="up"):
    """Sliced code in c-bit code space (float64), for one of the slicing rules.

    true_prefix     : prefix(q, r) * 2^(c-r) + delta_r          (MatGPTQ App. A.1)
    truncate        : prefix(q, r) * 2^(c-r)                     (MatGPTQ App. A.1)
    matquant_round  : clamp(round(q / 2^(c-r)), 0, 2^r-1) * 2^(c-r)
                      ("Matryoshka Quantization | Summary", §3.2)
    extra_precision : round(q / 2^(c-r)) * 2^(c-r), no clamp   (same page, §7 Errata)
    """
    _check_width(r)
    q = _as_codes(q)
    step = float(1 << (C_BITS - r))
    if mode == "true_prefix":
        return (q >> (C_BITS - r)).astype(np.float64) * step + delta(r, delta_rule)
    if mode == "truncate":
        return (q >> (C_BITS - r)).astype(np.float64) * step
    if mode in ("matquant_round", "extra_precision"):
        level = _round_half(q.astype(np.float64) / step, tie)
        if mode == "matquant_round":
            level = np.clip(level, 0.0, float((1 << r) - 1))
        return level * step
    raise ValueError(f"unknown slicing mode {mode!r}")


def _group_expand(a, group, K):
    a = np.asarray(a)
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    if a.shape[-1] != K // group:
        raise ValueError("per-group metadata has the wrong number of groups")
    return np.repeat(a.astype(np.float64), group, axis=-1)


def dequant(q, scale, zero, r, group, mode="true_prefix", delta_rule="code_mean", tie="up"):
    """W_hat[n, k] = s[n, k // group] * (q_hat[n, k] - z[n, k // group]) in fp64.

    ``q``: [N, K] codes; ``scale``: [N, K/group] (fp16 values); ``zero``: [N, K/group]
    codes.  "Matryoshka Quantization | Summary" §3.1 (MinMax scale and zero point);
    scale and zero shared by every width (MatGPTQ §1; MatQuant rebuttal, S.P. item 2).
    """
    q = _as_codes(q)
    N, K = q.shape
    s = _group_expand(scale, group, K)
    z = _group_expand(zero, group, K)
    return s * (reconstruct(q, r, mode, delta_rule, tie) - z)


def linear(x, q, scale, zero, r, group, mode="true_prefix", delta_rule="code_mean", tie="up"):
    """y[m, n] = sum_k x[m, k] * W_hat[n, k] in fp64 (MatGPTQ §4: Y = X W_D, Linear layout)."""
    x = np.asarray(x, dtype=np.float64)
    w = dequant(q, scale, zero, r, group, mode, delta_rule, tie)
    if x.shape[-1] != w.shape[1]:
        raise ValueError("x and W disagree on K")
    return x @ w.T


def linear_loops(x, q, scale, zero, r, group, mode="true_prefix"):
    """The same product written as a scalar triple loop (tiny shapes only)."""
    x = np.asarray(x, dtype=np.float64)
    q = _as_codes(q)
    M, K = x.shape
    N = q.shape[0]
    scale = np.asarray(scale, dtype=np.float64)
    zero = np.asarray(zero, dtype=np.float64)
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                g = k // group
                qh = float(reconstruct(np.array([q[n, k]]), r, mode)[0])
                acc += x[m, k] * (scale[n, g] * (qh - zero[n, g]))
            y[m, n] = acc
    return y


def linear_group_sums(x, q, scale, zero, r, group, delta_rule="code_mean"):
    """True-prefix product regrouped by K-group (delta folded into the zero point).

    y[m, n] = sum_g s[n, g] * ( 2^(c-r) * sum_{k in g} x[m, k] * p[n, k]
                                + (delta_r - z[n, g]) * sum_{k in g} x[m, k] )
    MatGPTQ App. A.1: delta_r can be absorbed into the zero point.
    """
    x = np.asarray(x, dtype=np.float64)
    p = prefix(q, r).astype(np.float64)
    N, K = p.shape
    M = x.shape[0]
    G = K // group
    xs = x.reshape(M, G, group)
    ps = p.reshape(N, G, group)
    dot = np.einsum("mgk,ngk->mng", xs, ps)             # sum_k x * p per group
    xsum = xs.sum(axis=2)                                 # [M, G]
    s = np.asarray(scale, dtype=np.float64)              # [N, G]
    z = np.asarray(zero, dtype=np.float64)
    step = float(1 << (C_BITS - r))
    d = delta(r, delta_rule)
    per_group = s[None] * (step * dot + (d - z)[None] * xsum[:, None, :])
    return per_group.sum(axis=2)


def bits_read_per_weight(r, mode="true_prefix"):
    """Bits of the parent code a width-r slice must read per weight.

    True-prefix slicing reads exactly r bits (MatGPTQ §4: serving r bits reads
    exactly r bits per weight); the rounding rule needs the (r+1)-th bit too
    (MatGPTQ App. A.1, second paragraph; §2.3).
    """
    _check_width(r)
    if mode in ("true_prefix", "truncate"):
        return r
    return min(r + 1, C_BITS)


# ---------------------------------------------------------------------------
# Mix'n'Match stack glue (reading stated in the module docstring)
# ---------------------------------------------------------------------------

def rmsnorm(h, eps=1e-5):
    """n = h / sqrt(mean(h^2, last axis) + eps), unit gain, fp64."""
    h = np.asarray(h, dtype=np.float64)
    return h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)


def silu(t):
    """SiLU(t) = t * sigmoid(t) = t / (1 + exp(-t)), fp64."""
    t = np.asarray(t, dtype=np.float64)
    return t / (1.0 + np.exp(-t))


def gated_product(gate, up):
    """a = silu(gate) * up (the SiLU-gated product between the two FFN halves)."""
    return silu(gate) * np.asarray(up, dtype=np.float64)


def ffn_block(h, layer, r, group, eps=1e-5):
    """One Mix'n'Match FFN block at width r; ``layer`` maps 'gate'/'up'/'down' to (q, s, z).

    h <- h + down(silu(gate(n)) * up(n)),  n = rmsnorm(h).
    """
    n = rmsnorm(h, eps)
    g = linear(n, *layer["gate"], r, group)
    u = linear(n, *layer["up"], r, group)
    a = gated_product(g, u)
    return np.asarray(h, dtype=np.float64) + linear(a, *layer["down"], r, group)


def mixnmatch_effective_bits(widths, sizes=None):
    """Average bits per weight of a per-layer width allocation ("Matryoshka
    Quantization | Summary" §4.3: effective bits per FFN parameter)."""
    widths = np.asarray(widths, dtype=np.float64)
    if sizes is None:
        return float(widths.mean())
    sizes = np.asarray(sizes, dtype=np.float64)
    return float((widths * sizes).sum() / sizes.sum())


def choose_codes(w, scale, zero, group, widths=(3, 4, 8), lambdas=None, mode="true_prefix"):
    """Parent codes chosen for several widths at once ("MatGPTQ: Efficient and Accurate
    Inference over Nested Quantized Models", §3.2 item 2 and App. A.2, the brute-force
    quant_MatGPTQ step of Algorithm 2).

    Every weight w[n, k] tries all 2^c candidate codes q.  Each candidate is dequantised at
    every target width r with the weight's shared group scale s and zero point z,
    w_hat_r(q) = s * (reconstruct(q, r, mode) - z), and scored with
    lambda_r * (w - w_hat_r(q))^2, summed over the widths in the order given.  The code with
    the smallest total is kept; on a tie the smallest code (argmin's first occurrence).

    Arithmetic: fp32 with every operation rounded on its own, the precision the page gives
    for the candidate errors (App. A.2, runtime and memory: the 2^c x rows matrix is held in
    FP32).  w_hat_r is exact in fp32 (an 11-bit scale times a half-integer below 256), so the
    roundings are those of e = w - w_hat_r, e * e, lambda_r * (e * e) and the running sum.

    widths: strictly ascending widths from WIDTHS.  lambdas: one finite non-negative weight
    per width (default: equal weights summing to one, the normalised lambda of §3.2 item 3).
    Returns uint8 codes [N, K].
    """
    widths = tuple(int(r) for r in widths)
    if not widths or any(r not in WIDTHS for r in widths) or any(a >= b for a, b in zip(widths, widths[1:])):
        raise ValueError("widths must be a strictly ascending subset of (2, 3, 4, 6, 8)")
    if lambdas is None:
        lambdas = [1.0 / len(widths)] * len(widths)
    lam = np.asarray(lambdas, dtype=np.float32)
    if lam.shape != (len(widths),) or not np.all(np.isfinite(lam)) or np.any(lam < 0):
        raise ValueError("one finite, non-negative lambda per width")
    w32 = np.asarray(w, dtype=np.float32)
    if w32.ndim != 2:
        raise ValueError("w must be [N, K]")
    N, K = w32.shape
    s32 = np.repeat(np.asarray(scale, dtype=np.float16).astype(np.float32), group, axis=1)
    z32 = np.repeat(np.asarray(zero, dtype=np.uint8).astype(np.float32), group, axis=1)
    if s32.shape != (N, K) or z32.shape != (N, K):
        raise ValueError("per-group metadata has the wrong shape")
    cand = np.arange(1 << C_BITS, dtype=np.uint8)
    qhat = {r: reconstruct(cand, r, mode).astype(np.float32)[:, None, None] for r in widths}
    out = np.empty((N, K), dtype=np.uint8)
    rows = max(1, (1 << 24) // ((1 << C_BITS) * max(K, 1)))  # bounds the candidate matrix
    for n0 in range(0, N, rows):
        sl = slice(n0, min(N, n0 + rows))
        wv, sv, zv = w32[sl][None], s32[sl][None], z32[sl][None]
        total = None
        for r, lr in zip(widths, lam):
            e = wv - sv * (qhat[r] - zv)
            t = lr * (e * e)
            total = t if total is None else total + t
        out[sl] = np.argmin(total, axis=0)
    return out
