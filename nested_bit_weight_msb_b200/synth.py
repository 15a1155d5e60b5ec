"""Seeded synthetic inputs for the sliced r-bit linear layer.

This module only draws inputs: Gaussian weights turned into 8-bit parent codes
with a per-group MinMax (asymmetric, round-to-nearest) quantizer, and Gaussian
bf16 activations.  It holds none of the slicing, dequantisation or product
arithmetic, and it imports nothing from the CUDA binding or the oracle, so
both sides can share its outputs as data.

Recipe (all seeded through ``numpy.random.SeedSequence([seed, layer, proj, kind])``):

* weights: W = 0.02 * standard_normal([N, K]) in fp32.  Per group of ``group``
  consecutive inputs of a row: mn = min(min(w), 0), mx = max(max(w), 0),
  s = fp16((mx - mn) / 255), z = clip(rint(-mn / s), 0, 255),
  q = clip(rint(w / s) + z, 0, 255).  MinMax scale / zero point as in
  "Matryoshka Quantization | Summary" §3.1; asymmetric as in MatGPTQ §5.2.
  The pages measure real Llama-3.1-8B / Qwen3-8B / Gemma-2-9B matrices; these
  synthetic weights of the same shapes stand in for them.
* activations: standard normal, optionally with a fraction of outlier input
  channels (the same channels for every row) multiplied by ``outlier_mult``,
  rounded to bf16 (round to nearest even).
* Mix'n'Match widths: a seeded permutation of [2]*11 + [3]*10 + [4]*11
  (32 layers, average exactly 3 bits).
"""

from __future__ import annotations

import numpy as np

PROJ = {"gate": 0, "up": 1, "down": 2}
KIND_WEIGHT = 0
KIND_ACT = 1


def _rng(seed, layer, proj, kind):
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(layer), int(proj), int(kind)]))


def bf16_round(a):
    """Round fp32 values to bf16 (nearest even); returns (uint16 bits, fp32 values)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    u = u.astype(np.uint32)
    return (u >> 16).astype(np.uint16), u.view(np.float32)


def quantize_minmax(w, group):
    """Per-group asymmetric MinMax round-to-nearest 8-bit codes (input recipe only)."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    if K % group:
        raise ValueError("K must be a multiple of group")
    wg = w.reshape(N, K // group, group)
    mn = np.minimum(wg.min(axis=2), 0.0)
    mx = np.maximum(wg.max(axis=2), 0.0)
    s = ((mx - mn) / np.float32(255.0)).astype(np.float16)
    tiny = np.float16(np.finfo(np.float16).tiny)
    s = np.where(s > 0, s, tiny).astype(np.float16)
    s32 = s.astype(np.float32)
    z = np.clip(np.rint(-mn / s32), 0, 255)
    q = np.clip(np.rint(wg / s32[:, :, None]) + z[:, :, None], 0, 255)
    return q.reshape(N, K).astype(np.uint8), s, z.astype(np.uint8)


def _float_w(N, K, seed, layer, proj, std):
    rng = _rng(seed, layer, PROJ.get(proj, proj), KIND_WEIGHT)
    return (np.float32(std) * rng.standard_normal((N, K), dtype=np.float32)).astype(np.float32)


def parent_weights(N, K, group, seed=0, layer=0, proj="gate", std=0.02):
    """Seeded parent codes [N, K] u8, fp16 scales [N, K/group], u8 zeros [N, K/group]."""
    return quantize_minmax(_float_w(N, K, seed, layer, proj, std), group)


def float_weights(N, K, group, seed=0, layer=0, proj="gate", std=0.02):
    """The fp32 weights [N, K] behind parent_weights (same arguments, same weights) with their
    per-group MinMax fp16 scales and u8 zero points: the inputs of a parent-code choice."""
    w = _float_w(N, K, seed, layer, proj, std)
    _, s, z = quantize_minmax(w, group)
    return w, s, z


def activations(M, K, seed=0, layer=0, proj="gate", outlier_frac=0.0, outlier_mult=20.0):
    """Seeded bf16 activations [M, K]: returns (uint16 bits, fp32 values).

    ``outlier_frac`` of the K input channels (round(outlier_frac * K) of them,
    chosen without replacement) are multiplied by ``outlier_mult`` in fp32
    before the bf16 rounding; the same channels for every row.
    """
    rng = _rng(seed, layer, PROJ.get(proj, proj), KIND_ACT)
    x = rng.standard_normal((M, K), dtype=np.float32)
    n_out = int(round(outlier_frac * K))
    if n_out:
        cols = rng.choice(K, n_out, replace=False)
        x[:, cols] *= np.float32(outlier_mult)
    return bf16_round(x)


def random_codes(shape, seed=0):
    """Uniform random 8-bit codes (for layout / round-trip tests)."""
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), 7]))
    return rng.integers(0, 256, size=shape, dtype=np.uint8)


def mixnmatch_widths(seed=0, layers=32):
    """Per-layer widths: a seeded permutation of [2]*11 + [3]*10 + [4]*11 (32 layers)."""
    if layers != 32:
        raise ValueError("the recipe is defined for 32 layers")
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), 32]))
    return rng.permutation(np.array([2] * 11 + [3] * 10 + [4] * 11, dtype=np.int64))
