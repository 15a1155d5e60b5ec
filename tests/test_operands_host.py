"""The bit-level unpack of plane words into fp16 MMA operands (csrc/operands.cuh, used by the
decode and the prefill kernels), compiled for the host and checked against the plane layout
documented in include/matq.h and the true-prefix definition ("MatGPTQ: Efficient and Accurate
Inference over Nested Quantized Models", App. A.1: the r-bit prefix p = q >> (8 - r)).

operands.cuh is compiled unchanged next to a host stand-in for common.cuh that gives the three
bit helpers it uses their documented meaning -- and_or(a, b, c) = (a & b) | c, bitsel(a, b, m)
= (a & m) | (b & ~m), and the default-mode byte permute of PTX prmt.b32 (each selector nibble
picks byte n of the 8-byte pool {b:a}, a = bytes 0..3; its top bit replicates that byte's sign).
The lane words are read from the bytes of the NumPy layout model (tests/layout_model.py, written
from the header text and also the reference for the pack kernel's output) at the lane offsets
the kernels load them from.  Every fp16 half of every operand register, for every lane, block
and width, must equal 1024 + sigma * v with v the prefix (r <= 4) or the prefix shifted back
(r = 6, 8) of its weight's code, and sigma the register's documented power of two.  No GPU
needed.
"""

import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle as O
from layout_model import field_coords as _field_coords, layout_model, tile_lane_words

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "nested_bit_weight_msb_b200", "csrc", "operands.cuh")
BUILD = os.path.join(ROOT, "tests", "_build", "operands")

COMMON_STUB = r"""
#pragma once
#include <cstdint>
#include <cstring>
#define __device__
#define __host__
#define __forceinline__ inline
namespace matq {
struct uint4 { uint32_t x, y, z, w; };
struct PlaneGeom { int N, K, RT, KC; unsigned long long off[5]; };
inline uint4 ldg_stream(const void* p) { uint4 v; std::memcpy(&v, p, 16); return v; }
inline uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) { return (a & b) | c; }
inline uint32_t bitsel(uint32_t a, uint32_t b, uint32_t m) { return (a & m) | (b & ~m); }
inline uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  const uint64_t pool = ((uint64_t)b << 32) | a;
  uint32_t d = 0;
  for (int i = 0; i < 4; ++i) {
    const uint32_t s = (sel >> (4 * i)) & 0xF;
    uint32_t byte = (uint32_t)(pool >> (8 * (s & 7))) & 0xFF;
    if (s & 8) byte = (byte & 0x80) ? 0xFF : 0x00;
    d |= byte << (8 * i);
  }
  return d;
}
}  // namespace matq
"""

DRIVER = r"""
#include "operands.cuh"
template <int R, int W>
static void one(const matq::LaneWords& L, uint32_t* out) {
  uint32_t A[2][4];
  matq::build_operands<R, W>(L, A);
  for (int j = 0; j < 2; ++j)
    for (int rho = 0; rho < 4; ++rho) out[4 * j + rho] = A[j][rho];
}
template <int R>
static void by_block(int W, const matq::LaneWords& L, uint32_t* out) {
  switch (W) {
    case 0: one<R, 0>(L, out); break;
    case 1: one<R, 1>(L, out); break;
    case 2: one<R, 2>(L, out); break;
    case 3: one<R, 3>(L, out); break;
    case 4: one<R, 4>(L, out); break;
    case 5: one<R, 5>(L, out); break;
    case 6: one<R, 6>(L, out); break;
    default: one<R, 7>(L, out); break;
  }
}
template <int KIND, int WB>
static void one_bf16(const matq::HalfWords& H, uint32_t* out) {
  uint32_t A[2][4];
  matq::build_bf16<KIND, WB>(H, A);
  for (int j = 0; j < 2; ++j)
    for (int rho = 0; rho < 4; ++rho) out[4 * j + rho] = A[j][rho];
}
template <int KIND>
static void bf16_by_block(int wb, const matq::HalfWords& H, uint32_t* out) {
  switch (wb) {
    case 0: one_bf16<KIND, 0>(H, out); break;
    case 1: one_bf16<KIND, 1>(H, out); break;
    case 2: one_bf16<KIND, 2>(H, out); break;
    default: one_bf16<KIND, 3>(H, out); break;
  }
}
// bf16 operands of block W (0..7) of an operand kind, from the same lane words (the decode path
// loads them half a chunk at a time: blocks 4*hc .. 4*hc + 3)
extern "C" void build_bf16_host(int kind, int W, const uint32_t* words, uint32_t* out) {
  const int hc = W >> 2, wb = W & 3;
  matq::HalfWords H;
  for (int i = 0; i < 4; ++i) { H.p0[i] = words[4 * hc + i]; H.p3[i] = words[16 + 4 * hc + i]; H.p4[i] = words[24 + 4 * hc + i]; }
  for (int i = 0; i < 2; ++i) { H.p1[i] = words[8 + 2 * hc + i]; H.p2[i] = words[12 + 2 * hc + i]; }
  switch (kind) {
    case 0: bf16_by_block<0>(wb, H, out); break;
    case 1: bf16_by_block<1>(wb, H, out); break;
    case 2: bf16_by_block<2>(wb, H, out); break;
    case 3: bf16_by_block<3>(wb, H, out); break;
    default: bf16_by_block<4>(wb, H, out); break;
  }
}
// words: p0[8], p1[4], p2[4], p3[8], p4[8] of one lane; out: A[j][rho] at 4*j + rho
extern "C" void build_host(int r, int W, const uint32_t* words, uint32_t* out) {
  matq::LaneWords L;
  for (int i = 0; i < 8; ++i) { L.p0[i] = words[i]; L.p3[i] = words[16 + i]; L.p4[i] = words[24 + i]; }
  for (int i = 0; i < 4; ++i) { L.p1[i] = words[8 + i]; L.p2[i] = words[12 + i]; }
  switch (r) {
    case 2: by_block<2>(W, L, out); break;
    case 3: by_block<3>(W, L, out); break;
    case 4: by_block<4>(W, L, out); break;
    case 6: by_block<6>(W, L, out); break;
    default: by_block<8>(W, L, out); break;
  }
}
"""


@pytest.fixture(scope="module")
def build_host():
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("needs g++")
    os.makedirs(BUILD, exist_ok=True)
    shutil.copy(SRC, os.path.join(BUILD, "operands.cuh"))
    with open(os.path.join(BUILD, "common.cuh"), "w") as f:
        f.write(COMMON_STUB)
    cpp = os.path.join(BUILD, "operands_host.cpp")
    with open(cpp, "w") as f:
        f.write(DRIVER)
    lib = os.path.join(BUILD, "liboperands_host.so")
    subprocess.run([gxx, "-O2", "-std=c++17", "-shared", "-fPIC", "-I", BUILD, "-o", lib, cpp], check=True)
    so = ctypes.CDLL(lib)
    vp = ctypes.c_void_p

    def run(r, W, words):
        words = np.ascontiguousarray(words, dtype=np.uint32)
        out = np.zeros(8, dtype=np.uint32)
        so.build_host(r, W, words.ctypes.data_as(vp), out.ctypes.data_as(vp))
        return out

    def run_bf16(kind, W, words):
        words = np.ascontiguousarray(words, dtype=np.uint32)
        out = np.zeros(8, dtype=np.uint32)
        so.build_bf16_host(kind, W, words.ctypes.data_as(vp), out.ctypes.data_as(vp))
        return out
    run.bf16 = run_bf16
    return run


# ---- lane words of one 16 x 256 tile: the bytes of the layout model, read at the lane offsets ----

def _lane_words_of(codes):
    tile = layout_model(codes, 8)
    return {(gid, tg): tile_lane_words(tile, 4 * gid + tg) for gid in range(8) for tg in range(4)}


def _sigma(r, rho):
    if r == 2:
        return 4 ** rho
    if r in (3, 4):
        return 16 if rho >= 2 else 1
    return 1


@pytest.mark.parametrize("r", O.WIDTHS)
def test_operands_are_exact_prefix_values(build_host, r):
    rng = np.random.default_rng(r)
    codes = rng.integers(0, 256, (16, 256), dtype=np.int64)
    codes[0, :16] = [0, 255, 0x55, 0xAA, 1, 2, 4, 8, 16, 32, 64, 128, 0x7F, 0x80, 234, 0xF0]
    p = O.prefix(codes, r)
    v = p if r <= 4 else p << (8 - r)
    lanes = _lane_words_of(codes)
    for gid in range(8):
        for tg in range(4):
            words = lanes[(gid, tg)]
            for W in range(8):
                regs = build_host(r, W, words)
                halves = regs.view(np.uint16).view(np.float16).astype(np.float64).reshape(8, 2)
                for j in range(2):
                    for rho in range(4):
                        for hi in range(2):
                            row, k = _field_coords(gid, tg, W, 8 * hi + 4 * j + rho)
                            want = 1024.0 + _sigma(r, rho) * float(v[row, k])
                            got = halves[4 * j + rho, hi]
                            assert got == want, (r, gid, tg, W, j, rho, hi, got, want)


def test_every_code_reaches_every_width(build_host):
    # 128 distinct codes in the fields of lane 0 (its share of the tile), high nibbles 0..15:
    # every operand half decodes back to its own code's prefix
    codes = np.zeros((16, 256), dtype=np.int64)
    for w in range(8):
        for f in range(16):
            row, k = _field_coords(0, 0, w, f)
            codes[row, k] = 16 * (w + 8 * (f >= 8)) % 256 + (f & 15)
    words = _lane_words_of(codes)[(0, 0)]
    for r in O.WIDTHS:
        seen = set()
        for W in range(8):
            halves = build_host(r, W, words).view(np.uint16).view(np.float16).astype(np.float64).reshape(8, 2)
            for j in range(2):
                for rho in range(4):
                    for hi in range(2):
                        row, k = _field_coords(0, 0, W, 8 * hi + 4 * j + rho)
                        val = (halves[4 * j + rho, hi] - 1024.0) / _sigma(r, rho)
                        q = int(codes[row, k])
                        assert val == (q >> (8 - r)) * (1 if r <= 4 else 1 << (8 - r))
                        seen.add(q)
        assert len(seen) == 128  # lane 0 holds 128 weights of the tile


# ---- bf16 operands of the decode path ---------------------------------------------------------
# kind -> (value of the weight's code the operand carries, alpha of row half h)
BF16_KINDS = {
    0: (lambda q: q >> 6, lambda h: 4 ** h),          # plane 0: bits 7..6 (width 2)
    1: (lambda q: q >> 5, lambda h: 1),               # planes 0, 1: bits 7..5 (width 3)
    2: (lambda q: q >> 4, lambda h: 1),               # planes 0..2: bits 7..4 (width 4; high part of 6, 8)
    3: (lambda q: (q >> 2) & 3, lambda h: 4 ** h),    # plane 3: bits 3..2 (low part of width 6)
    4: (lambda q: q & 15, lambda h: 1),               # planes 3, 4: bits 3..0 (low part of width 8)
}


def _bf16_values(regs):
    # bf16 bits -> float64 (exact: the upper half of an fp32 pattern)
    halves = regs.view(np.uint16).astype(np.uint32) << 16
    return halves.view(np.float32).astype(np.float64).reshape(8, 2)


@pytest.mark.parametrize("kind", sorted(BF16_KINDS))
def test_bf16_operands_are_exact_field_values(build_host, kind):
    """Every bf16 half of every register is 128 + alpha_h * v, v the kind's field of its weight's
    code, alpha fixed by the register's row half only (so the activations need no scaling)."""
    value, alpha = BF16_KINDS[kind]
    rng = np.random.default_rng(100 + kind)
    codes = rng.integers(0, 256, (16, 256), dtype=np.int64)
    codes[0, :16] = [0, 255, 0x55, 0xAA, 1, 2, 4, 8, 16, 32, 64, 128, 0x7F, 0x80, 234, 0xF0]
    lanes = _lane_words_of(codes)
    for gid in range(8):
        for tg in range(4):
            words = lanes[(gid, tg)]
            for W in range(8):
                halves = _bf16_values(build_host.bf16(kind, W, words))
                for j in range(2):
                    for rho in range(4):
                        for hi in range(2):
                            row, k = _field_coords(gid, tg, W, 8 * hi + 4 * j + rho)
                            want = 128.0 + alpha(rho & 1) * float(value(int(codes[row, k])))
                            got = halves[4 * j + rho, hi]
                            assert got == want, (kind, gid, tg, W, j, rho, hi, got, want)


def test_bf16_parts_rebuild_every_width(build_host):
    """The decode path's parts add up to the true prefix of every width: high nibble * 4 + bits
    3..2 is the 6-bit prefix, high nibble * 16 + low nibble the code (MatGPTQ App. A.1)."""
    codes = np.arange(16 * 256, dtype=np.int64).reshape(16, 256) % 256
    lanes = _lane_words_of(codes)
    for (gid, tg) in ((0, 0), (5, 3), (7, 1)):
        words = lanes[(gid, tg)]
        for W in range(8):
            parts = {kd: _bf16_values(build_host.bf16(kd, W, words)) for kd in BF16_KINDS}
            for j in range(2):
                for rho in range(4):
                    for hi in range(2):
                        row, k = _field_coords(gid, tg, W, 8 * hi + 4 * j + rho)
                        q = int(codes[row, k])
                        v = {kd: (parts[kd][4 * j + rho, hi] - 128.0) / BF16_KINDS[kd][1](rho & 1) for kd in parts}
                        assert v[0] == O.prefix(np.array([q]), 2)[0]
                        assert v[1] == O.prefix(np.array([q]), 3)[0]
                        assert v[2] == O.prefix(np.array([q]), 4)[0]
                        assert 4 * v[2] + v[3] == O.prefix(np.array([q]), 6)[0]
                        assert 16 * v[2] + v[4] == O.prefix(np.array([q]), 8)[0]
