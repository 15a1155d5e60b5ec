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

HARNESS = r"""
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
        f.write(HARNESS)
    lib = os.path.join(BUILD, "liboperands_host.so")
    subprocess.run([gxx, "-O2", "-std=c++17", "-shared", "-fPIC", "-I", BUILD, "-o", lib, cpp], check=True)
    so = ctypes.CDLL(lib)
    vp = ctypes.c_void_p

    def run(r, W, words):
        words = np.ascontiguousarray(words, dtype=np.uint32)
        out = np.zeros(8, dtype=np.uint32)
        so.build_host(r, W, words.ctypes.data_as(vp), out.ctypes.data_as(vp))
        return out
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
