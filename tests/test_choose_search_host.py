"""The cell search of the parent-code choice kernel, compiled for the host, against the oracle's
brute force over all 256 codes ("MatGPTQ: Efficient and Accurate Inference over Nested
Quantized Models", §3.2 item 2; App. A.2).

The device functions of csrc/choose.cu (from the parameter struct to choose_one) are compiled
with g++ under a few definitions that map the CUDA rounding intrinsics to plain IEEE fp32
operations (no contraction), so the search takes the same decisions as on the GPU.  The one
approximate operation, the division that estimates the nearest level, only places the search
window, whose correctness does not depend on it.  This runs the search on far more inputs than
the GPU tests do -- every width set, both reconstruction rules, weights placed on and next to
level boundaries, scales from the smallest fp16 subnormal to 300 -- without a GPU.  The oracle
shares no code with it.
"""

import ctypes
import itertools
import os
import re
import shutil
import subprocess

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "nested_bit_weight_msb_b200", "csrc", "choose.cu")
BUILD = os.path.join(ROOT, "tests", "_build")

PRELUDE = r"""
#include <algorithm>
#include <cmath>
#include <cstdint>
#define __device__
#define __forceinline__ inline
#define __noinline__ __attribute__((noinline))
struct __half { uint16_t x; };
static inline float __fsub_rn(float a, float b) { return a - b; }
static inline float __fadd_rn(float a, float b) { return a + b; }
static inline float __fmul_rn(float a, float b) { return a * b; }
static inline float __fdividef(float a, float b) { return a / b; }
static inline int __float2int_rn(float x) { return (int)std::nearbyint(x); }
using std::isnan; using std::max; using std::min;
namespace matq {
"""

HARNESS = r"""
}  // namespace matq
extern "C" void choose_host(const float* w, const float* s, const float* z, int n, int nw, const int* r,
                            const float* lam, int truncate, int force_scan, uint8_t* out) {
  matq::ChooseParams P{};
  P.nw = nw;
  P.fast = force_scan ? 0 : 1;
  for (int i = 0; i < nw; ++i) {
    P.r[i] = r[i];
    P.lam[i] = lam[i];
    P.delta[i] = truncate ? 0.f : (float)((1 << (8 - r[i])) - 1) * 0.5f;
    P.cell[i] = (float)(1 << (8 - r[i]));
    if (!(lam[i] <= 1e20f)) P.fast = 0;
  }
  for (int i = 0; i < n; ++i) {
    switch (nw) {
      case 1: out[i] = matq::choose_one<1>(w[i], s[i], z[i], P); break;
      case 2: out[i] = matq::choose_one<2>(w[i], s[i], z[i], P); break;
      case 3: out[i] = matq::choose_one<3>(w[i], s[i], z[i], P); break;
      case 4: out[i] = matq::choose_one<4>(w[i], s[i], z[i], P); break;
      default: out[i] = matq::choose_one<5>(w[i], s[i], z[i], P); break;
    }
  }
}
"""


def _search_source():
    text = open(SRC).read()
    start = text.index("struct ChooseParams")
    m = re.search(r"template <int NW>\n__device__ __forceinline__ uint8_t choose_one\(.*?\n}\n", text[start:], re.S)
    assert m, "choose_one not found in choose.cu"
    return text[start:start + m.end()]


@pytest.fixture(scope="module")
def search():
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("needs g++")
    os.makedirs(BUILD, exist_ok=True)
    cpp = os.path.join(BUILD, "choose_search_host.cpp")
    lib = os.path.join(BUILD, "libchoose_search_host.so")
    with open(cpp, "w") as f:
        f.write(PRELUDE + _search_source() + HARNESS)
    subprocess.run([gxx, "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
                    "-o", lib, cpp], check=True)
    so = ctypes.CDLL(lib)
    vp = ctypes.c_void_p

    def run(w, s32, z32, widths, lam, mode, force_scan=False):
        w = np.ascontiguousarray(w, dtype=np.float32).ravel()
        s32 = np.ascontiguousarray(s32, dtype=np.float32).ravel()
        z32 = np.ascontiguousarray(z32, dtype=np.float32).ravel()
        out = np.empty(w.size, dtype=np.uint8)
        r = (ctypes.c_int * len(widths))(*widths)
        lv = (ctypes.c_float * len(lam))(*[float(np.float32(v)) for v in lam])
        so.choose_host(w.ctypes.data_as(vp), s32.ctypes.data_as(vp), z32.ctypes.data_as(vp), w.size, len(widths),
                       r, lv, int(mode == "truncate"), int(force_scan), out.ctypes.data_as(vp))
        return out
    return run


SUBSETS = [c for n in range(1, 6) for c in itertools.combinations(O.WIDTHS, n)]
G = 64


def _problem(rng, N=8, K=128):
    s = (rng.choice([6e-8, 1e-5, 3e-4, 0.01, 2.0, 300.0], size=(N, K // G))
         * rng.uniform(0.5, 2.0, (N, K // G))).astype(np.float16)
    z = rng.integers(0, 256, (N, K // G)).astype(np.uint8)
    s32 = np.repeat(s.astype(np.float32), G, 1)
    z32 = np.repeat(z.astype(np.float32), G, 1)
    # code-space positions on and next to level boundaries and cell centres, inside and past
    # the grid
    base = rng.integers(-8, 264, (N, K)).astype(np.float64)
    frac = rng.choice([0.0, 0.5, 0.25, 1e-6, -1e-6, 0.5 + 1e-6, 0.5 - 1e-6], size=(N, K))
    frac = frac + rng.uniform(-0.02, 0.02, (N, K)) * (rng.random((N, K)) < 0.5)
    w = (s32 * (base + frac - z32)).astype(np.float32)
    return w, s, z, s32, z32


@pytest.mark.parametrize("mode", ["true_prefix", "truncate"])
def test_every_width_set_on_boundary_inputs(search, mode):
    rng = np.random.default_rng(0 if mode == "true_prefix" else 1)
    for widths in SUBSETS:
        for _ in range(3):
            w, s, z, s32, z32 = _problem(rng)
            lam = rng.choice([0.0, 0.3, 1.0, 1.0 / 3, 2.5], size=len(widths)).astype(np.float32)
            want = O.choose_codes(w, s, z, G, widths, lam, mode).ravel()
            got = search(w, s32, z32, widths, lam, mode)
            assert np.array_equal(got, want), (widths, mode, lam, int((got != want).sum()))


def test_scan_path_and_special_inputs(search):
    rng = np.random.default_rng(2)
    w, s, z, s32, z32 = _problem(rng)
    w[0, :6] = [np.nan, np.inf, -np.inf, 3e7, -3e7, 0.0]
    for widths, lam in (((3, 4, 8), [1 / 3] * 3), ((2, 8), [1.0, 1.0]), ((3, 8), [0.0, 0.0]),
                        ((2, 4, 8), [1e25, 1.0, 1.0]), ((4,), [1.0])):
        for mode in ("true_prefix", "truncate"):
            with np.errstate(invalid="ignore", over="ignore"):
                want = O.choose_codes(w, s, z, G, widths, lam, mode).ravel()
            assert np.array_equal(search(w, s32, z32, widths, lam, mode), want), (widths, lam, mode)
            # the literal 256-candidate scan gives the same codes everywhere
            assert np.array_equal(search(w, s32, z32, widths, lam, mode, force_scan=True), want)
