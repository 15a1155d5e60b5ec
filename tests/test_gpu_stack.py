"""GPU parity of the Mix'n'Match stack glue and of a small mixed-width FFN stack.

Each step is checked teacher-forced: the oracle gets the GPU's own input for that step
(RMSNorm of the GPU's residual stream, the projections of the GPU's normalised input, the
gated product of the GPU's gate/up outputs, the down projection of the GPU's product), at the
stated tolerance.  The end-to-end deviation of the whole stack from an fp64 run of the oracle
alone is reported (and only checked to be finite and small in a loose sense).
"""

import numpy as np
import pytest

import oracle as O
from helpers import check_close
from nested_bit_weight_msb_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from nested_bit_weight_msb_b200 import matq
    return matq


def _bf16(t):
    return t.float().cpu().numpy().astype(np.float64)


def _rne_bf16(a):
    """fp64 values rounded to the nearest bf16 (ties to even), as fp64."""
    return synth.bf16_round(np.asarray(a, dtype=np.float32))[1].astype(np.float64)


@pytest.mark.parametrize("Mt,D", [(1, 4096), (16, 4096), (33, 1000)])
def test_rmsnorm(M, Mt, D):
    import torch
    rng = np.random.default_rng(D + Mt)
    h = (rng.standard_normal((Mt, D)) * rng.uniform(0.1, 30)).astype(np.float32)
    n = M.rmsnorm(torch.from_numpy(h).cuda(), eps=1e-5)
    check_close(_bf16(n), O.rmsnorm(h, 1e-5), what="rmsnorm")


@pytest.mark.parametrize("Mt,F", [(1, 14336), (16, 14336), (3, 1001)])
def test_silu_mul(M, Mt, F):
    import torch
    rng = np.random.default_rng(F + Mt)
    gb, gv = synth.bf16_round((rng.standard_normal((Mt, F)) * 3).astype(np.float32))
    ub, uv = synth.bf16_round(rng.standard_normal((Mt, F)).astype(np.float32))
    g = torch.from_numpy(gb.view(np.int16)).cuda().view(torch.bfloat16)
    u = torch.from_numpy(ub.view(np.int16)).cuda().view(torch.bfloat16)
    a = M.silu_mul(g, u)
    check_close(_bf16(a), O.gated_product(gv, uv), what="silu_mul")


@pytest.mark.parametrize("Mt,F", [(1, 14336), (16, 14336), (3, 1001), (5, 24)])
def test_silu_mul_gu(M, Mt, F):
    """Gated product read from the two halves of one fused gate+up output [M, 2F]."""
    import torch
    rng = np.random.default_rng(F + 7 * Mt)
    gub, guv = synth.bf16_round((rng.standard_normal((Mt, 2 * F)) * 3).astype(np.float32))
    gu = torch.from_numpy(gub.view(np.int16)).cuda().view(torch.bfloat16)
    a = M.silu_mul_gu(gu)
    check_close(_bf16(a), O.gated_product(guv[:, :F], guv[:, F:]), what="silu_mul_gu")


@pytest.mark.parametrize("Mt,r", [(1, 2), (16, 4), (40, 3)])
def test_fused_gate_up_block(M, Mt, r):
    """One sliced linear over the row-concatenated [W_gate; W_up] pack, then the gated product
    from its halves: teacher-forced against the oracle's separate gate and up projections."""
    import torch
    D, F, G = 512, 1024, 128
    host = {name: synth.parent_weights(F, D, G, seed=4, layer=0, proj=name) for name in ("gate", "up")}
    q = np.concatenate([host["gate"][0], host["up"][0]], axis=0)
    s = np.concatenate([host["gate"][1], host["up"][1]], axis=0)
    z = np.concatenate([host["gate"][2], host["up"][2]], axis=0)
    planes = M.pack(torch.from_numpy(q).cuda(), r_keep=8)
    xb, xv = synth.activations(Mt, D, seed=6)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    gu = M.linear(x, planes, 8, torch.from_numpy(s.view(np.int16)).cuda(), torch.from_numpy(z).cuda(), 2 * F, r, G)
    g_ref = O.linear(xv.astype(np.float64), *host["gate"], r, G)
    u_ref = O.linear(xv.astype(np.float64), *host["up"], r, G)
    check_close(_bf16(gu)[:, :F], g_ref, what="fused gate half")
    check_close(_bf16(gu)[:, F:], u_ref, what="fused up half")
    a = M.silu_mul_gu(gu)
    check_close(_bf16(a), O.gated_product(_bf16(gu)[:, :F], _bf16(gu)[:, F:]), what="fused gated product")


def _interleave(a, b):
    """Rows 2i = a[i], 2i + 1 = b[i]."""
    out = np.empty((2 * a.shape[0],) + a.shape[1:], dtype=a.dtype)
    out[0::2] = a
    out[1::2] = b
    return out


@pytest.mark.parametrize("Mt,r,group", [(1, 2, 128), (5, 3, 64), (16, 8, 128), (17, 4, 128), (40, 6, 64),
                                        (300, 4, 128)])
def test_gated_output_mode(M, Mt, r, group):
    """MATQ_OUT_SILU_GATED: one call over the row-interleaved [gate; up] pack writes
    silu(gate) * up directly (decode path M <= 16, prefill above, ragged token tiles),
    compared with the fp64 oracle's separate projections and gated product."""
    import torch
    D, F = 512, 1000
    host = {nm: synth.parent_weights(F, D, group, seed=8, layer=1, proj=nm) for nm in ("gate", "up")}
    q, s, z = (_interleave(host["gate"][i], host["up"][i]) for i in range(3))
    planes = M.pack(torch.from_numpy(q).cuda(), r_keep=8)
    xb, xv = synth.activations(Mt, D, seed=10)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    a = M.linear(x, planes, 8, torch.from_numpy(s.view(np.int16)).cuda(), torch.from_numpy(z).cuda(), 2 * F, r,
                 group, y_mode=M.MATQ_OUT_SILU_GATED)
    assert tuple(a.shape) == (Mt, F) and a.dtype == torch.bfloat16
    g = O.linear(xv.astype(np.float64), *host["gate"], r, group)
    u = O.linear(xv.astype(np.float64), *host["up"], r, group)
    check_close(_bf16(a), O.gated_product(g, u), what=f"gated M={Mt} r={r}")


@pytest.mark.parametrize("Mt", [1, 16, 2048])
def test_gated_output_mode_8b_sampled(M, Mt):
    """The gated mode at the 8B FFN shape (interleaved [28672, 4096], group 128) in the bench's
    launch configuration.  Two checks per width: (1) the same call in fp32 output mode (the
    same accumulation) gives gate and up within the parity tolerance of the oracle, on sampled
    columns; (2) the gated output equals the fp64 gated product of those fp32 results up to its
    bf16 rounding, on every column.  (With the 1% outlier channels of the prefill workload, g
    and u reach tens to hundreds, and silu(g) * u multiplies g's admissible absolute error by
    |u|; a direct bound on the product would test conditioning, not the kernel.)"""
    import torch
    D, F, G = 4096, 14336, 128
    host = {nm: synth.parent_weights(F, D, G, seed=0, proj=nm) for nm in ("gate", "up")}
    q, s, z = (_interleave(host["gate"][i], host["up"][i]) for i in range(3))
    planes = M.pack(torch.from_numpy(q).cuda(), r_keep=8)
    ds, dz = torch.from_numpy(s.view(np.int16)).cuda(), torch.from_numpy(z).cuda()
    xb, xv = synth.activations(Mt, D, seed=0, outlier_frac=0.01 if Mt > 16 else 0.0)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    cols = np.sort(np.random.default_rng(Mt).choice(F, 256, replace=False))
    for r in ((2, 4, 8) if Mt <= 16 else (3, 4, 8)):
        a = M.linear(x, planes, 8, ds, dz, 2 * F, r, G, y_mode=M.MATQ_OUT_SILU_GATED)
        y32 = M.linear(x, planes, 8, ds, dz, 2 * F, r, G, y_mode=M.MATQ_OUT_F32).cpu().numpy().astype(np.float64)
        g32, u32 = y32[:, 0::2], y32[:, 1::2]
        check_close(g32[:, cols], O.linear(xv.astype(np.float64), *(h[cols] for h in host["gate"]), r, G),
                    what=f"gate M={Mt} r={r}")
        check_close(u32[:, cols], O.linear(xv.astype(np.float64), *(h[cols] for h in host["up"]), r, G),
                    what=f"up M={Mt} r={r}")
        ref = O.gated_product(g32, u32)
        err = np.abs(_bf16(a) - ref)
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-6), f"gated epilogue M={Mt} r={r}: {err.max():.3g}"


@pytest.mark.parametrize("alloc", ["fixed", "pyramid"])
@pytest.mark.parametrize("Mt", [1, 16, 40])
def test_mixnmatch_stack_teacher_forced(M, Mt, alloc):
    """A four-layer stack with one width per layer: a fixed mix, and the Pyramid allocation of
    4 effective bits over widths {2, 4, 8} (middle layers widest)."""
    import torch
    from nested_bit_weight_msb_b200 import mixnmatch
    D, F, G, L = 512, 1024, 128, 4
    widths = [2, 4, 3, 8] if alloc == "fixed" else mixnmatch.allocate_widths(L, 4.0, "pyramid", (2, 4, 8))
    layers = []
    for l in range(L):
        lay = {}
        for name, (N, K) in (("gate", (F, D)), ("up", (F, D)), ("down", (D, F))):
            q, s, z = synth.parent_weights(N, K, G, seed=3, layer=l, proj=name)
            dq = torch.from_numpy(q).cuda()
            lay[name] = dict(host=(q, s, z), planes=M.pack(dq, r_keep=widths[l]),
                             s=torch.from_numpy(s.view(np.int16)).cuda(), z=torch.from_numpy(z).cuda(), N=N)
        layers.append(lay)
    xb, xv = synth.activations(Mt, D, seed=5)
    h = torch.from_numpy(xv.copy()).cuda()           # fp32 residual stream
    ws = M.workspace(Mt, F, F, G)
    h_ref = xv.astype(np.float64)                     # oracle-only run, for the reported deviation
    for l, lay in enumerate(layers):
        r = widths[l]
        n = M.rmsnorm(h, eps=1e-5)
        check_close(_bf16(n), O.rmsnorm(h.cpu().numpy(), 1e-5), what=f"layer {l} rmsnorm")
        outs = {}
        for name in ("gate", "up"):
            p = lay[name]
            outs[name] = M.linear(n, p["planes"], r, p["s"], p["z"], p["N"], r, G, workspace=ws)
            check_close(_bf16(outs[name]), O.linear(_bf16(n), *p["host"], r, G), what=f"layer {l} {name}")
        a = M.silu_mul(outs["gate"], outs["up"])
        check_close(_bf16(a), O.gated_product(_bf16(outs["gate"]), _bf16(outs["up"])), what=f"layer {l} silu")
        h_before = h.cpu().numpy().astype(np.float64)
        p = lay["down"]
        M.linear(a, p["planes"], r, p["s"], p["z"], p["N"], r, G, y=h, y_mode=M.MATQ_OUT_F32_ACCUM, workspace=ws)
        check_close(h.cpu().numpy() - h_before, O.linear(_bf16(a), *p["host"], r, G), what=f"layer {l} down")
        h_ref = O.ffn_block(h_ref, {k: v["host"] for k, v in lay.items()}, r, G)
    assert M.workspace_status(ws) == 0
    dev = np.linalg.norm(h.cpu().numpy() - h_ref) / np.linalg.norm(h_ref)
    print(f"end-to-end stack deviation (M={Mt}): {dev:.3e}")
    assert np.isfinite(dev) and dev < 5e-2


@pytest.mark.parametrize("Mt", [1, 16, 512])
def test_mixnmatch_stack_8b_shapes_sampled(M, Mt):
    """The Mix'n'Match stack at the 8B FFN shapes (D = 4096, F = 14336, group 128), three layers
    with the first widths of the seeded {2 x 11, 3 x 10, 4 x 11} permutation, gate and up served
    by one fused call, the residual kept in fp32 by the accumulate mode.  Decode path for
    M = 1, 16, tcgen05 prefill path for M = 512.  Every step is checked teacher-forced: the
    projections on 512 sampled output columns, the elementwise gated product on all of them
    (a few dozen bf16-rounded values alone can exceed the Frobenius bar by chance)."""
    import torch
    D, F, G, L = 4096, 14336, 128, 3
    widths = synth.mixnmatch_widths(seed=0)[:L]
    rng = np.random.default_rng(Mt)
    xb, xv = synth.activations(Mt, D, seed=9)
    h = torch.from_numpy(xv.copy()).cuda()
    ws = M.workspace(Mt, F, 2 * F, G)
    for l in range(L):
        r = int(widths[l])
        host = {nm: synth.parent_weights(N, K, G, seed=1, layer=l, proj=nm)
                for nm, (N, K) in (("gate", (F, D)), ("up", (F, D)), ("down", (D, F)))}
        gu = tuple(np.concatenate([host["gate"][i], host["up"][i]], axis=0) for i in range(3))
        p_gu = M.pack(torch.from_numpy(gu[0]).cuda(), r_keep=4)      # mode A: keep 4 bits
        p_dn = M.pack(torch.from_numpy(host["down"][0]).cuda(), r_keep=4)
        n = M.rmsnorm(h, eps=1e-5)
        nv = _bf16(n)
        y_gu = M.linear(n, p_gu, 4, torch.from_numpy(gu[1].view(np.int16)).cuda(), torch.from_numpy(gu[2]).cuda(),
                        2 * F, r, G, workspace=ws)
        cols = np.sort(rng.choice(F, 512, replace=False))
        for half, nm in ((0, "gate"), (1, "up")):
            q, s, z = host[nm]
            got = _bf16(y_gu)[:, half * F + cols]
            check_close(got, O.linear(nv, q[cols], s[cols], z[cols], r, G), what=f"layer {l} {nm} M={Mt}")
        a = M.silu_mul_gu(y_gu)
        av = _bf16(a)
        gv = _bf16(y_gu)
        check_close(av, O.gated_product(gv[:, :F], gv[:, F:]), what=f"layer {l} silu M={Mt}")
        h_before = h.cpu().numpy().astype(np.float64)
        q, s, z = host["down"]
        M.linear(a, p_dn, 4, torch.from_numpy(s.view(np.int16)).cuda(), torch.from_numpy(z).cuda(), D, r, G,
                 y=h, y_mode=M.MATQ_OUT_F32_ACCUM, workspace=ws)
        dcols = np.sort(rng.choice(D, 512, replace=False))
        check_close(h.cpu().numpy()[:, dcols] - h_before[:, dcols], O.linear(av, q[dcols], s[dcols], z[dcols], r, G),
                    what=f"layer {l} down M={Mt}")
    assert M.workspace_status(ws) == 0


def test_stack32_decode_teacher_forced_sampled(M):
    """The 32-layer Mix'n'Match stack exactly as the stack benchmark serves it (8B FFN shapes,
    group 128, widths from the seeded {2 x 11, 3 x 10, 4 x 11} permutation, every layer packed
    keeping only its width's planes, gate+up in one gated call, down accumulating into the fp32
    residual) at M = 1, checked teacher-forced at every layer: the RMSNorm on all columns, the
    gated product on 256 sampled columns, the residual update on 256 sampled columns.  The whole
    pass replayed as the benchmark's CUDA graph must reproduce the layer-by-layer result bit for
    bit (the kernels sum their partial results in a fixed order)."""
    import torch
    import bench
    weights = bench.host_weights()
    sb = bench.StackBench(weights, torch.device("cuda", 0), 0)
    fused = bench.fused_weights(weights)
    perms = bench.stack_perms()
    D, F, G = bench.D_MODEL, bench.D_FF, bench.GROUP
    rng = np.random.default_rng(32)
    h = sb.h[1]
    h.copy_(sb.h0[1])
    for l, lay in enumerate(sb.layers):
        r = lay["r"]
        gu, dn = bench.stack_layer_host(fused, perms, l)
        h_in = h.cpu().numpy().astype(np.float64)
        sb.layer(lay, 1, h)
        torch.cuda.synchronize()
        nv = _bf16(sb.n[1])
        # both glue outputs are bf16 by definition (bf16 of the fp32 result), so the reference is
        # the oracle's value rounded to bf16 (unrounded, bf16's own spacing alone is ~2e-3 RMS)
        check_close(nv, _rne_bf16(O.rmsnorm(h_in, 1e-5)), what=f"layer {l} rmsnorm")
        cols = np.sort(rng.choice(F, 256, replace=False))
        g = O.linear(nv, gu[0][2 * cols], gu[1][2 * cols], gu[2][2 * cols], r, G)
        u = O.linear(nv, gu[0][2 * cols + 1], gu[1][2 * cols + 1], gu[2][2 * cols + 1], r, G)
        av = _bf16(sb.a[1])
        check_close(av[:, cols], _rne_bf16(O.gated_product(g, u)), what=f"layer {l} (r={r}) gated gate+up")
        dcols = np.sort(rng.choice(D, 256, replace=False))
        check_close(h.cpu().numpy().astype(np.float64)[:, dcols] - h_in[:, dcols],
                    O.linear(av, dn[0][dcols], dn[1][dcols], dn[2][dcols], r, G), what=f"layer {l} (r={r}) down")
    assert sb.matq.workspace_status(sb.ws) == 0
    h_eager = h.clone()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        sb.run(1)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            sb.run(1)
        h.zero_()
        graph.replay()
        torch.cuda.synchronize()
    assert torch.equal(h, h_eager)
    assert sb.matq.workspace_status(sb.ws) == 0
