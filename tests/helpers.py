"""Shared helpers of the GPU parity tests: problem setup and the parity bar.

The parity bar (fp outputs) is the one the target states: elementwise
|y - ref| <= 1e-2 * (|ref| + 1) and ||y - ref||_F / ||ref||_F <= 2e-3, with ref the
fp64 oracle.  Codes and prefixes are compared bit-exactly.
"""

import numpy as np

from nested_bit_weight_msb_b200 import synth

ELEM_TOL = 1e-2
FROB_TOL = 2e-3


def check_close(y, ref, elem_tol=ELEM_TOL, frob_tol=FROB_TOL, what=""):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = np.abs(y - ref)
    bound = elem_tol * (np.abs(ref) + 1.0)
    worst = float(np.max(err / bound)) if err.size else 0.0
    assert np.all(err <= bound), f"{what}: elementwise bound exceeded (worst ratio {worst:.3g})"
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(y - ref) / nref if nref > 0 else np.linalg.norm(y - ref)
    assert rel <= frob_tol, f"{what}: relative Frobenius error {rel:.3e} > {frob_tol}"
    return rel


def problem(M, N, K, group, seed=0, outlier_frac=0.0, layer=0, proj="gate"):
    q, s, z = synth.parent_weights(N, K, group, seed=seed, layer=layer, proj=proj)
    xb, xv = synth.activations(M, K, seed=seed, layer=layer, proj=proj, outlier_frac=outlier_frac)
    return q, s, z, xb, xv


def to_device(q, s, z, xb):
    import torch
    dq = torch.from_numpy(q).cuda()
    ds = torch.from_numpy(s.view(np.int16)).cuda()
    dz = torch.from_numpy(z).cuda()
    dx = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    return dq, ds, dz, dx
