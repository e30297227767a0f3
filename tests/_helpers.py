"""Shared test helpers: tolerance checks and oracle runs on synthetic layers.

The tolerance follows the spec of the layer's output: max |dY| <= 1e-2 rms(Y_ref)
for fp32 output, and for bf16 output the same bound plus half a bf16 ulp of the
reference value (the rounding of the output alone can exceed 1e-2 rms for
|y| > 2.56 rms).  A tighter fp32 bound, 1e-4 rms, follows from the arithmetic:
the kernel rounds each of at most 192 group updates at 2^-24 relative, which
gives errors of order 1e-6 of |y|.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import hsq_oracle as O

TOL_SPEC = 1e-2
TOL_F32_TIGHT = 1e-4


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def rms(a) -> float:
    a = np.asarray(a, dtype=np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


def check_y(Y_gpu: np.ndarray, Y_ref: np.ndarray, out_f32: bool, where: str = ""):
    """Assert the spec tolerance; return (max|dY|/rms, rms)."""
    Y_gpu = np.asarray(Y_gpu, dtype=np.float64)
    Y_ref = np.asarray(Y_ref, dtype=np.float64)
    assert Y_gpu.shape == Y_ref.shape, (Y_gpu.shape, Y_ref.shape)
    assert np.all(np.isfinite(Y_gpu)), f"non-finite output {where}"
    r = rms(Y_ref)
    d = np.abs(Y_gpu - Y_ref)
    if out_f32:
        assert d.max() <= TOL_SPEC * r, f"{where}: max|dY| = {d.max():.3e} > 1e-2 rms = {TOL_SPEC * r:.3e}"
        assert d.max() <= TOL_F32_TIGHT * r, f"{where}: max|dY| = {d.max():.3e} > 1e-4 rms"
    else:
        bound = TOL_SPEC * r + 0.5 * O.bf16_ulp(Y_ref)
        bad = d > bound
        assert not bad.any(), (f"{where}: {bad.sum()} elements beyond 1e-2 rms + ulp/2; worst "
                               f"{d.max():.3e} (rms {r:.3e})")
    return (float(d.max()) / r if r > 0 else float(d.max())), r


def oracle_layer(X, W, s, L1, L2, bias, rows=None, group=O.GROUP):
    """Oracle outputs for a layer given torch CPU tensors (bf16 / fp32).
    ``rows`` restricts the activation side to those token rows."""
    Xn = to_np(X)
    if rows is not None:
        Xn = Xn[rows]
    Wn, sn = to_np(W), to_np(s)
    L1n = None if L1 is None else to_np(L1)
    L2n = None if L2 is None else to_np(L2)
    bn = None if bias is None else to_np(bias)
    wc, ws = O.pack_weights(Wn, sn, L1n, L2n, group)
    xc, xs, U = O.quantize_act(Xn, sn, L1n, group)
    Y = O.linear_forward(xc, xs, U, wc, ws, L2n, bn, group)
    return dict(w_codes=wc, w_scales=ws, x_codes=xc, x_scales=xs, U=U, Y=Y)


def pad_scales(sc: np.ndarray, ld: int) -> np.ndarray:
    """Oracle scales [G, rows] -> the library's [G, ld] layout (zero padding)."""
    G, rows = sc.shape
    out = np.zeros((G, ld), dtype=np.float32)
    out[:, :rows] = sc
    return out
