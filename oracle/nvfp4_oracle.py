"""CPU oracle for the NVFP4 variant of the low-rank-assisted W4A4 layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only ``tests/`` (and, once the variant has kernels, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU baseline leg) use it.  It shares no code with the CUDA
library.

What the pages fix
------------------
"DiRotQ: Rotation-Aware Quantization for 4-bit Diffusion Transformers"
(papernotes.org), section on the loss / training strategy: besides INT4 W4A4
(groups of 64), the 4-bit floating-point W4A4 setting uses the standard NVFP4
format of Blackwell: groups of 16 values sharing an FP8 scale factor.  The
layer is otherwise the one of oracle.hsq_oracle (smoothed activations X_hat,
residual R = W diag(s) - (L1 L2)^T, high-precision low-rank branch), with both
4-bit operands in NVFP4 instead of group-64 INT4.

Readings where the page is silent:
  * element format E2M1 (sign, 2 exponent bits with bias 1, 1 mantissa bit):
    magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; a 4-bit code is sign << 3 | index
    (index = exponent << 1 | mantissa, i.e. the position in that list); values
    round to the nearest magnitude, ties to the even mantissa bit, and
    saturate at 6;
  * one scale per 16 consecutive K-values, stored as FP8 E4M3 (the finite
    format: bias 7, 3 mantissa bits, subnormals m * 2^-9, largest 448), and one
    fp32 scale per tensor, g = fp32(amax(|V|) / 2688) (2688 = 6 * 448), so that
    every block scale fits E4M3: block scale b = E4M3(fp32(amax_block / fp32(6 g)))
    rounded to nearest, ties to even, saturating at 448;
  * element code = E2M1(fp32(v / fp32(b * g))); an all-zero tensor has g = 0,
    a block whose scale rounds to 0 has codes 0;
  * K is zero-padded to a multiple of 16; two codes per byte, code 2j in bits
    0-3 and code 2j+1 in bits 4-7 (the INT4 packing);
  * the value of a code is E2M1(code) * b * g, and the layer's products and
    sums are taken in fp64 here.
"""
from __future__ import annotations

import numpy as np

f32 = np.float32
f64 = np.float64

BLOCK = 16
E2M1_MAX = 6.0
E4M3_MAX = 448.0
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=f64)


# ---------------------------------------------------------------- E4M3 scale
def e4m3_round(v):
    """Nearest finite E4M3 value of each v >= 0 (fp64 array), ties to an even
    mantissa, saturating at 448.  Normal values are (1 + m/8) * 2^e for
    e in [-6, 8]; subnormals m * 2^-9."""
    v = np.asarray(v, dtype=f64)
    out = np.zeros_like(v)
    pos = v > 0
    x = np.minimum(v[pos], E4M3_MAX)
    e = np.floor(np.log2(x))
    e = np.maximum(e, -6.0)            # below 2^-6: the subnormal spacing 2^-9
    step = np.exp2(e - 3.0)            # 3 mantissa bits
    q = x / step
    r = np.rint(q)                     # numpy rint: round half to even
    out[pos] = np.minimum(r * step, E4M3_MAX)
    return out


# ---------------------------------------------------------------- E2M1 element
def e2m1_encode(t):
    """4-bit E2M1 codes of fp64 values t: nearest magnitude of E2M1_GRID, ties to
    the even index (even mantissa bit), saturating at 6; sign in bit 3."""
    t = np.asarray(t, dtype=f64)
    a = np.minimum(np.abs(t), E2M1_MAX)
    d = np.abs(a[..., None] - E2M1_GRID)             # distance to every magnitude
    best = d.min(axis=-1, keepdims=True)
    ties = d == best
    # lowest even index among the nearest, else the (single) nearest index
    even = ties & (np.arange(8) % 2 == 0)
    idx = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(ties, axis=-1))
    sign = (t < 0) & (idx > 0)
    return (idx | (sign.astype(np.int64) << 3)).astype(np.uint8)


def e2m1_value(codes):
    codes = np.asarray(codes, dtype=np.int64)
    mag = E2M1_GRID[codes & 7]
    return np.where(codes & 8, -mag, mag)


# ---------------------------------------------------------------- quantizer
def quantize_nvfp4(V):
    """NVFP4 quantization of V [rows, K] along K: returns (codes [rows, Kp]
    uint8, block scales [rows, Kp/16] fp64 holding E4M3 values, tensor scale g
    as fp32).  Kp = K rounded up to 16; padding values are 0."""
    V = np.asarray(V, dtype=f32)
    rows, K = V.shape
    Kp = -(-K // BLOCK) * BLOCK
    Vp = np.zeros((rows, Kp), dtype=f32)
    Vp[:, :K] = V
    amax = f32(np.max(np.abs(Vp))) if Vp.size else f32(0)
    g = f32(amax / f32(6.0 * E4M3_MAX))
    blocks = Vp.reshape(rows, Kp // BLOCK, BLOCK)
    bmax = np.max(np.abs(blocks), axis=2).astype(f32)
    if g == 0:
        scales = np.zeros_like(bmax, dtype=f64)
    else:
        sb = (bmax / f32(f32(6.0) * g)).astype(f32)
        scales = e4m3_round(sb.astype(f64))
    denom = (scales.astype(f32) * g).astype(f32)        # fp32(b * g)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(denom[..., None] > 0, blocks / denom[..., None], f32(0)).astype(f32)
    t = t.reshape(rows, Kp)
    codes = np.zeros((rows, Kp), dtype=np.uint8)
    for i in range(0, rows, 256):  # in row slices, to bound the encoder's temporaries
        codes[i:i + 256] = e2m1_encode(t[i:i + 256].astype(f64))
    return codes, scales, g


def dequantize_nvfp4(codes, scales, g):
    rows, Kp = codes.shape
    vals = e2m1_value(codes).reshape(rows, Kp // BLOCK, BLOCK)
    return (vals * scales[..., None] * f64(g)).reshape(rows, Kp)


def pack_fp4(codes):
    """Two 4-bit codes per byte: code 2j in bits 0-3, code 2j+1 in bits 4-7."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


# ---------------------------------------------------------------- the layer
def nvfp4_quantize_act(X, s, L1):
    """The per-forward step: X_hat = fp32(X)/s exactly as oracle.hsq_oracle forms
    it, its NVFP4 codes, block scales and tensor scale, and U = X_hat L1 in fp64."""
    from . import hsq_oracle as H  # the INT4 oracle's smoothing step
    Xh = H.smooth_activation(X, s)
    c, sc, g = quantize_nvfp4(Xh)
    if L1 is None or np.asarray(L1).shape[1] == 0:
        U = np.zeros((Xh.shape[0], 0), dtype=f64)
    else:
        U = Xh.astype(f64) @ np.asarray(L1, dtype=f64)
    return c, sc, g, U


def nvfp4_pack_weights(W, s, L1, L2):
    """Offline: the residual R = W diag(s) - (L1 L2)^T as oracle.hsq_oracle forms
    it (fp64, fixed order, one fp32 rounding), then its NVFP4 codes, block scales
    and tensor scale."""
    from . import hsq_oracle as H  # the INT4 oracle's residual step
    return quantize_nvfp4(H.residual_weight(W, s, L1, L2))


def nvfp4_linear_forward(xc, xs, xg, U, wc, ws, wg, L2, bias, K):
    """Y = deq(x) deq(w)^T + U L2 + b in fp64, from the codes [rows, Kp] (one code
    per byte), block scales [rows, Kp/16] and tensor scales of both operands;
    K is the layer's true width (the padding is dropped)."""
    Xq = dequantize_nvfp4(xc, xs, xg)[:, :K]
    Rq = dequantize_nvfp4(wc, ws, wg)[:, :K]
    Y = Xq @ Rq.T
    if U is not None and np.asarray(U).shape[1] > 0:
        Y += np.asarray(U, dtype=f64) @ np.asarray(L2, dtype=f64)
    if bias is not None:
        Y += np.asarray(bias, dtype=f64)[None, :]
    return Y


def nvfp4_layer_forward(X, W, s, L1, L2, bias):
    """Y = deq(NVFP4(X_hat)) deq(NVFP4(R))^T + (X_hat L1) L2 + b, with X_hat and
    R formed exactly as in oracle.hsq_oracle (fp32 X_hat, fp32 residual) and the
    products and sums in fp64: the three steps above in order."""
    wc, ws, wg = nvfp4_pack_weights(W, s, L1, L2)
    xc, xs, xg, U = nvfp4_quantize_act(X, s, L1)
    return nvfp4_linear_forward(xc, xs, xg, U, wc, ws, wg, L2, bias, np.asarray(X).shape[1])
