"""CPU oracle for the low-rank-assisted W4A4 linear layer (H-SVDQuant forward).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg use it.  It shares no code with the CUDA library.

What it computes, and where the pages fix it
--------------------------------------------
Source: "Deflating the Hessian: Rank-4 W4A4 Quantization for Multimodal
Diffusion Transformers" (Wang, Zhao, Yuan; arXiv 2610.11315) as summarised on
shd-paper.top, thelatestinai.com and rit.work.

* Abstract: each weight is split into a low-bit residual plus a high-precision
  low-rank component, with 4-bit weights AND 4-bit activations (W4A4).
* Table 1 caption / Table 8 caption: all W4A4 results use group size 64.
* rit.work blog, section "How Hessian deflation separates the branches",
  paragraph on diagonal scaling: a diagonal rescaling moves range between
  weights and activations without changing the layer's full-precision map.

Together:  Y = Q4(X_hat) Q4(R)^T + (X_hat L1) L2 + b, with
X_hat = X diag(s)^-1 and R = W diag(s) - (L1 L2)^T  (W stored [N, K]).

Readings taken where the pages are silent:
  * symmetric signed INT4, codes in [-7, 7], scale = absmax / 7 in fp32 with
    IEEE division, code = round-half-even(fp32(x / scale)), clamp to [-7, 7];
  * an all-zero group has scale 0 and codes 0;
  * K is zero-padded up to a multiple of 64;
  * X_hat is fp32(fp32(X) / s_k) (division), and the same fp32 X_hat feeds
    both the quantizer and the low-rank branch;
  * R is formed in fp64 in a fixed order (sum over j of L1[k,j]*L2[j,n],
    each operation rounded, no fused multiply-add) and rounded once to fp32;
  * the branch (X_hat L1) L2 and the bias are evaluated here in fp64;
  * scales are stored group-major ([G][rows]); packed codes hold code 2j in
    bits 0-3 and code 2j+1 in bits 4-7 of byte j, 4-bit two's complement.

The quantizer decides integers from fp32 arithmetic, so those steps are done
in fp32 exactly as stated (numpy float32 division is IEEE round-to-nearest);
everything else is fp64.  Matrix products use numpy's BLAS as a primitive;
integer partial sums are exact in fp64 because |partial| <= 64*49 < 2^53.
"""
from __future__ import annotations

import numpy as np

GROUP = 64
QMAX = 7

f32 = np.float32
f64 = np.float64


def num_groups(K: int, group: int = GROUP) -> int:
    return -(-K // group)


def padded_k(K: int, group: int = GROUP) -> int:
    return num_groups(K, group) * group


# --------------------------------------------------------------------------
# smoothing  (rit.work blog: diagonal scaling keeps the FP transform)
# --------------------------------------------------------------------------
def smooth_activation(X, s, exact: bool = False):
    """X_hat = X diag(s)^-1.

    Default: fp32(fp32(X) / s) per element (the quantizer's input).
    ``exact=True`` returns the same quotient in fp64 (used by the invariant
    that the unquantized layer equals X W^T).
    """
    X = np.asarray(X)
    s = np.asarray(s, dtype=f32)
    if exact:
        return X.astype(f64) / s.astype(f64)[None, :]
    return X.astype(f32) / s[None, :]


def residual_weight(W, s, L1, L2, exact: bool = False):
    """R = W diag(s) - (L1 L2)^T   (Abstract: low-bit residual + low-rank part).

    W [N, K], s [K], L1 [K, r], L2 [r, N].  W_hat[n,k] = W[n,k]*s[k] is exact in
    fp64 (a bf16 times an fp32).  The low-rank term lr[n,k] = sum_j L1[k,j]*L2[j,n]
    is accumulated for j = 0..r-1 with one rounding per multiply and per add.
    Returned as fp32 (rounded once) unless ``exact``.
    """
    W = np.asarray(W, dtype=f64)
    s = np.asarray(s, dtype=f32).astype(f64)
    N, K = W.shape
    W_hat = W * s[None, :]
    lr = np.zeros((N, K), dtype=f64)
    if L1 is not None:
        L1 = np.asarray(L1, dtype=f64)
        L2 = np.asarray(L2, dtype=f64)
        for j in range(L1.shape[1]):
            lr = lr + np.outer(L2[j, :], L1[:, j])
    R = W_hat - lr
    return R if exact else R.astype(f32)


# --------------------------------------------------------------------------
# group-64 symmetric INT4 quantizer  (Abstract: W4A4; Table 1 caption: group-64)
# --------------------------------------------------------------------------
def quantize_groups(V, group: int = GROUP):
    """Quantize the rows of fp32 ``V`` [rows, K] in groups of ``group`` along K.

    Returns (codes int8 [rows, Kp], scales fp32 [rows, G]).  For each group:
    scale = fp32(absmax / 7); code = clamp(rint(fp32(v / scale)), -7, 7), ties to
    even; a group whose absmax is 0 gets scale 0 and codes 0.
    """
    V = np.asarray(V, dtype=f32)
    rows, K = V.shape
    G = num_groups(K, group)
    Kp = G * group
    Vp = np.zeros((rows, Kp), dtype=f32)
    Vp[:, :K] = V
    Vg = Vp.reshape(rows, G, group)
    absmax = np.abs(Vg).max(axis=2)
    scale = (absmax / f32(QMAX)).astype(f32)
    safe = np.where(scale == 0, f32(1), scale).astype(f32)
    ratio = (Vg / safe[:, :, None]).astype(f32)
    q = np.rint(ratio)
    q = np.where(scale[:, :, None] == 0, f32(0), q)
    q = np.clip(q, -QMAX, QMAX).astype(np.int8)
    return q.reshape(rows, Kp), scale


def dequantize_groups(codes, scales, group: int = GROUP):
    """codes [rows, Kp] int8, scales [rows, G] -> fp64 values code*scale."""
    codes = np.asarray(codes, dtype=f64)
    rows, Kp = codes.shape
    G = Kp // group
    sc = np.asarray(scales, dtype=f64).reshape(rows, G, 1)
    return (codes.reshape(rows, G, group) * sc).reshape(rows, Kp)


def pack_int4(codes):
    """Two 4-bit two's-complement codes per byte: code 2j -> bits 0-3, 2j+1 -> 4-7."""
    q = np.asarray(codes).astype(np.int16)
    lo = q[:, 0::2] & 0xF
    hi = q[:, 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(packed):
    """Inverse of pack_int4: uint8 [rows, Kp/2] -> int8 [rows, Kp]."""
    b = np.asarray(packed, dtype=np.uint8).astype(np.int16)
    lo = b & 0xF
    hi = b >> 4
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((b.shape[0], 2 * b.shape[1]), dtype=np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


# --------------------------------------------------------------------------
# the three calls of the layer
# --------------------------------------------------------------------------
def pack_weights(W, s, L1, L2, group: int = GROUP):
    """Offline: R = W diag(s) - (L1 L2)^T, quantized group-wise.

    Returns (w_codes uint8 [N, Kp/2], w_scales fp32 [G, N]) in the library's
    layouts (scales group-major).
    """
    R = residual_weight(W, s, L1, L2)
    q, sc = quantize_groups(R, group)
    return pack_int4(q), np.ascontiguousarray(sc.T)


def quantize_act(X, s, L1, group: int = GROUP):
    """Online: X_hat = X diag(s)^-1 quantized group-wise, plus U = X_hat L1.

    Returns (x_codes uint8 [M, Kp/2], x_scales fp32 [G, M], U fp64 [M, r]).
    U is the low-rank branch's down-projection of the same fp32 X_hat,
    evaluated in fp64.
    """
    Xh = smooth_activation(X, s)
    q, sc = quantize_groups(Xh, group)
    M = Xh.shape[0]
    if L1 is None or np.asarray(L1).shape[1] == 0:
        U = np.zeros((M, 0), dtype=f64)
    else:
        U = Xh.astype(f64) @ np.asarray(L1, dtype=f64)
    return pack_int4(q), np.ascontiguousarray(sc.T), U


def linear_forward(x_codes, x_scales, U, w_codes, w_scales, L2, bias, group: int = GROUP):
    """Y = sum_g sx[m,g] sw[n,g] P_g[m,n] + U L2 + b   (fp64).

    P_g[m,n] = sum_{k in group g} qx[m,k] qw[n,k] is the exact integer partial of
    group g; each is scaled by the product of the two group scales, which is the
    same as multiplying the dequantized operands Q4(X_hat) Q4(R)^T.
    """
    qx = unpack_int4(x_codes).astype(f64)
    qw = unpack_int4(w_codes).astype(f64)
    sx = np.asarray(x_scales, dtype=f64)   # [G, M]
    sw = np.asarray(w_scales, dtype=f64)   # [G, N]
    M, Kp = qx.shape
    N = qw.shape[0]
    G = Kp // group
    Y = np.zeros((M, N), dtype=f64)
    for g in range(G):
        ks = slice(g * group, (g + 1) * group)
        P = qx[:, ks] @ qw[:, ks].T
        Y += (sx[g][:, None] * sw[g][None, :]) * P
    if U is not None and np.asarray(U).shape[1] > 0:
        Y += np.asarray(U, dtype=f64) @ np.asarray(L2, dtype=f64)
    if bias is not None:
        Y += np.asarray(bias, dtype=f64)[None, :]
    return Y


def layer_forward(X, W, s, L1, L2, bias, group: int = GROUP):
    """All three steps in order: pack, quantize the activations, forward."""
    w_codes, w_scales = pack_weights(W, s, L1, L2, group)
    x_codes, x_scales, U = quantize_act(X, s, L1, group)
    return linear_forward(x_codes, x_scales, U, w_codes, w_scales, L2, bias, group)


def unquantized_forward(X, W, s, L1, L2, bias):
    """The same decomposition with quantization switched off, all in fp64:
    X_hat R^T + (X_hat L1) L2 + b.  By the smoothing paragraph of the rit.work
    blog this must equal the dense X W^T + b."""
    Xh = smooth_activation(X, s, exact=True)
    R = residual_weight(W, s, L1, L2, exact=True)
    Y = Xh @ R.T
    if L1 is not None and np.asarray(L1).shape[1] > 0:
        Y += (Xh @ np.asarray(L1, dtype=f64)) @ np.asarray(L2, dtype=f64)
    if bias is not None:
        Y += np.asarray(bias, dtype=f64)[None, :]
    return Y


def dense_forward(X, W, bias):
    """Plain fp64 X W^T + b (the layer before any decomposition)."""
    Y = np.asarray(X, dtype=f64) @ np.asarray(W, dtype=f64).T
    if bias is not None:
        Y += np.asarray(bias, dtype=f64)[None, :]
    return Y


def lowrank_init(W, s, r):
    """Plain truncated-SVD initialisation of the low-rank pair.

    The pages name it as the "Plain SVD" row of the L1-initialisation ablation
    (Table 6 of the paper, shd-paper.top): the protected subspace L1 is taken
    from the singular vectors of the smoothed weight.  Reading: L1 [K, r] holds
    the top-r right singular vectors of W_hat = W diag(s) (orthonormal columns,
    the protected subspace of Figure 1's caption) and L2 [r, N] = L1^T W_hat^T,
    its least-squares partner, so that (L1 L2)^T is the best rank-r
    approximation of W_hat (Eckart-Young).  Sign convention: each column of L1
    has its entry of largest magnitude positive (lowest index on ties).  All in
    fp64; returns (L1, L2, singular values of W_hat)."""
    What = np.asarray(W, dtype=f64) * np.asarray(s, dtype=f64)[None, :]
    _, sv, Vt = np.linalg.svd(What, full_matrices=False)
    L1 = Vt[:r].T.copy()
    for j in range(r):
        i = int(np.argmax(np.abs(L1[:, j])))
        if L1[i, j] < 0:
            L1[:, j] = -L1[:, j]
    L2 = L1.T @ What.T
    return L1, L2, sv


def bf16_ulp(y):
    """Spacing of bf16 numbers at |y| (fp64), used by the bf16-output tolerance.

    bf16 keeps 8 significant bits (7 stored) and the fp32 exponent range, so in
    the binade [2^E, 2^(E+1)) its spacing is 2^(E-7); below the smallest normal
    2^-126 the spacing stays 2^-133.  E is read exactly from the fp64 exponent
    (frexp), not from a rounded logarithm.
    """
    y = np.abs(np.asarray(y, dtype=f64))
    _, e = np.frexp(y)                    # y = m 2^e with m in [0.5, 1)
    E = np.maximum(np.where(y > 0, e - 1, -126), -126)
    return np.ldexp(np.ones_like(y), E - 7)
