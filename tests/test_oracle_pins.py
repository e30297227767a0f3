"""Pins for the CPU oracle: checks against what the method and plain
mathematics fix, not against the oracle itself.

Method source: "Deflating the Hessian: Rank-4 W4A4 Quantization for Multimodal
Diffusion Transformers" -- Abstract (residual + high-precision low-rank split,
W4A4), Table 1 / Table 8 captions (group 64), rit.work blog diagonal-scaling
paragraph (smoothing leaves the full-precision map unchanged).
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import hsq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")
f32 = np.float32


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _bf16_round(a):
    """Round fp32 values to bf16 (RNE) and return them as fp32 (test helper)."""
    a = np.asarray(a, dtype=f32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) >> 16) << 16
    return u.astype(np.uint32).view(f32)


def _on_grid(rng, rows, K, mant_bits=0, emin=-12, emax=6):
    """Rows whose every 64-group is q * scale with q in [-7, 7], a +-7 present,
    and scale = m * 2^e (m an odd integer of <= mant_bits bits)."""
    G = O.num_groups(K)
    q = rng.integers(-7, 8, size=(rows, G * 64))
    for r in range(rows):
        for g in range(G):
            hi = min(K, (g + 1) * 64)
            idx = rng.integers(g * 64, hi)
            q[r, idx] = 7 if rng.random() < 0.5 else -7
    q[:, K:] = 0
    e = rng.integers(emin, emax, size=(rows, G)).astype(np.float64)
    m = np.ones((rows, G))
    if mant_bits:
        m = rng.integers(1, 2 ** mant_bits, size=(rows, G)) | 1
    scale = (m * 2.0 ** e).astype(f32)
    x = (q.reshape(rows, G, 64) * scale[:, :, None].astype(np.float64)).reshape(rows, G * 64)
    return x[:, :K].astype(f32), q[:, :K].astype(np.int8), scale


# ---------------------------------------------------------------- quantizer
@pytest.mark.parametrize("mant_bits", [0, 20])
@pytest.mark.parametrize("K", [64, 96, 1152])
def test_on_grid_values_are_returned_exactly(mant_bits, K):
    rng = np.random.default_rng(1 + K + mant_bits)
    x, q, scale = _on_grid(rng, 7, K, mant_bits)
    codes, sc = O.quantize_groups(x)
    assert np.array_equal(sc, scale)
    assert np.array_equal(codes[:, :K], q)
    assert np.all(codes[:, K:] == 0)
    # dequantization returns the input bit for bit
    deq = O.dequantize_groups(codes, sc)[:, :K]
    assert np.array_equal(deq, x.astype(np.float64))


def test_round_half_even_ties_and_packing_worked_example():
    ex = _golden()["group_tie_breaking"]
    row = np.zeros((1, 64), dtype=f32)
    vals = np.array(ex["x_over_u"], dtype=np.float64) * ex["unit"]
    row[0, :len(vals)] = vals
    codes, sc = O.quantize_groups(row)
    assert sc[0, 0] == f32(ex["scale"])
    assert codes[0, :len(ex["codes"])].tolist() == ex["codes"]
    assert np.all(codes[0, len(ex["codes"]):] == 0)
    packed = O.pack_int4(codes)
    nb = len(ex["packed_first_bytes"])
    assert packed[0, :nb].tolist() == ex["packed_first_bytes"]
    assert np.all(packed[0, nb:] == 0)


def test_smoothing_worked_example():
    ex = _golden()
    g = ex["group_tie_breaking"]
    X = np.zeros((1, 64), dtype=f32)
    vals = np.array(g["x_over_u"], dtype=np.float64) * g["unit"] * ex["smoothing_by_two"]["s"]
    X[0, :len(vals)] = vals
    s = np.full(64, ex["smoothing_by_two"]["s"], dtype=f32)
    xc, xs, U = O.quantize_act(X, s, None)
    assert xs.shape == (1, 1) and xs[0, 0] == f32(g["scale"])
    assert O.unpack_int4(xc)[0, :len(g["codes"])].tolist() == g["codes"]


def test_rank1_forward_worked_example():
    ex = _golden()
    g, e = ex["group_tie_breaking"], ex["rank1_forward"]
    X = np.zeros((1, 64), dtype=f32)
    vals = np.array(g["x_over_u"], dtype=np.float64) * g["unit"]
    X[0, :len(vals)] = vals
    W = np.zeros((1, 64), dtype=f32); W[0, 0] = e["W00"]
    L1 = np.zeros((64, 1), dtype=f32); L1[0, 0] = e["L1_00"]
    L2 = np.array([[e["L2_00"]]], dtype=f32)
    b = np.array([e["bias"]], dtype=f32)
    s = np.ones(64, dtype=f32)
    wc, ws = O.pack_weights(W, s, L1, L2)
    assert O.unpack_int4(wc)[0, 0] == e["qw0"]
    assert ws[0, 0] == f32(1.25) / f32(7)
    xc, xs, U = O.quantize_act(X, s, L1)
    assert U[0, 0] == e["U"]
    Y = O.linear_forward(xc, xs, U, wc, ws, L2, b)
    want = (1 / 8) * float(f32(1.25) / f32(7)) * 49 + e["U"] * e["L2_00"] + e["bias"]
    assert Y[0, 0] == pytest.approx(want, rel=1e-15)
    assert Y[0, 0] == pytest.approx(e["dense_Y"], rel=1e-6)


def test_quantization_error_is_at_most_half_a_step():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((33, 200)) * np.exp(rng.uniform(-3, 3, (33, 1)))).astype(f32)
    codes, sc = O.quantize_groups(x)
    deq = O.dequantize_groups(codes, sc)[:, :200]
    step = np.repeat(sc.astype(np.float64), 64, axis=1)[:, :200]
    err = np.abs(deq - x.astype(np.float64))
    # round-to-nearest: half a step, plus the fp32 rounding of x/scale
    assert np.all(err <= 0.5 * step * (1 + 2 ** -20) + 1e-30)
    # every group reaches +-7 at its absmax element, so the range is used fully
    G = sc.shape[1]
    for g in range(G):
        blk = codes[:, g * 64:(g + 1) * 64]
        assert np.all(np.abs(blk).max(axis=1) == 7)


def test_all_zero_group_has_zero_scale_and_codes():
    x = np.zeros((2, 128), dtype=f32)
    x[1, 64:] = np.linspace(-1, 1, 64, dtype=f32)
    codes, sc = O.quantize_groups(x)
    assert sc[0, 0] == 0 and sc[0, 1] == 0 and sc[1, 0] == 0
    assert np.all(codes[0] == 0) and np.all(codes[1, :64] == 0)
    assert sc[1, 1] == f32(1) / f32(7)


def test_brute_force_quantizer_elementwise():
    """Element-by-element restatement with numpy fp32 scalars on small rows."""
    rng = np.random.default_rng(3)
    for K in (64, 96, 128):
        x = (rng.standard_normal((5, K)) * 3).astype(f32)
        codes, sc = O.quantize_groups(x)
        for r in range(5):
            for g in range(O.num_groups(K)):
                vals = [x[r, k] for k in range(g * 64, min(K, g * 64 + 64))]
                amax = f32(0)
                for v in vals:
                    amax = max(amax, abs(v))
                s = f32(amax / f32(7))
                assert sc[r, g] == s
                for i, v in enumerate(vals):
                    t = f32(v / s)
                    fl = np.floor(t)
                    d = t - fl
                    qq = fl + 1 if d > 0.5 else fl if d < 0.5 else (fl if fl % 2 == 0 else fl + 1)
                    qq = min(7, max(-7, int(qq)))
                    assert codes[r, g * 64 + i] == qq


# ---------------------------------------------------------------- packing
def test_nibble_packing_all_byte_patterns():
    allb = np.arange(256, dtype=np.uint8).reshape(1, 256)
    q = O.unpack_int4(allb)
    assert np.array_equal(O.pack_int4(q), allb)
    lo, hi = q[0, 0::2], q[0, 1::2]
    b = np.arange(256)
    want_lo = np.where((b & 15) >= 8, (b & 15) - 16, b & 15)
    want_hi = np.where((b >> 4) >= 8, (b >> 4) - 16, b >> 4)
    assert np.array_equal(lo, want_lo) and np.array_equal(hi, want_hi)


def test_nibble_packing_hand_rows():
    q = np.zeros((1, 64), dtype=np.int8)
    q[0, 0], q[0, 1] = 1, -1      # 0xF1
    q[0, 2], q[0, 3] = -8, 7      # 0x78
    q[0, 62], q[0, 63] = 3, 0     # last byte 0x03
    p = O.pack_int4(q)
    assert p.shape == (1, 32)
    assert p[0, 0] == 0xF1 and p[0, 1] == 0x78 and p[0, 31] == 0x03
    assert np.all(p[0, 2:31] == 0)


# ---------------------------------------------------------------- smoothing / residual
def test_unit_smoothing_is_identity():
    rng = np.random.default_rng(5)
    X = _bf16_round(rng.standard_normal((4, 100)))
    W = _bf16_round(rng.standard_normal((6, 100)) * 0.02)
    s = np.ones(100, dtype=f32)
    assert np.array_equal(O.smooth_activation(X, s), X)
    assert np.array_equal(O.residual_weight(W, s, None, None), W)


def test_unquantized_layer_equals_dense_product():
    """rit.work blog: the diagonal scaling leaves the layer's FP map unchanged,
    and the residual + low-rank split is exact before quantization:
    X_hat R^T + X_hat L1 L2 + b == X W^T + b."""
    rng = np.random.default_rng(11)
    M, K, N, r = 9, 160, 12, 4
    X = _bf16_round(rng.standard_normal((M, K)))
    W = _bf16_round(rng.standard_normal((N, K)) * 0.02)
    L1 = _bf16_round(rng.standard_normal((K, r)) * 0.5)
    L2 = _bf16_round(rng.standard_normal((r, N)) * 0.5)
    b = _bf16_round(rng.standard_normal(N))
    s = np.exp(rng.uniform(-2, 2, K)).astype(f32)
    Yq = O.unquantized_forward(X, W, s, L1, L2, b)
    Yd = O.dense_forward(X, W, b)
    assert np.max(np.abs(Yq - Yd)) <= 1e-12 * np.max(np.abs(Yd))
    # the low-rank part is really subtracted (a wrong sign or transpose fails this)
    R = O.residual_weight(W, s, L1, L2, exact=True)
    LR = (L1.astype(np.float64) @ L2.astype(np.float64)).T
    assert np.allclose(R + LR, W.astype(np.float64) * s.astype(np.float64)[None, :], rtol=0, atol=1e-15)


def test_residual_rounding_is_single_fp32_rounding_of_fixed_order_fp64():
    rng = np.random.default_rng(12)
    K, N, r = 64, 3, 3
    W = _bf16_round(rng.standard_normal((N, K)) * 0.02)
    L1 = _bf16_round(rng.standard_normal((K, r)) * 0.02)
    L2 = _bf16_round(rng.standard_normal((r, N)) * 0.02)
    s = np.exp(rng.uniform(-1, 1, K)).astype(f32)
    R = O.residual_weight(W, s, L1, L2)
    for n in range(N):
        for k in range(K):
            lr = 0.0
            for j in range(r):
                lr = lr + float(L1[k, j]) * float(L2[j, n])
            assert R[n, k] == f32(float(W[n, k]) * float(s[k]) - lr)


# ---------------------------------------------------------------- forward
def test_rank0_is_plain_w4a4_of_smoothed_operands():
    """r = 0: Y = Q4(X_hat) Q4(W diag(s))^T + b, i.e. the product of the two
    dequantized operands (a different formulation from per-group partials)."""
    rng = np.random.default_rng(13)
    M, K, N = 6, 200, 7
    X = _bf16_round(rng.standard_normal((M, K)))
    W = _bf16_round(rng.standard_normal((N, K)) * 0.02)
    b = _bf16_round(rng.standard_normal(N))
    s = np.exp(rng.uniform(-1, 1, K)).astype(f32)
    Y = O.layer_forward(X, W, s, None, None, b)
    qx, sx = O.quantize_groups(O.smooth_activation(X, s))
    What = (W.astype(np.float64) * s.astype(np.float64)[None, :]).astype(f32)
    qw, sw = O.quantize_groups(What)
    Yd = O.dequantize_groups(qx, sx) @ O.dequantize_groups(qw, sw).T + b.astype(np.float64)
    assert np.max(np.abs(Y - Yd)) <= 1e-13 * np.max(np.abs(Yd))


def test_identity_weight_closed_form():
    """N = K, W = I, s = 1, r = 0: each residual row holds a single 1, so its
    group scale is fl32(1/7), its code 7, and Y[m,n] = sx[m,g(n)]*qx[m,n]*7*fl32(1/7)."""
    rng = np.random.default_rng(17)
    K = 128
    X = _bf16_round(rng.standard_normal((3, K)))
    W = np.eye(K, dtype=f32)
    s = np.ones(K, dtype=f32)
    wc, ws = O.pack_weights(W, s, None, None)
    qw = O.unpack_int4(wc)
    assert np.array_equal(qw, 7 * np.eye(K, dtype=np.int8))
    for n in range(K):
        for g in range(2):
            assert ws[g, n] == (f32(1) / f32(7) if g == n // 64 else 0)
    xc, xs, U = O.quantize_act(X, s, None)
    Y = O.linear_forward(xc, xs, U, wc, ws, None, None)
    qx = O.unpack_int4(xc).astype(np.float64)
    for m in range(3):
        for n in range(K):
            want = float(xs[n // 64, m]) * qx[m, n] * 7 * float(f32(1) / f32(7))
            assert Y[m, n] == pytest.approx(want, rel=1e-15, abs=0)


def test_lossless_inputs_reproduce_dense_product():
    """s = 1, r = 0 and both operands on the INT4 grid of their own groups:
    quantization is lossless, so the layer equals the fp64 X W^T."""
    rng = np.random.default_rng(19)
    M, K, N = 5, 192, 9
    X, _, _ = _on_grid(rng, M, K)
    W, _, _ = _on_grid(rng, N, K)
    s = np.ones(K, dtype=f32)
    Y = O.layer_forward(X, W, s, None, None, None)
    Yd = O.dense_forward(X, W, None)
    assert np.max(np.abs(Y - Yd)) <= 1e-13 * np.max(np.abs(Yd))


def test_brute_force_tiny_layers():
    """Tiny shapes, every output by explicit loops over dequantized products."""
    rng = np.random.default_rng(23)
    for (M, N, K, r) in [(1, 1, 64, 0), (3, 5, 96, 1), (8, 2, 128, 4), (2, 8, 64, 4)]:
        X = _bf16_round(rng.standard_normal((M, K)) * 2)
        W = _bf16_round(rng.standard_normal((N, K)) * 0.02)
        L1 = _bf16_round(rng.standard_normal((K, r)) * 0.1) if r else None
        L2 = _bf16_round(rng.standard_normal((r, N)) * 0.1) if r else None
        b = _bf16_round(rng.standard_normal(N))
        s = np.exp(rng.uniform(-1, 1, K)).astype(f32)
        wc, ws = O.pack_weights(W, s, L1, L2)
        xc, xs, U = O.quantize_act(X, s, L1)
        Y = O.linear_forward(xc, xs, U, wc, ws, L2, b)
        qx, qw = O.unpack_int4(xc), O.unpack_int4(wc)
        Xh = O.smooth_activation(X, s)
        for m in range(M):
            for j in range(r):
                u = 0.0
                for k in range(K):
                    u += float(Xh[m, k]) * float(L1[k, j])
                assert U[m, j] == pytest.approx(u, rel=1e-12, abs=1e-15)
            for n in range(N):
                y = 0.0
                for k in range(qx.shape[1]):
                    g = k // 64
                    y += (float(xs[g, m]) * int(qx[m, k])) * (float(ws[g, n]) * int(qw[n, k]))
                for j in range(r):
                    y += U[m, j] * float(L2[j, n])
                y += float(b[n])
                assert Y[m, n] == pytest.approx(y, rel=1e-12, abs=1e-12)


# ---------------------------------------------------------------- groups of 128
# (Deflating the Hessian, Table 3 and Table 4 captions: the Qwen3-8B results use
# groups of 128 along K.)
def test_brute_force_quantizer_groups_of_128():
    """Element-by-element restatement of the quantizer with 128-wide groups,
    including a K that pads the last group."""
    rng = np.random.default_rng(31)
    for K in (128, 200, 256):
        x = (rng.standard_normal((3, K)) * 3).astype(f32)
        codes, sc = O.quantize_groups(x, 128)
        assert codes.shape == (3, O.num_groups(K, 128) * 128)
        for r in range(3):
            for g in range(O.num_groups(K, 128)):
                vals = [x[r, k] for k in range(g * 128, min(K, g * 128 + 128))]
                amax = f32(0)
                for v in vals:
                    amax = max(amax, abs(v))
                s = f32(amax / f32(7))
                assert sc[r, g] == s
                for i, v in enumerate(vals):
                    t = f32(v / s)
                    fl = np.floor(t)
                    d = t - fl
                    qq = fl + 1 if d > 0.5 else fl if d < 0.5 else (fl if fl % 2 == 0 else fl + 1)
                    assert codes[r, g * 128 + i] == min(7, max(-7, int(qq)))
            assert np.all(codes[r, K:] == 0)


def test_groups_of_128_agree_with_64_when_halves_share_the_absmax():
    """If both 64-halves of every 128-group have the same absmax, the two group
    sizes give the same codes and the 128-group scale equals both 64-group
    scales: a misplaced group boundary or a wrong group count breaks this."""
    rng = np.random.default_rng(37)
    x = (rng.standard_normal((4, 384)) * 2).astype(f32)
    x = np.clip(x, -5, 5).astype(f32)
    x[:, 0::64] = f32(6.5)  # the absmax of every 64-half, so also of every 128-group
    c64, s64 = O.quantize_groups(x, 64)
    c128, s128 = O.quantize_groups(x, 128)
    assert np.array_equal(c64, c128)
    assert np.array_equal(s128, s64[:, 0::2]) and np.array_equal(s128, s64[:, 1::2])
    x[:, 64] = f32(6.6)  # now the second half of group 0 is larger: only that group changes
    c64, s64 = O.quantize_groups(x, 64)
    c128, s128 = O.quantize_groups(x, 128)
    assert s128[0, 0] == f32(f32(6.6) / f32(7)) and s64[0, 0] == f32(f32(6.5) / f32(7))
    assert np.array_equal(c128[:, 128:], c64[:, 128:])


def test_brute_force_tiny_layers_groups_of_128():
    """Tiny layers with 128-wide groups, every output by explicit loops."""
    rng = np.random.default_rng(41)
    for (M, N, K, r) in [(2, 3, 128, 0), (3, 2, 200, 2), (1, 4, 256, 4)]:
        X = _bf16_round(rng.standard_normal((M, K)) * 2)
        W = _bf16_round(rng.standard_normal((N, K)) * 0.02)
        L1 = _bf16_round(rng.standard_normal((K, r)) * 0.1) if r else None
        L2 = _bf16_round(rng.standard_normal((r, N)) * 0.1) if r else None
        b = _bf16_round(rng.standard_normal(N))
        s = np.exp(rng.uniform(-1, 1, K)).astype(f32)
        wc, ws = O.pack_weights(W, s, L1, L2, 128)
        xc, xs, U = O.quantize_act(X, s, L1, 128)
        Y = O.linear_forward(xc, xs, U, wc, ws, L2, b, 128)
        qx, qw = O.unpack_int4(xc), O.unpack_int4(wc)
        assert xs.shape == (O.num_groups(K, 128), M) and ws.shape == (O.num_groups(K, 128), N)
        for m in range(M):
            for n in range(N):
                y = 0.0
                for k in range(qx.shape[1]):
                    g = k // 128
                    y += (float(xs[g, m]) * int(qx[m, k])) * (float(ws[g, n]) * int(qw[n, k]))
                for j in range(r):
                    y += U[m, j] * float(L2[j, n])
                y += float(b[n])
                assert Y[m, n] == pytest.approx(y, rel=1e-12, abs=1e-12)


# ---------------------------------------------------------------- truncated-SVD initialisation
def _orthonormal(rng, n, k):
    q, _ = np.linalg.qr(rng.standard_normal((n, k)))
    return q


def test_lowrank_init_recovers_a_planted_decomposition():
    """W_hat = U diag(sigma) V^T built from known orthonormal factors and known
    singular values: L1 spans V's first r columns, (L1 L2)^T leaves exactly the
    tail energy sqrt(sum_{i>r} sigma_i^2), and L1 is orthonormal."""
    rng = np.random.default_rng(5)
    N, K, r = 40, 24, 4
    U, V = _orthonormal(rng, N, K), _orthonormal(rng, K, K)
    sigma = np.array([50.0, 30.0, 20.0, 12.0] + list(np.linspace(3.0, 0.5, K - 4)))
    What = U @ np.diag(sigma) @ V.T
    s = rng.uniform(0.5, 2.0, K)
    W = What / s[None, :]  # so that W diag(s) is the planted matrix
    L1, L2, _ = O.lowrank_init(W, s, r)
    assert np.allclose(L1.T @ L1, np.eye(r), atol=1e-12)
    P1, Pv = L1 @ L1.T, V[:, :r] @ V[:, :r].T
    assert np.max(np.abs(P1 - Pv)) < 1e-10
    err = np.linalg.norm(What.T - L1 @ L2)
    assert abs(err - np.sqrt(np.sum(sigma[r:] ** 2))) < 1e-9 * err
    # sign convention: the largest-magnitude entry of each column is positive
    for j in range(r):
        assert L1[np.argmax(np.abs(L1[:, j])), j] > 0


def test_lowrank_init_exact_for_rank_r_weights():
    rng = np.random.default_rng(6)
    N, K, r = 30, 20, 3
    What = rng.standard_normal((N, r)) @ rng.standard_normal((r, K))
    L1, L2, _ = O.lowrank_init(What, np.ones(K), r)
    assert np.max(np.abs(L1 @ L2 - What.T)) < 1e-11 * np.max(np.abs(What))


def test_lowrank_init_picks_the_largest_axes_of_a_scaled_selection():
    """W with one nonzero per row in distinct columns: its singular vectors are
    coordinate axes, so L1's columns are the unit vectors of the r largest |W|
    entries (in that order, positive) and L2 holds those entries."""
    N, K, r = 6, 8, 3
    W = np.zeros((N, K))
    cols, vals = [5, 1, 7, 2, 0, 4], [2.0, -9.0, 4.0, -1.0, 6.5, 3.0]
    for n, (c, v) in enumerate(zip(cols, vals)):
        W[n, c] = v
    s = np.full(K, 0.5)  # smoothing scales every singular value by 0.5
    L1, L2, sv = O.lowrank_init(W, s, r)
    order = [1, 4, 2]  # rows with |v| = 9, 6.5, 4
    for j, n in enumerate(order):
        e = np.zeros(K)
        e[cols[n]] = 1.0
        assert np.allclose(L1[:, j], e, atol=1e-12)
        expect = np.zeros(N)
        expect[n] = 0.5 * vals[n]
        assert np.allclose(L2[j], expect, atol=1e-12)
    assert np.allclose(sv[:r], [4.5, 3.25, 2.0])


# --------------------------------------------------------------------------
# bf16_ulp: the spacing the bf16-output tolerance adds, fixed by the bf16 format
# --------------------------------------------------------------------------
def _bf16_values_from_bits(bits):
    """bf16 bit patterns (uint16) -> their values, decoded by torch's bfloat16."""
    t = torch.tensor(np.asarray(bits, dtype=np.int32).astype(np.int16), dtype=torch.int16)
    return t.view(torch.bfloat16).double().numpy()


def test_bf16_ulp_hand_values():
    # 8 significant bits: spacing 2^-7 in [1, 2), 2^-6 in [2, 4)
    assert O.bf16_ulp(np.array([1.0]))[0] == 2.0 ** -7
    assert O.bf16_ulp(np.array([1.5]))[0] == 2.0 ** -7
    assert O.bf16_ulp(np.array([2.0]))[0] == 2.0 ** -6
    assert O.bf16_ulp(np.array([-3.0]))[0] == 2.0 ** -6
    assert O.bf16_ulp(np.array([0.75]))[0] == 2.0 ** -8
    # just below a power of two stays in the lower binade (no rounding of a logarithm)
    assert O.bf16_ulp(np.array([2.0 - 2.0 ** -40]))[0] == 2.0 ** -7
    assert O.bf16_ulp(np.array([np.nextafter(1.0, 0.0)]))[0] == 2.0 ** -8
    # subnormal range: the spacing stays that of the smallest binade, 2^-133
    assert O.bf16_ulp(np.array([3 * 2.0 ** -130]))[0] == 2.0 ** -133
    assert O.bf16_ulp(np.array([0.0]))[0] == 2.0 ** -133
    assert O.bf16_ulp(np.array([2.0 ** -126]))[0] == 2.0 ** -133


def test_bf16_ulp_equals_gap_to_next_bf16_pattern():
    """For every positive finite bf16 value x except the largest, the gap to the
    next bit pattern is the spacing at x."""
    bits = np.arange(1, 0x7F7F, dtype=np.int64)  # 0x7F7F is the largest finite bf16
    lo = _bf16_values_from_bits(bits)
    hi = _bf16_values_from_bits(bits + 1)
    assert np.all(hi > lo)
    assert np.array_equal(O.bf16_ulp(lo), hi - lo)
    # and at a point inside each gap
    assert np.array_equal(O.bf16_ulp((lo + hi) / 2), hi - lo)
