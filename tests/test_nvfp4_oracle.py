"""Pins of the NVFP4-variant oracle (oracle/nvfp4_oracle.py) against what the
formats and the mathematics fix: an enumeration of every finite E4M3 value, the
E2M1 grid and its ties (derived by hand), a scalar re-derivation of the block
quantizer, on-grid round trips, and a lossless layer."""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as F

f32, f64 = np.float32, np.float64


def _e4m3_values():
    """Every finite, non-negative E4M3 value, enumerated from the bit fields
    (exponent bias 7, 3 mantissa bits, exponent field 0 subnormal, the all-ones
    pattern S.1111.111 is NaN)."""
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            vals.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(sorted(set(vals)))


def _nearest_even(v, grid, mantissa_of):
    d = np.abs(grid - v)
    i = np.flatnonzero(d == d.min())
    if len(i) == 1:
        return grid[i[0]]
    return grid[[j for j in i if mantissa_of(grid[j]) % 2 == 0][0]]


def _e4m3_mantissa(x):
    if x < 2.0 ** -6:
        return int(round(x / 2.0 ** -9))
    e = int(np.floor(np.log2(x)))
    return int(round((x / 2.0 ** e - 1) * 8))


def test_e4m3_rounding_matches_the_enumerated_format():
    grid = _e4m3_values()
    assert grid.max() == 448.0 and grid[1] == 2.0 ** -9
    rng = np.random.default_rng(1)
    mids = (grid[1:] + grid[:-1]) / 2  # every tie
    samples = np.concatenate([grid, mids, rng.uniform(0, 448, 2000), np.exp2(rng.uniform(-12, 9, 2000))])
    samples = samples[samples <= 448.0]
    want = np.array([_nearest_even(v, grid, _e4m3_mantissa) for v in samples])
    assert np.array_equal(F.e4m3_round(samples), want)
    assert F.e4m3_round(np.array([460.0, 1e6]))[0] == 448.0  # saturates


def test_e2m1_grid_and_hand_derived_ties():
    for i, v in enumerate(F.E2M1_GRID):
        assert F.e2m1_encode(np.array([v]))[0] == i
        if i:
            assert F.e2m1_encode(np.array([-v]))[0] == 8 | i
    # ties go to the even mantissa bit (the even index)
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for t, v in ties.items():
        assert F.e2m1_value(F.e2m1_encode(np.array([t])))[0] == v, t
        assert F.e2m1_value(F.e2m1_encode(np.array([-t])))[0] == -v, t
    assert F.e2m1_value(F.e2m1_encode(np.array([7.9, -100.0]))).tolist() == [6.0, -6.0]  # saturation
    assert F.e2m1_encode(np.array([-0.1]))[0] == 0  # no negative zero


def _scalar_quantize(V):
    """The block quantizer spelled out one value at a time (fp32 arithmetic via
    numpy scalars), independent of the vectorised oracle."""
    V = np.asarray(V, dtype=f32)
    rows, K = V.shape
    Kp = -(-K // 16) * 16
    grid = _e4m3_values()
    amax = f32(0)
    for v in V.ravel():
        amax = max(amax, f32(abs(v)))
    g = f32(amax / f32(2688.0))
    codes = np.zeros((rows, Kp), dtype=np.uint8)
    scales = np.zeros((rows, Kp // 16))
    for i in range(rows):
        for b in range(Kp // 16):
            blk = [V[i, k] if k < K else f32(0) for k in range(16 * b, 16 * b + 16)]
            bmax = f32(0)
            for v in blk:
                bmax = max(bmax, f32(abs(v)))
            if g == 0:
                continue
            sb = f32(bmax / f32(f32(6.0) * g))
            e = _nearest_even(min(f64(sb), 448.0), grid, _e4m3_mantissa)
            scales[i, b] = e
            den = f32(f32(e) * g)
            for j, v in enumerate(blk):
                t = f32(v / den) if den > 0 else f32(0)
                mag = _nearest_even(min(abs(f64(t)), 6.0), F.E2M1_GRID,
                                    lambda x: int(np.flatnonzero(F.E2M1_GRID == x)[0]))
                idx = int(np.flatnonzero(F.E2M1_GRID == mag)[0])
                codes[i, 16 * b + j] = idx | (8 if (t < 0 and idx) else 0)
    return codes, scales, g


@pytest.mark.parametrize("shape,seed", [((3, 40), 0), ((5, 16), 1), ((2, 67), 2)])
def test_block_quantizer_matches_a_scalar_derivation(shape, seed):
    rng = np.random.default_rng(seed)
    V = (rng.standard_normal(shape) * np.exp2(rng.integers(-6, 6, shape))).astype(f32)
    V[0, :5] = 0.0  # a partly zero block
    c, s, g = F.quantize_nvfp4(V)
    c2, s2, g2 = _scalar_quantize(V)
    assert g == g2 and np.array_equal(s, s2) and np.array_equal(c, c2)


def _on_grid(rows, K, rng, g=2.0 ** -10):
    """Values k * b * g with k on the E2M1 grid, b an E4M3 value per block, and
    in every block one |k| = 6 (so the block scale computes back to b), one
    block with b = 448 (so the tensor scale computes back to g)."""
    blocks = K // 16
    b = 448.0 * np.exp2(-rng.integers(0, 12, (rows, blocks)).astype(f64)) * rng.choice([1.0, 1.25, 1.5], (rows, blocks))
    b = F.e4m3_round(b)
    b[0, 0] = 448.0
    k = rng.choice(np.concatenate([F.E2M1_GRID, -F.E2M1_GRID]), (rows, blocks, 16))
    k[..., 0] = 6.0
    return (k * b[..., None] * g).reshape(rows, K), b, g


def test_on_grid_values_round_trip_exactly():
    rng = np.random.default_rng(3)
    V, b, g = _on_grid(4, 64, rng)
    c, s, gq = F.quantize_nvfp4(V)
    assert gq == f32(g) and np.array_equal(s, b)
    assert np.array_equal(F.dequantize_nvfp4(c, s, gq), V)
    p = F.pack_fp4(c)
    assert p.shape == (4, 32) and np.array_equal(p & 0xF, c[:, 0::2]) and np.array_equal(p >> 4, c[:, 1::2])


def test_lossless_layer_equals_the_dense_product():
    """s = 1, r = 0, X and W on the NVFP4 grid (exact in bf16 too): the NVFP4
    layer is exact, so it equals the fp64 X W^T + b."""
    rng = np.random.default_rng(4)
    X, _, _ = _on_grid(3, 48, rng, g=2.0 ** -8)
    W, _, _ = _on_grid(5, 48, rng, g=2.0 ** -11)
    bias = rng.standard_normal(5)
    Y = F.nvfp4_layer_forward(X.astype(f32), W.astype(f32), np.ones(48, dtype=f32), None, None, bias)
    assert np.array_equal(Y, X @ W.T + bias[None, :])


def test_lossless_layer_with_low_rank_branch_equals_the_dense_product():
    """s = 1, r = 2: the residual R = W - (L1 L2)^T and X are on the NVFP4 grid
    with values that are multiples of 2^-8, so W = R + (L1 L2)^T is exact in bf16
    and the quantization is lossless.  Then X R^T + (X L1) L2 = X W^T exactly:
    a dropped, transposed or sign-flipped branch fails."""
    rng = np.random.default_rng(5)
    K, M, N, r = 64, 3, 5, 2
    g = 2.0 ** -12
    # block scales that are multiples of 32, so every k b g is a multiple of 2^-8
    bvals = np.array([32.0, 64.0, 96.0, 128.0, 192.0, 256.0, 320.0, 384.0, 448.0])

    def grid(rows):
        b = rng.choice(bvals, (rows, K // 16))
        b[0, 0] = 448.0
        k = rng.choice(np.concatenate([F.E2M1_GRID, -F.E2M1_GRID]), (rows, K // 16, 16))
        k[..., 0] = 6.0
        return (k * b[..., None] * g).reshape(rows, K)

    X, R = grid(M), grid(N)
    L1 = rng.integers(-2, 3, (K, r)) * 2.0 ** -4
    L2 = rng.integers(-2, 3, (r, N)) * 2.0 ** -4
    W = R + (L1 @ L2).T
    Wb = torch.tensor(W, dtype=torch.float64).to(torch.bfloat16).double().numpy()
    assert np.array_equal(Wb, W), "W must be exact in bf16"
    bias = rng.standard_normal(N)
    Y = F.nvfp4_layer_forward(X.astype(f32), W.astype(f32), np.ones(K, dtype=f32), L1.astype(f32),
                              L2.astype(f32), bias)
    assert np.array_equal(Y, X @ W.T + bias[None, :])
    assert np.max(np.abs((X @ L1) @ L2)) > 0  # the branch is not trivially zero
