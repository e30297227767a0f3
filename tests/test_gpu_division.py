"""The activation kernel divides by a reciprocal with a correction step instead
of an IEEE division; these tests check that every value it decides (the fp32
smoothed activation through its group scale, and the codes) still matches the
oracle's IEEE division, for every finite bf16 input value."""
import numpy as np
import pytest
import torch

from oracle import hsq_oracle as O
from w4a4_rank_assisted_b200 import hsq

from _helpers import pad_scales, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _all_finite_bf16():
    """Every nonzero bf16 value whose smoothed value stays finite (|x| < 2^90)."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[np.isfinite(f) & (f != 0) & (np.abs(f) < 2.0 ** 90)]
    return f


def _run(X, s):
    M, K = X.shape
    act = hsq.ActBuffers(M, K, 0, DEV)
    Xt = torch.tensor(X).to(torch.bfloat16).to(DEV)
    st = torch.tensor(s).to(DEV)
    hsq.hsq_quantize_act(Xt, st, None, M, K, 0, act.x_codes, act.x_scales, None)
    torch.cuda.synchronize()
    xc, xs, _ = O.quantize_act(to_np(Xt.cpu()), s, None)
    return act, xc, xs


@pytest.mark.parametrize("K", [4096, 512])  # 512: enough rows for the many-row kernel
def test_every_bf16_value_through_its_group_scale(K):
    """One nonzero element per 64-group: the group's scale is fl(|fl(x/s)|/7),
    so a smoothed value off by one ulp would change the scale."""
    vals = _all_finite_bf16()
    G = K // 64
    M = -(-len(vals) // G)
    X = np.zeros((M, K), dtype=np.float32)
    flat = np.zeros(M * G, dtype=np.float32)
    flat[:len(vals)] = vals
    rng = np.random.default_rng(0)
    pos = rng.integers(0, 64, size=M * G)
    X.reshape(M * G, 64)[np.arange(M * G), pos] = flat
    s = np.exp(rng.uniform(np.log(0.05), np.log(50.0), K)).astype(np.float32)
    act, xc, xs = _run(X, s)
    assert np.array_equal(to_np(act.x_scales), pad_scales(xs, hsq.hsq_scales_ld(M)))
    assert np.array_equal(to_np(act.x_codes), xc)


@pytest.mark.parametrize("M", [512, 4400])  # 4400: the many-row kernel
def test_code_rounding_near_half_integers(M):
    """Groups whose elements sit at and around k + 1/2 steps of the group scale."""
    rng = np.random.default_rng(1)
    K = 1024
    X = np.zeros((M, K), dtype=np.float32)
    G = K // 64
    for m in range(M):
        for g in range(G):
            a = np.float32(rng.uniform(0.5, 8.0))
            blk = np.empty(64, dtype=np.float32)
            blk[0] = a
            sc = np.float32(a / np.float32(7))
            k = rng.integers(-7, 7, size=63)
            frac = rng.choice([0.5, 0.5 - 2 ** -9, 0.5 + 2 ** -9, 0.25, 0.75], size=63)
            blk[1:] = (k + frac) * sc
            X[m, g * 64:(g + 1) * 64] = blk
    s = np.ones(K, dtype=np.float32)
    act, xc, xs = _run(X, s)
    assert np.array_equal(to_np(act.x_scales), pad_scales(xs, hsq.hsq_scales_ld(M)))
    assert np.array_equal(to_np(act.x_codes), xc)


def test_extreme_values_and_smoothing_factors():
    """Rows that mix a normal group absmax with bf16 subnormals and values below
    2^-100, groups of such tiny values only, values above 2^100, all-zero groups,
    and channels whose smoothing factor lies outside [2^-24, 2^24] (in the last
    256-channel chunk only): every code and scale must still equal what the
    oracle's IEEE quotients give."""
    rng = np.random.default_rng(2)
    K, M = 1024, 4400  # enough rows for the many-row kernel
    G = K // 64
    X = rng.standard_normal((M, K)).astype(np.float32)
    tiny = np.array([2.0 ** -133, 2.0 ** -126, 2.0 ** -110, 2.0 ** -101, 2.0 ** -100, 3 * 2.0 ** -105],
                    dtype=np.float32)
    sign = lambda n: rng.choice(np.array([-1.0, 1.0], dtype=np.float32), n)
    for m in range(M):
        kind = m % 5
        if kind == 0:    # a normal absmax with tiny elements beside it
            idx = rng.choice(768, 40, replace=False)
            X[m, idx] = rng.choice(tiny, 40) * sign(40)
        elif kind == 1:  # one group of tiny values only
            g = rng.integers(12)
            X[m, g * 64:(g + 1) * 64] = rng.choice(tiny, 64) * sign(64)
        elif kind == 2:  # values above 2^100
            idx = rng.choice(768, 3, replace=False)
            X[m, idx] = (2.0 ** rng.uniform(100.0, 120.0, 3)).astype(np.float32) * sign(3)
        elif kind == 3:  # an all-zero group
            g = rng.integers(G)
            X[m, g * 64:(g + 1) * 64] = 0.0
    s = np.exp(rng.uniform(np.log(0.05), np.log(50.0), K)).astype(np.float32)
    s[900:904] = np.array([2.0 ** -30, 2.0 ** -25, 2.0 ** 25, 2.0 ** 30], dtype=np.float32)
    act, xc, xs = _run(X, s)
    assert np.array_equal(to_np(act.x_scales), pad_scales(xs, hsq.hsq_scales_ld(M)))
    assert np.array_equal(to_np(act.x_codes), xc)
