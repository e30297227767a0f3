"""The truncated-SVD helper (hsq_lowrank_init) on the GPU against the oracle's
exact SVD (oracle.hsq_oracle.lowrank_init)."""
import numpy as np
import pytest
import torch

from oracle import hsq_oracle as O
from w4a4_rank_assisted_b200 import hsq

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _planted(N, K, r, seed, top=(40.0, 25.0, 16.0, 10.0), tail=1.0):
    """W_hat = U diag(sigma) V^T with a clear gap after the r largest values;
    returns W (bf16) and s such that W diag(s) ~ W_hat."""
    rng = np.random.default_rng(seed)
    m = min(N, K)
    U, _ = np.linalg.qr(rng.standard_normal((N, m)))
    V, _ = np.linalg.qr(rng.standard_normal((K, m)))
    big = list(np.geomspace(top[0], top[-1], r)) if r != len(top) else list(top)
    sigma = np.array(big + list(np.linspace(tail, 0.1 * tail, m - r)))
    What = U @ np.diag(sigma) @ V.T
    s = rng.uniform(0.5, 2.0, K).astype(np.float32)
    W = torch.from_numpy(What / s[None, :]).to(torch.bfloat16)
    return W, torch.from_numpy(s)


def _run(W, s, r, iters=8, seed=1):
    L1, L2 = hsq.lowrank_init(W.to(DEV), s.to(DEV), r, iters=iters, seed=seed)
    torch.cuda.synchronize()
    return L1.float().cpu().numpy().astype(np.float64), L2.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("N,K,r", [(256, 128, 4), (300, 200, 8), (128, 512, 32)])
def test_planted_subspace_and_product_match_the_oracle(N, K, r):
    W, s = _planted(N, K, r, seed=N + K + r, top=(60.0, 30.0))
    L1, L2 = _run(W, s, r)
    ref1, ref2, _ = O.lowrank_init(W.float().numpy(), s.numpy(), r)
    # same subspace, same signs: columns agree to bf16 rounding (2^-8 relative)
    assert np.max(np.abs(L1 - ref1)) <= 2e-2 * np.max(np.abs(ref1)), "L1 differs"
    P, Pref = L1 @ L2, ref1 @ ref2
    rms = np.sqrt(np.mean(Pref ** 2))
    assert np.max(np.abs(P - Pref)) <= 2e-2 * np.max(np.abs(Pref)) + 1e-2 * rms, "L1 L2 differs"
    assert np.max(np.abs(L1.T @ L1 - np.eye(r))) <= 2e-2, "L1 not orthonormal"


def test_random_weights_reach_the_optimal_error():
    """Weights as the synthetic layers draw them (N(0, 0.02), no gap): the
    product's error is within 2 % of the Eckart-Young optimum."""
    g = torch.Generator().manual_seed(3)
    N, K, r = 1024, 512, 32
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    s = torch.rand(K, generator=g) * 1.5 + 0.5
    L1, L2 = _run(W, s, r, iters=12)
    What = W.double().numpy() * s.double().numpy()[None, :]
    _, _, sv = O.lowrank_init(W.float().numpy(), s.numpy(), r)
    opt = np.sqrt(np.sum(sv[r:] ** 2))
    err = np.linalg.norm(What.T - L1 @ L2)
    assert err <= 1.02 * opt, f"error {err:.4g} vs optimum {opt:.4g}"


def test_same_seed_same_result_and_status():
    W, s = _planted(200, 96, 4, seed=9)
    a = _run(W, s, 4, seed=7)
    b = _run(W, s, 4, seed=7)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK
