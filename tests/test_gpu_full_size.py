"""Full-size parity on the stated layer shapes (PixArt-Sigma, SANA-1.6B,
FLUX.1, Qwen3-8B linears), in the same launch configuration the benchmark
times.  The oracle packs every weight (codes and scales compared bit for bit)
and recomputes a sample of token rows -- the first, the last, and rows drawn
at random -- whose activation codes, scales, U and outputs are compared."""
import numpy as np
import pytest
import torch

from oracle import hsq_oracle as O
from w4a4_rank_assisted_b200 import hsq
from w4a4_rank_assisted_b200.synth import WORKLOADS, make_layer

from _helpers import check_y, pad_scales, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
LAYERS = [(w, i) for w, specs in WORKLOADS.items() for i in range(len(specs))]


def _sample_rows(M, n=40, seed=0):
    rng = np.random.default_rng(seed)
    rows = {0, M - 1} | set(rng.integers(0, M, size=min(n, M)).tolist())
    return np.array(sorted(rows))


@pytest.mark.parametrize("workload,idx", LAYERS, ids=[f"{w}-{i}" for w, i in LAYERS])
def test_full_size_layer(workload, idx):
    spec = WORKLOADS[workload][idx]
    layer = make_layer(spec)
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    pl = hsq.PackedLinear(layer.W.to(DEV), layer.s.to(DEV), layer.L1.to(DEV), layer.L2.to(DEV), None)
    act = hsq.ActBuffers(M, K, r, DEV)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    hsq.forward(pl, layer.X.to(DEV), act, Y, workspace=pl.workspace(M))
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK

    Wn, sn, L1n, L2n = to_np(layer.W), to_np(layer.s), to_np(layer.L1), to_np(layer.L2)
    wc, ws = O.pack_weights(Wn, sn, L1n, L2n)
    assert np.array_equal(to_np(pl.w_codes), wc)
    assert np.array_equal(to_np(pl.w_scales), pad_scales(ws, hsq.hsq_scales_ld(N)))

    rows = _sample_rows(M)
    xc, xs, U = O.quantize_act(to_np(layer.X)[rows], sn, L1n)
    assert np.array_equal(to_np(act.x_codes)[rows], xc)
    assert np.array_equal(to_np(act.x_scales)[:, rows], xs)
    U_gpu = to_np(act.U)[rows].astype(np.float64)
    assert np.max(np.abs(U_gpu - U)) <= 1e-5 * (np.abs(U).max() + 1e-30)
    Y_ref = O.linear_forward(xc, xs, U, wc, ws, L2n, None)
    check_y(to_np(Y)[rows], Y_ref, out_f32=False, where=spec.name)
