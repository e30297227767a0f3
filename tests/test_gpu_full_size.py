"""Full-size parity on the stated layer shapes (PixArt-Sigma, SANA-1.6B,
FLUX.1, Qwen3-8B linears), in the same launch configuration the benchmark
times.  The oracle packs every weight (codes and scales compared bit for bit)
and recomputes a sample of token rows -- the first, the last, and rows drawn
at random -- whose activation codes, scales, U and outputs are compared.

Every layer runs at its own quantization group (64, or 128 for the
``qwen3_8b_m*_g128`` workloads, the pages' Qwen3-8B setting) on both sides,
and the test asserts the group count of the packed scales, so that a
group-128 case cannot silently run at 64.  The decode workloads the benchmark
runs as one launch per layer (``hsq_linear_forward_fused``) are also checked
in that form."""
import numpy as np
import pytest
import torch

from oracle import hsq_oracle as O
from w4a4_rank_assisted_b200 import hsq
from w4a4_rank_assisted_b200.synth import WORKLOADS, make_layer

from _helpers import check_y, pad_scales, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
# the INT4 layers (the NVFP4 variant's full-size case is in test_gpu_nvfp4.py)
LAYERS = [(w, i) for w, specs in WORKLOADS.items() for i in range(len(specs)) if specs[i].fmt == "int4"]
FUSED_LAYERS = [(w, i) for w, i in LAYERS
                if hsq.fused_supported(WORKLOADS[w][i].M, WORKLOADS[w][i].K, WORKLOADS[w][i].r,
                                       WORKLOADS[w][i].group, N=WORKLOADS[w][i].N)]


def _sample_rows(M, n=40, seed=0):
    rng = np.random.default_rng(seed)
    rows = {0, M - 1} | set(rng.integers(0, M, size=min(n, M)).tolist())
    return np.array(sorted(rows))


def _packed(layer, spec):
    g = spec.group
    pl = hsq.PackedLinear(layer.W.to(DEV), layer.s.to(DEV), layer.L1.to(DEV), layer.L2.to(DEV), None, group=g)
    assert pl.group == g
    assert pl.w_scales.shape[0] == hsq.hsq_num_groups(spec.K, g)
    Wn, sn, L1n, L2n = to_np(layer.W), to_np(layer.s), to_np(layer.L1), to_np(layer.L2)
    wc, ws = O.pack_weights(Wn, sn, L1n, L2n, g)
    assert ws.shape[0] == O.num_groups(spec.K, g)
    assert np.array_equal(to_np(pl.w_codes), wc)
    assert np.array_equal(to_np(pl.w_scales), pad_scales(ws, hsq.hsq_scales_ld(spec.N)))
    return pl, (wc, ws, sn, L1n, L2n)


@pytest.mark.parametrize("workload,idx", LAYERS, ids=[f"{w}-{i}" for w, i in LAYERS])
def test_full_size_layer(workload, idx):
    spec = WORKLOADS[workload][idx]
    layer = make_layer(spec)
    M, K, N, r, g = spec.M, spec.K, spec.N, spec.r, spec.group
    pl, (wc, ws, sn, L1n, L2n) = _packed(layer, spec)
    act = hsq.ActBuffers(M, K, r, DEV, group=g)
    assert act.x_scales.shape[0] == hsq.hsq_num_groups(K, g)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    hsq.forward(pl, layer.X.to(DEV), act, Y, workspace=pl.workspace(M))
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK

    rows = _sample_rows(M)
    xc, xs, U = O.quantize_act(to_np(layer.X)[rows], sn, L1n, g)
    assert np.array_equal(to_np(act.x_codes)[rows], xc)
    assert np.array_equal(to_np(act.x_scales)[:, rows], xs)
    U_gpu = to_np(act.U)[rows].astype(np.float64)
    assert np.max(np.abs(U_gpu - U)) <= 1e-5 * (np.abs(U).max() + 1e-30)
    Y_ref = O.linear_forward(xc, xs, U, wc, ws, L2n, None, g)
    check_y(to_np(Y)[rows], Y_ref, out_f32=False, where=f"{spec.name} g{g}")


@pytest.mark.parametrize("workload,idx", FUSED_LAYERS, ids=[f"{w}-{i}" for w, i in FUSED_LAYERS])
def test_full_size_fused_layer(workload, idx):
    """The single-launch decode forward on the full-size decode layers (K up to
    12288), against the oracle and against the two-call path."""
    spec = WORKLOADS[workload][idx]
    layer = make_layer(spec)
    M, K, N, r, g = spec.M, spec.K, spec.N, spec.r, spec.group
    pl, (wc, ws, sn, L1n, L2n) = _packed(layer, spec)
    X = layer.X.to(DEV)
    Yf = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    hsq.forward_fused(pl, X, Yf)
    act = hsq.ActBuffers(M, K, r, DEV, group=g)
    Y2 = torch.empty_like(Yf)
    hsq.forward(pl, X, act, Y2, workspace=pl.workspace(M))
    torch.cuda.synchronize()
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK

    xc, xs, U = O.quantize_act(to_np(layer.X), sn, L1n, g)
    Y_ref = O.linear_forward(xc, xs, U, wc, ws, L2n, None, g)
    check_y(to_np(Yf), Y_ref, out_f32=False, where=f"fused {spec.name} g{g}")
    # the same codes and scales as the two calls, U and the group sums up to their
    # fp32 summation order: the two bf16 outputs differ by at most the one
    # rounding of the output, an ulp
    a, b = to_np(Yf).astype(np.float64), to_np(Y2).astype(np.float64)
    rms = np.sqrt(np.mean(Y_ref ** 2))
    tol = 1e-5 * rms + O.bf16_ulp(np.maximum(np.abs(a), np.abs(b)))
    assert np.all(np.abs(a - b) <= tol), "fused forward differs from the two calls"
