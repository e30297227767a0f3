"""hsq_linear_forward_noalloc: the forward that uses the library's built-in
scratch array instead of a caller workspace.

Checked through the C ABI against hsq_linear_forward (the regular entry point,
with a workspace the test allocates) on the same inputs, on two calls in a row
so that the second call starts from the scratch contents the first one left.
Both entry points run the same kernels with the same launch plan, and the
split-K reduction sums the partial tiles in a fixed order, so the outputs must
be equal bit for bit: a stale or mis-cleared scratch that disturbs even a few
outputs slightly fails the check.
Runs alone in a fresh process and after the other test files alike: it builds
all of its own inputs.
"""
import pytest
import torch

from w4a4_rank_assisted_b200 import hsq
from w4a4_rank_assisted_b200.synth import LayerSpec, make_layer

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _prepare(M, K, N, r, seed, group):
    spec = LayerSpec(f"na{M}x{K}x{N}", M, K, N, r, act="outlier", outlier_frac=0.01, outlier_mult=30.0,
                     seed=seed, bias=True)
    lay = make_layer(spec)
    d = lambda t: None if t is None else t.to(DEV).contiguous()
    pl = hsq.PackedLinear(d(lay.W), d(lay.s), d(lay.L1) if r else None, d(lay.L2) if r else None, d(lay.bias),
                          group=group)
    act = hsq.ActBuffers(M, K, r, DEV, group=group)
    hsq.hsq_quantize_act(d(lay.X), pl.s, pl.L1, M, K, r, act.x_codes, act.x_scales, act.U, group=group)
    return pl, act


def _regular(pl, act, M, K, N, r, group):
    Y = torch.empty((M, N), dtype=torch.float32, device=DEV)
    ws = pl.workspace(M)
    hsq.hsq_linear_forward(act.x_codes, act.x_scales, act.U, pl.w_codes, pl.w_scales, pl.L2, pl.bias,
                           M, N, K, r, Y, out=hsq.HSQ_OUT_F32, workspace=ws,
                           ws_bytes=0 if ws is None else ws.numel(), group=group)
    return Y


def _noalloc(pl, act, M, K, N, r, group):
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
    hsq.hsq_linear_forward_noalloc(act.x_codes, act.x_scales, act.U, pl.w_codes, pl.w_scales, pl.L2, pl.bias,
                                   M, N, K, r, Y, out=hsq.HSQ_OUT_F32, group=group)
    return Y


@pytest.mark.parametrize("M,K,N,r,group", [
    (16, 4096, 2048, 4, 64),    # split-K decode tiles: uses the scratch array
    (128, 2048, 1024, 4, 64),   # split-K 128x256 tiles: uses the scratch array
    (200, 224, 1160, 32, 64),   # whole tiles: no scratch
    (320, 640, 1024, 4, 64),    # more than 256 tokens: expanded codes in the scratch array (whole tiles)
    (128, 2048, 1024, 4, 128),  # groups of 128 above 64 tokens: expanded codes in the scratch array
])
def test_noalloc_matches_regular_entry_point_twice(M, K, N, r, group):
    pl, act = _prepare(M, K, N, r, seed=M + N, group=group)
    ref = _regular(pl, act, M, K, N, r, group)
    torch.cuda.synchronize()
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK
    for call in range(2):
        Y = _noalloc(pl, act, M, K, N, r, group)
        torch.cuda.synchronize()
        assert hsq.hsq_get_device_status() == hsq.HSQ_OK
        assert bool(torch.isfinite(Y).all()), f"call {call}: outputs left unwritten"
        ndiff = int((Y != ref).sum())
        assert ndiff == 0, f"call {call}: {ndiff} outputs differ from hsq_linear_forward's"


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 256 tokens x 4096 outputs: 32 tiles of 128x256 cut between CTAs, whose
    # partial tiles need more than the built-in array on a full-size GPU.
    M, K, N, r = 256, 4096, 4096, 4
    need = hsq.hsq_workspace_bytes(M, N, K, r)
    if need <= hsq.HSQ_NOALLOC_SCRATCH_BYTES:
        pytest.skip(f"this device needs only {need} bytes for the shape")
    # full-size buffers, so that nothing could be read out of bounds even if a launch happened
    x_codes = torch.zeros((M, K // 2), dtype=torch.uint8, device=DEV)
    x_scales = torch.zeros((K // 64, hsq.hsq_scales_ld(M)), dtype=torch.float32, device=DEV)
    U = torch.zeros((M, r), dtype=torch.float32, device=DEV)
    w_codes = torch.zeros((N, K // 2), dtype=torch.uint8, device=DEV)
    w_scales = torch.zeros((K // 64, hsq.hsq_scales_ld(N)), dtype=torch.float32, device=DEV)
    L2 = torch.zeros((r, N), dtype=torch.bfloat16, device=DEV)
    Y = torch.full((M, N), 7.0, dtype=torch.float32, device=DEV)
    with pytest.raises(hsq.HsqError) as e:
        hsq.hsq_linear_forward_noalloc(x_codes, x_scales, U, w_codes, w_scales, L2, None, M, N, K, r, Y,
                                       out=hsq.HSQ_OUT_F32)
    assert e.value.status == hsq.HSQ_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert bool(torch.all(Y == 7.0)), "a rejected call must launch nothing"
