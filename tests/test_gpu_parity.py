"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Codes, packed bytes and scales must match bit for bit; outputs must meet the
layer's tolerance (see tests/_helpers.py).  Small shapes are compared element
by element; shapes span several tiles and ragged tails in M, N and K.
"""
import numpy as np
import pytest
import torch

from oracle import hsq_oracle as O
from w4a4_rank_assisted_b200 import hsq
from w4a4_rank_assisted_b200.synth import LayerSpec, make_layer

from _helpers import check_y, oracle_layer, pad_scales, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run_gpu(layer, out=hsq.HSQ_OUT_F32, X=None, group=hsq.GROUP):
    X = layer.X if X is None else X
    M, K = X.shape
    N = layer.W.shape[0]
    r = layer.spec.r
    d = lambda t: None if t is None else t.to(DEV).contiguous()
    pl = hsq.PackedLinear(d(layer.W), d(layer.s), d(layer.L1) if r else None,
                          d(layer.L2) if r else None, d(layer.bias), group=group)
    act = hsq.ActBuffers(M, K, r, DEV, group=group)
    Y = torch.empty((M, N), dtype=torch.float32 if out == hsq.HSQ_OUT_F32 else torch.bfloat16, device=DEV)
    ws = pl.workspace(M)
    hsq.forward(pl, d(X), act, Y, workspace=ws, out=out)
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK
    torch.cuda.synchronize()
    return pl, act, Y, ws


def _spec(M, K, N, r, seed=0, bias=True, act="outlier"):
    return LayerSpec(f"t{M}x{K}x{N}r{r}", M, K, N, r, act=act, outlier_frac=0.01, outlier_mult=30.0,
                     seed=seed, bias=bias)


def _check_all(layer, pl, act, Y, out_f32, where, group=hsq.GROUP):
    ref = oracle_layer(layer.X, layer.W, layer.s, layer.L1 if layer.spec.r else None,
                       layer.L2 if layer.spec.r else None, layer.bias, group=group)
    M, N = Y.shape
    # weights: bit-exact codes and scales (with the zero padding of the layout)
    assert np.array_equal(to_np(pl.w_codes), ref["w_codes"]), f"{where}: weight codes differ"
    assert np.array_equal(to_np(pl.w_scales), pad_scales(ref["w_scales"], hsq.hsq_scales_ld(N))), \
        f"{where}: weight scales differ"
    # activations: bit-exact codes and scales; U within fp32 accumulation error
    assert np.array_equal(to_np(act.x_codes), ref["x_codes"]), f"{where}: activation codes differ"
    assert np.array_equal(to_np(act.x_scales), pad_scales(ref["x_scales"], hsq.hsq_scales_ld(M))), \
        f"{where}: activation scales differ"
    if layer.spec.r:
        U = to_np(act.U).astype(np.float64)
        scale = np.abs(ref["U"]).max() + 1e-30
        assert np.max(np.abs(U - ref["U"])) <= 1e-5 * scale, f"{where}: U differs"
    return check_y(to_np(Y), ref["Y"], out_f32, where)


SMALL_SHAPES = [
    # (M, K, N, r)   -- decode tiles, split-K, ragged M/N/K tails, large-M tiles
    (1, 64, 128, 4),
    (5, 96, 136, 1),
    (16, 1152, 1152, 4),
    (17, 256, 264, 4),
    (33, 320, 128, 0),
    (64, 512, 384, 32),
    (65, 192, 520, 4),
    (128, 1152, 256, 4),
    (200, 224, 1160, 4),
    (256, 1152, 1152, 4),
    (300, 640, 512, 32),
    (8, 12288, 4096, 4),     # weight stream whose ring reuses its slots, partial last stage, ragged last block
    (8, 16384, 2048, 2),     # ... four stages through two slots
    (16, 4096, 2048, 4),     # stream-K, decode tile
    (24, 4096, 2048, 4),     # stream-K, decode tile of 32 tokens
    (128, 2048, 1024, 4),    # stream-K, large tile
    (130, 320, 264, 15),     # largest rank of one tensor-core low-rank step
    (97, 192, 136, 16),      # two low-rank steps
    (96, 256, 200, 31),      # three low-rank steps, the last with one rank
    (300, 640, 512, 16),     # large tiles, two low-rank steps (one rank in the second)
    (520, 384, 776, 17),     # ... two ranks in the second: the many-rank kernels
    (200, 320, 264, 17),     # mid tiles, the many-rank kernels
    (2048, 128, 2560, 32),   # more tiles than SMs: later tiles' low-rank steps built ahead
    (129, 128, 256, 0),      # no low-rank pair: the step carries the bias alone
    (70, 200, 136, 8),       # rank 8: eight L1 rows per warp load, chunk of 200 channels
    (40, 328, 264, 8),       # few rows, rank 8, ragged last chunk
    (33, 328, 128, 7),       # generic odd rank, few rows
    (150, 584, 136, 5),      # generic odd rank, ragged rows and last chunk
    (4150, 1160, 136, 4),    # many-row activation kernel: ragged last block, lanes past the padded K
    (4150, 264, 136, 0),     # ... no low-rank branch
    (4200, 520, 136, 1),     # ... rank 1
    (4150, 2056, 136, 2),    # ... rank 2, a last chunk of 8 channels
    # M <= 8: the CUDA-core weight stream
    (2, 640, 264, 32),
    (3, 1152, 1160, 0),
    (4, 200, 136, 7),        # K = 200 pads to 256
    (8, 4096, 520, 4),
    (7, 12288, 256, 4),      # long rows: several load batches per row
    (8, 32768, 128, 4),      # activations too large for one block's shared memory: decode tiles
]


@pytest.mark.parametrize("M,K,N,r", SMALL_SHAPES)
@pytest.mark.parametrize("out", [hsq.HSQ_OUT_F32, hsq.HSQ_OUT_BF16])
def test_layer_matches_oracle(M, K, N, r, out):
    layer = make_layer(_spec(M, K, N, r, seed=M + K + N + r))
    pl, act, Y, _ = _run_gpu(layer, out)
    _check_all(layer, pl, act, Y, out == hsq.HSQ_OUT_F32, f"{M}x{K}x{N} r{r}")


# groups of 128 (the pages' Qwen3-8B setting): decode and large tiles, split-K,
# K that pads the last group, the tensor-core and CUDA-core low-rank paths
SHAPES_G128 = [
    (1, 256, 128, 4),
    (16, 4096, 1024, 4),     # stream-K decode tile
    (17, 200, 264, 2),       # K = 200 pads to 256
    (40, 640, 136, 32),
    (64, 384, 520, 0),
    (65, 1152, 256, 4),
    (130, 320, 264, 15),
    (200, 1024, 1160, 4),
    (128, 2048, 1024, 4),    # large tile, split-K or whole tiles
    (300, 640, 512, 32),
    (520, 640, 392, 20),     # the many-rank kernels, two low-rank steps
    (6, 640, 264, 16),       # the CUDA-core weight stream, four lanes per group
    (8, 1024, 1160, 4),
    (4150, 1160, 136, 2),    # many-row activation kernel
    (4160, 392, 136, 4),     # ... K = 392 pads to 512
]


@pytest.mark.parametrize("M,K,N,r", SHAPES_G128)
@pytest.mark.parametrize("out", [hsq.HSQ_OUT_F32, hsq.HSQ_OUT_BF16])
def test_layer_matches_oracle_groups_of_128(M, K, N, r, out):
    layer = make_layer(_spec(M, K, N, r, seed=7 * M + K + N + r))
    pl, act, Y, _ = _run_gpu(layer, out, group=128)
    assert pl.w_scales.shape[0] == hsq.hsq_num_groups(K, 128)
    _check_all(layer, pl, act, Y, out == hsq.HSQ_OUT_F32, f"g128 {M}x{K}x{N} r{r}", group=128)


FUSED_SHAPES = [
    # (M, K, N, r, group)  -- the single-launch decode forward
    (1, 4096, 1160, 4, 64),
    (2, 640, 264, 2, 64),
    (3, 200, 136, 1, 64),     # K = 200 pads to 256
    (4, 1152, 520, 0, 64),
    (1, 1024, 264, 4, 128),
    (4, 384, 136, 2, 128),
    # the decode-tile form (cooperative launch, the step shared out over the grid)
    (5, 640, 264, 2, 64),      # from 5 tokens
    (8, 4096, 1160, 4, 64),
    (16, 1152, 520, 0, 64),    # no low-rank branch
    (16, 2048, 2048, 32, 64),  # largest rank
    (12, 200, 136, 7, 64),     # K = 200 pads to 256, an odd rank
    (3, 1152, 520, 8, 64),     # a rank the weight stream's form does not take
    (1, 2048, 4096, 32, 64),   # one token, rank 32
    (16, 12288, 1024, 4, 64),  # stream-K over many stages
    (16, 1024, 264, 16, 128),
    (9, 384, 136, 2, 128),
]


@pytest.mark.parametrize("M,K,N,r,group", FUSED_SHAPES)
@pytest.mark.parametrize("out", [hsq.HSQ_OUT_F32, hsq.HSQ_OUT_BF16])
def test_fused_forward_matches_oracle_and_two_calls(M, K, N, r, group, out):
    layer = make_layer(_spec(M, K, N, r, seed=11 * M + K + N + r + group))
    pl, act, Y2, _ = _run_gpu(layer, out, group=group)  # the two calls
    Yf = torch.empty_like(Y2)
    hsq.forward_fused(pl, layer.X.to(DEV), Yf, out=out)
    torch.cuda.synchronize()
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK
    ref = oracle_layer(layer.X, layer.W, layer.s, layer.L1 if r else None, layer.L2 if r else None, layer.bias,
                       group=group)
    check_y(to_np(Yf), ref["Y"], out == hsq.HSQ_OUT_F32, f"fused {M}x{K}x{N} r{r} g{group}")
    # the same codes and scales; U and the group sums up to their fp32 summation
    # order (from 5 tokens the two calls run the weight stream or other decode
    # tiles), so bf16 outputs may differ by the one rounding of the output: an ulp
    a, b = to_np(Yf).astype(np.float64), to_np(Y2).astype(np.float64)
    rms = np.sqrt(np.mean(ref["Y"] ** 2))
    tol = 1e-5 * rms if out == hsq.HSQ_OUT_F32 else 1e-5 * rms + O.bf16_ulp(np.maximum(np.abs(a), np.abs(b)))
    assert np.all(np.abs(a - b) <= tol), "fused forward differs from the two calls"


def test_strong_low_rank_branch_and_zero_bias():
    """Scale up L1, L2 so that the branch carries a large share of Y: a dropped
    or transposed branch would fail the tolerance by a wide margin."""
    layer = make_layer(_spec(96, 256, 192, 4, seed=5, bias=False))
    layer.L1 = (layer.L1.float() * 40).to(torch.bfloat16)
    layer.L2 = (layer.L2.float() * 40).to(torch.bfloat16)
    pl, act, Y, _ = _run_gpu(layer)
    ratio, r = _check_all(layer, pl, act, Y, True, "strong branch")
    ref = oracle_layer(layer.X, layer.W, layer.s, layer.L1, layer.L2, None)
    branch = ref["U"] @ to_np(layer.L2).astype(np.float64)
    assert np.sqrt(np.mean(branch ** 2)) > 0.2 * r


def test_zero_rows_and_zero_groups():
    layer = make_layer(_spec(40, 192, 128, 4, seed=9))
    X = layer.X.clone()
    X[3] = 0           # an all-zero token: every group scale is 0
    X[7, 64:128] = 0   # one all-zero group
    layer.X = X
    pl, act, Y, _ = _run_gpu(layer)
    _check_all(layer, pl, act, Y, True, "zero rows")
    assert np.all(to_np(act.x_scales)[:, 3] == 0)


def test_unit_smoothing_lossless_grid_matches_dense_product():
    """s = 1, r = 0, both operands on their INT4 grids: the layer is exact, so
    the GPU output equals the fp64 X W^T up to fp32 accumulation."""
    rng = np.random.default_rng(4)
    M, K, N = 130, 256, 264
    def grid(rows):
        q = rng.integers(-7, 8, size=(rows, K))
        q[:, ::64] = 7
        sc = 2.0 ** rng.integers(-6, 2, size=(rows, K // 64))
        return (q.reshape(rows, -1, 64) * sc[:, :, None]).reshape(rows, K)
    X = torch.tensor(grid(M), dtype=torch.bfloat16)
    W = torch.tensor(grid(N), dtype=torch.bfloat16)
    grid_x = to_np(X)  # exact: every value is q * 2^e with |q| <= 7
    pl = hsq.PackedLinear(W.to(DEV), torch.ones(K, device=DEV), None, None)
    act = hsq.ActBuffers(M, K, 0, DEV)
    Y = torch.empty((M, N), dtype=torch.float32, device=DEV)
    hsq.forward(pl, X.to(DEV), act, Y, workspace=pl.workspace(M), out=hsq.HSQ_OUT_F32)
    torch.cuda.synchronize()
    dense = O.dense_forward(grid_x, to_np(W), None)
    assert np.max(np.abs(to_np(Y) - dense)) <= 1e-6 * np.abs(dense).max()


def test_repeated_calls_are_deterministic_and_reuse_workspace():
    layer = make_layer(_spec(24, 4096, 2048, 4, seed=2))
    pl, act, Y, ws = _run_gpu(layer)
    assert ws is not None  # stream-K path (tiles cut between CTAs)
    assert int(ws[:16].view(torch.int32).abs().sum()) == 0  # counters back at zero
    Y0 = Y.clone()
    for _ in range(3):
        hsq.forward(pl, layer.X.to(DEV), act, Y, workspace=ws, out=hsq.HSQ_OUT_F32)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y0)


def test_few_token_stream_is_deterministic_without_workspace():
    layer = make_layer(_spec(3, 4096, 2048, 4, seed=2))
    pl, act, Y, ws = _run_gpu(layer)
    assert ws is None  # up to 8 tokens: the CUDA-core weight stream, no scratch
    Y0 = Y.clone()
    for _ in range(3):
        hsq.forward(pl, layer.X.to(DEV), act, Y, workspace=None, out=hsq.HSQ_OUT_F32)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y0)


def test_forced_timeout_reports_status_and_library_recovers():
    layer = make_layer(_spec(24, 256, 256, 4, seed=3))  # a decode tile (the weight stream has no waits)
    pl, act, Y, ws = _run_gpu(layer)
    Y_ok = Y.clone()
    hsq.hsq_debug_force_timeout(1, 30)
    hsq.forward(pl, layer.X.to(DEV), act, Y, workspace=ws, out=hsq.HSQ_OUT_F32)
    assert hsq.hsq_get_device_status() == hsq.HSQ_ERR_TIMEOUT
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK  # the word is cleared by the read
    if ws is not None:
        ws.zero_()  # an aborted call may leave split-K counters behind
    hsq.forward(pl, layer.X.to(DEV), act, Y, workspace=ws, out=hsq.HSQ_OUT_F32)
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK
    assert torch.equal(Y, Y_ok)


def test_fused_decode_tiles_repeat_bit_exact_and_recover_from_a_timeout():
    """The decode-tile form of the single launch: its grid barrier and stream-K
    counters are back at zero after every call (also after a forced timeout),
    so repeated calls give the same bits."""
    layer = make_layer(_spec(16, 4096, 2048, 8, seed=5))
    assert hsq.hsq_fused_form(16, 2048, 4096, 8, 64) == 2
    pl, act, Y2, ws = _run_gpu(layer)
    X = layer.X.to(DEV)
    Y = torch.empty_like(Y2)
    hsq.forward_fused(pl, X, Y, out=hsq.HSQ_OUT_F32)
    torch.cuda.synchronize()
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK
    Y0 = Y.clone()
    for _ in range(3):
        hsq.forward_fused(pl, X, Y, out=hsq.HSQ_OUT_F32)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y0)
    hsq.hsq_debug_force_timeout(1, 30)  # the producer issues nothing: the drain's waits run out
    hsq.forward_fused(pl, X, Y, out=hsq.HSQ_OUT_F32)
    assert hsq.hsq_get_device_status() == hsq.HSQ_ERR_TIMEOUT
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK
    hsq.forward_fused(pl, X, Y, out=hsq.HSQ_OUT_F32)
    torch.cuda.synchronize()
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK
    assert torch.equal(Y, Y0)


@pytest.mark.parametrize("M,K,N,r,group", [
    (300, 640, 512, 32, 64),    # tokens x outputs tiles with expanded operands
    (4150, 1160, 136, 4, 64),
    (130, 320, 264, 15, 128),   # groups of 128 expand from 65 tokens
    (16, 4096, 2048, 4, 64),    # decode tiles: the copy is not used
])
def test_expanded_weight_copy_gives_the_same_bits(M, K, N, r, group):
    """hsq_linear_forward_pre with the weights' E4M3 copy (hsq_expand_weights,
    made once) against hsq_linear_forward, which expands them on every call."""
    layer = make_layer(_spec(M, K, N, r, seed=17 * M + K + N + r + group))
    pl, act, Y, ws = _run_gpu(layer, hsq.HSQ_OUT_F32, group=group)
    pl.expand()
    assert pl.w_e4m3.numel() == hsq.hsq_weights_e4m3_bytes(N, K, group)
    Y2 = torch.empty_like(Y)
    hsq.forward(pl, layer.X.to(DEV), act, Y2, workspace=pl.workspace(M), out=hsq.HSQ_OUT_F32)
    torch.cuda.synchronize()
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK
    assert torch.equal(Y, Y2)


@pytest.mark.parametrize("M,K,N,r,group", [
    (4150, 1160, 136, 4, 64),   # the activation kernel writes the GEMM's E4M3 tiles (padding rows, padded K)
    (4150, 1160, 136, 2, 128),
    (4160, 392, 264, 0, 64),
    (4200, 520, 136, 1, 64),
    (4150, 1160, 136, 8, 64),   # rank 8: the two steps, with the expansion kernel
    (300, 640, 512, 32, 64),    # few rows: the two steps
    (16, 4096, 2048, 4, 64),    # decode tiles
])
def test_forward_x_gives_the_bits_of_the_two_calls(M, K, N, r, group):
    """hsq_linear_forward_x (X in, Y out), with and without the weights' E4M3
    copy, against hsq_quantize_act + hsq_linear_forward: the same bits, also on
    a workspace first filled with 0xFF bytes (E4M3 NaN patterns), which the
    padding rows of the activations' tiles must not keep."""
    layer = make_layer(_spec(M, K, N, r, seed=19 * M + K + N + r + group))
    pl, act, Y, ws = _run_gpu(layer, hsq.HSQ_OUT_F32, group=group)
    X = layer.X.to(DEV)
    for expanded in (False, True):
        if expanded:
            pl.expand()
        wsx = pl.workspace_x(M)
        wsx.fill_(0xFF)
        Yx = torch.full_like(Y, float("nan"))
        hsq.forward_x(pl, X, Yx, wsx, out=hsq.HSQ_OUT_F32)
        torch.cuda.synchronize()
        assert hsq.hsq_get_device_status() == hsq.HSQ_OK
        assert torch.equal(Yx, Y), f"forward_x (weights' copy: {expanded}) differs from the two calls"
        hsq.forward_x(pl, X, Yx, wsx, out=hsq.HSQ_OUT_F32)  # again, on the same workspace
        torch.cuda.synchronize()
        assert torch.equal(Yx, Y)


def test_invalid_arguments_launch_nothing():
    layer = make_layer(_spec(8, 128, 64, 4, seed=1))
    pl, act, Y, ws = _run_gpu(layer)
    with pytest.raises(hsq.HsqError) as e:
        hsq.hsq_linear_forward(act.x_codes, act.x_scales, act.U, pl.w_codes, pl.w_scales, pl.L2, None,
                               8, 64, 128, 4, Y, group=96)
    assert e.value.status == hsq.HSQ_ERR_UNSUPPORTED
    # a shape that needs split-K scratch, called without it: rejected before any
    # launch (the buffers above are far too small for it, so nothing may run)
    big = hsq.hsq_workspace_bytes(24, 4096, 12288, 4)
    with pytest.raises(hsq.HsqError) as e:
        hsq.hsq_linear_forward(act.x_codes, act.x_scales, act.U, pl.w_codes, pl.w_scales, pl.L2, None,
                               24, 4096, 12288, 4, Y, workspace=None)
    assert big > 0 and e.value.status == hsq.HSQ_ERR_INVALID_ARG
