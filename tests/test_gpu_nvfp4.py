"""GPU parity of the NVFP4 variant (DiRotQ page: E2M1 values, one E4M3 scale per
16 values, fp32 tensor scale) against oracle/nvfp4_oracle.py, through the C ABI.

Codes, packed bytes, E4M3 block scales (in the library's 128-row x 64-K atom
layout, padding included) and the tensor scales must match bit for bit; U within
fp32 accumulation error; outputs within the layer tolerance of tests/_helpers.py.
Shapes span several 128 x 128 tiles, ragged M, N and K tails (K not a multiple
of 64, a last stage with fewer than four K = 64 chunks), ranks 0..32, and the
degenerate cases (an all-zero token, an all-zero block, an all-zero input)."""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as F
from w4a4_rank_assisted_b200 import hsq
from w4a4_rank_assisted_b200.synth import LayerSpec, make_layer

from _helpers import check_y, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _e4m3_byte_of():
    """Value -> byte of every finite non-negative E4M3 number (bias 7, 3 mantissa
    bits, exponent field 0 subnormal, 0x7F is NaN)."""
    table = {}
    for b in range(0x7F):
        e, m = b >> 3, b & 7
        table[m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)] = b
    return table


E4M3_BYTE = _e4m3_byte_of()


def sf_atoms(scales, rows, K):
    """Oracle block scales [rows, Kp16/16] (E4M3 values) -> the library's bytes:
    atoms [ceil(rows/128)][Kq/64][512], row 128t+i and K-block 4c+j at byte
    16 (i % 32) + 4 (i / 32) + j of atom (t, c); padding 0."""
    Kq = -(-K // 64) * 64
    T, C = -(-rows // 128), Kq // 64
    full = np.zeros((T * 128, Kq // 16), dtype=np.uint8)
    byte = np.vectorize(lambda v: E4M3_BYTE[float(v)])(scales) if scales.size else scales
    full[:rows, :scales.shape[1]] = byte
    out = np.zeros((T, C, 512), dtype=np.uint8)
    for i in range(128):
        for j in range(4):
            out[:, :, 16 * (i % 32) + 4 * (i // 32) + j] = full.reshape(T, 128, C, 4)[:, i, :, j]
    return out.reshape(-1)


def packed_codes(codes, K):
    """Oracle codes [rows, Kp16] -> packed bytes [rows, Kq/2] (zero padding)."""
    Kq = -(-K // 64) * 64
    c = np.zeros((codes.shape[0], Kq), dtype=np.uint8)
    c[:, :codes.shape[1]] = codes
    return F.pack_fp4(c)


def _spec(M, K, N, r, seed, bias=True):
    return LayerSpec(f"fp4_{M}x{K}x{N}r{r}", M, K, N, r, act="outlier", outlier_frac=0.01, outlier_mult=30.0,
                     seed=seed, bias=bias)


def _run(layer, out):
    M, K = layer.X.shape
    N = layer.W.shape[0]
    r = layer.spec.r
    d = lambda t: None if t is None else t.to(DEV).contiguous()
    pl = hsq.Fp4Linear(d(layer.W), d(layer.s), d(layer.L1) if r else None, d(layer.L2) if r else None,
                       d(layer.bias))
    act = hsq.Fp4ActBuffers(M, K, r, DEV)
    Y = torch.empty((M, N), dtype=torch.float32 if out == hsq.HSQ_OUT_F32 else torch.bfloat16, device=DEV)
    hsq.fp4_forward(pl, d(layer.X), act, Y, out=out)
    torch.cuda.synchronize()
    assert hsq.hsq_get_device_status() == hsq.HSQ_OK
    return pl, act, Y


def _check(layer, pl, act, Y, out, where):
    M, K = layer.X.shape
    r = layer.spec.r
    f = lambda t: None if t is None else to_np(t)
    L1 = f(layer.L1) if r else None
    L2 = f(layer.L2) if r else None
    wc, ws, wg = F.nvfp4_pack_weights(f(layer.W), f(layer.s), L1, L2)
    xc, xs, xg, U = F.nvfp4_quantize_act(f(layer.X), f(layer.s), L1)
    N = wc.shape[0]
    assert np.float32(to_np(pl.w_gs)[0]) == wg, f"{where}: weight tensor scale"
    assert np.float32(to_np(act.x_gs)[0]) == xg, f"{where}: activation tensor scale"
    assert np.array_equal(to_np(pl.w_codes), packed_codes(wc, K)), f"{where}: weight codes"
    assert np.array_equal(to_np(pl.w_sf), sf_atoms(ws, N, K)), f"{where}: weight block scales"
    assert np.array_equal(to_np(act.x_codes), packed_codes(xc, K)), f"{where}: activation codes"
    assert np.array_equal(to_np(act.x_sf), sf_atoms(xs, M, K)), f"{where}: activation block scales"
    if r:
        Ug = to_np(act.U).astype(np.float64)
        assert np.max(np.abs(Ug - U)) <= 1e-5 * (np.abs(U).max() + 1e-30), f"{where}: U"
    bias = f(layer.bias) if layer.bias is not None else None
    Y_ref = F.nvfp4_linear_forward(xc, xs, xg, U, wc, ws, wg, L2, bias, K)
    return check_y(to_np(Y), Y_ref, out == hsq.HSQ_OUT_F32, where)


SHAPES = [
    # (M, K, N, r)
    (1, 64, 128, 4),
    (5, 96, 136, 1),       # K pads to 64-multiples (96 -> 128), ragged N
    (128, 256, 128, 4),    # one tile, one full stage
    (130, 320, 264, 4),    # ragged M and N tiles, five K chunks (a partial last stage)
    (256, 1152, 1152, 4),
    (64, 2048, 384, 32),   # largest rank
    (300, 640, 512, 0),    # no low-rank branch
    (97, 192, 136, 15),
    # the many-row activation kernel in its NVFP4 form
    (4150, 1160, 136, 4),  # ragged last block of rows, K pads to 1216
    (4150, 264, 136, 0),
    (4200, 520, 136, 1),
    (4160, 392, 264, 2),
]


@pytest.mark.parametrize("M,K,N,r", SHAPES)
@pytest.mark.parametrize("out", [hsq.HSQ_OUT_F32, hsq.HSQ_OUT_BF16])
def test_nvfp4_layer_matches_oracle(M, K, N, r, out):
    layer = make_layer(_spec(M, K, N, r, seed=3 * M + K + N + r))
    pl, act, Y = _run(layer, out)
    _check(layer, pl, act, Y, out, f"nvfp4 {M}x{K}x{N} r{r}")


@pytest.mark.parametrize("M", [40, 4160])  # 4160: the many-row activation kernel
def test_nvfp4_zero_token_zero_block_and_zero_input(M):
    layer = make_layer(_spec(M, 192, 128, 4, seed=9))
    X = layer.X.clone()
    X[3] = 0            # an all-zero token: every block scale 0, codes 0
    X[7, 16:32] = 0     # one all-zero 16-value block
    layer.X = X
    pl, act, Y = _run(layer, hsq.HSQ_OUT_F32)
    _check(layer, pl, act, Y, hsq.HSQ_OUT_F32, "zero token / block")
    # an all-zero input: g = 0, every scale and code 0, Y = U L2 + b = b
    layer.X = torch.zeros_like(X)
    pl, act, Y = _run(layer, hsq.HSQ_OUT_F32)
    assert to_np(act.x_gs)[0] == 0.0
    assert not to_np(act.x_codes).any() and not to_np(act.x_sf).any()
    _check(layer, pl, act, Y, hsq.HSQ_OUT_F32, "zero input")


def test_nvfp4_full_size_flux_mlp_up_sampled_rows():
    """The FLUX.1 MLP-up shape (M = 4608, K = 3072, N = 12288, r = 4) in the launch
    configuration the benchmark times: weights bit-exact in full, activations and
    outputs on sampled token rows."""
    spec = LayerSpec("flux_mlp_up_fp4", 4608, 3072, 12288, 4, act="outlier", outlier_frac=0.005,
                     outlier_mult=50.0, seed=1)
    layer = make_layer(spec)
    pl, act, Y = _run(layer, hsq.HSQ_OUT_BF16)
    f = to_np
    wc, ws, wg = F.nvfp4_pack_weights(f(layer.W), f(layer.s), f(layer.L1), f(layer.L2))
    assert np.float32(f(pl.w_gs)[0]) == wg
    assert np.array_equal(f(pl.w_codes), packed_codes(wc, spec.K))
    assert np.array_equal(f(pl.w_sf), sf_atoms(ws, spec.N, spec.K))
    # the activation tensor scale depends on every row: take it from the full oracle step
    xc, xs, xg, U = F.nvfp4_quantize_act(f(layer.X), f(layer.s), f(layer.L1))
    assert np.float32(f(act.x_gs)[0]) == xg
    rows = np.array(sorted({0, spec.M - 1} | set(np.random.default_rng(0).integers(0, spec.M, 40).tolist())))
    assert np.array_equal(f(act.x_codes)[rows], packed_codes(xc[rows], spec.K))
    Y_ref = F.nvfp4_linear_forward(xc[rows], xs[rows], xg, U[rows], wc, ws, wg, f(layer.L2), None, spec.K)
    check_y(f(Y)[rows], Y_ref, False, "nvfp4 FLUX MLP up")


@pytest.mark.parametrize("huge", [False, True])  # values above 2^100 set g for the whole tensor
def test_nvfp4_extreme_values_and_smoothing_factors(huge):
    """Blocks that mix a normal absmax with bf16 subnormals and values below
    2^-100, blocks of such tiny values only, values above 2^100, and channels
    whose smoothing factor lies outside [2^-24, 2^24] (last 256-channel chunk
    only), at enough rows for the many-row kernel: codes, E4M3 scales and the
    tensor scale bit for bit."""
    rng = np.random.default_rng(4)
    M, K, N, r = 4400, 1024, 128, 4
    layer = make_layer(_spec(M, K, N, r, seed=13))
    X = layer.X.float().numpy()
    tiny = np.array([2.0 ** -133, 2.0 ** -126, 2.0 ** -110, 2.0 ** -101, 2.0 ** -100], dtype=np.float32)
    sign = lambda n: rng.choice(np.array([-1.0, 1.0], dtype=np.float32), n)
    for m in range(0, M, 7):
        kind = (m // 7) % 4
        if kind == 0:
            idx = rng.choice(768, 30, replace=False)
            X[m, idx] = rng.choice(tiny, 30) * sign(30)
        elif kind == 1:
            b = rng.integers(48)
            X[m, b * 16:(b + 1) * 16] = rng.choice(tiny, 16) * sign(16)
        elif kind == 2 and huge:
            idx = rng.choice(768, 2, replace=False)
            X[m, idx] = (2.0 ** rng.uniform(100.0, 110.0, 2)).astype(np.float32) * sign(2)
    s = layer.s.float().numpy().copy()
    s[900:904] = np.array([2.0 ** -30, 2.0 ** -25, 2.0 ** 25, 2.0 ** 30], dtype=np.float32)
    layer.X = torch.tensor(X).to(torch.bfloat16)
    layer.s = torch.tensor(s)
    pl, act, Y = _run(layer, hsq.HSQ_OUT_F32)
    f = to_np
    xc, xs, xg, U = F.nvfp4_quantize_act(f(layer.X), f(layer.s), f(layer.L1))
    assert np.float32(f(act.x_gs)[0]) == xg
    assert np.array_equal(f(act.x_codes), packed_codes(xc, K))
    assert np.array_equal(f(act.x_sf), sf_atoms(xs, M, K))
