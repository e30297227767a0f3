"""Host-side checks of the C ABI (no GPU needed): the library builds, loads and
exports every symbol that include/hsq.h declares; size helpers; argument
validation that rejects a call before anything is launched."""
import ctypes
import os
import re

import pytest

from w4a4_rank_assisted_b200 import hsq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hsq.h")

# fake, non-null device addresses: the calls below must fail validation before
# touching them
A = 1 << 20          # 16-byte aligned
MIS = (1 << 20) + 4  # misaligned


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hsq_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = hsq.load()
    declared = _declared()
    assert declared, "no declarations parsed"
    assert set(declared) == set(hsq.EXPORTED)
    for name in declared:
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_size_helpers():
    assert hsq.hsq_num_groups(64) == 1
    assert hsq.hsq_num_groups(96) == 2
    assert hsq.hsq_num_groups(5600) == 88
    assert hsq.hsq_codes_bytes(3, 96) == 3 * 64
    assert hsq.hsq_codes_bytes(4608, 3072) == 4608 * 1536
    assert hsq.hsq_scales_ld(1) == 4 and hsq.hsq_scales_ld(4) == 4 and hsq.hsq_scales_ld(5) == 8
    assert hsq.hsq_scales_bytes(5, 128) == 2 * 8 * 4
    assert hsq.load().hsq_num_groups(10, 0) == 0


def test_status_strings():
    names = [hsq.status_string(i) for i in range(6)]
    assert names == ["HSQ_OK", "HSQ_ERR_INVALID_ARG", "HSQ_ERR_ALIGNMENT", "HSQ_ERR_UNSUPPORTED",
                     "HSQ_ERR_CUDA", "HSQ_ERR_TIMEOUT"]


def _fwd(lib, **kw):
    a = dict(xc=A, xs=A, U=A, wc=A, ws=A, L2=A, b=None, M=16, N=64, K=64, r=4, g=64, Y=A, out=0,
             wsp=None, wsb=0)
    a.update(kw)
    return lib.hsq_linear_forward(a["xc"], a["xs"], a["U"], a["wc"], a["ws"], a["L2"], a["b"], a["M"],
                                  a["N"], a["K"], a["r"], a["g"], a["Y"], a["out"], a["wsp"], a["wsb"],
                                  None)


def test_forward_argument_validation():
    lib = hsq.load()
    assert _fwd(lib, g=96) == hsq.HSQ_ERR_UNSUPPORTED
    assert _fwd(lib, g=32) == hsq.HSQ_ERR_UNSUPPORTED
    assert _fwd(lib, r=33) == hsq.HSQ_ERR_UNSUPPORTED
    assert _fwd(lib, r=-1) == hsq.HSQ_ERR_INVALID_ARG
    assert _fwd(lib, K=100) == hsq.HSQ_ERR_UNSUPPORTED
    assert _fwd(lib, N=60) == hsq.HSQ_ERR_UNSUPPORTED
    assert _fwd(lib, M=0) == hsq.HSQ_ERR_INVALID_ARG
    assert _fwd(lib, N=0) == hsq.HSQ_ERR_INVALID_ARG
    assert _fwd(lib, K=(1 << 20) + 8) == hsq.HSQ_ERR_INVALID_ARG
    assert _fwd(lib, out=7) == hsq.HSQ_ERR_INVALID_ARG
    assert _fwd(lib, xc=None) == hsq.HSQ_ERR_INVALID_ARG
    assert _fwd(lib, Y=None) == hsq.HSQ_ERR_INVALID_ARG
    assert _fwd(lib, L2=None) == hsq.HSQ_ERR_INVALID_ARG          # r > 0 needs L2
    assert _fwd(lib, r=0) == hsq.HSQ_ERR_INVALID_ARG              # r == 0 wants L2 == U == NULL
    assert _fwd(lib, xs=MIS) == hsq.HSQ_ERR_ALIGNMENT
    assert _fwd(lib, b=MIS) == hsq.HSQ_ERR_ALIGNMENT


def test_fused_forward_argument_validation():
    lib = hsq.load()
    f = lib.hsq_linear_forward_fused

    def call(**kw):
        a = dict(X=A, s=A, L1=A, wc=A, ws=A, L2=A, b=None, M=1, N=64, K=64, r=4, g=64, Y=A, out=0)
        a.update(kw)
        return f(a["X"], a["s"], a["L1"], a["wc"], a["ws"], a["L2"], a["b"], a["M"], a["N"], a["K"], a["r"],
                 a["g"], a["Y"], a["out"], None)

    # (only shapes the library rejects before launching are called: fake
    # pointers must never reach a launch)
    assert call(M=17) == hsq.HSQ_ERR_UNSUPPORTED         # more than 16 tokens: the two-call path
    assert call(r=33) == hsq.HSQ_ERR_UNSUPPORTED
    assert call(M=16, K=1 << 20) == hsq.HSQ_ERR_UNSUPPORTED  # the codes alone overflow the library's array
    assert call(g=96) == hsq.HSQ_ERR_UNSUPPORTED
    assert call(M=0) == hsq.HSQ_ERR_INVALID_ARG
    assert call(X=None) == hsq.HSQ_ERR_INVALID_ARG
    assert call(L1=None) == hsq.HSQ_ERR_INVALID_ARG      # r > 0 needs L1 and L2
    assert call(r=0) == hsq.HSQ_ERR_INVALID_ARG          # r == 0 wants L1 == L2 == NULL
    assert call(X=MIS) == hsq.HSQ_ERR_ALIGNMENT


def test_expanded_weights_calls_validate_and_size():
    """The weights' E4M3 copy: its size (Kp x N rounded up to 256), and the
    argument checks of the expansion and of the forward that reads it (only
    calls rejected before any launch are made: fake pointers)."""
    lib = hsq.load()
    assert hsq.hsq_weights_e4m3_bytes(300, 200, 64) == 512 * 256
    assert hsq.hsq_weights_e4m3_bytes(12288, 3072, 64) == 12288 * 3072
    assert hsq.hsq_weights_e4m3_bytes(100, 200, 128) == 256 * 256
    assert hsq.hsq_weights_e4m3_bytes(0, 64, 64) == 0 and hsq.hsq_weights_e4m3_bytes(64, 64, 96) == 0
    ex = lib.hsq_expand_weights
    assert ex(None, 64, 64, 64, A, None) == hsq.HSQ_ERR_INVALID_ARG
    assert ex(A, 64, 64, 64, MIS, None) == hsq.HSQ_ERR_ALIGNMENT
    assert ex(A, 64, 64, 96, A, None) == hsq.HSQ_ERR_UNSUPPORTED
    pre = lib.hsq_linear_forward_pre
    args = [A, A, A, A, A, A, A, None, 300, 64, 64, 4, 64, A, 0, A, 1 << 30, None]
    call = lambda **kw: pre(*[kw.get(str(i), a) for i, a in enumerate(args)])
    assert call(**{"5": None}) == hsq.HSQ_ERR_INVALID_ARG   # the expanded copy is required
    assert call(**{"5": MIS}) == hsq.HSQ_ERR_ALIGNMENT
    assert call(**{"0": None}) == hsq.HSQ_ERR_INVALID_ARG
    # the workspace without the weights' part is smaller wherever the copy is used
    for M, N, K in ((300, 512, 640), (4608, 12288, 3072)):
        assert hsq.hsq_workspace_bytes_pre(M, N, K, 4) < hsq.hsq_workspace_bytes(M, N, K, 4)
    assert hsq.hsq_workspace_bytes_pre(16, 2048, 4096, 4) == hsq.hsq_workspace_bytes(16, 2048, 4096, 4)


def test_forward_x_validates_before_launching():
    """hsq_linear_forward_x: workspace required and large enough, alignment of
    every pointer; all checked before anything is launched (fake pointers)."""
    lib = hsq.load()
    fx = lib.hsq_linear_forward_x
    need = hsq.hsq_workspace_bytes_x(4608, 12288, 3072, 4, 64, True)
    assert need > 0
    assert hsq.hsq_workspace_bytes_x(4608, 12288, 3072, 4, 64, False) > need  # plus the weights' expansion
    assert hsq.hsq_workspace_bytes_x(0, 64, 64, 4, 64, True) == 0
    args = [A, A, A, A, A, A, A, None, 4608, 12288, 3072, 4, 64, A, 0, A, need, None]
    call = lambda **kw: fx(*[kw.get(str(i), a) for i, a in enumerate(args)])
    assert call(**{"15": None}) == hsq.HSQ_ERR_INVALID_ARG       # no workspace
    assert call(**{"16": need - 1}) == hsq.HSQ_ERR_INVALID_ARG   # too small
    assert call(**{"5": MIS}) == hsq.HSQ_ERR_ALIGNMENT
    assert call(**{"0": MIS}) == hsq.HSQ_ERR_ALIGNMENT
    assert call(**{"2": None}) == hsq.HSQ_ERR_INVALID_ARG        # r > 0 needs L1
    assert call(**{"12": 96}) == hsq.HSQ_ERR_UNSUPPORTED


def test_fused_form_query_and_its_python_restatement():
    """hsq_fused_form (host arithmetic, no launch) against fused_supported and
    the weight stream's shared-memory restatement, on both sides of each limit."""
    form = hsq.hsq_fused_form
    assert form(1, 12288, 4096, 4, 64) == 1 and form(4, 12288, 4096, 2, 128) == 1
    assert form(5, 12288, 4096, 4, 64) == 2 and form(16, 4096, 12288, 4, 64) == 2
    assert form(2, 4096, 4096, 8, 64) == 2 and form(16, 4096, 4096, 32, 128) == 2
    assert form(17, 4096, 4096, 4, 64) == 0 and form(16, 64, 1 << 20, 4, 64) == 0
    assert form(4, 4096, 4096, 33, 64) == 0 and form(4, 4096, 4100, 4, 64) == 0
    if hsq._sm_count() != 148:
        return
    # the weight stream's shared-memory limit, at its edge
    for N, M in ((4096, 4), (12288, 1), (12288, 4)):
        lo, hi = 64, 1 << 17
        while hi - lo > 64:  # the largest K (a multiple of 64) the restatement gives the stream
            mid = (lo + hi) // 2 // 64 * 64
            lo, hi = (mid, hi) if hsq.stream_smem_fits(M, N, mid, 64, nsm=148) else (lo, mid)
        assert form(M, N, lo, 4, 64) == 1 and form(M, N, lo + 64, 4, 64) == 2
    # the decode tiles' array limit, at its edge (K where the codes fill it)
    for N, M, r, g in ((4096, 16, 4, 64), (12288, 9, 32, 128), (128, 16, 0, 64)):
        lo, hi = 64, 1 << 20
        while hi - lo > 64:
            mid = (lo + hi) // 2 // 64 * 64
            lo, hi = (mid, hi) if hsq.fused_supported(M, mid, r, g, N=N, nsm=148) else (lo, mid)
        assert form(M, N, lo, r, g) == 2 and form(M, N, lo + 64, r, g) == 0
    for M, K, r, g, N in ((1, 4096, 4, 64, 12288), (3, 1152, 8, 64, 520), (16, 4096, 4, 64, 12288),
                          (12, 200, 7, 64, 136), (16, 1024, 16, 128, 264)):
        assert hsq.fused_supported(M, K, r, g, N=N, nsm=148) == (form(M, N, K, r, g) != 0)


def test_lowrank_helper_argument_validation():
    lib = hsq.load()
    f = lib.hsq_lowrank_init
    ws = hsq.hsq_lowrank_workspace_bytes(64, 32, 4)
    assert ws >= 4 * 64 * 32
    assert hsq.hsq_lowrank_workspace_bytes(64, 32, 0) == 0
    assert hsq.hsq_lowrank_workspace_bytes(64, 32, 33) == 0

    def call(**kw):
        a = dict(W=A, s=A, N=64, K=32, r=4, it=8, seed=0, L1=A, L2=A, ws=A, wsb=ws)
        a.update(kw)
        return f(a["W"], a["s"], a["N"], a["K"], a["r"], a["it"], a["seed"], a["L1"], a["L2"], a["ws"], a["wsb"],
                 None)

    assert call(r=0) == hsq.HSQ_ERR_UNSUPPORTED
    assert call(r=33) == hsq.HSQ_ERR_UNSUPPORTED
    assert call(N=16, K=8, r=9) == hsq.HSQ_ERR_UNSUPPORTED   # rank above min(N, K)
    assert call(it=65) == hsq.HSQ_ERR_INVALID_ARG
    assert call(ws=None) == hsq.HSQ_ERR_INVALID_ARG
    assert call(wsb=ws - 1) == hsq.HSQ_ERR_INVALID_ARG
    assert call(W=MIS) == hsq.HSQ_ERR_ALIGNMENT


def test_pack_and_act_argument_validation():
    lib = hsq.load()
    pk = lib.hsq_pack_weights
    assert pk(A, A, A, A, 64, 64, 4, 32, A, A, None) == hsq.HSQ_ERR_UNSUPPORTED
    assert pk(A, A, None, A, 64, 64, 4, 64, A, A, None) == hsq.HSQ_ERR_INVALID_ARG
    assert pk(A, A, A, A, 64, 66, 4, 64, A, A, None) == hsq.HSQ_ERR_UNSUPPORTED
    assert pk(A, A, A, A, 64, 64, 4, 64, MIS, A, None) == hsq.HSQ_ERR_ALIGNMENT
    assert pk(None, A, A, A, 64, 64, 4, 64, A, A, None) == hsq.HSQ_ERR_INVALID_ARG
    qa = lib.hsq_quantize_act
    assert qa(A, A, A, 8, 64, 4, 64, A, A, None, None) == hsq.HSQ_ERR_INVALID_ARG  # U missing
    assert qa(A, A, A, 8, 64, 40, 64, A, A, A, None) == hsq.HSQ_ERR_UNSUPPORTED
    assert qa(MIS, A, A, 8, 64, 4, 64, A, A, A, None) == hsq.HSQ_ERR_ALIGNMENT
    assert qa(A, A, A, 0, 64, 4, 64, A, A, A, None) == hsq.HSQ_ERR_INVALID_ARG


def test_workspace_needs_are_consistent():
    # More than 64 tokens: both code matrices expanded to E4M3 bytes, rows padded
    # to whole 128 x 256 tiles (no split-K: the 1728 tiles fill the device).
    assert hsq.hsq_workspace_bytes(4608, 12288, 3072, 4) == (4608 + 12288) * 3072
    # decode tiles: only split-K scratch (counters and partial tiles)
    assert 0 < hsq.hsq_workspace_bytes(16, 4096, 12288, 4) < 16 << 20
    # up to 8 tokens: the weight stream needs no workspace, unless K is too long
    # for one block's shared memory (then the decode tiles and their scratch)
    assert hsq.hsq_workspace_bytes(1, 4096, 12288, 4) == 0
    assert hsq.hsq_workspace_bytes(8, 12288, 4096, 4) == 0
    assert hsq.hsq_workspace_bytes(8, 4096, 32768, 4) > 0  # K = 32768
    assert hsq.hsq_workspace_bytes(0, 4096, 12288, 4) == 0


def test_fp4_size_helpers():
    # K rounded up to 64; scale atoms of 128 rows x 64 K (512 bytes)
    assert hsq.hsq_fp4_codes_bytes(3, 96) == 3 * 64
    assert hsq.hsq_fp4_codes_bytes(4608, 3072) == 4608 * 1536
    assert hsq.hsq_fp4_scales_bytes(1, 64) == 512
    assert hsq.hsq_fp4_scales_bytes(129, 200) == 2 * 4 * 512
    assert hsq.hsq_fp4_scales_bytes(12288, 3072) == 96 * 48 * 512


def test_fp4_argument_validation():
    lib = hsq.load()
    # weights: K % 8, rank, L1/L2 presence, alignment
    assert lib.hsq_fp4_pack_weights(A, A, A, A, 64, 60, 4, A, A, A, None) == hsq.HSQ_ERR_UNSUPPORTED
    assert lib.hsq_fp4_pack_weights(A, A, A, A, 64, 64, 33, A, A, A, None) == hsq.HSQ_ERR_UNSUPPORTED
    assert lib.hsq_fp4_pack_weights(A, A, None, A, 64, 64, 4, A, A, A, None) == hsq.HSQ_ERR_INVALID_ARG
    assert lib.hsq_fp4_pack_weights(A, A, A, A, 64, 64, 4, A, A, None, None) == hsq.HSQ_ERR_INVALID_ARG
    assert lib.hsq_fp4_pack_weights(A, A, A, A, 64, 64, 4, A, MIS, A, None) == hsq.HSQ_ERR_ALIGNMENT
    # activations
    assert lib.hsq_fp4_quantize_act(A, A, A, 0, 64, 4, A, A, A, A, None) == hsq.HSQ_ERR_INVALID_ARG
    assert lib.hsq_fp4_quantize_act(A, A, A, 8, 64, 4, A, A, A, None, None) == hsq.HSQ_ERR_INVALID_ARG
    assert lib.hsq_fp4_quantize_act(A, A, A, 8, 64, 4, A, A, MIS, A, None) == hsq.HSQ_ERR_ALIGNMENT
    # forward: N % 8, output type, scales present
    f = lib.hsq_fp4_linear_forward
    assert f(A, A, A, A, A, A, A, A, None, 16, 60, 64, 4, A, 0, None) == hsq.HSQ_ERR_UNSUPPORTED
    assert f(A, A, A, A, A, A, A, A, None, 16, 64, 64, 4, A, 7, None) == hsq.HSQ_ERR_INVALID_ARG
    assert f(A, None, A, A, A, A, A, A, None, 16, 64, 64, 4, A, 0, None) == hsq.HSQ_ERR_INVALID_ARG
    assert f(A, A, A, None, A, A, A, A, None, 16, 64, 64, 4, A, 0, None) == hsq.HSQ_ERR_INVALID_ARG
    assert f(A, A, A, A, A, A, A, A, MIS, 16, 64, 64, 4, A, 0, None) == hsq.HSQ_ERR_ALIGNMENT
