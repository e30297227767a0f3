"""Python binding of libhsq's C ABI (include/hsq.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libhsq.so``.  Tensors are torch CUDA tensors (torch supplies device memory and
streams); their ``data_ptr()`` values are handed to the C functions of the
same names.  There is no CPU fallback: if the library is missing or a call
fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

GROUP = 64

HSQ_OK = 0
HSQ_ERR_INVALID_ARG = 1
HSQ_ERR_ALIGNMENT = 2
HSQ_ERR_UNSUPPORTED = 3
HSQ_ERR_CUDA = 4
HSQ_ERR_TIMEOUT = 5
HSQ_ERR_SCRATCH_LIMIT = 6
#: Size of the built-in scratch array of hsq_linear_forward_noalloc.
HSQ_NOALLOC_SCRATCH_BYTES = 16 << 20
HSQ_OUT_BF16 = 0
HSQ_OUT_F32 = 1

#: Every symbol that include/hsq.h declares.
EXPORTED = (
    "hsq_num_groups", "hsq_codes_bytes", "hsq_scales_ld", "hsq_scales_bytes",
    "hsq_workspace_bytes", "hsq_pack_weights", "hsq_quantize_act",
    "hsq_linear_forward", "hsq_status_string", "hsq_get_device_status",
    "hsq_debug_force_timeout", "hsq_linear_forward_noalloc", "hsq_linear_forward_fused", "hsq_fused_form",
    "hsq_weights_e4m3_bytes", "hsq_expand_weights", "hsq_workspace_bytes_pre", "hsq_linear_forward_pre",
    "hsq_workspace_bytes_x", "hsq_linear_forward_x",
    "hsq_lowrank_workspace_bytes", "hsq_lowrank_init",
    "hsq_fp4_codes_bytes", "hsq_fp4_scales_bytes", "hsq_fp4_pack_weights", "hsq_fp4_quantize_act",
    "hsq_fp4_linear_forward",
)


class HsqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {status_string(status)}")


_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return _build.LIB_PATH


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libhsq.so (building it first if it is absent and nvcc is available)."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB_PATH
    if not os.path.exists(path):
        if not build_if_missing:
            raise RuntimeError(f"libhsq.so not built at {path}")
        _build.build()
    lib = ctypes.CDLL(path)
    c = ctypes
    vp, i, sz = c.c_void_p, c.c_int, c.c_size_t
    lib.hsq_num_groups.argtypes = [i, i]; lib.hsq_num_groups.restype = i
    lib.hsq_codes_bytes.argtypes = [i, i, i]; lib.hsq_codes_bytes.restype = sz
    lib.hsq_scales_ld.argtypes = [i]; lib.hsq_scales_ld.restype = i
    lib.hsq_scales_bytes.argtypes = [i, i, i]; lib.hsq_scales_bytes.restype = sz
    lib.hsq_workspace_bytes.argtypes = [i, i, i, i]; lib.hsq_workspace_bytes.restype = sz
    lib.hsq_pack_weights.argtypes = [vp, vp, vp, vp, i, i, i, i, vp, vp, vp]
    lib.hsq_pack_weights.restype = i
    lib.hsq_quantize_act.argtypes = [vp, vp, vp, i, i, i, i, vp, vp, vp, vp]
    lib.hsq_quantize_act.restype = i
    lib.hsq_linear_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp, sz, vp]
    lib.hsq_linear_forward.restype = i
    lib.hsq_linear_forward_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp]
    lib.hsq_linear_forward_fused.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp]
    lib.hsq_linear_forward_fused.restype = i
    lib.hsq_fused_form.argtypes = [i, i, i, i, i]
    lib.hsq_fused_form.restype = i
    lib.hsq_weights_e4m3_bytes.argtypes = [i, i, i]
    lib.hsq_weights_e4m3_bytes.restype = ctypes.c_size_t
    lib.hsq_expand_weights.argtypes = [vp, i, i, i, vp, vp]
    lib.hsq_expand_weights.restype = i
    lib.hsq_workspace_bytes_pre.argtypes = [i, i, i, i]
    lib.hsq_workspace_bytes_pre.restype = ctypes.c_size_t
    lib.hsq_linear_forward_pre.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp, ctypes.c_size_t, vp]
    lib.hsq_linear_forward_pre.restype = i
    lib.hsq_workspace_bytes_x.argtypes = [i, i, i, i, i, i]
    lib.hsq_workspace_bytes_x.restype = ctypes.c_size_t
    lib.hsq_linear_forward_x.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp, ctypes.c_size_t, vp]
    lib.hsq_linear_forward_x.restype = i
    lib.hsq_lowrank_workspace_bytes.argtypes = [i, i, i]; lib.hsq_lowrank_workspace_bytes.restype = sz
    lib.hsq_lowrank_init.argtypes = [vp, vp, i, i, i, i, c.c_ulonglong, vp, vp, vp, sz, vp]
    lib.hsq_lowrank_init.restype = i
    lib.hsq_linear_forward_noalloc.restype = i
    lib.hsq_status_string.argtypes = [i]; lib.hsq_status_string.restype = c.c_char_p
    lib.hsq_get_device_status.argtypes = [vp]; lib.hsq_get_device_status.restype = i
    lib.hsq_debug_force_timeout.argtypes = [i, i]; lib.hsq_debug_force_timeout.restype = None
    lib.hsq_fp4_codes_bytes.argtypes = [i, i]; lib.hsq_fp4_codes_bytes.restype = sz
    lib.hsq_fp4_scales_bytes.argtypes = [i, i]; lib.hsq_fp4_scales_bytes.restype = sz
    lib.hsq_fp4_pack_weights.argtypes = [vp, vp, vp, vp, i, i, i, vp, vp, vp, vp]
    lib.hsq_fp4_pack_weights.restype = i
    lib.hsq_fp4_quantize_act.argtypes = [vp, vp, vp, i, i, i, vp, vp, vp, vp, vp]
    lib.hsq_fp4_quantize_act.restype = i
    lib.hsq_fp4_linear_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, vp, i, vp]
    lib.hsq_fp4_linear_forward.restype = i
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().hsq_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libhsq takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("libhsq takes contiguous tensors only")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, what: str) -> None:
    if status != HSQ_OK:
        raise HsqError(status, what)


# ---------------------------------------------------------------- sizes
def hsq_num_groups(K: int, group: int = GROUP) -> int:
    return load().hsq_num_groups(K, group)


def hsq_codes_bytes(rows: int, K: int, group: int = GROUP) -> int:
    return load().hsq_codes_bytes(rows, K, group)


def hsq_scales_ld(rows: int) -> int:
    return load().hsq_scales_ld(rows)


def hsq_scales_bytes(rows: int, K: int, group: int = GROUP) -> int:
    return load().hsq_scales_bytes(rows, K, group)


def hsq_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return load().hsq_workspace_bytes(M, N, K, r)


# ---------------------------------------------------------------- the three calls
def hsq_pack_weights(W, s, L1, L2, N, K, r, w_codes, w_scales, group=GROUP, stream=None) -> None:
    _check(load().hsq_pack_weights(_ptr(W), _ptr(s), _ptr(L1), _ptr(L2), N, K, r, group,
                                   _ptr(w_codes), _ptr(w_scales), _stream(stream)), "hsq_pack_weights")


def hsq_quantize_act(X, s, L1, M, K, r, x_codes, x_scales, U, group=GROUP, stream=None) -> None:
    _check(load().hsq_quantize_act(_ptr(X), _ptr(s), _ptr(L1), M, K, r, group,
                                   _ptr(x_codes), _ptr(x_scales), _ptr(U), _stream(stream)),
           "hsq_quantize_act")


def hsq_linear_forward(x_codes, x_scales, U, w_codes, w_scales, L2, bias, M, N, K, r, Y,
                       out: int = HSQ_OUT_BF16, workspace=None, ws_bytes: int = 0,
                       group=GROUP, stream=None) -> None:
    _check(load().hsq_linear_forward(_ptr(x_codes), _ptr(x_scales), _ptr(U), _ptr(w_codes),
                                     _ptr(w_scales), _ptr(L2), _ptr(bias), M, N, K, r, group,
                                     _ptr(Y), int(out), _ptr(workspace), int(ws_bytes),
                                     _stream(stream)), "hsq_linear_forward")


def hsq_linear_forward_noalloc(x_codes, x_scales, U, w_codes, w_scales, L2, bias, M, N, K, r, Y,
                               out: int = HSQ_OUT_BF16, group=GROUP, stream=None) -> None:
    """hsq_linear_forward with the library's own scratch array instead of a
    workspace: for callers that must not allocate.  Calls that overlap on the
    GPU share that array and race; the first call on a device must come
    before any stream capture."""
    _check(load().hsq_linear_forward_noalloc(_ptr(x_codes), _ptr(x_scales), _ptr(U), _ptr(w_codes),
                                             _ptr(w_scales), _ptr(L2), _ptr(bias), M, N, K, r, group,
                                             _ptr(Y), int(out), _stream(stream)),
           "hsq_linear_forward_noalloc")


def hsq_weights_e4m3_bytes(N: int, K: int, group: int = GROUP) -> int:
    return int(load().hsq_weights_e4m3_bytes(N, K, group))


def hsq_expand_weights(w_codes, N, K, w_e4m3, group=GROUP, stream=None) -> None:
    _check(load().hsq_expand_weights(_ptr(w_codes), N, K, group, _ptr(w_e4m3), _stream(stream)),
           "hsq_expand_weights")


def hsq_workspace_bytes_pre(M: int, N: int, K: int, r: int) -> int:
    return int(load().hsq_workspace_bytes_pre(M, N, K, r))


def hsq_linear_forward_pre(x_codes, x_scales, U, w_codes, w_scales, w_e4m3, L2, bias, M, N, K, r, Y,
                           out: int = HSQ_OUT_BF16, workspace=None, ws_bytes: int = 0,
                           group=GROUP, stream=None) -> None:
    _check(load().hsq_linear_forward_pre(_ptr(x_codes), _ptr(x_scales), _ptr(U), _ptr(w_codes),
                                         _ptr(w_scales), _ptr(w_e4m3), _ptr(L2), _ptr(bias), M, N, K, r, group,
                                         _ptr(Y), int(out), _ptr(workspace), int(ws_bytes),
                                         _stream(stream)), "hsq_linear_forward_pre")


def hsq_workspace_bytes_x(M: int, N: int, K: int, r: int, group: int = GROUP, with_w_e4m3: bool = True) -> int:
    return int(load().hsq_workspace_bytes_x(M, N, K, r, group, 1 if with_w_e4m3 else 0))


def hsq_linear_forward_x(X, s, L1, w_codes, w_scales, w_e4m3, L2, bias, M, N, K, r, Y,
                         out: int = HSQ_OUT_BF16, workspace=None, ws_bytes: int = 0,
                         group=GROUP, stream=None) -> None:
    _check(load().hsq_linear_forward_x(_ptr(X), _ptr(s), _ptr(L1), _ptr(w_codes), _ptr(w_scales), _ptr(w_e4m3),
                                       _ptr(L2), _ptr(bias), M, N, K, r, group, _ptr(Y), int(out),
                                       _ptr(workspace), int(ws_bytes), _stream(stream)), "hsq_linear_forward_x")


def hsq_linear_forward_fused(X, s, L1, w_codes, w_scales, L2, bias, M, N, K, r, Y,
                             out: int = HSQ_OUT_BF16, group=GROUP, stream=None) -> None:
    """The activation step and the forward in one launch (M <= 4, r in
    {0, 1, 2, 4}); HSQ_ERR_UNSUPPORTED otherwise."""
    _check(load().hsq_linear_forward_fused(_ptr(X), _ptr(s), _ptr(L1), _ptr(w_codes), _ptr(w_scales),
                                           _ptr(L2), _ptr(bias), M, N, K, r, group, _ptr(Y), int(out),
                                           _stream(stream)),
           "hsq_linear_forward_fused")


def _sm_count() -> int:
    if torch.cuda.is_available():
        return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return 148


def _a16(v: int) -> int:
    return (v + 15) // 16 * 16


def stream_smem_fits(M: int, N: int, K: int, group: int = GROUP, nsm: Optional[int] = None) -> bool:
    """Whether the weight stream's shared memory fits one block for this shape:
    the restatement, in integer arithmetic, of the limit include/hsq.h gives for
    hsq_linear_forward_fused (no library call, so it can be asked without a GPU).
    T = M rounded up to 1, 2, 4 or 8; RB = rows per block = ceil(N / SMs) rounded
    up to 4; a ring of at least two stages (one if one stage holds all RB rows)
    of rs rows, rs = max(1, max(16384, min(RB Kp/4, budget/2)) // (Kp/2))."""
    nsm = nsm or _sm_count()
    G = -(-K // group)
    Kp = G * group
    T = 1 if M <= 1 else 2 if M <= 2 else 4 if M <= 4 else 8
    RB = (-(-N // nsm) + 3) // 4 * 4
    if RB > 256 or G > 256:  # the block's scales are one copy of at most 256 x 256
        return False
    rowbytes = Kp // 2
    fixed = _a16(G * RB * 4) + _a16(T * Kp) + _a16(G * T * 4) + _a16(T * 16) + _a16(16 * T * 16)
    budget = max(0, 227 * 1024 - fixed - 1024)
    target = max(16384, min(RB * rowbytes // 2, budget // 2))
    rs = min(RB, max(1, target // rowbytes))
    min_stages = 1 if -(-RB // rs) == 1 else 2
    return min_stages * rs * rowbytes <= budget


def _dec16_scratch_bytes(M: int, N: int, K: int, r: int, group: int, nsm: int) -> int:
    """Bytes of the library's array that the decode-tile form of
    hsq_linear_forward_fused uses for this shape (restated from the planner: the
    barrier's 256 bytes, stream-K counters and partials, codes, scales, U
    partials and per-CTA copies of U, each rounded up to 256)."""
    up = lambda v: -(-v // 256) * 256
    G = -(-K // group)
    Kp = G * group
    gps = 4 if group == 64 else 2          # scale groups per pipeline stage
    tiles = -(-N // 128)                   # 128 weight rows x 16 tokens
    S = -(-G // gps)
    waves = -(-tiles // nsm)
    fill = tiles / (waves * nsm)
    total = tiles * S
    if (tiles >= nsm and fill >= 0.9) or total <= nsm or total >= (1 << 30):
        grid = min(tiles, nsm)
    else:
        sl = -(-total // nsm)
        grid = -(-total // sl)
    counters = up(tiles * 4 * 4)
    partials = grid * 2 * 16 * 128 * 4
    ldx = (M + 3) // 4 * 4
    rr = max(r, 1)
    nchk = -(-Kp // 256)
    off = 256
    for b in (counters, partials, M * (Kp // 2), G * ldx * 4, M * nchk * rr * 4, grid * M * rr * 4):
        off = up(off + b)
    return off


FUSED_SCRATCH_BYTES = 8 << 20


def fused_supported(M: int, K: int, r: int, group: int = GROUP, N: int = 8, nsm: Optional[int] = None) -> bool:
    """Whether hsq_linear_forward_fused takes this shape (the limits stated in
    include/hsq.h, restated without a library call so it can be asked without a
    GPU): the weight stream for M <= 4, r in {0, 1, 2, 4} and a block's shared
    memory, else the decode tiles for M <= 16, r <= 32 and the library's array."""
    if M < 1 or M > 16 or r < 0 or r > 32 or group not in (64, 128) or K % 8 or N % 8:
        return False
    nsm = nsm or _sm_count()
    if M <= 4 and r in (0, 1, 2, 4) and stream_smem_fits(M, N, K, group, nsm):
        return True
    return _dec16_scratch_bytes(M, N, K, r, group, nsm) <= FUSED_SCRATCH_BYTES


def hsq_fused_form(M: int, N: int, K: int, r: int, group: int = GROUP) -> int:
    return int(load().hsq_fused_form(M, N, K, r, group))


def hsq_lowrank_workspace_bytes(N: int, K: int, r: int) -> int:
    return int(load().hsq_lowrank_workspace_bytes(N, K, r))


def lowrank_init(W: torch.Tensor, s: torch.Tensor, r: int, iters: int = 8, seed: int = 0, stream=None):
    """Plain truncated-SVD L1 [K, r], L2 [r, N] (bf16) of W diag(s) on the GPU
    (pack-time helper; see hsq_lowrank_init)."""
    N, K = W.shape
    ws = torch.empty(max(1, hsq_lowrank_workspace_bytes(N, K, r)), dtype=torch.uint8, device=W.device)
    L1 = torch.empty((K, r), dtype=torch.bfloat16, device=W.device)
    L2 = torch.empty((r, N), dtype=torch.bfloat16, device=W.device)
    _check(load().hsq_lowrank_init(_ptr(W), _ptr(s), N, K, r, iters, int(seed) & ((1 << 64) - 1), _ptr(L1),
                                   _ptr(L2), _ptr(ws), ws.numel(), _stream(stream)),
           "hsq_lowrank_init")
    return L1, L2


def hsq_get_device_status(stream=None) -> int:
    return load().hsq_get_device_status(_stream(stream))


def hsq_debug_force_timeout(flags: int, limit_ms: int) -> None:
    load().hsq_debug_force_timeout(int(flags), int(limit_ms))


# ---------------------------------------------------------------- buffers
def alloc_codes(rows: int, K: int, device, group: int = GROUP) -> torch.Tensor:
    Kp = hsq_num_groups(K, group) * group
    return torch.empty((rows, Kp // 2), dtype=torch.uint8, device=device)


def alloc_scales(rows: int, K: int, device, group: int = GROUP) -> torch.Tensor:
    return torch.empty((hsq_num_groups(K, group), hsq_scales_ld(rows)), dtype=torch.float32, device=device)


class PackedLinear:
    """A packed layer: INT4 residual codes and scales plus the low-rank pair,
    the smoothing vector and the bias, all resident on one device."""

    def __init__(self, W, s, L1, L2, bias=None, stream=None, group: int = GROUP):
        N, K = W.shape
        r = 0 if L1 is None else int(L1.shape[1])
        dev = W.device
        self.N, self.K, self.r, self.group = N, K, r, group
        self.s = s.contiguous()
        self.L1 = None if r == 0 else L1.contiguous()
        self.L2 = None if r == 0 else L2.contiguous()
        self.bias = None if bias is None else bias.contiguous()
        self.w_codes = alloc_codes(N, K, dev, group)
        self.w_scales = alloc_scales(N, K, dev, group)
        self.w_e4m3 = None  # the weights' expanded copy, once expand() has run
        hsq_pack_weights(W.contiguous(), self.s, self.L1, self.L2, N, K, r,
                         self.w_codes, self.w_scales, group=group, stream=stream)

    def expand(self, stream=None) -> None:
        """Keep the weights' E4M3-expanded copy (hsq_expand_weights): forwards
        with many tokens then skip re-expanding the weights on every call."""
        if self.w_e4m3 is None:
            self.w_e4m3 = torch.empty(hsq_weights_e4m3_bytes(self.N, self.K, self.group), dtype=torch.uint8,
                                      device=self.w_codes.device)
            hsq_expand_weights(self.w_codes, self.N, self.K, self.w_e4m3, group=self.group, stream=stream)

    def workspace_x(self, M: int) -> torch.Tensor:
        """Workspace of forward_x for M tokens."""
        n = hsq_workspace_bytes_x(M, self.N, self.K, self.r, self.group, self.w_e4m3 is not None)
        return torch.zeros(max(n, 16), dtype=torch.uint8, device=self.w_codes.device)

    def workspace(self, M: int) -> Optional[torch.Tensor]:
        n = (hsq_workspace_bytes(M, self.N, self.K, self.r) if self.w_e4m3 is None
             else hsq_workspace_bytes_pre(M, self.N, self.K, self.r))
        if n == 0:
            return None
        return torch.zeros(n, dtype=torch.uint8, device=self.w_codes.device)


class ActBuffers:
    """Per-forward buffers of the activation step for M tokens."""

    def __init__(self, M: int, K: int, r: int, device, group: int = GROUP):
        self.M, self.K, self.r, self.group = M, K, r, group
        self.x_codes = alloc_codes(M, K, device, group)
        self.x_scales = alloc_scales(M, K, device, group)
        self.U = torch.empty((M, r), dtype=torch.float32, device=device) if r > 0 else None


def forward_fused(layer: PackedLinear, X: torch.Tensor, Y: torch.Tensor, out: int = HSQ_OUT_BF16,
                  stream=None) -> torch.Tensor:
    """One forward of the layer in a single launch (decode sizes, see
    hsq_linear_forward_fused)."""
    hsq_linear_forward_fused(X, layer.s, layer.L1, layer.w_codes, layer.w_scales, layer.L2, layer.bias,
                             X.shape[0], layer.N, layer.K, layer.r, Y, out=out, group=layer.group,
                             stream=stream)
    return Y


def forward_x(layer: PackedLinear, X: torch.Tensor, Y: torch.Tensor, workspace: torch.Tensor,
              out: int = HSQ_OUT_BF16, stream=None) -> torch.Tensor:
    """The activation step and the forward in one call (hsq_linear_forward_x);
    `workspace` of at least layer.workspace_x(M) bytes."""
    M = X.shape[0]
    hsq_linear_forward_x(X, layer.s, layer.L1, layer.w_codes, layer.w_scales, layer.w_e4m3, layer.L2, layer.bias,
                         M, layer.N, layer.K, layer.r, Y, out=out, workspace=workspace, ws_bytes=workspace.numel(),
                         group=layer.group, stream=stream)
    return Y


def forward(layer: PackedLinear, X: torch.Tensor, act: ActBuffers, Y: torch.Tensor,
            workspace: Optional[torch.Tensor] = None, out: int = HSQ_OUT_BF16, stream=None) -> torch.Tensor:
    """One forward of the layer: the activation step, then the GEMM + epilogue."""
    M = X.shape[0]
    if act.group != layer.group:
        raise ValueError("activation buffers and packed layer use different group sizes")
    hsq_quantize_act(X, layer.s, layer.L1, M, layer.K, layer.r, act.x_codes, act.x_scales, act.U,
                     group=layer.group, stream=stream)
    ws_bytes = 0 if workspace is None else workspace.numel()
    if layer.w_e4m3 is not None:
        hsq_linear_forward_pre(act.x_codes, act.x_scales, act.U, layer.w_codes, layer.w_scales, layer.w_e4m3,
                               layer.L2, layer.bias, M, layer.N, layer.K, layer.r, Y, out=out, workspace=workspace,
                               ws_bytes=ws_bytes, group=layer.group, stream=stream)
    else:
        hsq_linear_forward(act.x_codes, act.x_scales, act.U, layer.w_codes, layer.w_scales, layer.L2,
                           layer.bias, M, layer.N, layer.K, layer.r, Y, out=out, workspace=workspace,
                           ws_bytes=ws_bytes, group=layer.group, stream=stream)
    return Y


# ---------------------------------------------------------------- NVFP4 variant
def hsq_fp4_codes_bytes(rows: int, K: int) -> int:
    return int(load().hsq_fp4_codes_bytes(rows, K))


def hsq_fp4_scales_bytes(rows: int, K: int) -> int:
    return int(load().hsq_fp4_scales_bytes(rows, K))


def hsq_fp4_pack_weights(W, s, L1, L2, N, K, r, w_codes, w_sf, w_gs, stream=None) -> None:
    _check(load().hsq_fp4_pack_weights(_ptr(W), _ptr(s), _ptr(L1), _ptr(L2), N, K, r, _ptr(w_codes),
                                       _ptr(w_sf), _ptr(w_gs), _stream(stream)), "hsq_fp4_pack_weights")


def hsq_fp4_quantize_act(X, s, L1, M, K, r, x_codes, x_sf, x_gs, U, stream=None) -> None:
    _check(load().hsq_fp4_quantize_act(_ptr(X), _ptr(s), _ptr(L1), M, K, r, _ptr(x_codes), _ptr(x_sf),
                                       _ptr(x_gs), _ptr(U), _stream(stream)), "hsq_fp4_quantize_act")


def hsq_fp4_linear_forward(x_codes, x_sf, x_gs, U, w_codes, w_sf, w_gs, L2, bias, M, N, K, r, Y,
                           out: int = HSQ_OUT_BF16, stream=None) -> None:
    _check(load().hsq_fp4_linear_forward(_ptr(x_codes), _ptr(x_sf), _ptr(x_gs), _ptr(U), _ptr(w_codes),
                                         _ptr(w_sf), _ptr(w_gs), _ptr(L2), _ptr(bias), M, N, K, r, _ptr(Y),
                                         int(out), _stream(stream)), "hsq_fp4_linear_forward")


def _fp4_kq(K: int) -> int:
    return -(-K // 64) * 64


class Fp4Linear:
    """A layer packed in the NVFP4 variant: E2M1 residual codes, E4M3 block
    scales and the tensor scale, plus the low-rank pair, smoothing and bias."""

    def __init__(self, W, s, L1, L2, bias=None, stream=None):
        N, K = W.shape
        r = 0 if L1 is None else int(L1.shape[1])
        dev = W.device
        self.N, self.K, self.r = N, K, r
        self.s = s.contiguous()
        self.L1 = None if r == 0 else L1.contiguous()
        self.L2 = None if r == 0 else L2.contiguous()
        self.bias = None if bias is None else bias.contiguous()
        self.w_codes = torch.empty((N, _fp4_kq(K) // 2), dtype=torch.uint8, device=dev)
        self.w_sf = torch.empty(hsq_fp4_scales_bytes(N, K), dtype=torch.uint8, device=dev)
        self.w_gs = torch.empty(4, dtype=torch.float32, device=dev)
        hsq_fp4_pack_weights(W.contiguous(), self.s, self.L1, self.L2, N, K, r, self.w_codes, self.w_sf,
                             self.w_gs, stream=stream)

    def workspace(self, M: int) -> None:
        """The NVFP4 forward needs no workspace."""
        return None


class Fp4ActBuffers:
    """Per-forward buffers of the NVFP4 activation step for M tokens."""

    def __init__(self, M: int, K: int, r: int, device):
        self.M, self.K, self.r = M, K, r
        self.x_codes = torch.empty((M, _fp4_kq(K) // 2), dtype=torch.uint8, device=device)
        self.x_sf = torch.empty(hsq_fp4_scales_bytes(M, K), dtype=torch.uint8, device=device)
        self.x_gs = torch.empty(4, dtype=torch.float32, device=device)
        self.U = torch.empty((M, r), dtype=torch.float32, device=device) if r > 0 else None


def fp4_forward(layer: Fp4Linear, X: torch.Tensor, act: Fp4ActBuffers, Y: torch.Tensor,
                out: int = HSQ_OUT_BF16, stream=None) -> torch.Tensor:
    """One NVFP4 forward: the activation step, then the block-scaled GEMM + epilogue."""
    M = X.shape[0]
    hsq_fp4_quantize_act(X, layer.s, layer.L1, M, layer.K, layer.r, act.x_codes, act.x_sf, act.x_gs, act.U,
                         stream=stream)
    hsq_fp4_linear_forward(act.x_codes, act.x_sf, act.x_gs, act.U, layer.w_codes, layer.w_sf, layer.w_gs,
                           layer.L2, layer.bias, M, layer.N, layer.K, layer.r, Y, out=out, stream=stream)
    return Y
