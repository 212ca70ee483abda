"""ctypes binding of the C ABI in ``include/fp8bl.h`` (``libfp8bl.so``, built
in-tree by ``fine_grained_block_token_b200.build``).  The binding only
marshals arguments: it allocates outputs with torch on the input's device,
passes raw device pointers, sizes and the current CUDA stream, and turns
status codes into exceptions.  Every step of the computation runs in the
library's CUDA kernels; there is no fallback path.  If the library is
missing the import of this module fails.

Method ("Fine-grained FP8" page of the transformers docs, opening bullet
list): weights quantized to e4m3 with one fp32 scale per 128 x 128 block,
activations quantized dynamically per token with one fp32 scale per group of
128 input channels, and a GEMM that applies both scale sets per 128-deep K
block and writes bf16.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "Fp8blError", "BLOCK", "lib_path", "quant_act", "quant_weight", "block_linear",
    "block_linear_fused", "block_linear_noalloc", "workspace_bytes", "fused_workspace_bytes",
    "check", "version", "quant_act_ue8m0", "quant_weight_ue8m0", "block_linear_ue8m0",
    "ue8m0_workspace_bytes",
    "quant_rowwise", "linear_rowwise", "quant_act_static", "grouped_linear_ue8m0",
    "grouped_ue8m0_workspace_bytes",
]

BLOCK = 128
_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libfp8bl.so")

if not os.path.exists(lib_path):
    raise ImportError(
        f"{lib_path} is missing: build it with `python -m fine_grained_block_token_b200.build`")

_lib = ctypes.CDLL(lib_path)
_i64, _vp, _sz = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
_lib.fp8_quant_act.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
_lib.fp8_quant_weight.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
_lib.fp8_block_linear.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _sz, _vp]
_lib.fp8_block_linear_fused.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _sz, _vp]
_lib.fp8_block_linear_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]
_lib.fp8_block_linear_workspace_bytes.argtypes = [_i64, _i64, _i64]
_lib.fp8_block_linear_workspace_bytes.restype = _sz
_lib.fp8_block_linear_fused_workspace_bytes.argtypes = [_i64, _i64, _i64]
_lib.fp8_block_linear_fused_workspace_bytes.restype = _sz
_lib.fp8_quant_act_ue8m0.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
_lib.fp8_quant_weight_ue8m0.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
_lib.fp8_block_linear_ue8m0.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]
_lib.fp8_block_linear_ue8m0_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _sz, _vp]
_lib.fp8_block_linear_ue8m0_workspace_bytes.argtypes = [_i64, _i64, _i64]
_lib.fp8_block_linear_ue8m0_workspace_bytes.restype = _sz
_lib.fp8_quant_rowwise.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp]
_lib.fp8_quant_act_static.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp, _vp]
_lib.fp8_grouped_linear_ue8m0.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp]
_lib.fp8_grouped_linear_ue8m0_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                             _vp, _sz, _vp]
_lib.fp8_grouped_linear_ue8m0_workspace_bytes.argtypes = [_i64, _i64, _i64, _i64]
_lib.fp8_grouped_linear_ue8m0_workspace_bytes.restype = _sz
_lib.fp8_linear_rowwise.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]
_lib.fp8bl_check.argtypes = [_vp]
_lib.fp8bl_status_string.argtypes = [ctypes.c_int]
_lib.fp8bl_status_string.restype = ctypes.c_char_p
_lib.fp8bl_version.restype = ctypes.c_int
for _f in ("fp8_quant_act", "fp8_quant_weight", "fp8_block_linear", "fp8_block_linear_fused",
           "fp8_block_linear_noalloc", "fp8bl_check", "fp8_quant_act_ue8m0",
           "fp8_quant_weight_ue8m0", "fp8_block_linear_ue8m0", "fp8_block_linear_ue8m0_ws",
           "fp8_quant_rowwise",
           "fp8_linear_rowwise", "fp8_quant_act_static", "fp8_grouped_linear_ue8m0",
           "fp8_grouped_linear_ue8m0_ws"):
    getattr(_lib, _f).restype = ctypes.c_int

STATUS = {0: "FP8BL_OK", 1: "FP8BL_ERR_NULL", 2: "FP8BL_ERR_SHAPE", 3: "FP8BL_ERR_ALIGN",
          4: "FP8BL_ERR_ARCH", 5: "FP8BL_ERR_CUDA", 6: "FP8BL_ERR_TIMEOUT",
          7: "FP8BL_ERR_WORKSPACE", 8: "FP8BL_ERR_OVERLAP"}


class Fp8blError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.fp8bl_status_string(status).decode()
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")


def _ok(status: int, where: str) -> None:
    if status != 0:
        raise Fp8blError(status, where)


def _stream(t: torch.Tensor):
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _u8(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.uint8) if t.dtype != torch.uint8 else t


# The C ABI takes raw pointers and sizes and cannot see strides, devices or
# dtypes, so every tensor is checked here before its pointer is passed: on
# the current CUDA device (that of the call's first input), dense
# (contiguous), of the expected dtype and shape.  Violations raise before
# anything is enqueued.
_CODES = (torch.float8_e4m3fn, torch.uint8)          # e4m3 codes, or their bytes
_E8M0 = (torch.float8_e8m0fnu, torch.uint8)          # ue8m0 scale codes, or their bytes
_F32 = (torch.float32,)
_BF16 = (torch.bfloat16,)


def _device_of(t, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device (got {t.device})")
    # the library launches on the current device: a tensor elsewhere would
    # hand another device's pointers to its kernels
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name} is on {t.device} but the current device is cuda:{cur}; "
                         f"call under `with torch.cuda.device({t.device.index}):`")
    return t.device


def _need(t, name: str, dtypes, shape, device) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {' or '.join(map(str, dtypes))}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_linear(q_a, s_a, q_w, s_w, y):
    """Checks the operands of the fp32-scale linear; returns (M, N, K)."""
    dev = _device_of(q_a, "q_a")
    M, K = _dims2(q_a, "q_a")
    N = _dims2(q_w, "q_w")[0]
    _need(q_a, "q_a", _CODES, (M, K), dev)
    _need(s_a, "s_a", _F32, (M, K // BLOCK), dev)
    _need(q_w, "q_w", _CODES, (N, K), dev)
    _need(s_w, "s_w", _F32, (N // BLOCK, K // BLOCK), dev)
    if y is not None:
        _need(y, "y", _BF16, (M, N), dev)
    return M, N, K


def _dims2(t, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    return t.shape


def version() -> int:
    return _lib.fp8bl_version()


def quant_act(x: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None):
    """bf16 [M, K] -> (e4m3 [M, K], fp32 [M, K/128]).  Outputs may be given."""
    dev = _device_of(x, "x")
    M, K = _dims2(x, "x")
    _need(x, "x", _BF16, (M, K), dev)
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    if s is None:
        s = torch.empty((M, K // BLOCK), dtype=torch.float32, device=x.device)
    _need(q, "q", _CODES, (M, K), dev)
    _need(s, "s", _F32, (M, K // BLOCK), dev)
    _ok(_lib.fp8_quant_act(_ptr(x), M, K, _ptr(q), _ptr(s), _stream(x)), "fp8_quant_act")
    return q, s


def quant_act_static(x: torch.Tensor, s_given: torch.Tensor, q: torch.Tensor | None = None,
                     s: torch.Tensor | None = None):
    """Static scheme: bf16 [M, K] with one given fp32 scale (a 1-element device
    tensor) -> (e4m3 [M, K], fp32 [M, K/128] filled with that scale), ready
    for block_linear."""
    dev = _device_of(x, "x")
    M, K = _dims2(x, "x")
    _need(x, "x", _BF16, (M, K), dev)
    if not isinstance(s_given, torch.Tensor) or s_given.numel() != 1:
        raise ValueError("s_given must be a one-element fp32 tensor")
    _need(s_given, "s_given", _F32, None, dev)
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    if s is None:
        s = torch.empty((M, K // BLOCK), dtype=torch.float32, device=x.device)
    _need(q, "q", _CODES, (M, K), dev)
    _need(s, "s", _F32, (M, K // BLOCK), dev)
    _ok(_lib.fp8_quant_act_static(_ptr(x), M, K, _ptr(s_given), _ptr(q), _ptr(s), _stream(x)),
        "fp8_quant_act_static")
    return q, s


def quant_weight(w: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None):
    """bf16 [N, K] -> (e4m3 [N, K], fp32 [N/128, K/128])."""
    dev = _device_of(w, "w")
    N, K = _dims2(w, "w")
    _need(w, "w", _BF16, (N, K), dev)
    if q is None:
        q = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=w.device)
    if s is None:
        s = torch.empty((N // BLOCK, K // BLOCK), dtype=torch.float32, device=w.device)
    _need(q, "q", _CODES, (N, K), dev)
    _need(s, "s", _F32, (N // BLOCK, K // BLOCK), dev)
    _ok(_lib.fp8_quant_weight(_ptr(w), N, K, _ptr(q), _ptr(s), _stream(w)), "fp8_quant_weight")
    return q, s


# UE8M0 variant ("UE8M0 scale format" section): scales are float8_e8m0fnu
# codes (one byte, value 2^(code - 127)), the fp32 scale rounded up to a
# power of two.


def quant_act_ue8m0(x: torch.Tensor, q: torch.Tensor | None = None,
                    s: torch.Tensor | None = None):
    """bf16 [M, K] -> (e4m3 [M, K], float8_e8m0fnu [M, K/128])."""
    dev = _device_of(x, "x")
    M, K = _dims2(x, "x")
    _need(x, "x", _BF16, (M, K), dev)
    if q is None:
        q = torch.empty((M, K), dtype=torch.float8_e4m3fn, device=x.device)
    if s is None:
        s = torch.empty((M, K // BLOCK), dtype=torch.float8_e8m0fnu, device=x.device)
    _need(q, "q", _CODES, (M, K), dev)
    _need(s, "s", _E8M0, (M, K // BLOCK), dev)
    _ok(_lib.fp8_quant_act_ue8m0(_ptr(x), M, K, _ptr(q), _ptr(s), _stream(x)),
        "fp8_quant_act_ue8m0")
    return q, s


def quant_weight_ue8m0(w: torch.Tensor, q: torch.Tensor | None = None,
                       s: torch.Tensor | None = None):
    """bf16 [N, K] -> (e4m3 [N, K], float8_e8m0fnu [N/128, K/128])."""
    dev = _device_of(w, "w")
    N, K = _dims2(w, "w")
    _need(w, "w", _BF16, (N, K), dev)
    if q is None:
        q = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=w.device)
    if s is None:
        s = torch.empty((N // BLOCK, K // BLOCK), dtype=torch.float8_e8m0fnu, device=w.device)
    _need(q, "q", _CODES, (N, K), dev)
    _need(s, "s", _E8M0, (N // BLOCK, K // BLOCK), dev)
    _ok(_lib.fp8_quant_weight_ue8m0(_ptr(w), N, K, _ptr(q), _ptr(s), _stream(w)),
        "fp8_quant_weight_ue8m0")
    return q, s


def block_linear_ue8m0(q_a, s_a, q_w, s_w, y=None, workspace=None, pairs=True) -> torch.Tensor:
    """(e4m3 [M,K], e8m0 [M,K/128], e4m3 [N,K], e8m0 [N/128,K/128]) -> bf16 [M,N],
    on the tensor core's block-scaled MMA.  With pairs=True (the default) the
    call goes through fp8_block_linear_ue8m0_ws, which runs M > 128 on CTA
    pairs with a workspace (allocated here unless given); pairs=False calls
    the workspace-free single-CTA fp8_block_linear_ue8m0."""
    dev = _device_of(q_a, "q_a")
    M, K = _dims2(q_a, "q_a")
    N = _dims2(q_w, "q_w")[0]
    _need(q_a, "q_a", _CODES, (M, K), dev)
    _need(s_a, "s_a", _E8M0, (M, K // BLOCK), dev)
    _need(q_w, "q_w", _CODES, (N, K), dev)
    _need(s_w, "s_w", _E8M0, (N // BLOCK, K // BLOCK), dev)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=q_a.device)
    _need(y, "y", _BF16, (M, N), dev)
    if not pairs:
        _ok(_lib.fp8_block_linear_ue8m0(_ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_w), _ptr(y), M, N, K,
                                        _stream(q_a)), "fp8_block_linear_ue8m0")
        return y
    ws, wsb = _workspace(ue8m0_workspace_bytes(M, N, K), q_a.device, workspace)
    _ok(_lib.fp8_block_linear_ue8m0_ws(_ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_w), _ptr(y), M, N, K,
                                       _ptr(ws), wsb, _stream(q_a)), "fp8_block_linear_ue8m0_ws")
    return y


def ue8m0_workspace_bytes(M: int, N: int, K: int) -> int:
    """Workspace bytes fp8_block_linear_ue8m0_ws needs for these sizes."""
    return int(_lib.fp8_block_linear_ue8m0_workspace_bytes(M, N, K))


def grouped_linear_ue8m0(q_a, s_a, q_w, s_w, expert_offsets, y=None, workspace=None,
                         pairs=True) -> torch.Tensor:
    """Grouped (MoE expert) UE8M0 linear: rows [off[e], off[e+1]) of
    (e4m3 [M,K], e8m0 [M,K/128]) times expert e of (e4m3 [E,N,K],
    e8m0 [E,N/128,K/128]); expert_offsets int32 [E+1] on the device.  With
    pairs=True (the default) the call goes through fp8_grouped_linear_ue8m0_ws,
    which runs M > 128 on CTA pairs with a workspace (allocated here unless
    given); pairs=False calls the single-CTA fp8_grouped_linear_ue8m0."""
    dev = _device_of(q_a, "q_a")
    M, K = _dims2(q_a, "q_a")
    if q_w.dim() != 3:
        raise ValueError(f"q_w must be 3-D [E, N, K], got shape {tuple(q_w.shape)}")
    E, N, _ = q_w.shape
    _need(q_a, "q_a", _CODES, (M, K), dev)
    _need(s_a, "s_a", _E8M0, (M, K // BLOCK), dev)
    _need(q_w, "q_w", _CODES, (E, N, K), dev)
    _need(s_w, "s_w", _E8M0, (E, N // BLOCK, K // BLOCK), dev)
    _need(expert_offsets, "expert_offsets", (torch.int32,), (E + 1,), dev)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=q_a.device)
    _need(y, "y", _BF16, (M, N), dev)
    if not pairs:
        _ok(_lib.fp8_grouped_linear_ue8m0(_ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_w),
                                          _ptr(expert_offsets), _ptr(y), M, N, K, E, _stream(q_a)),
            "fp8_grouped_linear_ue8m0")
        return y
    ws, wsb = _workspace(grouped_ue8m0_workspace_bytes(M, N, K, E), q_a.device, workspace)
    _ok(_lib.fp8_grouped_linear_ue8m0_ws(_ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_w),
                                         _ptr(expert_offsets), _ptr(y), M, N, K, E, _ptr(ws), wsb,
                                         _stream(q_a)), "fp8_grouped_linear_ue8m0_ws")
    return y


def grouped_ue8m0_workspace_bytes(M: int, N: int, K: int, E: int) -> int:
    """Workspace bytes fp8_grouped_linear_ue8m0_ws needs for these sizes."""
    return int(_lib.fp8_grouped_linear_ue8m0_workspace_bytes(M, N, K, E))


# Row-wise variant ("BFL (fp8r / nvfp4)" page): one fp32 scale per row of
# the activations and of the weight.


def quant_rowwise(x: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None):
    """bf16 [R, K] -> (e4m3 [R, K], fp32 [R]); K % 16 == 0."""
    dev = _device_of(x, "x")
    R, K = _dims2(x, "x")
    _need(x, "x", _BF16, (R, K), dev)
    if q is None:
        q = torch.empty((R, K), dtype=torch.float8_e4m3fn, device=x.device)
    if s is None:
        s = torch.empty((R,), dtype=torch.float32, device=x.device)
    _need(q, "q", _CODES, (R, K), dev)
    _need(s, "s", _F32, (R,), dev)
    _ok(_lib.fp8_quant_rowwise(_ptr(x), R, K, _ptr(q), _ptr(s), _stream(x)), "fp8_quant_rowwise")
    return q, s


def linear_rowwise(q_a, s_a, q_w, s_w, y=None) -> torch.Tensor:
    """(e4m3 [M,K], fp32 [M], e4m3 [N,K], fp32 [N]) -> bf16 [M,N]."""
    dev = _device_of(q_a, "q_a")
    M, K = _dims2(q_a, "q_a")
    N = _dims2(q_w, "q_w")[0]
    _need(q_a, "q_a", _CODES, (M, K), dev)
    _need(s_a, "s_a", _F32, (M,), dev)
    _need(q_w, "q_w", _CODES, (N, K), dev)
    _need(s_w, "s_w", _F32, (N,), dev)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=q_a.device)
    _need(y, "y", _BF16, (M, N), dev)
    _ok(_lib.fp8_linear_rowwise(_ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_w), _ptr(y), M, N, K,
                                _stream(q_a)), "fp8_linear_rowwise")
    return y


def workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.fp8_block_linear_workspace_bytes(M, N, K))


def fused_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.fp8_block_linear_fused_workspace_bytes(M, N, K))


def _workspace(nbytes: int, device, given):
    if given is not None:
        _need(given, "workspace", (torch.uint8,), None, device)
    if nbytes == 0:
        return given, 0 if given is None else given.numel() * given.element_size()
    if given is None:
        given = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return given, given.numel() * given.element_size()


def block_linear(q_a, s_a, q_w, s_w, y=None, workspace=None) -> torch.Tensor:
    """(e4m3 [M,K], fp32 [M,K/128], e4m3 [N,K], fp32 [N/128,K/128]) -> bf16 [M,N]."""
    M, N, K = _check_linear(q_a, s_a, q_w, s_w, y)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=q_a.device)
    ws, wsb = _workspace(workspace_bytes(M, N, K), q_a.device, workspace)
    _ok(_lib.fp8_block_linear(_ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_w), _ptr(y), M, N, K,
                              _ptr(ws), wsb, _stream(q_a)), "fp8_block_linear")
    return y


def block_linear_fused(x, q_w, s_w, y=None, workspace=None, in_kernel=False) -> torch.Tensor:
    """bf16 x [M,K] with quantized weights -> bf16 [M,N], bit-identical to
    quant_act + block_linear.  By default the codes are staged in a workspace
    (allocated here unless given); in_kernel=True (M > 64) passes no
    workspace, so that the GEMM quantizes each activation tile itself."""
    dev = _device_of(x, "x")
    M, K = _dims2(x, "x")
    N = _dims2(q_w, "q_w")[0]
    _need(x, "x", _BF16, (M, K), dev)
    _need(q_w, "q_w", _CODES, (N, K), dev)
    _need(s_w, "s_w", _F32, (N // BLOCK, K // BLOCK), dev)
    if y is not None:
        _need(y, "y", _BF16, (M, N), dev)
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if in_kernel:
        if M <= 64:
            raise ValueError("in_kernel=True needs M > 64 (decode sizes always stage)")
        ws, wsb = None, 0
    else:
        ws, wsb = _workspace(fused_workspace_bytes(M, N, K), x.device, workspace)
    _ok(_lib.fp8_block_linear_fused(_ptr(x), _ptr(q_w), _ptr(s_w), _ptr(y), M, N, K,
                                    _ptr(ws), wsb, _stream(x)), "fp8_block_linear_fused")
    return y


def block_linear_noalloc(q_a, s_a, q_w, s_w, y) -> torch.Tensor:
    """Decode-sized linear (1 <= M <= 64) with the library's built-in scratch:
    no workspace, and nothing is allocated here or in the library, so the
    output tensor ``y`` (bf16 [M, N]) must be given.  For callers that cannot
    allocate device memory where they run the layer."""
    if y is None:
        raise ValueError("block_linear_noalloc needs the output tensor y")
    M, N, K = _check_linear(q_a, s_a, q_w, s_w, y)
    _ok(_lib.fp8_block_linear_noalloc(_ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_w), _ptr(y), M, N, K,
                                      _stream(q_a)), "fp8_block_linear_noalloc")
    return y


def check(device=None) -> None:
    """Synchronise the current stream and raise if a kernel wait timed out."""
    st = torch.cuda.current_stream(device).cuda_stream
    _ok(_lib.fp8bl_check(st), "fp8bl_check")
