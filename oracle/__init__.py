"""CPU oracle for fine-grained block-scaled FP8 linear layers.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The CUDA
library never calls it, and it imports nothing from the CUDA package.

The arithmetic lives in ``fp8bl_oracle.c`` (plain C, fp64 GEMM, software e4m3
encoder written from the format definition); this module compiles it with gcc
(no fast-math, no FP contraction) and exposes numpy-level wrappers.

Sources (transformers docs, "Fine-grained FP8" page):
  * opening bullet list -- 128 x 128 weight blocks, per-token activation
    groups of 128 along the input channel;
  * "DeepGEMM fast path" section -- the dynamic activation scheme;
  * "UE8M0 scale format" section -- power-of-two scales stored as
    float8_e8m0fnu (the ``*_ue8m0`` functions).
Static activation scale (``quant_act_static``): the "DeepGEMM fast path" section's
static activation quantization.  Row-wise FP8 (the ``*_rowwise`` functions): "BFL (fp8r / nvfp4)" page of the
diffusers docs, first bullet of its list and its "Kernels" table.
The readings the pages leave open (scale formula, rounding, eps) are stated
in the header comment of ``fp8bl_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8bl_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_fp8bl.so")
_lock = threading.Lock()
_lib = None

BLOCK = 128
E4M3_MAX = 448.0
AMAX_EPS = np.float32(1e-10)


def build(force: bool = False) -> str:
    """Compile the oracle's C source into a shared library (gcc, -O2).

    ``-fno-fast-math -ffp-contract=off`` keep every fp32 division IEEE and stop
    gcc from fusing multiply-adds, so the code computes what it says."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
           "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def bind(path: str):
    """Load a compiled oracle library from ``path`` and declare its C signatures."""
    lib = ctypes.CDLL(path)
    i64, vp, ip = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_quant_act_rows.argtypes = [vp, i64, i64, vp, vp, i64, i64]
    lib.oracle_quant_act_rows.restype = None
    lib.oracle_quant_act.argtypes = [vp, i64, i64, vp, vp, ip]
    lib.oracle_quant_act.restype = None
    lib.oracle_quant_weight.argtypes = [vp, i64, i64, vp, vp]
    lib.oracle_quant_weight.restype = None
    lib.oracle_block_linear_rows.argtypes = [vp, vp, vp, vp, i64, i64, i64,
                                                 vp, i64, vp, ip]
    lib.oracle_block_linear_rows.restype = ctypes.c_int
    lib.oracle_ue8m0_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_ue8m0_decode.restype = ctypes.c_double
    lib.oracle_ue8m0_from_amax.argtypes = [ctypes.c_float]
    lib.oracle_ue8m0_from_amax.restype = ctypes.c_uint8
    lib.oracle_quant_act_ue8m0_rows.argtypes = [vp, i64, i64, vp, vp, i64, i64]
    lib.oracle_quant_act_ue8m0_rows.restype = None
    lib.oracle_quant_act_ue8m0.argtypes = [vp, i64, i64, vp, vp, ip]
    lib.oracle_quant_act_ue8m0.restype = None
    lib.oracle_quant_weight_ue8m0.argtypes = [vp, i64, i64, vp, vp]
    lib.oracle_quant_weight_ue8m0.restype = None
    lib.oracle_quant_rowwise_rows.argtypes = [vp, i64, vp, vp, i64, i64]
    lib.oracle_quant_rowwise_rows.restype = None
    lib.oracle_linear_rowwise_rows.argtypes = [vp, vp, vp, vp, i64, i64, vp, i64, vp]
    lib.oracle_linear_rowwise_rows.restype = ctypes.c_int
    lib.oracle_quant_act_static.argtypes = [vp, i64, i64, ctypes.c_float, vp, vp]
    lib.oracle_quant_act_static.restype = None
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = bind(build())
        return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _as_bf16_bits(x) -> np.ndarray:
    """Accept a uint16 array of bf16 bit patterns (or a torch bf16 CPU tensor)."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch  # noqa: F401  (torch is optional for the oracle)
        x = x.contiguous().view(dtype=__import__("torch").int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("bf16 input must be given as uint16 bit patterns")
    return x


def e4m3_decode(code: int) -> float:
    """Value of one e4m3 code (OCP FP8 E4M3, the 'fn' variant)."""
    return _load().oracle_e4m3_decode(int(code) & 0xFF)


def e4m3_decode_table() -> np.ndarray:
    """fp64 values of all 256 codes (NaN for 0x7F / 0xFF)."""
    lib = _load()
    return np.array([lib.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(v: float) -> int:
    """e4m3 code of one fp32 value: RNE to the even code, saturating."""
    return int(_load().oracle_e4m3_encode(float(np.float32(v))))


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    """Elementwise encode of an fp32 array (slow: one C call per element)."""
    lib = _load()
    flat = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.empty(flat.shape, dtype=np.uint8)
    for i, x in enumerate(flat.tolist()):
        out[i] = lib.oracle_e4m3_encode(x)
    return out.reshape(np.shape(v))


def quant_act(x_bf16, nthreads: int = 1):
    """Dynamic per-token activation quantization, groups of 128 channels.

    x_bf16: uint16 [M, K] bf16 bit patterns, K % 128 == 0.
    Returns (q uint8 [M, K] e4m3 codes, s float32 [M, K/128])."""
    x = _as_bf16_bits(x_bf16)
    M, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 128")
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M, K // BLOCK), dtype=np.float32)
    if M:
        _load().oracle_quant_act(_ptr(x), M, K, _ptr(q), _ptr(s), int(nthreads))
    return q, s


def quant_act_rows(x_bf16, m0: int, m1: int):
    """Quantize rows m0..m1-1 only (single thread).  Returns (q, s) for those rows."""
    x = _as_bf16_bits(x_bf16)
    M, K = x.shape
    sub = np.ascontiguousarray(x[m0:m1])
    q = np.empty((m1 - m0, K), dtype=np.uint8)
    s = np.empty((m1 - m0, K // BLOCK), dtype=np.float32)
    if m1 > m0:
        _load().oracle_quant_act_rows(_ptr(sub), m1 - m0, K, _ptr(q), _ptr(s), 0, m1 - m0)
    return q, s


def quant_weight(w_bf16):
    """128 x 128 block weight quantization.

    w_bf16: uint16 [N, K] bf16 bit patterns, N % 128 == K % 128 == 0.
    Returns (q uint8 [N, K], s float32 [N/128, K/128])."""
    w = _as_bf16_bits(w_bf16)
    N, K = w.shape
    if N % BLOCK or K % BLOCK:
        raise ValueError("N and K must be multiples of 128")
    q = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N // BLOCK, K // BLOCK), dtype=np.float32)
    _load().oracle_quant_weight(_ptr(w), N, K, _ptr(q), _ptr(s))
    return q, s


def block_linear(q_a, s_a, q_w, s_w, rows=None, nthreads: int = 1) -> np.ndarray:
    """fp64 result R of the block-scaled FP8 linear for the given rows.

    q_a uint8 [M, K], s_a float32 [M, K/128], q_w uint8 [N, K],
    s_w float32 [N/128, K/128].  ``rows``: iterable of row indices (default:
    all rows).  Returns float64 [len(rows), N]."""
    q_a = np.ascontiguousarray(q_a, dtype=np.uint8)
    q_w = np.ascontiguousarray(q_w, dtype=np.uint8)
    s_a = np.ascontiguousarray(s_a, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    M, K = q_a.shape
    N = q_w.shape[0]
    if q_w.shape[1] != K or K % BLOCK or N % BLOCK:
        raise ValueError("shape mismatch")
    if s_a.shape != (M, K // BLOCK) or s_w.shape != (N // BLOCK, K // BLOCK):
        raise ValueError("scale shape mismatch")
    r = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((len(r), N), dtype=np.float64)
    if len(r):
        rc = _load().oracle_block_linear_rows(_ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_w),
                                              M, N, K, _ptr(r), len(r), _ptr(y), int(nthreads))
        if rc != 0:
            raise MemoryError("oracle allocation failed")
    return y


# ------------------------------------------------------------ UE8M0 scales
# "Fine-grained FP8" page, "UE8M0 scale format" section: scales kept as
# float8_e8m0fnu (scale_fmt="ue8m0").  Readings R11-R13 in fp8bl_oracle.c:
# the scale is the fp32 scale rounded up to a power of two 2^e, stored as
# the byte e + 127, and q = e4m3(x * 2^-e).


def ue8m0_decode(codes) -> np.ndarray:
    """fp64 values 2^(c - 127) of ue8m0 codes (NaN for 255)."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib.oracle_ue8m0_decode(i) for i in range(256)], dtype=np.float64)
    return table[c]


def ue8m0_from_amax(amax: float) -> int:
    """ue8m0 code of the scale of a group whose largest magnitude is ``amax``."""
    return int(_load().oracle_ue8m0_from_amax(float(np.float32(amax))))


def quant_act_ue8m0(x_bf16, nthreads: int = 1):
    """Per-token 1 x 128 activation quantization with UE8M0 scales.

    Returns (q uint8 [M, K] e4m3 codes, s uint8 [M, K/128] ue8m0 codes)."""
    x = _as_bf16_bits(x_bf16)
    M, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 128")
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M, K // BLOCK), dtype=np.uint8)
    if M:
        _load().oracle_quant_act_ue8m0(_ptr(x), M, K, _ptr(q), _ptr(s), int(nthreads))
    return q, s


def quant_act_ue8m0_rows(x_bf16, m0: int, m1: int):
    """UE8M0 quantization of rows m0..m1-1 only (single thread)."""
    x = _as_bf16_bits(x_bf16)
    M, K = x.shape
    sub = np.ascontiguousarray(x[m0:m1])
    q = np.empty((m1 - m0, K), dtype=np.uint8)
    s = np.empty((m1 - m0, K // BLOCK), dtype=np.uint8)
    if m1 > m0:
        _load().oracle_quant_act_ue8m0_rows(_ptr(sub), m1 - m0, K, _ptr(q), _ptr(s), 0, m1 - m0)
    return q, s


def quant_weight_ue8m0(w_bf16):
    """128 x 128 block weight quantization with UE8M0 scales.

    Returns (q uint8 [N, K], s uint8 [N/128, K/128] ue8m0 codes)."""
    w = _as_bf16_bits(w_bf16)
    N, K = w.shape
    if N % BLOCK or K % BLOCK:
        raise ValueError("N and K must be multiples of 128")
    q = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N // BLOCK, K // BLOCK), dtype=np.uint8)
    _load().oracle_quant_weight_ue8m0(_ptr(w), N, K, _ptr(q), _ptr(s))
    return q, s


def block_linear_ue8m0(q_a, c_a, q_w, c_w, rows=None, nthreads: int = 1) -> np.ndarray:
    """fp64 result of the block-scaled linear whose scales are ue8m0 codes:
    the same sum as ``block_linear`` with s = 2^(c - 127) (exact in fp32)."""
    s_a = ue8m0_decode(c_a).astype(np.float32)
    s_w = ue8m0_decode(c_w).astype(np.float32)
    return block_linear(q_a, s_a, q_w, s_w, rows=rows, nthreads=nthreads)


# ------------------------------------------------------ row-wise FP8 (fp8r)
# "BFL (fp8r / nvfp4)" page: one fp32 scale per weight row and per
# activation row.  Readings R14-R15 in fp8bl_oracle.c.


def quant_rowwise(x_bf16, r0: int = 0, r1: int | None = None):
    """Row-wise e4m3 quantization of rows r0..r1-1 of a bf16 [R, K] matrix.

    Returns (q uint8 [r1 - r0, K], s float32 [r1 - r0])."""
    x = _as_bf16_bits(x_bf16)
    R, K = x.shape
    r1 = R if r1 is None else r1
    sub = np.ascontiguousarray(x[r0:r1])
    q = np.empty((r1 - r0, K), dtype=np.uint8)
    s = np.empty((r1 - r0,), dtype=np.float32)
    if r1 > r0:
        _load().oracle_quant_rowwise_rows(_ptr(sub), K, _ptr(q), _ptr(s), 0, r1 - r0)
    return q, s


def linear_rowwise(q_a, s_a, q_w, s_w, rows=None) -> np.ndarray:
    """fp64 result of the row-wise scaled linear for the given rows.

    q_a uint8 [M, K], s_a float32 [M], q_w uint8 [N, K], s_w float32 [N]."""
    q_a = np.ascontiguousarray(q_a, dtype=np.uint8)
    q_w = np.ascontiguousarray(q_w, dtype=np.uint8)
    s_a = np.ascontiguousarray(s_a, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    M, K = q_a.shape
    N = q_w.shape[0]
    if q_w.shape[1] != K or s_a.shape != (M,) or s_w.shape != (N,):
        raise ValueError("shape mismatch")
    r = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty((len(r), N), dtype=np.float64)
    if len(r):
        if _load().oracle_linear_rowwise_rows(_ptr(q_a), _ptr(s_a), _ptr(q_w), _ptr(s_w), N, K,
                                              _ptr(r), len(r), _ptr(y)) != 0:
            raise MemoryError("oracle allocation failed")
    return y


def quant_act_static(x_bf16, s: float):
    """Static activation quantization with one given fp32 scale (reading R16 in
    fp8bl_oracle.c).  Returns (q uint8 [M, K], s_a float32 [M, K/128] all = s)."""
    x = _as_bf16_bits(x_bf16)
    M, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 128")
    q = np.empty((M, K), dtype=np.uint8)
    sa = np.empty((M, K // BLOCK), dtype=np.float32)
    if M:
        _load().oracle_quant_act_static(_ptr(x), M, K, float(np.float32(s)), _ptr(q), _ptr(sa))
    return q, sa


def grouped_linear_ue8m0(q_a, c_a, q_w, c_w, offsets, rows=None, nthreads: int = 1) -> np.ndarray:
    """Grouped (MoE expert) UE8M0 linear, fp64 [M, N]: rows [off[e], off[e+1])
    times expert e's weights q_w[e] / c_w[e] (a contiguous grouping of the
    rows by expert, each segment the block linear of its expert).  Rows
    outside [off[0], off[E]), and rows not listed in ``rows`` when it is
    given, are NaN."""
    q_a = np.ascontiguousarray(q_a, dtype=np.uint8)
    q_w = np.ascontiguousarray(q_w, dtype=np.uint8)
    M, K = q_a.shape
    E, N, _ = q_w.shape
    off = [int(v) for v in offsets]
    if len(off) != E + 1 or off[0] < 0 or off[-1] > M or any(b < a for a, b in zip(off, off[1:])):
        raise ValueError("offsets must be non-decreasing within [0, M]")
    want = np.arange(M) if rows is None else np.unique(np.asarray(rows, dtype=np.int64))
    y = np.full((M, N), np.nan, dtype=np.float64)
    for e in range(E):
        r = want[(want >= off[e]) & (want < off[e + 1])]
        if len(r):
            y[r] = block_linear_ue8m0(q_a, c_a, q_w[e], c_w[e], rows=r, nthreads=nthreads)
    return y


def bf16_rne(y: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (nearest, ties to even), returned as fp64.

    Used for the bf16 view of the oracle's result: first to fp32 would add a
    second rounding, so the rounding is done from fp64 directly by scaling to
    the bf16 grid of each value's binade."""
    y = np.asarray(y, dtype=np.float64)
    out = np.zeros_like(y)
    nz = (y != 0) & np.isfinite(y)
    a = np.abs(y[nz])
    e = np.floor(np.log2(a))
    # guard log2 rounding at binade edges
    e = np.where(np.ldexp(1.0, e.astype(np.int64)) > a, e - 1, e)
    e = np.where(np.ldexp(1.0, (e + 1).astype(np.int64)) <= a, e + 1, e)
    e = np.maximum(e, -133.0 + 7)  # bf16 subnormal grid spacing is 2^-133
    spacing = np.ldexp(1.0, (e - 7).astype(np.int64))
    out[nz] = np.sign(y[nz]) * np.round(a / spacing) * spacing  # np.round is half-to-even
    out[~np.isfinite(y)] = y[~np.isfinite(y)]
    return out
