"""Host-side checks of the C-ABI library (no GPU needed).

The library must load, export every function declared in include/fp8bl.h,
and reject invalid arguments with the documented status BEFORE touching the
device.  Calls with valid arguments need a GPU and live in the gpu tests.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8bl.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(fp8\w*)\s*\(", txt, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from fine_grained_block_token_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_expected_calls():
    names = _declared()
    for n in ("fp8_quant_act", "fp8_quant_weight", "fp8_block_linear", "fp8_block_linear_fused",
              "fp8_block_linear_workspace_bytes", "fp8bl_check", "fp8bl_status_string",
              "fp8_quant_act_ue8m0", "fp8_quant_weight_ue8m0", "fp8_block_linear_ue8m0",
              "fp8_quant_rowwise", "fp8_linear_rowwise", "fp8_quant_act_static",
              "fp8_grouped_linear_ue8m0"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from fine_grained_block_token_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.strip()}
    for n in _declared():
        assert n in exported, n
        assert getattr(lib, n) is not None


def test_status_strings(lib):
    lib.fp8bl_status_string.restype = ctypes.c_char_p
    for s in range(9):
        assert lib.fp8bl_status_string(s)
    assert lib.fp8bl_status_string(99) == b"unknown status"


V = ctypes.c_void_p


def _p(v):
    return ctypes.c_void_p(v)


def test_quant_act_argument_errors(lib):
    f = lib.fp8_quant_act
    f.argtypes = [V, ctypes.c_int64, ctypes.c_int64, V, V, V]
    good = _p(0x10000)
    assert f(good, 4, 100, good, good, None) == 2          # K not multiple of 128
    assert f(good, -1, 128, good, good, None) == 2         # negative M
    assert f(good, 4, 0, good, good, None) == 2            # K == 0
    assert f(good, 1, (1 << 31) * 128, good, good, None) == 2  # beyond FP8BL_MAX_DIM
    assert f(good, 0, 128, None, None, None) == 0          # M == 0 is a no-op
    assert f(None, 4, 128, good, good, None) == 1          # null input
    assert f(_p(0x10008), 4, 128, good, _p(0x20000), None) == 3  # misaligned x
    assert f(good, 4, 128, _p(0x20001), _p(0x30000), None) == 3  # misaligned q
    assert f(good, 4, 128, _p(0x10100), _p(0x40000), None) == 8  # q overlaps x


def test_quant_weight_argument_errors(lib):
    f = lib.fp8_quant_weight
    f.argtypes = [V, ctypes.c_int64, ctypes.c_int64, V, V, V]
    g = _p(0x100000)
    assert f(g, 100, 128, _p(0x200000), _p(0x300000), None) == 2   # N not multiple of 128
    assert f(g, 128, 0, _p(0x200000), _p(0x300000), None) == 2
    assert f(g, 128, 128, None, _p(0x300000), None) == 1
    assert f(g, 128, 128, _p(0x200000), _p(0x300002), None) == 3  # misaligned scales


def test_block_linear_argument_errors(lib):
    f = lib.fp8_block_linear
    f.argtypes = [V, V, V, V, V, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, V,
                  ctypes.c_size_t, V]
    a, sa, w, sw, y = (_p(0x1000000 * (i + 1)) for i in range(5))
    assert f(a, sa, w, sw, y, 4, 100, 128, None, 0, None) == 2    # N % 128
    assert f(a, sa, w, sw, y, 4, 128, 130, None, 0, None) == 2    # K % 128
    assert f(a, sa, w, sw, y, 0, 128, 128, None, 0, None) == 0    # empty M
    assert f(None, sa, w, sw, y, 4, 128, 128, None, 0, None) == 1
    assert f(a, sa, w, sw, _p(0x5000008), 4, 128, 128, None, 0, None) == 3
    assert f(a, sa, w, sw, a, 4, 128, 128, None, 0, None) == 8    # y aliases q_a


def test_fused_argument_errors(lib):
    f = lib.fp8_block_linear_fused
    f.argtypes = [V, V, V, V, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, V, ctypes.c_size_t, V]
    x, w, sw, y = (_p(0x1000000 * (i + 1)) for i in range(4))
    assert f(x, w, sw, y, 4, 128, 120, None, 0, None) == 2
    assert f(x, None, sw, y, 4, 128, 128, None, 0, None) == 1
    assert f(x, w, sw, x, 4, 128, 128, None, 0, None) == 8


def test_ue8m0_argument_errors(lib):
    fa = lib.fp8_quant_act_ue8m0
    fa.argtypes = [V, ctypes.c_int64, ctypes.c_int64, V, V, V]
    g = _p(0x10000)
    assert fa(g, 4, 100, _p(0x20000), _p(0x30000), None) == 2     # K % 128
    assert fa(g, 0, 128, None, None, None) == 0                   # empty M
    assert fa(g, 4, 128, _p(0x20000), None, None) == 1            # null scales
    assert fa(_p(0x10008), 4, 128, _p(0x20000), _p(0x30000), None) == 3
    # byte scales need no alignment: a misaligned scale pointer is accepted
    # by the checks and reaches the device query (no GPU here: CUDA / ARCH)
    assert fa(g, 4, 128, _p(0x20000), _p(0x30001), None) in (4, 5)
    assert fa(g, 4, 128, _p(0x20000), _p(0x10010), None) == 8     # scales overlap x
    fw = lib.fp8_quant_weight_ue8m0
    fw.argtypes = [V, ctypes.c_int64, ctypes.c_int64, V, V, V]
    assert fw(g, 100, 128, _p(0x200000), _p(0x300000), None) == 2
    assert fw(g, 128, 128, None, _p(0x300000), None) == 1
    fl = lib.fp8_block_linear_ue8m0
    fl.argtypes = [V, V, V, V, V, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, V]
    a, sa, w, sw, y = (_p(0x1000000 * (i + 1)) for i in range(5))
    assert fl(a, sa, w, sw, y, 4, 100, 128, None) == 2
    assert fl(a, sa, w, sw, y, 4, 128, 130, None) == 2
    assert fl(a, sa, w, sw, y, 0, 128, 128, None) == 0
    assert fl(a, None, w, sw, y, 4, 128, 128, None) == 1
    assert fl(a, sa, w, sw, _p(0x5000008), 4, 128, 128, None) == 3
    assert fl(a, sa, w, sw, a, 4, 128, 128, None) == 8
    assert fl(a, sa, w, sw, sw, 4, 128, 128, None) == 8           # y over the weight scales


def test_rowwise_argument_errors(lib):
    fq = lib.fp8_quant_rowwise
    fq.argtypes = [V, ctypes.c_int64, ctypes.c_int64, V, V, V]
    g = _p(0x10000)
    assert fq(g, 4, 100, _p(0x20000), _p(0x30000), None) == 2      # K % 16
    assert fq(g, 0, 16, None, None, None) == 0                     # empty
    assert fq(g, 4, 16, None, _p(0x30000), None) == 1
    assert fq(g, 4, 16, _p(0x20000), _p(0x30002), None) == 3       # scales need 4 bytes
    assert fq(g, 4, 16, _p(0x10040), _p(0x30000), None) == 8       # q overlaps x
    fl = lib.fp8_linear_rowwise
    fl.argtypes = [V, V, V, V, V, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, V]
    a, sa, w, sw, y = (_p(0x1000000 * (i + 1)) for i in range(5))
    assert fl(a, sa, w, sw, y, 4, 24, 32, None) == 2               # N % 16
    assert fl(a, sa, w, sw, y, 4, 32, 24, None) == 2               # K % 16
    assert fl(a, sa, w, sw, y, 0, 32, 32, None) == 0
    assert fl(a, sa, None, sw, y, 4, 32, 32, None) == 1
    assert fl(a, sa, w, _p(0x4000004), y, 4, 32, 32, None) == 3    # s_w must be 16-byte aligned
    assert fl(a, sa, w, sw, w, 4, 32, 32, None) == 8


def test_static_argument_errors(lib):
    f = lib.fp8_quant_act_static
    f.argtypes = [V, ctypes.c_int64, ctypes.c_int64, V, V, V, V]
    g, sg, q, s = _p(0x10000), _p(0x90000), _p(0x20000), _p(0x30000)
    assert f(g, 4, 100, sg, q, s, None) == 2          # K % 128
    assert f(g, 0, 128, None, None, None, None) == 0  # empty
    assert f(g, 4, 128, None, q, s, None) == 1        # no given scale
    assert f(g, 4, 128, _p(0x90002), q, s, None) == 3 # given scale misaligned
    assert f(g, 4, 128, _p(0x20010), q, s, None) == 8 # given scale inside q


def test_grouped_argument_errors(lib):
    f = lib.fp8_grouped_linear_ue8m0
    f.argtypes = [V, V, V, V, V, V] + [ctypes.c_int64] * 4 + [V]
    a, sa, w, sw, off, y = (_p(0x1000000 * (i + 1)) for i in range(6))
    assert f(a, sa, w, sw, off, y, 4, 128, 128, 0, None) == 2        # E < 1
    assert f(a, sa, w, sw, off, y, 4, 128, 128, 1025, None) == 2     # E > 1024
    assert f(a, sa, w, sw, off, y, 4, 1 << 24, 128, 128, None) == 2  # E * N too large
    assert f(a, sa, w, sw, off, y, 4, 100, 128, 2, None) == 2        # N % 128
    assert f(a, sa, w, sw, off, y, 0, 128, 128, 2, None) == 0        # empty
    assert f(a, sa, w, sw, None, y, 4, 128, 128, 2, None) == 1       # no offsets
    assert f(a, sa, w, sw, _p(0x5000002), y, 4, 128, 128, 2, None) == 3
    assert f(a, sa, w, sw, off, off, 4, 128, 128, 2, None) == 8      # y over the offsets


def test_ue8m0_pair_workspace_sizes(lib):
    """Workspace of the CTA-pair schedules: none at M <= 128; otherwise, per
    K block, 512 bytes per packed group of 128 activation rows -- 2 per
    256-row block, and for E > 1 every expert's segment padded to 256 rows,
    bounded by 2 (ceil(M/256) + E) -- plus 512 bytes per 128-row weight
    block (2 per 256 output columns) of every expert."""
    fd = lib.fp8_block_linear_ue8m0_workspace_bytes
    fd.argtypes = [ctypes.c_int64] * 3
    fd.restype = ctypes.c_size_t
    fg = lib.fp8_grouped_linear_ue8m0_workspace_bytes
    fg.argtypes = [ctypes.c_int64] * 4
    fg.restype = ctypes.c_size_t
    cdiv = lambda a, b: -(-a // b)
    for M, N, K in [(129, 128, 128), (4096, 28672, 4096), (4096, 4096, 14336), (300, 384, 512)]:
        KB = K // 128
        assert fd(M, N, K) == KB * 2 * cdiv(M, 256) * 512 + KB * 2 * cdiv(N, 256) * 512, (M, N, K)
        assert fg(M, N, K, 1) == fd(M, N, K)
    for M, N, K, E in [(8192, 4096, 7168, 16), (8192, 7168, 2048, 16), (300, 256, 256, 3),
                       (4100, 256, 384, 256)]:
        KB = K // 128
        assert fg(M, N, K, E) == KB * 2 * (cdiv(M, 256) + E) * 512 + E * KB * 2 * cdiv(N, 256) * 512
    assert fd(128, 4096, 4096) == 0 and fg(128, 4096, 4096, 8) == 0
    assert fg(300, 256, 256, 0) == 0 and fg(300, 256, 256, 1025) == 0 and fg(300, 100, 256, 2) == 0


def test_grouped_workspace_argument_errors(lib):
    """fp8_grouped_linear_ue8m0_ws refuses a missing, short, misaligned or
    overlapping workspace before touching the device (M > 128 needs one)."""
    f = lib.fp8_grouped_linear_ue8m0_ws
    f.argtypes = [V, V, V, V, V, V] + [ctypes.c_int64] * 4 + [V, ctypes.c_size_t, V]
    fg = lib.fp8_grouped_linear_ue8m0_workspace_bytes
    fg.argtypes = [ctypes.c_int64] * 4
    fg.restype = ctypes.c_size_t
    M, N, K, E = 300, 256, 256, 3
    need = fg(M, N, K, E)
    a, sa, w, sw, off, y, ws = (_p(0x10000000 * (i + 1)) for i in range(7))
    assert f(a, sa, w, sw, off, y, M, N, K, E, None, 0, None) == 1            # no workspace
    assert f(a, sa, w, sw, off, y, M, N, K, E, ws, need - 16, None) == 7      # too small
    assert f(a, sa, w, sw, off, y, M, N, K, E, _p(0x70000008), need, None) == 3
    assert f(a, sa, w, sw, off, y, M, N, K, E, y, need, None) == 8            # workspace over y
    assert f(a, sa, w, sw, off, y, M, N, K, 0, ws, need, None) == 2           # E < 1
    assert f(a, sa, w, sw, off, y, 0, N, K, E, None, 0, None) == 0           # empty


def test_valid_call_without_gpu_reports_cuda_error(lib):
    """With no usable device the library answers FP8BL_ERR_CUDA (or ARCH on
    a non-B200 device) instead of crashing or falling back to the CPU."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    f = lib.fp8_quant_act
    f.argtypes = [V, ctypes.c_int64, ctypes.c_int64, V, V, V]
    assert f(_p(0x10000), 4, 128, _p(0x20000), _p(0x30000), None) in (4, 5)


def test_workspace_query_never_fails(lib):
    f = lib.fp8_block_linear_workspace_bytes
    f.argtypes = [ctypes.c_int64] * 3
    f.restype = ctypes.c_size_t
    assert f(4, 100, 128) == 0
    assert f(-1, 128, 128) == 0


def test_selftest_wait_timeout_rejects_bad_arguments(lib):
    """The failure-detection self-test validates its arguments on the host."""
    f = lib.fp8bl_selftest_wait_timeout
    f.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]
    f.restype = ctypes.c_int
    assert f(0, 0, None) == 2
    assert f((1 << 32) + 1, 0, None) == 2
    assert f(1000, 2, None) == 2
    assert f(1000, -1, None) == 2


def _decode_slots_needed(N, K, G):
    """Brute force over the stream-K partition of the decode schedule: CTA g
    streams units [g*U/G, (g+1)*U/G) of the flattened (weight block, K chunk)
    space (U = N/128 * K/128) and stores one partial per block it touches,
    in slot (block - first block of its range).  Returns the largest number
    of slots any CTA uses."""
    KB = K // 128
    U = (N // 128) * KB
    most = 0
    for g in range(G):
        lo, hi = g * U // G, (g + 1) * U // G
        if hi > lo:
            most = max(most, (hi - 1) // KB - lo // KB + 1)
    return most


@pytest.mark.parametrize("seed", range(6))
def test_decode_workspace_covers_every_partial_slot(lib, seed):
    """The workspace the library asks for must hold the per-block ready flags
    and counters plus, for each of the G CTAs, a partial [Mpad, 128] fp32 for every block
    its range touches; a smaller stride would let a CTA write past its
    slots (and the last CTA past the buffer).  Without a GPU the library
    plans for 148 SMs: G = min(148, U / ceil(KB / 8)) CTAs, or U / c when the
    least divisor c of KB with c >= ceil(KB / 8) and U / c <= 148 keeps at
    least 85 % of those CTAs (ranges that tile the weight blocks)."""
    import numpy as np
    f = lib.fp8_block_linear_workspace_bytes
    f.argtypes = [ctypes.c_int64] * 3
    f.restype = ctypes.c_size_t
    g = np.random.default_rng(seed)
    shapes = [(1, 128, 128), (64, 128, 128), (1, 256, 32768), (17, 28672, 4096), (64, 4096, 14336),
              (8, 1024, 4096), (33, 128, 1024 * 128)]
    shapes += [(int(g.integers(1, 65)), 128 * int(g.integers(1, 300)), 128 * int(g.integers(1, 200)))
               for _ in range(40)]
    for M, N, K in shapes:
        KB, U = K // 128, (N // 128) * (K // 128)
        G = max(1, min(148, U // ((KB + 7) // 8)))
        c = max((KB + 7) // 8, -(-U // 148))
        while c <= KB and KB % c:
            c += 1
        if c <= KB and (U // c) * 100 >= G * 85:
            G = U // c
        mpad = (M + 15) // 16 * 16
        # a 64-bit ready flag and a 32-bit counter per weight block
        counters = ((N // 128) * 12 + 255) // 256 * 256
        ws = f(M, N, K)
        per_slot = G * mpad * 128 * 4
        assert ws > counters and (ws - counters) % per_slot == 0, (M, N, K, ws)
        assert (ws - counters) // per_slot >= _decode_slots_needed(N, K, G), (M, N, K)
    assert f(65, 4096, 4096) == 0          # prefill sizes need no workspace


def test_fused_workspace_holds_the_staged_activations(lib):
    """The fused entry point's workspace holds the staged activations (codes
    M*K bytes, then scales M*K/128 fp32, each 256-byte aligned) after the
    decode schedule's own scratch (none at prefill sizes, where a smaller
    workspace selects the in-GEMM quantization instead)."""
    ws = lib.fp8_block_linear_workspace_bytes
    fw = lib.fp8_block_linear_fused_workspace_bytes
    for f in (ws, fw):
        f.argtypes = [ctypes.c_int64] * 3
        f.restype = ctypes.c_size_t
    up = lambda v: (v + 255) // 256 * 256
    for M, N, K in [(1, 128, 128), (7, 4096, 4096), (64, 28672, 4096), (33, 4096, 14336),
                    (64, 128, 1024 * 128), (65, 4096, 4096), (8192, 7168, 18432)]:
        assert fw(M, N, K) >= up(ws(M, N, K)) + up(M * K) + up(M * (K // 128) * 4), (M, N, K)
    for M, N, K in [(65, 4096, 4096), (8192, 7168, 18432)]:
        assert ws(M, N, K) == 0


def test_noalloc_scratch_covers_the_decode_workloads(lib):
    """The no-allocation entry point serves a decode shape only while its
    schedule's scratch fits the built-in array (FP8BL_NOALLOC_SCRATCH_BYTES,
    16 MiB).  Every Llama-3-8B and DeepSeek-V3 linear at the decode token
    counts must fit, so that a change to the schedule's geometry cannot
    silently turn those shapes into FP8BL_ERR_WORKSPACE.  (Planned for 148
    SMs, the B200's count, as the library does without a GPU.)"""
    f = lib.fp8_block_linear_workspace_bytes
    f.argtypes = [ctypes.c_int64] * 3
    f.restype = ctypes.c_size_t
    hdr = open(os.path.join(ROOT, "include", "fp8bl.h")).read()
    m = re.search(r"#define FP8BL_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", hdr)
    limit = int(m.group(1)) << int(m.group(2))
    llama3_8b = [(4096, 4096), (1024, 4096), (28672, 4096), (4096, 14336)]
    deepseek_v3 = [(18432, 7168), (7168, 18432), (2048, 7168), (7168, 2048), (4096, 7168)]
    for M in (1, 8, 32, 64):
        for N, K in llama3_8b + deepseek_v3:
            need = f(M, N, K)
            assert 0 < need <= limit, (M, N, K, need, limit)
