"""GPU test of fp8_block_linear_noalloc, the decode-sized linear that runs
on scratch memory built into the library instead of a caller workspace (for
callers that cannot allocate device memory where they run the layer).

The entry point is called through the C ABI and its output is compared with
fp8_block_linear's (same inputs, caller workspace) on two calls in a row:
the second call runs on scratch that still holds the first call's contents.
Both run the same deterministic decode schedule, so the outputs must be
equal bit for bit; one shape is also held to the oracle within the GEMM
tolerance of the other tests.  Sizes beyond what the built-in scratch or
the decode schedule cover must be refused.

This file sorts last so that a run that stops at the first failure has
already run every other test; it also passes on its own in a new process.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from tests.parity import FRO_REL, PW_REL, PW_RMS, check_gemm

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fine_grained_block_token_b200 as m
    return m


def _within_tolerance(y, ref, label):
    y = y.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(r * r)))
    assert np.all(np.abs(y - r) <= PW_REL * np.abs(r) + PW_RMS * rms), label
    nrm = float(np.linalg.norm(r))
    assert float(np.linalg.norm(y - r)) <= FRO_REL * max(nrm, 1e-30), label


def _c_call(fp8, q_a, s_a, q_w, s_w, y, M, N, K):
    lib = ctypes.CDLL(fp8.lib_path)
    f = lib.fp8_block_linear_noalloc
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int64] * 3 + [ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f(q_a.data_ptr(), s_a.data_ptr(), q_w.data_ptr(), s_w.data_ptr(), y.data_ptr(), M, N, K,
             torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (8, 1024, 4096), (37, 2048, 3072),
                                   (64, 28672, 4096), (64, 4096, 14336)])
def test_noalloc_matches_workspace_path_twice(fp8, M, N, K):
    xb = wl.normal((M, K), 1.0, 0, M + N)
    wb = wl.zero_blocks(wl.normal((N, K), 0.02, 1, M + N), 0.02)
    x, w = wl.to_torch_bf16(xb).cuda(), wl.to_torch_bf16(wb).cuda()
    q_a, s_a = fp8.quant_act(x)
    q_w, s_w = fp8.quant_weight(w)
    ref = fp8.block_linear(q_a, s_a, q_w, s_w)            # caller-provided workspace
    torch.cuda.synchronize()
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _c_call(fp8, q_a, s_a, q_w, s_w, y, M, N, K) == 0
        fp8.check()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), \
            f"noalloc call {call} {M}x{N}x{K} differs from fp8_block_linear"


def test_noalloc_against_the_oracle(fp8):
    """One decode shape with ragged tokens and zeroed weight blocks: the
    no-allocation output meets the GEMM tolerance against the oracle's fp64
    result computed from the same codes and scales."""
    import oracle
    M, N, K = 37, 2048, 3072
    xb = wl.normal((M, K), 1.0, 0, 91)
    wb = wl.zero_blocks(wl.normal((N, K), 0.02, 1, 91), 0.05)
    x, w = wl.to_torch_bf16(xb).cuda(), wl.to_torch_bf16(wb).cuda()
    q_a, s_a = fp8.quant_act(x)
    q_w, s_w = fp8.quant_weight(w)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _c_call(fp8, q_a, s_a, q_w, s_w, y, M, N, K) == 0
    fp8.check()
    R = oracle.block_linear(q_a.view(torch.uint8).cpu().numpy(), s_a.cpu().numpy(),
                            q_w.view(torch.uint8).cpu().numpy(), s_w.cpu().numpy(), nthreads=8)
    check_gemm(y.float().cpu().numpy(), R, "noalloc vs oracle")


def test_noalloc_binding_allocates_nothing(fp8):
    M, N, K = 16, 2048, 4096
    x = wl.to_torch_bf16(wl.normal((M, K), 1.0, 0, 5)).cuda()
    w = wl.to_torch_bf16(wl.normal((N, K), 0.02, 1, 5)).cuda()
    q_a, s_a = fp8.quant_act(x)
    q_w, s_w = fp8.quant_weight(w)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    fp8.block_linear_noalloc(q_a, s_a, q_w, s_w, y)
    fp8.block_linear_noalloc(q_a, s_a, q_w, s_w, y)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    _within_tolerance(y, fp8.block_linear(q_a, s_a, q_w, s_w), "binding")


def test_noalloc_refuses_what_it_cannot_serve(fp8):
    """Shapes outside the decode schedule or beyond the built-in scratch are
    refused on the host before anything is launched (real, in-bounds
    buffers are passed all the same)."""
    # more than 64 tokens: not the decode schedule (fp8_block_linear needs
    # no workspace there)
    M, N, K = 65, 128, 128
    q_a = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    s_a = torch.ones((M, K // 128), dtype=torch.float32, device="cuda")
    q_w = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    s_w = torch.ones((N // 128, K // 128), dtype=torch.float32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _c_call(fp8, q_a, s_a, q_w, s_w, y, M, N, K) == 2
    # many one-chunk weight blocks: the partials need ~73 MB > 16 MiB
    M, N, K = 64, 128 * 2048, 128
    assert fp8.workspace_bytes(M, N, K) > 16 << 20
    q_a = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    s_a = torch.ones((M, K // 128), dtype=torch.float32, device="cuda")
    q_w = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    s_w = torch.ones((N // 128, K // 128), dtype=torch.float32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _c_call(fp8, q_a, s_a, q_w, s_w, y, M, N, K) == 7
    fp8.check()
