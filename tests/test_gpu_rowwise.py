"""GPU parity of the row-wise FP8 variant (fp8r) against the oracle, through
the C ABI.

Method: "BFL (fp8r / nvfp4)" page of the diffusers docs (an E4M3 weight with
one fp32 scale per row; activations quantized per row at run time; a scaled
matmul with row-wise scales).  Codes and scales must match the oracle bit
for bit; the linear must meet the tolerance in tests/parity.py against the
oracle's fp64 result from the same codes.  Shapes cover K and N that are not
multiples of 128 (the tile's K tail reads zeros, the N tail is masked), rows
longer than the quantizer's register cache, and random codes with scales
spread over 2^+-20 per row and column.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import check_gemm, f32, to_dev, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fine_grained_block_token_b200 as m
    return m


@pytest.mark.parametrize("R,K", [(1, 16), (7, 144), (33, 4096), (5, 8192), (3, 8208), (2, 18432),
                                 (257, 1024)])
def test_quant_rowwise_shapes(fp8, R, K):
    bits = wl.student_t_outliers(R, K, 3.0, 0.01, 50.0, R + K) if K % 128 == 0 else \
        wl.normal((R, K), 1.0, 0, R + K)
    q, s = fp8.quant_rowwise(to_dev(bits))
    torch.cuda.synchronize()
    qo, so = oracle.quant_rowwise(bits)
    assert np.array_equal(f32(s).view(np.uint32), so.view(np.uint32))
    assert np.count_nonzero(u8(q) != qo) == 0


def test_quant_rowwise_edge_values(fp8):
    bits = wl.normal((8, 512), 1.0, 3)
    bits[0] = 0
    bits[1] = 0x8000
    bits[2] = 0x0001
    bits[3] = 0x7F7F
    bits[4] = wl.f32_to_bf16_bits(np.linspace(-3e30, 3e30, 512).astype(np.float32))
    bits[5] = wl.f32_to_bf16_bits(np.float32(2.0) ** -np.arange(512, dtype=np.float32) / 4)
    q, s = fp8.quant_rowwise(to_dev(bits))
    torch.cuda.synchronize()
    qo, so = oracle.quant_rowwise(bits)
    assert np.array_equal(f32(s).view(np.uint32), so.view(np.uint32))
    assert np.array_equal(u8(q), qo)


def test_quant_rowwise_empty(fp8):
    q, s = fp8.quant_rowwise(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"))
    assert q.shape == (0, 64) and s.shape == (0,)


def _run(fp8, xb, wb, rows=None):
    q_a, s_a = fp8.quant_rowwise(to_dev(xb))
    q_w, s_w = fp8.quant_rowwise(to_dev(wb))
    y = fp8.linear_rowwise(q_a, s_a, q_w, s_w)
    fp8.check()
    R = oracle.linear_rowwise(u8(q_a), f32(s_a), u8(q_w), f32(s_w), rows=rows)
    yv = f32(y) if rows is None else f32(y[torch.as_tensor(rows, device=y.device)])
    return yv, R, (q_a, s_a, q_w, s_w, y)


@pytest.mark.parametrize("M,N,K", [
    (1, 16, 16), (5, 48, 144), (127, 256, 384), (129, 640, 1040), (300, 528, 512),
    (64, 1024, 4096), (257, 784, 2048), (1000, 1152, 1168),
])
def test_ragged_shapes(fp8, M, N, K):
    xb = wl.normal((M, K), 1.0, 0, 5 * M + N + K)
    wb = wl.normal((N, K), 0.02, 1, 5 * M + N + K)
    y, R, _ = _run(fp8, xb, wb)
    check_gemm(y, R, f"{M}x{N}x{K}")


def test_scale_placement(fp8):
    g = np.random.default_rng(11)
    M, N, K = 300, 528, 784
    qa = g.integers(0, 256, (M, K), dtype=np.uint8)
    qw = g.integers(0, 256, (N, K), dtype=np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0
    qw[(qw & 0x7F) == 0x7F] = 0
    sa = np.exp2(g.uniform(-20, 20, M)).astype(np.float32)
    sw = np.exp2(g.uniform(-20, 20, N)).astype(np.float32)
    dev = lambda a: torch.from_numpy(a).cuda()
    y = fp8.linear_rowwise(dev(qa).view(torch.float8_e4m3fn), dev(sa), dev(qw).view(torch.float8_e4m3fn),
                           dev(sw))
    fp8.check()
    R = oracle.linear_rowwise(qa, sa, qw, sw)
    check_gemm(f32(y), R, "placement")


def test_deterministic(fp8):
    xb = wl.normal((300, 1024), 1.0, 3)
    wb = wl.normal((784, 1024), 0.02, 4)
    _, _, (q_a, s_a, q_w, s_w, y) = _run(fp8, xb, wb)
    for _ in range(3):
        y2 = fp8.linear_rowwise(q_a, s_a, q_w, s_w)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("which", ["gate_up", "down"])
def test_full_size_prefill(fp8, which):
    xb, wb = wl.llama3_prefill(which)
    g = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, xb.shape[0] - 1], g.choice(xb.shape[0], 16, replace=False)]))
    y, R, _ = _run(fp8, xb, wb, rows=rows)
    check_gemm(y, R, f"llama3 prefill {which}")


def test_no_timeout_recorded(fp8):
    fp8.check()


@pytest.mark.parametrize("M,N,K", [(129, 512, 1024), (255, 256, 2048), (256, 768, 512), (257, 256, 384),
                                   (4096, 2048, 4096)])
def test_pair_boundaries_and_repeated_runs(fp8, M, N, K):
    """M around the CTA-pair tile (256 rows: the odd CTA with no rows, a
    partial tile, several tiles): parity, then five more runs bit-identical
    (a hand-off race between the two CTAs would show up as differing runs)."""
    xb = wl.normal((M, K), 1.0, 0, 7 * M + N + K)
    wb = wl.normal((N, K), 0.02, 1, 7 * M + N + K)
    rows = None if M <= 300 else np.array([0, 1, 127, 128, 255, 256, 2047, 4095])
    y, R, (q_a, s_a, q_w, s_w, y0) = _run(fp8, xb, wb, rows=rows)
    check_gemm(y, R, f"{M}x{N}x{K}")
    for _ in range(5):
        y1 = fp8.linear_rowwise(q_a, s_a, q_w, s_w)
        torch.cuda.synchronize()
        assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    fp8.check()
