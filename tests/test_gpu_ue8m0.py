"""GPU parity of the UE8M0 (power-of-two scale) variant against the oracle,
through the C ABI.

Method: "Fine-grained FP8" page of the transformers docs, "UE8M0 scale
format" section (scales kept as float8_e8m0fnu).  Quantized codes and scale
codes must match the oracle bit for bit; the GEMM (on the tensor core's
block-scaled MMA) must meet the tolerance in tests/parity.py against the
oracle's fp64 result computed from the same codes.  The GEMM is also fed
random codes with per-row scale codes spread over 2^+-20, so that a scale
factor applied to the wrong row, column block or K block cannot hide in the
tolerance.
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


def _check_act(fp8, bits):
    q, s = fp8.quant_act_ue8m0(to_dev(bits))
    torch.cuda.synchronize()
    qo, so = oracle.quant_act_ue8m0(bits, nthreads=8)
    assert s.dtype == torch.float8_e8m0fnu
    assert np.array_equal(u8(s), so), "scale codes differ"
    bad = np.count_nonzero(u8(q) != qo)
    assert bad == 0, f"{bad} codes differ"


@pytest.mark.parametrize("M,K", [(32, 512), (1, 128), (3, 384), (129, 1024), (33, 7168),
                                 (64, 18432)])
def test_act_quant_shapes(fp8, M, K):
    _check_act(fp8, wl.normal((M, K), 1.0, 0, 31 * M + K))


def test_act_quant_edge_values(fp8):
    bits = wl.student_t_outliers(40, 1024, 3.0, 0.01, 100.0)
    bits[0, :128] = 0                       # all-zero group -> eps floor, code 85
    bits[1, 128:256] = 0x8000               # all -0.0
    bits[2, 256:384] = 0x0001               # bf16 denormals
    bits[3, 384:512] = 0x7F7F               # bf16 max -> code 247
    bits[4, 512:640] = wl.f32_to_bf16_bits(np.full(128, 1e-38, np.float32))
    bits[5, :] = wl.f32_to_bf16_bits(np.linspace(-3e30, 3e30, 1024).astype(np.float32))
    bits[6, 0:128] = wl.f32_to_bf16_bits(np.float32(2.0) ** -np.arange(128, dtype=np.float32))
    bits[7, 0:128] = wl.f32_to_bf16_bits(np.full(128, 448.0 * 2.0 ** -5, np.float32))  # exact power
    bits[8, 0:128] = wl.f32_to_bf16_bits(np.full(128, -448.0, np.float32))
    _check_act(fp8, bits)


def test_act_quant_16_byte_aligned_input(fp8):
    """The 16-byte-load kernel (input not 32-byte aligned)."""
    bits = wl.normal((17, 640), 2.0, 21)
    buf = torch.empty(17 * 640 + 8, dtype=torch.bfloat16, device="cuda")
    x = buf[8:].view(17, 640)
    x.copy_(to_dev(bits))
    assert x.data_ptr() % 32 == 16
    q, s = fp8.quant_act_ue8m0(x)
    torch.cuda.synchronize()
    qo, so = oracle.quant_act_ue8m0(bits)
    assert np.array_equal(u8(s), so) and np.array_equal(u8(q), qo)


def test_act_quant_empty(fp8):
    q, s = fp8.quant_act_ue8m0(torch.empty((0, 256), dtype=torch.bfloat16, device="cuda"))
    assert q.shape == (0, 256) and s.shape == (0, 2)


@pytest.mark.parametrize("N,K", [(128, 128), (256, 384), (1024, 4096), (384, 7168)])
def test_weight_quant_shapes(fp8, N, K):
    bits = wl.zero_blocks(wl.normal((N, K), 0.02, 1, N + K), 0.1)
    q, s = fp8.quant_weight_ue8m0(to_dev(bits))
    torch.cuda.synchronize()
    qo, so = oracle.quant_weight_ue8m0(bits)
    assert np.array_equal(u8(s), so)
    assert np.array_equal(u8(q), qo)


def _run(fp8, xbits, wbits, rows=None):
    x, w = to_dev(xbits), to_dev(wbits)
    q_a, s_a = fp8.quant_act_ue8m0(x)
    q_w, s_w = fp8.quant_weight_ue8m0(w)
    y = fp8.block_linear_ue8m0(q_a, s_a, q_w, s_w)
    fp8.check()
    R = oracle.block_linear_ue8m0(u8(q_a), u8(s_a), u8(q_w), u8(s_w), rows=rows, nthreads=8)
    yv = f32(y) if rows is None else f32(y[torch.as_tensor(rows, device=y.device)])
    return yv, R, (q_a, s_a, q_w, s_w, y)


def test_tiny(fp8):
    xb, wb = wl.tiny()
    y, R, _ = _run(fp8, xb, wb)
    check_gemm(y, R, "tiny")


@pytest.mark.parametrize("M,N,K", [
    (1, 128, 128), (5, 384, 256), (127, 256, 384), (129, 640, 1024), (300, 512, 512),
    (64, 1024, 4096), (257, 768, 2048), (1000, 1152, 1152),
])
def test_ragged_shapes(fp8, M, N, K):
    xb = wl.normal((M, K), 1.0, 0, 3 * M + N + K)
    wb = wl.normal((N, K), 0.02, 1, 3 * M + N + K)
    y, R, _ = _run(fp8, xb, wb)
    check_gemm(y, R, f"{M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (130, 384, 1280)])
def test_scale_factor_placement(fp8, M, N, K):
    """Random e4m3 codes with scale codes that differ by up to 2^40 between
    rows, weight blocks and K blocks: any scale factor read for the wrong
    row, block or slice changes the result by orders of magnitude."""
    g = np.random.default_rng(M + N + K)
    qa = g.integers(0, 256, (M, K), dtype=np.uint8)
    qw = g.integers(0, 256, (N, K), dtype=np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x00
    qw[(qw & 0x7F) == 0x7F] = 0x00
    ca = g.integers(107, 148, (M, K // 128), dtype=np.uint8)
    cw = g.integers(107, 148, (N // 128, K // 128), dtype=np.uint8)
    dev = lambda a: torch.from_numpy(a).cuda()
    y = fp8.block_linear_ue8m0(dev(qa).view(torch.float8_e4m3fn), dev(ca).view(torch.float8_e8m0fnu),
                               dev(qw).view(torch.float8_e4m3fn), dev(cw).view(torch.float8_e8m0fnu))
    fp8.check()
    R = oracle.block_linear_ue8m0(qa, ca, qw, cw, nthreads=8)
    check_gemm(f32(y), R, "placement")


def test_scale_extremes(fp8):
    M, N, K = 192, 512, 1024
    g = np.random.default_rng(5)
    x = g.standard_normal((M, K)).astype(np.float32) * np.exp(g.uniform(-9, 9, (M, 1))).astype(np.float32)
    xb = wl.f32_to_bf16_bits(x)
    xb[7, 256:384] = 0
    wb = wl.zero_blocks(wl.normal((N, K), 0.02, 2), 0.2)
    y, R, _ = _run(fp8, xb, wb)
    check_gemm(y, R, "extremes")


def test_deterministic(fp8):
    xb = wl.normal((300, 1024), 1.0, 3)
    wb = wl.normal((768, 1024), 0.02, 4)
    _, _, (q_a, s_a, q_w, s_w, y) = _run(fp8, xb, wb)
    for _ in range(3):
        y2 = fp8.block_linear_ue8m0(q_a, s_a, q_w, s_w)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def _sample_rows(M, n, seed=0):
    g = np.random.default_rng(seed)
    r = set([0, 1, M - 1, M // 2]) | set(g.choice(M, n, replace=False).tolist())
    return np.array(sorted(r), dtype=np.int64)


@pytest.mark.parametrize("which", ["gate_up", "down"])
def test_full_size_prefill(fp8, which):
    xb, wb = wl.llama3_prefill(which)
    rows = _sample_rows(xb.shape[0], 24)
    y, R, _ = _run(fp8, xb, wb, rows=rows)
    check_gemm(y, R, f"llama3 prefill {which}")


@pytest.mark.parametrize("M", [1, 8, 64])
def test_decode_sizes(fp8, M):
    xb, wb = wl.llama3_decode(M, "qo")
    y, R, _ = _run(fp8, xb, wb)
    check_gemm(y, R, f"decode qo M={M}")


def test_full_size_sweep(fp8):
    xb, wb = wl.sweep_x(8192), wl.sweep_w()
    rows = _sample_rows(8192, 16)
    y, R, _ = _run(fp8, xb, wb, rows=rows)
    check_gemm(y, R, "sweep 8192")


def test_no_timeout_recorded(fp8):
    fp8.check()


@pytest.mark.parametrize("M,N,K", [(129, 384, 384), (256, 512, 512), (300, 1152, 1280),
                                   (4096 + 128, 1024, 2048), (1000, 28672, 512)])
def test_pairs_equal_single_cta(fp8, M, N, K):
    """The CTA-pair schedule (fp8_block_linear_ue8m0_ws, M > 128) runs the
    same block-scaled MMAs in the same K order as the single-CTA kernel
    (fp8_block_linear_ue8m0): the outputs must be equal bit for bit, here on
    random codes with scale codes spread over 2^+-20 so that a scale factor
    copied to the wrong TMEM lane, column or slice shows."""
    g = np.random.default_rng(7 * M + N + K)
    qa = g.integers(0, 256, (M, K), dtype=np.uint8)
    qw = g.integers(0, 256, (N, K), dtype=np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x00
    qw[(qw & 0x7F) == 0x7F] = 0x00
    ca = g.integers(107, 148, (M, K // 128), dtype=np.uint8)
    cw = g.integers(107, 148, (N // 128, K // 128), dtype=np.uint8)
    dev = lambda a: torch.from_numpy(a).cuda()
    args = (dev(qa).view(torch.float8_e4m3fn), dev(ca).view(torch.float8_e8m0fnu),
            dev(qw).view(torch.float8_e4m3fn), dev(cw).view(torch.float8_e8m0fnu))
    assert fp8.ue8m0_workspace_bytes(M, N, K) > 0
    y_pair = fp8.block_linear_ue8m0(*args)
    y_single = fp8.block_linear_ue8m0(*args, pairs=False)
    fp8.check()
    assert torch.equal(y_pair.view(torch.int16), y_single.view(torch.int16)), (M, N, K)
    rows = _sample_rows(M, 8, seed=M)
    R = oracle.block_linear_ue8m0(qa, ca, qw, cw, rows=rows, nthreads=8)
    check_gemm(f32(y_pair[torch.as_tensor(rows, device=y_pair.device)]), R, f"pairs {M}x{N}x{K}")


def test_pairs_workspace_checks(fp8):
    M, N, K = 256, 256, 256
    need = fp8.ue8m0_workspace_bytes(M, N, K)
    assert need > 0 and fp8.ue8m0_workspace_bytes(128, N, K) == 0
    z = lambda *s: torch.zeros(s, dtype=torch.uint8, device="cuda")
    q_a, q_w = z(M, K).view(torch.float8_e4m3fn), z(N, K).view(torch.float8_e4m3fn)
    s_a = torch.full((M, K // 128), 127, dtype=torch.uint8, device="cuda").view(torch.float8_e8m0fnu)
    s_w = torch.full((N // 128, K // 128), 127, dtype=torch.uint8, device="cuda").view(torch.float8_e8m0fnu)
    with pytest.raises(fp8.Fp8blError) as ei:
        fp8.block_linear_ue8m0(q_a, s_a, q_w, s_w, workspace=z(need - 16))
    assert ei.value.status == 7
    fp8.check()
