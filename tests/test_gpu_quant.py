"""GPU parity: activation and weight quantization must match the oracle bit
for bit (codes and fp32 scales), through the C ABI.

Shapes cover the workloads ("Fine-grained FP8" page: 1x128 activation
groups, 128x128 weight blocks) plus ragged and degenerate cases: a single
row, odd row counts, one group per row, all-zero and negative-zero groups,
huge and tiny magnitudes.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import to_dev, u8, f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fine_grained_block_token_b200 as m
    return m


def _check_act(fp8, bits, nthreads=8):
    x = to_dev(bits)
    q, s = fp8.quant_act(x)
    torch.cuda.synchronize()
    qo, so = oracle.quant_act(bits, nthreads=nthreads)
    gq, gs = u8(q), f32(s)
    assert np.array_equal(gs.view(np.uint32), so.view(np.uint32)), "scales differ"
    bad = np.count_nonzero(gq != qo)
    assert bad == 0, f"{bad} codes differ"


@pytest.mark.parametrize("M,K", [(32, 512), (1, 128), (3, 384), (127, 256), (129, 1024),
                                 (1, 4096), (8, 14336), (33, 7168), (64, 18432)])
def test_act_quant_shapes(fp8, M, K):
    _check_act(fp8, wl.normal((M, K), 1.0, 0, M * 7 + K))


def test_act_quant_edge_values(fp8):
    bits = wl.student_t_outliers(40, 1024, 3.0, 0.01, 100.0)
    bits[0, :128] = 0                       # all-zero group
    bits[1, 128:256] = 0x8000               # all -0.0
    bits[2, 256:384] = 0x0001               # bf16 denormals
    bits[3, 384:512] = 0x7F7F               # bf16 max
    bits[4, 512:640] = wl.f32_to_bf16_bits(np.full(128, 1e-38, np.float32))
    bits[5, :] = wl.f32_to_bf16_bits(np.linspace(-3e30, 3e30, 1024).astype(np.float32))
    bits[6, 0:128] = wl.f32_to_bf16_bits(np.float32(2.0) ** -np.arange(128, dtype=np.float32))
    _check_act(fp8, bits)


def test_act_quant_empty(fp8):
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q, s = fp8.quant_act(x)
    assert q.shape == (0, 256) and s.shape == (0, 2)


@pytest.mark.parametrize("name", ["prefill_gate_up", "prefill_down", "sweep_16384"])
def test_act_quant_full_size(fp8, name):
    if name == "prefill_gate_up":
        bits, _ = wl.llama3_prefill("gate_up")
    elif name == "prefill_down":
        bits, _ = wl.llama3_prefill("down")
    else:
        bits = wl.sweep_x(16384)
    _check_act(fp8, bits)


def test_act_quant_deepseek_full_size(fp8):
    bits, _ = wl.deepseek_mlp("down")       # X [8192, 18432]
    _check_act(fp8, bits)


def _check_weight(fp8, bits):
    w = to_dev(bits)
    q, s = fp8.quant_weight(w)
    torch.cuda.synchronize()
    qo, so = oracle.quant_weight(bits)
    assert np.array_equal(f32(s).view(np.uint32), so.view(np.uint32))
    assert np.array_equal(u8(q), qo)


@pytest.mark.parametrize("N,K", [(256, 512), (128, 128), (384, 640), (1024, 4096)])
def test_weight_quant_shapes(fp8, N, K):
    bits = wl.normal((N, K), 0.02, 1, N + K)
    bits = wl.zero_blocks(bits, 0.1)
    _check_weight(fp8, bits)


def test_weight_quant_full_size(fp8):
    _, wbits = wl.deepseek_mlp("up")        # W [18432, 7168], 1% zero blocks
    _check_weight(fp8, wbits)


def test_act_quant_16_byte_aligned_input(fp8):
    """Inputs that are 16- but not 32-byte aligned take the 16-byte kernel;
    codes and scales must be identical to the oracle as well."""
    M, K = 77, 1536
    bits = wl.student_t_outliers(M, K, 3.0, 0.01, 100.0)
    base = torch.empty(M * K + 64, dtype=torch.bfloat16, device="cuda")
    x = base[8:8 + M * K].view(M, K)                    # +16 bytes
    assert x.data_ptr() % 32 == 16
    x.copy_(wl.to_torch_bf16(bits).cuda())
    q, s = fp8.quant_act(x)
    torch.cuda.synchronize()
    qo, so = oracle.quant_act(bits, nthreads=8)
    assert np.array_equal(f32(s).view(np.uint32), so.view(np.uint32))
    assert np.array_equal(u8(q), qo)


# ------------------------------------------------ static activation scale


@pytest.mark.parametrize("M,K,sc", [(32, 512, 0.01), (1, 128, 1.0), (129, 7168, 0.0037),
                                    (64, 18432, 2.5e-4)])
def test_act_quant_static(fp8, M, K, sc):
    bits = wl.student_t_outliers(M, K, 3.0, 0.01, 100.0, M + K)
    bits[0, :128] = 0x8000
    s_given = torch.tensor([sc], dtype=torch.float32, device="cuda")
    q, s = fp8.quant_act_static(to_dev(bits), s_given)
    torch.cuda.synchronize()
    qo, so = oracle.quant_act_static(bits, sc)
    assert np.array_equal(f32(s), so)
    assert np.count_nonzero(u8(q) != qo) == 0


def test_act_quant_static_16_byte_aligned_input(fp8):
    bits = wl.normal((9, 384), 3.0, 5)
    buf = torch.empty(9 * 384 + 8, dtype=torch.bfloat16, device="cuda")
    x = buf[8:].view(9, 384)
    x.copy_(to_dev(bits))
    s_given = torch.tensor([0.004], dtype=torch.float32, device="cuda")
    q, s = fp8.quant_act_static(x, s_given)
    torch.cuda.synchronize()
    qo, so = oracle.quant_act_static(bits, 0.004)
    assert np.array_equal(u8(q), qo) and np.array_equal(f32(s), so)


def test_static_then_block_linear(fp8):
    """The static outputs feed the block linear unchanged; parity with the
    oracle's block linear from the same codes and scales."""
    from tests.parity import check_gemm
    xb = wl.normal((200, 1024), 1.0, 6)
    wb = wl.normal((512, 1024), 0.02, 7)
    sc = float(np.abs(wl.bf16_bits_to_f32(xb)).max() / 448.0 * 0.5)   # half the range: some saturation
    q_a, s_a = fp8.quant_act_static(to_dev(xb), torch.tensor([sc], dtype=torch.float32, device="cuda"))
    q_w, s_w = fp8.quant_weight(to_dev(wb))
    y = fp8.block_linear(q_a, s_a, q_w, s_w)
    fp8.check()
    qo, so = oracle.quant_act_static(xb, sc)
    assert np.array_equal(u8(q_a), qo)
    R = oracle.block_linear(qo, so, u8(q_w), f32(s_w), nthreads=8)
    check_gemm(f32(y), R, "static + block linear")
