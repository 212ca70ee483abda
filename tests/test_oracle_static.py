"""Pins for the oracle's static activation scale scheme.

Method: "Fine-grained FP8" page, "DeepGEMM fast path" section (static
activation quantization exists next to the dynamic scheme; the page says no
more).  Reading: one given fp32 scale s per linear, q = e4m3(x / s) with the
saturating rounding of the dynamic scheme, and the linear is the block-scaled
one with every activation group scale equal to s.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl


def _expected(bits, s):
    x = wl.bf16_bits_to_f32(bits)
    t = (x / np.float32(s)).astype(np.float32)          # IEEE fp32 division
    t = np.clip(t, -448.0, 448.0)                        # the saturating rule (torch's cast gives NaN)
    return torch.from_numpy(np.ascontiguousarray(t)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@pytest.mark.parametrize("s", [0.01, 0.0071, 1.0, 3.3e-3])
def test_vs_library_composition(s):
    bits = wl.student_t_outliers(16, 512, 3.0, 0.01, 30.0, 1)
    bits[2, :128] = 0x8000
    q, sa = oracle.quant_act_static(bits, s)
    assert np.array_equal(q, _expected(bits, s))
    assert np.all(sa == np.float32(s)) and sa.shape == (16, 4)


def test_saturates_above_448_s():
    x = np.array([[448.0, 449.0, 464.0, 1e30, -1e30, -500.0, 0.5, -0.0] * 16], np.float32)
    q, _ = oracle.quant_act_static(wl.f32_to_bf16_bits(x), 1.0)
    assert list(q[0, :8]) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x30, 0x80]


def test_equals_dynamic_when_s_is_every_groups_scale():
    """Every 128-group carries the same largest magnitude a, so the dynamic
    scale of each group is fp32(a / 448); with that s the static codes are the
    pinned dynamic quantizer's."""
    bits = wl.normal((6, 768), 1.0, 2)
    x = wl.bf16_bits_to_f32(bits).copy()
    x[:, 5::128] = np.float32(9.0)
    bits = wl.f32_to_bf16_bits(x)
    qd, sd = oracle.quant_act(bits)
    s = np.float32(9.0) / np.float32(448.0)
    assert np.all(sd == s)
    qs, ss = oracle.quant_act_static(bits, s)
    assert np.array_equal(qs, qd) and np.array_equal(ss, sd)
