"""Pins for the oracle's UE8M0 (power-of-two scale) variant.

Method: transformers docs, "Fine-grained FP8" page, "UE8M0 scale format"
section (scales kept as float8_e8m0fnu, scale_fmt="ue8m0").  Reading: the
scale of a group or block is the smallest power of two 2^e with
max(amax, 1e-10) <= 448 * 2^e, stored as the byte e + 127, and
q = e4m3(x * 2^-e).

Each expectation is formed another way than the oracle forms it: torch's
float8_e8m0fnu and float8_e4m3fn casts, numpy's frexp of the quotient, the
already-pinned fp32 scales, closed forms at the binade edges.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

EPS = np.float32(1e-10)


def _f32(bits):
    return wl.bf16_bits_to_f32(bits)


def _ceil_log2_frexp(t):
    """ceil(log2 t) for positive fp64 t via frexp: t = f * 2^e, f in [0.5, 1)."""
    f, e = np.frexp(np.asarray(t, dtype=np.float64))
    return np.where(f == 0.5, e - 1, e)


def _expected_codes(g, c):
    """torch e4m3 cast of RN32(x * 2^-(c-127)) for groups g [..., 128]."""
    inv = np.ldexp(np.float32(1.0), (127 - c.astype(np.int64)))[..., None].astype(np.float32)
    t = (g.astype(np.float32) * inv).astype(np.float32)
    assert np.all(np.abs(t) <= 448.0)
    return torch.from_numpy(np.ascontiguousarray(t)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e8m0fnu).to(torch.float32).double().numpy()
    got = oracle.ue8m0_decode(codes)
    assert np.isnan(got[255]) and np.isnan(ref[255])
    assert np.array_equal(got[:255], ref[:255])


@pytest.mark.parametrize("k", [-30, -7, -1, 0, 1, 5, 40])
def test_scale_code_at_binade_edges(k):
    """448 * 2^k needs exactly 2^k; the next fp32 above it needs 2^(k+1);
    the fp32 below it still fits 2^k."""
    a = np.float32(np.ldexp(448.0, k))
    up = np.nextafter(a, np.float32(np.inf))
    down = np.nextafter(a, np.float32(0))
    assert oracle.ue8m0_from_amax(a) == 127 + k
    assert oracle.ue8m0_from_amax(up) == 128 + k
    assert oracle.ue8m0_from_amax(down) == 127 + k


def test_scale_code_zero_group_uses_eps():
    # 448 * 2^-43 < 1e-10 <= 448 * 2^-42
    assert np.ldexp(448.0, -43) < 1e-10 <= np.ldexp(448.0, -42)
    assert oracle.ue8m0_from_amax(0.0) == 127 - 42
    assert oracle.ue8m0_from_amax(np.float32(1e-12)) == 127 - 42


def test_scale_code_vs_frexp_random():
    rng = np.random.default_rng(5)
    a = np.exp(rng.uniform(np.log(1e-9), np.log(1e37), 4000)).astype(np.float32)
    got = np.array([oracle.ue8m0_from_amax(v) for v in a]).astype(np.int64) - 127
    exp = _ceil_log2_frexp(np.maximum(a, EPS).astype(np.float64) / 448.0)
    assert np.array_equal(got, exp)


def test_scale_code_every_bf16_amax():
    """Every positive finite bf16 magnitude (the amax values the bf16 input
    can produce): the code is minimal, and matches the frexp route."""
    bits = np.arange(1, 0x7F80, dtype=np.uint16)
    a = _f32(bits)
    got = np.array([oracle.ue8m0_from_amax(v) for v in a]).astype(np.int64) - 127
    am = np.maximum(a, EPS).astype(np.float64)
    assert np.all(am <= np.ldexp(448.0, got))
    assert np.all(am > np.ldexp(448.0, got - 1))
    assert np.array_equal(got, _ceil_log2_frexp(am / 448.0))


def test_act_vs_library_composition():
    bits = wl.student_t_outliers(24, 640, 3.0, 0.01, 30.0, 7)
    bits[2, 128:256] = 0
    bits[4, 0:128] = 0x8000
    q, c = oracle.quant_act_ue8m0(bits)
    x = _f32(bits).reshape(24, 5, 128)
    amax = np.abs(x).max(axis=2)
    e = _ceil_log2_frexp(np.maximum(amax, EPS).astype(np.float64) / 448.0)
    assert np.array_equal(c.astype(np.int64), e + 127)
    assert np.array_equal(q, _expected_codes(x, c).reshape(24, 640))
    assert np.all(q[2, 128:256] == 0) and np.all(q[4, 0:128] == 0x80)


def test_act_scales_bracket_fp32_scales():
    """s_fp32 <= 2^e < 2 s_fp32 (the power of two is the fp32 scale rounded
    up), against the pinned fp32 quantizer."""
    bits = wl.normal((16, 1024), 3.0, 11)
    _, s32 = oracle.quant_act(bits)
    _, c = oracle.quant_act_ue8m0(bits)
    p2 = oracle.ue8m0_decode(c)
    assert np.all(s32.astype(np.float64) <= p2)
    assert np.all(p2 < 2.0 * s32.astype(np.float64))


def test_act_amax_element_code_range():
    """The group's largest element lands in (224, 448] -- the top binade."""
    bits = wl.normal((8, 512), 1.0, 12)
    q, c = oracle.quant_act_ue8m0(bits)
    x = _f32(bits).reshape(8, 4, 128)
    qv = oracle.e4m3_decode_table()[q.reshape(8, 4, 128)]
    idx = np.abs(x).argmax(axis=2)
    top = np.take_along_axis(np.abs(qv), idx[..., None], axis=2)[..., 0]
    assert np.all(top > 224.0 - 1e-9) and np.all(top <= 448.0)


def test_act_rows_match_full():
    bits = wl.normal((9, 384), 0.5, 13)
    q, c = oracle.quant_act_ue8m0(bits, nthreads=3)
    q2, c2 = oracle.quant_act_ue8m0_rows(bits, 3, 7)
    assert np.array_equal(q[3:7], q2) and np.array_equal(c[3:7], c2)


def test_power_of_two_equivariance():
    """Scaling the input by 2^k shifts every code by k and leaves q alone."""
    bits = wl.normal((4, 256), 1.0, 14)
    x = _f32(bits)
    q0, c0 = oracle.quant_act_ue8m0(bits)
    q1, c1 = oracle.quant_act_ue8m0(wl.f32_to_bf16_bits(x * np.float32(8.0)))
    assert np.array_equal(q0, q1)
    assert np.array_equal(c1.astype(int), c0.astype(int) + 3)


def test_weight_vs_library_composition():
    bits = wl.normal((256, 384), 0.02, 15)
    bits = wl.zero_blocks(bits, 0.2)
    w = _f32(bits).reshape(2, 128, 3, 128) * np.array([1, 3, 7, 20, 50, 0.1], np.float32).reshape(2, 1, 3, 1)
    bits = wl.f32_to_bf16_bits(w.reshape(256, 384))
    q, c = oracle.quant_weight_ue8m0(bits)
    w = _f32(bits).reshape(2, 128, 3, 128)
    amax = np.abs(w).max(axis=(1, 3))
    e = _ceil_log2_frexp(np.maximum(amax, EPS).astype(np.float64) / 448.0)
    assert c.shape == (2, 3)
    assert np.array_equal(c.astype(np.int64), e + 127)
    blocks = w.transpose(0, 2, 1, 3)                     # [2, 3, 128, 128]
    qe = _expected_codes(blocks.reshape(2, 3, 128 * 128), c).reshape(2, 3, 128, 128)
    assert np.array_equal(q, qe.transpose(0, 2, 1, 3).reshape(256, 384))


def test_weight_equals_act_when_rows_share_amax():
    bits = wl.normal((128, 256), 0.02, 16)
    w = _f32(bits).copy()
    w[:, 7] = np.float32(0.75)
    w[:, 200] = np.float32(-3.0)
    bits = wl.f32_to_bf16_bits(w)
    qw, cw = oracle.quant_weight_ue8m0(bits)
    qa, ca = oracle.quant_act_ue8m0(bits)
    assert np.array_equal(qw, qa)
    assert np.array_equal(np.repeat(cw, 128, axis=0), ca)


def test_gemm_with_ue8m0_scales_vs_exact_sum():
    """With power-of-two scales every term is dyadic: the oracle's fp64
    result must be the correctly rounded exact sum (Python rationals)."""
    rng = np.random.default_rng(17)
    M, N, K = 3, 256, 384
    qa = rng.integers(0, 256, (M, K), dtype=np.uint8)
    qw = rng.integers(0, 256, (N, K), dtype=np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0
    qw[(qw & 0x7F) == 0x7F] = 0
    ca = rng.integers(100, 140, (M, K // 128), dtype=np.uint8)
    cw = rng.integers(100, 140, (N // 128, K // 128), dtype=np.uint8)
    y = oracle.block_linear_ue8m0(qa, ca, qw, cw)
    dec = oracle.e4m3_decode_table()
    # every e4m3 value is an integer multiple of 2^-9
    ia = np.rint(dec[qa] * 512).astype(np.int64)
    iw = np.rint(dec[qw] * 512).astype(np.int64)
    for m in range(M):
        for n in (0, 1, 77, 127, 128, 200, 255):
            tot = Fraction(0)
            for j in range(K // 128):
                b = int(np.dot(ia[m, j * 128:(j + 1) * 128], iw[n, j * 128:(j + 1) * 128]))
                tot += Fraction(b) * Fraction(2) ** (int(ca[m, j]) + int(cw[n // 128, j]) - 254 - 18)
            assert abs(Fraction(float(y[m, n])) - tot) <= abs(tot) * Fraction(1, 2 ** 51)
