"""Pins for the oracle's row-wise FP8 (fp8r) variant.

Method: "BFL (fp8r / nvfp4)" page of the diffusers docs, first bullet of its
list (E4M3 weight with one fp32 scale per row; activations quantized per row
at run time) and its "Kernels" table (a scaled matmul with row-wise scales).
Reading: the fine-grained scheme's scale rule with one group per row,
s = fp32(max(amax_row, 1e-10) / 448), q = e4m3(x / s), and
y[m,n] = s_a[m] s_w[n] sum_k q_a[m,k] q_w[n,k].

Expectations are formed another way: numpy row reductions, fp32 division and
torch's e4m3 cast; the pinned 1x128 block quantizer; exact rationals.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

EPS = np.float32(1e-10)


def _expected(bits):
    x = wl.bf16_bits_to_f32(bits)
    amax = np.abs(x).max(axis=1)
    s = (np.maximum(amax, EPS) / np.float32(448.0)).astype(np.float32)
    t = (x / s[:, None]).astype(np.float32)
    assert np.all(np.abs(t) < 464.0)
    q = torch.from_numpy(np.ascontiguousarray(t)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return q, s


@pytest.mark.parametrize("R,K,seed", [(8, 256, 0), (5, 4096, 1), (1, 16, 2), (3, 7168, 3)])
def test_quant_vs_library_composition(R, K, seed):
    bits = wl.student_t_outliers(R, K, 3.0, 0.01, 30.0, seed) if K % 128 == 0 else wl.normal((R, K), 1.0, seed)
    q, s = oracle.quant_rowwise(bits)
    qe, se = _expected(bits)
    assert np.array_equal(s, se) and np.array_equal(q, qe)


def test_zero_and_negative_zero_rows():
    bits = wl.normal((4, 512), 1.0, 4)
    bits[1] = 0
    bits[2] = 0x8000
    q, s = oracle.quant_rowwise(bits)
    assert s[1] == np.float32(EPS) / np.float32(448.0)
    assert np.all(q[1] == 0x00) and np.all(q[2] == 0x80)


def test_row_max_maps_to_448():
    bits = wl.normal((6, 1024), 2.0, 5)
    q, _ = oracle.quant_rowwise(bits)
    x = wl.bf16_bits_to_f32(bits)
    i = np.abs(x).argmax(axis=1)
    top = q[np.arange(6), i]
    assert np.all((top & 0x7F) == 0x7E)
    assert np.array_equal(top >> 7, (x[np.arange(6), i] < 0).astype(np.uint8))


def test_equals_block_quant_when_groups_share_the_row_max():
    """If every 1x128 group of a row holds the row's largest magnitude, the
    row scale equals each group scale, so the codes equal the pinned 1x128
    activation quantizer's."""
    bits = wl.normal((4, 640), 1.0, 6)
    x = wl.bf16_bits_to_f32(bits).copy()
    for r in range(4):
        x[r, 3::128] = np.float32(5.0 + r)
    bits = wl.f32_to_bf16_bits(x)
    qr, sr = oracle.quant_rowwise(bits)
    qb, sb = oracle.quant_act(bits)
    assert np.array_equal(qr, qb)
    assert np.array_equal(np.repeat(sr[:, None], 5, axis=1), sb)


def test_row_range_matches_full():
    bits = wl.normal((9, 384), 1.0, 7)
    q, s = oracle.quant_rowwise(bits)
    q2, s2 = oracle.quant_rowwise(bits, 2, 6)
    assert np.array_equal(q[2:6], q2) and np.array_equal(s[2:6], s2)


def _codes(shape, g):
    c = g.integers(0, 256, shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0
    return c


def test_linear_vs_exact_rationals():
    g = np.random.default_rng(8)
    M, N, K = 3, 5, 160
    qa, qw = _codes((M, K), g), _codes((N, K), g)
    sa = g.uniform(0.001, 2.0, M).astype(np.float32)
    sw = g.uniform(0.001, 2.0, N).astype(np.float32)
    y = oracle.linear_rowwise(qa, sa, qw, sw)
    dec = oracle.e4m3_decode_table()
    for m in range(M):
        for n in range(N):
            b = sum(Fraction(float(dec[qa[m, k]])) * Fraction(float(dec[qw[n, k]])) for k in range(K))
            exact = Fraction(float(sa[m])) * Fraction(float(sw[n])) * b
            assert abs(Fraction(float(y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 51)


def test_unit_scales_reduce_to_integer_matmul():
    g = np.random.default_rng(9)
    M, N, K = 7, 33, 512
    qa, qw = _codes((M, K), g), _codes((N, K), g)
    ones_a, ones_w = np.ones(M, np.float32), np.ones(N, np.float32)
    y = oracle.linear_rowwise(qa, ones_a, qw, ones_w)
    dec = oracle.e4m3_decode_table()
    ia = np.rint(dec[qa] * 512).astype(np.int64)
    iw = np.rint(dec[qw] * 512).astype(np.int64)
    assert np.array_equal(y * 2.0 ** 18, (ia @ iw.T).astype(np.float64))


def test_scale_index_per_row_and_column():
    """Doubling s_a[m] doubles row m only; doubling s_w[n] doubles column n only."""
    g = np.random.default_rng(10)
    M, N, K = 4, 6, 256
    qa, qw = _codes((M, K), g), _codes((N, K), g)
    sa, sw = g.uniform(0.5, 1, M).astype(np.float32), g.uniform(0.5, 1, N).astype(np.float32)
    y0 = oracle.linear_rowwise(qa, sa, qw, sw)
    sa2 = sa.copy(); sa2[2] *= 2
    sw2 = sw.copy(); sw2[4] *= 2
    y1 = oracle.linear_rowwise(qa, sa2, qw, sw)
    y2 = oracle.linear_rowwise(qa, sa, qw, sw2)
    e1 = y0.copy(); e1[2] *= 2
    e2 = y0.copy(); e2[:, 4] *= 2
    assert np.array_equal(y1, e1) and np.array_equal(y2, e2)
