"""Pins for the oracle's activation and weight quantizers.

Method (transformers docs, "Fine-grained FP8" page, opening bullet list):
per-token activation groups of 128 input channels, 128 x 128 weight blocks,
one fp32 scale each.  Scale reading: s = max(amax, 1e-10) / 448 in fp32, and
q = e4m3(x / s) with an IEEE fp32 division.

Each test computes its expectation another way than the oracle does (numpy
reductions and fp32 division, torch's e4m3 cast, closed-form invariants), so
that a dropped term, a transposed block index or a wrong rounding fails here.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

EPS = np.float32(1e-10)


def _f32(bits):
    return wl.bf16_bits_to_f32(bits)


def _expected_act(bits):
    """numpy amax per 1x128 group + numpy fp32 division + torch e4m3 cast."""
    x = _f32(bits)
    M, K = x.shape
    g = x.reshape(M, K // 128, 128)
    amax = np.abs(g).max(axis=2)
    s = (np.maximum(amax, EPS) / np.float32(448.0)).astype(np.float32)
    t = (g / s[:, :, None]).astype(np.float32)          # IEEE fp32 division
    assert np.all(np.abs(t) < 464.0)                    # torch cast is RNE there
    q = torch.from_numpy(t.reshape(M, K).copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return q, s


@pytest.mark.parametrize("shape,seed", [((32, 512), 0), ((7, 384), 3), ((1, 128), 4)])
def test_quant_act_vs_library_composition(shape, seed):
    bits = wl.normal(shape, 1.0, seed)
    q, s = oracle.quant_act(bits)
    qe, se = _expected_act(bits)
    assert np.array_equal(s, se)
    assert np.array_equal(q, qe)


def test_quant_act_heavy_tails_and_zero_groups():
    bits = wl.sweep_x(16, 1024)
    bits[3, 128:256] = 0
    bits[5, 0:128] = 0x8000                           # a group of -0.0
    q, s = oracle.quant_act(bits)
    qe, se = _expected_act(bits)
    assert np.array_equal(s, se) and np.array_equal(q, qe)
    assert s[3, 1] == np.float32(EPS) / np.float32(448.0)
    assert np.all(q[3, 128:256] == 0x00)
    assert np.all(q[5, 0:128] == 0x80)


def test_amax_element_maps_to_448():
    bits = wl.normal((64, 1024), 3.0, 11)
    x = _f32(bits).reshape(64, 8, 128)
    q, _ = oracle.quant_act(bits)
    q = q.reshape(64, 8, 128)
    idx = np.abs(x).argmax(axis=2)
    top = np.take_along_axis(q, idx[:, :, None], axis=2)[:, :, 0]
    sign = np.take_along_axis(x, idx[:, :, None], axis=2)[:, :, 0] < 0
    assert np.all(top == np.where(sign, 0xFE, 0x7E))


def test_round_trip_bound():
    """|x - dec(q) s| <= 2^-4 |x| (1 + 2^-19) + 2^-10 s  (3 mantissa bits,
    fp32 quotient rounding, subnormal spacing 2^-9)."""
    bits = wl.student_t_outliers(64, 1024, 3.0, 0.01, 100.0)
    x = _f32(bits).astype(np.float64)
    q, s = oracle.quant_act(bits)
    dec = oracle.e4m3_decode_table()[q]
    sx = np.repeat(s.astype(np.float64), 128, axis=1)
    err = np.abs(x - dec * sx)
    assert np.all(err <= 2.0 ** -4 * np.abs(x) * (1 + 2.0 ** -19) + 2.0 ** -10 * sx)


@pytest.mark.parametrize("k", [-12, -3, -1, 1, 5, 20])
def test_power_of_two_equivariance(k):
    bits = wl.normal((8, 512), 1.0, 5)
    x = _f32(bits)
    x2 = (x * np.float32(2.0 ** k)).astype(np.float32)   # exact: stays normal
    bits2 = wl.f32_to_bf16_bits(x2)
    assert np.array_equal(_f32(bits2), x2)
    q1, s1 = oracle.quant_act(bits)
    q2, s2 = oracle.quant_act(bits2)
    assert np.array_equal(q1, q2)
    assert np.array_equal(s2, (s1 * np.float32(2.0 ** k)).astype(np.float32))


def test_row_permutation():
    bits = wl.normal((16, 256), 1.0, 6)
    perm = np.random.default_rng(0).permutation(16)
    q, s = oracle.quant_act(bits)
    qp, sp = oracle.quant_act(bits[perm])
    assert np.array_equal(qp, q[perm]) and np.array_equal(sp, s[perm])


def test_quant_act_rows_matches_full():
    bits = wl.normal((9, 256), 1.0, 7)
    q, s = oracle.quant_act(bits, nthreads=3)
    q2, s2 = oracle.quant_act_rows(bits, 2, 7)
    assert np.array_equal(q[2:7], q2) and np.array_equal(s[2:7], s2)


# ------------------------------------------------------------- weight quant

def _expected_weight(bits):
    w = _f32(bits)
    N, K = w.shape
    b = w.reshape(N // 128, 128, K // 128, 128)
    amax = np.abs(b).max(axis=(1, 3))
    s = (np.maximum(amax, EPS) / np.float32(448.0)).astype(np.float32)
    t = (b / s[:, None, :, None]).astype(np.float32).reshape(N, K)
    q = torch.from_numpy(t.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return q, s


def test_quant_weight_vs_library_composition():
    bits = wl.normal((256, 384), 0.02, 1)
    bits = wl.zero_blocks(bits, 0.2)
    # give each block a different scale so a transposed block index fails
    w = _f32(bits).reshape(2, 128, 3, 128) * np.array([1, 3, 7, 20, 50, 0.1], np.float32).reshape(2, 1, 3, 1)
    bits = wl.f32_to_bf16_bits(w.reshape(256, 384))
    q, s = oracle.quant_weight(bits)
    qe, se = _expected_weight(bits)
    assert s.shape == (2, 3)
    assert np.array_equal(s, se) and np.array_equal(q, qe)


def test_quant_weight_equals_act_when_rows_share_amax():
    """If every 1x128 row-group of a 128x128 block has the block's amax, the
    block scale equals each group's scale, so weight quant == act quant."""
    bits = wl.normal((256, 256), 0.02, 9)
    w = _f32(bits).copy()
    for i in range(2):
        for j in range(2):
            blk = w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            m = np.float32(0.5 + i + 2 * j)
            blk[:, 5] = m
    bits = wl.f32_to_bf16_bits(w)
    qw, sw = oracle.quant_weight(bits)
    qa, sa = oracle.quant_act(bits)
    assert np.array_equal(qw, qa)
    assert np.array_equal(np.repeat(np.repeat(sw, 128, axis=0), 1, axis=1), sa)


def test_quant_weight_zero_block():
    bits = wl.normal((128, 256), 0.02, 2)
    bits[:, 128:] = 0
    q, s = oracle.quant_weight(bits)
    assert s[0, 1] == np.float32(EPS) / np.float32(448.0)
    assert np.all(q[:, 128:] == 0)
