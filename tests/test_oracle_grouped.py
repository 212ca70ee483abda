"""Pins for the oracle's grouped (MoE expert) UE8M0 linear.

Method: "Fine-grained FP8" page, "DeepGEMM fast path" section (MoE expert
matmuls through DeepGEMM) and "UE8M0 scale format" section (Blackwell's
expert kernels take UE8M0 scales).  Reading: rows sorted by expert, expert e
owns rows [off[e], off[e+1]) and multiplies them by its own weights.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _codes(shape, g):
    c = g.integers(0, 256, shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0
    return c


def _case(g, M, N, K, E):
    qa = _codes((M, K), g)
    qw = _codes((E, N, K), g)
    ca = g.integers(110, 140, (M, K // 128), dtype=np.uint8)
    cw = g.integers(110, 140, (E, N // 128, K // 128), dtype=np.uint8)
    return qa, ca, qw, cw


def test_vs_exact_rationals_with_an_empty_expert():
    g = np.random.default_rng(1)
    M, N, K, E = 7, 128, 256, 3
    qa, ca, qw, cw = _case(g, M, N, K, E)
    off = [0, 3, 3, 7]                     # expert 1 gets no rows
    y = oracle.grouped_linear_ue8m0(qa, ca, qw, cw, off)
    dec = oracle.e4m3_decode_table()
    owner = [0, 0, 0, 2, 2, 2, 2]
    for m in range(M):
        e = owner[m]
        for n in (0, 5, 127):
            tot = Fraction(0)
            for j in range(K // 128):
                b = sum(Fraction(float(dec[qa[m, k]])) * Fraction(float(dec[qw[e, n, k]]))
                        for k in range(128 * j, 128 * (j + 1)))
                tot += b * Fraction(2) ** (int(ca[m, j]) + int(cw[e, n // 128, j]) - 254)
            assert abs(Fraction(float(y[m, n])) - tot) <= abs(tot) * Fraction(1, 2 ** 51)


def test_one_expert_is_the_block_linear():
    g = np.random.default_rng(2)
    qa, ca, qw, cw = _case(g, 9, 256, 384, 1)
    y = oracle.grouped_linear_ue8m0(qa, ca, qw, cw, [0, 9])
    assert np.array_equal(y, oracle.block_linear_ue8m0(qa, ca, qw[0], cw[0]))


def test_rows_depend_only_on_their_expert():
    g = np.random.default_rng(3)
    qa, ca, qw, cw = _case(g, 12, 128, 256, 4)
    off = [0, 2, 7, 7, 12]
    y0 = oracle.grouped_linear_ue8m0(qa, ca, qw, cw, off)
    qw2 = qw.copy()
    qw2[1] = _codes(qw2[1].shape, g)
    y1 = oracle.grouped_linear_ue8m0(qa, ca, qw2, cw, off)
    assert np.array_equal(y0[:2], y1[:2]) and np.array_equal(y0[7:], y1[7:])
    assert not np.array_equal(y0[2:7], y1[2:7])


def test_rows_outside_the_segments_are_not_produced():
    g = np.random.default_rng(4)
    qa, ca, qw, cw = _case(g, 10, 128, 128, 2)
    y = oracle.grouped_linear_ue8m0(qa, ca, qw, cw, [2, 5, 8])
    assert np.all(np.isnan(y[:2])) and np.all(np.isnan(y[8:]))
    assert np.all(np.isfinite(y[2:8]))


def test_bad_offsets_raise():
    g = np.random.default_rng(5)
    qa, ca, qw, cw = _case(g, 4, 128, 128, 2)
    for off in ([0, 3, 2], [0, 2, 5], [-1, 2, 4]):
        with pytest.raises(ValueError):
            oracle.grouped_linear_ue8m0(qa, ca, qw, cw, off)


def test_row_subset_matches_full():
    g = np.random.default_rng(6)
    qa, ca, qw, cw = _case(g, 20, 128, 256, 3)
    off = [0, 6, 6, 20]
    y = oracle.grouped_linear_ue8m0(qa, ca, qw, cw, off)
    ys = oracle.grouped_linear_ue8m0(qa, ca, qw, cw, off, rows=[1, 5, 6, 19])
    assert np.array_equal(ys[[1, 5, 6, 19]], y[[1, 5, 6, 19]])
    assert np.all(np.isnan(ys[[0, 2, 7, 18]]))
