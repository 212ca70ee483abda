"""Pins for the oracle's block-scaled FP8 GEMM.

Definition (transformers docs, "Fine-grained FP8" page: 128 x 128 weight
blocks, per-token groups of 128 along the input channel; the block-scaled
GEMM applies both scale sets per 128-deep K block):
    y[m,n] = sum_j s_a[m,j] * s_w[n/128,j] * sum_{k in block j} a[m,k] w[n,k]

Expectations here come from exact rational arithmetic (fractions), integer
matmuls of the codes' integer values and closed-form properties, never from
the oracle's own loops.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as wl


def _int_val(code):
    """e4m3 value times 2^9, as an exact integer, from the OCP bit layout."""
    c = np.asarray(code, dtype=np.int64)
    s = np.where(c & 0x80, -1, 1)
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, m, (8 + m) << np.maximum(e - 1, 0))
    return s * mag


def _random_case(M, N, K, seed):
    rng = np.random.default_rng(seed)
    qa = rng.integers(0, 256, (M, K), dtype=np.uint8)
    qw = rng.integers(0, 256, (N, K), dtype=np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x3C            # no NaN codes
    qw[(qw & 0x7F) == 0x7F] = 0x41
    sa = (rng.random((M, K // 128)) * 2 + 1e-3).astype(np.float32)
    sw = (rng.random((N // 128, K // 128)) * 0.01 + 1e-5).astype(np.float32)
    return qa, sa, qw, sw


@pytest.mark.parametrize("K", [128, 256, 384])
def test_gemm_vs_exact_rationals(K):
    M, N = 3, 128
    qa, sa, qw, sw = _random_case(M, N, K, K)
    y = oracle.block_linear(qa, sa, qw, sw)
    ia, iw = _int_val(qa), _int_val(qw)
    cols = [0, 1, 63, 64, 127]
    for m in range(M):
        for n in cols:
            exact = Fraction(0)
            mag = Fraction(0)
            for j in range(K // 128):
                bj = sum(int(ia[m, k]) * int(iw[n, k]) for k in range(128 * j, 128 * j + 128))
                t = Fraction(float(sa[m, j])) * Fraction(float(sw[n // 128, j])) * Fraction(bj, 2 ** 18)
                exact += t
                mag += abs(t)
            # fp64 evaluation: two roundings per term and one per addition,
            # each at most 2^-53 relative to the magnitudes involved
            bound = 4 * (K // 128) * 2.0 ** -53 * float(mag)
            assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(bound), (m, n)


def test_unit_scales_reduce_to_integer_matmul():
    M, N, K = 5, 256, 512
    qa, _, qw, _ = _random_case(M, N, K, 1)
    sa = np.ones((M, K // 128), np.float32)
    sw = np.ones((N // 128, K // 128), np.float32)
    y = oracle.block_linear(qa, sa, qw, sw)
    exact = _int_val(qa) @ _int_val(qw).T            # int64, units 2^-18
    assert np.array_equal(y * 2.0 ** 18, exact.astype(np.float64))


def test_block_sums_exact_per_block():
    """With one non-zero K block at a time the fp64 result is exactly
    s_a * s_w * B_j, B_j the exact integer block sum."""
    M, N, K = 4, 128, 384
    qa, sa, qw, sw = _random_case(M, N, K, 2)
    for j in range(3):
        qw_j = np.zeros_like(qw)
        qw_j[:, 128 * j:128 * (j + 1)] = qw[:, 128 * j:128 * (j + 1)]
        y = oracle.block_linear(qa, sa, qw_j, sw)
        bj = _int_val(qa[:, 128 * j:128 * (j + 1)]) @ _int_val(qw[:, 128 * j:128 * (j + 1)]).T
        ref = (sa[:, j:j + 1].astype(np.float64) * sw[0, j].astype(np.float64)) * (bj.astype(np.float64) / 2.0 ** 18)
        assert np.array_equal(y, ref)


def test_zero_weight_blocks_contribute_zero():
    M, N, K = 3, 256, 256
    qa, sa, qw, sw = _random_case(M, N, K, 3)
    qw[128:, :] = 0
    y = oracle.block_linear(qa, sa, qw, sw)
    assert np.all(y[:, 128:] == 0.0)


def test_scale_linearity_and_block_index():
    """Doubling s_w of block (1, 0) doubles exactly the K-block-0 term of the
    columns 128..255 (catches a transposed s_w index)."""
    M, N, K = 2, 256, 256
    qa, sa, qw, sw = _random_case(M, N, K, 4)
    y = oracle.block_linear(qa, sa, qw, sw)
    sw2 = sw.copy()
    sw2[1, 0] *= 2
    y2 = oracle.block_linear(qa, sa, qw, sw2)
    b0 = _int_val(qa[:, :128]) @ _int_val(qw[128:, :128]).T / 2.0 ** 18
    term = sa[:, 0:1].astype(np.float64) * np.float64(sw[1, 0]) * b0
    assert np.allclose(y2[:, 128:] - y[:, 128:], term, rtol=1e-12, atol=1e-300)
    assert np.array_equal(y2[:, :128], y[:, :128])


def test_row_subset_matches_full():
    M, N, K = 6, 128, 256
    qa, sa, qw, sw = _random_case(M, N, K, 5)
    y = oracle.block_linear(qa, sa, qw, sw, nthreads=2)
    ys = oracle.block_linear(qa, sa, qw, sw, rows=[4, 1])
    assert np.array_equal(ys, y[[4, 1]])


def test_end_to_end_close_to_bf16_matmul():
    """Loose sanity bound: quantize-then-GEMM stays within e4m3 error of the
    plain bf16 matmul (the dequantize fallback the BFL page describes)."""
    xb, wb = wl.tiny()
    qa, sa = oracle.quant_act(xb)
    qw, sw = oracle.quant_weight(wb)
    y = oracle.block_linear(qa, sa, qw, sw)
    ref = wl.bf16_bits_to_f32(xb).astype(np.float64) @ wl.bf16_bits_to_f32(wb).astype(np.float64).T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 0.05
    # a transposed operand or dropped scale would be far off
    assert rel > 1e-4


def test_bf16_rne_view():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(200000) * np.exp2(rng.integers(-30, 30, 200000))).astype(np.float32)
    import torch
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.bf16_rne(v.astype(np.float64)), ref)


def _bf16_value(bits):
    """fp64 value of bf16 bit patterns (exact)."""
    b = np.asarray(bits, dtype=np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def test_bf16_rne_view_fp64_ties_and_near_ties():
    """fp64 inputs (the oracle's GEMM results are fp64): brute force over the
    bf16 grid around each value picks the nearest, ties to the even code.
    Cases include exact midpoints between neighbouring bf16 values and
    midpoints moved by a few fp64 ulps -- the values a detour through fp32
    would round twice (midpoint + 2^-40 relative becomes the midpoint in
    fp32, then rounds to even instead of up)."""
    rng = np.random.default_rng(7)
    lo_bits = rng.integers(0x0080, 0x7F00, 4000).astype(np.uint32)      # normal positive bf16
    lo, hi = _bf16_value(lo_bits), _bf16_value(lo_bits + 1)
    mid = (lo + hi) / 2                                                   # exact in fp64
    eps = np.abs(mid) * 2.0 ** -40
    vals = np.concatenate([mid, mid + eps, mid - eps, lo + (hi - lo) * rng.random(4000)])
    vals = np.concatenate([vals, -vals])
    got = oracle.bf16_rne(vals)
    a = np.abs(vals)
    base = (a.astype(np.float32).view(np.uint32) >> 16).astype(np.int64)  # within one code of the answer
    best = np.empty_like(a)
    for i in range(len(a)):
        cands = _bf16_value(np.arange(max(base[i] - 2, 0), base[i] + 3))
        d = np.abs(cands - a[i])
        k = np.flatnonzero(d == d.min())
        if len(k) > 1:                                                    # a tie: the even code
            codes = np.arange(max(base[i] - 2, 0), base[i] + 3)[k]
            k = k[codes % 2 == 0]
        best[i] = cands[k[0]]
    assert np.array_equal(got, np.sign(vals) * best)
    # the double-rounding trap is really exercised: fp32 first would differ
    via32 = np.asarray(oracle.bf16_rne(vals.astype(np.float32).astype(np.float64)))
    assert np.count_nonzero(via32 != got) > 1000
