"""The CUDA quantizers form a UE8M0 scale code from the correctly rounded
fp32 quotient t = RN32(max(amax, 1e-10) / 448) as (biased exponent field of
t) + (1 if t's mantissa field is non-zero), and scale the elements by the
fp32 number whose bits are (254 - code) << 23.  These tests replay that
sequence with numpy's IEEE binary32 arithmetic for every amax a bf16 input
can produce and check it against the oracle's exact definition (the least
power of two 2^e with max(amax, 1e-10) <= 448 * 2^e).  The fp32 quotient
itself is the one pinned exhaustively by test_quant_division."""
import numpy as np

import oracle
import workloads as wl


def _method_code(a):
    t = (np.maximum(a.astype(np.float32), np.float32(1e-10)) / np.float32(448.0)).astype(np.float32)
    b = t.view(np.uint32)
    return ((b >> 23) + ((b & 0x7FFFFF) != 0)).astype(np.int64)


def test_code_method_matches_definition_for_every_bf16_amax():
    bits = np.arange(0, 0x7F80, dtype=np.uint16)        # +0 .. largest finite bf16
    a = wl.bf16_bits_to_f32(bits)
    got = _method_code(a)
    ref = np.array([oracle.ue8m0_from_amax(v) for v in a], dtype=np.int64)
    assert np.array_equal(got, ref)
    assert got.min() == 85 and got.max() <= 247


def test_inverse_scale_bits_are_exact_powers_of_two():
    codes = np.arange(85, 248, dtype=np.uint32)
    inv = ((254 - codes) << 23).astype(np.uint32).view(np.float32).astype(np.float64)
    assert np.array_equal(inv, 1.0 / oracle.ue8m0_decode(codes.astype(np.uint8)))
