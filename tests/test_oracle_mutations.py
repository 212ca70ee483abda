"""Planted mistakes in copies of the oracle must fail the pins.

Each case compiles a mutated copy of oracle/fp8bl_oracle.c into a temporary
library, swaps it in for the real one, and checks that at least one pin of
the relevant kind fails.  This shows the pins are sensitive to the plausible
errors they are meant to catch (a dropped term, a transposed index, the
reciprocal instead of the division, a wrong rounding).  The grouped (MoE)
oracle is a Python composition, so its mutants are planted in a copy of that
Python function instead.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
import workloads as wl
from tests import test_oracle_gemm as tg
from tests import test_oracle_quant as tq
from tests import test_oracle_rowwise as trw
from tests import test_oracle_static as tst
from tests import test_oracle_ue8m0 as tu

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "fp8bl_oracle.c")


def _build_mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert old in src, old
    p = tmp_path / "mutant.c"
    p.write_text(src.replace(old, new, 1))
    so = str(tmp_path / "libmutant.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
                    "-fPIC", "-shared", "-pthread", str(p), "-o", so, "-lm"], check=True)
    return oracle.bind(so)


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


QUANT_MUTANTS = [
    # multiply by the reciprocal instead of dividing
    ("oracle_e4m3_encode(bf16_to_f32(xg[i]) / sc)", "oracle_e4m3_encode(bf16_to_f32(xg[i]) * (1.0f / sc))"),
    # amax taken without the absolute value
    ("float a = fabsf(bf16_to_f32(xg[i]));", "float a = bf16_to_f32(xg[i]);"),
    # scale off by the e4m3 max (uses 240, the e4m3fnuz max)
    ("#define OR_E4M3_MAX 448.0f", "#define OR_E4M3_MAX 240.0f"),
    # amax window misplaced (stride 64 instead of 128, stays in bounds)
    ("const uint16_t *xg = x + m * K + g * OR_BLOCK;", "const uint16_t *xg = x + m * K + g * 64;"),
]


@pytest.mark.parametrize("old,new", QUANT_MUTANTS)
def test_quant_pins_catch(tmp_path, monkeypatch, old, new):
    lib = _build_mutant(tmp_path, old, new)
    monkeypatch.setattr(oracle, "_lib", lib)
    checks = [
        lambda: tq.test_quant_act_vs_library_composition((32, 512), 0),
        lambda: tq.test_quant_act_heavy_tails_and_zero_groups(),
        lambda: tq.test_amax_element_maps_to_448(),
    ]
    assert any(_fails(c) for c in checks)


GEMM_MUTANTS = [
    # transposed weight-scale index
    ("(double)jb->sw[(n / OR_BLOCK) * KB + j]", "(double)jb->sw[j * (N / OR_BLOCK) + (n / OR_BLOCK) % KB]"),
    # activation scale of the wrong K block
    ("(double)jb->sa[m * KB + j]", "(double)jb->sa[m * KB]"),
    # dropped last K block
    ("for (int64_t j = 0; j < KB; ++j) {", "for (int64_t j = 0; j + 1 < KB; ++j) {"),
    # off-by-one K range inside a block
    ("k < (j + 1) * OR_BLOCK; ++k)", "k < (j + 1) * OR_BLOCK - 1; ++k)"),
]


@pytest.mark.parametrize("old,new", GEMM_MUTANTS)
def test_gemm_pins_catch(tmp_path, monkeypatch, old, new):
    lib = _build_mutant(tmp_path, old, new)
    monkeypatch.setattr(oracle, "_lib", lib)
    checks = [
        lambda: tg.test_gemm_vs_exact_rationals(256),
        lambda: tg.test_unit_scales_reduce_to_integer_matmul(),
        lambda: tg.test_block_sums_exact_per_block(),
        lambda: tg.test_scale_linearity_and_block_index(),
    ]
    assert any(_fails(c) for c in checks)


def test_real_oracle_passes_same_checks():
    tq.test_quant_act_vs_library_composition((32, 512), 0)
    tg.test_gemm_vs_exact_rationals(256)
    assert np.all(np.isfinite(oracle.block_linear(*tg._random_case(2, 128, 128, 0))))
    assert wl.tiny()[0].shape == (32, 512)


UE8M0_MUTANTS = [
    # rounds the exponent down at exact powers of two (<= instead of <)
    ("while (ldexp(448.0, e) < a)", "while (ldexp(448.0, e) <= a)"),
    # floor instead of ceil: the largest element may exceed 448
    ("while (ldexp(448.0, e - 1) >= a)\n        --e;\n    while (ldexp(448.0, e) < a)\n        ++e;",
     "e = (int)floor(log2(a / 448.0));"),
    # bias 128 instead of 127 when storing
    ("return (uint8_t)(e + 127);", "return (uint8_t)(e + 128);"),
    # multiplies by 2^e instead of 2^-e
    ("double v = (double)x * ldexp(1.0, 127 - (int)c);", "double v = (double)x * ldexp(1.0, (int)c - 127);"),
    # decode without the bias
    ("return ldexp(1.0, (int)c - 127);", "return ldexp(1.0, (int)c - 126);"),
]


@pytest.mark.parametrize("old,new", UE8M0_MUTANTS)
def test_ue8m0_pins_catch(tmp_path, monkeypatch, old, new):
    lib = _build_mutant(tmp_path, old, new)
    monkeypatch.setattr(oracle, "_lib", lib)
    checks = [
        tu.test_decode_all_codes_vs_torch,
        lambda: tu.test_scale_code_at_binade_edges(3),
        tu.test_scale_code_vs_frexp_random,
        tu.test_act_vs_library_composition,
        tu.test_weight_vs_library_composition,
    ]
    assert any(_fails(c) for c in checks)


ROWWISE_MUTANTS = [
    # amax over the first 128 elements only (the block rule leaking in)
    ("        for (int64_t k = 0; k < K; ++k) {\n            float a = fabsf(bf16_to_f32(xr[k]));",
     "        for (int64_t k = 0; k < (K < 128 ? K : 128); ++k) {\n            float a = fabsf(bf16_to_f32(xr[k]));"),
    # weight scale of the wrong index (the activation row's)
    ("y[r * N + n] = (double)sa[m] * (double)sw[n] * b;", "y[r * N + n] = (double)sa[m] * (double)sw[m % N] * b;"),
    # dropped last k term
    ("            for (int64_t k = 0; k < K; ++k)\n                b += arow[k] * dec[wr[k]];",
     "            for (int64_t k = 0; k + 1 < K; ++k)\n                b += arow[k] * dec[wr[k]];"),
]


@pytest.mark.parametrize("old,new", ROWWISE_MUTANTS)
def test_rowwise_pins_catch(tmp_path, monkeypatch, old, new):
    lib = _build_mutant(tmp_path, old, new)
    monkeypatch.setattr(oracle, "_lib", lib)
    checks = [
        lambda: trw.test_quant_vs_library_composition(5, 4096, 1),
        trw.test_row_max_maps_to_448,
        trw.test_linear_vs_exact_rationals,
        trw.test_unit_scales_reduce_to_integer_matmul,
        trw.test_scale_index_per_row_and_column,
    ]
    assert any(_fails(c) for c in checks)


STATIC_MUTANTS = [
    # multiplies by the scale instead of dividing
    ("q[i] = oracle_e4m3_encode(bf16_to_f32(x[i]) / s);", "q[i] = oracle_e4m3_encode(bf16_to_f32(x[i]) * s);"),
    # scale grid not filled with the given scale
    ("        sa[i] = s;", "        sa[i] = 1.0f;"),
]


@pytest.mark.parametrize("old,new", STATIC_MUTANTS)
def test_static_pins_catch(tmp_path, monkeypatch, old, new):
    lib = _build_mutant(tmp_path, old, new)
    monkeypatch.setattr(oracle, "_lib", lib)
    checks = [lambda: tst.test_vs_library_composition(0.01), tst.test_saturates_above_448_s,
              tst.test_equals_dynamic_when_s_is_every_groups_scale]
    assert any(_fails(c) for c in checks)


GROUPED_MUTANTS = [
    # segment end taken as inclusive
    ("(want < off[e + 1])", "(want <= off[e + 1])"),
    # segment start taken as exclusive
    ("(want >= off[e])", "(want > off[e])"),
    # the next expert's weights and scales
    ("q_w[e], c_w[e]", "q_w[min(e + 1, E - 1)], c_w[min(e + 1, E - 1)]"),
    # expert 0's weight scales for every expert
    ("q_w[e], c_w[e]", "q_w[e], c_w[0]"),
    # offsets no longer validated
    ('raise ValueError("offsets must be non-decreasing within [0, M]")', "pass"),
]


@pytest.mark.parametrize("old,new", GROUPED_MUTANTS)
def test_grouped_pins_catch(monkeypatch, old, new):
    """The grouped oracle is a Python composition of the pinned UE8M0 block
    linear, so its mutants are planted in a copy of that Python function."""
    import inspect
    from tests import test_oracle_grouped as tgr
    src = inspect.getsource(oracle.grouped_linear_ue8m0)
    assert old in src, old
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new, 1), "<grouped mutant>", "exec"), ns)
    monkeypatch.setattr(oracle, "grouped_linear_ue8m0", ns["grouped_linear_ue8m0"])
    checks = [tgr.test_vs_exact_rationals_with_an_empty_expert, tgr.test_one_expert_is_the_block_linear,
              tgr.test_rows_depend_only_on_their_expert, tgr.test_rows_outside_the_segments_are_not_produced,
              tgr.test_bad_offsets_raise, tgr.test_row_subset_matches_full]

    def fails(fn):
        try:
            fn()
        except (Exception, pytest.fail.Exception):   # a failed assertion, pytest.raises, or a crash
            return True
        return False
    assert any(fails(c) for c in checks)


def test_real_grouped_oracle_passes_the_same_checks():
    from tests import test_oracle_grouped as tgr
    for c in (tgr.test_vs_exact_rationals_with_an_empty_expert, tgr.test_one_expert_is_the_block_linear,
              tgr.test_rows_depend_only_on_their_expert, tgr.test_rows_outside_the_segments_are_not_produced,
              tgr.test_bad_offsets_raise, tgr.test_row_subset_matches_full):
        c()
