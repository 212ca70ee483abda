"""Pins for the oracle's e4m3 decode and encode.

The format is OCP FP8 E4M3 (the 'fn' variant): the BFL (fp8r / nvfp4) page
names E4M3 and the "Fine-grained FP8" page names fp8.  Nothing here compares
the oracle with itself: decode is checked against the OCP facts file and two
independent library casts (torch, ml_dtypes); encode against an exhaustive
brute-force nearest-value search and the same library casts inside their
non-saturating range.
"""
import math
import os
import subprocess

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")


def _golden_rows():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_format.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            code, val = line.split()[:2]
            rows.append((int(code, 16), float(val)))
    return rows


@pytest.mark.parametrize("code,val", _golden_rows())
def test_decode_ocp_facts(code, val):
    got = oracle.e4m3_decode(code)
    if math.isnan(val):
        assert math.isnan(got)
    else:
        assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val)


def test_decode_all_codes_vs_torch_and_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode_table()
    t = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    m = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for ref in (t, m):
        nan = np.isnan(ref)
        assert np.array_equal(np.isnan(ours), nan)
        assert np.array_equal(ours[~nan], ref[~nan])
        assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))
    assert np.isnan(ours).sum() == 2  # 0x7F and 0xFF only


def test_decode_monotone_and_symmetric():
    tab = oracle.e4m3_decode_table()
    pos = tab[:127]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(tab[128:255], -pos)


@pytest.mark.parametrize("v,code", [
    (448.0, 0x7E), (464.0, 0x7E),           # 464 is the tie 448|480: even code wins
    (470.0, 0x7E), (1e30, 0x7E),            # saturate (torch's cast gives NaN here)
    (float("inf"), 0x7E), (float("-inf"), 0xFE),
    (-0.0, 0x80), (0.0, 0x00),
    (2.0 ** -10, 0x00),                     # half of min subnormal: tie to even 0
    (1.5 * 2.0 ** -9, 0x02),                # tie between codes 1 and 2 -> 2
    (2.5 * 2.0 ** -9, 0x02),                # tie between codes 2 and 3 -> 2
    (-1e-30, 0x80),                         # negative underflow keeps the sign
    (1.0, 0x38), (1.0625, 0x38), (1.0625001, 0x39), (1.1875, 0x3A),
])
def test_encode_special_values(v, code):
    assert oracle.e4m3_encode(v) == code


def test_encode_nan():
    assert oracle.e4m3_encode(float("nan")) & 0x7F == 0x7F


def test_encode_vs_torch_and_ml_dtypes_in_range():
    """All bf16 values and 2^20 random fp32 values with |v| < 464, where the
    library casts are plain RNE (no saturation needed)."""
    bf = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    rng = np.random.default_rng(123)
    rnd = (rng.standard_normal(1 << 20) * np.exp2(rng.integers(-14, 9, 1 << 20))).astype(np.float32)
    v = np.concatenate([bf, rnd])
    v = v[np.isfinite(v) & (np.abs(v) <= 448.0)]
    # The per-element ctypes path is slow, so go through quant_act with a unit
    # scale: a group whose amax is exactly 448 gets s = 448/448 = 1, and then
    # q = encode(x / 1) = encode(x).
    n = len(v)
    G = (n + 126) // 127
    grp = np.zeros((G, 128), dtype=np.float32)
    flat = np.zeros(G * 127, dtype=np.float32)
    flat[:n] = v
    grp[:, :127] = flat.reshape(G, 127)
    grp[:, 127] = 448.0
    # only bf16-representable values can go through quant_act; keep those
    is_bf = (grp.view(np.uint32) & 0xFFFF) == 0
    keep_rows = is_bf.all(axis=1)
    bits = (grp[keep_rows].view(np.uint32) >> 16).astype(np.uint16)
    q, s = oracle.quant_act(bits)
    assert np.all(s == 1.0)
    vals = grp[keep_rows][:, :127].ravel()
    ours = q[:, :127].ravel()
    t = torch.from_numpy(vals.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    m = vals.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, t)
    assert np.array_equal(ours, m)
    # the non-bf16 random values: per-element path on a subsample
    sub = np.concatenate([rnd[np.abs(rnd) < 464.0][:20000],
                          np.linspace(448.0, 463.9, 64, dtype=np.float32)])
    ours2 = oracle.e4m3_encode_array(sub)
    t2 = torch.from_numpy(sub.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours2, t2)


def test_encode_exhaustive_bruteforce(tmp_path):
    """All 2^32 fp32 bit patterns against a nearest-of-table brute force
    (tests/brute_e4m3.c), about 10 s on 8 cores."""
    exe = str(tmp_path / "brute_e4m3")
    subprocess.run(["gcc", "-O2", "-pthread", os.path.join(HERE, "brute_e4m3.c"),
                    "-o", exe, "-ldl", "-lm"], check=True)
    lib = oracle.build()
    r = subprocess.run([exe, lib, str(os.cpu_count() or 4)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("mismatches 0")


def test_bruteforce_catches_planted_errors(tmp_path):
    """The brute force must fail on a plausible encoder mistake: build a copy
    of the oracle with ties rounded away from zero and check the brute force
    reports mismatches (run on a slice of the bit patterns)."""
    src = open(os.path.join(os.path.dirname(HERE), "oracle", "fp8bl_oracle.c")).read()
    bad = src.replace("(frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) != 0.0))", "(frac >= 0.5)")
    assert bad != src
    p = tmp_path / "bad.c"
    p.write_text(bad)
    so = str(tmp_path / "libbad.so")
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-pthread", str(p), "-o", so, "-lm"], check=True)
    exe = str(tmp_path / "brute_e4m3")
    subprocess.run(["gcc", "-O2", "-pthread", os.path.join(HERE, "brute_e4m3.c"),
                    "-o", exe, "-ldl", "-lm"], check=True)
    # top-16-bit range 0x3F88..0x3F89 starts at 1.0625, a tie between codes
    # 0x38 and 0x39
    r = subprocess.run([exe, so, "2", "0x3F88", "0x3F89"], capture_output=True, text=True)
    assert r.returncode == 1 and not r.stdout.startswith("mismatches 0")
