"""GPU parity of the grouped (MoE expert) UE8M0 linear against the oracle,
through the C ABI.

Method: "Fine-grained FP8" page ("DeepGEMM fast path": MoE expert matmuls;
"UE8M0 scale format": Blackwell expert kernels take UE8M0 scales), read as a
contiguous grouping of rows by expert.  Segment sizes cover empty experts,
segments shorter than a 128-row tile, and segments that end inside a tile;
malformed offsets are clamped by the kernel, and the test checks the clamped
meaning.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.parity import check_gemm, f32, to_dev, u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fine_grained_block_token_b200 as m
    return m


def _segments(g, M, E, p_empty=0.2):
    """Random non-negative counts summing to M, some experts empty."""
    w = g.exponential(1.0, E) * (g.random(E) > p_empty)
    if w.sum() == 0:
        w[0] = 1.0
    c = np.floor(w / w.sum() * M).astype(np.int64)
    c[np.argmax(w)] += M - c.sum()
    return np.concatenate([[0], np.cumsum(c)]).astype(np.int32)


def _quantized(fp8, M, N, K, E, seed):
    xb = wl.normal((M, K), 1.0, seed)
    wb = wl.normal((E * N, K), 0.02, seed + 1)
    q_a, s_a = fp8.quant_act_ue8m0(to_dev(xb))
    q_w, s_w = fp8.quant_weight_ue8m0(to_dev(wb))
    return q_a, s_a, q_w.view(E, N, K), s_w.view(E, N // 128, K // 128)


def _check(fp8, q_a, s_a, q_w, s_w, off, rows=None, label="", pairs=True):
    M = q_a.shape[0]
    y = torch.full((M, q_w.shape[1]), 7.0, dtype=torch.bfloat16, device="cuda")
    fp8.grouped_linear_ue8m0(q_a, s_a, q_w, s_w, torch.from_numpy(off).cuda(), y, pairs=pairs)
    fp8.check()
    R = oracle.grouped_linear_ue8m0(u8(q_a), u8(s_a), u8(q_w), u8(s_w), off, rows=rows, nthreads=8)
    covered = np.zeros(M, bool)
    covered[off[0]:off[-1]] = True
    Y = f32(y)
    assert np.all(Y[~covered] == 7.0), label + ": rows outside the segments were written"
    idx = np.nonzero(covered)[0] if rows is None else np.intersect1d(rows, np.nonzero(covered)[0])
    check_gemm(Y[idx], R[idx], label)


@pytest.mark.parametrize("pairs", [True, False])
@pytest.mark.parametrize("M,N,K,E,seed", [
    (300, 256, 256, 3, 0), (1000, 384, 512, 8, 1), (77, 256, 384, 5, 2), (2048, 512, 1024, 64, 3),
    (129, 128, 128, 1, 4),
])
def test_random_segments(fp8, M, N, K, E, seed, pairs):
    g = np.random.default_rng(seed)
    q_a, s_a, q_w, s_w = _quantized(fp8, M, N, K, E, 10 * seed)
    _check(fp8, q_a, s_a, q_w, s_w, _segments(g, M, E), label=f"{M}x{N}x{K} E={E} pairs={pairs}",
           pairs=pairs)


@pytest.mark.parametrize("M,N,K,E,seed", [
    (300, 256, 256, 3, 0), (1000, 384, 512, 8, 1), (2048, 512, 1024, 64, 3), (513, 256, 768, 16, 5),
    (4100, 1280, 640, 7, 6),
])
def test_pairs_equal_single_cta(fp8, M, N, K, E, seed):
    """The CTA-pair schedule (fp8_grouped_linear_ue8m0_ws, 256-row tiles in
    each expert's segment, scale factors packed per expert) runs the same
    block-scaled MMAs in the same K order as the single-CTA kernel: every
    output equal bit for bit, rows outside the segments untouched by both.
    Random codes with scale codes spread over 2^+-20, so that a factor taken
    from the wrong expert, row or K block shows."""
    g = np.random.default_rng(100 + seed)
    qa = g.integers(0, 256, (M, K), dtype=np.uint8)
    qw = g.integers(0, 256, (E * N, K), dtype=np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x00
    qw[(qw & 0x7F) == 0x7F] = 0x00
    ca = g.integers(107, 148, (M, K // 128), dtype=np.uint8)
    cw = g.integers(107, 148, (E * N // 128, K // 128), dtype=np.uint8)
    dev = lambda a: torch.from_numpy(a).cuda()
    q_a, s_a = dev(qa).view(torch.float8_e4m3fn), dev(ca).view(torch.float8_e8m0fnu)
    q_w = dev(qw).view(torch.float8_e4m3fn).view(E, N, K)
    s_w = dev(cw).view(torch.float8_e8m0fnu).view(E, N // 128, K // 128)
    off = _segments(g, M, E)
    off[0], off[-1] = min(int(off[1]), 5), max(int(off[-2]), M - 3)     # a few rows left out
    offd = torch.from_numpy(off).cuda()
    assert fp8.grouped_ue8m0_workspace_bytes(M, N, K, E) > 0
    ys = [torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    fp8.grouped_linear_ue8m0(q_a, s_a, q_w, s_w, offd, ys[0])
    fp8.grouped_linear_ue8m0(q_a, s_a, q_w, s_w, offd, ys[1], pairs=False)
    fp8.check()
    assert torch.equal(ys[0].view(torch.int16), ys[1].view(torch.int16)), (M, N, K, E)
    rows = np.unique(np.concatenate([off[:-1], np.maximum(off[1:] - 1, 0), g.choice(M, 6, replace=False)]))
    rows = rows[rows < M]
    R = oracle.grouped_linear_ue8m0(qa, ca, qw.reshape(E, N, K), cw.reshape(E, N // 128, K // 128),
                                    off, rows=rows, nthreads=8)
    covered = np.zeros(M, bool)
    covered[off[0]:off[-1]] = True
    Y = f32(ys[0])
    assert np.all(Y[~covered] == 3.0)
    idx = np.intersect1d(rows, np.nonzero(covered)[0])
    check_gemm(Y[idx], R[idx], f"grouped pairs {M}x{N}x{K} E={E}")


def test_pairs_many_experts(fp8):
    """256 experts over 4100 rows, a third of them empty and many of a few
    rows (so most 256-row pair tiles are mostly padding and the packed
    activation factors need the bound of ceil(M / 256) + E groups): pairs
    equal the single-CTA kernel bit for bit, sampled rows match the oracle."""
    M, N, K, E = 4100, 256, 384, 256
    g = np.random.default_rng(77)
    q_a, s_a, q_w, s_w = _quantized(fp8, M, N, K, E, 31)
    off = _segments(g, M, E, p_empty=0.33)
    offd = torch.from_numpy(off).cuda()
    ys = [torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    fp8.grouped_linear_ue8m0(q_a, s_a, q_w, s_w, offd, ys[0])
    fp8.grouped_linear_ue8m0(q_a, s_a, q_w, s_w, offd, ys[1], pairs=False)
    fp8.check()
    assert torch.equal(ys[0].view(torch.int16), ys[1].view(torch.int16))
    rows = np.unique(np.concatenate([off[:-1], np.maximum(off[1:] - 1, 0), g.choice(M, 8, replace=False)]))
    rows = rows[rows < M]
    R = oracle.grouped_linear_ue8m0(u8(q_a), u8(s_a), u8(q_w), u8(s_w), off, rows=rows, nthreads=8)
    check_gemm(f32(ys[0])[rows], R[rows], "grouped pairs 256 experts")


def test_pairs_workspace_checks(fp8):
    """The workspace call refuses a short or missing workspace before any
    launch, and needs none at M <= 128."""
    M, N, K, E = 300, 256, 256, 3
    need = fp8.grouped_ue8m0_workspace_bytes(M, N, K, E)
    assert need > 0 and fp8.grouped_ue8m0_workspace_bytes(128, N, K, E) == 0
    q_a, s_a, q_w, s_w = _quantized(fp8, M, N, K, E, 3)
    off = torch.tensor([0, 100, 200, 300], dtype=torch.int32, device="cuda")
    with pytest.raises(fp8.Fp8blError) as ei:
        fp8.grouped_linear_ue8m0(q_a, s_a, q_w, s_w, off,
                                 workspace=torch.zeros(need - 16, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == 7
    fp8.check()


def test_segments_not_covering_all_rows(fp8):
    q_a, s_a, q_w, s_w = _quantized(fp8, 400, 256, 256, 4, 7)
    _check(fp8, q_a, s_a, q_w, s_w, np.array([37, 100, 100, 250, 333], np.int32), label="partial")


def test_single_expert_equals_plain_call(fp8):
    q_a, s_a, q_w, s_w = _quantized(fp8, 333, 384, 512, 1, 8)
    y1 = fp8.block_linear_ue8m0(q_a, s_a, q_w[0], s_w[0])
    y2 = fp8.grouped_linear_ue8m0(q_a, s_a, q_w, s_w, torch.tensor([0, 333], dtype=torch.int32,
                                                                    device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_malformed_offsets_are_clamped(fp8):
    """Out-of-range and decreasing offsets: the kernel clamps each to [0, M]
    and takes a running maximum; the result is the grouping those define."""
    M = 300
    q_a, s_a, q_w, s_w = _quantized(fp8, M, 256, 256, 5, 9)
    raw = np.array([-50, 120, 80, 400, 250, 1000], np.int32)
    clamped = np.maximum.accumulate(np.clip(raw, 0, M)).astype(np.int32)
    y = torch.full((M, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    fp8.grouped_linear_ue8m0(q_a, s_a, q_w, s_w, torch.from_numpy(raw).cuda(), y)
    fp8.check()
    R = oracle.grouped_linear_ue8m0(u8(q_a), u8(s_a), u8(q_w), u8(s_w), clamped)
    check_gemm(f32(y)[clamped[0]:clamped[-1]], R[clamped[0]:clamped[-1]], "clamped")


def test_moe_sized(fp8):
    """DeepSeek-V3-like expert MLP up-projection shape: 16 experts, K 7168,
    N 2048, 8192 routed token rows; sampled rows against the oracle."""
    g = np.random.default_rng(12)
    M, N, K, E = 8192, 2048, 7168, 16
    q_a, s_a, q_w, s_w = _quantized(fp8, M, N, K, E, 120)
    off = _segments(g, M, E, p_empty=0.1)
    rows = np.unique(np.concatenate([off[:-1], np.maximum(off[1:] - 1, 0), g.choice(M, 24, replace=False)]))
    rows = rows[rows < M]
    _check(fp8, q_a, s_a, q_w, s_w, off, rows=rows, label="moe")


def test_no_timeout_recorded(fp8):
    fp8.check()
