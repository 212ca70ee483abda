"""GPU parity of the block-scaled FP8 GEMM against the oracle's fp64 result,
through the C ABI.

Definition ("Fine-grained FP8" page of the transformers docs): both scale
sets applied per 128-deep K block.  Quantized operands come from the GPU
quantizers, which the quant tests hold bit-exact to the oracle; the oracle
then computes R from the same codes and scales, and the GPU output must meet
the tolerance in tests/parity.py.  Small shapes compare every element; the
full workload sizes compare sampled rows (all N columns) in the launch
configuration the benchmark uses.
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


def _run(fp8, xbits, wbits, rows=None):
    x, w = to_dev(xbits), to_dev(wbits)
    q_a, s_a = fp8.quant_act(x)
    q_w, s_w = fp8.quant_weight(w)
    y = fp8.block_linear(q_a, s_a, q_w, s_w)
    fp8.check()
    qa, sa, qw, sw = u8(q_a), f32(s_a), u8(q_w), f32(s_w)
    R = oracle.block_linear(qa, sa, qw, sw, rows=rows, nthreads=8)
    yv = f32(y) if rows is None else f32(y[torch.as_tensor(rows, device=y.device)])
    return yv, R, (x, q_a, s_a, q_w, s_w, y)


def test_tiny(fp8):
    xb, wb = wl.tiny()
    y, R, _ = _run(fp8, xb, wb)
    check_gemm(y, R, "tiny")


@pytest.mark.parametrize("M,N,K", [
    (1, 128, 128), (5, 384, 256), (127, 256, 384), (129, 640, 1024), (300, 512, 512),
    (64, 1024, 4096), (257, 768, 2048),
])
def test_ragged_shapes(fp8, M, N, K):
    xb = wl.normal((M, K), 1.0, 0, M + N + K)
    wb = wl.normal((N, K), 0.02, 1, M + N + K)
    y, R, _ = _run(fp8, xb, wb)
    check_gemm(y, R, f"{M}x{N}x{K}")


def test_scale_extremes(fp8):
    """Per-token magnitudes spanning 1e-4..1e4 and zeroed weight blocks."""
    M, N, K = 192, 512, 1024
    g = np.random.default_rng(5)
    x = g.standard_normal((M, K)).astype(np.float32) * np.exp(g.uniform(-9, 9, (M, 1))).astype(np.float32)
    xb = wl.f32_to_bf16_bits(x)
    xb[7, 256:384] = 0
    wb = wl.zero_blocks(wl.normal((N, K), 0.02, 2), 0.2)
    y, R, _ = _run(fp8, xb, wb)
    check_gemm(y, R, "extremes")


def test_deterministic(fp8):
    xb = wl.normal((200, 1024), 1.0, 3)
    wb = wl.normal((768, 1024), 0.02, 4)
    _, _, (x, q_a, s_a, q_w, s_w, y) = _run(fp8, xb, wb)
    y2 = fp8.block_linear(q_a, s_a, q_w, s_w)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def _sample_rows(M, n=48, seed=0):
    g = np.random.default_rng(seed)
    r = set([0, 1, M - 1, M // 2]) | set(g.choice(M, n, replace=False).tolist())
    return np.array(sorted(r), dtype=np.int64)


@pytest.mark.parametrize("which", ["llama3_prefill_gate_up", "llama3_prefill_down"])
def test_full_size_prefill(fp8, which):
    xb, wb = wl.llama3_prefill(which.split("prefill_")[1])
    rows = _sample_rows(xb.shape[0], 24)
    y, R, _ = _run(fp8, xb, wb, rows=rows)
    check_gemm(y, R, which)


@pytest.mark.parametrize("name", ["qo", "kv", "gate_up", "down"])
@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_full_size_decode(fp8, name, M):
    xb, wb = wl.llama3_decode(M, name)
    y, R, _ = _run(fp8, xb, wb)
    check_gemm(y, R, f"decode {name} M={M}")


def test_full_size_deepseek_up(fp8):
    xb, wb = wl.deepseek_mlp("up")
    rows = _sample_rows(xb.shape[0], 12)
    y, R, _ = _run(fp8, xb, wb, rows=rows)
    check_gemm(y, R, "deepseek up")


def test_fused_bit_identical(fp8):
    for (M, N, K) in [(32, 256, 512), (129, 640, 1024), (1, 1024, 4096)]:
        xb = wl.sweep_x(M, K)
        wb = wl.normal((N, K), 0.02, 1)
        x, w = to_dev(xb), to_dev(wb)
        q_w, s_w = fp8.quant_weight(w)
        q_a, s_a = fp8.quant_act(x)
        y1 = fp8.block_linear(q_a, s_a, q_w, s_w)
        y2 = fp8.block_linear_fused(x, q_w, s_w)
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), (M, N, K)
        if M > 64:
            y3 = fp8.block_linear_fused(x, q_w, s_w, in_kernel=True)
            torch.cuda.synchronize()
            assert torch.equal(y1.view(torch.int16), y3.view(torch.int16)), (M, N, K)


def test_no_timeout_recorded(fp8):
    fp8.check()


@pytest.mark.parametrize("M", [1, 2, 15, 16, 17, 33, 48, 63, 64])
def test_decode_token_counts(fp8, M):
    """Every padded-token bucket of the decode schedule (16/32/48/64) with
    ragged counts; K spans 24 chunks so stream-K ranges cross blocks."""
    N, K = 1024, 3072
    xb = wl.normal((M, K), 1.0, 0, 100 + M)
    wb = wl.zero_blocks(wl.normal((N, K), 0.02, 1, 100 + M), 0.05)
    y, R, _ = _run(fp8, xb, wb)
    check_gemm(y, R, f"decode M={M}")


def test_decode_deterministic_and_small_shapes(fp8):
    for (M, N, K) in [(3, 128, 128), (8, 256, 384), (64, 384, 1280)]:
        xb = wl.normal((M, K), 1.0, 0, M + K)
        wb = wl.normal((N, K), 0.02, 1, M + K)
        y, R, (x, q_a, s_a, q_w, s_w, _) = _run(fp8, xb, wb)
        check_gemm(y, R, f"decode {M}x{N}x{K}")
        y2 = fp8.block_linear(q_a, s_a, q_w, s_w)
        y3 = fp8.block_linear(q_a, s_a, q_w, s_w)
        torch.cuda.synchronize()
        assert torch.equal(y2.view(torch.int16), y3.view(torch.int16))


def test_decode_workspace_too_small(fp8):
    M, N, K = 8, 512, 1024
    need = fp8.workspace_bytes(M, N, K)
    assert need > 0
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((N, K), dtype=torch.bfloat16, device="cuda")
    q_a, s_a = fp8.quant_act(x)
    q_w, s_w = fp8.quant_weight(w)
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fp8.Fp8blError) as ei:
        fp8.block_linear(q_a, s_a, q_w, s_w, workspace=small)
    assert ei.value.status == 7


@pytest.mark.parametrize("M", [512, 1024, 2048, 4096, 8192, 16384])
def test_full_size_sweep_unfused_and_fused(fp8, M):
    """Sweep workload: X [M, 7168] Student-t(3) with outlier channels and
    zeroed groups against W [2048, 7168]; the fused entry point must equal the
    unfused one bit for bit, and both meet the tolerance on sampled rows."""
    xb = wl.sweep_x(M)
    wb = wl.sweep_w()
    rows = _sample_rows(M, 16, seed=M)
    y, R, (x, q_a, s_a, q_w, s_w, y_full) = _run(fp8, xb, wb, rows=rows)
    check_gemm(y, R, f"sweep M={M}")
    for in_kernel in (False, True):
        y_fused = fp8.block_linear_fused(x, q_w, s_w, in_kernel=in_kernel)
        torch.cuda.synchronize()
        assert torch.equal(y_full.view(torch.int16), y_fused.view(torch.int16)), in_kernel


def test_full_size_deepseek_down(fp8):
    xb, wb = wl.deepseek_mlp("down")          # X [8192, 18432], W [7168, 18432]
    rows = _sample_rows(xb.shape[0], 8, seed=3)
    y, R, _ = _run(fp8, xb, wb, rows=rows)
    check_gemm(y, R, "deepseek down")


def test_fused_prefill_size_bit_identical(fp8):
    xb, wb = wl.llama3_prefill("down")        # X [4096, 14336], W [4096, 14336]
    x, w = to_dev(xb), to_dev(wb)
    q_w, s_w = fp8.quant_weight(w)
    q_a, s_a = fp8.quant_act(x)
    y1 = fp8.block_linear(q_a, s_a, q_w, s_w)
    for in_kernel in (False, True):
        y2 = fp8.block_linear_fused(x, q_w, s_w, in_kernel=in_kernel)
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), in_kernel


@pytest.mark.parametrize("M,N,K", [(8192, 2048, 1024), (4096, 4096, 2048), (640, 1280, 1152)])
def test_fused_repeated_runs_bit_identical(fp8, M, N, K):
    """The fused kernel at sizes where each CTA cluster processes several
    (row band, group of N-tiles) units -- with a partly empty last group
    (N = 1280) and an odd chunk count (K = 1152) -- run ten times: Y must
    equal the unfused result every time.  A hand-off race between the fused
    kernel's warps or CTAs shows up as an intermittent mismatch."""
    xb = wl.sweep_x(M, K)
    wb = wl.normal((N, K), 0.02, 1, M + N + K)
    x, w = to_dev(xb), to_dev(wb)
    q_w, s_w = fp8.quant_weight(w)
    q_a, s_a = fp8.quant_act(x)
    y1 = fp8.block_linear(q_a, s_a, q_w, s_w)
    y2 = torch.empty_like(y1)
    for rep in range(10):
        y2.fill_(0)
        fp8.block_linear_fused(x, q_w, s_w, y2, in_kernel=True)
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), (M, N, K, rep)
    fp8.check()


def test_decode_workspace_needs_no_clearing(fp8):
    """The decode schedule's hand-over flags count as set only when they hold
    the launch's own tag, so a workspace holding leftover bytes -- all ones,
    random bytes, or another shape's leftovers -- gives the same Y, bit for
    bit, as a fresh one, and calls that reuse one workspace across shapes
    stay exact."""
    shapes = [(1, 4096, 4096), (64, 1024, 4096), (17, 2048, 3072)]
    runs = []
    size = 0
    for M, N, K in shapes:
        xb = wl.normal((M, K), 1.0, 0, 7 + M)
        wb = wl.normal((N, K), 0.02, 1, 7 + M)
        x, w = to_dev(xb), to_dev(wb)
        q_a, s_a = fp8.quant_act(x)
        q_w, s_w = fp8.quant_weight(w)
        size = max(size, fp8.workspace_bytes(M, N, K))
        runs.append((q_a, s_a, q_w, s_w, M, N, K))
    shared = torch.empty(size, dtype=torch.uint8, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(11)
    for q_a, s_a, q_w, s_w, M, N, K in runs:
        ref = fp8.block_linear(q_a, s_a, q_w, s_w)
        R = oracle.block_linear(u8(q_a), f32(s_a), u8(q_w), f32(s_w), nthreads=8)
        check_gemm(f32(ref), R, f"decode {M}x{N}x{K}")
        for fill in ("ones", "random", "reuse", "reuse"):
            if fill == "ones":
                shared.fill_(255)
            elif fill == "random":
                shared.random_(0, 256, generator=g)
            y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            fp8.block_linear(q_a, s_a, q_w, s_w, y, shared[:fp8.workspace_bytes(M, N, K)])
            torch.cuda.synchronize()
            assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), (M, N, K, fill)
    fp8.check()


def test_decode_graph_replay_bit_identical(fp8):
    """A CUDA graph replays its decode launches with the arguments they were
    captured with (tags included); every completed launch leaves the flags
    it used cleared, so replays give the eager result bit for bit.  The graph holds the
    activation quantizer and the decode linear back to back (both launched
    with programmatic serialization), for two shapes on one workspace."""
    items = []
    size = 0
    for M, N, K in [(8, 4096, 4096), (64, 28672, 4096)]:
        x = to_dev(wl.normal((M, K), 1.0, 0, 21 + M))
        w = to_dev(wl.normal((N, K), 0.02, 1, 21 + M))
        q_w, s_w = fp8.quant_weight(w)
        q_a, s_a = fp8.quant_act(x)
        ref = fp8.block_linear(q_a, s_a, q_w, s_w)
        size = max(size, fp8.workspace_bytes(M, N, K))
        items.append(dict(x=x, q_w=q_w, s_w=s_w, q_a=torch.empty_like(q_a), s_a=torch.empty_like(s_a),
                          y=torch.empty_like(ref), ref=ref, M=M, N=N, K=K))
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")

    def step():
        for it in items:
            fp8.quant_act(it["x"], it["q_a"], it["s_a"])
            fp8.block_linear(it["q_a"], it["s_a"], it["q_w"], it["s_w"], it["y"],
                             ws[:fp8.workspace_bytes(it["M"], it["N"], it["K"])])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for rep in range(4):
        for it in items:
            it["y"].fill_(0)
        graph.replay()
        torch.cuda.synchronize()
        for it in items:
            assert torch.equal(it["y"].view(torch.int16), it["ref"].view(torch.int16)), (it["M"], rep)
    del graph
    fp8.check()


@pytest.mark.parametrize("M,N,K", [(7000, 640, 256), (4096, 4096, 512), (150, 2048, 384)])
def test_split_tail_wave(fp8, M, N, K):
    """Shapes whose last wave of 128x256 tiles is run as 128-column halves:
    7000x640 has 55x3 = 165 tiles on 148 CTAs (17 split, some of them in the
    partial last N tile), 4096x4096 has 512 (68 split), 150x2048 has 16 (all
    split).  Sampled rows against the oracle, and the in-GEMM quantization
    schedule (full tiles only) equal bit for bit: the split items must keep
    every element's K order and products."""
    xb = wl.sweep_x(M, K)
    wb = wl.normal((N, K), 0.02, 1, M + N + K)
    rows = _sample_rows(M, 24, seed=M + N)
    y, R, (x, q_a, s_a, q_w, s_w, y_full) = _run(fp8, xb, wb, rows=rows)
    check_gemm(y, R, f"split tail {M}x{N}x{K}")
    y_fused = fp8.block_linear_fused(x, q_w, s_w, in_kernel=True)
    torch.cuda.synchronize()
    assert torch.equal(y_full.view(torch.int16), y_fused.view(torch.int16))
