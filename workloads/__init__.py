"""Seeded synthetic inputs for the fine-grained FP8 linear workloads.

This module is shared by the tests, the benchmark and the smoke check, and it
holds none of the method's arithmetic: it only draws random numbers, rounds
them to bf16 (the input dtype) and returns bf16 bit patterns (uint16) plus a
torch view on request.

Workloads (shapes as N x K for weights, M x K for activations):
  tiny           X [32, 512] ~ N(0, 1); W [256, 512] ~ N(0, 0.02); seed 0.
  llama3_decode  M in {1, 8, 32, 64}; q/o 4096x4096, k/v 1024x4096,
                 gate+up 28672x4096, down 4096x14336; X ~ N(0,1), W ~ N(0,0.02).
  llama3_prefill M = 4096; gate+up 28672x4096, down 4096x14336;
                 X ~ Student-t(df=4) with 0.5% of channels scaled by 50;
                 W ~ N(0, 0.02).
  deepseek_mlp   M = 8192; up 18432x7168, down 7168x18432;
                 X ~ N(0,1) times a per-token LogNormal(0,1) factor;
                 W ~ N(0, 0.015) with 1% of the 128x128 blocks all zero.
  sweep          X [M, 7168], M in {512, 1024, ..., 16384}, Student-t(df=3),
                 0.1% of channels scaled by 100, 1% of the 1x128 groups all
                 zero; W [2048, 7168] ~ N(0, 0.02).
  deepseek_moe   16 experts of the DeepSeek-V3 expert MLP shape: up (gate
                 and up fused) 4096x7168, down 7168x2048, stacked [E, N, K];
                 8192 routed token rows sorted by expert, segment sizes a
                 multinomial draw with Dirichlet(1) expert shares (uneven,
                 some small); X ~ N(0,1) times a per-row LogNormal(0,1);
                 W ~ N(0, 0.015), drawn on the GPU by torch's seeded
                 generator (deepseek_moe_weights).

Seeds: X draws use seed 0, W draws seed 1, the selection of outlier
channels / zeroed blocks / zeroed groups seed 2 (one generator per role, so
changing one shape does not move the others).  "N(0, s)" means standard
deviation s.  Values are drawn in fp32 (fp64 for Student-t), scaled, then
rounded to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import numpy as np

SEED_X, SEED_W, SEED_SEL = 0, 1, 2
GROUP = 128

LLAMA3_8B_LINEARS = {          # name: (N, K)
    "qo": (4096, 4096),
    "kv": (1024, 4096),
    "gate_up": (28672, 4096),
    "down": (4096, 14336),
}
DECODE_M = (1, 8, 32, 64)
PREFILL_M = 4096
DEEPSEEK_M = 8192
DEEPSEEK_LINEARS = {"up": (18432, 7168), "down": (7168, 18432)}
SWEEP_K = 7168
SWEEP_N = 2048
SWEEP_M = (512, 1024, 2048, 4096, 8192, 16384)
MOE_EXPERTS = 16
MOE_ROWS = 8192
MOE_LINEARS = {"up": (4096, 7168), "down": (7168, 2048)}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    nan = np.isnan(x)
    # u + 0x7FFF + lsb stays below 2^32 for every non-NaN pattern (at most
    # 0xFF807FFF), so 32-bit arithmetic rounds exactly; NaNs are set below.
    r = ((u + np.uint32(0x7FFF) + ((u >> 16) & np.uint32(1))) >> 16).astype(np.uint16)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, salt: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, salt])


def normal(shape, std: float, seed: int, salt: int = 0) -> np.ndarray:
    g = _rng(seed, salt)
    return f32_to_bf16_bits(g.standard_normal(shape, dtype=np.float32) * np.float32(std))


def student_t_outliers(M: int, K: int, df: float, frac: float, factor: float,
                       seed: int = SEED_X, salt: int = 0) -> np.ndarray:
    """Student-t(df) activations with round(frac*K) channels scaled by factor."""
    g = _rng(seed, salt)
    x = g.standard_t(df, size=(M, K)).astype(np.float32)
    cols = _rng(SEED_SEL, salt).choice(K, int(round(frac * K)), replace=False)
    x[:, cols] *= np.float32(factor)
    return f32_to_bf16_bits(x)


def zero_groups(xbits: np.ndarray, frac: float, salt: int = 0) -> np.ndarray:
    """Zero round(frac * #groups) of the 1x128 groups of an [M, K] array."""
    M, K = xbits.shape
    G = M * (K // GROUP)
    n = int(round(frac * G))
    sel = _rng(SEED_SEL, 1000 + salt).choice(G, n, replace=False)
    v = xbits.reshape(M * (K // GROUP), GROUP)
    v[sel] = 0
    return xbits


def zero_blocks(wbits: np.ndarray, frac: float, salt: int = 0) -> np.ndarray:
    """Zero round(frac * #blocks) of the 128x128 blocks of an [N, K] array."""
    N, K = wbits.shape
    NB, KB = N // GROUP, K // GROUP
    n = int(round(frac * NB * KB))
    sel = _rng(SEED_SEL, 2000 + salt).choice(NB * KB, n, replace=False)
    for b in sel:
        i, j = divmod(int(b), KB)
        wbits[i * GROUP:(i + 1) * GROUP, j * GROUP:(j + 1) * GROUP] = 0
    return wbits


# ---------------------------------------------------------------- workloads

def tiny():
    """X [32, 512] ~ N(0,1) and W [256, 512] ~ N(0, 0.02)."""
    return normal((32, 512), 1.0, SEED_X), normal((256, 512), 0.02, SEED_W)


def llama3_decode(M: int, name: str):
    return llama3_decode_x(M, name), llama3_decode_w(name)


def llama3_decode_x(M: int, name: str):
    """X [M, K] of one decode linear (the same draw as llama3_decode)."""
    _, K = LLAMA3_8B_LINEARS[name]
    return normal((M, K), 1.0, SEED_X, hash_name(name))


def llama3_decode_w(name: str):
    """W [N, K] of one decode linear; it does not depend on M."""
    N, K = LLAMA3_8B_LINEARS[name]
    return normal((N, K), 0.02, SEED_W, hash_name(name))


def llama3_prefill(name: str, M: int = PREFILL_M):
    N, K = LLAMA3_8B_LINEARS[name]
    salt = hash_name(name)
    x = student_t_outliers(M, K, 4.0, 0.005, 50.0, SEED_X, salt)
    return x, normal((N, K), 0.02, SEED_W, salt)


def deepseek_mlp(name: str, M: int = DEEPSEEK_M):
    N, K = DEEPSEEK_LINEARS[name]
    salt = hash_name(name)
    g = _rng(SEED_X, salt)
    x = g.standard_normal((M, K), dtype=np.float32)
    x *= g.lognormal(0.0, 1.0, size=(M, 1)).astype(np.float32)
    w = normal((N, K), 0.015, SEED_W, salt)
    return f32_to_bf16_bits(x), zero_blocks(w, 0.01, salt)


def moe_offsets(E: int = MOE_EXPERTS, M: int = MOE_ROWS) -> np.ndarray:
    """int32 [E + 1] segment starts of M routed rows over E experts."""
    g = _rng(SEED_SEL, 3001)
    counts = g.multinomial(M, g.dirichlet(np.ones(E)))
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def deepseek_moe(name: str, E: int = MOE_EXPERTS, M: int = MOE_ROWS):
    """(X bits [M, K], offsets int32 [E + 1]) for the expert linear `name`;
    the weights come from deepseek_moe_weights."""
    N, K = MOE_LINEARS[name]
    g = _rng(SEED_X, hash_name("moe_" + name))
    x = g.standard_normal((M, K), dtype=np.float32)
    x *= g.lognormal(0.0, 1.0, size=(M, 1)).astype(np.float32)
    return f32_to_bf16_bits(x), moe_offsets(E, M)


def deepseek_moe_weights(name: str, device, E: int = MOE_EXPERTS):
    """Stacked expert weights [E * N, K] (expert e = rows e N .. e N + N - 1),
    N(0, 0.015) in bf16, drawn on `device` by torch's generator seeded with
    (SEED_W, salt): hundreds of millions of draws, which numpy on the host
    would take tens of seconds for."""
    import torch
    N, K = MOE_LINEARS[name]
    g = torch.Generator(device=device)
    g.manual_seed(SEED_W * 1_000_003 + hash_name("moe_" + name))
    w = torch.empty((E * N, K), dtype=torch.bfloat16, device=device)
    for e in range(E):
        w[e * N:(e + 1) * N] = (torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
                                * 0.015).to(torch.bfloat16)
    return w


def sweep_x(M: int, K: int = SWEEP_K):
    x = student_t_outliers(M, K, 3.0, 0.001, 100.0, SEED_X, 77)
    return zero_groups(x, 0.01, 77)


def sweep_w():
    return normal((SWEEP_N, SWEEP_K), 0.02, SEED_W, 77)


def hash_name(name: str) -> int:
    """Stable small integer per linear name (Python's hash() is salted)."""
    return sum((i + 1) * ord(c) for i, c in enumerate(name)) % 10007


def to_torch_bf16(bits: np.ndarray):
    """View bf16 bit patterns as a torch.bfloat16 CPU tensor (no copy)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
