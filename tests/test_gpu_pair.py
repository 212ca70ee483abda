"""GPU parity of the CTA-pair block-scaled GEMM (tcgen05.mma.cta_group::2,
256 x 256 tiles), which the library runs instead of the single-CTA kernel
when FP8BL_BLOCK_PAIRS=1 is set before it loads.  The switch is read once
per process, so the check runs in a child process: its outputs must meet
the GEMM tolerance against the oracle ("Fine-grained FP8" page: both scale
sets applied per 128-deep K block) and equal the single-CTA kernel's up to
the fp32 accumulation order."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import fine_grained_block_token_b200 as fp8
import oracle, workloads as wl
from tests.parity import check_gemm
for (M, N, K) in [(256, 512, 512), (300, 640, 1024), (129, 384, 384), (1024, 2304, 2048)]:
    xb = wl.normal((M, K), 1.0, 0, M + N + K)
    wb = wl.zero_blocks(wl.normal((N, K), 0.02, 1, M + N + K), 0.05)
    x, w = wl.to_torch_bf16(xb).cuda(), wl.to_torch_bf16(wb).cuda()
    q_a, s_a = fp8.quant_act(x)
    q_w, s_w = fp8.quant_weight(w)
    y = fp8.block_linear(q_a, s_a, q_w, s_w)
    fp8.check()
    R = oracle.block_linear(q_a.view(torch.uint8).cpu().numpy(), s_a.cpu().numpy(),
                            q_w.view(torch.uint8).cpu().numpy(), s_w.cpu().numpy(), nthreads=8)
    check_gemm(y.float().cpu().numpy(), R, f"pair {M}x{N}x{K}")
print("PAIR_OK")
'''


def test_pair_kernel_against_the_oracle():
    env = dict(os.environ, FP8BL_BLOCK_PAIRS="1")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "PAIR_OK" in r.stdout, r.stdout[-2000:] + r.stderr[-3000:]
