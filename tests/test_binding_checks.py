"""Argument checks of the Python binding.

The C ABI takes raw pointers and sizes, so the binding checks every tensor
(device, dtype, shape, contiguity) and raises before it passes a pointer on.
The CPU cases need no GPU: a tensor that is not on a CUDA device is refused
before the library is called.  The GPU cases build wrong operands on the
device and check that each is refused by the binding, and that the library
then still runs a correct call (nothing was enqueued by the refused ones).
A last CPU case checks that every ctypes signature in the binding has as
many arguments as its declaration in include/fp8bl.h.
"""
import pytest
import torch

import fine_grained_block_token_b200 as fp8

BF16 = torch.bfloat16
E4 = torch.float8_e4m3fn
E8 = torch.float8_e8m0fnu


def _cpu_calls():
    x = torch.zeros(4, 256, dtype=BF16)
    q = torch.zeros(4, 256, dtype=E4)
    s = torch.ones(4, 2, dtype=torch.float32)
    qw = torch.zeros(128, 256, dtype=E4)
    sw = torch.ones(1, 2, dtype=torch.float32)
    c = torch.full((4, 2), 127, dtype=torch.uint8).view(E8)
    cw = torch.full((1, 2), 127, dtype=torch.uint8).view(E8)
    off = torch.tensor([0, 4], dtype=torch.int32)
    y = torch.empty(4, 128, dtype=BF16)
    return {
        "quant_act": lambda: fp8.quant_act(x),
        "quant_act_static": lambda: fp8.quant_act_static(x, torch.ones(1)),
        "quant_weight": lambda: fp8.quant_weight(x),
        "quant_act_ue8m0": lambda: fp8.quant_act_ue8m0(x),
        "quant_weight_ue8m0": lambda: fp8.quant_weight_ue8m0(x),
        "quant_rowwise": lambda: fp8.quant_rowwise(x),
        "block_linear": lambda: fp8.block_linear(q, s, qw, sw),
        "block_linear_fused": lambda: fp8.block_linear_fused(x, qw, sw),
        "block_linear_noalloc": lambda: fp8.block_linear_noalloc(q, s, qw, sw, y),
        "block_linear_ue8m0": lambda: fp8.block_linear_ue8m0(q, c, qw, cw),
        "grouped_linear_ue8m0": lambda: fp8.grouped_linear_ue8m0(q, c, qw.view(1, 128, 256),
                                                                 cw.view(1, 1, 2), off),
        "linear_rowwise": lambda: fp8.linear_rowwise(q, s[:, 0].contiguous(), qw,
                                                     torch.ones(128)),
    }


@pytest.mark.parametrize("name", sorted(_cpu_calls()))
def test_host_tensors_refused(name):
    with pytest.raises(ValueError, match="CUDA device"):
        _cpu_calls()[name]()


def test_non_tensor_refused():
    with pytest.raises(TypeError):
        fp8.quant_act([[0.0] * 128])
    with pytest.raises(TypeError):
        fp8.block_linear(None, None, None, None)


@pytest.mark.gpu
def test_wrong_operands_refused_on_device():
    d = "cuda"
    x = torch.randn(64, 256, dtype=BF16, device=d)
    w = torch.randn(256, 256, dtype=BF16, device=d) * 0.02
    q_a, s_a = fp8.quant_act(x)
    q_w, s_w = fp8.quant_weight(w)
    bad = [
        (TypeError, lambda: fp8.quant_act(x.float())),                           # fp32 input
        (ValueError, lambda: fp8.quant_act(x.t())),                              # strided view
        (ValueError, lambda: fp8.quant_act(x[None])),                            # 3-D
        (ValueError, lambda: fp8.quant_act(x, s=torch.empty(64, 3, device=d))),  # scale shape
        (TypeError, lambda: fp8.quant_act(x, q=torch.empty(64, 256, dtype=torch.int8, device=d))),
        (TypeError, lambda: fp8.block_linear(q_a, s_a.double(), q_w, s_w)),
        (ValueError, lambda: fp8.block_linear(q_a, s_a, q_w[:, :128].contiguous(), s_w)),
        (ValueError, lambda: fp8.block_linear(q_a, s_a[:, :1], q_w, s_w)),
        (ValueError, lambda: fp8.block_linear(q_a, s_a, q_w, s_w,
                                              y=torch.empty(64, 128, dtype=BF16, device=d))),
        (ValueError, lambda: fp8.block_linear_noalloc(q_a, s_a, q_w, s_w, None)),
        (TypeError, lambda: fp8.block_linear_ue8m0(q_a, s_a, q_w, s_w)),         # fp32 scales
        (TypeError, lambda: fp8.grouped_linear_ue8m0(
            q_a, s_a.to(torch.uint8), q_w.view(1, 256, 256), s_w.to(torch.uint8).view(1, 2, 2),
            torch.tensor([0, 64], dtype=torch.int64, device=d))),                # int64 offsets
        (ValueError, lambda: fp8.grouped_linear_ue8m0(
            q_a, s_a.to(torch.uint8), q_w.view(1, 256, 256), s_w.to(torch.uint8).view(1, 2, 2),
            torch.tensor([0, 32, 64], dtype=torch.int32, device=d))),            # E + 1 mismatch
        (ValueError, lambda: fp8.linear_rowwise(q_a, s_a, q_w, s_w)),            # block scales
        (ValueError, lambda: fp8.quant_act_static(x, torch.ones(2, device=d))),
        (ValueError, lambda: fp8.quant_act_static(x, torch.ones(1))),            # host scale
    ]
    for i, (exc, call) in enumerate(bad):
        with pytest.raises(exc):
            call()
    y = fp8.block_linear(q_a, s_a, q_w, s_w)
    fp8.check()
    ref = (x.float() @ w.float().t())
    err = (y.float() - ref).norm() / ref.norm()
    assert float(err) < 0.1


def _header_param_counts():
    import os
    import re
    hdr = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fp8bl.h")
    txt = re.sub(r"/\*.*?\*/", "", open(hdr).read(), flags=re.S)
    out = {}
    for name, params in re.findall(r"\b(fp8\w*)\s*\(([^;{]*?)\)\s*;", txt, flags=re.S):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argtypes_match_the_header():
    """Every function the binding declares to ctypes takes as many arguments
    as its C declaration (a missing or extra one would shift every pointer
    after it)."""
    from fine_grained_block_token_b200 import _binding as b
    counts = _header_param_counts()
    checked = 0
    for name, n in counts.items():
        f = getattr(b._lib, name)
        if f.argtypes is None:
            continue
        assert len(f.argtypes) == n, (name, len(f.argtypes), n)
        checked += 1
    assert checked >= 15


def test_package_exports_every_binding_name():
    """Every public name of the ctypes binding is reachable from the package
    (its lazy re-export list), so a new entry point cannot go missing there."""
    import fine_grained_block_token_b200 as pkg
    from fine_grained_block_token_b200 import _binding
    missing = set(_binding.__all__) - set(pkg.__all__)
    assert not missing, missing
    for name in _binding.__all__:
        assert getattr(pkg, name) is getattr(_binding, name)
