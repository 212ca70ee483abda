"""fine_grained_block_token_b200 -- block-scaled FP8 linear layers for B200.

Weights quantized to e4m3 with one fp32 scale per 128 x 128 block,
activations quantized dynamically per token with one fp32 scale per group of
128 input channels, and a GEMM that applies both scale sets per 128-deep K
block and writes bf16 ("Fine-grained FP8" page of the transformers docs,
opening bullet list).  The ``*_ue8m0`` functions are the power-of-two scale
variant of the page's "UE8M0 scale format" section (float8_e8m0fnu scales),
whose GEMM runs on the tensor core's block-scaled MMA.  ``quant_rowwise`` /
``linear_rowwise`` are the row-wise FP8 scheme (fp8r) of the "BFL (fp8r /
nvfp4)" page: one fp32 scale per activation row and per weight row.
``quant_act_static`` is the static activation scheme (one given scale), and
``grouped_linear_ue8m0`` the grouped (MoE expert) form of the UE8M0 linear.

The functions below come from ``_binding`` (a ctypes binding of
``libfp8bl.so``), loaded on first use so that the ``build`` submodule can be
imported before the library exists.  Using any of them without the library
raises ImportError: there is no fallback path.
"""
__all__ = [
    "Fp8blError", "BLOCK", "STATUS", "lib_path", "quant_act", "quant_weight", "block_linear",
    "block_linear_fused", "block_linear_noalloc", "workspace_bytes", "fused_workspace_bytes",
    "check", "version", "quant_act_ue8m0", "quant_weight_ue8m0", "block_linear_ue8m0",
    "ue8m0_workspace_bytes", "quant_rowwise", "linear_rowwise", "quant_act_static",
    "grouped_linear_ue8m0", "grouped_ue8m0_workspace_bytes",
]


def __getattr__(name):
    if name in __all__:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
