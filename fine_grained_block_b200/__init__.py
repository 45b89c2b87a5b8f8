"""FP8 scaled quantization for B200: a thin Python binding over ``libfp8q.so``.

The CUDA library does all the work; this package only marshals arguments.
The binding is loaded on first use, so ``import fine_grained_block_b200.inputs``
works on a host without the library or a GPU.  Calling any entry point when
the library is missing raises; there is no CPU fallback.
"""

_BINDING_NAMES = (
    "fp8_quantize_per_tensor", "fp8_quantize_blockwise", "fp8_dequantize",
    "fp8_amax_history_update", "fp8_amax_history_update_ex", "fp8_fake_quantize", "fp8_amax", "fp8_scale_from_amax",
    "fp8_quantize_per_tensor_fused", "fused_workspace", "fp8_status_string", "FP8Error", "load_library",
    "fp8_quantize_mx", "fp8_dequantize_mx", "MX_FIT", "MX_OCP", "fp8_quantize_per_tensor_transpose", "fp8_quantize_blockwise_transpose",
    "fp8_gemm_blockwise", "fp8_quantize_delayed_step", "DelayedScaler",
    "fp8_quantize_blockwise_grouped", "FP8BlockTensor", "fp8_quantize_delayed_step_grouped", "FP8DelayedTensor",
    "fp8_quantize_per_tensor_grouped", "FP8CurrentTensor",
    "E4M3", "E5M2", "F32", "BF16",
)


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
