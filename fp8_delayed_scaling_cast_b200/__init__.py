"""B200-native FP8 delayed-scaling linear hot path.

The compute lives in ``libfp8ds.so`` (hand-written CUDA for sm_100a, C ABI in
``include/fp8ds.h``); ``binding`` is its thin ctypes binding.  Attributes of
the binding are re-exported lazily so that ``inputs`` (the seeded input
generators) can be imported on machines without the built library.
"""

__all__ = [
    "fp8_quantize", "fp8_cast_transpose_amax", "fp8_update_scales", "fp8_gemm", "fp8_gemm_ex",
    "fp8_gemm_workspace_size", "gemm_workspace",
    "fp8_linear_fwd", "fp8_linear_bwd", "fp8ds_last_error", "fp8ds_device_status",
    "fp8ds_version", "Fp8Meta", "Fp8Linear", "Fp8dsError", "E4M3", "E5M2",
]


def __getattr__(name):
    if name in __all__ or name in ("binding", "LIB_PATH"):
        import importlib
        binding = importlib.import_module(__name__ + ".binding")
        return binding if name == "binding" else getattr(binding, name)
    raise AttributeError(name)
