"""B200-native engine for the MiniMax H3 DiT block hot path.

The compute lives in ``libh3b.so`` (hand-written sm_100a CUDA behind the C
ABI declared in ``include/h3b.h``); ``h3b`` is its Python binding.  The
binding is loaded on first use of any of the names below; without the built
library that raises ImportError -- there is no CPU fallback.  Build with
``python -m audio_diffusion_transformer_dit_b200.build``.
"""
_EXPORTS = ("BF16", "INT8", "Block", "Dims", "Graph", "H3bError", "HostPipeline", "StackOpts", "Trace", "attention",
            "block_forward", "denoise", "denoise_ex", "device_error", "dims_of", "flow_step", "gelu", "gemm",
            "quantize_weights", "rmsnorm", "rope_table", "seq_len", "stack_forward", "stack_forward_ex",
            "stack_opts", "token_merge", "token_unmerge", "workspace", "workspace_bytes", "workspace_ex")


def __getattr__(name):
    if name == "h3b" or name in _EXPORTS:
        import importlib
        mod = importlib.import_module(__name__ + ".h3b")
        return mod if name == "h3b" else getattr(mod, name)
    raise AttributeError(name)
