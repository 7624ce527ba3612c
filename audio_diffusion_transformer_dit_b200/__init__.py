"""B200-native engine for the MiniMax H3 DiT block hot path.

The compute lives in ``libh3b.so`` (hand-written sm_100a CUDA behind the C
ABI declared in ``include/h3b.h``); ``h3b`` is its Python binding.  Importing
the package without the built library raises ImportError -- there is no CPU
fallback.  Build with ``python -m audio_diffusion_transformer_dit_b200.build``.
"""
from . import h3b  # noqa: F401
from .h3b import (BF16, INT8, Block, Dims, H3bError, Trace, attention, block_forward, denoise,  # noqa: F401
                  dims_of, flow_step, gemm, quantize_weights, rmsnorm, rope_table, seq_len, stack_forward,
                  token_merge, token_unmerge, workspace, workspace_bytes)
