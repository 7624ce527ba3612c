"""The allocation-free block forward (h3b_block_forward_noalloc).

It exists for callers that may not allocate device memory (an application
that owns all device memory through its own pool, or a latency-critical
thread that must not call cudaMalloc).  Its scratch is a fixed array inside
the library's device image; these tests call it through the C ABI twice in a
row -- the second call sees the first call's leftovers in that array -- and
require both results to equal, bit for bit, h3b_block_forward's result on a
caller-allocated workspace: the same kernels run on the same inputs with the
same arena plan, so nothing may differ.  The file is collected last so a failure here
leaves every other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wlmod

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("audio_diffusion_transformer_dit_b200.h3b")

_fn = h3b.lib.h3b_block_forward_noalloc
_fn.restype = ctypes.c_int
_fn.argtypes = [ctypes.POINTER(h3b.Dims), ctypes.POINTER(h3b.BlockWeights), ctypes.c_void_p, ctypes.c_int,
                ctypes.c_void_p]


def _noalloc(dm, blk, x, merged=False):
    return _fn(ctypes.byref(dm), ctypes.byref(blk.c), x.data_ptr(), int(merged), h3b._stream())


@pytest.mark.parametrize("int8,merged", [(False, False), (False, True), (True, False)])
def test_noalloc_matches_block_forward_twice(cuda_dev, int8, merged):
    wl = wlmod.WORKLOADS["block_d256_s288"]
    dm = h3b.dims_of(wl)
    w = wlmod.block_weights(wl, 0, cuda_dev)
    blk = h3b.Block.quantized(w) if int8 else h3b.Block.from_dict(w)
    S = h3b.seq_len(dm, merged)
    x0 = wlmod.initial_tokens(wl, cuda_dev, seq=S)

    ref = x0.clone()
    ws = h3b.workspace(dm, blk.dtype)
    h3b.block_forward(dm, blk, ref, ws, merged)

    for _ in range(2):
        x = x0.clone()
        assert _noalloc(dm, blk, x, merged) == 0
        torch.cuda.synchronize()
        assert h3b.device_error() == 0
        assert np.isfinite(x.cpu().numpy()).all()
        assert torch.equal(x, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_dev):
    wl = wlmod.WORKLOADS["block_d3072_s6400"]
    dm = h3b.dims_of(wl)
    assert h3b.workspace_bytes(dm) > (32 << 20)
    w = wlmod.block_weights(wlmod.WORKLOADS["block_d256_s288"], 0, cuda_dev)  # never read: rejected first
    blk = h3b.Block.from_dict(w)
    x = torch.zeros(8, device=cuda_dev)
    assert _noalloc(dm, blk, x) == -5  # H3B_ERR_WORKSPACE, nothing enqueued
