"""Whole library steps captured into a CUDA graph (``h3b.Graph``) and replayed:
a replay issues the same kernels with the same arguments as the eager calls,
so its result equals theirs bit for bit.  Every kernel on the path reduces in
a fixed order (split-K parts and key-split parts summed in part order, no
floating-point atomics), which makes the eager result itself reproducible.
Agreement with the oracle follows from the eager tests."""
import pytest
import torch

import workloads as wlmod

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("audio_diffusion_transformer_dit_b200.h3b")

TINY = wlmod.WORKLOADS["block_d256_s288"]


def eager_and_replayed(x0, call, replays=2):
    """``call(x)`` issues library calls that update x in place.  Returns x0
    after ``replays`` eager applications and after as many replays of one
    captured application (captured on its own buffer, which is reset to x0
    before the replays)."""
    xe = x0.clone()
    for _ in range(replays):
        call(xe)
    xg = x0.clone()
    call(xg)  # the library has run on this device and on these buffers before the capture
    torch.cuda.synchronize()
    g = h3b.Graph(lambda: call(xg))
    xg.copy_(x0)
    for _ in range(replays):
        g.replay()
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    return xe, xg


@pytest.mark.parametrize("int8,merged", [(False, False), (False, True), (True, False)])
def test_block_graph_replay_equals_eager(cuda_dev, int8, merged):
    w = wlmod.block_weights(TINY, 0, cuda_dev)
    blk = h3b.Block.quantized(w) if int8 else h3b.Block.from_dict(w)
    dm = h3b.dims_of(TINY)
    x0 = wlmod.initial_tokens(TINY, cuda_dev, seq=h3b.seq_len(dm, merged))
    ws = h3b.workspace(dm, h3b.INT8 if int8 else h3b.BF16)
    xe, xg = eager_and_replayed(x0, lambda x: h3b.block_forward(dm, blk, x, ws, merged))
    assert not torch.equal(xe, x0)
    assert torch.equal(xe, xg)


@pytest.mark.parametrize("int8", [False, True])
def test_stack_with_reduction_graph_replay_equals_eager(cuda_dev, int8):
    wl = TINY.with_(n_blocks=5, depth_scaled_init=True, seed=21, dtype=h3b.INT8 if int8 else h3b.BF16)
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(wl.n_blocks)]
    blocks = [h3b.Block.quantized(w) if int8 else h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    ws = h3b.workspace(dm, wl.dtype, True)
    xe, xg = eager_and_replayed(x0, lambda x: h3b.stack_forward(dm, blocks, x, ws, 1, 3))
    assert torch.equal(xe, xg)


def test_denoise_graph_replay_equals_eager(cuda_dev):
    wl = TINY.with_(n_blocks=4, depth_scaled_init=True, seed=22)
    blocks = [h3b.Block.from_dict(wlmod.block_weights(wl, l, cuda_dev)) for l in range(wl.n_blocks)]
    dm = h3b.dims_of(wl)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    v = torch.empty_like(x0)
    ws = h3b.workspace(dm, h3b.BF16, True)
    xe, xg = eager_and_replayed(x0, lambda x: h3b.denoise(dm, blocks, x, v, ws, 5, 2, 1, 2), replays=1)
    assert torch.equal(xe, xg)


def test_denoise_ex_condition_rows_core_reuse_graph_replay_equals_eager(cuda_dev):
    wl = TINY.with_(n_blocks=4, depth_scaled_init=True, seed=23)
    C, steps = 12, 5
    blocks = [h3b.Block.from_dict(wlmod.block_weights(wl, l, cuda_dev)) for l in range(4)]
    dm = h3b.dims_of(wl)
    mod = wlmod.normal_tensor((steps, 4, 2, 6, wl.d), 44, cuda_dev, 0.1)
    cond = wlmod.normal_tensor((C, wl.d), 45, cuda_dev)
    o = h3b.stack_opts(1, 2, unmerge_delta=True, core_first=1, core_last=2, cond_rows=cond, modulation=mod)
    ws = h3b.workspace_ex(dm, o)
    v = torch.empty((wl.seq + C, wl.d), device=cuda_dev)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    xe, xg = eager_and_replayed(
        x0, lambda x: h3b.denoise_ex(dm, blocks, x, v, ws, steps, o, reuse=1, core_reuse=2), replays=1)
    assert torch.equal(xe, xg)
