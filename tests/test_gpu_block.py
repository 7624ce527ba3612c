"""Block, stack and denoising-loop parity through the C ABI against the oracle.

Tolerances (per the block's stated bar): block output relative L2 <= 1e-2 and
max-abs <= 5e-2 for BF16; relative L2 <= 2e-2 for INT8 against the oracle
block run on the int8 round-trip of the weights, with element and per-token
bounds derived in check_int8.  The block update x2 - x is
also checked on its own (a stricter view: the residual dominates x2), with a
bound derived from the bf16 roundings on the path (u, qkv, P, o, u2, GELU out:
six roundings of 2^-9 relative each, attenuated through the GEMMs) -> 2e-2
for BF16; for INT8 the per-token activation codes add ~1% per GEMM -> 6e-2.
At full sizes the oracle computes a sample of output rows (all keys/values).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wlmod
from tests._util import np64, rel_l2, max_abs, host_weights

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("audio_diffusion_transformer_dit_b200.h3b")

TINY = wlmod.WORKLOADS["block_d256_s288"]


def make_block(wl, layer, dev, int8):
    w = wlmod.block_weights(wl, layer, dev)
    return w, (h3b.Block.quantized(w) if int8 else h3b.Block.from_dict(w))


def run_block(wl, layer, dev, int8=False, merged=False):
    w, blk = make_block(wl, layer, dev, int8)
    dm = h3b.dims_of(wl)
    S = h3b.seq_len(dm, merged)
    x0 = wlmod.initial_tokens(wl, dev, seq=S)
    x = x0.clone()
    ws = h3b.workspace(dm, h3b.INT8 if int8 else h3b.BF16)
    h3b.block_forward(dm, blk, x, ws, merged)
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    return np64(x0), np64(x), host_weights(w)


def check_bf16(x0, got, ref):
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) <= 1e-2
    assert max_abs(got, ref) <= 5e-2
    assert rel_l2(got - x0, ref - x0) <= 2e-2


def check_int8(x0, got, ref):
    """INT8 block output against the oracle block on the dequantised weights.

    Relative L2 <= 2e-2 (the INT8 bound) and update relative L2 <= 6e-2.  The
    per-token activation codes (a rounding of up to half a step, step = row
    max / 127, at every GEMM input; bf16 roundings before each quantiser flip
    codes too) make the error a sum of many small independent terms, so its
    largest element grows with the output's scale and the sample size: the
    element bound is 6 sigma of an error whose RMS is at the relative-L2 bound,
    6 * 2e-2 * rms(ref) (measured at d = 5120, S = 20640: max-abs 0.22 against
    0.35 allowed; 0.038 against 0.13 at d = 1024).  No token may be off by
    more than twice the global bound, which a badly quantised token (a wrong
    scale, a flipped sign) would break."""
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) <= 2e-2
    assert rel_l2(got - x0, ref - x0) <= 6e-2
    rms = float(np.sqrt(np.mean(np.asarray(ref, dtype=np.float64) ** 2)))
    assert max_abs(got, ref) <= 6 * 2e-2 * rms
    row_rel = np.linalg.norm(got - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-300)
    assert row_rel.max() <= 4e-2


@pytest.mark.parametrize("merged", [False, True])
def test_block_tiny_bf16(cuda_dev, merged):
    x0, got, w = run_block(TINY, 0, cuda_dev, merged=merged)
    check_bf16(x0, got, oracle.block_forward(x0, w, TINY, merged=merged))


def test_block_tiny_int8(cuda_dev):
    x0, got, w = run_block(TINY, 0, cuda_dev, int8=True)
    check_int8(x0, got, oracle.block_forward(x0, oracle.dequant_weights(w), TINY))


@pytest.mark.parametrize("int8", [False, True])
def test_block_medium(cuda_dev, int8):
    wl = wlmod.Workload("m", 3, 10, 12, 77, 1024, 8, 128, 4096, 1, 1 if int8 else 0, 11, False)
    x0, got, w = run_block(wl, 0, cuda_dev, int8=int8)
    if int8:
        check_int8(x0, got, oracle.block_forward(x0, oracle.dequant_weights(w), wl))
    else:
        check_bf16(x0, got, oracle.block_forward(x0, w, wl))


def test_block_head_dim_64(cuda_dev):
    wl = wlmod.Workload("h64", 2, 6, 8, 21, 512, 8, 64, 2048, 1, 0, 12, False)
    x0, got, w = run_block(wl, 0, cuda_dev)
    check_bf16(x0, got, oracle.block_forward(x0, w, wl))


def sample_rows(S, n_video, k=48, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, n_video - 1, n_video, S - 1]
    return np.unique(np.concatenate([fixed, rng.choice(S, size=k, replace=False)]))


@pytest.mark.slow
@pytest.mark.parametrize("name,layer,merged", [("block_d3072_s6400", 0, False),
                                               ("stack8_d5120_s6528", 0, False),
                                               ("stack8_d5120_s6528", 7, False),
                                               ("loop45_d5120_s6528", 20, True),
                                               ("preview40_d5120_s2784", 39, False)])
def test_block_full_size_sampled(cuda_dev, name, layer, merged):
    wl = wlmod.WORKLOADS[name]
    x0, got, w = run_block(wl, layer, cuda_dev, merged=merged)
    S = x0.shape[0]
    nv = wl.n_video // 2 if merged else wl.n_video
    rows = sample_rows(S, nv)
    ref = oracle.block_forward(x0, w, wl, merged=merged, rows=rows)
    check_bf16(x0[rows], got[rows], ref)


@pytest.mark.slow
def test_block_int8_full_size_sampled(cuda_dev):
    wl = wlmod.WORKLOADS["block_int8_d5120_s20640"]
    x0, got, w = run_block(wl, 0, cuda_dev, int8=True)
    rows = sample_rows(x0.shape[0], wl.n_video, k=32)
    ref = oracle.block_forward(x0, oracle.dequant_weights(w), wl, rows=rows)
    check_int8(x0[rows], got[rows], ref)


# ----------------------------------------------------------------------------- stack
def run_stack(wl, dev, mf=-1, ml=-1):
    ws_ = [wlmod.block_weights(wl, l, dev) for l in range(wl.n_blocks)]
    blocks = [h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    x0 = wlmod.initial_tokens(wl, dev)
    x = x0.clone()
    ws = h3b.workspace(dm, h3b.BF16, mf >= 0)
    h3b.stack_forward(dm, blocks, x, ws, mf, ml)
    torch.cuda.synchronize()
    return x0, x, ws_, blocks, ws


@pytest.mark.parametrize("mf,ml", [(-1, -1), (2, 4)])
def test_stack_small_vs_oracle(cuda_dev, mf, ml):
    wl = TINY.with_(n_blocks=6, depth_scaled_init=True, seed=5)
    x0, x, ws_, _, _ = run_stack(wl, cuda_dev, mf, ml)
    ref = oracle.stack_forward(np64(x0), [host_weights(w) for w in ws_], wl, mf, ml)
    check_bf16(np64(x0), np64(x), ref)


def test_stack_equals_block_sequence(cuda_dev):
    """h3b_stack_forward = merge + the same block calls + unmerge.  Inside the
    stack, consecutive blocks on the same token grid (blocks 1..3 in the merged
    window) take their RMSNorm1 folded into the QKV GEMM (the previous FC2
    leaves bf16(x * g) and the row sums of squares), where a lone block call
    normalises first: the two differ only by where one bf16 rounding of the
    normed operand falls (~2^-9 relative on the GEMM input), while a wrong
    merge, unmerge, row-sum table or stale bf16 copy would be off by O(1)."""
    wl = TINY.with_(n_blocks=5, depth_scaled_init=True, seed=6)
    x0, x, _, blocks, ws = run_stack(wl, cuda_dev, 1, 3)
    dm = h3b.dims_of(wl)
    y = x0.clone()
    for l in (0,):
        h3b.block_forward(dm, blocks[l], y, ws)
    ym = torch.empty((h3b.seq_len(dm, True), wl.d), device=cuda_dev)
    h3b.token_merge(dm, y, ym)
    for l in (1, 2, 3):
        h3b.block_forward(dm, blocks[l], ym, ws, merged=True)
    h3b.token_unmerge(dm, ym, y)
    h3b.block_forward(dm, blocks[4], y, ws)
    torch.cuda.synchronize()
    assert rel_l2(x, y) <= 2e-3 and max_abs(x, y) <= 2e-2
    assert rel_l2(x - x0, y - x0) <= 1e-2


def test_int8_stack_equals_block_sequence_bitexact(cuda_dev):
    """INT8 blocks normalise (and quantise) in their own pass inside a stack as
    in a lone block call, so the stack with a reduction window equals the
    explicit merge + block calls + unmerge bit for bit."""
    wl = TINY.with_(n_blocks=4, depth_scaled_init=True, seed=16, dtype=h3b.INT8)
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(4)]
    blocks = [h3b.Block.quantized(w) for w in ws_]
    dm = h3b.dims_of(wl)
    x = wlmod.initial_tokens(wl, cuda_dev)
    y = x.clone()
    ws = h3b.workspace(dm, h3b.INT8, True)
    h3b.stack_forward(dm, blocks, x, ws, 1, 2)
    h3b.block_forward(dm, blocks[0], y, ws)
    ym = torch.empty((h3b.seq_len(dm, True), wl.d), device=cuda_dev)
    h3b.token_merge(dm, y, ym)
    for l in (1, 2):
        h3b.block_forward(dm, blocks[l], ym, ws, merged=True)
    h3b.token_unmerge(dm, ym, y)
    h3b.block_forward(dm, blocks[3], y, ws)
    torch.cuda.synchronize()
    assert torch.equal(x, y)


@pytest.mark.slow
def test_stack8_full_size_equals_blocks(cuda_dev):
    """The benched 8-block stack against the same blocks called one by one
    (blocks 1..7 take the folded RMSNorm1 in the stack; see
    test_stack_equals_block_sequence), and the stack run twice is bit-identical
    (the folded norm sums its row partials in a fixed order)."""
    wl = wlmod.WORKLOADS["stack8_d5120_s6528"]
    x0, x, _, blocks, ws = run_stack(wl, cuda_dev)
    dm = h3b.dims_of(wl)
    y = x0.clone()
    for b in blocks:
        h3b.block_forward(dm, b, y, ws)
    x2 = x0.clone()
    h3b.stack_forward(dm, blocks, x2, ws)
    torch.cuda.synchronize()
    assert torch.isfinite(x).all()
    assert torch.equal(x, x2)
    assert rel_l2(x, y) <= 2e-3 and rel_l2(x - x0, y - x0) <= 1e-2


# ----------------------------------------------------------------------------- denoising loop
@pytest.mark.parametrize("steps,reuse,mf,ml", [(5, 2, 1, 2), (4, 1, -1, -1), (20, 3, -1, -1)])
def test_denoise_small_vs_oracle(cuda_dev, steps, reuse, mf, ml):
    wl = TINY.with_(n_blocks=4, depth_scaled_init=True, seed=7)
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(wl.n_blocks)]
    blocks = [h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    x = x0.clone()
    v = torch.empty_like(x)
    ws = h3b.workspace(dm, h3b.BF16, mf >= 0)
    nf = h3b.denoise(dm, blocks, x, v, ws, steps, reuse, mf, ml)
    torch.cuda.synchronize()
    ref, nf_ref = oracle.denoise(np64(x0), [host_weights(w) for w in ws_], wl, steps, reuse, mf, ml)
    assert nf == nf_ref == len(oracle.fresh_steps(steps, reuse))
    assert rel_l2(x, ref) <= 1e-2
    assert max_abs(x, ref) <= 5e-2


@pytest.mark.parametrize("steps,reuse", [(4, 1), (5, 2), (7, 3)])
def test_denoise_few_steps_layer_subset_vs_oracle(cuda_dev, steps, reuse):
    """The 4..7-step presets on the first L = 3 of a 5-block model (--layers):
    the loop is given only the active blocks."""
    wl = TINY.with_(n_blocks=5, depth_scaled_init=True, seed=11, frames=2, rows=6, cols=10, n_audio=24)
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(3)]
    blocks = [h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    x = x0.clone()
    v = torch.empty_like(x)
    nf = h3b.denoise(dm, blocks, x, v, h3b.workspace(dm), steps, reuse)
    torch.cuda.synchronize()
    ref, nf_ref = oracle.denoise(np64(x0), [host_weights(w) for w in ws_], wl, steps, reuse)
    assert nf == nf_ref
    assert rel_l2(x, ref) <= 1e-2 and max_abs(x, ref) <= 5e-2


@pytest.mark.slow
def test_loop45_full_size_equals_composition(cuda_dev):
    """The benched loop itself (45 blocks at d = 5120, S = 6528, tokens merged
    over blocks 15..29, 20 steps, whole-velocity reuse 2) equals, bit for bit,
    its definition written with the separately verified entry points: on a
    fresh step the velocity is the stack output of the current x, and every
    step is the Euler update over the sigma grid 1 - i/N."""
    wl = wlmod.WORKLOADS["loop45_d5120_s6528"]
    dm = h3b.dims_of(wl)
    blocks = [h3b.Block.from_dict(wlmod.block_weights(wl, l, cuda_dev)) for l in range(wl.n_blocks)]
    ws = h3b.workspace(dm, h3b.BF16, True)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    x = x0.clone()
    v = torch.empty_like(x)
    nf = h3b.denoise(dm, blocks, x, v, ws, wl.steps, wl.reuse, wl.merge_first, wl.merge_last)
    y = x0.clone()
    sig = oracle.sigmas(wl.steps)
    vel = None
    for i in range(wl.steps):
        if oracle.is_fresh(i, wl.steps, wl.reuse):
            vel = h3b.stack_forward(dm, blocks, y.clone(), ws, wl.merge_first, wl.merge_last)
        h3b.flow_step(y, vel, float(sig[i]), float(sig[i + 1]))
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    assert nf == len(oracle.fresh_steps(wl.steps, wl.reuse)) == 11
    assert torch.isfinite(x).all() and torch.equal(x, y)


def test_denoise_fresh_counts(cuda_dev):
    wl = TINY.with_(n_blocks=1)
    blocks = [h3b.Block.from_dict(wlmod.block_weights(wl, 0, cuda_dev))]
    dm = h3b.dims_of(wl)
    x = wlmod.initial_tokens(wl, cuda_dev)
    v = torch.empty_like(x)
    ws = h3b.workspace(dm)
    assert [h3b.denoise(dm, blocks, x, v, ws, 20, r) for r in (1, 2, 3)] == [20, 11, 8]


# ----------------------------------------------------------------------------- host-side errors on a GPU machine
def test_workspace_too_small_is_rejected(cuda_dev):
    dm = h3b.dims_of(TINY)
    _, blk = make_block(TINY, 0, cuda_dev, False)
    x = wlmod.initial_tokens(TINY, cuda_dev)
    ws = torch.empty(h3b.workspace_bytes(dm) - 256, dtype=torch.uint8, device=cuda_dev)
    with pytest.raises(h3b.H3bError) as e:
        h3b.block_forward(dm, blk, x, ws)
    assert e.value.status == -5


def test_misaligned_pointer_is_rejected(cuda_dev):
    dm = h3b.dims_of(TINY)
    _, blk = make_block(TINY, 0, cuda_dev, False)
    buf = torch.zeros(TINY.seq * TINY.d + 1, device=cuda_dev)
    ws = h3b.workspace(dm)
    st = h3b.lib.h3b_block_forward(h3b.ctypes.byref(dm), h3b.ctypes.byref(blk.c), buf.data_ptr() + 4, 0,
                                   ws.data_ptr(), ws.numel(), h3b._stream())
    assert st == -2


def test_bounded_wait_reports_and_context_survives(cuda_dev):
    """A device wait that can never complete gives up after its limit, sets the
    error word, and later work on the same context runs normally."""
    assert h3b.device_error() == 0
    assert h3b.lib.h3b_selftest_wait_timeout(2000, h3b._stream()) == 0
    torch.cuda.synchronize()
    assert h3b.device_error() == (3 << 8) | 1
    assert h3b.device_error() == 0  # cleared by the read
    x = torch.ones(1024, device=cuda_dev)
    h3b.flow_step(x, torch.ones_like(x), 1.0, 0.5)
    torch.cuda.synchronize()
    assert torch.all(x == 0.5)
    assert h3b.lib.h3b_selftest_wait_timeout(0, h3b._stream()) == -3


def test_host_pipeline_matches_device_calls(cuda_dev):
    """Pinned-host streaming with copies overlapped on separate streams gives
    the same tokens as the plain device calls, step by step."""
    wl = TINY
    dm = h3b.dims_of(wl)
    _, blk = make_block(wl, 0, cuda_dev, False)
    ws = h3b.workspace(dm)
    xs = [wlmod.normal_tensor((wl.seq, wl.d), 60 + i, "cpu").pin_memory() for i in range(5)]
    outs = [torch.empty_like(x).pin_memory() for x in xs]
    pipe = h3b.HostPipeline(dm, blk, ws, tuple(xs[0].shape))
    for x, o in zip(xs, outs):
        pipe.submit(x, o)
    pipe.synchronize()
    for x, o in zip(xs, outs):
        ref = x.to(cuda_dev)
        h3b.block_forward(dm, blk, ref, ws)
        torch.cuda.synchronize()
        assert torch.equal(o, ref.cpu())


# ----------------------------------------------------------------------------- next rows: delta unmerge, core reuse
def _identity_blocks(wl, n, dev):
    out = []
    for l in range(n):
        w = wlmod.block_weights(wl, l, dev)
        w["w_o"] = torch.zeros_like(w["w_o"])
        w["w_fc2"] = torch.zeros_like(w["w_fc2"])
        out.append(h3b.Block.from_dict(w))
    return out


def test_unmerge_delta_identity_blocks_bitexact(cuda_dev):
    """Blocks that change nothing: the delta unmerge returns x exactly, the
    plain unmerge returns the pair means."""
    wl = TINY.with_(n_blocks=3)
    dm = h3b.dims_of(wl)
    blocks = _identity_blocks(wl, 3, cuda_dev)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    for delta in (True, False):
        o = h3b.stack_opts(0, 1, unmerge_delta=delta)
        x = x0.clone()
        h3b.stack_forward_ex(dm, blocks, x, h3b.workspace_ex(dm, o), o)
        torch.cuda.synchronize()
        if delta:
            assert torch.equal(x, x0)
        else:
            ref = oracle.token_unmerge(oracle.token_merge(np64(x0), wl), wl).astype(np.float32)
            assert np.array_equal(x.cpu().numpy(), ref)


def test_stack_unmerge_delta_vs_oracle(cuda_dev):
    wl = TINY.with_(n_blocks=5, depth_scaled_init=True, seed=8)
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(5)]
    blocks = [h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    o = h3b.stack_opts(1, 3, unmerge_delta=True)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    x = x0.clone()
    h3b.stack_forward_ex(dm, blocks, x, h3b.workspace_ex(dm, o), o)
    torch.cuda.synchronize()
    ref = oracle.stack_forward_ex(np64(x0), [host_weights(w) for w in ws_], wl, 1, 3, unmerge_delta=True)
    check_bf16(np64(x0), np64(x), ref)


@pytest.mark.parametrize("core_reuse,delta", [(2, False), (4, True), (1, True)])
def test_denoise_core_reuse_vs_oracle(cuda_dev, core_reuse, delta):
    wl = TINY.with_(n_blocks=5, depth_scaled_init=True, seed=9)
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(5)]
    blocks = [h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    o = h3b.stack_opts(2, 3, unmerge_delta=delta, core_first=1, core_last=3)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    x = x0.clone()
    v = torch.empty_like(x)
    nf, nc = h3b.denoise_ex(dm, blocks, x, v, h3b.workspace_ex(dm, o), 6, o, reuse=1, core_reuse=core_reuse)
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    ref, nc_ref = oracle.denoise_core(np64(x0), [host_weights(w) for w in ws_], wl, 6, core_reuse, 1, 3, 2, 3,
                                      unmerge_delta=delta)
    assert nf == 6 and nc == nc_ref
    assert rel_l2(x, ref) <= 1e-2 and max_abs(x, ref) <= 5e-2


def test_denoise_core_counts(cuda_dev):
    wl = TINY.with_(n_blocks=3)
    blocks = [h3b.Block.from_dict(wlmod.block_weights(wl, l, cuda_dev)) for l in range(3)]
    dm = h3b.dims_of(wl)
    o = h3b.stack_opts(core_first=1, core_last=1)
    ws = h3b.workspace_ex(dm, o)
    x = wlmod.initial_tokens(wl, cuda_dev)
    v = torch.empty_like(x)
    got = [h3b.denoise_ex(dm, blocks, x, v, ws, 20, o, core_reuse=r) for r in (1, 4, 6)]
    assert got == [(20, 20), (20, 6), (20, 5)]
    assert [len(oracle.fresh_steps(20, r)) for r in (1, 4, 6)] == [20, 6, 5]


# ----------------------------------------------------------------------------- modulation and condition rows
def rand_mod(shape, seed, dev):
    """Modulation vectors [..., 2, 6, d]: shifts and scales ~ N(0, 0.1), gates ~ 1 + N(0, 0.1)."""
    m = wlmod.normal_tensor(shape, seed, dev, std=0.1)
    m[..., 2, :] += 1.0
    m[..., 5, :] += 1.0
    return m.contiguous()


@pytest.mark.parametrize("int8", [False, True])
def test_modulated_block_with_condition_rows_vs_oracle(cuda_dev, int8):
    wl = TINY
    C = 16
    w, blk = make_block(wl, 0, cuda_dev, int8)
    dm = h3b.dims_of(wl)
    mod = rand_mod((1, 2, 6, wl.d), 40, cuda_dev)
    x0 = wlmod.initial_tokens(wl, cuda_dev, seq=wl.seq + C)
    x = x0.clone()
    o = h3b.stack_opts(n_cond=C, modulation=mod)
    h3b.stack_forward_ex(dm, [blk], x, h3b.workspace_ex(dm, o, h3b.INT8 if int8 else h3b.BF16), o)
    torch.cuda.synchronize()
    hw = host_weights(w)
    ref = oracle.block_forward_cond(np64(x0), oracle.dequant_weights(hw) if int8 else hw, wl, np64(mod[0]), C)
    (check_int8 if int8 else check_bf16)(np64(x0), np64(x), ref)


@pytest.mark.parametrize("int8", [True, False])
def test_identity_modulation_is_bitexact(cuda_dev, int8):
    """Zero shifts and scales with unit gates reproduce the unmodulated stack.
    INT8 blocks normalise in a separate pass either way: bit for bit.  Without
    modulation, bf16 blocks fold their RMSNorms into the neighbouring GEMMs
    (the modulated norm is not a per-row scale and stays a separate pass), so
    the two bf16 runs differ only by where one bf16 rounding of each normed
    GEMM input falls."""
    wl = TINY.with_(n_blocks=3, depth_scaled_init=True, seed=12, dtype=h3b.INT8 if int8 else h3b.BF16)
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(3)]
    blocks = [h3b.Block.quantized(w) if int8 else h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    dt = h3b.INT8 if int8 else h3b.BF16
    ident = torch.zeros((3, 2, 6, wl.d), device=cuda_dev)
    ident[..., 2, :] = 1.0
    ident[..., 5, :] = 1.0
    x = wlmod.initial_tokens(wl, cuda_dev)
    x0 = x.clone()
    y = x.clone()
    o = h3b.stack_opts(0, 1, modulation=ident)
    h3b.stack_forward_ex(dm, blocks, x, h3b.workspace_ex(dm, o, dt), o)
    h3b.stack_forward(dm, blocks, y, h3b.workspace(dm, dt, True), 0, 1)
    torch.cuda.synchronize()
    if int8:
        assert torch.equal(x, y)
    else:
        assert rel_l2(x, y) <= 2e-3 and rel_l2(x - x0, y - x0) <= 1e-2


@pytest.mark.parametrize("delta", [False, True])
def test_condition_stack_with_reduction_vs_oracle(cuda_dev, delta):
    wl = TINY.with_(n_blocks=5, depth_scaled_init=True, seed=13)
    C = 24
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(5)]
    blocks = [h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    mod = rand_mod((5, 2, 6, wl.d), 41, cuda_dev)
    x0 = wlmod.initial_tokens(wl, cuda_dev, seq=wl.seq + C)
    x = x0.clone()
    o = h3b.stack_opts(1, 3, unmerge_delta=delta, n_cond=C, modulation=mod)
    h3b.stack_forward_ex(dm, blocks, x, h3b.workspace_ex(dm, o), o)
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    ref = oracle.stack_forward_cond(np64(x0), [host_weights(w) for w in ws_], wl, np64(mod), C, 1, 3,
                                    unmerge_delta=delta)
    check_bf16(np64(x0), np64(x), ref)


@pytest.mark.parametrize("delta", [False, True])
def test_condition_stack_without_modulation_vs_oracle(cuda_dev, delta):
    """Condition rows without modulation: the RMSNorms are folded into the
    GEMMs over every row, condition rows included (blocks 1..3 on the merged
    grid chain their norm-1 through the previous FC2)."""
    wl = TINY.with_(n_blocks=5, depth_scaled_init=True, seed=15)
    C = 20
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(5)]
    blocks = [h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    x0 = wlmod.initial_tokens(wl, cuda_dev, seq=wl.seq + C)
    x = x0.clone()
    o = h3b.stack_opts(1, 3, unmerge_delta=delta, n_cond=C)
    h3b.stack_forward_ex(dm, blocks, x, h3b.workspace_ex(dm, o), o)
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    ref = oracle.stack_forward_cond(np64(x0), [host_weights(w) for w in ws_], wl, None, C, 1, 3,
                                    unmerge_delta=delta)
    check_bf16(np64(x0), np64(x), ref)


@pytest.mark.parametrize("n_blocks", [1, 3])
def test_folded_norm_width_not_a_multiple_of_256(cuda_dev, n_blocks):
    """d = 384: the residual GEMMs' last 256-column tile holds one valid half,
    whose per-row sums of squares must count as zero in the folded norm."""
    wl = wlmod.Workload("w384", 2, 4, 6, 8, 384, 3, 128, 1536, n_blocks, 0, 16, True)
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(n_blocks)]
    blocks = [h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    x = x0.clone()
    h3b.stack_forward(dm, blocks, x, h3b.workspace(dm))
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    ref = oracle.stack_forward(np64(x0), [host_weights(w) for w in ws_], wl)
    check_bf16(np64(x0), np64(x), ref)


@pytest.mark.parametrize("reuse,core_reuse,per_step", [(2, 1, True), (1, 3, True), (3, 1, False)])
def test_denoise_with_condition_rows_and_modulation_vs_oracle(cuda_dev, reuse, core_reuse, per_step):
    wl = TINY.with_(n_blocks=4, depth_scaled_init=True, seed=14)
    C, steps = 12, 5
    ws_ = [wlmod.block_weights(wl, l, cuda_dev) for l in range(4)]
    blocks = [h3b.Block.from_dict(w) for w in ws_]
    dm = h3b.dims_of(wl)
    mod = rand_mod(((steps,) if per_step else ()) + (4, 2, 6, wl.d), 42, cuda_dev)
    cond = wlmod.normal_tensor((C, wl.d), 43, cuda_dev)
    core = core_reuse > 1
    o = h3b.stack_opts(1, 2, core_first=1 if core else -1, core_last=2 if core else -1, cond_rows=cond,
                       modulation=mod)
    x0 = wlmod.initial_tokens(wl, cuda_dev)
    x = x0.clone()
    v = torch.empty((wl.seq + C, wl.d), device=cuda_dev)
    nf, nc = h3b.denoise_ex(dm, blocks, x, v, h3b.workspace_ex(dm, o), steps, o, reuse=reuse, core_reuse=core_reuse)
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    ref, nf_ref, nc_ref = oracle.denoise_cond(np64(x0), [host_weights(w) for w in ws_], wl, steps, np64(cond),
                                              np64(mod), reuse, 1, 2, core_reuse=core_reuse,
                                              core_first=1 if core else -1, core_last=2 if core else -1)
    assert nf == nf_ref and (not core or nc == nc_ref)
    assert rel_l2(x, ref) <= 1e-2 and max_abs(x, ref) <= 5e-2
