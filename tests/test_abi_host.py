"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/h3b.h declares, and rejects bad arguments before it
touches the device."""
import ctypes

import pytest

import workloads as wlmod

h3b = pytest.importorskip("audio_diffusion_transformer_dit_b200.h3b")


def test_every_header_function_is_exported():
    names = h3b.header_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(h3b.lib, n), n


def test_index_checked_library_exports_the_same_symbols():
    """libh3b_check.so (built beside libh3b.so with -DH3B_CHECK=1) is a drop-in
    for the default library: it loads without a GPU and exports every entry
    point of include/h3b.h."""
    import ctypes
    import os
    path = os.path.join(os.path.dirname(h3b.LIB_PATH), "libh3b_check.so")
    assert os.path.exists(path), "libh3b_check.so not built"
    lib = ctypes.CDLL(path, mode=ctypes.RTLD_LOCAL)
    for n in h3b.header_functions():
        assert hasattr(lib, n), n


def test_status_strings():
    for code in range(0, -9, -1):
        assert h3b.lib.h3b_status_string(code).decode() != "unknown status"
    assert h3b.lib.h3b_status_string(-99).decode() == "unknown status"


def test_seq_len_and_workspace_plan():
    wl = wlmod.WORKLOADS["stack8_d5120_s6528"]
    dm = h3b.dims_of(wl)
    assert h3b.seq_len(dm) == 6528 and h3b.seq_len(dm, True) == 3456
    S, d, f = 6528, 5120, 20480
    ws = h3b.workspace_bytes(dm)
    # aliased arenas: max(qkv+o+u1, u2+g) = max(10dS, 2dS+2fS) bytes, plus scales, the RoPE table and,
    # for the folded RMSNorm, the next block's bf16 QKV input (2dS), two [S, 2 * d/256] partial-sum tables
    # and two [S] row-factor vectors
    arena = max(10 * d * S, 2 * d * S + 2 * f * S)
    folded = 2 * d * S + 2 * S * (2 * d // 256) * 4 + 2 * S * 4
    extra = ws - arena - folded
    assert 0 < extra < 3 * 4 * S + S * 64 * 8 + 12 * 256
    assert h3b.workspace_saved_bytes(dm) == (6 + 2 + 2 + 2) * d * S + 2 * f * S - arena
    wsr = h3b.workspace_bytes(dm, h3b.BF16, True)
    assert wsr - ws >= 3456 * d * 4 + 3456 * 64 * 8
    assert h3b.workspace_bytes(dm, h3b.INT8) > 0


def test_invalid_dims_rejected():
    base = dict(frames=2, rows=2, cols=2, n_audio=1, d=256, n_heads=2, head_dim=128, ffn=1024, eps=1e-6,
                rope_theta=1e4)
    assert h3b.lib.h3b_seq_len(ctypes.byref(h3b.Dims(**base)), 0) == 9
    for bad in (dict(head_dim=96, n_heads=3, d=288), dict(d=384), dict(ffn=1000), dict(eps=-1.0),
                dict(frames=-1), dict(frames=0, n_audio=0)):
        dm = h3b.Dims(**{**base, **bad})
        assert h3b.lib.h3b_seq_len(ctypes.byref(dm), 0) == -1
        assert h3b.lib.h3b_workspace_bytes(ctypes.byref(dm), 0, 0) == 0
    # the largest accepted sizes, and one past each
    for ok, bad in ((dict(d=8192, n_heads=64), dict(d=8320, n_heads=65)),
                    (dict(ffn=32768), dict(ffn=32896)),
                    (dict(frames=1, rows=1, cols=1 << 24, n_audio=0), dict(frames=1, rows=1, cols=1 << 24, n_audio=1))):
        assert h3b.lib.h3b_seq_len(ctypes.byref(h3b.Dims(**{**base, **ok})), 0) > 0
        assert h3b.lib.h3b_seq_len(ctypes.byref(h3b.Dims(**{**base, **bad})), 0) == -1
    odd = h3b.Dims(**{**base, "cols": 3})
    assert h3b.lib.h3b_seq_len(ctypes.byref(odd), 1) == -1
    assert h3b.lib.h3b_workspace_bytes(ctypes.byref(odd), 0, 1) == 0


def _weights(ptr, dtype=0):
    return h3b.BlockWeights(dtype, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr)


# Every call below fails validation on the host; none may reach a launch (the
# pointers are fake), so each case breaks at least one rule.
def test_block_forward_argument_errors_before_device():
    dm = h3b.dims_of(wlmod.WORKLOADS["block_d256_s288"])
    need = h3b.workspace_bytes(dm)
    fake = 1 << 20  # never dereferenced: validation fails first
    w = _weights(fake)
    f = h3b.lib.h3b_block_forward
    assert f(ctypes.byref(dm), ctypes.byref(w), None, 0, fake, need, None) == -1
    assert f(ctypes.byref(dm), ctypes.byref(w), fake + 4, 0, fake, need, None) == -2
    assert f(ctypes.byref(dm), ctypes.byref(w), fake, 0, fake, need - 1, None) == -5
    assert f(ctypes.byref(dm), ctypes.byref(_weights(fake, 7)), fake, 0, fake, need, None) == -4
    assert f(ctypes.byref(dm), ctypes.byref(_weights(fake, 1)), fake, 0, fake, need, None) == -5  # int8 needs more
    bad = h3b.Dims(dm.frames, dm.rows, dm.cols, dm.n_audio, 200, 2, 100, 800, 1e-6, 1e4)
    assert f(ctypes.byref(bad), ctypes.byref(w), fake, 0, fake, need, None) == -3


def test_stack_and_denoise_argument_errors():
    dm = h3b.dims_of(wlmod.WORKLOADS["block_d256_s288"])
    fake = 1 << 20
    arr = (h3b.BlockWeights * 3)(_weights(fake), _weights(fake), _weights(fake))
    need = h3b.workspace_bytes(dm, 0, 1)
    st = h3b.lib.h3b_stack_forward
    assert st(ctypes.byref(dm), arr, 3, 2, 1, fake, fake, need, None) == -3      # last < first
    assert st(ctypes.byref(dm), arr, 3, 1, 3, fake, fake, need, None) == -3      # last beyond stack
    assert st(ctypes.byref(dm), arr, 3, 0, 2, fake, fake, need - 256, None) == -5
    mixed = (h3b.BlockWeights * 2)(_weights(fake, 0), _weights(fake, 1))
    assert st(ctypes.byref(dm), mixed, 2, -1, -1, fake, fake, need, None) == -4
    dn = h3b.lib.h3b_denoise
    assert dn(ctypes.byref(dm), arr, 3, -1, -1, 0, 2, fake, fake, fake, need, None, None) == -3
    assert dn(ctypes.byref(dm), arr, 3, -1, -1, 20, 0, fake, fake, fake, need, None, None) == -3
    assert dn(ctypes.byref(dm), arr, 3, -1, -1, 20, 2, fake, None, fake, need, None, None) == -1


def test_gemm_argument_errors():
    g = h3b.lib.h3b_gemm
    fake = 1 << 20
    assert g(fake, fake, 128, 100, 128, 0, 0, fake, None, None, None, None, None, None, 0, None) == -3   # N % 32
    assert g(fake, fake, 128, 128, 96, 0, 0, fake, None, None, None, None, None, None, 0, None) == -3    # K % 64
    assert g(fake, fake, 128, 128, 64, 1, 0, fake, None, None, None, None, None, None, 0, None) == -3    # int8 K % 128
    assert g(fake, fake, 128, 128, 128, 0, 5, fake, None, None, None, None, None, None, 0, None) == -4   # I32 needs int8
    assert g(fake, fake, 128, 128, 128, 1, 0, fake, None, None, None, None, None, None, 0, None) == -1   # scales
    assert g(fake, fake, 128, 128, 128, 0, 9, fake, None, None, None, None, None, None, 0, None) == -4
    assert g(fake, fake + 8, 128, 128, 128, 0, 0, fake, None, None, None, None, None, None, 0, None) == -2


def test_empty_unit_calls_are_noops_before_device():
    """rows / M / S == 0: nothing is launched and NULL buffers are accepted
    (these return before any CUDA call, so they run without a GPU); the
    remaining arguments are still validated."""
    fake = 1 << 20
    lib = h3b.lib
    assert lib.h3b_quantize_weights(None, 0, 256, None, None, None) == 0
    assert lib.h3b_quantize_weights(None, 0, 250, None, None, None) == -3                 # k % 8
    assert lib.h3b_quantize_rows_absmax(None, None, 0, 1024, None, None, None) == 0
    assert lib.h3b_rmsnorm(None, None, 0, 256, 1e-6, None, None, h3b.BF16, None) == 0
    assert lib.h3b_rmsnorm(None, None, 0, 256, 1e-6, None, None, 7, None) == -4          # dtype
    assert lib.h3b_gemm(None, fake, 0, 128, 128, 0, 1, None, None, None, None, None, None, None, 0, None) == 0
    assert lib.h3b_gemm(None, fake, 0, 100, 128, 0, 1, None, None, None, None, None, None, None, 0, None) == -3
    assert lib.h3b_gemm(None, None, 0, 128, 128, 0, 1, None, None, None, None, None, None, None, 0, None) == -1
    assert lib.h3b_attention(None, 0, 4, 128, None, None, 0, None) == 0
    assert lib.h3b_attention(None, 0, 4, 96, None, None, 0, None) == -3                   # head_dim
    assert lib.h3b_flow_step(None, None, 0.5, 0.4, 0, None, None) == 0


def test_extended_options_argument_errors():
    dm = h3b.dims_of(wlmod.WORKLOADS["block_d256_s288"])
    fake = 1 << 20
    arr = (h3b.BlockWeights * 4)(*[_weights(fake) for _ in range(4)])
    dn = h3b.lib.h3b_denoise_ex
    o = h3b.stack_opts(core_first=1, core_last=2)
    need = h3b.lib.h3b_workspace_bytes_ex(ctypes.byref(dm), 0, ctypes.byref(o))
    assert need > h3b.workspace_bytes(dm)                                       # + cached core update
    # core reuse excludes whole-velocity reuse
    assert dn(ctypes.byref(dm), arr, 4, ctypes.byref(o), 20, 2, 4, fake, fake, fake, need, None, None, None) == -3
    # the reduction window partly overlapping the core window
    o2 = h3b.stack_opts(0, 1, core_first=1, core_last=2)
    need2 = h3b.lib.h3b_workspace_bytes_ex(ctypes.byref(dm), 0, ctypes.byref(o2))
    assert dn(ctypes.byref(dm), arr, 4, ctypes.byref(o2), 20, 1, 4, fake, fake, fake, need2, None, None, None) == -3
    # core window past the stack
    o3 = h3b.stack_opts(core_first=2, core_last=4)
    assert dn(ctypes.byref(dm), arr, 4, ctypes.byref(o3), 20, 1, 4, fake, fake, fake, need, None, None, None) == -3
    # workspace without room for the cached update
    small = h3b.workspace_bytes(dm)
    assert dn(ctypes.byref(dm), arr, 4, ctypes.byref(o), 20, 1, 4, fake, fake, fake, small, None, None, None) == -5
    assert h3b.lib.h3b_stack_forward_ex(ctypes.byref(dm), arr, 4, None, fake, fake, need, None) == -1


def test_condition_rows_and_modulation_argument_errors():
    """Every case here fails validation before anything is launched."""
    dm = h3b.dims_of(wlmod.WORKLOADS["block_d256_s288"])
    fake = 1 << 20
    arr = (h3b.BlockWeights * 4)(*[_weights(fake) for _ in range(4)])
    dn, sf = h3b.lib.h3b_denoise_ex, h3b.lib.h3b_stack_forward_ex
    wsx = h3b.lib.h3b_workspace_bytes_ex

    def opts(**kw):
        o = h3b.StackOpts(-1, -1, 0, -1, -1, 0, 0, None, None)
        for k, v in kw.items():
            setattr(o, k, v)
        return ctypes.byref(o)

    D = ctypes.byref(dm)
    need = wsx(D, 0, opts(n_cond=8))
    assert need > h3b.workspace_bytes(dm)                            # room for the condition rows
    assert wsx(D, 0, opts(n_cond=-1)) == 0
    assert sf(D, arr, 4, opts(n_cond=-1), fake, fake, need, None) == -3
    assert sf(D, arr, 4, opts(modulation=fake + 4, mod_steps=1), fake, fake, need, None) == -2
    assert sf(D, arr, 4, opts(modulation=fake, mod_steps=0), fake, fake, need, None) == -3
    # per-step slices must number 1 or n_steps
    assert dn(D, arr, 4, opts(modulation=fake, mod_steps=3), 20, 1, 1, fake, fake, fake, need, None, None,
              None) == -3
    # condition rows without their values, or misaligned
    assert dn(D, arr, 4, opts(n_cond=8), 20, 1, 1, fake, fake, fake, need, None, None, None) == -1
    assert dn(D, arr, 4, opts(n_cond=8, cond_rows=fake + 8), 20, 1, 1, fake, fake, fake, need, None, None,
              None) == -2
    # workspace sized without the condition rows
    assert sf(D, arr, 4, opts(n_cond=8), fake, fake, h3b.workspace_bytes(dm), None) == -5
