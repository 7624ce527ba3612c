"""Kernel-level parity: each h3b kernel, called through the C ABI, against the
CPU oracle on the same seeded inputs (ragged tails and several tiles)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wlmod
from tests._util import np64, rel_l2, max_abs, ulp_diff_f32

pytestmark = pytest.mark.gpu

h3b = pytest.importorskip("audio_diffusion_transformer_dit_b200.h3b")


def small_dims(F=2, H=4, W=6, A=5, d=256, heads=4, ffn=1024):
    return wlmod.Workload("t", F, H, W, A, d, heads, d // heads, ffn, 1, 0, 0, False)


# ----------------------------------------------------------------------------- Euler step
@pytest.mark.parametrize("n", [0, 1, 7, 4096, 1_000_003])
def test_flow_step(cuda_dev, n):
    x = wlmod.normal_tensor((n,), 1, cuda_dev)
    v = wlmod.normal_tensor((n,), 2, cuda_dev)
    x0 = x.clone()
    cp = torch.full_like(x, 7.0)
    s0, s1 = np.float32(0.65), np.float32(0.6)
    h3b.flow_step(x, v, float(s0), float(s1), x_copy=cp)
    torch.cuda.synchronize()
    ref = oracle.flow_step(np64(x0), np64(v), s0, s1).astype(np.float32)
    got = x.cpu().numpy()
    assert np.all(ulp_diff_f32(got, ref) <= 1)
    assert np.array_equal(cp.cpu().numpy(), got)


def test_flow_step_zero_velocity_identity(cuda_dev):
    x = wlmod.normal_tensor((12345,), 3, cuda_dev)
    x0 = x.clone()
    h3b.flow_step(x, torch.zeros_like(x), 0.9, 0.85)
    assert torch.equal(x, x0)


# ----------------------------------------------------------------------------- token reduction
@pytest.mark.parametrize("geom", [(2, 3, 4, 5, 128), (6, 32, 32, 384, 256), (1, 1, 2, 0, 128), (5, 48, 84, 480, 5120)])
def test_merge_unmerge_bitexact(cuda_dev, geom):
    F, H, W, A, d = geom
    wl = wlmod.Workload("g", F, H, W, A, d, d // 128, 128, 4 * d, 1, 0, 0, False)
    dm = h3b.dims_of(wl)
    x = wlmod.normal_tensor((F * H * W + A, d), 4, cuda_dev) * 3.0
    xm = torch.empty((F * H * W // 2 + A, d), dtype=torch.float32, device=cuda_dev)
    h3b.token_merge(dm, x, xm)
    torch.cuda.synchronize()
    ref = oracle.token_merge(np64(x), wl)
    assert np.array_equal(xm.cpu().numpy(), ref.astype(np.float32))
    back = torch.empty_like(x)
    h3b.token_unmerge(dm, xm, back)
    torch.cuda.synchronize()
    assert np.array_equal(back.cpu().numpy(), oracle.token_unmerge(ref, wl).astype(np.float32))


@pytest.mark.parametrize("geom", [(5, 48, 84, 480, 128), (2, 3, 4, 5, 256)])
def test_unmerge_delta_bitexact(cuda_dev, geom):
    """x_pre + (ym - xm0) broadcast: on values that are multiples of 2^-10
    below 2^8 in magnitude the fp32 subtraction and addition are exact, so the
    kernel equals the fp64 oracle bit for bit; audio rows are copied from ym."""
    F, H, W, A, d = geom
    wl = wlmod.Workload("g", F, H, W, A, d, d // 128, 128, 4 * d, 1, 0, 0, False)
    dm = h3b.dims_of(wl)
    S, Sm = F * H * W + A, F * H * W // 2 + A

    def grid(shape, seed):
        return torch.round(wlmod.normal_tensor(shape, seed, cuda_dev) * 1024.0 * 8.0) / 1024.0

    x = grid((S, d), 70)
    ym, xm0 = grid((Sm, d), 71), grid((Sm, d), 72)
    ref = oracle.token_unmerge_delta(np64(x), np64(ym), np64(xm0), wl)
    h3b.token_unmerge_delta(dm, x, ym, xm0)
    torch.cuda.synchronize()
    assert np.array_equal(x.cpu().numpy(), ref.astype(np.float32))


def test_merge_rejects_odd_width(cuda_dev):
    wl = wlmod.Workload("g", 2, 3, 5, 1, 128, 1, 128, 512, 1, 0, 0, False)
    x = torch.zeros((31, 128), device=cuda_dev)
    xm = torch.zeros((31, 128), device=cuda_dev)
    with pytest.raises(h3b.H3bError) as e:
        h3b.token_merge(h3b.dims_of(wl), x, xm)
    assert e.value.status == -3


def test_merge_unmerge_identity_pair_constant(cuda_dev):
    wl = small_dims(3, 4, 8, 7, 256, 2, 1024)
    dm = h3b.dims_of(wl)
    m = wlmod.normal_tensor((h3b.seq_len(dm, True), 256), 5, cuda_dev)
    x = torch.empty((h3b.seq_len(dm), 256), dtype=torch.float32, device=cuda_dev)
    h3b.token_unmerge(dm, m, x)
    m2 = torch.empty_like(m)
    h3b.token_merge(dm, x, m2)
    x2 = torch.empty_like(x)
    h3b.token_unmerge(dm, m2, x2)
    assert torch.equal(m2, m) and torch.equal(x2, x)


# ----------------------------------------------------------------------------- RoPE table
@pytest.mark.parametrize("merged", [False, True])
@pytest.mark.parametrize("hd", [64, 128])
def test_rope_table(cuda_dev, merged, hd):
    wl = small_dims(3, 5, 84, 37, 2 * hd, 2, 8 * hd)
    dm = h3b.dims_of(wl)
    tab = h3b.rope_table(dm, merged)
    torch.cuda.synchronize()
    ang = oracle.rope_angles(wl, merged)
    t = tab.cpu().double().numpy()
    assert t.shape[:2] == ang.shape
    assert np.max(np.abs(t[..., 0] - np.cos(ang))) < 1e-6
    assert np.max(np.abs(t[..., 1] - np.sin(ang))) < 1e-6


# ----------------------------------------------------------------------------- RMSNorm
@pytest.mark.parametrize("rows,d", [(1, 128), (37, 256), (300, 3072), (129, 5120), (3, 8192), (10000, 1024)])
def test_rmsnorm_bf16(cuda_dev, rows, d):
    x = wlmod.normal_tensor((rows, d), 6, cuda_dev) * 2.0
    g = wlmod.uniform_tensor((d,), 7, cuda_dev, 0.5, 1.5)
    u = h3b.rmsnorm(x, g, 1e-6)
    torch.cuda.synchronize()
    ref = oracle.rmsnorm(np64(x), np64(g), 1e-6)
    # one bf16 rounding of an fp32 value: relative error <= 2^-8
    assert np.all(np.abs(np64(u) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)


@pytest.mark.parametrize("rows,d", [(37, 256), (300, 5120), (7, 4096), (7, 6144), (10000, 1024), (5, 8192)])
def test_rmsnorm_int8(cuda_dev, rows, d):
    x = wlmod.normal_tensor((rows, d), 8, cuda_dev)
    g = torch.ones(d, device=cuda_dev)
    q, s = h3b.rmsnorm(x, g, 1e-6, int8=True)
    torch.cuda.synchronize()
    u = oracle.rmsnorm(np64(x), np.ones(d), 1e-6)
    qr, sr = oracle.quantize_rows(u)
    # the kernel's u is fp32 arithmetic, the oracle's fp64: scales agree to fp32
    # rounding, codes agree except at rare near-ties (never by more than 1)
    assert np.allclose(s.cpu().numpy(), sr, rtol=1e-6)
    dq = np.abs(q.cpu().numpy().astype(int) - qr.astype(int))
    assert dq.max() <= 1 and (dq > 0).mean() < 1e-3


# ----------------------------------------------------------------------------- quantisation
# rows of up to 32 KB (k <= 16384) stream through shared memory, ragged at
# 1032 and 6152, many rows per CTA at 12000 x 512; wider rows (20480, 32768)
# take the one-CTA-per-row register kernel
@pytest.mark.parametrize("rows,k", [(1, 8), (33, 256), (300, 5120), (17, 20480), (5, 32768), (37, 1024), (9, 1032),
                                    (41, 6144), (6, 6152), (12000, 512), (3, 16384)])
def test_quantize_weights_bitexact(cuda_dev, rows, k):
    w = (wlmod.normal_tensor((rows, k), 9, cuda_dev) * 0.02).to(torch.bfloat16)
    w[0, :] = 0  # zero row -> s = 0, q = 0
    q, s = h3b.quantize_weights(w)
    torch.cuda.synchronize()
    qr, sr = oracle.quantize_rows(w.float().cpu().numpy())
    assert np.array_equal(s.cpu().numpy(), sr)
    assert np.array_equal(q.cpu().numpy(), qr)


# one CTA per row for k a multiple of 16 up to 32768 (1..8 groups of 16 per
# thread, ragged at 12304); the 2-D grid path for k a multiple of 8 only
@pytest.mark.parametrize("rows,k", [(77, 1024), (13, 12288), (5, 20480), (3, 32768), (4, 12304), (6, 1000)])
def test_quantize_rows_absmax_bitexact(cuda_dev, rows, k):
    a = (wlmod.normal_tensor((rows, k), 10, cuda_dev) * 3).to(torch.bfloat16)
    amax = a.float().abs().amax(dim=1).contiguous()
    q, s = h3b.quantize_rows_absmax(a, amax)
    torch.cuda.synchronize()
    qr, sr = oracle.quantize_rows(a.float().cpu().numpy())
    assert np.array_equal(s.cpu().numpy(), sr) and np.array_equal(q.cpu().numpy(), qr)


def test_quantize_rows_absmax_below_true_max_bitexact(cuda_dev):
    """A caller-given row maximum smaller than the row's true maximum (half,
    a quarter) and a zero maximum: values beyond it clamp to +-127, the rest
    round as usual, bit for bit with the oracle's known-max rule."""
    rows, k = 24, 2048
    a = (wlmod.normal_tensor((rows, k), 12, cuda_dev) * 2).to(torch.bfloat16)
    true_max = a.float().abs().amax(dim=1)
    frac = torch.tensor([1.0, 0.5, 0.25, 0.0] * (rows // 4), device=cuda_dev)
    amax = (true_max * frac).contiguous()
    q, s = h3b.quantize_rows_absmax(a, amax)
    torch.cuda.synchronize()
    qr, sr = oracle.quantize_rows_known_max(a.float().cpu().numpy(), amax.cpu().numpy())
    assert np.array_equal(s.cpu().numpy(), sr) and np.array_equal(q.cpu().numpy(), qr)
    assert (np.abs(qr[1::4]) == 127).sum() > 0 and (qr[3::4] == 0).all()  # clamping and zero rows really occurred


# ----------------------------------------------------------------------------- GEMM
GEMM_SHAPES = [(1, 256, 64), (300, 768, 512), (129, 288, 1024), (1000, 1536, 3072), (6528, 512, 128)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_bf16_f32(cuda_dev, M, N, K):
    A = wlmod.normal_tensor((M, K), 11, cuda_dev, dtype=torch.bfloat16)
    B = wlmod.normal_tensor((N, K), 12, cuda_dev, 0.02, dtype=torch.bfloat16)
    C = torch.full((M, N), float("nan"), device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_F32, C)
    torch.cuda.synchronize()
    ref = oracle.linear(np64(A), np64(B))
    assert np.isfinite(C.cpu().numpy()).all()
    # fp32 accumulation of exact bf16 products
    assert max_abs(C, ref) <= 2e-5 * np.sqrt(K) * np.abs(ref).max() + 1e-6
    assert rel_l2(C, ref) < 1e-5


@pytest.mark.parametrize("M,N,K", [(1, 256, 128), (300, 512, 1024), (129, 288, 2048), (700, 1024, 5120)])
def test_gemm_int8_i32_bitexact(cuda_dev, M, N, K):
    A = wlmod.int8_tensor((M, K), 13, cuda_dev)
    B = wlmod.int8_tensor((N, K), 14, cuda_dev)
    C = torch.zeros((M, N), dtype=torch.int32, device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_I32, C)
    torch.cuda.synchronize()
    ref = oracle.int8_matmul(A.cpu().numpy(), B.cpu().numpy())
    assert np.array_equal(C.cpu().numpy().astype(np.int64), ref)


def test_gemm_int8_extremes_bitexact(cuda_dev):
    K = 4096
    A = torch.full((130, K), 127, dtype=torch.int8, device=cuda_dev)
    A[1::2] = -127
    B = torch.full((256, K), -127, dtype=torch.int8, device=cuda_dev)
    C = torch.zeros((130, 256), dtype=torch.int32, device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_I32, C)
    torch.cuda.synchronize()
    ref = oracle.int8_matmul(A.cpu().numpy(), B.cpu().numpy())
    assert np.array_equal(C.cpu().numpy().astype(np.int64), ref)


def test_gemm_int8_dequant(cuda_dev):
    M, N, K = 300, 512, 1024
    A = wlmod.int8_tensor((M, K), 15, cuda_dev)
    B = wlmod.int8_tensor((N, K), 16, cuda_dev)
    sa = wlmod.uniform_tensor((M,), 17, cuda_dev, 0.001, 0.01)
    sb = wlmod.uniform_tensor((N,), 18, cuda_dev, 0.001, 0.01)
    C = torch.empty((M, N), device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_F32, C, scale_a=sa, scale_b=sb)
    torch.cuda.synchronize()
    acc = oracle.int8_matmul(A.cpu().numpy(), B.cpu().numpy()).astype(np.float64)
    ref = acc * np64(sa)[:, None] * np64(sb)[None, :]
    assert rel_l2(C, ref) < 1e-6


@pytest.mark.parametrize("int8", [False, True])
def test_gemm_resid_and_gelu(cuda_dev, int8):
    M, N, K = 333, 768, 1024
    if int8:
        A, B = wlmod.int8_tensor((M, K), 19, cuda_dev), wlmod.int8_tensor((N, K), 20, cuda_dev)
        sa = wlmod.uniform_tensor((M,), 21, cuda_dev, 0.001, 0.003)
        sb = wlmod.uniform_tensor((N,), 22, cuda_dev, 0.001, 0.003)
        acc = oracle.int8_matmul(A.cpu().numpy(), B.cpu().numpy()) * np64(sa)[:, None] * np64(sb)[None, :]
    else:
        A = wlmod.normal_tensor((M, K), 19, cuda_dev, dtype=torch.bfloat16)
        B = wlmod.normal_tensor((N, K), 20, cuda_dev, 0.05, dtype=torch.bfloat16)
        sa = sb = None
        acc = oracle.linear(np64(A), np64(B))
    x = wlmod.normal_tensor((M, N), 23, cuda_dev)
    x0 = np64(x)
    h3b.gemm(A, B, h3b.EPI_RESID, x, scale_a=sa, scale_b=sb)
    g = torch.empty((M, N), dtype=torch.bfloat16, device=cuda_dev)
    amax = torch.zeros(M, device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_GELU, g, scale_a=sa, scale_b=sb, row_absmax=amax if int8 else None)
    torch.cuda.synchronize()
    assert rel_l2(np64(x) - x0, acc) < 1e-5
    ref_g = oracle.gelu(acc)
    assert np.all(np.abs(np64(g) - ref_g) <= 2.0 ** -8 * np.abs(ref_g) + 1e-5 * np.abs(acc).max())
    if int8:
        assert np.array_equal(amax.cpu().numpy(), g.float().abs().amax(dim=1).cpu().numpy())


@pytest.mark.parametrize("int8", [False, True])
@pytest.mark.parametrize("hd,merged", [(64, False), (128, False), (128, True)])
def test_gemm_qkv_rope(cuda_dev, int8, hd, merged):
    wl = small_dims(2, 4, 6, 19, 2 * hd, 2, 8 * hd)
    dm = h3b.dims_of(wl)
    S, d = h3b.seq_len(dm, merged), wl.d
    tab = h3b.rope_table(dm, merged)
    if int8:
        A, B = wlmod.int8_tensor((S, d), 24, cuda_dev), wlmod.int8_tensor((3 * d, d), 25, cuda_dev)
        sa = wlmod.uniform_tensor((S,), 26, cuda_dev, 0.001, 0.003)
        sb = wlmod.uniform_tensor((3 * d,), 27, cuda_dev, 0.001, 0.003)
        acc = oracle.int8_matmul(A.cpu().numpy(), B.cpu().numpy()) * np64(sa)[:, None] * np64(sb)[None, :]
    else:
        A = wlmod.normal_tensor((S, d), 24, cuda_dev, dtype=torch.bfloat16)
        B = wlmod.normal_tensor((3 * d, d), 25, cuda_dev, 0.05, dtype=torch.bfloat16)
        sa = sb = None
        acc = oracle.linear(np64(A), np64(B))
    C = torch.empty((S, 3 * d), dtype=torch.bfloat16, device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_QKV_ROPE, C, scale_a=sa, scale_b=sb, rope=tab, dims=dm)
    torch.cuda.synchronize()
    ang = oracle.rope_angles(wl, merged)
    ref = np.concatenate([oracle.apply_rope(acc[:, :d], ang, 2), oracle.apply_rope(acc[:, d:2 * d], ang, 2),
                          acc[:, 2 * d:]], axis=1)
    assert np.all(np.abs(np64(C) - ref) <= 2.0 ** -8 * np.abs(ref) + 2e-5 * np.abs(ref).max())


# ----------------------------------------------------------------------------- attention
@pytest.mark.parametrize("S,H,D", [(1, 1, 64), (100, 2, 64), (128, 2, 128), (288, 4, 64), (1000, 3, 128),
                                   (2049, 2, 128)])
def test_attention(cuda_dev, S, H, D):
    qkv = wlmod.normal_tensor((S, 3 * H * D), 28, cuda_dev, 1.5, dtype=torch.bfloat16)
    o = h3b.attention(qkv, H, D)
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    q = np64(qkv)
    d = H * D
    ref = oracle.attention(q[:, :d], q[:, d:2 * d], q[:, 2 * d:], H)
    assert np.isfinite(np64(o)).all()
    assert rel_l2(o, ref) < 1e-2
    assert max_abs(o, ref) < 3e-2


def test_attention_large_scores(cuda_dev):
    """Growing row maxima across key tiles exercise the lazy O rescale."""
    S, H, D = 700, 2, 128
    g = torch.Generator(device="cpu").manual_seed(3)
    qkv = torch.randn((S, 3 * H * D), generator=g) * 0.3
    qkv[:, :H * D] *= 6.0
    ramp = torch.linspace(0.2, 4.0, S)[:, None]
    qkv[:, H * D:2 * H * D] *= ramp  # later keys have larger norms -> maxima grow along the sweep
    qkv = qkv.to(torch.bfloat16).to(cuda_dev)
    o = h3b.attention(qkv, H, D)
    torch.cuda.synchronize()
    q = np64(qkv)
    d = H * D
    ref = oracle.attention(q[:, :d], q[:, d:2 * d], q[:, 2 * d:], H)
    assert rel_l2(o, ref) < 1e-2


def test_gelu_accuracy(cuda_dev):
    """The GEMM epilogue's GELU against the exact-erf form in fp64.  Budget:
    Abramowitz & Stegun 7.1.26 is within 1.5e-7 of erfc, i.e. 0.75e-7 * |x| in
    GELU; the fp32 evaluation adds a few ulp of erfc/2 (< 0.5) and of the
    result -- together below 2e-7 * |x| + 1e-6 * |GELU(x)|."""
    x = torch.cat([torch.linspace(-12.0, 12.0, 200001), wlmod.normal_tensor((100000,), 50, "cpu") * 4.0,
                   torch.tensor([0.0, -0.0, 1e-30, -1e-30, 30.0, -30.0, 3e4, -3e4])]).float().to(cuda_dev)
    y = h3b.gelu(x)
    torch.cuda.synchronize()
    xr = np64(x)
    ref = oracle.gelu(xr)
    err = np.abs(np64(y) - ref)
    assert np.all(err <= 2e-7 * np.abs(xr) + 1e-6 * np.abs(ref))
    assert np.all(np64(y)[xr >= 0] >= 0) and np.all(np64(y)[xr < 0] <= 0)


def test_exp2_poly_error_bound(cuda_dev):
    """The FMA-pipe exp2 of the attention kernel against 2^x in fp64."""
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001), torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0, 7.5])])
    x = x.float().to(cuda_dev)
    y = h3b.exp2_poly(x)
    torch.cuda.synchronize()
    ref = np.exp2(np64(x))
    rel = np.abs(np64(y) - ref) / ref
    assert rel.max() < 1e-4
    assert np64(h3b.exp2_poly(torch.tensor([-300.0, -126.0], device=cuda_dev))).max() < 2.0 ** -125


@pytest.mark.parametrize("ktail", [False, True])
@pytest.mark.parametrize("int8", [False, True])
def test_gemm_resid_split_tail(cuda_dev, int8, ktail):
    """A residual GEMM with a nearly empty last wave (300 pair tiles) splits its
    tail tiles along K; with and without scratch it matches the oracle, and two
    split runs agree bit for bit.  ktail: K ends on a half stage."""
    M, N = 6400, 3072
    K = (1152 if int8 else 1088) if ktail else 1024
    if int8:
        A, B = wlmod.int8_tensor((M, K), 31, cuda_dev), wlmod.int8_tensor((N, K), 32, cuda_dev)
        sa = wlmod.uniform_tensor((M,), 33, cuda_dev, 0.001, 0.003)
        sb = wlmod.uniform_tensor((N,), 34, cuda_dev, 0.001, 0.003)
        acc = (A.double() @ B.double().T).cpu().numpy() * np64(sa)[:, None] * np64(sb)[None, :]
    else:
        A = wlmod.normal_tensor((M, K), 31, cuda_dev, dtype=torch.bfloat16)
        B = wlmod.normal_tensor((N, K), 32, cuda_dev, 0.05, dtype=torch.bfloat16)
        sa = sb = None
        acc = oracle.linear(np64(A), np64(B))
    x0 = wlmod.normal_tensor((M, N), 35, cuda_dev)
    scratch = torch.empty(64 << 20, dtype=torch.uint8, device=cuda_dev)
    outs = []
    for sc in (None, scratch, scratch):
        x = x0.clone()
        h3b.gemm(A, B, h3b.EPI_RESID, x, scale_a=sa, scale_b=sb, scratch=sc)
        torch.cuda.synchronize()
        outs.append(x)
        assert rel_l2(np64(x) - np64(x0), acc) < 1e-5
    assert torch.equal(outs[1], outs[2])
    assert rel_l2(outs[1], outs[0]) < 1e-6


@pytest.mark.parametrize("S,H,D", [(6400, 24, 128), (6528, 40, 128), (3000, 52, 64)])
def test_attention_key_split_tail(cuda_dev, S, H, D):
    """Work-item counts whose last wave is nearly empty (e.g. 600 items on 148
    SMs) split the tail items along the keys: same result with and without the
    split (within bf16 rounding), bit-identical across runs, and sampled rows
    agree with the oracle."""
    qkv = wlmod.normal_tensor((S, 3 * H * D), 36, cuda_dev, 1.5, dtype=torch.bfloat16)
    scratch = torch.empty(64 << 20, dtype=torch.uint8, device=cuda_dev)
    o_plain = h3b.attention(qkv, H, D)
    o_split = h3b.attention(qkv, H, D, scratch=scratch)
    o_again = h3b.attention(qkv, H, D, scratch=scratch)
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    assert torch.equal(o_split, o_again)
    assert rel_l2(o_split, o_plain) < 4e-3
    rows = np.unique(np.concatenate([np.arange(S - 300, S), np.linspace(0, S - 1, 64).astype(int)]))
    q = np64(qkv)
    d = H * D
    ref = oracle.attention(q[rows, :d], q[:, d:2 * d], q[:, 2 * d:], H)
    assert rel_l2(np64(o_split)[rows], ref) < 1e-2


# shapes whose 256x256 tiles fill a wave of CTA pairs -> the 2-SM (cta_group::2) kernel
# the last two end K on a half stage (one 128-byte atom of the two a pair stage holds)
PAIR_SHAPES = [(2048, 2560, 1024), (2100, 2592, 512), (6528, 3072, 256), (2048, 2560, 192), (2100, 2592, 64)]


@pytest.mark.parametrize("M,N,K", PAIR_SHAPES)
def test_gemm_pair_bf16(cuda_dev, M, N, K):
    A = wlmod.normal_tensor((M, K), 41, cuda_dev, dtype=torch.bfloat16)
    B = wlmod.normal_tensor((N, K), 42, cuda_dev, 0.02, dtype=torch.bfloat16)
    C = torch.full((M, N), float("nan"), device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_F32, C)
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    ref = oracle.linear(np64(A), np64(B))
    assert np.isfinite(C.cpu().numpy()).all()
    assert rel_l2(C, ref) < 1e-5


@pytest.mark.parametrize("M,N,K", PAIR_SHAPES)
def test_gemm_pair_int8_i32_bitexact(cuda_dev, M, N, K):
    K = K if K % 128 == 0 else 2 * K  # int8 K steps are 128 wide: 192 -> 384 (1.5 stages), 64 -> 128
    A = wlmod.int8_tensor((M, K), 43, cuda_dev)
    B = wlmod.int8_tensor((N, K), 44, cuda_dev)
    C = torch.zeros((M, N), dtype=torch.int32, device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_I32, C)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(0, 8), np.arange(120, 136), np.arange(M - 140, M),
                                     np.linspace(0, M - 1, 40).astype(int)]))
    ref = oracle.int8_matmul(A.cpu().numpy()[rows], B.cpu().numpy())
    assert np.array_equal(C.cpu().numpy()[rows].astype(np.int64), ref)


@pytest.mark.parametrize("int8", [False, True])
def test_gemm_pair_epilogues(cuda_dev, int8):
    """RoPE, GELU(+row max) and residual epilogues on the pair kernel."""
    wl = wlmod.Workload("p", 4, 16, 30, 100, 1024, 8, 128, 4096, 1, 0, 0, False)  # S = 2020
    dm = h3b.dims_of(wl)
    S, d = h3b.seq_len(dm), wl.d
    tab = h3b.rope_table(dm)
    if int8:
        A, B = wlmod.int8_tensor((S, d), 45, cuda_dev), wlmod.int8_tensor((3 * d, d), 46, cuda_dev)
        sa = wlmod.uniform_tensor((S,), 47, cuda_dev, 0.001, 0.003)
        sb = wlmod.uniform_tensor((3 * d,), 48, cuda_dev, 0.001, 0.003)
        acc = (A.double() @ B.double().T).cpu().numpy() * np64(sa)[:, None] * np64(sb)[None, :]
    else:
        A = wlmod.normal_tensor((S, d), 45, cuda_dev, dtype=torch.bfloat16)
        B = wlmod.normal_tensor((3 * d, d), 46, cuda_dev, 0.05, dtype=torch.bfloat16)
        sa = sb = None
        acc = oracle.linear(np64(A), np64(B))
    C = torch.empty((S, 3 * d), dtype=torch.bfloat16, device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_QKV_ROPE, C, scale_a=sa, scale_b=sb, rope=tab, dims=dm)
    G = torch.empty((S, 3 * d), dtype=torch.bfloat16, device=cuda_dev)
    amax = torch.zeros(S, device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_GELU, G, scale_a=sa, scale_b=sb, row_absmax=amax if int8 else None)
    X0 = wlmod.normal_tensor((S, 3 * d), 49, cuda_dev)
    X = X0.clone()
    h3b.gemm(A, B, h3b.EPI_RESID, X, scale_a=sa, scale_b=sb)
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    ang = oracle.rope_angles(wl)
    ref = np.concatenate([oracle.apply_rope(acc[:, :d], ang, 8), oracle.apply_rope(acc[:, d:2 * d], ang, 8),
                          acc[:, 2 * d:]], axis=1)
    assert np.all(np.abs(np64(C) - ref) <= 2.0 ** -8 * np.abs(ref) + 2e-5 * np.abs(ref).max())
    ref_g = oracle.gelu(acc)
    assert np.all(np.abs(np64(G) - ref_g) <= 2.0 ** -8 * np.abs(ref_g) + 1e-5 * np.abs(acc).max())
    if int8:
        assert np.array_equal(amax.cpu().numpy(), G.float().abs().amax(dim=1).cpu().numpy())
    assert rel_l2(np64(X) - np64(X0), acc) < 1e-5


def test_quantize_ties_and_near_ties_bitexact(cuda_dev):
    """Rows scaled so that v/s is an exact half-integer (round-half-even ties),
    plus the neighbouring bf16 values on either side, through both row
    quantisation kernels: codes and scales equal the oracle's bit for bit."""
    rows = []
    for k in range(0, 6):                       # s = 2^-k exactly (row max 127 * 2^-k)
        sc = 2.0 ** -k
        halves = (np.arange(-127, 127) + 0.5) * sc
        rows.append(np.concatenate([[127 * sc], halves]))
    base = np.stack([r[:255] for r in rows]).astype(np.float32)
    t = torch.tensor(base).to(torch.bfloat16)
    bits = t.view(torch.int16)
    nb_up = (bits + 1).view(torch.bfloat16)
    nb_dn = (bits - 1).view(torch.bfloat16)
    nb_up[:, 0] = t[:, 0]
    nb_dn[:, 0] = t[:, 0]
    w = torch.cat([t, nb_up, nb_dn], dim=0)
    w = torch.cat([w, torch.zeros((w.shape[0], 1), dtype=torch.bfloat16)], dim=1)  # k = 256
    w = w.contiguous().to(cuda_dev)
    q, s = h3b.quantize_weights(w)
    amax = w.float().abs().amax(dim=1).contiguous()
    q2, s2 = h3b.quantize_rows_absmax(w, amax)
    torch.cuda.synchronize()
    qr, sr = oracle.quantize_rows(w.float().cpu().numpy())
    assert np.array_equal(s.cpu().numpy(), sr) and np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(s2.cpu().numpy(), sr) and np.array_equal(q2.cpu().numpy(), qr)
    assert set(np.abs(qr[0, 1:255]).tolist()) >= {0, 2, 126}  # half-even ties really occurred


# ----------------------------------------------------------------------------- maximum sizes
@pytest.mark.parametrize("M,N,K", [(130, 24576, 256), (130, 2048, 32768)])
def test_gemm_int8_max_sizes_extremes_bitexact(cuda_dev, M, N, K):
    """The largest operands the API accepts: N = 3 d at d = 8192 (QKV) and
    K = f = 32768 (FC2).  Codes of +-127 drive every int32 accumulator to
    +-127^2 K = 528,482,304 at K = 32768, still inside int32."""
    A = torch.full((M, K), 127, dtype=torch.int8, device=cuda_dev)
    A[1::2] = -127
    B = wlmod.int8_tensor((N, K), 60, cuda_dev)
    B[:64] = 127
    C = torch.zeros((M, N), dtype=torch.int32, device=cuda_dev)
    h3b.gemm(A, B, h3b.EPI_I32, C)
    torch.cuda.synchronize()
    ref = oracle.int8_matmul(A.cpu().numpy(), B.cpu().numpy())
    assert np.abs(ref).max() == 127 * 127 * K
    assert np.array_equal(C.cpu().numpy().astype(np.int64), ref)


def test_gemm_bf16_residual_max_k(cuda_dev):
    """FC2 at the largest MLP width (K = 32768) with the residual epilogue.
    The bf16 products are exact; the fp32 accumulation error grows like
    sqrt(K) (the K <= 3072 cases hold 1e-5, i.e. ~3.3e-5 at 32768), so the bar
    is 1e-4.  A lost or doubled 64-wide K block would show as ~sqrt(64/K) =
    4e-2; the int8 case at the same K is bit-exact."""
    M, N, K = 257, 2048, 32768
    A = wlmod.normal_tensor((M, K), 61, cuda_dev, dtype=torch.bfloat16)
    B = wlmod.normal_tensor((N, K), 62, cuda_dev, 0.01, dtype=torch.bfloat16)
    X0 = wlmod.normal_tensor((M, N), 63, cuda_dev)
    X = X0.clone()
    h3b.gemm(A, B, h3b.EPI_RESID, X)
    torch.cuda.synchronize()
    acc = oracle.linear(np64(A), np64(B))
    assert rel_l2(np64(X) - np64(X0), acc) < 1e-4


def test_attention_max_heads(cuda_dev):
    """d = 8192: 64 heads of 128, over a ragged 300-token sequence."""
    S, H, D = 300, 64, 128
    qkv = wlmod.normal_tensor((S, 3 * H * D), 64, cuda_dev, 1.5, dtype=torch.bfloat16)
    o = h3b.attention(qkv, H, D)
    torch.cuda.synchronize()
    assert h3b.device_error() == 0
    q = np64(qkv)
    d = H * D
    ref = oracle.attention(q[:, :d], q[:, d:2 * d], q[:, 2 * d:], H)
    assert rel_l2(o, ref) < 1e-2 and max_abs(o, ref) < 3e-2


def test_empty_inputs_launch_nothing(cuda_dev):
    """Zero rows / tokens through the binding: empty results, no launch, no
    device error."""
    d, k = 256, 1024
    g = torch.ones(d, device=cuda_dev)
    with h3b.Trace() as tr:
        u = h3b.rmsnorm(torch.empty((0, d), device=cuda_dev), g, 1e-6)
        q, s = h3b.rmsnorm(torch.empty((0, d), device=cuda_dev), g, 1e-6, int8=True)
        qw, sw = h3b.quantize_weights(torch.empty((0, k), dtype=torch.bfloat16, device=cuda_dev))
        qa, sa = h3b.quantize_rows_absmax(torch.empty((0, k), dtype=torch.bfloat16, device=cuda_dev),
                                          torch.empty(0, device=cuda_dev))
        B = torch.ones((128, k), dtype=torch.bfloat16, device=cuda_dev)
        c = h3b.gemm(torch.empty((0, k), dtype=torch.bfloat16, device=cuda_dev), B, h3b.EPI_BF16,
                     torch.empty((0, 128), dtype=torch.bfloat16, device=cuda_dev))
        o = h3b.attention(torch.empty((0, 3 * 2 * 128), dtype=torch.bfloat16, device=cuda_dev), 2, 128)
        torch.cuda.synchronize()
    assert tr.records == []
    assert [t.shape[0] for t in (u, q, s, qw, sw, qa, sa, c, o)] == [0] * 9
    assert h3b.device_error() == 0
