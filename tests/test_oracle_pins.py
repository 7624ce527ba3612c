"""Pins for the CPU oracle: each check ties an oracle function to something
other than itself (closed forms, pure-Python brute force on tiny inputs,
invariants, the fresh-evaluation counts printed on the pages)."""
import json
import math
import os
import random
import types

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def dims_of(F, H, W, A, d, h, ffn, eps=1e-6, theta=10000.0):
    return types.SimpleNamespace(frames=F, rows=H, cols=W, n_audio=A, d=d, n_heads=h,
                                 head_dim=d // h, ffn=ffn, eps=eps, rope_theta=theta)


# ----------------------------------------------------------------------------- RMSNorm / GELU
def test_rmsnorm_constant_rows_closed_form():
    eps = 1e-6
    for c in (0.0, 1e-4, 0.3, -2.5, 1e3):
        x = np.full((1, 16), c)
        u = oracle.rmsnorm(x, np.ones(16), eps)
        assert np.allclose(u, c / math.sqrt(c * c + eps), rtol=1e-15, atol=0)


def test_rmsnorm_unit_rms_and_gain():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(5, 64)) * 3.0
    u = oracle.rmsnorm(x, np.ones(64), 0.0)
    assert np.allclose(np.sqrt(np.mean(u * u, axis=1)), 1.0, rtol=1e-14)
    g = rng.uniform(0.5, 2.0, size=64)
    ug = oracle.rmsnorm(x, g, 0.0)
    assert np.allclose(ug, u * g, rtol=1e-14)


def test_gelu_closed_form_and_limits():
    for v in (-6.0, -1.7, -0.3, 0.0, 0.25, 1.0, 3.3):
        ref = 0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0)))
        assert abs(float(oracle.gelu(np.array([v]))[0]) - ref) < 1e-15
    assert oracle.gelu(np.array([40.0]))[0] == 40.0
    assert abs(oracle.gelu(np.array([-40.0]))[0]) < 1e-300
    xs = np.linspace(-5, 5, 1001)
    tanh_form = 0.5 * xs * (1 + np.tanh(math.sqrt(2 / math.pi) * (xs + 0.044715 * xs ** 3)))
    assert np.max(np.abs(oracle.gelu(xs) - tanh_form)) < 1e-3


# ----------------------------------------------------------------------------- RoPE
def test_rope_sections():
    assert oracle.rope_sections(64) == (16, 24, 24)
    assert oracle.rope_sections(128) == (32, 48, 48)


def test_rope_angles_hand_computed():
    dm = dims_of(3, 4, 5, 3, 128, 2, 512)  # D = 64
    th = 10000.0
    ang = oracle.rope_angles(dm)
    assert ang.shape == (3 * 4 * 5 + 3, 32)
    t = (2 * 4 + 3) * 5 + 4  # video token (f=2, r=3, c=4)
    assert ang[t, 0] == pytest.approx(2.0)                       # frame section, pair 0
    assert ang[t, 1] == pytest.approx(2.0 * th ** (-2 / 16))     # frame section, pair 1
    assert ang[t, 8] == pytest.approx(3.0)                       # row section starts at pair D/8
    assert ang[t, 9] == pytest.approx(3.0 * th ** (-2 / 24))
    assert ang[t, 20] == pytest.approx(4.0)                      # col section starts at pair D/8+3D/16
    assert ang[t, 31] == pytest.approx(4.0 * th ** (-22 / 24))
    a = 60 + 2  # audio token 2
    for j in (0, 5, 31):
        assert ang[a, j] == pytest.approx(2.0 * th ** (-2 * j / 64))
    # merged geometry: token (f=1, r=2, c'=1) sits at column 2*1+0.5
    angm = oracle.rope_angles(dm, merged=True)
    assert angm.shape == (3 * 4 * 2 + 3, 32)
    tm = (1 * 4 + 2) * 2 + 1
    assert angm[tm, 20] == pytest.approx(2.5)
    assert angm[tm, 0] == pytest.approx(1.0) and angm[tm, 8] == pytest.approx(2.0)


def test_apply_rope_rotates_interleaved_pairs():
    rng = np.random.default_rng(1)
    S, H, D = 3, 2, 16
    ang = rng.uniform(-3, 3, size=(S, D // 2))
    for s in range(S):
        for j in range(D // 2):
            e = np.zeros((S, H * D))
            e[s, D + 2 * j] = 1.0          # head 1, even element of pair j
            e[s, D + 2 * j + 1] = 0.5      # odd element
            out = oracle.apply_rope(e, ang, H)
            c, sn = math.cos(ang[s, j]), math.sin(ang[s, j])
            assert out[s, D + 2 * j] == pytest.approx(1.0 * c - 0.5 * sn, abs=1e-15)
            assert out[s, D + 2 * j + 1] == pytest.approx(1.0 * sn + 0.5 * c, abs=1e-15)
            others = np.delete(out[s], [D + 2 * j, D + 2 * j + 1])
            assert np.all(others == 0)


def test_rope_position_zero_identity_and_norms():
    dm = dims_of(2, 3, 4, 5, 128, 2, 512)
    ang = oracle.rope_angles(dm)
    rng = np.random.default_rng(2)
    t = rng.normal(size=(ang.shape[0], 128))
    out = oracle.apply_rope(t, ang, 2)
    assert np.array_equal(out[0], t[0])                 # video (0,0,0)
    assert np.array_equal(out[24], t[24])               # audio a = 0
    pn_in = t.reshape(-1, 64, 2)
    pn_out = out.reshape(-1, 64, 2)
    assert np.allclose(np.hypot(pn_in[..., 0], pn_in[..., 1]), np.hypot(pn_out[..., 0], pn_out[..., 1]), rtol=1e-13)


def test_rope_relative_position_property():
    """<R_p q, R_p' k> depends on p - p' only, section by section."""
    dm = dims_of(4, 6, 6, 8, 64, 1, 256)
    ang = oracle.rope_angles(dm)
    rng = np.random.default_rng(3)
    q, k = rng.normal(size=64), rng.normal(size=64)

    def idx(f, r, c):
        return (f * 6 + r) * 6 + c

    def dot(i, j):
        Q = oracle.apply_rope(q[None], ang[i:i + 1], 1)[0]
        K = oracle.apply_rope(k[None], ang[j:j + 1], 1)[0]
        return Q @ K

    base = dot(idx(1, 2, 3), idx(0, 4, 1))
    assert dot(idx(3, 3, 5), idx(2, 5, 3)) == pytest.approx(base, rel=1e-12)
    assert dot(idx(1, 2, 3), idx(0, 4, 2)) != pytest.approx(base, rel=1e-6)
    V = 4 * 6 * 6
    assert dot(V + 1, V + 5) == pytest.approx(dot(V + 3, V + 7), rel=1e-12)


# ----------------------------------------------------------------------------- attention
def brute_attention(q, k, v, H):
    Sq, HD = len(q), len(q[0])
    D = HD // H
    out = [[0.0] * HD for _ in range(Sq)]
    for h in range(H):
        for i in range(Sq):
            sc = [sum(q[i][h * D + e] * k[j][h * D + e] for e in range(D)) / math.sqrt(D) for j in range(len(k))]
            m = max(sc)
            w = [math.exp(s - m) for s in sc]
            z = sum(w)
            for e in range(D):
                out[i][h * D + e] = sum(w[j] * v[j][h * D + e] for j in range(len(k))) / z
    return np.array(out)


def test_attention_vs_bruteforce():
    rng = np.random.default_rng(4)
    for S, H, D in ((1, 1, 4), (7, 2, 4), (13, 3, 8)):
        q, k, v = (rng.normal(size=(S, H * D)) * 2 for _ in range(3))
        ref = brute_attention(q.tolist(), k.tolist(), v.tolist(), H)
        assert np.allclose(oracle.attention(q, k, v, H, chunk=4), ref, rtol=1e-12, atol=1e-13)


def test_attention_uniform_and_convex():
    rng = np.random.default_rng(5)
    S, H, D = 9, 2, 8
    k, v = rng.normal(size=(S, H * D)), rng.normal(size=(S, H * D))
    o = oracle.attention(np.zeros((S, H * D)), k, v, H)
    assert np.allclose(o, v.mean(axis=0, keepdims=True), rtol=1e-14)
    o1 = oracle.attention(rng.normal(size=(S, H * D)), k, np.ones((S, H * D)), H)
    assert np.allclose(o1, 1.0, rtol=1e-14)


# ----------------------------------------------------------------------------- block
def quant_row_py(vals):
    """Per-row symmetric int8 by the fp32 rule, element by element: s =
    fp32(max|v|) / 127 in fp32, code = round-half-even(fp32(v) / s) (IEEE fp32
    quotient) clamped to +-127; a zero row gives s = 0 and zero codes."""
    a32 = [np.float32(t) for t in vals]
    s = np.float32(max(abs(t) for t in a32) / np.float32(127.0))
    if s == 0:
        return [0] * len(a32), 0.0
    return [int(min(127, max(-127, round(float(t / s))))) for t in a32], float(s)


def brute_block(x, w, dm, merged=False, mod=None, n_cond=0, w8a8=False):
    """Pure-Python loops: RMSNorm, QKV, RoPE by explicit (f,r,c)/audio
    positions, softmax attention, output projection, RMSNorm, GELU MLP.
    With ``mod`` ([2][6][d] nested lists: shift/scale/gate for attention, then
    for the MLP; class 1 = the last n_cond rows) each normed row becomes
    u*(1+scale)+shift and each residual update is multiplied by its gate;
    the n_cond condition rows get no rotation.  With ``w8a8`` every GEMM takes
    int8 codes of its input row and of each weight row (quant_row_py) and
    returns float(exact integer dot product) * s_input * s_weight."""
    S, d, H, D, f = len(x), dm.d, dm.n_heads, dm.head_dim, dm.ffn
    if mod is None:
        ident = [[0.0] * d, [0.0] * d, [1.0] * d]
        mod = [ident + ident, ident + ident]

    def cls(i):
        return 1 if i >= S - n_cond else 0
    wqkv, wo, w1, w2 = (w[k].tolist() for k in ("w_qkv", "w_o", "w_fc1", "w_fc2"))
    wq = {id(W): [quant_row_py(r) for r in W] for W in (wqkv, wo, w1, w2)} if w8a8 else None

    def norm(row, g):
        r = 1.0 / math.sqrt(sum(a * a for a in row) / d + dm.eps)
        return [a * r * gg for a, gg in zip(row, g)]

    def mv(W, a):
        if w8a8:
            qa, sa = quant_row_py(a)
            return [float(sum(qa[i] * qw[i] for i in range(len(a)))) * sa * sw for qw, sw in wq[id(W)]]
        return [sum(wr[i] * a[i] for i in range(len(a))) for wr in W]

    F, Hr, Wc, A = dm.frames, dm.rows, dm.cols, dm.n_audio
    wc = Wc // 2 if merged else Wc
    nf, nr = D // 4, 3 * D // 8
    pos = []
    for fi in range(F):
        for ri in range(Hr):
            for ci in range(wc):
                pos.append(("v", fi, ri, 2 * ci + 0.5 if merged else ci))
    for a in range(A):
        pos.append(("a", a))
    for _ in range(n_cond):
        pos.append(("c",))

    def rot(vec, p):
        out = list(vec)
        if p[0] == "c":
            return out
        for h in range(H):
            for j in range(D // 2):
                if p[0] == "a":
                    ang = p[1] * dm.rope_theta ** (-2 * j / D)
                elif j < nf // 2:
                    ang = p[1] * dm.rope_theta ** (-2 * j / nf)
                elif j < (nf + nr) // 2:
                    ang = p[2] * dm.rope_theta ** (-2 * (j - nf // 2) / nr)
                else:
                    nc = D - nf - nr
                    ang = p[3] * dm.rope_theta ** (-2 * (j - (nf + nr) // 2) / nc)
                a0, a1 = vec[h * D + 2 * j], vec[h * D + 2 * j + 1]
                out[h * D + 2 * j] = a0 * math.cos(ang) - a1 * math.sin(ang)
                out[h * D + 2 * j + 1] = a0 * math.sin(ang) + a1 * math.cos(ang)
        return out

    def modulate(row, i, first):
        sh, sc = mod[cls(i)][first], mod[cls(i)][first + 1]
        return [a * (1.0 + sc[e]) + sh[e] for e, a in enumerate(row)]

    u = [modulate(norm(row, w["g_attn"].tolist()), i, 0) for i, row in enumerate(x)]
    qkv = [mv(wqkv, row) for row in u]
    q = [rot(r[:d], pos[i]) for i, r in enumerate(qkv)]
    k = [rot(r[d:2 * d], pos[i]) for i, r in enumerate(qkv)]
    v = [r[2 * d:] for r in qkv]
    o = brute_attention(q, k, v, H).tolist()
    x1 = [[a + gt * b for a, b, gt in zip(x[i], mv(wo, o[i]), mod[cls(i)][2])] for i in range(S)]
    out = []
    for i in range(S):
        hvec = mv(w1, modulate(norm(x1[i], w["g_mlp"].tolist()), i, 3))
        g = [0.5 * a * (1 + math.erf(a / math.sqrt(2))) for a in hvec]
        out.append([a + gt * b for a, b, gt in zip(x1[i], mv(w2, g), mod[cls(i)][5])])
    return np.array(out)


def rand_block(rng, d, f, scale=0.2):
    return {"w_qkv": rng.normal(size=(3 * d, d)) * scale, "w_o": rng.normal(size=(d, d)) * scale,
            "w_fc1": rng.normal(size=(f, d)) * scale, "w_fc2": rng.normal(size=(d, f)) * scale,
            "g_attn": rng.uniform(0.5, 1.5, size=d), "g_mlp": rng.uniform(0.5, 1.5, size=d)}


@pytest.mark.parametrize("merged", [False, True])
def test_block_vs_bruteforce(merged):
    dm = dims_of(1, 2, 4, 2, 32, 2, 64)   # D = 16 -> sections 4/6/6
    rng = np.random.default_rng(6)
    S = (4 if merged else 8) + 2
    x = rng.normal(size=(S, 32))
    w = rand_block(rng, 32, 64)
    ref = brute_block(x.tolist(), w, dm, merged)
    assert np.allclose(oracle.block_forward(x, w, dm, merged=merged), ref, rtol=1e-11, atol=1e-12)


def test_block_zero_weight_identities():
    dm = dims_of(2, 2, 2, 3, 64, 4, 128)
    rng = np.random.default_rng(7)
    x = rng.normal(size=(11, 64))
    w = rand_block(rng, 64, 128)
    w0 = dict(w, w_o=np.zeros((64, 64)), w_fc2=np.zeros((64, 128)))
    assert np.array_equal(oracle.block_forward(x, w0, dm), x)
    # zero QKV -> attention output is 0, block reduces to the MLP branch alone
    wq = dict(w, w_qkv=np.zeros((192, 64)))
    mlp = x + oracle.gelu(oracle.rmsnorm(x, w["g_mlp"], 1e-6) @ w["w_fc1"].T) @ w["w_fc2"].T
    assert np.allclose(oracle.block_forward(x, wq, dm), mlp, rtol=1e-14)


def test_block_permutation_equivariant_without_rope():
    dm = dims_of(2, 2, 2, 3, 64, 4, 128)
    rng = np.random.default_rng(8)
    x = rng.normal(size=(11, 64))
    w = rand_block(rng, 64, 128)
    perm = rng.permutation(11)
    a = oracle.block_forward(x, w, dm, rope=False)[perm]
    b = oracle.block_forward(x[perm], w, dm, rope=False)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-13)
    # with RoPE the positions break the symmetry
    c = oracle.block_forward(x[perm], w, dm)
    assert not np.allclose(oracle.block_forward(x, w, dm)[perm], c, rtol=1e-6)


def test_block_row_sampling_matches_full():
    dm = dims_of(2, 4, 4, 5, 64, 2, 128)
    rng = np.random.default_rng(9)
    x = rng.normal(size=(37, 64))
    w = rand_block(rng, 64, 128)
    rows = np.array([0, 5, 31, 32, 36])
    full = oracle.block_forward(x, w, dm)
    assert np.allclose(oracle.block_forward(x, w, dm, rows=rows), full[rows], rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------------------- modulation and condition rows
def rand_mod(rng, d, scale=0.3):
    m = rng.normal(size=(2, 6, d)) * scale
    m[:, 2, :] += 1.0   # gates around 1
    m[:, 5, :] += 1.0
    return m


@pytest.mark.parametrize("merged,n_cond", [(False, 0), (False, 3), (True, 2)])
def test_cond_block_vs_bruteforce(merged, n_cond):
    dm = dims_of(1, 2, 4, 2, 32, 2, 64)
    rng = np.random.default_rng(30 + n_cond)
    S = (4 if merged else 8) + 2 + n_cond
    x = rng.normal(size=(S, 32))
    w = rand_block(rng, 32, 64)
    mod = rand_mod(rng, 32)
    ref = brute_block(x.tolist(), w, dm, merged, mod.tolist(), n_cond)
    got = oracle.block_forward_cond(x, w, dm, mod, n_cond, merged=merged)
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_cond_block_identity_modulation_and_zero_gates():
    dm = dims_of(2, 2, 2, 3, 64, 4, 128)
    rng = np.random.default_rng(31)
    x = rng.normal(size=(11, 64))
    w = rand_block(rng, 64, 128)
    ident = np.zeros((2, 6, 64))
    ident[:, 2] = ident[:, 5] = 1.0
    assert np.allclose(oracle.block_forward_cond(x, w, dm, ident), oracle.block_forward(x, w, dm), rtol=1e-14)
    assert np.allclose(oracle.block_forward_cond(x, w, dm, None), oracle.block_forward(x, w, dm), rtol=1e-14)
    # zero gates: the block adds nothing, whatever the shifts and scales
    m = rand_mod(rng, 64)
    m[:, 2] = m[:, 5] = 0.0
    xc = rng.normal(size=(14, 64))
    assert np.array_equal(oracle.block_forward_cond(xc, w, dm, m, n_cond=3), xc)


def test_cond_block_scale_minus_one_closed_form():
    """scale_attn = -1 replaces every normed row by its class's shift, so the
    attention input holds two distinct rows (generated: s0, condition: s1);
    without RoPE each head's output is the softmax mix of the two value rows
    weighted by their counts.  MLP gate 0 isolates the attention branch."""
    dm = dims_of(2, 2, 2, 1, 16, 2, 32)
    rng = np.random.default_rng(32)
    Sg, C, d, H, D = 9, 4, 16, 2, 8
    x = rng.normal(size=(Sg + C, d))
    w = rand_block(rng, d, 32, scale=0.5)
    m = rand_mod(rng, d)
    m[:, 1] = -1.0
    m[:, 5] = 0.0
    got = oracle.block_forward_cond(x, w, dm, m, n_cond=C, rope=False)
    wq, wk, wv = w["w_qkv"][:d], w["w_qkv"][d:2 * d], w["w_qkv"][2 * d:]
    s0, s1 = m[0, 0], m[1, 0]
    k0, k1, v0, v1 = wk @ s0, wk @ s1, wv @ s0, wv @ s1
    for i in range(Sg + C):
        cl = 1 if i >= Sg else 0
        q = wq @ (s1 if cl else s0)
        o = np.zeros(d)
        for h in range(H):
            sl = slice(h * D, h * D + D)
            a0 = math.exp(float(q[sl] @ k0[sl]) / math.sqrt(D)) * Sg
            a1 = math.exp(float(q[sl] @ k1[sl]) / math.sqrt(D)) * C
            o[sl] = (a0 * v0[sl] + a1 * v1[sl]) / (a0 + a1)
        ref = x[i] + m[cl, 2] * (w["w_o"] @ o)
        assert np.allclose(got[i], ref, rtol=1e-12, atol=1e-13)


def test_cond_rows_unrotated_and_gated_by_their_class():
    dm = dims_of(2, 2, 4, 3, 32, 2, 64)
    rng = np.random.default_rng(33)
    Sg, C = 19, 5
    x = rng.normal(size=(Sg + C, 32))
    w = rand_block(rng, 32, 64)
    m = rand_mod(rng, 32)
    # condition rows carry no position: permuting them permutes their outputs
    # and leaves the generated rows unchanged (RoPE on)
    perm = np.concatenate([np.arange(Sg), Sg + rng.permutation(C)])
    a = oracle.block_forward_cond(x, w, dm, m, n_cond=C)
    b = oracle.block_forward_cond(x[perm], w, dm, m, n_cond=C)
    assert np.allclose(a[perm], b, rtol=1e-12, atol=1e-13)
    # class-1 gates 0: condition rows pass through, generated rows still see them
    m1 = m.copy()
    m1[1, 2] = m1[1, 5] = 0.0
    c = oracle.block_forward_cond(x, w, dm, m1, n_cond=C)
    assert np.array_equal(c[Sg:], x[Sg:])
    x2 = x.copy()
    x2[Sg:] += 1.0
    c2 = oracle.block_forward_cond(x2, w, dm, m1, n_cond=C)
    assert not np.allclose(c2[:Sg], c[:Sg], rtol=1e-6)


def test_cond_stack_merge_carries_condition_rows():
    dm = dims_of(1, 2, 4, 2, 32, 2, 64)
    rng = np.random.default_rng(34)
    C = 3
    x = rng.normal(size=(10 + C, 32))
    m = oracle.token_merge(x, dm)
    assert m.shape == (4 + 2 + C, 32) and np.array_equal(m[4:], x[8:])
    assert np.array_equal(oracle.token_unmerge(m, dm)[8:], x[8:])
    blocks = [rand_block(rng, 32, 64) for _ in range(3)]
    mods = [rand_mod(rng, 32) for _ in range(3)]
    for delta in (False, True):
        got = oracle.stack_forward_cond(x, blocks, dm, mods, C, 1, 1, unmerge_delta=delta)
        xm0 = oracle.token_merge(oracle.block_forward_cond(x, blocks[0], dm, mods[0], C), dm)
        ym = oracle.block_forward_cond(xm0, blocks[1], dm, mods[1], C, merged=True)
        x1 = oracle.block_forward_cond(x, blocks[0], dm, mods[0], C)
        mid = oracle.token_unmerge_delta(x1, ym, xm0, dm) if delta else oracle.token_unmerge(ym, dm)
        ref = oracle.block_forward_cond(mid, blocks[2], dm, mods[2], C)
        assert np.allclose(got, ref, rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------------------- token reduction
def test_merge_unmerge_explicit_indices():
    F, H, W, A, d = 2, 3, 4, 3, 5
    dm = dims_of(F, H, W, A, 8, 1, 8)
    rng = np.random.default_rng(10)
    x = rng.normal(size=(F * H * W + A, d))
    m = oracle.token_merge(x, dm)
    assert m.shape == (F * H * W // 2 + A, d)
    for f in range(F):
        for r in range(H):
            for c in range(W // 2):
                i = (f * H + r) * (W // 2) + c
                assert np.array_equal(m[i], (x[(f * H + r) * W + 2 * c] + x[(f * H + r) * W + 2 * c + 1]) * 0.5)
    assert np.array_equal(m[F * H * W // 2:], x[F * H * W:])
    u = oracle.token_unmerge(m, dm)
    for f in range(F):
        for r in range(H):
            for c in range(W):
                assert np.array_equal(u[(f * H + r) * W + c], m[(f * H + r) * (W // 2) + c // 2])
    assert np.array_equal(u[F * H * W:], x[F * H * W:])


def test_merge_unmerge_identity_on_pair_constant():
    dm = dims_of(3, 2, 6, 4, 8, 1, 8)
    rng = np.random.default_rng(11)
    m = rng.normal(size=(3 * 2 * 3 + 4, 7))
    x = oracle.token_unmerge(m, dm)           # pair-constant by construction
    assert np.array_equal(oracle.token_unmerge(oracle.token_merge(x, dm), dm), x)
    assert np.array_equal(oracle.token_merge(x, dm), m)


def test_merge_fp32_single_rounding():
    """The fp64 mean of two fp32 values, rounded once to fp32, equals the fp32
    (a + b) * 0.5 -- the property the bit-exact merge check relies on."""
    rng = np.random.default_rng(12)
    a = (rng.normal(size=100000) * 10.0 ** rng.integers(-30, 30, size=100000)).astype(np.float32)
    b = (rng.normal(size=100000) * 10.0 ** rng.integers(-30, 30, size=100000)).astype(np.float32)
    via64 = ((a.astype(np.float64) + b.astype(np.float64)) * 0.5).astype(np.float32)
    via32 = (a + b) * np.float32(0.5)
    assert np.array_equal(via64, via32)


# ----------------------------------------------------------------------------- INT8
def test_quantize_rows_hand_computed():
    q, s = oracle.quantize_rows(np.array([[127.0, 0.5, 1.5, 2.5, -0.5, -127.0],
                                          [0.0, 0.0, 0.0, 0.0, 0.0, 0.0],
                                          [2.0, -1.0, 0.25, 0.0, 1.0, -2.0]]))
    assert s[0] == 1.0 and s[1] == 0.0
    assert q[0].tolist() == [127, 0, 2, 2, 0, -127]          # half-even ties
    assert q[1].tolist() == [0] * 6
    s2 = np.float32(2.0) / np.float32(127.0)
    assert s[2] == s2
    assert q[2].tolist() == [127, int(np.rint(np.float32(-1.0) / s2)), int(np.rint(np.float32(0.25) / s2)), 0,
                             int(np.rint(np.float32(1.0) / s2)), -127]
    assert q[2].tolist() == [127, -64, 16, 0, 64, -127]


def test_quantize_rows_bounds_and_roundtrip():
    rng = np.random.default_rng(13)
    a = rng.normal(size=(50, 300)).astype(np.float32)
    q, s = oracle.quantize_rows(a)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert np.all(np.abs(q.astype(int)) <= 127)
    assert np.all(np.max(np.abs(q.astype(int)), axis=1) == 127)
    assert np.all(np.abs(oracle.dequantize_rows(q, s) - a) <= s[:, None] * 0.5 * (1 + 1e-6))


def test_int8_matmul_vs_python():
    rng = np.random.default_rng(14)
    qa = rng.integers(-127, 128, size=(5, 37)).astype(np.int8)
    qw = rng.integers(-127, 128, size=(6, 37)).astype(np.int8)
    acc = oracle.int8_matmul(qa, qw)
    for m in range(5):
        for n in range(6):
            assert acc[m, n] == sum(int(qa[m, k]) * int(qw[n, k]) for k in range(37))
    big_a = np.full((1, 4096), 127, np.int8)
    assert oracle.int8_matmul(big_a, -big_a)[0, 0] == -127 * 127 * 4096


@pytest.mark.parametrize("merged", [False, True])
def test_w8a8_block_vs_bruteforce(merged):
    """The W8A8 block against pure-Python loops with per-element fp32
    quantisation and exact integer dot products; row sampling = full rows."""
    dm = dims_of(1, 2, 4, 2, 32, 2, 64)
    rng = np.random.default_rng(16)
    S = (4 if merged else 8) + 2
    x = rng.normal(size=(S, 32))
    w = rand_block(rng, 32, 64)
    ref = brute_block(x.tolist(), w, dm, merged, w8a8=True)
    got = oracle.block_forward_w8a8(x, w, dm, merged=merged)
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-12)
    rows = np.array([0, 3, S - 1])
    assert np.allclose(oracle.block_forward_w8a8(x, w, dm, merged=merged, rows=rows), got[rows], rtol=1e-13,
                       atol=1e-13)


def test_w8a8_block_close_to_dequant_reference():
    dm = dims_of(2, 4, 4, 4, 128, 2, 512)
    rng = np.random.default_rng(15)
    x = rng.normal(size=(36, 128))
    w = rand_block(rng, 128, 512, scale=0.05)
    ref = oracle.block_forward(x, oracle.dequant_weights(w), dm)
    diag = oracle.block_forward_w8a8(x, w, dm)
    rel = np.linalg.norm(diag - ref) / np.linalg.norm(ref)
    assert 0 < rel < 2e-2


# ----------------------------------------------------------------------------- flow-matching loop
def test_fresh_counts_golden():
    g = json.load(open(os.path.join(GOLDEN, "fresh_counts.json")))
    for r, n in g["fresh_evaluations"].items():
        assert len(oracle.fresh_steps(g["n_steps"], int(r))) == n


def test_fresh_counts_closed_form_few_steps():
    """The 4..7-step presets and every other (N, r): the fresh steps are the
    multiples of r below N plus the last step, so their number is
    ceil((N-1)/r) + 1 for N >= 2 (and 1 for N = 1); the last step is always
    fresh and step 0 always is."""
    for n in range(1, 51):
        for r in range(1, 8):
            f = oracle.fresh_steps(n, r)
            assert len(f) == (1 if n == 1 else -(-(n - 1) // r) + 1)
            assert f[0] == 0 and f[-1] == n - 1
    # the presets with the control table's reuse levels
    assert [len(oracle.fresh_steps(n, 1)) for n in (4, 5, 6, 7)] == [4, 5, 6, 7]
    assert [len(oracle.fresh_steps(n, 3)) for n in (4, 5, 6, 7)] == [2, 3, 3, 3]


def test_sigmas_grid():
    s = oracle.sigmas(20)
    assert s.dtype == np.float32 and len(s) == 21
    assert s[0] == 1.0 and s[-1] == 0.0 and np.all(np.diff(s) < 0)
    assert s[5] == np.float32(0.75)


def test_flow_step_zero_velocity_and_closed_form():
    rng = np.random.default_rng(16)
    x = rng.normal(size=(4, 8))
    assert np.array_equal(oracle.flow_step(x, np.zeros_like(x), 0.7, 0.65), x)
    v = rng.normal(size=(4, 8))
    dt = float(np.float32(0.7)) - 0.75          # the fp32 sigma, exactly
    assert np.allclose(oracle.flow_step(x, v, np.float32(0.75), np.float32(0.7)),
                       x + dt * v, rtol=1e-15, atol=0)


def test_denoise_constant_velocity_and_reuse_pattern():
    dm = dims_of(1, 1, 2, 1, 4, 1, 4)
    x0 = np.arange(12.0).reshape(3, 4)
    c = np.full((3, 4), 2.0)
    for r in (1, 2, 3):
        xN, nf = oracle.denoise(x0, [None], dm, 20, r, block_fn=lambda x, w, d, merged: c)
        assert nf == {1: 20, 2: 11, 3: 8}[r]
        assert np.allclose(xN, x0 - c, atol=1e-12)
    # v = x on fresh steps only: hand-computed N = 3, reuse 2 -> fresh at 0 and 2
    s = oracle.sigmas(3).astype(np.float64)
    xN, nf = oracle.denoise(x0, [None], dm, 3, 2, block_fn=lambda x, w, d, merged: x)
    v0 = x0
    x1 = x0 + (s[1] - s[0]) * v0
    x2 = x1 + (s[2] - s[1]) * v0
    x3 = x2 + (s[3] - s[2]) * x2
    assert nf == 2 and np.allclose(xN, x3, rtol=1e-14)


def test_stack_merge_window():
    dm = dims_of(2, 2, 4, 3, 8, 1, 8)
    seen = []

    def fn(x, w, d, merged):
        seen.append((len(x), merged))
        return x * 1.0

    x = np.random.default_rng(17).normal(size=(19, 8))
    out = oracle.stack_forward(x, [None] * 6, dm, 2, 3, block_fn=fn)
    assert seen == [(19, False), (19, False), (11, True), (11, True), (19, False), (19, False)]
    assert np.allclose(out, oracle.token_unmerge(oracle.token_merge(x, dm), dm))


# ----------------------------------------------------------------------------- next rows: delta unmerge, core reuse
def test_unmerge_delta_explicit_and_special_cases():
    F, H, W, A, d = 2, 3, 4, 2, 5
    dm = dims_of(F, H, W, A, 8, 1, 8)
    rng = np.random.default_rng(20)
    x_pre = rng.normal(size=(F * H * W + A, d))
    xm0 = oracle.token_merge(x_pre, dm)
    ym = xm0 + rng.normal(size=xm0.shape)
    out = oracle.token_unmerge_delta(x_pre, ym, xm0, dm)
    for f in range(F):
        for r in range(H):
            for c in range(W):
                i = (f * H + r) * W + c
                j = (f * H + r) * (W // 2) + c // 2
                assert np.allclose(out[i], x_pre[i] + ym[j] - xm0[j], rtol=0, atol=1e-14)
    assert np.array_equal(out[F * H * W:], ym[F * H * W // 2:])
    assert np.allclose(oracle.token_unmerge_delta(x_pre, xm0, xm0, dm)[:F * H * W], x_pre[:F * H * W])
    pc = oracle.token_unmerge(rng.normal(size=xm0.shape), dm)          # pair-constant pre-merge tokens
    pm = oracle.token_merge(pc, dm)
    assert np.allclose(oracle.token_unmerge_delta(pc, ym, pm, dm), oracle.token_unmerge(ym, dm), atol=1e-13)


def test_denoise_core_reuse_one_is_plain_loop():
    dm = dims_of(1, 1, 2, 1, 4, 1, 4)
    x0 = np.random.default_rng(21).normal(size=(3, 4))
    fn = lambda x, w, d, merged: np.tanh(x * w)  # noqa: E731
    ws = [0.9, 1.1, 0.7, 1.3]
    a, na = oracle.denoise(x0, ws, dm, 6, 1, block_fn=fn)
    b, nb = oracle.denoise_core(x0, ws, dm, 6, 1, 1, 2, block_fn=fn)
    assert na == nb == 6 and np.allclose(a, b, rtol=1e-14)


def test_denoise_core_hand_computed():
    """pre x a, core x b, post x c; 3 steps, core reuse 2 -> core fresh at 0 and 2."""
    dm = dims_of(1, 1, 2, 1, 4, 1, 4)
    x0 = np.random.default_rng(22).normal(size=(3, 4))
    a, b, c = 0.8, 1.25, 0.6
    fn = lambda x, w, d, merged: x * w  # noqa: E731
    got, nc = oracle.denoise_core(x0, [a, b, c], dm, 3, 2, 1, 1, block_fn=fn)
    s = oracle.sigmas(3).astype(np.float64)
    delta = (b - 1) * a * x0
    x1 = x0 + (s[1] - s[0]) * c * b * a * x0
    x2 = x1 + (s[2] - s[1]) * c * (a * x1 + delta)
    x3 = x2 + (s[3] - s[2]) * c * b * a * x2
    assert nc == 2 and np.allclose(got, x3, rtol=1e-14)
    with pytest.raises(ValueError):
        oracle.denoise_core(x0, [a, b, c], dm, 3, 2, 1, 1, merge_first=0, merge_last=1, block_fn=fn)


def test_denoise_cond_reduces_to_plain_loops():
    dm = dims_of(1, 1, 2, 1, 4, 1, 4)
    x0 = np.random.default_rng(35).normal(size=(3, 4))
    fn = lambda x, w, d, merged: np.tanh(x * w)  # noqa: E731
    fc = lambda x, w, d, mod, n_cond, merged: np.tanh(x * w)  # noqa: E731
    ws = [0.9, 1.1, 0.7, 1.3]
    a, na = oracle.denoise(x0, ws, dm, 7, 3, block_fn=fn)
    b, nb, _ = oracle.denoise_cond(x0, ws, dm, 7, reuse=3, block_fn=fc)
    assert na == nb and np.allclose(a, b, rtol=1e-15)
    a, nc = oracle.denoise_core(x0, ws, dm, 6, 4, 1, 2, block_fn=fn)
    b, nf, nc2 = oracle.denoise_cond(x0, ws, dm, 6, core_reuse=4, core_first=1, core_last=2, block_fn=fc)
    assert nf == 6 and nc == nc2 and np.allclose(a, b, rtol=1e-15)


def test_denoise_cond_rows_refilled_each_evaluation():
    """A toy block that adds the mean of the condition rows to every row: the
    condition rows grow inside an evaluation, but each evaluation starts from
    the given values, so the velocity of the generated rows is
    L * x + (sum over blocks of the running condition mean) at every step."""
    dm = dims_of(1, 1, 2, 1, 4, 1, 4)
    rng = np.random.default_rng(36)
    x0, cond = rng.normal(size=(3, 4)), rng.normal(size=(2, 4))

    def fc(x, w, d, mod, n_cond, merged):
        return x + x[len(x) - n_cond:].mean(axis=0)

    got, nf, _ = oracle.denoise_cond(x0, [0, 0], dm, 4, cond_rows=cond, reuse=1, block_fn=fc)
    s = oracle.sigmas(4).astype(np.float64)
    c = cond.mean(axis=0)
    x = x0.copy()
    for i in range(4):
        # block 1: rows + c; block 2: rows + (c + c) -> generated rows x + 3c
        x = x + (s[i + 1] - s[i]) * (x + 3.0 * c)
    assert nf == 4 and np.allclose(got, x, rtol=1e-14)
    with pytest.raises(ValueError):
        oracle.denoise_cond(x0, [0, 0], dm, 4, reuse=2, core_first=0, core_last=0, block_fn=fc)


def test_quantize_known_max_clamps_beyond_the_given_max():
    """Known-max int8 rule by hand: with row max 2, s = 2/127; 0.5/s = 31.75
    rounds to 32, 2/s = 127, 3/s = 190.5 and -8/s = -508 clamp to +-127; a zero
    max gives s = 0 and zero codes; with the row's own max it is quantize_rows."""
    q, s = oracle.quantize_rows_known_max(np.array([[0.5, 2.0, 3.0, -8.0], [1.0, -1.0, 0.5, 0.25]]),
                                          np.array([2.0, 0.0]))
    assert s[0] == np.float32(np.float32(2.0) / np.float32(127.0)) and s[1] == 0
    assert q.tolist() == [[32, 127, 127, -127], [0, 0, 0, 0]]
    a = np.random.default_rng(3).normal(size=(5, 64)).astype(np.float32)
    q1, s1 = oracle.quantize_rows(a)
    q2, s2 = oracle.quantize_rows_known_max(a, np.abs(a).max(axis=1))
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


# ----------------------------------------------------------------------------- wiring of the reduction window
# Toy block: every row is scaled by its block's weight, and a block that runs
# on the merged (reduced) grid also adds C.  Merged and unmerged blocks differ,
# so the expected tokens below -- derived by hand for one 1x1x2 video grid
# (one horizontal pair v0, v1) plus one audio row -- change if the window moves
# by one block, if the merge or unmerge happens at the wrong place, or if the
# delta unmerge takes the wrong pre-merge or merged tokens.
_C = 0.3


def _toy(x, w, d, merged):
    return x * w + (_C if merged else 0.0)


def _toy_cond(x, w, d, mod, n_cond, merged):
    return _toy(x, w, d, merged)


def test_stack_delta_unmerge_wiring_hand_computed():
    """stack_forward_ex(unmerge_delta=True) on blocks a0 (full grid), a1, a2
    (merged, window 1..2), a3 (full grid).  By hand, with y = a0*x the tokens
    that enter the window, m = (y0 + y1)/2 the merged pair and
    Y = a2*(a1*m + C) + C its output, each video token leaves the window as
    y_c + (Y - m); the audio row leaves as a2*(a1*y_a + C) + C; block 3 scales
    everything by a3.  The plain broadcast gives a3*Y on both video tokens."""
    dm = dims_of(1, 1, 2, 1, 8, 1, 8)
    a = [1.7, 0.6, 1.3, 0.8]
    x = np.array([[0.9, -1.1], [-0.4, 2.0], [1.5, 0.25]])  # v0, v1, audio; two channels
    seen = []

    def fn(xx, w, d, merged):
        seen.append((w, len(xx), merged))
        return _toy(xx, w, d, merged)

    got = oracle.stack_forward_ex(x, a, dm, 1, 2, unmerge_delta=True, block_fn=fn)
    assert seen == [(a[0], 3, False), (a[1], 2, True), (a[2], 2, True), (a[3], 3, False)]
    y = a[0] * x
    m = (y[0] + y[1]) / 2.0
    Y = a[2] * (a[1] * m + _C) + _C
    Ya = a[2] * (a[1] * y[2] + _C) + _C
    want = a[3] * np.stack([y[0] + (Y - m), y[1] + (Y - m), Ya])
    assert np.allclose(got, want, rtol=1e-15, atol=1e-15)
    # plain broadcast, same window
    got_b = oracle.stack_forward_ex(x, a, dm, 1, 2, unmerge_delta=False, block_fn=_toy)
    assert np.allclose(got_b, a[3] * np.stack([Y, Y, Ya]), rtol=1e-15, atol=1e-15)
    # the two unmerges differ on these tokens (v0 != v1), so the test tells them apart
    assert not np.allclose(got, got_b)


def _eval_window_in_core(x, a, delta=None):
    """One evaluation of the 5-block toy stack with core blocks 1..3 and the
    reduction window 2..3 (inside the core), by hand.  Returns (velocity,
    core update).  With delta given, the core is skipped and delta re-added."""
    p = a[0] * x                                   # block 0, full grid
    if delta is None:
        q = a[1] * p                               # block 1, full grid (core)
        m = (q[0] + q[1]) / 2.0                    # merge before block 2
        Yv = a[3] * (a[2] * m + _C) + _C           # blocks 2, 3 on the merged grid
        Ya = a[3] * (a[2] * q[2] + _C) + _C
        core = np.stack([Yv, Yv, Ya])              # plain broadcast after block 3
        delta = core - p
    else:
        core = p + delta
    return a[4] * core, delta                      # block 4, full grid


def _eval_window_after_core(x, a, delta=None):
    """Same toy stack with core block 1 only and the reduction window 3..4
    (after the core, in the last segment)."""
    p = a[0] * x
    if delta is None:
        core = a[1] * p
        delta = core - p
    else:
        core = p + delta
    r = a[2] * core                                # block 2, full grid
    m = (r[0] + r[1]) / 2.0
    Yv = a[4] * (a[3] * m + _C) + _C
    Ya = a[4] * (a[3] * r[2] + _C) + _C
    return np.stack([Yv, Yv, Ya]), delta


@pytest.mark.parametrize("case", ["inside_core", "after_core"])
def test_denoise_core_reduction_window_rebased_hand_computed(case):
    """denoise_core with the reduction window strictly inside the core window
    (core 1..3, merge 2..3) or after it (core 1..1, merge 3..4): 3 steps, core
    reuse 2 -> the core runs at steps 0 and 2, step 1 re-adds the cached
    update.  The window is re-based onto the segment it lies in; an off-by-one
    there moves the merge and changes every step below."""
    dm = dims_of(1, 1, 2, 1, 8, 1, 8)
    a = [0.8, 1.25, 0.7, 1.4, 0.9]
    x0 = np.array([[1.0, -0.5], [0.2, 0.7], [-1.3, 0.4]])
    cf, cl, mf, ml, ev = ((1, 3, 2, 3, _eval_window_in_core) if case == "inside_core"
                          else (1, 1, 3, 4, _eval_window_after_core))
    got, n_core = oracle.denoise_core(x0, a, dm, 3, 2, cf, cl, merge_first=mf, merge_last=ml, block_fn=_toy)
    s = oracle.sigmas(3).astype(np.float64)
    v0, d0 = ev(x0, a)
    x1 = x0 + (s[1] - s[0]) * v0
    v1, _ = ev(x1, a, delta=d0)
    x2 = x1 + (s[2] - s[1]) * v1
    v2, _ = ev(x2, a)
    x3 = x2 + (s[3] - s[2]) * v2
    assert n_core == 2
    assert np.allclose(got, x3, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("case", ["inside_core", "after_core"])
def test_denoise_cond_reduction_window_rebased_hand_computed(case):
    """The same hand-computed loops through denoise_cond, with one condition
    row appended (the toy block treats it like the audio row; it is refilled
    every evaluation and left out of the Euler update), and the velocity-reuse
    branch of denoise_cond with the window at 2..3 on the whole stack."""
    dm = dims_of(1, 1, 2, 1, 8, 1, 8)
    a = [0.8, 1.25, 0.7, 1.4, 0.9]
    x0 = np.array([[1.0, -0.5], [0.2, 0.7], [-1.3, 0.4]])
    cond = np.array([[0.6, -0.9]])
    cf, cl, mf, ml, ev = ((1, 3, 2, 3, _eval_window_in_core) if case == "inside_core"
                          else (1, 1, 3, 4, _eval_window_after_core))
    got, n_fresh, n_core = oracle.denoise_cond(x0, a, dm, 3, cond_rows=cond, merge_first=mf, merge_last=ml,
                                               core_reuse=2, core_first=cf, core_last=cl, block_fn=_toy_cond)
    s = oracle.sigmas(3).astype(np.float64)
    # the toy block acts row by row, so the condition row leaves the generated rows' velocity unchanged
    v0, d0 = ev(x0, a)
    x1 = x0 + (s[1] - s[0]) * v0
    v1, _ = ev(x1, a, delta=d0)
    x2 = x1 + (s[2] - s[1]) * v1
    v2, _ = ev(x2, a)
    x3 = x2 + (s[3] - s[2]) * v2
    assert (n_fresh, n_core) == (3, 2)
    assert np.allclose(got, x3, rtol=1e-14, atol=1e-14)

    # velocity reuse 2 (no core window), reduction window 2..3 of the 5 blocks:
    # fresh at steps 0 and 2, velocity reused at step 1
    def ev_full(x):
        p = a[1] * (a[0] * x)
        m = (p[0] + p[1]) / 2.0
        Yv = a[3] * (a[2] * m + _C) + _C
        Ya = a[3] * (a[2] * p[2] + _C) + _C
        return a[4] * np.stack([Yv, Yv, Ya])

    got, n_fresh, _ = oracle.denoise_cond(x0, a, dm, 3, cond_rows=cond, reuse=2, merge_first=2, merge_last=3,
                                          block_fn=_toy_cond)
    v0 = ev_full(x0)
    x1 = x0 + (s[1] - s[0]) * v0
    x2 = x1 + (s[2] - s[1]) * v0
    x3 = x2 + (s[3] - s[2]) * ev_full(x2)
    assert n_fresh == 2 and np.allclose(got, x3, rtol=1e-14, atol=1e-14)


def test_denoise_core_delta_unmerge_inside_core_hand_computed():
    """denoise_core with the delta unmerge and the window inside the core
    (core 1..3, merge 2..3): the core's output video tokens are
    q_c + (Y - m) with q = a1*a0*x the tokens entering the window."""
    dm = dims_of(1, 1, 2, 1, 8, 1, 8)
    a = [0.8, 1.25, 0.7, 1.4, 0.9]
    x0 = np.array([[1.0, -0.5], [0.2, 0.7], [-1.3, 0.4]])

    def ev(x, delta=None):
        p = a[0] * x
        if delta is None:
            q = a[1] * p
            m = (q[0] + q[1]) / 2.0
            Yv = a[3] * (a[2] * m + _C) + _C
            Ya = a[3] * (a[2] * q[2] + _C) + _C
            core = np.stack([q[0] + Yv - m, q[1] + Yv - m, Ya])
            delta = core - p
        else:
            core = p + delta
        return a[4] * core, delta

    got, n_core = oracle.denoise_core(x0, a, dm, 3, 2, 1, 3, merge_first=2, merge_last=3, unmerge_delta=True,
                                      block_fn=_toy)
    s = oracle.sigmas(3).astype(np.float64)
    v0, d0 = ev(x0)
    x1 = x0 + (s[1] - s[0]) * v0
    v1, _ = ev(x1, d0)
    x2 = x1 + (s[2] - s[1]) * v1
    v2, _ = ev(x2)
    x3 = x2 + (s[3] - s[2]) * v2
    assert n_core == 2 and np.allclose(got, x3, rtol=1e-14, atol=1e-14)


def test_linear_vs_python_dot_products():
    """y[m, n] = sum_k a[m, k] W[n, k] for W stored [out, in], by explicit sums."""
    rng = random.Random(5)
    a = [[rng.uniform(-2, 2) for _ in range(7)] for _ in range(3)]
    w = [[rng.uniform(-2, 2) for _ in range(7)] for _ in range(4)]
    y = oracle.linear(np.array(a), np.array(w))
    assert y.shape == (3, 4)
    for m in range(3):
        for n in range(4):
            assert abs(y[m, n] - math.fsum(a[m][k] * w[n][k] for k in range(7))) < 1e-13
