"""Oracle for one dense single-stream DiT block, its stack, token reduction,
the INT8 W8A8 variant and the flow-matching Euler loop with velocity reuse.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources.  The MiniMax H3 / h3.c pages fix the block's context, not its
internals:
  * "MiniMax H3: video and audio generated together" (mobbang.com, model
    section): H3 is a dense single-stream omni transformer; all frames and the
    audio track are denoised at once, with attention across frames and
    modalities.
  * "h3.c MiniMax H3 inference engine for Mac" (jdon.com, 330B-parameter
    section): token reduction pairs adjacent video tokens; fused kernels;
    the QKV arena is reused for the attention heads, then the MLP input.
  * "antirez/h3.c" (siami.tw, speed/quality control table): reuse 1/2/3 gives
    20/11/8 fresh DiT evaluations at 20 steps; token reduction merges
    horizontal video tokens in the middle blocks.
  * same page, "data" section, and the 21cto.com page's M5 Max section: INT8
    weight quantisation of the MLP, QKV and attention-output GEMMs;
    jdon.com "speed vs quality" section: int8 FC2 with one activation scale
    per row.
The block form itself (pre-norm RMSNorm with eps 1e-6, QKV, 3D RoPE over
(frame, row, col) and 1D RoPE for audio, full bidirectional attention,
output projection + residual, RMSNorm, exact-erf GELU MLP + residual) is the
one the workload specification states.  Where the pages and the specification
are silent, the plainest reading is taken; each is named in ``READINGS``.

Precision: fp64 everywhere, int64 for the integer GEMM, and fp32 for the
quantisation rule (scale = max|row| / 127 in fp32, IEEE fp32 divide,
round-half-even), which the method fixes in fp32.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "READINGS", "PINS", "MOD_FIELDS", "block_forward_cond", "stack_forward_cond", "denoise_cond",
    "linear", "rmsnorm", "gelu", "rope_sections", "token_positions", "rope_angles", "apply_rope",
    "attention", "block_forward", "stack_forward", "token_merge", "token_unmerge",
    "quantize_rows", "quantize_rows_known_max", "dequantize_rows", "int8_matmul", "dequant_weights", "block_forward_w8a8",
    "sigmas", "is_fresh", "fresh_steps", "flow_step", "denoise",
    "token_unmerge_delta", "stack_forward_ex", "denoise_core",
]

# Readings taken where the pages (and the workload specification) leave a step open.
READINGS = {
    "block": "no biases, no QK-norm, no timestep modulation, no final norm (none is stated)",
    "gelu": "exact erf form 0.5*x*(1+erf(x/sqrt2))",
    "rope_pairs": "interleaved pairs (x[2j], x[2j+1]) within each head",
    "rope_sections": "video head dims split [frame D/4 | row 3D/8 | col 3D/8]; audio: one 1D section over D",
    "rope_freq": "pair j of a section of width n rotates by p * theta^(-2j/n), theta = 10000",
    "rope_positions": "integer (f, r, c) from 0; audio a = 0..A-1 independent of video",
    "merged_rope": "a merged token (f, r, c') sits at column position 2c'+0.5",
    "merge": "mean of the horizontally adjacent pair (2c', 2c'+1); audio rows pass through",
    "unmerge": "plain broadcast of the merged token to both columns",
    "merge_blocks": "blocks 15..29, 0-indexed, inclusive",
    "quant": "symmetric, s = max|row|/127 in fp32, q = rint(v/s) half-even, clamp [-127,127], zero row -> s=0,q=0",
    "int8_coverage": "QKV, attention-output, FC1 and FC2 GEMMs; attention stays bf16",
    "sigmas": "sigma_i = 1 - i/N, i = 0..N, computed in fp64 and stored fp32",
    "fresh": "step i is fresh iff i % reuse == 0 or i == N-1",
    "velocity": "the velocity is the stack output (no in/out projection is stated)",
    "euler": "x <- x + (sigma_{i+1} - sigma_i) * v over all S tokens at width d",
    "residual": "fp32 residual stream in every configuration",
    "unmerge_delta": "alternative unmerge: the pre-merge tokens plus the merged blocks' update broadcast to "
                     "both columns, x_pre + (y - m); audio rows take y",
    "core_reuse": "core residual reuse (exclusive with whole-velocity reuse): every step evaluates the stack, "
                  "but the core blocks run only on fresh-core steps (i % r == 0 or the last step); their update "
                  "(output - input of the core) is cached and added on the other steps",
    "layers": "--layers L: the stack is given the active blocks (the first L of the model in the workloads)",
    "modulation": "timestep conditioning as adaLN-style modulation (the pages give no form): per block and row "
                  "class, u = RMSNorm(x)*(1+scale)+shift before the QKV and FC1 GEMMs and x += gate*update "
                  "after the O-proj and FC2 GEMMs; class 0 = generated (video + audio) rows, class 1 = "
                  "condition rows",
    "condition_rows": "fixed condition rows (the siami.tw file list names a 0.999 condition augmentation and "
                      "fixed condition rows inside the DiT, without a form): C rows appended after the audio "
                      "tokens, given already augmented; "
                      "they take part in every block (joint attention) with no rotary embedding, every "
                      "evaluation starts them from the given values, and the Euler update leaves them out",
}

# What pins each function to something other than itself (tests/test_oracle_*.py).
PINS = {
    "rmsnorm": "closed form on constant rows; unit RMS with g = 1",
    "gelu": "math.erf closed form at scalar points; tanh approximation within 1e-3; limits",
    "rope_angles/apply_rope": "hand-computed rotations per section; position 0 = identity; pair norms; "
                              "relative-position invariance per section",
    "attention": "pure-Python brute-force softmax attention on tiny inputs; rows sum to 1; "
                 "uniform-attention closed form",
    "block_forward": "pure-Python loop block on a tiny case; zero-weight identities; "
                     "permutation equivariance without RoPE; row sampling = full rows",
    "token_merge/unmerge": "explicit (f, r, c) loops; unmerge(merge(x)) = x on pair-constant x",
    "quantize_rows": "hand-computed codes incl. half-even ties; zero row",
    "quantize_rows_known_max": "hand-computed codes with a given max below the row's (clamping), zero max; "
                               "equals quantize_rows at the row's own max",
    "int8_matmul": "pure-Python integer dot products",
    "block_forward_w8a8": "pure-Python loop block with per-element fp32 quantisation and exact integer dot "
                          "products; row sampling = full rows; close to block_forward on the dequantised weights",
    "sigmas/fresh/denoise": "fresh counts 20/11/8 at 20 steps (control table); v = 0 identity; "
                            "single-step closed form",
    "token_unmerge_delta": "explicit (f, r, c) loops; equals plain unmerge when x_pre is pair-constant; "
                           "identity when the merged blocks change nothing",
    "denoise_core": "core_reuse = 1 equals the plain loop; a core that adds a constant gives the closed form; "
                    "hand-computed 3-step case; hand-computed loops with the reduction window strictly inside "
                    "the core window and after it (window re-based onto its segment), plain and delta unmerge",
    "stack_forward_ex": "hand-computed tokens with a toy block whose merged and unmerged forms differ: where the "
                        "pre-merge tokens are taken, which merged input the delta subtracts, the window's blocks",
    "linear": "pure-Python dot products",
    "stack_forward": "scalar toy blocks: the blocks inside the reduction window see the merged rows, the others "
                     "the full rows, in order; identity blocks give unmerge(merge(x))",
    "stack_forward_cond": "merge window with condition rows equals the explicit composition of pinned parts "
                          "(block_forward_cond, token_merge, token_unmerge[_delta]); condition rows pass the merge",
    "flow_step": "zero velocity is the identity; x + (s1 - s0) v closed form",
    "dequantize_rows/dequant_weights": "|dequantised - input| <= s/2 per element; the W8A8 block is close to "
                                       "block_forward on the dequantised weights",
    "rope_sections/token_positions": "section widths D/4, 3D/8, 3D/8; hand-computed angles of a given (f, r, c), of "
                                     "an audio token and of a merged token at column 2c'+0.5",
    "block_forward_cond": "identity modulation without condition rows equals block_forward; zero gates give the "
                          "identity; scale = -1 makes every normed row equal to the shift (closed form without "
                          "RoPE); condition rows are permutation-equivariant among themselves (no rotation); a "
                          "class-1 zero gate leaves condition rows unchanged",
    "denoise_cond": "no condition rows and no modulation equals denoise / denoise_core; a toy block gives the "
                    "closed form that needs the condition rows refilled every evaluation; hand-computed loops with "
                    "the reduction window inside / after the core window and under velocity reuse",
}


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------- linear / norm / activation
def linear(a, w):
    """y = a W^T for W stored [out, in] (a library matmul in fp64)."""
    return _f64(a) @ _f64(w).T


def rmsnorm(x, g, eps):
    """u = x * 1/sqrt(mean_j x_j^2 + eps) * g, per row (token)."""
    x = _f64(x)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * _f64(g)


def gelu(x):
    """Exact GELU: 0.5 * x * (1 + erf(x / sqrt(2)))."""
    x = _f64(x)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


# ----------------------------------------------------------------------------- RoPE
def rope_sections(head_dim):
    """Widths of the (frame, row, col) sections of one head: D/4, 3D/8, the rest."""
    nf = head_dim // 4
    nr = 3 * head_dim // 8
    return nf, nr, head_dim - nf - nr


def token_positions(dims, merged=False):
    """(video positions [V', 3] as (f, r, c) floats, audio positions [A]).

    Video tokens are ordered (f*H + r)*W + c.  After token reduction the grid
    has W/2 columns and the merged token c' sits at column 2c' + 0.5."""
    F, H, W, A = dims.frames, dims.rows, dims.cols, dims.n_audio
    wc = W // 2 if merged else W
    f, r, c = np.meshgrid(np.arange(F), np.arange(H), np.arange(wc), indexing="ij")
    col = 2.0 * c + 0.5 if merged else c.astype(np.float64)
    video = np.stack([f.ravel().astype(np.float64), r.ravel().astype(np.float64), col.ravel()], axis=1)
    return video, np.arange(A, dtype=np.float64)


def rope_angles(dims, merged=False):
    """Rotation angle of every (token, pair) [S', D/2].

    Video: pair j of the section of width n that carries position p (frame,
    row or col) turns by p * theta^(-2j/n).  Audio: one section of width D
    carrying the audio index a."""
    D, theta = dims.head_dim, float(dims.rope_theta)
    video, audio = token_positions(dims, merged)
    cols = []
    for axis, n in enumerate(rope_sections(D)):
        j = np.arange(n // 2, dtype=np.float64)
        omega = theta ** (-2.0 * j / n)
        cols.append(video[:, axis:axis + 1] * omega[None, :])
    ang_v = np.concatenate(cols, axis=1)
    j = np.arange(D // 2, dtype=np.float64)
    ang_a = audio[:, None] * (theta ** (-2.0 * j / D))[None, :]
    return np.concatenate([ang_v, ang_a], axis=0)


def apply_rope(t, angles, n_heads):
    """Rotate each interleaved pair (t[2j], t[2j+1]) of every head by angles[:, j]."""
    t = _f64(t)
    S = t.shape[0]
    D = t.shape[1] // n_heads
    th = t.reshape(S, n_heads, D // 2, 2)
    c = np.cos(angles)[:, None, :]
    s = np.sin(angles)[:, None, :]
    x0, x1 = th[..., 0], th[..., 1]
    out = np.empty_like(th)
    out[..., 0] = x0 * c - x1 * s
    out[..., 1] = x0 * s + x1 * c
    return out.reshape(S, n_heads * D)


# ----------------------------------------------------------------------------- attention
def attention(q, k, v, n_heads, chunk=2048):
    """o = softmax(q k^T / sqrt(D)) v per head, every query against every key
    (bidirectional, no mask).  Query rows are independent; they are taken in
    chunks only to bound memory."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Sq = q.shape[0]
    D = q.shape[1] // n_heads
    out = np.empty((Sq, n_heads * D))
    scale = 1.0 / math.sqrt(D)
    for h in range(n_heads):
        sl = slice(h * D, (h + 1) * D)
        kh, vh = k[:, sl], v[:, sl]
        for r0 in range(0, Sq, chunk):
            sc = (q[r0:r0 + chunk, sl] @ kh.T) * scale
            sc -= sc.max(axis=1, keepdims=True)
            p = np.exp(sc)
            p /= p.sum(axis=1, keepdims=True)
            out[r0:r0 + chunk, sl] = p @ vh
    return out


# ----------------------------------------------------------------------------- block / stack
def block_forward(x, w, dims, merged=False, rows=None, rope=True):
    """One DiT block on the residual stream x [S', d]:

        u  = RMSNorm(x; g_attn)
        q, k, v = u W_qkv^T split in thirds; q, k <- RoPE(q), RoPE(k) per head
        x1 = x + softmax(q k^T / sqrt(D)) v  W_o^T
        x2 = x1 + GELU(RMSNorm(x1; g_mlp) W_fc1^T) W_fc2^T

    ``rows`` (optional index array) returns x2 only at those tokens; keys and
    values still cover every token, so the sampled rows equal the full
    result's rows.  ``rope=False`` leaves q and k unrotated (invariance tests).
    """
    x = _f64(x)
    S, d = x.shape
    H = dims.n_heads
    rows = np.arange(S) if rows is None else np.asarray(rows)
    wqkv = _f64(w["w_qkv"])
    u = rmsnorm(x, w["g_attn"], dims.eps)
    k = u @ wqkv[d:2 * d].T
    v = u @ wqkv[2 * d:3 * d].T
    q = u[rows] @ wqkv[:d].T
    if rope:
        ang = rope_angles(dims, merged)
        q = apply_rope(q, ang[rows], H)
        k = apply_rope(k, ang, H)
    o = attention(q, k, v, H)
    x1 = x[rows] + o @ _f64(w["w_o"]).T
    hmid = gelu(rmsnorm(x1, w["g_mlp"], dims.eps) @ _f64(w["w_fc1"]).T)
    return x1 + hmid @ _f64(w["w_fc2"]).T


def token_merge(x, dims):
    """Token reduction: the merged video token (f, r, c') is the mean of the
    horizontally adjacent pair (f, r, 2c') and (f, r, 2c'+1); the rows after
    the video rows (audio, then any condition rows) are carried unchanged after
    the merged video rows."""
    x = _f64(x)
    F, H, W = dims.frames, dims.rows, dims.cols
    V = F * H * W
    vid = x[:V].reshape(F, H, W, -1)
    m = (vid[:, :, 0::2, :] + vid[:, :, 1::2, :]) * 0.5
    return np.concatenate([m.reshape(V // 2, -1), x[V:]], axis=0)


def token_unmerge(xm, dims):
    """Inverse of the reduction: each merged token is broadcast back to both
    columns it came from; the rows after the video rows are carried unchanged."""
    xm = _f64(xm)
    F, H, W = dims.frames, dims.rows, dims.cols
    V = F * H * W
    vid = xm[:V // 2].reshape(F, H, W // 2, -1)
    full = np.repeat(vid, 2, axis=2)
    return np.concatenate([full.reshape(V, -1), xm[V // 2:]], axis=0)


def token_unmerge_delta(x_pre, ym, xm0, dims):
    """Delta-broadcast unmerge: full token (f, r, c) = x_pre(f, r, c) +
    (ym - xm0)(f, r, c // 2), where xm0 is the merged sequence that entered
    the merged blocks and ym what they returned; the rows after the video rows
    (audio, condition) take ym."""
    x_pre, ym, xm0 = _f64(x_pre), _f64(ym), _f64(xm0)
    F, H, W = dims.frames, dims.rows, dims.cols
    V = F * H * W
    dv = (ym[:V // 2] - xm0[:V // 2]).reshape(F, H, W // 2, -1)
    full = x_pre[:V].reshape(F, H, W, -1) + np.repeat(dv, 2, axis=2)
    return np.concatenate([full.reshape(V, -1), ym[V // 2:]], axis=0)


def stack_forward_ex(x, blocks, dims, merge_first=-1, merge_last=-1, unmerge_delta=False, block_fn=None):
    """stack_forward with the choice of unmerge: plain broadcast, or the
    delta-broadcast form (pre-merge tokens plus the merged blocks' update)."""
    if not unmerge_delta:
        return stack_forward(x, blocks, dims, merge_first, merge_last, block_fn)
    fn = block_forward if block_fn is None else block_fn
    x = _f64(x)
    x_pre = xm0 = None
    for layer, w in enumerate(blocks):
        if layer == merge_first:
            x_pre = x
            xm0 = token_merge(x, dims)
            x = xm0
        x = fn(x, w, dims, merged=merge_first >= 0 and merge_first <= layer <= merge_last)
        if layer == merge_last and merge_first >= 0:
            x = token_unmerge_delta(x_pre, x, xm0, dims)
    return x


def denoise_core(x0, blocks, dims, n_steps, core_reuse, core_first, core_last, merge_first=-1, merge_last=-1,
                 unmerge_delta=False, block_fn=None):
    """Flow-matching loop with core residual reuse: every step evaluates the
    stack; the core blocks [core_first, core_last] (with the token-reduction
    window, which lies inside the core or outside it) run only on fresh-core
    steps (i % core_reuse == 0 or the last step), where their update
    delta = core(v) - v is cached; other steps add the cached delta instead.
    Returns (x_N, number of fresh-core steps)."""
    inside = merge_first >= 0 and core_first <= merge_first and merge_last <= core_last
    if not (inside or merge_first < 0 or merge_last < core_first or merge_first > core_last):
        raise ValueError("the token-reduction window must lie inside the core window or outside it")
    sig = sigmas(n_steps)
    x = _f64(x0)
    delta = None
    n_core = 0

    def part(v, lo, hi):  # blocks lo..hi with the merge window re-based if it lies in them
        if lo > hi:
            return v
        mf, ml = (merge_first - lo, merge_last - lo) if merge_first >= 0 and lo <= merge_first <= hi else (-1, -1)
        return stack_forward_ex(v, blocks[lo:hi + 1], dims, mf, ml, unmerge_delta, block_fn)

    for i in range(n_steps):
        v = part(x, 0, core_first - 1)
        if is_fresh(i, n_steps, core_reuse):
            out = part(v, core_first, core_last)
            delta = out - v
            v = out
            n_core += 1
        else:
            v = v + delta
        v = part(v, core_last + 1, len(blocks) - 1)
        x = flow_step(x, v, sig[i], sig[i + 1])
    return x, n_core


def stack_forward(x, blocks, dims, merge_first=-1, merge_last=-1, block_fn=None):
    """Blocks 0..L-1 in order; with token reduction on, merge before block
    ``merge_first`` and unmerge after block ``merge_last`` (inclusive)."""
    fn = block_forward if block_fn is None else block_fn
    on = merge_first >= 0
    x = _f64(x)
    for layer, w in enumerate(blocks):
        if on and layer == merge_first:
            x = token_merge(x, dims)
        x = fn(x, w, dims, merged=on and merge_first <= layer <= merge_last)
        if on and layer == merge_last:
            x = token_unmerge(x, dims)
    return x


# ----------------------------------------------------------------------------- INT8 W8A8
def quantize_rows(a):
    """Per-row symmetric int8: s = max|row|/127 (fp32), q = rint(row/s) with an
    IEEE fp32 divide, half-even, clamped to [-127, 127]; an all-zero row gives
    s = 0 and q = 0.  Used for weights (per output channel) and for
    activations (per token)."""
    a32 = np.asarray(a, dtype=np.float32)
    return quantize_rows_known_max(a32, np.max(np.abs(a32), axis=1))


def quantize_rows_known_max(a, row_max):
    """The same rule with each row's maximum given (the FC2 input takes it from
    the FC1 epilogue): s = row_max/127 (fp32); values beyond row_max clamp to
    +-127; row_max = 0 gives s = 0 and q = 0."""
    a32 = np.asarray(a, dtype=np.float32)
    s = (np.asarray(row_max, dtype=np.float32) / np.float32(127.0)).astype(np.float32)
    q = np.zeros(a32.shape, dtype=np.float32)
    nz = s > 0
    q[nz] = np.rint(a32[nz] / s[nz, None])
    return np.clip(q, -127, 127).astype(np.int8), s


def dequantize_rows(q, s):
    return q.astype(np.float64) * _f64(s)[:, None]


def int8_matmul(qa, qw):
    """Exact integer GEMM: acc[m, n] = sum_k qa[m, k] * qw[n, k] in int64."""
    return qa.astype(np.int64) @ qw.astype(np.int64).T


def dequant_weights(w):
    """Block weights with each GEMM matrix replaced by its int8 round trip
    q * s_w (the reference the W8A8 block is held to)."""
    out = dict(w)
    for key in ("w_qkv", "w_o", "w_fc1", "w_fc2"):
        q, s = quantize_rows(w[key])
        out[key] = dequantize_rows(q, s)
    return out


def _w8a8_linear(a, wq, ws):
    qa, sa = quantize_rows(a)
    # integer sums are exact in fp64 here (|acc| < 2^53)
    acc = qa.astype(np.float64) @ wq.astype(np.float64).T
    return acc * _f64(sa)[:, None] * _f64(ws)[None, :]


def block_forward_w8a8(x, w, dims, merged=False, rope=True, rows=None):
    """Block with every GEMM input fake-quantised per token as well as the
    weights per output channel (the full W8A8 arithmetic in fp64).  ``rows``
    as in block_forward: x2 only at those tokens, keys and values over all
    (per-token quantisation keeps every row independent of the others)."""
    x = _f64(x)
    S, d, H = x.shape[0], x.shape[1], dims.n_heads
    rows = np.arange(S) if rows is None else np.asarray(rows)
    qw = {k: quantize_rows(w[k]) for k in ("w_qkv", "w_o", "w_fc1", "w_fc2")}
    u = rmsnorm(x, w["g_attn"], dims.eps)
    qa, sa = quantize_rows(u)
    wq, ws = qw["w_qkv"]
    k = (qa.astype(np.float64) @ wq[d:2 * d].astype(np.float64).T) * _f64(sa)[:, None] * _f64(ws[d:2 * d])[None, :]
    v = (qa.astype(np.float64) @ wq[2 * d:].astype(np.float64).T) * _f64(sa)[:, None] * _f64(ws[2 * d:])[None, :]
    q = (qa[rows].astype(np.float64) @ wq[:d].astype(np.float64).T) * _f64(sa[rows])[:, None] * _f64(ws[:d])[None, :]
    if rope:
        ang = rope_angles(dims, merged)
        q, k = apply_rope(q, ang[rows], H), apply_rope(k, ang, H)
    o = attention(q, k, v, H)
    x1 = x[rows] + _w8a8_linear(o, *qw["w_o"])
    g = gelu(_w8a8_linear(rmsnorm(x1, w["g_mlp"], dims.eps), *qw["w_fc1"]))
    return x1 + _w8a8_linear(g, *qw["w_fc2"])


# ----------------------------------------------------------------------------- modulation and condition rows
MOD_FIELDS = ("shift_attn", "scale_attn", "gate_attn", "shift_mlp", "scale_mlp", "gate_mlp")


def _mod_rows(mod, n_rows, n_cond, field):
    """[rows, d] view of one modulation field: class 0 for the generated rows,
    class 1 for the last n_cond (condition) rows."""
    mod = _f64(mod)
    i = MOD_FIELDS.index(field)
    cls = np.zeros(n_rows, dtype=np.int64)
    cls[n_rows - n_cond:] = 1
    return mod[cls, i, :]


def block_forward_cond(x, w, dims, mod=None, n_cond=0, merged=False, rows=None, rope=True):
    """block_forward over [generated rows ; n_cond condition rows] with
    adaLN-style modulation.  ``mod``: [2, 6, d] (row class, MOD_FIELDS) or
    None (scale 0, shift 0, gate 1):

        u  = RMSNorm(x; g_attn) * (1 + scale_attn) + shift_attn
        x1 = x + gate_attn * (Attn(RoPE(u W_qkv^T)) W_o^T)
        x2 = x1 + gate_mlp * (GELU((RMSNorm(x1; g_mlp) * (1 + scale_mlp) + shift_mlp) W_fc1^T) W_fc2^T)

    Condition rows carry no rotary embedding; every row attends to every row.
    ``rows`` returns x2 only at those rows (keys/values still cover all)."""
    x = _f64(x)
    S, d = x.shape
    Sg = S - n_cond
    H = dims.n_heads
    rows = np.arange(S) if rows is None else np.asarray(rows)
    if mod is None:
        mod = np.zeros((2, 6, d))
        mod[:, 2, :] = 1.0
        mod[:, 5, :] = 1.0
    f = {k: _mod_rows(mod, S, n_cond, k) for k in MOD_FIELDS}
    wqkv = _f64(w["w_qkv"])
    u = rmsnorm(x, w["g_attn"], dims.eps) * (1.0 + f["scale_attn"]) + f["shift_attn"]
    k = u @ wqkv[d:2 * d].T
    v = u @ wqkv[2 * d:3 * d].T
    q = u[rows] @ wqkv[:d].T
    if rope:
        ang = np.zeros((S, d // H // 2))
        ang[:Sg] = rope_angles(dims, merged)
        q = apply_rope(q, ang[rows], H)
        k = apply_rope(k, ang, H)
    o = attention(q, k, v, H)
    x1 = x[rows] + f["gate_attn"][rows] * (o @ _f64(w["w_o"]).T)
    h2 = rmsnorm(x1, w["g_mlp"], dims.eps) * (1.0 + f["scale_mlp"][rows]) + f["shift_mlp"][rows]
    return x1 + f["gate_mlp"][rows] * (gelu(h2 @ _f64(w["w_fc1"]).T) @ _f64(w["w_fc2"]).T)


def stack_forward_cond(x, blocks, dims, mods=None, n_cond=0, merge_first=-1, merge_last=-1, unmerge_delta=False,
                       block_fn=None):
    """Blocks in order on [generated ; condition] rows; block l takes
    ``mods[l]`` ([2, 6, d]) when ``mods`` is given.  Token reduction as in
    stack_forward_ex (condition rows are carried like the audio rows)."""
    fn = block_forward_cond if block_fn is None else block_fn
    on = merge_first >= 0
    x = _f64(x)
    x_pre = xm0 = None
    for layer, w in enumerate(blocks):
        if on and layer == merge_first:
            x_pre = x
            xm0 = token_merge(x, dims)
            x = xm0
        x = fn(x, w, dims, None if mods is None else mods[layer], n_cond,
               merged=on and merge_first <= layer <= merge_last)
        if on and layer == merge_last:
            x = token_unmerge_delta(x_pre, x, xm0, dims) if unmerge_delta else token_unmerge(x, dims)
    return x


def denoise_cond(x0, blocks, dims, n_steps, cond_rows=None, mods=None, reuse=1, merge_first=-1, merge_last=-1,
                 unmerge_delta=False, core_reuse=1, core_first=-1, core_last=-1, block_fn=None):
    """The flow-matching loop with fixed condition rows and per-step
    modulation.  x0: generated rows [S, d]; cond_rows: [C, d] (every
    evaluation starts from them; the Euler update covers the S generated rows
    only); mods: None, [n_blocks, 2, 6, d] for every step or
    [n_steps, n_blocks, 2, 6, d].  Velocity reuse (reuse) or, with
    core_first >= 0 and reuse = 1, core residual reuse as in denoise_core.
    Returns (x_N, stack evaluations, core evaluations)."""
    x = _f64(x0)
    S = x.shape[0]
    C = 0 if cond_rows is None else len(cond_rows)
    cond = np.zeros((0, x.shape[1])) if cond_rows is None else _f64(cond_rows)
    L = len(blocks)
    if core_first >= 0:
        if reuse != 1:
            raise ValueError("core reuse excludes whole-velocity reuse")
        inside = merge_first >= 0 and core_first <= merge_first and merge_last <= core_last
        if not (inside or merge_first < 0 or merge_last < core_first or merge_first > core_last):
            raise ValueError("the token-reduction window must lie inside the core window or outside it")

    def mods_at(i):
        if mods is None:
            return None
        m = _f64(mods)
        return m[i] if m.ndim == 5 else m

    def run(e, lo, hi, i):  # blocks lo..hi, the reduction window re-based when it lies in them
        if lo > hi:
            return e
        mf, ml = (merge_first - lo, merge_last - lo) if merge_first >= 0 and lo <= merge_first <= hi else (-1, -1)
        m = mods_at(i)
        return stack_forward_cond(e, blocks[lo:hi + 1], dims, None if m is None else m[lo:hi + 1], C, mf, ml,
                                  unmerge_delta, block_fn)

    sig = sigmas(n_steps)
    vel = delta = None
    n_fresh = n_core = 0
    for i in range(n_steps):
        if core_first >= 0:
            e = run(np.concatenate([x, cond], axis=0), 0, core_first - 1, i)
            if is_fresh(i, n_steps, core_reuse):
                out = run(e, core_first, core_last, i)
                delta = out - e
                e = out
                n_core += 1
            else:
                e = e + delta
            vel = run(e, core_last + 1, L - 1, i)[:S]
            n_fresh += 1
        elif is_fresh(i, n_steps, reuse):
            vel = run(np.concatenate([x, cond], axis=0), 0, L - 1, i)[:S]
            n_fresh += 1
        x = flow_step(x, vel, sig[i], sig[i + 1])
    return x, n_fresh, n_core


# ----------------------------------------------------------------------------- flow-matching loop
def sigmas(n_steps):
    """Linear grid 1 -> 0: sigma_i = 1 - i/N for i = 0..N (fp64, stored fp32)."""
    return (1.0 - np.arange(n_steps + 1, dtype=np.float64) / n_steps).astype(np.float32)


def is_fresh(i, n_steps, reuse):
    """Whole-velocity reuse: step i runs a fresh DiT evaluation iff
    i % reuse == 0 or it is the last step."""
    return i % reuse == 0 or i == n_steps - 1


def fresh_steps(n_steps, reuse):
    return [i for i in range(n_steps) if is_fresh(i, n_steps, reuse)]


def flow_step(x, v, sigma_cur, sigma_next):
    """Euler step of the flow ODE: x + (sigma_next - sigma_cur) * v."""
    return _f64(x) + (float(sigma_next) - float(sigma_cur)) * _f64(v)


def denoise(x0, blocks, dims, n_steps, reuse, merge_first=-1, merge_last=-1, block_fn=None):
    """N Euler steps over the sigma grid; the velocity is the stack output on
    fresh steps and the last fresh velocity otherwise.  Returns (x_N, number
    of fresh evaluations)."""
    sig = sigmas(n_steps)
    x = _f64(x0)
    v = None
    n_fresh = 0
    for i in range(n_steps):
        if is_fresh(i, n_steps, reuse):
            v = stack_forward(x, blocks, dims, merge_first, merge_last, block_fn)
            n_fresh += 1
        x = flow_step(x, v, sig[i], sig[i + 1])
    return x, n_fresh
