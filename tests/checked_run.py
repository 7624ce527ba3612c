"""One fixed set of library calls that reaches every kernel family and every
index path the hot path has: ragged tails of rows, keys and GEMM tiles, the
split-K tail of a residual GEMM, the key-split tail of attention with its
combine kernel, the folded RMSNorm of a bf16 stack, token reduction with the
plain and the delta unmerge, condition rows with modulation, the INT8 block,
the denoising loop and the unit kernels.  Saves every output and the device
error word to an .npz.

    python tests/checked_run.py OUT.npz

test_gpu_checked.py runs it once with the default library and once with
H3B_LIBRARY pointing at libh3b_check.so (every hand-indexed global access
checked against its buffer's extent) and compares the two."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402
from audio_diffusion_transformer_dit_b200 import h3b  # noqa: E402


def main(out_path: str) -> None:
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    res = {}

    def keep(name, t):
        torch.cuda.synchronize()
        res[name] = t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()

    tiny = W.WORKLOADS["block_d256_s288"]
    dm = h3b.dims_of(tiny)

    # blocks: bf16, merged geometry, INT8
    blk = h3b.Block.from_dict(W.block_weights(tiny, 0, dev))
    for merged in (False, True):
        x = W.initial_tokens(tiny, dev, seq=h3b.seq_len(dm, merged))
        h3b.block_forward(dm, blk, x, h3b.workspace(dm), merged=merged)
        keep(f"block_bf16_m{int(merged)}", x)
    t8 = tiny.with_(dtype=h3b.INT8)
    blk8 = h3b.Block.quantized(W.block_weights(t8, 0, dev))
    x = W.initial_tokens(t8, dev)
    h3b.block_forward(dm, blk8, x, h3b.workspace(dm, h3b.INT8))
    keep("block_int8", x)

    # stacks with a reduction window: bf16 (folded norms) and INT8
    for dt, name in ((h3b.BF16, "bf16"), (h3b.INT8, "int8")):
        wl = tiny.with_(n_blocks=5, depth_scaled_init=True, seed=7, dtype=dt)
        ws_ = [W.block_weights(wl, l, dev) for l in range(5)]
        blocks = [h3b.Block.quantized(w) if dt == h3b.INT8 else h3b.Block.from_dict(w) for w in ws_]
        x = W.initial_tokens(wl, dev)
        h3b.stack_forward(dm, blocks, x, h3b.workspace(dm, dt, True), 1, 3)
        keep(f"stack_{name}", x)

    # delta unmerge with condition rows and per-block modulation
    wl = tiny.with_(n_blocks=4, depth_scaled_init=True, seed=9)
    blocks = [h3b.Block.from_dict(W.block_weights(wl, l, dev)) for l in range(4)]
    C = 20
    mod = W.normal_tensor((4, 2, 6, wl.d), 31, dev, 0.1)
    o = h3b.stack_opts(1, 2, unmerge_delta=True, n_cond=C, modulation=mod)
    x = W.initial_tokens(wl, dev, seq=wl.seq + C)
    h3b.stack_forward_ex(dm, blocks, x, h3b.workspace_ex(dm, o), o)
    keep("stack_ex_delta_cond_mod", x)

    # denoising loop with velocity reuse and a reduction window (Euler step + fused copy)
    x = W.initial_tokens(wl, dev)
    v = torch.empty_like(x)
    h3b.denoise(dm, blocks, x, v, h3b.workspace(dm, h3b.BF16, True), 5, 2, 1, 2)
    keep("denoise", x)

    # attention: ragged key tails (D = 128 and 64) and the key-split tail + combine
    for S, H, D in ((300, 3, 128), (2049, 2, 64), (6400, 24, 128)):
        qkv = W.normal_tensor((S, 3 * H * D), 40 + S, dev, 1.5, dtype=torch.bfloat16)
        scr = torch.empty(2 * S * H * D, dtype=torch.float32, device=dev)
        keep(f"attention_{S}_{H}_{D}", h3b.attention(qkv, H, D, scratch=scr))

    # residual GEMM whose last wave is split along K (6400 x 3072: 300 pair tiles)
    A = W.normal_tensor((6400, 256), 51, dev, dtype=torch.bfloat16)
    B = W.normal_tensor((3072, 256), 52, dev, 0.05, dtype=torch.bfloat16)
    Cm = W.normal_tensor((6400, 3072), 53, dev)
    scr = torch.empty(6400 * 3072, dtype=torch.float32, device=dev)
    keep("gemm_resid_split", h3b.gemm(A, B, h3b.EPI_RESID, Cm, scratch=scr))
    # ragged single-CTA GEMMs: bf16 out and INT8 GELU with row maxima
    A = W.normal_tensor((300, 512), 54, dev, dtype=torch.bfloat16)
    B = W.normal_tensor((768, 512), 55, dev, 0.05, dtype=torch.bfloat16)
    keep("gemm_bf16_ragged", h3b.gemm(A, B, h3b.EPI_BF16, torch.empty((300, 768), dtype=torch.bfloat16, device=dev)))
    A8 = W.int8_tensor((129, 1024), 56, dev)
    B8 = W.int8_tensor((288, 1024), 57, dev)
    sa = W.uniform_tensor((129,), 58, dev, 1e-3, 2e-3)
    sb = W.uniform_tensor((288,), 59, dev, 1e-3, 2e-3)
    amax = torch.zeros(129, dtype=torch.float32, device=dev)
    g = h3b.gemm(A8, B8, h3b.EPI_GELU, torch.empty((129, 288), dtype=torch.bfloat16, device=dev), scale_a=sa,
                 scale_b=sb, row_absmax=amax)
    keep("gemm_int8_gelu", g)
    keep("gemm_int8_gelu_rowmax", amax)

    # norms and quantisers (row-per-CTA paths, the 8-element known-max path)
    x = W.normal_tensor((7, 5120), 60, dev)
    gain = W.uniform_tensor((5120,), 61, dev, 0.5, 1.5)
    q, s = h3b.rmsnorm(x, gain, 1e-6, int8=True)
    keep("rmsnorm_int8_q", q)
    keep("rmsnorm_int8_s", s)
    keep("rmsnorm_bf16", h3b.rmsnorm(x, gain, 1e-6))
    for k in (1000, 20480):
        a = (W.normal_tensor((5, k), 62 + k, dev) * 3).to(torch.bfloat16)
        q, s = h3b.quantize_rows_absmax(a, a.float().abs().amax(dim=1).contiguous())
        keep(f"quant_absmax_{k}_q", q)
        keep(f"quant_absmax_{k}_s", s)
    q, s = h3b.quantize_weights((W.normal_tensor((33, 5120), 63, dev) * 0.02).to(torch.bfloat16))
    keep("quant_rows_q", q)
    keep("quant_rows_s", s)

    # unit kernels: merge / unmerge, Euler step with copy, RoPE table, GELU
    x = W.initial_tokens(tiny, dev)
    xm = torch.empty((h3b.seq_len(dm, True), tiny.d), device=dev)
    h3b.token_merge(dm, x, xm)
    keep("merge", xm)
    y = torch.empty_like(x)
    h3b.token_unmerge(dm, xm, y)
    keep("unmerge", y)
    xc = torch.empty_like(x)
    h3b.flow_step(x, W.normal_tensor(x.shape, 64, dev), 0.75, 0.7, xc)
    keep("flow", x)
    keep("flow_copy", xc)
    keep("rope_merged", h3b.rope_table(dm, True))
    keep("gelu", h3b.gelu(W.normal_tensor((1001,), 65, dev, 4.0)))

    torch.cuda.synchronize()
    res["device_error"] = np.array([h3b.device_error()])
    # the check itself: an index past its extent, through the self-test kernel
    # (no memory is touched in either build)
    h3b.selftest_index_check(5, 5)
    torch.cuda.synchronize()
    res["selftest_error"] = np.array([h3b.device_error()])
    h3b.selftest_index_check(4, 5)
    torch.cuda.synchronize()
    res["selftest_in_range_error"] = np.array([h3b.device_error()])
    res["index_checked"] = np.array([int(h3b.index_checked())])
    np.savez(out_path, **res)


if __name__ == "__main__":
    main(sys.argv[1])
