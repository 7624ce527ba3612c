"""Python binding of the h3b C ABI (include/h3b.h).

Argument marshalling only: every step of the block path runs in the CUDA
kernels of ``libh3b.so``.  Tensors are torch tensors used as device memory;
calls enqueue on ``torch.cuda.current_stream()``.  There is no fallback: if
the library is missing, importing this module raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# H3B_LIBRARY names another build of the same library (e.g. libh3b_check.so,
# the index-checked build next to it); by default the in-tree libh3b.so is loaded.
LIB_PATH = os.environ.get("H3B_LIBRARY") or os.path.join(_HERE, "libh3b.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "h3b.h")

BF16, INT8 = 0, 1
EPI_F32, EPI_BF16, EPI_QKV_ROPE, EPI_RESID, EPI_GELU, EPI_I32 = range(6)

if not os.path.exists(LIB_PATH):
    raise ImportError(f"the h3b library is not built ({LIB_PATH}); run `python -m audio_diffusion_transformer_dit_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_i, _f, _p, _sz = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class Dims(ctypes.Structure):
    _fields_ = [("frames", _i), ("rows", _i), ("cols", _i), ("n_audio", _i), ("d", _i), ("n_heads", _i),
                ("head_dim", _i), ("ffn", _i), ("eps", _f), ("rope_theta", _f)]


class BlockWeights(ctypes.Structure):
    _fields_ = [("dtype", _i), ("w_qkv", _p), ("w_o", _p), ("w_fc1", _p), ("w_fc2", _p), ("s_qkv", _p),
                ("s_o", _p), ("s_fc1", _p), ("s_fc2", _p), ("g_attn", _p), ("g_mlp", _p)]


class StackOpts(ctypes.Structure):
    _fields_ = [("merge_first", _i), ("merge_last", _i), ("unmerge_delta", _i), ("core_first", _i),
                ("core_last", _i), ("n_cond", _i), ("mod_steps", _i), ("cond_rows", _p), ("modulation", _p)]


_SIGS = {
    "h3b_status_string": (ctypes.c_char_p, [_i]),
    "h3b_seq_len": (_i, [ctypes.POINTER(Dims), _i]),
    "h3b_workspace_bytes": (_sz, [ctypes.POINTER(Dims), _i, _i]),
    "h3b_workspace_saved_bytes": (_sz, [ctypes.POINTER(Dims), _i]),
    "h3b_block_forward": (_i, [ctypes.POINTER(Dims), ctypes.POINTER(BlockWeights), _p, _i, _p, _sz, _p]),
    "h3b_stack_forward": (_i, [ctypes.POINTER(Dims), ctypes.POINTER(BlockWeights), _i, _i, _i, _p, _p, _sz, _p]),
    "h3b_denoise": (_i, [ctypes.POINTER(Dims), ctypes.POINTER(BlockWeights), _i, _i, _i, _i, _i, _p, _p, _p, _sz,
                         ctypes.POINTER(_i), _p]),
    "h3b_workspace_bytes_ex": (_sz, [ctypes.POINTER(Dims), _i, ctypes.POINTER(StackOpts)]),
    "h3b_stack_forward_ex": (_i, [ctypes.POINTER(Dims), ctypes.POINTER(BlockWeights), _i, ctypes.POINTER(StackOpts),
                                  _p, _p, _sz, _p]),
    "h3b_denoise_ex": (_i, [ctypes.POINTER(Dims), ctypes.POINTER(BlockWeights), _i, ctypes.POINTER(StackOpts), _i, _i,
                            _i, _p, _p, _p, _sz, ctypes.POINTER(_i), ctypes.POINTER(_i), _p]),
    "h3b_quantize_weights": (_i, [_p, _i, _i, _p, _p, _p]),
    "h3b_token_merge": (_i, [ctypes.POINTER(Dims), _p, _p, _p]),
    "h3b_token_unmerge": (_i, [ctypes.POINTER(Dims), _p, _p, _p]),
    "h3b_token_unmerge_delta": (_i, [ctypes.POINTER(Dims), _p, _p, _p, _p]),
    "h3b_flow_step": (_i, [_p, _p, _f, _f, _sz, _p, _p]),
    "h3b_rope_table": (_i, [ctypes.POINTER(Dims), _i, _p, _p]),
    "h3b_rmsnorm": (_i, [_p, _p, _i, _i, _f, _p, _p, _i, _p]),
    "h3b_gemm": (_i, [_p, _p, _i, _i, _i, _i, _i, _p, _p, _p, _p, ctypes.POINTER(Dims), _p, _p, _sz, _p]),
    "h3b_quantize_rows_absmax": (_i, [_p, _p, _i, _i, _p, _p, _p]),
    "h3b_attention": (_i, [_p, _i, _i, _i, _p, _p, _sz, _p]),
    "h3b_exp2_poly": (_i, [_p, _p, _i, _p]),
    "h3b_gelu": (_i, [_p, _p, _sz, _p]),
    "h3b_device_error": (_i, [_p]),
    "h3b_selftest_wait_timeout": (_i, [_i, _p]),
    "h3b_selftest_index_check": (_i, [ctypes.c_longlong, ctypes.c_longlong, _p]),
    "h3b_index_checked": (_i, []),
    "h3b_trace_start": (_i, [_i]),
    "h3b_trace_stop": (_i, [ctypes.POINTER(_i)]),
    "h3b_trace_read": (_i, [_p, _p, _i]),
    "h3b_kernel_name": (ctypes.c_char_p, [_i]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class H3bError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: h3b status {status} ({lib.h3b_status_string(status).decode()})")


def header_functions() -> list:
    """Names of the functions include/h3b.h declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(h3b_\w+)\s*\(", src)))


def _check(status: int, what: str):
    if status != 0:
        raise H3bError(status, what)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def dims_of(wl) -> Dims:
    """Dims from any object with frames, rows, cols, n_audio, d, n_heads,
    head_dim, ffn, eps, rope_theta attributes."""
    return Dims(wl.frames, wl.rows, wl.cols, wl.n_audio, wl.d, wl.n_heads, wl.head_dim, wl.ffn,
                float(wl.eps), float(wl.rope_theta))


def seq_len(dims: Dims, merged: bool = False) -> int:
    return lib.h3b_seq_len(ctypes.byref(dims), int(merged))


def workspace_bytes(dims: Dims, dtype: int = BF16, token_reduction: bool = False) -> int:
    return lib.h3b_workspace_bytes(ctypes.byref(dims), dtype, int(token_reduction))


def workspace_saved_bytes(dims: Dims, dtype: int = BF16) -> int:
    return lib.h3b_workspace_saved_bytes(ctypes.byref(dims), dtype)


def workspace(dims: Dims, dtype: int = BF16, token_reduction: bool = False, device="cuda") -> torch.Tensor:
    n = workspace_bytes(dims, dtype, token_reduction)
    if n == 0:
        raise ValueError("invalid dims for workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)


class Block:
    """Device weights of one block plus the ABI struct that points at them.

    BF16: pass bf16 tensors.  INT8: pass int8 weights and fp32 per-row scales
    (``Block.quantized`` builds them with h3b_quantize_weights)."""

    KEYS = ("w_qkv", "w_o", "w_fc1", "w_fc2")

    def __init__(self, w_qkv, w_o, w_fc1, w_fc2, g_attn, g_mlp, scales=None):
        self.t = dict(w_qkv=w_qkv, w_o=w_o, w_fc1=w_fc1, w_fc2=w_fc2, g_attn=g_attn, g_mlp=g_mlp)
        int8 = w_qkv.dtype == torch.int8
        self.dtype = INT8 if int8 else BF16
        self.scales = scales or {}
        wt = torch.int8 if int8 else torch.bfloat16
        self.c = BlockWeights(self.dtype, *(_ptr(self.t[k], wt, k) for k in self.KEYS),
                              *((_ptr(self.scales[k], torch.float32, "s_" + k) if int8 else None) for k in self.KEYS),
                              _ptr(g_attn, torch.float32, "g_attn"), _ptr(g_mlp, torch.float32, "g_mlp"))

    @classmethod
    def from_dict(cls, w: dict) -> "Block":
        return cls(w["w_qkv"], w["w_o"], w["w_fc1"], w["w_fc2"], w["g_attn"], w["g_mlp"])

    @classmethod
    def quantized(cls, w: dict) -> "Block":
        qs, ss = {}, {}
        for k in cls.KEYS:
            qs[k], ss[k] = quantize_weights(w[k])
        return cls(qs["w_qkv"], qs["w_o"], qs["w_fc1"], qs["w_fc2"], w["g_attn"], w["g_mlp"], scales=ss)


def _blocks_array(blocks: Sequence[Block]):
    arr = (BlockWeights * max(1, len(blocks)))()
    for i, b in enumerate(blocks):
        arr[i] = b.c
    return arr


def block_forward(dims: Dims, block: Block, x: torch.Tensor, ws: torch.Tensor, merged: bool = False,
                  staging: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One block in place on x [S, d] fp32.  If x is a host tensor, it is
    copied into ``staging`` (a device buffer of the same shape), processed
    there and copied back into x (host-buffer entry point)."""
    if not x.is_cuda:
        if staging is None:
            staging = torch.empty(x.shape, dtype=torch.float32, device="cuda")
        staging.copy_(x, non_blocking=True)
        block_forward(dims, block, staging, ws, merged)
        x.copy_(staging, non_blocking=True)
        return x
    _check(lib.h3b_block_forward(ctypes.byref(dims), ctypes.byref(block.c), _ptr(x, torch.float32, "x"),
                                 int(merged), _ptr(ws, None, "ws"), ws.numel() * ws.element_size(), _stream()),
           "h3b_block_forward")
    return x


class HostPipeline:
    """Streams token batches that live in host memory through the block (or
    stack) on the device.  Copy-in of step i+1 and copy-out of step i-1 run on
    their own CUDA streams while step i computes, with ``depth`` device buffers
    in rotation; the workspace is used by one compute stream, in order.

    ``submit(x_in, x_out)`` enqueues one step: x_in (pinned host, [S, d] fp32)
    is copied in, processed, and the result copied to x_out (pinned host).
    The call returns at once; x_in must stay untouched and x_out is valid only
    after ``synchronize()`` (or once a later submit has reused its buffer).

    Three buffers (the default) let step i+1's copy-in start while step i-1's
    copy-out is still running; with two, that copy-in waits for it and the
    loop runs at compute + copy-out + copy-in per two steps."""

    def __init__(self, dims: Dims, blocks, ws: torch.Tensor, shape, depth: int = 3, merge_first: int = -1,
                 merge_last: int = -1):
        self.dims, self.ws = dims, ws
        self.blocks = list(blocks) if isinstance(blocks, (list, tuple)) else [blocks]
        self.mf, self.ml = merge_first, merge_last
        self.bufs = [torch.empty(shape, dtype=torch.float32, device="cuda") for _ in range(depth)]
        self.s_in, self.s_run, self.s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        self.ev_in = [torch.cuda.Event() for _ in range(depth)]
        self.ev_run = [torch.cuda.Event() for _ in range(depth)]
        self.ev_out = [torch.cuda.Event() for _ in range(depth)]
        self.i = 0

    def submit(self, x_in: torch.Tensor, x_out: torch.Tensor):
        b = self.i % len(self.bufs)
        buf = self.bufs[b]
        self.s_in.wait_event(self.ev_out[b])  # the previous copy-out from this buffer is done
        with torch.cuda.stream(self.s_in):
            buf.copy_(x_in, non_blocking=True)
            self.ev_in[b].record(self.s_in)
        self.s_run.wait_event(self.ev_in[b])
        with torch.cuda.stream(self.s_run):
            if len(self.blocks) == 1 and self.mf < 0:
                block_forward(self.dims, self.blocks[0], buf, self.ws)
            else:
                stack_forward(self.dims, self.blocks, buf, self.ws, self.mf, self.ml)
            self.ev_run[b].record(self.s_run)
        self.s_out.wait_event(self.ev_run[b])
        with torch.cuda.stream(self.s_out):
            x_out.copy_(buf, non_blocking=True)
            self.ev_out[b].record(self.s_out)
        self.i += 1

    def synchronize(self):
        self.s_out.synchronize()


def stack_forward(dims: Dims, blocks: Sequence[Block], x: torch.Tensor, ws: torch.Tensor,
                  merge_first: int = -1, merge_last: int = -1) -> torch.Tensor:
    arr = _blocks_array(blocks)
    _check(lib.h3b_stack_forward(ctypes.byref(dims), arr, len(blocks), merge_first, merge_last,
                                 _ptr(x, torch.float32, "x"), _ptr(ws, None, "ws"), ws.numel(), _stream()),
           "h3b_stack_forward")
    return x


def denoise(dims: Dims, blocks: Sequence[Block], x: torch.Tensor, v: torch.Tensor, ws: torch.Tensor, n_steps: int,
            reuse: int, merge_first: int = -1, merge_last: int = -1) -> int:
    arr = _blocks_array(blocks)
    nf = ctypes.c_int(0)
    _check(lib.h3b_denoise(ctypes.byref(dims), arr, len(blocks), merge_first, merge_last, n_steps, reuse,
                           _ptr(x, torch.float32, "x"), _ptr(v, torch.float32, "v"), _ptr(ws, None, "ws"),
                           ws.numel(), ctypes.byref(nf), _stream()), "h3b_denoise")
    return nf.value


def stack_opts(merge_first: int = -1, merge_last: int = -1, unmerge_delta: bool = False, core_first: int = -1,
               core_last: int = -1, n_cond: int = 0, cond_rows: Optional[torch.Tensor] = None,
               modulation: Optional[torch.Tensor] = None) -> StackOpts:
    """Options of the extended entry points.  cond_rows: fp32 [n_cond, d]
    (the loop's fixed condition rows); modulation: fp32 [n_blocks, 2, 6, d]
    (every step) or [n_steps, n_blocks, 2, 6, d] (one slice per step).  The
    tensors are kept referenced by the returned object."""
    if cond_rows is not None and n_cond == 0:
        n_cond = cond_rows.shape[0]
    mod_steps = 0
    if modulation is not None:
        if modulation.dim() not in (4, 5) or tuple(modulation.shape[-3:-1]) != (2, 6):
            raise ValueError("modulation must be [n_blocks, 2, 6, d] or [n_steps, n_blocks, 2, 6, d]")
        mod_steps = modulation.shape[0] if modulation.dim() == 5 else 1
    o = StackOpts(merge_first, merge_last, int(unmerge_delta), core_first, core_last, n_cond, mod_steps,
                  _ptr(cond_rows, torch.float32, "cond_rows"), _ptr(modulation, torch.float32, "modulation"))
    o._keep = (cond_rows, modulation)
    return o


def workspace_ex(dims: Dims, opts: StackOpts, dtype: int = BF16, device="cuda") -> torch.Tensor:
    n = lib.h3b_workspace_bytes_ex(ctypes.byref(dims), dtype, ctypes.byref(opts))
    if n == 0:
        raise ValueError("invalid dims / options for workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)


def stack_forward_ex(dims: Dims, blocks: Sequence[Block], x: torch.Tensor, ws: torch.Tensor,
                     opts: StackOpts) -> torch.Tensor:
    arr = _blocks_array(blocks)
    _check(lib.h3b_stack_forward_ex(ctypes.byref(dims), arr, len(blocks), ctypes.byref(opts),
                                    _ptr(x, torch.float32, "x"), _ptr(ws, None, "ws"), ws.numel(), _stream()),
           "h3b_stack_forward_ex")
    return x


def denoise_ex(dims: Dims, blocks: Sequence[Block], x: torch.Tensor, v: torch.Tensor, ws: torch.Tensor, n_steps: int,
               opts: StackOpts, reuse: int = 1, core_reuse: int = 1):
    """Returns (stack evaluations, core evaluations)."""
    arr = _blocks_array(blocks)
    nf, nc = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.h3b_denoise_ex(ctypes.byref(dims), arr, len(blocks), ctypes.byref(opts), n_steps, reuse, core_reuse,
                              _ptr(x, torch.float32, "x"), _ptr(v, torch.float32, "v"), _ptr(ws, None, "ws"),
                              ws.numel(), ctypes.byref(nf), ctypes.byref(nc), _stream()), "h3b_denoise_ex")
    return nf.value, nc.value


def quantize_weights(w: torch.Tensor):
    rows, k = w.shape
    q = torch.empty((rows, k), dtype=torch.int8, device=w.device)
    s = torch.empty(rows, dtype=torch.float32, device=w.device)
    _check(lib.h3b_quantize_weights(_ptr(w, torch.bfloat16, "w"), rows, k, q.data_ptr(), s.data_ptr(), _stream()),
           "h3b_quantize_weights")
    return q, s


def token_merge(dims: Dims, x: torch.Tensor, xm: torch.Tensor) -> torch.Tensor:
    _check(lib.h3b_token_merge(ctypes.byref(dims), _ptr(x, torch.float32, "x"), _ptr(xm, torch.float32, "xm"),
                               _stream()), "h3b_token_merge")
    return xm


def token_unmerge(dims: Dims, xm: torch.Tensor, x: torch.Tensor) -> torch.Tensor:
    _check(lib.h3b_token_unmerge(ctypes.byref(dims), _ptr(xm, torch.float32, "xm"), _ptr(x, torch.float32, "x"),
                                 _stream()), "h3b_token_unmerge")
    return x


def token_unmerge_delta(dims: Dims, x: torch.Tensor, ym: torch.Tensor, xm0: torch.Tensor) -> torch.Tensor:
    """x (the pre-merge tokens) += the merged blocks' update ym - xm0, broadcast to both columns of each pair."""
    _check(lib.h3b_token_unmerge_delta(ctypes.byref(dims), _ptr(x, torch.float32, "x"), _ptr(ym, torch.float32, "ym"),
                                       _ptr(xm0, torch.float32, "xm0"), _stream()), "h3b_token_unmerge_delta")
    return x


def flow_step(x: torch.Tensor, v: torch.Tensor, sigma_cur: float, sigma_next: float,
              x_copy: Optional[torch.Tensor] = None) -> torch.Tensor:
    _check(lib.h3b_flow_step(_ptr(x, torch.float32, "x"), _ptr(v, torch.float32, "v"), sigma_cur, sigma_next,
                             x.numel(), _ptr(x_copy, torch.float32, "x_copy"), _stream()), "h3b_flow_step")
    return x


def rope_table(dims: Dims, merged: bool = False, table: Optional[torch.Tensor] = None) -> torch.Tensor:
    if table is None:
        table = torch.empty((seq_len(dims, merged), dims.head_dim // 2, 2), dtype=torch.float32, device="cuda")
    _check(lib.h3b_rope_table(ctypes.byref(dims), int(merged), _ptr(table, torch.float32, "table"), _stream()),
           "h3b_rope_table")
    return table


def rmsnorm(x: torch.Tensor, g: torch.Tensor, eps: float, int8: bool = False):
    rows, d = x.shape
    if int8:
        out = torch.empty((rows, d), dtype=torch.int8, device=x.device)
        sc = torch.empty(rows, dtype=torch.float32, device=x.device)
    else:
        out = torch.empty((rows, d), dtype=torch.bfloat16, device=x.device)
        sc = None
    _check(lib.h3b_rmsnorm(_ptr(x, torch.float32, "x"), _ptr(g, torch.float32, "g"), rows, d, eps, out.data_ptr(),
                           None if sc is None else sc.data_ptr(), INT8 if int8 else BF16, _stream()), "h3b_rmsnorm")
    return (out, sc) if int8 else out


def gemm(A: torch.Tensor, B: torch.Tensor, epilogue: int, C: torch.Tensor, scale_a=None, scale_b=None,
         rope: Optional[torch.Tensor] = None, dims: Optional[Dims] = None, row_absmax=None,
         scratch: Optional[torch.Tensor] = None) -> torch.Tensor:
    M, K = A.shape
    N = B.shape[0]
    ab = INT8 if A.dtype == torch.int8 else BF16
    _check(lib.h3b_gemm(_ptr(A, None, "A"), _ptr(B, A.dtype, "B"), M, N, K, ab, epilogue, _ptr(C, None, "C"),
                        _ptr(scale_a, torch.float32, "scale_a"), _ptr(scale_b, torch.float32, "scale_b"),
                        _ptr(rope, torch.float32, "rope"), None if dims is None else ctypes.byref(dims),
                        _ptr(row_absmax, torch.float32, "row_absmax"), _ptr(scratch, None, "scratch"),
                        0 if scratch is None else scratch.numel() * scratch.element_size(), _stream()), "h3b_gemm")
    return C


def quantize_rows_absmax(a: torch.Tensor, absmax: torch.Tensor):
    rows, k = a.shape
    q = torch.empty((rows, k), dtype=torch.int8, device=a.device)
    s = torch.empty(rows, dtype=torch.float32, device=a.device)
    _check(lib.h3b_quantize_rows_absmax(_ptr(a, torch.bfloat16, "a"), _ptr(absmax, torch.float32, "absmax"), rows,
                                        k, q.data_ptr(), s.data_ptr(), _stream()), "h3b_quantize_rows_absmax")
    return q, s


def attention(qkv: torch.Tensor, n_heads: int, head_dim: int, o: Optional[torch.Tensor] = None,
              scratch: Optional[torch.Tensor] = None) -> torch.Tensor:
    S = qkv.shape[0]
    if o is None:
        o = torch.empty((S, n_heads * head_dim), dtype=torch.bfloat16, device=qkv.device)
    _check(lib.h3b_attention(_ptr(qkv, torch.bfloat16, "qkv"), S, n_heads, head_dim, _ptr(o, torch.bfloat16, "o"),
                             _ptr(scratch, None, "scratch"),
                             0 if scratch is None else scratch.numel() * scratch.element_size(), _stream()),
           "h3b_attention")
    return o


def exp2_poly(x: torch.Tensor) -> torch.Tensor:
    y = torch.empty_like(x)
    _check(lib.h3b_exp2_poly(_ptr(x, torch.float32, "x"), y.data_ptr(), x.numel(), _stream()), "h3b_exp2_poly")
    return y


def gelu(x: torch.Tensor) -> torch.Tensor:
    y = torch.empty_like(x)
    _check(lib.h3b_gelu(_ptr(x, torch.float32, "x"), y.data_ptr(), x.numel(), _stream()), "h3b_gelu")
    return y


def device_error() -> int:
    return lib.h3b_device_error(_stream())


def index_checked() -> bool:
    """True when the loaded library is the index-checked build (libh3b_check.so)."""
    return bool(lib.h3b_index_checked())


def selftest_index_check(i: int, n: int) -> None:
    """Passes index i of extent n through the kernels' index check without
    touching memory (records (4 << 8) | 99 in the checked build when i is out
    of range; nothing in the default build)."""
    _check(lib.h3b_selftest_index_check(i, n, _stream()), "h3b_selftest_index_check")


class Graph:
    """Library calls captured once into a CUDA graph and replayed with one
    host call per replay: the same kernels (with their programmatic-launch
    edges), arguments and buffers.  ``fn`` issues the calls on the current
    stream; every tensor it touches must stay alive and in place while the
    graph exists, and the library must have run once on this device before
    the capture (its first call sets up per-device state).  Tracing
    (``Trace``) does not see replayed launches."""

    def __init__(self, fn):
        self.g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g):
            fn()

    def replay(self):
        self.g.replay()


class Trace:
    """Per-launch CUDA-event tracing of every kernel the library launches."""

    def __init__(self, capacity: int = 4096):
        self.capacity = capacity
        self.records = []

    def __enter__(self):
        _check(lib.h3b_trace_start(self.capacity), "h3b_trace_start")
        return self

    def __exit__(self, *exc):
        n = ctypes.c_int(0)
        _check(lib.h3b_trace_stop(ctypes.byref(n)), "h3b_trace_stop")
        ids = (ctypes.c_int * max(1, n.value))()
        ms = (ctypes.c_float * max(1, n.value))()
        got = lib.h3b_trace_read(ids, ms, n.value)
        self.records = [(lib.h3b_kernel_name(ids[i]).decode(), ms[i]) for i in range(got)]
        return False

    def by_kernel(self) -> dict:
        out = {}
        for name, t in self.records:
            c, s = out.get(name, (0, 0.0))
            out[name] = (c + 1, s + t)
        return out
