"""ctypes binding of ``libtbik.so`` (argument marshalling only).

Every step of the computation runs in the library's CUDA kernels; this module
only turns torch tensors into device pointers and sizes, allocates workspaces
with torch (the library itself never allocates), and raises on a non-zero
status.  There is no fallback: if the library cannot be loaded, importing the
functions raises.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtbik.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "tbik.h")

TBIK_OK = 0
TBIK_ERR_ARG = 1
TBIK_ERR_SHAPE = 2
TBIK_ERR_ALIGN = 3
TBIK_ERR_WORKSPACE = 4
TBIK_ERR_CUDA = 5
TBIK_ERR_TIMEOUT = 6
TBIK_ERR_TARGET = 7
TBIK_ERR_POSITION = 8
TBIK_ERR_UNSUPPORTED = 9

EXACT = 0x1
TC = 0x2
NONINV = 0x4
B_KN = 0x00
B_NK = 0x10
OUT_F32 = 0x000
OUT_BF16 = 0x100
SWIGLU_OUT = 0x200
DEBUG_WITHHOLD_ACC_ARRIVE = 0x1
DEBUG_TILE128 = 0x2
VOCAB_LEAF = 64
T_MAX = 8

_lock = threading.Lock()
_lib = None


class TbikError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: tbik status {status} ({status_string(status)})")


class RopeSwigluArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("q_out", ctypes.c_void_p), ("k_out", ctypes.c_void_p),
        ("pos", ctypes.c_void_p), ("table", ctypes.c_void_p),
        ("tokens", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("max_pos", ctypes.c_int),
        ("g", ctypes.c_void_p), ("u", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("n", ctypes.c_longlong), ("in_f32", ctypes.c_int),
    ]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load ``libtbik.so`` (raises OSError if it is missing: build it first)."""
    global _lib
    with _lock:
        if _lib is not None and path == LIB_PATH:
            return _lib
        if not os.path.exists(path):
            raise OSError(f"{path} not found: run `python -m invariant_tree_ordered_b200.build`")
        lib = ctypes.CDLL(path)
        vp, i32, u32, sz, f32, f64, ull = (ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t,
                                            ctypes.c_float, ctypes.c_double, ctypes.c_ulonglong)
        sigs = {
            "tbik_version": (ctypes.c_char_p, []),
            "tbik_status_string": (ctypes.c_char_p, [i32]),
            "tbik_gemm_workspace": (sz, [i32, i32, i32, i32, i32, u32]),
            "tbik_gemm": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, u32, vp, sz, vp]),
            "tbik_gemm_residual": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, u32, vp, sz, vp]),
            "tbik_rmsnorm_residual": (i32, [vp, vp, vp, vp, vp, i32, i32, f32, i32, vp]),
            "tbik_rope_table": (i32, [vp, i32, i32, f64, vp]),
            "tbik_rope_swiglu_fp32": (i32, [ctypes.POINTER(RopeSwigluArgs), vp]),
            "tbik_logprob_workspace": (sz, [i32, i32, i32, i32, i32, u32]),
            "tbik_logprob": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, u32, vp, sz, vp]),
            "tbik_attention": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]),
            "tbik_attention_tc_workspace": (sz, [i32, i32, i32, i32, i32]),
            "tbik_attention_tc": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, sz, vp]),
            "tbik_embedding": (i32, [vp, vp, vp, i32, i32, i32, vp]),
            "tbik_transpose": (i32, [vp, vp, i32, i32, vp]),
            "tbik_tree_combine": (i32, [vp, vp, ctypes.c_longlong, i32, u32, vp, vp]),
            "tbik_logprob_partial_workspace": (sz, [i32, i32, i32, i32, i32, u32]),
            "tbik_logprob_partial": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, u32, vp, sz, vp]),
            "tbik_logprob_combine": (i32, [vp, vp, vp, i32, i32, i32, vp]),
            "tbik_get_error": (i32, [vp]),
            "tbik_debug_set": (i32, [u32, ull]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        if path == LIB_PATH:
            _lib = lib
        return lib


def declared_functions(header: str = HEADER):
    """Names of the functions ``include/tbik.h`` declares."""
    with open(header) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tbik_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    try:
        return load_library().tbik_status_string(status).decode()
    except OSError:
        return "library not loaded"


def _check(status: int, what: str):
    if status != TBIK_OK:
        raise TbikError(status, what)


# ------------------------------------------------------------ torch plumbing

def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need_out(t, dtype, shape, name="out"):
    """A caller-provided output: a contiguous CUDA tensor of this dtype and shape."""
    _need(t, dtype, name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _need(t, dtype, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _workspace(nbytes: int, device, workspace):
    torch = _torch()
    if nbytes == (1 << 64) - 1 or nbytes < 0:
        raise TbikError(TBIK_ERR_SHAPE, "workspace query")
    if nbytes == 0:
        return workspace, 0
    if workspace is not None:
        return workspace, workspace.numel() * workspace.element_size()
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, nbytes


# ---------------------------------------------------------------- entry points

def gemm_workspace(M, N, K, T, leaf, mode) -> int:
    return int(load_library().tbik_gemm_workspace(M, N, K, T, leaf, mode))


def gemm(A, B, *, T: int = 1, leaf: int = 256, tc: bool = True, noninv: bool = False, b_nk: bool = False,
         out_bf16: bool = False, swiglu: bool = False, residual=None, out=None, workspace=None, stream=None):
    """C = A @ B with the K reduction in tree order (see tbik_gemm in tbik.h).
    swiglu: B holds gate/up columns interleaved in blocks of 32 and C is the
    bf16 SwiGLU [M, N/2] of the fp32 roots (TBIK_SWIGLU_OUT).
    residual: bf16 [M, N]; C = bf16(root + residual) (tbik_gemm_residual);
    ``out`` may be the residual tensor itself (in place)."""
    torch = _torch()
    lib = load_library()
    _need(A, torch.bfloat16, "A")
    _need(B, torch.bfloat16, "B")
    M, K = A.shape
    N = B.shape[0] if b_nk else B.shape[1]
    kb = B.shape[1] if b_nk else B.shape[0]
    if kb != K:
        raise ValueError("inner dimensions differ")
    mode = (TC if tc else EXACT) | (NONINV if noninv else 0) | (B_NK if b_nk else B_KN)
    if residual is not None:
        if swiglu:
            raise ValueError("residual and swiglu outputs are exclusive")
        _need(residual, torch.bfloat16, "residual")
        if tuple(residual.shape) != (M, N):
            raise ValueError("residual must be [M, N]")
        if out is None:
            out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
        _need_out(out, torch.bfloat16, (M, N))
        ws, wsb = _workspace(lib.tbik_gemm_workspace(M, N, K, T, leaf, mode | OUT_BF16), A.device, workspace)
        _check(lib.tbik_gemm_residual(_ptr(A), _ptr(B), _ptr(residual), _ptr(out), M, N, K, T, leaf, mode,
                                      _ptr(ws), wsb, _stream_handle(stream)), "tbik_gemm_residual")
        return out
    mode |= OUT_BF16 if out_bf16 else OUT_F32
    if swiglu:
        mode |= SWIGLU_OUT
    out_dtype = torch.bfloat16 if (swiglu or out_bf16) else torch.float32
    out_shape = (M, N // 2) if swiglu else (M, N)
    if out is None:
        out = torch.empty(out_shape, dtype=out_dtype, device=A.device)
    _need_out(out, out_dtype, out_shape)
    ws, wsb = _workspace(lib.tbik_gemm_workspace(M, N, K, T, leaf, mode), A.device, workspace)
    _check(lib.tbik_gemm(_ptr(A), _ptr(B), _ptr(out), M, N, K, T, leaf, mode, _ptr(ws), wsb,
                         _stream_handle(stream)), "tbik_gemm")
    return out


def rmsnorm_residual(x, res, gamma, *, eps: float = 1e-6, T: int = 1, y=None, res_out=None, want_res_out=True,
                     stream=None):
    torch = _torch()
    lib = load_library()
    for t, n in ((x, "x"), (res, "res"), (gamma, "gamma")):
        if t is not None or n != "res":  # res None: no residual input, r = f32(x)
            _need(t, torch.bfloat16, n)
    if x.dim() != 2:
        raise ValueError("x must be [tokens, H]")
    tokens, H = x.shape
    if res is not None and res.shape != x.shape:
        raise ValueError("res must have the shape of x")
    if tuple(gamma.shape) != (H,):
        raise ValueError("gamma must be [H]")
    if y is None:
        y = torch.empty_like(x)
    _need_out(y, torch.bfloat16, x.shape, "y")
    if res_out is None and want_res_out:
        res_out = torch.empty_like(x)
    if res_out is not None:
        _need_out(res_out, torch.bfloat16, x.shape, "res_out")
    _check(lib.tbik_rmsnorm_residual(_ptr(x), _ptr(res), _ptr(gamma), _ptr(y), _ptr(res_out), tokens, H,
                                     float(eps), T, _stream_handle(stream)), "tbik_rmsnorm_residual")
    return y, res_out


def rope_table(max_pos: int, head_dim: int = 128, base: float = 1e6, device="cuda", stream=None):
    torch = _torch()
    lib = load_library()
    t = torch.empty((max_pos, head_dim // 2, 2), dtype=torch.float32, device=device)
    _check(lib.tbik_rope_table(_ptr(t), max_pos, head_dim, float(base), _stream_handle(stream)), "tbik_rope_table")
    return t


def rope_swiglu(*, q=None, k=None, pos=None, table=None, q_out=None, k_out=None, g=None, u=None, out=None,
                stream=None):
    """RoPE on q/k and/or SwiGLU on g/u in one call (see tbik_rope_swiglu_fp32)."""
    torch = _torch()
    lib = load_library()
    a = RopeSwigluArgs()
    if q is not None or k is not None:
        ref = q if q is not None else k
        _need(ref, torch.bfloat16, "q/k")
        _need(pos, torch.int32, "pos")
        _need(table, torch.float32, "table")
        if ref.dim() != 3:
            raise ValueError("q and k must be [tokens, heads, head_dim]")
        tokens, heads, hd = ref.shape
        for t, n in ((q, "q"), (k, "k")):
            if t is not None:
                _need(t, torch.bfloat16, n)
                if t.shape != ref.shape:
                    raise ValueError("q and k must share one shape")
        if pos.numel() != tokens:
            raise ValueError("pos must hold one position per token")
        if table.dim() != 3 or tuple(table.shape[1:]) != (hd // 2, 2):
            raise ValueError("table must be [max_pos, head_dim/2, 2]")
        if q is not None and q_out is None:
            q_out = torch.empty_like(q)
        if k is not None and k_out is None:
            k_out = torch.empty_like(k)
        if q is not None:
            _need_out(q_out, torch.bfloat16, ref.shape, "q_out")
        if k is not None:
            _need_out(k_out, torch.bfloat16, ref.shape, "k_out")
        a.q, a.k, a.q_out, a.k_out = _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out)
        a.pos, a.table = _ptr(pos), _ptr(table)
        a.tokens, a.heads, a.head_dim, a.max_pos = tokens, heads, hd, table.shape[0]
    if g is not None:
        if g.dtype not in (torch.bfloat16, torch.float32) or u.dtype != g.dtype:
            raise TypeError("g and u must both be bf16 or both fp32")
        _need(g, g.dtype, "g")
        _need(u, g.dtype, "u")
        if u.shape != g.shape:
            raise ValueError("g and u must share one shape")
        if out is None:
            out = torch.empty(g.shape, dtype=torch.bfloat16, device=g.device)
        _need_out(out, torch.bfloat16, g.shape)
        a.g, a.u, a.out, a.n, a.in_f32 = _ptr(g), _ptr(u), _ptr(out), g.numel(), int(g.dtype == torch.float32)
    _check(lib.tbik_rope_swiglu_fp32(ctypes.byref(a), _stream_handle(stream)), "tbik_rope_swiglu_fp32")
    return q_out, k_out, out


# keys per tree leaf: the exact mode's chunk and the tensor-core mode's leaf (two 64-key MMA chunks)
ATTENTION_CHUNK = 64
ATTENTION_TC_LEAF = 128


def attention_tc_workspace(batch, seq, heads, head_dim, chunk=ATTENTION_TC_LEAF) -> int:
    n = load_library().tbik_attention_tc_workspace(batch, seq, heads, head_dim, chunk)
    if n == (1 << 64) - 1:
        raise TbikError(TBIK_ERR_SHAPE, "tbik_attention_tc_workspace: unsupported shape")
    return n


def attention(q, k, v, *, out=None, chunk=None, tc: bool = False, workspace=None, stream=None):
    """Causal attention with the key reduction in tree order; q, k, v bf16
    [batch, seq, heads, head_dim].  tc=False: tbik_attention (exact order on
    the CUDA cores, leaves of `chunk` = 64 keys); tc=True: tbik_attention_tc
    (tensor cores, leaves of 128 keys; a workspace is allocated when none is
    given)."""
    if chunk is None:
        chunk = ATTENTION_TC_LEAF if tc else ATTENTION_CHUNK
    torch = _torch()
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share the shape [batch, seq, heads, head_dim]")
    B, S, NH, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    _need_out(out, torch.bfloat16, q.shape)
    if not tc:
        _check(lib.tbik_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, S, NH, D, chunk, _stream_handle(stream)),
               "tbik_attention")
        return out
    need = attention_tc_workspace(B, S, NH, D, chunk)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wsp, wsn = (_ptr(workspace), workspace.numel() * workspace.element_size()) if workspace is not None else (None, 0)
    _check(lib.tbik_attention_tc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, S, NH, D, chunk, wsp, wsn,
                                 _stream_handle(stream)), "tbik_attention_tc")
    return out


def embedding(ids, table, *, out=None, stream=None):
    """Rows of ``table`` (bf16 [V, d]) at ``ids`` (int32 [tokens]) (see tbik_embedding)."""
    torch = _torch()
    lib = load_library()
    _need(ids, torch.int32, "ids")
    _need(table, torch.bfloat16, "table")
    V, d = table.shape
    if out is None:
        out = torch.empty((ids.numel(), d), dtype=torch.bfloat16, device=table.device)
    _need_out(out, torch.bfloat16, (ids.numel(), d))
    _check(lib.tbik_embedding(_ptr(ids), _ptr(table), _ptr(out), ids.numel(), V, d, _stream_handle(stream)),
           "tbik_embedding")
    return out


def transpose(x, *, out=None, stream=None):
    """bf16 [rows, cols] -> [cols, rows] (see tbik_transpose)."""
    torch = _torch()
    lib = load_library()
    _need(x, torch.bfloat16, "x")
    rows, cols = x.shape
    if out is None:
        out = torch.empty((cols, rows), dtype=torch.bfloat16, device=x.device)
    _need_out(out, torch.bfloat16, (cols, rows))
    _check(lib.tbik_transpose(_ptr(x), _ptr(out), rows, cols, _stream_handle(stream)), "tbik_transpose")
    return out


def logprob_workspace(M, V, H, T, leaf, mode) -> int:
    return int(load_library().tbik_logprob_workspace(M, V, H, T, leaf, mode))


def _logprob_shapes(hidden, W, targets):
    if hidden.dim() != 2 or W.dim() != 2 or W.shape[1] != hidden.shape[1]:
        raise ValueError("hidden must be [M, H] and W_lm [V, H]")
    if targets.numel() != hidden.shape[0]:
        raise ValueError("targets must hold one index per row of hidden")


def logprob(hidden, W, targets, *, T: int = 1, leaf: int = 256, tc: bool = True, noninv: bool = False, out=None,
            workspace=None, stream=None):
    torch = _torch()
    lib = load_library()
    _need(hidden, torch.bfloat16, "hidden")
    _need(W, torch.bfloat16, "W_lm")
    _need(targets, torch.int32, "targets")
    M, H = hidden.shape
    V = W.shape[0]
    _logprob_shapes(hidden, W, targets)
    mode = (TC if tc else EXACT) | (NONINV if noninv else 0)
    if out is None:
        out = torch.empty(M, dtype=torch.float32, device=hidden.device)
    _need_out(out, torch.float32, (M,))
    ws, wsb = _workspace(lib.tbik_logprob_workspace(M, V, H, T, leaf, mode), hidden.device, workspace)
    _check(lib.tbik_logprob(_ptr(hidden), _ptr(W), _ptr(targets), _ptr(out), M, V, H, T, leaf, mode, _ptr(ws), wsb,
                            _stream_handle(stream)), "tbik_logprob")
    return out


# ------------------------------------------- shard level across GPUs (TP)

def vocab_shard(V: int, T: int, t: int):
    """Shard t of T of the padded vocabulary (tbik.h, vocabulary-parallel
    logprob): (v0, Vs, Lvs) = first vocabulary index, real columns, leaves."""
    step = VOCAB_LEAF * T_MAX
    vpad = ((V + step - 1) // step) * step
    if T not in (1, 2, 4, 8) or not 0 <= t < T:
        raise ValueError("T must be 1, 2, 4 or 8 and 0 <= t < T")
    width = vpad // T
    v0 = t * width
    vs = max(0, min(V - v0, width))
    return v0, vs, width // VOCAB_LEAF


def tree_combine(partials, *, noninv: bool = False, out_bf16: bool = False, residual=None, out=None, stream=None):
    """tbik_tree_combine: the shard level of the tree over fp32 partials [T, ...]
    gathered in rank order (left to right with noninv).  Returns fp32 or bf16
    of shape partials.shape[1:]; residual (bf16, that shape) is added to the
    fp32 root before the bf16 rounding."""
    torch = _torch()
    lib = load_library()
    _need(partials, torch.float32, "partials")
    T = partials.shape[0]
    shape = tuple(partials.shape[1:])
    mn = partials[0].numel()
    if residual is not None:
        out_bf16 = True
        _need_out(residual, torch.bfloat16, shape, "residual")
    dtype = torch.bfloat16 if out_bf16 else torch.float32
    if out is None:
        out = torch.empty(shape, dtype=dtype, device=partials.device)
    _need_out(out, dtype, shape)
    mode = (NONINV if noninv else 0) | (OUT_BF16 if out_bf16 else 0)
    _check(lib.tbik_tree_combine(_ptr(partials), _ptr(out), mn, T, mode, _ptr(residual), _stream_handle(stream)),
           "tbik_tree_combine")
    return out


def logprob_partial(hidden, W_shard, targets, *, v0: int, Lvs: int, leaf: int = 256, tc: bool = True, out=None,
                    workspace=None, stream=None):
    """tbik_logprob_partial: one vocabulary shard's per-row (m, s, z, own),
    fp32 [M, 4].  W_shard holds vocabulary rows [v0, v0 + Vs) (Vs may be 0)."""
    torch = _torch()
    lib = load_library()
    _need(hidden, torch.bfloat16, "hidden")
    _need(W_shard, torch.bfloat16, "W_shard")
    _need(targets, torch.int32, "targets")
    M, H = hidden.shape
    Vs = W_shard.shape[0]
    if W_shard.dim() != 2 or (Vs > 0 and W_shard.shape[1] != H):
        raise ValueError("W_shard must be [Vs, H]")
    if targets.numel() != M:
        raise ValueError("targets must hold one index per row of hidden")
    mode = TC if tc else EXACT
    if out is None:
        out = torch.empty((M, 4), dtype=torch.float32, device=hidden.device)
    _need_out(out, torch.float32, (M, 4))
    ws, wsb = _workspace(lib.tbik_logprob_partial_workspace(M, Vs, Lvs, H, leaf, mode), hidden.device, workspace)
    wptr = _ptr(W_shard) if Vs > 0 else None
    _check(lib.tbik_logprob_partial(_ptr(hidden), wptr, _ptr(targets), _ptr(out), M, Vs, v0, Lvs, H, leaf, mode,
                                    _ptr(ws), wsb, _stream_handle(stream)), "tbik_logprob_partial")
    return out


def logprob_combine(parts, targets, V: int, *, out=None, stream=None):
    """tbik_logprob_combine: parts fp32 [T, M, 4] (shard summaries in rank
    order) -> logprob fp32 [M]."""
    torch = _torch()
    lib = load_library()
    _need(parts, torch.float32, "parts")
    _need(targets, torch.int32, "targets")
    if parts.dim() != 3 or parts.shape[2] != 4:
        raise ValueError("parts must be [T, M, 4]")
    T, M = parts.shape[0], parts.shape[1]
    if targets.numel() != M:
        raise ValueError("targets must hold one index per row")
    if out is None:
        out = torch.empty(M, dtype=torch.float32, device=parts.device)
    _need_out(out, torch.float32, (M,))
    _check(lib.tbik_logprob_combine(_ptr(parts), _ptr(targets), _ptr(out), M, V, T, _stream_handle(stream)),
           "tbik_logprob_combine")
    return out


def get_error(stream=None) -> int:
    return int(load_library().tbik_get_error(_stream_handle(stream)))


def debug_set(flags: int = 0, wait_limit_ns: int = 0):
    _check(load_library().tbik_debug_set(flags, wait_limit_ns), "tbik_debug_set")


_noalloc_ready = False


def logprob_noalloc(hidden, W, targets, *, T: int = 1, leaf: int = 256, noninv: bool = False, out=None,
                    stream=None):
    """tbik_logprob_noalloc: tensor-core logprob whose scratch is the library's
    fixed device array, for callers that cannot allocate a workspace.  Only the
    output (when not given) is allocated here, by torch."""
    global _noalloc_ready
    torch = _torch()
    lib = load_library()
    if not _noalloc_ready:
        vp, i32, u32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
        lib.tbik_logprob_noalloc.restype = i32
        lib.tbik_logprob_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, u32, vp]
        _noalloc_ready = True
    _need(hidden, torch.bfloat16, "hidden")
    _need(W, torch.bfloat16, "W_lm")
    _need(targets, torch.int32, "targets")
    M, H = hidden.shape
    V = W.shape[0]
    _logprob_shapes(hidden, W, targets)
    mode = TC | (NONINV if noninv else 0)
    if out is None:
        out = torch.empty(M, dtype=torch.float32, device=hidden.device)
    _need_out(out, torch.float32, (M,))
    _check(lib.tbik_logprob_noalloc(_ptr(hidden), _ptr(W), _ptr(targets), _ptr(out), M, V, H, T, leaf, mode,
                                    _stream_handle(stream)), "tbik_logprob_noalloc")
    return out

