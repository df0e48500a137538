"""CPU oracle of the tree-ordered invariant kernels (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It wraps ``oracle.c`` (plain single-threaded C,
compiled on first use into ``liboracle.so`` beside it; ``build_all_cores``
makes an OpenMP build of the same file for timing on all host cores) with
numpy marshalling;
all arithmetic happens in the C file.  Nothing here is shared with the CUDA
library.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_FMA = None


def _so_path() -> str:
    # The -mfma variant only runs on CPUs with FMA; both give the same bits.
    return os.path.join(_HERE, "liboracle_fma.so" if _cpu_has_fma() else "liboracle.so")
_lock = threading.Lock()
_lib = None

VLEAF = 64  # vocabulary columns per logprob leaf


def _cpu_has_fma() -> bool:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("flags"):
                    return " fma " in f" {line.split(':', 1)[1]} "
    except OSError:
        pass
    return False


def build(force: bool = False) -> str:
    """Compile the oracle: -O2, no contraction, no fast-math, single thread.

    ``-mfma`` only lets gcc inline the correctly rounded ``fmaf`` the source
    calls (the value is the same either way); contraction stays off.
    """
    so = _so_path()
    if force or not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(_SRC):
        flags = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]
        if _cpu_has_fma():
            flags.append("-mfma")
        tmp = so + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *flags, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, so)
    return so


def build_all_cores(force: bool = False) -> str:
    """Compile the same oracle.c with -fopenmp into ``liboracle_omp.so``: the
    pragmas on the independent GEMM outputs and logprob rows spread them over
    the host's cores (each output is the same serial computation, so the bits
    equal the default build's).  Used only to time the oracle on all cores."""
    so = os.path.join(_HERE, "liboracle_omp.so")
    if force or not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(_SRC):
        flags = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-fopenmp"]
        if _cpu_has_fma():
            flags.append("-mfma")
        tmp = so + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *flags, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, so)
    return so


def _open(path: str) -> ctypes.CDLL:
    """Load an oracle build at ``path`` and declare its function signatures."""
    lib = ctypes.CDLL(path)
    vp, i32, i64, f32, f64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double)
    sig = {
        "oracle_bf16_rne": (ctypes.c_uint16, [f32]),
        "oracle_bf16_rne_array": (None, [vp, vp, i64]),
        "oracle_tree_sum": (f32, [vp, i32]),
        "oracle_exp": (f32, [f32]),
        "oracle_log": (f32, [f32]),
        "oracle_tree_ms": (None, [vp, vp, i32, vp, vp]),
        "oracle_gemm_tree": (i32, [vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]),
        "oracle_gemm_noninv": (i32, [vp, vp, i32, i32, i32, i32, i32, vp, vp]),
        "oracle_gemm_f64": (None, [vp, vp, i32, i32, i32, i32, vp]),
        "oracle_rmsnorm_residual": (i32, [vp, vp, vp, vp, vp, i32, i32, f32, i32]),
        "oracle_add_residual_bf16": (None, [vp, vp, vp, i64]),
        "oracle_rope_table": (None, [vp, i32, i32, f64]),
        "oracle_rope": (None, [vp, vp, vp, vp, i32, i32, i32]),
        "oracle_swiglu_bf16": (None, [vp, vp, vp, i64]),
        "oracle_swiglu_f32": (None, [vp, vp, vp, i64]),
        "oracle_logprob": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp]),
        "oracle_logprob_f64": (None, [vp, vp, vp, vp, i32, i32, i32]),
        "oracle_attention": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32]),
        "oracle_attention_f64": (None, [vp, vp, vp, vp, i32, i32, i32, i32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _open(build())
    return _lib


@contextlib.contextmanager
def library(path: str):
    """Run the wrappers against another build of oracle.c (a shared object at
    ``path``) for the duration of the block.  Test use only: the oracle's
    mutation tests compile copies of oracle.c with one mistake planted and
    check that the pins catch it."""
    global _lib
    other = _open(path)
    with _lock:
        saved = _lib
        _lib = other
    try:
        yield other
    finally:
        with _lock:
            _lib = saved


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile C source text (a variant of oracle.c) with the oracle's flags."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    flags = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]
    if _cpu_has_fma():
        flags.append("-mfma")
    subprocess.check_call(["gcc", *flags, "-o", out_path, src, "-lm"])
    return out_path


def source() -> str:
    """The text of oracle.c."""
    with open(_SRC) as f:
        return f.read()


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle rejected the shape for {what}")


# ------------------------------------------------------------------ scalars

def bf16_rne(x: float) -> int:
    return int(_load().oracle_bf16_rne(float(x)))


def bf16_rne_array(x) -> np.ndarray:
    """bf16 bits of float32 values, round to nearest even (element-wise)."""
    a, pa = _c(x, np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().oracle_bf16_rne_array(pa, out.ctypes.data, a.size)
    return out


def exp(x: float) -> float:
    return float(_load().oracle_exp(float(x)))


def log(x: float) -> float:
    return float(_load().oracle_log(float(x)))


def exp_array(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32).ravel()
    f = _load().oracle_exp
    return np.array([f(float(v)) for v in x], dtype=np.float32)


def log_array(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32).ravel()
    f = _load().oracle_log
    return np.array([f(float(v)) for v in x], dtype=np.float32)


def tree_sum(p) -> np.float32:
    p, ptr = _c(p, np.float32)
    return np.float32(_load().oracle_tree_sum(ptr, p.size))


def tree_ms(m, s):
    m, pm = _c(m, np.float32)
    s, ps = _c(s, np.float32)
    om, os_ = ctypes.c_float(), ctypes.c_float()
    _load().oracle_tree_ms(pm, ps, m.size, ctypes.byref(om), ctypes.byref(os_))
    return np.float32(om.value), np.float32(os_.value)


# ------------------------------------------------------------------ GEMM

def gemm_tree(a_bits, b_bits, *, b_nk: bool, T: int, leaf: int, shards: bool = False):
    """C fp32 [M,N] of the tree-ordered GEMM (and shard partials [T,M,N] if asked)."""
    a, pa = _c(a_bits, np.uint16)
    b, pb = _c(b_bits, np.uint16)
    M, K = a.shape
    N = b.shape[0] if b_nk else b.shape[1]
    c = np.empty((M, N), dtype=np.float32)
    q = np.empty((T, M, N), dtype=np.float32) if shards else None
    _check(_load().oracle_gemm_tree(pa, pb, int(b_nk), M, N, K, T, leaf, c.ctypes.data,
                                    q.ctypes.data if shards else None), "gemm_tree")
    return (c, q) if shards else c


def gemm_noninv(a_bits, b_bits, *, b_nk: bool, T: int, shards: bool = False):
    a, pa = _c(a_bits, np.uint16)
    b, pb = _c(b_bits, np.uint16)
    M, K = a.shape
    N = b.shape[0] if b_nk else b.shape[1]
    c = np.empty((M, N), dtype=np.float32)
    q = np.empty((T, M, N), dtype=np.float32) if shards else None
    _check(_load().oracle_gemm_noninv(pa, pb, int(b_nk), M, N, K, T, c.ctypes.data,
                                      q.ctypes.data if shards else None), "gemm_noninv")
    return (c, q) if shards else c


def add_residual_bf16(root, r_bits) -> np.ndarray:
    """bf16 bits of root + f32(R): one fp32 add, one RNE rounding."""
    c, pc = _c(root, np.float32)
    r, pr = _c(r_bits, np.uint16)
    if c.shape != r.shape:
        raise ValueError("root and residual shapes differ")
    out = np.empty(c.shape, dtype=np.uint16)
    _load().oracle_add_residual_bf16(pc, pr, out.ctypes.data, c.size)
    return out


def gemm_residual(a_bits, b_bits, r_bits, *, b_nk: bool, T: int, leaf: int, noninv: bool = False):
    """bf16 bits of the tree GEMM's fp32 root (or the baseline's) plus the residual R."""
    if noninv:
        root = gemm_noninv(a_bits, b_bits, b_nk=b_nk, T=T)
    else:
        root = gemm_tree(a_bits, b_bits, b_nk=b_nk, T=T, leaf=leaf)
    return add_residual_bf16(root, r_bits)


def gemm_f64(a_bits, b_bits, *, b_nk: bool):
    a, pa = _c(a_bits, np.uint16)
    b, pb = _c(b_bits, np.uint16)
    M, K = a.shape
    N = b.shape[0] if b_nk else b.shape[1]
    c = np.empty((M, N), dtype=np.float64)
    _load().oracle_gemm_f64(pa, pb, int(b_nk), M, N, K, c.ctypes.data)
    return c


# ------------------------------------------------------------ reductions

def rmsnorm_residual(x_bits, res_bits, gamma_bits, *, eps: float = 1e-6, T: int = 1):
    """y and res_out bf16 bits; res_bits None: no residual input (r = f32(x))."""
    x, px = _c(x_bits, np.uint16)
    pr = None
    if res_bits is not None:
        r, pr = _c(res_bits, np.uint16)
    g, pg = _c(gamma_bits, np.uint16)
    tokens, H = x.shape
    y = np.empty_like(x)
    ro = np.empty_like(x)
    _check(_load().oracle_rmsnorm_residual(px, pr, pg, y.ctypes.data, ro.ctypes.data, tokens, H,
                                           float(eps), T), "rmsnorm_residual")
    return y, ro


def rope_table(max_pos: int, head_dim: int = 128, base: float = 1e6) -> np.ndarray:
    t = np.empty((max_pos, head_dim // 2, 2), dtype=np.float32)
    _load().oracle_rope_table(t.ctypes.data, max_pos, head_dim, float(base))
    return t


def rope(x_bits, pos, table):
    x, px = _c(x_bits, np.uint16)
    p, pp = _c(pos, np.int32)
    t, pt = _c(table, np.float32)
    tokens, heads, hd = x.shape
    out = np.empty_like(x)
    _load().oracle_rope(px, pp, pt, out.ctypes.data, tokens, heads, hd)
    return out


def swiglu(g, u):
    """bf16 bits of SwiGLU; g/u are bf16 bit patterns (uint16) or float32."""
    if np.asarray(g).dtype == np.uint16:
        g, pg = _c(g, np.uint16)
        u, pu = _c(u, np.uint16)
        out = np.empty(g.shape, dtype=np.uint16)
        _load().oracle_swiglu_bf16(pg, pu, out.ctypes.data, g.size)
    else:
        g, pg = _c(g, np.float32)
        u, pu = _c(u, np.float32)
        out = np.empty(g.shape, dtype=np.uint16)
        _load().oracle_swiglu_f32(pg, pu, out.ctypes.data, g.size)
    return out


# --------------------------------------------------------------- logprob

def vpad_for(V: int, vleaf: int = VLEAF, tmax: int = 8) -> int:
    step = vleaf * tmax
    return ((V + step - 1) // step) * step


def logprob(hidden_bits, w_bits, targets, *, T: int = 1, leaf: int = 256, vleaf: int = VLEAF,
            vpad: int | None = None, noninv: bool = False, stats: bool = False):
    h, ph = _c(hidden_bits, np.uint16)
    w, pw = _c(w_bits, np.uint16)
    t, pt = _c(targets, np.int32)
    M, H = h.shape
    V = w.shape[0]
    vpad = vpad_for(V, vleaf) if vpad is None else vpad
    out = np.empty(M, dtype=np.float32)
    rm = np.empty(M, dtype=np.float32)
    rs = np.empty(M, dtype=np.float32)
    _check(_load().oracle_logprob(ph, pw, pt, out.ctypes.data, M, V, H, T, leaf, vleaf, vpad,
                                  int(noninv), rm.ctypes.data, rs.ctypes.data), "logprob")
    return (out, rm, rs) if stats else out


def logprob_f64(hidden_bits, w_bits, targets):
    h, ph = _c(hidden_bits, np.uint16)
    w, pw = _c(w_bits, np.uint16)
    t, pt = _c(targets, np.int32)
    M, H = h.shape
    V = w.shape[0]
    out = np.empty(M, dtype=np.float64)
    _load().oracle_logprob_f64(ph, pw, pt, out.ctypes.data, M, V, H)
    return out


def attention(q_bits, k_bits, v_bits, *, chunk: int = 64):
    """Causal attention, keys in chunks combined by the tree; bf16 [batch, seq, heads, head_dim] in and out."""
    q, pq = _c(q_bits, np.uint16)
    k, pk = _c(k_bits, np.uint16)
    v, pv = _c(v_bits, np.uint16)
    B, S, NH, D = q.shape
    out = np.empty_like(q)
    _check(_load().oracle_attention(pq, pk, pv, out.ctypes.data, B, S, NH, D, chunk), "attention")
    return out


def attention_f64(q_bits, k_bits, v_bits):
    q, pq = _c(q_bits, np.uint16)
    k, pk = _c(k_bits, np.uint16)
    v, pv = _c(v_bits, np.uint16)
    B, S, NH, D = q.shape
    out = np.empty(q.shape, dtype=np.float64)
    _load().oracle_attention_f64(pq, pk, pv, out.ctypes.data, B, S, NH, D)
    return out

