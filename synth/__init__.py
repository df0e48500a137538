"""Seeded synthetic inputs (SplitMix64 -> Box-Muller -> bf16 RNE).

The generator lives in ``synth.c`` and is compiled on first use into
``libsynth.so`` beside it.  It draws random numbers only; the method's
arithmetic lives in the CUDA library and, separately, in the oracle.

Arrays come back as numpy arrays; bf16 tensors are returned as ``uint16``
bit patterns (use :func:`as_torch_bf16` to view them as ``torch.bfloat16``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_SO = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``libsynth.so`` (OpenMP, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
            lib.synth_splitmix64.restype = u64
            lib.synth_splitmix64.argtypes = [u64, u64]
            lib.synth_normal_f64.argtypes = [u64, u64, i64, vp]
            lib.synth_normal_bf16.argtypes = [u64, u64, i64, dbl, dbl, vp]
            lib.synth_normal_f32.argtypes = [u64, u64, i64, dbl, dbl, vp]
            lib.synth_int_bf16.argtypes = [u64, u64, i64, ctypes.c_int, vp]
            lib.synth_uniform_int32.argtypes = [u64, u64, i64, i64, i64, vp]
            lib.synth_permutation.argtypes = [u64, i64, vp]
            for f in (lib.synth_normal_f64, lib.synth_normal_bf16, lib.synth_normal_f32,
                      lib.synth_int_bf16, lib.synth_uniform_int32, lib.synth_permutation):
                f.restype = None
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def splitmix64(seed: int, i: int) -> int:
    return int(_load().synth_splitmix64(seed, i))


def normal_f64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().synth_normal_f64(seed, offset, n, _ptr(out))
    return out


def normal_bf16(seed: int, shape, std: float = 1.0, mean: float = 0.0, offset: int = 0) -> np.ndarray:
    """bf16 bit patterns of mean + std * N(0,1), row-major ``shape``."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    _load().synth_normal_bf16(seed, offset, n, float(mean), float(std), _ptr(out))
    return out.reshape(shape)


def normal_f32(seed: int, shape, std: float = 1.0, mean: float = 0.0, offset: int = 0) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    _load().synth_normal_f32(seed, offset, n, float(mean), float(std), _ptr(out))
    return out.reshape(shape)


def int_bf16(seed: int, shape, amp: int, offset: int = 0) -> np.ndarray:
    """bf16 bit patterns of integers uniform in [-amp, amp]."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    _load().synth_int_bf16(seed, offset, n, int(amp), _ptr(out))
    return out.reshape(shape)


def uniform_int32(seed: int, n: int, lo: int, hi: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _load().synth_uniform_int32(seed, offset, n, int(lo), int(hi), _ptr(out))
    return out


def permutation(seed: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _load().synth_permutation(seed, n, _ptr(out))
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (a pure bit shift)."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def as_torch_bf16(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


# ---------------------------------------------------------------------------
# Workload recipes: seeds, shapes and distributions of the synthetic inputs.
# ---------------------------------------------------------------------------

def tiny_gemm_inputs():
    """A bf16 [4,256] then B bf16 [256,64] from one seed-0 stream, N(0,1)/sqrt(256)."""
    a = normal_bf16(0, (4, 256), std=1.0 / 16.0, offset=0)
    b = normal_bf16(0, (256, 64), std=1.0 / 16.0, offset=4 * 256)
    return a, b


def down_proj_weight(K: int = 14336, N: int = 4096, layout: str = "kn"):
    """down_proj weight, N(0, 0.02^2); ``kn`` = [K,N] row-major, ``nk`` = [N,K]."""
    if layout == "kn":
        return normal_bf16(13, (K, N), std=0.02)
    return normal_bf16(13, (N, K), std=0.02)


def gate_up_preacts(M: int, F: int = 14336, H: int = 4096):
    """Stand-ins for x.Wg and x.Wu with x ~ N(0,1) [M,H], W ~ N(0,0.02^2).

    Each entry of x.W is a sum of H products and is N(0, H * 0.02^2) to a very
    good approximation, so g and u are drawn directly from that normal
    (std 0.02*sqrt(H) = 1.28 at H = 4096) as float32.
    """
    std = 0.02 * float(np.sqrt(H))
    g = normal_f32(11, (M, F), std=std)
    u = normal_f32(12, (M, F), std=std)
    return g, u


def reduction_inputs(tokens: int, H: int = 4096, heads: int = 32, head_dim: int = 128,
                     F: int = 14336, max_pos: int = 32768):
    x = normal_bf16(20, (tokens, H))
    res = normal_bf16(21, (tokens, H))
    gamma = normal_bf16(22, (H,), std=0.1, mean=1.0)
    pos = uniform_int32(23, tokens, 0, max_pos)
    g = normal_bf16(24, (tokens, F))
    u = normal_bf16(25, (tokens, F))
    q = normal_bf16(26, (tokens, heads, head_dim))
    k = normal_bf16(27, (tokens, heads, head_dim))
    return dict(x=x, res=res, gamma=gamma, pos=pos, q=q, k=k, g=g, u=u)


def logprob_inputs(M: int, V: int = 151936, H: int = 4096, with_weight: bool = True):
    hidden = normal_bf16(30, (M, H))
    w = normal_bf16(31, (V, H), std=0.02) if with_weight else None
    targets = uniform_int32(32, M, 0, V)
    return hidden, w, targets


# ---------------------------------------------------------------------------
# End-to-end decoder (Llama-style, pre-norm): shapes, seeds and distributions.
# ---------------------------------------------------------------------------

DECODER_FULL = dict(d=2048, heads=16, head_dim=128, ffn=5632, vocab=32000, layers=4, batch=8, seq=2048,
                    leaf=256, leaf_ffn=176)
DECODER_SMALL = dict(d=256, heads=2, head_dim=128, ffn=512, vocab=1024, layers=2, batch=2, seq=80,
                     leaf=32, leaf_ffn=64)


def decoder_weights(cfg):
    """Random-init weights, every matrix N(0, 0.02^2) bf16, stored [in, out]
    row-major (the lm_head [vocab, d]); RMSNorm gammas 1.  Seeds 40 (embedding),
    41 (lm_head), 50 + 10*l + {0..6} (layer l: q, k, v, o, gate, up, down)."""
    d, f, V = cfg["d"], cfg["ffn"], cfg["vocab"]
    w = dict(emb=normal_bf16(40, (V, d), std=0.02), lm_head=normal_bf16(41, (V, d), std=0.02), layers=[])
    for layer in range(cfg["layers"]):
        s = 50 + 10 * layer
        w["layers"].append(dict(
            wq=normal_bf16(s, (d, d), std=0.02), wk=normal_bf16(s + 1, (d, d), std=0.02),
            wv=normal_bf16(s + 2, (d, d), std=0.02), wo=normal_bf16(s + 3, (d, d), std=0.02),
            wg=normal_bf16(s + 4, (d, f), std=0.02), wu=normal_bf16(s + 5, (d, f), std=0.02),
            wd=normal_bf16(s + 6, (f, d), std=0.02)))
    w["gamma"] = np.full(d, 0x3F80, dtype=np.uint16)  # bf16 1.0
    return w


def decoder_tokens(cfg, seed: int = 90):
    """Token ids and next-token targets, uniform in [0, vocab), [batch, seq]."""
    B, S, V = cfg["batch"], cfg["seq"], cfg["vocab"]
    ids = uniform_int32(seed, B * S, 0, V).reshape(B, S)
    targets = uniform_int32(seed + 1, B * S, 0, V).reshape(B, S)
    return ids, targets
