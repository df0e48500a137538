"""Oracle of the end-to-end decoder: the library's operations composed in a
Llama-style pre-norm decoder, each step one oracle routine (TEST
INFRASTRUCTURE ONLY; only the tests, smoke() and the benchmark's CPU leg may
use it).

Per layer: y = RMSNorm(h) -> q, k, v = y Wq, y Wk, y Wv (column-parallel:
the whole K tree, the same for every T) -> RoPE(q, k) -> causal attention
with key chunks of 64 combined by the tree -> o Wo (row-parallel: T shards of
K, combined by the tree, or the non-invariant chain-and-sum baseline) ->
residual -> RMSNorm -> gate/up (column-parallel, kept fp32) -> SwiGLU on the
fp32 values -> down (row-parallel) -> residual.  Then the final RMSNorm and
the lm_head logprob of each target (T splits the vocabulary).  Other GEMM
results are rounded to bf16 once; RMSNorm gammas are 1, eps 1e-6, RoPE base
1e6, positions 0..seq-1.
"""
import numpy as np

from . import (attention, bf16_rne_array, gemm_noninv, gemm_tree, logprob, rmsnorm_residual, rope, rope_table,
               swiglu)


def _dense(a, w, *, leaf, T=1, noninv=False):
    if noninv:
        c = gemm_noninv(a, w, b_nk=False, T=T)
    else:
        c = gemm_tree(a, w, b_nk=False, T=T, leaf=leaf)
    return bf16_rne_array(c)


def forward(cfg, w, ids, targets, *, T: int = 1, noninv: bool = False):
    """Per-token logprobs fp32 [batch, seq] of `targets` after `ids`."""
    B, S = ids.shape
    d, NH, HD = cfg["d"], cfg["heads"], cfg["head_dim"]
    n = B * S
    leaf, leaf_ffn = cfg["leaf"], cfg["leaf_ffn"]
    x = w["emb"][ids.reshape(-1)]
    res = np.zeros((n, d), dtype=np.uint16)
    gamma = w["gamma"]
    table = rope_table(S, HD, 1e6)
    pos = np.tile(np.arange(S, dtype=np.int32), B)
    y, res = rmsnorm_residual(x, res, gamma, eps=1e-6)
    for L in w["layers"]:
        q = _dense(y, L["wq"], leaf=leaf)
        k = _dense(y, L["wk"], leaf=leaf)
        v = _dense(y, L["wv"], leaf=leaf)
        q = rope(q.reshape(n, NH, HD), pos, table)
        k = rope(k.reshape(n, NH, HD), pos, table)
        o = attention(q.reshape(B, S, NH, HD), k.reshape(B, S, NH, HD), v.reshape(B, S, NH, HD), chunk=64)
        a = _dense(o.reshape(n, d), L["wo"], leaf=leaf, T=T, noninv=noninv)
        y, res = rmsnorm_residual(a, res, gamma, eps=1e-6)
        # gate and up stay fp32 until the SwiGLU: one rounding, at its output
        g = gemm_tree(y, L["wg"], b_nk=False, T=1, leaf=leaf)
        u = gemm_tree(y, L["wu"], b_nk=False, T=1, leaf=leaf)
        act = swiglu(g, u)
        m = _dense(act, L["wd"], leaf=leaf_ffn, T=T, noninv=noninv)
        y, res = rmsnorm_residual(m, res, gamma, eps=1e-6)
    lp = logprob(y, w["lm_head"], targets.reshape(-1).astype(np.int32), T=T, leaf=leaf, noninv=noninv)
    return lp.reshape(B, S)
