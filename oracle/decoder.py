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

from . import (attention, bf16_rne_array, gemm_noninv, gemm_residual, gemm_tree, logprob, rmsnorm_residual, rope,
               rope_table, swiglu)


def _dense(a, w, *, leaf, T=1, noninv=False):
    if noninv:
        c = gemm_noninv(a, w, b_nk=False, T=T)
    else:
        c = gemm_tree(a, w, b_nk=False, T=T, leaf=leaf)
    return bf16_rne_array(c)


def forward(cfg, w, ids, targets, *, T: int = 1, noninv: bool = False, fuse_residual: bool = False):
    """Per-token logprobs fp32 [batch, seq] of `targets` after `ids`.

    fuse_residual: the o and down projections return bf16(root + h) for the
    residual stream h (one fp32 add, one rounding) and the RMSNorms take h with
    no residual input; otherwise the projection is rounded to bf16 and the
    RMSNorm adds it to the residual in fp32."""
    B, S = ids.shape
    d, NH, HD = cfg["d"], cfg["heads"], cfg["head_dim"]
    n = B * S
    leaf, leaf_ffn = cfg["leaf"], cfg["leaf_ffn"]
    x = w["emb"][ids.reshape(-1)]
    gamma = w["gamma"]
    table = rope_table(S, HD, 1e6)
    pos = np.tile(np.arange(S, dtype=np.int32), B)

    def add_norm(a, wt, lf, res):
        if fuse_residual:
            h = gemm_residual(a, wt, res, b_nk=False, T=T, leaf=lf, noninv=noninv)
            return rmsnorm_residual(h, None, gamma, eps=1e-6)[0], h
        return rmsnorm_residual(_dense(a, wt, leaf=lf, T=T, noninv=noninv), res, gamma, eps=1e-6)

    if fuse_residual:
        res = x
        y = rmsnorm_residual(x, None, gamma, eps=1e-6)[0]
    else:
        y, res = rmsnorm_residual(x, np.zeros((n, d), dtype=np.uint16), gamma, eps=1e-6)
    for L in w["layers"]:
        q = _dense(y, L["wq"], leaf=leaf)
        k = _dense(y, L["wk"], leaf=leaf)
        v = _dense(y, L["wv"], leaf=leaf)
        q = rope(q.reshape(n, NH, HD), pos, table)
        k = rope(k.reshape(n, NH, HD), pos, table)
        o = attention(q.reshape(B, S, NH, HD), k.reshape(B, S, NH, HD), v.reshape(B, S, NH, HD), chunk=64)
        y, res = add_norm(o.reshape(n, d), L["wo"], leaf, res)
        # gate and up stay fp32 until the SwiGLU: one rounding, at its output
        g = gemm_tree(y, L["wg"], b_nk=False, T=1, leaf=leaf)
        u = gemm_tree(y, L["wu"], b_nk=False, T=1, leaf=leaf)
        act = swiglu(g, u)
        y, res = add_norm(act, L["wd"], leaf_ffn, res)
    lp = logprob(y, w["lm_head"], targets.reshape(-1).astype(np.int32), T=T, leaf=leaf, noninv=noninv)
    return lp.reshape(B, S)
