"""A Llama-style pre-norm decoder forward pass built from the library's calls,
returning the per-token logprob of given targets.  Every step runs in the
library's kernels; this module only allocates the activations (torch) and
sequences the calls.

Per layer: y = RMSNorm(h); q, k, v = y Wq, y Wk, y Wv (column-parallel: each
device holds whole output columns, so the K reduction is the full tree and the
same for every T); RoPE on q, k; causal attention with the keys in chunks of
64 combined by the tree (heads split across devices: per-head, so the same
for every T); o Wo (row-parallel: K = d split into T shards, combined by the
tree, or by the non-invariant chain-and-sum baseline); residual + RMSNorm;
gate and up as one column-parallel GEMM whose epilogue applies SwiGLU to the
fp32 roots (one bf16 rounding, after the SwiGLU); down (row-parallel);
residual.  Then the final RMSNorm and the lm_head logprob (T splits the
vocabulary).  Other GEMM outputs are rounded to bf16 once; gammas come with
the weights; eps 1e-6; RoPE base 1e6; positions 0..seq-1 in every sequence.
"""
from dataclasses import dataclass

import numpy as np

from . import _binding as tb


@dataclass
class DecoderConfig:
    d: int
    heads: int
    head_dim: int
    ffn: int
    vocab: int
    layers: int
    leaf: int = 256       # K leaf of the d-wide GEMMs
    leaf_ffn: int = 176   # K leaf of the down projection (ffn wide)
    w_out_in: bool = False  # projection weights stored [out, in] (the GEMMs' [N,K] operand) instead of [in, out]


class Decoder:
    """Weights are device bf16 tensors: ``emb`` and ``lm_head`` [vocab, d],
    ``gamma`` [d], and per layer ``wq wk wv wo`` [d, d], ``wgu`` [d, 2 ffn]
    (gate and up interleaved, see `interleave_gate_up`), ``wd`` [ffn, d]
    ([in, out] row-major), or each of them transposed ([out, in]) when
    ``cfg.w_out_in``: the same products, run by the tensor-core GEMM's
    192-column tiles, with the same bits."""

    def __init__(self, cfg: DecoderConfig, emb, lm_head, gamma, layers):
        self.cfg, self.emb, self.lm_head, self.gamma, self.layers = cfg, emb, lm_head, gamma, layers
        self._tables = {}

    def _table(self, seq, device):
        key = (seq, str(device))
        if key not in self._tables:
            self._tables[key] = tb.rope_table(seq, self.cfg.head_dim, 1e6, device=device)
        return self._tables[key]

    def forward(self, ids, targets, pos, *, T: int = 1, tc: bool = True, noninv: bool = False,
                fuse_residual: bool = False, attention_tc: bool = False, stream=None):
        """ids, targets: device int32 [batch, seq]; pos: device int32 [batch*seq]
        (the position of each token).  Returns fp32 logprobs [batch, seq].

        fuse_residual: the o and down projections add their fp32 root to the
        bf16 residual stream h in their last step (tbik_gemm_residual, one
        rounding: h = bf16(root + h)) and each RMSNorm normalises h with no
        residual input; otherwise the projection output is rounded to bf16
        and the RMSNorm adds it to the residual in fp32.

        attention_tc: the attention on the tensor cores (tbik_attention_tc,
        head_dim 128, seq a multiple of 128); otherwise the exact-order kernel."""
        torch = tb._torch()
        c = self.cfg
        B, S = ids.shape
        n = B * S
        dev = ids.device
        bf = torch.bfloat16

        nk = c.w_out_in

        def dense(a, w, leaf, shards=1, baseline=False):
            out = torch.empty((a.shape[0], w.shape[0] if nk else w.shape[1]), dtype=bf, device=dev)
            tb.gemm(a, w, T=shards, leaf=leaf, tc=tc, noninv=baseline, out_bf16=True, b_nk=nk, out=out,
                    stream=stream)
            return out

        def add_norm(w, a, leaf, res):
            """(y, res) after the row-parallel projection a @ w and its residual add."""
            if fuse_residual:  # res is the stream h, updated in place
                tb.gemm(a, w, T=T, leaf=leaf, tc=tc, noninv=noninv, residual=res, out=res, b_nk=nk, stream=stream)
                y, _ = tb.rmsnorm_residual(res, None, self.gamma, eps=1e-6, T=1, want_res_out=False, stream=stream)
                return y, res
            return tb.rmsnorm_residual(dense(a, w, leaf, T, noninv), res, self.gamma, eps=1e-6, T=1, stream=stream)

        x = tb.embedding(ids.reshape(-1), self.emb, stream=stream)
        table = self._table(S, dev)
        if fuse_residual:
            res = x
            y, _ = tb.rmsnorm_residual(x, None, self.gamma, eps=1e-6, T=1, want_res_out=False, stream=stream)
        else:
            res = torch.zeros((n, c.d), dtype=bf, device=dev)
            y, res = tb.rmsnorm_residual(x, res, self.gamma, eps=1e-6, T=1, stream=stream)
        for L in self.layers:
            q = dense(y, L["wq"], c.leaf)
            k = dense(y, L["wk"], c.leaf)
            v = dense(y, L["wv"], c.leaf)
            q3, k3 = q.view(n, c.heads, c.head_dim), k.view(n, c.heads, c.head_dim)
            tb.rope_swiglu(q=q3, k=k3, pos=pos, table=table, q_out=q3, k_out=k3, stream=stream)
            o = tb.attention(q.view(B, S, c.heads, c.head_dim), k.view(B, S, c.heads, c.head_dim),
                             v.view(B, S, c.heads, c.head_dim), tc=attention_tc, stream=stream)
            y, res = add_norm(L["wo"], o.view(n, c.d), c.leaf, res)
            act = torch.empty((n, c.ffn), dtype=bf, device=dev)
            tb.gemm(y, L["wgu"], T=1, leaf=c.leaf, tc=tc, swiglu=True, b_nk=nk, out=act, stream=stream)
            y, res = add_norm(L["wd"], act, c.leaf_ffn, res)
        lp = tb.logprob(y, self.lm_head, targets.reshape(-1), T=T, leaf=c.leaf, tc=tc, noninv=noninv, stream=stream)
        return lp.view(B, S)


def positions(batch: int, seq: int) -> np.ndarray:
    """Position of each token of a [batch, seq] block (0..seq-1 per sequence)."""
    return np.tile(np.arange(seq, dtype=np.int32), batch)


def interleave_gate_up(wg: np.ndarray, wu: np.ndarray) -> np.ndarray:
    """[K, F] gate and up weights -> [K, 2F] with blocks of 32 columns
    alternating (gate features 32j..32j+31, then the same up features), the
    layout the SwiGLU-output GEMM expects.  Data layout only."""
    K, F = wg.shape
    if wu.shape != wg.shape or F % 32:
        raise ValueError("gate and up must share the shape [K, F] with F % 32 == 0")
    out = np.empty((K, F // 32, 2, 32), dtype=wg.dtype)
    out[:, :, 0] = wg.reshape(K, F // 32, 32)
    out[:, :, 1] = wu.reshape(K, F // 32, 32)
    return out.reshape(K, 2 * F)

