"""Tree-ordered invariant kernels (TBIK-style) for NVIDIA B200, sm_100a.

A bf16 GEMM and the reductions around it (residual RMSNorm, RoPE and SwiGLU
with fp32 intermediates, lm_head -> log-softmax -> target logprob) whose fp32
reductions follow one fixed binary tree over fixed-size leaves, so results are
bitwise identical for any tensor-parallel shard count T and any batch size.

The computation lives in the C-ABI library ``libtbik.so`` (``include/tbik.h``);
this package is its Python binding.
"""
from ._binding import (  # noqa: F401
    B_KN, B_NK, SWIGLU_OUT, DEBUG_WITHHOLD_ACC_ARRIVE, DEBUG_TILE128, EXACT, NONINV, OUT_BF16, OUT_F32, T_MAX, TC,
    TBIK_ERR_ALIGN, TBIK_ERR_ARG, TBIK_ERR_CUDA, TBIK_ERR_POSITION, TBIK_ERR_SHAPE, TBIK_ERR_TARGET,
    TBIK_ERR_TIMEOUT, TBIK_ERR_UNSUPPORTED, TBIK_ERR_WORKSPACE, TBIK_OK, VOCAB_LEAF, TbikError, debug_set,
    attention, attention_tc_workspace, declared_functions, embedding, gemm, gemm_workspace, get_error, load_library, logprob, logprob_workspace,
    rmsnorm_residual, rope_swiglu, rope_table, status_string, transpose, tree_combine, logprob_partial,
    logprob_combine, vocab_shard,
)

__all__ = [
    "gemm", "gemm_workspace", "rmsnorm_residual", "rope_table", "rope_swiglu", "logprob", "logprob_workspace",
    "attention", "attention_tc_workspace", "embedding", "transpose", "get_error", "debug_set", "load_library", "declared_functions", "TbikError",
    "tree_combine", "logprob_partial", "logprob_combine", "vocab_shard",
]
