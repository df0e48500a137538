"""The gate/up projection fused with SwiGLU (TBIK_SWIGLU_OUT): the gate and up
roots stay fp32 and are rounded to bf16 only after the SwiGLU.  Exact mode is
bit-exact to the oracle (tree GEMMs in fp32, then the fp32-input SwiGLU); the
tensor-core epilogue gives the same bits as the tensor-core GEMM's fp32 output
followed by the standalone SwiGLU kernel, for every T and batch size."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, dev_f32, host_bits16, host_f32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402
from invariant_tree_ordered_b200.decoder import interleave_gate_up  # noqa: E402


def weights(seed, K, F):
    wg = synth.normal_bf16(seed, (K, F), std=0.05)
    wu = synth.normal_bf16(seed + 1, (K, F), std=0.05)
    return wg, wu


def split_roots(c, F):
    """gate and up columns of an interleaved [M, 2F] fp32 result."""
    c = c.reshape(c.shape[0], F // 32, 2, 32)
    return np.ascontiguousarray(c[:, :, 0].reshape(-1, F)), np.ascontiguousarray(c[:, :, 1].reshape(-1, F))


@pytest.mark.parametrize("M,K,F,leaf", [(1, 256, 64, 32), (37, 512, 96, 64), (300, 384, 160, 64)])
@pytest.mark.parametrize("b_nk", [False, True])
def test_fused_exact_bitwise_vs_oracle(M, K, F, leaf, b_nk):
    a = synth.normal_bf16(700 + M, (M, K))
    wg, wu = weights(710 + F, K, F)
    ref = oracle.swiglu(oracle.gemm_tree(a, wg, b_nk=False, T=1, leaf=leaf),
                        oracle.gemm_tree(a, wu, b_nk=False, T=1, leaf=leaf))
    b = interleave_gate_up(wg, wu)
    if b_nk:
        b = np.ascontiguousarray(b.T)
    for T in (1, 2):
        got = tbik.gemm(dev_bf16(a), dev_bf16(b), T=T, leaf=leaf, tc=False, b_nk=b_nk, swiglu=True)
        assert tuple(got.shape) == (M, F)
        assert np.array_equal(host_bits16(got), ref), T
    assert tbik.get_error() == tbik.TBIK_OK


@pytest.mark.parametrize("M", [16, 1024])  # 16: frontier-split (unfused) path; 1024: fused epilogue
@pytest.mark.parametrize("b_nk", [False, True])  # 128-column tiles; 192-column tiles (ragged last tile)
def test_fused_tc_equals_tc_roots_then_swiglu(M, b_nk):
    K, F = 2048, 2048
    a = dev_bf16(synth.normal_bf16(720, (M, K)))
    wg, wu = weights(730, K, F)
    bh = interleave_gate_up(wg, wu)
    b = dev_bf16(np.ascontiguousarray(bh.T) if b_nk else bh)
    fused = host_bits16(tbik.gemm(a, b, T=1, leaf=256, tc=True, swiglu=True, b_nk=b_nk))
    roots = host_f32(tbik.gemm(a, b, T=1, leaf=256, tc=True, b_nk=b_nk))
    g, u = split_roots(roots, F)
    _, _, sep = tbik.rope_swiglu(g=dev_f32(g), u=dev_f32(u))
    assert np.array_equal(fused, host_bits16(sep))
    for T in (2, 8):
        assert np.array_equal(host_bits16(tbik.gemm(a, b, T=T, leaf=256, tc=True, swiglu=True, b_nk=b_nk)),
                              fused), T
    if M > 1:
        part = host_bits16(tbik.gemm(a[3:M - 2].contiguous(), b, T=4, leaf=256, tc=True, swiglu=True, b_nk=b_nk))
        assert np.array_equal(part, fused[3:M - 2])
    assert tbik.get_error() == tbik.TBIK_OK


def test_fused_argument_errors():
    lib = tbik.load_library()
    a = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros((256, 96), dtype=torch.bfloat16, device="cuda")
    c = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    mode = tbik.TC | tbik.SWIGLU_OUT
    assert lib.tbik_gemm_workspace(4, 96, 256, 1, 32, mode) == (1 << 64) - 1  # N % 64 != 0
    assert lib.tbik_gemm(a.data_ptr(), b.data_ptr(), c.data_ptr(), 4, 96, 256, 1, 32, mode, None, 0, s) \
        == tbik.TBIK_ERR_SHAPE
    assert lib.tbik_gemm(a.data_ptr(), b.data_ptr(), c.data_ptr(), 4, 64, 256, 1, 32, mode | tbik.NONINV, None, 0,
                         s) == tbik.TBIK_ERR_ARG
