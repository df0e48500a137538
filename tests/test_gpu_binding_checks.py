"""The Python binding refuses tensors whose shapes do not fit the call before
anything is launched: the C ABI takes plain pointers, so a short companion
buffer (targets, positions, a residual, an output) would otherwise be read or
written past its end."""
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

import invariant_tree_ordered_b200 as tbik  # noqa: E402


def z(*shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype, device="cuda")


def test_gemm_outputs():
    a, b = z(8, 64), z(64, 32)
    with pytest.raises(ValueError):
        tbik.gemm(a, b, leaf=16, out=z(8, 16, dtype=torch.float32))
    with pytest.raises(TypeError):
        tbik.gemm(a, b, leaf=16, out=z(8, 32))  # fp32 output expected
    with pytest.raises(ValueError):
        tbik.gemm(a, b, leaf=16, swiglu=True, out=z(8, 32))  # SwiGLU output is [M, N/2]
    with pytest.raises(ValueError):
        tbik.gemm(a, b, leaf=16, residual=z(8, 32), out=z(4, 32))


def test_reduction_companions():
    x, g = z(4, 256), z(256)
    with pytest.raises(ValueError):
        tbik.rmsnorm_residual(x, z(2, 256), g)
    with pytest.raises(ValueError):
        tbik.rmsnorm_residual(x, x, z(128))
    with pytest.raises(ValueError):
        tbik.rmsnorm_residual(x, x, g, y=z(2, 256))
    tab = tbik.rope_table(16, 64, 1e4)
    q = z(3, 2, 64)
    with pytest.raises(ValueError):
        tbik.rope_swiglu(q=q, pos=z(2, dtype=torch.int32), table=tab)
    with pytest.raises(ValueError):
        tbik.rope_swiglu(q=q, k=z(3, 1, 64), pos=z(3, dtype=torch.int32), table=tab)
    with pytest.raises(ValueError):
        tbik.rope_swiglu(q=z(3, 2, 128), pos=z(3, dtype=torch.int32), table=tab)  # table built for head_dim 64
    with pytest.raises(ValueError):
        tbik.rope_swiglu(g=z(16), u=z(8))
    with pytest.raises(ValueError):
        tbik.rope_swiglu(g=z(16), u=z(16), out=z(8))
    assert tbik.get_error() == tbik.TBIK_OK


def test_logprob_attention_embedding_transpose():
    h, w = z(4, 256), z(1000, 256)
    with pytest.raises(ValueError):
        tbik.logprob(h, w, z(3, dtype=torch.int32))
    with pytest.raises(ValueError):
        tbik.logprob(h, z(1000, 128), z(4, dtype=torch.int32))
    with pytest.raises(ValueError):
        tbik.logprob(h, w, z(4, dtype=torch.int32), out=z(2, dtype=torch.float32))
    q = z(1, 8, 2, 64)
    with pytest.raises(ValueError):
        tbik.attention(q, q, q, out=z(1, 4, 2, 64))
    with pytest.raises(ValueError):
        tbik.embedding(z(5, dtype=torch.int32), z(10, 16), out=z(4, 16))
    with pytest.raises(ValueError):
        tbik.transpose(z(3, 5), out=z(3, 5))
    assert tbik.get_error() == tbik.TBIK_OK
