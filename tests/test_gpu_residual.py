"""The residual add fused into the last step of a row-parallel projection
(tbik_gemm_residual): C = bf16(root + f32(R)), one fp32 add and one rounding,
done in the GEMM epilogue when the tiles write C directly and in the kernel
that combines the shard partials otherwise.  Exact mode is bit-exact to the
oracle; tensor-core mode gives the bits of its own fp32 root plus R rounded
once, for every T and batch size; in place (C = R) gives the same bits.  Also
the RMSNorm without a residual input (r = f32(x)) that follows it."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, host_bits16, host_f32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402


def inputs(seed, M, N, K, b_nk=False):
    a = synth.normal_bf16(seed, (M, K))
    b = synth.normal_bf16(seed + 1, (N, K) if b_nk else (K, N), std=0.05)
    r = synth.normal_bf16(seed + 2, (M, N))
    return a, b, r


# (M, N, K, leaf): tiles that write C directly at T = 1 (1100 x 1088: 306 tiles
# of 64 x 64), frontier splits combined by the tree kernel (small M), ragged M, N
@pytest.mark.parametrize("M,N,K,leaf", [(1, 8, 64, 16), (37, 72, 256, 32), (300, 520, 512, 64),
                                        (1100, 1088, 256, 32)])
@pytest.mark.parametrize("b_nk", [False, True])
def test_exact_bitwise_vs_oracle(M, N, K, leaf, b_nk):
    a, b, r = inputs(900 + M, M, N, K, b_nk)
    da, db = dev_bf16(a), dev_bf16(b)
    for T in (1, 2, 8) if (K // leaf) % 8 == 0 else (1, 2):
        ref = oracle.gemm_residual(a, b, r, b_nk=b_nk, T=T, leaf=leaf)
        got = host_bits16(tbik.gemm(da, db, T=T, leaf=leaf, tc=False, b_nk=b_nk, residual=dev_bf16(r)))
        assert np.array_equal(got, ref), T
    # the non-invariant baseline adds R after its left-to-right shard sum
    ref = oracle.gemm_residual(a, b, r, b_nk=b_nk, T=2, leaf=leaf, noninv=True)
    got = host_bits16(tbik.gemm(da, db, T=2, leaf=leaf, tc=False, noninv=True, b_nk=b_nk, residual=dev_bf16(r)))
    assert np.array_equal(got, ref)
    assert tbik.get_error() == tbik.TBIK_OK


@pytest.mark.parametrize("M", [1, 200, 2048])  # 2048 x 2048: direct tiles at T = 1
def test_tc_is_its_fp32_root_plus_r_rounded_once(M):
    N, K = 2048, 1024
    a, b, r = inputs(930, M, N, K)
    da, db, dr = dev_bf16(a), dev_bf16(b), dev_bf16(r)
    root = host_f32(tbik.gemm(da, db, T=1, leaf=256, tc=True))
    ref = oracle.add_residual_bf16(root, r)
    for T in (1, 2, 4):
        got = host_bits16(tbik.gemm(da, db, T=T, leaf=256, tc=True, residual=dr))
        assert np.array_equal(got, ref), T
    # in place: the residual tensor receives the result
    h = dev_bf16(r)
    tbik.gemm(da, db, T=1, leaf=256, tc=True, residual=h, out=h)
    assert np.array_equal(host_bits16(h), ref)
    h = dev_bf16(r)
    tbik.gemm(da, db, T=4, leaf=256, tc=True, residual=h, out=h)
    assert np.array_equal(host_bits16(h), ref)
    if M > 4:  # rows are independent
        part = host_bits16(tbik.gemm(da[2:M - 1].contiguous(), db, T=2, leaf=256, tc=True,
                                     residual=dr[2:M - 1].contiguous()))
        assert np.array_equal(part, ref[2:M - 1])
    assert tbik.get_error() == tbik.TBIK_OK


def test_tc_noninv_baseline_adds_after_its_chain():
    M, N, K = 512, 1024, 2048
    a, b, r = inputs(950, M, N, K)
    da, db, dr = dev_bf16(a), dev_bf16(b), dev_bf16(r)
    for T in (1, 8):
        root = host_f32(tbik.gemm(da, db, T=T, leaf=256, tc=True, noninv=True))
        got = host_bits16(tbik.gemm(da, db, T=T, leaf=256, tc=True, noninv=True, residual=dr))
        assert np.array_equal(got, oracle.add_residual_bf16(root, r)), T


def test_rmsnorm_without_residual_bitwise():
    d = synth.reduction_inputs(333, H=4096, F=16)
    ref_y, _ = oracle.rmsnorm_residual(d["x"], None, d["gamma"], eps=1e-6)
    for T in (1, 8):
        y, ro = tbik.rmsnorm_residual(dev_bf16(d["x"]), None, dev_bf16(d["gamma"]), eps=1e-6, T=T)
        assert np.array_equal(host_bits16(y), ref_y), T
        assert np.array_equal(host_bits16(ro), d["x"])


def test_residual_argument_errors():
    lib = tbik.load_library()
    a = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros((256, 64), dtype=torch.bfloat16, device="cuda")
    r = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    c = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    ws = torch.empty(lib.tbik_gemm_workspace(4, 64, 256, 1, 32, tbik.TC | tbik.OUT_BF16) + 256,
                     dtype=torch.uint8, device="cuda")
    call = lib.tbik_gemm_residual
    args = (4, 64, 256, 1, 32)
    assert call(a.data_ptr(), b.data_ptr(), r.data_ptr(), c.data_ptr(), *args, tbik.TC | tbik.OUT_BF16,
                ws.data_ptr(), ws.numel(), s) == tbik.TBIK_ERR_ARG
    assert call(a.data_ptr(), b.data_ptr(), r.data_ptr(), c.data_ptr(), *args, tbik.TC | tbik.SWIGLU_OUT,
                ws.data_ptr(), ws.numel(), s) == tbik.TBIK_ERR_ARG
    assert call(a.data_ptr(), b.data_ptr(), None, c.data_ptr(), *args, tbik.TC, ws.data_ptr(), ws.numel(),
                s) == tbik.TBIK_ERR_ARG
    assert call(a.data_ptr(), b.data_ptr(), r.data_ptr() + 2, c.data_ptr(), *args, tbik.TC, ws.data_ptr(),
                ws.numel(), s) == tbik.TBIK_ERR_ALIGN
    with pytest.raises(ValueError):
        tbik.gemm(a, b, residual=r[:, :32].contiguous())
    assert tbik.get_error() == tbik.TBIK_OK
