"""GPU parity of tbik_gemm against the CPU oracle (through the C ABI).

Exact-order mode: bit-exact to the oracle.  Tensor-core mode: bitwise
identical to itself across T and M, and within 2e-5 relative Frobenius error
of the binary64 product.  The non-invariant baseline diverges across T.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, host_bits16, host_f32, oracle_rows, rel_frob, sample_rows, u32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402

TS = (1, 2, 4, 8)


def run(a, b, *, T, leaf, tc, b_nk=False, noninv=False, out_bf16=False):
    c = tbik.gemm(dev_bf16(a), dev_bf16(b), T=T, leaf=leaf, tc=tc, b_nk=b_nk, noninv=noninv, out_bf16=out_bf16)
    assert tbik.get_error() == tbik.TBIK_OK
    return host_bits16(c) if out_bf16 else host_f32(c)


# ------------------------------------------------------------- tiny config

@pytest.mark.parametrize("b_nk", [False, True])
def test_tiny_exact_bitwise_vs_oracle_all_T(b_nk):
    a, b = synth.tiny_gemm_inputs()
    bb = np.ascontiguousarray(b.T) if b_nk else b
    ref = oracle.gemm_tree(a, b, b_nk=False, T=1, leaf=32)
    for T in TS:
        got = run(a, bb, T=T, leaf=32, tc=False, b_nk=b_nk)
        assert np.array_equal(u32(got), u32(ref)), T


@pytest.mark.parametrize("b_nk", [False, True])
def test_tiny_tc_invariant_and_close(b_nk):
    a, b = synth.tiny_gemm_inputs()
    bb = np.ascontiguousarray(b.T) if b_nk else b
    c64 = oracle.gemm_f64(a, b, b_nk=False)
    outs = [run(a, bb, T=T, leaf=32, tc=True, b_nk=b_nk) for T in TS]
    for o in outs[1:]:
        assert np.array_equal(u32(o), u32(outs[0]))
    assert rel_frob(outs[0], c64) <= 2e-5


def test_tc_operand_layouts_agree():
    """[K,N] (MN-major descriptor) and [N,K] (K-major) B give the same bits."""
    M, N, K = 130, 200, 512
    a = synth.normal_bf16(100, (M, K))
    b = synth.normal_bf16(101, (K, N), std=0.05)
    c1 = run(a, b, T=2, leaf=64, tc=True, b_nk=False)
    c2 = run(a, np.ascontiguousarray(b.T), T=2, leaf=64, tc=True, b_nk=True)
    assert rel_frob(c1, oracle.gemm_f64(a, b, b_nk=False)) <= 2e-5
    assert np.array_equal(u32(c1), u32(c2))


# ------------------------------------------------------- ragged shapes

@pytest.mark.parametrize("M,N,K,leaf", [(1, 8, 16, 16), (3, 72, 96, 32), (129, 136, 256, 16),
                                        (200, 264, 1024, 64), (64, 128, 768, 96)])
@pytest.mark.parametrize("b_nk", [False, True])
def test_ragged_exact_bitwise_and_tc_tolerance(M, N, K, leaf, b_nk):
    a = synth.normal_bf16(110 + M, (M, K))
    b = synth.normal_bf16(111 + N, (N, K) if b_nk else (K, N), std=0.05)
    L = K // leaf
    ref = oracle.gemm_tree(a, b, b_nk=b_nk, T=1, leaf=leaf)
    c64 = oracle.gemm_f64(a, b, b_nk=b_nk)
    Ts = [T for T in TS if L % T == 0]
    tc_outs = []
    for T in Ts:
        got = run(a, b, T=T, leaf=leaf, tc=False, b_nk=b_nk)
        assert np.array_equal(u32(got), u32(ref)), ("exact", T)
        tc_outs.append(run(a, b, T=T, leaf=leaf, tc=True, b_nk=b_nk))
    for o in tc_outs[1:]:
        assert np.array_equal(u32(o), u32(tc_outs[0]))
    assert rel_frob(tc_outs[0], c64) <= 2e-5


@pytest.mark.parametrize("M,N", [(3, 5), (1, 7), (5, 9)])
def test_exact_frontier_split_with_odd_output_count(M, N):
    """M*N % 4 != 0 with the tree cut into frontier partials (few output tiles)
    and, for T > 1, per-shard buffers: the shard combine takes its element
    path (the buffers do not start on 16-byte boundaries).  Bit-exact for every
    T, fp32 and bf16 outputs, with and without the fused residual."""
    K, leaf = 256, 32
    a = synth.normal_bf16(125 + M, (M, K))
    b = synth.normal_bf16(126 + N, (K, N), std=0.1)
    r = synth.normal_bf16(127 + N, (M, N))
    ref = oracle.gemm_tree(a, b, b_nk=False, T=1, leaf=leaf)
    ref_bf = np.array([oracle.bf16_rne(float(v)) for v in ref.ravel()], dtype=np.uint16).reshape(ref.shape)
    ref_res = oracle.add_residual_bf16(ref, r)
    for T in TS:
        assert np.array_equal(u32(run(a, b, T=T, leaf=leaf, tc=False)), u32(ref)), T
        assert np.array_equal(run(a, b, T=T, leaf=leaf, tc=False, out_bf16=True), ref_bf), T
        got = tbik.gemm(dev_bf16(a), dev_bf16(b), T=T, leaf=leaf, tc=False, residual=dev_bf16(r))
        assert tbik.get_error() == tbik.TBIK_OK
        assert np.array_equal(host_bits16(got), ref_res), T


def test_exact_leaf_one_and_odd_leaf_counts():
    """Exact mode follows the tree for leaf = 1 and non-power-of-two leaf counts."""
    a = synth.normal_bf16(120, (5, 96))
    b = synth.normal_bf16(121, (96, 40))
    for leaf in (1, 3, 12, 32):
        ref = oracle.gemm_tree(a, b, b_nk=False, T=1, leaf=leaf)
        got = run(a, b, T=1, leaf=leaf, tc=False)
        assert np.array_equal(u32(got), u32(ref)), leaf


def test_bf16_output_is_one_rounding_of_fp32():
    M, N, K = 70, 96, 512
    a = synth.normal_bf16(130, (M, K))
    b = synth.normal_bf16(131, (K, N), std=0.05)
    for tc in (False, True):
        f = run(a, b, T=4, leaf=64, tc=tc)
        h = run(a, b, T=4, leaf=64, tc=tc, out_bf16=True)
        expect = np.array([oracle.bf16_rne(float(v)) for v in f.ravel()], dtype=np.uint16).reshape(f.shape)
        assert np.array_equal(h, expect)


# ---------------------------------------------------- non-invariant baseline

def test_noninv_exact_matches_oracle_and_diverges():
    M, N, K = 8, 96, 14336 // 4
    a = synth.normal_bf16(140, (M, K))
    b = synth.normal_bf16(141, (K, N), std=0.02)
    outs = []
    for T in TS:
        got = run(a, b, T=T, leaf=K // 8, tc=False, noninv=True)
        ref = oracle.gemm_noninv(a, b, b_nk=False, T=T)
        assert np.array_equal(u32(got), u32(ref)), T
        outs.append(got)
    assert any(not np.array_equal(u32(outs[0]), u32(o)) for o in outs[1:])


def test_noninv_tc_diverges_over_T_invariant_does_not():
    M, N, K = 256, 512, 14336
    a = synth.normal_bf16(150, (M, K))
    b = synth.normal_bf16(151, (K, N), std=0.02)
    non = [run(a, b, T=T, leaf=256, tc=True, noninv=True) for T in TS]
    inv = [run(a, b, T=T, leaf=256, tc=True) for T in TS]
    assert any(not np.array_equal(u32(non[0]), u32(o)) for o in non[1:])
    for o in inv[1:]:
        assert np.array_equal(u32(o), u32(inv[0]))


# ---------------------------------------------------- down_proj shape

@pytest.fixture(scope="module")
def down_proj():
    K, N = 14336, 4096
    b = synth.down_proj_weight(K, N, "kn")
    g, u = synth.gate_up_preacts(4096, K)
    a = oracle.swiglu(g, u)  # A = bf16(silu(x.Wg) * (x.Wu)), fixed as input bytes
    return a, b


def test_down_proj_exact_small_M_bitwise(down_proj):
    a, b = down_proj
    for M in (1, 16):
        ref = oracle.gemm_tree(a[:M], b, b_nk=False, T=1, leaf=256)
        for T in (1, 8):
            got = run(a[:M], b, T=T, leaf=256, tc=False)
            assert np.array_equal(u32(got), u32(ref)), (M, T)


def test_down_proj_tc_invariance_over_T_and_M(down_proj):
    a, b = down_proj
    full = {T: run(a, b, T=T, leaf=256, tc=True) for T in TS}
    for T in TS[1:]:
        assert np.array_equal(u32(full[T]), u32(full[1])), T
    for M in (1, 16, 128, 1024):
        part = run(a[:M], b, T=2 if M > 1 else 8, leaf=256, tc=True)
        assert np.array_equal(u32(part), u32(full[1][:M])), M
    # row i sits in a different tile position when the batch is shifted
    sub = run(a[5:133], b, T=4, leaf=256, tc=True)
    assert np.array_equal(u32(sub), u32(full[1][5:133]))
    rows = sample_rows(35, 4096, 64, must=(0, 1, 255, 256, 4095))
    c64 = oracle_rows(lambda rs: oracle.gemm_f64(a[rs], b, b_nk=False), rows)
    assert rel_frob(full[1][rows], c64) <= 2e-5


def test_down_proj_tile_widths_agree_bitwise(down_proj):
    """The 192-column tile kernel (two TMEM accumulators, the pending 2-leaf
    value in registers, a split 3-4 leaf slot; B [K,N] in 64-byte-swizzle
    atoms, B [N,K] K-major) and the 128-column one (three accumulators, TMEM
    and shared-memory slots; the test hook forces it): different storage
    plans and operand layouts for the same 56-leaf tree.  All must give the
    same bits, at T = 1 and T = 8 and for a shifted batch."""
    a, b = down_proj
    bt = np.ascontiguousarray(b.T)
    for T in (1, 8):
        kn = run(a, b, T=T, leaf=256, tc=True)
        nk = run(a, bt, T=T, leaf=256, tc=True, b_nk=True)
        try:
            tbik.debug_set(tbik.DEBUG_TILE128, 0)
            kn128 = run(a, b, T=T, leaf=256, tc=True)
        finally:
            tbik.debug_set(0, 0)
        assert np.array_equal(u32(kn), u32(nk)), T
        assert np.array_equal(u32(kn), u32(kn128)), T
    sub = run(a[7:300], b, T=2, leaf=256, tc=True)
    assert np.array_equal(u32(sub), u32(kn[7:300]))
    assert tbik.get_error() == tbik.TBIK_OK


def test_down_proj_exact_sampled_rows_full_M(down_proj):
    """64 seeded rows (tile edges included) of the exact-mode 4096-row launch at
    T = 8, bit-exact to the oracle."""
    a, b = down_proj
    got = run(a, b, T=8, leaf=256, tc=False)
    rows = sample_rows(36, 4096, 64, must=(0, 63, 64, 2049, 4095))
    ref = oracle_rows(lambda rs: oracle.gemm_tree(a[rs], b, b_nk=False, T=1, leaf=256), rows)
    assert np.array_equal(u32(got[rows]), u32(ref))


# --------------------------------------------------------------- errors

def test_host_side_argument_errors():
    a = dev_bf16(synth.normal_bf16(1, (4, 256)))
    b = dev_bf16(synth.normal_bf16(2, (256, 64)))
    c = torch.empty((4, 64), dtype=torch.float32, device="cuda")
    lib = tbik.load_library()
    s = torch.cuda.current_stream().cuda_stream

    def call(M=4, N=64, K=256, T=1, leaf=32, mode=tbik.TC, ws=None, wsb=0, A=a, C=c):
        return lib.tbik_gemm(A.data_ptr(), b.data_ptr(), C.data_ptr(), M, N, K, T, leaf, mode, ws, wsb, s)

    assert call(T=3) == tbik.TBIK_ERR_SHAPE
    assert call(leaf=24) == tbik.TBIK_ERR_SHAPE           # TC needs leaf % 16 == 0
    assert call(leaf=100) == tbik.TBIK_ERR_SHAPE          # K % leaf
    assert call(T=8, leaf=64) == tbik.TBIK_ERR_SHAPE      # 4 leaves, 8 shards
    assert call(mode=tbik.TC | tbik.EXACT) == tbik.TBIK_ERR_ARG
    assert call(mode=0x80000) == tbik.TBIK_ERR_ARG
    assert call(M=-1) == tbik.TBIK_ERR_ARG
    assert call(M=0) == tbik.TBIK_OK
    ws_need = lib.tbik_gemm_workspace(4, 64, 256, 8, 32, tbik.TC)
    assert ws_need > 0
    assert call(T=8) == tbik.TBIK_ERR_WORKSPACE
    off = torch.empty(64 * 4 + 4, dtype=torch.uint8, device="cuda")
    assert lib.tbik_gemm(off.data_ptr() + 2, b.data_ptr(), c.data_ptr(), 4, 64, 256, 1, 32, tbik.TC, None, 0, s) \
        == tbik.TBIK_ERR_ALIGN
    assert tbik.get_error() == tbik.TBIK_OK
