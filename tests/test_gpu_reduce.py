"""GPU parity of residual RMSNorm, RoPE and SwiGLU against the CPU oracle:
bit-exact (same fp32 operation sequence and one bf16 rounding on both sides)."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, dev_f32, dev_i32, host_bits16, host_f32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402


@pytest.mark.parametrize("tokens", [1, 16, 128, 1024, 3000])  # 3000: CTAs loop over several tokens
def test_rmsnorm_bitwise_all_T(tokens):
    d = synth.reduction_inputs(tokens, F=8)
    y_ref, r_ref = oracle.rmsnorm_residual(d["x"], d["res"], d["gamma"], eps=1e-6)
    x, res, gamma = dev_bf16(d["x"]), dev_bf16(d["res"]), dev_bf16(d["gamma"])
    for T in (1, 2, 4, 8):
        y, ro = tbik.rmsnorm_residual(x, res, gamma, eps=1e-6, T=T)
        assert np.array_equal(host_bits16(y), y_ref), T
        assert np.array_equal(host_bits16(ro), r_ref), T
    assert tbik.get_error() == tbik.TBIK_OK


@pytest.mark.parametrize("H", [256, 1024, 8192])
def test_rmsnorm_other_widths(H):
    x = synth.normal_bf16(200, (9, H))
    res = synth.normal_bf16(201, (9, H))
    gamma = synth.normal_bf16(202, (H,), std=0.1, mean=1.0)
    y_ref, r_ref = oracle.rmsnorm_residual(x, res, gamma, eps=1e-5, T=8)
    y, ro = tbik.rmsnorm_residual(dev_bf16(x), dev_bf16(res), dev_bf16(gamma), eps=1e-5, T=8)
    assert np.array_equal(host_bits16(y), y_ref)
    assert np.array_equal(host_bits16(ro), r_ref)


def test_rmsnorm_full_size_sampled_and_batch_invariant():
    d = synth.reduction_inputs(8192, F=8)
    x, res, gamma = dev_bf16(d["x"]), dev_bf16(d["res"]), dev_bf16(d["gamma"])
    y, _ = tbik.rmsnorm_residual(x, res, gamma, T=4)
    rows = [0, 1, 4097, 8191]
    y_ref, _ = oracle.rmsnorm_residual(d["x"][rows], d["res"][rows], d["gamma"])
    assert np.array_equal(host_bits16(y)[rows], y_ref)
    y1, _ = tbik.rmsnorm_residual(x[4097:4098].contiguous(), res[4097:4098].contiguous(), gamma, T=1)
    assert np.array_equal(host_bits16(y1)[0], host_bits16(y)[4097])


def test_rope_table_bitwise_and_full_position_sweep():
    tab_ref = oracle.rope_table(32768, 128, 1e6)
    tab = tbik.rope_table(32768, 128, 1e6)
    assert np.array_equal(host_f32(tab).view(np.uint32), tab_ref.view(np.uint32))
    # every position 0..32767 once
    pos = np.arange(32768, dtype=np.int32)
    q = synth.normal_bf16(26, (32768, 2, 128))
    k = synth.normal_bf16(27, (32768, 2, 128))
    qo, ko, _ = tbik.rope_swiglu(q=dev_bf16(q), k=dev_bf16(k), pos=dev_i32(pos), table=tab)
    assert np.array_equal(host_bits16(qo), oracle.rope(q, pos, tab_ref))
    assert np.array_equal(host_bits16(ko), oracle.rope(k, pos, tab_ref))
    assert tbik.get_error() == tbik.TBIK_OK


@pytest.mark.parametrize("tokens", [1, 16, 128, 1024])
def test_rope_config_shapes_bitwise(tokens):
    d = synth.reduction_inputs(tokens, F=8)
    tab = tbik.rope_table(32768, 128, 1e6)
    tab_ref = oracle.rope_table(32768, 128, 1e6)
    qo, ko, _ = tbik.rope_swiglu(q=dev_bf16(d["q"]), k=dev_bf16(d["k"]), pos=dev_i32(d["pos"]), table=tab)
    assert np.array_equal(host_bits16(qo), oracle.rope(d["q"], d["pos"], tab_ref))
    assert np.array_equal(host_bits16(ko), oracle.rope(d["k"], d["pos"], tab_ref))


def test_rope_in_place_and_bad_position():
    tab = tbik.rope_table(64, 64, 1e4)
    q = synth.normal_bf16(5, (3, 4, 64))
    pos = np.array([1, 63, 7], dtype=np.int32)
    qd = dev_bf16(q)
    tbik.rope_swiglu(q=qd, pos=dev_i32(pos), table=tab, q_out=qd)
    assert np.array_equal(host_bits16(qd), oracle.rope(q, pos, oracle.rope_table(64, 64, 1e4)))
    qo, _, _ = tbik.rope_swiglu(q=dev_bf16(q), pos=dev_i32(np.array([1, 64, 2], dtype=np.int32)), table=tab)
    assert tbik.get_error() == tbik.TBIK_ERR_POSITION
    got = host_bits16(qo)
    assert np.all(np.isnan(synth.bf16_bits_to_f32(got[1])))
    assert np.array_equal(got[0], oracle.rope(q[:1], pos[:1], oracle.rope_table(64, 64, 1e4))[0])
    assert tbik.get_error() == tbik.TBIK_OK


@pytest.mark.parametrize("tokens", [1, 128, 1024])
def test_swiglu_bitwise_bf16_inputs(tokens):
    d = synth.reduction_inputs(tokens)
    _, _, out = tbik.rope_swiglu(g=dev_bf16(d["g"]), u=dev_bf16(d["u"]))
    assert np.array_equal(host_bits16(out), oracle.swiglu(d["g"], d["u"]))


def test_swiglu_bitwise_fp32_inputs_and_special_values():
    g, u = synth.gate_up_preacts(64, 14336)
    _, _, out = tbik.rope_swiglu(g=dev_f32(g), u=dev_f32(u))
    assert np.array_equal(host_bits16(out), oracle.swiglu(g, u))
    sp = np.array([0.0, -0.0, 1e-30, -1e-30, 88.0, 89.5, -87.0, -104.5, 200.0, -200.0, np.inf, -np.inf, 1.0, -1.0,
                   3.0, -3.0], dtype=np.float32)
    ones = np.ones_like(sp)
    _, _, out = tbik.rope_swiglu(g=dev_f32(sp), u=dev_f32(ones))
    ref = oracle.swiglu(sp, ones)
    got = host_bits16(out)
    same = (got == ref) | (np.isnan(synth.bf16_bits_to_f32(got)) & np.isnan(synth.bf16_bits_to_f32(ref)))
    assert np.all(same)


def test_swiglu_every_bf16_gate_value():
    """Every one of the 65536 bf16 bit patterns as the gate (NaNs, infinities,
    subnormals, both zeros included) against the oracle, with two up values:
    the kernel pairs elements for its packed arithmetic, so each pattern is
    checked in both lanes (even and odd positions)."""
    g = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    g2 = np.concatenate([g, np.roll(g, 1)])  # each pattern at an even and an odd index
    for u_val in (1.0, -2.5):
        u = np.full(g2.shape, np.float32(u_val), dtype=np.float32)
        ub = (u.view(np.uint32) >> 16).astype(np.uint16)
        _, _, out = tbik.rope_swiglu(g=dev_bf16(g2), u=dev_bf16(ub))
        ref = oracle.swiglu(g2, ub)
        got = host_bits16(out)
        same = (got == ref) | (np.isnan(synth.bf16_bits_to_f32(got)) & np.isnan(synth.bf16_bits_to_f32(ref)))
        assert np.all(same), u_val
        # bf16 gates read silu(g) from the library's table; the same values as
        # fp32 inputs take the computed path: the two give the same bits
        _, _, out32 = tbik.rope_swiglu(g=dev_f32(synth.bf16_bits_to_f32(g2)), u=dev_f32(synth.bf16_bits_to_f32(ub)))
        got32 = host_bits16(out32)
        same32 = (got == got32) | (np.isnan(synth.bf16_bits_to_f32(got)) & np.isnan(synth.bf16_bits_to_f32(got32)))
        assert np.all(same32), u_val


def test_rope_swiglu_argument_errors():
    lib = tbik.load_library()
    a = tbik._binding.RopeSwigluArgs()
    g = torch.zeros(12, dtype=torch.bfloat16, device="cuda")
    a.g, a.u, a.out, a.n = g.data_ptr(), g.data_ptr(), g.data_ptr(), 12
    s = torch.cuda.current_stream().cuda_stream
    import ctypes
    assert lib.tbik_rope_swiglu_fp32(ctypes.byref(a), s) == tbik.TBIK_ERR_SHAPE
    x = torch.zeros((2, 4096), dtype=torch.bfloat16, device="cuda")
    gm = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    assert lib.tbik_rmsnorm_residual(x.data_ptr(), x.data_ptr(), gm.data_ptr(), x.data_ptr(), None, 2, 4096, 1e-6, 3,
                                     s) == tbik.TBIK_ERR_SHAPE
    assert lib.tbik_rmsnorm_residual(x.data_ptr(), x.data_ptr(), gm.data_ptr(), x.data_ptr(), None, 2, 4000, 1e-6, 1,
                                     s) == tbik.TBIK_ERR_SHAPE
