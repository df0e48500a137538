"""End-to-end decoder (Llama-style, pre-norm) built from the library's calls:
per-token logprobs bit-exact to the oracle decoder in exact-order mode (small
configuration, with the residual add in the RMSNorm or fused into the o and
down projections), and in tensor-core mode bitwise identical across T in
{1,2,4,8} and across batch compositions at the full configuration (4 layers,
d 2048, 16 heads of 128, ffn 5632, vocab 32000, batch 8 x seq 2048), while the
non-invariant baseline diverges with T."""
import numpy as np
import pytest

import oracle.decoder as odec
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
from tests.gpu_util import dev_bf16, dev_i32, host_f32, u32  # noqa: E402

import invariant_tree_ordered_b200 as tbik  # noqa: E402
from invariant_tree_ordered_b200.decoder import Decoder, DecoderConfig, interleave_gate_up, positions  # noqa: E402


def build(cfg, out_in=False):
    """The decoder on device; out_in: projection weights stored [out, in]."""
    w = synth.decoder_weights(cfg)
    lay = (lambda a: np.ascontiguousarray(a.T)) if out_in else (lambda a: a)  # noqa: E731
    layers = []
    for L in w["layers"]:
        dl = {k: dev_bf16(lay(L[k])) for k in ("wq", "wk", "wv", "wo", "wd")}
        dl["wgu"] = dev_bf16(lay(interleave_gate_up(L["wg"], L["wu"])))
        layers.append(dl)
    dc = DecoderConfig(d=cfg["d"], heads=cfg["heads"], head_dim=cfg["head_dim"], ffn=cfg["ffn"],
                       vocab=cfg["vocab"], layers=cfg["layers"], leaf=cfg["leaf"], leaf_ffn=cfg["leaf_ffn"],
                       w_out_in=out_in)
    return w, Decoder(dc, dev_bf16(w["emb"]), dev_bf16(w["lm_head"]), dev_bf16(w["gamma"]), layers)


def run(dec, ids, tg, **kw):
    B, S = ids.shape
    return host_f32(dec.forward(dev_i32(ids), dev_i32(tg), dev_i32(positions(B, S)), **kw))


@pytest.fixture(scope="module")
def small():
    cfg = synth.DECODER_SMALL
    w, dec = build(cfg)
    ids, tg = synth.decoder_tokens(cfg)
    return cfg, w, dec, ids, tg


def test_small_exact_matches_oracle_decoder(small):
    cfg, w, dec, ids, tg = small
    for T, noninv in ((1, False), (8, False), (4, True)):
        got = run(dec, ids, tg, T=T, tc=False, noninv=noninv)
        ref = odec.forward(cfg, w, ids, tg, T=T, noninv=noninv)
        assert np.array_equal(u32(got), u32(ref)), (T, noninv)
    assert tbik.get_error() == tbik.TBIK_OK


def test_small_fused_residual_exact_matches_oracle_decoder(small):
    cfg, w, dec, ids, tg = small
    for T, noninv in ((1, False), (8, False), (4, True)):
        got = run(dec, ids, tg, T=T, tc=False, noninv=noninv, fuse_residual=True)
        ref = odec.forward(cfg, w, ids, tg, T=T, noninv=noninv, fuse_residual=True)
        assert np.array_equal(u32(got), u32(ref)), (T, noninv)
    outs = [run(dec, ids, tg, T=T, tc=True, fuse_residual=True) for T in (1, 2, 8)]
    for o in outs[1:]:
        assert np.array_equal(u32(o), u32(outs[0]))
    assert tbik.get_error() == tbik.TBIK_OK


def test_small_out_in_weights_exact_and_tc_bits(small):
    """Weights stored [out, in] (the tensor-core GEMM's 192-column tiles): exact
    mode stays bit-exact to the oracle decoder, tensor-core mode gives the same
    bits as the [in, out] layout."""
    cfg, w, dec, ids, tg = small
    _, dec_t = build(cfg, out_in=True)
    ref = odec.forward(cfg, w, ids, tg, T=1)
    assert np.array_equal(u32(run(dec_t, ids, tg, T=2, tc=False)), u32(ref))
    for T in (1, 8):
        assert np.array_equal(u32(run(dec_t, ids, tg, T=T, tc=True)), u32(run(dec, ids, tg, T=T, tc=True))), T
    assert np.array_equal(u32(run(dec_t, ids, tg, T=1, tc=True, fuse_residual=True)),
                          u32(run(dec, ids, tg, T=1, tc=True, fuse_residual=True)))


def test_small_tc_invariant_and_close_to_oracle(small):
    cfg, w, dec, ids, tg = small
    outs = [run(dec, ids, tg, T=T, tc=True) for T in (1, 2, 4, 8)]
    for o in outs[1:]:
        assert np.array_equal(u32(o), u32(outs[0]))
    ref = odec.forward(cfg, w, ids, tg, T=1)
    # the tensor-core leaves round differently from the exact chains, and each
    # layer rounds its activations to bf16 (a flipped rounding moves a value
    # by one bf16 ulp, 2^-8 relative), so the two paths agree only to that scale
    assert np.max(np.abs(outs[0] - ref)) <= 2e-2
    assert np.mean(np.abs(outs[0] - ref)) <= 2e-3


@pytest.fixture(scope="module")
def full():
    cfg = synth.DECODER_FULL
    w, dec = build(cfg)
    ids, tg = synth.decoder_tokens(cfg)
    return cfg, dec, ids, tg


def test_full_config_tc_invariant_over_T_and_batch(full):
    cfg, dec, ids, tg = full
    base = run(dec, ids, tg, T=1, tc=True)
    assert np.all(np.isfinite(base))
    for T in (2, 4, 8):
        assert np.array_equal(u32(run(dec, ids, tg, T=T, tc=True)), u32(base)), T
    perm = synth.permutation(33, cfg["batch"])
    shuf = run(dec, ids[perm].copy(), tg[perm].copy(), T=4, tc=True)
    assert np.array_equal(u32(shuf), u32(base[perm]))
    sub = run(dec, ids[[6, 1]].copy(), tg[[6, 1]].copy(), T=8, tc=True)
    assert np.array_equal(u32(sub), u32(base[[6, 1]]))
    # a plausible scale for random init: close to -ln(vocab)
    assert abs(float(base.mean()) + np.log(cfg["vocab"])) < 0.5
    # the residual add fused into the o and down projections: invariant too,
    # and within bf16 rounding of the unfused composition
    fused = run(dec, ids, tg, T=1, tc=True, fuse_residual=True)
    assert np.array_equal(u32(run(dec, ids, tg, T=8, tc=True, fuse_residual=True)), u32(fused))
    assert float(np.mean(np.abs(fused - base))) < 2e-2
    assert tbik.get_error() == tbik.TBIK_OK


def test_full_config_tc_attention_invariant_and_close(full):
    """The attention on the tensor cores (tbik_attention_tc): the decoder stays
    bitwise identical across T and batch compositions, and its logprobs stay
    close to those with the exact-order attention (the per-layer bf16
    activations differ by about one rounding, 2^-8 relative)."""
    cfg, dec, ids, tg = full
    base = run(dec, ids, tg, T=1, tc=True, attention_tc=True)
    assert np.all(np.isfinite(base))
    for T in (2, 8):
        assert np.array_equal(u32(run(dec, ids, tg, T=T, tc=True, attention_tc=True)), u32(base)), T
    sub = run(dec, ids[[5, 2]].copy(), tg[[5, 2]].copy(), T=4, tc=True, attention_tc=True)
    assert np.array_equal(u32(sub), u32(base[[5, 2]]))
    ref = run(dec, ids, tg, T=1, tc=True)
    assert float(np.mean(np.abs(base - ref))) < 2e-2
    assert tbik.get_error() == tbik.TBIK_OK


def test_full_config_noninv_baseline_diverges_over_T(full):
    cfg, dec, ids, tg = full
    outs = {T: run(dec, ids, tg, T=T, tc=True, noninv=True) for T in (1, 2, 4, 8)}
    diffs = {T: float(np.max(np.abs(outs[T] - outs[1]))) for T in (2, 4, 8)}
    print("non-invariant baseline: max |logprob(T) - logprob(1)|", diffs)
    assert any(d > 0.0 for d in diffs.values())
