"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against something the pages or mathematics fix:
hand-evaluated fixtures under tests/golden/, exact integer arithmetic, textbook
special cases (sequential and pairwise summation), error bounds against binary64,
closed forms, and libm/torch routines.  A plausible mistake in the oracle (a
dropped term, a wrong index, a transposed operand, a different tree shape)
fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F = synth.bf16_bits_to_f32


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def bits(a):
    return np.asarray(a, dtype=np.float32).view(np.uint32)


# ---------------------------------------------------------------- generator

def test_splitmix64_published_first_output():
    # SplitMix64 seeded with 0: first output 0xE220A8397B1DCDAF (Vigna's reference
    # implementation of Steele-Lea-Flood).
    assert synth.splitmix64(0, 0) == 0xE220A8397B1DCDAF


def test_generator_is_thread_count_independent_and_offsettable():
    a = synth.normal_bf16(7, (1000,), std=0.5)
    b = synth.normal_bf16(7, (500,), std=0.5, offset=500)
    assert np.array_equal(a[500:], b)
    z = synth.normal_f64(3, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01


# ------------------------------------------------------------------- bf16

def test_bf16_rne_matches_torch():
    torch = pytest.importorskip("torch")
    x = np.concatenate([synth.normal_f32(5, (20000,), std=3.0),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.4e38, -3.4e38, 1e-40],
                                 dtype=np.float32)])
    ours = np.array([oracle.bf16_rne(float(v)) for v in x], dtype=np.uint16)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ----------------------------------------------------------- associativity

def test_associativity_counterexamples():
    g = load("associativity.json")
    a, b, c = g["f64"]["a"], g["f64"]["b"], g["f64"]["c"]
    assert ((a + b) + c).hex() == g["f64"]["left_first"]
    assert (a + (b + c)).hex() == g["f64"]["right_first"]
    f = np.float32
    a, b, c = f(g["f32"]["a"]), f(g["f32"]["b"]), f(g["f32"]["c"])
    assert (a + b) + c == f(g["f32"]["left_first"])
    assert a + (b + c) == f(g["f32"]["right_first"])
    # The decimal example is associative in binary32 (both groupings agree).
    x, y, z = f(0.1), f(0.2), f(0.3)
    assert (x + y) + z == x + (y + z) == f(float.fromhex(g["f32_decimal_example_is_associative"]["value_hex"]))
    # The oracle's tree realises the left-first order on the binary32 case.
    assert oracle.tree_sum([a, b, c]) == f(g["f32"]["left_first"])


# -------------------------------------------------------------- tree shape

def test_tree_shape_golden_cases():
    for case in load("tree_shape.json")["cases"]:
        assert float(oracle.tree_sum(case["leaves"])) == case["tree"], case["why"]


def _halving_lca_depth(n, i, j):
    """Depth of the lowest common ancestor of leaves i and j in the halving tree."""
    lo, depth = 0, 0
    while True:
        h = (n + 1) // 2
        li, lj = i < lo + h, j < lo + h
        if li != lj:
            return depth
        if li:
            n = h
        else:
            lo, n = lo + h, n - h
        depth += 1


@pytest.mark.parametrize("n", [3, 5, 7, 12, 56])
def test_tree_grouping_structural_probe(n):
    """Cancel +-1e8 at leaves (i, j) and put 1 at leaf l, zeros elsewhere.

    The tree returns 1 exactly when i and j meet strictly below the node where l
    joins them (the pair cancels before the 1 can be absorbed into 1e8), else 0.
    The expectation uses only the interval structure of the halving tree.
    """
    rng = np.random.default_rng(n)
    for _ in range(200):
        i, j, l = rng.choice(n, size=3, replace=False)
        p = np.zeros(n, dtype=np.float32)
        p[i], p[j], p[l] = 1e8, -1e8, 1.0
        d_ij = _halving_lca_depth(n, min(i, j), max(i, j))
        d_il = _halving_lca_depth(n, min(i, l), max(i, l))
        expect = 1.0 if d_ij > d_il else 0.0
        assert float(oracle.tree_sum(p)) == expect, (n, i, j, l)


def test_pairwise_special_case_leaf1_power_of_two():
    """leaf = 1 with L = 2^k is textbook pairwise summation (level by level)."""
    rng = np.random.default_rng(1)
    for L in (2, 8, 64, 256):
        a = synth.normal_bf16(40 + L, (3, L))
        b = synth.normal_bf16(41 + L, (L, 5))
        c = oracle.gemm_tree(a, b, b_nk=False, T=1, leaf=1)
        fa, fb = F(a), F(b)
        for i in range(3):
            for n in range(5):
                v = (fa[i, :] * fb[:, n]).astype(np.float32)  # bf16 x bf16 is exact in fp32
                while v.size > 1:
                    v = (v[0::2] + v[1::2]).astype(np.float32)
                assert bits(c[i, n]) == bits(v[0])


def test_sequential_special_case_leaf_equals_K():
    """leaf = K is the naive ascending dot product."""
    a = synth.normal_bf16(50, (2, 96))
    b = synth.normal_bf16(51, (7, 96))
    c = oracle.gemm_tree(a, b, b_nk=True, T=1, leaf=96)
    fa, fb = F(a), F(b)
    for i in range(2):
        for n in range(7):
            acc = np.float32(0.0)
            for k in range(96):
                acc = np.float32(acc + np.float32(fa[i, k] * fb[n, k]))
            assert bits(c[i, n]) == bits(acc)


# ------------------------------------------------------------------- GEMM

@pytest.mark.parametrize("b_nk", [False, True])
def test_gemm_integer_inputs_exact(b_nk):
    """Integer-valued bf16 inputs (|x| <= 16): every partial sum is an integer below
    2^24, so every tree gives the exact int64 product."""
    M, N, K = 5, 9, 512
    a = synth.int_bf16(60, (M, K), 16)
    b = synth.int_bf16(61, (N, K) if b_nk else (K, N), 16)
    ai = F(a).astype(np.int64)
    bi = F(b).astype(np.int64)
    exact = ai @ (bi.T if b_nk else bi)
    for T in (1, 2, 4, 8):
        for leaf in (1, 16, 64):
            c = oracle.gemm_tree(a, b, b_nk=b_nk, T=T, leaf=leaf)
            assert np.array_equal(c.astype(np.int64), exact)


def test_gemm_within_higham_bound():
    """|c_hat - c| <= gamma_{leaf-1+ceil(log2 L)} * sum|a b| (Higham, Accuracy and Stability
    of Numerical Algorithms, ch. 4: recursive summation error bound)."""
    M, N, K, leaf = 6, 11, 1024, 32
    a = synth.normal_bf16(70, (M, K))
    b = synth.normal_bf16(71, (K, N), std=0.02)
    c = oracle.gemm_tree(a, b, b_nk=False, T=1, leaf=leaf).astype(np.float64)
    c64 = oracle.gemm_f64(a, b, b_nk=False)
    absprod = np.abs(F(a).astype(np.float64)) @ np.abs(F(b).astype(np.float64))
    L = K // leaf
    n = leaf - 1 + math.ceil(math.log2(L))
    u = 2.0 ** -24
    gamma = n * u / (1 - n * u)
    assert np.all(np.abs(c - c64) <= gamma * absprod)
    # and the double reference itself matches an independent numpy product
    assert np.allclose(c64, F(a).astype(np.float64) @ F(b).astype(np.float64), rtol=0, atol=1e-12)


def test_gemm_layouts_agree_and_transposition_matters():
    M, N, K = 4, 6, 64
    a = synth.normal_bf16(80, (M, K))
    b_kn = synth.normal_bf16(81, (K, N))
    b_nk = np.ascontiguousarray(b_kn.T)
    c1 = oracle.gemm_tree(a, b_kn, b_nk=False, T=2, leaf=16)
    c2 = oracle.gemm_tree(a, b_nk, b_nk=True, T=2, leaf=16)
    assert np.array_equal(bits(c1), bits(c2))


def test_gemm_invariant_over_T_and_batch_split():
    a, b = synth.tiny_gemm_inputs()
    base, shards = oracle.gemm_tree(a, b, b_nk=False, T=1, leaf=32, shards=True)
    for T in (2, 4, 8):
        c, q = oracle.gemm_tree(a, b, b_nk=False, T=T, leaf=32, shards=True)
        assert np.array_equal(bits(c), bits(base))
        # shard t's partial is the TREE over its own leaves: leaf-wise equal to a
        # GEMM restricted to that K range.
        Ks = 256 // T
        for t in range(T):
            sub = oracle.gemm_tree(a[:, t * Ks:(t + 1) * Ks], b[t * Ks:(t + 1) * Ks], b_nk=False, T=1, leaf=32)
            assert np.array_equal(bits(q[t]), bits(sub))
    # rows are independent: any split or permutation of the batch gives the same rows
    perm = np.array([2, 0, 3, 1])
    cp = oracle.gemm_tree(a[perm], b, b_nk=False, T=4, leaf=32)
    assert np.array_equal(bits(cp), bits(base[perm]))
    for i in range(4):
        ci = oracle.gemm_tree(a[i:i + 1], b, b_nk=False, T=8, leaf=32)
        assert np.array_equal(bits(ci[0]), bits(base[i]))


def test_noninv_baseline_structure_and_divergence():
    M, N, K = 8, 16, 14336 // 8
    a = synth.normal_bf16(90, (M, K))
    b = synth.normal_bf16(91, (K, N), std=0.02)
    # T = 1: one fma chain over K == the tree with a single leaf
    assert np.array_equal(bits(oracle.gemm_noninv(a, b, b_nk=False, T=1)),
                          bits(oracle.gemm_tree(a, b, b_nk=False, T=1, leaf=K)))
    # its shard partials are single-leaf chains over each shard's range
    for T in (2, 4, 8):
        _, q = oracle.gemm_noninv(a, b, b_nk=False, T=T, shards=True)
        _, q2 = oracle.gemm_tree(a, b, b_nk=False, T=T, leaf=K // T, shards=True)
        assert np.array_equal(bits(q), bits(q2))
    outs = [oracle.gemm_noninv(a, b, b_nk=False, T=T) for T in (1, 2, 4, 8)]
    assert any(not np.array_equal(bits(outs[0]), bits(o)) for o in outs[1:])


def test_residual_add_integer_exact_and_single_rounding():
    """bf16(root + R): with integer inputs the sum is an integer below 256, exactly
    representable, so it must equal the int64 result (a dropped R or a wrong sign
    fails); a root just below a bf16 rounding midpoint plus a small R rounds up,
    while rounding the root first would round down (one rounding, not two)."""
    M, N, K = 6, 10, 16
    a = synth.int_bf16(95, (M, K), 3)
    b = synth.int_bf16(96, (K, N), 3)
    r = synth.int_bf16(97, (M, N), 100)
    exact = F(a).astype(np.int64) @ F(b).astype(np.int64) + F(r).astype(np.int64)
    for T, leaf in ((1, 16), (2, 4), (4, 2)):
        c = oracle.gemm_residual(a, b, r, b_nk=False, T=T, leaf=leaf)
        assert np.array_equal(F(c).astype(np.int64), exact)
    one = oracle.bf16_rne
    a1 = np.array([[one(1.0), one(2.0 ** -8), one(-(2.0 ** -12)), 0]], dtype=np.uint16)
    b1 = np.full((4, 1), one(1.0), dtype=np.uint16)
    r1 = np.array([[one(2.0 ** -11)]], dtype=np.uint16)
    c1 = oracle.gemm_residual(a1, b1, r1, b_nk=False, T=1, leaf=4)
    assert F(c1)[0, 0] == 1.0 + 2.0 ** -7
    twice = one(float(np.float32(F(np.array([one(1.0 + 2.0 ** -8 - 2.0 ** -12)]))[0]) + np.float32(2.0 ** -11)))
    assert F(np.array([twice]))[0] == 1.0


def test_residual_add_zero_operands():
    """B = 0: root = +0 and C = R (a -0 residual becomes +0, as +0 + -0 = +0);
    R = +0: C is the single rounding of the root."""
    M, N, K = 3, 8, 64
    a = synth.normal_bf16(98, (M, K))
    r = synth.normal_bf16(99, (M, N))
    r[0, 0] = 0x8000  # -0
    c = oracle.gemm_residual(a, np.zeros((K, N), dtype=np.uint16), r, b_nk=False, T=2, leaf=16)
    expect = r.copy()
    expect[0, 0] = 0
    assert np.array_equal(c, expect)
    b = synth.normal_bf16(100, (K, N), std=0.1)
    for noninv in (False, True):
        root = (oracle.gemm_noninv(a, b, b_nk=False, T=4) if noninv
                else oracle.gemm_tree(a, b, b_nk=False, T=4, leaf=16))
        c0 = oracle.gemm_residual(a, b, np.zeros((M, N), dtype=np.uint16), b_nk=False, T=4, leaf=16, noninv=noninv)
        assert np.array_equal(c0, oracle.bf16_rne_array(root))


def test_rmsnorm_without_residual_input():
    """res = None means r = f32(x): the same as a +0 residual for rows without -0,
    and y = gamma for a row of ones (r = 1, ms = 1, inv = 1 with eps = 0)."""
    d = synth.reduction_inputs(7, H=1024, F=16)
    zero = np.zeros_like(d["x"])
    y0, r0 = oracle.rmsnorm_residual(d["x"], zero, d["gamma"], eps=1e-6)
    y1, r1 = oracle.rmsnorm_residual(d["x"], None, d["gamma"], eps=1e-6)
    assert np.array_equal(y0, y1) and np.array_equal(r1, d["x"]) and np.array_equal(r0, r1)
    x = np.full((1, 1024), oracle.bf16_rne(1.0), dtype=np.uint16)
    y, _ = oracle.rmsnorm_residual(x, None, d["gamma"], eps=0.0)
    assert np.array_equal(y[0], d["gamma"])


# ---------------------------------------------------------------- exp / log

def test_exp_log_specs_against_libm():
    xs = np.linspace(-87.0, 88.0, 40001).astype(np.float32)
    e = oracle.exp_array(xs).astype(np.float64)
    ref = np.exp(xs.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(e - ref) / ulp) <= 1.0
    ys = np.exp(np.linspace(-87, 88, 40001)).astype(np.float32)
    lg = oracle.log_array(ys).astype(np.float64)
    ref = np.log(ys.astype(np.float64))
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(lg - ref) / np.maximum(ulp, 1e-45)) <= 2.0
    assert oracle.exp(0.0) == 1.0 and oracle.log(1.0) == 0.0
    assert oracle.exp(-math.inf) == 0.0 and oracle.exp(math.inf) == math.inf
    assert math.isnan(oracle.exp(math.nan)) and oracle.log(0.0) == -math.inf
    # subnormal results and arguments
    assert oracle.exp(-100.0) == pytest.approx(math.exp(-100.0), rel=2e-3)
    assert oracle.log(1e-42) == pytest.approx(math.log(np.float32(1e-42)), rel=1e-6)


# ---------------------------------------------------------------- RMSNorm

def _rms_f64(x, res, gamma, eps):
    r = (F(x).astype(np.float64) + F(res).astype(np.float64))
    inv = 1.0 / np.sqrt(np.mean(r * r, axis=1, keepdims=True) + eps)
    return r * inv * F(gamma).astype(np.float64), r


def test_rmsnorm_against_f64_and_T_invariance():
    d = synth.reduction_inputs(6, H=4096, F=16)
    y, ro = oracle.rmsnorm_residual(d["x"], d["res"], d["gamma"], eps=1e-6, T=1)
    yf, r = _rms_f64(d["x"], d["res"], d["gamma"], 1e-6)
    # within 1 bf16 ulp of the binary64 value (fp32 intermediates, one rounding)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(yf), 1e-30))) - 7)
    assert np.all(np.abs(F(y).astype(np.float64) - yf) <= 1.0 * ulp)
    # res_out is the rounded fp32 sum
    assert np.array_equal(ro, np.array([oracle.bf16_rne(v) for v in r.ravel().astype(np.float32)],
                                       dtype=np.uint16).reshape(ro.shape))
    for T in (2, 4, 8):
        y2, ro2 = oracle.rmsnorm_residual(d["x"], d["res"], d["gamma"], eps=1e-6, T=T)
        assert np.array_equal(y, y2) and np.array_equal(ro, ro2)


def test_rmsnorm_constant_and_integer_rows():
    H = 256
    gamma = synth.normal_bf16(22, (H,), std=0.1, mean=1.0)
    for c in (3.0, -0.5):
        x = np.full((1, H), oracle.bf16_rne(c), dtype=np.uint16)
        res = np.zeros((1, H), dtype=np.uint16)
        y, _ = oracle.rmsnorm_residual(x, res, gamma, eps=0.0)
        expect = [oracle.bf16_rne(float(np.float32(math.copysign(1.0, c)) * g)) for g in F(gamma)]
        assert np.array_equal(y[0], np.array(expect, dtype=np.uint16))
    # all-ones row plus all-ones residual: r = 2, ms = 4, inv = 1/2 exactly -> y = gamma
    x = np.full((1, H), oracle.bf16_rne(1.0), dtype=np.uint16)
    y, ro = oracle.rmsnorm_residual(x, x, gamma, eps=0.0)
    assert np.array_equal(y[0], gamma) and np.all(F(ro) == 2.0)


# -------------------------------------------------------------------- RoPE

def test_rope_table_and_rotation():
    tab = oracle.rope_table(64, 128, 1e6)
    assert np.all(tab[0, :, 0] == 1.0) and np.all(tab[0, :, 1] == 0.0)
    i = np.arange(64)
    for p in (1, 17, 63):
        ang = p * (1e6 ** (-(2.0 * i) / 128.0))
        assert np.array_equal(tab[p, :, 0], np.cos(ang).astype(np.float32))
        assert np.array_equal(tab[p, :, 1], np.sin(ang).astype(np.float32))
    x = synth.normal_bf16(26, (5, 4, 128))
    pos = np.array([0, 0, 0, 0, 0], dtype=np.int32)
    assert np.array_equal(oracle.rope(x, pos, tab), x)  # position 0 is the identity


def test_rope_against_f64_and_norm():
    max_pos = 32768
    tab = oracle.rope_table(max_pos, 128, 1e6)
    x = synth.normal_bf16(26, (9, 3, 128))
    pos = np.array([0, 1, 2, 100, 4095, 16384, 30000, 32766, 32767], dtype=np.int32)
    out = oracle.rope(x, pos, tab)
    xf = F(x).astype(np.float64)
    c = tab[pos, :, 0].astype(np.float64)[:, None, :]
    s = tab[pos, :, 1].astype(np.float64)[:, None, :]
    o1 = xf[..., :64] * c - xf[..., 64:] * s
    o2 = xf[..., 64:] * c + xf[..., :64] * s
    ref = np.concatenate([o1, o2], axis=-1)
    got = F(out).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(got - ref) <= ulp * 1.0 + 1e-30)
    # rotation preserves each (i, i+64) pair's norm up to the bf16 roundings
    n_in = xf[..., :64] ** 2 + xf[..., 64:] ** 2
    n_out = got[..., :64] ** 2 + got[..., 64:] ** 2
    assert np.allclose(n_out, n_in, rtol=2e-2, atol=1e-4)


# ------------------------------------------------------------------ SwiGLU

def test_swiglu_against_f64_and_special_values():
    g = synth.normal_bf16(24, (4000,))
    u = synth.normal_bf16(25, (4000,))
    out = oracle.swiglu(g, u)
    gf, uf = F(g).astype(np.float64), F(u).astype(np.float64)
    ref = gf / (1.0 + np.exp(-gf)) * uf
    got = F(out).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(got - ref) <= ulp + 1e-30)
    z = np.zeros(3, dtype=np.uint16)
    assert np.all(F(oracle.swiglu(z, synth.normal_bf16(1, (3,)))) == 0.0)
    big = np.array([oracle.bf16_rne(30.0)], dtype=np.uint16)
    one = np.array([oracle.bf16_rne(1.0)], dtype=np.uint16)
    assert F(oracle.swiglu(big, one))[0] == 30.0  # silu(g) = g for large g
    gf32 = synth.normal_f32(11, (1000,), std=1.28)
    uf32 = synth.normal_f32(12, (1000,), std=1.28)
    ref = gf32.astype(np.float64) / (1.0 + np.exp(-gf32.astype(np.float64))) * uf32
    got = F(oracle.swiglu(gf32, uf32)).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(got - ref) <= ulp + 1e-30)


# ----------------------------------------------------------------- logprob

def test_logprob_against_f64():
    M, V, H = 3, 1000, 512
    h = synth.normal_bf16(30, (M, H))
    w = synth.normal_bf16(31, (V, H), std=0.02)
    t = synth.uniform_int32(32, M, 0, V)
    out = oracle.logprob(h, w, t, T=1, leaf=256)
    ref = oracle.logprob_f64(h, w, t)
    assert np.max(np.abs(out - ref)) <= 1e-5
    # and the binary64 reference agrees with an independent numpy log-softmax
    z = F(h).astype(np.float64) @ F(w).astype(np.float64).T
    ls = z - z.max(1, keepdims=True)
    ls = ls - np.log(np.exp(ls).sum(1, keepdims=True))
    assert np.allclose(ref, ls[np.arange(M), t], atol=1e-12)


def test_logprob_zero_weight_is_minus_log_V():
    V, H = 151936, 256
    h = synth.normal_bf16(30, (1, H))
    w = np.zeros((V, H), dtype=np.uint16)
    out = oracle.logprob(h, w, np.array([12345], dtype=np.int32), leaf=256)
    assert abs(float(out[0]) - (-11.931214658529285)) <= 1e-6


def test_logprob_normalises():
    V, H = 700, 256
    h = synth.normal_bf16(33, (1, H))
    w = synth.normal_bf16(34, (V, H), std=0.05)
    hh = np.repeat(h, V, axis=0)
    t = np.arange(V, dtype=np.int32)
    out = oracle.logprob(hh, w, t, leaf=128).astype(np.float64)
    assert abs(np.exp(out).sum() - 1.0) <= 1e-5
    assert np.all(out == out[0] + (out - out[0]))  # finite


def test_logprob_combine_identity_is_exact_and_T_batch_invariance():
    m = np.array([1.5, -np.inf, 0.25, -np.inf], dtype=np.float32)
    s = np.array([3.0, 0.0, 7.0, 0.0], dtype=np.float32)
    cm, cs = oracle.tree_ms(m[:1], s[:1])
    cm2, cs2 = oracle.tree_ms(m[:2], s[:2])
    assert bits(cm) == bits(cm2) and bits(cs) == bits(cs2)
    M, V, H = 4, 2000, 256
    h = synth.normal_bf16(35, (M, H))
    w = synth.normal_bf16(36, (V, H), std=0.02)
    t = synth.uniform_int32(37, M, 0, V)
    base = oracle.logprob(h, w, t, T=1, leaf=128)
    for T in (2, 4, 8):
        assert np.array_equal(bits(base), bits(oracle.logprob(h, w, t, T=T, leaf=128)))
    perm = synth.permutation(33, M)
    assert np.array_equal(bits(oracle.logprob(h[perm], w, t[perm], T=4, leaf=128)), bits(base[perm]))
    one = oracle.logprob(h[2:3], w, t[2:3], T=8, leaf=128)
    assert bits(one[0]) == bits(base[2])
    bad = oracle.logprob(h[:1], w, np.array([V], dtype=np.int32), leaf=128)
    assert math.isnan(bad[0])


def test_logprob_noninv_diverges_over_T():
    M, V, H = 6, 8192, 256
    h = synth.normal_bf16(38, (M, H))
    w = synth.normal_bf16(39, (V, H), std=0.3)
    t = synth.uniform_int32(40, M, 0, V)
    outs = [oracle.logprob(h, w, t, T=T, leaf=128, noninv=True) for T in (1, 2, 4, 8)]
    assert any(not np.array_equal(bits(outs[0]), bits(o)) for o in outs[1:])


# ------------------------------------------------------------- attention

def _bf16_of(x):
    """bf16 bits of values that bf16 represents exactly (checked)."""
    f = np.asarray(x, dtype=np.float32)
    b = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(synth.bf16_bits_to_f32(b), f)
    return b


def test_attention_single_key_is_v():
    q = synth.normal_bf16(60, (2, 1, 3, 128))
    k = synth.normal_bf16(61, (2, 1, 3, 128))
    v = synth.normal_bf16(62, (2, 1, 3, 128))
    assert np.array_equal(oracle.attention(q, k, v), v)  # p = exp(0) = 1, s = 1, o = v


def test_attention_chunk_tree_grouping_and_causality():
    # equal scores (identical keys) make every p = 1 and every combine factor
    # exp(0) = 1, so o is a plain fp32 sum of v in the chunk tree's grouping:
    # keys [1, 2^27, -2^27] as three 1-key chunks: TREE(3) = (c0 + c1) + c2 = 0
    # (2^27 + 1 rounds to 2^27); the other grouping would give 1.
    S = 3
    q = synth.normal_bf16(63, (1, S, 1, 128))
    k = np.tile(synth.normal_bf16(64, (1, 1, 1, 128)), (1, S, 1, 1))
    vals = np.array([1.0, 2.0**27, -2.0**27], dtype=np.float32)
    v = np.zeros((1, S, 1, 128), dtype=np.float32)
    v[0, :, 0, 0] = vals
    v[0, :, 0, 1] = 2.0  # mean 2 exactly
    vb = _bf16_of(v)
    out = synth.bf16_bits_to_f32(oracle.attention(q, k, vb, chunk=1))
    assert out[0, 2, 0, 0] == 0.0
    assert out[0, 1, 0, 0] == np.float32(np.float32(1.0 + 2.0**27) / 2)  # (1 + 2^27) / 2 over keys 0..1
    assert np.all(out[0, :, 0, 1] == 2.0)
    # one 3-key chunk: o accumulates keys in ascending order by fma, same grouping here
    out3 = synth.bf16_bits_to_f32(oracle.attention(q, k, vb, chunk=4))
    assert out3[0, 2, 0, 0] == 0.0
    # causality: keys and values after position i never change output i
    k2, v2 = k.copy(), vb.copy()
    k2[0, 2] = synth.normal_bf16(65, (1, 128))
    v2[0, 2] = synth.normal_bf16(66, (1, 128))
    o1 = oracle.attention(q, k, vb, chunk=1)
    o2 = oracle.attention(q, k2, v2, chunk=1)
    assert np.array_equal(o1[0, :2], o2[0, :2])


@pytest.mark.parametrize("chunk", [1, 7, 64])
def test_attention_within_binary64_softmax(chunk):
    B, S, NH, D = 2, 150, 2, 128
    q = synth.normal_bf16(67, (B, S, NH, D))
    k = synth.normal_bf16(68, (B, S, NH, D))
    v = synth.normal_bf16(69, (B, S, NH, D))
    got = synth.bf16_bits_to_f32(oracle.attention(q, k, v, chunk=chunk)).astype(np.float64)
    ref = oracle.attention_f64(q, k, v)
    # one bf16 rounding (half an ulp of 2^-7 relative) plus fp32 reduction error
    tol = np.abs(ref) * (2.0**-8 + 2e-5) + 1e-6
    assert np.all(np.abs(got - ref) <= tol)


# ----------------------------------------------------------------- decoder

def test_decoder_zero_layers_leave_the_residual_stream_unchanged():
    """With every layer weight zero, attention gives exactly 0 (v = 0) and so does
    the FFN (silu(0) * 0 = 0), so the oracle decoder must reduce to
    RMSNorm(embedding[ids]) followed by the logprob of the targets, with the
    residual add in the RMSNorm or fused into the projections alike (a residual
    added twice, a misaligned target or a skipped norm fails); a zero lm_head on
    top gives -ln V for every token."""
    import oracle.decoder as odec
    cfg = synth.DECODER_SMALL
    w = synth.decoder_weights(cfg)
    for layer in w["layers"]:
        for k in layer:
            layer[k] = np.zeros_like(layer[k])
    ids, tg = synth.decoder_tokens(cfg)
    x = w["emb"][ids.reshape(-1)]
    y, _ = oracle.rmsnorm_residual(x, None, w["gamma"], eps=1e-6)
    expect = oracle.logprob(y, w["lm_head"], tg.reshape(-1).astype(np.int32), T=1,
                            leaf=cfg["leaf"]).reshape(ids.shape)
    for fuse in (False, True):
        got = odec.forward(cfg, w, ids, tg, T=2, fuse_residual=fuse)
        assert np.array_equal(bits(got), bits(expect)), fuse
    w["lm_head"] = np.zeros_like(w["lm_head"])
    got = odec.forward(cfg, w, ids, tg, T=1)
    assert np.allclose(got, -math.log(cfg["vocab"]), rtol=0, atol=1e-6)


# ------------------------------------------------------ ordering probes
# Hand-derived outputs (tests/golden/ordering_probes.json) on inputs where the
# reduction order, the leaf size or the place of eps changes the result far
# beyond rounding; tests/test_oracle_mutants.py shows each planted mistake fails.

def test_baseline_combine_is_left_to_right():
    from tests import ordering_probes
    ordering_probes.check_baseline_shard_sum()


def test_logprob_baseline_logits_are_summed_left_to_right():
    from tests import ordering_probes
    ordering_probes.check_logprob_baseline_logit_sum()


def test_rmsnorm_leaf_size_mean_and_eps_placement():
    from tests import ordering_probes
    ordering_probes.check_rmsnorm_cancellation()


def test_vocab_leaf_sum_is_ascending():
    from tests import ordering_probes
    ordering_probes.check_vocab_leaf_ascending_sum()


def test_rmsnorm_eps_inside_square_root_closed_form():
    """A row of magnitude ~1e-3 with eps = 1e-6: 1/sqrt(ms + eps) and
    1/(sqrt(ms) + eps) differ by ~30 %; the oracle follows the first within
    one bf16 ulp of the binary64 closed form."""
    H = 4096
    c = 2.0 ** -10
    x = np.full((1, H), c, dtype=np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    gamma = np.full(H, 0x3F80, dtype=np.uint16)
    y, _ = oracle.rmsnorm_residual(xb, None, gamma, eps=1e-6)
    want = c / math.sqrt(c * c + float(np.float32(1e-6)))
    wrong = c / (c + float(np.float32(1e-6)))
    got = float(F(y[0, :1])[0])
    assert abs(got - want) <= want * 2 ** -8
    assert abs(got - wrong) > 0.25 * wrong
