"""Pins of the CPU oracle against what the MixLLM text and mathematics fix.

Each test checks the oracle against something other than itself: hand-worked
closed-form examples, a library conversion (numpy's binary16), pure-Python brute
force, a textbook integer GEMM, exactly representable inputs whose dequantized
product is a plain fp64 matmul, and invariants (round-trip bounds, permutation).
"""
import numpy as np
import pytest

from mixed_precision_quantized_mx_b200 import inputs


def f16bits(v):
    return int(np.array([v], np.float16).view(np.uint16)[0])


# --------------------------------------------------------------- binary16
def test_fp16_round_matches_numpy(orc):
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(4000) * 10.0 ** rng.integers(-9, 6, 4000),
        rng.uniform(-70000, 70000, 500),
        np.ldexp(1.0, np.arange(-30, 17)),
    ]).astype(np.float32)
    with np.errstate(over="ignore"):
        wants = vals.astype(np.float16).astype(np.float64)
    for v, want in zip(vals, wants):
        got = orc.fp16_round(float(v))
        assert got == want or (np.isinf(want) and np.isinf(got) and np.sign(want) == np.sign(got)), v
        if np.isfinite(want):
            assert orc.fp16_bits(got) == f16bits(want)
            assert orc.fp16_value(orc.fp16_bits(got)) == want


def test_fp16_round_hand_values(orc):
    # largest finite, the half-ulp overflow boundary, subnormals, ties to even
    assert orc.fp16_round(65504.0) == 65504.0
    assert orc.fp16_round(65519.0) == 65504.0
    assert np.isinf(orc.fp16_round(65520.0))
    assert orc.fp16_round(2.0 ** -24) == 2.0 ** -24
    assert orc.fp16_round(2.0 ** -25) == 0.0                 # tie between 0 and 2^-24 -> even (0)
    assert orc.fp16_round(1.5 * 2.0 ** -24) == 2.0 ** -23    # tie -> even mantissa 2
    assert orc.fp16_round(1.0 + 2.0 ** -11) == 1.0           # tie -> even
    assert orc.fp16_round(1.0 + 3 * 2.0 ** -11) == 1.0 + 2.0 ** -9
    assert orc.fp16_bits(1.0) == 0x3C00
    assert orc.fp16_bits(-2.0) == 0xC000
    assert orc.fp16_bits(65504.0) == 0x7BFF
    assert orc.fp16_bits(2.0 ** -24) == 0x0001
    assert orc.fp16_bits(2.0 ** -14) == 0x0400


# --------------------------------------------------------------- symmetric 8-bit
def test_sym8_ties_half_even(orc):
    # s = 127/127 = 1 exactly: codes are round-half-even of x
    q, s = orc.quant_sym8([127, 2.5, 3.5, -2.5, 0.5, -0.5, 1.5, -127])
    assert s == 0x3C00
    assert q.tolist() == [127, 2, 4, -2, 0, 0, 2, -127]


def test_sym8_scale_is_rounded_fp16(orc):
    # amax = 1 -> 1/127 = 0.0078740.. -> nearest fp16 0.00787353515625 (0x2008)
    q, s = orc.quant_sym8([1.0, -0.25])
    assert s == 0x2008
    assert q.tolist() == [127, round(-0.25 / 0.00787353515625)]


def test_sym8_degenerate(orc):
    q, s = orc.quant_sym8(np.zeros(128))
    assert s == 0x3C00 and not q.any()                         # zero group: s = 1
    q, s = orc.quant_sym8(np.full(64, 1e-10))
    assert s == 0x3C00 and not q.any()                         # fp16 underflow: s = 1
    q, s = orc.quant_sym8(np.array([1e7, -3e6], np.float32))
    assert s == 0x7BFF                                          # saturates at 65504
    assert q.tolist() == [127, -46]                             # 3e6/65504 = 45.8 -> 46


def test_sym8_round_trip_bound(orc):
    rng = np.random.default_rng(2)
    for t in range(300):
        x = (rng.standard_normal(128) * 10.0 ** rng.uniform(-4, 3)).astype(np.float32)
        if t % 7 == 0:
            x[rng.integers(128)] *= 50
        q, sb = orc.quant_sym8(x)
        s = orc.fp16_value(sb)
        err = np.abs(x.astype(np.float64) - q.astype(np.float64) * s)
        i = int(np.argmax(np.abs(x)))
        if s >= 2.0 ** -14:
            # normal fp16 scale: relative rounding <= 2^-11, so nothing clamps
            assert err.max() <= s / 2 * (1 + 1e-12)
            assert abs(int(q[i])) == 127                        # the absmax element hits the edge
        else:
            # subnormal scale: coarse rounding may push |x|/s past 127.5; only those clamp
            inner = np.abs(q.astype(np.int64)) < 127
            assert err[inner].max(initial=0) <= s / 2 * (1 + 1e-12)
            assert (np.abs(x[~inner]) >= 126.5 * s * (1 - 1e-7)).all()


def test_sym8_idempotent_on_grid(orc):
    rng = np.random.default_rng(3)
    for _ in range(200):
        s = float(np.float16(10.0 ** rng.uniform(-5, 1)))
        codes = rng.integers(-127, 128, 128)
        codes[rng.integers(128)] = 127 * rng.choice([-1, 1])
        x = (codes * s).astype(np.float32)
        assert np.array_equal(x.astype(np.float64), codes * s)   # exact in fp32
        q, sb = orc.quant_sym8(x)
        assert sb == f16bits(s)
        assert np.array_equal(q, codes.astype(np.int8))


# --------------------------------------------------------------- asymmetric 4-bit
def test_asym4_hand_example(orc):
    # lo=-1, hi=2: s = fp16(3/15) = 0.199951171875 (0x3266); z = round(5.0012) = 5
    q, z, s = orc.quant_asym4([-1.0, 2.0])
    assert (s, z) == (0x3266, 5)
    assert q.tolist() == [0, 15]


def test_asym4_ties_and_clamp(orc):
    # range 15 -> s = 1, z = round_half_even(7.5) = 8; 7.5 -> 8 + 8 = 16 clamps to 15
    q, z, s = orc.quant_asym4([-7.5, 7.5, 0.5, 1.5, 2.5, -0.5, -1.5])
    assert (s, z) == (0x3C00, 8)
    assert q.tolist() == [0, 15, 8, 10, 10, 8, 6]


def test_asym4_zero_in_range(orc):
    q, z, s = orc.quant_asym4(np.linspace(0.5, 3.0, 64))      # all positive: lo = 0
    assert z == 0 and q.min() >= 0
    q, z, s = orc.quant_asym4(-np.linspace(0.5, 3.0, 64))     # all negative: hi = 0
    assert z == 15
    q, z, s = orc.quant_asym4(np.zeros(128))
    assert (s, z) == (0x3C00, 0) and not q.any()
    q, z, s = orc.quant_asym4(np.full(32, 2.0))                # constant group
    sv = orc.fp16_value(s)
    assert z == 0 and sv == float(np.float16(np.float32(2.0) / np.float32(15)))
    assert set(q.tolist()) == {15}


def test_asym4_round_trip_bound(orc):
    rng = np.random.default_rng(4)
    clamp_hits = 0
    for t in range(400):
        x = (rng.standard_normal(128) * 0.02 + rng.uniform(-0.02, 0.02)).astype(np.float32)
        if t % 5 == 0:
            x[rng.integers(128)] *= 10
        q, z, sb = orc.quant_asym4(x)
        s = orc.fp16_value(sb)
        assert 0 <= z <= 15 and q.min() >= 0 and q.max() <= 15
        err = np.abs(x.astype(np.float64) - (q.astype(np.float64) - z) * s)
        # <= s/2 unless the top code clamps, where fp16 rounding of s adds at most 15 s 2^-10
        assert err.max() <= s * (0.5 + 15 * 2.0 ** -10)
        unclamped = q < 15
        assert err[unclamped].max() <= s / 2 * (1 + 1e-12)
        clamp_hits += int((err > s / 2 * (1 + 1e-12)).any())
    assert clamp_hits < 40


def test_asym4_idempotent_on_grid(orc):
    rng = np.random.default_rng(5)
    for _ in range(200):
        s = float(np.float16(10.0 ** rng.uniform(-4, 0)))
        zz = int(rng.integers(0, 16))
        codes = rng.integers(0, 16, 128)
        codes[0], codes[1] = 0, 15
        rng.shuffle(codes)
        x = ((codes - zz) * s).astype(np.float32)
        q, z, sb = orc.quant_asym4(x)
        assert (z, sb) == (zz, f16bits(s))
        assert np.array_equal(q, codes.astype(np.uint8))


# --------------------------------------------------------------- activations
def test_quant_act_per_token_and_group(orc):
    rng = np.random.default_rng(6)
    M, K = 5, 512
    codes = rng.integers(-127, 128, (M, K))
    codes[:, 7] = 127
    scales = np.array([float(np.float16(v)) for v in 10.0 ** rng.uniform(-3, 0, M)])
    X = (codes * scales[:, None]).astype(np.float32)
    Aq, sa = orc.quant_act(X)
    assert np.array_equal(Aq, codes.astype(np.int8))
    assert [orc.fp16_value(b) for b in sa] == scales.tolist()
    # group mode: every 128-column slice is its own symmetric group
    Xr = rng.standard_normal((M, K)).astype(np.float32)
    Aq_g, sa_g = orc.quant_act(Xr, act_group=128)
    assert sa_g.shape == (M, 4)
    for m in range(M):
        for j in range(4):
            sl = Xr[m, j * 128:(j + 1) * 128].astype(np.float64)
            s = orc.fp16_value(sa_g[m, j])
            assert np.abs(sl - Aq_g[m, j * 128:(j + 1) * 128] * s).max() <= s / 2 * (1 + 1e-12)
            assert np.abs(Aq_g[m, j * 128:(j + 1) * 128]).max() == 127


# --------------------------------------------------------------- packing
def test_pack_permutation(orc):
    L = inputs.tiny_layer(0)
    c = orc.pack(L.W, L.is8, 128)
    assert c.n8 == 51 == int(L.is8.sum())
    assert sorted(c.perm.tolist()) == list(range(512))
    assert c.perm[:51].tolist() == np.flatnonzero(L.is8).tolist()
    assert c.perm[51:].tolist() == np.flatnonzero(L.is8 == 0).tolist()


def test_pack_permutation_invariance(orc):
    rng = np.random.default_rng(7)
    N, K = 96, 256
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    mask = (rng.random(N) < 0.3).astype(np.uint8)
    pi = rng.permutation(N)
    c = orc.pack(W, mask, 64)
    cp = orc.pack(W[pi], mask[pi], 64)
    assert np.array_equal(orc.dequant_weights(cp), orc.dequant_weights(c)[pi])


def test_pack_degenerate_fractions(orc):
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((40, 256)) * 0.02).astype(np.float32)
    c0 = orc.pack(W, np.zeros(40, np.uint8), 128)
    c1 = orc.pack(W, np.ones(40, np.uint8), 128)
    assert c0.n8 == 0 and c0.codes4.shape == (40, 256) and c0.perm.tolist() == list(range(40))
    assert c1.n8 == 40 and c1.codes8.shape == (40, 256) and c1.codes4.shape == (0, 256)
    W0 = orc.dequant_weights(c0)
    W1 = orc.dequant_weights(c1)
    # each dequantized element is within half a step of the original
    s0 = np.repeat(orc.fp16_values(c0.scales4), 128, axis=1)
    s1 = np.repeat(orc.fp16_values(c1.scales8), 128, axis=1)
    assert (np.abs(W0 - W) <= s0 * (0.5 + 15 * 2.0 ** -10)).all()
    assert (np.abs(W1 - W) <= s1 * 0.5 * (1 + 1e-12)).all()


# --------------------------------------------------------------- integer partials
def _brute_partials(Aq, c):
    """Pure-Python int arithmetic straight from the two-step definition."""
    M, K, g, G = Aq.shape[0], c.K, c.group, c.G
    pos = {int(n): j for j, n in enumerate(c.perm)}
    P = np.zeros((M, c.N, G), np.int64)
    for m in range(M):
        for n in range(c.N):
            j = pos[n]
            for gi in range(G):
                acc = 0
                for k in range(gi * g, (gi + 1) * g):
                    if j < c.n8:
                        w = int(c.codes8[j, k])
                    else:
                        w = int(c.codes4[j - c.n8, k]) - int(c.zeros4[j - c.n8, gi])
                    acc += int(Aq[m, k]) * w
                P[m, n, gi] = acc
    return P


def test_partials_brute_force(orc):
    rng = np.random.default_rng(9)
    M, N, K, g = 3, 12, 256, 64
    X = rng.standard_normal((M, K)).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    mask = np.zeros(N, np.uint8)
    mask[[1, 4, 5, 11]] = 1
    Aq, sa = orc.quant_act(X)
    c = orc.pack(W, mask, g)
    P, pmax = orc.partials(Aq, c)
    assert np.array_equal(P, _brute_partials(Aq, c))
    assert pmax == np.abs(P).max()


def test_partials_textbook_gemm(orc):
    rng = np.random.default_rng(10)
    M, N, K = 7, 33, 512
    Aq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    for frac in (0.0, 1.0):
        c = orc.pack(W, np.full(N, frac, np.uint8), 128)
        P, _ = orc.partials(Aq, c)
        if frac:
            Wi = c.codes8.astype(np.int64)
        else:
            Wi = c.codes4.astype(np.int64) - np.repeat(c.zeros4.astype(np.int64), 128, axis=1)
        ref = Aq.astype(np.int64) @ Wi.T           # plain integer GEMM over all K
        assert np.array_equal(P.sum(axis=2)[:, c.perm], ref)


def test_partials_fast_i2f_window(orc):
    # worst case of the group-128 int8 dot product stays inside the 2^22 half-window
    K, g = 128, 128
    Aq = np.full((2, K), 127, np.int8)
    Aq[1] = -127
    W = np.full((2, K), 1.0, np.float32)
    c = orc.pack(W, np.array([1, 0], np.uint8), g)
    P, pmax = orc.partials(Aq, c)
    assert pmax == 127 * 127 * 128 < 2 ** 22


# --------------------------------------------------------------- Y
def test_gemm_two_ways_agree(orc):
    L = inputs.tiny_layer(0)
    Aq, sa = orc.quant_act(L.X)
    c = orc.pack(L.W, L.is8, L.group)
    yd, yt = orc.gemm(Aq, sa, c)
    assert np.abs(yd - yt).max() <= 1e-12 * np.abs(yt).max()
    # sampled entries equal the full matrix
    rng = np.random.default_rng(0)
    m = rng.integers(0, 16, 50)
    n = rng.integers(0, 512, 50)
    sd, st = orc.gemm(Aq, sa, c, pairs=(m, n))
    assert np.array_equal(sd, yd[m, n]) and np.array_equal(st, yt[m, n])


def _grid_layer(rng, M, N, K, g, n8):
    """X and W exactly on their quantization grids, so dequant(quant(.)) is the identity."""
    codes = rng.integers(-127, 128, (M, K))
    codes[np.arange(M), rng.integers(0, K, M)] = 127
    sa = np.array([float(np.float16(v)) for v in 10.0 ** rng.uniform(-2, 0, M)])
    X = codes * sa[:, None]
    W = np.zeros((N, K))
    mask = np.zeros(N, np.uint8)
    mask[rng.choice(N, n8, replace=False)] = 1
    for n in range(N):
        for gi in range(K // g):
            s = float(np.float16(10.0 ** rng.uniform(-3, -1)))
            sl = slice(gi * g, (gi + 1) * g)
            if mask[n]:
                q = rng.integers(-127, 128, g)
                q[rng.integers(g)] = 127
                W[n, sl] = q * s
            else:
                z = int(rng.integers(0, 16))
                q = rng.integers(0, 16, g)
                q[:2] = (0, 15)
                W[n, sl] = (q - z) * s
    return X.astype(np.float32), W.astype(np.float32), mask


def test_gemm_exact_grid_equals_fp64_matmul(orc):
    rng = np.random.default_rng(11)
    for (M, N, K, g, n8) in [(4, 24, 256, 128, 5), (3, 16, 256, 64, 0), (2, 10, 128, 128, 10)]:
        X, W, mask = _grid_layer(rng, M, N, K, g, n8)
        Aq, sa = orc.quant_act(X)
        c = orc.pack(W, mask, g)
        assert np.array_equal(orc.dequant_weights(c), W.astype(np.float64))
        yd, yt = orc.gemm(Aq, sa, c)
        ref = X.astype(np.float64) @ W.astype(np.float64).T
        scale = np.abs(ref).max()
        assert np.abs(yd - ref).max() <= 1e-12 * scale
        assert np.abs(yt - ref).max() <= 1e-12 * scale


def test_gemm_group_activations(orc):
    rng = np.random.default_rng(12)
    M, N, K, g = 3, 20, 256, 128
    X = rng.standard_normal((M, K)).astype(np.float32)
    X[:, 3] *= 20
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    mask = (rng.random(N) < 0.2).astype(np.uint8)
    c = orc.pack(W, mask, g)
    Aq, sa = orc.quant_act(X, act_group=g)
    yd, yt = orc.gemm(Aq, sa, c, act_group=g)
    assert np.abs(yd - yt).max() <= 1e-12 * np.abs(yt).max()
    # dequantized product in fp64 with numpy (library matmul)
    Xd = Aq.astype(np.float64) * np.repeat(orc.fp16_values(sa), g, axis=1)
    ref = Xd @ orc.dequant_weights(c).T
    assert np.abs(yd - ref).max() <= 1e-12 * np.abs(ref).max()
    # group-wise scales lose less than one scale per token when an outlier sits in one group
    Aq_t, sa_t = orc.quant_act(X)
    Xt = Aq_t.astype(np.float64) * orc.fp16_values(sa_t)[:, None]
    err_group = np.linalg.norm(Xd - X)
    err_token = np.linalg.norm(Xt - X)
    assert err_group < err_token


# --------------------------------------------------------------- global saliency (precision search)
def _asym4_grid_rows(rng, N, K, g):
    """W whose every group is exactly on its 4-bit asymmetric grid (codes 0 and 15 present)."""
    W = np.zeros((N, K))
    for n in range(N):
        for gi in range(K // g):
            s = float(np.float16(10.0 ** rng.uniform(-3, -1)))
            z = int(rng.integers(0, 16))
            q = rng.integers(0, 16, g)
            q[:2] = (0, 15)
            rng.shuffle(q)
            W[n, gi * g:(gi + 1) * g] = (q - z) * s
    return W.astype(np.float32)


def test_saliency_vanishes_on_the_4bit_grid(orc):
    # quantize() is the 4-bit asymmetric quantizer: on its grid dW = 0, whatever G is.
    # An 8-bit (or any other) quantizer would not reproduce these values exactly.
    rng = np.random.default_rng(40)
    W = _asym4_grid_rows(rng, 12, 512, 128)
    G = rng.standard_normal(W.shape).astype(np.float32) * 100.0
    assert np.array_equal(orc.saliency(W, G, 128), np.zeros(12))
    W8 = (rng.integers(-127, 128, (12, 512)) * 0.01).astype(np.float32)   # on an 8-bit grid only
    assert (orc.saliency(W8, G, 128) > 0).any()


def test_saliency_unit_gradient_is_one_element_error(orc):
    # G = e_k in row n: S1 is that element's quantization error d, S = |d + d^2/2|
    rng = np.random.default_rng(41)
    W = (rng.standard_normal((3, 256)) * 0.05).astype(np.float32)
    for n, k in ((0, 5), (1, 200), (2, 129)):
        G = np.zeros_like(W)
        G[n, k] = 1.0
        g0 = (k // 128) * 128
        q, z, sb = orc.quant_asym4(W[n, g0:g0 + 128])
        d = (float(q[k - g0]) - z) * orc.fp16_value(sb) - float(W[n, k])
        S = orc.saliency(W, G, 128)
        assert S[n] == pytest.approx(abs(d + 0.5 * d * d), rel=1e-15, abs=0)
        assert np.array_equal(np.delete(S, n), np.zeros(2))


def test_saliency_first_and_second_order_terms(orc):
    # flipping G flips S1: S(G) = |S1 + S1^2/2|, S(-G) = |-S1 + S1^2/2|.  For 0 < |S1| < 2
    # both are S1-linear plus or minus the same square: their half-sum is |S1| and their
    # difference is S1^2 (a dropped or mis-scaled second-order term fails this)
    rng = np.random.default_rng(42)
    W = (rng.standard_normal((8, 384)) * 0.02).astype(np.float32)
    G = (rng.standard_normal(W.shape) * 10.0).astype(np.float32)
    Sp, Sm = orc.saliency(W, G, 128), orc.saliency(W, -G, 128)
    s1 = 0.5 * (Sp + Sm)
    assert (s1 > 1e-3).all() and (s1 < 2).all()
    assert np.allclose(np.abs(Sp - Sm), s1 * s1, rtol=1e-9, atol=0)
    # and S1 is linear in G: doubling G doubles |S1|
    S2p, S2m = orc.saliency(W, 2 * G, 128), orc.saliency(W, -2 * G, 128)
    assert np.allclose(0.5 * (S2p + S2m), 2 * s1, rtol=1e-9, atol=0)


def test_saliency_group_sizes_and_zero_gradient(orc):
    rng = np.random.default_rng(43)
    W = (rng.standard_normal((5, 256)) * 0.02).astype(np.float32)
    assert np.array_equal(orc.saliency(W, np.zeros_like(W), 64), np.zeros(5))
    with pytest.raises(ValueError):
        orc.saliency(W[:, :200], np.zeros((5, 200), np.float32), 128)   # K not a multiple of g


def test_select_top_brute_force(orc):
    # the n_top largest scores, ties to the lower index: against an exhaustive check of
    # every index subset on tiny inputs
    import itertools
    rng = np.random.default_rng(44)
    for _ in range(200):
        n = int(rng.integers(1, 8))
        s = rng.integers(0, 4, n).astype(np.float64)        # many ties
        k = int(rng.integers(0, n + 1))
        best = None
        for sub in itertools.combinations(range(n), k):      # lexicographically first optimum
            key = (sum(s[list(sub)]), [-i for i in sub])
            if best is None or key > best[0]:
                best = (key, sub)
        want = np.zeros(n, np.uint8)
        want[list(best[1])] = 1
        assert np.array_equal(orc.select_top(s, k), want), (s, k)
