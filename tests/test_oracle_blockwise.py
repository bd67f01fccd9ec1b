"""Pins of the block-wise bit-width oracle (ScaleBITS blog page: section 1.2.2, one
bit width per 64 x 128 block; section 3.2, 2-bit metadata per block; section 4.2,
widths from {1, 2, 3, 4, 6, 8}) against what the text and mathematics fix.

Each check is independent of the code it pins: hand-worked examples, brute force
over every grid level, the reduction of uniform and row-uniform width maps to the
MixLLM packing (pinned in test_oracle.py), numpy's own binary16 conversion and
fp64 matmul for the plain definition of Y, and closed forms.
"""
import numpy as np
import pytest

from mixed_precision_quantized_mx_b200 import inputs

BR, BC = 64, 128


def f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


# --------------------------------------------------------------- the b-bit quantizer
def test_quant_asym_worked_examples(orc):
    # 2 bits, x in [-1, 2]: s = 3 / 3 = 1, z = round(1) = 1, q = clamp(round(x) + 1, 0, 3),
    # ties to even (round(-0.5) = -0, round(0.5) = 0, round(1.5) = 2)
    x = [-1.0, -0.5, 0.0, 0.5, 1.0, 1.5, 2.0, 0.49, 0.51]
    q, z, s = orc.quant_asym(x, 2)
    assert list(q) == [0, 1, 1, 1, 2, 3, 3, 1, 2] and z == 1 and s == 0x3C00
    # 1 bit, x in [-0.3, 0.7]: s = 1, z = round(0.3) = 0, q = clamp(round(x), 0, 1)
    q, z, s = orc.quant_asym([-0.3, 0.2, 0.7], 1)
    assert list(q) == [0, 0, 1] and z == 0 and s == 0x3C00
    # 3 bits, x in [0, 7]: s = 1, z = 0, round(3.5) = 4
    q, z, s = orc.quant_asym([0.0, 0.7, 3.5, 7.0], 3)
    assert list(q) == [0, 1, 4, 7] and z == 0 and s == 0x3C00
    # 6 bits, all negative: lo = -6.3, hi = 0, s = fp16(6.3 / 63) = fp16(0.1), z = round(63) = 63
    q, z, s = orc.quant_asym([-6.3, -0.1, 0.0], 6)
    assert z == 63 and s == int(np.array([0.1], np.float16).view(np.uint16)[0])
    assert list(q) == [0, 62, 63]


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7])
def test_quant_asym_is_nearest_level(orc, bits):
    # with s and z fixed, the code is the nearest of the 2^b grid levels (j - z) s, found
    # here by brute force over j; the tolerance covers the fp32 rounding of x / s
    rng = np.random.default_rng(bits)
    qmax = (1 << bits) - 1
    for trial in range(40):
        x = (rng.standard_normal(128) * 10.0 ** rng.uniform(-3, 1)).astype(np.float32)
        if trial % 4 == 1:
            x = np.abs(x)
        elif trial % 4 == 2:
            x = -np.abs(x)
        q, z, sb = orc.quant_asym(x, bits)
        s = float(f16(sb))
        assert 0 <= z <= qmax and q.max() <= qmax
        levels = (np.arange(qmax + 1) - z) * s
        best = np.abs(x[:, None].astype(np.float64) - levels[None, :]).min(1)
        got = np.abs(x.astype(np.float64) - (q.astype(np.float64) - z) * s)
        assert (got <= best + 1e-6 * s).all()
        # the grid spans the group's range to within one step (0 is in the range)
        assert levels[0] <= min(0.0, x.min()) + s and levels[-1] >= max(0.0, x.max()) - s


def test_quant_asym_4_bits_is_the_mixllm_quantizer(orc):
    rng = np.random.default_rng(3)
    for _ in range(50):
        x = (rng.standard_normal(128) * 0.05).astype(np.float32)
        q, z, s = orc.quant_asym(x, 4)
        q4, z4, s4 = orc.quant_asym4(x)
        assert np.array_equal(q, q4) and z == z4 and s == s4


def test_quant_asym_rejects_widths_outside_1_to_7(orc):
    for b in (0, 8, 9):
        with pytest.raises(ValueError):
            orc.quant_asym([1.0, 2.0], b)


# --------------------------------------------------------------- metadata
def test_block_code_packing_worked_example(orc):
    codes = np.array([[0, 1, 2, 3], [3, 2, 1, 0], [1, 1, 0, 0]])
    # byte 0: 0 | 1 << 2 | 2 << 4 | 3 << 6 = 0xE4; byte 1: 3 | 2 << 2 | 1 << 4 = 0x1B;
    # byte 2: 1 | 1 << 2 = 0x05
    assert list(orc.pack_block_codes(codes)) == [0xE4, 0x1B, 0x05]
    assert list(orc.pack_block_codes(np.array([[2, 1, 3, 0, 1]]))) == [0x36, 0x01]


def test_bits_per_weight_closed_form(orc):
    W = np.zeros((128, 256), np.float32)
    b = orc.pack_blockwise(W, [[0, 1], [2, 3]], [2, 3, 4, 8])
    # blocks of 64 x 128 at 2, 3, 4 and 8 bits, plus four 2-bit codes
    assert orc.bits_per_weight(b) == pytest.approx((2 + 3 + 4 + 8) / 4 + 8 / (128 * 256), rel=1e-15)
    # a short last row block counts its rows only: 70 rows = 64 + 6
    b = orc.pack_blockwise(np.zeros((70, 128), np.float32), [[1], [0]], [2, 6, 4, 8])
    assert orc.bits_per_weight(b) == pytest.approx((64 * 6 + 6 * 2) / 70 + 4 / (70 * 128), rel=1e-15)


# --------------------------------------------------------------- packing
def test_each_block_uses_its_own_width(orc):
    # N = 200 (a short last row block), K = 512: the codes, zeros and scales of every
    # (row, 128-column) group equal that group quantized alone at its block's width
    rng = np.random.default_rng(5)
    N, K = 200, 512
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    codes = inputs.block_codes(rng, N, K)
    table = np.array([1, 2, 6, 8], np.uint8)
    b = orc.pack_blockwise(W, codes, table)
    assert b.q.shape == (N, K) and b.zeros.shape == (N, K // BC)
    for n in range(N):
        for kb in range(K // BC):
            width = int(table[codes[n // BR, kb]])
            x = W[n, kb * BC:(kb + 1) * BC]
            if width == 8:
                q, s = orc.quant_sym8(x)
                z = 0
            else:
                q, z, s = orc.quant_asym(x, width)
            assert np.array_equal(b.q[n, kb * BC:(kb + 1) * BC], q.astype(np.int16)), (n, kb)
            assert b.zeros[n, kb] == z and b.scales[n, kb] == s
            vals = b.q[n, kb * BC:(kb + 1) * BC]
            if width == 8:
                assert np.abs(vals).max() <= 127
            else:
                assert vals.min() >= 0 and vals.max() <= (1 << width) - 1


def test_changing_one_block_changes_only_that_block(orc):
    rng = np.random.default_rng(6)
    N, K = 192, 384
    W = inputs.weights(rng, N, K)
    codes = np.zeros((3, 3), np.uint8)
    table = [2, 4, 6, 8]
    a = orc.pack_blockwise(W, codes, table)
    codes2 = codes.copy()
    codes2[1, 2] = 3                                   # row block 1, column block 2 -> 8 bits
    c = orc.pack_blockwise(W, codes2, table)
    diff = a.q != c.q
    assert diff[64:128, 256:384].any()
    diff[64:128, 256:384] = False
    assert not diff.any()
    zd = a.scales != c.scales
    assert zd[64:128, 2].all()
    zd[64:128, 2] = False
    assert not zd.any()


def test_uniform_widths_reduce_to_mixllm_packing(orc):
    # every block 4-bit = MixLLM with no 8-bit rows; every block 8-bit = all rows 8-bit;
    # row blocks at 8 then 4 bits = MixLLM with those rows selected (output-feature
    # mixed precision is the row-uniform special case of block-wise widths)
    rng = np.random.default_rng(7)
    N, K, M = 128, 384, 5
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    X = inputs.activations(rng, M, K, 2, dtype=np.float32)
    Aq, sa = orc.quant_act(X)
    for codes, is8 in ((np.zeros((2, 3)), np.zeros(N)), (np.full((2, 3), 3), np.ones(N)),
                       (np.array([[3, 3, 3], [0, 0, 0]]), np.arange(N) < 64)):
        b = orc.pack_blockwise(W, codes, [4, 2, 6, 8])
        yd, yt, P, pmax = orc.gemm_blockwise(Aq, sa, b)
        c = orc.pack(W, is8.astype(np.uint8), 128)
        yd_m, yt_m = orc.gemm(Aq, sa, c)
        P_m, _ = orc.partials(Aq, c)
        assert np.array_equal(P, P_m)
        assert np.array_equal(yt, yt_m) and np.array_equal(yd, yd_m)


# --------------------------------------------------------------- the GEMM
def test_gemm_blockwise_plain_definition(orc):
    # Y against numpy: both operands dequantized with numpy's binary16 conversion, then
    # an fp64 matmul; the partials against a pure-Python integer loop
    rng = np.random.default_rng(8)
    N, K, M = 100, 256, 4
    W = inputs.weights(rng, N, K, outlier_frac=0.01)
    X = inputs.activations(rng, M, K, 3, dtype=np.float32)
    b = orc.pack_blockwise(W, inputs.block_codes(rng, N, K), [1, 3, 4, 8])
    Aq, sa = orc.quant_act(X)
    yd, yt, P, pmax = orc.gemm_blockwise(Aq, sa, b)
    KB = K // BC
    Wd = (b.q.astype(np.float64) - np.repeat(b.zeros.astype(np.float64), BC, 1)) * np.repeat(f16(b.scales), BC, 1)
    Xd = Aq.astype(np.float64) * f16(sa)[:, None]
    ref = Xd @ Wd.T
    assert np.allclose(yd, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(yt, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    for m, n in ((0, 0), (3, 99), (1, 64), (2, 63)):
        for kb in range(KB):
            want = sum(int(Aq[m, k]) * (int(b.q[n, k]) - int(b.zeros[n, kb])) for k in range(kb * BC, (kb + 1) * BC))
            assert P[m, n, kb] == want
    assert pmax < 2 ** 22                     # the window the fast int-to-float conversion needs
    # sampled pairs give the same values as the full product
    pm = np.array([0, 3, 2]), np.array([5, 99, 64])
    yd2, yt2, P2, _ = orc.gemm_blockwise(Aq, sa, b, pairs=pm)
    assert np.array_equal(yd2, yd[pm]) and np.array_equal(P2, P[pm])


def test_dequantization_error_shrinks_with_width(orc):
    rng = np.random.default_rng(9)
    N, K = 128, 256
    W = inputs.weights(rng, N, K)
    errs = []
    for width in (1, 2, 3, 4, 6, 8):
        b = orc.pack_blockwise(W, np.zeros((2, 2)), [width, width, width, width])
        Wd = (b.q.astype(np.float64) - np.repeat(b.zeros.astype(np.float64), BC, 1)) * np.repeat(f16(b.scales), BC, 1)
        err = np.abs(Wd - W)
        # half a step, plus at the ends of the range what the fp16 rounding of s (at most
        # 2^-11 of it) takes off the qmax steps of the grid
        qmax = 127 if width == 8 else (1 << width) - 1
        step = np.repeat(f16(b.scales), BC, 1)
        assert (err <= step * (0.5 + qmax * 2.0 ** -11) * (1 + 1e-6)).all()
        errs.append(err.mean())
    assert all(e1 > e2 for e1, e2 in zip(errs, errs[1:]))


def test_pack_blockwise_rejects_bad_arguments(orc):
    W = np.zeros((64, 200), np.float32)               # K not a multiple of 128
    with pytest.raises((ValueError, AssertionError)):
        orc.pack_blockwise(W, np.zeros((1, 1)), [2, 3, 4, 8])
    with pytest.raises(ValueError):                   # a width outside 1..8
        orc.pack_blockwise(np.zeros((64, 128), np.float32), np.zeros((1, 1)), [2, 3, 4, 9])
