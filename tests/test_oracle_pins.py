"""Pins for the CPU oracle: each check rests on something other than the oracle itself
(exact rational arithmetic, closed forms, invariants of the definitions, brute force,
hand-derived fixtures).  No GPU needed.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import inputs
from oracle import awq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# exact fp16 rounding, built from the IEEE binary16 definition
# ----------------------------------------------------------------------------

def _all_finite_fp16():
    """Sorted (value as Fraction, bit pattern) for every finite non-negative fp16."""
    vals = []
    for bits in range(0x7C00):            # +0 .. largest finite
        e = bits >> 10
        f = bits & 0x3FF
        if e == 0:
            v = Fraction(f, 1 << 24)
        else:
            v = Fraction(1024 + f, 1 << 10) * Fraction(2) ** (e - 15)
        vals.append((v, bits))
    return vals


_FP16 = _all_finite_fp16()
_FP16_VALUES = [v for v, _ in _FP16]
_FP16_MAX = _FP16_VALUES[-1]
_FP16_OVERFLOW = _FP16_MAX + Fraction(1, 2) * Fraction(2) ** (15 - 10)   # 65520: rounds to inf


def exact_round_fp16(x: float) -> float:
    """Round the exact value of a double to binary16, nearest-even, by search."""
    import bisect
    q = Fraction(x)
    sign = -1 if q < 0 else 1
    a = abs(q)
    if a >= _FP16_OVERFLOW:
        return sign * math.inf
    i = bisect.bisect_left(_FP16_VALUES, a)
    if i < len(_FP16_VALUES) and _FP16_VALUES[i] == a:
        return sign * float(a)
    lo_v, lo_b = _FP16[i - 1]
    hi_v, hi_b = _FP16[i] if i < len(_FP16) else (Fraction(65536), 0x7C00)
    d_lo, d_hi = a - lo_v, hi_v - a
    if d_lo < d_hi or (d_lo == d_hi and lo_b % 2 == 0):
        return sign * float(lo_v)
    return sign * (math.inf if hi_b == 0x7C00 else float(hi_v))


def test_fp16_rn_matches_exact_rounding_for_doubles():
    g = np.random.Generator(np.random.PCG64(7))
    xs = list(g.standard_normal(3000) * np.exp(g.uniform(-18, 11, 3000)))
    # values straddling fp16 midpoints by less than a float32 ulp: a double->float->half
    # detour would round these the wrong way
    for v, _ in _FP16[1000:31000:97]:
        nxt = _FP16_VALUES[_FP16_VALUES.index(v) + 1]
        mid = (v + nxt) / 2
        for eps in (Fraction(0), Fraction(1, 2 ** 40), -Fraction(1, 2 ** 40)):
            xs.append(float(mid * (1 + eps)))
    got = O.fp16_rn(np.array(xs, dtype=np.float64)).astype(np.float64)
    want = np.array([exact_round_fp16(x) for x in xs])
    assert np.array_equal(got, want)


def test_fp16_rn_matches_exact_rounding_for_float32():
    g = np.random.Generator(np.random.PCG64(8))
    xs = (g.standard_normal(4000) * np.exp(g.uniform(-18, 11, 4000))).astype(np.float32)
    got = O.fp16_rn(xs).astype(np.float64)
    want = np.array([exact_round_fp16(float(x)) for x in xs])
    assert np.array_equal(got, want)


# ----------------------------------------------------------------------------
# activation statistic, alpha grid, s
# ----------------------------------------------------------------------------

def test_act_absmean_is_the_exact_mean():
    X = inputs.activations(37, 96, seed=11)
    m = O.act_absmean(X)
    for k in range(0, 96, 5):
        exact = sum(Fraction(abs(float(v))) for v in X[:, k]) / 37
        assert m[k] == float(exact)       # float(Fraction) rounds once, to nearest


def test_act_absmean_order_independent():
    X = inputs.activations(512, 64, seed=12)
    a = O.act_absmean(X)
    b = O.act_absmean(X[::-1].copy())
    assert np.array_equal(a, b)


def test_alpha_grid_closed_form():
    a = O.alpha_grid(20)
    assert len(a) == 20 and a[0] == 0.0 and a[10] == 0.5 and a[-1] == 0.95
    assert np.all(np.diff(a) > 0) and a.max() < 1.0


def test_scales_for_alpha_special_values():
    m = np.array([4.0, 0.25, 9.0, 0.0, 1.0, 3.7])
    assert np.all(O.scales_for_alpha(m, 0.0) == 1.0)           # pow(m, 0) = 1, pow(0, 0) = 1
    s = O.scales_for_alpha(m, 0.5)
    assert s[0] == 2.0 and s[1] == 0.5 and s[2] == 3.0 and s[4] == 1.0
    assert float(s[3]) == 2.0 ** -14                            # floor for m = 0
    assert s.dtype == np.float16


def test_scales_for_alpha_rounds_pow_once():
    g = np.random.Generator(np.random.PCG64(13))
    m = g.uniform(0.01, 30, 500)
    for alpha in (0.05, 0.35, 0.95):
        s = O.scales_for_alpha(m, alpha).astype(np.float64)
        want = [exact_round_fp16(max(math.pow(float(v), alpha), 2.0 ** -14)) for v in m]
        assert np.array_equal(s, np.array(want))
    # m chosen so that m^alpha sits 2^-30 (relative) above an fp16 midpoint: only a pow
    # evaluated in double and rounded once to fp16 lands on the upper neighbour
    mids = []
    for v, _ in _FP16[15400:16800:37]:          # fp16 values around 0.5 .. 2
        nxt = _FP16_VALUES[_FP16_VALUES.index(v) + 1]
        mids.append(float((v + nxt) / 2))
    for alpha, power in ((0.5, 2), (0.25, 4)):
        m = np.array([(x * (1 + 2.0 ** -30)) ** power for x in mids])
        s = O.scales_for_alpha(m, alpha).astype(np.float64)
        want = [exact_round_fp16(math.pow(float(v), alpha)) for v in m]
        assert np.array_equal(s, np.array(want))


# ----------------------------------------------------------------------------
# group quantisation
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "handworked_groups.json")))["cases"],
                         ids=lambda c: c["name"])
def test_handworked_groups(case):
    G = case["group_size"]
    fill = case.get("fill_value", 0.0)
    w = np.full(G, fill, dtype=np.float64)
    w[:len(case["w_head"])] = case["w_head"]
    W = np.tile(w.astype(np.float16), (2, 1))
    codes, scale16, zeros = O.quantize_groups(W, None, G, case["zero_point"])
    assert float(scale16[0, 0]) == case["scale"]
    assert int(zeros[0, 0]) == case["zero"]
    head = case["codes_head"]
    assert list(codes[0, :len(head)]) == head
    if case["code_of_zero_fill"] is not None:
        assert np.all(codes[0, len(head):] == case["code_of_zero_fill"])
    else:
        assert np.all(codes[0] == head[0])


def _groups_straddling_zero(ws, G):
    N, K = ws.shape
    g = ws.reshape(N, K // G, G)
    return (g.min(axis=2) <= 0) & (g.max(axis=2) >= 0)


@pytest.mark.parametrize("G", O.GROUP_SIZES)
@pytest.mark.parametrize("zp", [True, False])
def test_error_bound_invariant(G, zp):
    W = inputs.weights(24, 1024, 0.02, seed=21 + G)
    s = O.scales_for_alpha(O.act_absmean(inputs.activations(16, 1024, seed=22)), 0.5)
    codes, scale16, zeros = O.quantize_groups(W, s, G, zp)
    ws = W.astype(np.float64) * s.astype(np.float64)[None, :]
    N, K = W.shape
    q = codes.astype(np.float64).reshape(N, K // G, G)
    sc = scale16.astype(np.float64)[:, :, None]
    deq = (q - zeros.astype(np.float64)[:, :, None]) * sc
    err = np.abs(deq - ws.reshape(N, K // G, G))
    if zp:
        ok = _groups_straddling_zero(ws, G)
        bound = sc * (0.5 + 2.0 ** -6)
        assert np.all((err <= bound)[ok])
        assert ok.mean() > 0.99
        # the scale is the group range over 15, up to one fp16 rounding
        g = ws.reshape(N, K // G, G)
        rng = g.max(axis=2) - g.min(axis=2)
        assert np.all(np.abs(scale16.astype(np.float64) * 15 - rng) <= rng * 2.0 ** -10)
    else:
        assert np.all(err <= sc * 0.5 * (1 + 2.0 ** -9))
        amax = np.abs(ws.reshape(N, K // G, G)).max(axis=2)
        assert np.all(np.abs(scale16.astype(np.float64) * 7 - amax) <= amax * 2.0 ** -10)
        assert np.all(zeros == 8)


@pytest.mark.parametrize("G", O.GROUP_SIZES)
@pytest.mark.parametrize("zp", [True, False])
def test_weights_on_the_grid_round_trip(G, zp):
    """ws = (c - z) * sigma with sigma a power of two and both extreme codes present:
    the oracle must return scale = sigma, zero = z and the codes c exactly."""
    g = np.random.Generator(np.random.PCG64(31 + G))
    N, K = 6, 4 * G
    ng = K // G
    sigma = 2.0 ** g.integers(-10, -3, size=(N, ng))
    if zp:
        z = g.integers(0, 16, size=(N, ng))
        c = g.integers(0, 16, size=(N, ng, G))
        c[:, :, 0] = 0
        c[:, :, 1] = 15
    else:
        z = np.full((N, ng), 8)
        c = g.integers(1, 16, size=(N, ng, G))          # c - 8 in [-7, 7]
        c[:, :, 0] = 1
        c[:, :, 1] = 15
    w = (c - z[:, :, None]) * sigma[:, :, None]
    W = w.reshape(N, K).astype(np.float16)
    assert np.array_equal(W.astype(np.float64), w.reshape(N, K))    # exact in fp16
    codes, scale16, zeros = O.quantize_groups(W, None, G, zp)
    assert np.array_equal(scale16.astype(np.float64), sigma)
    assert np.array_equal(zeros.astype(np.int64), z)
    assert np.array_equal(codes.reshape(N, ng, G).astype(np.int64), c)


@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("zp", [True, False])
def test_brute_force_nearest_code(G, zp):
    """K=128, N=64: each code is the nearest of the 16 grid points (q - zero) * scale,
    ties resolved half-to-even on q - zero."""
    W = inputs.weights(64, 128, 0.02, seed=41 + G)
    s = O.scales_for_alpha(O.act_absmean(inputs.activations(8, 128, seed=42)), 0.4)
    codes, scale16, zeros = O.quantize_groups(W, s, G, zp)
    ws = W.astype(np.float64) * s.astype(np.float64)[None, :]
    for n in range(64):
        for k in range(128):
            gi = k // G
            sc = float(scale16[n, gi])
            z = int(zeros[n, gi])
            d = [abs(ws[n, k] - (c - z) * sc) for c in range(16)]
            best = min(d)
            cands = [c for c in range(16) if d[c] == best]
            q = int(codes[n, k])
            if len(cands) == 1:
                # the only allowed miss: the fp32 quotient w/scale rounded across a
                # half-way point (distances then differ by < 2^-20 * scale)
                assert q == cands[0] or abs(d[q] - best) < sc * 2.0 ** -20
            else:
                assert q in cands and (q - z) % 2 == 0


def test_symmetric_mode_is_odd():
    W = inputs.weights(16, 512, 0.02, seed=51)
    for G in O.GROUP_SIZES:
        qa, sa, za = O.quantize_pack(W, None, G, False)
        qb, sb, zb = O.quantize_pack(-W, None, G, False)
        da = O.dequantize(qa, sa, za, 512, G, False)
        db = O.dequantize(qb, sb, zb, 512, G, False)
        assert np.array_equal(da, -db)
    zeros_only = np.zeros((2, 64), dtype=np.float16)
    codes, _, _ = O.quantize_groups(zeros_only, None, 32, False)
    assert np.all(codes == 8)


# ----------------------------------------------------------------------------
# packing
# ----------------------------------------------------------------------------

def test_pack_bit_positions():
    codes = np.array([[1, 2, 3, 4, 5, 6, 7, 8, 15, 0, 0, 0, 0, 0, 0, 9]], dtype=np.uint8)
    words = O.pack_nibbles(codes)
    assert words.dtype == np.uint32
    assert list(words[0]) == [0x87654321, 0x9000000F]
    ragged = O.pack_nibbles(np.array([[3, 10, 12]], dtype=np.uint8))
    assert list(ragged[0]) == [0x00000CA3]


def test_code_pack_bit_positions():
    """qweight order: code j of a word in nibble (0, 4, 1, 5, 2, 6, 3, 7)[j]."""
    codes = np.array([[1, 2, 3, 4, 5, 6, 7, 8, 15, 0, 0, 0, 0, 0, 0, 9]], dtype=np.uint8)
    words = O.pack_codes(codes)
    assert words.dtype == np.uint32
    assert list(words[0]) == [0x86427531, 0x9000000F]
    assert list(O.pack_codes(np.array([[3, 10, 12]], dtype=np.uint8))[0]) == [0x000A00C3]
    # the point of the order: one mask of a word gives an adjacent pair (k, k+1) in its halves
    c = inputs.random_codes((1, 8 * 64), seed=62)
    w = O.pack_codes(c)[0]
    for i, word in enumerate(w):
        word = int(word)
        k = 8 * i
        assert (word & 0xF, (word >> 16) & 0xF) == (c[0, k], c[0, k + 1])
        assert ((word >> 4) & 0xF, (word >> 20) & 0xF) == (c[0, k + 2], c[0, k + 3])
        assert ((word >> 8) & 0xF, (word >> 24) & 0xF) == (c[0, k + 4], c[0, k + 5])
        assert ((word >> 12) & 0xF, (word >> 28) & 0xF) == (c[0, k + 6], c[0, k + 7])


def test_pack_unpack_identity():
    for C in (8, 16, 24, 128, 4096, 3, 11):
        c = inputs.random_codes((5, C), seed=60 + C)
        assert np.array_equal(O.unpack_nibbles(O.pack_nibbles(c), C), c)
        assert np.array_equal(O.unpack_codes(O.pack_codes(c), C), c)
    words = np.random.Generator(np.random.PCG64(61)).integers(0, 2 ** 32, size=(4, 16), dtype=np.uint64).astype(np.uint32)
    assert np.array_equal(O.pack_nibbles(O.unpack_nibbles(words, 128)), words)
    assert np.array_equal(O.pack_codes(O.unpack_codes(words, 128)), words)


def test_quantize_pack_shapes():
    W = inputs.weights(8, 512, seed=62)
    for G in O.GROUP_SIZES:
        q, s, z = O.quantize_pack(W, None, G, True)
        ng = 512 // G
        assert q.shape == (8, 64) and s.shape == (8, ng) and z.shape == (8, (ng + 7) // 8)
        q2, s2, z2 = O.quantize_pack(W, None, G, False)
        assert z2 is None


# ----------------------------------------------------------------------------
# linear
# ----------------------------------------------------------------------------

def test_linear_against_naive_loop():
    K, N, M, G = 64, 5, 3, 32
    W = inputs.weights(N, K, seed=71)
    X = inputs.activations(M, K, seed=72)
    for zp in (True, False):
        q, s, z = O.quantize_pack(W, None, G, zp)
        y = O.linear(X, q, s, z, K, G, zp)
        codes = O.unpack_codes(q, K)
        zer = O.unpack_nibbles(z, K // G) if zp else np.full((N, K // G), 8)
        for m in range(M):
            for n in range(N):
                acc = Fraction(0)
                for k in range(K):
                    acc += Fraction(float(X[m, k])) * (int(codes[n, k]) - int(zer[n, k // G])) * Fraction(float(s[n, k // G]))
                assert abs(y[m, n] - float(acc)) <= 1e-12 * (abs(float(acc)) + 1)


def test_linear_on_grid_weights_is_exact():
    G, N, K = 64, 4, 256
    g = np.random.Generator(np.random.PCG64(73))
    sigma = 2.0 ** g.integers(-9, -5, size=(N, K // G))
    z = g.integers(0, 16, size=(N, K // G))
    c = g.integers(0, 16, size=(N, K // G, G))
    c[:, :, 0], c[:, :, 1] = 0, 15
    W = ((c - z[:, :, None]) * sigma[:, :, None]).reshape(N, K).astype(np.float16)
    X = inputs.activations(3, K, seed=74)
    q, s, zz = O.quantize_pack(W, None, G, True)
    y = O.linear(X, q, s, zz, K, G, True)
    assert np.array_equal(y, X.astype(np.float64) @ W.astype(np.float64).T)


def test_fold_inverse_scale():
    X = inputs.activations(4, 64, seed=75)
    ones = np.ones(64, dtype=np.float16)
    assert np.array_equal(O.fold_inverse_scale(X, ones), X)
    pow2 = (2.0 ** np.random.Generator(np.random.PCG64(76)).integers(-3, 4, 64)).astype(np.float16)
    assert np.array_equal(O.fold_inverse_scale(X, pow2).astype(np.float64),
                          X.astype(np.float64) / pow2.astype(np.float64)[None, :])
    s = inputs.uniform_fp16(64, 0.3, 7.0, seed=77)
    got = O.fold_inverse_scale(X, s).astype(np.float64)
    for j in range(0, 64, 3):
        q32 = float(np.float32(Fraction(float(X[1, j])) / Fraction(float(s[j]))))   # the fp32 quotient
        assert got[1, j] == exact_round_fp16(q32)


# ----------------------------------------------------------------------------
# scale search
# ----------------------------------------------------------------------------

def _brute_delta(W, s, G, zp):
    """Independent per-group quantiser: scale/zero from per-group Python float32 scalars,
    codes by scanning all 16 grid points."""
    N, K = W.shape
    ws = W.astype(np.float32) * s.astype(np.float32)[None, :]
    deq = np.zeros((N, K))
    for n in range(N):
        for gi in range(K // G):
            grp = ws[n, gi * G:(gi + 1) * G]
            if zp:
                sc32 = np.float32(np.float32(grp.max()) - np.float32(grp.min())) / np.float32(15)
                sc = float(np.float16(max(sc32, np.float32(1e-5))))
                z = min(max(round(float(-grp.min()) / sc), 0), 15)   # Python round() is half-even
            else:
                sc32 = np.float32(np.abs(grp).max()) / np.float32(7)
                sc = float(np.float16(max(sc32, np.float32(1e-5))))
                z = 8
            for j, v in enumerate(grp):
                d = [abs(float(v) - (c - z) * sc) for c in range(16)]
                c = min(range(16), key=lambda cc: (d[cc], (cc - z) % 2))
                deq[n, gi * G + j] = (c - z) * sc
    return deq / s.astype(np.float64)[None, :] - W.astype(np.float64)


@pytest.mark.parametrize("zp", [True, False])
def test_search_loss_against_gram_form(zp):
    """loss = trace(dW (X^T X) dW^T) / (M N) with dW from the brute-force quantiser."""
    M, K, N, G = 16, 128, 8, 32
    X = inputs.activations(M, K, seed=81)
    W = inputs.weights(N, K, seed=82)
    m = O.act_absmean(X)
    Xd = X.astype(np.float64)
    gram = Xd.T @ Xd
    for alpha in (0.0, 0.3, 0.85):
        s = O.scales_for_alpha(m, alpha)
        dW = _brute_delta(W, s, G, zp)
        want = np.trace(dW @ gram @ dW.T) / (M * N)
        got = O.search_loss(X, W, s, G, zp)
        assert abs(got - want) <= 1e-9 * want


def test_scale_search_properties():
    M, K, N = 32, 256, 16
    X = inputs.activations(M, K, seed=83)
    W = inputs.weights(N, K, seed=84)
    for zp in (True, False):
        best, alpha, s, losses = O.scale_search(X, W, 64, zp, n_grid=20)
        assert best == int(np.argmin(losses)) and alpha == best / 20
        assert losses[best] <= losses[0]
        assert np.array_equal(s, O.scales_for_alpha(O.act_absmean(X), alpha))
        # alpha = 0 is plain round-to-nearest: codes equal the unscaled quantisation
        s0 = O.scales_for_alpha(O.act_absmean(X), 0.0)
        a = O.quantize_pack(W, s0, 64, zp)
        b = O.quantize_pack(W, None, 64, zp)
        assert all(np.array_equal(x, y) for x, y in zip(a, b) if x is not None)
    # outlier channels make scaling pay off: the search should pick alpha > 0
    assert best > 0


def test_scale_search_ties_go_to_the_smaller_alpha():
    """An exact tie: with |X| = 1 everywhere, m_k = 1 and s = pow(1, alpha) = 1 for every
    alpha, so every alpha quantises the same weights the same way and all losses are the
    same number.  The search must then return the first index (alpha = 0)."""
    g = np.random.Generator(np.random.PCG64(85))
    X = np.where(g.random((8, 128)) < 0.5, -1.0, 1.0).astype(np.float16)
    W = inputs.weights(8, 128, seed=86)
    for zp in (True, False):
        best, alpha, s, losses = O.scale_search(X, W, 32, zp, n_grid=20)
        assert np.all(losses == losses[0]) and losses[0] > 0
        assert best == 0 and alpha == 0.0
        assert np.all(s.astype(np.float32) == 1.0)


# ----------------------------------------------------------------------------
# duo_scaling
# ----------------------------------------------------------------------------

def exact_round_fp16_q(q: Fraction) -> float:
    """exact_round_fp16 for an exact rational."""
    import bisect
    sign = -1 if q < 0 else 1
    a = abs(q)
    if a >= _FP16_OVERFLOW:
        return sign * math.inf
    i = bisect.bisect_left(_FP16_VALUES, a)
    if i < len(_FP16_VALUES) and _FP16_VALUES[i] == a:
        return sign * float(a)
    lo_v, lo_b = _FP16[i - 1]
    hi_v, hi_b = _FP16[i] if i < len(_FP16) else (Fraction(65536), 0x7C00)
    d_lo, d_hi = a - lo_v, hi_v - a
    if d_lo < d_hi or (d_lo == d_hi and lo_b % 2 == 0):
        return sign * float(lo_v)
    return sign * float(hi_v)


def test_weight_absmean_is_the_exact_mean():
    W = inputs.weights(37, 24, 0.3, seed=90)
    got = O.weight_absmean(W)
    for k in range(24):
        want = sum(abs(Fraction(float(v))) for v in W[:, k]) / 37
        assert got[k] == float(want)


def test_duo_scales_closed_form():
    """s = fp16(min(max(a / b, 2^-14), 65504)), a = max(m^alpha, 2^-14), b = max(w^(1-alpha),
    2^-14), against 40-digit decimal arithmetic rounded exactly to fp16 (cases within 1e-12 of
    an fp16 midpoint are skipped); includes the clamps (tiny w, zero m)."""
    from decimal import Decimal, getcontext
    getcontext().prec = 40
    g = np.random.Generator(np.random.PCG64(91))
    m = np.concatenate([g.uniform(0.05, 30.0, 40), [0.0, 3.0, 1e-7, 30.0]])
    w = np.concatenate([g.uniform(1e-3, 0.5, 40), [0.02, 1e-12, 0.01, 1e-12]])
    checked = 0
    for alpha in (0.0, 0.05, 0.35, 0.5, 0.95):
        got = O.duo_scales_for_alpha(m, w, alpha).astype(np.float64)
        lo = Decimal(2) ** -14
        for k in range(len(m)):
            al = Decimal(float(np.float64(alpha)))
            a = Decimal(float(m[k])) ** al if m[k] > 0 else (Decimal(1) if alpha == 0 else Decimal(0))
            b = Decimal(float(w[k])) ** (1 - al)
            v = min(max(max(a, lo) / max(b, lo), lo), Decimal(65504))
            q = Fraction(str(v))
            want = exact_round_fp16_q(q)
            if q != Fraction(want):             # skip values within 1e-12 of an fp16 midpoint
                nxt = np.nextafter(np.float16(want), np.float16(np.inf)).astype(np.float64)
                prv = np.nextafter(np.float16(want), np.float16(0)).astype(np.float64)
                mids = [(Fraction(want) + Fraction(float(x))) / 2 for x in (nxt, prv) if np.isfinite(x)]
                if min(abs(q - mm) for mm in mids) <= q * Fraction(1, 10 ** 12):
                    continue
            assert got[k] == want, (alpha, k, got[k], want)
            checked += 1
    assert checked > 150


def test_duo_search_with_unit_weight_statistic_is_the_plain_search():
    """With |W| = 1 everywhere the weight statistic is 1, and duo scaling reduces to the
    plain search exactly: the same s for every alpha, the same losses and index."""
    g = np.random.Generator(np.random.PCG64(92))
    W = np.where(g.random((24, 256)) < 0.5, -1.0, 1.0).astype(np.float16)
    X = inputs.activations(32, 256, seed=93)
    m = O.act_absmean(X)
    w = O.weight_absmean(W)
    assert np.all(w == 1.0)
    for a in O.alpha_grid(20):
        assert np.array_equal(O.duo_scales_for_alpha(m, w, a), O.scales_for_alpha(m, a))
    for zp in (True, False):
        d = O.scale_search_duo(X, W, 64, zp, 20)
        p = O.scale_search(X, W, 64, zp, 20)
        assert d[0] == p[0] and np.array_equal(d[2], p[2]) and np.array_equal(d[3], p[3])


def test_duo_search_properties():
    X = inputs.activations(32, 256, seed=94)
    W = inputs.weights(16, 256, seed=95)
    m, w = O.act_absmean(X), O.weight_absmean(W)
    for zp in (True, False):
        best, alpha, s, losses = O.scale_search_duo(X, W, 64, zp, 20)
        assert best == int(np.argmin(losses)) and losses[best] <= losses.min()
        assert np.array_equal(s, O.duo_scales_for_alpha(m, w, alpha))
        # every loss is the plain search's loss function at the duo s of that alpha
        for i in (0, 7, 19):
            assert losses[i] == O.search_loss(X, W, O.duo_scales_for_alpha(m, w, i / 20), 64, zp)
    # alpha = 0: s = fp16(1 / w) (the weights alone set the scale)
    s0 = O.duo_scales_for_alpha(m, w, 0.0).astype(np.float64)
    for k in range(0, 256, 17):
        assert s0[k] == exact_round_fp16_q(1 / Fraction(float(w[k])))


# ----------------------------------------------------------------------------
# apply_clip
# ----------------------------------------------------------------------------

def test_clip_ratios_closed_form():
    r = O.clip_ratios(20, 10)
    assert r.dtype == np.float32 and len(r) == 10
    for j in range(10):
        assert r[j] == np.float32(Fraction(20 - j, 20))


def test_clip_with_one_ratio_is_plain_quantisation():
    """n_clip = 1: the only ratio is 1 (clamping at the group's own max|ws|), so the
    result is awq_quantize_pack of W s, bit for bit."""
    X = inputs.activations(16, 256, seed=96)
    W = inputs.weights(12, 256, seed=97)
    s = O.scales_for_alpha(O.act_absmean(X), 0.5)
    for G in (32, 128):
        for zp in (True, False):
            idx, err, packed = O.clip_search(X, W, s, G, zp, 20, 1)
            assert np.all(idx == 0)
            ref = O.quantize_pack(W, s, G, zp)
            assert all(np.array_equal(a, b) for a, b in zip(packed, ref) if a is not None)


def test_clip_error_of_one_group_is_the_search_loss():
    """With K = G there is one group: sum_n err[n, 0, 0] / (M N) is the search loss."""
    X = inputs.activations(24, 64, seed=98)
    W = inputs.weights(10, 64, seed=99)
    s = O.scales_for_alpha(O.act_absmean(X), 0.4)
    for zp in (True, False):
        err = O.clip_errors(X, W, s, 64, zp, 20, 3)
        want = O.search_loss(X, W, s, 64, zp)
        assert abs(err[:, 0, 0].sum() / (24 * 10) - want) <= 1e-12 * want


def _brute_clip_err(X, W, s, G, zp, ratio):
    """Independent per-group clip + quantise by scanning all 16 codes, then the group's
    output error with Python sums."""
    N, K = W.shape
    ws = W.astype(np.float32) * s.astype(np.float32)[None, :]
    Xd = X.astype(np.float64)
    out = np.zeros((N, K // G))
    for n in range(N):
        for gi in range(K // G):
            grp = ws[n, gi * G:(gi + 1) * G]
            c = np.float32(np.float32(ratio) * np.float32(max(abs(float(v)) for v in grp)))
            grp = np.array([min(max(float(v), -float(c)), float(c)) for v in grp], dtype=np.float32)
            if zp:
                sc32 = np.float32(np.float32(grp.max()) - np.float32(grp.min())) / np.float32(15)
                sc = float(np.float16(max(sc32, np.float32(1e-5))))
                z = min(max(round(float(np.float32(-grp.min()) / np.float32(sc))), 0), 15)
            else:
                sc32 = np.float32(np.abs(grp).max()) / np.float32(7)
                sc = float(np.float16(max(sc32, np.float32(1e-5))))
                z = 8
            dw = []
            for j, v in enumerate(grp):
                d = [abs(float(v) - (c_ - z) * sc) for c_ in range(16)]
                c_ = min(range(16), key=lambda cc: (d[cc], (cc - z) % 2))
                k = gi * G + j
                dw.append((c_ - z) * sc / float(s[k]) - float(W[n, k]))
            e = [sum(Xd[t, gi * G + j] * dw[j] for j in range(G)) for t in range(X.shape[0])]
            out[n, gi] = sum(v * v for v in e)
    return out


@pytest.mark.parametrize("zp", [True, False])
def test_clip_errors_against_brute_force(zp):
    X = inputs.activations(6, 64, seed=100)
    W = inputs.weights(3, 64, seed=101)
    W[1, :32] = np.linspace(-0.05, 0.03, 32).astype(np.float16)
    s = O.scales_for_alpha(O.act_absmean(X), 0.3)
    err = O.clip_errors(X, W, s, 32, zp, 20, 6)
    for j in range(6):
        want = _brute_clip_err(X, W, s, 32, zp, np.float32(Fraction(20 - j, 20)))
        assert np.allclose(err[:, :, j], want, rtol=1e-9, atol=0)


def test_clip_search_properties():
    """The chosen ratio has the smallest error of its group (first one on ties: an all-zero
    group has equal errors for every ratio and keeps ratio 1), and the packed result is the
    quantisation of the group clipped at that ratio; clipping can only lower the error."""
    X = inputs.activations(32, 256, seed=102)
    W = inputs.weights(16, 256, seed=103)
    W[4] = 0
    s = O.scales_for_alpha(O.act_absmean(X), 0.5)
    for zp in (True, False):
        idx, err, packed = O.clip_search(X, W, s, 64, zp, 20, 10)
        chosen = np.take_along_axis(err, idx[:, :, None], axis=2)[:, :, 0]
        assert np.all(chosen == err.min(axis=2)) and np.all(chosen <= err[:, :, 0])
        assert np.all(idx[4] == 0)
        assert np.any(idx > 0)              # some group prefers clipping
        ref = O.quantize_pack_clipped(W, s, 64, zp, idx, 20)
        assert all(np.array_equal(a, b) for a, b in zip(packed, ref) if a is not None)
