"""Pins of the oracle: checks against what the pages and the mathematics fix.

Each ``pin_*`` takes an oracle object (the C oracle, or a build of it with a
planted mistake) and raises ``AssertionError`` when the oracle disagrees with
a value that is fixed independently of it:

* golden fixtures printed by the pages (``tests/golden``);
* closed forms worked out by hand below (exact dyadic inputs, so every fp32
  step is exact and the expected value follows from the definition alone);
* invariants (sign flip, power-of-two scaling, odd symmetry);
* brute force over every ternary row of length 8;
* the exact rational mean computed with Python integers.

Definitions followed: "Microsoft BitNet 深度研究报告" (BitNet research report),
技术原理 items 2-3 (absmean Q(w), the stored 2-bit value, add/subtract form);
the BitNet b1.58 2B4T model card, 模型详情 -> 量化 (per-token absmax int8
activations); the 2B4T technical-report write-up, GPU kernel section (four
ternaries per byte).
"""

from __future__ import annotations

import itertools
import json
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def f32(v) -> np.float32:
    return np.float32(v)


def f32_bits(u: int) -> np.float32:
    return np.array([u], dtype=np.uint32).view(np.float32)[0]


HALF_MINUS = f32_bits(0x3EFFFFFF)   # 0.5 - 2^-25, the largest float below 0.5
HALF_PLUS = f32_bits(0x3F000001)    # 0.5 + 2^-24
ONE_MINUS = f32_bits(0x3F7FFFFF)    # 1 - 2^-24


# ------------------------------------------------------------------ codes
def pin_code_table(R):
    """Stored value of each ternary weight is the page's table."""
    tab = _golden("code_table.json")["stored_value"]
    for q, code in tab.items():
        assert R.code_of(int(q)) == code, (q, code)
        assert R.value_of(code) == int(q)
    assert R.value_of(3) == -2, "code 3 is never written and must be rejected"


# Boundary matrix with sum |w| = 32 over 32 entries, so gamma = 1 exactly and
# w / gamma = w.  Expected codes follow from round(clamp(w, -1, 1)) with
# halves rounded away from zero.
_BOUNDARY = [
    (f32(0.5), 1), (f32(-0.5), 2), (HALF_MINUS, 0), (-HALF_MINUS, 0), (HALF_PLUS, 1),
    (f32(1.0), 1), (f32(-1.0), 2), (f32(1.5), 1), (f32(-1.5), 2), (f32(0.0), 0), (f32(-0.0), 0),
    (f32(0.25), 0), (f32(-0.75), 2), (f32(0.75), 1), (f32(3.0), 1), (f32(-3.0), 2),
    (f32(0.125), 0), (f32(-0.125), 0), (f32(0.625), 1), (f32(-0.625), 2), (f32(2.0), 1),
    (f32(-2.0), 2), (f32(0.375), 0), (f32(-0.375), 0), (f32(1.25), 1), (f32(-1.25), 2),
    (f32(0.5), 1), (f32(-0.5), 2), (f32(0.0), 0), (f32(0.0), 0), (f32(0.0), 0), (f32(7.0), 1),
]

# sum |w| = 12 over 16 entries: gamma = 0.75; w / 0.75 is exact for these w.
_BOUNDARY_075 = [
    (f32(0.375), 1), (f32(-0.375), 2), (f32(0.75), 1), (f32(-0.75), 2), (f32(1.5), 1),
    (f32(-1.5), 2), (f32(0.1875), 0), (f32(-0.5625), 2), (f32(0.0), 0), (f32(0.0), 0),
    (f32(2.25), 1), (f32(-2.25), 2), (f32(0.75), 1), (f32(0.75), 1), (f32(0.0), 0), (f32(0.0), 0),
]


def _codes_of(R, W):
    packed, g = R.quantize_weights(W)
    return R.unpack_codes(packed, W.shape[1]), packed, g


def pin_weight_boundaries(R):
    for table, gamma in ((_BOUNDARY, 1.0), (_BOUNDARY_075, 0.75)):
        W = np.array([[w for w, _ in table]], dtype=np.float32)
        want = np.array([[c for _, c in table]], dtype=np.uint8)
        codes, _, g = _codes_of(R, W)
        assert g == f32(gamma), (g, gamma)
        assert np.array_equal(codes, want), (codes, want)
        # power-of-two scaling: gamma scales exactly, codes unchanged
        for k in (-20, -3, 5):
            Ws = (W * f32(2.0 ** k)).astype(np.float32)
            cs, _, gs = _codes_of(R, Ws)
            assert gs == f32(gamma * 2.0 ** k), (k, gs)
            assert np.array_equal(cs, want)
        # sign flip: same gamma, codes 1 <-> 2
        cn, _, gn = _codes_of(R, -W)
        assert gn == g
        assert np.array_equal(cn, np.array([0, 2, 1], dtype=np.uint8)[want])


def pin_weight_special(R):
    K = 32
    z = np.zeros((3, K), dtype=np.float32)
    packed, g = R.quantize_weights(z)
    assert g == 0.0 and not packed.any(), "W = 0 must give gamma 0 and all-zero codes"
    packed, g = R.quantize_weights(np.ones((3, K), dtype=np.float32))
    assert g == 1.0 and np.all(packed == 0x55), "W = +1: every code 1 -> bytes 0b01010101"
    packed, g = R.quantize_weights(-np.ones((3, K), dtype=np.float32))
    assert g == 1.0 and np.all(packed == 0xAA), "W = -1: every code 2 -> bytes 0b10101010"


def _exact_mean_to_f32(W: np.ndarray) -> np.float32:
    """fp32 nearest (ties to even) to the exact rational mean of |W|."""
    tot = sum((Fraction(float(abs(v))) for v in W.ravel()), Fraction(0))
    q = tot / W.size
    c = np.float32(float(q))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    err = [abs(Fraction(float(x)) - q) for x in cands]
    best = min(err)
    winners = [x for x, e in zip(cands, err) if e == best]
    if len(winners) > 1:
        winners = [x for x in winners if int(np.array([x]).view(np.uint32)[0]) % 2 == 0]
    return np.float32(winners[0])


def pin_gamma_exact(R):
    """gamma equals the correctly rounded exact mean of |W| (Fractions)."""
    for seed, (N, K) in enumerate(((3, 16), (7, 48), (16, 64), (33, 160))):
        rng = np.random.default_rng(1000 + seed)
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        W[0, :4] = [0.0, -0.0, 1e-30, -3.5]
        assert R.absmean_gamma(W) == _exact_mean_to_f32(W), (N, K)


def pin_gamma_statistics(R):
    """Latent N(0, sigma): gamma ~ sigma*sqrt(2/pi), zeros ~ 2*Phi(0.5*sqrt(2/pi)) - 1."""
    from math import erf, pi, sqrt
    rng = np.random.default_rng(7)
    sigma = 0.02
    W = (rng.standard_normal((128, 2560)) * sigma).astype(np.float32)
    packed, g = R.quantize_weights(W)
    assert abs(g / (sigma * sqrt(2 / pi)) - 1) < 0.01
    q = R.unpack_weights(packed, W.shape[1])
    p0 = erf(0.5 * sqrt(2 / pi) / sqrt(2))  # P(|z| < 0.5*sqrt(2/pi)) = 0.3101
    assert abs((q == 0).mean() - p0) < 0.005, (q == 0).mean()
    assert abs((q == 1).mean() - (q == -1).mean()) < 0.01


# ------------------------------------------------------------------ packing
def pin_pack_words(R):
    """Hand-computed words: element 16g + 4j + i sits at bits [8i + 2j, +2)."""
    cases = [
        ({0: 1}, [0x01, 0x00, 0x00, 0x00]),
        ({1: 2}, [0x00, 0x02, 0x00, 0x00]),
        ({4: 1}, [0x04, 0x00, 0x00, 0x00]),        # i=0, j=1 -> bit 2
        ({15: 2}, [0x00, 0x00, 0x00, 0x80]),       # i=3, j=3 -> bit 30
        ({0: 1, 1: 2, 4: 2, 8: 1, 12: 2}, [0x01 | 0x08 | 0x10 | 0x80, 0x02, 0x00, 0x00]),
        ({3: 1, 7: 1, 11: 1, 15: 1}, [0x00, 0x00, 0x00, 0x55]),
    ]
    for elems, want in cases:
        codes = np.zeros((1, 32), dtype=np.uint8)
        for e, c in elems.items():
            codes[0, 16 + e] = c   # second group: also checks the group offset
        packed = R.pack_codes(codes)
        assert list(packed[0, 4:8]) == want, (elems, list(packed[0]))
        assert not packed[0, :4].any()
        assert np.array_equal(R.unpack_codes(packed, 32), codes)


def pin_pack_exhaustive(R):
    """All 81 valid byte patterns at each of the 4 byte positions round-trip."""
    valid = [b for b in range(256) if all(((b >> (2 * t)) & 3) != 3 for t in range(4))]
    assert len(valid) == 81
    for i in range(4):
        packed = np.zeros((81, 4), dtype=np.uint8)
        packed[:, i] = valid
        codes = R.unpack_codes(packed, 16)
        for r, b in enumerate(valid):
            want = np.zeros(16, dtype=np.uint8)
            for j in range(4):
                want[4 * j + i] = (b >> (2 * j)) & 3
            assert np.array_equal(codes[r], want), (i, b)
        assert np.array_equal(R.pack_codes(codes), packed)


def pin_density(R):
    d = _golden("packing_density.json")
    K = 64
    packed, _ = R.quantize_weights(np.ones((2, K), dtype=np.float32))
    assert packed.shape[1] * d["weights_per_byte"] == K
    assert abs(np.log2(3) - d["entropy_bits_per_weight"]) < 0.005


# ------------------------------------------------------------------ activations
def pin_act_ties(R):
    # amax = 127 -> s = 1 exactly, v = x: halves round away from zero.
    a = [127.0, 0.5, -0.5, 1.5, 2.5, -2.5, float(HALF_MINUS), 126.5, -126.5, -127.0,
         3.5, -0.0, 0.0, 64.5, -64.5, 100.25]
    ea = [127, 1, -1, 2, 3, -3, 0, 127, -127, -127, 4, 0, 0, 65, -65, 100]
    # amax = 254 -> s = 0.5 exactly.
    b = [254.0, 1.0, 3.0, 5.0, -5.0, -254.0, float(ONE_MINUS), 253.0, 0.0, 2.0, -1.0, -3.0,
         7.0, 9.0, -11.0, 0.5]
    eb = [127, 1, 2, 3, -3, -127, 0, 127, 0, 1, -1, -2, 4, 5, -6, 0]
    c = [0.0] * 16
    X = np.array([a, b, c], dtype=np.float32)
    xq, s = R.quantize_act(X)
    assert list(s) == [1.0, 0.5, 1.0], s
    assert list(xq[0]) == ea, xq[0]
    assert list(xq[1]) == eb, xq[1]
    assert not xq[2].any(), "all-zero row -> xq = 0 (and s = 1)"


def pin_act_amax_position(R):
    rng = np.random.default_rng(3)
    K = 48
    for pos in (0, 17, K - 1):
        for sign in (1, -1):
            x = rng.uniform(-1, 1, (1, K)).astype(np.float32)
            x[0, pos] = f32(sign * 3.0)
            xq, s = R.quantize_act(x)
            assert s[0] == f32(127.0) / f32(3.0)
            assert xq[0, pos] == sign * 127
            assert np.abs(xq).max() == 127 and np.count_nonzero(np.abs(xq) == 127) >= 1


def pin_act_symmetry_scaling(R):
    rng = np.random.default_rng(4)
    X = rng.standard_t(3, (5, 64)).astype(np.float32)
    xq, s = R.quantize_act(X)
    xn, sn = R.quantize_act(-X)
    assert np.array_equal(xn, -xq) and np.array_equal(sn, s)
    for k in (-8, 6):
        xk, sk = R.quantize_act((X * f32(2.0 ** k)).astype(np.float32))
        assert np.array_equal(xk, xq)
        assert np.array_equal(sk, (s * f32(2.0 ** -k)).astype(np.float32))


# ------------------------------------------------------------------ contraction
def pin_brute_force(R):
    """Every ternary row of length 8 (3^8 rows), placed at two position sets."""
    rng = np.random.default_rng(5)
    xq = rng.integers(-127, 128, (3, 16)).astype(np.int8)
    digits = np.array(list(itertools.product((0, 1, -1), repeat=8)), dtype=np.int8)  # [6561, 8]
    code = {0: 0, 1: 1, -1: 2}
    for positions in ((0, 1, 2, 3, 4, 5, 6, 7), (3, 15, 4, 8, 13, 1, 10, 6)):
        q = np.zeros((len(digits), 16), dtype=np.int8)
        q[:, list(positions)] = digits
        codes = np.vectorize(code.get)(q).astype(np.uint8)
        packed = R.pack_codes(codes)
        acc = R.matmul_acc(xq, packed, q.shape[0], 16)
        want = np.zeros_like(acc)
        for m in range(3):
            for d, pos in enumerate(positions):
                want[m] += xq[m, pos].astype(np.int32) * digits[:, d].astype(np.int32)
        assert np.array_equal(acc, want)


def pin_addsub(R):
    """Page's add/subtract identity, one weight at a time."""
    cases = _golden("addsub_identity.json")["cases"]
    code = {0: 0, 1: 1, -1: 2}
    xq = np.array([[37] + [0] * 15, [-91] + [0] * 15], dtype=np.int8)
    for c in cases:
        codes = np.zeros((1, 16), dtype=np.uint8)
        codes[0, 0] = code[c["w"]]
        acc = R.matmul_acc(xq, R.pack_codes(codes), 1, 16)
        assert list(acc[:, 0]) == [37 * c["delta_of_C_per_unit_A"], -91 * c["delta_of_C_per_unit_A"]]


def pin_ones_and_zero(R):
    rng = np.random.default_rng(6)
    K, N = 64, 5
    X = rng.standard_normal((4, K)).astype(np.float32)
    packed, g = R.quantize_weights(np.ones((N, K), dtype=np.float32))
    out = R.bitlinear(X, packed, g, N)
    rowsum = out["xq"].astype(np.int64).sum(axis=1)
    assert np.array_equal(out["acc"], np.repeat(rowsum[:, None], N, axis=1))
    assert np.array_equal(out["y"], (out["acc"].astype(np.float32) * (f32(1.0) / out["s"])[:, None]))
    packed, g = R.quantize_weights(np.zeros((N, K), dtype=np.float32))
    out = R.bitlinear(X, packed, g, N, relu2=True)
    assert not out["acc"].any() and not out["y"].any(), "W = 0 must give y = 0"


def pin_sign_flip(R):
    rng = np.random.default_rng(8)
    K, N = 96, 40
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    X = rng.standard_normal((3, K)).astype(np.float32)
    p, g = R.quantize_weights(W)
    pn, gn = R.quantize_weights(-W)
    a = R.bitlinear(X, p, g, N)
    b = R.bitlinear(X, pn, gn, N)
    c = R.bitlinear(-X, p, g, N)
    assert np.array_equal(b["acc"], -a["acc"]) and np.array_equal(b["y"], -a["y"])
    assert np.array_equal(c["acc"], -a["acc"]) and np.array_equal(c["y"], -a["y"])


# ------------------------------------------------------------------ epilogue
def pin_epilogue(R):
    acc = np.array([[3, -4, 0], [8, -8, 1]], dtype=np.int32)
    s = np.array([0.25, 2.0], dtype=np.float32)
    y = R.epilogue(acc, s, 0.5)           # r = gamma / s = [2, 0.25]
    assert np.array_equal(y, np.array([[6, -8, 0], [2, -2, 0.25]], dtype=np.float32)), y
    y2 = R.epilogue(acc, s, 0.5, relu2=True)
    assert np.array_equal(y2, np.array([[36, 0, 0], [4, 0, 0.0625]], dtype=np.float32)), y2


def pin_bf16(R):
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20, -1.5, 0.0,
                     -0.0, 65280.0 + 128.0], dtype=np.float32)
    want = [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xBFC0, 0x0000, 0x8000, 0x4780]
    assert [int(v) for v in R.to_bf16(vals)] == want


# ------------------------------------------------------------------ rms norm (chain glue)
def _rms_norm_exact(row):
    """x / sqrt(mean(x^2) + 1e-6) in 50-digit decimal arithmetic, with the
    stand-in's epsilon taken as the double nearest 1e-6."""
    from decimal import Decimal, getcontext
    getcontext().prec = 50
    xs = [Decimal(float(v)) for v in row]
    ms = sum(v * v for v in xs) / len(xs) + Decimal(1e-6)
    inv = 1 / ms.sqrt()
    return [float(v * inv) for v in xs]


def pin_rms_norm(R):
    """The weightless per-token RMS normalisation that stands in for the
    model card's subln (模型详情 -> 架构; no formula on the pages), against
    high-precision values, within 2 fp32 ulps: rows of 1e-3 (where the
    epsilon doubles the mean square), a lone 1 among zeros (mean over K, not
    the sum), 3 and 4, a zero row (stays zero), and a random row whose
    output mean square is 1."""
    rows = [np.full(4, 1e-3, dtype=np.float32), np.array([1, 0, 0, 0], dtype=np.float32),
            np.array([3, 4], dtype=np.float32), np.zeros(3, dtype=np.float32),
            np.random.default_rng(5).standard_normal(64).astype(np.float32)]
    for row in rows:
        got = R.rms_norm(row[None, :])[0]
        want = np.array(_rms_norm_exact(row))
        tol = 2 * np.spacing(np.abs(want).astype(np.float32)).astype(np.float64)
        assert np.all(np.abs(got.astype(np.float64) - want) <= tol), (row[:4], got[:4], want[:4])
    big = rows[-1]
    y = R.rms_norm(big[None, :])[0].astype(np.float64)
    assert abs(np.mean(y * y) - 1.0) < 1e-5


ALL_PINS = [
    pin_code_table, pin_weight_boundaries, pin_weight_special, pin_gamma_exact,
    pin_gamma_statistics, pin_pack_words, pin_pack_exhaustive, pin_density, pin_act_ties,
    pin_act_amax_position, pin_act_symmetry_scaling, pin_brute_force, pin_addsub,
    pin_ones_and_zero, pin_sign_flip, pin_epilogue, pin_bf16, pin_rms_norm,
]
