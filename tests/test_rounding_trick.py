"""The two float-to-int8 roundings the activation quantisers run on the GPU,
restated in float32 numpy (every step is one IEEE round-to-nearest-even
operation, as on the device), against round-half-away-from-zero computed
exactly in fp64.  No CUDA code is imported: this pins the arithmetic the
kernels were designed on.

  magic  (every quantiser but the bulk one): r = (v + 1.5*2^23) - 1.5*2^23 is
         v rounded to nearest even; a remainder of exactly 1/2 moves r one
         step away from zero; clamp to [-127, 127]; the integer is read from
         the low bits of r + 1.5*2^23.
  branch (the warp-per-row bulk quantiser): q is read from the bits of
         t = v + 1.5*2^23; d = v - (t - 1.5*2^23); a tie (|d| = 1/2) that went
         toward zero (q = 0, or sign(d) = sign(q)) moves q one step away.  No
         clamp: in contract |v| <= 127 * (1 + 2^-24) rounds to at most
         127.0000077.

The full range |v| <= 127.00002 (2.2e9 floats) was checked the same way off
line; here: every tie k + 1/2 with 64 floats on each side, every 97th float
up to 1/64 (dense near zero), and 4 M random bit patterns in range."""

import numpy as np

MAGIC = np.float32(12582912.0)  # 1.5 * 2^23
F32 = np.float32


def ref_round(v):
    a = np.abs(v.astype(np.float64))
    q = np.sign(v.astype(np.float64)) * np.floor(a + 0.5)
    return np.clip(q, -127, 127).astype(np.int64)


def magic(v):
    r = ((v + MAGIC).astype(F32) - MAGIC).astype(F32)
    d = (v - r).astype(F32)
    tie = np.abs(d) == F32(0.5)
    r = np.where(tie, (v + np.copysign(F32(0.5), v)).astype(F32), r).astype(F32)
    r = np.minimum(np.maximum(r, F32(-127)), F32(127))
    return (r + MAGIC).astype(F32).view(np.uint32).astype(np.int64) - 0x4B400000


def branch(v):
    t = (v + MAGIC).astype(F32)
    q = t.view(np.uint32).astype(np.int64) - 0x4B400000
    d = (v - (t - MAGIC).astype(F32)).astype(F32)
    fix = (np.abs(d) == F32(0.5)) & ((q == 0) | ((d > 0) == (q > 0)))
    return q + np.where(fix, np.where(d > 0, 1, -1), 0)


def _values():
    top = int(np.array([127.00002], dtype=F32).view(np.uint32)[0])
    # ties and their neighbourhoods, both signs
    ties = np.arange(0, 127, dtype=np.float64) + 0.5
    tb = ties.astype(F32).view(np.uint32).astype(np.int64)
    around = (tb[:, None] + np.arange(-64, 65)[None, :]).ravel()
    # every 97th float from 0 to 1/64
    small = np.arange(0, int(np.array([1 / 64], dtype=F32).view(np.uint32)[0]) + 1, 97, dtype=np.int64)
    # random bit patterns in range
    rnd = np.random.default_rng(0).integers(0, top + 1, 4_000_000, dtype=np.int64)
    bits = np.concatenate([around, small, rnd, [top]]).astype(np.uint32)
    v = bits.view(F32)
    return np.concatenate([v, -v])


def test_magic_number_rounding_matches_half_away():
    v = _values()
    assert np.array_equal(magic(v), ref_round(v))


def test_branch_light_rounding_matches_half_away():
    v = _values()
    assert np.array_equal(branch(v), ref_round(v))


def test_ties_are_exercised():
    v = _values()
    t = (v + MAGIC).astype(F32)
    d = (v - (t - MAGIC).astype(F32)).astype(F32)
    assert np.count_nonzero(np.abs(d) == F32(0.5)) >= 2 * 127


def test_in_contract_products_never_reach_127_and_a_half():
    """|x * s| for |x| <= amax and s = fl(127 / amax) stays at or below
    127.0000077, so the clamp is a no-op within the contract."""
    rng = np.random.default_rng(1)
    amax = (np.abs(rng.standard_normal(1_000_000)) *
            F32(10.0) ** rng.integers(-30, 30, 1_000_000)).astype(F32)
    amax = amax[np.isfinite(amax) & (amax > 0)]
    s = (F32(127.0) / amax).astype(F32)
    ok = np.isfinite(s)
    top = (amax[ok] * s[ok]).astype(F32)
    assert float(top.max()) <= 127.0000077
    assert np.array_equal(branch(top), np.full(top.shape, 127))
