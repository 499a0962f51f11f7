"""Numpy restatement of the BitLinear forward.  TEST INFRASTRUCTURE.

Written independently of ``bitnet_ref.c`` to cross-check it: it reaches the
same numbers by other routes.

* gamma: ``np.cumsum`` (a sequential running sum) over |W| in fp64, row by
  row and then over the row sums, mean taken in fp64, rounded once to fp32.
  ("Microsoft BitNet 深度研究报告", technical principles, item 2.)
* ternary values: numpy fp32 division and clipping, rounding half away from
  zero as sign(t) * floor(|t| + 0.5) evaluated in fp64 (exact for |t| <= 1).
* codes and packing: the 2-bit value table of the same item; the word layout
  is built with vectorised shifts over all 16 positions at once.
* activations: per-token absmax in fp32, s = float32(127) / amax, v = x * s
  in fp32, rounded half away in fp64 and clipped to [-127, 127].  (Model card
  of BitNet b1.58 2B4T, "模型详情", quantisation bullets.)
* contraction: the add/subtract identity of item 3 of the research report:
  acc = sum over w=+1 of xq  -  sum over w=-1 of xq, as two int64 matrix
  products with 0/1 masks.
* epilogue: r = float32(gamma) / s in fp32, y = float32(acc) * r in fp32;
  ReLU^2; bf16 by round-to-nearest-even on the bit pattern.
"""

from __future__ import annotations

import numpy as np


def absmean_gamma(W: np.ndarray) -> np.float32:
    a = np.abs(np.asarray(W, dtype=np.float32).astype(np.float64))
    row = np.cumsum(a, axis=1)[:, -1]
    total = np.cumsum(row)[-1]
    return np.float32(total / np.float64(a.size))


def _round_half_away(t: np.ndarray) -> np.ndarray:
    t = t.astype(np.float64)
    return np.sign(t) * np.floor(np.abs(t) + 0.5)


def ternary_values(W: np.ndarray, gamma: np.float32) -> np.ndarray:
    W = np.asarray(W, dtype=np.float32)
    if gamma == np.float32(0):
        return np.zeros(W.shape, dtype=np.int8)
    t = np.clip(W / np.float32(gamma), np.float32(-1), np.float32(1)).astype(np.float32)
    return _round_half_away(t).astype(np.int8)


_CODE = np.array([2, 0, 1], dtype=np.uint32)  # value -1, 0, +1 -> stored 2, 0, 1


def pack(q: np.ndarray) -> np.ndarray:
    """Ternary values [N, K] (K % 16 == 0) -> packed bytes [N, K/4]."""
    q = np.asarray(q, dtype=np.int64)
    N, K = q.shape
    codes = _CODE[q + 1].reshape(N, K // 16, 4, 4)  # [..., j, i]: element 4j + i
    i = np.arange(4, dtype=np.uint32)[None, None, None, :]
    j = np.arange(4, dtype=np.uint32)[None, None, :, None]
    words = np.bitwise_or.reduce((codes << (8 * i + 2 * j)).reshape(N, K // 16, 16), axis=2)
    return words.astype("<u4").view(np.uint8).reshape(N, K // 4)


def unpack(packed: np.ndarray, K: int) -> np.ndarray:
    """Packed bytes [N, K/4] -> ternary values [N, K]; raises on a code 3."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    words = packed.view("<u4").reshape(N, K // 16, 1, 1).astype(np.uint32)
    i = np.arange(4, dtype=np.uint32)[None, None, None, :]
    j = np.arange(4, dtype=np.uint32)[None, None, :, None]
    codes = ((words >> (8 * i + 2 * j)) & np.uint32(3)).reshape(N, K)
    if (codes == 3).any():
        raise ValueError("code 3 in packed weights")
    lut = np.array([0, 1, -1], dtype=np.int8)
    return lut[codes]


def quantize_weights(W: np.ndarray):
    g = absmean_gamma(W)
    return pack(ternary_values(W, g)), g


def quantize_act(X: np.ndarray):
    X = np.asarray(X, dtype=np.float32)
    amax = np.max(np.abs(X), axis=1)
    zero = amax == np.float32(0)
    s = np.where(zero, np.float32(1), np.float32(127) / np.where(zero, np.float32(1), amax))
    s = s.astype(np.float32)
    v = (X * s[:, None]).astype(np.float32)
    xq = np.clip(_round_half_away(v), -127, 127).astype(np.int8)
    xq[zero] = 0
    return xq, s


def matmul_acc(xq: np.ndarray, packed: np.ndarray, K: int) -> np.ndarray:
    q = unpack(packed, K)
    x = np.asarray(xq, dtype=np.int64)
    plus = (q == 1).astype(np.int64)
    minus = (q == -1).astype(np.int64)
    acc = x @ plus.T - x @ minus.T
    assert np.all(np.abs(acc) < 2**31)
    return acc.astype(np.int32)


def epilogue(acc: np.ndarray, s: np.ndarray, gamma, relu2: bool = False) -> np.ndarray:
    r = (np.float32(gamma) / np.asarray(s, dtype=np.float32)).astype(np.float32)
    y = (np.asarray(acc).astype(np.float32) * r[:, None]).astype(np.float32)
    if relu2:
        y = np.where(y > np.float32(0), y, np.float32(0)).astype(np.float32)
        y = (y * y).astype(np.float32)
    return y


def to_bf16(y: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(y, dtype=np.float32).view(np.uint32).astype(np.uint64)
    out = ((u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16))
    return out.astype(np.uint16)


def bitlinear(X, packed, gamma, K: int, relu2: bool = False) -> dict:
    xq, s = quantize_act(X)
    acc = matmul_acc(xq, packed, K)
    return dict(xq=xq, s=s, acc=acc, y=epilogue(acc, s, gamma, relu2))
