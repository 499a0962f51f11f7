"""ctypes wrapper of the C oracle (``bitnet_ref.c``).  TEST INFRASTRUCTURE.

Every function takes and returns numpy arrays.  bf16 values enter as fp32
(widening bf16 to fp32 is exact) and leave as uint16 bit patterns.

Parity pins (what fixes each function other than itself; see tests/):

* ``absmean_gamma``   -- exact rational mean (Python integers) on small
  matrices; hand-made matrices (all zero, all +-1, power-of-two scaling).
* ``ternary`` / codes -- closed form of Q(w) at the gamma/2 boundary and at
  +-gamma, codes table, sign flip.
* ``pack`` / ``unpack`` -- hand-computed words, exhaustive round trip of all
  81 valid byte patterns at every position.
* ``quantize_act``    -- hand-made rows with exact ties (+-0.5, +-1.5,
  +-2.5 after scaling), the largest float below 0.5, all-zero rows, the
  amax position, odd symmetry, power-of-two invariance.
* ``matmul_acc``      -- brute force over all 3^8 ternary rows at K = 8 (in a
  K = 16 word), W = +1 (row sums), sign flip, the numpy add/subtract
  restatement.
* ``epilogue``        -- closed form from acc; ReLU^2 of negatives is 0.
* ``bitlinear`` end to end -- parity unpinned against an external value:
  the pages print no worked example; pinned only by the pieces above and by
  bit-for-bit agreement with the numpy restatement.
"""

from __future__ import annotations

import ctypes as C

import numpy as np

from .build import build

OK, ERR_ARG, ERR_RANGE, ERR_CODE, ERR_OVERFLOW = 0, 1, 2, 3, 4


class OracleError(RuntimeError):
    pass


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _check(st: int, what: str):
    if st != OK:
        raise OracleError(f"{what}: oracle status {st}")


class COracle:
    """One loaded build of ``bitnet_ref.c`` (the real one, or a test mutant)."""

    def __init__(self, path: str):
        L = C.CDLL(path)
        P = C.c_void_p
        i64 = C.c_int64
        sig = {
            "ref_absmean_gamma": ([P, i64, i64], C.c_float),
            "ref_ternary": ([C.c_float, C.c_float], C.c_int),
            "ref_code_of": ([C.c_int], C.c_uint),
            "ref_value_of": ([C.c_uint], C.c_int),
            "ref_pack_row": ([P, i64, P], None),
            "ref_unpack_code": ([P, i64], C.c_uint),
            "ref_quantize_weights": ([P, i64, i64, P, P], C.c_int),
            "ref_unpack_weights": ([P, i64, i64, P], C.c_int),
            "ref_quantize_act": ([P, i64, i64, P, P], C.c_int),
            "ref_matmul_acc": ([P, P, i64, i64, i64, P], C.c_int),
            "ref_epilogue": ([P, P, C.c_float, i64, i64, C.c_int, P], None),
            "ref_bf16_bits": ([C.c_float], C.c_uint16),
            "ref_to_bf16": ([P, i64, P], None),
            "ref_bitlinear": ([P, i64, i64, P, C.c_float, i64, C.c_int, P, P, P, P], C.c_int),
            "ref_rms_norm": ([P, i64, i64, P], None),
            "ref_num_threads": ([], C.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        self.L = L
        self.path = path

    def absmean_gamma(self, W) -> np.float32:
        W = _f32(W)
        N, K = W.shape
        return np.float32(self.L.ref_absmean_gamma(_p(W), N, K))

    def ternary(self, w: float, gamma: float) -> int:
        return int(self.L.ref_ternary(float(np.float32(w)), float(np.float32(gamma))))

    def code_of(self, q: int) -> int:
        return int(self.L.ref_code_of(int(q)))

    def value_of(self, code: int) -> int:
        return int(self.L.ref_value_of(int(code)))

    def pack_codes(self, codes) -> np.ndarray:
        """codes [N, K] uint8 in {0,1,2,3} -> packed [N, K/4] uint8."""
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        N, K = codes.shape
        out = np.zeros((N, K // 4), dtype=np.uint8)
        for n in range(N):
            self.L.ref_pack_row(_p(codes[n]), K, _p(out[n]))
        return out

    def unpack_codes(self, packed, K: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint8)
        N = packed.shape[0]
        out = np.zeros((N, K), dtype=np.uint8)
        for n in range(N):
            row = _p(packed[n])
            for k in range(K):
                out[n, k] = self.L.ref_unpack_code(row, k)
        return out

    def quantize_weights(self, W):
        """-> (packed [N, K/4] uint8, gamma float32)."""
        W = _f32(W)
        N, K = W.shape
        packed = np.zeros((N, K // 4), dtype=np.uint8)
        g = np.zeros(1, dtype=np.float32)
        _check(self.L.ref_quantize_weights(_p(W), N, K, _p(packed), _p(g)), "quantize_weights")
        return packed, g[0]

    def unpack_weights(self, packed, K: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint8)
        N = packed.shape[0]
        q = np.zeros((N, K), dtype=np.int8)
        _check(self.L.ref_unpack_weights(_p(packed), N, K, _p(q)), "unpack_weights")
        return q

    def quantize_act(self, X):
        """-> (xq [M, K] int8, s [M] float32)."""
        X = _f32(X)
        M, K = X.shape
        xq = np.zeros((M, K), dtype=np.int8)
        s = np.zeros(M, dtype=np.float32)
        _check(self.L.ref_quantize_act(_p(X), M, K, _p(xq), _p(s)), "quantize_act")
        return xq, s

    def matmul_acc(self, xq, packed, N: int, K: int) -> np.ndarray:
        xq = np.ascontiguousarray(xq, dtype=np.int8)
        packed = np.ascontiguousarray(packed, dtype=np.uint8)
        M = xq.shape[0]
        acc = np.zeros((M, N), dtype=np.int32)
        _check(self.L.ref_matmul_acc(_p(xq), _p(packed), M, N, K, _p(acc)), "matmul_acc")
        return acc

    def epilogue(self, acc, s, gamma, relu2: bool = False) -> np.ndarray:
        acc = np.ascontiguousarray(acc, dtype=np.int32)
        s = _f32(s)
        M, N = acc.shape
        y = np.zeros((M, N), dtype=np.float32)
        self.L.ref_epilogue(_p(acc), _p(s), float(np.float32(gamma)), M, N, int(relu2), _p(y))
        return y

    def to_bf16(self, y) -> np.ndarray:
        y = _f32(y)
        out = np.zeros(y.shape, dtype=np.uint16)
        self.L.ref_to_bf16(_p(y), y.size, _p(out))
        return out

    def bitlinear(self, X, packed, gamma, N: int, relu2: bool = False) -> dict:
        """Whole forward.  Returns xq, s, acc (int32) and y (fp32)."""
        X = _f32(X)
        packed = np.ascontiguousarray(packed, dtype=np.uint8)
        M, K = X.shape
        xq = np.zeros((M, K), dtype=np.int8)
        s = np.zeros(M, dtype=np.float32)
        acc = np.zeros((M, N), dtype=np.int32)
        y = np.zeros((M, N), dtype=np.float32)
        _check(self.L.ref_bitlinear(_p(X), M, K, _p(packed), float(np.float32(gamma)), N,
                                    int(relu2), _p(xq), _p(s), _p(acc), _p(y)), "bitlinear")
        return dict(xq=xq, s=s, acc=acc, y=y)

    def rms_norm(self, X) -> np.ndarray:
        X = _f32(X)
        M, K = X.shape
        Y = np.zeros_like(X)
        self.L.ref_rms_norm(_p(X), M, K, _p(Y))
        return Y

    def num_threads(self) -> int:
        return int(self.L.ref_num_threads())


def decode_chain(x0, layers, d: int, oracle=None) -> list:
    """A stack of decoder layers' BitLinear projections for one token, in
    bf16 between projections (TEST INFRASTRUCTURE, composed of the functions
    above only).  Per layer: q = BitLinear_qkv(x)[:, :d]; o = BitLinear_o(q);
    u = ReLU^2(BitLinear_up(o)); v = BitLinear_down(u); x <- rms_norm(v).
    (Model card of BitNet b1.58 2B4T, 模型详情 -> 架构: ReLU^2 in the FFN and a
    "subln" normalisation without a formula; the weightless RMS
    normalisation is the plain stand-in, and the first d columns of the QKV
    output stand in for attention, which is not part of the path.)

    x0: fp32 [1, K] (bf16-exact values); layers: per layer four
    (packed, gamma, N, relu2).  Returns per layer the bf16 bit patterns of
    [qkv, o, up, down, normalised] outputs."""
    R = oracle or default()
    x = np.ascontiguousarray(x0, dtype=np.float32)
    outs = []
    for proj in layers:
        bits = []
        inp = x
        for pi, (packed, gamma, N, relu2) in enumerate(proj):
            y = R.to_bf16(R.bitlinear(inp, packed, gamma, N, relu2=relu2)["y"])
            bits.append(y)
            f = (y.astype(np.uint32) << 16).view(np.float32)
            inp = f[:, :d] if pi == 0 else f
        n = R.to_bf16(R.rms_norm(inp))
        bits.append(n)
        x = (n.astype(np.uint32) << 16).view(np.float32)
        outs.append(bits)
    return outs


_default = None


def default() -> COracle:
    global _default
    if _default is None:
        _default = COracle(build())
    return _default


def __getattr__(name):
    # module-level shortcuts: ref.quantize_weights(...) etc. use the real build
    if name.startswith("_"):
        raise AttributeError(name)
    return getattr(default(), name)
