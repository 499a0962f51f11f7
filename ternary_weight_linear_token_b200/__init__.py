"""Thin Python binding of ``libbitnet158.so``, the B200 (sm_100a) C-ABI
library for the BitNet b1.58 BitLinear forward (W1.58A8).

Argument marshalling only: every function below checks the torch tensors it
is given (device, dtype, contiguity, shape), passes their device pointers and
the current CUDA stream to the C entry point of the same name, and raises
``BitnetError`` on a non-OK status.  All arithmetic runs in the library's
CUDA kernels; there is no CPU fallback.  Importing this module fails loudly
if the library has not been built (``python -m
ternary_weight_linear_token_b200.build``).
"""

from __future__ import annotations

import ctypes as C
import functools
import os

import torch

from .build import LIB as LIB_PATH

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m ternary_weight_linear_token_b200.build`"
        " (the BitLinear forward has no CPU fallback)")

lib = C.CDLL(LIB_PATH)

# ---------------------------------------------------------------- constants
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_MISALIGNED, ERR_CUDA, ERR_TIMEOUT, ERR_RANGE, \
    ERR_WORKSPACE = range(8)
F32, BF16, I8, I32 = 0, 1, 2, 3
EPI_NONE, EPI_RELU2 = 0, 1
FLAG_WEIGHTS_STATIC = 1
FLAG_WEIGHTS_EXPANDED = 2
FLAG_TABLE_LOOKUP = 4
FLAG_PREP_IN_KERNEL = 8
PATH_NONE, PATH_ROWS, PATH_MMA_TOKENS, PATH_MMA_WEIGHTS, PATH_TENSOR_CORE, PATH_GENERIC = range(6)
PATH_NAMES = {PATH_NONE: "none", PATH_ROWS: "rows", PATH_MMA_TOKENS: "mma_tokens",
              PATH_MMA_WEIGHTS: "mma_weights", PATH_TENSOR_CORE: "tensor_core",
              PATH_GENERIC: "generic"}

_DTYPE = {torch.float32: F32, torch.bfloat16: BF16, torch.int8: I8, torch.int32: I32}

_P = C.c_void_p
_I64 = C.c_int64
_SZ = C.c_size_t
_ST = C.c_int

_SIGS = {
    "bitnet_version": ([], C.c_int),
    "bitnet_status_string": ([_ST], C.c_char_p),
    "bitnet_get_device_status": ([_P], _ST),
    "bitnet_quantize_weights_workspace_size": ([_I64, _I64], _SZ),
    "bitnet_quantize_weights": ([_P, _ST, _I64, _I64, _P, _P, _P, _SZ, _P], _ST),
    "bitnet_quantize_act": ([_P, _ST, _I64, _I64, _P, _P, _P], _ST),
    "bitnet_w158a8_matmul_workspace_size": ([_I64, _I64, _I64, _ST], _SZ),
    "bitnet_w158a8_matmul_path": ([_I64, _I64, _I64, _ST], _ST),
    "bitnet_w158a8_matmul_host": ([_P, _ST, _P, _P, _P, _I64, _I64, _I64, _ST, _P, _P, _ST, _P, _SZ,
                                   C.c_uint32, _P], _ST),
    "bitnet_w158a8_matmul": ([_P, _ST, _P, _P, _P, _I64, _I64, _I64, _ST, _P, _ST, _P, _SZ,
                              C.c_uint32, _P], _ST),
    "bitnet_rms_norm": ([_P, _ST, _I64, _I64, _P, _ST, _P], _ST),
    "bitnet_rms_norm_w158a8_matmul": ([_P, _ST, _P, _P, _P, _I64, _I64, _I64, _ST, _P, _ST, _P,
                                       _SZ, C.c_uint32, _P], _ST),
    "bitnet_w158a8_matmul_noalloc": ([_P, _ST, _P, _P, _P, _I64, _I64, _I64, _ST, _P, _ST,
                                      C.c_uint32, _P], _ST),
    "bitnet_host_plan_create": ([_P, _ST, _P, _P, _P, _I64, _I64, _I64, _ST, _P, _P, _ST, _P, _SZ,
                                 C.c_uint32, _P, C.POINTER(_P)], _ST),
    "bitnet_host_plan_run": ([_P], _ST),
    "bitnet_host_plan_destroy": ([_P], None),
}


class ChainStep(C.Structure):
    """``bitnet_chain_step`` of the C header."""
    _fields_ = [("packed", C.c_void_p), ("gamma", C.c_void_p), ("N", C.c_int64),
                ("K", C.c_int64), ("flags", C.c_uint32), ("Y", C.c_void_p),
                ("X_normed", C.c_void_p)]


STEP_RELU2, STEP_NORM_IN = 1, 2
CHAIN_MAX_STEPS = 256
_SIGS["bitnet_decode_chain_workspace_size"] = ([C.POINTER(ChainStep), C.c_int], _SZ)
_SIGS["bitnet_decode_chain"] = ([C.POINTER(ChainStep), C.c_int, _P, _P, _P, _SZ, _P], _ST)

for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res


class BitnetError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib.bitnet_status_string(status).decode()} (status {status})")


def _check(status: int, what: str):
    if status != OK:
        raise BitnetError(status, what)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtypes=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the BitLinear path has no CPU fallback)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} must have dtype in {dtypes}, got {t.dtype}")


def version() -> int:
    return lib.bitnet_version()


def status_string(status: int) -> str:
    return lib.bitnet_status_string(status).decode()


def bitnet_get_device_status(stream=None) -> int:
    return lib.bitnet_get_device_status(_stream(stream))


# ---------------------------------------------------------------- weights
def bitnet_quantize_weights_workspace_size(N: int, K: int) -> int:
    return lib.bitnet_quantize_weights_workspace_size(N, K)


def bitnet_quantize_weights(W: torch.Tensor, packed: torch.Tensor | None = None,
                            gamma: torch.Tensor | None = None,
                            workspace: torch.Tensor | None = None, stream=None):
    """W [N, K] fp32/bf16 -> (packed [N, K/4] uint8, gamma [1] fp32)."""
    _dev(W, "W", (torch.float32, torch.bfloat16))
    N, K = W.shape
    if packed is None:
        packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    need = bitnet_quantize_weights_workspace_size(N, K)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=W.device)
    _dev(packed, "packed", (torch.uint8,))
    _dev(gamma, "gamma", (torch.float32,))
    st = lib.bitnet_quantize_weights(_ptr(W), _DTYPE[W.dtype], N, K, _ptr(packed), _ptr(gamma),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream))
    _check(st, "bitnet_quantize_weights")
    return packed, gamma


# ---------------------------------------------------------------- activations
def bitnet_quantize_act(X: torch.Tensor, xq: torch.Tensor | None = None,
                        s: torch.Tensor | None = None, stream=None):
    """X [M, K] fp32/bf16 -> (xq [M, K] int8, s [M] fp32)."""
    _dev(X, "X", (torch.float32, torch.bfloat16))
    M, K = X.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8, device=X.device)
    if s is None:
        s = torch.empty(M, dtype=torch.float32, device=X.device)
    _dev(xq, "xq", (torch.int8,))
    _dev(s, "s", (torch.float32,))
    st = lib.bitnet_quantize_act(_ptr(X), _DTYPE[X.dtype], M, K, _ptr(xq), _ptr(s),
                                 _stream(stream))
    _check(st, "bitnet_quantize_act")
    return xq, s


# ---------------------------------------------------------------- matmul
@functools.lru_cache(maxsize=256)
def _workspace_size(M: int, N: int, K: int, xd: int) -> int:
    return lib.bitnet_w158a8_matmul_workspace_size(M, N, K, xd)


def bitnet_w158a8_matmul_workspace_size(M: int, N: int, K: int, x_dtype) -> int:
    # a pure function of its arguments: remembered, so that a call per forward costs no
    # second trip through ctypes
    xd = _DTYPE[x_dtype] if isinstance(x_dtype, torch.dtype) else int(x_dtype)
    return _workspace_size(int(M), int(N), int(K), xd)


def bitnet_w158a8_matmul_path(M: int, N: int, K: int, x_dtype) -> int:
    """The kernel path a call of these sizes takes on the current device
    (one of the PATH_* constants)."""
    xd = _DTYPE[x_dtype] if isinstance(x_dtype, torch.dtype) else int(x_dtype)
    return lib.bitnet_w158a8_matmul_path(M, N, K, xd)


def bitnet_w158a8_matmul(X: torch.Tensor, packed: torch.Tensor, gamma: torch.Tensor,
                         s: torch.Tensor | None = None, relu2: bool = False,
                         out_dtype: torch.dtype = torch.bfloat16, Y: torch.Tensor | None = None,
                         workspace: torch.Tensor | None = None, weights_static: bool = False,
                         weights_expanded: bool = False, table_lookup: bool = False,
                         prep_in_kernel: bool = False, stream=None) -> torch.Tensor:
    """Y = BitLinear(X).  X is fp32/bf16 [M, K] (quantised inside the call) or
    int8 xq [M, K] with its scales ``s`` [M].  out_dtype fp32/bf16, or int32
    for the raw accumulators (relu2 must then be False).  ``weights_expanded``
    promises that ``workspace`` still holds the int8 weight copy of an
    earlier tensor-core-path call with the same weights and input kind;
    ``table_lookup`` runs the table-lookup comparison kernel (M <= 8);
    ``prep_in_kernel`` the tensor-core kernel that prepares its own operands."""
    _dev(X, "X", (torch.float32, torch.bfloat16, torch.int8))
    _dev(packed, "packed", (torch.uint8,))
    _dev(gamma, "gamma", (torch.float32,))
    M, K = X.shape
    N = packed.shape[0]
    if packed.shape[1] * 4 != K:
        raise ValueError(f"packed has {packed.shape[1]} bytes per row, expected K/4 = {K // 4}")
    if s is not None:
        _dev(s, "s", (torch.float32,))
    if Y is None:
        Y = torch.empty((M, N), dtype=out_dtype, device=X.device)
    _dev(Y, "Y", (torch.float32, torch.bfloat16, torch.int32))
    need = 0 if table_lookup else bitnet_w158a8_matmul_workspace_size(M, N, K, X.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.bitnet_w158a8_matmul(_ptr(X), _DTYPE[X.dtype], _ptr(s), _ptr(packed), _ptr(gamma),
                                  M, N, K, EPI_RELU2 if relu2 else EPI_NONE, _ptr(Y),
                                  _DTYPE[Y.dtype], _ptr(workspace), ws_bytes,
                                  (FLAG_WEIGHTS_STATIC if weights_static else 0)
                                  | (FLAG_WEIGHTS_EXPANDED if weights_expanded else 0)
                                  | (FLAG_TABLE_LOOKUP if table_lookup else 0)
                                  | (FLAG_PREP_IN_KERNEL if prep_in_kernel else 0),
                                  _stream(stream))
    _check(st, "bitnet_w158a8_matmul")
    return Y


def _host_call_args(X_host, packed, gamma, X_dev, Y_dev, Y_host, relu2, workspace,
                    weights_static, stream):
    """Checks the arguments of bitnet_w158a8_matmul_host and returns them as
    the C call takes them (plus the workspace tensor, kept alive by the caller)."""
    if X_host.is_cuda or Y_host.is_cuda:
        raise ValueError("X_host and Y_host must be host (CPU) tensors")
    if not (X_host.is_contiguous() and Y_host.is_contiguous()):
        raise ValueError("X_host and Y_host must be contiguous")
    _dev(X_dev, "X_dev", (X_host.dtype,))
    _dev(Y_dev, "Y_dev", (Y_host.dtype,))
    _dev(packed, "packed", (torch.uint8,))
    _dev(gamma, "gamma", (torch.float32,))
    M, K = X_host.shape
    N = packed.shape[0]
    if X_dev.shape != X_host.shape or Y_dev.shape != Y_host.shape or Y_host.shape != (M, N):
        raise ValueError("X_dev/Y_dev must match the shapes of X_host [M, K] and Y_host [M, N]")
    need = bitnet_w158a8_matmul_workspace_size(M, N, K, X_host.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=X_dev.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (_ptr(X_host), _DTYPE[X_host.dtype], _ptr(X_dev), _ptr(packed), _ptr(gamma), M, N, K,
            EPI_RELU2 if relu2 else EPI_NONE, _ptr(Y_dev), _ptr(Y_host), _DTYPE[Y_host.dtype],
            _ptr(workspace), ws_bytes, FLAG_WEIGHTS_STATIC if weights_static else 0, _stream(stream))
    return args, workspace


def bitnet_w158a8_matmul_host(X_host: torch.Tensor, packed: torch.Tensor, gamma: torch.Tensor,
                              X_dev: torch.Tensor, Y_dev: torch.Tensor, Y_host: torch.Tensor,
                              relu2: bool = False, workspace: torch.Tensor | None = None,
                              weights_static: bool = False, stream=None) -> torch.Tensor:
    """Y_host = BitLinear(X_host) in one C call: X_host (CPU, fp32/bf16, best
    pinned) is copied to X_dev, the product writes Y_dev, which is copied to
    Y_host (CPU, pinned); returns once Y_host holds the result."""
    args, _ws = _host_call_args(X_host, packed, gamma, X_dev, Y_dev, Y_host, relu2, workspace,
                                weights_static, stream)
    _check(lib.bitnet_w158a8_matmul_host(*args), "bitnet_w158a8_matmul_host")
    return Y_host


class HostMatmulPlan:
    """bitnet_w158a8_matmul_host over fixed buffers, for a projection that
    runs again and again (a decode loop): the arguments are checked once,
    here, and with page-locked X_host and Y_host the copy in, the product and
    the copy out are recorded once as a CUDA graph (bitnet_host_plan_create);
    each call then launches it and waits (bitnet_host_plan_run).  With
    pageable host buffers each call is the one bitnet_w158a8_matmul_host call.
    The caller refills X_host before a call and reads Y_host after it; the
    tensors must stay alive and in place as long as the plan is used."""

    def __init__(self, X_host: torch.Tensor, packed: torch.Tensor, gamma: torch.Tensor,
                 X_dev: torch.Tensor, Y_dev: torch.Tensor, Y_host: torch.Tensor,
                 relu2: bool = False, workspace: torch.Tensor | None = None,
                 weights_static: bool = False, stream=None):
        self._plan = None
        self._args, self._ws = _host_call_args(X_host, packed, gamma, X_dev, Y_dev, Y_host, relu2,
                                               workspace, weights_static, stream)
        self._keep = (X_host, packed, gamma, X_dev, Y_dev, Y_host)
        self.Y_host = Y_host
        self.graph = False
        if X_host.is_pinned() and Y_host.is_pinned():
            h = _P()
            st = lib.bitnet_host_plan_create(*self._args, C.byref(h))
            if st == OK:
                self._plan = h
                self.graph = True
            elif st != ERR_CUDA:  # argument errors raise; a graph that could not be
                _check(st, "bitnet_host_plan_create")  # made leaves the per-call path
        self._run = lib.bitnet_host_plan_run
        self._call = lib.bitnet_w158a8_matmul_host

    def __call__(self) -> torch.Tensor:
        st = self._run(self._plan) if self._plan is not None else self._call(*self._args)
        if st != OK:
            raise BitnetError(st, "bitnet_host_plan_run" if self._plan is not None
                              else "bitnet_w158a8_matmul_host")
        return self.Y_host

    def close(self) -> None:
        """Frees the CUDA graph (also done when the plan is collected)."""
        if self._plan is not None:
            lib.bitnet_host_plan_destroy(self._plan)
            self._plan = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def bitnet_rms_norm_w158a8_matmul(X: torch.Tensor, packed: torch.Tensor, gamma: torch.Tensor,
                                  X_normed: torch.Tensor | None = None, relu2: bool = False,
                                  out_dtype: torch.dtype = torch.bfloat16,
                                  Y: torch.Tensor | None = None,
                                  workspace: torch.Tensor | None = None,
                                  weights_static: bool = False, stream=None) -> torch.Tensor:
    """Y = BitLinear(rms_norm(X)) for fp32/bf16 X [M, K].  X_normed (same
    dtype and shape as X) receives the normalised input; it may be omitted
    for M <= 8 and is allocated here otherwise."""
    _dev(X, "X", (torch.float32, torch.bfloat16))
    _dev(packed, "packed", (torch.uint8,))
    _dev(gamma, "gamma", (torch.float32,))
    M, K = X.shape
    N = packed.shape[0]
    if packed.shape[1] * 4 != K:
        raise ValueError(f"packed has {packed.shape[1]} bytes per row, expected K/4 = {K // 4}")
    if X_normed is None and M > 8:
        X_normed = torch.empty_like(X)
    if X_normed is not None:
        _dev(X_normed, "X_normed", (X.dtype,))
    if Y is None:
        Y = torch.empty((M, N), dtype=out_dtype, device=X.device)
    _dev(Y, "Y", (torch.float32, torch.bfloat16, torch.int32))
    need = bitnet_w158a8_matmul_workspace_size(M, N, K, X.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.bitnet_rms_norm_w158a8_matmul(_ptr(X), _DTYPE[X.dtype], _ptr(X_normed), _ptr(packed),
                                           _ptr(gamma), M, N, K,
                                           EPI_RELU2 if relu2 else EPI_NONE, _ptr(Y),
                                           _DTYPE[Y.dtype], _ptr(workspace), ws_bytes,
                                           FLAG_WEIGHTS_STATIC if weights_static else 0,
                                           _stream(stream))
    _check(st, "bitnet_rms_norm_w158a8_matmul")
    return Y


STATIC_SCRATCH_BYTES = 32 << 20


def bitnet_w158a8_matmul_noalloc(X: torch.Tensor, packed: torch.Tensor, gamma: torch.Tensor,
                                 s: torch.Tensor | None = None, relu2: bool = False,
                                 out_dtype: torch.dtype = torch.bfloat16,
                                 Y: torch.Tensor | None = None, weights_static: bool = False,
                                 stream=None) -> torch.Tensor:
    """bitnet_w158a8_matmul with the library's built-in scratch array instead
    of a workspace, for callers that cannot allocate device memory (the output
    Y is still the caller's)."""
    _dev(X, "X", (torch.float32, torch.bfloat16, torch.int8))
    _dev(packed, "packed", (torch.uint8,))
    _dev(gamma, "gamma", (torch.float32,))
    M, K = X.shape
    N = packed.shape[0]
    if packed.shape[1] * 4 != K:
        raise ValueError(f"packed has {packed.shape[1]} bytes per row, expected K/4 = {K // 4}")
    if s is not None:
        _dev(s, "s", (torch.float32,))
    if Y is None:
        Y = torch.empty((M, N), dtype=out_dtype, device=X.device)
    _dev(Y, "Y", (torch.float32, torch.bfloat16, torch.int32))
    st = lib.bitnet_w158a8_matmul_noalloc(_ptr(X), _DTYPE[X.dtype], _ptr(s), _ptr(packed),
                                          _ptr(gamma), M, N, K, EPI_RELU2 if relu2 else EPI_NONE,
                                          _ptr(Y), _DTYPE[Y.dtype],
                                          FLAG_WEIGHTS_STATIC if weights_static else 0,
                                          _stream(stream))
    _check(st, "bitnet_w158a8_matmul_noalloc")
    return Y


# ---------------------------------------------------------------- glue
def bitnet_rms_norm(X: torch.Tensor, Y: torch.Tensor | None = None,
                    out_dtype: torch.dtype | None = None, stream=None) -> torch.Tensor:
    """Weightless per-token RMS normalisation (decode-chain glue)."""
    _dev(X, "X", (torch.float32, torch.bfloat16))
    M, K = X.shape
    if Y is None:
        Y = torch.empty((M, K), dtype=out_dtype or X.dtype, device=X.device)
    _dev(Y, "Y", (torch.float32, torch.bfloat16))
    st = lib.bitnet_rms_norm(_ptr(X), _DTYPE[X.dtype], M, K, _ptr(Y), _DTYPE[Y.dtype],
                             _stream(stream))
    _check(st, "bitnet_rms_norm")
    return Y


# ---------------------------------------------------------------- decode chain
def bitnet_decode_chain_steps(steps) -> C.Array:
    """Descriptor array for ``bitnet_decode_chain``: one dict per step with
    ``packed`` [N, K/4] uint8, ``gamma`` [1] fp32, ``Y`` bf16 with N elements
    and optionally ``relu2``, ``norm_in`` and ``X_normed`` (bf16, K elements).
    The tensors must outlive every call that uses the array."""
    arr = (ChainStep * len(steps))()
    for i, d in enumerate(steps):
        packed, gamma, Y = d["packed"], d["gamma"], d["Y"]
        _dev(packed, f"steps[{i}].packed", (torch.uint8,))
        _dev(gamma, f"steps[{i}].gamma", (torch.float32,))
        _dev(Y, f"steps[{i}].Y", (torch.bfloat16,))
        N, K = packed.shape[0], packed.shape[1] * 4
        if Y.numel() != N:
            raise ValueError(f"steps[{i}].Y has {Y.numel()} elements, expected N = {N}")
        xn = d.get("X_normed")
        if xn is not None:
            _dev(xn, f"steps[{i}].X_normed", (torch.bfloat16,))
            if xn.numel() != K:
                raise ValueError(f"steps[{i}].X_normed has {xn.numel()} elements, expected K = {K}")
        flags = (STEP_RELU2 if d.get("relu2") else 0) | (STEP_NORM_IN if d.get("norm_in") else 0)
        arr[i] = ChainStep(packed.data_ptr(), gamma.data_ptr(), N, K, flags, Y.data_ptr(),
                           None if xn is None else xn.data_ptr())
    return arr


def bitnet_decode_chain_workspace_size(steps) -> int:
    arr = steps if isinstance(steps, C.Array) else bitnet_decode_chain_steps(steps)
    return lib.bitnet_decode_chain_workspace_size(arr, len(arr))


def bitnet_decode_chain(steps, x0: torch.Tensor, workspace: torch.Tensor,
                        y_norm: torch.Tensor | None = None, stream=None) -> None:
    """Runs a chain of M = 1 BitLinear projections in one launch.  ``steps``
    is a list of step dicts (see ``bitnet_decode_chain_steps``) or a prebuilt
    descriptor array; x0 is the bf16 input of the first step; ``workspace``
    is a uint8 tensor of ``bitnet_decode_chain_workspace_size`` bytes,
    zero-filled once and then kept for every call of this chain; y_norm
    (optional, bf16) receives the RMS normalisation of the last output."""
    arr = steps if isinstance(steps, C.Array) else bitnet_decode_chain_steps(steps)
    _dev(x0, "x0", (torch.bfloat16,))
    _dev(workspace, "workspace", (torch.uint8,))
    if x0.numel() != arr[0].K:
        raise ValueError(f"x0 has {x0.numel()} elements, expected K = {arr[0].K}")
    if y_norm is not None:
        _dev(y_norm, "y_norm", (torch.bfloat16,))
        if y_norm.numel() != arr[len(arr) - 1].N:
            raise ValueError("y_norm must have the last step's N elements")
    st = lib.bitnet_decode_chain(arr, len(arr), _ptr(x0), _ptr(y_norm), _ptr(workspace),
                                 workspace.numel(), _stream(stream))
    _check(st, "bitnet_decode_chain")
