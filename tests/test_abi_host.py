"""The C-ABI library on the host, without a GPU: it loads, exports every
function that include/bitnet158.h declares, and rejects bad arguments with the
documented status before it would touch the device."""

import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitnet158.h")


@pytest.fixture(scope="module")
def tw():
    from __graft_entry__ import load_builder
    load_builder().build()
    import ternary_weight_linear_token_b200 as tw
    return tw


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(bitnet_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("bitnet_quantize_weights", "bitnet_quantize_act", "bitnet_w158a8_matmul",
                 "bitnet_status_string", "bitnet_get_device_status"):
        assert must in names


def test_every_declared_symbol_is_exported(tw):
    for name in declared_functions():
        assert hasattr(tw.lib, name), name


def test_status_strings_and_version(tw):
    for st in range(8):
        assert isinstance(tw.status_string(st), str) and tw.status_string(st)
    assert tw.status_string(99) == "unknown status"
    m = re.search(r"#define BITNET_VERSION (\d+)", open(HEADER).read())
    assert m and tw.version() == int(m.group(1)) == 10100  # the library is the header's


# Fake, suitably aligned device addresses: the calls below must be rejected by
# the host checks and never dereference them.
A = C.c_void_p(0x10000000)
B = C.c_void_p(0x20000000)
Cc = C.c_void_p(0x30000000)
G = C.c_void_p(0x40000000)
WS = C.c_void_p(0x50000000)
MIS = C.c_void_p(0x20000004)


def mm(tw, X=A, xd=1, s=None, P=B, g=G, M=4, N=8, K=64, epi=0, Y=Cc, yd=1, ws=None, wsb=0,
       flags=0):
    return tw.lib.bitnet_w158a8_matmul(X, xd, s, P, g, M, N, K, epi, Y, yd, ws, wsb, flags, None)


def test_matmul_rejects_bad_arguments(tw):
    assert mm(tw, X=None) == tw.ERR_INVALID_ARG
    assert mm(tw, P=None) == tw.ERR_INVALID_ARG
    assert mm(tw, g=None) == tw.ERR_INVALID_ARG
    assert mm(tw, Y=None) == tw.ERR_INVALID_ARG
    assert mm(tw, xd=3) == tw.ERR_INVALID_ARG            # int32 activations
    assert mm(tw, yd=2) == tw.ERR_INVALID_ARG            # int8 output
    assert mm(tw, epi=2) == tw.ERR_INVALID_ARG
    assert mm(tw, yd=3, epi=1) == tw.ERR_INVALID_ARG     # raw int32 with ReLU^2
    assert mm(tw, flags=16) == tw.ERR_INVALID_ARG        # unknown flag bit
    assert mm(tw, M=-1) == tw.ERR_INVALID_ARG
    assert mm(tw, K=0) == tw.ERR_INVALID_ARG
    assert mm(tw, K=40) == tw.ERR_UNSUPPORTED_SHAPE      # not a multiple of 16
    assert mm(tw, K=(1 << 24) + 16) == tw.ERR_UNSUPPORTED_SHAPE
    assert mm(tw, xd=2) == tw.ERR_INVALID_ARG            # int8 input needs s
    assert mm(tw, s=G) == tw.ERR_INVALID_ARG             # float input takes no s
    assert mm(tw, X=MIS) == tw.ERR_MISALIGNED
    assert mm(tw, Y=C.c_void_p(0x30000008)) == tw.ERR_MISALIGNED
    assert mm(tw, g=C.c_void_p(0x40000002)) == tw.ERR_MISALIGNED
    # Y overlapping X
    assert mm(tw, Y=C.c_void_p(0x10000010)) == tw.ERR_INVALID_ARG
    # prefill-sized float input needs the quantisation workspace
    assert mm(tw, M=4096, N=6912, K=2560) == tw.ERR_WORKSPACE
    need = tw.lib.bitnet_w158a8_matmul_workspace_size(4096, 6912, 2560, tw.BF16)
    assert mm(tw, M=4096, N=6912, K=2560, ws=WS, wsb=need - 1) == tw.ERR_WORKSPACE
    assert mm(tw, M=4096, N=6912, K=2560, ws=C.c_void_p(0x50000010), wsb=need) == tw.ERR_MISALIGNED
    # empty calls succeed without touching the device
    assert mm(tw, M=0) == tw.OK
    assert mm(tw, N=0) == tw.OK


def test_workspace_sizes(tw):
    f = tw.lib.bitnet_w158a8_matmul_workspace_size
    assert f(1, 2560, 2560, tw.BF16) == 0          # decode, M <= 3: fused, no scratch
    assert f(3, 6912, 2560, tw.F32) == 0
    assert f(4, 6912, 2560, tw.F32) == 4 * 2560 + 256      # M >= 4: quantised once
    assert f(8, 6912, 2560, tw.F32) == 8 * 2560 + 256
    assert f(8, 6912, 2560, tw.I8) == 0                   # xq given
    assert f(32, 2560, 6912, tw.BF16) == 32 * 6912 + 256
    assert f(16, 2560, 6912, tw.I8) == 0            # xq given, mma.sync path
    # tensor-core path: xq and s (float input only), then the int8 weights,
    # then 32 bytes of readiness counter per 128 tokens and per 256 features
    ready = (4096 // 128 + (6912 + 255) // 256) * 32   # 1888 -> 2048
    assert f(4096, 6912, 2560, tw.I8) == 6912 * 2560 + 2048
    assert f(4096, 6912, 2560, tw.BF16) == 4096 * 2560 + 4096 * 4 + 6912 * 2560 + 2048
    assert ready <= 2048
    assert f(33, 7, 64, tw.F32) == 2304 + 256 + 512 + 256  # each part rounded up to 256
    assert f(40, 33, 80, tw.I8) == 0                # K % 64 != 0: generic kernel
    assert f(5, 64, 48, tw.F32) == 0                # M <= 8 and K % 64 != 0: fused kernel
    assert f(9, 64, 48, tw.F32) == 512 + 256        # generic path (M > 8, K % 64 != 0)
    assert tw.lib.bitnet_quantize_weights_workspace_size(2560, 2560) == 2560 * 8
    assert tw.lib.bitnet_quantize_weights_workspace_size(3, 16) == 256


def test_quantizers_reject_bad_arguments(tw):
    q = tw.lib.bitnet_quantize_weights
    assert q(None, 0, 4, 64, B, G, WS, 256, None) == tw.ERR_INVALID_ARG
    assert q(A, 2, 4, 64, B, G, WS, 256, None) == tw.ERR_INVALID_ARG      # int8 weights
    assert q(A, 0, 0, 64, B, G, WS, 256, None) == tw.ERR_INVALID_ARG      # empty matrix
    assert q(A, 0, 4, 24, B, G, WS, 256, None) == tw.ERR_UNSUPPORTED_SHAPE
    assert q(A, 0, 4, 64, B, G, None, 0, None) == tw.ERR_WORKSPACE
    assert q(MIS, 0, 4, 64, B, G, WS, 256, None) == tw.ERR_MISALIGNED
    a = tw.lib.bitnet_quantize_act
    assert a(A, 0, 4, 64, None, G, None) == tw.ERR_INVALID_ARG
    assert a(A, 3, 4, 64, B, G, None) == tw.ERR_INVALID_ARG
    assert a(A, 0, 4, 20, B, G, None) == tw.ERR_UNSUPPORTED_SHAPE
    assert a(A, 0, 4, 64, MIS, G, None) == tw.ERR_MISALIGNED
    assert a(A, 0, 0, 64, B, G, None) == tw.OK
    r = tw.lib.bitnet_rms_norm
    assert r(A, 1, 4, 64, A, 0, None) == tw.ERR_INVALID_ARG             # in place, dtype change
    assert r(A, 1, 4, 64, C.c_void_p(0x10000010), 1, None) == tw.ERR_INVALID_ARG
    assert r(A, 1, 0, 64, B, 1, None) == tw.OK


def chain(tw, shapes, flags=None, xn=None):
    """Descriptor array with fake aligned device addresses."""
    arr = (tw.ChainStep * len(shapes))()
    for i, (N, K) in enumerate(shapes):
        f = 0 if flags is None else flags[i]
        x = None if xn is None else xn[i]
        arr[i] = tw.ChainStep(0x20000000 + (i << 20), 0x40000000 + 256 * i, N, K, f,
                              0x60000000 + (i << 20), x)
    return arr


def dc(tw, arr, n=None, x0=A, y=None, ws=WS, wsb=1 << 20):
    return tw.lib.bitnet_decode_chain(arr, len(arr) if n is None else n, x0, y, ws, wsb, None)


def test_decode_chain_rejects_bad_arguments(tw):
    ok = chain(tw, [(3840, 2560), (2560, 2560), (6912, 2560), (2560, 6912)])
    assert dc(tw, ok, n=0) == tw.ERR_INVALID_ARG
    assert dc(tw, ok, n=257) == tw.ERR_INVALID_ARG
    assert dc(tw, ok, x0=None) == tw.ERR_INVALID_ARG
    assert dc(tw, ok, x0=MIS) == tw.ERR_MISALIGNED
    assert dc(tw, chain(tw, [(64, 96)])) == tw.ERR_UNSUPPORTED_SHAPE       # K % 64
    assert dc(tw, chain(tw, [(64, 8256)])) == tw.ERR_UNSUPPORTED_SHAPE     # K > 8192
    assert dc(tw, chain(tw, [(100, 64), (64, 128)])) == tw.ERR_INVALID_ARG  # K > previous N
    assert dc(tw, chain(tw, [(0, 64)])) == tw.ERR_INVALID_ARG
    assert dc(tw, chain(tw, [(64, 64)], flags=[4])) == tw.ERR_INVALID_ARG
    # X_normed without the normalisation flag
    assert dc(tw, chain(tw, [(64, 64)], xn=[0x70000000])) == tw.ERR_INVALID_ARG
    assert dc(tw, chain(tw, [(64, 64)], flags=[2], xn=[0x70000008])) == tw.ERR_MISALIGNED
    # y_norm needs N % 16 == 0
    assert dc(tw, chain(tw, [(100, 64)]), y=C.c_void_p(0x70000000)) == tw.ERR_UNSUPPORTED_SHAPE
    # an output overlapping the chain input
    assert dc(tw, chain(tw, [(64, 64)]), x0=C.c_void_p(0x60000000)) == tw.ERR_INVALID_ARG
    need = tw.lib.bitnet_decode_chain_workspace_size(ok, 4)
    assert dc(tw, ok, wsb=need - 1) == tw.ERR_WORKSPACE
    assert dc(tw, ok, ws=None) == tw.ERR_WORKSPACE
    assert dc(tw, ok, ws=C.c_void_p(0x50000008), wsb=need) == tw.ERR_MISALIGNED


def test_decode_chain_workspace_size(tw):
    f = tw.lib.bitnet_decode_chain_workspace_size
    layer = [(3840, 2560), (2560, 2560), (6912, 2560), (2560, 6912)]
    # 256-byte header (the launch and done counters); then, for every step
    # but the last, one 4-byte tagged word per value the next step reads
    assert f(chain(tw, layer), 4) == 256 + 4 * (2560 + 2560 + 6912)
    assert f(chain(tw, [(333, 64)]), 1) == 256
    assert f(chain(tw, [(333, 64), (64, 320)]), 2) == 256 + 4 * 320
    assert f(chain(tw, [(64, 40)]), 1) == 0          # invalid descriptors
    assert f(chain(tw, layer * 30), 120) == 256 + 4 * (30 * (2560 + 2560 + 6912 + 2560) - 2560)


def test_rms_norm_matmul_rejects_bad_arguments(tw):
    f = tw.lib.bitnet_rms_norm_w158a8_matmul

    def call(X=A, xd=1, Xn=None, P=B, g=G, M=4, N=8, K=64, epi=0, Y=Cc, yd=1, ws=None, wsb=0,
             flags=0):
        return f(X, xd, Xn, P, g, M, N, K, epi, Y, yd, ws, wsb, flags, None)

    assert call(xd=2) == tw.ERR_INVALID_ARG                       # int8 input
    assert call(yd=2) == tw.ERR_INVALID_ARG
    assert call(K=40) == tw.ERR_UNSUPPORTED_SHAPE
    assert call(M=9, ws=WS, wsb=1 << 20) == tw.ERR_INVALID_ARG    # M > 8 needs X_normed
    assert call(Xn=MIS) == tw.ERR_MISALIGNED
    assert call(Xn=C.c_void_p(0x10000000)) == tw.ERR_INVALID_ARG  # X_normed overlapping X
    assert call(Xn=C.c_void_p(0x30000000)) == tw.ERR_INVALID_ARG  # X_normed overlapping Y
    assert call(M=0) == tw.OK


def test_table_lookup_flag_checks(tw):
    """The table-lookup comparison kernel takes 1..8 tokens and no workspace;
    larger M is an unsupported shape, and the normalising variant refuses
    the flag.  All decided before any device access."""
    assert mm(tw, M=9, K=64, flags=4) == tw.ERR_UNSUPPORTED_SHAPE
    assert mm(tw, M=1, N=8, K=1 << 20, flags=4) == tw.ERR_UNSUPPORTED_SHAPE  # tables too big
    assert mm(tw, M=0, flags=4) == tw.OK
    f = tw.lib.bitnet_rms_norm_w158a8_matmul
    assert f(A, 1, None, B, G, 4, 8, 64, 0, Cc, 1, None, 0, 4, None) == tw.ERR_INVALID_ARG


def test_matmul_path_query(tw):
    """Which kernel path a call takes: host logic for every path; the
    tensor-core path also needs the driver's tensor-map encoder, which this
    GPU-less host lacks, so calls of that shape report the dp4a fallback
    instead of running it silently."""
    f = tw.lib.bitnet_w158a8_matmul_path
    assert f(1, 2560, 2560, tw.BF16) == tw.PATH_ROWS
    assert f(3, 6912, 2560, tw.F32) == tw.PATH_ROWS
    assert f(8, 2560, 2560, tw.BF16) == tw.PATH_MMA_TOKENS
    assert f(32, 2560, 6912, tw.BF16) == tw.PATH_MMA_TOKENS
    assert f(16, 2560, 2560, tw.I8) == tw.PATH_MMA_WEIGHTS
    assert f(8, 2560, 2560, tw.I8) == tw.PATH_ROWS        # caller's int8, up to 8 tokens
    assert f(5, 64, 48, tw.F32) == tw.PATH_ROWS           # K % 64 != 0, M <= 8
    assert f(9, 64, 48, tw.F32) == tw.PATH_GENERIC        # K % 64 != 0, M > 8
    assert f(0, 64, 64, tw.F32) == tw.PATH_NONE
    assert f(4, 64, 40, tw.F32) == tw.PATH_NONE
    assert f(4, 64, 64, 3) == tw.PATH_NONE                # int32 activations
    import torch
    want = tw.PATH_TENSOR_CORE if torch.cuda.is_available() else tw.PATH_GENERIC
    assert f(4096, 6912, 2560, tw.BF16) == want
    assert f(4096, 6912, 2560, tw.I8) == want


def test_noalloc_checks_arguments_before_its_size_limit(tw):
    """A bad dtype, flag or size is an invalid argument, even where the call
    would also need more than the built-in scratch array; the size limit is
    checked next; nothing reaches the device."""
    f = tw.lib.bitnet_w158a8_matmul_noalloc

    def call(X=A, xd=1, s=None, M=4096, N=6912, K=2560, epi=0, Y=Cc, yd=1, flags=0):
        return f(X, xd, s, B, G, M, N, K, epi, Y, yd, flags, None)

    assert call(xd=3) == tw.ERR_INVALID_ARG
    assert call(xd=7) == tw.ERR_INVALID_ARG
    assert call(yd=2) == tw.ERR_INVALID_ARG
    assert call(flags=16) == tw.ERR_INVALID_ARG
    assert call(M=1 << 40) == tw.ERR_INVALID_ARG
    assert call(K=40) == tw.ERR_UNSUPPORTED_SHAPE
    assert call(X=MIS) == tw.ERR_MISALIGNED
    assert call(M=8192) == tw.ERR_WORKSPACE               # (8192 + 6912) * 2560 > 32 MiB
    assert call(M=0) == tw.OK


def test_host_entry_point_checks(tw):
    """The host-to-host entry point: the matmul's checks on the device
    buffers, host pointers required, no int8 input; all before any CUDA call."""
    f = tw.lib.bitnet_w158a8_matmul_host
    H = C.c_void_p(0x7000000)

    def call(Xh=H, xd=1, Xd=A, M=1, N=8, K=64, Yd=Cc, Yh=H, yd=1, flags=0):
        return f(Xh, xd, Xd, B, G, M, N, K, 0, Yd, Yh, yd, None, 0, flags, None)

    assert call(Xh=None) == tw.ERR_INVALID_ARG
    assert call(Yh=None) == tw.ERR_INVALID_ARG
    assert call(xd=2) == tw.ERR_INVALID_ARG      # int8 input: its scales would need a copy
    assert call(Xd=MIS) == tw.ERR_MISALIGNED
    assert call(K=40) == tw.ERR_UNSUPPORTED_SHAPE
    assert call(flags=16) == tw.ERR_INVALID_ARG
    assert call(M=4096, N=6912, K=2560) == tw.ERR_WORKSPACE
    assert call(M=0) == tw.OK


def test_host_plan_checks(tw):
    """A plan takes the host entry point's checks, all before any CUDA call,
    and refuses a null plan pointer and an empty call; running or freeing a
    null plan is safe."""
    f = tw.lib.bitnet_host_plan_create
    H = C.c_void_p(0x7000000)

    def create(Xh=H, xd=1, Xd=A, M=1, N=8, K=64, Yd=Cc, Yh=H, flags=0, out=True):
        h = C.c_void_p(0x1234)
        st = f(Xh, xd, Xd, B, G, M, N, K, 0, Yd, Yh, 1, None, 0, flags, None,
               C.byref(h) if out else None)
        if out:
            assert h.value is None  # NULL on every error
        return st

    assert create(out=False) == tw.ERR_INVALID_ARG
    assert create(Xh=None) == tw.ERR_INVALID_ARG
    assert create(xd=2) == tw.ERR_INVALID_ARG
    assert create(Xd=MIS) == tw.ERR_MISALIGNED
    assert create(K=40) == tw.ERR_UNSUPPORTED_SHAPE
    assert create(flags=16) == tw.ERR_INVALID_ARG
    assert create(M=0) == tw.ERR_INVALID_ARG
    assert tw.lib.bitnet_host_plan_run(None) == tw.ERR_INVALID_ARG
    tw.lib.bitnet_host_plan_destroy(None)


def test_binding_refuses_host_tensors_for_device_buffers(tw):
    """The Python binding (and the host-to-host plan) refuse CPU tensors where
    device buffers belong, before any C call: there is no CPU fallback."""
    import torch
    x = torch.zeros(1, 64, dtype=torch.bfloat16)
    y = torch.zeros(1, 16, dtype=torch.bfloat16)
    packed = torch.zeros(16, 16, dtype=torch.uint8)
    gamma = torch.ones(1, dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        tw.bitnet_w158a8_matmul(x, packed, gamma)
    with pytest.raises(ValueError, match="CUDA tensor"):
        tw.bitnet_w158a8_matmul_host(x, packed, gamma, x.clone(), y.clone(), y)
    with pytest.raises(ValueError, match="CUDA tensor"):
        tw.HostMatmulPlan(x, packed, gamma, x.clone(), y.clone(), y)
