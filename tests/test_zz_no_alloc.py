"""bitnet_w158a8_matmul_noalloc: the BitLinear product for callers that
cannot allocate device memory (a plugin whose host framework owns all device
memory, a serving loop that must not call cudaMalloc because it can block
until the device is idle).  It uses the library's built-in scratch array
instead of a caller workspace.

Checked through the C ABI against the regular entry point on the same
inputs, within the tolerances of the parity tests (bf16 within 1 ulp, int32
exact), on two calls in a row with different inputs, so that whatever the
first call leaves in the shared array cannot leak into the second.  This file
is collected last so that a run stopping at the first failure has run every
other test first; it also passes alone in a fresh process.
"""

import ctypes as C

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def tw():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from __graft_entry__ import load_builder
    load_builder().build()
    import ternary_weight_linear_token_b200 as tw
    return tw


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).astype(np.int32)


def _within_one_ulp(a, b):
    def ordered(x):
        return np.where(x & 0x8000, -(x & 0x7FFF), x & 0x7FFF)
    return int(np.abs(ordered(a) - ordered(b)).max(initial=0)) <= 1


def _noalloc_raw(tw, X, packed, gamma, Y, relu2=False, s=None):
    """Direct call of the C entry point (no Python-side allocation)."""
    M, K = X.shape
    N = packed.shape[0]
    ptr = lambda t: None if t is None else C.c_void_p(t.data_ptr())
    xd = {torch.bfloat16: tw.BF16, torch.float32: tw.F32, torch.int8: tw.I8}[X.dtype]
    yd = {torch.bfloat16: tw.BF16, torch.float32: tw.F32, torch.int32: tw.I32}[Y.dtype]
    return tw.lib.bitnet_w158a8_matmul_noalloc(
        ptr(X), xd, ptr(s), ptr(packed), ptr(gamma), M, N, K,
        tw.EPI_RELU2 if relu2 else tw.EPI_NONE, ptr(Y), yd, 0,
        C.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M,N,K,relu2", [(300, 600, 2560, False), (4096, 512, 2560, True),
                                         (129, 257, 2624, False), (1, 2560, 2560, False),
                                         (40, 33, 80, True)])
def test_noalloc_matches_regular_entry_point_twice(tw, M, N, K, relu2):
    rng = np.random.default_rng(M + 3 * N + 7 * K)
    W = torch.from_numpy(synth.latent_weights(rng, N, K)).to(DEV)
    packed, gamma = tw.bitnet_quantize_weights(W)
    for call in range(2):  # two calls in a row, different activations
        x = rng.standard_t(3, (M, K)).astype(np.float32) * (1 + 5 * call)
        X = torch.from_numpy(synth.f32_to_bf16_bits(x).view(np.int16)).to(DEV).view(torch.bfloat16)
        want = tw.bitnet_w158a8_matmul(X, packed, gamma, relu2=relu2)
        got = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _noalloc_raw(tw, X, packed, gamma, got, relu2=relu2) == tw.OK
        torch.cuda.synchronize()
        assert _within_one_ulp(_bits(got), _bits(want)), (M, N, K, call)
        acc_want = tw.bitnet_w158a8_matmul(X, packed, gamma, out_dtype=torch.int32)
        acc_got = torch.zeros((M, N), dtype=torch.int32, device=DEV)
        assert _noalloc_raw(tw, X, packed, gamma, acc_got) == tw.OK
        torch.cuda.synchronize()
        assert torch.equal(acc_got, acc_want), (M, N, K, call)
    assert tw.bitnet_get_device_status() == tw.OK


def test_noalloc_binding_and_size_limit(tw):
    K = 4096
    W = torch.ones((64, K), device=DEV)
    packed, gamma = tw.bitnet_quantize_weights(W)
    X = torch.randn((128, K), device=DEV).to(torch.bfloat16)
    y = tw.bitnet_w158a8_matmul_noalloc(X, packed, gamma)
    assert torch.equal(y, tw.bitnet_w158a8_matmul(X, packed, gamma))
    # the scratch need of this call (M*K bytes of int8 + scales) is above the
    # built-in scratch: rejected with the workspace status, nothing launched
    M_big = (tw.STATIC_SCRATCH_BYTES // K) + 64
    need = tw.bitnet_w158a8_matmul_workspace_size(M_big, 64, K, torch.bfloat16)
    assert need > tw.STATIC_SCRATCH_BYTES
    Xb = torch.zeros((M_big, K), dtype=torch.bfloat16, device=DEV)
    Yb = torch.zeros((M_big, 64), dtype=torch.bfloat16, device=DEV)
    assert _noalloc_raw(tw, Xb, packed, gamma, Yb) == tw.ERR_WORKSPACE
    with pytest.raises(tw.BitnetError):
        tw.bitnet_w158a8_matmul_noalloc(Xb, packed, gamma, Y=Yb)
