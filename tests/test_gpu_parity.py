"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Integers (packed codes, xq, s, int32 accumulators) must be bit-exact.
Floating-point outputs: fp32 within 1e-6 relative, bf16 within 1 ulp (the
tolerances of the benchmark spec); the kernels apply the same operations in
the same order as the oracle, so exact agreement is also counted and reported.

Sizes span several tiles and ragged tails of every kernel path: the fused
decode kernel (M <= 32, 16-row blocks, 256-element K units), the tcgen05
prefill kernel (128 x 256 tiles, 128-byte K stages) and the dp4a generic
kernel (K % 64 != 0).  The full-size prefill workload is checked on every
output.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_util import (DEV, as_x, assert_bf16_within_ulp, assert_f32_close,
                      assert_f32_within_ulp, bf16_bits_of, bf16_t,
                      f32_t, np_of, quantize_weights_both, x_tensor)
from oracle import ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tw():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from __graft_entry__ import load_builder
    load_builder().build()
    import ternary_weight_linear_token_b200 as tw
    return tw


def _latent(N, K, seed):
    return synth.latent_weights(np.random.default_rng(seed), N, K)


# --------------------------------------------------------------- weights
WEIGHT_CASES = {
    "tiny": lambda: synth.config_inputs("tiny")["W"],
    "decode": lambda: synth.config_inputs("decode")["W"],
    "qkv": lambda: synth.config_inputs("sweep", proj=0)["W"],
    "up": lambda: synth.config_inputs("sweep", proj=2)["W"],
    "down": lambda: synth.config_inputs("sweep", proj=3)["W"],
    "ragged_37x48": lambda: _latent(37, 48, 1),
    "one_row_16": lambda: _latent(1, 16, 2),
    "rows_129_k_272": lambda: _latent(129, 272, 3),
    "zeros": lambda: np.zeros((20, 64), dtype=np.float32),
    "ones": lambda: np.ones((20, 64), dtype=np.float32),
    "minus_ones": lambda: -np.ones((20, 64), dtype=np.float32),
}


@pytest.mark.parametrize("name", sorted(WEIGHT_CASES))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_weights_bitexact(tw, name, dtype):
    W = WEIGHT_CASES[name]()
    pd, gd, po, go = quantize_weights_both(W, dtype)
    torch.cuda.synchronize()
    assert np_of(gd)[0].view(np.uint32) == np.float32(go).view(np.uint32), (np_of(gd)[0], go)
    assert np.array_equal(np_of(pd), po)


def test_quantize_weights_boundaries(tw):
    """The hand-made boundary rows of the oracle pins, on the GPU."""
    from pins import _BOUNDARY, _BOUNDARY_075
    for table in (_BOUNDARY, _BOUNDARY_075):
        W = np.array([[w for w, _ in table]], dtype=np.float32)
        pd, gd, po, go = quantize_weights_both(W)
        assert np.array_equal(np_of(pd), po) and np_of(gd)[0] == go


# --------------------------------------------------------------- activations
def _act_cases():
    yield "tiny", synth.config_inputs("tiny")["x"], "f32"
    yield "decode", synth.config_inputs("decode", weights=False)["x"], "bf16"
    yield "sweep_M32_K6912", synth.config_inputs("sweep", M=32, proj=3, weights=False)["x"], "bf16"
    # bf16 rows whose products x * s round onto ties (v = +-63.5 hundreds of
    # times): 200 rows take the warp-per-row kernel, 100 the CTA-per-row one
    yield "prefill_rows", synth.config_inputs("prefill", weights=False)["x"][:200], "bf16"
    yield "prefill_rows_few", synth.config_inputs("prefill", weights=False)["x"][:100], "bf16"
    rng = np.random.default_rng(11)
    x = rng.standard_t(3, (7, 48)).astype(np.float32)
    x[2] = 0.0
    yield "ragged_zero_row", x, "f32"
    ties = np.array([[127.0, 0.5, -0.5, 1.5, 2.5, -2.5, 126.5, -126.5, 64.5, -64.5, 3.5, 0.0,
                      -0.0, 100.25, 1.0, -127.0],
                     [254.0, 1.0, 3.0, 5.0, -5.0, -254.0, 253.0, 0.0, 2.0, -1.0, -3.0, 7.0, 9.0,
                      -11.0, 0.5, 0.25]], dtype=np.float32)
    yield "ties", ties, "f32"
    yield "ties_bf16", ties, "bf16"


@pytest.mark.parametrize("name,x,dtype", list(_act_cases()), ids=lambda v: v if isinstance(v, str) else "")
def test_quantize_act_bitexact(tw, name, x, dtype):
    xd, xexact = as_x(x, dtype)
    xq, s = tw.bitnet_quantize_act(xd)
    xq_o, s_o = ref.quantize_act(xexact)
    torch.cuda.synchronize()
    assert np.array_equal(np_of(s).view(np.uint32), s_o.view(np.uint32))
    assert np.array_equal(np_of(xq), xq_o)


# --------------------------------------------------------------- matmul
# (M, N, K): low-latency shapes (M <= 8, any K % 16 == 0, several CTAs per
# SM, K beyond the register window), decode shapes (8 < M <= 32, K % 64 ==
# 0), prefill shapes (several 128 x 256 tiles, ragged M, N, K), generic
# shapes (M > 8, K % 64 != 0).
SHAPES = [
    (1, 272, 320), (2, 275, 320), (3, 17, 64), (4, 40, 48), (1, 33, 8704), (4, 21, 10240),
    (2, 5, 16), (5, 100, 6912), (8, 160, 2560), (7, 3000, 80), (6, 2561, 2560), (9, 33, 256),
    (16, 48, 1024), (17, 31, 192), (24, 64, 2560), (31, 47, 640), (32, 96, 6912),
    (33, 300, 192), (128, 256, 128), (129, 257, 2624), (300, 600, 2560), (256, 520, 64),
    (384, 300, 640), (1000, 512, 2560), (640, 1100, 384),
    (5, 77, 48), (40, 33, 80), (1, 19, 2576), (130, 70, 208),
    # 4..8 tokens quantised inside the mma.sync kernel: one K step (fewer than
    # the warps), N below one 8-row block, an odd step count, the largest K
    (4, 7, 64), (7, 9, 192), (4, 2000, 1088), (5, 1201, 4096), (8, 2560, 4160),
    # more than 148 tokens: the quantiser's warp-per-row kernel keeps a bf16
    # row in registers up to K = 3072 and loops in two passes above it
    (200, 24, 3072), (150, 24, 3136), (160, 40, 6912),
]


def _run_all_outputs(tw, Xd, sd, packed_d, gamma_d, M, N, K, want_acc, s_o, gamma_o,
                     table_lookup=False):
    exact = {}
    for out_dtype, relu2 in ((torch.int32, False), (torch.float32, False), (torch.float32, True),
                             (torch.bfloat16, False), (torch.bfloat16, True)):
        Y = tw.bitnet_w158a8_matmul(Xd, packed_d, gamma_d, s=sd, relu2=relu2, out_dtype=out_dtype,
                                    table_lookup=table_lookup)
        torch.cuda.synchronize()
        if out_dtype == torch.int32:
            assert np.array_equal(np_of(Y), want_acc), "int32 accumulators differ"
            continue
        y_o = ref.epilogue(want_acc, s_o, gamma_o, relu2)
        if out_dtype == torch.float32:
            got = np_of(Y)
            assert_f32_close(got, y_o, 1e-6)
            exact[("f32", relu2)] = bool(np.array_equal(got.view(np.uint32), y_o.view(np.uint32)))
        else:
            got = bf16_bits_of(Y)
            want = ref.to_bf16(y_o)
            assert_bf16_within_ulp(got, want, 1)
            exact[("bf16", relu2)] = bool(np.array_equal(got, want))
    return exact


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("xdtype", ["f32", "bf16", "i8"])
def test_matmul_parity(tw, M, N, K, xdtype):
    rng = np.random.default_rng(M * 7919 + N * 31 + K)
    W = synth.latent_weights(rng, N, K)
    x = rng.standard_t(3, (M, K)).astype(np.float32)
    packed_d, gamma_d, packed_o, gamma_o = quantize_weights_both(W)
    assert np.array_equal(np_of(packed_d), packed_o)
    if xdtype == "i8":
        xq_o, s_o = ref.quantize_act(x)
        Xd = torch.from_numpy(xq_o).to(DEV)
        sd = torch.from_numpy(s_o).to(DEV)
    else:
        Xd, xexact = as_x(x, xdtype)
        sd = None
        xq_o, s_o = ref.quantize_act(xexact)
    acc_o = ref.matmul_acc(xq_o, packed_o, N, K)
    exact = _run_all_outputs(tw, Xd, sd, packed_d, gamma_d, M, N, K, acc_o, s_o, gamma_o)
    assert all(exact.values()), f"within tolerance but not bit-identical: {exact}"


# The extremes of the accepted sizes, kept cheap for the oracle by the other
# dimensions: K up to 2^22 (|acc| <= 127 K stays far inside int32; the
# activations no longer fit any kernel's shared-memory window) for 1, 3, 8
# and 40 tokens; 2^17 tokens (1024 row tiles of the tensor-core path); and
# 1.1 M tokens on the dp4a kernel (K % 64 != 0), more token blocks than a
# grid's y dimension holds.
EXTREME_SHAPES = [(1, 7, 1 << 20), (3, 5, 1 << 22), (8, 9, 1 << 20), (40, 6, 1 << 20),
                  (1 << 17, 24, 64), (100003, 3, 128), (1100000, 3, 16)]


@pytest.mark.parametrize("M,N,K", EXTREME_SHAPES)
def test_matmul_parity_extreme_sizes(tw, M, N, K):
    """Every kernel path at the largest sizes the checks accept that still fit
    a test: int32 accumulators and bf16 outputs bit-exact, bf16 input."""
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    W = synth.latent_weights(rng, N, K)
    x = rng.standard_t(3, (M, K)).astype(np.float32)
    packed_d, gamma_d, packed_o, gamma_o = quantize_weights_both(W)
    assert np.array_equal(np_of(packed_d), packed_o)
    Xd, xexact = as_x(x, "bf16")
    xq_o, s_o = ref.quantize_act(xexact)
    acc_o = ref.matmul_acc(xq_o, packed_o, N, K)
    Y = tw.bitnet_w158a8_matmul(Xd, packed_d, gamma_d, out_dtype=torch.int32)
    torch.cuda.synchronize()
    assert np.array_equal(np_of(Y), acc_o), "int32 accumulators differ"
    Y = tw.bitnet_w158a8_matmul(Xd, packed_d, gamma_d, relu2=True)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits_of(Y), ref.to_bf16(ref.epilogue(acc_o, s_o, gamma_o, True)))
    assert tw.bitnet_get_device_status() == tw.OK


PREP_SHAPES = [(33, 300, 192), (128, 256, 128), (129, 257, 2624), (300, 600, 2560),
               (256, 520, 64), (1000, 512, 2560), (640, 1100, 384), (130, 70, 208)]


@pytest.mark.parametrize("M,N,K", [sh for sh in PREP_SHAPES if sh[2] % 64 == 0])
@pytest.mark.parametrize("xdtype", ["f32", "bf16", "i8"])
def test_prep_in_kernel_parity(tw, M, N, K, xdtype):
    """The tensor-core path with its operands prepared inside the kernel
    (BITNET_FLAG_PREP_IN_KERNEL): single CTAs and CTA pairs, ragged M, N and
    K, every input dtype; int32 accumulators and outputs bit-exact."""
    rng = np.random.default_rng(M * 7907 + N * 13 + K)
    W = synth.latent_weights(rng, N, K)
    x = rng.standard_t(3, (M, K)).astype(np.float32)
    packed_d, gamma_d, packed_o, gamma_o = quantize_weights_both(W)
    if xdtype == "i8":
        xq_o, s_o = ref.quantize_act(x)
        Xd, sd = torch.from_numpy(xq_o).to(DEV), torch.from_numpy(s_o).to(DEV)
    else:
        Xd, xexact = as_x(x, xdtype)
        sd = None
        xq_o, s_o = ref.quantize_act(xexact)
    assert tw.bitnet_w158a8_matmul_path(M, N, K, Xd.dtype) == tw.PATH_TENSOR_CORE
    acc_o = ref.matmul_acc(xq_o, packed_o, N, K)
    for out_dtype, relu2 in ((torch.int32, False), (torch.bfloat16, True), (torch.float32, False)):
        Y = tw.bitnet_w158a8_matmul(Xd, packed_d, gamma_d, s=sd, relu2=relu2, out_dtype=out_dtype,
                                    prep_in_kernel=True)
        torch.cuda.synchronize()
        if out_dtype == torch.int32:
            assert np.array_equal(np_of(Y), acc_o)
        elif out_dtype == torch.float32:
            assert np.array_equal(np_of(Y), ref.epilogue(acc_o, s_o, gamma_o, relu2))
        else:
            assert np.array_equal(bf16_bits_of(Y), ref.to_bf16(ref.epilogue(acc_o, s_o, gamma_o, relu2)))
    assert tw.bitnet_get_device_status() == tw.OK


# the table-lookup comparison kernel: 1..8 tokens, several CTAs' rows, K
# ragged against the 32-lane word loop, K of the down projection (one
# token's tables per batch), more tokens than fit in one table batch
LUT_SHAPES = [(1, 2560, 2560), (2, 275, 320), (3, 17, 64), (4, 40, 48), (8, 160, 2560),
              (5, 100, 6912), (1, 19, 2576), (8, 6912, 2560), (7, 3000, 80)]


@pytest.mark.parametrize("M,N,K", LUT_SHAPES)
@pytest.mark.parametrize("xdtype", ["f32", "bf16", "i8"])
def test_table_lookup_kernel_parity(tw, M, N, K, xdtype):
    """The table-lookup kernel (BITNET_FLAG_TABLE_LOOKUP) against the oracle:
    int32 accumulators and every output dtype bit-exact."""
    rng = np.random.default_rng(M * 104729 + N * 17 + K)
    W = synth.latent_weights(rng, N, K)
    x = rng.standard_t(3, (M, K)).astype(np.float32)
    packed_d, gamma_d, packed_o, gamma_o = quantize_weights_both(W)
    if xdtype == "i8":
        xq_o, s_o = ref.quantize_act(x)
        Xd, sd = torch.from_numpy(xq_o).to(DEV), torch.from_numpy(s_o).to(DEV)
    else:
        Xd, xexact = as_x(x, xdtype)
        sd = None
        xq_o, s_o = ref.quantize_act(xexact)
    acc_o = ref.matmul_acc(xq_o, packed_o, N, K)
    exact = _run_all_outputs(tw, Xd, sd, packed_d, gamma_d, M, N, K, acc_o, s_o, gamma_o,
                             table_lookup=True)
    assert all(exact.values()), f"within tolerance but not bit-identical: {exact}"
    assert tw.bitnet_get_device_status() == tw.OK


def test_matmul_degenerate(tw):
    K, N = 256, 48
    x = np.random.default_rng(5).standard_normal((3, K)).astype(np.float32)
    x[1] = 0.0  # all-zero token row -> s = 1, y row = 0
    for path_M in (3, 6, 40):  # fused one-launch kernels and the prefill path
        xm = np.resize(x, (path_M, K)).astype(np.float32)
        Xd = f32_t(xm)
        for Wv, label in ((np.zeros((N, K), np.float32), "zero"), (np.ones((N, K), np.float32), "ones")):
            pd, gd = tw.bitnet_quantize_weights(f32_t(Wv))
            Y = np_of(tw.bitnet_w158a8_matmul(Xd, pd, gd, out_dtype=torch.float32))
            if label == "zero":
                assert not Y.any(), "W = 0 must give y = 0"
            else:
                xq, s = ref.quantize_act(xm)
                want = (xq.astype(np.int64).sum(axis=1).astype(np.float32) *
                        (np.float32(1.0) / s))[:, None].repeat(N, axis=1)
                assert np.array_equal(Y, want.astype(np.float32)), "W = +1 must give row sums"
        # zero activation row gives a zero output row
        pd, gd = tw.bitnet_quantize_weights(f32_t(synth.latent_weights(np.random.default_rng(1), N, K)))
        Y = np_of(tw.bitnet_w158a8_matmul(Xd, pd, gd, out_dtype=torch.float32))
        zero_rows = ~xm.any(axis=1)
        assert zero_rows.any() and not Y[zero_rows].any()
    # empty batch: no launch, no error
    empty = torch.empty((0, K), dtype=torch.bfloat16, device=DEV)
    Y = tw.bitnet_w158a8_matmul(empty, pd, gd)
    assert Y.shape == (0, N)
    assert tw.bitnet_get_device_status() == tw.OK


def test_sign_flip_on_gpu(tw):
    rng = np.random.default_rng(9)
    W = synth.latent_weights(rng, 300, 2560)
    x = rng.standard_normal((40, 2560)).astype(np.float32)
    for M in (4, 40):
        Xd = f32_t(x[:M])
        p, g = tw.bitnet_quantize_weights(f32_t(W))
        pn, gn = tw.bitnet_quantize_weights(f32_t(-W))
        a = np_of(tw.bitnet_w158a8_matmul(Xd, p, g, out_dtype=torch.int32))
        b = np_of(tw.bitnet_w158a8_matmul(Xd, pn, gn, out_dtype=torch.int32))
        c = np_of(tw.bitnet_w158a8_matmul(f32_t(-x[:M]), p, g, out_dtype=torch.int32))
        assert np.array_equal(b, -a) and np.array_equal(c, -a)


def test_workspace_too_small_raises(tw):
    X = torch.zeros((64, 256), dtype=torch.bfloat16, device=DEV)
    p, g = tw.bitnet_quantize_weights(torch.ones((32, 256), device=DEV))
    need = tw.bitnet_w158a8_matmul_workspace_size(64, 32, 256, torch.bfloat16)
    ws = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(tw.BitnetError) as e:
        tw.bitnet_w158a8_matmul(X, p, g, workspace=ws)
    assert e.value.status == tw.ERR_WORKSPACE


# --------------------------------------------------------------- workloads at full size
def test_decode_workload_full(tw):
    """Decode GEMV, M=1, K=N=2560, bf16 in/out: every output against the oracle,
    plain, with the static-weights flag, and replayed from a CUDA graph."""
    d = synth.config_inputs("decode")
    pd, gd, po, go = quantize_weights_both(d["W"])
    want = ref.to_bf16(ref.bitlinear(d["x"], po, go, d["N"])["y"])
    Xd = x_tensor(d)
    for ws in (False, True):
        Y = tw.bitnet_w158a8_matmul(Xd, pd, gd, weights_static=ws)
        assert_bf16_within_ulp(bf16_bits_of(Y), want)
        assert np.array_equal(bf16_bits_of(Y), want)
    Y = torch.empty((1, d["N"]), dtype=torch.bfloat16, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        tw.bitnet_w158a8_matmul(Xd, pd, gd, Y=Y, weights_static=True)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    Y.zero_()
    with torch.cuda.graph(graph):
        for _ in range(4):
            tw.bitnet_w158a8_matmul(Xd, pd, gd, Y=Y, weights_static=True)
    graph.replay()
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits_of(Y), want)


@pytest.mark.parametrize("M", [1, 8, 32])
def test_sweep_workload_full(tw, M):
    """One decoder layer's four projections at M = 1, 8, 32 (Student-t bf16)."""
    for proj in range(4):
        d = synth.config_inputs("sweep", M=M, proj=proj)
        pd, gd, po, go = quantize_weights_both(d["W"])
        want = ref.to_bf16(ref.bitlinear(d["x"], po, go, d["N"], relu2=d["relu2"])["y"])
        Y = tw.bitnet_w158a8_matmul(x_tensor(d), pd, gd, relu2=d["relu2"], weights_static=True)
        assert np.array_equal(bf16_bits_of(Y), want), (M, proj)


def test_prefill_workload_full_size(tw):
    """Prefill, M=4096, K=2560, N=6912, bf16, in the launch configuration the
    bench times (CTA-pair tcgen05 kernel on 256 x 256 tiles, weights expanded
    into the workspace): every one of the 4096 x 6912 int32 accumulators and
    bf16 outputs against the oracle (about 1.4e11 ops on the host cores),
    and the quantised activations the path left in its workspace.  Then the
    same call with the expansion skipped (BITNET_FLAG_WEIGHTS_EXPANDED) on
    that workspace, and the int8-input form, must give the same outputs."""
    d = synth.config_inputs("prefill")
    pd, gd, po, go = quantize_weights_both(d["W"])
    assert tw.bitnet_w158a8_matmul_path(4096, 6912, 2560, torch.bfloat16) == tw.PATH_TENSOR_CORE
    Xd = x_tensor(d)
    need = tw.bitnet_w158a8_matmul_workspace_size(4096, 6912, 2560, torch.bfloat16)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    Y = tw.bitnet_w158a8_matmul(Xd, pd, gd, workspace=ws, weights_static=True)
    Yi = tw.bitnet_w158a8_matmul(Xd, pd, gd, workspace=ws, out_dtype=torch.int32)
    torch.cuda.synchronize()
    out = ref.bitlinear(d["x"], po, go, d["N"])
    acc = np_of(Yi)
    bad = np.argwhere(acc != out["acc"])
    assert bad.size == 0, f"{len(bad)} int32 accumulators differ, first at {bad[:4].tolist()}"
    want = ref.to_bf16(out["y"])
    got = bf16_bits_of(Y)
    assert_bf16_within_ulp(got, want)
    assert np.array_equal(got, want)
    # the quantised activations the prefill path wrote into its workspace, kept
    # there in the K order of the kernel's weight unpack (inside each
    # 16-element group: elements 0,8,1,9, 4,12,5,13, 2,10,3,11, 6,14,7,15)
    perm = np.array([0, 8, 1, 9, 4, 12, 5, 13, 2, 10, 3, 11, 6, 14, 7, 15])
    stored = np_of(ws[: 4096 * 2560]).view(np.int8).reshape(4096, 160, 16)
    natural = np.empty_like(stored)
    natural[:, :, perm] = stored
    assert np.array_equal(natural.reshape(4096, 2560), out["xq"])
    # the expansion skipped on the same workspace: same outputs
    Y2 = tw.bitnet_w158a8_matmul(Xd, pd, gd, workspace=ws, weights_static=True,
                                 weights_expanded=True)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits_of(Y2), want)
    # the tensor-core kernel preparing its own operands (quantiser and
    # expansion inside the kernel, BITNET_FLAG_PREP_IN_KERNEL): same outputs
    ws2 = torch.empty(need, dtype=torch.uint8, device=DEV)
    Y4 = tw.bitnet_w158a8_matmul(Xd, pd, gd, workspace=ws2, weights_static=True,
                                 prep_in_kernel=True)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits_of(Y4), want)
    # int8 activations from the caller (natural K order, its own expansion),
    # then again with that expansion kept
    xq, sq = tw.bitnet_quantize_act(Xd)
    need8 = tw.bitnet_w158a8_matmul_workspace_size(4096, 6912, 2560, torch.int8)
    ws8 = torch.empty(need8, dtype=torch.uint8, device=DEV)
    for expanded in (False, True):
        Y3 = tw.bitnet_w158a8_matmul(xq, pd, gd, s=sq, workspace=ws8, weights_expanded=expanded)
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits_of(Y3), want), expanded
    assert tw.bitnet_get_device_status() == tw.OK


def test_chain_link_by_link(tw):
    """Two layers of the 30-layer decode chain: every projection's GPU output
    against the oracle fed the GPU's own input to that projection."""
    from ternary_weight_linear_token_b200.chain import DecodeChain
    layers = []
    for layer in range(2):
        layers.append([(f32_t(synth.layer_weights(layer, p)), synth.PROJECTIONS[p][3])
                       for p in range(4)])
    chain = DecodeChain(layers)
    x0 = synth.config_inputs("chain", weights=False)
    chain.run(x_tensor(x0))
    torch.cuda.synchronize()
    x_in = bf16_bits_of(chain.x_in)
    for li, (proj, bufs) in enumerate(zip(chain.layers, chain.outs)):
        inputs = [x_in, bf16_bits_of(bufs[0])[:, :chain.d], bf16_bits_of(bufs[1]),
                  bf16_bits_of(bufs[2])]
        for pi in range(4):
            W = synth.layer_weights(li, pi)
            po, go = ref.quantize_weights(W)
            assert np.array_equal(np_of(proj[pi]["packed"]), po)
            xin = synth.bf16_bits_to_f32(inputs[pi])
            want = ref.to_bf16(ref.bitlinear(xin, po, go, proj[pi]["N"], relu2=proj[pi]["relu2"])["y"])
            assert np.array_equal(bf16_bits_of(bufs[pi]), want), (li, pi)
        norm_in = synth.bf16_bits_to_f32(bf16_bits_of(bufs[3]))
        assert_bf16_within_ulp(bf16_bits_of(bufs[4]), ref.to_bf16(ref.rms_norm(norm_in)), 1)
        x_in = bf16_bits_of(bufs[4])
    # graph replay reproduces the eager run bit for bit
    eager = bf16_bits_of(chain.outs[-1][4]).copy()
    chain.capture()
    chain.graph.replay()
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits_of(chain.outs[-1][4]), eager)


def test_quantize_act_rounding_near_every_tie(tw):
    """Every row has max |x| = 127, so s = 127 / 127 = 1 exactly and x * s = x:
    the kernel's rounding is seen directly.  Rows hold every tie k + 0.5
    (k = -127..126) with the 64 floats on each side of it, plus uniform
    values; xq must equal the oracle's round-half-away-from-zero bit for bit."""
    vals = []
    for k in range(-127, 127):
        t = np.float32(k + 0.5)
        lo = hi = t
        vals.append(t)
        for _ in range(64):
            lo = np.nextafter(lo, np.float32(-np.inf), dtype=np.float32)
            hi = np.nextafter(hi, np.float32(np.inf), dtype=np.float32)
            vals += [lo, hi]
    vals = np.array(vals, dtype=np.float32)
    vals = vals[np.abs(vals) <= 127.0]
    rng = np.random.default_rng(5)
    K = 4096
    body = np.concatenate([vals, rng.uniform(-127, 127, 64 * K).astype(np.float32)])
    M = (body.size + K - 2) // (K - 1)
    body = np.resize(body, M * (K - 1)).reshape(M, K - 1)
    x = np.concatenate([np.full((M, 1), 127.0, np.float32), body], axis=1)
    xq, sc = tw.bitnet_quantize_act(f32_t(x))
    torch.cuda.synchronize()
    wq, ws = ref.quantize_act(x)
    assert np.all(ws == np.float32(1.0)) and np.array_equal(np_of(sc), ws)
    assert np.array_equal(np_of(xq), wq)


def test_fused_prologue_rounding_near_every_tie(tw):
    """The quantiser inside the fused few-token kernel, seen directly: W is
    the K x K identity (gamma = 1/K, every diagonal code +1, the rest 0), so
    the int32 accumulators are the int8 activations themselves.  Rows hold
    every tie k + 0.5 (k = -127..126) with the 64 floats on each side and
    max |x| = 127 (s = 1 exactly), 1..3 tokens per call (the fused path), fp32
    and bf16 input; every accumulator must equal the oracle's quantised
    activation."""
    K = 4096
    vals = []
    for k in range(-127, 127):
        t = np.float32(k + 0.5)
        lo = hi = t
        vals.append(t)
        for _ in range(64):
            lo = np.nextafter(lo, np.float32(-np.inf), dtype=np.float32)
            hi = np.nextafter(hi, np.float32(np.inf), dtype=np.float32)
            vals += [lo, hi]
    vals = np.array(vals, dtype=np.float32)
    vals = vals[np.abs(vals) <= 127.0]
    rows = (vals.size + K - 2) // (K - 1)
    body = np.resize(vals, rows * (K - 1)).reshape(rows, K - 1)
    x = np.concatenate([np.full((rows, 1), 127.0, np.float32), body], axis=1)
    pd, gd = tw.bitnet_quantize_weights(f32_t(np.eye(K, dtype=np.float32)))
    for dt in ("f32", "bf16"):
        for r0 in range(0, rows, 3):
            xs = x[r0:r0 + 3]
            Xd, xexact = as_x(xs, dt)
            assert tw.bitnet_w158a8_matmul_path(xs.shape[0], K, K, Xd.dtype) == tw.PATH_ROWS
            acc = tw.bitnet_w158a8_matmul(Xd, pd, gd, out_dtype=torch.int32)
            torch.cuda.synchronize()
            want, _ = ref.quantize_act(xexact)
            assert np.array_equal(np_of(acc), want.astype(np.int32)), (dt, r0)


# (M, N, K, input dtype, ReLU^2): one-launch fused path for M <= 8, a
# normalisation kernel and then the matmul for larger M
NORM_SHAPES = [(1, 2560, 2560, "bf16", False), (1, 3840, 2560, "bf16", False),
               (3, 640, 2560, "f32", True), (8, 300, 320, "bf16", True), (5, 77, 48, "f32", False),
               (2, 6912, 2560, "bf16", True), (9, 200, 512, "bf16", False),
               (33, 128, 256, "f32", True)]


@pytest.mark.parametrize("M,N,K,dt,relu2", NORM_SHAPES)
def test_rms_norm_matmul(tw, M, N, K, dt, relu2):
    """Y = BitLinear(rms_norm(X)): the normalised input against the oracle's
    normalisation, and Y bit-exact against the oracle's BitLinear of the
    kernel's own normalised input.

    Tolerance of the normalisation (glue, outside the bit-exact contract):
    both sides sum the squares in fp64 (each square exact there) and compute
    the factor 1/sqrt(ss/K + 1e-6) in fp64, rounded once to fp32; then
    y = x * factor in fp32.  The sums differ only in order, by a few fp64
    ulps, so the fp32 factors are equal unless the exact factor lies within
    that distance of an fp32 rounding boundary (about 1e-7 per token); then
    they differ by one fp32 ulp, and y by at most 2 fp32 ulps (1 bf16 ulp
    after rounding to bf16).  So: every token within 2 fp32 ulps / 1 bf16
    ulp, and at most one token of a call not bit-identical."""
    rng = np.random.default_rng(M * 131 + N + K)
    W = synth.latent_weights(rng, N, K)
    x = (3.0 * rng.standard_t(3, (M, K))).astype(np.float32)
    X, xf = as_x(x, dt)
    pd, gd = tw.bitnet_quantize_weights(f32_t(W))
    po, go = ref.quantize_weights(W)
    Xn = torch.empty_like(X)
    ydt = torch.float32 if dt == "f32" else torch.bfloat16
    Y = tw.bitnet_rms_norm_w158a8_matmul(X, pd, gd, X_normed=Xn, relu2=relu2, out_dtype=ydt)
    torch.cuda.synchronize()
    want_n = ref.rms_norm(xf)
    if dt == "bf16":
        got_n = bf16_bits_of(Xn)
        assert_bf16_within_ulp(got_n, ref.to_bf16(want_n), 1)
        differ = int((got_n != ref.to_bf16(want_n)).any(axis=1).sum())
        want = ref.to_bf16(ref.bitlinear(synth.bf16_bits_to_f32(got_n), po, go, N, relu2=relu2)["y"])
        assert np.array_equal(bf16_bits_of(Y), want)
    else:
        got_n = np_of(Xn)
        assert_f32_within_ulp(got_n, want_n, 2)
        differ = int((got_n != want_n).any(axis=1).sum())
        want = ref.bitlinear(got_n, po, go, N, relu2=relu2)["y"]
        assert_f32_close(np_of(Y), want)
    assert differ <= 1, f"{differ} of {M} normalised tokens not bit-identical"
    if M <= 8:  # without X_normed: the same result
        Y2 = tw.bitnet_rms_norm_w158a8_matmul(X, pd, gd, relu2=relu2, out_dtype=ydt)
        torch.cuda.synchronize()
        assert torch.equal(Y2, Y)
    assert tw.bitnet_get_device_status() == tw.OK


@pytest.mark.parametrize("M,N,K,dt", [(1, 2560, 2560, "bf16"), (8, 300, 320, "f32"),
                                      (300, 600, 2560, "bf16"), (1000, 1600, 2560, "bf16"),
                                      (916, 1100, 1024, "f32")])
def test_host_entry_point(tw, M, N, K, dt):
    """bitnet_w158a8_matmul_host (pinned host input and output, one call)
    gives exactly the device entry point's output, on the fused, mma.sync and
    tensor-core paths, and the oracle's; so does a HostMatmulPlan, whose
    graph for the last two shapes is a pipeline of 128-token chunks (the last
    chunk 104 tokens on the tensor-core path, or 20 tokens on the mma.sync
    path)."""
    rng = np.random.default_rng(M + N + K)
    W = synth.latent_weights(rng, N, K)
    x = rng.standard_t(3, (M, K)).astype(np.float32)
    Xd, xexact = as_x(x, dt)
    pd, gd, po, go = quantize_weights_both(W)
    ydt = torch.float32 if dt == "f32" else torch.bfloat16
    want_d = tw.bitnet_w158a8_matmul(Xd, pd, gd, out_dtype=ydt)
    Xh = Xd.cpu().pin_memory()
    Yh = torch.empty((M, N), dtype=ydt).pin_memory()
    X2 = torch.empty_like(Xd)
    Y2 = torch.empty((M, N), dtype=ydt, device=DEV)
    for _ in range(2):
        Yh.zero_()
        tw.bitnet_w158a8_matmul_host(Xh, pd, gd, X2, Y2, Yh, weights_static=True)
        assert torch.equal(Yh, want_d.cpu())
    want_o = ref.bitlinear(xexact, po, go, N)["y"]
    if dt == "f32":
        assert np.array_equal(Yh.numpy(), want_o)
    else:
        assert np.array_equal(Yh.view(torch.int16).numpy().view(np.uint16), ref.to_bf16(want_o))
    # the same call through a plan (arguments checked once), with the host input refilled
    plan = tw.HostMatmulPlan(Xh, pd, gd, X2, Y2, Yh, weights_static=True)
    assert plan.graph  # page-locked buffers: recorded once as a CUDA graph
    for r in range(2):
        x2 = rng.standard_t(3, (M, K)).astype(np.float32)
        Xd2, xexact2 = as_x(x2, dt)
        Xh.copy_(Xd2.cpu())
        Yh.zero_()
        assert plan() is Yh
        want2 = ref.bitlinear(xexact2, po, go, N)["y"]
        got2 = Yh.numpy() if dt == "f32" else Yh.view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got2, want2 if dt == "f32" else ref.to_bf16(want2)), r
    plan.close()
    assert tw.bitnet_get_device_status() == tw.OK


def test_host_plan_pageable_buffers(tw):
    """A HostMatmulPlan over pageable host tensors records no graph and makes
    the host entry point's call each time (the driver stages the copies);
    the results are the oracle's."""
    M, N, K = 1, 640, 1024
    rng = np.random.default_rng(4242)
    W = synth.latent_weights(rng, N, K)
    pd, gd, po, go = quantize_weights_both(W)
    Xh = torch.empty((M, K), dtype=torch.bfloat16)
    Yh = torch.empty((M, N), dtype=torch.bfloat16)
    assert not Xh.is_pinned() and not Yh.is_pinned()
    X2 = torch.empty((M, K), dtype=torch.bfloat16, device=DEV)
    Y2 = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    plan = tw.HostMatmulPlan(Xh, pd, gd, X2, Y2, Yh, relu2=True)
    assert not plan.graph
    for r in range(2):
        x = rng.standard_t(3, (M, K)).astype(np.float32)
        Xd, xexact = as_x(x, "bf16")
        Xh.copy_(Xd.cpu())
        plan()
        want = ref.bitlinear(xexact, po, go, N, relu2=True)["y"]
        assert np.array_equal(Yh.view(torch.int16).numpy().view(np.uint16), ref.to_bf16(want)), r
    plan.close()
    assert tw.bitnet_get_device_status() == tw.OK


def test_repeatable(tw):
    d = synth.config_inputs("sweep", M=8, proj=0)
    pd, gd = tw.bitnet_quantize_weights(f32_t(d["W"]))
    a = bf16_bits_of(tw.bitnet_w158a8_matmul(x_tensor(d), pd, gd))
    b = bf16_bits_of(tw.bitnet_w158a8_matmul(x_tensor(d), pd, gd))
    assert np.array_equal(a, b)
    assert tw.bitnet_get_device_status() == tw.OK
