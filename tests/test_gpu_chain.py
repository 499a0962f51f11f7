"""The persistent decode chain (bitnet_decode_chain) against the CPU oracle,
link by link: every step's bf16 output must equal the oracle's BitLinear of
the step's actual bf16 input (bit-exact); a normalised input (BITNET_STEP_NORM_IN)
must be within 1 bf16 ulp of the oracle's RMS normalisation of the previous
output (both sum the squares in fp64 and round the factor once, so in
practice it is bit-identical), and the oracle's BitLinear is then fed the
kernel's own normalised values.  Shapes cover odd N (a half-filled last
32-bit store), K smaller than the previous N, CTAs that own no row of a step
(N < number of SMs), both epilogues, repeated launches on one workspace and
CUDA-graph replay; and the configured 30-layer stack in both chain forms."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from gpu_util import DEV, assert_bf16_within_ulp, bf16_bits_of, bf16_t, f32_t, np_of
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


def build_chain(tw, specs, seed):
    """specs: (N, K, relu2, norm_in) per step -> step dicts and latent weights."""
    rng = np.random.default_rng(seed)
    steps, Ws = [], []
    for N, K, relu2, norm in specs:
        W = synth.latent_weights(rng, N, K)
        packed, gamma = tw.bitnet_quantize_weights(f32_t(W))
        st = dict(packed=packed, gamma=gamma, relu2=relu2,
                  Y=torch.full((N,), float("nan"), dtype=torch.bfloat16, device=DEV))
        if norm:
            st.update(norm_in=True, X_normed=torch.empty(K, dtype=torch.bfloat16, device=DEV))
        steps.append(st)
        Ws.append(W)
    return steps, Ws


def x0_bits(K, seed):
    x = np.random.default_rng(seed).standard_t(3, K).astype(np.float32)
    return synth.f32_to_bf16_bits(x)


def check_links(steps, Ws, x0, y_norm=None):
    prev = x0
    for i, (st, W) in enumerate(zip(steps, Ws)):
        N, K = st["packed"].shape[0], st["packed"].shape[1] * 4
        po, go = ref.quantize_weights(W)
        assert np.array_equal(np_of(st["packed"]), po), i
        xin = prev[:K]
        if st.get("norm_in"):
            xn = bf16_bits_of(st["X_normed"])
            want_n = ref.to_bf16(ref.rms_norm(synth.bf16_bits_to_f32(xin)[None, :]))[0]
            assert_bf16_within_ulp(xn, want_n, 1)
            xin = xn
        want = ref.to_bf16(ref.bitlinear(synth.bf16_bits_to_f32(xin)[None, :], po, go, N,
                                         relu2=st["relu2"])["y"])[0]
        got = bf16_bits_of(st["Y"])
        bad = np.flatnonzero(got != want)
        assert bad.size == 0, (f"step {i}: {bad.size} of {N} outputs differ, first at {bad[:4]}: "
                               f"got {got[bad[:4]]} want {want[bad[:4]]}")
        prev = got
    if y_norm is not None:
        want = ref.to_bf16(ref.rms_norm(synth.bf16_bits_to_f32(prev)[None, :]))[0]
        assert_bf16_within_ulp(bf16_bits_of(y_norm), want, 1)
    return prev


# (N, K, relu2, norm_in)
SHAPES_A = [(333, 256, True, False),     # odd N: the last exchange word holds one value
            (1000, 320, False, True),    # K < previous N; normalised input
            (5000, 960, True, False),    # wide: ~34 rows per CTA
            (64, 4992, False, True),     # fewer rows than CTAs
            (8192, 64, True, False),     # the largest K the next step may use
            (160, 8192, False, True),    # K = 8192
            (304, 64, True, False)]      # 2 or 4 rows of 4 packed words per CTA: a row's
                                         # pieces fewer than the warps between them
SHAPES_B = [(3840, 2560, False, False), (2560, 2560, False, False), (6912, 2560, True, False),
            (2560, 6912, False, False), (1, 2560, False, True)]  # one output row


@pytest.mark.parametrize("specs,seed,final_norm", [(SHAPES_A, 11, True), (SHAPES_B, 12, False)],
                         ids=["ragged", "one_layer_then_one_row"])
def test_decode_chain_links(tw, specs, seed, final_norm):
    steps, Ws = build_chain(tw, specs, seed)
    arr = tw.bitnet_decode_chain_steps(steps)
    ws = torch.zeros(tw.bitnet_decode_chain_workspace_size(arr), dtype=torch.uint8, device=DEV)
    y_norm = (torch.empty(specs[-1][0], dtype=torch.bfloat16, device=DEV) if final_norm else None)
    for launch in range(3):  # the launch counter in the workspace advances every time
        x0 = x0_bits(specs[0][1], seed + launch)
        for st in steps:
            st["Y"].fill_(float("nan"))
        tw.bitnet_decode_chain(arr, bf16_t(x0), ws, y_norm=y_norm)
        torch.cuda.synchronize()
        check_links(steps, Ws, x0, y_norm)
    assert tw.bitnet_get_device_status() == tw.OK


def test_decode_chain_graph_replay(tw):
    """Captured in a CUDA graph, each replay is a new launch (new tag) and
    recomputes every link from the current input."""
    steps, Ws = build_chain(tw, SHAPES_A[:3], 21)
    arr = tw.bitnet_decode_chain_steps(steps)
    ws = torch.zeros(tw.bitnet_decode_chain_workspace_size(arr), dtype=torch.uint8, device=DEV)
    x_in = torch.empty(SHAPES_A[0][1], dtype=torch.bfloat16, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        x_in.copy_(bf16_t(x0_bits(SHAPES_A[0][1], 0)))
        tw.bitnet_decode_chain(arr, x_in, ws)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        tw.bitnet_decode_chain(arr, x_in, ws)
    for r in range(3):
        x0 = x0_bits(SHAPES_A[0][1], 100 + r)
        x_in.copy_(bf16_t(x0))
        g.replay()
        torch.cuda.synchronize()
        check_links(steps, Ws, x0)
    assert tw.bitnet_get_device_status() == tw.OK


def test_decode_chain_matches_per_launch_chain(tw):
    """Two layers of the 30-layer stack run both ways: the BitLinear links
    agree with the oracle in both, and where the normalisations agree bit for
    bit, so do all later outputs."""
    from ternary_weight_linear_token_b200.chain import DecodeChain
    layers = [[(f32_t(synth.layer_weights(li, p)), synth.PROJECTIONS[p][3]) for p in range(4)]
              for li in range(2)]
    x0 = synth.config_inputs("chain", weights=False)
    x = bf16_t(x0["x_bits"])
    per = DecodeChain(layers)
    per.run(x)
    pers = DecodeChain(layers, persistent=True)
    pers.run(x)
    torch.cuda.synchronize()
    # the first layer has no normalisation: identical outputs
    for pi in range(4):
        assert np.array_equal(bf16_bits_of(per.outs[0][pi]), bf16_bits_of(pers.outs[0][pi])), pi
    # every persistent link against the oracle
    steps = [dict(packed=p["packed"], relu2=p["relu2"], Y=pers.outs[li][pi].view(-1))
             for li, proj in enumerate(pers.layers) for pi, p in enumerate(proj)]
    for li in range(1, 2):
        steps[4 * li].update(norm_in=True, X_normed=pers.outs[li - 1][4].view(-1))
    Ws = [synth.layer_weights(li, p) for li in range(2) for p in range(4)]
    check_links(steps, Ws, x0["x_bits"].reshape(-1), pers.outs[-1][4].view(-1))
    assert tw.bitnet_get_device_status() == tw.OK


def test_decode_chain_launch_tag_wraps(tw):
    """The 16-bit tag of launch T is (T mod 65535) + 1: with the launch
    counter pre-set just below a multiple of 65535 the tags run 65535, 1, 2,
    each launch's values are told apart from the previous launch's, and the
    zero-filled tagged words (tag 0) are never taken for values."""
    steps, Ws = build_chain(tw, SHAPES_A[:3], 41)
    arr = tw.bitnet_decode_chain_steps(steps)
    ws = torch.zeros(tw.bitnet_decode_chain_workspace_size(arr), dtype=torch.uint8, device=DEV)
    ws.view(torch.int32)[0] = 65533          # the launch counter: next launch is T = 65534
    done = 65533 * torch.cuda.get_device_properties(DEV).multi_processor_count
    ws.view(torch.int32)[128 // 4] = done     # the done counter of those launches
    for launch in range(3):
        x0 = x0_bits(SHAPES_A[0][1], 500 + launch)
        for st in steps:
            st["Y"].fill_(float("nan"))
        tw.bitnet_decode_chain(arr, bf16_t(x0), ws)
        torch.cuda.synchronize()
        check_links(steps, Ws, x0)
        assert int(ws.view(torch.int32)[0].item()) == 65534 + launch
    assert tw.bitnet_get_device_status() == tw.OK


def test_decode_chain_bounded_wait_reports_timeout(tw):
    """A wait that never completes gives up (about 2 s) and is reported, with
    no fault: the done counter in a zero-filled workspace starts at 2^30, so
    it never equals the count CTA 0 waits for at the end (the number of
    CTAs), and only grows, so that count never appears.  (A start below the
    awaited count would not do: the count could pass through it.)  Only CTA
    0 waits on that counter; every link is computed before that and is still
    right, the device status is BITNET_ERR_TIMEOUT, and the launch counter
    is not advanced (zero the workspace again after a timeout, as the header
    says)."""
    steps, Ws = build_chain(tw, SHAPES_A[:2], 31)
    arr = tw.bitnet_decode_chain_steps(steps)
    ws = torch.zeros(tw.bitnet_decode_chain_workspace_size(arr), dtype=torch.uint8, device=DEV)
    ws.view(torch.int32)[128 // 4] = 1 << 30  # the done counter
    assert tw.bitnet_get_device_status() == tw.OK
    x0 = x0_bits(SHAPES_A[0][1], 7)
    tw.bitnet_decode_chain(arr, bf16_t(x0), ws)
    assert tw.bitnet_get_device_status() == tw.ERR_TIMEOUT
    check_links(steps, Ws, x0)
    assert int(ws.view(torch.int32)[0].item()) == 0  # launch counter unchanged
    assert tw.bitnet_get_device_status() == tw.OK   # reading the status cleared it


# ------------------------------------------------------------------ the 30-layer stack
@pytest.fixture(scope="module")
def stack30(tw):
    """The configured 30-layer decode stack (per layer qkv 2560->3840, o
    2560->2560, up 2560->6912 + ReLU^2, down 6912->2560; 1.55 B ternary
    weights): latent weights made one layer at a time, quantised on the GPU
    and by the oracle (codes and gamma must agree), and both chain forms
    sharing the GPU's packed weights.  Also the oracle's own run of the whole
    stack from the chain input."""
    from ternary_weight_linear_token_b200.chain import DecodeChain
    layers = 30
    oracle_layers = []

    def gen():
        for li in range(layers):
            dev_w, proj = [], []
            for p in range(4):
                W = synth.layer_weights(li, p)
                po, go = ref.quantize_weights(W)
                proj.append((po, go, W.shape[0], synth.PROJECTIONS[p][3]))
                dev_w.append((f32_t(W), synth.PROJECTIONS[p][3]))
            oracle_layers.append(proj)
            yield dev_w

    per = DecodeChain(gen())
    for li in range(layers):
        for p in range(4):
            po, go = oracle_layers[li][p][:2]
            assert np.array_equal(np_of(per.layers[li][p]["packed"]), po), (li, p)
            assert np_of(per.layers[li][p]["gamma"])[0] == go, (li, p)
    pers = DecodeChain(None, persistent=True, quantized=per.layers)
    x0 = synth.config_inputs("chain", weights=False)
    want = ref.decode_chain(x0["x"], oracle_layers, per.d)
    return dict(per=per, pers=pers, oracle=oracle_layers, x0=x0, want=want)


def check_stack(chain, oracle_layers, x0_bits):
    """Every link of a chain run: each projection's bf16 output bit-exact
    against the oracle's BitLinear of the projection's actual bf16 input;
    each normalised vector within 1 bf16 ulp of the oracle's normalisation
    of the actual down output.  Returns how many normalised vectors are
    bit-identical to the oracle's."""
    d = chain.d
    x_in = x0_bits.reshape(1, -1)
    exact_norms = 0
    for li, bufs in enumerate(chain.outs):
        inputs = [x_in, bf16_bits_of(bufs[0])[:, :d], bf16_bits_of(bufs[1]), bf16_bits_of(bufs[2])]
        for pi in range(4):
            po, go, N, relu2 = oracle_layers[li][pi]
            xin = synth.bf16_bits_to_f32(inputs[pi])
            want = ref.to_bf16(ref.bitlinear(xin, po, go, N, relu2=relu2)["y"])
            got = bf16_bits_of(bufs[pi])
            bad = np.flatnonzero(got != want)
            assert bad.size == 0, (li, pi, bad[:4], got.ravel()[bad[:4]], want.ravel()[bad[:4]])
        want_n = ref.to_bf16(ref.rms_norm(synth.bf16_bits_to_f32(bf16_bits_of(bufs[3]))))
        got_n = bf16_bits_of(bufs[4])
        assert_bf16_within_ulp(got_n, want_n, 1)
        exact_norms += int(np.array_equal(got_n, want_n))
        x_in = got_n
    return exact_norms


def test_stack30_per_launch_links_and_end_to_end(tw, stack30):
    """The per-launch form (121 launches per token) of the 30-layer stack:
    all 120 BitLinear links and 30 normalisations against the oracle, then
    the whole run against the oracle's own run from the chain input.  The
    normalisation computes the oracle's fp64 sum and factor, so it is
    bit-identical except where two fp64 summation orders straddle an fp32
    rounding boundary of the factor (about 1e-7 per token); with every link
    exact the whole stack then equals the oracle's run bit for bit.  Then a
    CUDA-graph replay of the whole token reproduces the eager run."""
    chain, x0 = stack30["per"], stack30["x0"]
    chain.run(bf16_t(x0["x_bits"]).view(1, -1))
    torch.cuda.synchronize()
    exact = check_stack(chain, stack30["oracle"], x0["x_bits"])
    assert exact >= 29, exact
    if exact == 30:
        for li, (bufs, want) in enumerate(zip(chain.outs, stack30["want"])):
            for pi in range(5):
                assert np.array_equal(bf16_bits_of(bufs[pi]), want[pi]), (li, pi)
    eager = [bf16_bits_of(b).copy() for bufs in chain.outs for b in bufs]
    for bufs in chain.outs:
        for b in bufs:
            b.fill_(float("nan"))
    chain.capture()
    chain.graph.replay()
    torch.cuda.synchronize()
    again = [bf16_bits_of(b) for bufs in chain.outs for b in bufs]
    assert all(np.array_equal(a, b) for a, b in zip(eager, again))
    assert tw.bitnet_get_device_status() == tw.OK


def test_stack30_persistent_links(tw, stack30):
    """The persistent form (one bitnet_decode_chain launch per token, 120
    steps, the weight ring of shared-memory slots wrapping many times) of
    the 30-layer stack: every link against the oracle and the whole first
    run against the oracle's own run (as for the per-launch form), on two
    launches in a row (the second with another input) and on a CUDA-graph
    replay."""
    chain, x0 = stack30["pers"], stack30["x0"]
    for r in range(2):
        bits = x0["x_bits"] if r == 0 else x0_bits(2560, 77)
        chain.run(bf16_t(bits).view(1, -1))
        torch.cuda.synchronize()
        exact = check_stack(chain, stack30["oracle"], bits)
        assert exact >= 29, exact
        if r == 0 and exact == 30:  # the whole run equals the oracle's own run
            for li, (bufs, want) in enumerate(zip(chain.outs, stack30["want"])):
                for pi in range(5):
                    assert np.array_equal(bf16_bits_of(bufs[pi]), want[pi]), (li, pi)
    eager = [bf16_bits_of(b).copy() for bufs in chain.outs for b in bufs]
    chain.capture()
    for bufs in chain.outs:
        for b in bufs:
            b.fill_(float("nan"))
    chain.graph.replay()
    torch.cuda.synchronize()
    assert all(np.array_equal(a, bf16_bits_of(b)) for a, b in
               zip(eager, [b for bufs in chain.outs for b in bufs]))
    assert tw.bitnet_get_device_status() == tw.OK
