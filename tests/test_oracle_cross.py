"""C oracle vs the independent numpy restatement, bit for bit, on the
workloads' own seeded inputs (sizes the CPU finishes in seconds)."""

import numpy as np
import pytest

from oracle import ref, ref_np
import synth


def _cases():
    yield "tiny", synth.config_inputs("tiny")
    yield "decode", synth.config_inputs("decode")
    yield "sweep_up_M8", synth.config_inputs("sweep", M=8, proj=2)
    yield "sweep_down_M1", synth.config_inputs("sweep", M=1, proj=3)
    d = synth.config_inputs("prefill")
    d["x"] = d["x"][:8]
    d["M"] = 8
    yield "prefill_rows0_8", d


@pytest.mark.parametrize("name,d", list(_cases()), ids=lambda v: v if isinstance(v, str) else "")
def test_c_vs_numpy(name, d):
    R = ref.default()
    W, X, N, K = d["W"], d["x"], d["N"], d["K"]
    p_c, g_c = R.quantize_weights(W)
    p_n, g_n = ref_np.quantize_weights(W)
    assert g_c == g_n
    assert np.array_equal(p_c, p_n)
    out_c = R.bitlinear(X, p_c, g_c, N, relu2=d["relu2"])
    out_n = ref_np.bitlinear(X, p_n, g_n, K, relu2=d["relu2"])
    for key in ("xq", "s", "acc", "y"):
        assert np.array_equal(out_c[key], out_n[key]), key
    assert np.array_equal(R.to_bf16(out_c["y"]), ref_np.to_bf16(out_n["y"]))


def test_generator_recipe():
    """The seeded inputs have the recipe's shapes and distributions."""
    d = synth.config_inputs("decode")
    assert d["x"].shape == (1, 2560) and d["W"].shape == (2560, 2560)
    assert d["x_bits"] is not None and d["x_bits"].dtype == np.uint16
    assert np.array_equal(synth.bf16_bits_to_f32(d["x_bits"]), d["x"])
    big = np.abs(d["x"]) > 6
    assert 0 < big.sum() < 12  # ~0.1% of 2560 entries scaled by 20
    t = synth.config_inputs("tiny")
    assert t["x_bits"] is None and t["W"].dtype == np.float32
    again = synth.config_inputs("tiny")
    assert np.array_equal(t["W"], again["W"]) and np.array_equal(t["x"], again["x"])
