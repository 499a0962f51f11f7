"""Helpers shared by the GPU parity tests: move seeded inputs to the device,
run the oracle on the host, compare within the stated tolerances."""

from __future__ import annotations

import numpy as np
import torch

import synth

DEV = "cuda:0"


def f32_t(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def bf16_t(bits: np.ndarray) -> torch.Tensor:
    """bf16 device tensor from uint16 bit patterns (exact)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def x_tensor(d: dict) -> torch.Tensor:
    """The workload's activations in their storage dtype."""
    return bf16_t(d["x_bits"]) if d["x_bits"] is not None else f32_t(d["x"])


def as_x(x: np.ndarray, dtype: str) -> tuple[torch.Tensor, np.ndarray]:
    """Device tensor in `dtype` plus the exact fp32 values the kernel sees."""
    if dtype == "f32":
        return f32_t(x), np.ascontiguousarray(x, dtype=np.float32)
    bits = synth.f32_to_bf16_bits(x)
    return bf16_t(bits), synth.bf16_bits_to_f32(bits)


def bf16_bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def np_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def assert_f32_close(got: np.ndarray, want: np.ndarray, rel: float = 1e-6):
    """fp32 outputs: |got - want| <= rel * |want| element by element."""
    got = np.asarray(got, dtype=np.float32)
    want = np.asarray(want, dtype=np.float32)
    assert got.shape == want.shape
    err = np.abs(got.astype(np.float64) - want.astype(np.float64))
    bound = rel * np.abs(want.astype(np.float64))
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} of {bad.size} fp32 outputs outside {rel} relative; "
                           f"first at {np.argwhere(bad)[0]}: got {got[bad][0]!r} want {want[bad][0]!r}")


def assert_f32_within_ulp(got: np.ndarray, want: np.ndarray, ulps: int):
    """fp32 outputs: at most `ulps` units in the last place apart."""
    g = np.asarray(got, dtype=np.float32).view(np.int32).astype(np.int64)
    w = np.asarray(want, dtype=np.float32).view(np.int32).astype(np.int64)
    assert g.shape == w.shape

    def ordered(b):  # monotone integer image of the fp32 value line
        return np.where(b < 0, -(b & 0x7FFFFFFF), b)
    diff = np.abs(ordered(g) - ordered(w))
    bad = diff > ulps
    assert not bad.any(), (f"{bad.sum()} of {bad.size} fp32 outputs more than {ulps} ulp apart; "
                           f"first at {np.argwhere(bad)[0]}")


def assert_bf16_within_ulp(got_bits: np.ndarray, want_bits: np.ndarray, ulps: int = 1):
    """bf16 outputs: at most `ulps` units in the last place apart (same sign
    or both zero)."""
    g = np.asarray(got_bits, dtype=np.uint16).astype(np.int32)
    w = np.asarray(want_bits, dtype=np.uint16).astype(np.int32)
    assert g.shape == w.shape

    def ordered(b):  # monotone integer image of the bf16 value line
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    diff = np.abs(ordered(g) - ordered(w))
    bad = diff > ulps
    assert not bad.any(), (f"{bad.sum()} of {bad.size} bf16 outputs more than {ulps} ulp apart; "
                           f"first at {np.argwhere(bad)[0]}")


def quantize_weights_both(W: np.ndarray, dtype: str = "f32"):
    """Quantise on the GPU (product) and on the host (oracle) from the same W."""
    import ternary_weight_linear_token_b200 as tw
    from oracle import ref
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(W)
        Wd = bf16_t(bits)
        Wexact = synth.bf16_bits_to_f32(bits)
    else:
        Wd = f32_t(W)
        Wexact = W
    packed_d, gamma_d = tw.bitnet_quantize_weights(Wd)
    packed_o, gamma_o = ref.quantize_weights(Wexact)
    return packed_d, gamma_d, packed_o, gamma_o
