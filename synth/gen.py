"""Seeded input generators for the five BitLinear workloads.

Every tensor is drawn from its own numpy ``Generator`` whose seed is
``SeedSequence(0, spawn_key=(workload, layer, projection, role))``, so a tensor
can be regenerated alone, in any order, on any machine.  The tiny workload
follows its stated recipe literally: ``default_rng(0)``, weights first, then
activations.

Distributions (the workload recipe, not the method):

* latent weights: N(0, 0.02) in fp32.  Absmean quantisation of such a matrix
  leaves about 31% zeros (2*Phi(0.5*sqrt(2/pi)) - 1 = 0.3101).
* tiny activations: N(0, 1) fp32.
* decode activations: N(0, 1), with each entry independently multiplied by 20
  with probability 0.001 (outliers), then rounded to bf16.
* sweep / chain activations: Student-t with 3 degrees of freedom, bf16.
* prefill activations: N(0, 1), bf16.

Rounding to bf16 here is input preparation (round-to-nearest-even on the fp32
bit pattern); nothing in this module quantises, packs or multiplies the way the
method does.
"""

from __future__ import annotations

import numpy as np

# (name, in_features K, out_features N, relu2 epilogue) of one decoder layer's
# BitLinear projections, in the order a token passes through them.
PROJECTIONS = (
    ("qkv", 2560, 3840, False),
    ("o", 2560, 2560, False),
    ("up", 2560, 6912, True),
    ("down", 6912, 2560, False),
)

CONFIGS = {
    "tiny": dict(index=0, M=4, K=256, N=512, x="normal", x_dtype="f32", y_dtype="f32"),
    "decode": dict(index=1, M=1, K=2560, N=2560, x="normal_outliers", x_dtype="bf16", y_dtype="bf16"),
    "sweep": dict(index=2, Ms=(1, 8, 32), x="student_t", x_dtype="bf16", y_dtype="bf16"),
    "prefill": dict(index=3, M=4096, K=2560, N=6912, x="normal", x_dtype="bf16", y_dtype="bf16"),
    "chain": dict(index=4, M=1, layers=30, x="student_t", x_dtype="bf16", y_dtype="bf16"),
}

ROLE_W = 0
ROLE_X = 1


def rng_for(*key: int) -> np.random.Generator:
    """Independent generator for one tensor, keyed by small non-negative ints."""
    return np.random.default_rng(np.random.SeedSequence(0, spawn_key=tuple(int(k) for k in key)))


# ---------------------------------------------------------------- bf16 storage
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = ((u[nan] >> np.uint64(16)) | np.uint64(0x0040)).astype(np.uint16)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------- draws
def latent_weights(rng: np.random.Generator, N: int, K: int, sigma: float = 0.02) -> np.ndarray:
    """Latent (pre-quantisation) weight matrix [N, K] fp32 ~ N(0, sigma)."""
    return rng.standard_normal((N, K), dtype=np.float32) * np.float32(sigma)


def acts_normal(rng: np.random.Generator, M: int, K: int) -> np.ndarray:
    return rng.standard_normal((M, K), dtype=np.float32)


def acts_normal_outliers(rng: np.random.Generator, M: int, K: int,
                         frac: float = 0.001, scale: float = 20.0) -> np.ndarray:
    x = rng.standard_normal((M, K), dtype=np.float32)
    hit = rng.random((M, K)) < frac
    x[hit] *= np.float32(scale)
    return x


def acts_student_t(rng: np.random.Generator, M: int, K: int, df: float = 3.0) -> np.ndarray:
    return rng.standard_t(df, size=(M, K)).astype(np.float32)


_ACTS = {"normal": acts_normal, "normal_outliers": acts_normal_outliers, "student_t": acts_student_t}


def _as_storage(x: np.ndarray, dtype: str) -> dict:
    if dtype == "f32":
        return {"x": x, "x_bits": None}
    bits = f32_to_bf16_bits(x)
    return {"x": bf16_bits_to_f32(bits), "x_bits": bits}


def config_inputs(name: str, M: int | None = None, proj: int = 0, layer: int = 0,
                  weights: bool = True) -> dict:
    """Inputs of one BitLinear call of a workload.

    Returns ``W`` (fp32 [N, K]), ``x`` (fp32 [M, K], the exact values the
    kernel sees), ``x_bits`` (uint16 bf16 bits or None), and the shape / dtype
    metadata.  For "sweep" and "chain", ``proj`` indexes PROJECTIONS and
    ``layer`` the decoder layer (chain only).
    """
    cfg = CONFIGS[name]
    idx = cfg["index"]
    if name == "tiny":
        rng = np.random.default_rng(0)
        N, K, M = cfg["N"], cfg["K"], cfg["M"]
        W = latent_weights(rng, N, K)
        x = acts_normal(rng, M, K)
        out = dict(W=W, **_as_storage(x, "f32"), M=M, N=N, K=K, relu2=False,
                   x_dtype="f32", y_dtype="f32")
        return out
    if name in ("decode", "prefill"):
        N, K = cfg["N"], cfg["K"]
        M = cfg["M"] if M is None else M
        relu2 = False
    else:
        pname, K, N, relu2 = PROJECTIONS[proj]
        M = (cfg["M"] if name == "chain" else (M if M is not None else cfg["Ms"][0]))
    W = latent_weights(rng_for(idx, layer, proj, ROLE_W), N, K) if weights else None
    x = _ACTS[cfg["x"]](rng_for(idx, layer, proj, ROLE_X, M), M, K)
    out = dict(W=W, **_as_storage(x, cfg["x_dtype"]), M=M, N=N, K=K, relu2=relu2,
               x_dtype=cfg["x_dtype"], y_dtype=cfg["y_dtype"])
    return out


def layer_weights(layer: int, proj: int) -> np.ndarray:
    """Latent weights of one projection of one layer of the 30-layer chain."""
    _, K, N, _ = PROJECTIONS[proj]
    return latent_weights(rng_for(CONFIGS["chain"]["index"], layer, proj, ROLE_W), N, K)
