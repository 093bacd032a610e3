"""Seeded synthetic inputs for the layer-pruning path.

This module only draws random numbers and rounds them to the storage type.  It
holds none of the pruning arithmetic, so both the CUDA path and the fp64
oracle can consume the same bytes without sharing any of the method.

Every draw is addressable: row ``k`` of ``W`` comes from
``default_rng([seed, 0, k])`` (layer ``l > 0`` of a decoder block:
``default_rng([seed, 100 + l, k])``) and feature row ``i`` of the activations of
input ``a`` (the pages' ``X`` is ``b x n`` with examples as columns, "Pruning LLMs
with Thanos", section "The layer-reconstruction lens") comes from
``default_rng([seed, 1 + a, i])``, so any subset of rows can be regenerated
without drawing the rest.  Outlier features are chosen by
``default_rng([seed, 99, a])``.

Workloads mirror the shapes the pages work with: LLaMA-7B linear layers and a
calibration set of 2048-token sequences (128 sequences of C4 on the pages;
here fewer Gaussian or Laplace sequences stand in for that dataset).
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "workload", "make_W", "make_X_features",
    "make_X_tokens", "f64_to_bf16_bits", "bf16_bits_to_f64", "bf16_bits_to_f32",
    "custom", "decoder_block", "BLOCK_INPUTS", "BLOCK_LAYERS",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    c: int                 # output rows of W
    b: int                 # input features (columns of W, rows of the pages' X)
    n: int                 # calibration tokens
    dtype: str             # "fp32" or "bf16" storage of W and X
    x_dist: str            # "gaussian" or "laplace"
    outlier_frac: float    # fraction of input features scaled up
    outlier_scale: float
    pattern: str           # "unstructured" or "nm"
    nm: tuple              # (n, m) for N:M
    sparsity: float
    block: int
    damp: float = 0.01
    seed: int = 0
    input_id: int = 0      # which activation stream feeds this layer
    w_id: int = 0          # which weight stream (layers of one decoder block differ)


WORKLOADS = {
    # single fp32 layer, small enough for the oracle to finish in well under a second
    "layer128x256_fp32": Workload("layer128x256_fp32", 128, 256, 512, "fp32", "gaussian",
                                  0.02, 20.0, "unstructured", (0, 0), 0.5, 32),
    # LLaMA-7B-shaped q_proj, 8 x 2048 tokens
    "q_proj4096x4096": Workload("q_proj4096x4096", 4096, 4096, 16384, "bf16", "gaussian",
                                0.005, 50.0, "unstructured", (0, 0), 0.5, 128),
    # LLaMA-7B-shaped up_proj, 16 x 2048 tokens, 2:4
    "up_proj11008x4096_2of4": Workload("up_proj11008x4096_2of4", 11008, 4096, 32768, "bf16",
                                       "gaussian", 0.005, 50.0, "nm", (2, 4), 0.5, 128),
    # LLaMA-7B-shaped down_proj, 16 x 2048 tokens of heavy-tailed activations, 4:8
    "down_proj4096x11008_4of8": Workload("down_proj4096x11008_4of8", 4096, 11008, 32768, "bf16",
                                         "laplace", 0.0, 1.0, "nm", (4, 8), 0.5, 128),
}


# One LLaMA-7B-shaped decoder block, 128 x 2048 calibration tokens: four activation
# inputs (q, k, v read the attention input; gate and up the MLP input) and seven layers,
# all at 50% unstructured with the global budget, B = 128.
BLOCK_TOKENS = 128 * 2048
BLOCK_INPUTS = {          # name: (b, distribution, outlier fraction, outlier scale, input id)
    "attn_in": (4096, "gaussian", 0.005, 50.0, 1),
    "o_in": (4096, "gaussian", 0.005, 50.0, 2),
    "mlp_in": (4096, "gaussian", 0.005, 50.0, 3),
    "down_in": (11008, "laplace", 0.0, 1.0, 4),
}
BLOCK_LAYERS = [          # (name, input, c); the layer's index is its weight stream
    ("q_proj", "attn_in", 4096), ("k_proj", "attn_in", 4096), ("v_proj", "attn_in", 4096),
    ("o_proj", "o_in", 4096), ("gate_proj", "mlp_in", 11008), ("up_proj", "mlp_in", 11008),
    ("down_proj", "down_in", 4096),
]


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def decoder_block(n: int = BLOCK_TOKENS):
    """{layer name: (input name, Workload)} of the decoder block; layers that read the
    same input have identical activation parameters, so make_X_tokens gives one X."""
    out = {}
    for l, (name, inp, c) in enumerate(BLOCK_LAYERS):
        b, dist, frac, scale, a = BLOCK_INPUTS[inp]
        out[name] = (inp, Workload(f"block_{name}", c, b, n, "bf16", dist, frac, scale, "unstructured",
                                   (0, 0), 0.5, 128, 0.01, 0, a, l))
    return out


def custom(c, b, n, dtype="fp32", x_dist="gaussian", outlier_frac=0.0, outlier_scale=1.0,
           pattern="unstructured", nm=(0, 0), sparsity=0.5, block=32, damp=0.01, seed=0,
           input_id=0, name="custom") -> Workload:
    return Workload(name, c, b, n, dtype, x_dist, outlier_frac, outlier_scale, pattern,
                    tuple(nm), sparsity, block, damp, seed, input_id)


# ---------------------------------------------------------------------------- storage rounding

def f64_to_bf16_bits(x) -> np.ndarray:
    """Round fp64 values once, to nearest-even, to bfloat16; return the 16-bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    bits = x.view(np.uint64)
    drop = np.uint64(45)                      # 52 fp64 mantissa bits -> 7 bf16 mantissa bits
    lower = bits & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    keep = bits >> drop
    up = (lower > half) | ((lower == half) & ((keep & np.uint64(1)) == np.uint64(1)))
    keep = keep + up.astype(np.uint64)
    y = (keep << drop).view(np.float64)
    ay = np.abs(y)
    if np.any((ay != 0) & (ay < 1.1754943508222875e-38)) or np.any(ay > 3.3e38):
        raise ValueError("value outside the normal bfloat16 range")
    return (y.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(u16) -> np.ndarray:
    u = np.ascontiguousarray(u16, dtype=np.uint16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(u16) -> np.ndarray:
    return bf16_bits_to_f32(u16).astype(np.float64)


def _store(x64: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "fp32":
        return x64.astype(np.float32)
    if dtype == "bf16":
        return f64_to_bf16_bits(x64)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------- draws

def make_W(wl: Workload, rows=None) -> np.ndarray:
    """W (c x b), rows ~ N(0, 0.02^2); fp32 array or bf16 bit patterns (uint16)."""
    rows = range(wl.c) if rows is None else rows
    rows = list(rows)
    out = np.empty((len(rows), wl.b), dtype=np.float64)
    stream = 0 if wl.w_id == 0 else 100 + wl.w_id
    for i, k in enumerate(rows):
        out[i] = np.random.default_rng([wl.seed, stream, int(k)]).normal(0.0, 0.02, wl.b)
    return _store(out, wl.dtype)


def outlier_features(wl: Workload) -> np.ndarray:
    k = int(round(wl.outlier_frac * wl.b))
    if k == 0:
        return np.zeros(0, dtype=np.int64)
    rng = np.random.default_rng([wl.seed, 99, wl.input_id])
    return np.sort(rng.choice(wl.b, size=k, replace=False))


def _feature_row(wl: Workload, i: int, scale: float) -> np.ndarray:
    rng = np.random.default_rng([wl.seed, 1 + wl.input_id, int(i)])
    if wl.x_dist == "gaussian":
        v = rng.normal(0.0, 1.0, wl.n)
    elif wl.x_dist == "laplace":
        # unit-variance Laplace; 30% of entries shrunk by 1e-2 (near-zero gate outputs)
        v = rng.laplace(0.0, 1.0 / np.sqrt(2.0), wl.n)
        near_zero = rng.random(wl.n) < 0.3
        v = np.where(near_zero, v * 1e-2, v)
    else:
        raise ValueError(wl.x_dist)
    return v * scale


def make_X_features(wl: Workload, features=None) -> np.ndarray:
    """Feature rows of the pages' X (b x n): shape [len(features), n], storage dtype."""
    feats = range(wl.b) if features is None else features
    feats = list(feats)
    outl = set(outlier_features(wl).tolist())
    out = np.empty((len(feats), wl.n), dtype=np.float64)
    for r, i in enumerate(feats):
        out[r] = _feature_row(wl, i, wl.outlier_scale if i in outl else 1.0)
    return _store(out, wl.dtype)


def make_X_tokens(wl: Workload, chunk: int = 512, threads: int = 1) -> np.ndarray:
    """Token-major activations [n, b] (PyTorch activation layout), storage dtype.  With
    threads > 1 feature chunks are drawn concurrently (each feature row has its own
    generator, so the result is the same)."""
    dt = np.float32 if wl.dtype == "fp32" else np.uint16
    out = np.empty((wl.n, wl.b), dtype=dt)

    def fill(f0, f1):
        out[:, f0:f1] = make_X_features(wl, range(f0, f1)).T

    if threads <= 1:
        for f0 in range(0, wl.b, chunk):
            fill(f0, min(wl.b, f0 + chunk))
        return out
    step = 64
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(lambda f0: fill(f0, min(wl.b, f0 + step)), range(0, wl.b, step)))
    return out


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values to fp64."""
    return bf16_bits_to_f64(a) if dtype == "bf16" else np.asarray(a, dtype=np.float64)
