"""Seeded synthetic inputs for the top-k MoE FFN forward.

This module only draws numbers and names shapes.  It holds none of the
layer's arithmetic (no routing, no softmax, no expert maths), so both the
float64 oracle and the CUDA path can be fed from it without sharing any
computation.

Workloads follow the shapes of the published problems:

* the Flax exercise "Mixture-of-Experts FFN" (crackedaicode.com, section
  "Problem"): Dense(F)->ReLU->Dense(D) experts with biases and a biased
  Dense(E) router, x float32 of shape (T, D);
* mojolearn.MoEBlock (section "Examples"): a Mixtral-style SiLU-gated block
  whose example input is ``default_rng(0).random((4, 16, 64), float32)``;
* three bf16 layers of Mixtral-8x7B, fine-grained many-expert and decode
  shapes.

Recipe:

* small float32 workloads draw from ONE ``numpy.random.default_rng(seed)``
  in the order x, router, [router_bias], gate_up_proj, down_proj, [b1, b2];
* large bf16 workloads draw each tensor in fixed 4 Mi-element chunks, chunk
  ``c`` of tensor ``i`` from ``default_rng([seed, i, c])``, so the values do
  not depend on how many threads produce them; float32 draws are rounded to
  bf16 (round to nearest, ties to even) once.
* weights ~ N(0, 0.02^2); biases 0.01*N(0, 1); x ~ U[0, 1) (float32
  workloads) or N(0, 1) (bf16 workloads); the fine-grained workload adds a
  fixed router bias 2*log(1/rank) = -2*ln(e+1) that skews expert load.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from functools import lru_cache

import numpy as np

WEIGHT_STD = 0.02
BIAS_SCALE = 0.01
CHUNK = 1 << 22

ACT_SILU_GATED = "silu_gated"
ACT_RELU = "relu"


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    D: int
    F: int
    E: int
    K: int
    act: str
    dtype: str              # "f32" or "bf16": the dtype of x, weights and out
    norm_topk_prob: bool
    seed: int
    x_dist: str             # "uniform01" or "normal"
    x_shape: tuple = field(default=())
    router_offset: str | None = None   # "zipf": -2*ln(e+1)
    biases: bool = False    # Dense/ReLU experts carry b1, b2 and a router bias

    @property
    def R(self) -> int:
        """Routed rows, T*K."""
        return self.T * self.K

    @property
    def shape_x(self) -> tuple:
        return self.x_shape if self.x_shape else (self.T, self.D)

    def with_K(self, K: int, name: str | None = None) -> "Workload":
        d = dict(self.__dict__)
        d["K"] = K
        d["name"] = name or f"{self.name}_k{K}"
        return Workload(**d)

    def routed_flops(self) -> float:
        """Routed FLOPs of one forward: experts on the selected rows only,
        plus the router; bias adds are not counted."""
        per_row = 6 * self.D * self.F if self.act == ACT_SILU_GATED else 4 * self.D * self.F
        return float(self.R * per_row + 2 * self.T * self.D * self.E)


WORKLOADS: dict[str, Workload] = {}


def _reg(w: Workload) -> Workload:
    WORKLOADS[w.name] = w
    return w


# The Flax exercise: Dense/ReLU experts with biases, router Dense(E)+bias.
DENSE_RELU = _reg(Workload(
    name="dense_relu_t64_d32_f64_e4_k2_f32", T=64, D=32, F=64, E=4, K=2,
    act=ACT_RELU, dtype="f32", norm_topk_prob=True, seed=0,
    x_dist="uniform01", biases=True))

# mojolearn.MoEBlock(64, 128, 8, 2) on its own example input (4, 16, 64).
SILU_SMALL = _reg(Workload(
    name="silu_gated_t64_d64_f128_e8_k2_f32", T=64, D=64, F=128, E=8, K=2,
    act=ACT_SILU_GATED, dtype="f32", norm_topk_prob=True, seed=0,
    x_dist="uniform01", x_shape=(4, 16, 64)))

# One Mixtral-8x7B-shaped layer.
MIXTRAL = _reg(Workload(
    name="mixtral8x7b_t4096_d4096_f14336_e8_k2_bf16", T=4096, D=4096, F=14336,
    E=8, K=2, act=ACT_SILU_GATED, dtype="bf16", norm_topk_prob=True, seed=1,
    x_dist="normal"))

# Fine-grained many-expert layer with a Zipf-skewed expert load.
FINE_GRAINED = _reg(Workload(
    name="fine_grained_t16384_d2048_f1408_e64_k6_zipf_bf16", T=16384, D=2048,
    F=1408, E=64, K=6, act=ACT_SILU_GATED, dtype="bf16", norm_topk_prob=True,
    seed=2, x_dist="normal", router_offset="zipf"))

# A Mixtral-shaped layer cut to 2 experts (704 MB of weights, still larger
# than L2): the size at which a full counter capture of one grouped-GEMM
# launch stays within a few GB of device memory.
MIXTRAL_E2 = _reg(Workload(
    name="mixtral_shape_t2048_d4096_f14336_e2_k2_bf16", T=2048, D=4096, F=14336, E=2, K=2,
    act=ACT_SILU_GATED, dtype="bf16", norm_topk_prob=True, seed=5, x_dist="normal"))

# The same cut with 1024 routed rows per expert, as in the Mixtral layer.
MIXTRAL_E2_T1024 = _reg(Workload(
    name="mixtral_shape_t1024_d4096_f14336_e2_k2_bf16", T=1024, D=4096, F=14336, E=2, K=2,
    act=ACT_SILU_GATED, dtype="bf16", norm_topk_prob=True, seed=5, x_dist="normal"))

# Decode-like weight streaming: 32 tokens, swept over top_k.
DECODE = {k: _reg(Workload(
    name=f"decode_t32_d4096_f14336_e8_k{k}_bf16", T=32, D=4096, F=14336, E=8,
    K=k, act=ACT_SILU_GATED, dtype="bf16", norm_topk_prob=True, seed=3,
    x_dist="normal")) for k in (1, 2, 8)}


# ---------------------------------------------------------------- bf16 bits
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits (uint16) to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def as_float32(a: np.ndarray) -> np.ndarray:
    """float32 view of an input array: bf16 bits are widened exactly."""
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a)
    return np.asarray(a, dtype=np.float32)


# ------------------------------------------------------------ chunked draws
def _chunked_bf16(seed: int, tensor_id: int, shape: tuple, kind: str,
                  scale: float) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    nchunks = (n + CHUNK - 1) // CHUNK

    def work(c: int) -> None:
        lo, hi = c * CHUNK, min(n, (c + 1) * CHUNK)
        rng = np.random.default_rng([seed, tensor_id, c])
        if kind == "normal":
            v = rng.standard_normal(hi - lo, dtype=np.float32)
        else:
            v = rng.random(hi - lo, dtype=np.float32)
        if scale != 1.0:
            v *= np.float32(scale)
        out[lo:hi] = f32_to_bf16_bits(v)

    workers = max(1, min(nchunks, os.cpu_count() or 1))
    if workers == 1:
        for c in range(nchunks):
            work(c)
    else:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(work, range(nchunks)))
    return out.reshape(shape)


def zipf_router_offset(E: int) -> np.ndarray:
    """The fixed per-expert logit offset 2*log(1/rank), rank = e+1."""
    return (2.0 * np.log(1.0 / np.arange(1, E + 1, dtype=np.float64))).astype(np.float32)


def _make(w: Workload) -> dict:
    gu_rows = 2 * w.F if w.act == ACT_SILU_GATED else w.F
    if w.dtype == "f32":
        rng = np.random.default_rng(w.seed)
        if w.x_dist == "uniform01":
            x = rng.random(w.shape_x, dtype=np.float32)
        else:
            x = rng.standard_normal(w.shape_x, dtype=np.float32)
        router = (rng.standard_normal((w.E, w.D), dtype=np.float32) * np.float32(WEIGHT_STD))
        router_bias = None
        if w.biases:
            router_bias = rng.standard_normal(w.E, dtype=np.float32) * np.float32(BIAS_SCALE)
        gate_up = rng.standard_normal((w.E, gu_rows, w.D), dtype=np.float32) * np.float32(WEIGHT_STD)
        down = rng.standard_normal((w.E, w.D, w.F), dtype=np.float32) * np.float32(WEIGHT_STD)
        b1 = b2 = None
        if w.biases:
            b1 = rng.standard_normal((w.E, w.F), dtype=np.float32) * np.float32(BIAS_SCALE)
            b2 = rng.standard_normal((w.E, w.D), dtype=np.float32) * np.float32(BIAS_SCALE)
    else:
        kind = "random" if w.x_dist == "uniform01" else "normal"
        x = _chunked_bf16(w.seed, 0, w.shape_x, kind, 1.0)
        router = _chunked_bf16(w.seed, 1, (w.E, w.D), "normal", WEIGHT_STD)
        gate_up = _chunked_bf16(w.seed, 2, (w.E, gu_rows, w.D), "normal", WEIGHT_STD)
        down = _chunked_bf16(w.seed, 3, (w.E, w.D, w.F), "normal", WEIGHT_STD)
        router_bias = b1 = b2 = None
        if w.biases:
            rng = np.random.default_rng([w.seed, 4])
            router_bias = rng.standard_normal(w.E, dtype=np.float32) * np.float32(BIAS_SCALE)
            b1 = rng.standard_normal((w.E, w.F), dtype=np.float32) * np.float32(BIAS_SCALE)
            b2 = rng.standard_normal((w.E, w.D), dtype=np.float32) * np.float32(BIAS_SCALE)
    if w.router_offset == "zipf":
        off = zipf_router_offset(w.E)
        router_bias = off if router_bias is None else (router_bias + off).astype(np.float32)
    return {"x": x, "router": router, "router_bias": router_bias,
            "gate_up_proj": gate_up, "down_proj": down, "b1": b1, "b2": b2}


@lru_cache(maxsize=4)
def _cached(T: int, D: int, F: int, E: int, act: str, dtype: str,
            seed: int, x_dist: str, x_shape: tuple, router_offset, biases) -> dict:
    w = Workload(name="", T=T, D=D, F=F, E=E, K=1, act=act, dtype=dtype,
                 norm_topk_prob=True, seed=seed, x_dist=x_dist, x_shape=x_shape,
                 router_offset=router_offset, biases=biases)
    d = _make(w)
    for v in d.values():
        if v is not None:
            v.setflags(write=False)
    return d


def make_inputs(w: Workload) -> dict:
    """Inputs of workload ``w`` as numpy arrays (bf16 as uint16 bits).

    K does not enter the draw, so the decode sweep over top_k shares one set
    of tensors.  Arrays are cached and read-only."""
    return _cached(w.T, w.D, w.F, w.E, w.act, w.dtype, w.seed, w.x_dist,
                   tuple(w.x_shape), w.router_offset, w.biases)


def random_case(seed: int, T: int, D: int, F: int, E: int, act: str = ACT_SILU_GATED,
                dtype: str = "f32", biases: bool | None = None,
                x_dist: str = "normal", weight_std: float = 0.1) -> dict:
    """A small seeded case of arbitrary shape (property and edge-case tests)."""
    rng = np.random.default_rng(seed)
    if biases is None:
        biases = act == ACT_RELU
    gu_rows = 2 * F if act == ACT_SILU_GATED else F
    if x_dist == "uniform01":
        x = rng.random((T, D), dtype=np.float32)
    else:
        x = rng.standard_normal((T, D), dtype=np.float32)
    router = rng.standard_normal((E, D), dtype=np.float32) * np.float32(weight_std)
    gate_up = rng.standard_normal((E, gu_rows, D), dtype=np.float32) * np.float32(weight_std)
    down = rng.standard_normal((E, D, F), dtype=np.float32) * np.float32(weight_std)
    rb = b1 = b2 = None
    if biases:
        rb = rng.standard_normal(E, dtype=np.float32) * np.float32(BIAS_SCALE * 10)
        b1 = rng.standard_normal((E, F), dtype=np.float32) * np.float32(BIAS_SCALE * 10)
        b2 = rng.standard_normal((E, D), dtype=np.float32) * np.float32(BIAS_SCALE * 10)
    d = {"x": x, "router": router, "router_bias": rb, "gate_up_proj": gate_up,
         "down_proj": down, "b1": b1, "b2": b2}
    if dtype == "bf16":
        for k in ("x", "router", "gate_up_proj", "down_proj"):
            d[k] = f32_to_bf16_bits(d[k])
    return d
