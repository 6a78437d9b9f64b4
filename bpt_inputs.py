"""Seeded synthetic inputs for one BPT layer forward.

This module draws the random tensors that both the fp64 oracle and the GPU
library consume. It holds none of the method's arithmetic: it only produces
x, the projection weights and the biases, rounded to the precision that the
call under test receives.

Generator (a counter-based stream, so any element can be drawn on its own):

* splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): the n-th output of a stream whose state starts
  at ``key`` is ``mix64(key + n * GAMMA)`` for n = 1, 2, ... (mod 2**64),
  with GAMMA = 0x9E3779B97F4A7C15 and mix64 the variant-13 finaliser below.
* Each tensor has its own stream: ``key = mix64(seed * GAMMA + tensor_id + 1)``
  with tensor ids in the fixed order x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2.
* Element j of a tensor takes outputs 2j+1 and 2j+2 of its stream, turns
  each into a uniform double from its top 53 bits, and applies the
  Box-Muller transform (Box and Muller, 1958), keeping the cosine branch:
  ``z = sqrt(-2 ln u1) * cos(2 pi u2)`` with u1 in (0, 1], u2 in [0, 1).
* The normal draw is scaled by the tensor's standard deviation in fp64, then
  rounded to fp32 (round to nearest even) and, for bf16 workloads, from fp32
  to bf16 (round to nearest even).

Distributions (the layer's synthetic workload): x ~ N(0, 1);
weights ~ N(0, 1/fan_in), i.e. std 1/sqrt(fan_in) with fan_in = h for Wqkv,
Wo and W1 and 4h for W2; biases ~ N(0, 0.02**2), i.e. std 0.02.

Weights are stored ``[in, out]`` row-major so that a projection reads
``x @ W`` (the row-vector convention of the position-wise FFN
``max(0, x W1 + b1) W2 + b2``).
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK = (1 << 64) - 1

TENSOR_IDS = {"x": 0, "Wqkv": 1, "bqkv": 2, "Wo": 3, "bo": 4, "W1": 5, "b1": 6, "W2": 7, "b2": 8}

_CHUNK = 1 << 22


def mix64_int(z: int) -> int:
    """splitmix64 finaliser on a Python int (mod 2**64)."""
    z &= _MASK
    z = ((z ^ (z >> 30)) * _M1) & _MASK
    z = ((z ^ (z >> 27)) * _M2) & _MASK
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    return mix64_int(seed * GAMMA + tensor_id + 1)


def _mix64_arr(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
    return z ^ (z >> np.uint64(31))


def _normal_chunk(key: int, start: int, count: int) -> np.ndarray:
    j = np.arange(start, start + count, dtype=np.uint64)
    n1 = j * np.uint64(2) + np.uint64(1)
    with np.errstate(over="ignore"):
        s1 = np.uint64(key) + n1 * np.uint64(GAMMA)
        s2 = s1 + np.uint64(GAMMA)
        r1 = _mix64_arr(s1)
        r2 = _mix64_arr(s2)
    scale = 2.0 ** -53
    u1 = 1.0 - (r1 >> np.uint64(11)).astype(np.float64) * scale
    u2 = (r2 >> np.uint64(11)).astype(np.float64) * scale
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def normal_f64(seed: int, tensor_id: int, n: int, threads: int | None = None) -> np.ndarray:
    """The first n standard-normal draws of a tensor's stream, in fp64."""
    key = stream_key(seed, tensor_id)
    out = np.empty(n, dtype=np.float64)
    starts = list(range(0, n, _CHUNK))
    if len(starts) <= 1:
        if n:
            out[:] = _normal_chunk(key, 0, n)
        return out

    def work(st):
        cnt = min(_CHUNK, n - st)
        out[st:st + cnt] = _normal_chunk(key, st, cnt)

    workers = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=workers) as ex:
        list(ex.map(work, starts))
    return out


def normal_scalar(seed: int, tensor_id: int, j: int) -> float:
    """Draw j of a tensor's stream with plain Python integers (for testing)."""
    key = stream_key(seed, tensor_id)
    r1 = mix64_int(key + (2 * j + 1) * GAMMA)
    r2 = mix64_int(key + (2 * j + 2) * GAMMA)
    u1 = 1.0 - (r1 >> 11) * 2.0 ** -53
    u2 = (r2 >> 11) * 2.0 ** -53
    return math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


@dataclass(frozen=True)
class LayerShape:
    b: int
    s: int
    h: int
    heads: int
    q_block: int
    kv_block: int
    causal: bool
    dtype: str = "bf16"  # "bf16" or "f32": the precision the inputs are rounded to
    ffn: int = 0  # FFN width; 0 means the pages' 4h

    @property
    def dh(self) -> int:
        return self.h // self.heads

    @property
    def f(self) -> int:
        return self.ffn if self.ffn else 4 * self.h


def tensor_shapes(shape: LayerShape) -> dict:
    h, f = shape.h, shape.f
    return {
        "x": (shape.b, shape.s, h),
        "Wqkv": (h, 3 * h), "bqkv": (3 * h,),
        "Wo": (h, h), "bo": (h,),
        "W1": (h, f), "b1": (f,),
        "W2": (f, h), "b2": (h,),
    }


def tensor_std(name: str, shape: LayerShape) -> float:
    if name == "x":
        return 1.0
    if name.startswith("b"):
        return 0.02
    fan_in = shape.f if name == "W2" else shape.h
    return 1.0 / math.sqrt(fan_in)


def make_inputs(shape: LayerShape, seed: int = 0, threads: int | None = None) -> dict:
    """Draw every tensor of the layer.

    Returns a dict name -> array. For dtype "bf16" the arrays are uint16 bf16
    bit patterns; for "f32" they are float32. ``to_f64`` gives the exact
    values as fp64 for the oracle.
    """
    out = {}
    for name, shp in tensor_shapes(shape).items():
        n = int(np.prod(shp))
        v = normal_f64(seed, TENSOR_IDS[name], n, threads) * tensor_std(name, shape)
        v32 = v.astype(np.float32)
        del v
        if shape.dtype == "bf16":
            out[name] = f32_to_bf16_bits(v32).reshape(shp)
        elif shape.dtype == "f32":
            out[name] = v32.reshape(shp)
        else:
            raise ValueError(f"unknown dtype {shape.dtype!r}")
    return out


def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact fp64 values of a generated tensor (bf16 bit patterns or fp32)."""
    if a.dtype == np.uint16:
        return bf16_bits_to_f64(a)
    return a.astype(np.float64)


# The five workloads of the layer forward, by what they are.
WORKLOADS = {
    "small_fp32_s256_h256": LayerShape(1, 256, 256, 4, 64, 64, False, "f32"),
    "causal_b2_s2048_h1024": LayerShape(2, 2048, 1024, 16, 128, 128, True),
    "gpt1b_s8192_h2048": LayerShape(1, 8192, 2048, 16, 512, 512, True),
    "gpt7b_s32768_h4096": LayerShape(1, 32768, 4096, 32, 1024, 2048, True),
}
SWEEP_BLOCKS = (64, 128, 256, 512, 1024, 2048)


def sweep_shape(block: int, causal: bool) -> LayerShape:
    """Block-size sweep point: b 1, s 16384, h 2048, 16 heads of 128."""
    return LayerShape(1, 16384, 2048, 16, block, block, causal)


def to_torch(a: np.ndarray, device="cuda"):
    """A generated tensor as a torch tensor (bf16 for bit patterns, else fp32)."""
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


PARAM_NAMES = ("Wqkv", "bqkv", "Wo", "bo", "W1", "b1", "W2", "b2")


def oracle_args(inp: dict) -> tuple:
    """(x, Wqkv, bqkv, Wo, bo, W1, b1, W2, b2) as exact fp64 arrays."""
    return tuple(to_f64(inp[k]) for k in ("x",) + PARAM_NAMES)
