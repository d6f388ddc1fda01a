"""Seeded synthetic inputs for the LiftQuant decode operator.

This module only draws random numbers and rounds them to the storage dtypes;
it holds none of the operator's arithmetic. Both the CUDA path and the CPU
oracle take their inputs from here.

Recipe (fixed draw order, numpy PCG64):
  weights generator  PCG64([seed, layer])        : sign, M, bits, s
  input generator    PCG64([seed, layer, batch]) : x, then outlier positions
  sign  in {+1,-1}^K, uniform                   (whitening sign vector sigma)
  M     [d][D] float32 ~ N(0, 1/D)              (mapping matrix)
  b     [N][G*D] int8 in {+1,-1}, uniform       (stored lifted codes, G = ceil(K/d))
  s     [N] ~ U(0.5, 1.5) (divided by sqrt(K) where the workload says so), rounded to
        the storage dtype
  x     [batch][K] ~ N(0, 1) drawn in float32; optional outliers: on even token rows,
        round(0.01*K) distinct positions multiplied by 20; then rounded (round to nearest
        even) to the storage dtype.
The layer shapes are those of Llama-2-7B / Llama-3-70B linear layers; no trained weights
or datasets are involved.
"""
from dataclasses import dataclass, field
import math

import numpy as np
import torch

F32, F16, BF16 = "f32", "f16", "bf16"


def round_to(x_f32: np.ndarray, dtype: str):
    """Round float32 values to a storage dtype; returns (raw array, exact float32 values).

    raw is float32 / float16, or uint16 holding bf16 bit patterns.
    """
    x_f32 = np.ascontiguousarray(x_f32, dtype=np.float32)
    if dtype == F32:
        return x_f32, x_f32
    if dtype == F16:
        h = x_f32.astype(np.float16)
        return h, h.astype(np.float32)
    if dtype == BF16:
        t = torch.from_numpy(x_f32).to(torch.bfloat16)
        raw = t.view(torch.int16).numpy().view(np.uint16).copy()
        return raw, t.to(torch.float32).numpy()
    raise ValueError(dtype)


def random_signs(rng, shape):
    """Uniform +1/-1 int8 entries drawn from random bytes."""
    n = int(np.prod(shape))
    raw = np.frombuffer(rng.bytes((n + 7) // 8), dtype=np.uint8)
    bits = np.unpackbits(raw)[:n]
    return (1 - 2 * bits.astype(np.int8)).reshape(shape)


@dataclass
class Layer:
    """One synthetic quantized linear layer and a batch of inputs for it."""
    name: str
    K: int
    N: int
    d: int
    D: int
    block: int              # Hadamard block of T (0 = identity)
    sign: np.ndarray        # [K] int8 +1/-1
    M: np.ndarray           # [d][D] float32
    b: np.ndarray           # [N][G*D] int8 +1/-1 (None if not materialised)
    s_raw: np.ndarray       # [N] float16 or float32
    s_dtype: str
    s: np.ndarray           # [N] float32, exact values of s_raw
    x_raw: np.ndarray       # [batch][K] float32 / float16 / uint16(bf16 bits)
    x_dtype: str
    x: np.ndarray           # [batch][K] float32, exact values of x_raw
    chan_scale: np.ndarray = None
    meta: dict = field(default_factory=dict)

    @property
    def G(self):
        return (self.K + self.d - 1) // self.d

    @property
    def lifted(self):
        return self.G * self.D

    @property
    def batch(self):
        return self.x.shape[0]


def make_weights(seed, layer, K, N, d, D, s_dtype=F16, s_div_sqrt_k=True, with_bits=True):
    rng = np.random.Generator(np.random.PCG64([seed, layer]))
    sign = random_signs(rng, (K,))
    M = (rng.standard_normal((d, D)) / math.sqrt(D)).astype(np.float32)
    G = (K + d - 1) // d
    b = random_signs(rng, (N, G * D)) if with_bits else None
    if not with_bits:
        rng.bytes((N * G * D + 7) // 8)          # keep the draw order of s unchanged
    s = rng.uniform(0.5, 1.5, N)
    if s_div_sqrt_k:
        s = s / math.sqrt(K)
    s_raw, s_exact = round_to(s.astype(np.float32), s_dtype)
    return sign, M, b, s_raw, s_exact


def make_inputs(seed, layer, batch, K, x_dtype=BF16, outliers=False):
    rng = np.random.Generator(np.random.PCG64([seed, layer, batch]))
    x = rng.standard_normal((batch, K)).astype(np.float32)
    if outliers:
        n_out = int(round(0.01 * K))
        for t in range(0, batch, 2):
            pos = rng.choice(K, size=n_out, replace=False)
            x[t, pos] *= 20.0
    return round_to(x, x_dtype)


def make_layer(name, seed, layer, K, N, d, D, batch, block=256, x_dtype=BF16, s_dtype=F16,
               s_div_sqrt_k=True, outliers=False, with_bits=True):
    sign, M, b, s_raw, s = make_weights(seed, layer, K, N, d, D, s_dtype, s_div_sqrt_k,
                                        with_bits)
    x_raw, x = make_inputs(seed, layer, batch, K, x_dtype, outliers)
    return Layer(name=name, K=K, N=N, d=d, D=D, block=block, sign=sign, M=M, b=b,
                 s_raw=s_raw, s_dtype=s_dtype, s=s, x_raw=x_raw, x_dtype=x_dtype, x=x,
                 meta=dict(seed=seed, layer=layer, outliers=outliers))


# The five workloads: (name, seed, layer, K, N, d, D, batch, extra kwargs).
SWEEP_CODES = [(1, 2), (2, 4), (2, 5), (3, 8), (10, 24), (10, 25), (4, 12)]


def workload_specs(cfg: int):
    """Layer specs of one workload, in a fixed order."""
    if cfg == 1:
        return [("tiny_256x128_d2D5_b1", 0, 0, 256, 128, 2, 5, 1,
                 dict(x_dtype=F32, s_dtype=F32, s_div_sqrt_k=False))]
    if cfg == 2:
        return [("llama2_7b_qproj_4096x4096_d10D24_b1", 1, 0, 4096, 4096, 10, 24, 1, {})]
    if cfg == 3:
        out = []
        for li, (nm, K, N) in enumerate([("gateup", 8192, 28672), ("down", 28672, 8192)]):
            for bt in (1, 4, 16):
                out.append((f"llama3_70b_{nm}_{K}x{N}_d10D24_b{bt}", 2, li, K, N, 10, 24, bt,
                            {}))
        return out
    if cfg == 4:
        out = []
        for li, (d, D) in enumerate(SWEEP_CODES):
            for bt in (1, 8):
                out.append((f"sweep_8192x8192_d{d}D{D}_b{bt}", 3, li, 8192, 8192, d, D, bt,
                            dict(outliers=True)))
        return out
    if cfg == 5:
        return [("prefill_8192x28672_d10D24_b2048", 4, 0, 8192, 28672, 10, 24, 2048, {})]
    raise ValueError(cfg)


def build(spec, with_bits=True):
    name, seed, layer, K, N, d, D, batch, kw = spec
    return make_layer(name, seed, layer, K, N, d, D, batch, with_bits=with_bits, **kw)
