"""Seeded synthetic inputs for AQLM layers (shared by the tests and the bench).

This module only draws random numbers; it holds none of the method's
arithmetic.  The distributions stand in for trained Llama-2 AQLM layers:

  codebooks  fp16 ~ N(0, 0.02)        [M][2^B][8]
  codes      uniform over 0..2^B-1    [d_out][d_in/8][M]  (uint8 for B=8,
                                       int16 bit patterns for B=16)
  scales     fp16 ~ U[0.5, 1.5]       [d_out]
  x          N(0, 1), fp16 (decode) or bf16 bit patterns (prefill) [T][d_in]

Draw order from one numpy Generator(PCG64(seed)): codebooks, codes, scales,
x.  Every fp16 value is the round-to-nearest-even conversion of the float64
draw (numpy's astype), every bf16 value the RNE conversion of the float32
draw (torch's conversion).
"""
from dataclasses import dataclass

import numpy as np

GROUP = 8


@dataclass(frozen=True)
class LayerSpec:
    d_out: int
    d_in: int
    M: int
    B: int

    @property
    def groups(self):
        return self.d_in // GROUP

    @property
    def K(self):
        return 1 << self.B

    @property
    def name(self):
        return f"{self.M}x{self.B} {self.d_out}x{self.d_in}"

    def code_bytes(self):
        return self.d_out * self.groups * self.M * self.B // 8

    def codebook_bytes(self):
        return self.M * self.K * GROUP * 2


def _codes(rng, spec):
    shape = (spec.d_out, spec.groups, spec.M)
    if spec.B == 8:
        return rng.integers(0, 256, size=shape, dtype=np.uint8)
    return rng.integers(0, 65536, size=shape, dtype=np.uint16).view(np.int16)


def bf16_bits(a):
    """float array -> bfloat16 bit patterns (uint16), round to nearest even."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def make_layer(spec, seed=0, tokens=1, x_dtype="fp16"):
    """Return dict(codes, codebooks, scales, x) for one layer, numpy on the host."""
    rng = np.random.Generator(np.random.PCG64(seed))
    codebooks = rng.normal(0.0, 0.02, size=(spec.M, spec.K, GROUP)).astype(np.float16)
    codes = _codes(rng, spec)
    scales = rng.uniform(0.5, 1.5, size=(spec.d_out,)).astype(np.float16)
    x = make_x(rng, tokens, spec.d_in, x_dtype) if tokens > 0 else None
    return {"codes": codes, "codebooks": codebooks, "scales": scales, "x": x}


def make_x(rng, tokens, d_in, x_dtype="fp16"):
    xs = rng.normal(0.0, 1.0, size=(tokens, d_in))
    if x_dtype == "fp16":
        return xs.astype(np.float16)
    if x_dtype == "bf16":
        return bf16_bits(xs.astype(np.float32))
    raise ValueError(x_dtype)


# The workloads, named by what they are.
SMALL_2X8 = LayerSpec(256, 512, 2, 8)
LLAMA7B_SHAPES = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                  ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
LLAMA70B_SHAPES = [("attn", 8192, 8192), ("gate_up", 28672, 8192), ("down", 8192, 28672)]
PREFILL_SHAPES = [(11008, 4096), (4096, 11008)]
PREFILL_TOKENS = 2048
FORMATS = {"1x16": (1, 16), "2x8": (2, 8), "2x16": (2, 16)}
