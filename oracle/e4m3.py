"""E4M3 codes to numbers, for the oracle -- TEST INFRASTRUCTURE ONLY.

The 8-bit floating point format E4M3 of the OCP 8-bit floating point
specification (the format torch calls ``float8_e4m3fn``): bit 7 is the sign
s, bits 6-3 the exponent field e (bias 7), bits 2-0 the mantissa field m.

    e = 0          value = (-1)^s * (m / 8) * 2^(1 - 7)      zero and subnormals
    0 < e          value = (-1)^s * (1 + m / 8) * 2^(e - 7)
    e = 15, m = 7  NaN (the format has no infinities)

An fp8 latent KV cache is read as these codes times one per-tensor scale
(the reading of kernelbot-amd-mixed-mla submission 588924's fp8 KV remark,
which fixes no format).  Everything here is fp64 and exact: a code's value
has at most 4 significant bits and the scale is an fp32 number, so their
product is exact in fp64.
"""
from __future__ import annotations

import math

import torch


def value(code: int) -> float:
    """The number an E4M3 code stands for (the definition above)."""
    if not 0 <= code <= 255:
        raise ValueError("an E4M3 code is one byte")
    s = (code >> 7) & 1
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 15 and m == 7:
        return math.nan
    mag = (m / 8.0) * 2.0 ** (1 - 7) if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


_TABLE = torch.tensor([value(c) for c in range(256)], dtype=torch.float64)


def decode(codes: torch.Tensor) -> torch.Tensor:
    """fp64 values of a tensor of codes (uint8, or float8_e4m3fn read as its bytes)."""
    if codes.dtype != torch.uint8:
        codes = codes.view(torch.uint8)
    return _TABLE[codes.long()]


def dequantize(codes: torch.Tensor, scale: float) -> torch.Tensor:
    """scale * value(code), elementwise, in fp64."""
    return decode(codes) * float(scale)
