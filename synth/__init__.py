"""Seeded synthetic inputs shared by the CUDA path's tests/bench and by the oracle.

This module holds no attention arithmetic.  It only draws numbers and rounds
them to the storage types the library consumes, so that both sides see the
very same bytes:

* ``normal_f32``   -- N(0, 1) fp32 from numpy's Philox4x32-10 counter-based
  generator, keyed by ``(seed, tensor_id)`` so every tensor has its own stream.
* ``to_bf16_bits`` -- fp32 -> bf16 bit patterns, round-to-nearest-even
  (torch's CPU cast), and ``bf16_bits_to_f64`` for the exact values.
* ``quantize_e4m3`` -- per-tensor amax scaling to float8 e4m3 (the reading of
  "FP8 with per-tensor scales" taken for the FP8 forward): s = 448 / amax,
  x8 = e4m3(RNE(x * s)), descale = 1 / s.  Returns the bytes, the descale and
  the exact dequantised fp64 values (x8 * descale) the oracle consumes.

The workloads are the attention configurations of the exact IO-aware attention
explainers (FlashAttention): Q, K, V, dO ~ N(0, 1), layout [B, H, N, d] with d
innermost; an optional power-of-two multiplier on Q (exact in fp32) widens the
score range to force running-max rescales.
"""
from __future__ import annotations

import numpy as np
import torch

# Tensor ids: one independent Philox stream per tensor of a configuration.
TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "do": 4}


def normal_f32(seed: int, tensor_id: int, shape) -> np.ndarray:
    """N(0,1) float32 of ``shape`` from Philox keyed by (seed, tensor_id)."""
    bitgen = np.random.Philox(key=[int(seed) & 0xFFFFFFFFFFFFFFFF, int(tensor_id)])
    rng = np.random.Generator(bitgen)
    return rng.standard_normal(size=tuple(shape), dtype=np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> uint16 bf16 bit patterns, round to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> the exact float64 values."""
    u32 = bits.astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


def e4m3_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """uint8 e4m3 (fn variant: no inf, 0x7f/0xff are NaN) -> exact float64."""
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def quantize_e4m3(x: np.ndarray):
    """Per-tensor amax quantisation to e4m3.

    Returns ``(bits uint8, descale float, dequantised float64)``.  The scaled
    values are <= 448 in magnitude, so the cast never saturates.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    amax = float(np.max(np.abs(x))) if x.size else 0.0
    if amax == 0.0:
        scale = np.float32(1.0)
    else:
        scale = np.float32(448.0) / np.float32(amax)
    xs = torch.from_numpy(x) * torch.tensor(scale, dtype=torch.float32)
    bits = xs.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    descale = float(np.float32(1.0) / scale)
    deq = e4m3_bits_to_f64(bits) * descale
    return bits, descale, deq


def attention_inputs(B: int, H: int, N: int, d: int, seed: int, q_mult: float = 1.0,
                     with_grad: bool = True, storage: str = "bf16", want_f64: bool = True):
    """Seeded Q, K, V (and dO) for one attention configuration.

    ``storage`` is ``"bf16"`` (Q, K, V, dO rounded to bf16) or ``"e4m3"`` (Q, K,
    V quantised with per-tensor scales; no dO).  The returned dict holds, per
    tensor name, the raw storage bits (``"<name>_bits"``) and the exact float64
    values the device will see (``"<name>"``).  For e4m3 it also holds
    ``"<name>_descale"``.  With ``want_f64=False`` the float64 copies are
    skipped (large shapes); ``head_f64`` converts one head on demand.
    """
    shape = (B, H, N, d)
    out = {"shape": shape, "seed": seed, "q_mult": q_mult, "storage": storage}
    names = ["q", "k", "v"] + (["do"] if (with_grad and storage == "bf16") else [])
    for name in names:
        x = normal_f32(seed, TENSOR_IDS[name], shape)
        if name == "q" and q_mult != 1.0:
            x = x * np.float32(q_mult)
        if storage == "bf16":
            bits = to_bf16_bits(x)
            out[name + "_bits"] = bits
            if want_f64:
                out[name] = bf16_bits_to_f64(bits)
        elif storage == "e4m3":
            bits, descale, deq = quantize_e4m3(x)
            out[name + "_bits"] = bits
            out[name + "_descale"] = descale
            if want_f64:
                out[name] = deq
        else:
            raise ValueError(f"unknown storage {storage!r}")
    return out


def decode_inputs(B: int, H: int, Nq: int, Nk: int, d: int, seed: int, q_mult: float = 1.0,
                  want_f64: bool = True):
    """Seeded bf16 inputs for decode against a KV cache: Q [B,H,Nq,d] (the
    newest Nq positions) and K, V [B,H,Nk,d] (the cache), N(0,1) like the
    square workloads.  Same dict layout as ``attention_inputs``."""
    out = {"shape": (B, H, Nq, Nk, d), "seed": seed, "q_mult": q_mult, "storage": "bf16"}
    for name, n in (("q", Nq), ("k", Nk), ("v", Nk)):
        x = normal_f32(seed, TENSOR_IDS[name], (B, H, n, d))
        if name == "q" and q_mult != 1.0:
            x = x * np.float32(q_mult)
        bits = to_bf16_bits(x)
        out[name + "_bits"] = bits
        if want_f64:
            out[name] = bf16_bits_to_f64(bits)
    return out


def head_f64(inp, name: str, b: int, h: int) -> np.ndarray:
    """Exact float64 values of one head of tensor ``name``."""
    bits = inp[name + "_bits"][b, h]
    if inp["storage"] == "bf16":
        return bf16_bits_to_f64(bits)
    return e4m3_bits_to_f64(bits) * inp[name + "_descale"]


def attention_inputs_f32_to_bf16(B, H, N, d, seed):
    """The fp32-drawn variant of the single-head reference case: the fp32 draws
    are returned too, and the bf16 rounding of them is what both sides use."""
    shape = (B, H, N, d)
    out = attention_inputs(B, H, N, d, seed)
    out["f32"] = {n: normal_f32(seed, TENSOR_IDS[n], shape) for n in ("q", "k", "v", "do")}
    return out
