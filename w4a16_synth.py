"""Seeded synthetic inputs for the W4A16 group-128 linear layer.

This module is the one place that makes inputs.  Both the CPU oracle (under
``oracle/``) and the CUDA library are fed from it; it contains none of the
layer's own arithmetic (no unpacking, no dequantisation, no matmul).  It does
hold the *input recipe*:

* activations ``x``: float32 draws rounded to BF16 (round-to-nearest-even),
  optionally with 1 % of the entries multiplied by 20 before rounding;
* weights: float32 ``W ~ N(0, 0.02)`` quantised per 128-wide K group with the
  affine min/max quantiser (``scale = (max - min) / 15``, ``bias = min``, both
  rounded to BF16 first, then ``q = clamp(rint((w - bias) / scale), 0, 15)``),
  packed eight 4-bit codes per uint32 with k % 8 == 0 in bits 0-3.

The pages fix the format as 4-bit weights, group size 128, BF16 activations,
quantisation parameters and output (tiny-llm, "Week 2 Day 6: SIMD-Matrix
Prefill", the list under the introduction and Task 3).  The packing order and
the quantiser are this library's format definition.

BF16 values travel as ``uint16`` bit patterns so that nothing here depends on a
framework's BF16 type.  Randomness is numpy's PCG64 seeded with
``[seed, M, N, K]`` for a shape, so every shape has its own stream.
"""
from __future__ import annotations

import numpy as np

GROUP = 128  # K values per scale/bias pair
PACK = 8     # 4-bit codes per uint32 word


def bf16_bits(a) -> np.ndarray:
    """float32 -> BF16 bit patterns, round to nearest, ties to even."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = a.view(np.uint32).astype(np.uint64)
    nan = (u & 0x7F800000) == 0x7F800000
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r = np.where(nan & ((u & 0x007FFFFF) != 0), ((u >> 16) | 0x40).astype(np.uint16), r)
    r = np.where(nan & ((u & 0x007FFFFF) == 0), (u >> 16).astype(np.uint16), r)
    return r.astype(np.uint16)


def bf16_to_f32(bits) -> np.ndarray:
    """BF16 bit patterns -> float32 (exact widening)."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


def pack_nibbles(q: np.ndarray) -> np.ndarray:
    """uint8 codes [N, K] in 0..15 -> uint32 words [N, K/8], low nibble first."""
    q = np.asarray(q)
    N, K = q.shape
    if K % PACK:
        raise ValueError("K must be a multiple of 8")
    if q.min(initial=0) < 0 or q.max(initial=0) > 15:
        raise ValueError("codes must lie in 0..15")
    q = q.astype(np.uint32).reshape(N, K // PACK, PACK)
    shifts = (4 * np.arange(PACK, dtype=np.uint32))[None, None, :]
    return np.bitwise_or.reduce(q << shifts, axis=2).astype(np.uint32)


def quantize_w4_g128(W: np.ndarray):
    """Affine min/max quantiser, one (scale, bias) per row and 128-wide K group.

    Returns ``(wq uint32 [N, K/8], scales uint16 [N, K/128], biases uint16
    [N, K/128])`` with BF16 bit patterns for scales and biases.  A constant
    group (max == min) gets scale 0 and codes 0, so it reproduces ``bias``.
    """
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    Wg = W.reshape(N, K // GROUP, GROUP)
    mn = Wg.min(axis=2)
    mx = Wg.max(axis=2)
    s_bits = bf16_bits((mx - mn) / np.float32(15))
    b_bits = bf16_bits(mn)
    s = bf16_to_f32(s_bits)[..., None]
    b = bf16_to_f32(b_bits)[..., None]
    safe = np.where(s == 0, np.float32(1), s)
    q = np.rint((Wg - b) / safe)
    q = np.where(s == 0, 0, q)
    q = np.clip(q, 0, 15).astype(np.uint8).reshape(N, K)
    return pack_nibbles(q), s_bits, b_bits


def shape_rng(M: int, N: int, K: int, seed: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, M, N, K])


def make_x(rng: np.random.Generator, M: int, K: int, outliers: bool = False,
           std: float = 1.0) -> np.ndarray:
    """BF16 activations [M, K]; with ``outliers`` 1 % of entries are scaled by 20."""
    x = rng.standard_normal((M, K), dtype=np.float32) * np.float32(std)
    if outliers:
        hit = rng.random((M, K)) < 0.01
        x = np.where(hit, x * np.float32(20), x).astype(np.float32)
    return bf16_bits(x)


def make_weights(rng: np.random.Generator, N: int, K: int, std: float = 0.02):
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(std)
    return quantize_w4_g128(W)


def make_problem(M: int, N: int, K: int, seed: int = 0, outliers: bool = False,
                 rng: np.random.Generator | None = None) -> dict:
    """One seeded problem: x [M,K] bf16 bits, wq [N,K/8], scales/biases [N,K/128]."""
    rng = shape_rng(M, N, K, seed) if rng is None else rng
    x = make_x(rng, M, K, outliers=outliers)
    wq, s, b = make_weights(rng, N, K)
    return {"x": x, "wq": wq, "scales": s, "biases": b, "M": M, "N": N, "K": K}


def make_pr1_problem() -> dict:
    """The small reference problem: M=32, K=256, N=64, seed 0 (x drawn first, then W)."""
    return make_problem(32, 64, 256, rng=np.random.default_rng(0))


def make_integer_problem(M: int, N: int, K: int, seed: int = 0) -> dict:
    """Integer-valued inputs whose products and sums are exact in FP32.

    x in {-4..4}, scale in {1, 2}, bias in {-8..0}, codes in 0..15.  With
    K <= 1024 every partial sum (in any order, and with any per-group
    factoring of scale and bias) is an integer below 2**24 in magnitude, so
    FP32 arithmetic on it is exact and only the final BF16 rounding remains.
    Returns the problem plus the integer arrays used to build it.
    """
    rng = shape_rng(M, N, K, seed + 7919)
    G = K // GROUP
    xi = rng.integers(-4, 5, size=(M, K)).astype(np.int64)
    qi = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    si = rng.integers(1, 3, size=(N, G)).astype(np.int64)
    bi = rng.integers(-8, 1, size=(N, G)).astype(np.int64)
    return {
        "x": bf16_bits(xi.astype(np.float32)),
        "wq": pack_nibbles(qi),
        "scales": bf16_bits(si.astype(np.float32)),
        "biases": bf16_bits(bi.astype(np.float32)),
        "M": M, "N": N, "K": K,
        "xi": xi, "qi": qi.astype(np.int64), "si": si, "bi": bi,
    }


# Projection shapes (name, K, N) of a Qwen3-4B decoder layer, plus the vocabulary
# projection, as the benchmark ledger of "Week 2 Day 6: SIMD-Matrix Prefill"
# sweeps them (Benchmark Analysis: q k v o gate up down).
QWEN3_4B_PROJECTIONS = (
    ("q", 2560, 4096),
    ("k", 2560, 1024),
    ("v", 2560, 1024),
    ("o", 4096, 2560),
    ("gate", 2560, 9728),
    ("up", 2560, 9728),
    ("down", 9728, 2560),
)
QWEN3_4B_LM_HEAD = ("lm_head", 2560, 151936)


# ---------------------------------------------------------------- edge-case inputs
# Inputs built to reach the corners of the layer's definition; none of this computes the
# layer itself.  Each returns a problem dict like make_problem.

def make_x_positive(rng: np.random.Generator, M: int, K: int, kind: str = "abs4") -> np.ndarray:
    """Non-zero-mean BF16 activations: ``abs4`` = |N(0,1)| * 4 (mean about 3.2), ``swiglu`` =
    silu(a) * b with a ~ N(0,1) + 1 and b ~ |N(0,1)| (the mostly positive input of a down
    projection after the gated activation)."""
    if kind == "abs4":
        x = np.abs(rng.standard_normal((M, K), dtype=np.float32)) * np.float32(4)
    elif kind == "swiglu":
        a = rng.standard_normal((M, K), dtype=np.float32) + np.float32(1)
        b = np.abs(rng.standard_normal((M, K), dtype=np.float32))
        x = (a / (np.float32(1) + np.exp(-a)) * b).astype(np.float32)
    else:
        raise ValueError(kind)
    return bf16_bits(x)


def make_edge_problem(M: int, N: int, K: int, x_kind: str = "normal", seed: int = 0) -> dict:
    """A problem whose weights hit the quantiser's corners and whose activations are chosen
    by ``x_kind`` (``normal``, ``abs4``, ``swiglu``).

    Weights: W ~ N(0, 0.02), then every 7th (row, group) pair is made constant (the quantiser
    gives scale 0 and bias = the value, so the group reproduces its bias), and after
    quantisation every 5th (row, group) pair gets all codes 15 and every 11th all codes 0
    (scales and biases kept).
    """
    rng = shape_rng(M, N, K, seed + 104729)
    if x_kind == "normal":
        x = make_x(rng, M, K)
    else:
        x = make_x_positive(rng, M, K, x_kind)
    G = K // GROUP
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    Wg = W.reshape(N, G, GROUP)
    idx = np.arange(N * G).reshape(N, G)
    const = (idx % 7) == 3
    Wg[const] = Wg[const][:, :1]                      # constant group: every value equal
    wq, s, b = quantize_w4_g128(Wg.reshape(N, K))
    words = wq.reshape(N, G, GROUP // PACK)
    words[(idx % 5) == 1] = np.uint32(0xFFFFFFFF)     # all codes 15
    words[(idx % 11) == 2] = np.uint32(0)             # all codes 0
    return {"x": x, "wq": words.reshape(N, K // PACK).copy(), "scales": s, "biases": b,
            "M": M, "N": N, "K": K, "const_groups": int(const.sum())}


def make_overflow_problem(M: int, N: int, K: int, sign: float = 1.0, exponent: int = 122,
                          positive_w: bool = True, seed: int = 0) -> dict:
    """Huge activations |x| = 2^exponent .. 2^(exponent+1) of one sign.

    With ``positive_w`` (W = 0.05 + |N(0, 0.02)|) every term x * w has the sign of ``sign``,
    so for exponent 122 the FP32 sum of the plain definition overflows to +-inf for every
    output.  With W ~ N(0, 0.02) instead, the terms cancel and the plain sums stay finite
    (about 2^exponent in size) while sums of x alone do not fit FP32 for exponent >= 121."""
    rng = shape_rng(M, N, K, seed + 15485863)
    mag = np.float32(2.0 ** exponent) * (np.float32(1) + rng.random((M, K), dtype=np.float32))
    x = bf16_bits(np.float32(sign) * mag)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    if positive_w:
        W = np.float32(0.05) + np.abs(W)
    wq, s, b = quantize_w4_g128(W)
    return {"x": x, "wq": wq, "scales": s, "biases": b, "M": M, "N": N, "K": K}


def interleave_gate_up(gate, up):
    """Row-interleave two [N2, ...] arrays (a packed layer's codes, scales or biases) in blocks
    of 8 for the fused gate/up projection: gate rows 8 b .. 8 b + 7, then up rows 8 b .. 8 b + 7
    (a layout only, no arithmetic)."""
    gate, up = np.asarray(gate), np.asarray(up)
    if gate.shape != up.shape or gate.shape[0] % 8:
        raise ValueError("gate and up need the same shape and a row count divisible by 8")
    n2 = gate.shape[0]
    return np.stack([gate.reshape(n2 // 8, 8, -1), up.reshape(n2 // 8, 8, -1)], axis=1).reshape(2 * n2, -1)


# ---------------------------------------------------------------- other bit widths
# The same affine format with b-bit codes (b in {2, 4, 8}): 32 / b codes per uint32, low first,
# scale = (max - min) / (2^b - 1), q clamped to 0 .. 2^b - 1; wq is [N, K * b / 32].

def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    """uint8 codes [N, K] in 0 .. 2^bits - 1 -> uint32 words [N, K * bits / 32], low first."""
    q = np.asarray(q)
    N, K = q.shape
    per = 32 // bits
    if bits not in (2, 4, 8) or K % per:
        raise ValueError("bits must be 2, 4 or 8 and K a multiple of 32 / bits")
    if q.min(initial=0) < 0 or q.max(initial=0) > (1 << bits) - 1:
        raise ValueError("codes out of range")
    q = q.astype(np.uint32).reshape(N, K // per, per)
    shifts = (bits * np.arange(per, dtype=np.uint32))[None, None, :]
    return np.bitwise_or.reduce(q << shifts, axis=2).astype(np.uint32)


def quantize_affine_g128(W: np.ndarray, bits: int):
    """The min/max recipe of quantize_w4_g128 for b-bit codes (2^b - 1 steps per group)."""
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    top = (1 << bits) - 1
    Wg = W.reshape(N, K // GROUP, GROUP)
    mn = Wg.min(axis=2)
    mx = Wg.max(axis=2)
    s_bits = bf16_bits((mx - mn) / np.float32(top))
    b_bits = bf16_bits(mn)
    s = bf16_to_f32(s_bits)[..., None]
    b = bf16_to_f32(b_bits)[..., None]
    safe = np.where(s == 0, np.float32(1), s)
    q = np.rint((Wg - b) / safe)
    q = np.where(s == 0, 0, q)
    q = np.clip(q, 0, top).astype(np.uint8).reshape(N, K)
    return pack_codes(q, bits), s_bits, b_bits


def make_problem_bits(M: int, N: int, K: int, bits: int, seed: int = 0, outliers: bool = False) -> dict:
    """make_problem with b-bit codes (its own stream per shape and bit width)."""
    rng = np.random.default_rng([seed, M, N, K, bits])
    x = make_x(rng, M, K, outliers=outliers)
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    wq, s, b = quantize_affine_g128(W, bits)
    return {"x": x, "wq": wq, "scales": s, "biases": b, "M": M, "N": N, "K": K, "bits": bits}


def make_integer_problem_bits(M: int, N: int, K: int, bits: int, seed: int = 0) -> dict:
    """Integer-valued inputs with b-bit codes whose FP32 sums are exact (see make_integer_problem):
    x in {-4..4}, scale in {1, 2}, bias in {-8..0}, codes in 0 .. 2^bits - 1, K <= 1024 for
    bits <= 4 and K <= 256 for 8 bits (|partial sums| < 2^24)."""
    rng = np.random.default_rng([seed + 7919, M, N, K, bits])
    G = K // GROUP
    xi = rng.integers(-4, 5, size=(M, K)).astype(np.int64)
    qi = rng.integers(0, 1 << bits, size=(N, K)).astype(np.uint8)
    si = rng.integers(1, 3, size=(N, G)).astype(np.int64)
    bi = rng.integers(-8, 1, size=(N, G)).astype(np.int64)
    return {
        "x": bf16_bits(xi.astype(np.float32)), "wq": pack_codes(qi, bits),
        "scales": bf16_bits(si.astype(np.float32)), "biases": bf16_bits(bi.astype(np.float32)),
        "M": M, "N": N, "K": K, "bits": bits,
        "xi": xi, "qi": qi.astype(np.int64), "si": si, "bi": bi,
    }
