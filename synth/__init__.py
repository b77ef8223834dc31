"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module only draws random bytes and numbers; it holds none of the Q4_K
arithmetic (no scale unpacking, no dequantisation, no matmul, no routing).
Both sides receive the same packed bytes and re-derive everything from them.

Q4_K blocks are drawn field by field as uniform random bytes:

* bytes 0-1 and 2-3 (``d`` and ``dmin``): ``|N(0,1)| * 1e-3`` computed in
  fp64, cast to IEEE binary16 (round to nearest even), stored little-endian;
* bytes 4-15 (the packed six-bit scale/min pairs) and 16-143 (the 4-bit
  quants): independent uniform bytes.

Every bit of the scale field and of the quant field belongs to exactly one
six-bit scale, six-bit min or four-bit quant, so uniform random bytes give
each ``q`` uniform on 0..15 and each ``sc``/``m`` uniform on 0..63,
independently -- the distribution the workloads ask for -- without this module
knowing where the bits go.

Activations are ``N(0,1)`` drawn in fp32 and rounded to bf16 (nearest even),
returned as their raw 16-bit patterns (``uint16``). Router logits are fp32.
"""
from __future__ import annotations

import numpy as np

BLOCK_WEIGHTS = 256  # weights per Q4_K super-block
BLOCK_BYTES = 144    # bytes per Q4_K super-block

# Workload shapes (dense decode, dense prefill, MoE layer).
DENSE_DECODE = dict(gate_up=(34816, 5120), down=(5120, 17408), Ms=(1, 4, 8, 16, 32))
DENSE_PREFILL = dict(N=17408, K=5120, Ms=(512, 4096))
MOE = dict(E=128, topk=8, H=2048, F=768)
MOE_DECODE_MS = (1, 8, 32)
MOE_PREFILL_M = 4096
MOE_HOT = 16
MOE_HOT_BIAS = 1.5
MOE_LOGIT_SIGMA = 2.0


def q4k_random_blocks(rng: np.random.Generator, nrows: int, K: int) -> np.ndarray:
    """Random Q4_K matrix of ``nrows`` x ``K`` weights: uint8 ``[nrows][K/256][144]``.

    Draw order: d, dmin, scale bytes, quant bytes (each over all blocks in
    row-major block order).
    """
    if K % BLOCK_WEIGHTS:
        raise ValueError("K must be a multiple of 256")
    nb = nrows * (K // BLOCK_WEIGHTS)
    d = (np.abs(rng.standard_normal(nb)) * 1e-3).astype(np.float16)
    dmin = (np.abs(rng.standard_normal(nb)) * 1e-3).astype(np.float16)
    sc = rng.integers(0, 256, size=(nb, 12), dtype=np.uint8)
    qs = rng.integers(0, 256, size=(nb, 128), dtype=np.uint8)
    out = np.empty((nb, BLOCK_BYTES), dtype=np.uint8)
    out[:, 0:2] = d.astype("<f2").view(np.uint8).reshape(nb, 2)
    out[:, 2:4] = dmin.astype("<f2").view(np.uint8).reshape(nb, 2)
    out[:, 4:16] = sc
    out[:, 16:144] = qs
    return out.reshape(nrows, K // BLOCK_WEIGHTS, BLOCK_BYTES)


Q5_BLOCK_BYTES = 176  # bytes per Q5_K super-block


def q5k_random_blocks(rng: np.random.Generator, nrows: int, K: int) -> np.ndarray:
    """Random Q5_K matrix: uint8 ``[nrows][K/256][176]``, drawn like Q4_K blocks
    (d, dmin, scale bytes) and then the 32 fifth-bit bytes and the 128 nibble
    bytes as uniform bytes, so every five-bit quant is uniform on 0..31."""
    if K % BLOCK_WEIGHTS:
        raise ValueError("K must be a multiple of 256")
    nb = nrows * (K // BLOCK_WEIGHTS)
    d = (np.abs(rng.standard_normal(nb)) * 1e-3).astype(np.float16)
    dmin = (np.abs(rng.standard_normal(nb)) * 1e-3).astype(np.float16)
    sc = rng.integers(0, 256, size=(nb, 12), dtype=np.uint8)
    qh = rng.integers(0, 256, size=(nb, 32), dtype=np.uint8)
    qs = rng.integers(0, 256, size=(nb, 128), dtype=np.uint8)
    out = np.empty((nb, Q5_BLOCK_BYTES), dtype=np.uint8)
    out[:, 0:2] = d.astype("<f2").view(np.uint8).reshape(nb, 2)
    out[:, 2:4] = dmin.astype("<f2").view(np.uint8).reshape(nb, 2)
    out[:, 4:16] = sc
    out[:, 16:48] = qh
    out[:, 48:176] = qs
    return out.reshape(nrows, K // BLOCK_WEIGHTS, Q5_BLOCK_BYTES)


Q80_BLOCK_BYTES = 34  # bytes per Q8_0 block of 32 weights


def q80_random_blocks(rng: np.random.Generator, nrows: int, K: int) -> np.ndarray:
    """Random Q8_0 matrix: uint8 ``[nrows][K/32][34]``. Draw order: d (as for
    Q4_K blocks), then the 32 quant bytes of every block as uniform bytes (each
    signed quant uniform on -128..127)."""
    if K % BLOCK_WEIGHTS:
        raise ValueError("K must be a multiple of 256")
    nb = nrows * (K // 32)
    d = (np.abs(rng.standard_normal(nb)) * 1e-3).astype(np.float16)
    qs = rng.integers(0, 256, size=(nb, 32), dtype=np.uint8)
    out = np.empty((nb, Q80_BLOCK_BYTES), dtype=np.uint8)
    out[:, 0:2] = d.astype("<f2").view(np.uint8).reshape(nb, 2)
    out[:, 2:34] = qs
    return out.reshape(nrows, K // 32, Q80_BLOCK_BYTES)


Q6_BLOCK_BYTES = 210  # bytes per Q6_K super-block


def q6k_random_blocks(rng: np.random.Generator, nrows: int, K: int) -> np.ndarray:
    """Random Q6_K matrix: uint8 ``[nrows][K/256][210]``. Draw order: the 192 quant
    bytes (ql then qh, uniform: every six-bit quant uniform), the 16 scale bytes
    (uniform: signed scales uniform on -128..127), then d as for Q4_K blocks."""
    if K % BLOCK_WEIGHTS:
        raise ValueError("K must be a multiple of 256")
    nb = nrows * (K // BLOCK_WEIGHTS)
    qb = rng.integers(0, 256, size=(nb, 192), dtype=np.uint8)
    sc = rng.integers(0, 256, size=(nb, 16), dtype=np.uint8)
    d = (np.abs(rng.standard_normal(nb)) * 1e-3).astype(np.float16)
    out = np.empty((nb, Q6_BLOCK_BYTES), dtype=np.uint8)
    out[:, 0:192] = qb
    out[:, 192:208] = sc
    out[:, 208:210] = d.astype("<f2").view(np.uint8).reshape(nb, 2)
    return out.reshape(nrows, K // BLOCK_WEIGHTS, Q6_BLOCK_BYTES)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round to nearest even (torch CPU cast)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32 values (exact widening)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_normal(rng: np.random.Generator, shape) -> np.ndarray:
    """N(0,1) drawn in fp32, rounded to bf16; returns uint16 bit patterns."""
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def gemv_small(seed: int = 0, N: int = 256, K: int = 2048, M: int = 1):
    """Single-matrix GEMV case (default: 256 x 2048, one token). Order: W, X."""
    rng = np.random.default_rng(seed)
    W = q4k_random_blocks(rng, N, K)
    X = bf16_normal(rng, (M, K))
    return W, X


def dense_decode(seed: int = 1, Mmax: int = 32, scale_rows: float = 1.0):
    """Dense decode projections: gate+up (34816 x 5120) and down (5120 x 17408).

    Order: W_gate_up, W_down, X_gate_up [Mmax][5120], X_down [Mmax][17408].
    A call with M tokens uses the first M rows of X. ``scale_rows`` < 1 shrinks
    the row counts (kept a multiple of 16) for quick tests.
    """
    rng = np.random.default_rng(seed)
    (ngu, kgu), (ndn, kdn) = DENSE_DECODE["gate_up"], DENSE_DECODE["down"]
    ngu = max(16, int(ngu * scale_rows) // 16 * 16)
    ndn = max(16, int(ndn * scale_rows) // 16 * 16)
    Wgu = q4k_random_blocks(rng, ngu, kgu)
    Wdn = q4k_random_blocks(rng, ndn, kdn)
    Xgu = bf16_normal(rng, (Mmax, kgu))
    Xdn = bf16_normal(rng, (Mmax, kdn))
    return dict(W_gate_up=Wgu, W_down=Wdn, X_gate_up=Xgu, X_down=Xdn)


def gemv_small_q5(seed: int = 0, N: int = 256, K: int = 2048, M: int = 1):
    """Single-matrix Q5_K GEMV case. Order: W, X."""
    rng = np.random.default_rng(seed)
    W = q5k_random_blocks(rng, N, K)
    X = bf16_normal(rng, (M, K))
    return W, X


def dense_decode_q5(seed: int = 5, Mmax: int = 32):
    """The dense decode shapes with Q5_K weights (gate+up 34816 x 5120, down
    5120 x 17408). Order: W_gate_up, W_down, X_gate_up, X_down."""
    rng = np.random.default_rng(seed)
    (ngu, kgu), (ndn, kdn) = DENSE_DECODE["gate_up"], DENSE_DECODE["down"]
    Wgu = q5k_random_blocks(rng, ngu, kgu)
    Wdn = q5k_random_blocks(rng, ndn, kdn)
    Xgu = bf16_normal(rng, (Mmax, kgu))
    Xdn = bf16_normal(rng, (Mmax, kdn))
    return dict(W_gate_up=Wgu, W_down=Wdn, X_gate_up=Xgu, X_down=Xdn)


def gemv_small_q80(seed: int = 0, N: int = 256, K: int = 2048, M: int = 1):
    """Single-matrix Q8_0 GEMV case. Order: W, X."""
    rng = np.random.default_rng(seed)
    W = q80_random_blocks(rng, N, K)
    X = bf16_normal(rng, (M, K))
    return W, X


def dense_decode_q80(seed: int = 6, Mmax: int = 32):
    """The dense decode shapes with Q8_0 weights. Order: W_gate_up, W_down, X_gate_up, X_down."""
    rng = np.random.default_rng(seed)
    (ngu, kgu), (ndn, kdn) = DENSE_DECODE["gate_up"], DENSE_DECODE["down"]
    Wgu = q80_random_blocks(rng, ngu, kgu)
    Wdn = q80_random_blocks(rng, ndn, kdn)
    Xgu = bf16_normal(rng, (Mmax, kgu))
    Xdn = bf16_normal(rng, (Mmax, kdn))
    return dict(W_gate_up=Wgu, W_down=Wdn, X_gate_up=Xgu, X_down=Xdn)


def gemv_small_q6(seed: int = 0, N: int = 256, K: int = 2048, M: int = 1):
    """Single-matrix Q6_K GEMV case. Order: W, X."""
    rng = np.random.default_rng(seed)
    W = q6k_random_blocks(rng, N, K)
    X = bf16_normal(rng, (M, K))
    return W, X


def dense_decode_q6(seed: int = 7, Mmax: int = 32):
    """The dense decode shapes with Q6_K weights. Order: W_gate_up, W_down, X_gate_up, X_down."""
    rng = np.random.default_rng(seed)
    (ngu, kgu), (ndn, kdn) = DENSE_DECODE["gate_up"], DENSE_DECODE["down"]
    Wgu = q6k_random_blocks(rng, ngu, kgu)
    Wdn = q6k_random_blocks(rng, ndn, kdn)
    Xgu = bf16_normal(rng, (Mmax, kgu))
    Xdn = bf16_normal(rng, (Mmax, kdn))
    return dict(W_gate_up=Wgu, W_down=Wdn, X_gate_up=Xgu, X_down=Xdn)


def dense_prefill(seed: int = 2, M: int = 4096, N: int = 17408, K: int = 5120):
    """Dense prefill GEMM: W [N][K] in Q4_K, X [M][K] bf16. Order: W, X."""
    rng = np.random.default_rng(seed)
    W = q4k_random_blocks(rng, N, K)
    X = bf16_normal(rng, (M, K))
    return W, X


def moe_layer(seed: int, M: int, E: int = 128, H: int = 2048, F: int = 768,
              hot: int = 0, hot_bias: float = MOE_HOT_BIAS,
              sigma: float = MOE_LOGIT_SIGMA):
    """MoE layer inputs.

    Order: hot expert ids (only if ``hot`` > 0: ``rng.choice(E, hot, replace=False)``),
    router logits ``N(0,1)*sigma`` fp32 [M][E] (+``hot_bias`` on the hot columns),
    X bf16 [M][H], W_gate_up [E][2F][H/256] blocks (gate rows first, then up rows),
    W_down [E][H][F/256] blocks.
    """
    rng = np.random.default_rng(seed)
    hot_ids = np.sort(rng.choice(E, hot, replace=False)) if hot > 0 else np.zeros(0, np.int64)
    logits = (rng.standard_normal((M, E)) * sigma).astype(np.float32)
    if hot > 0:
        logits[:, hot_ids] += np.float32(hot_bias)
    X = bf16_normal(rng, (M, H))
    Wgu = q4k_random_blocks(rng, E * 2 * F, H).reshape(E, 2 * F, H // 256, BLOCK_BYTES)
    Wdn = q4k_random_blocks(rng, E * H, F).reshape(E, H, F // 256, BLOCK_BYTES)
    return dict(logits=logits, X=X, W_gate_up=Wgu, W_down=Wdn, hot_ids=hot_ids,
                E=E, H=H, F=F)


def router_weights(seed: int, E: int = 128, H: int = 2048, sigma: float = MOE_LOGIT_SIGMA):
    """bf16 router weights [E][H] drawn N(0, sigma^2 / H), so that with N(0,1)
    activations the logits are about N(0, sigma^2) (the logit distribution of the
    MoE workloads)."""
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits((rng.standard_normal((E, H)) * (sigma / np.sqrt(H))).astype(np.float32))


def moe_decode(seed: int = 3, M: int = 32):
    return moe_layer(seed, M)


def moe_prefill(seed: int = 4, M: int = MOE_PREFILL_M):
    return moe_layer(seed, M, hot=MOE_HOT)
