"""CPU oracle for the Q4_K weight-only matrix products (test infrastructure).

This module is test infrastructure: only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it. The product path
(the CUDA library and its Python binding) never calls it, and it shares no
code, table or constant with the CUDA sources.

Everything here is plain numpy in fp64 (bf16/fp32 roundings where the method
defines them go through torch CPU casts), written to be checked by eye
against the definitions it cites:

* Q4_K super-block format and dequantisation -- hipEngine 0.3.0 README,
  section "GGUF Support" (GGUF Q4_K tensors, "its own quant readers"); the
  byte layout is the llama.cpp-style K-quant block: 256 weights in 144 bytes
  (fp16 ``d``, fp16 ``dmin``, 12 bytes packing eight six-bit (scale, min)
  pairs, 128 bytes of nibbles), ``w = d*sc*q - dmin*m``.
* GEMV for decode / GEMM for prefill -- hipEngine 0.3.0 README, sections
  "GGUF Support" ("bulk-prefill path") and "Quickstart" (the
  "WMMA-prefill/GEMV-decode" session profile).
* Top-k routing, token permutation, grouped expert matmul and weighted
  combine -- hipEngine 0.3.0 README, "Architecture at a glance" (``moe``
  kernel family) and "Core principles" (fused ``gate_combine_residual``);
  hipster README, claims table ("MoE grouped GEMM").

Readings taken where the pages are silent are marked ``Reading Rn`` and are
listed, with the same numbers, in the design notes.
"""
from __future__ import annotations

import numpy as np

QK = 256          # weights per super-block
BLOCK_BYTES = 144
SUB = 32          # weights per sub-block (one six-bit scale/min pair)
REL_TOL = 2e-3    # matmul tolerance: |y - y_ref| <= REL_TOL * sum_k |w*x|


# --------------------------------------------------------------------------
# Block fields (Q4_K super-block, llama.cpp-style layout)
# --------------------------------------------------------------------------

def block_d_dmin(blocks: np.ndarray):
    """``d`` and ``dmin`` of each block as fp64 (bytes 0-1 and 2-3, binary16 LE)."""
    b = np.ascontiguousarray(blocks, dtype=np.uint8)
    d = b[..., 0:2].copy().view("<f2")[..., 0].astype(np.float64)
    dmin = b[..., 2:4].copy().view("<f2")[..., 0].astype(np.float64)
    return d, dmin


def scale_min_pairs(blocks: np.ndarray):
    """Eight six-bit (sc, m) pairs from bytes 4..15 of each block (Reading R1).

    With ``s`` = those 12 bytes:
      j = 0..3: sc_j = s[j] & 63,                    m_j = s[j+4] & 63
      j = 4..7: sc_j = (s[j+4] & 15) | (s[j-4] >> 6) << 4,
                m_j  = (s[j+4] >> 4) | (s[j]   >> 6) << 4
    Returns int64 arrays of shape ``[..., 8]``.
    """
    s = np.asarray(blocks, dtype=np.uint8)[..., 4:16].astype(np.int64)
    sc = np.empty(s.shape[:-1] + (8,), dtype=np.int64)
    m = np.empty_like(sc)
    for j in range(4):
        sc[..., j] = s[..., j] & 63
        m[..., j] = s[..., j + 4] & 63
    for j in range(4, 8):
        sc[..., j] = (s[..., j + 4] & 15) | ((s[..., j - 4] >> 6) << 4)
        m[..., j] = (s[..., j + 4] >> 4) | ((s[..., j] >> 6) << 4)
    return sc, m


def quants(blocks: np.ndarray) -> np.ndarray:
    """The 256 four-bit quants of each block, in weight order.

    Weight ``i = 64*c + 32*h + l`` (chunk c=0..3, half h=0..1, lane l=0..31)
    is the low nibble (h=0) or high nibble (h=1) of quant byte ``32*c + l``
    (block byte ``16 + 32*c + l``).
    """
    qs = np.asarray(blocks, dtype=np.uint8)[..., 16:144].astype(np.int64)
    q = np.empty(qs.shape[:-1] + (QK,), dtype=np.int64)
    for c in range(4):
        for h in range(2):
            q[..., 64 * c + 32 * h: 64 * c + 32 * h + 32] = (qs[..., 32 * c: 32 * c + 32] >> (4 * h)) & 15
    return q


def dequant_exact(blocks: np.ndarray) -> np.ndarray:
    """Exact dequantised weights in fp64: ``w_i = d*sc_j*q_i - dmin*m_j`` with ``j = i // 32``.

    ``blocks`` is ``[..., nb, 144]``; the result is ``[..., nb*256]``. Every
    term is an integer multiple of 2^-24 below 2^16, so fp64 holds it exactly.
    """
    d, dmin = block_d_dmin(blocks)
    sc, m = scale_min_pairs(blocks)
    q = quants(blocks)
    j = np.arange(QK) // SUB
    w = d[..., None] * sc[..., j] * q - dmin[..., None] * m[..., j]
    return w.reshape(w.shape[:-2] + (w.shape[-2] * QK,))


def dequant_f32(blocks: np.ndarray) -> np.ndarray:
    """fp32 dequant: the exact value rounded once to fp32 (nearest even)."""
    return dequant_exact(blocks).astype(np.float32)


def dequant_bf16_bits(blocks: np.ndarray) -> np.ndarray:
    """bf16 dequant (Reading R2): RN_bf16(RN_fp32(w_exact)), as uint16 bit patterns."""
    import torch

    f = torch.from_numpy(dequant_f32(blocks))
    return f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """RN_bf16(RN_fp32(a)) as uint16 bit patterns."""
    import torch

    f = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64).astype(np.float32))
    return f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------
# Q5_K super-block (sibling K-quant; hipEngine 0.3.0 README, "GGUF Support":
# the tensor-family table lists Q5_K beside Q4_K, Q8_0 and Q6_K). Reading R19:
# the pages give no byte layout; the one taken is the llama.cpp-style K-quant
# block of 256 weights in 176 bytes: fp16 d, fp16 dmin, the same 12-byte
# six-bit (scale, min) packing as Q4_K (bytes 4..15), 32 bytes qh of fifth
# bits (bytes 16..47) and the 128 bytes of low nibbles laid out as Q4_K's
# (bytes 48..175). Weight i = 64c + 32h + l takes its low four bits from
# nibble h of byte 48 + 32c + l and its fifth bit from bit 2c + h of qh[l]:
# q = nibble + 16 * bit in 0..31, w = d*sc_j*q - dmin*m_j with j = i // 32.
# --------------------------------------------------------------------------

Q5_BLOCK_BYTES = 176


def quants_q5(blocks: np.ndarray) -> np.ndarray:
    """The 256 five-bit quants (0..31) of each Q5_K block, in weight order."""
    b = np.asarray(blocks, dtype=np.uint8)
    qh = b[..., 16:48].astype(np.int64)
    qs = b[..., 48:176].astype(np.int64)
    q = np.empty(qs.shape[:-1] + (QK,), dtype=np.int64)
    for c in range(4):
        for h in range(2):
            low = (qs[..., 32 * c: 32 * c + 32] >> (4 * h)) & 15
            high = (qh >> (2 * c + h)) & 1
            q[..., 64 * c + 32 * h: 64 * c + 32 * h + 32] = low + 16 * high
    return q


def dequant_exact_q5(blocks: np.ndarray) -> np.ndarray:
    """Exact Q5_K weights in fp64 (``[..., nb, 176]`` -> ``[..., nb*256]``); every
    term is an integer multiple of 2^-24 below 2^17, so fp64 holds it exactly."""
    d, dmin = block_d_dmin(blocks)
    sc, m = scale_min_pairs(blocks)
    q = quants_q5(blocks)
    j = np.arange(QK) // SUB
    w = d[..., None] * sc[..., j] * q - dmin[..., None] * m[..., j]
    return w.reshape(w.shape[:-2] + (w.shape[-2] * QK,))


def matmul_ref_q5(W_blocks: np.ndarray, X_bits: np.ndarray):
    """``matmul_ref`` for Q5_K weights ``[N][K/256][176]``: ``(Y, S)`` in fp64."""
    W = dequant_exact_q5(W_blocks)
    X = bf16_to_f64(X_bits)
    return X @ W.T, np.abs(X) @ np.abs(W).T


def matmul_rows_ref_q5(W_blocks: np.ndarray, X_bits: np.ndarray, rows: np.ndarray):
    return matmul_ref_q5(np.asarray(W_blocks)[rows], X_bits)


# --------------------------------------------------------------------------
# Q8_0 block (sibling quant; the same tensor-family table). Reading R20: the
# llama.cpp-style block of 32 weights in 34 bytes -- fp16 d (little-endian),
# then 32 signed bytes q (two's complement) -- with w = d * q. A row of K
# weights is K/32 consecutive blocks.
# --------------------------------------------------------------------------

Q80_BLOCK_BYTES = 34
Q80_WEIGHTS = 32


def dequant_exact_q80(blocks: np.ndarray) -> np.ndarray:
    """Exact Q8_0 weights in fp64: ``[..., nb, 34]`` -> ``[..., nb*32]`` (d*q is exact)."""
    b = np.ascontiguousarray(blocks, dtype=np.uint8)
    d = b[..., 0:2].copy().view("<f2")[..., 0].astype(np.float64)
    q = b[..., 2:34].view(np.int8).astype(np.float64)
    w = d[..., None] * q
    return w.reshape(w.shape[:-2] + (w.shape[-2] * Q80_WEIGHTS,))


def matmul_ref_q80(W_blocks: np.ndarray, X_bits: np.ndarray):
    """``matmul_ref`` for Q8_0 weights ``[N][K/32][34]``: ``(Y, S)`` in fp64."""
    W = dequant_exact_q80(W_blocks)
    X = bf16_to_f64(X_bits)
    return X @ W.T, np.abs(X) @ np.abs(W).T


def matmul_rows_ref_q80(W_blocks: np.ndarray, X_bits: np.ndarray, rows: np.ndarray):
    return matmul_ref_q80(np.asarray(W_blocks)[rows], X_bits)


def make_block_q80(d: float, q) -> np.ndarray:
    """One 34-byte Q8_0 block from d (rounded to binary16) and 32 values in -128..127."""
    b = np.zeros(Q80_BLOCK_BYTES, dtype=np.uint8)
    b[0:2] = np.array([d], dtype="<f2").view(np.uint8)
    b[2:34] = np.asarray(q, dtype=np.int64).astype(np.int8).view(np.uint8)
    return b


# --------------------------------------------------------------------------
# Q6_K super-block (the remaining sibling of the tensor-family table). Reading
# R23: the llama.cpp-style block of 256 weights in 210 bytes -- ql[128] (bytes
# 0..127, low four bits), qh[64] (bytes 128..191, high two bits), 16 signed
# byte scales (bytes 192..207), fp16 d (bytes 208..209). Weight i = 128n + 32u
# + l (half n, quarter u, lane l) takes nibble u // 2 of ql[64n + 32(u % 2) + l]
# and bits 2u, 2u+1 of qh[32n + l]; q = those six bits - 32 in -32..31 and
# w = d * scale[i // 16] * q.
# --------------------------------------------------------------------------

Q6_BLOCK_BYTES = 210


def quants_q6(blocks: np.ndarray) -> np.ndarray:
    """The 256 six-bit quants (-32..31) of each Q6_K block, in weight order."""
    b = np.asarray(blocks, dtype=np.uint8)
    ql = b[..., 0:128].astype(np.int64)
    qh = b[..., 128:192].astype(np.int64)
    q = np.empty(b.shape[:-1] + (QK,), dtype=np.int64)
    for n in range(2):
        for u in range(4):
            low = (ql[..., 64 * n + 32 * (u % 2): 64 * n + 32 * (u % 2) + 32] >> (4 * (u // 2))) & 15
            high = (qh[..., 32 * n: 32 * n + 32] >> (2 * u)) & 3
            q[..., 128 * n + 32 * u: 128 * n + 32 * u + 32] = (low | (high << 4)) - 32
    return q


def dequant_exact_q6(blocks: np.ndarray) -> np.ndarray:
    """Exact Q6_K weights in fp64 (``[..., nb, 210]`` -> ``[..., nb*256]``)."""
    b = np.ascontiguousarray(blocks, dtype=np.uint8)
    d = b[..., 208:210].copy().view("<f2")[..., 0].astype(np.float64)
    sc = b[..., 192:208].view(np.int8).astype(np.float64)
    q = quants_q6(b)
    w = d[..., None] * sc[..., np.arange(QK) // 16] * q
    return w.reshape(w.shape[:-2] + (w.shape[-2] * QK,))


def matmul_ref_q6(W_blocks: np.ndarray, X_bits: np.ndarray):
    """``matmul_ref`` for Q6_K weights ``[N][K/256][210]``: ``(Y, S)`` in fp64."""
    W = dequant_exact_q6(W_blocks)
    X = bf16_to_f64(X_bits)
    return X @ W.T, np.abs(X) @ np.abs(W).T


def make_block_q6(d: float, scales, q) -> np.ndarray:
    """One 210-byte Q6_K block from d (rounded to binary16), 16 scales in -128..127
    and 256 quants in -32..31 (Reading R23)."""
    q6 = np.asarray(q, dtype=np.int64) + 32
    b = np.zeros(Q6_BLOCK_BYTES, dtype=np.uint8)
    ql = np.zeros(128, dtype=np.int64)
    qh = np.zeros(64, dtype=np.int64)
    for n in range(2):
        for u in range(4):
            v = q6[128 * n + 32 * u: 128 * n + 32 * u + 32]
            ql[64 * n + 32 * (u % 2): 64 * n + 32 * (u % 2) + 32] |= (v & 15) << (4 * (u // 2))
            qh[32 * n: 32 * n + 32] |= (v >> 4) << (2 * u)
    b[0:128] = ql.astype(np.uint8)
    b[128:192] = qh.astype(np.uint8)
    b[192:208] = np.asarray(scales, dtype=np.int64).astype(np.int8).view(np.uint8)
    b[208:210] = np.array([d], dtype="<f2").view(np.uint8)
    return b


# --------------------------------------------------------------------------
# Q8 activation lane (the pages' "fast" GEMV lane policy, dp4a route, accuracy
# traded). Reading R22: the pages give no format; the one taken is int8
# activations with one fp32 scale per 256-wide column of X (the super-block
# width of the weights, so that the integer dot products of a whole super-block
# can be summed with the six-bit scales exactly). Per token row and column kb:
#   amax = max |x_k|;  d_x = RN_fp32(amax / 127);  inv = RN_fp32(127 / amax);
#   q_k = clamp(rint_even(RN_fp32(x_k * inv)), -127, 127)   (amax = 0: all zero)
# and the lane's product is y = sum_kb d_x * sum_k w_k * q_k (w exact).
# --------------------------------------------------------------------------

def quantize_x_q8(X_bits: np.ndarray):
    """Int8 activations of the Q8 lane: ``(q int64 [M][K], d_x float32 [M][K/256])``,
    every decision taken in fp32 exactly as written above."""
    x = bf16_to_f64(X_bits).astype(np.float32)  # exact: bf16 values are fp32 values
    M, K = x.shape
    xb = x.reshape(M, K // QK, QK)
    amax = np.abs(xb).max(axis=2)
    with np.errstate(divide="ignore"):
        d_x = np.where(amax > 0, np.float32(amax / np.float32(127)), np.float32(0)).astype(np.float32)
        inv = np.where(amax > 0, np.float32(np.float32(127) / amax), np.float32(0)).astype(np.float32)
    prod = (xb * inv[..., None]).astype(np.float32)  # one fp32 rounding per product
    q = np.clip(np.rint(prod), -127, 127).astype(np.int64)
    return q.reshape(M, K), d_x


def matmul_ref_q8lane(W_blocks: np.ndarray, X_bits: np.ndarray):
    """The Q8 lane's product in fp64: ``(Y, S)`` with Y = sum_kb d_x * w . q over the
    quantised activations, S = sum |w| * |d_x * q| (the lane's own scale)."""
    W = dequant_exact(W_blocks)
    q, d_x = quantize_x_q8(X_bits)
    xh = q.astype(np.float64) * np.repeat(d_x.astype(np.float64), QK, axis=1)
    return xh @ W.T, np.abs(xh) @ np.abs(W).T


# --------------------------------------------------------------------------
# Dense matmul: Y[m, n] = sum_k W[n, k] * X[m, k]
# --------------------------------------------------------------------------

def matmul_ref(W_blocks: np.ndarray, X_bits: np.ndarray):
    """Reference product and its absolute-value scale, both fp64.

    ``W_blocks``: ``[N][K/256][144]``; ``X_bits``: bf16 ``[M][K]``.
    Returns ``(Y, S)`` with ``Y = X @ W^T`` and ``S = |X| @ |W|^T``, ``[M][N]``.
    The GPU result passes when ``|Y_gpu - Y| <= 2e-3 * S`` elementwise.
    """
    W = dequant_exact(W_blocks)
    X = bf16_to_f64(X_bits)
    return X @ W.T, np.abs(X) @ np.abs(W).T


def matmul_rows_ref(W_blocks: np.ndarray, X_bits: np.ndarray, rows: np.ndarray):
    """``matmul_ref`` restricted to output columns (weight rows) ``rows``."""
    return matmul_ref(np.asarray(W_blocks)[rows], X_bits)


def check_tolerance(y_gpu: np.ndarray, Y: np.ndarray, S: np.ndarray, rel: float = REL_TOL):
    """Return (ok, worst err/S ratio) for the matmul tolerance."""
    err = np.abs(np.asarray(y_gpu, dtype=np.float64) - Y)
    ratio = err / np.maximum(S, 1e-300)
    ok = bool(np.all(err <= rel * S))
    return ok, float(ratio.max()) if ratio.size else 0.0


# --------------------------------------------------------------------------
# MoE: routing, permutation, grouped expert FFN, combine
# --------------------------------------------------------------------------

def route_topk(logits: np.ndarray, topk: int):
    """Top-k routing of each token (Readings R3, R4).

    Experts are ranked by fp32 router logit, descending, equal logits going
    to the lower expert id; the first ``topk`` in that order are taken, and
    their weights are the softmax over the selected logits (equal to the
    full softmax renormalised over the selected experts), in fp64.
    Returns ``ids`` int32 ``[M][topk]`` and ``w`` fp64 ``[M][topk]``.
    """
    logits = np.asarray(logits, dtype=np.float32)
    M, E = logits.shape
    ids = np.empty((M, topk), dtype=np.int32)
    w = np.empty((M, topk), dtype=np.float64)
    expert = np.arange(E)
    for t in range(M):
        lt = logits[t].astype(np.float64)
        order = np.lexsort((expert, -lt))  # last key is primary: -logit, then id
        sel = order[:topk]
        e = np.exp(lt[sel] - lt[sel].max())
        ids[t] = sel
        w[t] = e / e.sum()
    return ids, w


def router_logits_ref(X_bits: np.ndarray, Wr_bits: np.ndarray):
    """Router logits of the routing front (hipEngine 0.3.0 README, "Architecture at a
    glance": moe kernels): ``(L, S)`` with ``L = X @ Wr^T`` and ``S = |X| @ |Wr|^T``
    in fp64, X bf16 [M][H], Wr bf16 [E][H]. Reading R21: the router weights are bf16
    like the activations; the pages do not give their type."""
    X = bf16_to_f64(X_bits)
    W = bf16_to_f64(Wr_bits)
    return X @ W.T, np.abs(X) @ np.abs(W).T


def permute(ids: np.ndarray, E: int):
    """Stable counting sort of the (token, slot) pairs by expert (Reading R6).

    The flat index ``f = t*topk + j`` is sorted by (expert, f). Returns
    ``expert_offsets`` [E+1], ``perm`` (sorted row -> f), ``inv_perm``
    (f -> sorted row) and ``row_token`` (sorted row -> token), all int32.
    """
    ids = np.asarray(ids)
    topk = ids.shape[1]
    flat = ids.reshape(-1).astype(np.int64)
    perm = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    inv_perm = np.empty_like(perm)
    inv_perm[perm] = np.arange(perm.size)
    row_token = perm // topk
    return (offsets.astype(np.int32), perm.astype(np.int32), inv_perm.astype(np.int32),
            row_token.astype(np.int32))


def grouped_ref(W_experts: np.ndarray, A_bits: np.ndarray, expert_offsets: np.ndarray,
                row_gather=None, rows=None):
    """Grouped expert product, reference and scale in fp64.

    Row ``r`` of the sorted order belongs to the expert ``e`` with
    ``offsets[e] <= r < offsets[e+1]``; its input is ``A[row_gather[r]]``
    (or ``A[r]`` when ``row_gather`` is None) and its output
    ``A_row @ W_e^T``. ``rows`` restricts the result to those sorted rows.
    Returns ``(Y, S)`` of shape ``[len(rows)][N]``.
    """
    offs = np.asarray(expert_offsets, dtype=np.int64)
    total = int(offs[-1])
    rows = np.arange(total) if rows is None else np.asarray(rows)
    expert_of_row = np.searchsorted(offs, rows, side="right") - 1
    N = W_experts.shape[1]
    Y = np.empty((rows.size, N))
    S = np.empty((rows.size, N))
    for e in np.unique(expert_of_row):
        sel = np.nonzero(expert_of_row == e)[0]
        src = rows[sel] if row_gather is None else np.asarray(row_gather)[rows[sel]]
        Y[sel], S[sel] = matmul_ref(W_experts[e], np.asarray(A_bits)[src])
    return Y, S


def silu_mul(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """SiLU(g) * u = g / (1 + exp(-g)) * u, fp64."""
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g)) * np.asarray(u, dtype=np.float64)


def swiglu_bf16_ref(GU: np.ndarray, F: int) -> np.ndarray:
    """h = SiLU(gate) * up from a gate_up row block (gate columns 0..F-1, up F..2F-1;
    Reading R8), rounded RN_bf16(RN_fp32(.)) (Reading R7). Returns uint16 bits."""
    GU = np.asarray(GU, dtype=np.float64)
    return f64_to_bf16_bits(silu_mul(GU[:, :F], GU[:, F:2 * F]))


def combine_ref(O: np.ndarray, inv_perm: np.ndarray, w: np.ndarray):
    """y[t] = sum_j w[t,j] * O[inv_perm[t*topk + j]], in fixed j order, fp64.

    Returns ``(y, S)`` with ``S[t] = sum_j |w[t,j] * O[...]|``.
    """
    w = np.asarray(w, dtype=np.float64)
    M, topk = w.shape
    O = np.asarray(O, dtype=np.float64)
    inv = np.asarray(inv_perm).reshape(M, topk)
    y = np.zeros((M, O.shape[1]))
    S = np.zeros_like(y)
    for j in range(topk):
        term = w[:, j:j + 1] * O[inv[:, j]]
        y += term
        S += np.abs(term)
    return y, S


def combine_residual_ref(O: np.ndarray, inv_perm: np.ndarray, w: np.ndarray, R: np.ndarray):
    """The gate_combine_residual composite (hipEngine 0.3.0 README, "Core
    principles"): y[t] = R[t] + sum_j w[t,j] * O[inv_perm[t*topk + j]], fp64.

    Reading R18: the pages name the fused composite but not its order of
    operations; the sum over j is formed first (as in ``combine_ref``) and the
    residual added last. Returns ``(y, S)`` with ``S = |R| + sum_j |w*O|``.
    """
    y, S = combine_ref(O, inv_perm, w)
    R = np.asarray(R, dtype=np.float64)
    return R + y, np.abs(R) + S


def moe_layer_ref(logits, X_bits, W_gate_up, W_down, topk: int):
    """End-to-end fp64 MoE layer (no intermediate rounding): y[t] =
    sum_j w[t,j] * W_down[e_j] @ (SiLU(W_gate[e_j] x_t) * (W_up[e_j] x_t))."""
    E, twoF = W_gate_up.shape[0], W_gate_up.shape[1]
    F = twoF // 2
    ids, w = route_topk(logits, topk)
    X = bf16_to_f64(X_bits)
    y = np.zeros((X.shape[0], W_down.shape[1]))
    for e in np.unique(ids):
        tok, slot = np.nonzero(ids == e)
        Wgu = dequant_exact(W_gate_up[e])
        Wdn = dequant_exact(W_down[e])
        gu = X[tok] @ Wgu.T
        h = silu_mul(gu[:, :F], gu[:, F:])
        o = h @ Wdn.T
        np.add.at(y, tok, w[tok, slot][:, None] * o)
    return y


# --------------------------------------------------------------------------
# Encoding side (used only by the oracle's own pins)
# --------------------------------------------------------------------------

def pack_scale_min(sc: np.ndarray, m: np.ndarray) -> np.ndarray:
    """Inverse of ``scale_min_pairs``: eight (sc, m) pairs in 0..63 -> 12 bytes."""
    sc = np.asarray(sc, dtype=np.int64)
    m = np.asarray(m, dtype=np.int64)
    s = np.zeros(sc.shape[:-1] + (12,), dtype=np.int64)
    for j in range(4):
        s[..., j] = (sc[..., j] & 63) | ((sc[..., j + 4] >> 4) << 6)
        s[..., j + 4] = (m[..., j] & 63) | ((m[..., j + 4] >> 4) << 6)
        s[..., j + 8] = (sc[..., j + 4] & 15) | ((m[..., j + 4] & 15) << 4)
    return s.astype(np.uint8)


def pack_quants(q: np.ndarray) -> np.ndarray:
    """Inverse of ``quants``: 256 values in 0..15 -> 128 bytes."""
    q = np.asarray(q, dtype=np.int64)
    qs = np.zeros(q.shape[:-1] + (128,), dtype=np.int64)
    for c in range(4):
        qs[..., 32 * c: 32 * c + 32] = q[..., 64 * c: 64 * c + 32] | (q[..., 64 * c + 32: 64 * c + 64] << 4)
    return qs.astype(np.uint8)


def make_block(d: float, dmin: float, sc, m, q) -> np.ndarray:
    """Assemble one 144-byte block (d, dmin rounded to binary16)."""
    b = np.zeros(BLOCK_BYTES, dtype=np.uint8)
    b[0:2] = np.array([d], dtype="<f2").view(np.uint8)
    b[2:4] = np.array([dmin], dtype="<f2").view(np.uint8)
    b[4:16] = pack_scale_min(np.asarray(sc), np.asarray(m))
    b[16:144] = pack_quants(np.asarray(q))
    return b


def make_block_q5(d: float, dmin: float, sc, m, q) -> np.ndarray:
    """Assemble one 176-byte Q5_K block from d, dmin (rounded to binary16), eight
    (sc, m) pairs and 256 quants in 0..31 (Reading R19)."""
    q = np.asarray(q, dtype=np.int64)
    b = np.zeros(Q5_BLOCK_BYTES, dtype=np.uint8)
    b[0:2] = np.array([d], dtype="<f2").view(np.uint8)
    b[2:4] = np.array([dmin], dtype="<f2").view(np.uint8)
    b[4:16] = pack_scale_min(np.asarray(sc), np.asarray(m))
    qh = np.zeros(32, dtype=np.int64)
    for c in range(4):
        for h in range(2):
            qh |= ((q[64 * c + 32 * h: 64 * c + 32 * h + 32] >> 4) & 1) << (2 * c + h)
    b[16:48] = qh.astype(np.uint8)
    b[48:176] = pack_quants(q & 15)
    return b


def quantize_brute_force(w: np.ndarray, d: float, dmin: float):
    """Search, per sub-block, every (sc, m) in 0..63 x 0..63 and q in 0..15 for
    an exact representation of the 256 fp64 weights ``w`` given ``d``, ``dmin``.

    Returns ``(sc[8], m[8], q[256])`` or raises ``ValueError`` if a sub-block
    has no exact representation.
    """
    d = float(np.float16(d))
    dmin = float(np.float16(dmin))
    sc_out = np.zeros(8, dtype=np.int64)
    m_out = np.zeros(8, dtype=np.int64)
    q_out = np.zeros(QK, dtype=np.int64)
    qv = np.arange(16, dtype=np.float64)
    for j in range(8):
        wj = np.asarray(w[SUB * j: SUB * (j + 1)], dtype=np.float64)
        found = False
        for sc in range(64):
            for mm in range(64):
                cand = d * sc * qv - dmin * mm            # the 16 values this pair can give
                hit = wj[:, None] == cand[None, :]
                if hit.any(axis=1).all():
                    sc_out[j], m_out[j] = sc, mm
                    q_out[SUB * j: SUB * (j + 1)] = hit.argmax(axis=1)
                    found = True
                    break
            if found:
                break
        if not found:
            raise ValueError(f"sub-block {j} has no exact Q4_K representation")
    return sc_out, m_out, q_out


# --------------------------------------------------------------------------
# Load-time decode repack (hipEngine 0.3.0 README, "GGUF Support": the
# "decode-repacked" layouts). Reading R17: the pages name repacked layouts
# but give none; the layout taken here is a pure byte permutation (the same
# 144 bytes per super-block):
#   * rows are grouped in tiles of 128; tile T's super-block column kb is the
#     contiguous run of rows 128T .. 128T+127, so the output is indexed
#     [T][kb][r][144];
#   * inside a row-block, bytes 0..15 (d, dmin, packed scales) stay, and the
#     quant byte at 16 + 32c + 8t + e (chunk c, quarter t, e = 0..7) moves to
#     16 + 32t + 8c + e;
#   * rows past N, up to the next multiple of 128, are zero bytes.
# --------------------------------------------------------------------------

REPACK_ROWS = 128


def repack_ref(W_blocks: np.ndarray) -> np.ndarray:
    """The repacked byte array (flat uint8) of W_blocks [N][K/256][144]."""
    N, nkb, _ = W_blocks.shape
    tiles = -(-N // REPACK_ROWS)
    out = np.zeros((tiles, nkb, REPACK_ROWS, BLOCK_BYTES), dtype=np.uint8)
    for n in range(N):
        T, r = divmod(n, REPACK_ROWS)
        for kb in range(nkb):
            src = W_blocks[n, kb]
            dst = out[T, kb, r]
            dst[:16] = src[:16]
            for c in range(4):
                for t in range(4):
                    dst[16 + 32 * t + 8 * c:16 + 32 * t + 8 * c + 8] = src[16 + 32 * c + 8 * t:16 + 32 * c + 8 * t + 8]
    return out.reshape(-1)


def unrepack_ref(Wr: np.ndarray, N: int, K: int) -> np.ndarray:
    """Inverse of repack_ref: the [N][K/256][144] blocks back from the flat bytes."""
    nkb = K // QK
    tiles = -(-N // REPACK_ROWS)
    R = Wr.reshape(tiles, nkb, REPACK_ROWS, BLOCK_BYTES)
    out = np.zeros((N, nkb, BLOCK_BYTES), dtype=np.uint8)
    for n in range(N):
        T, r = divmod(n, REPACK_ROWS)
        for kb in range(nkb):
            src = R[T, kb, r]
            dst = out[n, kb]
            dst[:16] = src[:16]
            for c in range(4):
                for t in range(4):
                    dst[16 + 32 * c + 8 * t:16 + 32 * c + 8 * t + 8] = src[16 + 32 * t + 8 * c:16 + 32 * t + 8 * c + 8]
    return out
