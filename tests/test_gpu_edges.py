"""GPU parity on edge inputs: extreme Q4_K blocks through the matmul kernels, and
activation columns with a wide dynamic range, all-zero columns, bf16 subnormals and
large magnitudes; the grouped tensor-core path's fp16 range latch.

Bounds as in test_gpu_parity: |y - y_ref| <= 2e-3 * sum|w*x| per fp32 output against
the fp64 oracle; the expected values come from oracle/ only.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import q4k as O
from tests.gpu_util import dev, host

pytestmark = pytest.mark.gpu

q = pytest.importorskip("q4_weight_only_super_b200")

RANGE = 10  # Q4K_ERR_DEVICE_RANGE


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    q.lib()
    assert q.q4k_last_device_status() == 0
    yield
    assert q.q4k_last_device_status() == 0


def _assert_tol(y, Y, S, what=""):
    ok, ratio = O.check_tolerance(y, Y, S)
    assert ok, f"{what}: worst err/S = {ratio:.3e} (limit 2e-3)"


# ---------------------------------------------------------------- edge weights --
# (d, dmin) pairs at the ends of binary16 (65504, subnormal 6e-8, zero, negative) and
# (sc, m, q) patterns at the ends of their fields; every block is a legal Q4_K block.

_DD = [(65504.0, 0.0), (6e-8, 6e-8), (1.0, 65504.0), (0.0, 0.0), (-2.0, -1.5),
       (1e-3, -1e-3), (-65504.0, 65504.0), (0.5, 0.25)]
_PAT = [(63, 63, 15), (1, 0, 1), (0, 63, 0), (0, 0, 15), (63, 0, 15), (5, 7, None)]


def _edge_pool(rng, limit=None):
    """Edge blocks; with `limit`, only blocks whose every sub-block keeps the grouped
    tensor-core path's range bound 15 * |d * sc| + |dmin * m| <= limit (the fp16 range
    check is made on that bound, not on the weights actually present)."""
    pool = []
    for d, dmin in _DD:
        for sc, m, qv in _PAT:
            qs = rng.integers(0, 16, 256) if qv is None else [qv] * 256
            if limit is not None and 15 * abs(float(np.float16(d)) * sc) + abs(float(np.float16(dmin)) * m) > limit:
                continue
            pool.append(O.make_block(d, dmin, [sc] * 8, [m] * 8, qs))
    return np.stack(pool)


def _edge_matrix(seed, N, K, limit=None):
    """N x K Q4_K matrix: about half its blocks from the edge pool, the rest random."""
    rng = np.random.default_rng(seed)
    pool = _edge_pool(rng, limit)
    W = synth.q4k_random_blocks(rng, N, K)
    pick = rng.random(W.shape[:2]) < 0.5
    idx = rng.integers(0, len(pool), W.shape[:2])
    W[pick] = pool[idx[pick]]
    return W


def _bits(a):
    return synth.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _edge_activations(seed, M, K):
    """bf16 rows: N(0,1); per 256-column an outlier 2^15 among values ~2^-15 (ratio 2^30);
    alternate all-zero columns; bf16 subnormals k * 2^-133; N(0,1) * 1e4; all negative;
    one non-zero per column; then N(0,1) rows."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((max(M, 8), K)).astype(np.float32)
    nkb = K // 256
    wide = rng.standard_normal(K).astype(np.float32) * 2.0 ** -15
    wide[np.arange(nkb) * 256 + rng.integers(0, 256, nkb)] = 2.0 ** 15
    X[1] = wide
    X[2, :] = rng.standard_normal(K)
    for kb in range(0, nkb, 2):
        X[2, kb * 256:(kb + 1) * 256] = 0.0
    X[3] = (rng.integers(1, 128, K) * rng.choice([-1.0, 1.0], K)).astype(np.float64) * 2.0 ** -133
    X[4] = rng.standard_normal(K) * 1e4
    X[5] = -np.abs(rng.standard_normal(K))
    one = np.zeros(K, np.float32)
    one[np.arange(nkb) * 256 + rng.integers(0, 256, nkb)] = rng.standard_normal(nkb)
    X[6] = one
    return _bits(X[:M])


@pytest.mark.parametrize("M", [1, 8, 9, 17, 32])
def test_gemv_edge_weights_and_activations(M):
    N, K = 272, 256 * 7
    W = _edge_matrix(900 + M, N, K)
    X = _edge_activations(910 + M, M, K)
    Wd, Xd = dev(W), dev(X)
    Y, S = O.matmul_ref(W, X)
    _assert_tol(host(q.q4k_gemv(Wd, Xd, N, K)), Y, S, f"edge gemv M={M}")
    _assert_tol(host(q.q4k_gemv_repacked(q.q4k_repack(Wd, N, K), Xd, N, K)), Y, S, f"edge repacked M={M}")


@pytest.mark.parametrize("row", range(7))
def test_gemv_edge_activation_rows_one_token(row):
    """Each edge activation row alone (the one-token path)."""
    N, K = 1040, 256 * 69
    W = synth.q4k_random_blocks(np.random.default_rng(920), N, K)
    X = _edge_activations(921, 8, K)[row:row + 1]
    Y, S = O.matmul_ref(W, X)
    _assert_tol(host(q.q4k_gemv(dev(W), dev(X), N, K)), Y, S, f"edge row {row}")


@pytest.mark.parametrize("M", [1, 9, 32])
def test_q5k_q80_gemv_edge_blocks(M):
    rng = np.random.default_rng(930 + M)
    N, K = 272, 256 * 5
    pool5 = []
    for d, dmin in _DD:
        for sc, m, qv in [(63, 63, 31), (1, 0, 16), (0, 63, 0), (63, 0, 31), (9, 3, None)]:
            qs = rng.integers(0, 32, 256) if qv is None else [qv] * 256
            pool5.append(O.make_block_q5(d, dmin, [sc] * 8, [m] * 8, qs))
    pool5 = np.stack(pool5)
    W5 = synth.q5k_random_blocks(rng, N, K)
    pick = rng.random(W5.shape[:2]) < 0.5
    W5[pick] = pool5[rng.integers(0, len(pool5), W5.shape[:2])[pick]]
    X = _edge_activations(940 + M, M, K)
    Y, S = O.matmul_ref_q5(W5, X)
    _assert_tol(host(q.q5k_gemv(dev(W5), dev(X), N, K)), Y, S, f"edge q5k M={M}")

    pool8 = np.stack([O.make_block_q80(d, qv) for d in (65504.0, -65504.0, 6e-8, 0.0, -1.0, 1e-3)
                      for qv in ([127] * 32, [-128] * 32, [0] * 32, list(range(-16, 16)))])
    W8 = synth.q80_random_blocks(rng, N, K)
    pick = rng.random(W8.shape[:2]) < 0.5
    W8[pick] = pool8[rng.integers(0, len(pool8), W8.shape[:2])[pick]]
    Y8, S8 = O.matmul_ref_q80(W8, X)
    _assert_tol(host(q.q80_gemv(dev(W8), dev(X), N, K)), Y8, S8, f"edge q80 M={M}")


@pytest.mark.parametrize("M", [1, 32])
def test_q8lane_edge_blocks(M):
    """The Q8 lane on edge blocks: tight against its own product (the lane's integer sums
    are exact; fp32 for the rest), zero columns give zero codes."""
    N, K = 272, 256 * 7
    W = _edge_matrix(950 + M, N, K)
    X = _edge_activations(951 + M, M, K)
    y = host(q.q4k_gemv_q8(dev(W), dev(X), N, K)).astype(np.float64)
    Yl, Sl = O.matmul_ref_q8lane(W, X)
    assert np.all(np.abs(y - Yl) <= 3e-5 * Sl + 1e-30)


def test_gemm_edge_weights():
    """Prefill GEMM (bf16 tensor-core operands) on edge blocks with N(0,1), wide-range,
    zero-column, large and one-hot activation rows.

    The GEMM multiplies bf16 weights RN_bf16(RN_fp32(w)) (Reading R2). bf16 keeps 8
    significant bits (unit roundoff 2^-8), so where one product dominates an output (the
    one-hot row) the weight rounding alone reaches ~3.5e-3 * sum|w*x| on these blocks,
    beyond the 2e-3 of the random workloads. The kernel is therefore pinned to the
    defined product itself: against sum_k RN_bf16(w) * x in fp64 it may differ only by
    fp32 accumulation (K * 2^-23 * sum|w*x|), and against the exact product by at most
    the bf16 rounding bound plus that."""
    M, N, K = 300, 512, 256 * 7
    W = _edge_matrix(960, N, K)
    X = _edge_activations(961, M, K)
    X[3] = _bits(np.random.default_rng(962).standard_normal(K))  # subnormal products: separate test
    Y, S = O.matmul_ref(W, X)
    y = host(q.q4k_gemm(dev(W), dev(X), N, K)).astype(np.float64)
    Yb = O.bf16_to_f64(X) @ O.bf16_to_f64(O.dequant_bf16_bits(W)).T   # the bf16-weight product
    acc = K * 2.0 ** -23  # fp32 accumulation, truncating adds allowed
    assert np.all(np.abs(y - Yb) <= acc * S + 1e-30), float((np.abs(y - Yb) / np.maximum(S, 1e-300)).max())
    assert np.all(np.abs(y - Y) <= (2.0 ** -8 + acc) * S + 1e-30)
    rnd = np.random.default_rng(963)                 # the workloads' kind of data: within 2e-3
    Xr = synth.bf16_normal(rnd, (64, K))
    Yr, Sr = O.matmul_ref(W, Xr)
    _assert_tol(host(q.q4k_gemm(dev(W), dev(Xr), N, K)), Yr, Sr, "edge gemm, N(0,1) activations")


def test_gemm_subnormal_activations():
    """bf16 subnormal activations (k * 2^-133) against ordinary weights: products and sums
    lie in the fp32 subnormal range; the result is checked with an absolute floor of a few
    fp32 subnormal steps (2^-149) per input."""
    M, N, K = 8, 256, 1024
    W = synth.q4k_random_blocks(np.random.default_rng(963), N, K)
    rng = np.random.default_rng(964)
    X = _bits((rng.integers(1, 128, (M, K)) * rng.choice([-1.0, 1.0], (M, K))) * 2.0 ** -133)
    Y, S = O.matmul_ref(W, X)
    y = host(q.q4k_gemm(dev(W), dev(X), N, K)).astype(np.float64)
    assert np.all(np.abs(y - Y) <= 2e-3 * S + K * 2.0 ** -149)


# ------------------------------------------------------------ grouped expert path --

def _grouped_case(seed, E, N, K, rows, limit):
    rng = np.random.default_rng(seed)
    W = np.stack([_edge_matrix(seed + e, N, K, limit=limit) for e in range(E)])
    counts = rng.multinomial(rows, np.ones(E) / E)
    offs = np.r_[0, np.cumsum(counts)].astype(np.int32)
    A = _edge_activations(seed + 99, rows, K)
    A[3] = _bits(rng.standard_normal(K))  # keep subnormal products out of the fp16 tensor path
    A[4] = _bits(rng.standard_normal(K) * 3e3)  # |x| <= 65504 for the fp16 operands
    return W, A, offs


@pytest.mark.parametrize("hint", [32, 64])
def test_grouped_edge_weights(hint):
    """Decode (GEMV, hint <= 32 = the largest expert's rows) and tensor-core grouped
    paths on edge blocks whose weights fit fp16."""
    E, N, K, rows = 4, 256, 512, 40
    W, A, offs = _grouped_case(970 + hint, E, N, K, rows, limit=65504.0)
    assert int(np.diff(offs).max()) <= 32
    Wd, Ad, od = dev(W), dev(A), dev(offs)
    out = host(q.moe_q4k_grouped(Wd, E, N, K, Ad, od, rows, hint, q.ACT_NONE))
    Y, S = O.grouped_ref(W, A, offs)
    _assert_tol(out, Y, S, f"edge grouped hint={hint}")


def test_grouped_range_latch_weights():
    """A weight beyond the fp16 range on the tensor-core grouped path latches
    Q4K_ERR_DEVICE_RANGE (no fault); the next valid call is correct and clean."""
    E, N, K, rows = 2, 256, 512, 64
    W, A, offs = _grouped_case(980, E, N, K, rows, limit=65504.0)
    bad = W.copy()
    bad[1, 7, 1] = O.make_block(65504.0, 0.0, [1] * 8, [0] * 8, [2] * 256)  # w = 131008 > 65504
    Wd, Ad, od = dev(bad), dev(A), dev(offs)
    q.moe_q4k_grouped(Wd, E, N, K, Ad, od, rows, rows, q.ACT_NONE)
    assert q.q4k_last_device_status() == RANGE
    out = host(q.moe_q4k_grouped(dev(W), E, N, K, Ad, od, rows, rows, q.ACT_NONE))
    assert q.q4k_last_device_status() == 0
    Y, S = O.grouped_ref(W, A, offs)
    _assert_tol(out, Y, S, "after range latch")


def test_grouped_range_latch_activations():
    """An activation above 65504 (a legal bf16) on the tensor-core grouped path latches
    Q4K_ERR_DEVICE_RANGE."""
    E, N, K, rows = 2, 256, 512, 64
    W, A, offs = _grouped_case(981, E, N, K, rows, limit=65504.0)
    A2 = A.copy()
    A2[5, 17] = _bits(np.array([1.0e5]))[0]
    q.moe_q4k_grouped(dev(W), E, N, K, dev(A2), dev(offs), rows, rows, q.ACT_NONE)
    assert q.q4k_last_device_status() == RANGE
