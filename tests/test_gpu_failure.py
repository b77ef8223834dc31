"""Failure detection on the GPU without a fault: a bounded wait is made to expire.

The library's test hook (q4k_test_wait_fault) shortens the wait limit to 200 us and
makes the weight producer of every CTA skip its first stage -- no copy and no arrival
-- so the roles waiting for it reach the limit. The kernel must return (no hang, no
trap), latch Q4K_ERR_DEVICE_TIMEOUT (7) in the status word, leave the context usable,
and the next normal call must be correct (fail closed: hipEngine 0.3.0 README, "Core
principles").
"""
import numpy as np
import pytest

import synth
from oracle import q4k as O
from tests.gpu_util import dev, host

pytestmark = pytest.mark.gpu

q = pytest.importorskip("q4_weight_only_super_b200")

TIMEOUT = 7  # Q4K_ERR_DEVICE_TIMEOUT


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    q.lib()
    q.q4k_test_wait_fault(-1, 0)
    assert q.q4k_last_device_status() == 0
    yield
    q.q4k_test_wait_fault(-1, 0)
    assert q.q4k_last_device_status() == 0


def _run(op):
    if op == "moe_route_gate_up":  # routing inside the grouped GEMV (MoE decode, one launch)
        inp = synth.moe_layer(997, 4, E=16, H=1536, F=256)
        E, H, F = inp["E"], inp["H"], inp["F"]
        Lg, Xd, Wd = dev(inp["logits"]), dev(inp["X"]), dev(inp["W_gate_up"])
        call = lambda: q.moe_route_gate_up(Lg, 2, Wd, 2 * F, H, Xd)[1]
        return call, inp, None
    if op == "moe_dec":  # grouped stationary GEMV (MoE decode)
        rng = np.random.default_rng(996)
        E, N, K = 4, 256, 2048
        W = np.stack([synth.q4k_random_blocks(rng, N, K) for _ in range(E)])
        X = synth.bf16_normal(rng, (12, K))
        offs = np.array([0, 3, 3, 11, 12], dtype=np.int32)
        Wd, Xd, od = dev(W), dev(X), dev(offs)
        call = lambda: q.moe_q4k_grouped(Wd, E, N, K, Xd, od, 12, 8, q.ACT_NONE)
        return call, (W, offs), X
    if op.startswith("gemv"):
        M = 1 if op == "gemv_1tok" else 17  # 1..8 tokens: stationary kernel; 17..32: ring kernel
        N, K = 272, 256 * 69                 # K split over a cluster in both kernels
        W, X = synth.gemv_small(990 + M, N=N, K=K, M=M)
        return (lambda: q.q4k_gemv(dev(W), dev(X), N, K)), W, X
    M, N, K = 300, 256, 1024
    W, X = synth.gemv_small(995, N=N, K=K, M=M)
    return (lambda: q.q4k_gemm(dev(W), dev(X), N, K)), W, X


@pytest.mark.parametrize("op", ["gemv_1tok", "gemv_17tok", "gemm", "moe_dec", "moe_route_gate_up"])
def test_bounded_wait_expires_and_recovers(op):
    call, W, X = _run(op)
    assert q.q4k_last_device_status() == 0
    try:
        q.q4k_test_wait_fault(0, 200_000)  # skip stage 0 everywhere; 200 us limit
        call()
        assert q.q4k_last_device_status() == TIMEOUT
    finally:
        q.q4k_test_wait_fault(-1, 0)
    assert q.q4k_last_device_status() == 0
    y = host(call())
    assert q.q4k_last_device_status() == 0
    if op == "moe_route_gate_up":  # h after the timeout equals the two-call path's
        inp = W
        r = q.moe_route_permute(dev(inp["logits"]), 2)
        h_ref = host(q.moe_q4k_grouped(dev(inp["W_gate_up"]), inp["E"], 2 * inp["F"], inp["H"], dev(inp["X"]),
                                       r["expert_offsets"], 8, 4, q.ACT_SWIGLU, row_gather=r["row_token"]))
        assert np.array_equal(y.view(np.uint16), h_ref.view(np.uint16))
        return
    Y, S = O.grouped_ref(W[0], X, W[1]) if op == "moe_dec" else O.matmul_ref(W, X)
    ok, ratio = O.check_tolerance(y, Y, S)
    assert ok, f"{op} after a timeout: worst err/S = {ratio:.3e}"
