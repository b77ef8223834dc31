"""GPU parity of the decode form of the grouped expert matmul (moe_q4k_grouped with
max_rows_hint <= 32): the grouped stationary GEMV (K up to 20 super-blocks) and the
grouped ring GEMV (longer K), against the oracle, against the dense decode GEMV of
each expert (bit for bit: same operands, same summation order), and with offsets
that its own checks must refuse.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import q4k as O
from tests.gpu_util import bf16_ulp, dev, host

pytestmark = pytest.mark.gpu

q = pytest.importorskip("q4_weight_only_super_b200")

BOUNDS = 8  # Q4K_ERR_DEVICE_BOUNDS


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    q.lib()
    yield
    assert q.q4k_last_device_status() == 0


def _assert_tol(y, Y, S, what=""):
    ok, ratio = O.check_tolerance(y, Y, S)
    assert ok, f"{what}: worst err/S = {ratio:.3e} (limit 2e-3)"
    return ratio


def _case(seed, E, N, K, counts, A_rows=None):
    """Experts' weights, activation rows and a gather over them, rows sorted by expert."""
    rng = np.random.default_rng(seed)
    W = np.stack([synth.q4k_random_blocks(rng, N, K) for _ in range(E)])
    offs = np.r_[0, np.cumsum(counts)].astype(np.int32)
    rows = int(offs[-1])
    A_rows = A_rows or max(1, rows // 2)
    A = synth.bf16_normal(rng, (A_rows, K))
    gather = rng.integers(0, A_rows, size=rows).astype(np.int32)
    return W, A, offs, gather


def _check_both(W, A, offs, gather, hint, what):
    E, N, K = W.shape[0], W.shape[1], W.shape[2] * 256
    rows = int(offs[-1])
    Wd, Ad, od, gd = dev(W), dev(A), dev(offs), dev(gather)
    y = host(q.moe_q4k_grouped(Wd, E, N, K, Ad, od, rows, hint, q.ACT_NONE, row_gather=gd))
    Y, S = O.grouped_ref(W, A, offs, row_gather=gather)
    ratio = _assert_tol(y, Y, S, what)
    h = host(q.moe_q4k_grouped(Wd, E, N, K, Ad, od, rows, hint, q.ACT_SWIGLU, row_gather=gd))
    h_ref = O.swiglu_bf16_ref(y, N // 2)
    ulps = np.abs(O.bf16_to_f64(h) - O.bf16_to_f64(h_ref)) / bf16_ulp(h_ref)
    assert np.all(ulps <= 1.0), f"{what} SwiGLU: max {ulps.max():.1f} bf16 ulp"
    return y, ratio


@pytest.mark.parametrize("K", [256, 768, 2048, 2816, 4096, 5120])
def test_grouped_decode_shapes(K):
    """One and two super-blocks a warp (K <= 2560 and 2816..5120), ragged experts,
    empty experts, a gather with repeats."""
    counts = [3, 0, 8, 1, 0, 0, 5, 2]
    W, A, offs, gather = _case(700 + K // 256, len(counts), 288, K, counts)
    _check_both(W, A, offs, gather, 8, f"K={K}")


def test_grouped_decode_many_rows_per_expert():
    """Experts with more than 8 rows: several token groups stream the same weights."""
    counts = [30, 9, 0, 17, 1, 8, 32, 0]
    W, A, offs, gather = _case(711, len(counts), 256, 2048, counts, A_rows=40)
    _check_both(W, A, offs, gather, 32, "rows per expert up to 32")


def test_grouped_decode_ring_path_long_k():
    """K beyond one CTA's warps (24 super-blocks): the grouped ring GEMV."""
    counts = [2, 7, 0, 4]
    W, A, offs, gather = _case(712, len(counts), 256, 24 * 256, counts)
    _check_both(W, A, offs, gather, 8, "ring K=6144")


def test_grouped_decode_equals_dense_per_expert():
    """Each expert's rows equal the dense 1..8-token GEMV of that expert's matrix on
    the same activation rows, bit for bit (the decode shapes of the MoE layer)."""
    for N, K in [(1536, 2048), (2048, 768)]:
        counts = [1, 8, 0, 3, 5]
        W, A, offs, gather = _case(713 + K, len(counts), N, K, counts)
        Wd, Ad, od, gd = dev(W), dev(A), dev(offs), dev(gather)
        rows = int(offs[-1])
        y = host(q.moe_q4k_grouped(Wd, len(counts), N, K, Ad, od, rows, 8, q.ACT_NONE, row_gather=gd))
        for e in range(len(counts)):
            a, b = offs[e], offs[e + 1]
            if b == a:
                continue
            ye = host(q.q4k_gemv(dev(W[e]), dev(A[gather[a:b]]), N, K))
            assert np.array_equal(y[a:b].view(np.uint32), ye.view(np.uint32)), f"expert {e} (N={N}, K={K})"


def test_grouped_decode_batch_invariant():
    """A row's result does not depend on the other rows of its expert or the batch."""
    N, K = 1536, 2048
    W, A, offs, gather = _case(714, 4, N, K, [6, 2, 8, 3])
    Wd, Ad = dev(W), dev(A)
    y = host(q.moe_q4k_grouped(Wd, 4, N, K, Ad, dev(offs), int(offs[-1]), 8, q.ACT_NONE,
                               row_gather=dev(gather)))
    # each row alone, as the only row of its expert
    for r in [0, 5, 7, 13, 18]:
        e = int(np.searchsorted(offs, r, side="right") - 1)
        o1 = np.zeros(5, np.int32)
        o1[e + 1:] = 1
        y1 = host(q.moe_q4k_grouped(Wd, 4, N, K, Ad, dev(o1), 1, 1, q.ACT_NONE,
                                    row_gather=dev(gather[r:r + 1])))
        assert np.array_equal(y1[0].view(np.uint32), y[r].view(np.uint32)), f"row {r}"


def test_grouped_decode_moe_shapes_sampled_dense_equal():
    """The MoE decode layer's stages at 32 tokens: every (token, expert) row of gate_up
    equals the dense GEMV of its expert."""
    inp = synth.moe_decode(3, 32)
    E, H, F = inp["E"], inp["H"], inp["F"]
    r = q.moe_route_permute(dev(inp["logits"]), 8)
    offs = host(r["expert_offsets"])
    rt = host(r["row_token"])
    Wgu, X = dev(inp["W_gate_up"]), dev(inp["X"])
    rows = 32 * 8
    gu = host(q.moe_q4k_grouped(Wgu, E, 2 * F, H, X, r["expert_offsets"], rows, 32, q.ACT_NONE,
                                row_gather=r["row_token"]))
    busiest = np.argsort(np.diff(offs))[::-1][:3]
    for e in busiest:
        a, b = offs[e], offs[e + 1]
        for c0 in range(a, b, 8):  # the dense GEMV takes up to 8 tokens in one class
            c1 = min(b, c0 + 8)
            ye = host(q.q4k_gemv(dev(inp["W_gate_up"][e]), dev(inp["X"][rt[c0:c1]]), 2 * F, H))
            assert np.array_equal(gu[c0:c1].view(np.uint32), ye.view(np.uint32)), f"expert {e}"


@pytest.mark.parametrize("bad", ["decreasing", "past_rows", "negative"])
def test_grouped_decode_bad_offsets_latch(bad):
    """Offsets that are not a non-decreasing sequence inside [0, rows]: the kernel's own
    check latches Q4K_ERR_DEVICE_BOUNDS and writes nothing; the next call is clean."""
    counts = [3, 2, 4]
    W, A, offs, gather = _case(715, 3, 256, 2048, counts)
    rows = int(offs[-1])
    o = offs.copy()
    if bad == "decreasing":
        o[2] = o[1] - 1
    elif bad == "past_rows":
        o[3] = rows + 5
    else:
        o[0] = -1
    Wd, Ad, gd = dev(W), dev(A), dev(gather)
    out = torch.full((rows, 256), 7.0, dtype=torch.float32, device="cuda")
    q.moe_q4k_grouped(Wd, 3, 256, 2048, Ad, dev(o), rows, 8, q.ACT_NONE, row_gather=gd, out=out)
    assert q.q4k_last_device_status() == BOUNDS
    assert torch.all(out == 7.0).item(), "nothing is written"
    assert q.q4k_last_device_status() == 0
    y = host(q.moe_q4k_grouped(Wd, 3, 256, 2048, Ad, dev(offs), rows, 8, q.ACT_NONE, row_gather=gd))
    assert q.q4k_last_device_status() == 0
    _assert_tol(y, *O.grouped_ref(W, A, offs, row_gather=gather), "after the latch")


# ------------------------------------------------ routing + gate_up, one launch --

@pytest.mark.parametrize("case", ["M1", "M8", "M32", "E16_top3", "E256_top8"])
def test_route_gate_up_equals_the_two_calls(case):
    """moe_route_gate_up == moe_route_permute then moe_q4k_grouped (SwiGLU), bit for bit:
    every routing output and the bf16 h."""
    if case == "E16_top3":
        M, topk, inp = 20, 3, synth.moe_layer(21, 20, E=16, H=1536, F=512)
    elif case == "E256_top8":
        M, topk, inp = 12, 8, synth.moe_layer(22, 12, E=256, H=1536, F=256)
    else:
        M, topk = int(case[1:]), 8
        inp = synth.moe_decode(3, M)
    E, H, F = inp["E"], inp["H"], inp["F"]
    L, X, Wgu = dev(inp["logits"]), dev(inp["X"]), dev(inp["W_gate_up"])
    r = q.moe_route_permute(L, topk)
    h_ref = host(q.moe_q4k_grouped(Wgu, E, 2 * F, H, X, r["expert_offsets"], M * topk, M, q.ACT_SWIGLU,
                                   row_gather=r["row_token"]))
    for _ in range(2):
        rr, h = q.moe_route_gate_up(L, topk, Wgu, 2 * F, H, X)
        for k in ("topk_ids", "expert_offsets", "perm", "inv_perm", "row_token"):
            assert np.array_equal(host(rr[k]), host(r[k])), k
        assert np.array_equal(host(rr["topk_w"]).view(np.uint32), host(r["topk_w"]).view(np.uint32))
        assert np.array_equal(host(h).view(np.uint16), h_ref.view(np.uint16))
    assert q.q4k_last_device_status() == 0


def test_route_gate_up_no_tokens():
    """M == 0: only the expert offsets are cleared."""
    E = 128
    offs = torch.full((E + 1,), 7, dtype=torch.int32, device="cuda")
    L = torch.empty(0, E, dtype=torch.float32, device="cuda")
    W = torch.empty(16, dtype=torch.uint8, device="cuda")
    X = torch.empty(0, 2048, dtype=torch.int16, device="cuda")
    out = {k: torch.empty(16, dtype=torch.int32, device="cuda")
           for k in ("topk_ids", "perm", "inv_perm", "row_token")}
    out["topk_w"] = torch.empty(16, dtype=torch.float32, device="cuda")
    out["expert_offsets"] = offs
    q.moe_route_gate_up(L, 8, W, 1536, 2048, X, out=out, h=torch.empty(16, dtype=torch.bfloat16, device="cuda"))
    assert int(torch.count_nonzero(offs)) == 0
