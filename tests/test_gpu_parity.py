"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Bit-exact for dequantised weights, routing ids, offsets and permutations;
|y - y_ref| <= 2e-3 * sum|w*x| per fp32 matmul output; routing weights within
1e-6; combine within 1e-6 * sum|w*O|; SwiGLU output within one bf16 ulp of the
value rounded from the GPU's own gate/up products.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import q4k as O
from tests.gpu_util import bf16_ulp, dev, host, sample_rows

pytestmark = pytest.mark.gpu

q = pytest.importorskip("q4_weight_only_super_b200")


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    q.lib()
    yield
    assert q.q4k_last_device_status() == 0


def _assert_tol(y, Y, S, what=""):
    ok, ratio = O.check_tolerance(y, Y, S)
    assert ok, f"{what}: worst err/S = {ratio:.3e} (limit 2e-3)"
    return ratio


# ------------------------------------------------------------------ dequant --

def _edge_blocks():
    blocks = []
    for d, dmin in [(65504.0, 0.0), (6e-8, 6e-8), (1.0, 65504.0), (0.0, 0.0), (-2.0, -1.5)]:
        for (sc, m, qv) in [(63, 63, 15), (1, 0, 1), (0, 63, 0)]:
            blocks.append(O.make_block(d, dmin, [sc] * 8, [m] * 8, [qv] * 256))
    return np.stack(blocks)


@pytest.mark.parametrize("out_bf16", [False, True])
def test_dequant_bit_exact(out_bf16):
    W, _ = synth.gemv_small(0)
    blocks = np.concatenate([W.reshape(-1, 144), _edge_blocks()])
    out = host(q.q4k_dequant(dev(blocks), out_bf16=out_bf16))
    if out_bf16:
        ref = O.dequant_bf16_bits(blocks[None])[0]
        assert np.array_equal(out, ref)
    else:
        ref = O.dequant_f32(blocks[None])[0]
        assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))


def test_dequant_empty():
    out = torch.empty(16, dtype=torch.float32, device="cuda")
    assert q.lib().q4k_dequant(out.data_ptr(), 0, 0, out.data_ptr(), None) == 0


# --------------------------------------------------------------------- GEMV --

def test_gemv_single_matrix_full():
    W, X = synth.gemv_small(0)
    y = host(q.q4k_gemv(dev(W), dev(X), 256, 2048))
    Y, S = O.matmul_ref(W, X)
    _assert_tol(y, Y, S, "256x2048 M=1")


@pytest.mark.parametrize("N,K", [(16, 256), (48, 512), (80, 1792), (272, 4096), (1040, 256 * 69)])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16, 17, 32])
def test_gemv_shapes(N, K, M):
    W, X = synth.gemv_small(100 + M, N=N, K=K, M=M)
    y = host(q.q4k_gemv(dev(W), dev(X), N, K))
    Y, S = O.matmul_ref(W, X)
    _assert_tol(y, Y, S, f"N={N} K={K} M={M}")


@pytest.fixture(scope="module")
def decode_inputs():
    inp = synth.dense_decode(1)
    d = {k: dev(v) for k, v in inp.items()}
    return inp, d


def _full_ref(W, X, chunk=2048):
    """The oracle's product and scale over every output, computed in row chunks."""
    Y = np.empty((X.shape[0], W.shape[0]))
    S = np.empty_like(Y)
    for r0 in range(0, W.shape[0], chunk):
        Y[:, r0:r0 + chunk], S[:, r0:r0 + chunk] = O.matmul_ref(W[r0:r0 + chunk], X)
    return Y, S


@pytest.fixture(scope="module")
def decode_refs(decode_inputs):
    """Full fp64 references of both decode projections for all 32 tokens (the token
    counts below use the first M rows of the same draw)."""
    inp, _ = decode_inputs
    return {proj: _full_ref(inp[f"W_{proj}"], inp[f"X_{proj}"]) for proj in ("gate_up", "down")}


@pytest.mark.parametrize("proj", ["gate_up", "down"])
@pytest.mark.parametrize("M", [1, 4, 8, 16, 32])
def test_gemv_dense_decode_full(decode_inputs, decode_refs, proj, M):
    """Every output of the decode projections (34816 x 5120 and 5120 x 17408) against the oracle."""
    inp, d = decode_inputs
    W = inp[f"W_{proj}"]
    N, K = W.shape[0], W.shape[1] * 256
    y = host(q.q4k_gemv(d[f"W_{proj}"], d[f"X_{proj}"][:M], N, K))
    Y, S = decode_refs[proj]
    _assert_tol(y, Y[:M], S[:M], f"{proj} M={M}")


def test_gemv_batch_invariance_and_determinism(decode_inputs):
    """Within a token class (1..8 tokens: the super-block-stationary kernel; 9..16: the
    ring kernel's subnormal-nibble operand; 17..32: its fp16 sc*q operand), row m of an
    M-token call is bit-identical to the same token in any other call of that class;
    repeated calls are bit-identical."""
    inp, d = decode_inputs
    for proj in ("down", "gate_up"):
        N, K = inp[f"W_{proj}"].shape[0], inp[f"W_{proj}"].shape[1] * 256
        W, X = d[f"W_{proj}"], d[f"X_{proj}"]
        y8 = q.q4k_gemv(W, X[:8], N, K)
        assert torch.equal(y8, q.q4k_gemv(W, X[:8], N, K))
        for M in (1, 4, 5):
            assert torch.equal(q.q4k_gemv(W, X[:M], N, K), y8[:M]), (proj, M)
        for m in (0, 3, 7):
            assert torch.equal(q.q4k_gemv(W, X[m:m + 1], N, K)[0], y8[m]), (proj, m)
        assert torch.equal(q.q4k_gemv(W, X[2:6], N, K), y8[2:6]), proj
    N, K = inp["W_down"].shape[0], inp["W_down"].shape[1] * 256
    W, X = d["W_down"], d["X_down"]
    y16 = q.q4k_gemv(W, X[:16], N, K)
    assert torch.equal(y16, q.q4k_gemv(W, X[:16], N, K))
    assert torch.equal(q.q4k_gemv(W, X[:9], N, K), y16[:9])
    assert torch.equal(q.q4k_gemv(W, X[5:16], N, K), y16[5:16])
    y32 = q.q4k_gemv(W, X[:32], N, K)
    assert torch.equal(y32, q.q4k_gemv(W, X[:32], N, K))
    assert torch.equal(q.q4k_gemv(W, X[:17], N, K), y32[:17])
    assert torch.equal(q.q4k_gemv(W, X[13:30], N, K), y32[13:30])


# ---------------------------------------------------------------- Q5_K GEMV --

@pytest.mark.parametrize("N,K", [(16, 256), (48, 512), (272, 4096), (1040, 256 * 69)])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16, 17, 32])
def test_q5k_gemv_shapes(N, K, M):
    W, X = synth.gemv_small_q5(400 + M, N=N, K=K, M=M)
    y = host(q.q5k_gemv(dev(W), dev(X), N, K))
    Y, S = O.matmul_ref_q5(W, X)
    _assert_tol(y, Y, S, f"Q5_K N={N} K={K} M={M}")


def test_q5k_gemv_without_fifth_bits_equals_q4k():
    """A Q5_K matrix whose fifth bits are all zero holds the same weights as the
    Q4_K matrix with the same header and nibbles; both GEMVs take the same
    arithmetic in the same order, so the results are bit-identical."""
    W4, X = synth.gemv_small(410, N=272, K=4096, M=32)
    W5 = np.zeros(W4.shape[:-1] + (176,), np.uint8)
    W5[..., 0:16] = W4[..., 0:16]
    W5[..., 48:176] = W4[..., 16:144]
    W4d, W5d, Xd = dev(W4), dev(W5), dev(X)
    for M in (9, 17, 32):  # token counts where q4k_gemv runs the same ring kernel as q5k_gemv
        assert torch.equal(q.q5k_gemv(W5d, Xd[:M], 272, 4096), q.q4k_gemv(W4d, Xd[:M], 272, 4096)), M


@pytest.fixture(scope="module")
def decode_inputs_q5():
    inp = synth.dense_decode_q5(5)
    d = {k: dev(v) for k, v in inp.items()}
    return inp, d


@pytest.mark.parametrize("proj", ["gate_up", "down"])
@pytest.mark.parametrize("M", [1, 8, 16, 32])
def test_q5k_gemv_dense_decode_sampled(decode_inputs_q5, proj, M):
    inp, d = decode_inputs_q5
    W, X = inp[f"W_{proj}"], inp[f"X_{proj}"][:M]
    N, K = W.shape[0], W.shape[1] * 256
    y = host(q.q5k_gemv(d[f"W_{proj}"], d[f"X_{proj}"][:M], N, K))
    rows = sample_rows(N, 384, seed=50 + M)
    Y, S = O.matmul_rows_ref_q5(W, X, rows)
    _assert_tol(y[:, rows], Y, S, f"Q5_K {proj} M={M}")


# ---------------------------------------------------------------- Q6_K GEMV --

@pytest.mark.parametrize("N,K", [(16, 256), (48, 512), (272, 4096), (1040, 256 * 69)])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16, 17, 32])
def test_q6k_gemv_shapes(N, K, M):
    W, X = synth.gemv_small_q6(800 + M, N=N, K=K, M=M)
    y = host(q.q6k_gemv(dev(W), dev(X), N, K))
    Y, S = O.matmul_ref_q6(W, X)
    _assert_tol(y, Y, S, f"Q6_K N={N} K={K} M={M}")


def test_q6k_gemv_odd_block_count_rows():
    """K = 256 * 69 (odd super-block count): every other row starts 2 bytes off a word."""
    W, X = synth.gemv_small_q6(820, N=64, K=256 * 69, M=5)
    y = host(q.q6k_gemv(dev(W), dev(X), 64, 256 * 69))
    Y, S = O.matmul_ref_q6(W, X)
    _assert_tol(y, Y, S, "Q6_K odd block count")


@pytest.mark.parametrize("M", [3, 9])  # the stationary form (1..8 tokens) and the 9..16 class
def test_q6k_gemv_edge_blocks(M):
    """Extreme Q6_K blocks: d = +-65504, subnormal d, zero; scales -128, 127, 0; q = -32, 31, 0."""
    rng = np.random.default_rng(830)
    N, K = 272, 256 * 5
    pool = np.stack([O.make_block_q6(d, sc, qv) for d in (65504.0, -65504.0, 6e-8, 0.0, -1.5)
                     for sc in ([-128] * 16, [127] * 16, [0] * 16, list(range(-8, 8)))
                     for qv in ([-32] * 256, [31] * 256, [0] * 256, list(rng.integers(-32, 32, 256)))])
    W = synth.q6k_random_blocks(rng, N, K)
    pick = rng.random(W.shape[:2]) < 0.5
    W[pick] = pool[rng.integers(0, len(pool), W.shape[:2])[pick]]
    X = synth.bf16_normal(rng, (M, K))
    Y, S = O.matmul_ref_q6(W, X)
    _assert_tol(host(q.q6k_gemv(dev(W), dev(X), N, K)), Y, S, "Q6_K edge blocks")


@pytest.fixture(scope="module")
def decode_inputs_q6():
    inp = synth.dense_decode_q6(7)
    d = {k: dev(v) for k, v in inp.items()}
    return inp, d


@pytest.mark.parametrize("proj", ["gate_up", "down"])
@pytest.mark.parametrize("M", [1, 4, 8, 16, 32])
def test_q6k_gemv_dense_decode_full(decode_inputs_q6, proj, M):
    """Every output of the decode projections in Q6_K against the oracle, in row chunks."""
    inp, d = decode_inputs_q6
    W, X = inp[f"W_{proj}"], inp[f"X_{proj}"][:M]
    N, K = W.shape[0], W.shape[1] * 256
    y = host(q.q6k_gemv(d[f"W_{proj}"], d[f"X_{proj}"][:M], N, K))
    for r0 in range(0, N, 4096):
        Y, S = O.matmul_ref_q6(W[r0:r0 + 4096], X)
        _assert_tol(y[:, r0:r0 + 4096], Y, S, f"Q6_K {proj} M={M} rows {r0}..")


def test_q6k_gemv_batch_invariance():
    """Within a token class a token's result does not depend on the rest of the batch."""
    W, X = synth.gemv_small_q6(840, N=1040, K=256 * 69, M=32)
    Wd, Xd = dev(W), dev(X)
    y8 = q.q6k_gemv(Wd, Xd[:8], 1040, 256 * 69)
    assert torch.equal(q.q6k_gemv(Wd, Xd[3:4], 1040, 256 * 69)[0], y8[3])
    y32 = q.q6k_gemv(Wd, Xd, 1040, 256 * 69)
    assert torch.equal(q.q6k_gemv(Wd, Xd[5:27], 1040, 256 * 69), y32[5:27])


# ------------------------------------------------------------------ Q8 lane --

def _q8lane_check(W, X, y, what):
    """Tight parity with the lane's own product (int32-exact super-block sums, fp32 for
    the rest: 3e-5 of its absolute scale), and the accuracy bound against the exact one."""
    Yl, Sl = O.matmul_ref_q8lane(W, X)
    err = np.abs(y.astype(np.float64) - Yl)
    assert np.all(err <= 3e-5 * Sl + 1e-30), f"{what}: lane parity, worst {float((err / np.maximum(Sl, 1e-300)).max()):.2e}"
    Ye, _ = O.matmul_ref(W, X)
    q, d_x = O.quantize_x_q8(X)
    xq = q * np.repeat(d_x.astype(np.float64), 256, axis=1)
    bound = (np.abs(O.bf16_to_f64(X) - xq) @ np.abs(O.dequant_exact(W)).T)
    assert np.all(np.abs(y - Ye) <= bound + 3e-5 * Sl + 1e-30), f"{what}: accuracy bound"


@pytest.mark.parametrize("N,K", [(16, 256), (48, 512), (272, 4096), (1040, 256 * 69)])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16, 17, 32])
def test_q8lane_gemv_shapes(N, K, M):
    W, X = synth.gemv_small(600 + M, N=N, K=K, M=M)
    y = host(q.q4k_gemv_q8(dev(W), dev(X), N, K))
    _q8lane_check(W, X, y, f"Q8 lane N={N} K={K} M={M}")


@pytest.mark.parametrize("proj", ["gate_up", "down"])
@pytest.mark.parametrize("M", [1, 32])
def test_q8lane_gemv_dense_decode_sampled(decode_inputs, proj, M):
    inp, d = decode_inputs
    W, X = inp[f"W_{proj}"], inp[f"X_{proj}"][:M]
    N, K = W.shape[0], W.shape[1] * 256
    y = host(q.q4k_gemv_q8(d[f"W_{proj}"], d[f"X_{proj}"][:M], N, K))
    rows = sample_rows(N, 256, seed=70 + M)
    _q8lane_check(W[rows], X, y[:, rows], f"Q8 lane {proj} M={M}")


def test_q8lane_batch_invariance():
    """Integer super-block sums and the same fp32 epilogue per token at every token
    count: row m of any call equals that token's row of a 32-token call."""
    W, X = synth.gemv_small(620, N=1040, K=256 * 69, M=32)
    Wd, Xd = dev(W), dev(X)
    y32 = q.q4k_gemv_q8(Wd, Xd, 1040, 256 * 69)
    for lo, hi in ((0, 1), (0, 8), (3, 12), (0, 16), (5, 22)):
        assert torch.equal(q.q4k_gemv_q8(Wd, Xd[lo:hi], 1040, 256 * 69), y32[lo:hi]), (lo, hi)


# ---------------------------------------------------------------- Q8_0 GEMV --

@pytest.mark.parametrize("N,K", [(16, 256), (48, 512), (272, 4096), (1040, 256 * 69)])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16, 17, 32])
def test_q80_gemv_shapes(N, K, M):
    W, X = synth.gemv_small_q80(500 + M, N=N, K=K, M=M)
    y = host(q.q80_gemv(dev(W), dev(X), N, K))
    Y, S = O.matmul_ref_q80(W, X)
    _assert_tol(y, Y, S, f"Q8_0 N={N} K={K} M={M}")


@pytest.fixture(scope="module")
def decode_inputs_q80():
    inp = synth.dense_decode_q80(6)
    d = {k: dev(v) for k, v in inp.items()}
    return inp, d


@pytest.mark.parametrize("proj", ["gate_up", "down"])
@pytest.mark.parametrize("M", [1, 8, 16, 32])
def test_q80_gemv_dense_decode_sampled(decode_inputs_q80, proj, M):
    inp, d = decode_inputs_q80
    W, X = inp[f"W_{proj}"], inp[f"X_{proj}"][:M]
    N, K = W.shape[0], W.shape[1] * 32
    y = host(q.q80_gemv(d[f"W_{proj}"], d[f"X_{proj}"][:M], N, K))
    rows = sample_rows(N, 384, seed=60 + M)
    Y, S = O.matmul_rows_ref_q80(W, X, rows)
    _assert_tol(y[:, rows], Y, S, f"Q8_0 {proj} M={M}")


def test_q80_gemv_batch_invariance():
    """Q8_0 takes the same per-token arithmetic at every token count: row m of any
    call equals that token's row in a 32-token call; repeated calls are identical."""
    W, X = synth.gemv_small_q80(520, N=1040, K=256 * 69, M=32)
    Wd, Xd = dev(W), dev(X)
    y32 = q.q80_gemv(Wd, Xd, 1040, 256 * 69)
    assert torch.equal(y32, q.q80_gemv(Wd, Xd, 1040, 256 * 69))
    for lo, hi in ((0, 1), (0, 8), (3, 12), (0, 16), (5, 22), (0, 17)):
        assert torch.equal(q.q80_gemv(Wd, Xd[lo:hi], 1040, 256 * 69), y32[lo:hi]), (lo, hi)


# ------------------------------------------------------------ decode repack --

@pytest.mark.parametrize("N,K", [(16, 256), (200, 512), (1040, 256 * 69)])
def test_repack_matches_reference(N, K):
    W, _ = synth.gemv_small(300, N=N, K=K, M=1)
    Wr = host(q.q4k_repack(dev(W), N, K))
    assert np.array_equal(Wr, O.repack_ref(W))


@pytest.mark.parametrize("N,K", [(16, 256), (272, 4096), (1040, 256 * 69)])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16, 17, 32])
def test_gemv_repacked_equals_raw_and_oracle(N, K, M):
    """Within tolerance; from 9 tokens on q4k_gemv runs the ring kernel the repacked
    GEMV shares, with the same arithmetic in the same order: bit-identical there."""
    W, X = synth.gemv_small(310 + M, N=N, K=K, M=M)
    Wd, Xd = dev(W), dev(X)
    y_raw = q.q4k_gemv(Wd, Xd, N, K)
    y_rep = q.q4k_gemv_repacked(q.q4k_repack(Wd, N, K), Xd, N, K)
    if M > 8:
        assert torch.equal(y_rep, y_raw)
    Y, S = O.matmul_ref(W, X)
    _assert_tol(host(y_rep), Y, S, f"repacked N={N} K={K} M={M}")


@pytest.mark.parametrize("proj", ["gate_up", "down"])
@pytest.mark.parametrize("M", [1, 8, 32])
def test_gemv_repacked_dense_decode(decode_inputs, decode_refs, proj, M):
    inp, d = decode_inputs
    W = inp[f"W_{proj}"]
    N, K = W.shape[0], W.shape[1] * 256
    Wr = q.q4k_repack(d[f"W_{proj}"], N, K)
    X = d[f"X_{proj}"][:M]
    y = q.q4k_gemv_repacked(Wr, X, N, K)
    Y, S = decode_refs[proj]
    _assert_tol(host(y), Y[:M], S[:M], f"repacked {proj} M={M}")
    if M > 8:
        assert torch.equal(y, q.q4k_gemv(d[f"W_{proj}"], X, N, K))


# ---------------------------------------------------------------- MoE route --

def _route_and_check(logits, topk=8):
    E = logits.shape[1]
    r = q.moe_route_permute(dev(logits), topk)
    ids, w = O.route_topk(logits, topk)
    offs, perm, inv, rt = O.permute(ids, E)
    assert np.array_equal(host(r["topk_ids"]), ids)
    assert np.abs(host(r["topk_w"]).astype(np.float64) - w).max() <= 1e-6
    assert np.array_equal(host(r["expert_offsets"]), offs)
    assert np.array_equal(host(r["perm"]), perm)
    assert np.array_equal(host(r["inv_perm"]), inv)
    assert np.array_equal(host(r["row_token"]), rt)
    return r


@pytest.mark.parametrize("M", [1, 8, 32, 33, 100])
def test_route_permute_decode(M):
    _route_and_check(synth.moe_layer(3, M, E=128, H=256, F=256)["logits"])


def test_route_permute_prefill_skewed():
    inp = synth.moe_layer(4, 4096, E=128, H=256, F=256, hot=16)
    _route_and_check(inp["logits"])


def test_route_ties_and_small_E():
    rng = np.random.default_rng(9)
    L = (rng.standard_normal((70, 128)) * 2).astype(np.float32)
    L[0] = 0.25
    L[1, [5, 77, 99]] = 7.0
    L[2, ::2] = L[2, 1::2]
    _route_and_check(L)
    _route_and_check((rng.standard_normal((50, 40))).astype(np.float32), topk=3)
    _route_and_check((rng.standard_normal((9, 1000))).astype(np.float32), topk=16)


def test_route_zero_tokens():
    offs = torch.full((129,), -1, dtype=torch.int32, device="cuda")
    st = q.lib().moe_route_permute(None, 0, 128, 8, None, None, offs.data_ptr(), None, None, None,
                                   None, 0, None)
    assert st == 0 and torch.count_nonzero(offs).item() == 0


@pytest.mark.parametrize("M", [1, 8, 32, 300])
def test_route_from_hidden(M):
    """Router logits within the fp32 summation bound of the oracle ((H-1) * 2^-24 * sum|x*w|);
    then routing and permutation bit-exact against the oracle run on those logits."""
    E, H, topk = 128, 2048, 8
    X = synth.bf16_normal(np.random.default_rng(700 + M), (M, H))
    Wr = synth.router_weights(22, E, H)
    r = q.moe_route_permute_hidden(dev(X), dev(Wr), topk)
    L, S = O.router_logits_ref(X, Wr)
    lg = host(r["logits"]).astype(np.float64)
    assert np.all(np.abs(lg - L) <= (H - 1) * 2.0 ** -24 * S)
    ids, w = O.route_topk(host(r["logits"]), topk)
    assert np.array_equal(host(r["topk_ids"]), ids)
    assert np.abs(host(r["topk_w"]).astype(np.float64) - w).max() <= 1e-6
    offs, perm, inv, rt = O.permute(ids, E)
    for name, ref in (("expert_offsets", offs), ("perm", perm), ("inv_perm", inv), ("row_token", rt)):
        assert np.array_equal(host(r[name]), ref), name


# -------------------------------------------------------------- MoE combine --

def test_combine():
    rng = np.random.default_rng(4)
    M, topk, H = 37, 8, 2048
    Od = rng.standard_normal((M * topk, H)).astype(np.float32)
    inv = rng.permutation(M * topk).astype(np.int32)
    w = rng.random((M, topk)).astype(np.float32)
    y = host(q.moe_combine(dev(Od), dev(inv), dev(w), M, topk, H))
    Y, S = O.combine_ref(Od, inv, w)
    assert np.all(np.abs(y - Y) <= 1e-6 * S + 1e-30)


def test_combine_residual():
    """Within tolerance of the oracle; bit-identical to the plain combine followed
    by an fp32 add of the residual; in place (Y = residual) gives the same."""
    rng = np.random.default_rng(6)
    M, topk, H = 37, 8, 2048
    Od = rng.standard_normal((M * topk, H)).astype(np.float32)
    inv = rng.permutation(M * topk).astype(np.int32)
    w = rng.random((M, topk)).astype(np.float32)
    R = rng.standard_normal((M, H)).astype(np.float32)
    Odd, invd, wd, Rd = dev(Od), dev(inv), dev(w), dev(R)
    y = q.moe_combine_residual(Odd, invd, wd, Rd, M, topk, H)
    Y, S = O.combine_residual_ref(Od, inv, w, R)
    assert np.all(np.abs(host(y) - Y) <= 1e-6 * S + 1e-30)
    assert torch.equal(y, Rd + q.moe_combine(Odd, invd, wd, M, topk, H))
    Ri = Rd.clone()
    q.moe_combine_residual(Odd, invd, wd, Ri, M, topk, H, Y=Ri)
    assert torch.equal(Ri, y)


def test_combine_bad_index_latches_status():
    M, topk, H = 2, 2, 8
    Od = torch.zeros(M * topk, H, device="cuda")
    inv = torch.tensor([0, 1, 2, 99], dtype=torch.int32, device="cuda")
    w = torch.ones(M, topk, device="cuda")
    q.moe_combine(Od, inv, w, M, topk, H)
    assert q.q4k_last_device_status() == 8  # Q4K_ERR_DEVICE_BOUNDS
    assert q.q4k_last_device_status() == 0


# ------------------------------------------------------- MoE expert matmuls --

def _moe_stagewise(inp, M, hint=None):
    """Run route -> gate_up (fp32 and SwiGLU) -> down -> combine; check every stage."""
    E, H, F, topk = inp["E"], inp["H"], inp["F"], 8
    r = _route_and_check(inp["logits"], topk)
    rows = M * topk
    hint = M if hint is None else hint
    Wgu, Wdn, X = dev(inp["W_gate_up"]), dev(inp["W_down"]), dev(inp["X"])
    offs_h = host(r["expert_offsets"])
    rt_h = host(r["row_token"])
    sample = sample_rows(rows, 384, seed=M) if rows > 512 else np.arange(rows)

    GU = q.moe_q4k_grouped(Wgu, E, 2 * F, H, X, r["expert_offsets"], rows, hint, q.ACT_NONE,
                           row_gather=r["row_token"])
    Yg, Sg = O.grouped_ref(inp["W_gate_up"], inp["X"], offs_h, row_gather=rt_h, rows=sample)
    ratio_gu = _assert_tol(host(GU)[sample], Yg, Sg, "gate_up")

    h = q.moe_q4k_grouped(Wgu, E, 2 * F, H, X, r["expert_offsets"], rows, hint, q.ACT_SWIGLU,
                          row_gather=r["row_token"])
    h_ref = O.swiglu_bf16_ref(host(GU)[sample], F)
    diff = np.abs(O.bf16_to_f64(host(h)[sample]) - O.bf16_to_f64(h_ref))
    ulps = diff / bf16_ulp(h_ref)
    assert np.all(ulps <= 1.0), f"SwiGLU: {int((ulps > 1).sum())} values beyond one bf16 ulp (max {ulps.max():.1f})"

    Od = q.moe_q4k_grouped(Wdn, E, H, F, h, r["expert_offsets"], rows, hint, q.ACT_NONE)
    Yd, Sd = O.grouped_ref(inp["W_down"], host(h), offs_h, rows=sample)
    ratio_dn = _assert_tol(host(Od)[sample], Yd, Sd, "down")

    y = host(q.moe_combine(Od, r["inv_perm"], r["topk_w"], M, topk, H))
    tok = np.arange(M) if M <= 64 else sample_rows(M, 64, seed=1)
    Yc, Sc = O.combine_ref(host(Od), host(r["inv_perm"]), host(r["topk_w"]))
    assert np.all(np.abs(y[tok] - Yc[tok]) <= 1e-6 * Sc[tok] + 1e-30)
    return ratio_gu, ratio_dn


@pytest.mark.parametrize("M", [1, 8, 32])
def test_moe_decode_layer(M):
    _moe_stagewise(synth.moe_decode(3, M), M)


def test_moe_decode_small_experts_tc_path():
    """The tensor-core grouped path on a small ragged problem (hint forces it)."""
    inp = synth.moe_layer(13, 40, E=16, H=512, F=256)
    _moe_stagewise(inp, 40, hint=40)


def test_moe_prefill_layer():
    _moe_stagewise(synth.moe_prefill(4), 4096)


# -------------------------------------------------------------------- GEMM --

@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (100, 512, 512), (256, 256, 1024),
                                   (300, 768, 2048), (513, 1024, 5120)])
def test_gemm_small(M, N, K):
    W, X = synth.gemv_small(200 + M, N=N, K=K, M=M)
    y = host(q.q4k_gemm(dev(W), dev(X), N, K))
    Y, S = O.matmul_ref(W, X)
    _assert_tol(y, Y, S, f"gemm M={M} N={N} K={K}")


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (300, 768, 2048), (513, 1024, 5120)])
def test_gemm_fused_equals_unfused_chain(M, N, K):
    """q4k_gemm (dequantise into shared memory, then tcgen05) is bit-identical to the
    unfused chain q4k_dequant(bf16) -> bf16w_gemm over the same tiles and MMA order
    (hipEngine 0.3.0 README, "Core principles": fused composites have numerically
    equivalent unfused chains)."""
    W, X = synth.gemv_small(230 + M, N=N, K=K, M=M)
    Wd, Xd = dev(W), dev(X)
    fused = q.q4k_gemm(Wd, Xd, N, K)
    Wb = q.q4k_dequant(Wd.reshape(-1), out_bf16=True).view(N, K)
    unfused = q.bf16w_gemm(Wb, Xd, N, K)
    assert torch.equal(fused, unfused)


@pytest.fixture(scope="module")
def prefill_inputs():
    W, X = synth.dense_prefill(2)
    return W, X, dev(W), dev(X)


def test_gemm_dense_prefill_full_512(prefill_inputs):
    """Every output of the 512-token prefill GEMM (512 x 17408) against the oracle."""
    W, X, Wd, Xd = prefill_inputs
    N, K = W.shape[0], W.shape[1] * 256
    y = q.q4k_gemm(Wd, Xd[:512], N, K)
    Y, S = _full_ref(W, X[:512])
    _assert_tol(host(y), Y, S, "prefill M=512")
    assert torch.equal(y, q.q4k_gemm(Wd, Xd[:512], N, K))  # deterministic


def test_gemm_dense_prefill_sampled_4096(prefill_inputs):
    """4096 tokens: every weight row for 64 sampled tokens (all N outputs of each)."""
    W, X, Wd, Xd = prefill_inputs
    N, K = W.shape[0], W.shape[1] * 256
    M = 4096
    y = q.q4k_gemm(Wd, Xd[:M], N, K)
    toks = sample_rows(M, 64, seed=M + 1)
    yh = host(y[torch.from_numpy(toks).cuda()])
    Y, S = _full_ref(W, X[toks])
    _assert_tol(yh, Y, S, f"prefill M={M}")
    assert torch.equal(y, q.q4k_gemm(Wd, Xd[:M], N, K))  # deterministic
