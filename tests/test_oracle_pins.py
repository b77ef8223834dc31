"""Pins for the CPU oracle: checks against facts fixed outside the oracle itself.

Each test pins one part of the oracle to a hand-derived value, an exhaustive
brute force, a closed form or an invariant, chosen so that a plausible slip
(a swapped nibble, a wrong bit of the six-bit packing, a dropped min term, a
transposed operand, a wrong tie-break) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

from oracle import q4k as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "q4k_block_handmade.txt")


def _read_golden():
    header, pairs, ws = None, {}, {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "header":
                header = bytes(int(t, 16) for t in tok[1:])
            elif tok[0] == "pair":
                pairs[int(tok[1])] = (int(tok[2]), int(tok[3]))
            elif tok[0] == "w":
                ws[int(tok[1])] = float(tok[2])
    block = np.zeros(144, np.uint8)
    block[:16] = np.frombuffer(header, np.uint8)
    block[16:] = np.arange(128, dtype=np.uint8)
    return block, pairs, ws


def _golden_ok(mod):
    block, pairs, ws = _read_golden()
    sc, m = mod.scale_min_pairs(block)
    if any((int(sc[j]), int(m[j])) != pairs[j] for j in range(8)):
        return False
    w = mod.dequant_exact(block[None, :])
    return all(w[i] == v for i, v in ws.items())


def test_golden_handmade_block():
    """Hand-packed block (tests/golden/q4k_block_handmade.txt) decodes to the hand-worked weights."""
    assert _golden_ok(O)


def test_scale_bits_each_owned_once():
    """Every one of the 96 bits of the scale field moves exactly one six-bit value by 2^b,
    and every (value, bit) pair is hit exactly once: the packing is a bijection."""
    base = np.zeros(144, np.uint8)
    sc0, m0 = O.scale_min_pairs(base)
    seen = set()
    for byte in range(12):
        for bit in range(8):
            b = base.copy()
            b[4 + byte] ^= np.uint8(1 << bit)
            sc, m = O.scale_min_pairs(b)
            diff = np.concatenate([sc - sc0, m - m0])
            nz = np.nonzero(diff)[0]
            assert nz.size == 1
            v = int(diff[nz[0]])
            assert v > 0 and (v & (v - 1)) == 0 and v < 64
            key = (int(nz[0]), v.bit_length() - 1)
            assert key not in seen
            seen.add(key)
    assert len(seen) == 96


def test_scale_pack_unpack_exhaustive():
    """All 8 x 64 x 64 (j, sc, m) values round-trip through the packer/unpacker,
    with the other seven pairs random."""
    rng = np.random.default_rng(123)
    for j in range(8):
        scv, mv = np.meshgrid(np.arange(64), np.arange(64), indexing="ij")
        n = scv.size
        sc = rng.integers(0, 64, (n, 8))
        m = rng.integers(0, 64, (n, 8))
        sc[:, j] = scv.ravel()
        m[:, j] = mv.ravel()
        blocks = np.zeros((n, 144), np.uint8)
        blocks[:, 4:16] = O.pack_scale_min(sc, m)
        sc2, m2 = O.scale_min_pairs(blocks)
        assert np.array_equal(sc2, sc) and np.array_equal(m2, m)


def test_one_hot_nibble_positions():
    """Setting only nibble h of quant byte 32c+l changes only weight 64c+32h+l, by d*sc_j*v."""
    sc = np.arange(1, 9)
    base = O.make_block(1.0, 0.0, sc, np.zeros(8, int), np.zeros(256, int))
    w0 = O.dequant_exact(base[None])
    assert np.all(w0 == 0)
    for c in range(4):
        for h in range(2):
            for l in range(32):
                for v in (1, 9, 15):
                    b = base.copy()
                    b[16 + 32 * c + l] = np.uint8(v << (4 * h))
                    w = O.dequant_exact(b[None])
                    i = 64 * c + 32 * h + l
                    expect = np.zeros(256)
                    expect[i] = 1.0 * sc[i // 32] * v
                    assert np.array_equal(w, expect), (c, h, l, v)


def test_closed_form_constant_block():
    """Constant q=c, sc=s, m=t in every position: w = d*s*c - dmin*t everywhere,
    and y = w * sum(x) exactly."""
    rng = np.random.default_rng(7)
    for (d, dmin, s, c, t) in [(1e-3, 2e-3, 17, 5, 40), (0.25, 0.125, 63, 15, 63), (3e-4, 0.0, 1, 1, 0)]:
        blk = O.make_block(d, dmin, [s] * 8, [t] * 8, [c] * 256)
        dh, dmh = float(np.float16(d)), float(np.float16(dmin))
        w = O.dequant_exact(np.stack([blk, blk])[None])  # one row, two blocks
        assert np.all(w == dh * s * c - dmh * t)
        X = synth.bf16_normal(rng, (3, 512))
        Y, S = O.matmul_ref(np.stack([blk, blk])[None], X)
        xs = O.bf16_to_f64(X).sum(axis=1)
        np.testing.assert_allclose(Y[:, 0], (dh * s * c - dmh * t) * xs, rtol=1e-13, atol=1e-15)


def test_quantize_dequantize_round_trip():
    """Weights built from known (d, dmin, sc, m, q) are found again by a brute-force
    quantizer, and its packed block dequantises to the same weights bit for bit."""
    rng = np.random.default_rng(11)
    for _ in range(3):
        d = float(np.float16(abs(rng.standard_normal()) * 1e-3))
        dmin = float(np.float16(abs(rng.standard_normal()) * 1e-3))
        sc = rng.integers(0, 64, 8)
        m = rng.integers(0, 64, 8)
        q = rng.integers(0, 16, 256)
        j = np.arange(256) // 32
        w = d * sc[j] * q - dmin * m[j]          # representable by construction
        sc2, m2, q2 = O.quantize_brute_force(w, d, dmin)
        blk = O.make_block(d, dmin, sc2, m2, q2)
        assert np.array_equal(O.dequant_exact(blk[None]), w)


def test_dequant_f32_bf16_single_rounding():
    """fp32 dequant is the exact value rounded once; bf16 is RN of that fp32 value."""
    W, _ = synth.gemv_small(0, N=8, K=512)
    ex = O.dequant_exact(W)
    f = O.dequant_f32(W)
    assert np.all(np.abs(f.astype(np.float64) - ex) <= np.abs(ex) * 2.0 ** -24)
    bf = O.bf16_to_f64(O.dequant_bf16_bits(W))
    assert np.all(np.abs(bf - f.astype(np.float64)) <= np.abs(f.astype(np.float64)) * 2.0 ** -8)


def _scalar_weight(block, i):
    """Scalar restatement used only as brute force for the matmul pins."""
    d = float(np.frombuffer(bytes(block[0:2]), "<f2")[0])
    dmin = float(np.frombuffer(bytes(block[2:4]), "<f2")[0])
    s = [int(v) for v in block[4:16]]
    j = i // 32
    if j < 4:
        sc, m = s[j] & 63, s[j + 4] & 63
    else:
        sc = (s[j + 4] & 0xF) | ((s[j - 4] >> 6) << 4)
        m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4)
    c, rem = divmod(i, 64)
    h, l = divmod(rem, 32)
    q = (int(block[16 + 32 * c + l]) >> (4 * h)) & 0xF
    return d * sc * q - dmin * m


def test_matmul_brute_force_tiny():
    """Two rows x one block x two tokens, every product enumerated, exact fsum."""
    W, X = synth.gemv_small(5, N=2, K=256, M=2)
    Y, S = O.matmul_ref(W, X)
    xf = O.bf16_to_f64(X)
    for n in range(2):
        for mtok in range(2):
            prods = [_scalar_weight(W[n, 0], i) * xf[mtok, i] for i in range(256)]
            assert abs(Y[mtok, n] - math.fsum(prods)) <= 1e-12 * math.fsum(abs(p) for p in prods)
            assert abs(S[mtok, n] - math.fsum(abs(p) for p in prods)) <= 1e-12 * S[mtok, n]


def test_matmul_orientation_and_linearity():
    """Y[m, n] pairs token m with weight row n (not transposed), and Y is linear in X."""
    W, X = synth.gemv_small(9, N=4, K=512, M=3)
    Wd = O.dequant_exact(W)
    xf = O.bf16_to_f64(X)
    Y, _ = O.matmul_ref(W, X)
    assert Y.shape == (3, 4)
    for mtok in range(3):
        for n in range(4):
            assert abs(Y[mtok, n] - math.fsum(Wd[n] * xf[mtok])) < 1e-12 * np.abs(Wd[n] * xf[mtok]).sum()
    # linearity: X = X1 + X2 exactly representable (bf16 * 2 stays bf16)
    X2 = synth.f32_to_bf16_bits(2.0 * O.bf16_to_f64(X).astype(np.float32))
    Y2, _ = O.matmul_ref(W, X2)
    np.testing.assert_allclose(Y2, 2 * Y, rtol=1e-13, atol=1e-14)


def test_batch_rows_independent():
    """Row m of an M-token product equals the one-token product of row m."""
    W, X = synth.gemv_small(3, N=16, K=512, M=5)
    Y, _ = O.matmul_ref(W, X)
    for mtok in range(5):
        y1, _ = O.matmul_ref(W, X[mtok:mtok + 1])
        np.testing.assert_allclose(Y[mtok], y1[0], rtol=1e-14, atol=1e-15)


def test_routing_brute_force_and_ties():
    rng = np.random.default_rng(21)
    L = (rng.standard_normal((40, 128)) * 2).astype(np.float32)
    L[0, :] = 0.5                      # all equal -> experts 0..7
    L[1, [3, 70, 90, 100]] = 9.0       # tie among the top
    L[2, ::2] = L[2, 1::2]             # pairwise duplicates
    ids, w = O.route_topk(L, 8)
    for t in range(L.shape[0]):
        ranked = sorted(range(128), key=lambda e: (-float(L[t, e]), e))[:8]
        assert list(ids[t]) == ranked
        full = np.exp(L[t].astype(np.float64) - L[t].max())
        full /= full.sum()
        ren = full[ranked] / full[ranked].sum()
        np.testing.assert_allclose(w[t], ren, rtol=1e-12)
        assert abs(w[t].sum() - 1.0) < 1e-12
    assert list(ids[0]) == list(range(8))
    assert list(ids[1][:4]) == [3, 70, 90, 100]


def test_permutation_invariants():
    rng = np.random.default_rng(5)
    L = (rng.standard_normal((64, 128)) * 2).astype(np.float32)
    ids, _ = O.route_topk(L, 8)
    offs, perm, inv, row_tok = O.permute(ids, 128)
    flat = ids.reshape(-1)
    assert sorted(perm.tolist()) == list(range(flat.size))
    exp_of_row = flat[perm]
    assert np.all(np.diff(exp_of_row) >= 0)
    for e in range(128):
        seg = perm[offs[e]:offs[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)
    assert np.array_equal(np.diff(offs), np.bincount(flat, minlength=128))
    assert np.array_equal(inv[perm], np.arange(flat.size))
    assert np.array_equal(row_tok, perm // 8)


def _small_moe(seed, M=6, E=4, H=256, F=256, topk=2):
    return synth.moe_layer(seed, M, E=E, H=H, F=F), topk


def test_combine_linear_and_gather():
    rng = np.random.default_rng(2)
    M, topk, H = 5, 3, 16
    O1 = rng.standard_normal((M * topk, H))
    O2 = rng.standard_normal((M * topk, H))
    inv = rng.permutation(M * topk).astype(np.int32)
    w = rng.random((M, topk))
    y1, _ = O.combine_ref(O1, inv, w)
    y2, _ = O.combine_ref(O2, inv, w)
    y12, _ = O.combine_ref(2.0 * O1 - O2, inv, w)
    np.testing.assert_allclose(y12, 2 * y1 - y2, rtol=1e-12, atol=1e-12)
    onehot = np.zeros((M, topk))
    onehot[:, 1] = 1.0
    yg, _ = O.combine_ref(O1, inv, onehot)
    np.testing.assert_array_equal(yg, O1[inv.reshape(M, topk)[:, 1]])


def test_combine_residual_reduces_and_adds():
    """Zero weights give the residual itself; a zero residual gives the plain
    combine; the residual enters once, unscaled, whatever the weights."""
    rng = np.random.default_rng(5)
    M, topk, H = 4, 3, 8
    Od = rng.standard_normal((M * topk, H))
    inv = rng.permutation(M * topk).astype(np.int32)
    w = rng.random((M, topk))
    R = rng.standard_normal((M, H))
    y0, S0 = O.combine_residual_ref(Od, inv, np.zeros((M, topk)), R)
    np.testing.assert_array_equal(y0, R)
    np.testing.assert_array_equal(S0, np.abs(R))
    yc, _ = O.combine_ref(Od, inv, w)
    yz, _ = O.combine_residual_ref(Od, inv, w, np.zeros((M, H)))
    np.testing.assert_array_equal(yz, yc)
    # one-hot weights: residual plus the gathered row, element by element
    onehot = np.zeros((M, topk))
    onehot[:, 2] = 1.0
    yg, _ = O.combine_residual_ref(Od, inv, onehot, R)
    for t in range(M):
        for hh in range(H):
            assert yg[t, hh] == R[t, hh] + Od[inv[t * topk + 2], hh]


def test_moe_layer_token_permutation_and_expert_relabel():
    inp, topk = _small_moe(31)
    y = O.moe_layer_ref(inp["logits"], inp["X"], inp["W_gate_up"], inp["W_down"], topk)
    p = np.random.default_rng(0).permutation(inp["logits"].shape[0])
    yp = O.moe_layer_ref(inp["logits"][p], inp["X"][p], inp["W_gate_up"], inp["W_down"], topk)
    np.testing.assert_allclose(yp, y[p], rtol=1e-12, atol=1e-14)
    # relabel experts: permute the weight stacks and logit columns together
    # (ties are impossible with continuous logits, so the chosen set is unchanged)
    r = np.array([2, 0, 3, 1])
    yr = O.moe_layer_ref(inp["logits"][:, r], inp["X"], inp["W_gate_up"][r], inp["W_down"][r], topk)
    np.testing.assert_allclose(yr, y, rtol=1e-12, atol=1e-14)


def test_moe_single_expert_is_dense_swiglu_ffn():
    """E=1, top-1: the layer reduces to down(SiLU(gate x) * up x) with weight 1."""
    inp = synth.moe_layer(41, 3, E=1, H=256, F=256)
    y = O.moe_layer_ref(inp["logits"], inp["X"], inp["W_gate_up"], inp["W_down"], 1)
    G, _ = O.matmul_ref(inp["W_gate_up"][0][:256], inp["X"])
    U, _ = O.matmul_ref(inp["W_gate_up"][0][256:], inp["X"])
    h = G / (1 + np.exp(-G)) * U
    Wd = O.dequant_exact(inp["W_down"][0])
    np.testing.assert_allclose(y, h @ Wd.T, rtol=1e-12, atol=1e-12)


def test_stagewise_pipeline_matches_end_to_end():
    """Routing -> permutation -> grouped gate_up -> SwiGLU -> grouped down -> combine
    (all in fp64, no bf16 step) equals the end-to-end layer."""
    inp, topk = _small_moe(17, M=7, E=5)
    ids, w = O.route_topk(inp["logits"], topk)
    offs, perm, inv, row_tok = O.permute(ids, 5)
    GU, _ = O.grouped_ref(inp["W_gate_up"], inp["X"], offs, row_gather=row_tok)
    F = inp["F"]
    h = O.silu_mul(GU[:, :F], GU[:, F:])
    Od = np.empty((perm.size, inp["H"]))
    offs64 = offs.astype(np.int64)
    for e in range(5):
        a, b = offs64[e], offs64[e + 1]
        if b > a:
            Od[a:b] = h[a:b] @ O.dequant_exact(inp["W_down"][e]).T
    y, _ = O.combine_ref(Od, inv, w)
    y_ref = O.moe_layer_ref(inp["logits"], inp["X"], inp["W_gate_up"], inp["W_down"], topk)
    np.testing.assert_allclose(y, y_ref, rtol=1e-11, atol=1e-13)


def test_synth_fields_distribution():
    """The generator's random bytes decode to q in 0..15 and sc, m in 0..63, all values hit."""
    W, _ = synth.gemv_small(0)
    sc, m = O.scale_min_pairs(W)
    q = O.quants(W)
    assert set(np.unique(q)) == set(range(16))
    assert set(np.unique(sc)) == set(range(64)) and set(np.unique(m)) == set(range(64))


# ---- planted mistakes: each mutant of the oracle must fail a pin -----------------

class _Mutant:
    def __init__(self, **over):
        self.__dict__.update({k: getattr(O, k) for k in ("scale_min_pairs", "quants", "block_d_dmin")})
        self.__dict__.update(over)

    def dequant_exact(self, blocks):
        d, dmin = self.block_d_dmin(blocks)
        sc, m = self.scale_min_pairs(blocks)
        q = self.quants(blocks)
        j = np.arange(256) // 32
        w = d[..., None] * sc[..., j] * q - dmin[..., None] * m[..., j]
        return w.reshape(w.shape[:-2] + (w.shape[-2] * 256,))


def _swap_nibbles(blocks):
    q = O.quants(blocks)
    out = q.copy()
    for c in range(4):
        out[..., 64 * c:64 * c + 32], out[..., 64 * c + 32:64 * c + 64] = q[..., 64 * c + 32:64 * c + 64], q[..., 64 * c:64 * c + 32]
    return out


def _swap_sc_m(blocks):
    sc, m = O.scale_min_pairs(blocks)
    return m, sc


def _hi_bits_wrong(blocks):
    sc, m = O.scale_min_pairs(blocks)
    sc2, m2 = sc.copy(), m.copy()
    sc2[..., 4:], m2[..., 4:] = (sc[..., 4:] & 15) | (m[..., 4:] & 48), (m[..., 4:] & 15) | (sc[..., 4:] & 48)
    return sc2, m2


def _d_dmin_swapped(blocks):
    d, dmin = O.block_d_dmin(blocks)
    return dmin, d


@pytest.mark.parametrize("mut", [dict(quants=_swap_nibbles), dict(scale_min_pairs=_swap_sc_m),
                                 dict(scale_min_pairs=_hi_bits_wrong), dict(block_d_dmin=_d_dmin_swapped)])
def test_planted_mistakes_are_caught(mut):
    assert not _golden_ok(_Mutant(**mut))


# ------------------------------------------------------------ decode repack --
# repack_ref is a byte permutation; these pins check it against properties the
# layout definition fixes, each chosen so that a plausible slip (chunk and
# quarter swapped, rows and blocks swapped in the tile order, the header moved,
# padding rows not zero) fails one of them.

def _tagged_blocks(N, nkb):
    """Blocks whose header names (row, block) and whose quant bytes are 0..127."""
    W = np.zeros((N, nkb, O.BLOCK_BYTES), dtype=np.uint8)
    for n in range(N):
        for kb in range(nkb):
            W[n, kb, 0] = n & 255
            W[n, kb, 1] = n >> 8
            W[n, kb, 2] = kb
            W[n, kb, 3] = 0xA5
            W[n, kb, 16:] = np.arange(128, dtype=np.uint8)
    return W


def test_repack_tile_order_and_padding():
    N, nkb = 200, 3  # two tiles, the second ragged (72 rows)
    Wr = O.repack_ref(_tagged_blocks(N, nkb))
    assert Wr.size == 2 * nkb * 128 * 144
    for n, kb in [(0, 0), (1, 0), (127, 2), (128, 0), (130, 1), (199, 2)]:
        off = ((n // 128 * nkb + kb) * 128 + n % 128) * 144
        assert Wr[off] == n & 255 and Wr[off + 1] == n >> 8 and Wr[off + 2] == kb and Wr[off + 3] == 0xA5
    # rows 200..255 of the second tile are zero
    R = Wr.reshape(2, nkb, 128, 144)
    assert not R[1, :, 72:, :].any()


def test_repack_quarter_runs():
    """A GEMV thread t reads 32 consecutive bytes at 16 + 32t: quant bytes
    [8t, 8t+8) of chunks 0, 1, 2, 3 in that order (byte values 0..127 = index)."""
    R = O.repack_ref(_tagged_blocks(1, 1)).reshape(128, 144)[0]
    expect = {0: [0, 32, 64, 96], 1: [8, 40, 72, 104], 2: [16, 48, 80, 112], 3: [24, 56, 88, 120]}
    for t, starts in expect.items():
        run = R[16 + 32 * t:16 + 32 * t + 32]
        assert list(run) == [s + e for s in starts for e in range(8)]


def test_repack_round_trip_and_byte_multisets():
    rng = np.random.default_rng(17)
    N, nkb = 300, 4
    W = rng.integers(0, 256, size=(N, nkb, 144), dtype=np.uint8)
    Wr = O.repack_ref(W)
    assert np.array_equal(O.unrepack_ref(Wr, N, nkb * 256), W)
    R = Wr.reshape(-1, nkb, 128, 144)
    for n in (0, 77, 128, 299):
        for kb in range(nkb):
            blk = R[n // 128, kb, n % 128]
            assert np.array_equal(blk[:16], W[n, kb, :16])
            assert np.array_equal(np.sort(blk[16:]), np.sort(W[n, kb, 16:]))


# ------------------------------------------------------------------ Q5_K --

def _scalar_weight_q5(block, i):
    """Scalar restatement of one Q5_K weight, used only as brute force (Reading R19)."""
    d = float(np.frombuffer(bytes(block[0:2]), "<f2")[0])
    dmin = float(np.frombuffer(bytes(block[2:4]), "<f2")[0])
    s = [int(v) for v in block[4:16]]
    j = i // 32
    if j < 4:
        sc, m = s[j] & 63, s[j + 4] & 63
    else:
        sc = (s[j + 4] & 0xF) | ((s[j - 4] >> 6) << 4)
        m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4)
    c, rem = divmod(i, 64)
    h, l = divmod(rem, 32)
    low = (int(block[48 + 32 * c + l]) >> (4 * h)) & 0xF
    fifth = (int(block[16 + l]) >> (2 * c + h)) & 1
    return d * sc * (low + 16 * fifth) - dmin * m


def test_q5_one_hot_fifth_bits_and_nibbles():
    """Bit 2c+h of qh[l] alone adds 16*d*sc_j to weight 64c+32h+l and to no other;
    nibble h of byte 48+32c+l alone adds d*sc_j*v to that same weight."""
    sc = np.arange(3, 11)
    base = O.make_block_q5(1.0, 0.0, sc, np.zeros(8, int), np.zeros(256, int))
    assert np.all(O.dequant_exact_q5(base[None]) == 0)
    for c in range(4):
        for h in range(2):
            for l in range(32):
                i = 64 * c + 32 * h + l
                b = base.copy()
                b[16 + l] = np.uint8(1 << (2 * c + h))
                expect = np.zeros(256)
                expect[i] = 16.0 * sc[i // 32]
                assert np.array_equal(O.dequant_exact_q5(b[None]), expect), (c, h, l)
                b = base.copy()
                b[48 + 32 * c + l] = np.uint8(7 << (4 * h))
                expect[i] = 7.0 * sc[i // 32]
                assert np.array_equal(O.dequant_exact_q5(b[None]), expect), (c, h, l)


def test_q5_closed_form_and_q4_agreement():
    """All quants 31 (every nibble 15, every fifth bit set): w = d*s*31 - dmin*t.
    With no fifth bit set a Q5_K block dequantises like the Q4_K block with the
    same header and nibbles."""
    for (d, dmin, s, t) in [(1e-3, 2e-3, 17, 40), (0.25, 0.125, 63, 63)]:
        blk = O.make_block_q5(d, dmin, [s] * 8, [t] * 8, [31] * 256)
        assert np.all(blk[16:176] == 0xFF)
        dh, dmh = float(np.float16(d)), float(np.float16(dmin))
        assert np.all(O.dequant_exact_q5(blk[None]) == dh * s * 31 - dmh * t)
    rng = np.random.default_rng(11)
    W4 = synth.q4k_random_blocks(rng, 3, 512)
    W5 = np.zeros(W4.shape[:-1] + (176,), np.uint8)
    W5[..., 0:16] = W4[..., 0:16]
    W5[..., 48:176] = W4[..., 16:144]
    np.testing.assert_array_equal(O.dequant_exact_q5(W5), O.dequant_exact(W4))


def test_q5_encode_round_trip_and_brute_force_matmul():
    rng = np.random.default_rng(12)
    q = rng.integers(0, 32, 256)
    sc, m = rng.integers(0, 64, 8), rng.integers(0, 64, 8)
    blk = O.make_block_q5(3e-3, 1e-3, sc, m, q)
    np.testing.assert_array_equal(O.quants_q5(blk[None])[0], q)
    W, X = synth.gemv_small_q5(13, N=2, K=256, M=2)
    Y, S = O.matmul_ref_q5(W, X)
    xf = O.bf16_to_f64(X)
    for n in range(2):
        for t in range(2):
            prods = [_scalar_weight_q5(W[n, 0], i) * xf[t, i] for i in range(256)]
            assert abs(Y[t, n] - math.fsum(prods)) <= 1e-12 * math.fsum(abs(p) for p in prods)
            assert abs(S[t, n] - math.fsum(abs(p) for p in prods)) <= 1e-12 * S[t, n]


def test_q5_synth_quants_cover_0_to_31():
    W, _ = synth.gemv_small_q5(14, N=64, K=512, M=1)
    q = O.quants_q5(W)
    assert q.min() == 0 and q.max() == 31
    counts = np.bincount(q.ravel(), minlength=32)
    assert counts.min() > 0.8 * counts.mean()


# ------------------------------------------------------------------ Q8_0 --

def test_q80_one_hot_and_signs():
    """A block with one nonzero quant v at position l gives w = d*v at weight 32b+l
    only; the sign follows two's complement (byte 0x80 is -128, 0xFF is -1)."""
    for l in (0, 1, 17, 31):
        for v, byte in ((1, 0x01), (127, 0x7F), (-1, 0xFF), (-128, 0x80)):
            blk = np.zeros(34, np.uint8)
            blk[0:2] = np.array([0.5], dtype="<f2").view(np.uint8)
            blk[2 + l] = byte
            W = np.stack([np.zeros(34, np.uint8), blk])[None]  # one row, two blocks
            W[0, 0, 0:2] = np.array([1.0], dtype="<f2").view(np.uint8)
            w = O.dequant_exact_q80(W)[0]
            expect = np.zeros(64)
            expect[32 + l] = 0.5 * v
            assert np.array_equal(w, expect), (l, v)


def test_q80_encode_closed_form_and_brute_force():
    rng = np.random.default_rng(15)
    q = rng.integers(-128, 128, 32)
    blk = O.make_block_q80(3e-3, q)
    dh = float(np.float16(3e-3))
    np.testing.assert_array_equal(O.dequant_exact_q80(blk[None]), dh * q)
    W, X = synth.gemv_small_q80(16, N=2, K=256, M=2)
    Y, S = O.matmul_ref_q80(W, X)
    xf = O.bf16_to_f64(X)
    for n in range(2):
        for t in range(2):
            prods = []
            for i in range(256):
                b = W[n, i // 32]
                d = float(np.frombuffer(bytes(b[0:2]), "<f2")[0])
                qv = int(b[2 + i % 32])
                qv = qv - 256 if qv >= 128 else qv
                prods.append(d * qv * xf[t, i])
            assert abs(Y[t, n] - math.fsum(prods)) <= 1e-12 * math.fsum(abs(p) for p in prods)
    Wq, _ = synth.gemv_small_q80(17, N=64, K=512, M=1)
    qv = Wq[..., 2:34].view(np.int8)
    assert qv.min() == -128 and qv.max() == 127


# --------------------------------------------------------------- router --

def test_router_logits_brute_force_and_one_hot():
    """Every logit enumerated for a tiny case; a one-hot activation row selects a
    column of the router weights."""
    rng = np.random.default_rng(19)
    X = synth.bf16_normal(rng, (3, 16))
    Wr = synth.bf16_normal(rng, (5, 16))
    L, S = O.router_logits_ref(X, Wr)
    xf, wf = O.bf16_to_f64(X), O.bf16_to_f64(Wr)
    for t in range(3):
        for e in range(5):
            prods = [xf[t, k] * wf[e, k] for k in range(16)]
            assert abs(L[t, e] - math.fsum(prods)) <= 1e-14 * math.fsum(abs(p) for p in prods)
            assert abs(S[t, e] - math.fsum(abs(p) for p in prods)) <= 1e-14 * S[t, e]
    onehot = np.zeros((1, 16), np.uint16)
    onehot[0, 7] = 0x3F80  # bf16 1.0
    L1, _ = O.router_logits_ref(onehot, Wr)
    np.testing.assert_array_equal(L1[0], wf[:, 7])


def test_router_weights_give_the_workload_logit_spread():
    rng = np.random.default_rng(20)
    X = synth.bf16_normal(rng, (64, 2048))
    L, _ = O.router_logits_ref(X, synth.router_weights(21))
    assert 1.8 < L.std() < 2.2


# -------------------------------------------------------------- Q8 lane --

def test_q8lane_quantizer_codes_and_error():
    """Codes lie in -127..127; each column's largest magnitude maps to +-127; a zero
    column gives zero codes and scale; every value is recovered within half a step
    (plus the fp32 rounding of the scale and of its reciprocal)."""
    rng = np.random.default_rng(23)
    X = synth.bf16_normal(rng, (4, 1024))
    X[1, 256:512] = 0
    q, d_x = O.quantize_x_q8(X)
    assert q.min() >= -127 and q.max() <= 127
    x = O.bf16_to_f64(X)
    for t in range(4):
        for kb in range(4):
            seg = x[t, 256 * kb: 256 * kb + 256]
            qs = q[t, 256 * kb: 256 * kb + 256]
            if not seg.any():
                assert d_x[t, kb] == 0 and not qs.any()
                continue
            i = np.argmax(np.abs(seg))
            assert abs(qs[i]) == 127 and np.sign(qs[i]) == np.sign(seg[i])
            # half a step, plus |q| <= 127 times the gap between d_x = RN(amax/127) and
            # 1/RN(127/amax) (a few fp32 ulps): d_x * (0.5 + 2e-5)
            err = np.abs(seg - qs * float(d_x[t, kb]))
            assert err.max() <= float(d_x[t, kb]) * (0.5 + 2e-5) + 1e-30


def test_q8lane_integer_form_and_accuracy_bound():
    """The lane's product equals the integer form used on the GPU -- per super-block
    d * sum_j sc_j * (q_w . q_x) - dmin * sum_j m_j * bsum_j, times d_x -- and stays
    within sum |w| * |x - d_x q| of the exact product."""
    W, X = synth.gemv_small(24, N=3, K=512, M=2)
    Y, S = O.matmul_ref_q8lane(W, X)
    q, d_x = O.quantize_x_q8(X)
    d, dmin = O.block_d_dmin(W)
    sc, m = O.scale_min_pairs(W)
    qw = O.quants(W)
    for t in range(2):
        for n in range(3):
            tot = 0.0
            for kb in range(2):
                qx = q[t, 256 * kb: 256 * kb + 256]
                I = sum(int(sc[n, kb, j]) * int(np.dot(qw[n, kb, 32 * j: 32 * j + 32], qx[32 * j: 32 * j + 32]))
                        for j in range(8))
                Im = sum(int(m[n, kb, j]) * int(qx[32 * j: 32 * j + 32].sum()) for j in range(8))
                tot += float(d_x[t, kb]) * (d[n, kb] * I - dmin[n, kb] * Im)
            assert abs(Y[t, n] - tot) <= 1e-12 * S[t, n]
    Ye, _ = O.matmul_ref(W, X)
    xq = q * np.repeat(d_x.astype(np.float64), 256, axis=1)
    bound = np.abs(O.dequant_exact(W)) @ np.abs(O.bf16_to_f64(X) - xq).T
    assert np.all(np.abs(Y - Ye) <= bound.T * (1 + 1e-9) + 1e-30)


# ------------------------------------------------------------------ Q6_K --

def test_q6_one_hot_bits():
    """Setting one bit of ql or qh changes exactly one weight, by d*scale*(bit value):
    nibble u//2 of ql[64n+32(u%2)+l] and bits 2u, 2u+1 of qh[32n+l] belong to weight
    128n+32u+l, whose scale is scale[i // 16]."""
    scales = np.arange(1, 17)
    base = O.make_block_q6(1.0, scales, np.full(256, -32))  # all six-bit fields zero
    assert not base[0:192].any()
    w0 = O.dequant_exact_q6(base[None])
    assert np.array_equal(w0, -32.0 * scales[np.arange(256) // 16])
    for n in range(2):
        for u in range(4):
            for l in (0, 5, 31):
                i = 128 * n + 32 * u + l
                for bit in range(6):
                    b = base.copy()
                    if bit < 4:
                        b[64 * n + 32 * (u % 2) + l] = np.uint8(1 << (bit + 4 * (u // 2)))
                    else:
                        b[128 + 32 * n + l] = np.uint8(1 << (2 * u + bit - 4))
                    diff = O.dequant_exact_q6(b[None]) - w0
                    expect = np.zeros(256)
                    expect[i] = float(1 << bit) * scales[i // 16]
                    assert np.array_equal(diff, expect), (n, u, l, bit)


def test_q6_round_trip_signs_and_brute_force():
    rng = np.random.default_rng(25)
    q = rng.integers(-32, 32, 256)
    sc = rng.integers(-128, 128, 16)
    blk = O.make_block_q6(2e-3, sc, q)
    np.testing.assert_array_equal(O.quants_q6(blk[None])[0], q)
    dh = float(np.float16(2e-3))
    np.testing.assert_array_equal(O.dequant_exact_q6(blk[None]), dh * sc[np.arange(256) // 16] * q)
    W = synth.q6k_random_blocks(rng, 2, 256)
    X = synth.bf16_normal(rng, (2, 256))
    Y, S = O.matmul_ref_q6(W, X)
    xf = O.bf16_to_f64(X)
    wq = O.quants_q6(W)
    for n in range(2):
        d = float(np.frombuffer(bytes(W[n, 0, 208:210]), "<f2")[0])
        s = W[n, 0, 192:208].view(np.int8)
        for t in range(2):
            prods = [d * int(s[i // 16]) * int(wq[n, 0, i]) * xf[t, i] for i in range(256)]
            assert abs(Y[t, n] - math.fsum(prods)) <= 1e-12 * math.fsum(abs(p) for p in prods)
    allq = O.quants_q6(synth.q6k_random_blocks(rng, 64, 512))
    assert allq.min() == -32 and allq.max() == 31


# ---------------------------------------------------------------- SiLU / SwiGLU --
# silu_mul and swiglu_bf16_ref (Reading R16: SiLU(g) = g * sigma(g), the gate of
# the SwiGLU expert FFN; Reading R8: gate columns first, then up) pinned by values
# the mathematics fixes, not by a restatement of the formula:
#   silu(0) = 0;  silu(1) = 1 / (1 + e^-1) = 0.7310585786300049;
#   silu(-1) = -1 / (1 + e) = -0.2689414213699951;
#   silu(g) - silu(-g) = g (sigma(g) + sigma(-g) = 1);
#   silu(g) > g / 2 for g > 0 (sigma(g) > 1/2 there);
#   silu(g) -> g as g -> +inf, silu(g) -> 0 from below as g -> -inf;
# and the logistic function of an independent library (scipy.special.expit).

SILU_1 = 0.7310585786300049    # 1 / (1 + 1/e), e = 2.718281828459045
SILU_M1 = -0.2689414213699951  # -1 / (1 + e)


def _silu_pins_hold(silu_mul) -> bool:
    from scipy.special import expit

    one = np.ones(1)
    if silu_mul(np.zeros(1), one)[0] != 0.0:
        return False
    if abs(silu_mul(one, one)[0] - SILU_1) > 1e-15 or abs(silu_mul(-one, one)[0] - SILU_M1) > 1e-15:
        return False
    g = np.linspace(-12.0, 12.0, 241)
    s, s_neg = silu_mul(g, np.ones_like(g)), silu_mul(-g, np.ones_like(g))
    if np.max(np.abs((s - s_neg) - g)) > 1e-13:
        return False
    pos = g > 0
    if not np.all(s[pos] > g[pos] / 2):
        return False
    if np.max(np.abs(s - g * expit(g))) > 1e-14:
        return False
    big = np.array([40.0, 100.0])
    if not np.all(silu_mul(big, np.ones(2)) == big):           # sigma(40) = 1 - 4e-18 -> 1.0
        return False
    tail = silu_mul(-big, np.ones(2))
    if not (np.all(tail < 0) and np.all(tail > -1e-15)):        # -40 e^-40 ~ -1.7e-16
        return False
    u = np.array([3.0, -0.5])                                   # linear in u
    return bool(np.all(np.abs(silu_mul(np.array([1.0, 1.0]), u) - SILU_1 * u) <= 1e-15))


def test_silu_pinned():
    assert _silu_pins_hold(O.silu_mul)


@pytest.mark.parametrize("mutant", [
    lambda g, u: g / (1.0 + np.exp(g)) * u,            # sigma(-g) in place of sigma(g)
    lambda g, u: 1.0 / (1.0 + np.exp(-g)) * u,         # sigmoid without the factor g
    lambda g, u: g / (1.0 + np.exp(-2.0 * g)) * u,     # a different slope
    lambda g, u: g * np.tanh(g) * u,                   # a different gate
])
def test_silu_mutants_are_caught(mutant):
    assert not _silu_pins_hold(mutant)


def test_swiglu_bf16_hand_values():
    """h = RN_bf16(RN_fp32(silu(gate) * up)) on hand-worked rows, gate columns first.

    gate 1, up 2: 2 * 0.7310585786300049 = 1.4621171572600098; bf16 spacing in [1, 2) is 2^-7,
    1.46211.../2^-7 = 187.15 -> 187 -> 1.4609375 = 0x3FBB.
    gate 2, up 1: 2 / (1 + e^-2) = 1.7615941559557646 -> 225.48 * 2^-7 -> 225 -> 1.7578125 = 0x3FE1
    (the same row read up-first would give 0x3FBB: the column order is pinned).
    gate 0, up 5: 0 -> 0x0000.  gate -1, up -4: 4 * 0.2689414213699951 = 1.0757656854799804
    -> 137.70 * 2^-7 -> 138 -> 1.078125 = 0x3F8A.
    """
    GU = np.array([[1.0, 2.0, 0.0, -1.0, 2.0, 1.0, 5.0, -4.0]])
    h = O.swiglu_bf16_ref(GU, 4)
    assert h.dtype == np.uint16
    assert [int(v) for v in h[0]] == [0x3FBB, 0x3FE1, 0x0000, 0x3F8A]


# ---------------------------------------------------- bf16 round to nearest even --
# Reading R2 (bf16 weights = RN_bf16(RN_fp32(w))) and the h rounding of Reading R7
# both rest on round-to-nearest-EVEN. Ties are built by hand: 1 + 2^-8 lies exactly
# halfway between the bf16 neighbours 1.0 (0x3F80, even) and 1 + 2^-7 (0x3F81, odd);
# 1 + 3*2^-8 halfway between 0x3F81 and 1 + 2^-6 (0x3F82, even). Round-half-away,
# round-half-up and truncation each get at least one of these wrong.

def _f32(v):
    return np.array([v], dtype=np.float64)


_RNE_CASES = [
    (1.0 + 2.0 ** -8, 0x3F80),                    # tie -> even (down)
    (1.0 + 3 * 2.0 ** -8, 0x3F82),                # tie -> even (up)
    (-(1.0 + 2.0 ** -8), 0xBF80),                 # sign symmetric
    (-(1.0 + 3 * 2.0 ** -8), 0xBF82),
    (1.0 + 2.0 ** -8 - 2.0 ** -23, 0x3F80),       # largest fp32 below the tie
    (1.0 + 2.0 ** -8 + 2.0 ** -23, 0x3F81),       # smallest fp32 above it
    # bf16 subnormals are k * 2^-133 (k < 128); fp32 holds these ties exactly
    (2.0 ** -133 * 1.5, 0x0002),                  # tie between k = 1 and 2 -> even (2)
    (2.0 ** -133 * 2.5, 0x0002),                  # tie between k = 2 and 3 -> even (2)
]


def _rne_pins_hold(to_bf16) -> bool:
    return all(int(to_bf16(_f32(v))[0]) == bits for v, bits in _RNE_CASES)


def test_bf16_rne_ties_and_neighbours():
    assert _rne_pins_hold(O.f64_to_bf16_bits)


def _f32_bits(a):
    return np.ascontiguousarray(a, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)


@pytest.mark.parametrize("mutant", [
    lambda a: ((_f32_bits(a) + 0x8000) >> 16).astype(np.uint16),             # ties away from zero
    lambda a: (_f32_bits(a) >> 16).astype(np.uint16),                         # truncation
    lambda a: ((_f32_bits(a) + 0x7FFF) >> 16).astype(np.uint16),             # ties toward zero
])
def test_bf16_rounding_mutants_are_caught(mutant):
    assert not _rne_pins_hold(mutant)


def test_bf16_double_rounding_through_fp32():
    """RN_bf16(RN_fp32(w)): 1 + 2^-8 + 2^-30 rounds to the tie 1 + 2^-8 in fp32 (2^-30 is
    below half an fp32 ulp of 1, 2^-24), then to the even 0x3F80 -- a direct rounding
    of the fp64 value would give 0x3F81."""
    assert int(O.f64_to_bf16_bits(_f32(1.0 + 2.0 ** -8 + 2.0 ** -30))[0]) == 0x3F80
    assert int(O.f64_to_bf16_bits(_f32(1.0 + 2.0 ** -8 + 2.0 ** -23))[0]) == 0x3F81


def test_dequant_bf16_ties_on_blocks():
    """Blocks whose weights are exact bf16 ties: d = 1 + 2^-8 and 1 + 3*2^-8 are fp16 values
    (10 mantissa bits), sc = q = 1, dmin = m = 0, so w = d exactly; bf16 must be the even
    neighbour. With q = 2 the weight 2d = 2 + 2^-7 is again a tie (spacing 2^-6 in [2, 4)):
    0x4000 (even). A min term reaching a tie from below: d = 1, sc = q = 1, dmin = 2^-8,
    m = 1 gives 1 - 2^-8, exactly representable in bf16 (spacing 2^-8 in [0.5, 1)): 0x3F7F."""
    blocks = np.stack([
        O.make_block(1.0 + 2.0 ** -8, 0.0, [1] * 8, [0] * 8, [1] * 256),
        O.make_block(1.0 + 3 * 2.0 ** -8, 0.0, [1] * 8, [0] * 8, [1] * 256),
        O.make_block(1.0 + 2.0 ** -8, 0.0, [1] * 8, [0] * 8, [2] * 256),
        O.make_block(1.0, 2.0 ** -8, [1] * 8, [1] * 8, [1] * 256),
    ])[:, None, :]                                    # four rows of one block each
    bits = O.dequant_bf16_bits(blocks)
    assert np.all(bits[0] == 0x3F80)
    assert np.all(bits[1] == 0x3F82)
    assert np.all(bits[2] == 0x4000)
    assert np.all(bits[3] == 0x3F7F)
    f32 = O.dequant_f32(blocks)
    assert np.all(f32[0] == np.float32(1.0 + 2.0 ** -8))
