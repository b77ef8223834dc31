"""CPU checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "q4k.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(?:q4k_status|size_t|int64_t|const char\*)\s+(\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from q4_weight_only_super_b200 import build
    build.build()
    import q4_weight_only_super_b200 as q
    return q.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("q4k_gemv", "q4k_gemm", "moe_route_permute", "moe_q4k_grouped", "moe_combine",
              "q4k_repack", "q4k_repacked_bytes", "q4k_gemv_repacked", "moe_combine_residual", "q5k_gemv",
              "q80_gemv", "moe_route_permute_hidden", "q4k_gemv_q8"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    import q4_weight_only_super_b200 as q
    for name in _declared():
        assert hasattr(L, name), name
        assert name in q.EXPORTS, f"binding lacks {name}"


def test_status_strings(L):
    assert L.q4k_status_string(0) == b"ok"
    assert b"unsupported" in L.q4k_status_string(4)


def test_argument_errors_return_before_launch(L):
    fake = 4096  # never dereferenced: every call below fails validation first
    big = 1 << 30
    # K not a multiple of 256
    assert L.q4k_gemv(fake, fake, fake, 1, 16, 100, fake, big, None) == 3
    # null pointers (weights, workspace)
    assert L.q4k_gemv(None, fake, fake, 1, 16, 256, fake, big, None) == 1
    assert L.q4k_gemv(fake, fake, fake, 1, 16, 256, None, big, None) == 1
    # misaligned pointer
    assert L.q4k_gemv(fake + 4, fake, fake, 1, 16, 256, fake, big, None) == 2
    # M > 32 is not a GEMV shape
    assert L.q4k_gemv(fake, fake, fake, 33, 16, 256, fake, big, None) == 4
    # N not a multiple of 16
    assert L.q4k_gemv(fake, fake, fake, 1, 24, 256, fake, big, None) == 4
    # workspace too small
    assert L.q4k_gemv(fake, fake, fake, 1, 16, 256, fake, 64, None) == 5
    assert L.q5k_gemv(fake, fake, fake, 1, 16, 256, fake, 64, None) == 5
    # Q5_K GEMV: K not a multiple of 256, more than 32 tokens, N % 16
    assert L.q5k_gemv(fake, fake, fake, 1, 16, 300, fake, 1 << 20, None) == 3
    assert L.q5k_gemv(fake, fake, fake, 33, 16, 256, fake, 1 << 20, None) == 4
    assert L.q5k_gemv(fake, fake, fake, 1, 24, 256, fake, 1 << 20, None) == 4
    # Q8 lane: the q4k_gemv checks
    assert L.q4k_gemv_q8(fake, fake, fake, 1, 16, 100, fake, big, None) == 3
    assert L.q4k_gemv_q8(fake, fake, fake, 33, 16, 256, fake, big, None) == 4
    assert L.q4k_gemv_q8(fake, fake, fake, 1, 16, 256, fake, 64, None) == 5
    # Q8_0 GEMV: K must be a multiple of 256 (eight 32-weight blocks per column)
    assert L.q80_gemv(fake, fake, fake, 1, 16, 96, fake, 1 << 20, None) == 3
    assert L.q80_gemv(fake, fake, fake, 1, 16, 256, fake, 64, None) == 5
    assert L.q80_gemv(None, None, None, 0, 16, 256, None, 0, None) == 0
    # router front: H not a multiple of 8; too many experts; M == 0 writes zero offsets only
    assert L.moe_route_permute_hidden(fake, fake, 1, 128, 100, 8, fake, fake, fake, fake, fake, fake, fake,
                                      fake, big, None) == 3
    assert L.moe_route_permute_hidden(fake, fake, 1, 2048, 256, 8, fake, fake, fake, fake, fake, fake, fake,
                                      fake, big, None) == 4
    # GEMM N not a multiple of 256
    assert L.q4k_gemm(fake, fake, fake, 4, 128, 256, None, 0, None) == 4
    # routing: too many experts / top-k
    assert L.moe_route_permute(fake, 4, 2048, 8, fake, fake, fake, fake, fake, fake, fake, 1 << 20,
                               None) == 4
    assert L.moe_route_permute(fake, 4, 128, 17, fake, fake, fake, fake, fake, fake, fake, 1 << 20,
                               None) == 4
    # routing: workspace too small
    assert L.moe_route_permute(fake, 64, 128, 8, fake, fake, fake, fake, fake, fake, fake, 16,
                               None) == 5
    # grouped: bad activation code, combine: H % 4
    assert L.moe_q4k_grouped(fake, 4, 64, 256, fake, None, fake, 8, 8, 7, fake, None, 0, None) == 4
    assert L.moe_combine(fake, fake, fake, 2, 2, 6, fake, None) == 4
    assert L.moe_combine_residual(fake, fake, fake, fake, 2, 2, 6, fake, None) == 4
    assert L.moe_combine_residual(fake, fake, fake, None, 2, 2, 8, fake, None) == 1
    assert L.moe_combine_residual(None, None, None, None, 0, 2, 8, None, None) == 0
    # routing + gate_up in one launch: more than 32 tokens, more than 256 experts, K below
    # six super-blocks or above 5120, K not a multiple of 256 (no fallback)
    rg = L.moe_route_gate_up
    assert rg(fake, 33, 128, 8, fake, fake, fake, fake, fake, fake, fake, 1536, 2048, fake, fake, None) == 4
    assert rg(fake, 4, 512, 8, fake, fake, fake, fake, fake, fake, fake, 1536, 2048, fake, fake, None) == 4
    assert rg(fake, 4, 128, 8, fake, fake, fake, fake, fake, fake, fake, 1536, 1280, fake, fake, None) == 4
    assert rg(fake, 4, 128, 8, fake, fake, fake, fake, fake, fake, fake, 1536, 24 * 256, fake, fake, None) == 4
    assert rg(fake, 4, 128, 8, fake, fake, fake, fake, fake, fake, fake, 1536, 2000, fake, fake, None) == 3
    assert rg(fake, 4, 128, 8, fake, fake, None, fake, fake, fake, fake, 1536, 2048, fake, fake, None) == 1
    # empty problems are no-ops
    assert L.q4k_gemv(None, None, None, 0, 16, 256, None, 0, None) == 0
    assert L.moe_combine(None, None, None, 0, 2, 8, None, None) == 0


def test_workspace_size(L):
    assert L.q4k_workspace_bytes(2, 4096, 0, 0, 128, 8) == 128 * 128 * 4
    assert L.q4k_workspace_bytes(2, 1, 0, 0, 128, 8) == 128 * 4
    assert L.q4k_workspace_bytes(1, 4096, 17408, 5120, 0, 0) == 0
    # GEMV: (K/256) blocks x (M + 32 padding rows) x 576-byte records
    assert L.q4k_workspace_bytes(4, 1, 34816, 5120, 0, 0) == 20 * 33 * 576
    assert L.q4k_workspace_bytes(3, 256, 1536, 2048, 128, 8) == 8 * 288 * 576


def test_repack_arguments(L):
    fake = 4096
    big = 1 << 30
    # 128-row tiles x (K/256) super-blocks x 144 bytes; N padded to the tile
    assert L.q4k_repacked_bytes(200, 512) == 2 * 2 * 128 * 144
    assert L.q4k_repacked_bytes(128, 256) == 128 * 144
    assert L.q4k_repacked_bytes(0, 256) == 0 and L.q4k_repacked_bytes(16, 100) == 0
    assert L.q4k_repack(fake, 16, 100, fake, None) == 3       # K % 256
    assert L.q4k_repack(None, 16, 256, fake, None) == 1
    assert L.q4k_repack(fake, 16, 256, fake + 8, None) == 2   # misaligned
    assert L.q4k_repack(None, 0, 256, None, None) == 0        # empty: no-op
    assert L.q4k_gemv_repacked(fake, fake, fake, 33, 16, 256, fake, big, None) == 4
    assert L.q4k_gemv_repacked(fake, fake, fake, 1, 24, 256, fake, big, None) == 4
    assert L.q4k_gemv_repacked(fake, fake, fake, 1, 16, 256, fake, 64, None) == 5
    assert L.q4k_gemv_repacked(None, None, None, 0, 16, 256, None, 0, None) == 0
