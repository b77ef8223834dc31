"""The no-allocation routing entry point, checked on the GPU against the
regular one.

moe_route_permute_noalloc exists for callers that cannot allocate device
memory when they call the library -- for example a runtime whose device
memory is owned by a host framework that gives this library no allocator,
or a serving loop that bans cudaMalloc after start-up because it can
synchronise the device. It keeps its scratch in a fixed array inside the
library instead of a caller-provided workspace, so it must give exactly the
results of moe_route_permute, call after call, even though the array still
holds the previous call's data.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from tests.gpu_util import dev, host

pytestmark = pytest.mark.gpu

q = pytest.importorskip("q4_weight_only_super_b200")

ROUTE_W_TOL = 1e-6  # routing-weight tolerance used by the routing parity tests


def _outputs(M, E, topk):
    return dict(
        topk_ids=torch.empty(M, topk, dtype=torch.int32, device="cuda"),
        topk_w=torch.empty(M, topk, dtype=torch.float32, device="cuda"),
        expert_offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
        perm=torch.empty(M * topk, dtype=torch.int32, device="cuda"),
        inv_perm=torch.empty(M * topk, dtype=torch.int32, device="cuda"),
        row_token=torch.empty(M * topk, dtype=torch.int32, device="cuda"),
    )


def _noalloc_via_c_abi(logits, topk):
    """Call the entry point through the C ABI directly (ctypes, raw pointers)."""
    L = q.lib()
    M, E = logits.shape
    out = _outputs(M, E, topk)
    st = L.moe_route_permute_noalloc(
        ctypes.c_void_p(logits.data_ptr()), M, E, topk,
        ctypes.c_void_p(out["topk_ids"].data_ptr()), ctypes.c_void_p(out["topk_w"].data_ptr()),
        ctypes.c_void_p(out["expert_offsets"].data_ptr()), ctypes.c_void_p(out["perm"].data_ptr()),
        ctypes.c_void_p(out["inv_perm"].data_ptr()), ctypes.c_void_p(out["row_token"].data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


def _compare(logits_np, topk):
    logits = dev(logits_np)
    ref = q.moe_route_permute(logits, topk)
    st, got = _noalloc_via_c_abi(logits, topk)
    assert st == 0
    for key in ("topk_ids", "expert_offsets", "perm", "inv_perm", "row_token"):
        assert torch.equal(got[key], ref[key]), (logits_np.shape, topk, key)
    dw = np.abs(host(got["topk_w"]).astype(np.float64) - host(ref["topk_w"]).astype(np.float64))
    assert dw.max() <= ROUTE_W_TOL


def test_noalloc_route_matches_workspace_entry_point(cuda_ok):
    # Calls back to back on the shared scratch: a large skewed prefill batch, then
    # smaller batches that read the array the earlier calls filled. Up to 32 tokens
    # the regular entry point routes in one CTA while this one always runs the
    # per-tile kernels (one tile there), so those token counts pair the two paths.
    rng = np.random.default_rng(77)
    cases = [(synth.moe_layer(4, 4096, E=128, H=256, F=256, hot=16)["logits"], 8),
             (synth.moe_layer(5, 37, E=128, H=256, F=256)["logits"], 8)]
    cases += [(synth.moe_layer(3, M, E=128, H=256, F=256)["logits"], 8) for M in (1, 8, 32)]
    cases += [((rng.standard_normal((70, 40)) * 2).astype(np.float32), 3),     # E = 40, top-3, 3 tiles
              ((rng.standard_normal((9, 1000))).astype(np.float32), 16),       # E = 1000, top-16, 1 tile
              (synth.moe_layer(3, 1, E=128, H=256, F=256)["logits"], 8)]       # again after those
    for logits_np, topk in cases:
        _compare(logits_np, topk)
    assert q.q4k_last_device_status() == 0


def test_noalloc_route_zero_tokens(cuda_ok):
    """M = 0: only the expert offsets are written, all zero."""
    L = q.lib()
    offs = torch.full((129,), -1, dtype=torch.int32, device="cuda")
    st = L.moe_route_permute_noalloc(None, 0, 128, 8, None, None, ctypes.c_void_p(offs.data_ptr()), None, None,
                                     None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    assert torch.count_nonzero(offs).item() == 0


def test_noalloc_route_rejects_problems_beyond_its_scratch(cuda_ok):
    # ceil(M/32) * E = 513 * 128 > 65536 histogram entries: refused before any launch.
    M, E = 32 * 513, 128
    logits = torch.zeros(M, E, dtype=torch.float32, device="cuda")
    st, _ = _noalloc_via_c_abi(logits, 8)
    assert st == 11  # Q4K_ERR_TOO_LARGE
