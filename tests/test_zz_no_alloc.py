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


def test_noalloc_route_matches_workspace_entry_point(cuda_ok):
    # Two calls in a row on the shared scratch: a large skewed prefill batch,
    # then a small decode batch that reads the array the first call filled.
    cases = [synth.moe_layer(4, 4096, E=128, H=256, F=256, hot=16)["logits"],
             synth.moe_layer(5, 37, E=128, H=256, F=256)["logits"]]
    for logits_np in cases:
        logits = dev(logits_np)
        ref = q.moe_route_permute(logits, 8)
        st, got = _noalloc_via_c_abi(logits, 8)
        assert st == 0
        for key in ("topk_ids", "expert_offsets", "perm", "inv_perm", "row_token"):
            assert torch.equal(got[key], ref[key]), key
        dw = np.abs(host(got["topk_w"]).astype(np.float64) - host(ref["topk_w"]).astype(np.float64))
        assert dw.max() <= ROUTE_W_TOL
    assert q.q4k_last_device_status() == 0


def test_noalloc_route_rejects_problems_beyond_its_scratch(cuda_ok):
    # ceil(M/32) * E = 513 * 128 > 65536 histogram entries: refused before any launch.
    M, E = 32 * 513, 128
    logits = torch.zeros(M, E, dtype=torch.float32, device="cuda")
    st, _ = _noalloc_via_c_abi(logits, 8)
    assert st == 11  # Q4K_ERR_TOO_LARGE
