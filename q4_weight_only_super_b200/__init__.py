"""Q4_K weight-only matrix products for NVIDIA B200 (sm_100a).

Thin ctypes binding over ``libq4k.so`` (C ABI in ``include/q4k.h``). Every
function here only marshals arguments: tensors are passed as raw device
pointers, the current torch CUDA stream is passed as the stream, and any
non-zero status raises :class:`Q4KError`. All computation happens in the
library's CUDA kernels; there is no CPU path.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "Q4KError", "lib", "q4k_dequant", "q4k_gemv", "q4k_gemv_q8", "q5k_gemv", "q80_gemv", "q6k_gemv", "q4k_repack", "q4k_gemv_repacked", "q4k_gemm", "bf16w_gemm",
    "moe_route_permute",
    "moe_route_permute_noalloc", "moe_route_permute_hidden", "moe_route_gate_up",
    "moe_q4k_grouped", "moe_combine", "moe_combine_residual", "q4k_workspace_bytes", "q4k_last_device_status",
    "q4k_test_wait_fault",
    "ACT_NONE", "ACT_SWIGLU", "OP_GEMM", "OP_ROUTE", "OP_GROUPED", "OP_GEMV", "EXPORTS",
]

ACT_NONE, ACT_SWIGLU = 0, 1
OP_GEMM, OP_ROUTE, OP_GROUPED, OP_GEMV = 1, 2, 3, 4
BLOCK_BYTES = 144
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libq4k.so")

_p, _i, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
# name -> (restype, argtypes); mirrors include/q4k.h
EXPORTS = {
    "q4k_dequant": (_i, [_p, _i64, _i, _p, _p]),
    "q4k_gemv": (_i, [_p, _p, _p, _i, _i, _i, _p, _sz, _p]),
    "q5k_gemv": (_i, [_p, _p, _p, _i, _i, _i, _p, _sz, _p]),
    "q80_gemv": (_i, [_p, _p, _p, _i, _i, _i, _p, _sz, _p]),
    "q6k_gemv": (_i, [_p, _p, _p, _i, _i, _i, _p, _sz, _p]),
    "q4k_gemv_q8": (_i, [_p, _p, _p, _i, _i, _i, _p, _sz, _p]),
    "q4k_repacked_bytes": (_i64, [_i, _i]),
    "q4k_repack": (_i, [_p, _i, _i, _p, _p]),
    "q4k_gemv_repacked": (_i, [_p, _p, _p, _i, _i, _i, _p, _sz, _p]),
    "q4k_gemm": (_i, [_p, _p, _p, _i, _i, _i, _p, _sz, _p]),
    "bf16w_gemm": (_i, [_p, _p, _p, _i, _i, _i, _p]),
    "moe_route_permute": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "moe_route_permute_noalloc": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p]),
    "moe_route_permute_hidden": (_i, [_p, _p, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "moe_q4k_grouped": (_i, [_p, _i, _i, _i, _p, _p, _p, _i, _i, _i, _p, _p, _sz, _p]),
    "moe_route_gate_up": (_i, [_p, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _i, _i, _p, _p, _p]),
    "moe_combine": (_i, [_p, _p, _p, _i, _i, _i, _p, _p]),
    "moe_combine_residual": (_i, [_p, _p, _p, _p, _i, _i, _i, _p, _p]),
    "q4k_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "q4k_last_device_status": (_i, [_p]),
    "q4k_test_wait_fault": (_i, [_i, ctypes.c_uint64]),
    "q4k_status_string": (ctypes.c_char_p, [_i]),
}

_LIB = None


class Q4KError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: status {status} ({lib().q4k_status_string(status).decode()})")


def lib() -> ctypes.CDLL:
    """Load libq4k.so (fails loudly if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m q4_weight_only_super_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, st):
    if st != 0:
        raise Q4KError(fn, st)


def _bits16(x):
    """bf16 activations may be given as bfloat16 or as their int16 bit patterns."""
    assert x.dtype in (torch.bfloat16, torch.int16, torch.uint16), x.dtype
    return x


def q4k_dequant(W, out_bf16: bool = False, out=None, stream=None):
    """W: uint8 [..., 144] Q4_K blocks on the GPU -> fp32 (or bf16) weights [nblocks*256]."""
    nb = W.numel() // BLOCK_BYTES
    if out is None:
        out = torch.empty(nb * 256, dtype=torch.bfloat16 if out_bf16 else torch.float32, device=W.device)
    _check("q4k_dequant", lib().q4k_dequant(_ptr(W), nb, int(out_bf16), _ptr(out), _stream(stream)))
    return out


def _scratch(nbytes: int, device, ws=None):
    if ws is not None:
        return ws
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def q4k_gemv(W, X, N: int, K: int, Y=None, ws=None, stream=None):
    """Y[M][N] = X[M][K] @ W^T for 1 <= M <= 32 (W: Q4_K [N][K/256][144])."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=X.device)
    ws = _scratch(q4k_workspace_bytes(OP_GEMV, M, N, K), X.device, ws)
    _check("q4k_gemv", lib().q4k_gemv(_ptr(W), _ptr(_bits16(X)), _ptr(Y), M, N, K, _ptr(ws), ws.numel(),
                                      _stream(stream)))
    return Y


def q4k_gemv_q8(W, X, N: int, K: int, Y=None, ws=None, stream=None):
    """The Q8 activation lane of q4k_gemv (int8 activations per 256-wide column; accuracy traded)."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=X.device)
    ws = _scratch(q4k_workspace_bytes(OP_GEMV, M, N, K), X.device, ws)
    _check("q4k_gemv_q8", lib().q4k_gemv_q8(_ptr(W), _ptr(_bits16(X)), _ptr(Y), M, N, K, _ptr(ws), ws.numel(),
                                            _stream(stream)))
    return Y


def q5k_gemv(W, X, N: int, K: int, Y=None, ws=None, stream=None):
    """q4k_gemv over Q5_K weights W [N][K/256][176]."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=X.device)
    ws = _scratch(q4k_workspace_bytes(OP_GEMV, M, N, K), X.device, ws)
    _check("q5k_gemv", lib().q5k_gemv(_ptr(W), _ptr(_bits16(X)), _ptr(Y), M, N, K, _ptr(ws), ws.numel(),
                                      _stream(stream)))
    return Y


def q80_gemv(W, X, N: int, K: int, Y=None, ws=None, stream=None):
    """q4k_gemv over Q8_0 weights W [N][K/32][34]."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=X.device)
    ws = _scratch(q4k_workspace_bytes(OP_GEMV, M, N, K), X.device, ws)
    _check("q80_gemv", lib().q80_gemv(_ptr(W), _ptr(_bits16(X)), _ptr(Y), M, N, K, _ptr(ws), ws.numel(),
                                      _stream(stream)))
    return Y


def q6k_gemv(W, X, N: int, K: int, Y=None, ws=None, stream=None):
    """Decode GEMV over Q6_K weights [N][K/256][210]: Y[M][N] = X @ W^T."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=X.device)
    need = q4k_workspace_bytes(OP_GEMV, M, N, K)
    ws = _scratch(need, X.device, ws)
    _check("q6k_gemv", lib().q6k_gemv(_ptr(W), _ptr(_bits16(X)), _ptr(Y), M, N, K, _ptr(ws), ws.numel(),
                                      _stream(stream)))
    return Y


def q4k_repack(W, N: int, K: int, Wr=None, stream=None):
    """Repacked copy of Q4_K weights W [N][K/256][144] for q4k_gemv_repacked (uint8, flat)."""
    nb = lib().q4k_repacked_bytes(N, K)
    if nb <= 0:
        raise ValueError(f"q4k_repack: bad shape N={N} K={K}")
    if Wr is None:
        Wr = torch.empty(nb, dtype=torch.uint8, device=W.device)
    _check("q4k_repack", lib().q4k_repack(_ptr(W), N, K, _ptr(Wr), _stream(stream)))
    return Wr


def q4k_gemv_repacked(Wr, X, N: int, K: int, Y=None, ws=None, stream=None):
    """q4k_gemv on weights from q4k_repack (bit-identical results)."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=X.device)
    ws = _scratch(q4k_workspace_bytes(OP_GEMV, M, N, K), X.device, ws)
    _check("q4k_gemv_repacked", lib().q4k_gemv_repacked(_ptr(Wr), _ptr(_bits16(X)), _ptr(Y), M, N, K, _ptr(ws),
                                                        ws.numel(), _stream(stream)))
    return Y


def q4k_gemm(W, X, N: int, K: int, Y=None, stream=None):
    """Prefill GEMM Y[M][N] = X[M][K] @ W^T on tcgen05 tensor cores."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=X.device)
    _check("q4k_gemm", lib().q4k_gemm(_ptr(W), _ptr(_bits16(X)), _ptr(Y), M, N, K, None, 0,
                                      _stream(stream)))
    return Y


def bf16w_gemm(Wb, X, N: int, K: int, Y=None, stream=None):
    """Y = X @ Wb^T with bf16 weights Wb [N][K] (the unfused chain's GEMM)."""
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.float32, device=X.device)
    _check("bf16w_gemm", lib().bf16w_gemm(_ptr(_bits16(Wb)), _ptr(_bits16(X)), _ptr(Y), M, N, K, _stream(stream)))
    return Y


def q4k_workspace_bytes(op: int, M: int, N: int = 0, K: int = 0, E: int = 0, topk: int = 0) -> int:
    return lib().q4k_workspace_bytes(op, M, N, K, E, topk)


def moe_route_permute_hidden(X, W_router, topk: int, out=None, ws=None, stream=None):
    """Router logits X @ W_router^T (bf16 in, fp32 out) then moe_route_permute. Returns
    the routing dict plus "logits"."""
    M, H = X.shape
    E = W_router.shape[0]
    dev = X.device
    if out is None:
        rows = M * topk
        out = {"logits": torch.empty(M, E, dtype=torch.float32, device=dev),
               "topk_ids": torch.empty(M, topk, dtype=torch.int32, device=dev),
               "topk_w": torch.empty(M, topk, dtype=torch.float32, device=dev),
               "expert_offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
               "perm": torch.empty(rows, dtype=torch.int32, device=dev),
               "inv_perm": torch.empty(rows, dtype=torch.int32, device=dev),
               "row_token": torch.empty(rows, dtype=torch.int32, device=dev)}
    ws = _scratch(q4k_workspace_bytes(OP_ROUTE, M, 0, 0, E, topk), dev, ws)
    st = lib().moe_route_permute_hidden(
        _ptr(_bits16(X)), _ptr(_bits16(W_router)), M, E, H, topk, _ptr(out["logits"]), _ptr(out["topk_ids"]),
        _ptr(out["topk_w"]), _ptr(out["expert_offsets"]), _ptr(out["perm"]), _ptr(out["inv_perm"]),
        _ptr(out["row_token"]), _ptr(ws), ws.numel(), _stream(stream))
    _check("moe_route_permute_hidden", st)
    return out


def moe_route_permute(logits, topk: int, out=None, ws=None, stream=None):
    """Top-k routing + stable permutation by expert. Returns a dict of device tensors:
    topk_ids, topk_w, expert_offsets, perm, inv_perm, row_token."""
    M, E = logits.shape
    dev = logits.device
    if out is None:
        out = dict(
            topk_ids=torch.empty(M, topk, dtype=torch.int32, device=dev),
            topk_w=torch.empty(M, topk, dtype=torch.float32, device=dev),
            expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
            perm=torch.empty(M * topk, dtype=torch.int32, device=dev),
            inv_perm=torch.empty(M * topk, dtype=torch.int32, device=dev),
            row_token=torch.empty(M * topk, dtype=torch.int32, device=dev),
        )
    need = q4k_workspace_bytes(OP_ROUTE, M, E=E, topk=topk)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    st = lib().moe_route_permute(
        _ptr(logits), M, E, topk, _ptr(out["topk_ids"]), _ptr(out["topk_w"]),
        _ptr(out["expert_offsets"]), _ptr(out["perm"]), _ptr(out["inv_perm"]),
        _ptr(out["row_token"]), _ptr(ws), ws.numel(), _stream(stream))
    _check("moe_route_permute", st)
    return out


def moe_route_permute_noalloc(logits, topk: int, out=None, stream=None):
    """moe_route_permute with the library's fixed scratch instead of a workspace
    (for callers that cannot allocate device memory at call time; see q4k.h)."""
    M, E = logits.shape
    dev = logits.device
    if out is None:
        out = dict(
            topk_ids=torch.empty(M, topk, dtype=torch.int32, device=dev),
            topk_w=torch.empty(M, topk, dtype=torch.float32, device=dev),
            expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
            perm=torch.empty(M * topk, dtype=torch.int32, device=dev),
            inv_perm=torch.empty(M * topk, dtype=torch.int32, device=dev),
            row_token=torch.empty(M * topk, dtype=torch.int32, device=dev),
        )
    st = lib().moe_route_permute_noalloc(
        _ptr(logits), M, E, topk, _ptr(out["topk_ids"]), _ptr(out["topk_w"]),
        _ptr(out["expert_offsets"]), _ptr(out["perm"]), _ptr(out["inv_perm"]),
        _ptr(out["row_token"]), _stream(stream))
    _check("moe_route_permute_noalloc", st)
    return out


def moe_q4k_grouped(W_experts, E: int, N: int, K: int, A, expert_offsets, rows: int,
                    max_rows_hint: int, act: int = ACT_NONE, row_gather=None, out=None, ws=None,
                    stream=None):
    """Grouped expert matmul over rows sorted by expert (see include/q4k.h)."""
    if out is None:
        if act == ACT_SWIGLU:
            out = torch.empty(rows, N // 2, dtype=torch.bfloat16, device=A.device)
        else:
            out = torch.empty(rows, N, dtype=torch.float32, device=A.device)
    if ws is None and 0 < max_rows_hint <= 32:  # only the decode kernel uses scratch
        ws = _scratch(q4k_workspace_bytes(OP_GROUPED, rows, N, K, E), A.device)
    st = lib().moe_q4k_grouped(_ptr(W_experts), E, N, K, _ptr(_bits16(A)), _ptr(row_gather),
                               _ptr(expert_offsets), rows, max_rows_hint, act, _ptr(out), _ptr(ws),
                               0 if ws is None else ws.numel(), _stream(stream))
    _check("moe_q4k_grouped", st)
    return out


def moe_route_gate_up(logits, topk: int, W_gate_up, N: int, K: int, X, out=None, h=None, stream=None):
    """Routing + permutation and the grouped gate_up SwiGLU GEMV in one launch (decode,
    M <= 32; see include/q4k.h). Returns (routing dict as moe_route_permute's, h)."""
    M, E = logits.shape
    dev = logits.device
    if out is None:
        out = dict(
            topk_ids=torch.empty(M, topk, dtype=torch.int32, device=dev),
            topk_w=torch.empty(M, topk, dtype=torch.float32, device=dev),
            expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
            perm=torch.empty(M * topk, dtype=torch.int32, device=dev),
            inv_perm=torch.empty(M * topk, dtype=torch.int32, device=dev),
            row_token=torch.empty(M * topk, dtype=torch.int32, device=dev),
        )
    if h is None:
        h = torch.empty(M * topk, N // 2, dtype=torch.bfloat16, device=dev)
    st = lib().moe_route_gate_up(_ptr(logits), M, E, topk, _ptr(out["topk_ids"]), _ptr(out["topk_w"]),
                                 _ptr(out["expert_offsets"]), _ptr(out["perm"]), _ptr(out["inv_perm"]),
                                 _ptr(out["row_token"]), _ptr(W_gate_up), N, K, _ptr(_bits16(X)), _ptr(h),
                                 _stream(stream))
    _check("moe_route_gate_up", st)
    return out, h


def moe_combine(O, inv_perm, topk_w, M: int, topk: int, H: int, Y=None, stream=None):
    """y[t] = sum_j topk_w[t,j] * O[inv_perm[t*topk+j]]."""
    if Y is None:
        Y = torch.empty(M, H, dtype=torch.float32, device=O.device)
    _check("moe_combine", lib().moe_combine(_ptr(O), _ptr(inv_perm), _ptr(topk_w), M, topk, H,
                                            _ptr(Y), _stream(stream)))
    return Y


def moe_combine_residual(O, inv_perm, topk_w, residual, M: int, topk: int, H: int, Y=None, stream=None):
    """y[t] = residual[t] + sum_j topk_w[t,j] * O[inv_perm[t*topk+j]] (Y may be residual)."""
    if Y is None:
        Y = torch.empty(M, H, dtype=torch.float32, device=O.device)
    _check("moe_combine_residual", lib().moe_combine_residual(_ptr(O), _ptr(inv_perm), _ptr(topk_w), _ptr(residual),
                                                              M, topk, H, _ptr(Y), _stream(stream)))
    return Y


def q4k_last_device_status(stream=None) -> int:
    """Synchronise the stream, return and clear the device status word (0 = ok)."""
    return lib().q4k_last_device_status(_stream(stream))


def q4k_test_wait_fault(drop_stage: int = -1, wait_limit_ns: int = 0) -> None:
    """Test hook: make the weight producers skip stage `drop_stage` (-1: off) and set the
    bounded-wait limit (0: the 2 s default). Synchronous; see include/q4k.h."""
    _check("q4k_test_wait_fault", lib().q4k_test_wait_fault(int(drop_stage), int(wait_limit_ns)))
