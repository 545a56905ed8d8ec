"""Thin ctypes binding of libcsa2 (declared in include/csa2.h).

Argument marshalling only: each function checks dtypes/devices/shapes of the
torch tensors it is given, passes raw device pointers and the current CUDA
stream to the C entry point of the same name, and raises ``Csa2Error`` on a
non-zero status. Every step of the computation runs in libcsa2's kernels.
Importing this module loads the library and raises if it is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcsa2.so")

POOL_BLOCKS = 2048
BLOCK_TOKENS = 8
TOPK = 512
N_WIN = 128
# Rows of at most this many candidates are selected by one single-CTA kernel
# inside the decode step; longer rows take a compaction and a finishing kernel.
TOPK_SHORT_ROW = 65536
# csa2_full_select holds a row of block scores (and of pooled token scores) in
# shared memory: at most this many of each.
FULL_SELECT_MAX = 16384
# The decode stack launches the attention of a layer group (a Full or Reindex
# layer and the Reuse layers after it, up to ATTN_GROUP_MAX layers) as one
# kernel when the tensor-core cluster kernel takes the shape (512 channels, 64
# heads, fewer than ATTN_ROWS_MIN query rows); otherwise one kernel per layer.
ATTN_GROUP_MAX = 8
ATTN_ROWS_MIN = 64
MODE_FULL, MODE_REINDEX, MODE_REUSE = 0, 1, 2


class Csa2Error(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} failed with status {status}: {text}")
        self.status = status


if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libcsa2.so is not built ({_LIB_PATH}); build it with "
                      "`python -m sparse_attention_fp4_kv_b200.build`")

lib = ctypes.CDLL(_LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float


class csa2_layer(ctypes.Structure):
    _fields_ = [("mode", _I), ("q_idx", _P), ("q", _P), ("swa", _P), ("out", _P), ("topk", _P)]


_SIGS = {
    "csa2_status_string": (ctypes.c_char_p, [_I]),
    "csa2_abi_version": (_I, []),
    "csa2_device_status": (_I, [_I]),
    "csa2_selftest_wait_timeout": (_I, [_I, _P]),
    "csa2_kv_append_fp4": (_I, [_P, _I, _I, _I, _P, _I64, _P, _P, _P]),
    "csa2_kv_append_mxfp4": (_I, [_P, _I, _I, _I, _P, _I64, _P, _P, _P]),
    "csa2_index_full": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _P, _P, _P, _P]),
    "csa2_topk_workspace_size": (_SZ, [_I, _I64, _I]),
    "csa2_topk": (_I, [_P, _P, _P, _I, _I64, _I, _P, _P, _SZ, _P]),
    "csa2_pool_gather": (_I, [_P, _P, _P, _P, _I, _I, _I, _I64, _P, _P, _P]),
    "csa2_full_select": (_I, [_P, _P, _P, _P, _P, _I, _I, _I64, _I, _I, _P, _P, _P]),
    "csa2_index_reindex": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I64, _I, _P, _P, _P]),
    "csa2_sparse_attn_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "csa2_sparse_attn_decode": (_I, [_P, _P, _P, _I64, _P, _I, _P, _P, _I, _P, _I, _I, _I, _I,
                                     _I, _F, _P, _P, _SZ, _P]),
    "csa2_sparse_attn_decode_mxfp4": (_I, [_P, _P, _P, _I64, _P, _I, _P, _P, _I, _P, _I, _I, _I,
                                           _I, _I, _F, _P, _P, _SZ, _P]),
    "csa2_decode_stack_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I64]),
    "csa2_decode_stack": (_I, [ctypes.POINTER(csa2_layer), _I, _P, _P, _P, _P, _P, _I64, _P, _P,
                               _I, _I, _I, _I, _I, _I, _F, _P, _I, _P, _P, _SZ, _P]),
    "csa2_decode_stack_noalloc": (_I, [ctypes.POINTER(csa2_layer), _I, _P, _P, _P, _P, _P, _I64,
                                       _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _I, _P]),
    "csa2_attn_resident_clusters": (_I, [_I]),
    "csa2_workspace_status": (_I, [_P, _I, _P]),
    "csa2_selftest_workspace_timeout": (_I, [_I, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def exported_symbols() -> List[str]:
    return list(_SIGS)


def status_string(status: int) -> str:
    return lib.csa2_status_string(status).decode()


def _check(name: str, st: int):
    if st != 0:
        raise Csa2Error(name, st, status_string(st))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libcsa2 must be contiguous")
    return _P(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return _P(stream.cuda_stream)


def _want(t: torch.Tensor, dtype, name: str):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


# ----------------------------------------------------------------------------- calls
def csa2_kv_append_fp4(kv_bf16: torch.Tensor, start_pos: torch.Tensor, kv_fp4: torch.Tensor,
                       kv_sf: torch.Tensor, stream=None, mx: bool = False) -> None:
    """kv_bf16 [B][n_new][C] bf16; start_pos [B] int64; kv_fp4 [B][cap][C/2] uint8;
    kv_sf [B][cap][C/16] uint8 (E4M3), or with mx the MXFP4 variant's
    [B][cap][C/32] E8M0 (csa2_kv_append_mxfp4)."""
    _want(kv_bf16, torch.bfloat16, "kv_bf16")
    _want(start_pos, torch.int64, "start_pos")
    _want(kv_fp4, torch.uint8, "kv_fp4")
    _want(kv_sf, torch.uint8, "kv_sf")
    B, n, C = kv_bf16.shape
    cap = kv_fp4.shape[1]
    assert kv_fp4.shape == (B, cap, C // 2) and kv_sf.shape == (B, cap, C // (32 if mx else 16))
    name = "csa2_kv_append_mxfp4" if mx else "csa2_kv_append_fp4"
    _check(name, getattr(lib, name)(
        _ptr(kv_bf16), B, n, C, _ptr(start_pos), cap, _ptr(kv_fp4), _ptr(kv_sf), _stream(stream)))


def csa2_index_full(q_idx, k_idx, k_scale, ctx_len, blk_score, tok_score=None, n_blk=None,
                    q_pos=None, stream=None) -> None:
    """q_idx [B][Nq][H][D] int8; k_idx [B][cap][H][D] int8; k_scale [B][cap] fp32;
    ctx_len [B] int64; blk_score [B][Nq][ceil(cap/8)] fp32; tok_score [B][Nq][cap]
    fp32 or None; n_blk [B][Nq] int32 or None; q_pos [B][Nq] int64 or None."""
    _want(q_idx, torch.int8, "q_idx")
    _want(k_idx, torch.int8, "k_idx")
    B, Nq, H, D = q_idx.shape
    cap = k_idx.shape[1]
    assert k_idx.shape == (B, cap, H, D) and k_scale.shape == (B, cap)
    assert blk_score.shape == (B, Nq, (cap + 7) // 8)
    if tok_score is not None:
        assert tok_score.shape == (B, Nq, cap)
    _check("csa2_index_full", lib.csa2_index_full(
        _ptr(q_idx), _ptr(k_idx), _ptr(k_scale), _ptr(ctx_len), _ptr(q_pos), B, Nq, H, D, cap,
        _ptr(tok_score), _ptr(blk_score), _ptr(n_blk), _stream(stream)))


def csa2_topk(score, k: int, out, cand_pos=None, n_valid=None, ws=None, stream=None) -> None:
    """score [R][n] fp32; out [R][k] int32; cand_pos [R][n] int32 or None;
    n_valid [R] int32 or None."""
    _want(score, torch.float32, "score")
    _want(out, torch.int32, "out")
    R, n = score.shape
    assert out.shape == (R, k)
    need = lib.csa2_topk_workspace_size(R, n, k)
    wsb = 0
    if need:
        if ws is None:
            raise ValueError(f"csa2_topk needs {need} workspace bytes")
        wsb = ws.numel() * ws.element_size()
    _check("csa2_topk", lib.csa2_topk(_ptr(score), _ptr(cand_pos), _ptr(n_valid), R, n, k,
                                      _ptr(out), _ptr(ws) if need else None, wsb, _stream(stream)))


def csa2_pool_gather(tok_score, pool, ctx_len, pool_score, pool_pos, q_pos=None,
                     stream=None) -> None:
    """tok_score [B][Nq][cap] fp32; pool [B][Nq][P] int32; pool_score/pool_pos [B][Nq][8P]."""
    B, Nq, cap = tok_score.shape
    P = pool.shape[2]
    assert pool_score.shape == (B, Nq, 8 * P) and pool_pos.shape == (B, Nq, 8 * P)
    _check("csa2_pool_gather", lib.csa2_pool_gather(
        _ptr(tok_score), _ptr(pool), _ptr(ctx_len), _ptr(q_pos), B, Nq, P, cap,
        _ptr(pool_score), _ptr(pool_pos), _stream(stream)))


def workspace_status(ws: torch.Tensor, clear: bool = False, stream=None) -> int:
    """Status of the call whose workspace is ws (its error word): 0, or
    CSA2_ERR_DEVICE_TIMEOUT (-7) if a kernel of that call gave up a wait."""
    return lib.csa2_workspace_status(_ptr(ws), int(clear), _stream(stream))


def attn_resident_clusters(heads_per_cluster: int) -> int:
    """8-CTA attention clusters that fit on the current device at once with
    heads_per_cluster (16, 32 or 64) query heads each."""
    return lib.csa2_attn_resident_clusters(heads_per_cluster)


def device_status(clear: bool = False) -> int:
    """CSA2_OK, or CSA2_ERR_DEVICE_TIMEOUT if a kernel gave up a bounded wait
    (synchronizes the device; clear resets the flags)."""
    return lib.csa2_device_status(1 if clear else 0)


def selftest_wait_timeout(limit_us: int = 1000, stream=None) -> None:
    """Launch one CTA whose wait nothing completes; it records a timeout."""
    _check("csa2_selftest_wait_timeout", lib.csa2_selftest_wait_timeout(limit_us, _stream(stream)))


def csa2_full_select(blk_score, n_blk, tok_score, ctx_len, pool, top, q_pos=None,
                     stream=None) -> None:
    """blk_score [B][Nq][ceil(cap/8)] fp32; n_blk [B][Nq] int32; tok_score [B][Nq][cap] fp32;
    pool [B][Nq][P] int32; top [B][Nq][K] int32."""
    _want(blk_score, torch.float32, "blk_score")
    _want(tok_score, torch.float32, "tok_score")
    _want(n_blk, torch.int32, "n_blk")
    B, Nq, cap = tok_score.shape
    P, K = pool.shape[2], top.shape[2]
    assert blk_score.shape == (B, Nq, (cap + 7) // 8) and n_blk.shape == (B, Nq)
    assert pool.shape[:2] == (B, Nq) and top.shape[:2] == (B, Nq)
    _check("csa2_full_select", lib.csa2_full_select(
        _ptr(blk_score), _ptr(n_blk), _ptr(tok_score), _ptr(ctx_len), _ptr(q_pos), B, Nq, cap, P, K,
        _ptr(pool), _ptr(top), _stream(stream)))


def csa2_index_reindex(q_idx, k_idx, k_scale, pool, ctx_len, pool_score, pool_pos, q_pos=None,
                       stream=None) -> None:
    """q_idx [B][Nq][H][D] int8; pool [B][Nq][P] int32; pool_score/pool_pos [B][Nq][8P]."""
    _want(q_idx, torch.int8, "q_idx")
    B, Nq, H, D = q_idx.shape
    cap = k_idx.shape[1]
    P = pool.shape[2]
    assert pool_score.shape == (B, Nq, 8 * P) and pool_pos.shape == (B, Nq, 8 * P)
    _check("csa2_index_reindex", lib.csa2_index_reindex(
        _ptr(q_idx), _ptr(k_idx), _ptr(k_scale), _ptr(pool), _ptr(ctx_len), _ptr(q_pos), B, Nq,
        H, D, cap, P, _ptr(pool_score), _ptr(pool_pos), _stream(stream)))


def sparse_attn_workspace_size(B, Nq, Hq, C, K, n_win=N_WIN) -> int:
    return lib.csa2_sparse_attn_workspace_size(B, Nq, Hq, C, K, n_win)


def csa2_sparse_attn_decode(q_bf16, kv_fp4, kv_sf, topk, swa_bf16, swa_pos0, out, softmax_scale,
                            q_pos=None, n_win=N_WIN, ws=None, stream=None, mx: bool = False) -> None:
    """q_bf16 [B][Nq][Hq][C]; topk [B][Nq][K] int32; swa_bf16 [B][rows][C] bf16;
    swa_pos0 [B] int64; out [B][Nq][Hq][C] fp32; with mx the cache is the MXFP4
    variant (csa2_sparse_attn_decode_mxfp4)."""
    _want(q_bf16, torch.bfloat16, "q_bf16")
    _want(out, torch.float32, "out")
    B, Nq, Hq, C = q_bf16.shape
    cap = kv_fp4.shape[1]
    K = topk.shape[2]
    rows = swa_bf16.shape[1] if swa_bf16 is not None else 0
    need = sparse_attn_workspace_size(B, Nq, Hq, C, K, n_win)
    if need and ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=q_bf16.device)
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    name = "csa2_sparse_attn_decode_mxfp4" if mx else "csa2_sparse_attn_decode"
    _check(name, getattr(lib, name)(
        _ptr(q_bf16), _ptr(kv_fp4), _ptr(kv_sf), cap, _ptr(topk), K, _ptr(swa_bf16),
        _ptr(swa_pos0), rows, _ptr(q_pos), n_win, B, Nq, Hq, C, float(softmax_scale), _ptr(out),
        _ptr(ws), wsb, _stream(stream)))


def decode_stack_workspace_size(B, Hq, C, H, D, cap) -> int:
    return lib.csa2_decode_stack_workspace_size(B, Hq, C, H, D, cap)


class DecodeStack:
    """Pre-marshalled arguments of csa2_decode_stack for a fixed set of device
    buffers, so that a decode step is one C call."""

    def __init__(self, modes: Sequence[int], q_idx: Sequence[Optional[torch.Tensor]],
                 q: Sequence[torch.Tensor], swa: Sequence[torch.Tensor],
                 out: Sequence[torch.Tensor], topk: Sequence[Optional[torch.Tensor]],
                 k_idx: torch.Tensor, k_scale: torch.Tensor, kv_fp4: torch.Tensor,
                 kv_sf: torch.Tensor, ctx_len: torch.Tensor, swa_pos0: torch.Tensor,
                 pool: torch.Tensor, softmax_scale: float, ws: Optional[torch.Tensor] = None,
                 kv_new: Optional[torch.Tensor] = None, pool_ready: bool = False):
        n = len(modes)
        self.layers = (csa2_layer * n)()
        self._keep = [q_idx, q, swa, out, topk, k_idx, k_scale, kv_fp4, kv_sf, ctx_len, swa_pos0,
                      pool, kv_new]
        for l in range(n):
            self.layers[l] = csa2_layer(int(modes[l]), _ptr(q_idx[l]), _ptr(q[l]), _ptr(swa[l]),
                                        _ptr(out[l]), _ptr(topk[l]))
        B, cap, H, D = k_idx.shape
        Hq, C = q[0].shape[-2], q[0].shape[-1]
        self.dims = (B, Hq, C, H, D, cap)
        need = decode_stack_workspace_size(B, Hq, C, H, D, cap)
        if ws is None:
            ws = torch.empty(need, dtype=torch.uint8, device=k_idx.device)
        assert ws.numel() >= need
        self.ws = ws
        self.args = (self.layers, n, _ptr(kv_new), _ptr(k_idx), _ptr(k_scale), _ptr(kv_fp4), _ptr(kv_sf), cap,
                     _ptr(ctx_len), _ptr(swa_pos0), swa[0].shape[1], B, Hq, C, H, D,
                     float(softmax_scale), _ptr(pool), int(bool(pool_ready)))
        self.ws_args = (_ptr(ws), ws.numel())

    def call_noalloc(self, stream=None) -> int:
        """The same decode step through csa2_decode_stack_noalloc, which uses
        the library's own scratch array instead of self.ws (for callers that
        cannot allocate). Returns the C status code."""
        return lib.csa2_decode_stack_noalloc(*self.args, _stream(stream))

    def __call__(self, stream=None, scan_events=None) -> None:
        """One decode step. scan_events: optional (start, end) torch.cuda.Event
        pair recorded around the first Full layer's indexer scan."""
        ev = None
        if scan_events is not None:
            ev = (_P * 2)(_P(scan_events[0].cuda_event), _P(scan_events[1].cuda_event))
        _check("csa2_decode_stack", lib.csa2_decode_stack(*self.args, ev, *self.ws_args,
                                                          _stream(stream)))
