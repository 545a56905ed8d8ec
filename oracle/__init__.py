"""CPU oracle for the CSA2 decode hot path.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers. The product library
never imports, links or runs anything here, and nothing here imports the
product package.

The arithmetic lives in ``csa2_oracle.c`` (exact E2M1/E4M3 conversion from the
format definitions, int64 indexer dot products, full-sort top-k, fp64
attention). This module marshals numpy arrays into it and strings the steps
together in the order the pages give them:

* "DeepSeek-V4.1-Flash: 890 Bytes Per Token, 437x Smaller KV Cache", section
  "CSA2: Sharing Main KV, Indexer K, and Top-K Indices Across Layers": Full
  layers score the context, build the candidate pool of up to 2,048 blocks of
  8 tokens and select a fresh top-512; Reindex layers rescore the pool with
  their own indexer Q; Reuse layers take the indices of the nearest
  Full/Reindex layer. Decoder groups: 1 Full + 3 Reuse, then four groups of
  1 Reindex + 3 Reuse. Encoder groups: three groups of 1 Full + 5 Reuse.
* "DeepSeek V4.1 Flash KV Cache: 890 Bytes per Token Explained", indexer and
  FP4 sections: pool of 2,048 blocks of 8 tokens, best 512 candidates per
  query, FP4 E2M1 values with one E4M3 scale per 16 channels.
* "890 bytes per token: how DeepSeek V4.1-Flash's KV cache works", mechanism 4:
  attention runs only over the selected candidates.

Parity pins: every function here is checked by ``tests/test_oracle_formats.py``,
``tests/test_oracle_selection.py`` and ``tests/test_oracle_attention.py``
against closed forms, the ml_dtypes format library, numpy/torch library
routines, brute force on tiny inputs and the invariants the pages fix;
``tests/test_oracle_mutants.py`` plants single mistakes in copies of the oracle
and checks that those pins catch each one.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libcsa2_oracle.so")
_LIB_OMP_PATH = os.path.join(_HERE, "_build", "libcsa2_oracle_omp.so")

# Constants the pages fix.
POOL_BLOCKS = 2048      # candidate pool: 2,048 blocks ...
BLOCK_TOKENS = 8        # ... of 8 tokens (16,384 positions)
TOPK = 512              # each query keeps its best 512
N_WIN = 128             # sliding window: the last 128 tokens
FP4_GROUP = 16          # one E4M3 scale per 16 channels
MX_GROUP = 32           # MXFP4 variant: one E8M0 scale per 32 channels

FULL, REINDEX, REUSE = "full", "reindex", "reuse"


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math: IEEE fp32 division
    and conversion must be exact). Returns the path of the shared library.
    CSA2_ORACLE_LIB names a library to load instead of the plain build (the
    mutation tests build copies of this source with one planted mistake each).
    openmp=True builds the timing variant (-fopenmp): the same source, its
    independent outer loops shared among threads, results identical."""
    override = os.environ.get("CSA2_ORACLE_LIB")
    if override and not openmp:
        return override
    path = _LIB_OMP_PATH if openmp else _LIB_PATH
    if force or not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(path), exist_ok=True)
        tmp = path + f".tmp{os.getpid()}"
        flags = ["-fopenmp"] if openmp else []
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
                               *flags, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, path)
    return path


_lib = None
_use_openmp = False


def use_openmp(on: bool = True) -> int:
    """Route every oracle call through the OpenMP timing build (on=True) or the
    plain build. Returns the number of threads the loaded build uses."""
    global _lib, _use_openmp
    if on != _use_openmp:
        _use_openmp = on
        _lib = None
    return num_threads()


def num_threads() -> int:
    """Threads the loaded oracle build shares its outer loops among (1 for the
    plain build)."""
    return int(_L().orc_num_threads())


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build(openmp=_use_openmp))
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_num_threads.argtypes = []
        c_i64, c_int, c_dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        P = ctypes.c_void_p
        lib.orc_e4m3_value.restype = c_dbl
        lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
        lib.orc_e2m1_value.restype = c_dbl
        lib.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        lib.orc_e2m1_encode.restype = ctypes.c_uint8
        lib.orc_e2m1_encode.argtypes = [ctypes.c_float]
        lib.orc_e4m3_encode_n.restype = None
        lib.orc_e4m3_encode_n.argtypes = [P, c_i64, P]
        lib.orc_e2m1_encode_n.restype = None
        lib.orc_e2m1_encode_n.argtypes = [P, c_i64, P]
        lib.orc_fp4_quantize.restype = None
        lib.orc_fp4_quantize.argtypes = [P, c_i64, c_int, P, P]
        lib.orc_fp4_dequantize.restype = None
        lib.orc_fp4_dequantize.argtypes = [P, P, c_i64, c_int, P]
        lib.orc_e8m0_value.restype = c_dbl
        lib.orc_e8m0_value.argtypes = [ctypes.c_uint8]
        lib.orc_mx_shared_exp.restype = c_int
        lib.orc_mx_shared_exp.argtypes = [c_dbl]
        lib.orc_mxfp4_quantize.restype = None
        lib.orc_mxfp4_quantize.argtypes = [P, c_i64, c_int, P, P]
        lib.orc_mxfp4_dequantize.restype = None
        lib.orc_mxfp4_dequantize.argtypes = [P, P, c_i64, c_int, P]
        lib.orc_index_dots.restype = None
        lib.orc_index_dots.argtypes = [P, P, c_i64, c_int, P]
        lib.orc_index_scores.restype = c_int
        lib.orc_index_scores.argtypes = [P, P, P, c_i64, c_int, P]
        lib.orc_block_max.restype = None
        lib.orc_block_max.argtypes = [P, c_i64, P]
        lib.orc_topk.restype = c_i64
        lib.orc_topk.argtypes = [P, P, c_i64, c_i64, P]
        lib.orc_attention.restype = None
        lib.orc_attention.argtypes = [P, c_int, c_int, P, c_i64, c_dbl, P]
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


# ----------------------------------------------------------------------------
# Number formats
# ----------------------------------------------------------------------------
def e4m3_value(code: int) -> float:
    return _L().orc_e4m3_value(int(code))


def e4m3_encode(x: float) -> int:
    return int(_L().orc_e4m3_encode(float(x)))


def e2m1_value(code: int) -> float:
    return _L().orc_e2m1_value(int(code))


def e2m1_encode(v: float) -> int:
    return int(_L().orc_e2m1_encode(float(v)))


def e2m1_encode_array(v: np.ndarray) -> np.ndarray:
    """Element-wise E2M1 encode of an fp32 array."""
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.empty(v.size, dtype=np.uint8)
    _L().orc_e2m1_encode_n(_p(v), v.size, _p(out))
    return out


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    """Element-wise E4M3 encode of an fp32 array."""
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.empty(v.size, dtype=np.uint8)
    _L().orc_e4m3_encode_n(_p(v), v.size, _p(out))
    return out


# ----------------------------------------------------------------------------
# FP4 main KV
# ----------------------------------------------------------------------------
def fp4_quantize(x_bf16: np.ndarray):
    """x_bf16: uint16 bf16 bit patterns [..., C]. Returns (packed uint8 [..., C/2],
    scales uint8 E4M3 [..., C/16])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    C = x.shape[-1]
    assert C % FP4_GROUP == 0
    rows = x.size // C
    packed = np.empty(x.shape[:-1] + (C // 2,), dtype=np.uint8)
    sf = np.empty(x.shape[:-1] + (C // FP4_GROUP,), dtype=np.uint8)
    _L().orc_fp4_quantize(_p(x), rows, C, _p(packed), _p(sf))
    return packed, sf


def fp4_dequantize(packed: np.ndarray, sf: np.ndarray) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    C = packed.shape[-1] * 2
    rows = packed.size // (C // 2)
    out = np.empty(packed.shape[:-1] + (C,), dtype=np.float64)
    _L().orc_fp4_dequantize(_p(packed), _p(sf), rows, C, _p(out))
    return out


def e8m0_value(code: int) -> float:
    return _L().orc_e8m0_value(int(code))


def mx_shared_exp(amax: float) -> int:
    return int(_L().orc_mx_shared_exp(float(amax)))


def mxfp4_quantize(x_bf16: np.ndarray):
    """MXFP4 variant. x_bf16: uint16 bf16 bit patterns [..., C], C % 32 == 0.
    Returns (packed uint8 [..., C/2], scales uint8 E8M0 [..., C/32])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    C = x.shape[-1]
    assert C % MX_GROUP == 0
    rows = x.size // C
    packed = np.empty(x.shape[:-1] + (C // 2,), dtype=np.uint8)
    sf = np.empty(x.shape[:-1] + (C // MX_GROUP,), dtype=np.uint8)
    _L().orc_mxfp4_quantize(_p(x), rows, C, _p(packed), _p(sf))
    return packed, sf


def mxfp4_dequantize(packed: np.ndarray, sf: np.ndarray) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    C = packed.shape[-1] * 2
    rows = packed.size // (C // 2)
    out = np.empty(packed.shape[:-1] + (C,), dtype=np.float64)
    _L().orc_mxfp4_dequantize(_p(packed), _p(sf), rows, C, _p(out))
    return out


def fp4_row_bytes(C: int) -> int:
    """Bytes per token of the FP4 main KV: C/2 element bytes + C/16 scale bytes."""
    return C // 2 + C // FP4_GROUP


# ----------------------------------------------------------------------------
# Indexer and selection
# ----------------------------------------------------------------------------
def index_dots(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """Exact integer dot products S[t] = sum q * k[t] (int64). q: [H, D] int8,
    k: [n, H, D] int8."""
    q = np.ascontiguousarray(q, dtype=np.int8).ravel()
    HD = q.size
    k = np.ascontiguousarray(k, dtype=np.int8).reshape(-1, HD)
    S = np.empty(k.shape[0], dtype=np.int64)
    _L().orc_index_dots(_p(q), _p(k), k.shape[0], HD, _p(S))
    return S


def index_scores(q: np.ndarray, k: np.ndarray, kscale: np.ndarray) -> np.ndarray:
    """fp32 scores score[t] = fp32(S[t]) * kscale[t]."""
    q = np.ascontiguousarray(q, dtype=np.int8).ravel()
    HD = q.size
    k = np.ascontiguousarray(k, dtype=np.int8).reshape(-1, HD)
    ks = np.ascontiguousarray(kscale, dtype=np.float32).ravel()
    assert ks.size == k.shape[0]
    out = np.empty(k.shape[0], dtype=np.float32)
    rc = _L().orc_index_scores(_p(q), _p(k), _p(ks), k.shape[0], HD, _p(out))
    if rc != 0:
        raise OverflowError("indexer dot product outside the int32 range")
    return out


def block_scores(score: np.ndarray, n_visible: int) -> np.ndarray:
    s = np.ascontiguousarray(score, dtype=np.float32)
    assert s.size >= n_visible
    nblk = (n_visible + BLOCK_TOKENS - 1) // BLOCK_TOKENS
    blk = np.empty(nblk, dtype=np.float32)
    if n_visible > 0:
        _L().orc_block_max(_p(s), n_visible, _p(blk))
    return blk


def topk(score: np.ndarray, pos: np.ndarray, k: int) -> np.ndarray:
    """Top-k of candidates (score desc, pos asc), ascending positions, -1 padded
    to k entries (int64)."""
    s = np.ascontiguousarray(score, dtype=np.float32).ravel()
    p = np.ascontiguousarray(pos, dtype=np.int64).ravel()
    assert s.size == p.size
    out = np.empty(k, dtype=np.int64)
    _L().orc_topk(_p(s), _p(p), s.size, k, _p(out))
    return out


def pooled_positions(pool: np.ndarray, n_visible: int) -> np.ndarray:
    """Token positions covered by the pool's blocks (in pool order), limited to
    the visible context."""
    blocks = pool[pool >= 0].astype(np.int64)
    pos = (blocks[:, None] * BLOCK_TOKENS + np.arange(BLOCK_TOKENS)[None, :]).ravel()
    return pos[pos < n_visible]


def full_layer(q_idx, k_idx, k_scale, n_visible, pool_blocks=POOL_BLOCKS, k_top=TOPK):
    """Full-mode indexing for one query that sees positions [0, n_visible).

    1. score every visible token with the layer's indexer Q;
    2. block score = max over each block of 8;
    3. pool = the best min(pool_blocks, nblk) blocks;
    4. top-k = the best k_top tokens among the pooled positions.
    Returns dict(tok_score, blk_score, pool (int64 [pool_blocks], ascending,
    -1 padded), top (int64 [k_top], ascending, -1 padded))."""
    tok = index_scores(q_idx, k_idx[:n_visible], k_scale[:n_visible])
    blk = block_scores(tok, n_visible)
    pool = topk(blk, np.arange(blk.size, dtype=np.int64), pool_blocks)
    ppos = pooled_positions(pool, n_visible)
    top = topk(tok[ppos], ppos, k_top)
    return dict(tok_score=tok, blk_score=blk, pool=pool, top=top)


def reindex_layer(q_idx, k_idx, k_scale, pool, n_visible, k_top=TOPK):
    """Reindex-mode indexing: rescore the pooled positions with this layer's
    own indexer Q and keep the best k_top. Returns (top, pooled positions,
    their scores)."""
    ppos = pooled_positions(np.asarray(pool), n_visible)
    sc = index_scores(q_idx, k_idx[ppos], k_scale[ppos])
    return topk(sc, ppos, k_top), ppos, sc


# ----------------------------------------------------------------------------
# Attention
# ----------------------------------------------------------------------------
def bf16_to_f64(x_bf16: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(x_bf16, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def attention(q_bf16: np.ndarray, kv: np.ndarray, scale: float) -> np.ndarray:
    """q_bf16: [Hq, C] uint16; kv: [n, C] float64 (K = V). Returns [Hq, C] fp64."""
    q = np.ascontiguousarray(q_bf16, dtype=np.uint16)
    Hq, C = q.shape
    kv = np.ascontiguousarray(kv, dtype=np.float64).reshape(-1, C)
    out = np.empty((Hq, C), dtype=np.float64)
    _L().orc_attention(_p(q), Hq, C, _p(kv), kv.shape[0], float(scale), _p(out))
    return out


def window_rows(q_pos: int, swa_pos0: int, swa_rows: int, n_win: int = N_WIN):
    """Rows of the per-layer SWA tensor that a query at position q_pos sees:
    positions max(0, q_pos - n_win + 1) .. q_pos, where row r holds position
    swa_pos0 + r."""
    lo = max(0, q_pos - n_win + 1, swa_pos0)
    hi = min(q_pos, swa_pos0 + swa_rows - 1)
    return np.arange(lo - swa_pos0, hi - swa_pos0 + 1, dtype=np.int64)


def sparse_attention(q_bf16, kv_bf16_rows_of, top, swa_bf16, q_pos, swa_pos0, scale,
                     n_win=N_WIN, kv_format="nvfp4"):
    """One query (all heads) attends the selected main-KV tokens (quantized to
    FP4 by this oracle, then dequantized) followed by its sliding-window rows.

    kv_bf16_rows_of(positions) -> uint16 bf16 rows [len, C] of the main KV
    before quantization; swa_bf16: [swa_rows, C] uint16 of this layer;
    kv_format: "nvfp4" (E4M3 per 16 channels) or "mxfp4" (E8M0 per 32)."""
    sel = np.asarray(top, dtype=np.int64)
    sel = sel[sel >= 0]
    if kv_format == "mxfp4":
        packed, sf = mxfp4_quantize(kv_bf16_rows_of(sel))
        main = mxfp4_dequantize(packed, sf)
    else:
        packed, sf = fp4_quantize(kv_bf16_rows_of(sel))
        main = fp4_dequantize(packed, sf)
    rows = window_rows(int(q_pos), int(swa_pos0), swa_bf16.shape[0], n_win)
    swa = bf16_to_f64(np.asarray(swa_bf16)[rows])
    return attention(q_bf16, np.concatenate([main, swa], axis=0), scale)


# ----------------------------------------------------------------------------
# Layer schedules
# ----------------------------------------------------------------------------
def decoder_schedule():
    """20 decoder layers in five groups of 4: 1 Full + 3 Reuse, then four
    groups of 1 Reindex + 3 Reuse."""
    return [FULL, REUSE, REUSE, REUSE] + [REINDEX, REUSE, REUSE, REUSE] * 4


def encoder_schedule():
    """18 CSA2 encoder layers in three groups of 6: 1 Full + 5 Reuse."""
    return [FULL] + [REUSE] * 5 + [FULL] + [REUSE] * 5 + [FULL] + [REUSE] * 5


def stack_indices(modes, q_idx_of, k_idx, k_scale, n_visible):
    """Run the indexing side of a layer stack for one query.

    modes: list of FULL/REINDEX/REUSE; q_idx_of(l): indexer Q of layer l (only
    asked for Full and Reindex layers). The pool used by Reindex layers is the
    one built by the most recent Full layer. Returns (list of top-k index
    arrays, one per layer; dict of per-layer pools for Full layers)."""
    tops, pools = [], {}
    pool, top = None, None
    for l, m in enumerate(modes):
        if m == FULL:
            r = full_layer(q_idx_of(l), k_idx, k_scale, n_visible)
            pool, top = r["pool"], r["top"]
            pools[l] = pool
        elif m == REINDEX:
            if pool is None:
                raise ValueError("a Reindex layer needs a preceding Full layer's pool")
            top, _, _ = reindex_layer(q_idx_of(l), k_idx, k_scale, pool, n_visible)
        elif m == REUSE:
            if top is None:
                raise ValueError("a Reuse layer needs a preceding Full or Reindex layer")
        else:
            raise ValueError(m)
        tops.append(top)
    return tops, pools
