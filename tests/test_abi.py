"""CPU tests of the C ABI: the library loads, exports every function that
include/csa2.h declares, and rejects bad arguments on the host with the
documented status codes (no kernel is launched on those paths, so no GPU is
needed)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")
LIB = os.path.join(ROOT, "sparse_attention_fp4_kv_b200", "libcsa2.so")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_fp4_kv_b200 import build
    build.build()
    return ctypes.CDLL(LIB)


def test_every_declared_function_is_exported(lib):
    names = _declared()
    assert len(names) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (csa2_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(lib, n)


def test_binding_covers_the_header():
    from sparse_attention_fp4_kv_b200 import binding
    assert set(binding.exported_symbols()) == set(_declared())
    assert binding.lib.csa2_abi_version() == 1


def test_status_strings():
    from sparse_attention_fp4_kv_b200 import binding as B
    for st in (0, -1, -2, -3, -4, -5, -6, -7):
        assert B.status_string(st) and B.status_string(st) != "unknown status"
    assert B.status_string(-99) == "unknown status"


def test_host_validation_codes():
    from sparse_attention_fp4_kv_b200 import binding as B
    L = B.lib
    P = ctypes.c_void_p
    good = P(4096)        # any 16-byte aligned non-null value; never dereferenced
    odd = P(4096 + 8)
    # NULL pointers
    assert L.csa2_kv_append_fp4(None, 1, 1, 512, good, 10, good, good, None) == -1
    assert L.csa2_index_full(None, good, good, good, None, 1, 1, 16, 128, 10, None, good, None,
                             None) == -1
    assert L.csa2_topk(None, None, None, 1, 10, 5, good, None, 0, None) == -1
    # shapes
    assert L.csa2_kv_append_fp4(good, 1, 1, 40, good, 10, good, good, None) == -2
    assert L.csa2_index_full(good, good, good, good, None, 1, 1, 3, 5, 10, None, good, None,
                             None) == -2
    assert L.csa2_topk(good, None, None, 1, 10, 5000, good, None, 0, None) == -2
    assert L.csa2_topk(good, None, None, 1, 0, 5, good, None, 0, None) == -2
    assert L.csa2_sparse_attn_decode(good, good, good, 10, good, 512, good, good, 128, None, 128,
                                     1, 1, 64, 48, ctypes.c_float(0.1), good, None, 0,
                                     None) == -2
    # alignment
    assert L.csa2_kv_append_fp4(odd, 1, 1, 512, good, 10, good, good, None) == -3
    need = L.csa2_sparse_attn_workspace_size(1, 1, 64, 512, 512, 128)
    assert need > 0
    assert L.csa2_sparse_attn_decode(good, good, good, 1000, good, 512, good, good, 128, None, 128,
                                     1, 1, 64, 512, ctypes.c_float(0.04), good, odd, need + 64,
                                     None) == -3
    assert L.csa2_index_full(odd, good, good, good, None, 1, 1, 16, 128, 10, None, good, None,
                             None) == -3
    # empty work is a no-op
    assert L.csa2_kv_append_fp4(good, 0, 1, 512, good, 10, good, good, None) == 0
    assert L.csa2_index_full(good, good, good, good, None, 0, 1, 16, 128, 10, None, good, None,
                             None) == 0
    assert L.csa2_topk(good, None, None, 0, 10, 5, good, None, 0, None) == 0
    # the wait-timeout self-test checks its bound on the host
    assert L.csa2_selftest_wait_timeout(0, None) == -4
    assert L.csa2_selftest_wait_timeout(2000000, None) == -4
    # fused Full-layer selection: NULL, the shared-memory row limits, empty work
    fs = L.csa2_full_select
    assert fs(None, good, good, good, None, 1, 1, 4096, 2048, 512, good, good, None) == -1
    assert fs(good, good, good, good, None, 1, 1, 8 * 16384 + 8, 2048, 512, good, good, None) == -2
    assert fs(good, good, good, good, None, 1, 1, 4096, 4096, 512, good, good, None) == -2
    assert fs(good, good, good, good, None, 1, 1, 4096, 64, 600, good, good, None) == -2
    assert fs(good, good, good, good, None, 1, 1, 4096, 2048, 0, good, good, None) == -2
    assert fs(good, good, good, good, None, 0, 1, 4096, 2048, 512, good, good, None) == 0


def test_decode_stack_schedule_checks():
    from sparse_attention_fp4_kv_b200 import binding as B
    P = ctypes.c_void_p
    good = P(4096)
    layers = (B.csa2_layer * 2)()
    layers[0] = B.csa2_layer(B.MODE_REUSE, None, good, good, good, None)
    layers[1] = B.csa2_layer(B.MODE_FULL, good, good, good, good, good)
    ws_need = B.lib.csa2_decode_stack_workspace_size(2, 64, 512, 16, 128, 1000)
    assert ws_need > 0
    args = [good, good, good, good, 1000, good, good, 128, 2, 64, 512, 16, 128, ctypes.c_float(0.04),
            good, 0, None, good, ws_need, None]
    # a Reuse layer with no producer before it
    assert B.lib.csa2_decode_stack(layers, 2, None, *args) == -4
    # a Reindex layer with no pool
    layers[0] = B.csa2_layer(B.MODE_REINDEX, good, good, good, good, good)
    assert B.lib.csa2_decode_stack(layers, 2, None, *args) == -4
    # workspace too small
    layers[0] = B.csa2_layer(B.MODE_FULL, good, good, good, good, good)
    small = list(args)
    small[-2] = ws_need - 1
    assert B.lib.csa2_decode_stack(layers, 2, None, *small) == -5
    # workspace not 16-byte aligned: rejected before anything is launched
    odd = list(args)
    odd[-3] = P(4096 + 8)
    assert B.lib.csa2_decode_stack(layers, 2, None, *odd) == -3
    # unknown mode
    layers[1] = B.csa2_layer(7, good, good, good, good, good)
    assert B.lib.csa2_decode_stack(layers, 2, None, *args) == -4


def _attn_slot_bytes(hpc):
    # one cluster's exchange slot: 8 CTAs' partial O [hpc][512] fp32, row maxima and sums
    return (8 * hpc * 512 + 2 * 8 * hpc) * 4


def test_attention_workspace_covers_every_head_split(lib):
    """The launcher splits the 64 heads into clusters of 16, 32 or 64 (one
    layer at a time, or a whole layer group per launch, at most 18 clusters);
    the workspace holds the exchange slots of the largest of those splits."""
    ws = lib.csa2_sparse_attn_workspace_size
    ws.restype = ctypes.c_size_t
    ws.argtypes = [ctypes.c_int] * 6
    for B, Nq in [(1, 1), (2, 1), (3, 1), (4, 1), (5, 1), (7, 1), (8, 1), (9, 1), (16, 1), (4, 4),
                  (63, 1), (64, 1)]:
        rows = B * Nq
        need = [min(rows * (64 // hpc), 18) * _attn_slot_bytes(hpc) for hpc in (16, 32, 64)]
        got = ws(B, Nq, 64, 512, 512, 128)
        assert got == 256 + max(need), (B, Nq, got, need)   # error word + exchange slots
    # more than 640 keys: the per-row kernel, which has bounded waits but no slots
    assert ws(2, 1, 64, 512, 1024, 128) == 256
    # the tensor-core kernels need no workspace outside their shape, nor does the general kernel
    assert ws(2, 1, 8, 128, 512, 128) == 0


def test_workspace_status_rejects_a_null_workspace(lib):
    """The per-call error word is read from the workspace; a NULL workspace is
    rejected on the host before any CUDA call."""
    assert lib.csa2_workspace_status(None, 0, None) == -1
    assert lib.csa2_selftest_workspace_timeout(1000, None, None) == -1
