"""GPU test of csa2_decode_stack_noalloc, the decode step for callers that
cannot allocate device memory: code running under CUDA graph capture, plugin
hosts that own every allocation, or latency-critical loops that cannot afford
cudaMalloc's synchronisation. That entry point keeps its scratch in a fixed
24 MiB array inside the library instead of a caller-provided workspace.

The test runs the same decode step through the regular entry point
(csa2_decode_stack, with a workspace) and then twice in a row through the
no-alloc entry point, called through the C ABI, and checks that the no-alloc
results match: indices and pools bit for bit, attention outputs within the
tolerance the other tests use. It also checks that a problem larger than the
scratch array is rejected before anything runs. This file is collected last,
so a failure here comes after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_cases import assert_attn_close
from sparse_attention_fp4_kv_b200 import synth

pytestmark = pytest.mark.gpu


def _snapshot(wl):
    return ([o.clone() for o in wl.out], [t.clone() for t in wl.topk if t is not None],
            wl.pool.clone())


def _scramble(wl, ref_pool):
    for o in wl.out:
        o.fill_(float("nan"))
    for t in wl.topk:
        if t is not None:
            t.fill_(-7)
    if wl.pool_ready:
        wl.pool.copy_(ref_pool)   # a Reindex group reads the pool as an input
    else:
        wl.pool.fill_(-7)         # a stack with a Full layer writes it


@pytest.mark.parametrize("name,kw", [("decoder_stack20_b4_ctx1m", dict(B=2, ctx=20003)),
                                     ("reindex_group_b32_ctx256k", dict(B=3, ctx=30001))])
def test_noalloc_matches_regular_entry_point(name, kw):
    from sparse_attention_fp4_kv_b200.workload import DecodeWorkload
    wl = DecodeWorkload(synth.scaled(synth.WORKLOADS[name], **kw), "cuda")
    wl.step()                                  # regular entry point, caller workspace
    torch.cuda.synchronize()
    ref_out, ref_top, ref_pool = _snapshot(wl)
    for call in range(2):                      # two no-alloc calls in a row
        _scramble(wl, ref_pool)
        st = wl.stack.call_noalloc()
        assert st == 0, f"csa2_decode_stack_noalloc returned {st}"
        torch.cuda.synchronize()
        assert torch.equal(wl.pool, ref_pool), f"pool differs (call {call})"
        tops = [t for t in wl.topk if t is not None]
        for a, b in zip(tops, ref_top):
            assert torch.equal(a, b), f"top-512 differs (call {call})"
        for l, (a, b) in enumerate(zip(wl.out, ref_out)):
            assert_attn_close(a.cpu().numpy(), b.cpu().numpy(), f"layer {l} call {call}")
    del wl
    torch.cuda.empty_cache()


def test_noalloc_rejects_problems_beyond_the_scratch_limit():
    from sparse_attention_fp4_kv_b200 import binding as B
    # every device pointer is NULL: the size check comes first and returns
    # CSA2_ERR_WORKSPACE; were it ever to run later, the NULL checks would stop
    # the call on the host (CSA2_ERR_NULL) before any kernel could launch
    layers = (B.csa2_layer * 1)(B.csa2_layer(B.MODE_FULL, None, None, None, None, None))
    B_, cap = 8, 1 << 20                       # needs ~38 MB of scratch
    need = B.lib.csa2_decode_stack_workspace_size(B_, 64, 512, 16, 128, cap)
    assert need > (24 << 20)
    st = B.lib.csa2_decode_stack_noalloc(layers, 1, None, None, None, None, None, cap, None, None,
                                         128, B_, 64, 512, 16, 128, ctypes.c_float(0.04), None, 0,
                                         None)
    assert st == -5 and B.status_string(st) == "workspace missing or too small"
