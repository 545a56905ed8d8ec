"""GPU parity of the chunked-prefill path (one Full layer, many causal
queries per sequence) against the oracle: FP4 append of the new rows, causal
tensor-core indexer scoring, per-query pool and top-512, and attention over
the 512 rows plus each query's own window.

Pools and indices must match bit for bit; attention within rel-L2 1e-3 and
max-abs 5e-3. The small case checks every query; the full-size workload
(4096 queries at 64K) checks sampled queries, which the oracle recomputes
one by one over their whole visible context.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_cases import assert_attn_close, bf16_np
from sparse_attention_fp4_kv_b200 import synth

pytestmark = pytest.mark.gpu


def _check_queries(pw, queries):
    w = pw.w
    for b in range(w.B):
        kn = pw.k_idx[b].cpu().numpy()
        sn = pw.k_scale[b].cpu().numpy()
        kvb = bf16_np(pw.kv_bf16[b])
        swa = bf16_np(pw.swa[b])
        pos0 = int(pw.swa_pos0[b])
        for i in queries:
            p = pw.ctx0 + i
            r = oracle.full_layer(pw.q_idx[b, i].cpu().numpy(), kn, sn, p + 1)
            assert np.array_equal(pw.pool[b, i].cpu().numpy(), r["pool"]), f"pool b={b} i={i}"
            assert np.array_equal(pw.top[b, i].cpu().numpy(), r["top"]), f"top b={b} i={i}"
            ref = oracle.sparse_attention(bf16_np(pw.q[b, i]), lambda P: kvb[P], r["top"], swa, p,
                                          pos0, pw.scale)
            assert_attn_close(pw.out[b, i].cpu().numpy(), ref, f"attention b={b} i={i}")


def _fp4_matches_oracle(pw):
    w = pw.w
    for b in range(w.B):
        packed, sf = oracle.fp4_quantize(bf16_np(pw.kv_new[b]))
        assert np.array_equal(pw.kv_fp4[b, pw.ctx0:].cpu().numpy(), packed)
        assert np.array_equal(pw.kv_sf[b, pw.ctx0:].cpu().numpy(), sf)


@pytest.mark.parametrize("ctx0,n", [(3000, 300), (1000, 129)])
def test_prefill_small_all_queries(ctx0, n):
    from sparse_attention_fp4_kv_b200.workload import PrefillWorkload
    w = synth.scaled(synth.WORKLOADS["prefill_4096_at_64k"], B=2, ctx=ctx0 + n, n_new=n,
                     prefill_queries=n)
    pw = PrefillWorkload(w, "cuda", keep_kv_bf16=True)
    pw.step()
    torch.cuda.synchronize()
    _fp4_matches_oracle(pw)
    _check_queries(pw, range(n))
    del pw
    torch.cuda.empty_cache()


def test_prefill_4096_at_64k_sampled():
    from sparse_attention_fp4_kv_b200.workload import PrefillWorkload
    from sparse_attention_fp4_kv_b200 import binding
    binding.device_status(clear=True)
    pw = PrefillWorkload(synth.WORKLOADS["prefill_4096_at_64k"], "cuda", keep_kv_bf16=True)
    pw.step()
    torch.cuda.synchronize()
    assert binding.device_status() == 0  # no kernel gave up a bounded wait
    _fp4_matches_oracle(pw)
    _check_queries(pw, [0, 1, 127, 128, 2049, 4095])
    del pw
    torch.cuda.empty_cache()


def test_multi_token_decode_sampled():
    """Four speculative tokens per sequence at 1M context: the tensor-core scan
    with a mostly padded query tile, the three-call selection (the rows are too
    long for the fused kernel) and split-key attention; sampled queries."""
    from sparse_attention_fp4_kv_b200.workload import PrefillWorkload
    from sparse_attention_fp4_kv_b200 import binding
    w = synth.scaled(synth.WORKLOADS["decode_mtp4_b4_ctx1m"], B=2, ctx=200003 + 4)
    pw = PrefillWorkload(w, "cuda", keep_kv_bf16=True)
    assert not pw.fused_select
    binding.device_status(clear=True)
    pw.step()
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    _fp4_matches_oracle(pw)
    _check_queries(pw, [0, 3])
    del pw
    torch.cuda.empty_cache()
