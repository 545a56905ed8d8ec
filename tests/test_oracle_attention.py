"""Pins for the oracle's attention and the end-to-end decode composition.

References outside the oracle: torch's scaled_dot_product_attention in fp64
(a library routine), closed forms (one key gives that key's row; equal logits
give the mean row), permutation invariance, and "dense equals sparse" when the
selection covers the whole context.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_fp4_kv_b200 import synth


def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _sdpa(q64, kv64, scale):
    q = torch.from_numpy(q64)[None, :, None, :]          # [1, Hq, 1, C]
    kv = torch.from_numpy(kv64)[None, None, :, :]        # [1, 1, n, C]
    kv = kv.expand(1, q.shape[1], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(q, kv, kv, scale=scale)
    return o[0, :, 0, :].numpy()


def test_attention_matches_library_sdpa():
    g = torch.Generator().manual_seed(0)
    qb = _bf16_bits(torch.randn(8, 64, generator=g))
    kv = torch.randn(100, 64, generator=g, dtype=torch.float64).numpy()
    out = oracle.attention(qb, kv, 0.125)
    ref = _sdpa(oracle.bf16_to_f64(qb), kv, 0.125)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_attention_closed_forms():
    g = torch.Generator().manual_seed(1)
    qb = _bf16_bits(torch.randn(4, 32, generator=g))
    kv = torch.randn(1, 32, generator=g, dtype=torch.float64).numpy()
    out = oracle.attention(qb, kv, 0.3)
    assert np.array_equal(out, np.repeat(kv, 4, 0))        # single key -> that row
    kv = torch.randn(37, 32, generator=g, dtype=torch.float64).numpy()
    zq = np.zeros((4, 32), np.uint16)                       # equal logits -> mean row
    np.testing.assert_allclose(oracle.attention(zq, kv, 1.0), np.repeat(kv.mean(0, keepdims=True), 4, 0),
                               rtol=1e-13, atol=1e-14)
    perm = np.random.default_rng(2).permutation(37)
    np.testing.assert_allclose(oracle.attention(qb, kv[perm], 0.3), oracle.attention(qb, kv, 0.3),
                               rtol=1e-12, atol=1e-14)


def test_attention_without_keys_is_zero():
    """A query that attends no key (every index masked, no window row) has no
    softmax; its output is zero by definition, and the oracle's sparse path
    reaches that case from masked indices and an empty window."""
    qb = _bf16_bits(torch.randn(4, 32, generator=torch.Generator().manual_seed(3)))
    out = oracle.attention(qb, np.zeros((0, 32)), 0.3)
    assert out.shape == (4, 32) and np.array_equal(out, np.zeros((4, 32)))
    rows = np.zeros((10, 32), np.uint16)
    swa = np.zeros((128, 32), np.uint16)
    out = oracle.sparse_attention(qb, lambda p: rows[p], -np.ones(8, np.int32), swa, 500, 373, 0.3,
                                  n_win=0)
    assert np.array_equal(out, np.zeros((4, 32)))


def test_window_rows():
    assert oracle.window_rows(999, 872, 128).tolist() == list(range(128))
    assert oracle.window_rows(99, 0, 100).tolist() == list(range(100))
    # prefill: query at position p sees rows for positions p-127..p
    assert oracle.window_rows(65536, 65409, 4223).tolist() == list(range(0, 128))
    assert oracle.window_rows(69631, 65409, 4223).tolist() == list(range(4095, 4223))


@pytest.mark.parametrize("ctx", [200, 512])
def test_dense_equals_sparse_when_selection_covers_context(ctx):
    w = synth.scaled(synth.WORKLOADS["full_b1_ctx4k"], ctx=ctx)
    kv = synth.main_kv_bf16(w, 0, 0, ctx, "cpu")
    kvb = kv.view(torch.int16).numpy().view(np.uint16)
    kidx = synth.indexer_keys(w, 0, ctx, "cpu").numpy()
    ksc = synth.indexer_key_scale(w, 0, ctx, "cpu").numpy()
    qidx = synth.indexer_q(w, 0, 1, "cpu").numpy()[0, 0]
    q = synth.main_q(w, 0, 1, "cpu")[0, 0]
    qb = q.view(torch.int16).numpy().view(np.uint16)
    swa_rows = min(128, ctx)
    swa = synth.swa_kv(w, 0, swa_rows, "cpu")[0]
    swab = swa.view(torch.int16).numpy().view(np.uint16)
    r = oracle.full_layer(qidx, kidx, ksc, ctx)
    assert np.array_equal(r["top"][r["top"] >= 0], np.arange(ctx))
    scale = 1.0 / np.sqrt(w.C)
    out = oracle.sparse_attention(qb, lambda p: kvb[p], r["top"], swab, ctx - 1, ctx - swa_rows, scale)
    # textbook dense attention over every main-KV row (FP4 round trip) plus the window
    packed, sf = oracle.fp4_quantize(kvb)
    dense_kv = np.concatenate([oracle.fp4_dequantize(packed, sf), oracle.bf16_to_f64(swab)], 0)
    ref = _sdpa(oracle.bf16_to_f64(qb), dense_kv, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_planted_blocks_reach_reindex_top512():
    """Scaled-down Reindex workload: the planted blocks (keys correlated 0.9
    with the Reindex query) land in the pool of the Full layer built from a
    query correlated 0.7, and all their tokens make the Reindex top-512."""
    w = synth.scaled(synth.WORKLOADS["reindex_group_b32_ctx256k"], B=1, ctx=40000)
    qr = synth.indexer_q(w, 0, 1, "cpu")[0, 0]
    qf = synth.pool_builder_q(w, qr)
    k = synth.indexer_keys(w, 0, w.ctx, "cpu")
    blocks = synth.plant(w, 0, k, qr)
    s = synth.indexer_key_scale(w, 0, w.ctx, "cpu").numpy()
    full = oracle.full_layer(qf.numpy(), k.numpy(), s, w.ctx)
    assert set(blocks.tolist()) <= set(full["pool"].tolist())
    top, _, _ = oracle.reindex_layer(qr.numpy(), k.numpy(), s, full["pool"], w.ctx)
    planted_tokens = {8 * j + r for j in blocks.tolist() for r in range(8)}
    assert planted_tokens <= set(top.tolist())
