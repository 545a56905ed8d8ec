"""Pins for the oracle's indexer scores, block scores, pool, top-k and layer
schedule.

Checks come from outside the oracle: closed forms (unit-vector queries), a
library routine (numpy int64 matmul, numpy lexsort), an independent O(n*k)
selection on tiny inputs, the constants the pages state (pool of 2,048 blocks
of 8, top-512, the decoder and encoder schedules) and the theorem that the
pool-restricted top-512 equals the whole-context top-512.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _layout():
    vals = {}
    for line in open(os.path.join(GOLDEN, "csa2_layout.txt")):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            vals[k] = v
    return vals


def test_constants_match_pages():
    L = _layout()
    assert oracle.POOL_BLOCKS == int(L["pool_blocks"][0])
    assert oracle.BLOCK_TOKENS == int(L["block_tokens"][0])
    assert oracle.POOL_BLOCKS * oracle.BLOCK_TOKENS == int(L["pool_positions"][0]) == 16384
    assert oracle.TOPK == int(L["topk"][0])
    assert oracle.N_WIN == int(L["n_win"][0])
    assert oracle.FP4_GROUP == int(L["fp4_group"][0])


def test_schedules_match_pages():
    L = _layout()
    name = {"F": oracle.FULL, "Ri": oracle.REINDEX, "U": oracle.REUSE}
    assert oracle.decoder_schedule() == [name[m] for m in L["decoder"]]
    assert oracle.encoder_schedule() == [name[m] for m in L["encoder"]]
    # the benchmark workloads use the same schedules
    from sparse_attention_fp4_kv_b200 import synth
    code = {synth.FULL: oracle.FULL, synth.REINDEX: oracle.REINDEX, synth.REUSE: oracle.REUSE}
    assert [code[m] for m in synth.DECODER_MODES] == oracle.decoder_schedule()
    assert [code[m] for m in synth.ENCODER_MODES] == oracle.encoder_schedule()
    assert len(oracle.decoder_schedule()) == 20 and len(oracle.encoder_schedule()) == 18


# ----------------------------------------------------------------------------- indexer
def test_index_dots_unit_vector_closed_form():
    rng = np.random.default_rng(0)
    k = rng.integers(-127, 128, (50, 4, 64), dtype=np.int8)
    for h, d in [(0, 0), (1, 17), (3, 63)]:
        q = np.zeros((4, 64), np.int8)
        q[h, d] = 1
        assert np.array_equal(oracle.index_dots(q, k), k[:, h, d].astype(np.int64))
        q[h, d] = -1
        assert np.array_equal(oracle.index_dots(q, k), -k[:, h, d].astype(np.int64))


def test_index_dots_match_library_matmul():
    rng = np.random.default_rng(1)
    q = rng.integers(-128, 128, (16, 128), dtype=np.int8)
    k = rng.integers(-128, 128, (300, 16, 128), dtype=np.int8)
    ref = k.reshape(300, -1).astype(np.int64) @ q.reshape(-1).astype(np.int64)
    assert np.array_equal(oracle.index_dots(q, k), ref)


def test_index_scores_fp32_rounding_and_scale():
    # S = 2^24 + 1 is a tie between 2^24 and 2^24 + 2: round to even -> 2^24.
    # S = 2^24 + 3 is a tie between 2^24 + 2 and 2^24 + 4: round to even -> 2^24 + 4.
    HD = 132105
    q = np.ones(HD, np.int8)
    k1 = np.full(HD, 127, np.int8)
    k1[-1] = 9                              # 132104 * 127 + 9 = 2^24 + 1
    k2 = k1.copy()
    k2[-1] = 11                             # 2^24 + 3
    ks = np.ones(2, np.float32)
    sc = oracle.index_scores(q, np.stack([k1, k2]), ks)
    assert oracle.index_dots(q, np.stack([k1, k2])).tolist() == [2 ** 24 + 1, 2 ** 24 + 3]
    assert sc.tolist() == [2.0 ** 24, 2.0 ** 24 + 4]
    # general case against numpy's own int64 -> fp32 cast and fp32 multiply
    rng = np.random.default_rng(2)
    q = rng.integers(-127, 128, (16, 128), dtype=np.int8)
    k = rng.integers(-127, 128, (500, 16, 128), dtype=np.int8)
    s = (0.5 + rng.random(500)).astype(np.float32)
    ref = (k.reshape(500, -1).astype(np.int64) @ q.reshape(-1).astype(np.int64)).astype(np.float32) * s
    assert np.array_equal(oracle.index_scores(q, k, s).view(np.uint32), ref.view(np.uint32))


def test_index_scores_reject_int32_overflow():
    HD = 131073
    q = np.full(HD, -128, np.int8)
    k = np.full((1, HD), -128, np.int8)       # 131073 * 16384 > 2^31 - 1
    with pytest.raises(OverflowError):
        oracle.index_scores(q, k, np.ones(1, np.float32))


# ----------------------------------------------------------------------------- blocks
def test_block_scores_hand_example_and_ragged_tail():
    s = np.array([1, 5, 2, 2, 0, 0, 0, 0, -3, -1, -2, -9, -9, -9, -9, -9, 7, 8, 100], np.float32)
    assert oracle.block_scores(s, 16).tolist() == [5.0, -1.0]
    assert oracle.block_scores(s, 18).tolist() == [5.0, -1.0, 8.0]   # partial block sees 16, 17 only
    assert oracle.block_scores(s, 19).tolist() == [5.0, -1.0, 100.0]
    assert oracle.block_scores(s, 0).size == 0


# ----------------------------------------------------------------------------- top-k
def _brute_topk(score, pos, k):
    """Independent selection: repeatedly take the best remaining candidate
    (higher score, then lower position)."""
    left = list(zip(score.tolist(), pos.tolist()))
    out = []
    for _ in range(min(k, len(left))):
        best = max(left, key=lambda sp: (sp[0], -sp[1]))
        out.append(best[1])
        left.remove(best)
    return sorted(out) + [-1] * (k - len(out))


def test_topk_matches_brute_force_on_tie_heavy_inputs():
    rng = np.random.default_rng(5)
    for n in (1, 5, 16, 40, 97):
        for k in (1, 3, 16, 64):
            score = rng.integers(0, 4, n).astype(np.float32)     # many ties
            pos = rng.permutation(1000)[:n]
            assert oracle.topk(score, pos, k).tolist() == _brute_topk(score, pos, k)


def test_topk_matches_lexsort_on_large_inputs():
    rng = np.random.default_rng(6)
    n = 50000
    score = np.round(rng.standard_normal(n) * 50).astype(np.float32)
    pos = np.arange(n) * 3
    order = np.lexsort((pos, -score.astype(np.float64)))
    for k in (512, 2048):
        assert np.array_equal(oracle.topk(score, pos, k), np.sort(pos[order[:k]]))


def test_topk_special_cases():
    n = 5000
    eq = np.zeros(n, np.float32)
    assert np.array_equal(oracle.topk(eq, np.arange(n), 512), np.arange(512))
    inc = np.arange(n, dtype=np.float32)
    assert np.array_equal(oracle.topk(inc, np.arange(n), 512), np.arange(n - 512, n))
    short = oracle.topk(inc[:10], np.arange(10), 16)
    assert short.tolist() == list(range(10)) + [-1] * 6


# ----------------------------------------------------------------------------- layers
def _indexer_case(ctx, H=4, D=32, seed=0, levels=None):
    rng = np.random.default_rng(seed)
    k = rng.integers(-127, 128, (ctx, H, D), dtype=np.int8)
    if levels is not None:                       # coarse keys -> many tied scores
        k = (k // levels * levels).astype(np.int8)
    q = rng.integers(-127, 128, (H, D), dtype=np.int8)
    s = (0.5 + rng.random(ctx)).astype(np.float32)
    if levels is not None:
        s[:] = 1.0
    return q, k, s


@pytest.mark.parametrize("ctx", [1, 7, 8, 9, 100, 4096, 16384, 16385, 20003])
def test_pool_size_and_topk_count(ctx):
    q, k, s = _indexer_case(ctx, H=2, D=16, seed=ctx)
    r = oracle.full_layer(q, k, s, ctx)
    nblk = -(-ctx // 8)
    pool = r["pool"]
    assert pool.size == 2048
    assert (pool >= 0).sum() == min(2048, nblk)
    valid = pool[pool >= 0]
    assert np.all(np.diff(valid) > 0) and valid.max() < nblk
    top = r["top"]
    assert top.size == 512 and (top >= 0).sum() == min(512, ctx)
    tv = top[top >= 0]
    assert np.all(np.diff(tv) > 0) and tv.max() < ctx
    assert set(tv.tolist()) <= set(oracle.pooled_positions(pool, ctx).tolist())


@pytest.mark.parametrize("ctx,levels", [(20000, None), (33333, None), (20000, 64)])
def test_pooled_top512_equals_whole_context_top512(ctx, levels):
    q, k, s = _indexer_case(ctx, seed=ctx, levels=levels)
    r = oracle.full_layer(q, k, s, ctx)
    sc = r["tok_score"]
    order = np.lexsort((np.arange(ctx), -sc.astype(np.float64)))
    assert np.array_equal(r["top"], np.sort(order[:512]))
    # and the pool is the top min(2048, nblk) blocks by (block max desc, block asc)
    blk = r["blk_score"]
    bo = np.lexsort((np.arange(blk.size), -blk.astype(np.float64)))
    assert np.array_equal(r["pool"][r["pool"] >= 0], np.sort(bo[:2048]))


@pytest.mark.parametrize("ctx,levels", [(20000, None), (33333, None), (20000, 64)])
def test_top512_tokens_lie_in_top512_blocks(ctx, levels):
    """Every one of the best 512 tokens lies in one of the best 512 blocks (by
    block max desc, block asc): each block ranked ahead of a token's block holds
    a token ranked ahead of that token. The decode selection gathers only the
    pooled blocks that reach the 512th block's histogram bin, a superset of
    those blocks."""
    q, k, s = _indexer_case(ctx, seed=ctx + 1, levels=levels)
    r = oracle.full_layer(q, k, s, ctx)
    blk = r["blk_score"]
    bo = np.lexsort((np.arange(blk.size), -blk.astype(np.float64)))
    best = set(bo[:512].tolist())
    tv = r["top"][r["top"] >= 0]
    assert set((tv // 8).tolist()) <= best


def test_reindex_subset_of_pool_and_identity_with_full_query():
    ctx = 30000
    q, k, s = _indexer_case(ctx, seed=9)
    r = oracle.full_layer(q, k, s, ctx)
    top_same, ppos, _ = oracle.reindex_layer(q, k, s, r["pool"], ctx)
    assert np.array_equal(top_same, r["top"])
    q2 = np.random.default_rng(10).integers(-127, 128, q.shape, dtype=np.int8)
    top2, ppos2, sc2 = oracle.reindex_layer(q2, k, s, r["pool"], ctx)
    assert set(top2[top2 >= 0].tolist()) <= set(ppos2.tolist())
    assert ppos2.size == 16384
    # rescoring really uses the new query: exact scores of the chosen tokens
    assert np.array_equal(sc2, oracle.index_scores(q2, k[ppos2], s[ppos2]))


def test_stack_reuse_layers_take_producer_indices():
    ctx = 20000
    rng = np.random.default_rng(12)
    k = rng.integers(-127, 128, (ctx, 4, 32), dtype=np.int8)
    s = (0.5 + rng.random(ctx)).astype(np.float32)
    qs = {l: rng.integers(-127, 128, (4, 32), dtype=np.int8) for l in range(20)}
    modes = oracle.decoder_schedule()
    tops, pools = oracle.stack_indices(modes, lambda l: qs[l], k, s, ctx)
    assert list(pools) == [0]
    # the Full layer's pool and indices, as the layer alone computes them (ascending, -1 padded)
    full = oracle.full_layer(qs[0], k, s, ctx)
    assert np.array_equal(pools[0], full["pool"]) and np.array_equal(tops[0], full["top"])
    assert np.all(np.diff(pools[0][pools[0] >= 0]) > 0)
    for l, m in enumerate(modes):
        producer = max(i for i in range(l + 1) if modes[i] != oracle.REUSE)
        assert np.array_equal(tops[l], tops[producer])
        if m == oracle.REINDEX:
            ref, _, _ = oracle.reindex_layer(qs[l], k, s, pools[0], ctx)
            assert np.array_equal(tops[l], ref)
    with pytest.raises(ValueError):
        oracle.stack_indices([oracle.REUSE], lambda l: qs[l], k, s, ctx)
    with pytest.raises(ValueError):
        oracle.stack_indices([oracle.REINDEX], lambda l: qs[l], k, s, ctx)
