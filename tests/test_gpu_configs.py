"""GPU parity of whole decode steps (csa2_decode_stack, the call bench.py
times) against the oracle, on the benchmark workloads at full size and on
scaled-down variants with ragged shapes.

At full size the oracle recomputes sampled sequences one by one: the Full
layer's scan over the whole context, the pool, every layer's top-512, and
every layer's attention for those sequences. Pools and indices must match bit
for bit; attention within rel-L2 1e-3 / max-abs 5e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_cases import assert_attn_close, bf16_np
from sparse_attention_fp4_kv_b200 import synth

pytestmark = pytest.mark.gpu

NAMES = {synth.FULL: oracle.FULL, synth.REINDEX: oracle.REINDEX, synth.REUSE: oracle.REUSE}


def _oracle_sequence(wl, b):
    """Oracle indices and attention outputs of sequence b for every layer."""
    w = wl.w
    ctx = w.ctx
    kn = wl.k_idx[b].cpu().numpy()
    sn = wl.k_scale[b].cpu().numpy()
    kvb = bf16_np(wl.kv_bf16[b])
    pool = None
    if wl.pool_ready:
        pool = oracle.full_layer(wl.pool_q_idx[b, 0].cpu().numpy(), kn, sn, ctx)["pool"]
    tops, pools, outs = [], [], []
    top = None
    for l, m in enumerate(wl.modes):
        mode = NAMES[m]
        if mode == oracle.FULL:
            r = oracle.full_layer(wl.q_idx[l][b, 0].cpu().numpy(), kn, sn, ctx)
            pool, top = r["pool"], r["top"]
        elif mode == oracle.REINDEX:
            top, _, _ = oracle.reindex_layer(wl.q_idx[l][b, 0].cpu().numpy(), kn, sn, pool, ctx)
        tops.append(top)
        pools.append(pool)
        outs.append(oracle.sparse_attention(bf16_np(wl.q[l][b, 0]), lambda P: kvb[P], top,
                                            bf16_np(wl.swa[l][b]), ctx - 1, ctx - wl.swa_rows,
                                            wl.scale))
    return tops, pools, outs


def _check(wl, seqs):
    wl.step()
    torch.cuda.synchronize()
    producers = [l for l, m in enumerate(wl.modes) if m != synth.REUSE]
    for b in seqs:
        tops, pools, outs = _oracle_sequence(wl, b)
        assert np.array_equal(wl.pool[b].cpu().numpy(), pools[-1]), f"pool b={b}"
        for l in range(len(wl.modes)):
            prod = max(p for p in producers if p <= l)
            assert np.array_equal(wl.topk[prod][b].cpu().numpy(), tops[l]), f"top-512 b={b} l={l}"
            assert_attn_close(wl.out[l][b, 0].cpu().numpy(), outs[l], f"attention b={b} l={l}")


def _workload(name, **kw):
    from sparse_attention_fp4_kv_b200.workload import DecodeWorkload
    w = synth.WORKLOADS[name] if not kw else synth.scaled(synth.WORKLOADS[name], **kw)
    return DecodeWorkload(w, "cuda", keep_kv_bf16=True)


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- scaled variants (ragged)
@pytest.mark.parametrize("name,kw", [
    ("decoder_stack20_b4_ctx1m", dict(B=3, ctx=20003)),
    ("decoder_stack20_b4_ctx1m", dict(B=2, ctx=16389)),
    # an indexer of 4 x 64 channels (the rescoring's generic row shapes)
    ("decoder_stack20_b4_ctx1m", dict(B=2, ctx=20003, H_idx=4, D_idx=64)),
    ("decoder_group1_b8_ctx128k", dict(B=5, ctx=3001)),
    ("decoder_group1_b8_ctx128k", dict(B=1, ctx=100)),
    ("reindex_group_b32_ctx256k", dict(B=3, ctx=50001)),
    # pools of 38 and 2 blocks: every pooled token is selected (fewer than 512)
    ("reindex_group_b32_ctx256k", dict(B=2, ctx=300)),
    ("reindex_group_b32_ctx256k", dict(B=1, ctx=9)),
    # more rows than resident clusters: clusters take whole rows (64 heads) one
    # after another and run every layer of a row before the next
    ("reindex_group_b32_ctx256k", dict(B=20, ctx=9001)),
    ("encoder_stack18_b4_ctx1m", dict(B=2, ctx=40007)),
    ("full_b1_ctx4k", dict(B=2, ctx=777)),
])
def test_scaled_stack(name, kw):
    wl = _workload(name, **kw)
    _check(wl, range(wl.w.B))
    del wl
    _free()


def test_stack_with_64_sequences_takes_the_per_row_attention():
    """64 sequences: the stack's attention runs one launch per layer on the
    one-CTA-per-row kernel (the cluster kernel serves fewer rows); a Full group
    and a Reindex group, every ninth sequence checked."""
    wl = _workload("decoder_stack20_b4_ctx1m", B=64, ctx=2001, modes=list(synth.DECODER_MODES[:8]))
    _check(wl, range(0, 64, 9))
    del wl
    _free()


def test_stack_reuse_run_longer_than_one_attention_launch():
    """A Full layer followed by 10 Reuse layers: the attention of the first 8
    layers runs as one launch and the last 3 as a second launch led by a Reuse
    layer (it gathers its rows before its dependency wait)."""
    wl = _workload("decoder_stack20_b4_ctx1m", B=3, ctx=9001, modes=[synth.FULL] + [synth.REUSE] * 10)
    _check(wl, range(wl.w.B))
    del wl
    _free()


@pytest.mark.parametrize("levels", [1, 3])
def test_stack_tie_heavy_keys(levels):
    """Coarse indexer keys give many equal scores: with levels=1 every score is
    zero (the whole candidate list ties and the order falls to positions); with
    levels=3 the threshold bins hold long runs of equal scores."""
    wl = _workload("decoder_stack20_b4_ctx1m", B=2, ctx=30011)
    g = torch.Generator(device="cuda").manual_seed(levels)
    wl.k_idx.copy_(torch.randint(0, levels, wl.k_idx.shape, generator=g, device="cuda",
                                 dtype=torch.int8))
    wl.k_scale.fill_(1.0)
    _check(wl, range(wl.w.B))
    del wl
    _free()


@pytest.mark.parametrize("levels", [0, 1])
def test_stack_ragged_long_rows(levels):
    """Sequences of 532,000, 300,001 and 9 tokens in one step over a
    532,000-token cache: the pool selection takes its many-CTA form (rows of
    more than 65,536 blocks), whose CTAs past a short row's end only take the
    row's ticket, and whose last CTA per row finishes the row. levels=1 makes
    every indexer score zero, so the pool's threshold bin holds the whole row
    (more ties than the compacted tie list holds)."""
    ctxs = [532000, 300001, 9]
    wl = _workload("decoder_stack20_b4_ctx1m", B=3, ctx=ctxs[0], modes=[synth.FULL, synth.REUSE])
    if levels:
        wl.k_idx.zero_()
    rows = wl.swa_rows
    for b, c in enumerate(ctxs):
        wl.ctx_len[b] = c
        wl.swa_pos0[b] = c - rows  # the window's last row is position c - 1
        wl.kv_bf16[b, c - 1] = wl.kv_new[b]  # the step appends the new token at c - 1
    wl.step()
    torch.cuda.synchronize()
    for b, c in enumerate(ctxs):
        kn, sn = wl.k_idx[b].cpu().numpy(), wl.k_scale[b].cpu().numpy()
        r = oracle.full_layer(wl.q_idx[0][b, 0].cpu().numpy(), kn, sn, c)
        assert np.array_equal(wl.pool[b].cpu().numpy(), r["pool"]), f"pool b={b}"
        assert np.array_equal(wl.topk[0][b].cpu().numpy(), r["top"]), f"top-512 b={b}"
        kvb = bf16_np(wl.kv_bf16[b, :c])
        for l in range(2):
            ref = oracle.sparse_attention(bf16_np(wl.q[l][b, 0]), lambda P: kvb[P], r["top"],
                                          bf16_np(wl.swa[l][b]), c - 1, c - rows, wl.scale)
            assert_attn_close(wl.out[l][b, 0].cpu().numpy(), ref, f"attention b={b} l={l}")
    del wl
    _free()


@pytest.mark.parametrize("ctx", [524288, 524296])
def test_stack_pool_path_boundary(ctx):
    """The Full layer's pool selection at the edge of its two forms: 65,536
    blocks (the largest row one CTA selects) and 65,537 blocks (the many-CTA
    compaction, whose last slice holds one block)."""
    wl = _workload("decoder_stack20_b4_ctx1m", B=1, ctx=ctx, modes=[synth.FULL, synth.REUSE])
    _check(wl, [0])
    del wl
    _free()


@pytest.mark.parametrize("ctx", [30000, 600000])
def test_launches_per_step_matches_profiler(ctx):
    """The kernel count the benchmark reports equals the libcsa2 kernels the
    CUDA profiler sees in one step (600K tokens: the pool selection's rows are
    long enough to take the many-CTA compaction whose last CTA per row
    finishes it)."""
    wl = _workload("decoder_stack20_b4_ctx1m", B=1, ctx=ctx)
    wl.step()
    torch.cuda.synchronize()
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        wl.step()
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    ours = [n for n in names if "csa2::" in n]
    assert len(ours) == wl.launches_per_step(), sorted(set(ours))
    del wl
    _free()


def test_decode_step_replays_as_a_cuda_graph():
    """The step captured as a CUDA graph (dependent launches become graph
    edges) gives the same pools, indices and outputs, bit for bit, as the
    directly launched step."""
    wl = _workload("decoder_stack20_b4_ctx1m", B=2, ctx=30011)
    wl.step()
    torch.cuda.synchronize()
    ref = [t.clone() for t in wl.topk if t is not None] + [o.clone() for o in wl.out] + [wl.pool.clone()]
    for t in [t for t in wl.topk if t is not None] + list(wl.out):
        t.zero_()
    g = wl.capture_step_graph()
    g.replay()
    torch.cuda.synchronize()
    got = [t for t in wl.topk if t is not None] + list(wl.out) + [wl.pool]
    for x, y in zip(ref, got):
        assert torch.equal(x, y)
    from sparse_attention_fp4_kv_b200 import binding
    assert binding.device_status() == 0
    del g, wl
    _free()


def test_decode_step_is_deterministic():
    wl = _workload("decoder_stack20_b4_ctx1m", B=2, ctx=30000)
    wl.step()
    torch.cuda.synchronize()
    first = [t.clone() for t in wl.topk if t is not None] + [o.clone() for o in wl.out]
    for _ in range(2):
        wl.step()
        torch.cuda.synchronize()
        again = [t for t in wl.topk if t is not None] + list(wl.out)
        for x, y in zip(first, again):
            assert torch.equal(x, y)
    del wl
    _free()


# ---------------------------------------------------------------- benchmark workloads, full size
def test_full_b1_ctx4k():
    wl = _workload("full_b1_ctx4k")
    _check(wl, [0])
    del wl
    _free()


def test_decoder_group1_b8_ctx128k_sampled():
    wl = _workload("decoder_group1_b8_ctx128k")
    _check(wl, [0, 7])
    del wl
    _free()


def test_reindex_group_b32_ctx256k_sampled():
    wl = _workload("reindex_group_b32_ctx256k")
    _check(wl, [0, 31])
    # the planted blocks' tokens are all selected by the Reindex layer
    for b in (0, 31):
        top = set(wl.topk[0][b].cpu().tolist())
        planted = {8 * j + r for j in wl.planted[b].tolist() for r in range(8)}
        assert planted <= top
    del wl
    _free()


def test_decoder_stack20_b4_ctx1m_sampled():
    from sparse_attention_fp4_kv_b200 import binding
    binding.device_status(clear=True)
    wl = _workload("decoder_stack20_b4_ctx1m")
    _check(wl, [0, 3])
    assert binding.device_status() == 0  # no kernel gave up a bounded wait
    del wl
    _free()
