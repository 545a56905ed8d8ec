"""GPU parity of each libcsa2 entry point against the CPU oracle, at sizes the
oracle finishes in seconds that still span several tiles and a ragged tail.

Bit-exact: packed FP4 bytes, E4M3 scales, token and block scores (fp32 bits),
block counts, pool and top-k indices. Attention: rel-L2 <= 1e-3 and
max-abs <= 5e-3 against the fp64 oracle.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_cases import assert_attn_close, bf16_np, f32_bits
from sparse_attention_fp4_kv_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def B():
    from sparse_attention_fp4_kv_b200 import binding
    return binding


# ----------------------------------------------------------------------------- a1 append
def _append_and_compare(B, x_bf16: torch.Tensor, cap_extra=3, start=None):
    """x_bf16: [Bn, n, C] on device. Appends at start positions and compares
    every written row with the oracle's quantizer."""
    Bn, n, C = x_bf16.shape
    cap = n + cap_extra
    if start is None:
        start = torch.arange(Bn, dtype=torch.int64) % (cap_extra + 1)
    start = start.to(DEV)
    fp4 = torch.full((Bn, cap, C // 2), 0xAB, dtype=torch.uint8, device=DEV)
    sf = torch.full((Bn, cap, C // 16), 0xCD, dtype=torch.uint8, device=DEV)
    B.csa2_kv_append_fp4(x_bf16, start, fp4, sf)
    torch.cuda.synchronize()
    xp, xs = oracle.fp4_quantize(bf16_np(x_bf16))
    g4, gs = fp4.cpu().numpy(), sf.cpu().numpy()
    for b in range(Bn):
        s0 = int(start[b])
        assert np.array_equal(g4[b, s0:s0 + n], xp[b]), f"packed bytes differ (b={b})"
        assert np.array_equal(gs[b, s0:s0 + n], xs[b]), f"scales differ (b={b})"
        # rows outside the written range are untouched
        assert np.all(g4[b, :s0] == 0xAB) and np.all(g4[b, s0 + n:] == 0xAB)


def test_append_synthetic_rows(B):
    w = synth.scaled(synth.WORKLOADS["decoder_group1_b8_ctx128k"], ctx=300)
    x = torch.stack([synth.main_kv_bf16(w, b, 0, 300, DEV) for b in range(3)])
    _append_and_compare(B, x)


def test_append_random_bit_patterns(B):
    g = torch.Generator(device=DEV).manual_seed(5)
    bits = torch.randint(0, 1 << 16, (4, 257, 512), generator=g, device=DEV, dtype=torch.int32)
    bits = bits.to(torch.int16)
    x = bits.view(torch.bfloat16)
    finite = torch.isfinite(x.float())
    x = torch.where(finite, x, torch.zeros_like(x))
    _append_and_compare(B, x.contiguous())


def test_append_ties_zeros_and_tiny_groups(B):
    rows = []
    e4 = [oracle.e4m3_value(c) for c in range(0x01, 0x7F)]
    mult = np.array([6, .25, .75, 1.25, 1.75, 2.5, 3.5, 5, -.25, -.75, -1.25, -2.5, -5, 0, -0.0, 6.5])
    for s in e4:
        rows.append(mult * s)
    rows.append(np.zeros(16))
    rows.append(-np.zeros(16))                      # negative zeros: scale 0, codes +0
    rows.append(np.full(16, 2.0 ** -13))            # amax/6 below the smallest E4M3 subnormal
    rows.append(np.full(16, -(2.0 ** -12)))
    rows.append(np.array([3e38] + [1.0] * 15))       # scale saturates at 448
    arr = np.concatenate(rows).astype(np.float32)
    pad = (-arr.size) % 128
    arr = np.concatenate([arr, np.zeros(pad, np.float32)]).reshape(1, -1, 128)
    x = torch.from_numpy(arr).to(torch.bfloat16).to(DEV)
    _append_and_compare(B, x.contiguous(), cap_extra=0)


@pytest.mark.parametrize("C", [16, 48, 128, 1024])
def test_append_channel_counts(B, C):
    g = torch.Generator(device=DEV).manual_seed(C)
    x = (torch.randn(2, 33, C, generator=g, device=DEV) * 3).to(torch.bfloat16)
    _append_and_compare(B, x)


def test_append_out_of_range_positions_are_skipped(B):
    x = torch.ones(2, 4, 32, dtype=torch.bfloat16, device=DEV)
    fp4 = torch.zeros(2, 4, 16, dtype=torch.uint8, device=DEV)
    sf = torch.zeros(2, 4, 2, dtype=torch.uint8, device=DEV)
    start = torch.tensor([2, -3], dtype=torch.int64, device=DEV)
    B.csa2_kv_append_fp4(x, start, fp4, sf)
    torch.cuda.synchronize()
    sfn = sf.cpu().numpy()
    assert np.all(sfn[0, 2:] != 0) and np.all(sfn[0, :2] == 0)
    assert np.all(sfn[1, :1] != 0) and np.all(sfn[1, 1:] == 0)


# ----------------------------------------------------------------------------- MXFP4 variant
def _append_mx_and_compare(B, x_bf16: torch.Tensor, cap_extra=3):
    """MXFP4 append (E8M0 per 32 channels) against the oracle, bit for bit."""
    Bn, n, C = x_bf16.shape
    cap = n + cap_extra
    start = (torch.arange(Bn, dtype=torch.int64) % (cap_extra + 1)).to(DEV)
    fp4 = torch.full((Bn, cap, C // 2), 0xAB, dtype=torch.uint8, device=DEV)
    sf = torch.full((Bn, cap, C // 32), 0xCD, dtype=torch.uint8, device=DEV)
    B.csa2_kv_append_fp4(x_bf16, start, fp4, sf, mx=True)
    torch.cuda.synchronize()
    xp, xs = oracle.mxfp4_quantize(bf16_np(x_bf16))
    g4, gs = fp4.cpu().numpy(), sf.cpu().numpy()
    for b in range(Bn):
        s0 = int(start[b])
        assert np.array_equal(g4[b, s0:s0 + n], xp[b]), f"packed bytes differ (b={b})"
        assert np.array_equal(gs[b, s0:s0 + n], xs[b]), f"E8M0 scales differ (b={b})"
        assert np.all(g4[b, :s0] == 0xAB) and np.all(gs[b, s0 + n:] == 0xCD)


def test_append_mxfp4_synthetic_rows_and_random_bits(B):
    w = synth.scaled(synth.WORKLOADS["decoder_group1_b8_ctx128k"], ctx=300)
    _append_mx_and_compare(B, torch.stack([synth.main_kv_bf16(w, b, 0, 300, DEV) for b in range(3)]))
    g = torch.Generator(device=DEV).manual_seed(15)
    bits = torch.randint(0, 1 << 16, (3, 129, 512), generator=g, device=DEV, dtype=torch.int32)
    x = bits.to(torch.int16).view(torch.bfloat16)
    x = torch.where(torch.isfinite(x.float()), x, torch.zeros_like(x))
    _append_mx_and_compare(B, x.contiguous())


def test_append_mxfp4_special_blocks(B):
    """Zero and negative-zero blocks, subnormal and near-maximum amax, amax at
    and just below powers of two, E2M1 ties and the saturation band (6, 8)."""
    rows = [np.zeros(32), -np.zeros(32), np.full(32, 2.0 ** -130), np.full(32, -(2.0 ** -133)),
            np.array([3.0e38] + [1.0] * 31), np.array([2.0 ** 10] + [3.0] * 31),
            np.array([2.0 ** 10 - 4.0] + [-3.0] * 31)]
    for k in range(-6, 7, 3):
        s = 2.0 ** k
        ties = np.array([.25, .75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.0, 7.75, -0.25, -2.5, -5.0,
                         4.0, 0.0, -0.0] * 2) * s
        rows.append(ties)
    x = torch.from_numpy(np.stack(rows).astype(np.float32)).to(torch.bfloat16).to(DEV)
    _append_mx_and_compare(B, x.view(1, -1, 32).contiguous(), cap_extra=0)


@pytest.mark.parametrize("C", [32, 96, 512])
def test_append_mxfp4_channel_counts(B, C):
    g = torch.Generator(device=DEV).manual_seed(C + 1)
    _append_mx_and_compare(B, (torch.randn(2, 17, C, generator=g, device=DEV) * 5).to(torch.bfloat16))


@pytest.mark.parametrize("Bn,ctx,C,Hq,K,Nq", [(3, 4000, 512, 64, 512, 1),     # split-key clusters
                                              (7, 3000, 512, 64, 512, 1),      # 32-head groups
                                              (70, 900, 512, 64, 512, 1),      # one CTA per row
                                              (2, 2000, 128, 8, 512, 1)])      # general kernel
def test_sparse_attention_mxfp4(B, Bn, ctx, C, Hq, K, Nq):
    _attention_case(B, Bn, ctx, C, Hq, K, 128, seed=Bn + ctx + 3, Nq=Nq, drop=7, mx=True)


# ----------------------------------------------------------------------------- a2/a3 scan
def _index_inputs(Bn, cap, H, D, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    k = torch.randint(-127, 128, (Bn, cap, H, D), generator=g, device=DEV, dtype=torch.int8)
    q = torch.randint(-127, 128, (Bn, 1, H, D), generator=g, device=DEV, dtype=torch.int8)
    s = 0.5 + torch.rand((Bn, cap), generator=g, device=DEV)
    return q, k, s


@pytest.mark.parametrize("H,D,ctxs", [(16, 128, [4100, 8, 1]), (4, 64, [4096, 3001, 17]),
                                      (3, 32, [1000, 999, 64]), (8, 128, [2049, 77, 5])])
def test_index_full_scores_bitexact(B, H, D, ctxs):
    cap = max(ctxs) + 5
    Bn = len(ctxs)
    q, k, s = _index_inputs(Bn, cap, H, D, seed=H * D)
    ctx = torch.tensor(ctxs, dtype=torch.int64, device=DEV)
    nb = (cap + 7) // 8
    blk = torch.full((Bn, 1, nb), -7.0, device=DEV)
    tok = torch.full((Bn, 1, cap), -7.0, device=DEV)
    nblk = torch.zeros((Bn, 1), dtype=torch.int32, device=DEV)
    B.csa2_index_full(q, k, s, ctx, blk, tok, nblk)
    torch.cuda.synchronize()
    qn, kn, sn = q.cpu().numpy(), k.cpu().numpy(), s.cpu().numpy()
    for b, c in enumerate(ctxs):
        ref_tok = oracle.index_scores(qn[b, 0], kn[b, :c], sn[b, :c])
        ref_blk = oracle.block_scores(ref_tok, c)
        assert np.array_equal(f32_bits(tok[b, 0, :c]), f32_bits(ref_tok))
        assert np.array_equal(f32_bits(blk[b, 0, :ref_blk.size]), f32_bits(ref_blk))
        assert int(nblk[b, 0]) == ref_blk.size
        assert np.all(tok[b, 0, c:].cpu().numpy() == -7.0)     # not written beyond ctx
        assert np.all(blk[b, 0, ref_blk.size:].cpu().numpy() == -7.0)


def test_index_full_extreme_values_int32_exact(B):
    # all +-127 / -128 keys: |S| up to 2048 * 16384; fp32 conversion rounds
    Bn, cap, H, D = 2, 64, 16, 128
    q = torch.full((Bn, 1, H, D), -128, dtype=torch.int8, device=DEV)
    k = torch.full((Bn, cap, H, D), -128, dtype=torch.int8, device=DEV)
    k[:, 1::2] = 127
    k[:, 5, :, :7] = -3
    s = torch.full((Bn, cap), 1.0, device=DEV)
    s[:, 3] = 0.75
    ctx = torch.tensor([64, 61], dtype=torch.int64, device=DEV)
    blk = torch.zeros((Bn, 1, 8), device=DEV)
    tok = torch.zeros((Bn, 1, cap), device=DEV)
    B.csa2_index_full(q, k, s, ctx, blk, tok)
    torch.cuda.synchronize()
    for b, c in enumerate([64, 61]):
        ref = oracle.index_scores(q[b, 0].cpu().numpy(), k[b, :c].cpu().numpy(), s[b, :c].cpu().numpy())
        assert np.array_equal(f32_bits(tok[b, 0, :c]), f32_bits(ref))


def test_index_full_causal_multi_query(B):
    Bn, cap, H, D, Nq = 2, 3000, 4, 64, 5
    g = torch.Generator(device=DEV).manual_seed(9)
    k = torch.randint(-127, 128, (Bn, cap, H, D), generator=g, device=DEV, dtype=torch.int8)
    q = torch.randint(-127, 128, (Bn, Nq, H, D), generator=g, device=DEV, dtype=torch.int8)
    s = 0.5 + torch.rand((Bn, cap), generator=g, device=DEV)
    ctx = torch.tensor([3000, 2500], dtype=torch.int64, device=DEV)
    qpos = torch.tensor([[0, 7, 8, 1234, 2999], [100, 2499, 2600, 9, 10]], dtype=torch.int64,
                        device=DEV)
    nb = (cap + 7) // 8
    blk = torch.zeros((Bn, Nq, nb), device=DEV)
    tok = torch.zeros((Bn, Nq, cap), device=DEV)
    nblk = torch.zeros((Bn, Nq), dtype=torch.int32, device=DEV)
    B.csa2_index_full(q, k, s, ctx, blk, tok, nblk, q_pos=qpos)
    torch.cuda.synchronize()
    for b in range(Bn):
        for i in range(Nq):
            V = min(int(qpos[b, i]) + 1, int(ctx[b]))
            ref = oracle.index_scores(q[b, i].cpu().numpy(), k[b, :V].cpu().numpy(), s[b, :V].cpu().numpy())
            rb = oracle.block_scores(ref, V)
            assert np.array_equal(f32_bits(tok[b, i, :V]), f32_bits(ref))
            assert np.array_equal(f32_bits(blk[b, i, :rb.size]), f32_bits(rb))
            assert int(nblk[b, i]) == rb.size


# ----------------------------------------------------------------------------- a4/a5 top-k
def _topk_ref(score, pos, valid, k):
    sel = pos >= 0
    if valid is not None:
        sel &= np.arange(score.size) < valid
    return oracle.topk(score[sel], pos[sel], k)


@pytest.mark.parametrize("n,k,levels", [(131072, 2048, None), (20000, 512, 7), (16384, 512, None),
                                        (5000, 512, 1), (300, 512, None), (70000, 2048, 3),
                                        (9000, 4096, None), (1, 1, None)])
def test_topk_bitexact(B, n, k, levels):
    R = 3
    g = torch.Generator(device=DEV).manual_seed(n + k)
    if levels is None:
        score = torch.randn((R, n), generator=g, device=DEV) * 1e5
    else:
        score = torch.randint(0, levels, (R, n), generator=g, device=DEV).float() - 1.0
    score[0, : n // 3] = -0.0 if levels == 1 else score[0, : n // 3]
    out = torch.empty((R, k), dtype=torch.int32, device=DEV)
    nv = torch.tensor([n, max(n // 2, 1), max(n - 17, 1)], dtype=torch.int32, device=DEV)
    B.csa2_topk(score, k, out, n_valid=nv)
    torch.cuda.synchronize()
    sc = score.cpu().numpy()
    for r in range(R):
        ref = _topk_ref(sc[r], np.arange(n), int(nv[r]), k)
        assert np.array_equal(out[r].cpu().numpy(), ref), f"row {r}"


def test_topk_with_candidate_positions(B):
    R, n, k = 4, 16384, 512
    g = torch.Generator(device=DEV).manual_seed(77)
    score = torch.randint(-50, 50, (R, n), generator=g, device=DEV).float()
    pos = torch.randperm(10 * n, generator=g, device=DEV)[: R * n].view(R, n).to(torch.int32)
    pos[:, ::5] = -1
    out = torch.empty((R, k), dtype=torch.int32, device=DEV)
    B.csa2_topk(score, k, out, cand_pos=pos)
    torch.cuda.synchronize()
    for r in range(R):
        ref = _topk_ref(score[r].cpu().numpy(), pos[r].cpu().numpy().astype(np.int64), None, k)
        assert np.array_equal(out[r].cpu().numpy(), ref)


# ----------------------------------------------------------------------------- Full / Reindex
def _full_layer_gpu(B, q, k, s, ctx):
    Bn, cap = s.shape
    nb = (cap + 7) // 8
    tok = torch.empty((Bn, 1, cap), device=DEV)
    blk = torch.empty((Bn, 1, nb), device=DEV)
    nblk = torch.empty((Bn, 1), dtype=torch.int32, device=DEV)
    B.csa2_index_full(q, k, s, ctx, blk, tok, nblk)
    pool = torch.empty((Bn, 1, 2048), dtype=torch.int32, device=DEV)
    B.csa2_topk(blk.view(Bn, nb), 2048, pool.view(Bn, 2048), n_valid=nblk.view(Bn))
    ps = torch.empty((Bn, 1, 16384), device=DEV)
    pp = torch.empty((Bn, 1, 16384), dtype=torch.int32, device=DEV)
    B.csa2_pool_gather(tok, pool, ctx, ps, pp)
    top = torch.empty((Bn, 1, 512), dtype=torch.int32, device=DEV)
    B.csa2_topk(ps.view(Bn, -1), 512, top.view(Bn, 512), cand_pos=pp.view(Bn, -1))
    torch.cuda.synchronize()
    return pool, top


@pytest.mark.parametrize("ctxs", [[20003, 4096, 100], [40000, 16384, 16385], [600, 7, 1]])
def test_full_layer_pool_and_topk_bitexact(B, ctxs):
    H, D = 16, 128
    cap = max(ctxs)
    q, k, s = _index_inputs(len(ctxs), cap, H, D, seed=sum(ctxs))
    ctx = torch.tensor(ctxs, dtype=torch.int64, device=DEV)
    pool, top = _full_layer_gpu(B, q, k, s, ctx)
    for b, c in enumerate(ctxs):
        r = oracle.full_layer(q[b, 0].cpu().numpy(), k[b].cpu().numpy(), s[b].cpu().numpy(), c)
        assert np.array_equal(pool[b, 0].cpu().numpy(), r["pool"])
        assert np.array_equal(top[b, 0].cpu().numpy(), r["top"])


# ----------------------------------------------------------------------------- fused Full-layer selection
def _full_select_check(B, q, k, s, ctx, q_pos=None, P=2048, K=512, oracle_rows=()):
    """csa2_full_select against csa2_topk -> csa2_pool_gather -> csa2_topk on the
    same scan outputs (bit for bit), and against the oracle on sampled rows."""
    Bn, Nq = q.shape[0], q.shape[1]
    cap = s.shape[1]
    nb = (cap + 7) // 8
    tok = torch.full((Bn, Nq, cap), -7.0, device=DEV)
    blk = torch.full((Bn, Nq, nb), -7.0, device=DEV)
    nblk = torch.zeros((Bn, Nq), dtype=torch.int32, device=DEV)
    B.csa2_index_full(q, k, s, ctx, blk, tok, nblk, q_pos=q_pos)
    pool_f = torch.full((Bn, Nq, P), -9, dtype=torch.int32, device=DEV)
    top_f = torch.full((Bn, Nq, K), -9, dtype=torch.int32, device=DEV)
    B.csa2_full_select(blk, nblk, tok, ctx, pool_f, top_f, q_pos=q_pos)
    pool_c = torch.empty((Bn, Nq, P), dtype=torch.int32, device=DEV)
    B.csa2_topk(blk.view(Bn * Nq, nb), P, pool_c.view(Bn * Nq, P), n_valid=nblk.view(-1))
    ps = torch.empty((Bn, Nq, 8 * P), device=DEV)
    pp = torch.empty((Bn, Nq, 8 * P), dtype=torch.int32, device=DEV)
    B.csa2_pool_gather(tok, pool_c, ctx, ps, pp, q_pos=q_pos)
    top_c = torch.empty((Bn, Nq, K), dtype=torch.int32, device=DEV)
    B.csa2_topk(ps.view(Bn * Nq, -1), K, top_c.view(Bn * Nq, K), cand_pos=pp.view(Bn * Nq, -1))
    torch.cuda.synchronize()
    assert torch.equal(pool_f, pool_c), "pool differs from the three-call composition"
    assert torch.equal(top_f, top_c), "top-k differs from the three-call composition"
    kn, sn, qn = k.cpu().numpy(), s.cpu().numpy(), q.cpu().numpy()
    for b, i in oracle_rows:
        V = int(ctx[b]) if q_pos is None else min(int(q_pos[b, i]) + 1, int(ctx[b]))
        r = oracle.full_layer(qn[b, i], kn[b], sn[b], V)
        if P == 2048 and K == 512:
            assert np.array_equal(pool_f[b, i].cpu().numpy(), r["pool"]), f"pool b={b} i={i}"
            assert np.array_equal(top_f[b, i].cpu().numpy(), r["top"]), f"top b={b} i={i}"


@pytest.mark.parametrize("ctxs,H,D", [([20003, 4096, 100, 1], 16, 128), ([16385, 16384, 7], 4, 64)])
def test_full_select_decode_rows(B, ctxs, H, D):
    cap = max(ctxs)
    q, k, s = _index_inputs(len(ctxs), cap, H, D, seed=sum(ctxs))
    ctx = torch.tensor(ctxs, dtype=torch.int64, device=DEV)
    _full_select_check(B, q, k, s, ctx, oracle_rows=[(b, 0) for b in range(len(ctxs))])


def test_full_select_largest_row(B):
    """131,072 positions: 16,384 blocks, the most one CTA holds."""
    cap = 131072
    q, k, s = _index_inputs(1, cap, 4, 32, seed=5)
    ctx = torch.tensor([cap], dtype=torch.int64, device=DEV)
    _full_select_check(B, q, k, s, ctx, oracle_rows=[(0, 0)])


def test_full_select_causal_queries(B):
    Bn, Nq, ctx0, H, D = 2, 64, 3000, 16, 128
    cap = ctx0 + Nq
    g = torch.Generator(device=DEV).manual_seed(9)
    k = torch.randint(-127, 128, (Bn, cap, H, D), generator=g, device=DEV, dtype=torch.int8)
    q = torch.randint(-127, 128, (Bn, Nq, H, D), generator=g, device=DEV, dtype=torch.int8)
    s = 0.5 + torch.rand((Bn, cap), generator=g, device=DEV)
    ctx = torch.tensor([cap, cap - 5], dtype=torch.int64, device=DEV)
    qpos = (ctx0 + torch.arange(Nq, device=DEV)).repeat(Bn, 1).contiguous()
    _full_select_check(B, q, k, s, ctx, q_pos=qpos, oracle_rows=[(0, 0), (1, 63), (1, 31)])


@pytest.mark.parametrize("levels", [1, 2, 5])
def test_full_select_tie_heavy(B, levels):
    """Coarse keys and unit scales: long runs of equal block and token scores
    (levels = 1: every score is zero), decided by position."""
    ctxs = [30000, 9001]
    cap = max(ctxs)
    g = torch.Generator(device=DEV).manual_seed(levels)
    k = torch.randint(0, levels, (2, cap, 4, 32), generator=g, device=DEV, dtype=torch.int8)
    q = torch.randint(-3, 4, (2, 1, 4, 32), generator=g, device=DEV, dtype=torch.int8)
    s = torch.ones((2, cap), device=DEV)
    ctx = torch.tensor(ctxs, dtype=torch.int64, device=DEV)
    _full_select_check(B, q, k, s, ctx, oracle_rows=[(0, 0), (1, 0)])


def test_full_select_other_sizes(B):
    """A smaller pool and a ragged k (the shapes the call accepts besides 2048 / 512)."""
    ctxs = [5000, 300]
    q, k, s = _index_inputs(2, 5000, 8, 64, seed=77)
    ctx = torch.tensor(ctxs, dtype=torch.int64, device=DEV)
    _full_select_check(B, q, k, s, ctx, P=64, K=100)
    _full_select_check(B, q, k, s, ctx, P=2048, K=4000)


def test_reindex_bitexact(B):
    ctxs = [30000, 20001, 9000]
    H, D = 16, 128
    cap = max(ctxs)
    q, k, s = _index_inputs(len(ctxs), cap, H, D, seed=3)
    q2 = torch.randint(-127, 128, q.shape, device=DEV, dtype=torch.int8,
                       generator=torch.Generator(device=DEV).manual_seed(4))
    ctx = torch.tensor(ctxs, dtype=torch.int64, device=DEV)
    kn, sn = k.cpu().numpy(), s.cpu().numpy()
    # the oracle's own pool (oracle output -> GPU input is allowed; not the reverse)
    pools = [oracle.full_layer(q[b, 0].cpu().numpy(), kn[b], sn[b], c)["pool"] for b, c in enumerate(ctxs)]
    pool = torch.from_numpy(np.stack(pools).astype(np.int32)).view(len(ctxs), 1, 2048).to(DEV)
    ps = torch.empty((len(ctxs), 1, 16384), device=DEV)
    pp = torch.empty((len(ctxs), 1, 16384), dtype=torch.int32, device=DEV)
    B.csa2_index_reindex(q2, k, s, pool, ctx, ps, pp)
    top = torch.empty((len(ctxs), 512), dtype=torch.int32, device=DEV)
    B.csa2_topk(ps.view(len(ctxs), -1), 512, top, cand_pos=pp.view(len(ctxs), -1))
    torch.cuda.synchronize()
    for b, c in enumerate(ctxs):
        ref_top, ppos, psc = oracle.reindex_layer(q2[b, 0].cpu().numpy(), kn[b], sn[b], pools[b], c)
        g_pos = pp[b, 0].cpu().numpy()
        valid = g_pos >= 0
        assert np.array_equal(g_pos[valid], ppos)
        assert np.array_equal(f32_bits(ps[b, 0].cpu().numpy()[valid]), f32_bits(psc))
        assert np.array_equal(top[b].cpu().numpy(), ref_top)


# ----------------------------------------------------------------------------- a8 attention
def _attention_case(B, Bn, ctx, C, Hq, K, n_win, seed, q_pos=None, Nq=1, drop=0, mx=False,
                    q_mul=None):
    """q_mul [Hq]: factors applied to Q per head (then rounded to bf16, the
    values both sides see)."""
    w = synth.scaled(synth.WORKLOADS["decoder_group1_b8_ctx128k"], B=Bn, ctx=ctx, C=C, Hq=Hq,
                     seed=seed)
    kv = torch.stack([synth.main_kv_bf16(w, b, 0, ctx, DEV) for b in range(Bn)])
    fp4 = torch.empty((Bn, ctx, C // 2), dtype=torch.uint8, device=DEV)
    sf = torch.empty((Bn, ctx, C // (32 if mx else 16)), dtype=torch.uint8, device=DEV)
    B.csa2_kv_append_fp4(kv, torch.zeros(Bn, dtype=torch.int64, device=DEV), fp4, sf, mx=mx)
    q = synth.main_q(w, 0, Nq, DEV)
    if q_mul is not None:
        q = (q.float() * q_mul.to(DEV).view(1, 1, Hq, 1)).to(torch.bfloat16)
    g = torch.Generator(device=DEV).manual_seed(seed)
    kk = min(K, ctx)
    top = torch.stack([torch.stack([torch.randperm(ctx, generator=g, device=DEV)[:kk].sort().values
                                    for _ in range(Nq)]) for _ in range(Bn)]).to(torch.int32)
    if kk < K:
        top = torch.cat([top, torch.full((Bn, Nq, K - kk), -1, dtype=torch.int32, device=DEV)], 2)
    if drop:
        top[:, :, ::drop] = -1
    rows = min(n_win, ctx) if q_pos is None else ctx
    swa = synth.swa_kv(w, 0, rows, DEV)
    pos0 = torch.full((Bn,), ctx - rows, dtype=torch.int64, device=DEV)
    out = torch.empty((Bn, Nq, Hq, C), device=DEV)
    scale = 1.0 / math.sqrt(C)
    B.csa2_sparse_attn_decode(q, fp4, sf, top.contiguous(), swa, pos0, out, scale, q_pos=q_pos,
                              n_win=n_win, mx=mx)
    torch.cuda.synchronize()
    kvn, qn, topn, swan = bf16_np(kv), bf16_np(q), top.cpu().numpy(), bf16_np(swa)
    for b in range(Bn):
        for i in range(Nq):
            p = (ctx - 1) if q_pos is None else int(q_pos[b, i])
            ref = oracle.sparse_attention(qn[b, i], lambda P: kvn[b][P], topn[b, i], swan[b], p,
                                          ctx - rows, scale, n_win,
                                          kv_format="mxfp4" if mx else "nvfp4")
            assert_attn_close(out[b, i].cpu().numpy(), ref, f"b={b} i={i}")


@pytest.mark.parametrize("Bn,ctx,C,Hq,K", [(3, 5000, 512, 64, 512), (2, 3000, 512, 64, 488),
                                           (2, 3000, 512, 64, 100),
                                           (2, 3000, 128, 8, 512),
                                           (1, 300, 512, 64, 512), (2, 100, 256, 16, 512),
                                           (1, 2000, 64, 3, 100)])
def test_sparse_attention_matches_oracle(B, Bn, ctx, C, Hq, K):
    _attention_case(B, Bn, ctx, C, Hq, K, 128, seed=ctx + C)


# The general kernel (shapes outside the tensor-core kernels'): keys split over a
# cluster of up to 8 CTAs, 8 heads per CTA, key rows staged in chunks of at
# most 96 KB. Odd pair counts per lane (96 channels), a partial last head
# group (13 heads), few keys (3 CTAs), the largest row (1024 channels: 48-key
# chunks, 11 of them per CTA at K = 4096), no window, masked slots and causal
# positions.
@pytest.mark.parametrize("Bn,ctx,C,Hq,K,n_win,drop", [(2, 3000, 96, 5, 300, 128, 0),
                                                      (2, 3000, 128, 13, 20, 128, 3),
                                                      (1, 6000, 1024, 2, 4096, 128, 5),
                                                      (3, 2000, 256, 8, 512, 0, 0),
                                                      (1, 2000, 32, 1, 512, 64, 2),
                                                      (2, 700, 128, 8, 1024, 100, 0)])
def test_sparse_attention_general_kernel(B, Bn, ctx, C, Hq, K, n_win, drop):
    _attention_case(B, Bn, ctx, C, Hq, K, n_win, seed=ctx + C + Hq, drop=drop)


def test_sparse_attention_general_kernel_causal_positions(B):
    ctx = 1300
    q_pos = torch.tensor([[1299, 700, 129, 128, 5, 0], [1000, 1001, 64, 3, 1250, 600]],
                         dtype=torch.int64, device=DEV)
    _attention_case(B, 2, ctx, 128, 8, 512, 128, seed=21, q_pos=q_pos, Nq=6, drop=4)
    _attention_case(B, 2, ctx, 128, 8, 512, 128, seed=22, q_pos=q_pos, Nq=6, mx=True)


def test_sparse_attention_skips_negative_indices_and_short_window(B):
    _attention_case(B, 2, 2500, 512, 64, 512, 128, seed=1, drop=3)
    _attention_case(B, 1, 50, 512, 64, 512, 128, seed=2)


def test_sparse_attention_window_only_and_no_keys(B):
    """K = 0: the window rows alone, on the split-key clusters, the per-row
    kernel and the general kernel; then every index masked and no window: no
    key at all, a zero output."""
    _attention_case(B, 2, 1000, 512, 64, 0, 128, seed=41)
    _attention_case(B, 1, 1000, 512, 64, 0, 128, seed=42, Nq=64)
    _attention_case(B, 2, 1000, 128, 8, 0, 100, seed=43)
    _attention_case(B, 2, 1000, 512, 64, 512, 0, seed=44, drop=1)
    _attention_case(B, 1, 1000, 512, 64, 512, 0, seed=45, Nq=64, drop=1)
    _attention_case(B, 2, 1000, 128, 8, 100, 0, seed=46, drop=1)


def test_sparse_attention_prefill_positions(B):
    ctx = 1200
    q_pos = torch.tensor([[1199, 1100, 600, 130]], dtype=torch.int64, device=DEV)
    _attention_case(B, 1, ctx, 512, 64, 512, 128, seed=3, q_pos=q_pos, Nq=4)


# The split-key cluster kernel divides the 64 heads of a row into groups with few
# rows: 16 heads per cluster up to 4 rows, 32 up to 9, all 64 beyond (clusters
# then loop over rows). Each grouping, with masked slots and short windows.
@pytest.mark.parametrize("Bn,Nq,drop,n_win", [(1, 1, 0, 128), (2, 2, 4, 128), (5, 1, 0, 128),
                                              (3, 3, 6, 100), (10, 1, 0, 128), (19, 1, 9, 64)])
def test_sparse_attention_head_groups(B, Bn, Nq, drop, n_win):
    _attention_case(B, Bn, 2600, 512, 64, 512, n_win, seed=31 * Bn + Nq, Nq=Nq, drop=drop)


# One CTA per query row: calls with 64 or more rows (and any call with more than
# 640 keys per row) take the per-row kernel; its window tiles, masked slots and
# online-softmax rescaling are covered here (the 20- to 40-row cases run the
# split-key kernel with all 64 heads per cluster).
@pytest.mark.parametrize("Bn,Nq,K,n_win,drop", [(20, 1, 512, 128, 0), (24, 1, 512, 128, 5),
                                                (2, 1, 1024, 128, 0), (20, 1, 512, 0, 0),
                                                (3, 8, 576, 64, 7)])
def test_sparse_attention_one_cta_per_row(B, Bn, Nq, K, n_win, drop):
    _attention_case(B, Bn, 3000, 512, 64, K, n_win, seed=7 * Bn + K + n_win, Nq=Nq, drop=drop)


def test_sparse_attention_one_cta_per_row_q_magnitudes(B):
    """Heads whose Q lies anywhere from 2^-60 to 2^66 times N(0, 1): softmax from
    uniform to one-hot, on the per-row kernel (40-row calls) and the split-key
    clusters (one row)."""
    mul = torch.tensor([2.0 ** e for e in range(-60, 68, 2)], dtype=torch.float32)
    _attention_case(B, 2, 3000, 512, 64, 512, 128, seed=13, Nq=40, q_mul=mul)
    _attention_case(B, 1, 3000, 512, 64, 512, 128, seed=14, drop=5, q_mul=mul)


def test_sparse_attention_one_cta_per_row_causal_positions(B):
    ctx = 1500
    pos = [1499, 1400, 900, 200, 127, 126, 64, 63, 5, 0] + list(range(1000, 1030))
    q_pos = torch.tensor([pos], dtype=torch.int64, device=DEV)
    _attention_case(B, 1, ctx, 512, 64, 512, 128, seed=11, q_pos=q_pos, Nq=len(pos))


# ----------------------------------------------------------------------------- a9 prefill scan
@pytest.mark.parametrize("Nq,ctx0,H,D", [(300, 5000, 16, 128), (129, 2048, 8, 128), (40, 777, 4, 64),
                                         (256, 7936, 16, 128), (2, 3000, 16, 128), (4, 5001, 16, 128),
                                         (7, 1234, 8, 128)])
def test_index_full_multi_query_tensor_core_path(B, Nq, ctx0, H, D):
    """Nq >= 2 runs the tcgen05 kind::i8 kernel (a few queries: speculative
    decode tokens): causal scores and block maxima must equal the oracle bit
    for bit, and equal the per-query dp4a scan."""
    Bn = 2
    cap = ctx0 + Nq
    g = torch.Generator(device=DEV).manual_seed(Nq + ctx0)
    k = torch.randint(-127, 128, (Bn, cap, H, D), generator=g, device=DEV, dtype=torch.int8)
    q = torch.randint(-127, 128, (Bn, Nq, H, D), generator=g, device=DEV, dtype=torch.int8)
    s = 0.5 + torch.rand((Bn, cap), generator=g, device=DEV)
    ctx = torch.tensor([cap, cap - 3], dtype=torch.int64, device=DEV)
    qpos = (ctx0 + torch.arange(Nq, device=DEV)).repeat(Bn, 1).contiguous()
    nb = (cap + 7) // 8
    blk = torch.full((Bn, Nq, nb), -7.0, device=DEV)
    tok = torch.full((Bn, Nq, cap), -7.0, device=DEV)
    nblk = torch.zeros((Bn, Nq), dtype=torch.int32, device=DEV)
    B.csa2_index_full(q, k, s, ctx, blk, tok, nblk, q_pos=qpos)
    # the same queries one at a time (Nq = 1 runs the dp4a scan kernel)
    blk1 = torch.full_like(blk, -7.0)
    tok1 = torch.full_like(tok, -7.0)
    nblk1 = torch.zeros_like(nblk)
    for i in range(Nq):
        b1 = torch.empty((Bn, 1, nb), device=DEV)
        t1 = torch.empty((Bn, 1, cap), device=DEV)
        n1 = torch.empty((Bn, 1), dtype=torch.int32, device=DEV)
        B.csa2_index_full(q[:, i:i + 1].contiguous(), k, s, ctx, b1, t1, n1,
                          q_pos=qpos[:, i:i + 1].contiguous())
        blk1[:, i] = b1[:, 0]
        tok1[:, i] = t1[:, 0]
        nblk1[:, i] = n1[:, 0]
    torch.cuda.synchronize()
    for b in range(Bn):
        for i in range(Nq):
            V = min(int(qpos[b, i]) + 1, int(ctx[b]))
            nv = (V + 7) // 8
            assert int(nblk[b, i]) == nv == int(nblk1[b, i])
            assert torch.equal(tok[b, i, :V], tok1[b, i, :V]), f"tok b={b} i={i}"
            assert torch.equal(blk[b, i, :nv], blk1[b, i, :nv]), f"blk b={b} i={i}"
            assert bool((tok[b, i, V:] == -7.0).all()) and bool((blk[b, i, nv:] == -7.0).all())
    kn, sn, qn = k.cpu().numpy(), s.cpu().numpy(), q.cpu().numpy()
    for b in range(Bn):
        for i in sorted({0, 1, Nq // 2, Nq - 1}):
            V = min(int(qpos[b, i]) + 1, int(ctx[b]))
            ref = oracle.index_scores(qn[b, i], kn[b, :V], sn[b, :V])
            assert np.array_equal(f32_bits(tok[b, i, :V]), f32_bits(ref))
            assert np.array_equal(f32_bits(blk[b, i, :(V + 7) // 8]), f32_bits(oracle.block_scores(ref, V)))


# ----------------------------------------------------------------------------- device-side status
def test_device_status_reports_a_bounded_wait_timeout(B):
    """A kernel whose wait nothing completes gives up at its bound, records it,
    and returns; the host reads the flag and the context stays usable."""
    B.device_status(clear=True)
    assert B.device_status() == 0
    B.selftest_wait_timeout(2000)
    assert B.device_status() == -7
    assert B.device_status(clear=True) == -7
    assert B.device_status() == 0
    score = torch.arange(100, device=DEV, dtype=torch.float32).view(1, 100)
    out = torch.empty((1, 10), dtype=torch.int32, device=DEV)
    B.csa2_topk(score, 10, out)
    assert out.cpu().tolist() == [list(range(90, 100))]


def test_workspace_error_word_attributes_a_timeout_to_its_call(B):
    """The error word at the start of a call's workspace: a kernel that gives up
    a bounded wait sets it (besides the library flag), another call's word on
    another stream stays clear, and a decode step clears its own word."""
    B.device_status(clear=True)
    ws_a = torch.zeros(256, dtype=torch.uint8, device=DEV)
    ws_b = torch.zeros(256, dtype=torch.uint8, device=DEV)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    assert B.lib.csa2_selftest_workspace_timeout(2000, B._ptr(ws_a), B._stream(s1)) == 0
    assert B.workspace_status(ws_a, stream=s1) == -7
    assert B.workspace_status(ws_b, stream=s2) == 0
    assert B.workspace_status(ws_a, clear=True, stream=s1) == -7
    assert B.workspace_status(ws_a, stream=s1) == 0
    assert B.device_status(clear=True) == -7          # the library flag saw it too
    # a decode step clears its word and leaves it clear when every wait completes
    from sparse_attention_fp4_kv_b200 import synth
    from sparse_attention_fp4_kv_b200.workload import DecodeWorkload
    wl = DecodeWorkload(synth.scaled(synth.WORKLOADS["decoder_stack20_b4_ctx1m"], B=2, ctx=9001), DEV)
    wl.stack.ws[:4].fill_(1)
    wl.step()
    assert B.workspace_status(wl.stack.ws) == 0
    assert B.device_status() == 0
