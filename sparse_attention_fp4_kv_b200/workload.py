"""Device-resident decode workloads: the caches, per-layer tensors and output
buffers of one CSA2 decode step, laid out in HBM for libcsa2.

HBM layout (per workload; B sequences, capacity = context length):
  k_idx    int8 [B][ctx][H_idx][D_idx]   indexer keys (2 KB per token at 16x128)
  k_scale  fp32 [B][ctx]
  kv_fp4   uint8 [B][ctx][C/2]           E2M1 codes, two per byte
  kv_sf    uint8 [B][ctx][C/16]          E4M3 scales
  per layer: q bf16 [B][1][Hq][C], swa bf16 [B][128][C], out fp32 [B][1][Hq][C],
             q_idx int8 [B][1][H_idx][D_idx] and topk int32 [B][512] (Full/Reindex)
  pool int32 [B][2048], workspace for the decode step.
The FP4 cache is filled with libcsa2's own append kernel from the seeded bf16
rows; the last position (ctx - 1) is the token each decode step appends.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import binding as csa2
from . import synth


class DecodeWorkload:
    def __init__(self, w: synth.Workload, device="cuda", keep_kv_bf16: bool = False):
        self.w = w
        B, ctx, C, Hq, H, D = w.B, w.ctx, w.C, w.Hq, w.H_idx, w.D_idx
        dev = torch.device(device)
        self.device = dev
        self.cap = ctx
        self.k_idx = torch.empty((B, ctx, H, D), dtype=torch.int8, device=dev)
        self.k_scale = torch.empty((B, ctx), dtype=torch.float32, device=dev)
        for b in range(B):
            self.k_idx[b] = synth.indexer_keys(w, b, ctx, dev)
            self.k_scale[b] = synth.indexer_key_scale(w, b, ctx, dev)
        self.kv_fp4 = torch.empty((B, ctx, C // 2), dtype=torch.uint8, device=dev)
        self.kv_sf = torch.empty((B, ctx, C // 16), dtype=torch.uint8, device=dev)
        self.kv_bf16: Optional[torch.Tensor] = None
        if keep_kv_bf16:
            self.kv_bf16 = torch.empty((B, ctx, C), dtype=torch.bfloat16, device=dev)
        zero = torch.zeros(1, dtype=torch.int64, device=dev)
        chunk = 65536
        for b in range(B):
            for t0 in range(0, ctx - 1, chunk):
                t1 = min(ctx - 1, t0 + chunk)
                rows = synth.main_kv_bf16(w, b, t0, t1, dev)
                if self.kv_bf16 is not None:
                    self.kv_bf16[b, t0:t1] = rows
                csa2.csa2_kv_append_fp4(rows.unsqueeze(0).contiguous(), zero + t0,
                                        self.kv_fp4[b:b + 1], self.kv_sf[b:b + 1])
        # the token this decode step appends (position ctx - 1)
        self.kv_new = torch.stack([synth.main_kv_bf16(w, b, ctx - 1, ctx, dev)[0] for b in range(B)])
        if self.kv_bf16 is not None:
            self.kv_bf16[:, ctx - 1] = self.kv_new
        self.ctx_len = torch.full((B,), ctx, dtype=torch.int64, device=dev)
        rows = min(w.n_win, ctx)
        self.swa_rows = rows
        self.swa_pos0 = torch.full((B,), ctx - rows, dtype=torch.int64, device=dev)
        L = w.n_layers
        self.modes = list(w.modes)
        self.q = [synth.main_q(w, l, 1, dev) for l in range(L)]
        self.swa = [synth.swa_kv(w, l, rows, dev) for l in range(L)]
        self.out = [torch.empty((B, 1, Hq, C), dtype=torch.float32, device=dev) for _ in range(L)]
        self.q_idx = [synth.indexer_q(w, l, 1, dev) if m != synth.REUSE else None
                      for l, m in enumerate(self.modes)]
        self.topk = [torch.empty((B, csa2.TOPK), dtype=torch.int32, device=dev)
                     if m != synth.REUSE else None for m in self.modes]
        self.pool = torch.empty((B, csa2.POOL_BLOCKS), dtype=torch.int32, device=dev)
        self.scale = 1.0 / math.sqrt(C)
        self.pool_ready = False
        self.planted = None
        self.pool_q_idx = None
        if self.modes[0] == synth.REINDEX:
            self._build_pool()
        self.stack = csa2.DecodeStack(self.modes, self.q_idx, self.q, self.swa, self.out,
                                      self.topk, self.k_idx, self.k_scale, self.kv_fp4, self.kv_sf,
                                      self.ctx_len, self.swa_pos0, self.pool, self.scale,
                                      kv_new=self.kv_new, pool_ready=self.pool_ready)

    def _build_pool(self):
        """A Reindex group starts from the pool of a preceding Full layer: plant
        the correlated blocks, then run that Full layer once (set-up)."""
        w = self.w
        q_r = self.q_idx[0]
        self.planted = [synth.plant(w, b, self.k_idx[b], q_r[b, 0]) if w.planted_blocks else None
                        for b in range(w.B)]
        self.pool_q_idx = synth.pool_builder_q(w, q_r)
        out = torch.empty_like(self.out[0])
        topk = torch.empty_like(self.topk[0])
        setup = csa2.DecodeStack([synth.FULL], [self.pool_q_idx], [self.q[0]], [self.swa[0]],
                                 [out], [topk], self.k_idx, self.k_scale, self.kv_fp4, self.kv_sf,
                                 self.ctx_len, self.swa_pos0, self.pool, self.scale,
                                 kv_new=self.kv_new)
        setup()
        torch.cuda.synchronize(self.device)
        self.pool_ready = True

    def step(self, stream=None):
        """One decode step: append the new token, then every layer of the stack."""
        self.stack(stream)

    def capture_step_graph(self):
        """One decode step (the csa2_decode_stack call) captured as a CUDA graph
        on a side stream; replay() runs the step again on the same buffers.
        Call a step first, outside the capture (one-time kernel set-up)."""
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.graph(graph, stream=side):
            self.stack(side)
        torch.cuda.current_stream(self.device).wait_stream(side)
        return graph

    def io_set(self):
        """A second set of the per-step inputs (new KV row, main and indexer Q)
        and outputs (attention outputs, top-k indices) with its own decode
        stack over the same caches, pool and window rows, so that one step's
        host copies can overlap another step's compute. Returns (stack,
        inputs, outputs)."""
        kv_new = self.kv_new.clone()
        q = [t.clone() for t in self.q]
        q_idx = [t.clone() if t is not None else None for t in self.q_idx]
        out = [torch.empty_like(t) for t in self.out]
        topk = [torch.empty_like(t) if t is not None else None for t in self.topk]
        stack = csa2.DecodeStack(self.modes, q_idx, q, self.swa, out, topk, self.k_idx,
                                 self.k_scale, self.kv_fp4, self.kv_sf, self.ctx_len, self.swa_pos0,
                                 self.pool, self.scale, kv_new=kv_new, pool_ready=self.pool_ready)
        inputs = [kv_new] + q + [t for t in q_idx if t is not None]
        outputs = out + [t for t in topk if t is not None]
        return stack, inputs, outputs

    def io_tensors(self):
        """The per-step inputs and outputs of the workload's own stack (same
        order as io_set)."""
        inputs = [self.kv_new] + list(self.q) + [t for t in self.q_idx if t is not None]
        outputs = list(self.out) + [t for t in self.topk if t is not None]
        return inputs, outputs

    def launches_per_step(self) -> int:
        """libcsa2 kernels one step launches: the step-begin kernel (the new
        rows' append and the zeroing of the step's counters), then per Full layer
        the scan and one selection of the pool and its top tokens; per Reindex
        layer the rescoring and the token selection. Attention: one
        kernel per layer group (a Full or Reindex layer and the Reuse layers
        after it, at most ATTN_GROUP_MAX layers per kernel) where the
        tensor-core cluster kernel takes the shape, else one per layer. A
        selection is one kernel for rows of at most TOPK_SHORT_ROW candidates,
        else two (compaction + finish)."""
        def sel(n):
            return 1 if n <= csa2.TOPK_SHORT_ROW else 2
        w = self.w
        pooled = csa2.POOL_BLOCKS * csa2.BLOCK_TOKENS
        grouped = w.C == 512 and w.Hq == 64 and w.B < csa2.ATTN_ROWS_MIN
        n = 1
        run = 0  # layers in the current attention launch
        for m in self.modes:
            n += {synth.FULL: 2, synth.REINDEX: 1 + sel(pooled), synth.REUSE: 0}[m]
            if grouped and m == synth.REUSE and 0 < run < csa2.ATTN_GROUP_MAX:
                run += 1
            else:
                n += 1
                run = 1
        return n

    # ---- algorithmic bytes of one step (what the method must move)
    def step_bytes(self) -> dict:
        w = self.w
        B, ctx, C, Hq = w.B, w.ctx, w.C, w.Hq
        HD = w.H_idx * w.D_idx
        scan = attn = reindex = 0
        nblk = (ctx + 7) // 8
        for m in self.modes:
            if m == synth.FULL:
                scan += B * ctx * (HD + 4) + B * ctx * 4 + B * nblk * 4   # keys+scales, scores
            elif m == synth.REINDEX:
                pooled = min(2048, nblk) * 8
                reindex += B * pooled * (HD + 4)
            attn += B * (512 * (C // 2 + C // 16) + self.swa_rows * C * 2 + Hq * C * 2 + Hq * C * 4)
        append = B * (C * 2 + C // 2 + C // 16)
        return dict(scan=scan, reindex=reindex, attn=attn, append=append,
                    total=scan + reindex + attn + append)


class PrefillWorkload:
    """Chunked prefill of one Full layer: n_new tokens appended to a context
    of ctx - n_new, each new token a query that sees positions <= its own.

    One step = FP4 append of the n_new rows, causal indexer scoring of every
    query against every visible key (tensor-core kernel), per-query pool of
    2048 blocks and top-512, then attention of each query over its 512 rows
    plus its own 128-token window. Buffers per sequence: token scores
    [n_new][ctx] fp32 (1.1 GB at 4096 x 69632), block scores, pools, pooled
    scores/positions, indices and outputs [n_new][64][512] fp32."""

    def __init__(self, w: synth.Workload, device="cuda", keep_kv_bf16: bool = False):
        self.w = w
        B, cap, C, Hq, H, D, n = w.B, w.ctx, w.C, w.Hq, w.H_idx, w.D_idx, w.n_new
        dev = torch.device(device)
        self.device = dev
        self.ctx0 = cap - n
        self.k_idx = torch.empty((B, cap, H, D), dtype=torch.int8, device=dev)
        self.k_scale = torch.empty((B, cap), dtype=torch.float32, device=dev)
        for b in range(B):
            self.k_idx[b] = synth.indexer_keys(w, b, cap, dev)
            self.k_scale[b] = synth.indexer_key_scale(w, b, cap, dev)
        self.kv_fp4 = torch.zeros((B, cap, C // 2), dtype=torch.uint8, device=dev)
        self.kv_sf = torch.zeros((B, cap, C // 16), dtype=torch.uint8, device=dev)
        self.kv_bf16 = (torch.empty((B, cap, C), dtype=torch.bfloat16, device=dev)
                        if keep_kv_bf16 else None)
        zero = torch.zeros(1, dtype=torch.int64, device=dev)
        chunk = 65536
        for b in range(B):
            for t0 in range(0, self.ctx0, chunk):
                t1 = min(self.ctx0, t0 + chunk)
                rows = synth.main_kv_bf16(w, b, t0, t1, dev)
                if self.kv_bf16 is not None:
                    self.kv_bf16[b, t0:t1] = rows
                csa2.csa2_kv_append_fp4(rows.unsqueeze(0).contiguous(), zero + t0,
                                        self.kv_fp4[b:b + 1], self.kv_sf[b:b + 1])
        self.kv_new = torch.stack([synth.main_kv_bf16(w, b, self.ctx0, cap, dev) for b in range(B)])
        if self.kv_bf16 is not None:
            self.kv_bf16[:, self.ctx0:] = self.kv_new
        self.start = torch.full((B,), self.ctx0, dtype=torch.int64, device=dev)
        self.ctx_len = torch.full((B,), cap, dtype=torch.int64, device=dev)
        self.q_pos = (self.ctx0 + torch.arange(n, device=dev, dtype=torch.int64)).repeat(B, 1).contiguous()
        self.q_idx = synth.indexer_q(w, 0, n, dev)
        self.q = synth.main_q(w, 0, n, dev)
        lo = max(0, self.ctx0 - (w.n_win - 1))
        self.swa_rows = cap - lo
        self.swa = synth.swa_kv(w, 0, self.swa_rows, dev)
        self.swa_pos0 = torch.full((B,), lo, dtype=torch.int64, device=dev)
        nb = (cap + 7) // 8
        self.tok = torch.empty((B, n, cap), dtype=torch.float32, device=dev)
        self.blk = torch.empty((B, n, nb), dtype=torch.float32, device=dev)
        self.nblk = torch.empty((B, n), dtype=torch.int32, device=dev)
        self.pool = torch.empty((B, n, csa2.POOL_BLOCKS), dtype=torch.int32, device=dev)
        P8 = csa2.POOL_BLOCKS * csa2.BLOCK_TOKENS
        # one fused selection kernel when a row fits in shared memory, else
        # block top-k, pool gather and token top-k
        self.fused_select = nb <= csa2.FULL_SELECT_MAX
        if not self.fused_select:
            self.pscore = torch.empty((B, n, P8), dtype=torch.float32, device=dev)
            self.ppos = torch.empty((B, n, P8), dtype=torch.int32, device=dev)
        self.top = torch.empty((B, n, csa2.TOPK), dtype=torch.int32, device=dev)
        self.out = torch.empty((B, n, Hq, C), dtype=torch.float32, device=dev)
        self.scale = 1.0 / math.sqrt(C)

    def step(self, stream=None, scan_events=None):
        w = self.w
        B, n = w.B, w.n_new
        csa2.csa2_kv_append_fp4(self.kv_new, self.start, self.kv_fp4, self.kv_sf, stream=stream)
        if scan_events is not None:
            scan_events[0].record(stream or torch.cuda.current_stream())
        csa2.csa2_index_full(self.q_idx, self.k_idx, self.k_scale, self.ctx_len, self.blk, self.tok,
                             self.nblk, q_pos=self.q_pos, stream=stream)
        if scan_events is not None:
            scan_events[1].record(stream or torch.cuda.current_stream())
        if self.fused_select:
            csa2.csa2_full_select(self.blk, self.nblk, self.tok, self.ctx_len, self.pool, self.top,
                                  q_pos=self.q_pos, stream=stream)
        else:
            csa2.csa2_topk(self.blk.view(B * n, -1), csa2.POOL_BLOCKS, self.pool.view(B * n, -1),
                           n_valid=self.nblk.view(-1), stream=stream)
            csa2.csa2_pool_gather(self.tok, self.pool, self.ctx_len, self.pscore, self.ppos,
                                  q_pos=self.q_pos, stream=stream)
            csa2.csa2_topk(self.pscore.view(B * n, -1), csa2.TOPK, self.top.view(B * n, -1),
                           cand_pos=self.ppos.view(B * n, -1), stream=stream)
        csa2.csa2_sparse_attn_decode(self.q, self.kv_fp4, self.kv_sf, self.top, self.swa,
                                     self.swa_pos0, self.out, self.scale, q_pos=self.q_pos,
                                     stream=stream)

    def launches_per_step(self) -> int:
        """append, scan, selection (one fused kernel, or three), attention."""
        return 4 if self.fused_select else 6

    def index_ops(self) -> int:
        """int8 multiply-adds x 2 of the causal scoring (every query x every
        visible key x H*D)."""
        w = self.w
        vis = sum(min(self.ctx0 + i + 1, w.ctx) for i in range(w.n_new))
        return 2 * w.B * vis * w.H_idx * w.D_idx
