"""Seeded synthetic inputs for the CSA2 decode hot path.

This module only draws random tensors with the shapes and value distributions
of the workloads; it holds none of the method's arithmetic (no quantization,
no scoring, no selection, no attention). Both the CUDA path and the CPU oracle
consume the tensors it returns (the oracle after a copy to host memory).

All draws use ``torch.Generator`` objects seeded from (workload seed, tensor
id, layer, sequence), so a tensor can be re-drawn on its own. Values drawn on
different device types differ; a comparison always draws once and copies.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import torch

FULL, REINDEX, REUSE = 0, 1, 2

# Decoder layer schedule: five groups of four layers, the first 1 Full + 3
# Reuse, the other four 1 Reindex + 3 Reuse ("DeepSeek-V4.1-Flash: 890 Bytes
# Per Token, 437x Smaller KV Cache", CSA2 section).
DECODER_MODES = [FULL, REUSE, REUSE, REUSE] + [REINDEX, REUSE, REUSE, REUSE] * 4
# Encoder CSA2 layers: three groups of six, each 1 Full + 5 Reuse (same section).
ENCODER_MODES = ([FULL] + [REUSE] * 5) * 3


@dataclass
class Workload:
    name: str
    B: int                  # sequences
    ctx: int                # context length (tokens visible to the decode query)
    C: int                  # main-KV channels (= main Q head dim)
    Hq: int                 # main Q heads
    H_idx: int              # indexer heads
    D_idx: int              # indexer dims per head
    modes: List[int]        # per-layer CSA2 mode
    outlier_frac: float     # fraction of main-KV channels scaled up
    outlier_mult: float
    seed: int
    n_win: int = 128
    planted_blocks: int = 0  # blocks per sequence with keys correlated to the Reindex Q
    planted_corr: float = 0.9
    full_q_corr: float = 0.7  # correlation of the pool-building Full Q with the Reindex Q
    n_new: int = 1            # tokens appended this step (decode: 1)
    prefill_queries: int = 0  # >0: chunked-prefill workload with this many queries
    extra: dict = field(default_factory=dict)

    @property
    def n_layers(self) -> int:
        return len(self.modes)

    @property
    def HD(self) -> int:
        return self.H_idx * self.D_idx


WORKLOADS = {
    # Single Full layer, batch 1, 4K context, small dims.
    "full_b1_ctx4k": Workload("full_b1_ctx4k", B=1, ctx=4096, C=128, Hq=8, H_idx=4, D_idx=64,
                              modes=[FULL], outlier_frac=0.02, outlier_mult=8.0, seed=0),
    # First decoder group (Full + 3 Reuse), batch 8, 128K context.
    "decoder_group1_b8_ctx128k": Workload("decoder_group1_b8_ctx128k", B=8, ctx=131072, C=512,
                                          Hq=64, H_idx=16, D_idx=128,
                                          modes=[FULL, REUSE, REUSE, REUSE],
                                          outlier_frac=0.01, outlier_mult=16.0, seed=1),
    # Reindex group (Reindex + 3 Reuse) over a pool built by a Full layer, batch 32, 256K.
    "reindex_group_b32_ctx256k": Workload("reindex_group_b32_ctx256k", B=32, ctx=262144, C=512,
                                          Hq=64, H_idx=16, D_idx=128,
                                          modes=[REINDEX, REUSE, REUSE, REUSE],
                                          outlier_frac=0.01, outlier_mult=16.0, seed=2,
                                          planted_blocks=8),
    # Full 20-layer decoder attention stack, batch 4, 1M context.
    "decoder_stack20_b4_ctx1m": Workload("decoder_stack20_b4_ctx1m", B=4, ctx=1048576, C=512,
                                         Hq=64, H_idx=16, D_idx=128, modes=list(DECODER_MODES),
                                         outlier_frac=0.01, outlier_mult=16.0, seed=3),
    # The same stack at 256K context: its Reindex, selection and attention
    # launches are those of the 1M stack (the pool is 2,048 blocks either way)
    # with a quarter of the scan; small enough on the device for multi-pass
    # profiler captures.
    "decoder_stack20_b4_ctx256k": Workload("decoder_stack20_b4_ctx256k", B=4, ctx=262144, C=512,
                                           Hq=64, H_idx=16, D_idx=128, modes=list(DECODER_MODES),
                                           outlier_frac=0.01, outlier_mult=16.0, seed=7),
    # The 18 CSA2 encoder layers of a decode step, batch 4, 1M context.
    "encoder_stack18_b4_ctx1m": Workload("encoder_stack18_b4_ctx1m", B=4, ctx=1048576, C=512,
                                         Hq=64, H_idx=16, D_idx=128, modes=list(ENCODER_MODES),
                                         outlier_frac=0.01, outlier_mult=16.0, seed=5),
    # Multi-token decode (speculative / MTP tokens): 4 new tokens per sequence
    # appended to a 1M context, each a causal query of one Full layer.
    "decode_mtp4_b4_ctx1m": Workload("decode_mtp4_b4_ctx1m", B=4, ctx=1048576 + 4, C=512, Hq=64,
                                     H_idx=16, D_idx=128, modes=[FULL], outlier_frac=0.01,
                                     outlier_mult=16.0, seed=6, n_new=4, prefill_queries=4),
    # Chunked prefill: 4096 new tokens appended to a 65536-token context.
    "prefill_4096_at_64k": Workload("prefill_4096_at_64k", B=1, ctx=65536 + 4096, C=512, Hq=64,
                                    H_idx=16, D_idx=128, modes=[FULL], outlier_frac=0.01,
                                    outlier_mult=16.0, seed=4, n_new=4096,
                                    prefill_queries=4096),
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    d = dict(w.__dict__)
    d.update(kw)
    d["modes"] = list(d["modes"])
    d["extra"] = dict(d["extra"])
    return Workload(**d)


# Tensor ids for seeding.
_T_KV, _T_KIDX, _T_KSCALE, _T_Q, _T_SWA, _T_QIDX, _T_OUTL, _T_PLANT, _T_PLANTU, _T_FULLQ = range(10)


def _gen(w: Workload, tensor: int, a: int = 0, b: int = 0, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    key = ((w.seed * 1_000_003 + tensor) * 1_000_033 + a) * 1_000_037 + b
    g.manual_seed(key % (1 << 63))
    return g


def outlier_channels(w: Workload) -> torch.Tensor:
    """Main-KV channels scaled by outlier_mult: round(frac * C) of them, by a
    seeded permutation (same channels for every token and sequence)."""
    n = int(round(w.outlier_frac * w.C))
    perm = torch.randperm(w.C, generator=_gen(w, _T_OUTL))
    return perm[:n].sort().values


def main_kv_bf16(w: Workload, b: int, t0: int, t1: int, device) -> torch.Tensor:
    """bf16 main-KV rows [t1 - t0, C] of sequence b, before quantization:
    N(0, 1) with the outlier channels multiplied. Rows are drawn in chunks of
    8192 tokens so any range can be re-drawn alone."""
    CH = 8192
    out = torch.empty((t1 - t0, w.C), dtype=torch.bfloat16, device=device)
    oc = outlier_channels(w).to(device)
    c0 = t0 // CH
    while c0 * CH < t1:
        g = _gen(w, _T_KV, b, c0, device=str(torch.device(device).type))
        x = torch.randn((CH, w.C), generator=g, device=device, dtype=torch.float32)
        if oc.numel():
            x[:, oc] *= w.outlier_mult
        lo, hi = max(t0, c0 * CH), min(t1, (c0 + 1) * CH)
        out[lo - t0:hi - t0] = x[lo - c0 * CH:hi - c0 * CH].to(torch.bfloat16)
        c0 += 1
    return out


def indexer_keys(w: Workload, b: int, n: int, device) -> torch.Tensor:
    """int8 indexer keys [n, H_idx, D_idx] of sequence b, uniform in [-127, 127]."""
    g = _gen(w, _T_KIDX, b, device=str(torch.device(device).type))
    return torch.randint(-127, 128, (n, w.H_idx, w.D_idx), generator=g, device=device,
                         dtype=torch.int8)


def indexer_key_scale(w: Workload, b: int, n: int, device) -> torch.Tensor:
    """fp32 per-token indexer key scale, U(0.5, 1.5)."""
    g = _gen(w, _T_KSCALE, b, device=str(torch.device(device).type))
    return 0.5 + torch.rand((n,), generator=g, device=device, dtype=torch.float32)


def main_q(w: Workload, layer: int, nq: int, device) -> torch.Tensor:
    """bf16 main Q [B, nq, Hq, C], N(0, 1)."""
    g = _gen(w, _T_Q, layer, device=str(torch.device(device).type))
    return torch.randn((w.B, nq, w.Hq, w.C), generator=g, device=device).to(torch.bfloat16)


def swa_kv(w: Workload, layer: int, rows: int, device) -> torch.Tensor:
    """bf16 per-layer sliding-window KV [B, rows, C], N(0, 1)."""
    g = _gen(w, _T_SWA, layer, device=str(torch.device(device).type))
    return torch.randn((w.B, rows, w.C), generator=g, device=device).to(torch.bfloat16)


def indexer_q(w: Workload, layer: int, nq: int, device) -> torch.Tensor:
    """int8 indexer Q [B, nq, H_idx, D_idx], uniform in [-127, 127]."""
    g = _gen(w, _T_QIDX, layer, device=str(torch.device(device).type))
    return torch.randint(-127, 128, (w.B, nq, w.H_idx, w.D_idx), generator=g, device=device,
                         dtype=torch.int8)


def _mix_int8(a: torch.Tensor, corr: float, g: torch.Generator) -> torch.Tensor:
    """clip(round(corr * a + sqrt(1 - corr^2) * u)) with u a fresh uniform int8
    tensor: an int8 tensor correlated `corr` with a."""
    u = torch.randint(-127, 128, a.shape, generator=g, device=a.device, dtype=torch.int8)
    y = corr * a.float() + (1.0 - corr * corr) ** 0.5 * u.float()
    return y.round().clamp(-127, 127).to(torch.int8)


def pool_builder_q(w: Workload, q_reindex: torch.Tensor) -> torch.Tensor:
    """Indexer Q of the Full layer that builds the pool a Reindex workload
    starts from: correlated full_q_corr with the Reindex layer's Q."""
    g = _gen(w, _T_FULLQ, device=str(q_reindex.device.type))
    return _mix_int8(q_reindex, w.full_q_corr, g)


def planted_blocks(w: Workload, b: int) -> torch.Tensor:
    """Block ids (sorted) of the planted blocks of sequence b."""
    nblk = (w.ctx + 7) // 8
    g = _gen(w, _T_PLANT, b)
    return torch.randperm(nblk, generator=g)[: w.planted_blocks].sort().values


def plant(w: Workload, b: int, k_idx_b: torch.Tensor, q_reindex_b: torch.Tensor) -> torch.Tensor:
    """Overwrite the indexer keys of sequence b's planted blocks with keys
    correlated planted_corr with the Reindex query (per head and dim).
    k_idx_b: [ctx, H, D] int8 (modified in place); q_reindex_b: [H, D]."""
    blocks = planted_blocks(w, b)
    g = _gen(w, _T_PLANTU, b, device=str(k_idx_b.device.type))
    for j in blocks.tolist():
        t0, t1 = 8 * j, min(8 * j + 8, k_idx_b.shape[0])
        base = q_reindex_b.unsqueeze(0).expand(t1 - t0, -1, -1)
        k_idx_b[t0:t1] = _mix_int8(base.contiguous(), w.planted_corr, g)
    return blocks
