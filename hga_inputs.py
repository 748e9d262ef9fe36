"""Seeded synthetic inputs for one routed-HGA attention layer.

This module only draws random numbers and plants structure (per-chunk key
offsets, needle groups).  It holds none of the method's arithmetic, so both the
CUDA path and the CPU oracle can be fed from it without sharing code.

Workloads (shapes of the Qwen3-8B attention layer: 32 query heads, 8 KV heads,
head dim 128; chunk 64, group 8, query block 64 as in "Long-Context
Fine-Tuning with Limited VRAM", pith.science free-parameter ledger and
Figure 1 caption; segment 2048 tokens as the TBPTT segment length there):

* ``tiny_f32``   1 x (4 q / 1 kv) heads, 1024 history + 256 segment tokens,
                 top-4 chunks / top-8 groups, float32, chunk offsets of scale 1.
* ``ctx4k``      4096 context = 2048 history + 2048 segment, top-16 / top-64, bf16.
* ``ctx16k``     16384 context = 14336 history + 2048 segment, top-16 / top-64, bf16.
* ``ctx8k``, ``ctx12k``  the same layer at history 6144 / 10240 (earlier segment positions of
                 the 16K sequence; ``ctx4k`` is the one at history 2048).
* ``ctx16k_kc8``, ``ctx16k_kc32``  the 16K layer with routing budgets 8 / 32 and 32 / 128
                 (the pages' sweep of the routed chunk count from 8 to 32).
* ``ctx131k``    131072 context = 129024 history + 2048 segment, top-32 / top-128,
                 bf16, forward only, 64 planted needle groups.
* ``ctx16k_b4``  the 16K layer at batch 4 (tiered-history workload shape).

Value distributions: Q, V, dO ~ N(0, 1); K = N(0, 1) + s * o_c where o_c ~ N(0, I)
is one offset per (batch, KV head, 64-token chunk) of the context (history
and segment alike) and s is the workload's offset scale.  Tensors are drawn in
float32 on the CPU from a ``torch.Generator`` seeded with ``seed`` and then
rounded (round-to-nearest-even) to the workload dtype, so every consumer sees
identical values.

Needles: for each of ``needles`` distinct (KV head, query block) targets a
random unit direction u is drawn; ``needle_q`` * u is added to every query of
the target block in the KV head's query heads, and ``needle_k`` * u to the 8
keys of one randomly chosen history group (distinct groups).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    hist_len: int
    seg_len: int
    top_chunks: int
    top_groups: int
    dtype: str                 # "f32" | "bf16"
    offset_scale: float
    chunk: int = 64
    group: int = 8
    qblock: int = 64
    backward: bool = True
    needles: int = 0
    needle_q: float = 1.0
    needle_k: float = 32.0
    n_sink: int = 0            # sink-window tokens at the start of the history (multiple of chunk)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def nblk(self) -> int:
        return self.seg_len // self.qblock

    @property
    def nch(self) -> int:
        return self.hist_len // self.chunk

    @property
    def ngr(self) -> int:
        return self.hist_len // self.group

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 4, 1, 128, 1024, 256, 4, 8, "f32", 1.0),
    "ctx4k": Workload("ctx4k", 1, 32, 8, 128, 2048, 2048, 16, 64, "bf16", 0.5),
    "ctx16k": Workload("ctx16k", 1, 32, 8, 128, 14336, 2048, 16, 64, "bf16", 0.5),
    # the 16K layer's earlier segment positions (history 6144 and 10240; 2048 is ctx4k)
    "ctx8k": Workload("ctx8k", 1, 32, 8, 128, 6144, 2048, 16, 64, "bf16", 0.5),
    "ctx12k": Workload("ctx12k", 1, 32, 8, 128, 10240, 2048, 16, 64, "bf16", 0.5),
    # routing-budget sweep of the 16K layer (k_c = 8 and 32 with k_g = 4 k_c; 16 / 64 is ctx16k)
    "ctx16k_kc8": Workload("ctx16k_kc8", 1, 32, 8, 128, 14336, 2048, 8, 32, "bf16", 0.5),
    "ctx16k_kc32": Workload("ctx16k_kc32", 1, 32, 8, 128, 14336, 2048, 32, 128, "bf16", 0.5),
    "ctx131k": Workload("ctx131k", 1, 32, 8, 128, 129024, 2048, 32, 128, "bf16", 0.5,
                        backward=False, needles=64),
    "ctx16k_b4": Workload("ctx16k_b4", 4, 32, 8, 128, 14336, 2048, 16, 64, "bf16", 0.5),
}


def make_inputs(w: Workload, seed: int = 0, device: str | torch.device = "cpu") -> dict:
    """Draw q [B,Hq,S,D], k_hist/v_hist [B,Hkv,H,D], k_seg/v_seg [B,Hkv,S,D], d_o [B,Hq,S,D].

    Returns a dict of tensors (dtype ``w.torch_dtype``) plus ``needles``: a long tensor
    [n, 3] of (kv head, query block, history group) for planted needles (batch 0)."""
    g = torch.Generator().manual_seed(int(seed))
    B, Hq, Hkv, D, H, S = w.B, w.Hq, w.Hkv, w.D, w.hist_len, w.seg_len
    C = w.chunk

    def normal(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32)

    q = normal(B, Hq, S, D)
    # one offset per (b, kv head, chunk) of the whole context [history | segment]
    n_ctx_chunks = (H + S + C - 1) // C
    offs = normal(B, Hkv, n_ctx_chunks, D) * w.offset_scale
    per_tok = offs.repeat_interleave(C, dim=2)[:, :, : H + S]
    k_hist = normal(B, Hkv, H, D) + per_tok[:, :, :H]
    k_seg = normal(B, Hkv, S, D) + per_tok[:, :, H:]
    v_hist = normal(B, Hkv, H, D)
    v_seg = normal(B, Hkv, S, D)
    d_o = normal(B, Hq, S, D)

    needles = torch.zeros(0, 3, dtype=torch.long)
    if w.needles:
        G = Hq // Hkv
        n = w.needles
        targets = torch.randperm(Hkv * w.nblk, generator=g)[:n]
        groups = torch.randperm(w.ngr, generator=g)[:n]
        dirs = normal(n, D)
        dirs = dirs / dirs.norm(dim=1, keepdim=True)
        rows = []
        for i in range(n):
            kh, blk = int(targets[i]) // w.nblk, int(targets[i]) % w.nblk
            j = int(groups[i])
            q[0, kh * G:(kh + 1) * G, blk * w.qblock:(blk + 1) * w.qblock] += w.needle_q * dirs[i]
            k_hist[0, kh, j * w.group:(j + 1) * w.group] += w.needle_k * dirs[i]
            rows.append((kh, blk, j))
        needles = torch.tensor(rows, dtype=torch.long)

    dt = w.torch_dtype
    out = dict(q=q, k_hist=k_hist, v_hist=v_hist, k_seg=k_seg, v_seg=v_seg, d_o=d_o)
    out = {k: v.to(dt).contiguous().to(device) for k, v in out.items()}
    out["needles"] = needles
    return out


def prev_block_q(w: Workload, seed: int) -> torch.Tensor:
    """The previous segment's last query block [B, Hq, qblock, D] for strictly causal routing: one
    query block drawn like ``make_inputs`` queries, with its own seed (seed + 100)."""
    return make_inputs(w.with_(hist_len=w.chunk, seg_len=w.qblock, n_sink=0, needles=0), seed + 100)["q"]


def sample_ids(n_total: int, n: int, seed: int) -> torch.Tensor:
    """``n`` distinct ids in [0, n_total), sorted, from a seeded generator (for sampled checks)."""
    g = torch.Generator().manual_seed(int(seed) + 7919)
    n = min(n, n_total)
    return torch.randperm(n_total, generator=g)[:n].sort().values


# Small and edge-case shapes used by the parity tests (all fit the oracle in seconds).
WORKLOADS["small_bf16"] = Workload("small_bf16", 2, 8, 2, 128, 1024, 512, 4, 16, "bf16", 0.5)

EDGE_WORKLOADS = {
    # a single history chunk, a single query block, budget of one chunk / one group
    "one_chunk_f32": WORKLOADS["tiny_f32"].with_(name="one_chunk_f32", hist_len=64, seg_len=64,
                                                 top_chunks=1, top_groups=1),
    # 5 groups = 40 routed keys: a ragged routed tile
    "ragged_groups_f32": WORKLOADS["tiny_f32"].with_(name="ragged_groups_f32", top_groups=5),
    # one query head per KV head, batch 2, 9 groups (72 routed keys), bf16
    "gqa1_b2_bf16": Workload("gqa1_b2_bf16", 2, 2, 2, 128, 512, 128, 2, 9, "bf16", 1.0),
    # eight query heads per KV head, budget covering the whole history (dense equivalence)
    "gqa8_dense_f32": Workload("gqa8_dense_f32", 1, 8, 1, 128, 256, 192, 4, 32, "f32", 1.0),
    # tiny layer with every chunk and group selected (dense equivalence)
    "dense_tiny_f32": WORKLOADS["tiny_f32"].with_(name="dense_tiny_f32", top_chunks=16, top_groups=128),
    # maximal group budget for the chosen chunks (k_g = 8 k_c), bf16
    "max_groups_bf16": WORKLOADS["small_bf16"].with_(name="max_groups_bf16", B=1, top_groups=32),
    # two query heads per KV head (one 128-row query tile per CTA), 7 query blocks (a ragged
    # 64-key last tile of the dK/dV kernel), 20 groups = 160 routed keys (ragged routed tiles), bf16
    "gqa2_ragged_bf16": Workload("gqa2_ragged_bf16", 1, 4, 2, 128, 1024, 448, 3, 20, "bf16", 1.0),
    # sink windows: two chunks (float32), one chunk (bf16, four query heads per KV head) and one
    # chunk with two query heads per KV head and a ragged routed tile (bf16)
    "sink_f32": WORKLOADS["tiny_f32"].with_(name="sink_f32", n_sink=128),
    "sink_bf16": WORKLOADS["small_bf16"].with_(name="sink_bf16", n_sink=64),
    "sink_gqa2_bf16": Workload("sink_gqa2_bf16", 1, 4, 2, 128, 1024, 448, 3, 20, "bf16", 1.0, n_sink=128),
    # eight query heads per KV head (two CTAs per query block), 5 query blocks, bf16
    "gqa8_bf16": Workload("gqa8_bf16", 1, 8, 1, 128, 512, 320, 4, 12, "bf16", 1.0),
    # six query heads per KV head: three 2-head forward CTAs per query block, three head pairs per
    # dQ unit list, three heads per paired dK/dV CTA; 7 query blocks, ragged routed tiles, bf16
    "gqa6_bf16": Workload("gqa6_bf16", 1, 12, 2, 128, 1024, 448, 3, 20, "bf16", 1.0),
    # many (batch, KV head) units of short segments: as many dK/dV key tiles as SMs or more, so
    # every CTA sums all of its KV head's query heads alone; ragged 64-key last tile, bf16
    "wide_bf16": Workload("wide_bf16", 16, 16, 8, 128, 256, 192, 2, 8, "bf16", 1.0),
}
