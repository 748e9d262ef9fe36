"""Segment-wise training over long sequences ("Long-Context Fine-Tuning with Limited VRAM",
gist.science Technical Summary 2.2 "Segment-wise Backward and Tiered Storage"; pith.science
review, "What carries the argument"): the sequence is processed in segments of S tokens; each
segment's attention reads the detached history of all earlier segments through the HGA routing,
the loss of the segment is back-propagated at once (truncated backpropagation through time), and
at the segment boundary the segment's K/V are appended to the history without their graph.

``HGAHistory`` is one attention layer's history: K/V buffers of a fixed capacity (device memory,
or pinned host memory for tiered storage) and their summaries in device memory, appended to at
every segment boundary (only the new chunks' summaries are computed).  ``segment_attention`` is
the differentiable attention of one segment against it (gradients for q, k_seg and v_seg only).

Budgets early in a sequence: with no history the first segment attends its causal prefix only; while
the history holds fewer chunks than the budget, the routing takes every chunk that is not sink
(k_c' = min(k_c, routable chunks), k_g' = min(k_g, 8 k_c')), and the sink keeps at least one chunk
routable.
"""
from __future__ import annotations

import torch

from . import _capi as C
from .api import _need, new_workspace

_DT = {torch.float32: C.HGA_F32, torch.bfloat16: C.HGA_BF16}


class HGAHistory:
    """Detached history of one attention layer: K/V [B, Hkv, capacity, D] in device memory
    (``tiered=False``) or pinned host memory (``tiered=True``), group / chunk summaries
    [B, Hkv, capacity / 8 (/ 64), D] float32 in device memory, and the number of valid tokens."""

    def __init__(self, B: int, Hq: int, Hkv: int, capacity: int, dtype=torch.bfloat16, D: int = 128,
                 device="cuda", tiered: bool = False, n_sink_tokens: int = 0):
        if capacity % 64:
            raise ValueError("capacity must be a multiple of the 64-token chunk")
        dev = torch.device(device)
        self.B, self.Hq, self.Hkv, self.D, self.capacity = B, Hq, Hkv, D, capacity
        self.dtype, self.device, self.tiered, self.n_sink_tokens = dtype, dev, tiered, n_sink_tokens
        self.length = 0
        kw = dict(dtype=dtype, device="cpu", pin_memory=True) if tiered else dict(dtype=dtype, device=dev)
        self.k = torch.empty(B, Hkv, capacity, D, **kw)
        self.v = torch.empty(B, Hkv, capacity, D, **kw)
        self.group_sum = torch.empty(B, Hkv, capacity // 8, D, dtype=torch.float32, device=dev)
        self.chunk_sum = torch.empty(B, Hkv, capacity // 64, D, dtype=torch.float32, device=dev)

    def config(self, seg_len: int, top_chunks: int, top_groups: int, softmax_scale: float = 0.0) -> C.HGAConfig:
        """The configuration of a segment against the current history, budgets clamped to it."""
        H = self.length
        if H == 0:
            kc = kg = ns = 0
        else:
            ns = min(self.n_sink_tokens, H - 64)
            kc = min(top_chunks, H // 64 - ns // 64)
            kg = min(top_groups, 8 * kc)
        return C.make_config(self.B, self.Hq, self.Hkv, H, seg_len, kc, kg, dtype=_DT[self.dtype], D=self.D,
                             softmax_scale=softmax_scale, n_sink_tokens=ns, hist_capacity=self.capacity)

    @torch.no_grad()
    def append(self, k_seg: torch.Tensor, v_seg: torch.Tensor) -> None:
        """Segment boundary: append the segment's K/V [B, Hkv, S, D] (detached) and the summaries of
        its chunks.  Asynchronous on the current stream."""
        B, Hkv, S, D = k_seg.shape
        _need(k_seg, "k_seg", (self.B, self.Hkv, S, self.D), self.dtype)
        _need(v_seg, "v_seg", (self.B, self.Hkv, S, self.D), self.dtype)
        L = self.length
        if S % 64 or L + S > self.capacity:
            raise ValueError(f"cannot append {S} tokens to a history of {L} / {self.capacity}")
        self.k[:, :, L:L + S].copy_(k_seg.detach(), non_blocking=True)
        self.v[:, :, L:L + S].copy_(v_seg.detach(), non_blocking=True)
        st = torch.cuda.current_stream(self.device).cuda_stream
        if self.tiered:
            # the new keys are still in device memory: summarise them there, then place the summaries
            cfg = C.make_config(B, self.Hq, Hkv, S, 64, 1, 1, dtype=_DT[self.dtype], D=D)
            gs = torch.empty(B, Hkv, S // 8, D, dtype=torch.float32, device=self.device)
            cs = torch.empty(B, Hkv, S // 64, D, dtype=torch.float32, device=self.device)
            C.build_summaries(cfg, k_seg.data_ptr(), gs.data_ptr(), cs.data_ptr(), None, st)
            self.group_sum[:, :, L // 8:(L + S) // 8].copy_(gs)
            self.chunk_sum[:, :, L // 64:(L + S) // 64].copy_(cs)
        else:
            cfg = C.make_config(B, self.Hq, Hkv, L + S, 64, 1, 1, dtype=_DT[self.dtype], D=D,
                                hist_capacity=self.capacity)
            C.append_summaries(cfg, self.k.data_ptr(), self.group_sum.data_ptr(), self.chunk_sum.data_ptr(), L,
                               None, st)
        self.length = L + S


class _SegmentAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k_seg, v_seg, hist: HGAHistory, top_chunks, top_groups, softmax_scale, causal, q_prev):
        B, Hq, S, D = q.shape
        cfg = hist.config(S, top_chunks, top_groups, float(softmax_scale or 0.0))
        dev = q.device
        st = torch.cuda.current_stream(dev).cuda_stream
        ws = new_workspace(cfg, dev)
        nblk = S // 64
        ci = torch.empty(B, hist.Hkv, nblk, max(cfg.top_chunks, 1), dtype=torch.int32, device=dev)
        gi = torch.empty(B, hist.Hkv, nblk, max(cfg.top_groups, 1), dtype=torch.int32, device=dev)
        with torch.no_grad():                           # routing carries no gradient
            if causal:
                C.route_causal(cfg, q.data_ptr(), q_prev.data_ptr() if q_prev is not None else None,
                               hist.group_sum.data_ptr(), hist.chunk_sum.data_ptr(), ci.data_ptr(), gi.data_ptr(),
                               ws.data_ptr(), st)
            else:
                C.route(cfg, q.data_ptr(), hist.group_sum.data_ptr(), hist.chunk_sum.data_ptr(), ci.data_ptr(),
                        gi.data_ptr(), ws.data_ptr(), st)
        acfg, kh, vh, agi = cfg, hist.k, hist.v, gi
        if hist.tiered and cfg.hist_len > 0:
            # bring the routed groups of the host-resident history into a compact device cache
            acfg = C.tier_cache_config(cfg)
            cap = acfg.hist_len // 8
            used = torch.empty(B, hist.Hkv, cap, dtype=torch.int32, device=dev)
            n_used = torch.empty(B * hist.Hkv, dtype=torch.int32, device=dev)
            agi = torch.empty_like(gi)
            C.tier_plan(cfg, gi.data_ptr(), used.data_ptr(), n_used.data_ptr(), agi.data_ptr(), ws.data_ptr(), st)
            kh = torch.empty(B, hist.Hkv, acfg.hist_len, D, dtype=q.dtype, device=dev)
            vh = torch.empty_like(kh)
            C.tier_gather(cfg, hist.k.data_ptr(), hist.v.data_ptr(), used.data_ptr(), n_used.data_ptr(),
                          kh.data_ptr(), vh.data_ptr(), st)
        o = torch.empty_like(q)
        lse = torch.empty(B, Hq, S, dtype=torch.float32, device=dev)
        hp = (kh.data_ptr(), vh.data_ptr(), agi.data_ptr()) if cfg.hist_len > 0 else (None, None, None)
        C.attn_fwd(acfg, q.data_ptr(), hp[0], hp[1], k_seg.data_ptr(), v_seg.data_ptr(), hp[2], o.data_ptr(),
                   lse.data_ptr(), ws.data_ptr(), st)
        ctx.acfg, ctx.hp = acfg, hp
        ctx.save_for_backward(q, k_seg, v_seg, o, lse, ws, kh, vh, agi, gi)
        ctx.mark_non_differentiable(gi)
        return o, gi

    @staticmethod
    def backward(ctx, d_o, _dgi):
        q, k_seg, v_seg, o, lse, ws, _kh, _vh, _agi, _gi = ctx.saved_tensors
        d_o = d_o.contiguous()
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k_seg), torch.empty_like(v_seg)
        hp = ctx.hp
        C.attn_bwd(ctx.acfg, q.data_ptr(), hp[0], hp[1], k_seg.data_ptr(), v_seg.data_ptr(), hp[2], o.data_ptr(),
                   lse.data_ptr(), d_o.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(),
                   torch.cuda.current_stream(q.device).cuda_stream)
        return dq, dk, dv, None, None, None, None, None, None


def segment_attention(q, k_seg, v_seg, history: HGAHistory, top_chunks: int, top_groups: int,
                      softmax_scale: float | None = None, causal: bool = False, q_prev=None):
    """Attention of one segment (q [B,Hq,S,D], k_seg / v_seg [B,Hkv,S,D], contiguous) over the sink,
    the routed groups of ``history`` and its own causal prefix.  Returns (o, group_idx); o is
    differentiable in q, k_seg and v_seg; the history is detached.  ``causal`` selects the strictly
    causal routing (block n routed with block n-1's query, block 0 with ``q_prev``)."""
    for name, t in (("q", q), ("k_seg", k_seg), ("v_seg", v_seg)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != history.dtype:
            raise ValueError(f"{name} must be a contiguous CUDA {history.dtype} tensor")
    return _SegmentAttention.apply(q, k_seg, v_seg, history, top_chunks, top_groups, softmax_scale, causal, q_prev)
