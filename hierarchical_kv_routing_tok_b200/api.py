"""PyTorch-facing wrapper of the routed-HGA C ABI.

PyTorch provides device memory and the current CUDA stream; every computation
runs in ``libhga.so``.  Tensors must be CUDA, contiguous, in the layouts of
``include/hga.h``: q/o/d_o/dq ``[B, Hq, S, D]``, history K/V ``[B, Hkv, H, D]``,
segment K/V and their gradients ``[B, Hkv, S, D]``.

Method: "Long-Context Fine-Tuning with Limited VRAM" (gist.science Technical
Summary 2.1-2.2; pith.science review Figures 1-2).  Routing runs without
gradient; the history K/V are detached; only q and the active segment get
gradients.
"""
from __future__ import annotations

import math
import time

import torch

from . import _capi as C

_DT = {torch.float32: C.HGA_F32, torch.bfloat16: C.HGA_BF16}


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _need(t: torch.Tensor, name: str, shape, dtype) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def make_config(q: torch.Tensor, k_hist: torch.Tensor, top_chunks: int, top_groups: int,
                softmax_scale: float | None = None, n_sink_tokens: int = 0, wait_limit_ns: int = 0) -> C.HGAConfig:
    """Configuration from q [B,Hq,S,D] and k_hist [B,Hkv,H,D]; ``n_sink_tokens`` (a multiple of 64)
    history tokens at the start form the sink window every query attends; ``wait_limit_ns`` bounds
    the tensor-core kernels' on-chip waits (0: 2 s)."""
    if q.dtype not in _DT:
        raise ValueError(f"unsupported dtype {q.dtype}")
    B, Hq, S, D = q.shape
    Hkv, H = k_hist.shape[1], k_hist.shape[2]
    return C.make_config(B, Hq, Hkv, H, S, top_chunks, top_groups, dtype=_DT[q.dtype], D=D,
                         softmax_scale=float(softmax_scale or 0.0), n_sink_tokens=n_sink_tokens,
                         wait_limit_ns=wait_limit_ns)


def _tdtype(cfg) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == C.HGA_BF16 else torch.float32


def new_workspace(cfg, device) -> torch.Tensor:
    """Zero-initialised workspace (the leading status word must start at 0)."""
    return torch.zeros(C.workspace_size(cfg), dtype=torch.uint8, device=device)


def build_summaries(cfg, k_hist, group_sum=None, chunk_sum=None, workspace=None):
    B, Hkv, H, D = cfg.B, cfg.Hkv, cfg.hist_len, cfg.D
    _need(k_hist, "k_hist", (B, Hkv, H, D), _tdtype(cfg))
    dev = k_hist.device
    if group_sum is None:
        group_sum = torch.empty(B, Hkv, H // cfg.group, D, dtype=torch.float32, device=dev)
    if chunk_sum is None:
        chunk_sum = torch.empty(B, Hkv, H // cfg.chunk, D, dtype=torch.float32, device=dev)
    _need(group_sum, "group_sum", (B, Hkv, H // cfg.group, D), torch.float32)
    _need(chunk_sum, "chunk_sum", (B, Hkv, H // cfg.chunk, D), torch.float32)
    C.build_summaries(cfg, k_hist.data_ptr(), group_sum.data_ptr(), chunk_sum.data_ptr(),
                      workspace.data_ptr() if workspace is not None else None, _stream(k_hist))
    return group_sum, chunk_sum


def route(cfg, q, group_sum, chunk_sum, chunk_idx=None, group_idx=None, workspace=None, causal: bool = False,
          q_prev=None):
    """Two-level routing of every query block.  causal=True: the strictly causal variant -- block n
    is routed with block n-1's query, block 0 with q_prev [B, Hq, 64, D] (the previous segment's
    last query block) or, when q_prev is None, a zero query."""
    B, Hq, Hkv, S, D = cfg.B, cfg.Hq, cfg.Hkv, cfg.seg_len, cfg.D
    nblk = S // cfg.qblock
    _need(q, "q", (B, Hq, S, D), _tdtype(cfg))
    dev = q.device
    if chunk_idx is None:
        chunk_idx = torch.empty(B, Hkv, nblk, cfg.top_chunks, dtype=torch.int32, device=dev)
    if group_idx is None:
        group_idx = torch.empty(B, Hkv, nblk, cfg.top_groups, dtype=torch.int32, device=dev)
    _need(group_sum, "group_sum", (B, Hkv, cfg.hist_len // cfg.group, D), torch.float32)
    _need(chunk_sum, "chunk_sum", (B, Hkv, cfg.hist_len // cfg.chunk, D), torch.float32)
    _need(chunk_idx, "chunk_idx", (B, Hkv, nblk, cfg.top_chunks), torch.int32)
    _need(group_idx, "group_idx", (B, Hkv, nblk, cfg.top_groups), torch.int32)
    ws = workspace.data_ptr() if workspace is not None else None
    if causal:
        if q_prev is not None:
            _need(q_prev, "q_prev", (B, Hq, cfg.qblock, D), _tdtype(cfg))
        C.route_causal(cfg, q.data_ptr(), q_prev.data_ptr() if q_prev is not None else None,
                       group_sum.data_ptr(), chunk_sum.data_ptr(), chunk_idx.data_ptr(), group_idx.data_ptr(), ws,
                       _stream(q))
    elif q_prev is not None:
        raise ValueError("q_prev is only used by the causal routing")
    else:
        C.route(cfg, q.data_ptr(), group_sum.data_ptr(), chunk_sum.data_ptr(), chunk_idx.data_ptr(),
                group_idx.data_ptr(), ws, _stream(q))
    return chunk_idx, group_idx


def _check_layer(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx):
    B, Hq, Hkv, S, H, D = cfg.B, cfg.Hq, cfg.Hkv, cfg.seg_len, cfg.hist_len, cfg.D
    dt = _tdtype(cfg)
    _need(q, "q", (B, Hq, S, D), dt)
    _need(k_hist, "k_hist", (B, Hkv, H, D), dt)
    _need(v_hist, "v_hist", (B, Hkv, H, D), dt)
    _need(k_seg, "k_seg", (B, Hkv, S, D), dt)
    _need(v_seg, "v_seg", (B, Hkv, S, D), dt)
    _need(group_idx, "group_idx", (B, Hkv, S // cfg.qblock, cfg.top_groups), torch.int32)


def attn_fwd(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx, o=None, lse=None, workspace=None):
    _check_layer(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(cfg.B, cfg.Hq, cfg.seg_len, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(cfg, q.device)
    _need(o, "o", q.shape, q.dtype)
    _need(lse, "lse", (cfg.B, cfg.Hq, cfg.seg_len), torch.float32)
    C.attn_fwd(cfg, q.data_ptr(), k_hist.data_ptr(), v_hist.data_ptr(), k_seg.data_ptr(), v_seg.data_ptr(),
               group_idx.data_ptr(), o.data_ptr(), lse.data_ptr(), workspace.data_ptr(), _stream(q))
    return o, lse


def attn_bwd(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o, dq=None, dk_seg=None, dv_seg=None,
             workspace=None):
    _check_layer(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx)
    _need(o, "o", q.shape, q.dtype)
    _need(d_o, "d_o", q.shape, q.dtype)
    _need(lse, "lse", (cfg.B, cfg.Hq, cfg.seg_len), torch.float32)
    dq = torch.empty_like(q) if dq is None else dq
    dk_seg = torch.empty_like(k_seg) if dk_seg is None else dk_seg
    dv_seg = torch.empty_like(v_seg) if dv_seg is None else dv_seg
    _need(dq, "dq", q.shape, q.dtype)
    _need(dk_seg, "dk_seg", k_seg.shape, k_seg.dtype)
    _need(dv_seg, "dv_seg", v_seg.shape, v_seg.dtype)
    if workspace is None:
        workspace = new_workspace(cfg, q.device)
    C.attn_bwd(cfg, q.data_ptr(), k_hist.data_ptr(), v_hist.data_ptr(), k_seg.data_ptr(), v_seg.data_ptr(),
               group_idx.data_ptr(), o.data_ptr(), lse.data_ptr(), d_o.data_ptr(), dq.data_ptr(),
               dk_seg.data_ptr(), dv_seg.data_ptr(), workspace.data_ptr(), _stream(q))
    return dq, dk_seg, dv_seg


def read_status(workspace: torch.Tensor) -> int:
    return C.read_status(workspace.data_ptr(), _stream(workspace))


class _HGAFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k_seg, v_seg, k_hist, v_hist, top_chunks, top_groups, softmax_scale):
        cfg = make_config(q, k_hist, top_chunks, top_groups, softmax_scale)
        ws = new_workspace(cfg, q.device)
        with torch.no_grad():                       # routing carries no gradient
            gs, cs = build_summaries(cfg, k_hist, workspace=ws)
            _, gi = route(cfg, q, gs, cs, workspace=ws)
        o, lse = attn_fwd(cfg, q, k_hist, v_hist, k_seg, v_seg, gi, workspace=ws)
        ctx.cfg = cfg
        ctx.save_for_backward(q, k_seg, v_seg, k_hist, v_hist, gi, o, lse, ws)
        ctx.mark_non_differentiable(lse, gi)
        return o, lse, gi

    @staticmethod
    def backward(ctx, d_o, _dlse, _dgi):
        q, k_seg, v_seg, k_hist, v_hist, gi, o, lse, ws = ctx.saved_tensors
        dq, dk, dv = attn_bwd(ctx.cfg, q, k_hist, v_hist, k_seg, v_seg, gi, o, lse, d_o.contiguous(),
                              workspace=ws)
        return dq, dk, dv, None, None, None, None, None


def hga_attention(q, k_seg, v_seg, k_hist, v_hist, top_chunks: int, top_groups: int,
                  softmax_scale: float | None = None):
    """Routed HGA attention of the active segment.  Returns (o, lse, group_idx).

    Differentiable in q, k_seg, v_seg; k_hist / v_hist are treated as detached history."""
    return _HGAFunction.apply(q, k_seg, v_seg, k_hist.detach(), v_hist.detach(), top_chunks, top_groups,
                              softmax_scale)


class LayerStep:
    """One full pass of the hot path (summaries, routing, forward, backward) over preallocated
    buffers, for a fixed configuration.  Used by the benchmark and the smoke check."""

    def __init__(self, cfg, device="cuda", causal_routing: bool = False, summaries_from: int | None = None):
        """summaries_from: None rebuilds the summaries of the whole history every step; a token
        index (a multiple of the chunk) makes the step compute only those of history tokens
        [summaries_from, H) -- the segment appended last -- with ``hga_append_summaries``, the
        summaries of the earlier tokens being already in ``group_sum`` / ``chunk_sum`` (run
        ``build_all_summaries`` once first)."""
        self.cfg = cfg
        self.causal_routing = causal_routing
        if summaries_from is not None and not (0 <= summaries_from <= cfg.hist_len
                                               and summaries_from % cfg.chunk == 0):
            raise ValueError(f"summaries_from={summaries_from}: a multiple of {cfg.chunk} in [0, {cfg.hist_len}]")
        self.summaries_from = summaries_from
        dev = torch.device(device)
        B, Hq, Hkv, S, H, D = cfg.B, cfg.Hq, cfg.Hkv, cfg.seg_len, cfg.hist_len, cfg.D
        dt = _tdtype(cfg)
        nblk = S // cfg.qblock
        self.ws = new_workspace(cfg, dev)
        self.group_sum = torch.empty(B, Hkv, H // cfg.group, D, dtype=torch.float32, device=dev)
        self.chunk_sum = torch.empty(B, Hkv, H // cfg.chunk, D, dtype=torch.float32, device=dev)
        self.chunk_idx = torch.empty(B, Hkv, nblk, cfg.top_chunks, dtype=torch.int32, device=dev)
        self.group_idx = torch.empty(B, Hkv, nblk, cfg.top_groups, dtype=torch.int32, device=dev)
        self.o = torch.empty(B, Hq, S, D, dtype=dt, device=dev)
        self.lse = torch.empty(B, Hq, S, dtype=torch.float32, device=dev)
        self.dq = torch.empty(B, Hq, S, D, dtype=dt, device=dev)
        self.dk = torch.empty(B, Hkv, S, D, dtype=dt, device=dev)
        self.dv = torch.empty(B, Hkv, S, D, dtype=dt, device=dev)

    def calls(self, x: dict, stream: int | None = None, cfg: "C.HGAConfig | None" = None):
        """The step as a list of (kernel name, zero-argument C-ABI call), one kernel each, in order.
        Pointers are bound once so the timed loop does no tensor bookkeeping.  ``cfg`` overrides the
        step's configuration (same shapes; e.g. another wait limit)."""
        cfg, ws = (self.cfg if cfg is None else cfg), self.ws.data_ptr()
        st = torch.cuda.current_stream(self.o.device).cuda_stream if stream is None else stream
        p = {k: v.data_ptr() for k, v in x.items() if isinstance(v, torch.Tensor) and v.is_cuda}
        gs, cs, ci, gi = (t.data_ptr() for t in (self.group_sum, self.chunk_sum, self.chunk_idx, self.group_idx))
        o, lse, dq, dk, dv = (t.data_ptr() for t in (self.o, self.lse, self.dq, self.dk, self.dv))
        first = self.summaries_from
        return [
            ("summaries", (lambda: C.build_summaries(cfg, p["k_hist"], gs, cs, ws, st)) if first is None
             else (lambda: C.append_summaries(cfg, p["k_hist"], gs, cs, first, ws, st))),
            ("route", (lambda: C.route_causal(cfg, p["q"], p.get("q_prev"), gs, cs, ci, gi, ws, st))
             if self.causal_routing else (lambda: C.route(cfg, p["q"], gs, cs, ci, gi, ws, st))),
            ("attn_fwd", lambda: C.attn_fwd(cfg, p["q"], p["k_hist"], p["v_hist"], p["k_seg"], p["v_seg"], gi, o,
                                            lse, ws, st)),
            # dq first: it also forms delta = rowsum(d_o * o), which dkdv reads
            ("bwd_dq", lambda: C.attn_bwd_dq(cfg, p["q"], p["k_hist"], p["v_hist"], p["k_seg"], p["v_seg"], gi,
                                             o, lse, p["d_o"], dq, ws, st)),
            ("bwd_dkdv", lambda: C.attn_bwd_dkdv(cfg, p["q"], p["k_seg"], p["v_seg"], lse, p["d_o"], dk, dv, ws,
                                                 st)),
        ]

    def build_all_summaries(self, x: dict) -> None:
        """Summaries of the whole history of x into this step's buffers (the state an appending
        step starts from)."""
        C.build_summaries(self.cfg, x["k_hist"].data_ptr(), self.group_sum.data_ptr(), self.chunk_sum.data_ptr(),
                          self.ws.data_ptr(), torch.cuda.current_stream(self.o.device).cuda_stream)

    def forward(self, x: dict) -> None:
        for _, call in self.calls(x)[:3]:
            call()

    def backward(self, x: dict) -> None:
        for _, call in self.calls(x)[3:]:
            call()

    def __call__(self, x: dict) -> None:
        for _, call in self.calls(x):
            call()

    def capture(self, x: dict, stream: "torch.cuda.Stream | None" = None, warmup: int = 2) -> "torch.cuda.CUDAGraph":
        """The whole step on the buffers of ``x`` as a CUDA graph: ``graph.replay()`` runs the same
        kernels (with their dependent launches) without the per-call host work of the C ABI (argument
        checks, tensor maps, launches).  The step is first run ``warmup`` times on ``stream`` (a
        side stream by default), then captured there; replay on any stream of the same device.
        The buffers of ``x`` and of this step must stay alive and in place while the graph is used."""
        dev = self.o.device
        s = stream if stream is not None else torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        calls = self.calls(x, s.cuda_stream)
        with torch.cuda.stream(s):
            for _ in range(warmup):
                for _, call in calls:
                    call()
        g = torch.cuda.CUDAGraph()
        # thread-local capture: CUDA calls of other host threads (a collective library's proxy
        # thread, say) neither join nor invalidate it
        with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
            for _, call in calls:
                call()
        torch.cuda.current_stream(dev).wait_stream(s)
        return g


class GroupSummaryCache:
    """Device cache of the group summaries of a history whose group-summary table lives in host
    memory ("Technical Summary" 2.1 Group Selection: group summaries are cached in device memory and
    the missing ones fetched from host memory; the chunk summaries stay in device memory).  Each of
    the ``cap_chunks`` slots per (batch, KV head) holds the 8 group summaries of one chunk; a step
    routes level 1 on the device chunk summaries, fetches the chosen chunks the cache lacks (least
    recently used slots make room) and routes level 2 from the cache, giving the same indices as
    the routing over the full table.

    group_sum_host: pinned CPU float32 [B, Hkv, Hs/8, D] (Hs = the history's capacity in tokens)."""

    CHUNK_BYTES = 8 * 128 * 4          # one slot: 8 group summaries of 128 float32

    def __init__(self, cfg, group_sum_host, cap_chunks: int, device="cuda"):
        dev = torch.device(device)
        B, Hkv, D = cfg.B, cfg.Hkv, cfg.D
        hs = cfg.hist_capacity or cfg.hist_len
        if group_sum_host.is_cuda or not group_sum_host.is_pinned():
            raise ValueError("group_sum_host must be pinned host memory")
        if (tuple(group_sum_host.shape) != (B, Hkv, hs // cfg.group, D) or group_sum_host.dtype != torch.float32
                or not group_sum_host.is_contiguous()):
            raise ValueError(f"group_sum_host: expected contiguous float32 {(B, Hkv, hs // cfg.group, D)}")
        self.cfg, self.dev, self.cap = cfg, dev, int(cap_chunks)
        self.host = group_sum_host
        i32 = dict(dtype=torch.int32, device=dev)
        self.slot_of = torch.full((B, Hkv, hs // cfg.chunk), -1, **i32)
        self.chunk_of = torch.full((B, Hkv, self.cap), -1, **i32)
        self.stamp = torch.full((B, Hkv, self.cap), -1, **i32)
        self.miss_chunk = torch.empty(B, Hkv, self.cap, **i32)
        self.miss_slot = torch.empty(B, Hkv, self.cap, **i32)
        self.counts = torch.zeros(B * Hkv, 2, **i32)
        self.gcache = torch.empty(B, Hkv, self.cap, 8, D, dtype=torch.float32, device=dev)
        self.qb = torch.empty(B, Hkv, cfg.seg_len // cfg.qblock, D, dtype=torch.float32, device=dev)
        self.step = 0

    def route(self, q, chunk_sum, chunk_idx, group_idx, workspace, stream: int | None = None) -> None:
        """Both routing levels of one step through the cache (asynchronous on ``stream``)."""
        cfg, cap = self.cfg, self.cap
        st = torch.cuda.current_stream(self.dev).cuda_stream if stream is None else stream
        ws = workspace.data_ptr()
        C.route_chunks(cfg, q.data_ptr(), chunk_sum.data_ptr(), chunk_idx.data_ptr(), self.qb.data_ptr(), ws, st)
        C.gcache_plan(cfg, cap, chunk_idx.data_ptr(), self.slot_of.data_ptr(), self.chunk_of.data_ptr(),
                      self.stamp.data_ptr(), self.step, self.miss_chunk.data_ptr(), self.miss_slot.data_ptr(),
                      self.counts.data_ptr(), ws, st)
        C.gcache_fetch(cfg, cap, self.host.data_ptr(), self.miss_chunk.data_ptr(), self.miss_slot.data_ptr(),
                       self.counts.data_ptr(), self.gcache.data_ptr(), st)
        C.route_groups_cached(cfg, self.qb.data_ptr(), chunk_idx.data_ptr(), self.slot_of.data_ptr(), cap,
                              self.gcache.data_ptr(), group_idx.data_ptr(), ws, st)
        self.step += 1

    def stats(self) -> dict:
        """Hits and misses of the last step (chunks, summed over batch and KV heads) and the bytes of
        group summaries it fetched from host memory (synchronises)."""
        c = self.counts.sum(dim=0).tolist()
        return {"hits": int(c[0]), "misses": int(c[1]), "host_bytes": int(c[1]) * self.CHUNK_BYTES,
                "cap_chunks": self.cap}


class TieredLayerStep:
    """One layer step with the detached history K/V in pinned host memory (tiered storage,
    "Technical Summary" 2.2): the summaries and the routing stay in device memory; per step only
    the K/V of the routed groups are gathered into a compact device cache.  The gather runs one
    batch element at a time on a side stream, so the copy of element b+1 over the host link
    overlaps the forward and backward of element b on the caller's stream.

    k_hist_host / v_hist_host: pinned CPU tensors [B, Hkv, H, D] (``pin_memory=True``);
    group_sum / chunk_sum: the device summaries of that history (built when it was written);
    group_cache: a GroupSummaryCache over the history's group summaries in host memory -- the
    routing then reads the group summaries through it (group_sum may be None), so that only the
    chunk summaries stay in device memory, as in the pages' three tiers."""

    def __init__(self, cfg, k_hist_host, v_hist_host, group_sum, chunk_sum, device="cuda",
                 group_cache: "GroupSummaryCache | None" = None):
        dev = torch.device(device)
        B, Hq, Hkv, S, H, D = cfg.B, cfg.Hq, cfg.Hkv, cfg.seg_len, cfg.hist_len, cfg.D
        dt = _tdtype(cfg)
        for name, t in (("k_hist_host", k_hist_host), ("v_hist_host", v_hist_host)):
            if t.is_cuda or not t.is_pinned():
                raise ValueError(f"{name} must be pinned host memory")
            if tuple(t.shape) != (B, Hkv, H, D) or t.dtype != dt or not t.is_contiguous():
                raise ValueError(f"{name}: expected contiguous {dt} {(B, Hkv, H, D)}, got {t.dtype} "
                                 f"{tuple(t.shape)}")
        self.cfg, self.dev = cfg, dev
        self.ccfg = C.tier_cache_config(cfg)
        self.cfg1 = C.make_config(1, Hq, Hkv, H, S, cfg.top_chunks, cfg.top_groups, dtype=cfg.dtype, D=D,
                                  softmax_scale=cfg.softmax_scale, n_sink_tokens=cfg.n_sink_tokens,
                                  wait_limit_ns=cfg.wait_limit_ns)
        self.ccfg1 = C.tier_cache_config(self.cfg1)
        self.cap = self.ccfg.hist_len // cfg.group
        nblk = S // cfg.qblock
        self.k_host, self.v_host = k_hist_host, v_hist_host
        self.group_sum, self.chunk_sum = group_sum, chunk_sum
        self.group_cache = group_cache
        if group_sum is None and group_cache is None:
            raise ValueError("group_sum is needed unless a group_cache is given")
        i32 = dict(dtype=torch.int32, device=dev)
        self.chunk_idx = torch.empty(B, Hkv, nblk, cfg.top_chunks, **i32)
        self.group_idx = torch.empty(B, Hkv, nblk, cfg.top_groups, **i32)
        self.compact_idx = torch.empty(B, Hkv, nblk, cfg.top_groups, **i32)
        self.used_groups = torch.empty(B, Hkv, self.cap, **i32)
        self.n_used = torch.empty(B * Hkv, **i32)
        self.k_cache = torch.empty(B, Hkv, self.cap * cfg.group, D, dtype=dt, device=dev)
        self.v_cache = torch.empty_like(self.k_cache)
        self.ws = new_workspace(cfg, dev)
        self.ws1 = [new_workspace(self.cfg1, dev) for _ in range(B)]
        self.o = torch.empty(B, Hq, S, D, dtype=dt, device=dev)
        self.lse = torch.empty(B, Hq, S, dtype=torch.float32, device=dev)
        self.dq = torch.empty_like(self.o)
        self.dk = torch.empty(B, Hkv, S, D, dtype=dt, device=dev)
        self.dv = torch.empty_like(self.dk)
        self.side = torch.cuda.Stream(dev)
        self.planned = torch.cuda.Event()
        self.gathered = [torch.cuda.Event() for _ in range(B)]
        self.done = torch.cuda.Event()

    def __call__(self, x: dict, backward: bool = True) -> None:
        """Enqueue one step (routing, plan, per-element gather + forward [+ backward]) for
        x = {q, k_seg, v_seg[, d_o]} on the current stream; returns without synchronising."""
        cfg, c1 = self.cfg, self.ccfg1
        main = torch.cuda.current_stream(self.dev)
        st, side = main.cuda_stream, self.side.cuda_stream
        ws = self.ws.data_ptr()
        if self.group_cache is not None:
            self.group_cache.route(x["q"], self.chunk_sum, self.chunk_idx, self.group_idx, self.ws, st)
        else:
            C.route(cfg, x["q"].data_ptr(), self.group_sum.data_ptr(), self.chunk_sum.data_ptr(),
                    self.chunk_idx.data_ptr(), self.group_idx.data_ptr(), ws, st)
        C.tier_plan(cfg, self.group_idx.data_ptr(), self.used_groups.data_ptr(), self.n_used.data_ptr(),
                    self.compact_idx.data_ptr(), ws, st)
        self.planned.record(main)
        self.side.wait_event(self.planned)
        for b in range(cfg.B):
            C.tier_gather(self.cfg1, self.k_host[b].data_ptr(), self.v_host[b].data_ptr(),
                          self.used_groups[b].data_ptr(), self.n_used[b * cfg.Hkv:].data_ptr(),
                          self.k_cache[b].data_ptr(), self.v_cache[b].data_ptr(), side)
            self.gathered[b].record(self.side)
        for b in range(cfg.B):
            main.wait_event(self.gathered[b])
            w1 = self.ws1[b].data_ptr()
            q, ks, vs = x["q"][b].data_ptr(), x["k_seg"][b].data_ptr(), x["v_seg"][b].data_ptr()
            kc, vc, gi = self.k_cache[b].data_ptr(), self.v_cache[b].data_ptr(), self.compact_idx[b].data_ptr()
            o, lse = self.o[b].data_ptr(), self.lse[b].data_ptr()
            C.attn_fwd(c1, q, kc, vc, ks, vs, gi, o, lse, w1, st)
            if backward:
                C.attn_bwd(c1, q, kc, vc, ks, vs, gi, o, lse, x["d_o"][b].data_ptr(), self.dq[b].data_ptr(),
                           self.dk[b].data_ptr(), self.dv[b].data_ptr(), w1, st)
        self.done.record(main)

    def wait(self, timeout_s: float = 30.0) -> None:
        """Host-side wait for the last enqueued step with a deadline: raises TimeoutError instead of
        blocking forever if the host link or the device stalls; raises on a device status error."""
        deadline = time.monotonic() + timeout_s
        while not self.done.query():
            if time.monotonic() > deadline:
                raise TimeoutError(f"tiered layer step not finished after {timeout_s} s")
            time.sleep(50e-6)
        for w in [self.ws, *self.ws1]:
            code = read_status(w)
            if code != 0:
                raise C.HGAError("tiered step (device status)", code)

    def gather_bytes(self) -> int:
        """Bytes of history K/V the last step copied into the cache (K and V)."""
        esz = 2 if self.cfg.dtype == C.HGA_BF16 else 4
        return int(self.n_used.sum().item()) * self.cfg.group * self.cfg.D * esz * 2


def default_scale(D: int = 128) -> float:
    return 1.0 / math.sqrt(D)
