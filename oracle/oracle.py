"""ctypes wrapper of the plain CPU oracle for routed HGA attention (``hga_oracle.c``).

TEST INFRASTRUCTURE ONLY: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  The CUDA library never
imports it and has no fallback to it.

Every function takes and returns numpy float64 arrays in the contiguous
``[B, heads, tokens, D]`` layout (torch tensors are accepted and converted).
The method follows "Long-Context Fine-Tuning with Limited VRAM": gist.science
Technical Summary section 2.1 (chunk selection, group selection, exact-token
attention) and 2.2 (detached history), and the pith.science review (Figure 1,
Figure 2 captions; chunk 64 / group 8 in the free-parameter ledger).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hga_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhga_oracle.so")
_lib = None

_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_dbl = ctypes.c_double
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C99, no fast-math, no FP contraction)."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.hgo_span_means.argtypes = [_i64, _i64, _i64, _i64, _i64, _i32, _p, _p]
        lib.hgo_block_query.argtypes = [_i64, _i64, _i64, _i64, _i64, _i64, _i32, _p, _p]
        lib.hgo_topk.argtypes = [_i64, _p, _i64, _p, _p]
        lib.hgo_route.argtypes = [_i64, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _i64, _i32,
                                  _p, _p, _p, _p, _p, _p, _p]
        lib.hgo_attn_fwd.argtypes = [_i64] * 10 + [_dbl] + [_p] * 6 + [_i64, _p, _p, _p]
        lib.hgo_attn_bwd.argtypes = ([_i64] * 10 + [_dbl] + [_p] * 7
                                     + [_i64, _p, _p, _i64, _p, _p, _p])
        for f in (lib.hgo_span_means, lib.hgo_block_query, lib.hgo_topk, lib.hgo_route,
                  lib.hgo_attn_fwd, lib.hgo_attn_bwd):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments")


# --------------------------------------------------------------------------- summaries
def group_summaries(k_hist, group: int = 8, prec: int = 64) -> np.ndarray:
    """Mean of every ``group`` consecutive history keys: [B,Hkv,H,D] -> [B,Hkv,H/group,D]."""
    k = _f64(k_hist)
    B, Hkv, H, D = k.shape
    out = np.empty((B, Hkv, H // group, D))
    _check(_load().hgo_span_means(B, Hkv, H, D, group, prec, _ptr(k), _ptr(out)), "group_summaries")
    return out


def chunk_summaries(k_hist, chunk: int = 64, prec: int = 64) -> np.ndarray:
    """Mean of every ``chunk`` consecutive history keys: [B,Hkv,H,D] -> [B,Hkv,H/chunk,D]."""
    k = _f64(k_hist)
    B, Hkv, H, D = k.shape
    out = np.empty((B, Hkv, H // chunk, D))
    _check(_load().hgo_span_means(B, Hkv, H, D, chunk, prec, _ptr(k), _ptr(out)), "chunk_summaries")
    return out


def block_query(q, Hkv: int, qblock: int = 64, prec: int = 64) -> np.ndarray:
    """Mean over the query heads of each KV head and the positions of each block."""
    qq = _f64(q)
    B, Hq, S, D = qq.shape
    out = np.empty((B, Hkv, S // qblock, D))
    _check(_load().hgo_block_query(B, Hq, Hkv, S, D, qblock, prec, _ptr(qq), _ptr(out)), "block_query")
    return out


# --------------------------------------------------------------------------- routing
def topk(score, k: int):
    """Indices (ascending) of the k largest scores, ties to the lower index; and the boundary gap."""
    s = _f64(score).reshape(-1)
    sel = np.empty(k, dtype=np.int64)
    gap = np.empty(1)
    _check(_load().hgo_topk(s.size, _ptr(s), k, _ptr(sel), _ptr(gap)), "topk")
    return sel, float(gap[0])


def route(qb, gs, cs, top_chunks: int, top_groups: int, prec: int = 64, n_sink_chunks: int = 0):
    """Two-level routing from summaries.  Returns chunk_idx, group_idx (int32, ascending) and the
    score gaps at the chunk and group selection boundaries, each [B,Hkv,nblk].  The first
    ``n_sink_chunks`` chunks (the fixed sink window) are not routable."""
    qb, gs, cs = _f64(qb), _f64(gs), _f64(cs)
    B, Hkv, nblk, D = qb.shape
    nch = cs.shape[2]
    gpc = gs.shape[2] // nch
    ci = np.empty((B, Hkv, nblk, top_chunks), dtype=np.int32)
    gi = np.empty((B, Hkv, nblk, top_groups), dtype=np.int32)
    cgap = np.empty((B, Hkv, nblk))
    ggap = np.empty((B, Hkv, nblk))
    _check(_load().hgo_route(B, Hkv, nblk, D, nch, gpc, n_sink_chunks, top_chunks, top_groups, prec,
                             _ptr(qb), _ptr(gs), _ptr(cs), _ptr(ci), _ptr(gi), _ptr(cgap), _ptr(ggap)),
           "route")
    return ci, gi, cgap, ggap


def route_from_inputs(q, k_hist, Hkv: int, top_chunks: int, top_groups: int, chunk: int = 64,
                      group: int = 8, qblock: int = 64, prec: int = 32, n_sink: int = 0) -> dict:
    """Summaries, block query and routing in one call (decisions taken in ``prec`` bits);
    ``n_sink`` sink tokens (a multiple of ``chunk``) are excluded from routing."""
    if n_sink % chunk:
        raise ValueError("n_sink must be a multiple of the chunk size")
    gs = group_summaries(k_hist, group, prec)
    cs = chunk_summaries(k_hist, chunk, prec)
    qb = block_query(q, Hkv, qblock, prec)
    ci, gi, cgap, ggap = route(qb, gs, cs, top_chunks, top_groups, prec, n_sink // chunk)
    return dict(group_sum=gs, chunk_sum=cs, qb=qb, chunk_idx=ci, group_idx=gi,
                chunk_gap=cgap, group_gap=ggap)


def route_causal_from_inputs(q, k_hist, Hkv: int, top_chunks: int, top_groups: int, q_prev=None,
                             chunk: int = 64, group: int = 8, qblock: int = 64, prec: int = 32,
                             n_sink: int = 0) -> dict:
    """Strictly causal routing (the variant the pages name as future work, Technical Summary
    section 5 "Causal Leakage"; reading: block n is routed with the block query of block n-1, so
    its routing depends on no token at or after the start of block n).  Block 0 uses the block
    query of ``q_prev`` [B, Hq, qblock, D] (the previous segment's last query block), or a zero
    query if ``q_prev`` is None."""
    if n_sink % chunk:
        raise ValueError("n_sink must be a multiple of the chunk size")
    gs = group_summaries(k_hist, group, prec)
    cs = chunk_summaries(k_hist, chunk, prec)
    qb = block_query(q, Hkv, qblock, prec)
    if q_prev is None:
        first = np.zeros_like(qb[:, :, :1])
    else:
        first = block_query(q_prev, Hkv, qblock, prec)
        if first.shape[2] != 1:
            raise ValueError("q_prev must hold exactly one query block")
    qbc = np.concatenate([first, qb[:, :, :-1]], axis=2)
    ci, gi, cgap, ggap = route(qbc, gs, cs, top_chunks, top_groups, prec, n_sink // chunk)
    return dict(group_sum=gs, chunk_sum=cs, qb=qbc, chunk_idx=ci, group_idx=gi,
                chunk_gap=cgap, group_gap=ggap)


# --------------------------------------------------------------------------- attention
def _layer(q, k_hist, v_hist, k_seg, v_seg, group_idx):
    q, kh, vh, ks, vs = (_f64(t) for t in (q, k_hist, v_hist, k_seg, v_seg))
    gi = np.ascontiguousarray(np.asarray(group_idx.cpu() if hasattr(group_idx, "cpu") else group_idx),
                              dtype=np.int32)
    return q, kh, vh, ks, vs, gi


def attn_fwd(q, k_hist, v_hist, k_seg, v_seg, group_idx, scale: float | None = None,
             group: int = 8, qblock: int = 64, rows=None, n_sink: int = 0):
    """Sink + routed + causal-local attention forward.  Returns (o, lse).

    rows=None: o [B,Hq,S,D], lse [B,Hq,S].  rows = array of flat row ids (b*Hq+h)*S+t:
    o [len(rows), D], lse [len(rows)]."""
    q, kh, vh, ks, vs, gi = _layer(q, k_hist, v_hist, k_seg, v_seg, group_idx)
    B, Hq, S, D = q.shape
    Hkv, H = kh.shape[1], kh.shape[2]
    kg = gi.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if rows is None:
        o = np.empty((B, Hq, S, D)); lse = np.empty((B, Hq, S)); rp = None; nr = 0
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        o = np.empty((r.size, D)); lse = np.empty(r.size); rp = _ptr(r); nr = r.size
    _check(_load().hgo_attn_fwd(B, Hq, Hkv, H, S, D, qblock, group, kg, n_sink, scale,
                                _ptr(q), _ptr(kh), _ptr(vh), _ptr(ks), _ptr(vs), _ptr(gi),
                                nr, rp, _ptr(o), _ptr(lse)), "attn_fwd")
    return o, lse


def attn_bwd(q, k_hist, v_hist, k_seg, v_seg, group_idx, d_o, scale: float | None = None,
             group: int = 8, qblock: int = 64, rows=None, keys=None, n_sink: int = 0):
    """Gradients (dq, dk_seg, dv_seg) of sum(o * d_o); history K/V and routing get none.

    rows/keys select flat ids (b*Hq+h)*S+t for dq and (b*Hkv+kh)*S+u for dk/dv; None = all."""
    q, kh, vh, ks, vs, gi = _layer(q, k_hist, v_hist, k_seg, v_seg, group_idx)
    do = _f64(d_o)
    B, Hq, S, D = q.shape
    Hkv, H = kh.shape[1], kh.shape[2]
    kg = gi.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if rows is None:
        dq = np.empty((B, Hq, S, D)); rp = None; nr = 0
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64); dq = np.empty((r.size, D)); rp = _ptr(r); nr = r.size
    if keys is None:
        dk = np.empty((B, Hkv, S, D)); dv = np.empty((B, Hkv, S, D)); kp = None; nk = 0
    else:
        kk = np.ascontiguousarray(keys, dtype=np.int64)
        dk = np.empty((kk.size, D)); dv = np.empty((kk.size, D)); kp = _ptr(kk); nk = kk.size
    _check(_load().hgo_attn_bwd(B, Hq, Hkv, H, S, D, qblock, group, kg, n_sink, scale,
                                _ptr(q), _ptr(kh), _ptr(vh), _ptr(ks), _ptr(vs), _ptr(gi), _ptr(do),
                                nr, rp, _ptr(dq), nk, kp, _ptr(dk), _ptr(dv)), "attn_bwd")
    return dq, dk, dv
