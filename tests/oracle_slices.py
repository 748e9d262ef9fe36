"""The CPU oracle's attention at sampled rows and keys of a large layer, one (batch, KV head) slice
per host thread.

Each (batch, KV head) slice of a layer -- its G query heads, its history and segment K/V and its
routing -- is computed independently of every other slice (routing and attention are per KV
head), so the oracle's value for a row or key equals its value on that row's slice alone.  The
oracle's C calls release the GIL, so the slices run on all host cores.  This module only indexes
and reassembles; all arithmetic happens in the oracle."""
from __future__ import annotations

import concurrent.futures as cf
import os

import numpy as np


def _arr(t) -> np.ndarray:
    if hasattr(t, "detach"):
        t = t.detach().cpu()
        if t.dtype.is_floating_point:
            t = t.double()
        return t.numpy()
    return np.asarray(t)


def attn_sampled(oracle, q, k_hist, v_hist, k_seg, v_seg, group_idx, d_o=None, rows=(), keys=(), n_sink=0):
    """Oracle outputs at flat row ids (b*Hq + h)*S + t and key ids (b*Hkv + kh)*S + u.

    Returns a dict with o [len(rows), D] and lse [len(rows)], and with d_o also dq [len(rows), D],
    dk, dv [len(keys), D], in the order the ids are given."""
    q, kh_, vh_, ks_, vs_, gi = (_arr(t) for t in (q, k_hist, v_hist, k_seg, v_seg, group_idx))
    do = _arr(d_o) if d_o is not None else None
    B, Hq, S, D = q.shape
    Hkv = ks_.shape[1]
    G = Hq // Hkv
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    keys = np.asarray(keys, dtype=np.int64).reshape(-1)
    r_b, r_h, r_t = rows // (Hq * S), (rows // S) % Hq, rows % S
    r_kh = r_h // G
    k_b, k_kh, k_u = keys // (Hkv * S), (keys // S) % Hkv, keys % S
    jobs = sorted(set(zip(r_b.tolist(), r_kh.tolist())) | set(zip(k_b.tolist(), k_kh.tolist())))

    def run(b, kh):
        hs = slice(kh * G, (kh + 1) * G)
        sl = (q[b:b + 1, hs], kh_[b:b + 1, kh:kh + 1], vh_[b:b + 1, kh:kh + 1], ks_[b:b + 1, kh:kh + 1],
              vs_[b:b + 1, kh:kh + 1], np.ascontiguousarray(gi[b:b + 1, kh:kh + 1]))
        mr = np.nonzero((r_b == b) & (r_kh == kh))[0]
        mk = np.nonzero((k_b == b) & (k_kh == kh))[0]
        lr = (r_h[mr] - kh * G) * S + r_t[mr]
        out = {}
        if mr.size:
            out["o"], out["lse"] = oracle.attn_fwd(*sl, rows=lr, n_sink=n_sink)
        if do is not None and (mr.size or mk.size):
            # placeholders where a slice needs no rows / no keys: the cheapest row and key (the last
            # key is seen only by the last query of each head)
            dq, dk, dv = oracle.attn_bwd(*sl, do[b:b + 1, hs], rows=lr if mr.size else np.array([0]),
                                         keys=k_u[mk] if mk.size else np.array([S - 1]), n_sink=n_sink)
            out["dq"], out["dk"], out["dv"] = dq, dk, dv
        return mr, mk, out

    res = {"o": np.empty((rows.size, D)), "lse": np.empty(rows.size)}
    if do is not None:
        res.update(dq=np.empty((rows.size, D)), dk=np.empty((keys.size, D)), dv=np.empty((keys.size, D)))
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        for mr, mk, out in ex.map(lambda j: run(*j), jobs):
            if mr.size:
                res["o"][mr], res["lse"][mr] = out["o"], out["lse"]
                if do is not None:
                    res["dq"][mr] = out["dq"]
            if do is not None and mk.size:
                res["dk"][mk], res["dv"][mk] = out["dk"], out["dv"]
    return res
