"""Tiered history (history K/V in pinned host memory, compact device cache per step) on a B200:
the tiered step matches the oracle over the whole history (routing bit-exact, outputs within the
bars of the resident path), the plan is the exact union of the routed groups with
order-preserving positions, the gather copies exactly those rows, and the whole tiered step
equals the step over device-resident history bit for bit."""
import numpy as np
import pytest
import torch

import hga_inputs as HI
from oracle_slices import attn_sampled

TOL = {"f32": 1e-4, "bf16": 2e-2}
LSE_TOL = {"f32": 1e-4, "bf16": 1e-3}

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_kv_routing_tok_b200 as H
    H.load()
    return H


def _wl(name):
    return HI.WORKLOADS.get(name) or HI.EDGE_WORKLOADS[name]


def _resident(hga, w, xd):
    cfg = hga.make_config(xd["q"], xd["k_hist"], w.top_chunks, w.top_groups, n_sink_tokens=w.n_sink)
    step = hga.LayerStep(cfg)
    step(xd)
    torch.cuda.synchronize()
    assert hga.read_status(step.ws) == 0
    return cfg, step


def _tiered(hga, cfg, step, x, xd):
    kh = x["k_hist"].pin_memory()
    vh = x["v_hist"].pin_memory()
    t = hga.TieredLayerStep(cfg, kh, vh, step.group_sum, step.chunk_sum)
    t(xd)
    t.wait(timeout_s=60)
    return t


def _tiered_only(hga, w, x):
    """The tiered step alone: summaries built on the device while the history keys are there (as
    when the history is written), then K/V kept only in pinned host memory."""
    xd = {k: x[k].cuda() for k in ("q", "k_seg", "v_seg", "d_o")}
    cfg = hga.make_config(xd["q"], x["k_hist"], w.top_chunks, w.top_groups, n_sink_tokens=w.n_sink)
    gs, cs = hga.build_summaries(cfg, x["k_hist"].cuda())
    t = hga.TieredLayerStep(cfg, x["k_hist"].pin_memory(), x["v_hist"].pin_memory(), gs, cs)
    t(xd)
    t.wait(timeout_s=120)
    return t


@pytest.mark.parametrize("name", ["small_bf16", "sink_bf16", "gqa2_ragged_bf16", "tiny_f32"])
def test_tiered_step_matches_oracle(hga, oracle, name):
    """The tiered step against the oracle over the whole history, element by element."""
    w = _wl(name)
    x = HI.make_inputs(w, 0)
    t = _tiered_only(hga, w, x)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32, n_sink=w.n_sink)
    assert np.array_equal(t.chunk_idx.cpu().numpy(), r["chunk_idx"])
    assert np.array_equal(t.group_idx.cpu().numpy(), r["group_idx"])
    args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
    o, lse = oracle.attn_fwd(*args, n_sink=w.n_sink)
    dq, dk, dv = oracle.attn_bwd(*args, x["d_o"], n_sink=w.n_sink)
    err = lambda a, b: float(np.abs(a.float().cpu().numpy() - b).max())
    errs = dict(o=err(t.o, o), dq=err(t.dq, dq), dk=err(t.dk, dk), dv=err(t.dv, dv))
    assert max(errs.values()) <= TOL[w.dtype], errs
    assert err(t.lse, lse) <= LSE_TOL[w.dtype]


def test_tiered_16k_batch4_matches_oracle_sampled(hga, oracle):
    """The tiered-history workload itself (the 16K layer at batch 4, 224 MiB of history K/V in
    pinned host memory): every routing index bit-exact, sampled rows of every batch element (block
    ends included) and the keys at both ends of every 128-key tile of four (batch, KV head) slices."""
    w = HI.WORKLOADS["ctx16k_b4"]
    x = HI.make_inputs(w, 11)             # seed with routing margins >= MIN_GAP (checked on the CPU)
    t = _tiered_only(hga, w, x)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32)
    assert np.array_equal(t.chunk_idx.cpu().numpy(), r["chunk_idx"])
    assert np.array_equal(t.group_idx.cpu().numpy(), r["group_idx"])
    ids = set(HI.sample_ids(w.B * w.Hq * w.seg_len, 96, 7).tolist())
    for b in range(w.B):
        for h in (0, w.Hq - 1):
            for blk in (0, w.nblk - 1):
                base = (b * w.Hq + h) * w.seg_len + blk * 64
                ids |= {base, base + 63}
    rows = np.array(sorted(ids), dtype=np.int64)
    us = sorted({u for t0 in range(0, w.seg_len, 128) for u in (t0, t0 + 127)})
    keys = np.array([(b * w.Hkv + kh) * w.seg_len + u for b in (0, w.B - 1) for kh in (0, w.Hkv - 1) for u in us],
                    dtype=np.int64)
    ref = attn_sampled(oracle, x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"], x["d_o"],
                       rows=rows, keys=keys)
    D = w.D
    got = lambda t_, ids_: t_.reshape(-1, D)[torch.as_tensor(ids_, device=t_.device)].float().cpu().numpy()
    e = dict(o=np.abs(got(t.o, rows) - ref["o"]).max(), dq=np.abs(got(t.dq, rows) - ref["dq"]).max(),
             dk=np.abs(got(t.dk, keys) - ref["dk"]).max(), dv=np.abs(got(t.dv, keys) - ref["dv"]).max(),
             lse=np.abs(t.lse.reshape(-1)[torch.as_tensor(rows, device=t.lse.device)].cpu().numpy()
                        - ref["lse"]).max())
    assert e["lse"] <= 1e-3 and max(e["o"], e["dq"], e["dk"], e["dv"]) <= 2e-2, e


@pytest.mark.parametrize("name", ["small_bf16", "sink_bf16", "tiny_f32", "gqa2_ragged_bf16", "sink_f32"])
def test_tiered_step_equals_resident_step_bitwise(hga, name):
    w = _wl(name)
    x = HI.make_inputs(w, 0)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    cfg, step = _resident(hga, w, xd)
    t = _tiered(hga, cfg, step, x, xd)
    assert torch.equal(t.group_idx, step.group_idx)
    for a, b in [(t.o, step.o), (t.lse, step.lse), (t.dq, step.dq), (t.dk, step.dk), (t.dv, step.dv)]:
        assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["small_bf16", "sink_bf16", "ctx4k"])
def test_tier_plan_is_the_union_of_routed_groups(hga, name):
    w = _wl(name)
    x = HI.make_inputs(w, 0)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    cfg, step = _resident(hga, w, xd)
    t = _tiered(hga, cfg, step, x, xd)
    gi = step.group_idx.cpu().numpy()
    used = t.used_groups.cpu().numpy()
    n_used = t.n_used.cpu().numpy().reshape(w.B, w.Hkv)
    compact = t.compact_idx.cpu().numpy()
    nsg = w.n_sink // 8
    for b in range(w.B):
        for kh in range(w.Hkv):
            want = np.unique(np.concatenate([np.arange(nsg), gi[b, kh].ravel()]))
            assert n_used[b, kh] == want.size <= t.cap
            assert np.array_equal(used[b, kh, :want.size], want)
            assert np.array_equal(compact[b, kh], np.searchsorted(want, gi[b, kh]))
            # the cache rows are the history rows of the used groups, in that order
            rows = (want[:, None] * 8 + np.arange(8)[None, :]).ravel()
            kc = t.k_cache[b, kh, :rows.size].cpu()
            assert torch.equal(kc, x["k_hist"][b, kh, torch.as_tensor(rows)])
    # the gathered bytes are what the plan asked for
    assert t.gather_bytes() == int(n_used.sum()) * 8 * w.D * (2 if w.dtype == "bf16" else 4) * 2


def test_tier_gather_rejects_pageable_host_memory(hga):
    from hierarchical_kv_routing_tok_b200 import _capi as C
    w = HI.WORKLOADS["small_bf16"]
    x = HI.make_inputs(w, 0)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    cfg, step = _resident(hga, w, xd)
    kh = x["k_hist"].clone()                                   # pageable: not readable by the device
    assert not kh.is_pinned()
    cap = C.tier_cache_config(cfg).hist_len // 8
    used = torch.zeros(w.B, w.Hkv, cap, dtype=torch.int32, device="cuda")
    n_used = torch.zeros(w.B * w.Hkv, dtype=torch.int32, device="cuda")
    kc = torch.empty(w.B, w.Hkv, cap * 8, w.D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(C.HGAError) as e:
        C.tier_gather(cfg, kh.data_ptr(), kh.data_ptr(), used.data_ptr(), n_used.data_ptr(), kc.data_ptr(),
                      kc.data_ptr(), 0)
    assert e.value.code == C.HGA_ERR_ARG


def test_tiered_wait_gives_up_at_its_deadline(hga):
    """The host-side wait raises TimeoutError when the step is not done by the deadline (here it is
    queued behind a bounded device sleep), and the step still completes afterwards."""
    w = HI.WORKLOADS["small_bf16"]
    x = HI.make_inputs(w, 0)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    cfg, step = _resident(hga, w, xd)
    t = hga.TieredLayerStep(cfg, x["k_hist"].pin_memory(), x["v_hist"].pin_memory(), step.group_sum,
                            step.chunk_sum)
    torch.cuda._sleep(1_000_000_000)              # ~0.5 s of device spin on the current stream
    t(xd)
    with pytest.raises(TimeoutError):
        t.wait(timeout_s=0.01)
    t.wait(timeout_s=60)
    assert torch.equal(t.o, step.o)
