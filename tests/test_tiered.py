"""Tiered history (history K/V in pinned host memory, compact device cache per step) on a B200:
the plan is the exact union of the routed groups with order-preserving positions, the gather
copies exactly those rows, and the whole tiered step equals the step over device-resident
history bit for bit (hence the oracle parity of the resident step carries over)."""
import numpy as np
import pytest
import torch

import hga_inputs as HI

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
