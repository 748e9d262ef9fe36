"""The device cache of group summaries (history's group-summary table in pinned host memory, a
fixed number of chunk slots per (batch, KV head) in device memory, misses fetched per step) on a
B200: over several steps that route different queries against one history, with caches smaller
than the history, the routing equals the oracle's bit for bit, the slot assignment and the hit /
miss counts equal a plain least-recently-used model of the cache, and the cached summaries are the
host table's values; the tiered layer step routed through the cache matches the oracle."""
import numpy as np
import pytest
import torch

import hga_inputs as HI

pytestmark = pytest.mark.gpu

# 2 batches x 2 KV heads, 4096 history tokens (64 chunks), 4 query blocks choosing 4 chunks each:
# a step chooses 13-16 chunks per (batch, KV head), so 24 slots hold one step but not two
SMALL = HI.Workload("gcache_small", 2, 8, 2, 128, 4096, 256, 4, 16, "bf16", 1.0)


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_kv_routing_tok_b200 as H
    H.load()
    return H


def lru_model(steps, cap, nch):
    """The cache policy in plain Python: per step, the chosen chunks (ascending) that hold a slot
    are hits (their slot's stamp becomes the step); the others take, in ascending chunk order, the
    slots holding no chosen chunk in (stamp, slot) order -- empty slots have stamp -1 -- and those
    slots' old chunks lose their slot."""
    slot_of, chunk_of, stamp = [-1] * nch, [-1] * cap, [-1] * cap
    out = []
    for step, need in enumerate(steps):
        needset = set(need)
        hits, misses = 0, []
        for c in need:
            s = slot_of[c]
            if s >= 0:
                stamp[s] = step
                hits += 1
            else:
                misses.append(c)
        free = sorted((s for s in range(cap) if chunk_of[s] < 0 or chunk_of[s] not in needset),
                      key=lambda s: (stamp[s], s))
        placed = min(len(misses), len(free))
        evicted = 0
        for i in range(placed):
            s = free[i]
            if chunk_of[s] >= 0:
                slot_of[chunk_of[s]] = -1
                evicted += 1
            chunk_of[s], slot_of[misses[i]], stamp[s] = misses[i], s, step
        out.append((hits, placed, list(slot_of), list(chunk_of), evicted))
    return out


def _run_steps(hga, oracle, w, cap, q_seeds, hist_seed=0):
    C = hga._capi
    xh = HI.make_inputs(w, hist_seed)
    kh_dev = xh["k_hist"].cuda()
    cfg = hga.make_config(xh["q"], kh_dev, w.top_chunks, w.top_groups)
    gs, cs = hga.build_summaries(cfg, kh_dev)
    gs_host = gs.cpu().pin_memory()                       # the group-summary table lives in host memory
    cache = hga.GroupSummaryCache(cfg, gs_host, cap)
    ws = hga.new_workspace(cfg, kh_dev.device)
    ci = torch.empty(w.B, w.Hkv, w.nblk, w.top_chunks, dtype=torch.int32, device="cuda")
    gi = torch.empty(w.B, w.Hkv, w.nblk, w.top_groups, dtype=torch.int32, device="cuda")
    unions = {(b, kh): [] for b in range(w.B) for kh in range(w.Hkv)}
    gpu = []
    for s in q_seeds:
        q = HI.make_inputs(w, s)["q"]
        cache.route(q.cuda(), cs, ci, gi, ws)
        torch.cuda.synchronize()
        assert hga.read_status(ws) == C.HGA_OK
        r = oracle.route_from_inputs(q, xh["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32)
        assert np.array_equal(ci.cpu().numpy(), r["chunk_idx"]), s
        assert np.array_equal(gi.cpu().numpy(), r["group_idx"]), s
        for b in range(w.B):
            for kh in range(w.Hkv):
                unions[(b, kh)].append(sorted(set(r["chunk_idx"][b, kh].ravel().tolist())))
        gpu.append((cache.counts.cpu().numpy().reshape(w.B, w.Hkv, 2), cache.slot_of.cpu().numpy(),
                    cache.chunk_of.cpu().numpy()))
    return cache, gs_host, unions, gpu


def test_cached_routing_over_steps_matches_oracle_and_lru_model(hga, oracle):
    w, cap = SMALL, 24
    cache, gs_host, unions, gpu = _run_steps(hga, oracle, w, cap, q_seeds=[0, 1, 2, 3, 4, 5])
    evictions = 0
    for b in range(w.B):
        for kh in range(w.Hkv):
            model = lru_model(unions[(b, kh)], cap, w.nch)
            for step, (hits, placed, slot_of, chunk_of, evicted) in enumerate(model):
                counts, so, co = gpu[step]
                assert counts[b, kh].tolist() == [hits, placed], (b, kh, step)
                assert hits + placed == len(unions[(b, kh)][step])
                assert so[b, kh].tolist() == slot_of and co[b, kh].tolist() == chunk_of, (b, kh, step)
                evictions += evicted
    assert evictions > 0                                  # the cache is smaller than the steps' chunks
    # every occupied slot holds its chunk's 8 group summaries exactly as in the host table
    gc = cache.gcache.cpu()
    co = cache.chunk_of.cpu()
    for b in range(w.B):
        for kh in range(w.Hkv):
            for s in range(cap):
                c = int(co[b, kh, s])
                if c >= 0:
                    assert torch.equal(gc[b, kh, s], gs_host[b, kh, 8 * c:8 * c + 8])


def test_cached_routing_16k_below_history_size(hga, oracle):
    """The 16K layer with 216 chunk slots per KV head (1728 of its 1792 group summaries): three steps,
    routing bit-exact to the oracle, counts equal to the model's."""
    w, cap = HI.WORKLOADS["ctx16k"], 216
    _, _, unions, gpu = _run_steps(hga, oracle, w, cap, q_seeds=[0, 2, 1])
    for kh in range(w.Hkv):
        model = lru_model(unions[(0, kh)], cap, w.nch)
        for step, (hits, placed, slot_of, _, _) in enumerate(model):
            counts, so, _ = gpu[step]
            assert counts[0, kh].tolist() == [hits, placed]
            assert so[0, kh].tolist() == slot_of


def test_cache_smaller_than_a_step_is_reported(hga):
    """8 slots for a step that chooses 13-16 chunks: the plan records HGA_ERR_ARG, the level-2 routing
    reads only slots that exist and records it too; nothing is read out of bounds."""
    C = hga._capi
    w = SMALL
    xh = HI.make_inputs(w, 0)
    kh_dev = xh["k_hist"].cuda()
    q = xh["q"].cuda()
    cfg = hga.make_config(q, kh_dev, w.top_chunks, w.top_groups)
    gs, cs = hga.build_summaries(cfg, kh_dev)
    cache = hga.GroupSummaryCache(cfg, gs.cpu().pin_memory(), 8)
    ws = hga.new_workspace(cfg, q.device)
    ci = torch.empty(w.B, w.Hkv, w.nblk, w.top_chunks, dtype=torch.int32, device="cuda")
    gi = torch.empty(w.B, w.Hkv, w.nblk, w.top_groups, dtype=torch.int32, device="cuda")
    cache.route(q, cs, ci, gi, ws)
    torch.cuda.synchronize()
    assert hga.read_status(ws) == C.HGA_ERR_ARG
    assert (cache.counts[:, 1] <= 8).all()


@pytest.mark.parametrize("name", ["small_bf16", "sink_bf16"])
def test_tiered_step_through_group_cache_matches_oracle(hga, oracle, name):
    """The pages' three tiers: chunk summaries in device memory, group summaries in host memory behind
    the device cache, K/V in host memory gathered per step."""
    w = HI.WORKLOADS.get(name) or HI.EDGE_WORKLOADS[name]
    x = HI.make_inputs(w, 0)
    xd = {k: x[k].cuda() for k in ("q", "k_seg", "v_seg", "d_o")}
    cfg = hga.make_config(xd["q"], x["k_hist"], w.top_chunks, w.top_groups, n_sink_tokens=w.n_sink)
    gs, cs = hga.build_summaries(cfg, x["k_hist"].cuda())
    nch_routable = (w.hist_len - w.n_sink) // 64
    cap = min(nch_routable, w.nblk * w.top_chunks)        # always holds a step's chosen chunks
    cache = hga.GroupSummaryCache(cfg, gs.cpu().pin_memory(), cap)
    del gs                                                # no device copy of the group summaries
    t = hga.TieredLayerStep(cfg, x["k_hist"].pin_memory(), x["v_hist"].pin_memory(), None, cs,
                            group_cache=cache)
    t(xd)
    t.wait(timeout_s=120)
    st = cache.stats()
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32, n_sink=w.n_sink)
    assert np.array_equal(t.group_idx.cpu().numpy(), r["group_idx"])
    nchosen = sum(len(set(r["chunk_idx"][b, kh].ravel().tolist())) for b in range(w.B) for kh in range(w.Hkv))
    assert st["hits"] == 0 and st["misses"] == nchosen and st["host_bytes"] == nchosen * 4096   # a cold cache
    args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
    o, lse = oracle.attn_fwd(*args, n_sink=w.n_sink)
    dq, dk, dv = oracle.attn_bwd(*args, x["d_o"], n_sink=w.n_sink)
    err = lambda a, b: float(np.abs(a.float().cpu().numpy() - b).max())
    assert max(err(t.o, o), err(t.dq, dq), err(t.dk, dk), err(t.dv, dv)) <= 2e-2
    assert err(t.lse, lse) <= 1e-3
    t(xd)                                                 # the same step again: every chosen chunk hits
    t.wait(timeout_s=120)
    st = cache.stats()
    assert st["misses"] == 0 and st["hits"] == nchosen
    assert torch.equal(t.group_idx.cpu(), torch.as_tensor(r["group_idx"]))
