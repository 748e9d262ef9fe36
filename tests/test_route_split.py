"""Routing of long histories in three launches (block queries; every chunk of a (batch, KV head)
scored against all of its block queries in one pass; selection and the group level) on a B200: it
computes each score with the same float32 operations in the same order as the single launch (the
same four-term lane products, summed over the lanes in the same pairing), so both give the same
chunk and group indices bit for bit, with and without sink chunks, for the standard and the
strictly causal routing, at ragged sizes (routable chunks not a multiple of 4, block counts not a
multiple of 32, odd G) and at the full 131K layer.  The 131K parity tests route through the
workspace, so this path is also checked against the oracle there."""
import numpy as np
import pytest
import torch

import hga_inputs as HI

pytestmark = pytest.mark.gpu

RAGGED = [
    # B, Hq, Hkv, history, segment, top_chunks, top_groups, sink
    HI.Workload("split_ragged", 2, 6, 2, 128, 64 * 514 + 128, 192, 5, 17, "bf16", 0.5, n_sink=128),
    HI.Workload("split_f32", 1, 4, 2, 128, 64 * 515, 2048 + 64, 9, 40, "f32", 0.5),
    HI.Workload("split_min", 1, 8, 4, 128, 64 * 512, 64, 1, 1, "bf16", 0.5),
]


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_kv_routing_tok_b200 as H
    H.load()
    return H


def _both(hga, w, seed=0, causal=False):
    C = hga._capi
    x = HI.make_inputs(w, seed)
    q = x["q"].cuda()
    kh = x["k_hist"].cuda()
    cfg = hga.make_config(q, kh, w.top_chunks, w.top_groups, n_sink_tokens=w.n_sink)
    ws = hga.new_workspace(cfg, q.device)
    assert hga._capi.route_launches(cfg) == 3           # long enough for the three launches
    gs, cs = hga.build_summaries(cfg, kh, workspace=ws)
    q_prev = torch.randn(w.B, w.Hq, 64, w.D, generator=torch.Generator().manual_seed(seed + 7)).to(q.dtype).cuda() \
        if causal else None
    split = hga.route(cfg, q, gs, cs, workspace=ws, causal=causal, q_prev=q_prev)
    single = hga.route(cfg, q, gs, cs, workspace=None, causal=causal, q_prev=q_prev)
    torch.cuda.synchronize()
    assert hga.read_status(ws) == C.HGA_OK
    return [t.cpu().numpy() for t in split], [t.cpu().numpy() for t in single], x


@pytest.mark.parametrize("w", RAGGED, ids=lambda w: w.name)
@pytest.mark.parametrize("causal", [False, True])
def test_split_equals_single_launch_ragged(hga, w, causal):
    (ci_s, gi_s), (ci_1, gi_1), _ = _both(hga, w, causal=causal)
    assert np.array_equal(ci_s, ci_1) and np.array_equal(gi_s, gi_1)
    assert (np.diff(gi_s, axis=-1) > 0).all()           # ascending, no repeats


@pytest.mark.parametrize("name", ["ctx131k"])
def test_split_equals_single_launch_full_size(hga, name):
    (ci_s, gi_s), (ci_1, gi_1), _ = _both(hga, HI.WORKLOADS[name])
    assert np.array_equal(ci_s, ci_1) and np.array_equal(gi_s, gi_1)


def test_split_ragged_matches_oracle(hga, oracle):
    """The ragged sink case against the oracle deciding in float32 (seed with margins: every
    selection boundary's float64 gap at least 4e-6 and the float32 and float64 routings equal)."""
    w = RAGGED[0]
    (ci_s, gi_s), _, x = _both(hga, w, seed=1)
    r32 = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32, n_sink=w.n_sink)
    r64 = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=64, n_sink=w.n_sink)
    assert np.array_equal(r32["group_idx"], r64["group_idx"]) and np.array_equal(r32["chunk_idx"], r64["chunk_idx"])
    assert r64["chunk_gap"].min() >= 4e-6 and r64["group_gap"].min() >= 4e-6
    assert np.array_equal(ci_s, r32["chunk_idx"]) and np.array_equal(gi_s, r32["group_idx"])


@pytest.mark.parametrize("fill", [0.25, 0.0])
def test_large_selection_ties_go_to_lower_index(hga, fill):
    """All history keys equal, so every score ties: 600 routable chunks (more candidates than a CTA
    has threads, so the filtered selection falls back to the radix select) and 320 candidate groups
    (filtered, then ranked): the lowest indices are selected, by the three launches and by one."""
    w = HI.Workload("split_ties", 1, 4, 2, 128, 64 * 600, 128, 40, 300, "bf16", 0.5)
    x = HI.make_inputs(w, 0)
    q = x["q"].cuda()
    kh = torch.full_like(x["k_hist"], fill).cuda()
    cfg = hga.make_config(q, kh, w.top_chunks, w.top_groups)
    ws = hga.new_workspace(cfg, q.device)
    gs, cs = hga.build_summaries(cfg, kh, workspace=ws)
    for workspace in (ws, None):
        ci, gi = hga.route(cfg, q, gs, cs, workspace=workspace)
        torch.cuda.synchronize()
        assert (ci.cpu() == torch.arange(w.top_chunks, dtype=torch.int32)).all()
        assert (gi.cpu() == torch.arange(w.top_groups, dtype=torch.int32)).all()


def test_layer_step_with_split_routing_and_paired_dkdv_matches_oracle(hga, oracle):
    """A whole layer step (summaries, three-launch routing, forward, backward) on one workspace whose
    region after the delta rows serves first as the routing scratch and then as the dK/dV exchange
    area (4 key tiles x 2 KV heads = 8 units, so the dK/dV kernel pairs CTAs): routing bit-exact,
    outputs and gradients within the bf16 bars of the oracle."""
    w = HI.Workload("split_step", 1, 8, 2, 128, 64 * 520, 512, 8, 32, "bf16", 0.5)
    x = HI.make_inputs(w, 0)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    cfg = hga.make_config(xd["q"], xd["k_hist"], w.top_chunks, w.top_groups)
    assert hga._capi.route_launches(cfg) == 3
    step = hga.LayerStep(cfg)
    step(xd)
    torch.cuda.synchronize()
    assert hga.read_status(step.ws) == hga._capi.HGA_OK
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32)
    assert np.array_equal(step.chunk_idx.cpu().numpy(), r["chunk_idx"])
    assert np.array_equal(step.group_idx.cpu().numpy(), r["group_idx"])
    args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
    o, lse = oracle.attn_fwd(*args)
    dq, dk, dv = oracle.attn_bwd(*args, x["d_o"])
    err = lambda a, b: float(np.abs(a.float().cpu().numpy() - b).max())
    assert max(err(step.o, o), err(step.dq, dq), err(step.dk, dk), err(step.dv, dv)) <= 2e-2
    assert err(step.lse, lse) <= 1e-3
