"""Segment-wise training (TBPTT with a growing detached history) on a B200: incremental summaries,
per-segment attention against the history of all earlier segments, a two-layer model trained
segment by segment against the same model on the oracle, tiered history and causal routing."""
import numpy as np
import pytest
import torch

import hga_inputs as HI

pytestmark = pytest.mark.gpu
MIN_GAP = 4e-6


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_kv_routing_tok_b200 as H
    H.load()
    return H


def _sequence(B, Hq, Hkv, S, nseg, dtype, seed):
    """nseg segments of q, k, v, d_o drawn like the benchmark inputs (per-chunk key offsets)."""
    w = HI.Workload("seq", B, Hq, Hkv, 128, (nseg - 1) * S, S, 1, 1, dtype, 1.0)
    x = HI.make_inputs(w, seed)
    ks = torch.cat([x["k_hist"], x["k_seg"]], dim=2)
    vs = torch.cat([x["v_hist"], x["v_seg"]], dim=2)
    g = torch.Generator().manual_seed(seed + 1)
    segs = []
    for s in range(nseg):
        q = torch.randn(B, Hq, S, 128, generator=g).to(x["q"].dtype)
        d_o = torch.randn(B, Hq, S, 128, generator=g).to(x["q"].dtype)
        segs.append(dict(q=q, k=ks[:, :, s * S:(s + 1) * S].contiguous(), v=vs[:, :, s * S:(s + 1) * S].contiguous(),
                         d_o=d_o))
    return segs


@pytest.mark.parametrize("dtype,tiered", [("f32", False), ("bf16", False), ("bf16", True)])
def test_incremental_summaries_equal_full_rebuild(hga, dtype, tiered):
    from hierarchical_kv_routing_tok_b200 import _capi as C
    B, Hq, Hkv, S, nseg = 2, 8, 2, 256, 4
    segs = _sequence(B, Hq, Hkv, S, nseg, dtype, 3)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    hist = hga.HGAHistory(B, Hq, Hkv, nseg * S, dtype=tdt, tiered=tiered)
    for s, seg in enumerate(segs):
        hist.append(seg["k"].cuda(), seg["v"].cuda())
        L = (s + 1) * S
        full = torch.cat([t["k"] for t in segs[:s + 1]], dim=2).cuda()
        cfg = C.make_config(B, Hq, Hkv, L, 64, 1, 1, dtype=C.HGA_BF16 if dtype == "bf16" else C.HGA_F32)
        gs, cs = hga.build_summaries(cfg, full)
        torch.cuda.synchronize()
        assert torch.equal(hist.group_sum[:, :, :L // 8], gs)
        assert torch.equal(hist.chunk_sum[:, :, :L // 64], cs)
        assert torch.equal(hist.k[:, :, :L].cpu(), full.cpu())


def _clamped(L, kc, kg, n_sink):
    if L == 0:
        return 0, 0, 0
    ns = min(n_sink, L - 64)
    kc2 = min(kc, L // 64 - ns // 64)
    return kc2, min(kg, 8 * kc2), ns


@pytest.mark.parametrize("dtype,n_sink", [("f32", 0), ("bf16", 0), ("bf16", 128)])
def test_segments_match_oracle(hga, oracle, dtype, n_sink):
    """Each segment: routing bit-exact and outputs / gradients against the oracle over the history
    of all earlier segments (the first segment has none: causal prefix only)."""
    B, Hq, Hkv, S, nseg, kc, kg = 1, 4, 1, 128, 4, 2, 12
    segs = _sequence(B, Hq, Hkv, S, nseg, dtype, 5)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    tol = 1e-4 if dtype == "f32" else 2e-2
    hist = hga.HGAHistory(B, Hq, Hkv, nseg * S, dtype=tdt, n_sink_tokens=n_sink)
    for s, seg in enumerate(segs):
        L = s * S
        q, k, v = (seg[n].cuda().requires_grad_(True) for n in ("q", "k", "v"))
        o, gi = hga.segment_attention(q, k, v, hist, kc, kg)
        (o * seg["d_o"].cuda()).sum().backward()
        kc2, kg2, ns = _clamped(L, kc, kg, n_sink)
        kh = torch.cat([t["k"] for t in segs[:s]], dim=2) if s else torch.zeros(B, Hkv, 0, 128, dtype=tdt)
        vh = torch.cat([t["v"] for t in segs[:s]], dim=2) if s else torch.zeros(B, Hkv, 0, 128, dtype=tdt)
        if s:
            r32 = oracle.route_from_inputs(seg["q"], kh, Hkv, kc2, kg2, prec=32, n_sink=ns)
            r64 = oracle.route_from_inputs(seg["q"], kh, Hkv, kc2, kg2, prec=64, n_sink=ns)
            assert np.array_equal(r32["group_idx"], r64["group_idx"])
            assert r64["chunk_gap"].min() >= MIN_GAP and r64["group_gap"].min() >= MIN_GAP
            ogi = r32["group_idx"]
            assert np.array_equal(gi.cpu().numpy(), ogi)
        else:
            ogi = np.zeros((B, Hkv, S // 64, 0), dtype=np.int32)
        args = (seg["q"], kh, vh, seg["k"], seg["v"], ogi)
        o_ref, _ = oracle.attn_fwd(*args, n_sink=ns)
        dq, dk, dv = oracle.attn_bwd(*args, seg["d_o"], n_sink=ns)
        for a, b in [(o, o_ref), (q.grad, dq), (k.grad, dk), (v.grad, dv)]:
            assert float(np.abs(a.detach().float().cpu().numpy() - b).max()) <= tol
        hist.append(k.detach(), v.detach())


def test_tiered_history_equals_device_history(hga):
    B, Hq, Hkv, S, nseg, kc, kg = 2, 8, 2, 256, 3, 3, 16
    segs = _sequence(B, Hq, Hkv, S, nseg, "bf16", 7)
    out = []
    for tiered in (False, True):
        hist = hga.HGAHistory(B, Hq, Hkv, nseg * S, dtype=torch.bfloat16, tiered=tiered, n_sink_tokens=64)
        res = []
        for seg in segs:
            q, k, v = (seg[n].cuda().requires_grad_(True) for n in ("q", "k", "v"))
            o, _ = hga.segment_attention(q, k, v, hist, kc, kg)
            (o * seg["d_o"].cuda()).sum().backward()
            res.append([o.detach(), q.grad, k.grad, v.grad])
            hist.append(k.detach(), v.detach())
        out.append(res)
    for a, b in zip(*out):
        for x, y in zip(a, b):
            assert torch.equal(x, y)


def test_causal_routing_across_segments(hga, oracle):
    """Strictly causal routing with q_prev = the previous segment's last query block."""
    B, Hq, Hkv, S, nseg, kc, kg = 1, 4, 1, 128, 3, 2, 8
    segs = _sequence(B, Hq, Hkv, S, nseg, "f32", 9)
    hist = hga.HGAHistory(B, Hq, Hkv, nseg * S, dtype=torch.float32)
    prev = None
    for s, seg in enumerate(segs):
        q, k, v = (seg[n].cuda() for n in ("q", "k", "v"))
        o, gi = hga.segment_attention(q, k, v, hist, kc, kg, causal=True, q_prev=prev)
        if s:
            kh = torch.cat([t["k"] for t in segs[:s]], dim=2)
            kc2, kg2, _ = _clamped(s * S, kc, kg, 0)
            qp = segs[s - 1]["q"][:, :, -64:]
            r = oracle.route_causal_from_inputs(seg["q"], kh, Hkv, kc2, kg2, q_prev=qp, prec=32)
            assert np.array_equal(gi.cpu().numpy(), r["group_idx"])
        hist.append(k, v)
        prev = q[:, :, -64:].contiguous()


# ----------------------------------------------------------------------------- two-layer model
class _OracleAttention(torch.autograd.Function):
    """The same attention on the CPU oracle (float64), for given routing."""

    @staticmethod
    def forward(ctx, q, k, v, kh, vh, gi, oracle):
        ctx.save_for_backward(q, k, v)
        ctx.kh, ctx.vh, ctx.gi, ctx.oracle = kh, vh, gi, oracle
        o, _ = oracle.attn_fwd(q, kh, vh, k, v, gi)
        return torch.as_tensor(o)

    @staticmethod
    def backward(ctx, d_o):
        q, k, v = ctx.saved_tensors
        dq, dk, dv = ctx.oracle.attn_bwd(q, ctx.kh, ctx.vh, k, v, ctx.gi, d_o)
        return torch.as_tensor(dq), torch.as_tensor(dk), torch.as_tensor(dv), None, None, None, None


def test_two_layer_model_trained_segment_by_segment(hga, oracle):
    """A two-layer residual model with HGA attention, trained by TBPTT over four segments (loss
    back-propagated per segment, each layer's K/V appended to its history at the boundary): the
    per-segment losses and every parameter gradient equal those of the same model whose attention
    is the float64 oracle, run with the routing the GPU chose.  That routing is itself checked: each
    layer's GPU routing of each segment equals the oracle's float32 routing of the same projected q
    and history keys (copied to the host), whose selection margins are checked to be >= MIN_GAP."""
    B, Hq, Hkv, D, S, nseg, dm, kc, kg = 1, 4, 1, 128, 128, 4, 32, 2, 8
    g = torch.Generator().manual_seed(21)
    params = {n: torch.randn(*shape, generator=g, dtype=torch.float64) * 0.3
              for n, shape in [("wq0", (dm, Hq * D)), ("wk0", (dm, Hkv * D)), ("wv0", (dm, Hkv * D)),
                               ("wo0", (Hq * D, dm)), ("wq1", (dm, Hq * D)), ("wk1", (dm, Hkv * D)),
                               ("wv1", (dm, Hkv * D)), ("wo1", (Hq * D, dm))]}
    xs = [torch.randn(B, S, dm, generator=g, dtype=torch.float64) for _ in range(nseg)]
    tgt = [torch.randn(B, S, dm, generator=g, dtype=torch.float64) for _ in range(nseg)]

    def heads(t, n):
        return t.view(B, S, n, D).transpose(1, 2).contiguous()

    # GPU model (float32)
    pg = {n: p.float().cuda().requires_grad_(True) for n, p in params.items()}
    hists = [hga.HGAHistory(B, Hq, Hkv, nseg * S, dtype=torch.float32) for _ in range(2)]
    losses_gpu, routing = [], []
    past_k = [[], []]                                     # host copies of each layer's earlier keys
    for s in range(nseg):
        h = xs[s].float().cuda()
        kv, gis = [], []
        for l in range(2):
            q, k, v = (heads(h @ pg[f"w{c}{l}"], n) for c, n in (("q", Hq), ("k", Hkv), ("v", Hkv)))
            o, gi = hga.segment_attention(q, k, v, hists[l], kc, kg)
            h = h + o.transpose(1, 2).reshape(B, S, Hq * D) @ pg[f"wo{l}"]
            kv.append((k.detach(), v.detach()))
            if hists[l].length:
                # the routing the GPU chose, against the oracle on the same float32 q and history keys
                kc2, kg2, _ = _clamped(hists[l].length, kc, kg, 0)
                qh, kh = q.detach().cpu(), torch.cat(past_k[l], dim=2)
                r32 = oracle.route_from_inputs(qh, kh, Hkv, kc2, kg2, prec=32)
                r64 = oracle.route_from_inputs(qh, kh, Hkv, kc2, kg2, prec=64)
                assert np.array_equal(r32["group_idx"], r64["group_idx"])
                assert r64["chunk_gap"].min() >= MIN_GAP and r64["group_gap"].min() >= MIN_GAP
                assert np.array_equal(gi.cpu().numpy(), r32["group_idx"]), (s, l)
                gis.append(r32["group_idx"])
            else:
                gis.append(np.zeros((B, Hkv, S // 64, 0), np.int32))
            past_k[l].append(k.detach().cpu())
        loss = ((h - tgt[s].float().cuda()) ** 2).mean()
        loss.backward()                                   # truncated: history is detached
        losses_gpu.append(loss.item())
        routing.append(gis)
        for l in range(2):
            hists[l].append(*kv[l])

    # the same model on the oracle (float64, CPU), with the GPU's routing
    pc = {n: p.clone().requires_grad_(True) for n, p in params.items()}
    hk = [[], []]
    losses_ref = []
    for s in range(nseg):
        h = xs[s]
        for l in range(2):
            q, k, v = (heads(h @ pc[f"w{c}{l}"], n) for c, n in (("q", Hq), ("k", Hkv), ("v", Hkv)))
            kh = torch.cat([a for a, _ in hk[l]], dim=2) if hk[l] else torch.zeros(B, Hkv, 0, D, dtype=torch.float64)
            vh = torch.cat([b for _, b in hk[l]], dim=2) if hk[l] else torch.zeros(B, Hkv, 0, D, dtype=torch.float64)
            o = _OracleAttention.apply(q, k, v, kh, vh, routing[s][l], oracle)
            h = h + o.transpose(1, 2).reshape(B, S, Hq * D) @ pc[f"wo{l}"]
            hk[l].append((k.detach(), v.detach()))
        loss = ((h - tgt[s]) ** 2).mean()
        loss.backward()
        losses_ref.append(loss.item())
    np.testing.assert_allclose(losses_gpu, losses_ref, rtol=1e-4)
    for n in params:
        a, b = pg[n].grad.double().cpu(), pc[n].grad
        assert float((a - b).abs().max()) <= 1e-3 * float(b.abs().max()), n   # float32 vs float64
