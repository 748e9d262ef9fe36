"""Pins of the CPU oracle against things other than itself (CPU only).

Each test names what fixes the expected result: a closed form, brute force on a
tiny input, a library routine the method reduces to (torch
``scaled_dot_product_attention`` in float64, with GQA head mapping and autograd),
finite differences, or the hand-derived worked example in
``tests/golden/worked_example.json``.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import hga_inputs as HI

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- summaries
@pytest.mark.parametrize("prec", [64, 32])
def test_summaries_closed_form_offset_plus_zero_mean_pattern(oracle, prec):
    """Keys = per-chunk constant + a pattern whose every 8-row group sums to exactly 0
    (rows a,-a,b,-b,...): group and chunk summaries equal the constant exactly."""
    rng = np.random.default_rng(1)
    B, Hkv, H, D = 2, 3, 256, 16
    c = rng.integers(-64, 64, size=(B, Hkv, H // 64, D)) / 8.0
    half = rng.integers(-100, 100, size=(B, Hkv, H // 2, D)) / 4.0
    pattern = np.stack([half, -half], axis=3).reshape(B, Hkv, H, D)
    k = np.repeat(c, 64, axis=2) + pattern
    gs = oracle.group_summaries(k, 8, prec)
    cs = oracle.chunk_summaries(k, 64, prec)
    assert np.array_equal(gs, np.repeat(c, 8, axis=2))
    assert np.array_equal(cs, c)


def test_summaries_one_hot_position(oracle):
    """A single non-zero key at position t0 lands in group t0//8 (value/8) and chunk t0//64
    (value/64); every other summary is 0."""
    B, Hkv, H, D = 1, 2, 256, 4
    for kh, t0 in [(0, 0), (1, 7), (0, 8), (1, 63), (0, 64), (1, 255)]:
        k = np.zeros((B, Hkv, H, D))
        k[0, kh, t0] = [8.0, -16.0, 64.0, 1.0]
        gs = oracle.group_summaries(k)
        cs = oracle.chunk_summaries(k)
        eg = np.zeros_like(gs); eg[0, kh, t0 // 8] = k[0, kh, t0] / 8
        ec = np.zeros_like(cs); ec[0, kh, t0 // 64] = k[0, kh, t0] / 64
        assert np.array_equal(gs, eg) and np.array_equal(cs, ec)


def test_chunk_summary_is_mean_of_its_group_summaries(oracle):
    """Closed-form relation: a 64-token mean equals the mean of its eight 8-token means."""
    x = HI.make_inputs(HI.WORKLOADS["tiny_f32"], 3)
    gs = oracle.group_summaries(x["k_hist"])
    cs = oracle.chunk_summaries(x["k_hist"])
    B, Hkv, ngr, D = gs.shape
    np.testing.assert_allclose(gs.reshape(B, Hkv, ngr // 8, 8, D).mean(axis=3), cs, rtol=0, atol=1e-14)


def test_block_query_one_hot_gqa_mapping(oracle):
    """One non-zero query (h0, t0) with Hq=4, Hkv=2 lands only in KV head h0 // 2 and block
    t0 // 64, divided by G*qblock = 128 (query head h belongs to KV head h // G)."""
    B, Hq, Hkv, S, D = 1, 4, 2, 128, 3
    for h0, t0 in itertools.product(range(4), (0, 63, 64, 127)):
        q = np.zeros((B, Hq, S, D))
        q[0, h0, t0] = [128.0, -256.0, 1.0]
        qb = oracle.block_query(q, Hkv)
        e = np.zeros((B, Hkv, 2, D)); e[0, h0 // 2, t0 // 64] = q[0, h0, t0] / 128
        assert np.array_equal(qb, e)


# --------------------------------------------------------------------------- top-k
def test_topk_equals_best_subset_brute_force(oracle):
    """For distinct scores the top-k set is the k-subset with the largest sum (enumerated)."""
    rng = np.random.default_rng(2)
    for n in range(1, 8):
        for k in range(1, n + 1):
            s = rng.standard_normal(n)
            best = max(itertools.combinations(range(n), k), key=lambda c: s[list(c)].sum())
            sel, gap = oracle.topk(s, k)
            assert list(sel) == sorted(best)
            srt = np.sort(s)[::-1]
            assert gap == (srt[k - 1] - srt[k] if k < n else math.inf)


def test_topk_ties_go_to_lower_index(oracle):
    assert list(oracle.topk([1, 3, 3, 2], 2)[0]) == [1, 2]
    assert list(oracle.topk([1, 3, 3, 2], 1)[0]) == [1]
    assert list(oracle.topk([5, 5, 5, 5, 5], 3)[0]) == [0, 1, 2]
    assert list(oracle.topk([0.0, -0.0, 1.0], 2)[0]) == [0, 2]
    assert list(oracle.topk([-0.0, 0.0, -1.0], 1)[0]) == [0]
    assert list(oracle.topk([2, 7, 2, 2, 7], 3)[0]) == [0, 1, 4]


# --------------------------------------------------------------------------- routing
@pytest.mark.parametrize("prec", [64, 32])
def test_route_brute_force_tiny(oracle, prec):
    """Chunk set = best kc-subset of chunk scores; group set = best kg-subset of the groups of
    the chosen chunks (scores by numpy dot products), for random tiny summaries."""
    rng = np.random.default_rng(3)
    B, Hkv, nblk, D, nch, gpc, kc, kg = 1, 2, 3, 8, 6, 4, 2, 3
    for _ in range(10):
        qb = rng.standard_normal((B, Hkv, nblk, D)).astype(np.float32).astype(np.float64)
        gs = rng.standard_normal((B, Hkv, nch * gpc, D)).astype(np.float32).astype(np.float64)
        cs = rng.standard_normal((B, Hkv, nch, D)).astype(np.float32).astype(np.float64)
        ci, gi, _, _ = oracle.route(qb, gs, cs, kc, kg, prec)
        for kh, n in itertools.product(range(Hkv), range(nblk)):
            sc = cs[0, kh] @ qb[0, kh, n]
            best_c = max(itertools.combinations(range(nch), kc), key=lambda c: sc[list(c)].sum())
            assert list(ci[0, kh, n]) == sorted(best_c)
            cand = [c * gpc + r for c in best_c for r in range(gpc)]
            sg = gs[0, kh] @ qb[0, kh, n]
            best_g = max(itertools.combinations(cand, kg), key=lambda c: sg[list(c)].sum())
            assert list(gi[0, kh, n]) == sorted(best_g)


def test_route_planted_chunks_are_selected(oracle):
    """Block n's queries and the keys of one history chunk i_n share a strong direction u_n:
    chunk i_n is selected for block n and its planted group is among the selected groups."""
    g = torch.Generator().manual_seed(5)
    B, Hq, Hkv, D, H, S = 1, 4, 2, 32, 1024, 256
    q = torch.randn(B, Hq, S, D, generator=g) * 0.1
    k = torch.randn(B, Hkv, H, D, generator=g) * 0.1
    planted = {}
    for kh in range(Hkv):
        chunks = torch.randperm(H // 64, generator=g)[: S // 64]
        for n in range(S // 64):
            u = torch.randn(D, generator=g); u /= u.norm()
            i = int(chunks[n]); j = i * 8 + int(torch.randint(8, (1,), generator=g))
            q[0, kh * 2:(kh + 1) * 2, n * 64:(n + 1) * 64] += u
            k[0, kh, j * 8:(j + 1) * 8] += 8 * u
            planted[(kh, n)] = (i, j)
    r = oracle.route_from_inputs(q, k, Hkv, 2, 4, prec=64)
    for (kh, n), (i, j) in planted.items():
        assert i in r["chunk_idx"][0, kh, n]
        assert j in r["group_idx"][0, kh, n]


def test_route_invariants_tiny_workload(oracle):
    w = HI.WORKLOADS["tiny_f32"]
    x = HI.make_inputs(w, 0)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups)
    ci, gi = r["chunk_idx"], r["group_idx"]
    assert ci.shape == (1, 1, w.nblk, w.top_chunks) and gi.shape == (1, 1, w.nblk, w.top_groups)
    for n in range(w.nblk):
        c, gg = ci[0, 0, n], gi[0, 0, n]
        assert (np.diff(c) > 0).all() and (np.diff(gg) > 0).all()
        assert c.min() >= 0 and c.max() < w.nch
        assert set(gg // 8) <= set(c)                       # groups lie in the chosen chunks
        assert gg.max() * 8 + 7 < w.hist_len                # history only


def test_route_permutation_equivariance(oracle):
    """Reordering the history chunks reorders the selection the same way."""
    w = HI.WORKLOADS["tiny_f32"]
    x = HI.make_inputs(w, 1)
    perm = torch.randperm(w.nch, generator=torch.Generator().manual_seed(9))
    kp = x["k_hist"].reshape(1, 1, w.nch, 64, w.D)[:, :, perm].reshape(x["k_hist"].shape)
    r0 = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=64)
    r1 = oracle.route_from_inputs(x["q"], kp, w.Hkv, w.top_chunks, w.top_groups, prec=64)
    inv = torch.argsort(perm).numpy()                      # old chunk id -> new position
    for n in range(w.nblk):
        assert sorted(inv[r0["chunk_idx"][0, 0, n]]) == list(r1["chunk_idx"][0, 0, n])
        old = r0["group_idx"][0, 0, n]
        assert sorted(inv[old // 8] * 8 + old % 8) == list(r1["group_idx"][0, 0, n])


# --------------------------------------------------------------------------- attention
def _small_layer(seed, B=1, Hq=4, Hkv=2, D=16, H=256, S=128):
    g = torch.Generator().manual_seed(seed)
    t = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)
    return dict(q=t(B, Hq, S, D), k_hist=t(B, Hkv, H, D), v_hist=t(B, Hkv, H, D),
                k_seg=t(B, Hkv, S, D), v_seg=t(B, Hkv, S, D), d_o=t(B, Hq, S, D))


def _mask_from_groups(group_idx, B, Hq, Hkv, H, S, group=8, qblock=64, n_sink=0):
    """Boolean [B, Hq, S, H+S]: history position p visible to query t iff p < n_sink or p // group
    is one of the block's routed groups; segment key u visible iff u <= t."""
    G = Hq // Hkv
    m = torch.zeros(B, Hq, S, H + S, dtype=torch.bool)
    m[:, :, :, :n_sink] = True
    gi = torch.as_tensor(np.asarray(group_idx), dtype=torch.long)
    for b, h in itertools.product(range(B), range(Hq)):
        for n in range(S // qblock):
            for j in gi[b, h // G, n].tolist():
                m[b, h, n * qblock:(n + 1) * qblock, j * group:(j + 1) * group] = True
    m[:, :, :, H:] = torch.tril(torch.ones(S, S, dtype=torch.bool))
    return m


def _sdpa_reference(x, mask, scale):
    """Library routine: torch SDPA over [history | segment] with the given mask and GQA
    head mapping, float64, autograd for q and the segment K/V only (history detached)."""
    q = x["q"].clone().requires_grad_(True)
    ks = x["k_seg"].clone().requires_grad_(True)
    vs = x["v_seg"].clone().requires_grad_(True)
    k = torch.cat([x["k_hist"].detach(), ks], dim=2)
    v = torch.cat([x["v_hist"].detach(), vs], dim=2)
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale, enable_gqa=True)
    (o * x["d_o"]).sum().backward()
    G = q.shape[1] // k.shape[1]
    logits = torch.einsum("bhsd,bhtd->bhst", q.detach(), k.repeat_interleave(G, dim=1).detach()) * scale
    lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1)
    return o.detach(), lse, q.grad, ks.grad, vs.grad


def _check_against_sdpa(oracle, x, group_idx, H, S, n_sink=0):
    B, Hq = x["q"].shape[:2]
    Hkv = x["k_hist"].shape[1]
    scale = 1 / math.sqrt(x["q"].shape[-1])
    mask = _mask_from_groups(group_idx, B, Hq, Hkv, H, S, n_sink=n_sink)
    o_ref, lse_ref, dq_ref, dk_ref, dv_ref = _sdpa_reference(x, mask, scale)
    o, lse = oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], group_idx,
                             n_sink=n_sink)
    dq, dk, dv = oracle.attn_bwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"],
                                 group_idx, x["d_o"], n_sink=n_sink)
    for a, b in [(o, o_ref), (lse, lse_ref), (dq, dq_ref), (dk, dk_ref), (dv, dv_ref)]:
        np.testing.assert_allclose(a, b.numpy(), rtol=1e-10, atol=1e-10)


def test_dense_equivalence_with_full_budget(oracle):
    """k_c = all chunks, k_g = all groups: routed HGA == dense causal attention over
    [history | segment] (torch SDPA), forward, LSE and gradients."""
    H, S = 256, 128
    x = _small_layer(0, H=H, S=S)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], 2, H // 64, H // 8, prec=64)
    assert (r["group_idx"] == np.arange(H // 8)).all()
    _check_against_sdpa(oracle, x, r["group_idx"], H, S)


def test_routed_attention_equals_masked_dense_attention(oracle):
    """Any routing: output == masked dense attention with mask = key set (torch SDPA)."""
    H, S = 256, 128
    x = _small_layer(1, H=H, S=S)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], 2, 2, 5, prec=64)
    _check_against_sdpa(oracle, x, r["group_idx"], H, S)
    g = torch.Generator().manual_seed(4)
    rand_gi = np.stack([np.sort(torch.randperm(H // 8, generator=g)[:3].numpy())
                        for _ in range(2 * (S // 64))]).reshape(1, 2, S // 64, 3).astype(np.int32)
    _check_against_sdpa(oracle, x, rand_gi, H, S)


def test_sink_window_dense_equivalence_with_full_budget(oracle):
    """Sink of two chunks + every other chunk and group routed: HGA == dense causal attention
    over [history | segment]; the sink chunks are never routed."""
    H, S, ns = 256, 128, 128
    x = _small_layer(5, H=H, S=S)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], 2, (H - ns) // 64, (H - ns) // 8, prec=64, n_sink=ns)
    assert (r["chunk_idx"] >= ns // 64).all()
    assert (r["group_idx"] == np.arange(ns // 8, H // 8)).all()
    _check_against_sdpa(oracle, x, r["group_idx"], H, S, n_sink=ns)


def test_sink_window_equals_masked_dense_attention(oracle):
    """Sink tokens are visible to every query, next to the routed groups and the causal prefix."""
    H, S, ns = 256, 128, 64
    x = _small_layer(6, H=H, S=S)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], 2, 2, 5, prec=64, n_sink=ns)
    assert (r["chunk_idx"] >= 1).all() and (r["group_idx"] >= ns // 8).all()
    _check_against_sdpa(oracle, x, r["group_idx"], H, S, n_sink=ns)
    # the sink changes the output (it is attended, not ignored)
    o0, _ = oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
    o1, _ = oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"],
                            n_sink=ns)
    assert np.abs(o0 - o1).max() > 1e-3


def test_route_brute_force_with_sink(oracle):
    """With n_sink_chunks sink chunks the chunk set is the best kc-subset of the other chunks."""
    rng = np.random.default_rng(8)
    B, Hkv, nblk, D, nch, gpc, nsc, kc, kg = 1, 1, 3, 8, 7, 4, 2, 2, 3
    for _ in range(10):
        qb = rng.standard_normal((B, Hkv, nblk, D))
        gs = rng.standard_normal((B, Hkv, nch * gpc, D))
        cs = rng.standard_normal((B, Hkv, nch, D))
        cs[..., :nsc, :] += 10 * qb[..., :1, :]        # sink chunks would win if they were routable
        ci, gi, _, _ = oracle.route(qb, gs, cs, kc, kg, 64, n_sink_chunks=nsc)
        for n in range(nblk):
            sc = cs[0, 0] @ qb[0, 0, n]
            best_c = max(itertools.combinations(range(nsc, nch), kc), key=lambda c: sc[list(c)].sum())
            assert list(ci[0, 0, n]) == sorted(best_c)
            cand = [c * gpc + r for c in best_c for r in range(gpc)]
            sg = gs[0, 0] @ qb[0, 0, n]
            best_g = max(itertools.combinations(cand, kg), key=lambda c: sg[list(c)].sum())
            assert list(gi[0, 0, n]) == sorted(best_g)


def test_gradients_match_finite_differences(oracle):
    """Central differences of L = sum(o * d_o) in float64 on a tiny layer."""
    B, Hq, Hkv, D, H, S, grp, qblk = 1, 2, 1, 4, 8, 4, 2, 2
    g = torch.Generator().manual_seed(11)
    t = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64).numpy()
    x = dict(q=t(B, Hq, S, D), k_hist=t(B, Hkv, H, D), v_hist=t(B, Hkv, H, D),
             k_seg=t(B, Hkv, S, D), v_seg=t(B, Hkv, S, D))
    do = t(B, Hq, S, D)
    gi = np.array([[[[0, 2], [1, 3]]]], dtype=np.int32)

    def loss(xx):
        o, _ = oracle.attn_fwd(xx["q"], xx["k_hist"], xx["v_hist"], xx["k_seg"], xx["v_seg"], gi,
                               group=grp, qblock=qblk)
        return float((o * do).sum())

    dq, dk, dv = oracle.attn_bwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], gi, do,
                                 group=grp, qblock=qblk)
    eps = 1e-6
    for name, grad in [("q", dq), ("k_seg", dk), ("v_seg", dv)]:
        fd = np.zeros_like(x[name])
        for idx in np.ndindex(x[name].shape):
            xp = {k: v.copy() for k, v in x.items()}; xp[name][idx] += eps
            xm = {k: v.copy() for k, v in x.items()}; xm[name][idx] -= eps
            fd[idx] = (loss(xp) - loss(xm)) / (2 * eps)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8)


def test_worked_example_golden(oracle):
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        ex = json.load(f)
    sh, inp, exp = ex["shape"], ex["inputs"], ex["expected"]
    a = {k: np.asarray(v, dtype=np.float64)[None, None] for k, v in inp.items()}
    scale = math.log(3) / 2
    gs = oracle.group_summaries(a["k_hist"], sh["group"])
    cs = oracle.chunk_summaries(a["k_hist"], sh["chunk"])
    qb = oracle.block_query(a["q"], sh["Hkv"], sh["qblock"])
    ci, gi, cgap, ggap = oracle.route(qb, gs, cs, sh["top_chunks"], sh["top_groups"])
    assert list(ci.ravel()) == exp["chunk_idx"] and list(gi.ravel()) == exp["group_idx"]
    assert cgap.ravel()[0] == exp["chunk_gap"] and ggap.ravel()[0] == exp["group_gap"]
    kw = dict(scale=scale, group=sh["group"], qblock=sh["qblock"])
    o, lse = oracle.attn_fwd(a["q"], a["k_hist"], a["v_hist"], a["k_seg"], a["v_seg"], gi, **kw)
    np.testing.assert_allclose(o[0, 0], exp["o"], atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], [math.log(4), math.log(5)], atol=1e-12)
    dq, dk, dv = oracle.attn_bwd(a["q"], a["k_hist"], a["v_hist"], a["k_seg"], a["v_seg"], gi,
                                 a["d_o"], **kw)
    np.testing.assert_allclose(dq[0, 0] / scale, exp["dq_over_scale"], atol=1e-12)
    np.testing.assert_allclose(dk[0, 0] / scale, exp["dk_seg_over_scale"], atol=1e-12)
    np.testing.assert_allclose(dv[0, 0], exp["dv_seg"], atol=1e-12)


def test_softmax_rows_sum_to_one(oracle):
    """Reconstruct every row's probabilities from LSE over its key set: they sum to 1."""
    H, S = 256, 128
    x = _small_layer(2, H=H, S=S)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], 2, 2, 4, prec=64)
    o, lse = oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
    mask = _mask_from_groups(r["group_idx"], 1, 4, 2, H, S)
    k = torch.cat([x["k_hist"], x["k_seg"]], dim=2).repeat_interleave(2, dim=1)
    logits = torch.einsum("bhsd,bhtd->bhst", x["q"], k) / 4.0
    p = torch.exp(logits - torch.as_tensor(lse)[..., None]) * mask
    np.testing.assert_allclose(p.sum(-1).numpy(), 1.0, atol=1e-12)
    assert mask.sum(-1).min() >= 4 * 8 + 1                 # routed tokens + itself


def test_no_future_information_across_blocks(oracle):
    """Changing segment K/V at u changes no output row t < u; changing a query of block n
    leaves the routing and outputs of blocks < n bit-identical."""
    w = HI.WORKLOADS["tiny_f32"]
    x = HI.make_inputs(w, 2)
    base = oracle.route_from_inputs(x["q"], x["k_hist"], 1, w.top_chunks, w.top_groups)
    o0, _ = oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], base["group_idx"])
    y = {k: v.clone() for k, v in x.items() if k != "needles"}
    y["k_seg"][0, 0, 130] += 3.0
    y["v_seg"][0, 0, 130] -= 3.0
    o1, _ = oracle.attn_fwd(y["q"], y["k_hist"], y["v_hist"], y["k_seg"], y["v_seg"], base["group_idx"])
    assert np.array_equal(o0[:, :, :130], o1[:, :, :130])
    assert not np.array_equal(o0[:, :, 130:], o1[:, :, 130:])
    z = {k: v.clone() for k, v in x.items() if k != "needles"}
    z["q"][0, :, 128:192] = torch.randn(4, 64, w.D, generator=torch.Generator().manual_seed(3)) * 5
    rz = oracle.route_from_inputs(z["q"], z["k_hist"], 1, w.top_chunks, w.top_groups)
    assert np.array_equal(rz["group_idx"][:, :, :2], base["group_idx"][:, :, :2])
    oz, _ = oracle.attn_fwd(z["q"], z["k_hist"], z["v_hist"], z["k_seg"], z["v_seg"], rz["group_idx"])
    assert np.array_equal(oz[:, :, :128], o0[:, :, :128])


def test_within_block_side_channel_is_present(oracle):
    """Documented behaviour (Technical Summary section 5, 'Causal Leakage'): the routing of a block
    depends on all of its queries, so a later query can change an earlier query's output."""
    w = HI.WORKLOADS["tiny_f32"]
    x = HI.make_inputs(w, 0)
    base = oracle.route_from_inputs(x["q"], x["k_hist"], 1, w.top_chunks, w.top_groups)
    z = {k: v.clone() for k, v in x.items() if k != "needles"}
    # push the block-0 mean towards the summary of a chunk that block 0 did not select
    cs = oracle.chunk_summaries(x["k_hist"])[0, 0]
    other = next(i for i in range(w.nch) if i not in base["chunk_idx"][0, 0, 0])
    z["q"][0, 0, 63] += torch.as_tensor(cs[other] * 400.0, dtype=z["q"].dtype)
    rz = oracle.route_from_inputs(z["q"], z["k_hist"], 1, w.top_chunks, w.top_groups)
    assert other in rz["chunk_idx"][0, 0, 0]
    o0, _ = oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], base["group_idx"])
    oz, _ = oracle.attn_fwd(z["q"], z["k_hist"], z["v_hist"], z["k_seg"], z["v_seg"], rz["group_idx"])
    assert not np.allclose(oz[0, 1, :63], o0[0, 1, :63])   # earlier queries of another head moved


def test_causal_routing_closes_the_within_block_side_channel(oracle):
    """Strictly causal variant (block n routed with block n-1's query): the perturbation that moves
    earlier outputs under the standard routing leaves every earlier output of the block unchanged;
    it reaches only the next block's routing, whose queries all come after it."""
    w = HI.WORKLOADS["tiny_f32"]
    x = HI.make_inputs(w, 0)
    qp = HI.make_inputs(w.with_(hist_len=64, seg_len=64), 1)["q"]          # previous segment's last block
    base = oracle.route_causal_from_inputs(x["q"], x["k_hist"], 1, w.top_chunks, w.top_groups, q_prev=qp)
    z = {k: v.clone() for k, v in x.items() if k != "needles"}
    cs = oracle.chunk_summaries(x["k_hist"])[0, 0]
    std = oracle.route_from_inputs(x["q"], x["k_hist"], 1, w.top_chunks, w.top_groups)
    other = next(i for i in range(w.nch) if i not in std["chunk_idx"][0, 0, 0])
    z["q"][0, 0, 63] += torch.as_tensor(cs[other] * 400.0, dtype=z["q"].dtype)
    rz = oracle.route_causal_from_inputs(z["q"], z["k_hist"], 1, w.top_chunks, w.top_groups, q_prev=qp)
    assert np.array_equal(rz["group_idx"][:, :, 0], base["group_idx"][:, :, 0])
    assert other in rz["chunk_idx"][0, 0, 1]                  # the next block's routing moved
    o0, _ = oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], base["group_idx"])
    oz, _ = oracle.attn_fwd(z["q"], z["k_hist"], z["v_hist"], z["k_seg"], z["v_seg"], rz["group_idx"])
    assert np.array_equal(oz[:, :, :63], o0[:, :, :63])       # nothing before the change moved


def test_causal_routing_is_strictly_causal_at_every_position(oracle):
    """Changing every query at or after position t (all heads) leaves all outputs before t equal."""
    w = HI.WORKLOADS["tiny_f32"]
    x = HI.make_inputs(w, 2)
    r0 = oracle.route_causal_from_inputs(x["q"], x["k_hist"], 1, w.top_chunks, w.top_groups)
    o0, _ = oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r0["group_idx"])
    g = torch.Generator().manual_seed(3)
    for t in (1, 63, 64, 100, 200):
        q = x["q"].clone()
        q[:, :, t:] = torch.randn(q[:, :, t:].shape, generator=g) * 3
        r = oracle.route_causal_from_inputs(q, x["k_hist"], 1, w.top_chunks, w.top_groups)
        o, _ = oracle.attn_fwd(q, x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
        assert np.array_equal(o[:, :, :t], o0[:, :, :t])


def test_causal_routing_is_the_previous_blocks_routing(oracle):
    """Block n >= 1 gets the standard routing of block n-1; block 0 that of q_prev, or with no
    q_prev a zero query, whose all-equal scores take the lowest routable indices."""
    w = HI.WORKLOADS["tiny_f32"].with_(n_sink=128)
    x = HI.make_inputs(w, 4)
    qp = HI.make_inputs(w.with_(hist_len=64, seg_len=64), 5)["q"]
    std = oracle.route_from_inputs(x["q"], x["k_hist"], 1, w.top_chunks, w.top_groups, n_sink=128)
    c = oracle.route_causal_from_inputs(x["q"], x["k_hist"], 1, w.top_chunks, w.top_groups, q_prev=qp,
                                        n_sink=128)
    assert np.array_equal(c["group_idx"][:, :, 1:], std["group_idx"][:, :, :-1])
    assert np.array_equal(c["chunk_idx"][:, :, 1:], std["chunk_idx"][:, :, :-1])
    q0 = torch.cat([qp, x["q"][:, :, 64:]], dim=2)              # a segment whose block 0 is q_prev
    std0 = oracle.route_from_inputs(q0, x["k_hist"], 1, w.top_chunks, w.top_groups, n_sink=128)
    assert np.array_equal(c["group_idx"][:, :, 0], std0["group_idx"][:, :, 0])
    z = oracle.route_causal_from_inputs(x["q"], x["k_hist"], 1, w.top_chunks, w.top_groups, n_sink=128)
    assert list(z["chunk_idx"][0, 0, 0]) == [2, 3, 4, 5]
    assert list(z["group_idx"][0, 0, 0]) == list(range(16, 24))


def test_row_and_key_subsets_match_full(oracle):
    w = HI.WORKLOADS["tiny_f32"]
    x = HI.make_inputs(w, 4)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], 1, w.top_chunks, w.top_groups)
    args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
    o, lse = oracle.attn_fwd(*args)
    dq, dk, dv = oracle.attn_bwd(*args, x["d_o"])
    rows = HI.sample_ids(4 * 256, 37, 0).numpy()
    keys = HI.sample_ids(256, 29, 1).numpy()
    os_, ls_ = oracle.attn_fwd(*args, rows=rows)
    dqs, dks, dvs = oracle.attn_bwd(*args, x["d_o"], rows=rows, keys=keys)
    assert np.array_equal(os_, o.reshape(-1, w.D)[rows]) and np.array_equal(ls_, lse.reshape(-1)[rows])
    assert np.array_equal(dqs, dq.reshape(-1, w.D)[rows])
    assert np.array_equal(dks, dk.reshape(-1, w.D)[keys]) and np.array_equal(dvs, dv.reshape(-1, w.D)[keys])


def test_invalid_arguments_raise(oracle):
    k = np.zeros((1, 1, 128, 4))
    with pytest.raises(ValueError):
        oracle.group_summaries(np.zeros((1, 1, 100, 4)), 8)
    qb = np.zeros((1, 1, 1, 4)); gs = oracle.group_summaries(k); cs = oracle.chunk_summaries(k)
    with pytest.raises(ValueError):
        oracle.route(qb, gs, cs, 3, 4)          # k_c > number of chunks
    with pytest.raises(ValueError):
        oracle.route(qb, gs, cs, 1, 9)          # k_g > groups of the chosen chunks
    with pytest.raises(ValueError):
        oracle.route(qb, gs, cs, 2, 4, n_sink_chunks=1)   # k_c > chunks outside the sink
    with pytest.raises(ValueError):
        oracle.route(qb, gs, cs, 1, 4, n_sink_chunks=2)   # the sink covers every chunk
    x = _small_layer(0, H=128, S=64)
    gi = np.array([[[[3, 9]], [[8, 9]]]], dtype=np.int32)
    with pytest.raises(ValueError):                        # group 3 lies in a 64-token sink
        oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], gi, n_sink=64)
    with pytest.raises(ValueError):                        # group 16 is beyond the history
        oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], gi + 7)


# --------------------------------------------------------------------------- inputs used by GPU parity
PARITY_SEEDS = {"tiny_f32": [0, 1, 2, 3, 4], "small_bf16": [0, 1], "ctx4k": [0, 1], "ctx16k": [0, 2],
                "ctx16k_kc8": [0], "ctx16k_kc32": [0], "ctx131k": [0], "ctx16k_b4": [11]}
PARITY_SEEDS.update({name: [0] for name in HI.EDGE_WORKLOADS})
MIN_GAP = 4e-6


@pytest.mark.parametrize("name", ["tiny_f32", "small_bf16", "ctx4k", "ctx16k", "ctx16k_kc8", "ctx16k_kc32",
                                  "ctx16k_b4", *HI.EDGE_WORKLOADS])
def test_parity_seeds_have_routing_margins(oracle, name):
    """For the seeds the GPU parity tests use, the fp32 routing equals the fp64 routing and every
    selection boundary has a score gap >= MIN_GAP (far above fp32 rounding of these scores,
    whose magnitude is < 10), so summation order cannot flip a selection."""
    w = HI.WORKLOADS.get(name) or HI.EDGE_WORKLOADS[name]
    for seed in PARITY_SEEDS[name]:
        x = HI.make_inputs(w, seed)
        r32 = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32,
                                       n_sink=w.n_sink)
        r64 = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=64,
                                       n_sink=w.n_sink)
        assert np.array_equal(r32["chunk_idx"], r64["chunk_idx"])
        assert np.array_equal(r32["group_idx"], r64["group_idx"])
        assert r64["chunk_gap"].min() >= MIN_GAP and r64["group_gap"].min() >= MIN_GAP


@pytest.mark.parametrize("name,q_seeds", [("gcache_small", [0, 1, 2, 3, 4, 5]), ("ctx16k", [0, 2, 1])])
def test_cache_test_steps_have_routing_margins(oracle, name, q_seeds):
    """The group-summary cache tests route the queries of several seeds against the history of seed
    0; every such step has the same margins as the other parity inputs."""
    w = (HI.Workload("gcache_small", 2, 8, 2, 128, 4096, 256, 4, 16, "bf16", 1.0) if name == "gcache_small"
         else HI.WORKLOADS[name])
    kh = HI.make_inputs(w, 0)["k_hist"]
    for s in q_seeds:
        q = HI.make_inputs(w, s)["q"]
        r32 = oracle.route_from_inputs(q, kh, w.Hkv, w.top_chunks, w.top_groups, prec=32)
        r64 = oracle.route_from_inputs(q, kh, w.Hkv, w.top_chunks, w.top_groups, prec=64)
        assert np.array_equal(r32["chunk_idx"], r64["chunk_idx"])
        assert np.array_equal(r32["group_idx"], r64["group_idx"])
        assert r64["chunk_gap"].min() >= MIN_GAP and r64["group_gap"].min() >= MIN_GAP


@pytest.mark.parametrize("name", ["small_bf16", "sink_bf16", "ctx16k"])
def test_causal_parity_inputs_have_routing_margins(oracle, name):
    """Block 0 of the causal routing in the GPU tests is routed with a separately drawn previous
    block; its selection boundaries have the same margins as the other parity inputs."""
    w = HI.WORKLOADS.get(name) or HI.EDGE_WORKLOADS[name]
    x = HI.make_inputs(w, 0)
    qp = HI.prev_block_q(w, 0)
    kw = dict(q_prev=qp, n_sink=w.n_sink)
    r32 = oracle.route_causal_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32, **kw)
    r64 = oracle.route_causal_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=64, **kw)
    assert np.array_equal(r32["chunk_idx"], r64["chunk_idx"])
    assert np.array_equal(r32["group_idx"], r64["group_idx"])
    assert r64["chunk_gap"].min() >= MIN_GAP and r64["group_gap"].min() >= MIN_GAP


def test_needles_recovered_at_131k(oracle):
    """131072-token workload: every planted needle group is routed to its target block."""
    w = HI.WORKLOADS["ctx131k"]
    x = HI.make_inputs(w, PARITY_SEEDS["ctx131k"][0])
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32)
    hits = [j in r["group_idx"][0, kh, n] for kh, n, j in x["needles"].tolist()]
    assert len(hits) == 64 and all(hits)
    r64 = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=64)
    assert np.array_equal(r["group_idx"], r64["group_idx"])
    assert r64["chunk_gap"].min() >= MIN_GAP and r64["group_gap"].min() >= MIN_GAP
