"""Parity of the CUDA path (through the C ABI) with the CPU oracle on a B200.

Bars: routing indices bit-exact (both sides decide in float32 on inputs whose selection
margins the CPU tests verify); float32 path max |err| <= 1e-4; bfloat16 path (float32
accumulation) max |err| <= 2e-2 on O, dQ, dK, dV; summaries relative error <= 1e-5.
Small workloads are compared element by element over the whole output; the benchmark
workload (16K context) and the 131K forward are compared on every routing index and on
sampled output rows / keys, in the launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import hga_inputs as HI
from oracle_slices import attn_sampled

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
LSE_TOL = {"f32": 1e-4, "bf16": 1e-3}


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_kv_routing_tok_b200 as H
    H.load()
    return H


def _wl(name):
    return HI.WORKLOADS.get(name) or HI.EDGE_WORKLOADS[name]


def run_gpu(hga, w, x, backward=True, group_idx=None):
    """Whole hot path on cuda:0 through the C ABI; returns CPU copies of every output."""
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    cfg = hga.make_config(xd["q"], xd["k_hist"], w.top_chunks, w.top_groups, n_sink_tokens=w.n_sink)
    step = hga.LayerStep(cfg)
    step.forward(xd)
    if group_idx is not None:          # attention on a given routing (routing-independent check)
        step.group_idx.copy_(torch.as_tensor(group_idx))
        hga.attn_fwd(cfg, xd["q"], xd["k_hist"], xd["v_hist"], xd["k_seg"], xd["v_seg"], step.group_idx,
                     step.o, step.lse, step.ws)
    if backward:
        step.backward(xd)
    torch.cuda.synchronize()
    assert hga.read_status(step.ws) == 0
    out = dict(gs=step.group_sum, cs=step.chunk_sum, ci=step.chunk_idx, gi=step.group_idx, o=step.o,
               lse=step.lse, dq=step.dq, dk=step.dk, dv=step.dv)
    return {k: v.float().cpu() if v.dtype != torch.int32 else v.cpu() for k, v in out.items()}


def maxerr(a, b):
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))))


# ----------------------------------------------------------------------------- small: full compare
FULL = ["tiny_f32", "small_bf16", *HI.EDGE_WORKLOADS]


@pytest.mark.parametrize("name", FULL)
def test_full_path_matches_oracle(hga, oracle, name):
    w = _wl(name)
    x = HI.make_inputs(w, 0)
    g = run_gpu(hga, w, x)
    # summaries
    gs = oracle.group_summaries(x["k_hist"])
    cs = oracle.chunk_summaries(x["k_hist"])
    np.testing.assert_allclose(g["gs"].numpy(), gs, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(g["cs"].numpy(), cs, rtol=1e-5, atol=1e-6)
    # routing: bit-exact against the oracle deciding in float32
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32,
                                 n_sink=w.n_sink)
    assert np.array_equal(g["ci"].numpy(), r["chunk_idx"])
    assert np.array_equal(g["gi"].numpy(), r["group_idx"])
    # forward / backward
    args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
    o, lse = oracle.attn_fwd(*args, n_sink=w.n_sink)
    dq, dk, dv = oracle.attn_bwd(*args, x["d_o"], n_sink=w.n_sink)
    tol = TOL[w.dtype]
    errs = dict(o=maxerr(g["o"], o), dq=maxerr(g["dq"], dq), dk=maxerr(g["dk"], dk), dv=maxerr(g["dv"], dv))
    assert max(errs.values()) <= tol, errs
    assert maxerr(g["lse"], lse) <= LSE_TOL[w.dtype]


@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_tiny_f32_more_seeds(hga, oracle, seed):
    w = HI.WORKLOADS["tiny_f32"]
    x = HI.make_inputs(w, seed)
    g = run_gpu(hga, w, x)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32)
    assert np.array_equal(g["gi"].numpy(), r["group_idx"])
    args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
    o, _ = oracle.attn_fwd(*args)
    dq, dk, dv = oracle.attn_bwd(*args, x["d_o"])
    assert max(maxerr(g["o"], o), maxerr(g["dq"], dq), maxerr(g["dk"], dk), maxerr(g["dv"], dv)) <= 1e-4


def test_attention_on_arbitrary_routing(hga, oracle):
    """Attention kernels on a routing the router did not produce (unsorted-free random sets)."""
    w = HI.WORKLOADS["small_bf16"]
    x = HI.make_inputs(w, 1)
    gen = torch.Generator().manual_seed(3)
    gi = torch.stack([torch.randperm(w.ngr, generator=gen)[:w.top_groups].sort().values
                      for _ in range(w.B * w.Hkv * w.nblk)]).reshape(w.B, w.Hkv, w.nblk, w.top_groups)
    gi = gi.to(torch.int32)
    g = run_gpu(hga, w, x, group_idx=gi)
    args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], gi.numpy())
    o, lse = oracle.attn_fwd(*args)
    dq, dk, dv = oracle.attn_bwd(*args, x["d_o"])
    assert max(maxerr(g["o"], o), maxerr(g["dq"], dq), maxerr(g["dk"], dk), maxerr(g["dv"], dv)) <= 2e-2


def test_bwd_outputs_only_16_byte_aligned(hga, oracle):
    """The interface promises 16-byte alignment only: dQ, dK, dV placed 16 bytes past a 32-byte
    boundary give the same bits as the aligned buffers (the dQ kernel stores 32-byte vectors only
    into a 32-byte aligned dQ) and match the oracle."""
    w = HI.WORKLOADS["small_bf16"]
    x = HI.make_inputs(w, 2)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    cfg = hga.make_config(xd["q"], xd["k_hist"], w.top_chunks, w.top_groups)
    step = hga.LayerStep(cfg)
    step(xd)

    def off16(like):
        buf = torch.empty(like.numel() + 8, dtype=like.dtype, device=like.device)
        t = buf[8:].view(like.shape)
        assert t.data_ptr() % 32 == 16
        return t

    dq, dk, dv = off16(step.dq), off16(step.dk), off16(step.dv)
    hga.attn_bwd(cfg, xd["q"], xd["k_hist"], xd["v_hist"], xd["k_seg"], xd["v_seg"], step.group_idx, step.o,
                 step.lse, xd["d_o"], dq, dk, dv, step.ws)
    torch.cuda.synchronize()
    assert hga.read_status(step.ws) == 0
    for got, ref in ((dq, step.dq), (dk, step.dk), (dv, step.dv)):
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], step.group_idx.cpu().numpy())
    rdq, rdk, rdv = oracle.attn_bwd(*args, x["d_o"])
    assert max(maxerr(dq.float().cpu(), rdq), maxerr(dk.float().cpu(), rdk), maxerr(dv.float().cpu(), rdv)) <= 2e-2


# ----------------------------------------------------------------------------- ties
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_routing_ties_go_to_lower_index(hga, dtype):
    """All history keys equal (scores tie exactly on both levels; with zero keys every score is
    +-0): the lowest chunk and group indices are selected."""
    w = HI.WORKLOADS["tiny_f32"].with_(dtype=dtype)
    x = HI.make_inputs(w, 0)
    for fill in (0.25, 0.0):
        x["k_hist"] = torch.full_like(x["k_hist"], fill)
        g = run_gpu(hga, w, x, backward=False)
        assert (g["ci"] == torch.arange(w.top_chunks, dtype=torch.int32)).all()
        assert (g["gi"] == torch.arange(w.top_groups, dtype=torch.int32)).all()


def test_routing_tie_between_duplicate_chunks(hga, oracle):
    """Chunks 9 and 3 hold identical keys aligned with every block query: with k_c = 1 the lower
    index (3) wins, and the groups come from chunk 3."""
    w = HI.WORKLOADS["tiny_f32"].with_(top_chunks=1, top_groups=8)
    x = HI.make_inputs(w, 0)
    u = x["q"].mean(dim=(1, 2))[0]
    blockk = x["k_hist"][0, 0, 9 * 64:10 * 64].clone() * 0.01 + 50 * u
    x["k_hist"][0, 0, 9 * 64:10 * 64] = blockk
    x["k_hist"][0, 0, 3 * 64:4 * 64] = blockk
    g = run_gpu(hga, w, x, backward=False)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32)
    assert (g["ci"] == 3).all() and np.array_equal(g["ci"].numpy(), r["chunk_idx"])
    assert np.array_equal(g["gi"].numpy(), r["group_idx"])


# ----------------------------------------------------------------------------- full-size, sampled
def _sampled_rows(w, n, seed):
    """Random rows plus the first/last row of sampled blocks (block and tile boundaries)."""
    ids = HI.sample_ids(w.B * w.Hq * w.seg_len, n, seed).tolist()
    for blk in (0, 1, w.nblk // 2, w.nblk - 1):
        for h in (0, w.Hq - 1):
            base = h * w.seg_len + blk * 64
            ids += [base, base + 63]
    return np.array(sorted(set(ids)), dtype=np.int64)


def _sampled_keys(w):
    """Segment keys of every (batch, KV head): both ends of every 128-key tile of the dK/dV kernel
    (so every CTA, and both CTAs of every cluster pair, is looked at) plus two keys inside tiles."""
    us = sorted({u for t in range(0, w.seg_len, 128) for u in (t, min(t + 127, w.seg_len - 1))}
                | {min(64, w.seg_len - 1), w.seg_len // 2 + 37})
    return np.array([(b * w.Hkv + kh) * w.seg_len + u for b in range(w.B) for kh in range(w.Hkv) for u in us],
                    dtype=np.int64)


@pytest.mark.parametrize("name,seed", [("ctx4k", 0), ("ctx4k", 1), ("ctx16k", 0), ("ctx16k", 2),
                                       ("ctx16k_kc8", 0), ("ctx16k_kc32", 0)])
def test_full_size_layer_sampled(hga, oracle, name, seed):
    w = HI.WORKLOADS[name]
    x = HI.make_inputs(w, seed)
    g = run_gpu(hga, w, x)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32)
    assert np.array_equal(g["ci"].numpy(), r["chunk_idx"])
    assert np.array_equal(g["gi"].numpy(), r["group_idx"])
    rows = _sampled_rows(w, 96, seed)
    keys = _sampled_keys(w)
    ref = attn_sampled(oracle, x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"], x["d_o"],
                       rows=rows, keys=keys)
    o, lse, dq, dk, dv = (ref[k] for k in ("o", "lse", "dq", "dk", "dv"))
    D = w.D
    e = dict(o=maxerr(g["o"].reshape(-1, D)[rows], o), lse=maxerr(g["lse"].reshape(-1)[rows], lse),
             dq=maxerr(g["dq"].reshape(-1, D)[rows], dq), dk=maxerr(g["dk"].reshape(-1, D)[keys], dk),
             dv=maxerr(g["dv"].reshape(-1, D)[keys], dv))
    assert e["lse"] <= 1e-3 and max(e["o"], e["dq"], e["dk"], e["dv"]) <= 2e-2, e


def test_131k_forward_routing_and_needles(hga, oracle):
    w = HI.WORKLOADS["ctx131k"]
    x = HI.make_inputs(w, 0)
    g = run_gpu(hga, w, x, backward=False)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32)
    assert np.array_equal(g["ci"].numpy(), r["chunk_idx"])
    assert np.array_equal(g["gi"].numpy(), r["group_idx"])
    hits = [j in g["gi"][0, kh, n].tolist() for kh, n, j in x["needles"].tolist()]
    assert len(hits) == 64 and all(hits)
    rows = _sampled_rows(w, 64, 5)
    o, lse = oracle.attn_fwd(x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"], rows=rows)
    assert maxerr(g["o"].reshape(-1, w.D)[rows], o) <= 2e-2
    assert maxerr(g["lse"].reshape(-1)[rows], lse) <= 1e-3


# ----------------------------------------------------------------------------- API-level
def test_repeat_runs_are_bitwise_identical(hga):
    w = HI.WORKLOADS["small_bf16"]
    x = HI.make_inputs(w, 0)
    a = run_gpu(hga, w, x)
    b = run_gpu(hga, w, x)
    for k in a:
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("name", ["small_bf16", "tiny_f32"])
def test_captured_step_replays_bitwise(hga, name):
    """LayerStep.capture: a CUDA-graph replay of the whole step gives bitwise the outputs of the
    step launched call by call, on new inputs copied into the captured buffers too."""
    w = _wl(name)
    x = {k: v.cuda() for k, v in HI.make_inputs(w, 0).items() if k != "needles"}
    cfg = hga.make_config(x["q"], x["k_hist"], w.top_chunks, w.top_groups)
    step = hga.LayerStep(cfg)
    outs = lambda: [t.clone() for t in (step.group_idx, step.o, step.lse, step.dq, step.dk, step.dv)]
    g = step.capture(x)
    for seed in (1, 2):
        x2 = {k: v.cuda() for k, v in HI.make_inputs(w, seed).items() if k != "needles"}
        for k in x:
            x[k].copy_(x2[k])
        g.replay()
        torch.cuda.synchronize()
        got = outs()
        step(x)
        torch.cuda.synchronize()
        assert hga.read_status(step.ws) == 0
        for a, b in zip(got, outs()):
            assert torch.equal(a, b)


def test_autograd_function_matches_oracle(hga, oracle):
    w = HI.WORKLOADS["small_bf16"]
    x = HI.make_inputs(w, 1)
    q = x["q"].cuda().requires_grad_(True)
    ks = x["k_seg"].cuda().requires_grad_(True)
    vs = x["v_seg"].cuda().requires_grad_(True)
    o, lse, gi = hga.hga_attention(q, ks, vs, x["k_hist"].cuda(), x["v_hist"].cuda(), w.top_chunks, w.top_groups)
    o.backward(x["d_o"].cuda())
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32)
    assert np.array_equal(gi.cpu().numpy(), r["group_idx"])
    args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
    oo, _ = oracle.attn_fwd(*args)
    dq, dk, dv = oracle.attn_bwd(*args, x["d_o"])
    assert maxerr(o.detach().float().cpu(), oo) <= 2e-2
    assert maxerr(q.grad.float().cpu(), dq) <= 2e-2
    assert maxerr(ks.grad.float().cpu(), dk) <= 2e-2
    assert maxerr(vs.grad.float().cpu(), dv) <= 2e-2


def test_api_rejects_wrong_dtype_and_shape(hga):
    w = HI.WORKLOADS["small_bf16"]
    x = {k: v.cuda() for k, v in HI.make_inputs(w, 0).items() if k != "needles"}
    cfg = hga.make_config(x["q"], x["k_hist"], w.top_chunks, w.top_groups)
    with pytest.raises(ValueError):
        hga.build_summaries(cfg, x["k_hist"].float())
    with pytest.raises(ValueError):
        hga.build_summaries(cfg, x["k_hist"][:, :, :512].contiguous())


def test_out_of_range_group_index_is_reported_not_read(hga):
    """A caller-supplied group index >= H/8 is caught by the kernels' own bounds check: the status
    word reports HGA_ERR_ARG and the outputs stay finite."""
    w = HI.WORKLOADS["tiny_f32"]
    x = {k: v.cuda() for k, v in HI.make_inputs(w, 0).items() if k != "needles"}
    cfg = hga.make_config(x["q"], x["k_hist"], w.top_chunks, w.top_groups)
    ws = hga.new_workspace(cfg, x["q"].device)
    gi = torch.zeros(w.B, w.Hkv, w.nblk, w.top_groups, dtype=torch.int32, device="cuda")
    gi[0, 0, 1, 3] = w.ngr + 5
    o, lse = hga.attn_fwd(cfg, x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], gi, workspace=ws)
    torch.cuda.synchronize()
    assert hga.read_status(ws) == -1
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert hga.read_status(ws) == 0          # read clears it
