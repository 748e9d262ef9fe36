"""Strictly causal routing (block n routed with block n-1's query) on a B200: routing indices
bit-exact against the oracle, the full path within the usual tolerances, and the leakage probe
of the pages ("mask a later token and check whether earlier-token predictions change"): under the
standard routing a later query of a block moves earlier outputs, under the causal one it cannot."""
import numpy as np
import pytest
import torch

import hga_inputs as HI

pytestmark = pytest.mark.gpu
CAUSAL_CASES = [("small_bf16", True), ("tiny_f32", False), ("sink_bf16", True), ("ctx16k", True)]


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_kv_routing_tok_b200 as H
    H.load()
    return H


def _wl(name):
    return HI.WORKLOADS.get(name) or HI.EDGE_WORKLOADS[name]


def _run(hga, w, xd, causal, q_prev=None):
    cfg = hga.make_config(xd["q"], xd["k_hist"], w.top_chunks, w.top_groups, n_sink_tokens=w.n_sink)
    step = hga.LayerStep(cfg, causal_routing=causal)
    x = dict(xd)
    if q_prev is not None:
        x["q_prev"] = q_prev
    step(x)
    torch.cuda.synchronize()
    assert hga.read_status(step.ws) == 0
    return step


@pytest.mark.parametrize("name,with_prev", CAUSAL_CASES)
def test_causal_routing_matches_oracle(hga, oracle, name, with_prev):
    w = _wl(name)
    x = HI.make_inputs(w, 0)
    qp = HI.prev_block_q(w, 0) if with_prev else None
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    step = _run(hga, w, xd, True, qp.cuda() if qp is not None else None)
    r = oracle.route_causal_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, q_prev=qp,
                                        prec=32, n_sink=w.n_sink)
    assert np.array_equal(step.chunk_idx.cpu().numpy(), r["chunk_idx"])
    assert np.array_equal(step.group_idx.cpu().numpy(), r["group_idx"])
    if w.seg_len * w.Hq * w.B <= 2 * 8 * 512:        # small layers: whole outputs against the oracle
        args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
        o, lse = oracle.attn_fwd(*args, n_sink=w.n_sink)
        dq, dk, dv = oracle.attn_bwd(*args, x["d_o"], n_sink=w.n_sink)
        tol = 1e-4 if w.dtype == "f32" else 2e-2
        for a, b in [(step.o, o), (step.dq, dq), (step.dk, dk), (step.dv, dv)]:
            assert float(np.abs(a.float().cpu().numpy() - b).max()) <= tol


def test_leakage_probe(hga, oracle):
    """Push the last query of block 0 towards a chunk block 0 did not select: with the standard
    routing the earlier outputs of the block move; with the causal routing they stay bit for bit."""
    w = HI.WORKLOADS["small_bf16"]
    x = HI.make_inputs(w, 0)
    std = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups)
    cs = oracle.chunk_summaries(x["k_hist"])[0, 0]
    other = next(i for i in range(w.nch) if i not in std["chunk_idx"][0, 0, 0])
    z = {k: v.clone() for k, v in x.items() if k != "needles"}
    z["q"][0, 0, 63] += torch.as_tensor(cs[other] * 400.0, dtype=z["q"].dtype)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    zd = {k: v.cuda() for k, v in z.items()}
    s0, s1 = _run(hga, w, xd, False), _run(hga, w, zd, False)
    assert not torch.equal(s0.o[0, :, :63], s1.o[0, :, :63])          # the side channel
    c0, c1 = _run(hga, w, xd, True), _run(hga, w, zd, True)
    assert torch.equal(c0.group_idx[:, :, 0], c1.group_idx[:, :, 0])
    assert torch.equal(c0.o[:, :, :63], c1.o[:, :, :63])               # closed
    assert torch.equal(c0.lse[:, :, :63], c1.lse[:, :, :63])
