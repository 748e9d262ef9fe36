"""Failure detection on the device without a GPU fault: every on-chip pipeline wait of the
tensor-core kernels is bounded.  A call whose wait limit (``wait_limit_ns``) is shorter than a tile
load's latency must give up along the kernels' own abort path -- set HGA_ERR_TIMEOUT in the status
word, let its own copies and MMAs land, free its tensor memory and return -- and leave the
context usable: the next call with the default limit gives the exact results again.  Nothing is
broken on purpose and nothing waits without a bound (the drains keep their own 2 s limit)."""
import time

import numpy as np
import pytest
import torch

import hga_inputs as HI

pytestmark = pytest.mark.gpu

KERNELS = ["attn_fwd", "bwd_dq", "bwd_dkdv"]


@pytest.fixture(scope="module")
def hga():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import hierarchical_kv_routing_tok_b200 as H
    H.load()
    return H


def _outputs(step):
    return [t.clone() for t in (step.group_idx, step.o, step.lse, step.dq, step.dk, step.dv)]


def _short_limit(C, cfg, ns=1):
    return C.make_config(cfg.B, cfg.Hq, cfg.Hkv, cfg.hist_len, cfg.seg_len, cfg.top_chunks, cfg.top_groups,
                         dtype=cfg.dtype, D=cfg.D, softmax_scale=cfg.softmax_scale,
                         n_sink_tokens=cfg.n_sink_tokens, hist_capacity=cfg.hist_capacity, wait_limit_ns=ns)


# small_bf16: 16 (batch, KV head, key tile) units, so the dK/dV kernel runs in CTA pairs (clusters);
# the same layer at batch 19 has 152 units, at least one per SM, and runs it unpaired
@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("batch", [2, 19])
def test_expired_wait_reports_timeout_and_next_call_is_exact(hga, oracle, kernel, batch):
    C = hga._capi
    w = HI.WORKLOADS["small_bf16"].with_(B=batch)
    x = HI.make_inputs(w, 0)
    xd = {k: v.cuda() for k, v in x.items() if k != "needles"}
    cfg = hga.make_config(xd["q"], xd["k_hist"], w.top_chunks, w.top_groups)
    step = hga.LayerStep(cfg)
    step(xd)                                               # the whole step with the default limit
    torch.cuda.synchronize()
    assert hga.read_status(step.ws) == C.HGA_OK
    ref = _outputs(step)

    # one kernel of the step with a 1 ns limit: its first wait that is not already satisfied expires
    call = dict(step.calls(xd, cfg=_short_limit(C, cfg)))[kernel]
    t0 = time.monotonic()
    call()
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    assert hga.read_status(step.ws) == C.HGA_ERR_TIMEOUT
    assert elapsed < 30.0                                  # it returned (drains are bounded at 2 s)

    # the context is intact: the step again with the default limit reproduces its earlier outputs
    step(xd)
    torch.cuda.synchronize()
    assert hga.read_status(step.ws) == C.HGA_OK
    for a, b in zip(_outputs(step), ref):
        assert torch.equal(a, b)
    if batch == 2:                                         # and they match the oracle
        r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32)
        assert np.array_equal(step.group_idx.cpu().numpy(), r["group_idx"])
        args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
        o, lse = oracle.attn_fwd(*args)
        dq, dk, dv = oracle.attn_bwd(*args, x["d_o"])
        for got, want in ((step.o, o), (step.dq, dq), (step.dk, dk), (step.dv, dv)):
            assert float(np.abs(got.float().cpu().numpy() - want).max()) <= 2e-2
        assert float(np.abs(step.lse.cpu().numpy() - lse).max()) <= 1e-3

