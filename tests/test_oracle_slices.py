"""The sliced, threaded oracle helper that the large GPU parity tests use gives bit for bit the
oracle's own values on the whole layer (it only indexes: every (batch, KV head) slice is computed
independently by the method)."""
import numpy as np
import pytest

import hga_inputs as HI
from oracle_slices import attn_sampled


@pytest.mark.parametrize("name", ["small_bf16", "sink_bf16", "gqa6_bf16"])
def test_sliced_oracle_equals_whole_layer_oracle(oracle, name):
    w = HI.WORKLOADS.get(name) or HI.EDGE_WORKLOADS[name]
    x = HI.make_inputs(w, 0)
    r = oracle.route_from_inputs(x["q"], x["k_hist"], w.Hkv, w.top_chunks, w.top_groups, prec=32, n_sink=w.n_sink)
    args = (x["q"], x["k_hist"], x["v_hist"], x["k_seg"], x["v_seg"], r["group_idx"])
    rows = HI.sample_ids(w.B * w.Hq * w.seg_len, 40, 1).numpy()[::-1].copy()       # any order
    keys = HI.sample_ids(w.B * w.Hkv * w.seg_len, 24, 2).numpy()
    got = attn_sampled(oracle, *args, x["d_o"], rows=rows, keys=keys, n_sink=w.n_sink)
    o, lse = oracle.attn_fwd(*args, rows=rows, n_sink=w.n_sink)
    dq, dk, dv = oracle.attn_bwd(*args, x["d_o"], rows=rows, keys=keys, n_sink=w.n_sink)
    for k, want in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert np.array_equal(got[k], want), k
    # forward only
    fwd = attn_sampled(oracle, *args, rows=rows, n_sink=w.n_sink)
    assert np.array_equal(fwd["o"], o) and "dq" not in fwd
