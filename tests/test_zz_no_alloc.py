"""hga_attn_bwd_noalloc: the backward for callers that cannot allocate device memory (a host that
owns the whole device through its own pool, or code that must not risk the device
synchronisation cudaMalloc/cudaFree can cause).  It must give the same gradients as
hga_attn_bwd with a caller workspace, on consecutive calls that reuse its fixed scratch, and
refuse problems larger than that scratch.  Collected last on purpose."""
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


# small_bf16: its caller workspace pairs dK/dV CTAs; ctx4k (the 4K layer, B*Hq*S = 65536 rows):
# its 16 MiB exchange area would not fit the fixed array either -- this entry never pairs CTAs, so
# both compare the unpaired tensor-core dK/dV path with the paired one of the workspace backward
@pytest.mark.parametrize("name,tol", [("small_bf16", 2e-2), ("tiny_f32", 1e-4), ("ctx4k", 2e-2)])
def test_noalloc_backward_matches_workspace_backward(hga, name, tol):
    C = hga._capi
    w = HI.WORKLOADS[name]
    x = {k: v.cuda() for k, v in HI.make_inputs(w, 0).items() if k != "needles"}
    cfg = hga.make_config(x["q"], x["k_hist"], w.top_chunks, w.top_groups)
    step = hga.LayerStep(cfg)
    step(x)                                           # forward + backward with a workspace
    torch.cuda.synchronize()
    ref = (step.dq.clone(), step.dk.clone(), step.dv.clone())
    st = torch.cuda.current_stream().cuda_stream
    for _ in range(2):                                # second call finds the first call's scratch
        dq, dk, dv = (torch.full_like(t, float("nan")) for t in ref)
        C.attn_bwd_noalloc(cfg, x["q"].data_ptr(), x["k_hist"].data_ptr(), x["v_hist"].data_ptr(),
                           x["k_seg"].data_ptr(), x["v_seg"].data_ptr(), step.group_idx.data_ptr(),
                           step.o.data_ptr(), step.lse.data_ptr(), x["d_o"].data_ptr(), dq.data_ptr(),
                           dk.data_ptr(), dv.data_ptr(), st)
        assert C.noalloc_read_status(st) == 0          # no device-side error (read and cleared)
        for got, want in zip((dq, dk, dv), ref):
            assert torch.isfinite(got).all()
            assert (got.float() - want.float()).abs().max().item() <= tol


def test_noalloc_rejects_problem_beyond_scratch(hga):
    C = hga._capi
    rows = C.HGA_NOALLOC_MAX_ROWS
    cfg = C.make_config(B=rows // (32 * 2048) + 1, Hq=32, Hkv=8, hist_len=2048, seg_len=2048, top_chunks=4,
                        top_groups=16)
    with pytest.raises(C.HGAError) as e:
        C.attn_bwd_noalloc(cfg, *([1 << 20] * 12), 0)
    assert e.value.code == C.HGA_ERR_TOO_LARGE
