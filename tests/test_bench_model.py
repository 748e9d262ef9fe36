"""The benchmark's algorithmic work per kernel (the numerator of every roofline fraction), pinned
to values computed by hand from the 16K workload's shapes: Hq = 32 query heads, S = 2048 segment
queries, D = 128, k_g = 64 routed groups of 8 keys, history H = 14336, Hkv = 8 KV heads."""
import bench
import hga_inputs as HI


def test_work_model_16k():
    wm = bench.work_model(HI.WORKLOADS["ctx16k"])
    Hq, Hkv, S, D, H = 32, 8, 2048, 128, 14336
    routed = Hq * S * 8 * 64                     # (query, routed key) pairs: 33.5 M
    local = Hq * S * (S + 1) // 2                # causal (query, segment key) pairs: 67.1 M
    assert routed == 33_554_432 and local == 67_141_632
    # forward: S = Q K^T and O = P V, 2 flops per multiply-add each
    assert wm["attn_fwd"] == ("tensor", 4 * D * (routed + local))
    assert abs(wm["attn_fwd"][1] / 1e9 - 51.56) < 0.01
    # backward at the method's work (the FlashAttention-form backward over the same key sets, no
    # history gradient): S, dP and dQ over routed and local pairs, charged to the dQ kernel ...
    assert wm["bwd_dq"] == ("tensor", 6 * D * (routed + local))
    assert abs(wm["bwd_dq"][1] / 1e9 - 77.34) < 0.01
    # ... and dV = P^T dO, dK = dS^T Q over the local pairs, charged to the dK/dV kernel; S and dP of
    # a local pair are not booked twice
    assert wm["bwd_dkdv"] == ("tensor", 4 * D * local)
    assert abs(wm["bwd_dkdv"][1] / 1e9 - 34.37) < 0.01
    # the backward as a whole: 25.8 GFLOP routed (1.5 x the forward's 17.2) + 85.9 local (2.5 x 34.4)
    bwd = wm["bwd_dq"][1] + wm["bwd_dkdv"][1]
    assert bwd == 6 * D * routed + 10 * D * local
    assert abs(bwd / 1e9 - 111.7) < 0.05
    assert abs(bench.method_flops(HI.WORKLOADS["ctx16k"]) / 1e9 - 163.3) < 0.05
    # what the dK/dV kernel executes: it recomputes S^T and dP^T
    assert bench.executed_flops(HI.WORKLOADS["ctx16k"])["bwd_dkdv"] == 8 * D * local
    # summaries: read the bf16 history keys once, write float32 group and chunk means
    assert wm["summaries"] == ("hbm", Hkv * H * D * 2 + Hkv * (H // 8 + H // 64) * D * 4)
    # routing: read the bf16 queries and both float32 summary tables, write both index lists
    assert wm["route"] == ("hbm", Hq * S * D * 2 + Hkv * (H // 64 + H // 8) * D * 4 + Hkv * (S // 64) * (16 + 64) * 4)


def test_work_model_scales_with_batch_and_budget():
    base = bench.work_model(HI.WORKLOADS["ctx16k"])
    b4 = bench.work_model(HI.WORKLOADS["ctx16k_b4"])
    for k in base:
        assert b4[k][1] == 4 * base[k][1]
    kc32 = bench.work_model(HI.WORKLOADS["ctx16k_kc32"])
    routed_extra = 32 * 2048 * 8 * 64            # 64 more routed groups per block
    assert kc32["attn_fwd"][1] - base["attn_fwd"][1] == 4 * 128 * routed_extra
    assert kc32["bwd_dkdv"][1] == base["bwd_dkdv"][1]   # routing never reaches dK/dV
