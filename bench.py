#!/usr/bin/env python
"""Benchmark of the routed-HGA hot path: one Qwen3-8B-shaped attention layer at 16K context.

Workload (default ``ctx16k``): batch 1, 32 query / 8 KV heads, head dim 128, bf16 with fp32
accumulation; 14336 detached history tokens + 2048 active-segment tokens; chunk 64, group 8,
query block 64; top-16 chunks then top-64 groups (512 routed tokens per block).  One step =
the whole hot path on synthetic inputs already in HBM: key summaries, routing, forward,
backward dQ, backward dK/dV (5 kernels, captured once as a CUDA graph and replayed per step).
Metric: active-segment tokens per second, forward + backward.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

With N > 1 (torchrun, one process per GPU) every rank runs its own layer (different seed):
the KV heads / batches of the method are independent, so there is no collective in the data
path ("scaling": "weak"); the timed region is bracketed by barriers and the step time is
the max over ranks.  ``--impl reference`` times the float64 CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import hga_inputs as HI  # noqa: E402

METRIC = "routed HGA attn tokens/sec fwd+bwd per layer at 16K ctx; % of HBM/tensor roofline"
L2_FLUSH_BYTES = 512 << 20          # > 126 MB L2: written between timed steps
L2_DRAIN_BYTES = 256 << 20          # then read, evicting the flush's dirty lines (written back here)


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), src="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, src="fallback")


NOMINAL_HBM_GBS = 8000.0   # the B200 datasheet figure, for context next to the measured copy rate


def work_model(w) -> dict:
    """Algorithmic work of each kernel of one step (bytes or flops per launch).

    The backward is booked at the method's own work (FlashAttention-form backward over the routed
    and local pairs, no history gradient): S and dP of a local pair count once, charged to the dQ
    kernel (S, dP, dQ over routed + local pairs); the dK/dV kernel is charged its dK and dV products
    only.  Its recomputation of S^T and dP^T is real work but not the method's: ``executed_flops``
    lists it."""
    B, Hq, Hkv, D, H, S = w.B, w.Hq, w.Hkv, w.D, w.hist_len, w.seg_len
    esz = 2 if w.dtype == "bf16" else 4
    routed_pairs = B * Hq * S * 8 * w.top_groups            # (query, routed key) pairs
    local_pairs = B * Hq * S * (S + 1) // 2                 # causal (query, segment key) pairs
    nch, ngr, nblk = H // 64, H // 8, S // 64
    return {
        "summaries": ("hbm", B * Hkv * H * D * esz + B * Hkv * (ngr + nch) * D * 4),
        "route": ("hbm", B * Hq * S * D * esz + B * Hkv * (nch + ngr) * D * 4
                  + B * Hkv * nblk * (w.top_chunks + w.top_groups) * 4),
        "attn_fwd": ("tensor", 4 * D * (routed_pairs + local_pairs)),
        "bwd_dq": ("tensor", 6 * D * (routed_pairs + local_pairs)),
        "bwd_dkdv": ("tensor", 4 * D * local_pairs),
    }


def executed_flops(w) -> dict:
    """Flops the tensor-core kernels issue, recomputation included: the dK/dV kernel recomputes
    S^T = K Q^T and dP^T = V dO^T over the local pairs (the dQ kernel already formed S and dP)."""
    local_pairs = w.B * w.Hq * w.seg_len * (w.seg_len + 1) // 2
    wm = work_model(w)
    return {"attn_fwd": wm["attn_fwd"][1], "bwd_dq": wm["bwd_dq"][1], "bwd_dkdv": 8 * w.D * local_pairs}


def method_flops(w) -> int:
    """The method's flops per step: forward 4 D (routed + local pairs), backward 6 D (routed +
    local) for S, dP, dQ plus 4 D local for dK, dV (no history gradient)."""
    wm = work_model(w)
    return wm["attn_fwd"][1] + wm["bwd_dq"][1] + wm["bwd_dkdv"][1]


class ClockSampler:
    """SM clock and throttle-reason samples of one GPU taken DURING the timed region.

    Polls NVML from a background thread every ~2 ms (the timed region is tens of milliseconds);
    reports nothing (``clocks: null``) when the NVML bindings are missing."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []          # (sm_mhz, reasons_mask)
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self._nvml = None

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self._physical_index())
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._nvml = nv
        except Exception:
            return self
        self._stop = threading.Event()

        def poll():
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((float(sm), int(rs)))
                except Exception:
                    pass
                time.sleep(0.002)

        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()
        time.sleep(0.01)
        return self

    def _physical_index(self) -> int:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                return int(vis.split(",")[self.gpu])
            except (ValueError, IndexError):
                pass
        return self.gpu

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        if self._nvml is not None:
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return None
        reasons = sorted(n for n, bit in self.REASONS.items() if any(r & bit for _, r in self.samples))
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml, 2 ms poll"}


def dist_setup():
    """One process per GPU (torchrun env).  NCCL where CUDA is present; gloo otherwise, which is
    all the CPU-only reference arm needs."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def all_max(v: float, world: int, device) -> float:
    """Max of v over the ranks (device times are reported as the slowest rank's)."""
    if world == 1:
        return v
    import torch.distributed as dist
    if dist.get_backend() != "nccl":
        device = "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def host_cores() -> int:
    """Cores this process may run on (affinity / cgroup aware where the OS tells)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_layer_pass(w, x, workers: int, n_slices: int | None = None, stages: dict | None = None) -> float:
    """The CPU oracle, as it stands, over the first n_slices (batch, KV head) slices of the layer
    (all of them by default), on `workers` host threads, in three phases of concurrent tasks (the
    oracle's C calls release the GIL): summaries and float32-decision routing per slice; the
    float64 forward of every (slice, 64-query block) unit; the dK/dV of every slice and the dQ of
    every unit.  A slice -- its G query heads with their history, segment K/V and routing -- is
    independent of every other slice.  Returns seconds (wall clock); `stages`, when given, receives
    each phase's seconds."""
    import concurrent.futures as cf

    import numpy as np

    from oracle import oracle as O
    t0 = time.perf_counter()
    f64 = {k: v.double().numpy() for k, v in x.items() if k != "needles"}
    G, S, nblk = w.Hq // w.Hkv, w.seg_len, w.seg_len // 64
    slices = [(b, kh) for b in range(w.B) for kh in range(w.Hkv)][:n_slices]

    def sl(b, kh):
        hs = slice(kh * G, (kh + 1) * G)
        return (f64["q"][b:b + 1, hs], f64["k_hist"][b:b + 1, kh:kh + 1], f64["v_hist"][b:b + 1, kh:kh + 1],
                f64["k_seg"][b:b + 1, kh:kh + 1], f64["v_seg"][b:b + 1, kh:kh + 1]), f64["d_o"][b:b + 1, hs]

    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        def route(b, kh):
            (q, kh_, *_), _ = sl(b, kh)
            return O.route_from_inputs(q, kh_, 1, w.top_chunks, w.top_groups, prec=32)["group_idx"]
        gi = dict(zip(slices, ex.map(lambda j: route(*j), slices)))
        t1 = time.perf_counter()
        block_rows = [np.array([hh * S + n * 64 + t for hh in range(G) for t in range(64)], dtype=np.int64)
                      for n in range(nblk)]
        fwd = []
        for b, kh in slices:
            args, _ = sl(b, kh)
            for rows in block_rows:               # forward of the block's G x 64 rows
                fwd.append(ex.submit(O.attn_fwd, *args, gi[(b, kh)], rows=rows))
        for t in fwd:
            t.result()
        t2 = time.perf_counter()
        bwd = []
        for b, kh in slices:                     # dK/dV of a slice: the longest tasks, queued first
            args, do = sl(b, kh)
            bwd.append(ex.submit(O.attn_bwd, *args, gi[(b, kh)], do, rows=np.array([0]),
                                 keys=np.arange(S)))
        for b, kh in slices:
            args, do = sl(b, kh)
            for rows in block_rows:               # dQ of the block's G x 64 rows
                bwd.append(ex.submit(O.attn_bwd, *args, gi[(b, kh)], do, rows=rows, keys=np.array([S - 1])))
        for t in bwd:
            t.result()
        t3 = time.perf_counter()
    if stages is not None:
        stages.update(summaries_and_route_s=t1 - t0, fwd_s=t2 - t1, bwd_s=t3 - t2)
    return t3 - t0


ORACLE_SAMPLE = ("the CPU oracle as it stands (plain C, float32-decision routing, float64 attention) over {what}, "
                 "in three phases of concurrent tasks on {workers} host threads: summaries and routing per (batch, "
                 "KV head); forward per (batch, KV head, 64-query block) unit; dK/dV per (batch, KV head) and dQ per "
                 "unit; wall clock")


def _oracle_baseline(w, x, warm: bool = True) -> dict:
    """The oracle over the whole layer on all host cores; when that takes longer than ~8 s, over the
    first (batch, KV head) slices only, as many as fit ~8 s, scaled to the whole layer's tokens."""
    workers = host_cores()
    total = w.B * w.Hkv
    n = total
    if warm:
        t1 = oracle_layer_pass(w, x, workers, n)
        if t1 > 8.0:
            n = max(1, min(total, int(total * 8.0 / t1)))
    stages = {}
    t = oracle_layer_pass(w, x, workers, n, stages)
    what = "the whole layer" if n == total else f"{n} of the layer's {total} (batch, KV head) slices"
    tokens = w.B * w.seg_len * n / total
    return {"value": tokens / t, "unit": "tokens/s", "cores": workers,
            "kind": "oracle", "sample": ORACLE_SAMPLE.format(what=what, workers=workers), "seconds": t,
            "stages_seconds": {k: round(v, 3) for k, v in stages.items()}, "slices": n, "host_cores": workers}


def run_reference(args, w, world, rank):
    """The reference arm: the CPU oracle as it stands, one layer pass (or the bounded slice sample
    of _oracle_baseline) per step, on the host cores; rank 0 only."""
    if rank != 0:
        return
    x = HI.make_inputs(w, args.seed)
    workers = host_cores()
    total = w.B * w.Hkv
    n = total
    for i in range(args.warmup):
        t1 = oracle_layer_pass(w, x, workers, n)
        if i == 0 and t1 > 8.0:                  # keep the whole run within a few minutes
            n = max(1, min(total, int(total * 8.0 / t1)))
    ts = [oracle_layer_pass(w, x, workers, n) for _ in range(args.steps)]
    t_step = statistics.mean(ts)
    tokens = w.B * w.seg_len * n / total
    value = tokens / t_step
    what = "the whole layer" if n == total else f"{n} of the layer's {total} (batch, KV head) slices"
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": _config(w, args), "gpu_launches": 0,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": workers, "kind": "oracle",
                             "sample": ORACLE_SAMPLE.format(what=what, workers=workers)},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _time_layer(H, w, seed, dev, stream, flush_l2, steps=5, warmup=3, causal=False, summaries_from=None) -> float:
    """Mean device time (ms) of one whole layer step of workload w, L2 flushed before each step
    (causal: with the strictly causal routing, the previous segment's last block as q_prev;
    summaries_from: the step computes the summaries of history tokens [summaries_from, H) only)."""
    x = {k: v.to(dev) for k, v in HI.make_inputs(w, seed).items() if k != "needles"}
    if causal:
        x["q_prev"] = HI.prev_block_q(w, seed).to(dev)
    cfg = H.make_config(x["q"], x["k_hist"], w.top_chunks, w.top_groups)
    step = H.LayerStep(cfg, dev, causal_routing=causal, summaries_from=summaries_from)
    if summaries_from is not None:
        step.build_all_summaries(x)
    graph = step.capture(x, warmup=warmup)            # replayed like the headline's step
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush_l2()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    if H.read_status(step.ws) != 0:
        raise RuntimeError(f"device status word set while timing {w.name}")
    return sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps


def _leakage_probe(H, w, seed, dev) -> dict:
    """The pages' probe of the within-block side channel: change a later query of a block and see
    whether earlier outputs move.  The last query of block 0 (head 0) is pushed towards a chunk block
    0 did not select; reported is the largest change of any output before it, under the standard and
    under the strictly causal routing."""
    x = {k: v.to(dev) for k, v in HI.make_inputs(w, seed).items() if k != "needles"}
    x["q_prev"] = HI.prev_block_q(w, seed).to(dev)
    cfg = H.make_config(x["q"], x["k_hist"], w.top_chunks, w.top_groups)
    out = {}
    for name, causal in (("standard", False), ("strictly_causal", True)):
        s0 = H.LayerStep(cfg, dev, causal_routing=causal)
        s0.forward(x)
        torch.cuda.synchronize(dev)
        if name == "standard":
            chosen = set(s0.chunk_idx[0, 0, 0].tolist())
            other = next(i for i in range(w.nch) if i not in chosen)
            z = dict(x)
            z["q"] = x["q"].clone()
            z["q"][0, 0, w.qblock - 1] += (400.0 * s0.chunk_sum[0, 0, other]).to(z["q"].dtype)
        s1 = H.LayerStep(cfg, dev, causal_routing=causal)
        s1.forward(z)
        torch.cuda.synchronize(dev)
        d = (s0.o[:, :, :w.qblock - 1].float() - s1.o[:, :, :w.qblock - 1].float()).abs().max().item()
        out[f"{name}_max_abs_change_before"] = d
    out["perturbed"] = f"query {w.qblock - 1} of head 0 (last of block 0), pushed towards an unselected chunk"
    return out


def _time_tiered(H, w, seed, dev, stream, flush_l2, world, steps=5, warmup=2) -> dict:
    """The layer of workload w with its history K/V in pinned host memory (TieredLayerStep), and the
    same layer with the history resident in device memory, both timed per step on the device; then
    the pages' three tiers: also the group summaries in pinned host memory behind a device cache
    smaller than the history (GroupSummaryCache), the chunk summaries alone resident, with two query
    sets alternating from step to step so that steps fetch the chunks the cache lacks."""
    x = HI.make_inputs(w, seed)
    xd = {k: x[k].to(dev) for k in ("q", "k_seg", "v_seg", "d_o")}
    kh, vh = x["k_hist"].pin_memory(), x["v_hist"].pin_memory()
    cfg = H.make_config(xd["q"], x["k_hist"], w.top_chunks, w.top_groups)
    # summaries are built when the history is written, while its keys are still on the device
    gs, cs = H.build_summaries(cfg, x["k_hist"].to(dev))
    step = H.TieredLayerStep(cfg, kh, vh, gs, cs, dev)

    def timed(st, inputs):
        for i in range(warmup):
            st(inputs[i % len(inputs)])
        st.wait(timeout_s=60)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i, (e0, e1) in enumerate(ev):
            flush_l2()
            e0.record(stream)
            st(inputs[i % len(inputs)])
            e1.record(stream)
        st.wait(timeout_s=60)
        return all_max(sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps, world, dev)

    ms = timed(step, [xd])
    nbytes = step.gather_bytes()
    resident_ms = all_max(_time_layer(H, w, seed, dev, stream, flush_l2), world, dev)
    tokens = w.B * w.seg_len * world
    # the three tiers: group summaries in host memory behind the device cache, 4 chunk slots short of
    # the whole history (a step of these inputs chooses at most 215 of the 224 chunks of a KV head)
    cap = max(1, w.nch - 4)
    gcache = H.GroupSummaryCache(cfg, gs.cpu().pin_memory(), cap, dev)
    step3 = H.TieredLayerStep(cfg, kh, vh, None, cs, dev, group_cache=gcache)
    xd2 = dict(xd, q=HI.make_inputs(w, seed + 1)["q"].to(dev))
    step3([xd, xd2][0])
    step3.wait(timeout_s=60)
    cold = gcache.stats()
    ms3 = timed(step3, [xd2, xd])
    warm = gcache.stats()
    return {"workload": f"{w.name}: the 16K layer at batch {w.B}, history K/V ({2 * kh.numel() * kh.element_size() >> 20}"
                        " MiB) in pinned host memory, summaries in device memory",
            "ms_per_step": ms, "tokens_per_s": tokens / (ms * 1e-3),
            "gather_bytes_per_step": nbytes, "host_link_GBps": nbytes / (ms * 1e-3) / 1e9,
            "resident_ms_per_step": resident_ms, "resident_tokens_per_s": tokens / (resident_ms * 1e-3),
            "group_summary_cache": {
                "layout": f"chunk summaries in device memory; group summaries ({gs.numel() * 4 >> 20} MiB) in pinned "
                          f"host memory behind a device cache of {cap} of the {w.nch} chunks per (batch, KV head) "
                          "(8 group summaries = 4 KB per chunk slot, least recently used replaced); K/V as above; "
                          "two query sets alternate from step to step",
                "cap_chunks": cap, "ms_per_step": ms3, "tokens_per_s": tokens / (ms3 * 1e-3),
                "first_step": cold, "last_step": warm,
                "host_bytes_per_step": warm["host_bytes"] + step3.gather_bytes()}}


def _time_forward_131k(H, w, seed, dev, stream, flush_l2, world, steps=5, warmup=3) -> dict:
    """Evaluation-length forward, no backward: the summaries of the whole history built on the
    device, routing, and the routed + causal forward.  Each kernel is bracketed by CUDA events (so
    the kernels do not overlap through dependent launch here), L2 flushed before every step; also
    reports how many planted needle groups the routing recovered."""
    xc = HI.make_inputs(w, seed)
    needles = xc.pop("needles")
    x = {k: v.to(dev) for k, v in xc.items()}
    cfg = H.make_config(x["q"], x["k_hist"], w.top_chunks, w.top_groups)
    step = H.LayerStep(cfg, dev)
    calls = step.calls(x, stream.cuda_stream)[:3]          # summaries, route, attn_fwd
    for _ in range(warmup):
        for _, c in calls:
            c()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(steps)]
    for e in ev:
        flush_l2()
        e[0].record(stream)
        for j, (_, c) in enumerate(calls):
            c()
            e[j + 1].record(stream)
    torch.cuda.synchronize(dev)
    if H.read_status(step.ws) != 0:
        raise RuntimeError(f"device status word set while timing {w.name}")
    ms = all_max(sum(e[0].elapsed_time(e[-1]) for e in ev) / steps, world, dev)
    per_us = {n: 1e3 * sum(e[j].elapsed_time(e[j + 1]) for e in ev) / steps for j, (n, _) in enumerate(calls)}
    wm, pk = work_model(w), _peaks()
    frac = {n: wm[n][1] / (per_us[n] * 1e-6) / ((pk["bf16"] * 1e12) if wm[n][0] == "tensor" else (pk["hbm"] * 1e9))
            for n in per_us}
    gi = step.group_idx.cpu()
    hits = sum(int(j) in gi[0, kh, n].tolist() for kh, n, j in needles.tolist())
    return {"workload": f"{w.name}: B={w.B}, Hq={w.Hq}, Hkv={w.Hkv}, history={w.hist_len}, segment={w.seg_len}, "
                        f"top_chunks={w.top_chunks}, top_groups={w.top_groups}, {w.dtype}, forward only",
            "ms_per_step": ms, "tokens_per_s": w.B * w.seg_len * world / (ms * 1e-3),
            "per_kernel_us": per_us, "per_kernel_frac": frac,
            "needles_recovered": f"{hits}/{len(needles)}"}


def _config(w, args):
    return {"workload": f"{w.name}: routed HGA layer, B={w.B}, Hq={w.Hq}, Hkv={w.Hkv}, D={w.D}, "
                        f"history={w.hist_len}, segment={w.seg_len}, chunk=64, group=8, qblock=64, "
                        f"top_chunks={w.top_chunks}, top_groups={w.top_groups}, {w.dtype}",
            "global_batch": w.B * args.gpus, "seq_len": w.hist_len + w.seg_len, "active_segment": w.seg_len,
            "parallelism": f"independent layer per GPU x{args.gpus}",
            "l2": (f"flushed before every timed step: {L2_FLUSH_BYTES >> 20} MiB written, then "
                   f"{L2_DRAIN_BYTES >> 20} MiB read so the flush's dirty lines are written back before "
                   "the step starts (L2 holds none of the step's data)")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="hga", choices=["hga", "reference"])
    ap.add_argument("--workload", default="ctx16k", choices=sorted(HI.WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-tiered", action="store_true", help="skip the tiered-history (batch 4) measurement")
    ap.add_argument("--no-131k", action="store_true", help="skip the 131K-context forward measurement")
    ap.add_argument("--no-positions", action="store_true",
                    help="skip timing the 16K layer at its earlier segment positions and other budgets")
    args = ap.parse_args()
    w = HI.WORKLOADS[args.workload]
    world, rank, local = dist_setup()
    if args.gpus != world and world > 1:
        args.gpus = world
    if args.impl == "reference":
        run_reference(args, w, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import hierarchical_kv_routing_tok_b200 as H
    from hierarchical_kv_routing_tok_b200 import _capi as C

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    x_cpu = HI.make_inputs(w, args.seed + rank)
    x = {k: v.to(dev) for k, v in x_cpu.items() if k != "needles"}
    cfg = H.make_config(x["q"], x["k_hist"], w.top_chunks, w.top_groups)
    step = H.LayerStep(cfg, dev)
    stream = torch.cuda.current_stream(dev)
    calls = step.calls(x, stream.cuda_stream)
    names = [n for n, _ in calls]
    # the routing call launches one kernel, or three for a long history (block queries, chunk scores
    # of all blocks at once, selection + group level)
    launches_per_step = len(calls) - 1 + H._capi.route_launches(cfg, with_workspace=True)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    drain = torch.ones(L2_DRAIN_BYTES // 4, dtype=torch.float32, device=dev)
    drain_out = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        torch.sum(drain, dim=0, out=drain_out)

    for _ in range(max(args.warmup, 3)):
        for _, c in calls:
            c()
    torch.cuda.synchronize(dev)
    if H.read_status(step.ws) != 0:
        raise RuntimeError("device status word set during warm-up")

    K = args.steps
    ev_step = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize(dev)
    # the step captured once as a CUDA graph (the same kernels and dependent launches, without the
    # per-call host work of the C ABI); the headline replays it
    graph = step.capture(x)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        # the headline: K graph replays of the step, events at the step boundaries only (an event
        # between two kernels would cost its own time and keep the next kernel from starting early)
        for i in range(K):
            flush_l2()
            ev_step[i][0].record(stream)
            graph.replay()
            ev_step[i][1].record(stream)
        torch.cuda.synchronize(dev)
        # the per-kernel device times for the roofline: K more steps, an event after every kernel
        for i in range(K):
            flush_l2()
            ev[i][0].record(stream)
            for j, (_, c) in enumerate(calls):
                c()
                ev[i][j + 1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    step_ms = [e0.elapsed_time(e1) for e0, e1 in ev_step]
    kern_ms = {n: [ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)] for j, n in enumerate(names)}
    t_step = all_max(sum(step_ms) / K, world, dev) * 1e-3
    t_step_kernel_events = all_max(sum(ev[i][0].elapsed_time(ev[i][-1]) for i in range(K)) / K, world, dev)
    tokens = w.B * w.seg_len * world
    value = tokens / t_step
    if H.read_status(step.ws) != 0:
        raise RuntimeError("device status word set during the timed region")

    # the same layer at the earlier segment positions of a 16K sequence (history 2048 / 6144 /
    # 10240 / 14336): attention work per token is flat, only summaries and chunk scoring grow
    # (timed alike: events at step boundaries only)
    positions = None
    if w.name == "ctx16k" and not args.no_positions:
        positions = {}
        for pname in ("ctx4k", "ctx8k", "ctx12k", "ctx16k"):
            pw = HI.WORKLOADS[pname]
            ms = all_max(_time_layer(H, pw, args.seed + rank, dev, stream, flush_l2), world, dev)
            positions[f"history_{pw.hist_len}"] = {"ms_per_step": ms,
                                                   "tokens_per_s": pw.B * pw.seg_len * world / (ms * 1e-3)}
    # routing-budget sweep of the same layer (the pages vary the routed chunk count from 8 to 32)
    budgets = None
    if w.name == "ctx16k" and not args.no_positions:
        budgets = {}
        for pname in ("ctx16k_kc8", "ctx16k", "ctx16k_kc32"):
            pw = HI.WORKLOADS[pname]
            ms = all_max(_time_layer(H, pw, args.seed + rank, dev, stream, flush_l2), world, dev)
            budgets[f"top_chunks_{pw.top_chunks}_top_groups_{pw.top_groups}"] = {
                "ms_per_step": ms, "tokens_per_s": pw.B * pw.seg_len * world / (ms * 1e-3)}

    # the same step with the summaries built incrementally: only the 2048 tokens of the segment that
    # closed last are summarised (the rest of the history's summaries are kept from earlier steps)
    incremental = None
    if w.hist_len >= w.seg_len and not args.no_positions:
        ms = all_max(_time_layer(H, w, args.seed + rank, dev, stream, flush_l2,
                                 summaries_from=w.hist_len - w.seg_len), world, dev)
        incremental = {"ms_per_step": ms, "tokens_per_s": w.B * w.seg_len * world / (ms * 1e-3),
                       "summaries": f"history tokens [{w.hist_len - w.seg_len}, {w.hist_len}) only "
                                    "(hga_append_summaries of the segment that closed last)"}

    # strictly causal routing (block n routed with block n-1's query): same kernels, other routing
    causal = None
    if w.name == "ctx16k" and not args.no_positions:
        ms = all_max(_time_layer(H, w, args.seed + rank, dev, stream, flush_l2, causal=True), world, dev)
        causal = {"ms_per_step": ms, "tokens_per_s": w.B * w.seg_len * world / (ms * 1e-3),
                  "leakage_probe": _leakage_probe(H, w, args.seed + rank, dev)}

    # tiered-history variant of the 16K layer at batch 4: history K/V in pinned host memory, the
    # summaries in device memory, the routed groups gathered per batch element on a side stream
    tiered = None
    if w.name == "ctx16k" and not args.no_tiered:
        tiered = _time_tiered(H, HI.WORKLOADS["ctx16k_b4"], args.seed + rank, dev, stream, flush_l2, world)

    # evaluation-length forward (131K context, routing over 129,024 history tokens, planted needles)
    fwd131k = None
    if w.name == "ctx16k" and not args.no_131k:
        fwd131k = _time_forward_131k(H, HI.WORKLOADS["ctx131k"], args.seed + rank, dev, stream, flush_l2, world)

    # roofline of the dominant kernel
    wm = work_model(w)
    pk = _peaks()
    dom = max(names, key=lambda n: sum(kern_ms[n]))
    avg_s = sum(kern_ms[dom]) / K * 1e-3
    bound, work = wm[dom]
    if bound == "tensor":
        achieved, peak, unit = work / avg_s / 1e12, pk["bf16"], "TFLOP/s"
    else:
        achieved, peak, unit = work / avg_s / 1e9, pk["hbm"], "GB/s"
    traffic = None
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            tr = json.load(f).get(f"{w.name}:{dom}")
        if tr and tr.get("kernel_source_sha") == _kernel_sha(dom):
            traffic = tr["dram_bytes_per_launch"]
    except (OSError, ValueError):
        pass
    mflops = method_flops(w)
    ex = executed_flops(w)
    per_us = {n: 1e3 * sum(v) / K for n, v in kern_ms.items()}
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": traffic, "kernel": dom, "peak_source": f"{pk['src']} (burst)",
                "per_kernel_us": per_us,
                "per_kernel_pass": f"a second pass of {K} steps, L2 flushed alike, with an event after every kernel "
                                   f"({t_step_kernel_events:.4f} ms per step with those events)",
                "per_kernel_frac": {n: (wm[n][1] / (sum(kern_ms[n]) / K * 1e-3)
                                        / ((pk["bf16"] * 1e12) if wm[n][0] == "tensor" else (pk["hbm"] * 1e9)))
                                    for n in names},
                "per_kernel_executed_frac": {n: ex[n] / (per_us[n] * 1e-6) / (pk["bf16"] * 1e12) for n in ex},
                # the memory-bound kernels also against the nominal 8 TB/s of the part
                "per_kernel_frac_nominal_hbm": {n: wm[n][1] / (per_us[n] * 1e-6) / (NOMINAL_HBM_GBS * 1e9)
                                                for n in names if wm[n][0] == "hbm"},
                "work_booking": "backward at the method's work: S, dP, dQ over routed + local pairs charged to "
                                "bwd_dq, dK and dV over local pairs to bwd_dkdv (its S^T, dP^T recomputation "
                                "is in per_kernel_executed_frac only)"}
    # the whole step against the method's flops (forward + backward, S and dP counted once)
    method = {"gflop_per_step": mflops / 1e9, "achieved_tflops": mflops / t_step / 1e12,
              "frac_burst": mflops / t_step / (pk["bf16"] * 1e12),
              "frac_sustained": mflops / t_step / (pk["bf16_sustained"] * 1e12),
              "peaks": f"{pk['src']}: {pk['bf16']} TFLOP/s burst, {pk['bf16_sustained']} sustained"}

    # end to end through the public API with pinned host buffers: every step copies its inputs in
    # and its outputs out.  Steps are pipelined the way a stream of steps would run: two sets of
    # device buffers, the host->device copy of step i+1 and the device->host copy of step i-1 (two
    # copy engines, two streams) overlap the compute of step i.  The workload keeps the detached
    # history's K/V resident in HBM (it is device state that successive segments append to, not a
    # per-step input), so the headline copies the active segment's q, k_seg, v_seg, d_o per step;
    # the same pipeline with the history K/V copied in every step as well is reported beside it.
    e2e = None
    if not args.no_e2e:
        x_host = {k: x_cpu[k].pin_memory() for k in ("q", "k_hist", "v_hist", "k_seg", "v_seg", "d_o")}
        outs_of = lambda st_b: [st_b.o, st_b.dq, st_b.dk, st_b.dv]
        host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs_of(step)]
        d2h = sum(t.numel() * t.element_size() for t in host_out)
        K2 = max(3, min(K, 10))
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def time_e2e(in_names):
            sets = []
            for b in range(2):
                xs = x if b == 0 else {k: (v.clone() if k in in_names else v) for k, v in x.items()}
                st_b = step if b == 0 else H.LayerStep(cfg, dev)
                sets.append((xs, st_b, st_b.capture(xs)))

            def run_e2e(n):
                ev = lambda: torch.cuda.Event()
                copied, computed, drained = [None] * n, [None] * n, [None] * n
                for i in range(n):
                    xs, st_b, g_b = sets[i % 2]
                    with torch.cuda.stream(s_in):            # inputs of step i (set i % 2 free after step i-2)
                        if i >= 2:
                            s_in.wait_event(computed[i - 2])
                        for k in in_names:
                            xs[k].copy_(x_host[k], non_blocking=True)
                        copied[i] = ev(); copied[i].record(s_in)
                    stream.wait_event(copied[i])             # compute of step i
                    if i >= 2:
                        stream.wait_event(drained[i - 2])    # its output buffers were read out
                    g_b.replay()
                    computed[i] = ev(); computed[i].record(stream)
                    with torch.cuda.stream(s_out):           # outputs of step i
                        s_out.wait_event(computed[i])
                        for d, h in zip(outs_of(st_b), host_out):
                            h.copy_(d, non_blocking=True)
                        drained[i] = ev(); drained[i].record(s_out)
                stream.wait_event(drained[n - 1])

            run_e2e(2)
            torch.cuda.synchronize(dev)
            barrier(world)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run_e2e(K2)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier(world)
            t = all_max(e0.elapsed_time(e1) / K2, world, dev) * 1e-3
            h2d = sum(x_host[k].numel() * x_host[k].element_size() for k in in_names)
            return t, h2d

        t_e2e, h2d = time_e2e(["q", "k_seg", "v_seg", "d_o"])
        t_all, h2d_all = time_e2e(["q", "k_hist", "v_hist", "k_seg", "v_seg", "d_o"])
        e2e = {"value": tokens / t_e2e, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": t_e2e * 1e3,
               "per_step_inputs": "q, k_seg, v_seg, d_o copied in, o, dq, dk, dv copied out every step; the "
                                  "history K/V resident in HBM (device state the segments append to)",
               "pipelining": "host->device copy of step i+1 and device->host copy of step i-1 overlap step i",
               "history_copied_every_step": {"value": tokens / t_all, "unit": "tokens/s",
                                             "h2d_bytes_per_step": h2d_all, "d2h_bytes_per_step": d2h,
                                             "ms_per_step": t_all * 1e3}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = _oracle_baseline(w, x_cpu, warm=False)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
                "config": _config(w, args), "roofline": roofline, "method_frac": method["frac_burst"],
                "method_roofline": method, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": K * launches_per_step, "clocks": clk.summary(),
                "step_launch": "one CUDA graph replay per step: the step's kernels and their dependent "
                               "launches, captured once through the C ABI (the per-kernel pass launches "
                               "them one by one)",
                "kernels_per_step": names,
                "route_launches": launches_per_step - (len(calls) - 1)}
        if incremental:
            line["incremental_summaries"] = incremental
        if positions:
            line["segment_positions"] = positions
        if budgets:
            line["routing_budget_sweep"] = budgets
        if causal:
            line["strictly_causal_routing"] = causal
        if tiered:
            line["tiered_history"] = tiered
        if fwd131k:
            line["forward_131k"] = fwd131k
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# The sources each timed kernel is compiled from (its file, the shared device helpers it includes).
KERNEL_SOURCES = {
    "summaries": ("summaries.cu", "common.cuh"),
    "route": ("route.cu", "common.cuh"),
    "attn_fwd": ("attn_tc_fwd.cu", "tc_common.cuh", "common.cuh"),
    "bwd_dq": ("attn_tc_bwd.cu", "tc_common.cuh", "common.cuh"),
    "bwd_dkdv": ("attn_tc_bwd.cu", "tc_common.cuh", "common.cuh"),
}


def _kernel_sha(kernel: str) -> str:
    """Hash of the sources of one kernel: a DRAM-traffic record in profiles/traffic.json is used
    only while this matches the hash stored with it."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hierarchical_kv_routing_tok_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    main()
