"""ctypes binding of the routed-HGA C ABI (``include/hga.h``, ``libhga.so``).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libhga.so``.  If the library is missing, loading raises; there is no fallback.
Pointer arguments are plain integers (device addresses); ``stream`` is a
``cudaStream_t`` as an integer (0 = legacy default stream).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhga.so")

HGA_OK = 0
HGA_ERR_ARG = -1
HGA_ERR_ALIGN = -2
HGA_ERR_UNSUPPORTED = -3
HGA_ERR_CUDA = -4
HGA_ERR_TIMEOUT = -5
HGA_ERR_WORKSPACE = -6
HGA_ERR_TOO_LARGE = -7
HGA_NOALLOC_MAX_ROWS = 1 << 20
HGA_F32 = 0
HGA_BF16 = 1

#: every entry point declared in include/hga.h
EXPORTS = ("hga_workspace_size", "hga_route_launches", "hga_build_summaries", "hga_append_summaries", "hga_route", "hga_route_causal", "hga_attn_fwd",
           "hga_attn_bwd",
           "hga_attn_bwd_preprocess", "hga_attn_bwd_dkdv", "hga_attn_bwd_dq", "hga_attn_bwd_noalloc",
           "hga_noalloc_read_status", "hga_tier_cache_config", "hga_route_chunks", "hga_gcache_plan",
           "hga_gcache_fetch", "hga_route_groups_cached", "hga_tier_plan", "hga_tier_gather",
           "hga_read_status", "hga_strerror", "hga_version")


class HGAConfig(ctypes.Structure):
    """Mirror of ``hga_config_t``."""
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
                ("hist_len", ctypes.c_int64), ("seg_len", ctypes.c_int64),
                ("chunk", ctypes.c_int32), ("group", ctypes.c_int32), ("qblock", ctypes.c_int32),
                ("top_chunks", ctypes.c_int32), ("top_groups", ctypes.c_int32),
                ("n_sink_tokens", ctypes.c_int32), ("dtype", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("hist_capacity", ctypes.c_int64), ("wait_limit_ns", ctypes.c_int64)]

    def __repr__(self):
        return "HGAConfig(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class HGAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {strerror(code)} (code {code})")
        self.code = code


_lib = None


def load() -> ctypes.CDLL:
    """Load libhga.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m hierarchical_kv_routing_tok_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, C = ctypes.c_void_p, ctypes.POINTER(HGAConfig)
    sig = {
        "hga_workspace_size": [C, ctypes.POINTER(ctypes.c_size_t)],
        "hga_route_launches": [C, ctypes.c_int, ctypes.POINTER(ctypes.c_int32)],
        "hga_build_summaries": [C, P, P, P, P, P],
        "hga_append_summaries": [C, P, P, P, ctypes.c_int64, P, P],
        "hga_route": [C, P, P, P, P, P, P, P],
        "hga_route_causal": [C, P, P, P, P, P, P, P, P],
        "hga_attn_fwd": [C, P, P, P, P, P, P, P, P, P, P],
        "hga_attn_bwd": [C, P, P, P, P, P, P, P, P, P, P, P, P, P, P],
        "hga_attn_bwd_preprocess": [C, P, P, P, P],
        "hga_attn_bwd_dkdv": [C, P, P, P, P, P, P, P, P, P],
        "hga_attn_bwd_dq": [C, P, P, P, P, P, P, P, P, P, P, P, P],
        "hga_attn_bwd_noalloc": [C, P, P, P, P, P, P, P, P, P, P, P, P, P],
        "hga_noalloc_read_status": [P, ctypes.POINTER(ctypes.c_int32)],
        "hga_tier_cache_config": [C, C],
        "hga_route_chunks": [C, P, P, P, P, P, P],
        "hga_gcache_plan": [C, ctypes.c_int32, P, P, P, P, ctypes.c_int32, P, P, P, P, P],
        "hga_gcache_fetch": [C, ctypes.c_int32, P, P, P, P, P, P],
        "hga_route_groups_cached": [C, P, P, P, ctypes.c_int32, P, P, P, P],
        "hga_tier_plan": [C, P, P, P, P, P, P],
        "hga_tier_gather": [C, P, P, P, P, P, P, P],
        "hga_read_status": [P, P, ctypes.POINTER(ctypes.c_int32)],
        "hga_strerror": [ctypes.c_int],
        "hga_version": [],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_char_p if name == "hga_strerror" else ctypes.c_int
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().hga_strerror(int(code)).decode()


def version() -> int:
    return load().hga_version()


def _call(name: str, *args) -> None:
    rc = getattr(load(), name)(*args)
    if rc != HGA_OK:
        raise HGAError(name, rc)


def make_config(B: int, Hq: int, Hkv: int, hist_len: int, seg_len: int, top_chunks: int, top_groups: int,
                dtype: int = HGA_BF16, D: int = 128, softmax_scale: float = 0.0, chunk: int = 64,
                group: int = 8, qblock: int = 64, n_sink_tokens: int = 0, hist_capacity: int = 0,
                wait_limit_ns: int = 0) -> HGAConfig:
    return HGAConfig(B, Hq, Hkv, D, hist_len, seg_len, chunk, group, qblock, top_chunks, top_groups,
                     n_sink_tokens, dtype, softmax_scale, hist_capacity, wait_limit_ns)


def route_launches(cfg: HGAConfig, with_workspace: bool = True) -> int:
    out = ctypes.c_int32()
    _call("hga_route_launches", ctypes.byref(cfg), 1 if with_workspace else 0, ctypes.byref(out))
    return out.value


def workspace_size(cfg: HGAConfig) -> int:
    out = ctypes.c_size_t(0)
    _call("hga_workspace_size", ctypes.byref(cfg), ctypes.byref(out))
    return int(out.value)


def build_summaries(cfg, k_hist, group_sum, chunk_sum, workspace, stream=0) -> None:
    _call("hga_build_summaries", ctypes.byref(cfg), k_hist, group_sum, chunk_sum, workspace, stream)


def append_summaries(cfg, k_hist, group_sum, chunk_sum, first_token, workspace, stream=0) -> None:
    _call("hga_append_summaries", ctypes.byref(cfg), k_hist, group_sum, chunk_sum, int(first_token), workspace,
          stream)


def route(cfg, q, group_sum, chunk_sum, chunk_idx, group_idx, workspace, stream=0) -> None:
    _call("hga_route", ctypes.byref(cfg), q, group_sum, chunk_sum, chunk_idx, group_idx, workspace, stream)


def route_causal(cfg, q, q_prev, group_sum, chunk_sum, chunk_idx, group_idx, workspace, stream=0) -> None:
    """Strictly causal routing: block n routed with block n-1's query (block 0: q_prev, or 0 = none)."""
    _call("hga_route_causal", ctypes.byref(cfg), q, q_prev, group_sum, chunk_sum, chunk_idx, group_idx, workspace,
          stream)


def attn_fwd(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, workspace, stream=0) -> None:
    _call("hga_attn_fwd", ctypes.byref(cfg), q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, workspace,
          stream)


def attn_bwd(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o, dq, dk_seg, dv_seg, workspace,
             stream=0) -> None:
    _call("hga_attn_bwd", ctypes.byref(cfg), q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o, dq,
          dk_seg, dv_seg, workspace, stream)


def attn_bwd_preprocess(cfg, o, d_o, workspace, stream=0) -> None:
    _call("hga_attn_bwd_preprocess", ctypes.byref(cfg), o, d_o, workspace, stream)


def attn_bwd_dkdv(cfg, q, k_seg, v_seg, lse, d_o, dk_seg, dv_seg, workspace, stream=0) -> None:
    _call("hga_attn_bwd_dkdv", ctypes.byref(cfg), q, k_seg, v_seg, lse, d_o, dk_seg, dv_seg, workspace, stream)


def attn_bwd_dq(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o, dq, workspace, stream=0) -> None:
    """dq; also leaves delta = rowsum(d_o * o) in the workspace for attn_bwd_dkdv."""
    _call("hga_attn_bwd_dq", ctypes.byref(cfg), q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o, dq,
          workspace, stream)


def attn_bwd_noalloc(cfg, q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o, dq, dk_seg, dv_seg,
                     stream=0) -> None:
    """hga_attn_bwd without a workspace: for callers that cannot allocate device memory (the
    library's fixed per-device scratch is used instead; overlapping calls race)."""
    _call("hga_attn_bwd_noalloc", ctypes.byref(cfg), q, k_hist, v_hist, k_seg, v_seg, group_idx, o, lse, d_o,
          dq, dk_seg, dv_seg, stream)


def noalloc_read_status(stream=0) -> int:
    """Device-side status of the last attn_bwd_noalloc call on the current device (read and cleared)."""
    out = ctypes.c_int32(0)
    _call("hga_noalloc_read_status", stream, ctypes.byref(out))
    return int(out.value)


def route_chunks(cfg, q, chunk_sum, chunk_idx, qb, workspace, stream=0) -> None:
    """Level 1 of the routing only: chunk_idx and the block queries qb."""
    _call("hga_route_chunks", ctypes.byref(cfg), q, chunk_sum, chunk_idx, qb, workspace, stream)


def gcache_plan(cfg, cap_chunks, chunk_idx, slot_of, chunk_of, stamp, step, miss_chunk, miss_slot, counts,
                workspace, stream=0) -> None:
    _call("hga_gcache_plan", ctypes.byref(cfg), int(cap_chunks), chunk_idx, slot_of, chunk_of, stamp, int(step),
          miss_chunk, miss_slot, counts, workspace, stream)


def gcache_fetch(cfg, cap_chunks, group_sum_src, miss_chunk, miss_slot, counts, gcache, stream=0) -> None:
    _call("hga_gcache_fetch", ctypes.byref(cfg), int(cap_chunks), group_sum_src, miss_chunk, miss_slot, counts,
          gcache, stream)


def route_groups_cached(cfg, qb, chunk_idx, slot_of, cap_chunks, gcache, group_idx, workspace, stream=0) -> None:
    _call("hga_route_groups_cached", ctypes.byref(cfg), qb, chunk_idx, slot_of, int(cap_chunks), gcache, group_idx,
          workspace, stream)


def tier_cache_config(cfg) -> HGAConfig:
    """Configuration of the attention calls over the compact history cache of a tiered step."""
    out = HGAConfig()
    _call("hga_tier_cache_config", ctypes.byref(cfg), ctypes.byref(out))
    return out


def tier_plan(cfg, group_idx, used_groups, n_used, compact_idx, workspace, stream=0) -> None:
    _call("hga_tier_plan", ctypes.byref(cfg), group_idx, used_groups, n_used, compact_idx, workspace, stream)


def tier_gather(cfg, k_hist, v_hist, used_groups, n_used, k_cache, v_cache, stream=0) -> None:
    _call("hga_tier_gather", ctypes.byref(cfg), k_hist, v_hist, used_groups, n_used, k_cache, v_cache, stream)


def read_status(workspace, stream=0) -> int:
    out = ctypes.c_int32(0)
    _call("hga_read_status", workspace, stream, ctypes.byref(out))
    return int(out.value)
