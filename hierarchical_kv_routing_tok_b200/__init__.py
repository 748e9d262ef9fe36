"""Routed Hierarchical Global Attention (HGA) for B200 (sm_100a).

The hot path of one attention layer over a detached history plus an active
segment ("Long-Context Fine-Tuning with Limited VRAM"): key summaries, two-level
top-k routing, and routed + causal-local attention forward and backward, all in
the CUDA library ``libhga.so`` behind the C ABI of ``include/hga.h``; with the
history K/V either in device memory (``LayerStep``) or in pinned host memory
(``TieredLayerStep``, optionally with the group summaries in host memory behind a device cache,
``GroupSummaryCache``).
"""
from . import _capi
from ._capi import HGAConfig, HGAError, load
from .api import (GroupSummaryCache, LayerStep, TieredLayerStep, attn_bwd, attn_fwd, build_summaries, hga_attention,
                  make_config, new_workspace, read_status, route)
from .segment import HGAHistory, segment_attention

__all__ = ["GroupSummaryCache", "HGAConfig", "HGAError", "HGAHistory", "LayerStep", "TieredLayerStep", "attn_bwd", "attn_fwd",
           "build_summaries", "hga_attention", "load", "make_config", "new_workspace", "read_status", "route",
           "segment_attention", "_capi"]
