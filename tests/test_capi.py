"""The C-ABI library: it loads, exports every symbol include/hga.h declares, its config struct
matches the C layout, and argument validation rejects bad calls before anything is launched
(these calls need no GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from hierarchical_kv_routing_tok_b200 import _capi as C
from hierarchical_kv_routing_tok_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hga.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return C.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"HGA_API\s+[\w\s\*]*?\b(hga_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 8
    assert sorted(C.EXPORTS) == names
    out = subprocess.run(["nm", "-D", "--defined-only", C.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (hga_\w+)", out))
    assert set(names) <= exported
    for n in names:
        assert hasattr(lib, n)


def test_version_and_strerror(lib):
    hdr = open(HEADER).read()
    assert C.version() == int(re.search(r"#define HGA_VERSION (\d+)", hdr).group(1))
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert C.strerror(code) and C.strerror(code) != "unknown status"
    assert C.strerror(12345) == "unknown status"


def test_config_struct_layout_matches_c(tmp_path):
    src = tmp_path / "layout.c"
    fields = [n for n, _ in C.HGAConfig._fields_]
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "hga.h"\nint main(void){\n'
                   '  printf("%zu\\n", sizeof(hga_config_t));\n'
                   + "".join(f'  printf("%zu\\n", offsetof(hga_config_t, {f}));\n' for f in fields)
                   + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    vals = [int(v) for v in subprocess.check_output([str(exe)], text=True).split()]
    assert vals[0] == ctypes.sizeof(C.HGAConfig)
    assert vals[1:] == [getattr(C.HGAConfig, f).offset for f in fields]


def cfg(**kw):
    base = dict(B=1, Hq=32, Hkv=8, hist_len=14336, seg_len=2048, top_chunks=16, top_groups=64)
    base.update(kw)
    return C.make_config(**base)


def _expected_ws(B, Hq, Hkv, S, bf16=True, sms=148, hist=14336, sink=0):
    """Status word, delta rows, then one region shared by (a) the dK/dV exchange area (bf16
    tensor-core path, fewer (batch, KV head, 128-key tile) units than SMs: the kernel pairs CTAs;
    2 x 64 KB per unit) and (b) the scratch of the three-launch routing (at least 128 routable
    chunks: a float32 block query and a row of chunk-score keys, padded to 4, per (batch, KV head,
    block)); the region is the larger of the two."""
    r256 = lambda x: (x + 255) // 256 * 256
    delta = B * Hq * S * 4
    units = B * Hkv * ((S + 127) // 128)
    paired = bf16 and (Hq // Hkv) % 2 == 0 and units < sms
    xchg = units * 2 * 64 * 256 * 4 if paired else 0
    nblk, nc1 = S // 64, hist // 64 - sink // 64
    blocks = B * Hkv * nblk
    split = nc1 >= 512 and (nblk + 31) // 32 * 32 * 512 <= 200 * 1024
    route = blocks * 128 * 4 + blocks * ((nc1 + 3) // 4 * 4) * 4 if split else 0
    return 256 + r256(delta) + max(xchg, route)


def test_workspace_size(lib):
    assert C.workspace_size(cfg()) == _expected_ws(1, 32, 8, 2048)
    assert C.workspace_size(cfg(B=3, Hq=4, Hkv=1, seg_len=64)) == _expected_ws(3, 4, 1, 64)
    assert C.workspace_size(cfg(B=3, Hq=4, Hkv=1, seg_len=64)) % 256 == 0
    # float32, odd G and many units: no exchange area
    assert C.workspace_size(cfg(dtype=C.HGA_F32)) == 256 + 1 * 32 * 2048 * 4
    # a long history routes in three launches and needs routing scratch (a shorter one does not)
    assert C.workspace_size(cfg(dtype=C.HGA_F32, hist_len=64 * 511)) == 256 + 1 * 32 * 2048 * 4
    assert C.workspace_size(cfg(dtype=C.HGA_F32, hist_len=64 * 512)) == (
        256 + 1 * 32 * 2048 * 4 + 8 * 32 * (128 + 512) * 4)
    assert C.workspace_size(cfg(dtype=C.HGA_F32, hist_len=64 * 515, n_sink_tokens=64)) == _expected_ws(
        1, 32, 8, 2048, bf16=False, hist=64 * 515, sink=64)
    assert C.workspace_size(cfg(hist_len=64 * 2016)) == _expected_ws(1, 32, 8, 2048, hist=64 * 2016)
    assert C.workspace_size(cfg(Hq=24)) == _expected_ws(1, 24, 8, 2048, sms=0)
    assert C.workspace_size(cfg(B=4)) == _expected_ws(4, 32, 8, 2048, sms=0)


def test_route_launches(lib):
    """Three launches with a workspace and at least 512 routable chunks, one without a workspace or
    for a shorter history (the 16K layer has 224 chunks), none without a history."""
    long = dict(hist_len=64 * 2016, top_chunks=32, top_groups=128)
    assert C.route_launches(cfg()) == 1
    assert C.route_launches(cfg(**long)) == 3
    assert C.route_launches(cfg(**long), with_workspace=False) == 1
    assert C.route_launches(cfg(hist_len=64 * 511)) == 1
    assert C.route_launches(cfg(hist_len=64 * 512)) == 3
    assert C.route_launches(cfg(hist_len=64 * 512, n_sink_tokens=64)) == 1   # 511 routable
    # the 400 block queries of a 25,600-token segment would need 208 KB of shared memory
    assert C.route_launches(cfg(seg_len=64 * 400, **long)) == 1
    assert C.route_launches(cfg(seg_len=64 * 384, **long)) == 3
    assert C.route_launches(cfg(hist_len=0, top_chunks=0, top_groups=0)) == 0   # first segment: no history


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=30), C.HGA_ERR_ARG),                     # Hq not a multiple of Hkv
    (dict(B=0), C.HGA_ERR_ARG),
    (dict(D=64), C.HGA_ERR_UNSUPPORTED),
    (dict(chunk=32), C.HGA_ERR_UNSUPPORTED),
    (dict(group=4), C.HGA_ERR_UNSUPPORTED),
    (dict(qblock=128), C.HGA_ERR_UNSUPPORTED),
    (dict(n_sink_tokens=4), C.HGA_ERR_ARG),           # sink not a whole number of chunks
    (dict(n_sink_tokens=-64), C.HGA_ERR_ARG),
    (dict(n_sink_tokens=14336), C.HGA_ERR_ARG),       # sink covers the whole history
    (dict(n_sink_tokens=13312, top_chunks=17), C.HGA_ERR_ARG),  # k_c > the 16 chunks left to route
    (dict(hist_len=14300), C.HGA_ERR_ARG),            # open chunk
    (dict(hist_len=0), C.HGA_ERR_ARG),
    (dict(seg_len=2000), C.HGA_ERR_ARG),
    (dict(top_chunks=0), C.HGA_ERR_ARG),
    (dict(top_chunks=225), C.HGA_ERR_ARG),            # more chunks than the history has
    (dict(top_groups=129), C.HGA_ERR_ARG),            # more groups than the chosen chunks hold
    (dict(top_groups=0), C.HGA_ERR_ARG),
    (dict(dtype=7), C.HGA_ERR_ARG),
    (dict(softmax_scale=-1.0), C.HGA_ERR_ARG),
    (dict(softmax_scale=float("nan")), C.HGA_ERR_ARG),
    (dict(wait_limit_ns=-1), C.HGA_ERR_ARG),          # the bounded-wait limit: 0 (2 s) or positive
    (dict(hist_len=64 * 40000, top_chunks=16), C.HGA_ERR_UNSUPPORTED),
])
def test_config_validation(lib, kw, code):
    with pytest.raises(C.HGAError) as e:
        C.workspace_size(cfg(**kw))
    assert e.value.code == code


def test_sink_window_config_accepted(lib):
    assert C.workspace_size(cfg(n_sink_tokens=64)) == _expected_ws(1, 32, 8, 2048)
    assert C.workspace_size(cfg(n_sink_tokens=13312, top_chunks=16)) == _expected_ws(1, 32, 8, 2048)


def test_tier_cache_config(lib):
    """The compact history cache holds every group a step can route to, in whole chunks."""
    c = C.tier_cache_config(cfg())                                  # 32 blocks x 64 > 1792 groups
    assert (c.hist_len, c.top_chunks, c.top_groups) == (14336, 8, 64)
    c = C.tier_cache_config(cfg(hist_len=129024, top_chunks=32, top_groups=128))
    assert c.hist_len == 32 * 128 * 8 and c.top_chunks == 16     # 4096 groups of 16128
    c = C.tier_cache_config(cfg(seg_len=64, top_chunks=4, top_groups=20))
    assert c.hist_len == 24 * 8                                    # 20 groups -> 3 whole chunks
    c = C.tier_cache_config(cfg(seg_len=128, top_chunks=4, top_groups=20, n_sink_tokens=128))
    assert c.hist_len == (16 + 40) * 8 and c.n_sink_tokens == 128   # sink + 2 blocks x 20
    c = C.tier_cache_config(cfg(seg_len=64, top_chunks=2, top_groups=1))
    assert c.hist_len == 64 and c.top_chunks == 1                  # at least one chunk
    assert C.workspace_size(c) > 0                                   # a valid configuration


def test_entry_points_reject_bad_pointers_before_launch(lib):
    c = cfg()
    ok, odd = 1 << 20, (1 << 20) + 8             # never dereferenced: validation fails first
    calls = {
        "summaries": lambda p: C.build_summaries(c, p[0], p[1], p[2], ok),
        "route": lambda p: C.route(c, p[0], p[1], p[2], p[3], p[4], ok),
        "fwd": lambda p: C.attn_fwd(c, p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7], p[8]),
        "bwd": lambda p: C.attn_bwd(c, *p[:13]),
    }
    for name, call in calls.items():
        for i in range(3):
            ptrs = [ok] * 13
            ptrs[i] = None
            with pytest.raises(C.HGAError) as e:
                call(ptrs)
            assert e.value.code == C.HGA_ERR_ARG, name
            ptrs[i] = odd
            with pytest.raises(C.HGAError) as e:
                call(ptrs)
            assert e.value.code == C.HGA_ERR_ALIGN, name
    with pytest.raises(C.HGAError) as e:
        C.attn_fwd(c, ok, ok, ok, ok, ok, ok, ok, ok, None)
    assert e.value.code == C.HGA_ERR_WORKSPACE
    with pytest.raises(C.HGAError) as e:
        C.attn_bwd(c, *([ok] * 12), None)
    assert e.value.code == C.HGA_ERR_WORKSPACE
    bad = cfg(top_chunks=300)
    with pytest.raises(C.HGAError) as e:
        C.route(bad, ok, ok, ok, ok, ok, ok)
    assert e.value.code == C.HGA_ERR_ARG


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """No CPU or library fallback: without libhga.so every call raises."""
    monkeypatch.setattr(C, "LIB_PATH", os.path.join(tmp_path, "libhga.so"))
    monkeypatch.setattr(C, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        C.load()
    with pytest.raises(RuntimeError, match="missing"):
        C.workspace_size(cfg())


def test_group_cache_entry_points_validate_before_launch(lib):
    """The group-summary cache calls reject a slot count outside [1, min(4096, history chunks)] and
    missing pointers or workspace before anything is launched."""
    c = cfg()                                       # 224 history chunks
    ok = 1 << 20
    for cap in (0, -1, 225, 5000):
        with pytest.raises(C.HGAError) as e:
            C.gcache_plan(c, cap, ok, ok, ok, ok, 0, ok, ok, ok, ok)
        assert e.value.code == C.HGA_ERR_ARG, cap
        with pytest.raises(C.HGAError) as e:
            C.route_groups_cached(c, ok, ok, ok, cap, ok, ok, ok)
        assert e.value.code == C.HGA_ERR_ARG, cap
    with pytest.raises(C.HGAError) as e:
        C.gcache_plan(c, 16, ok, ok, ok, ok, 0, ok, ok, ok, None)
    assert e.value.code == C.HGA_ERR_WORKSPACE
    with pytest.raises(C.HGAError) as e:
        C.route_groups_cached(c, ok, ok, ok, 16, ok, ok, None)
    assert e.value.code == C.HGA_ERR_WORKSPACE
    with pytest.raises(C.HGAError) as e:
        C.route_chunks(c, ok, ok, ok, None, None)      # no block-query buffer
    assert e.value.code == C.HGA_ERR_ARG
    with pytest.raises(C.HGAError) as e:
        C.gcache_fetch(c, 16, ok, None, ok, ok, ok)
    assert e.value.code == C.HGA_ERR_ARG
