"""Host logic of the segment-wise driver, no GPU: the configuration a segment is run with while the
history is still short.  Budgets are clamped to what the history holds (k_c' = min(k_c, routable
chunks), k_g' = min(k_g, 8 k_c')), the sink keeps at least one chunk routable, the first segment
routes nothing; every configuration produced must pass the C library's own validation."""
import pytest

from hierarchical_kv_routing_tok_b200 import _capi as C
from hierarchical_kv_routing_tok_b200 import build as B
from hierarchical_kv_routing_tok_b200.segment import HGAHistory


@pytest.fixture(scope="module")
def lib():
    B.build()
    return C.load()


def _history(capacity, n_sink):
    # K/V and summary buffers on the host: only the configuration logic is exercised here
    return HGAHistory(1, 8, 2, capacity, device="cpu", n_sink_tokens=n_sink)


@pytest.mark.parametrize("n_sink", [0, 64, 192])
@pytest.mark.parametrize("top_chunks,top_groups", [(1, 1), (4, 16), (16, 64), (16, 128)])
def test_clamped_budgets_are_valid_configurations(lib, n_sink, top_chunks, top_groups):
    hist = _history(64 * 40, n_sink)
    for length in range(0, 64 * 40 + 1, 64):
        hist.length = length
        cfg = hist.config(128, top_chunks, top_groups)
        assert cfg.hist_len == length and cfg.hist_capacity == 64 * 40
        if length == 0:
            assert (cfg.top_chunks, cfg.top_groups, cfg.n_sink_tokens) == (0, 0, 0)
        else:
            ns = cfg.n_sink_tokens
            routable = length // 64 - ns // 64
            assert ns % 64 == 0 and ns <= n_sink and routable >= 1
            assert ns == min(n_sink, length - 64)
            assert cfg.top_chunks == min(top_chunks, routable)
            assert cfg.top_groups == min(top_groups, 8 * cfg.top_chunks)
        assert C.workspace_size(cfg) > 0          # accepted by the library's validation


def test_unclamped_once_the_history_is_long_enough(lib):
    hist = _history(64 * 300, 64)
    hist.length = 64 * 300
    cfg = hist.config(2048, 16, 64)
    assert (cfg.top_chunks, cfg.top_groups, cfg.n_sink_tokens, cfg.seg_len) == (16, 64, 64, 2048)


def test_capacity_must_be_whole_chunks():
    with pytest.raises(ValueError):
        HGAHistory(1, 8, 2, 100, device="cpu")
