"""Host-side logic of the post-transition streaming (CPU only)."""
import pytest

from kv_cache_absorption_b200.streaming import kv_cache_bytes


def test_kv_cache_accounting():
    """KV bytes at the last streaming chunk of the 1.3B workload: 30 F-Layers
    hold 18.40 GB; 15 F + 15 L hold 9.78 GB (-46.9%)."""
    from kv_cache_absorption_b200.streaming import kv_cache_bytes
    all_f = kv_cache_bytes(30, 0, 1560, 93600, 4680, 1536)
    ispa_b = kv_cache_bytes(15, 15, 1560, 93600, 4680, 1536)
    assert all_f == 30 * 99840 * 1536 * 2 * 2
    assert abs(all_f / 1e9 - 18.40) < 0.01 and abs(ispa_b / 1e9 - 9.78) < 0.01
    assert abs(1 - ispa_b / all_f - 0.469) < 0.001


def test_kv_cache_bytes_counts_layers_and_tokens():
    # one F-Layer: (sink + history + chunk) tokens x d x (K, V) x bf16
    assert kv_cache_bytes(1, 0, 3, 5, 7, 4) == 15 * 4 * 2 * 2
    # one L-Layer drops the history
    assert kv_cache_bytes(0, 1, 3, 5, 7, 4) == 10 * 4 * 2 * 2
    assert kv_cache_bytes(2, 3, 3, 5, 7, 4, bytes_per_elem=1) == (2 * 15 + 3 * 10) * 4 * 2
