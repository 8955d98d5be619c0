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


def test_kv_cache_append_layout_and_bytes():
    import torch
    from kv_cache_absorption_b200.streaming import KVCache
    H, hd, sink, chunk = 2, 4, 3, 5
    tok = lambda n, base: (torch.arange(n * H * hd, dtype=torch.float32).reshape(n, H, hd) + base
                           ).to(torch.bfloat16)
    max_hist = 4 + 2 * chunk                 # the preloaded frames and two chunks
    f = KVCache(H, hd, sink, chunk, max_hist=max_hist, full=True, device="cpu")
    l = KVCache(H, hd, sink, chunk, max_hist=max_hist, full=False, device="cpu")
    assert f.nbytes == (sink + chunk + max_hist) * H * hd * 2 * 2 and l.nbytes == (sink + chunk) * H * hd * 2 * 2
    for c in (f, l):
        c.set_sink(tok(sink, 1000), tok(sink, 2000))
    f.set_history(tok(4, 0), tok(4, 100))
    for i in range(3):                       # three chunks of 5 tokens; the F-Layer keeps them all
        k, v = tok(chunk, 10 * (i + 1)), tok(chunk, 500 + i)
        f.append(k, v)
        l.append(k, v)
        cf, cl = f.chunk_inputs(None), l.chunk_inputs(None)
        assert torch.equal(cf["k_loc"], k) and torch.equal(cl["k_loc"], k)
        assert torch.equal(cf["v_loc"], v) and torch.equal(cl["v_loc"], v)
        assert cf["k_hist"].shape[0] == 4 + chunk * i and cl["k_hist"].shape[0] == 0
        assert torch.equal(cf["k_sink"], tok(sink, 1000)) and torch.equal(cl["v_sink"], tok(sink, 2000))
    # history = preloaded frames, then the first two chunks, in order
    assert torch.equal(cf["k_hist"][:4], tok(4, 0))
    assert torch.equal(cf["k_hist"][4:9], tok(chunk, 10)) and torch.equal(cf["k_hist"][9:], tok(chunk, 20))
    with pytest.raises(ValueError):
        f.append(tok(chunk, 0), tok(chunk, 0))       # a fourth chunk: 19 history + 5 > 14 + 5
    with pytest.raises(ValueError):
        l.set_history(tok(1, 0), tok(1, 0))
    f.rewind()                                       # the transition state again
    f.append(tok(chunk, 10), tok(chunk, 500))
    cf = f.chunk_inputs(None)
    assert cf["k_hist"].shape[0] == 4 and torch.equal(cf["k_loc"], tok(chunk, 10))
