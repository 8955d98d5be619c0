"""The seeded workload generator: determinism, AR(1) statistics and the
frame roles of each workload geometry."""
import math

import pytest
import torch

from ispa_synth import C0, C1, C2, C3, C4, ar1_stream, layer_streams, projection, scaled


def test_streams_are_deterministic_and_layer_specific():
    a = ar1_stream(3, 8, 16, 0.9, seed=0, layer=0, tensor="K")
    b = ar1_stream(3, 8, 16, 0.9, seed=0, layer=0, tensor="K")
    c = ar1_stream(3, 8, 16, 0.9, seed=0, layer=1, tensor="K")
    d = ar1_stream(3, 8, 16, 0.9, seed=0, layer=0, tensor="V")
    assert a.dtype == torch.bfloat16
    assert torch.equal(a, b) and not torch.equal(a, c) and not torch.equal(a, d)


def test_ar1_statistics():
    x = ar1_stream(12, 256, 256, 0.9, seed=3, layer=0, tensor="Q").float()
    assert abs(x.std().item() - 1.0) < 0.02
    r = (x[1:] * x[:-1]).mean() / (x[:-1] * x[:-1]).mean()
    assert abs(r.item() - 0.9) < 0.01


def test_projection_scale():
    w = projection(512, 0, 0)
    assert w.dtype == torch.float32
    assert abs(w.std().item() * math.sqrt(512) - 1.0) < 0.02


def test_chunk_geometry_13b():
    # 1.3B single chunk: sink 1560, local 4680, history 14040 (9 frames)
    assert C1.chunk_frames_of(0) == [10, 11, 12]
    assert len(C1.history_frames_of(0)) * C1.tokens_per_frame == 14040
    assert C1.sink_tokens == 1560 and C1.chunk_tokens == 4680 and C1.d == 1536
    # full warmup: history grows 0, 3, 6, 9 frames; 18720 rows per layer
    assert [len(C2.history_frames_of(c)) for c in range(4)] == [0, 3, 6, 9]
    assert C2.warmup_rows == 18720 and C3.warmup_rows == 18720 and C3.d == 5120
    # the last warmup chunk of the full warmup is the single-chunk workload
    assert C2.chunk_frames_of(3) == C1.chunk_frames_of(0)
    assert C2.history_frames_of(3) == C1.history_frames_of(0)
    # streaming ends with 60 frames (93600 tokens) of history
    last = C4.n_chunks + C4.stream_chunks - 1
    assert len(C4.history_frames_of(last)) * C4.tokens_per_frame == 93600


def test_chunk_geometry_tiny():
    assert [C0.chunk_frames_of(c)[0] for c in range(8)] == list(range(5, 13))
    assert all(len(C0.history_frames_of(c)) == 4 for c in range(8))
    st = layer_streams(C0, 0)
    ch = st.chunk(0)
    assert ch["q"].shape == (64, 2, 64) and ch["k_sink"].shape == (16, 2, 64)
    assert ch["k_hist"].shape == (256, 2, 64) and ch["k_loc"].shape == (64, 2, 64)
    # local keys and queries come from the same frame of their own streams
    assert torch.equal(ch["k_loc"], st.k[5].reshape(64, 2, 64))
    assert torch.equal(ch["k_hist"], st.k[1:5].reshape(256, 2, 64))


def test_empty_history_chunk():
    cfg = scaled(C2, tokens_per_frame=8, heads=1, head_dim=16, layers=1)
    st = layer_streams(cfg, 0)
    ch = st.chunk(0)
    assert ch["k_hist"].shape == (0, 1, 16) and ch["q"].shape == (24, 1, 16)


def test_stacked_streams_are_the_per_layer_streams():
    """All layers' streams in one tensor per Q, K, V: each layer's stream is a
    view of it with the draws of layer_streams, and stacked_chunk(c) holds
    chunk c of every layer as [L, tokens, heads, head_dim] views whose layers
    are contiguous and one stream apart."""
    import dataclasses
    from ispa_synth import stacked_chunk, stacked_layer_streams
    cfg = dataclasses.replace(C0, layers=3)
    sts, (Q, K, V) = stacked_layer_streams(cfg, [0, 1, 2], seed=5)
    for i, st in enumerate(sts):
        ref = layer_streams(cfg, i, seed=5)
        assert torch.equal(st.q, ref.q) and torch.equal(st.k, ref.k) and torch.equal(st.v, ref.v)
        assert st.k.data_ptr() == K[i].data_ptr()
    for c in range(cfg.n_chunks):
        sc = stacked_chunk(cfg, (Q, K, V), c)
        for key, x in sc.items():
            assert x.shape[0] == 3
            for l in range(3):
                assert torch.equal(x[l], sts[l].chunk(c)[key]), (c, key)
                assert x[l].is_contiguous()
            if x.shape[1]:
                assert x.untyped_storage().data_ptr() in {t.untyped_storage().data_ptr()
                                                          for t in (Q, K, V)}
                assert x.stride(0) == Q[0].numel()


def test_warmup_layer_groups():
    """The warmup driver's groups of layers per attention launch cover every
    layer once, in order, the last group short (host logic; CPU buffers)."""
    from kv_cache_absorption_b200.warmup import LayerWarmup
    mk = lambda L, g: LayerWarmup(2, 64, 64, 16, 64, 256, n_layers=L, device="cpu", n_slots=2,
                                  group=g)
    assert mk(30, 10).layer_groups() == [(0, 10), (10, 10), (20, 10)]
    assert mk(5, 2).layer_groups() == [(0, 2), (2, 2), (4, 1)]
    assert mk(3, 8).layer_groups() == [(0, 3)]                # a group no larger than the layers
    r = mk(4, 1)
    assert r.group == 1 and r.group_slots == []
    with pytest.raises(ValueError):                           # built without groups
        r.layers_chunks_stacked([])
