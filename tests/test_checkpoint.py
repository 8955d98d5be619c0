"""The transition-state checkpoint (kv_cache_absorption_b200/checkpoint.py):
a round trip through a file keeps every tensor bit for bit, and a file of
another format or geometry is refused. CPU only."""
import pytest
import torch

from kv_cache_absorption_b200.checkpoint import FORMAT, load_transition, save_transition


def state(L=4, d=128, sink=16, H=2, hd=64, with_hist=True):
    g = torch.Generator().manual_seed(7)
    r = lambda *s: torch.randn(*s, generator=g)
    sel = torch.tensor([1, 0, 1, 0], dtype=torch.uint8)[:L]
    kw = dict(dW=r(L, d, d), lam=r(L).abs(), err=r(L, 2).double().abs(),
              perm=torch.randperm(L, generator=g).int(), selected=sel,
              sink_k=[r(sink, H, hd).bfloat16() for _ in range(L)],
              sink_v=[r(sink, H, hd).bfloat16() for _ in range(L)])
    if with_hist:
        kw["hist_k"] = [None if sel[l] else r(40 + l, H, hd).bfloat16() for l in range(L)]
        kw["hist_v"] = [None if sel[l] else r(40 + l, H, hd).bfloat16() for l in range(L)]
    return kw


@pytest.mark.parametrize("with_hist", [True, False])
def test_round_trip_is_exact(tmp_path, with_hist):
    kw = state(with_hist=with_hist)
    p = str(tmp_path / "t.pt")
    save_transition(p, **kw, meta={"workload": "tiny"})
    got = load_transition(p, device="cpu", d=128, layers=4)
    assert got["format"] == FORMAT and got["meta"] == {"workload": "tiny"}
    for key, name in (("dW", "dW"), ("lam", "lambda"), ("err", "err"), ("perm", "perm")):
        assert torch.equal(got[name], kw[key].to(got[name].dtype)), key
    assert got["selected"].tolist() == kw["selected"].bool().tolist()
    for l in range(4):
        assert torch.equal(got["sink_k"][l], kw["sink_k"][l])
        assert torch.equal(got["sink_v"][l], kw["sink_v"][l])
        if with_hist:
            if kw["hist_k"][l] is None:
                assert got["hist_k"][l] is None
            else:
                assert torch.equal(got["hist_k"][l], kw["hist_k"][l])
                assert torch.equal(got["hist_v"][l], kw["hist_v"][l])
    assert ("hist_k" in got) == with_hist


def test_refuses_other_files_and_geometries(tmp_path):
    p = str(tmp_path / "t.pt")
    save_transition(p, **state())
    with pytest.raises(ValueError):
        load_transition(p, device="cpu", d=256)
    with pytest.raises(ValueError):
        load_transition(p, device="cpu", layers=5)
    q = str(tmp_path / "other.pt")
    torch.save({"format": "something else"}, q)
    with pytest.raises(ValueError):
        load_transition(q, device="cpu")


def test_rejects_inconsistent_states(tmp_path):
    p = str(tmp_path / "t.pt")
    kw = state()
    with pytest.raises(ValueError):
        save_transition(p, **dict(kw, lam=kw["lam"][:3]))
    bad = state()
    bad["hist_k"][0] = torch.zeros(3, 2, 64, dtype=torch.bfloat16)   # layer 0 is an L-Layer
    with pytest.raises(ValueError):
        save_transition(p, **bad)
