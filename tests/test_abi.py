"""The C-ABI library: it builds, loads without a GPU, exports exactly what
include/ispa.h declares, and rejects bad arguments on the host before any
device work. CPU only."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ispa.h")


@pytest.fixture(scope="module")
def ispa():
    from kv_cache_absorption_b200 import build
    build.build()
    from kv_cache_absorption_b200 import ispa as m
    m._load()
    return m


def declared():
    text = open(HEADER).read()
    return set(re.findall(r"^ISPA_API [\w\s\*]+?\b(ispa_\w+)\(", text, flags=re.M))


def exported():
    out = subprocess.run(["nm", "-D", "--defined-only", os.path.join(
        ROOT, "kv_cache_absorption_b200", "libispa.so")], capture_output=True, text=True).stdout
    return {line.split()[-1] for line in out.splitlines() if " T " in line}


def test_exports_match_header(ispa):
    names = declared()
    assert len(names) == 29
    assert names == exported()
    assert names == set(ispa.EXPORTED)
    lib = ctypes.CDLL(ispa.LIB_PATH)
    for n in names:
        assert getattr(lib, n) is not None


def test_version_and_status_strings(ispa):
    assert ispa.ispa_version() == 100
    assert ispa.ispa_kernel_launches() == 0   # nothing launched in a CPU-only process
    for code in (0, -1, -2, -3, -4, -5, 1, 2, 4, 8):
        assert ispa.ispa_status_string(code) != "unknown status"
    assert ispa.ispa_status_string(12345) == "unknown status"


def test_workspace_sizes(ispa):
    def r256(x):
        return (x + 255) // 256 * 256
    nq, H, hd = 4680, 12, 128
    out = r256(nq * H * hd * 4)
    lse = r256(H * nq * 4)
    cnt = r256(H * 19 * 4)                    # 19 query-tile pairs per head
    loc_tiles = 13 + 37                       # 1560 sink + 4680 local keys

    def bound(hist):                          # most key ranges any candidate plan uses
        t = -(-hist // 128)
        if t == 0:
            return 4
        base = 1 if t <= 3 * loc_tiles else min(64, -(-t // (2 * loc_tiles)))
        return 4 + min(base + 2, t)
    # one completion counter per (head, pair), an LSE block and an fp32
    # output per key range, for the most ranges any candidate plan may use
    sizes = []
    for hist in (0, 4680, 9360, 14040, 18720, 93600):
        want = cnt + bound(hist) * (lse + out) + 256
        assert ispa.ispa_dual_attention_workspace_size(nq, 1560, 4680, hist, H, hd) == want
        assert ispa.ispa_full_attention_workspace_size(nq, 1560, 4680, hist, H, hd) == want
        units, ls, hs = ispa.ispa_attention_units(nq, 1560, 4680, hist, H)
        assert ls + hs <= bound(hist)
        sizes.append(want)
    # non-decreasing in the history length: sized for the longest, fits all
    assert sizes == sorted(sizes)
    # one key tile and no history: one unit per (head, pair), no scratch
    assert ispa.ispa_attention_units(10, 1, 0, 0, 1) == (1, 1, 0)
    assert ispa.ispa_dual_attention_workspace_size(10, 1, 0, 0, 1, 64) == 256
    assert ispa.ispa_dual_attention_workspace_size(1, -1, 1, 1, 1, 64) == 0
    n = 1536
    assert ispa.ispa_absorb_workspace_size(n) >= 2 * n * n * 4
    assert ispa.ispa_absorb_workspace_size(0) == 0
    assert ispa.ispa_layer_error_workspace_size(128) >= 40


def test_attention_plan(ispa):
    """The unit decomposition: key ranges cover each branch without empty
    ranges, long histories are cut (split-KV), the counts can be forced, and
    the plan follows the shape (host only)."""
    nq, H = 4680, 12
    per = H * 19
    for hist in (0, 4680, 9360, 14040, 93600):
        units, ls, hs = ispa.ispa_attention_units(nq, 1560, 4680, hist, H)
        assert units == per * (ls + hs)
        assert 1 <= ls <= 4 and ls <= 50           # 13 sink + 37 local key tiles
        assert (hs == 0) == (hist == 0)
    assert ispa.ispa_attention_units(nq, 1560, 4680, 93600, H)[2] >= 8   # 732 history tiles
    # a branch of one key tile cannot be cut
    assert ispa.ispa_attention_units(64, 0, 64, 0, 2)[1:] == (1, 0)
    assert ispa.ispa_attention_units(1, 0, 0, 0, 1)[0] == 0               # no keys: invalid
    try:
        ispa.ispa_attention_set_splits(2, 3)
        assert ispa.ispa_attention_units(nq, 1560, 4680, 14040, H) == (per * 5, 2, 3)
        assert ispa.ispa_attention_units(nq, 1560, 4680, 0, H) == (per * 2, 2, 0)
        # more ranges than tiles: one range per tile
        assert ispa.ispa_attention_units(64, 16, 64, 128, 2)[1:] == (2, 1)
        # joint units (hist_splits -1) need A_loc as an output, which this
        # plan query does not assume: one history range then
        ispa.ispa_attention_set_splits(1, -1)
        assert ispa.ispa_attention_units(nq, 1560, 4680, 14040, H) == (per * 2, 1, 1)
    finally:
        ispa.ispa_attention_set_splits(0, 0)
    with pytest.raises(ispa.IspaError):
        ispa.ispa_attention_set_splits(-1, 0)
    with pytest.raises(ispa.IspaError):
        ispa.ispa_attention_set_splits(1, -2)


def _kv(ispa, n, addr=0x10000):
    return ispa.IspaKV(addr, addr, n)


def _dual(ispa, q=0x1000, nq=64, heads=2, hd=64, sink=16, loc=64, hist=256, scale=0.125,
          a_loc=0x2000, d_out=0x3000, ws=0x100000, ws_bytes=1 << 30, status=0x4000):
    lib = ispa._load()
    return lib.ispa_dual_attention(q, nq, heads, hd, _kv(ispa, sink), _kv(ispa, loc),
                                   _kv(ispa, hist), scale, a_loc, d_out, None, None, None, None,
                                   ws, ws_bytes, status, None)


def test_dual_attention_host_checks(ispa):
    assert _dual(ispa, q=0) == ispa.ISPA_ERR_ARG
    assert _dual(ispa, a_loc=0) == ispa.ISPA_ERR_ARG
    assert _dual(ispa, status=0) == ispa.ISPA_ERR_ARG
    assert _dual(ispa, nq=-1) == ispa.ISPA_ERR_ARG
    assert _dual(ispa, heads=0) == ispa.ISPA_ERR_ARG
    assert _dual(ispa, hd=96) == ispa.ISPA_ERR_UNSUPPORTED
    assert _dual(ispa, scale=0.0) == ispa.ISPA_ERR_ARG
    assert _dual(ispa, scale=float("nan")) == ispa.ISPA_ERR_ARG
    assert _dual(ispa, sink=0, loc=0) == ispa.ISPA_ERR_ARG
    assert _dual(ispa, hist=-5) == ispa.ISPA_ERR_ARG
    assert _dual(ispa, q=0x1004) == ispa.ISPA_ERR_UNSUPPORTED
    assert _dual(ispa, ws=0) == ispa.ISPA_ERR_WORKSPACE
    assert _dual(ispa, ws_bytes=100) == ispa.ISPA_ERR_WORKSPACE
    assert _dual(ispa, ws=0x100010) == ispa.ISPA_ERR_WORKSPACE
    # arguments that pass every host check then need an sm_100 device
    import torch
    rc = _dual(ispa)
    if not torch.cuda.is_available():
        assert rc in (ispa.ISPA_ERR_CUDA, ispa.ISPA_ERR_NO_DEVICE)


def _dual_layers(ispa, L=3, q=0x1000, qs=64 * 128, nq=64, heads=2, hd=64, sink=16, loc=64,
                 hist=256, kvs=None, outs=64 * 128, lses=2 * 64, a_loc=0x2000, d_out=0x3000,
                 ws=0x100000, ws_bytes=1 << 30, status=0x4000):
    lib = ispa._load()
    d = heads * hd
    kvs = kvs or {"sink": sink * d, "loc": loc * d, "hist": hist * d}
    kv = lambda n, s: ispa.IspaKVLayers(0x10000, 0x20000, n, s) if n else \
        ispa.IspaKVLayers(None, None, 0, 0)
    return lib.ispa_dual_attention_layers(
        L, q, qs, nq, heads, hd, kv(sink, kvs["sink"]), kv(loc, kvs["loc"]),
        kv(hist, kvs["hist"]), 0.125, a_loc, d_out, None, outs, None, None, None, lses, ws,
        ws_bytes, status, None)


def test_dual_attention_layers_host_checks(ispa):
    """The batched entry: layer counts and strides are checked before any
    device work (layers may not overlap, rows stay 16-byte aligned), and the
    workspace is one single-layer workspace per layer."""
    one = ispa.ispa_dual_attention_workspace_size(4680, 1560, 4680, 14040, 12, 128)
    assert ispa.ispa_dual_attention_layers_workspace_size(30, 4680, 1560, 4680, 14040, 12,
                                                          128) == 30 * one
    assert ispa.ispa_dual_attention_layers_workspace_size(0, 4680, 1560, 4680, 0, 12, 128) == 0
    assert _dual_layers(ispa, L=0) == ispa.ISPA_ERR_ARG
    assert _dual_layers(ispa, qs=64 * 128 - 8) == ispa.ISPA_ERR_ARG          # layers overlap
    assert _dual_layers(ispa, outs=64 * 128 - 8) == ispa.ISPA_ERR_ARG
    assert _dual_layers(ispa, lses=2 * 64 - 1) == ispa.ISPA_ERR_ARG
    assert _dual_layers(ispa, kvs={"sink": 16 * 128, "loc": 64 * 128 - 8,
                                   "hist": 256 * 128}) == ispa.ISPA_ERR_ARG
    assert _dual_layers(ispa, qs=64 * 128 + 4) == ispa.ISPA_ERR_UNSUPPORTED  # 16-byte rows
    assert _dual_layers(ispa, outs=64 * 128 + 4) == ispa.ISPA_ERR_UNSUPPORTED
    assert _dual_layers(ispa, ws_bytes=1000) == ispa.ISPA_ERR_WORKSPACE
    # one layer: strides are not used
    assert _dual_layers(ispa, L=1, qs=0, outs=0, lses=0, ws_bytes=100) == ispa.ISPA_ERR_WORKSPACE
    import torch
    rc = _dual_layers(ispa)
    if not torch.cuda.is_available():
        assert rc in (ispa.ISPA_ERR_CUDA, ispa.ISPA_ERR_NO_DEVICE)


def test_dual_attention_layers_binding_checks(ispa):
    """The binding of the several-layer call rejects inputs the C ABI could
    not address before any device work: tensors off the GPU, layers that are
    not contiguous, keys and values at different layer strides, outputs of
    another shape. CPU tensors are enough to reach these checks."""
    import torch
    L, nq, H, hd = 2, 64, 2, 64
    bf = lambda *shape: torch.zeros(*shape, dtype=torch.bfloat16)
    q = bf(L, nq, H, hd)
    with pytest.raises(ValueError):                       # [L, nq, H, hd] expected
        ispa.ispa_dual_attention_layers(bf(nq, H, hd), bf(L, 16, H, hd), bf(L, 16, H, hd),
                                        bf(L, nq, H, hd), bf(L, nq, H, hd))
    with pytest.raises(ValueError):                       # q's layers not contiguous
        ispa.ispa_dual_attention_layers(q.transpose(1, 2), bf(L, 16, H, hd), bf(L, 16, H, hd),
                                        bf(L, nq, H, hd), bf(L, nq, H, hd))
    with pytest.raises(ValueError):                       # keys on the host
        ispa._kv_layers(bf(L, 16, H, hd), bf(L, 16, H, hd), L, H, hd, "sink")
    assert ispa._kv_layers(None, None, L, H, hd, "history").len == 0
    assert ispa._kv_layers(bf(L, 0, H, hd), bf(L, 0, H, hd), L, H, hd, "history").len == 0


def test_other_entry_points_host_checks(ispa):
    lib = ispa._load()
    P = 0x1000
    assert lib.ispa_gram_accumulate(P, P, 100, 100, P, 0, 1, P, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert lib.ispa_gram_accumulate(P, P, -1, 128, P, 0, 1, P, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_gram_accumulate(None, P, 10, 128, P, 0, 1, P, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_gram_accumulate(P, P, 10, 128, None, 0, 1, P, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_gram_accumulate(P, P, 10, 128, P, 0, 1, None, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_absorb_solve(P, P, 128, float("nan"), P, P, None, P, 1 << 30, P, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_absorb_solve(P, P, 100, 0.0, P, P, None, P, 1 << 30, P, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert lib.ispa_absorb_solve(P, P, 128, 0.0, P, P, None, P, 16, P, None) == ispa.ISPA_ERR_WORKSPACE
    assert lib.ispa_layer_error(P, P, P, P, None, 128, P, P, 256, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_layer_error(P, P, P, P, P, 128, P, P, 8, None) == ispa.ISPA_ERR_WORKSPACE
    dd = 128 * 128
    assert lib.ispa_weight_gram_batched(2, P, dd, 100, P, dd, P, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert lib.ispa_weight_gram_batched(2, P, dd - 4, 128, P, dd, P, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_weight_gram_batched(2, P, dd, 128, P, dd + 2, P, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_weight_gram_batched(0, P, dd, 128, P, dd, P, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_weight_gram_batched(1, P + 4, dd, 128, P, dd, P, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert lib.ispa_layer_error_wwt_batched(2, P, 4 * dd, P, dd, P, dd, P, dd, P, 128, P, P, 256,
                                            None) == ispa.ISPA_ERR_WORKSPACE
    assert lib.ispa_layer_error_wwt_batched(2, P, dd, P, dd, P, dd, P, dd, P, 128, P, P, 512,
                                            None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_layer_error_wwt_batched(1, P, 4 * dd, None, dd, P, dd, P, dd, P, 128, P, P, 256,
                                            None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_project(P, 10, 100, P, P, 0, P, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert lib.ispa_project(P, -1, 128, P, P, 0, P, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_project(None, 10, 128, P, P, 0, P, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_project(P + 8, 10, 128, P, P, 0, P, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert lib.ispa_absorbed_weight(P, None, 96, P, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert lib.ispa_quantize_weight_int8(P, None, 96, P, P, None) == ispa.ISPA_ERR_UNSUPPORTED
    assert lib.ispa_quantize_weight_int8(None, None, 128, P, P, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_project_w8a8(P, 10, 128, P, P, P, 0, P, 16, P, None) == ispa.ISPA_ERR_WORKSPACE
    assert lib.ispa_project_w8a8(P, 10, 100, P, P, P, 0, P, 1 << 20, P, None) == \
        ispa.ISPA_ERR_UNSUPPORTED
    assert lib.ispa_project_w8a8(P, -1, 128, P, P, P, 0, P, 1 << 20, P, None) == ispa.ISPA_ERR_ARG
    assert ispa.ispa_project_w8a8_workspace_size(4680, 1536) >= 4680 * 1536 + 4680 * 4
    assert lib.ispa_absorbed_weight(None, None, 128, P, None) == ispa.ISPA_ERR_ARG
    kv = ispa.IspaKV(0x10000, 0x10000, 64)
    assert lib.ispa_full_attention(P, 64, 2, 64, kv, kv, kv, 0.125, None, None, P, 1 << 30, P,
                                   None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_full_attention(P, 64, 2, 96, kv, kv, kv, 0.125, P, None, P, 1 << 30, P,
                                   None) == ispa.ISPA_ERR_UNSUPPORTED
    assert lib.ispa_rank_layers(P, 4, 5, P, None, None) == ispa.ISPA_ERR_ARG
    assert lib.ispa_rank_layers(P, 0, 0, P, None, None) == ispa.ISPA_ERR_ARG


def test_binding_fails_loudly_without_library(tmp_path):
    code = ("import kv_cache_absorption_b200.ispa as m; m.LIB_PATH = '/nonexistent/libispa.so';\n"
            "try:\n    m._load()\nexcept RuntimeError as e:\n    print('LOUD', e)\n")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert "LOUD" in out.stdout and "missing" in out.stdout


def test_product_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "kv_cache_absorption_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in re.sub(r"#.*|//.*", "", text), f
