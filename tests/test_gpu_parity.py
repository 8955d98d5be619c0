"""GPU parity: the CUDA path through the C ABI against the float64 oracle on
the same seeded inputs.

Tolerances (fixed for this path): attention outputs max-abs <= 2e-2 and
relative Frobenius <= 5e-3 (bf16 inputs, fp32 accumulation); G and R
relative Frobenius <= 1e-3; Delta W relative Frobenius <= 2e-3; identical
layer ranking. LSEs: absolute <= 1e-3 (fp32 running max and sum with an
approximate exp2 of relative error ~2^-22; derived bound far below this).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from ispa_synth import (C0, C1, attention_like, gaussian, layer_streams, scaled,
                        stacked_chunk, stacked_layer_streams)

pytestmark = pytest.mark.gpu

ATT_MAXABS, ATT_RELFRO = 2e-2, 5e-3
GR_RELFRO, DW_RELFRO = 1e-3, 2e-3
LSE_ABS = 1e-3


def rel_fro(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check_attention(out, ref, tag=""):
    for key, gkey in (("a_loc", "a_loc"), ("d", "d"), ("a_full", "a_full")):
        got = f64(out[gkey])
        r = ref[key]
        if key == "d" and np.linalg.norm(r) == 0:
            assert np.max(np.abs(got)) == 0.0, tag
            continue
        assert np.max(np.abs(got - r)) <= ATT_MAXABS, (tag, key)
        tol = ATT_RELFRO
        assert rel_fro(got, r) <= tol, (tag, key, rel_fro(got, r))
    for key in ("lse_loc", "lse_hist", "lse_full"):
        got, r = f64(out[key]), ref[key]
        fin = np.isfinite(r)
        assert np.array_equal(np.isfinite(got), fin), (tag, key)
        assert np.array_equal(got[~fin], r[~fin]), (tag, key)
        if fin.any():
            assert np.max(np.abs(got[fin] - r[fin])) <= LSE_ABS, (tag, key)


def to_dev(ch):
    return {k: v.cuda() for k, v in ch.items()}


def run_dual(lib, ch):
    return lib.ispa_dual_attention(ch["q"], ch["k_sink"], ch["v_sink"], ch["k_loc"], ch["v_loc"],
                                   ch.get("k_hist"), ch.get("v_hist"))


def ref_dual(ch):
    return oracle.dual_attention(ch["q"], ch["k_sink"], ch["v_sink"], ch["k_loc"], ch["v_loc"],
                                 ch["k_hist"], ch["v_hist"])


def random_chunk(nq, sink, loc, hist, H, hd, seed):
    g = lambda n, i: gaussian((n, H, hd), seed + 17 * i, 0, "X").to(torch.bfloat16)
    return {"q": g(nq, 0), "k_sink": g(sink, 1), "v_sink": g(sink, 2), "k_loc": g(loc, 3),
            "v_loc": g(loc, 4), "k_hist": g(hist, 5), "v_hist": g(hist, 6)}


# ---------------------------------------------------------------- attention

def _stack_layers(chunks, key, pad_rows=0):
    """[L, len + pad_rows, H, hd] bf16 on the device, layer l's rows first:
    the layers at a stride wider than one layer's rows."""
    t = torch.stack([ch[key] for ch in chunks]).cuda()
    if pad_rows:
        pad = torch.zeros(t.shape[0], pad_rows, *t.shape[2:], dtype=t.dtype, device=t.device)
        t = torch.cat([t, pad], dim=1)
    return t


@pytest.mark.parametrize("hd", [128, 64])
def test_joint_units_equal_the_two_range_plan(lib, hd):
    """A joint unit per (head, query pair) (the local keys, A_loc stored where
    the history starts, then the history from a fresh state, merged in the
    epilogue) gives the same bits as the plan with one local and one history
    range merged by the later unit: single-layer and over three layers, with
    ragged query pairs and a partial last tile in every branch."""
    L, nq, H = 3, 700, 4
    chunks = [random_chunk(nq, 300, 600, 2000, H, hd, seed=60 + 5 * l) for l in range(L)]
    keys = ("a_loc", "d", "a_full", "lse_loc", "lse_hist", "lse_full")
    q = _stack_layers(chunks, "q")
    kv = [_stack_layers(chunks, k) for k in ("k_sink", "v_sink", "k_loc", "v_loc", "k_hist",
                                            "v_hist")]
    outs = {}
    try:
        for tag, hs in (("two", 1), ("joint", -1)):
            lib.ispa_attention_set_splits(1, hs)
            outs[tag + "1"] = [run_dual(lib, to_dev(ch)) for ch in chunks]
            outs[tag + "L"] = lib.ispa_dual_attention_layers(q, *kv, lse=True)
            torch.cuda.synchronize()
    finally:
        lib.ispa_attention_set_splits(0, 0)
    for l in range(L):
        for key in keys:
            assert torch.equal(outs["joint1"][l][key], outs["two1"][l][key]), (l, key)
            assert torch.equal(outs["jointL"][key][l], outs["two1"][l][key]), (l, key)
    assert lib.read_status(outs["jointL"]["status"]) == 0
    check_attention(outs["joint1"][0], ref_dual(chunks[0]), "joint unit")


@pytest.mark.parametrize("hist", [0, 2000])
def test_dual_attention_layers_equals_single_layer_calls(lib, hist):
    """One launch over three layers (ragged query pairs; with a history the
    key ranges are forced to a split with several ranges, so the merge runs
    per layer) equals three single-layer calls with the same split bit for
    bit; inputs and outputs at strides wider than a layer. Without forcing,
    the launch's own split matches the oracle."""
    L, nq, H, hd = 3, 700, 4, 128
    chunks = [random_chunk(nq, 300, 600, hist, H, hd, seed=40 + 7 * l) for l in range(L)]
    st = lambda key, n: _stack_layers(chunks, key, pad_rows=n)[:, :chunks[0][key].shape[0]]
    q = st("q", 8)
    ks, vs, kl, vl = st("k_sink", 16), st("v_sink", 16), st("k_loc", 0), st("v_loc", 0)
    kh, vh = (st("k_hist", 24), st("v_hist", 24)) if hist else (None, None)
    d = H * hd
    outs = [torch.empty(L, nq + 4, d, dtype=dt, device="cuda")[:, :nq]
            for dt in (torch.float32, torch.float32, torch.bfloat16)]
    lse = [torch.empty(L, H * nq + 16, device="cuda")[:, :H * nq].view(L, H, nq) for _ in range(3)]
    lib.ispa_attention_set_splits(2, 2 if hist else 0)
    try:
        got = lib.ispa_dual_attention_layers(q, ks, vs, kl, vl, kh, vh, a_loc=outs[0],
                                             d_out=outs[1], a_full=outs[2], lse=lse)
        torch.cuda.synchronize()
        assert lib.read_status(got["status"]) == 0
        for l in range(L):
            one = run_dual(lib, to_dev(chunks[l]))
            torch.cuda.synchronize()
            for key in ("a_loc", "d", "a_full", "lse_loc", "lse_hist", "lse_full"):
                assert torch.equal(got[key][l], one[key]), (l, key)
    finally:
        lib.ispa_attention_set_splits(0, 0)
    # the launch's own split, every layer against the oracle
    got = lib.ispa_dual_attention_layers(q, ks, vs, kl, vl, kh, vh, lse=True)
    torch.cuda.synchronize()
    assert lib.read_status(got["status"]) == 0
    for l in range(L):
        check_attention({k: v[l] for k, v in got.items() if k != "status"}, ref_dual(chunks[l]),
                        f"layer {l} of {L}")


def test_dual_attention_tiny_workload_all_chunks(lib):
    st = layer_streams(C0, 0, seed=0)
    for c in range(C0.n_chunks):
        ch = st.chunk(c)
        out = run_dual(lib, to_dev(ch))
        torch.cuda.synchronize()
        assert lib.read_status(out["status"]) == 0
        check_attention(out, ref_dual(ch), f"chunk {c}")


@pytest.mark.parametrize("nq,sink,loc,hist,H,hd", [
    (200, 16, 100, 300, 3, 128),    # ragged everywhere, several tiles
    (128, 128, 128, 128, 1, 64),    # exact tiles
    (1, 1, 0, 0, 1, 64),            # single query, single key
    (5, 0, 37, 0, 2, 128),          # no sink, no history
    (300, 24, 0, 1000, 2, 64),      # no local keys, long history
    (129, 7, 130, 257, 4, 128),     # one row / one key past a tile boundary
])
def test_dual_attention_shapes(lib, nq, sink, loc, hist, H, hd):
    ch = random_chunk(nq, sink, loc, hist, H, hd, seed=nq + sink + hist)
    out = run_dual(lib, to_dev(ch))
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    check_attention(out, ref_dual(ch), str((nq, sink, loc, hist, H, hd)))


@pytest.mark.parametrize("ls,hs", [(1, 1), (2, 1), (3, 2), (4, 7), (1, 0), (3, 0)])
def test_dual_attention_forced_key_ranges(lib, ls, hs):
    """Each (head, query pair) cut into ls local and hs history key ranges
    (hs = 0: automatic history ranges); the unit that finishes last merges the
    ranges by their log-sum-exps. Every cut gives the oracle's results."""
    ch = random_chunk(300, 200, 513, 1000, 3, 128, seed=11)
    lib.ispa_attention_set_splits(ls, hs)
    try:
        assert lib.ispa_attention_units(300, 200, 513, 1000, 3)[1] == ls
        out = run_dual(lib, to_dev(ch))
        torch.cuda.synchronize()
    finally:
        lib.ispa_attention_set_splits(0, 0)
    assert lib.read_status(out["status"]) == 0
    check_attention(out, ref_dual(ch), f"key ranges {ls}/{hs}")
    ch0 = dict(ch, k_hist=ch["k_hist"][:0], v_hist=ch["v_hist"][:0])   # no history
    lib.ispa_attention_set_splits(ls, 0)
    try:
        out0 = run_dual(lib, to_dev(ch0))
        torch.cuda.synchronize()
    finally:
        lib.ispa_attention_set_splits(0, 0)
    check_attention(out0, ref_dual(ch0), f"local ranges {ls}, no history")


def test_dual_attention_bit_identical_across_calls(lib):
    """Whichever unit of a (head, pair) finishes last applies the merge, and
    the finishing order varies from call to call; the outputs must not: every
    slot is read back exactly as stored and summed in slot order."""
    st = layer_streams(C1, 0, seed=3)
    ch = to_dev(st.chunk(0))
    outs = [run_dual(lib, ch) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        for k in ("a_loc", "d", "a_full", "lse_loc", "lse_hist", "lse_full"):
            assert torch.equal(o[k], outs[0][k]), k


def test_empty_history_gives_zero_discrepancy(lib):
    ch = random_chunk(70, 16, 64, 0, 2, 64, seed=3)
    out = run_dual(lib, to_dev(ch))
    torch.cuda.synchronize()
    assert torch.all(out["d"] == 0)
    assert torch.all(torch.isneginf(out["lse_hist"]))
    assert torch.equal(out["lse_full"], out["lse_loc"])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_local_attention(lib, dtype):
    ch = random_chunk(150, 16, 140, 0, 2, 128, seed=11)
    dc = to_dev(ch)
    out = lib.ispa_local_attention(dc["q"], dc["k_sink"], dc["v_sink"], dc["k_loc"], dc["v_loc"],
                                   out_dtype=dtype, want_lse=True)
    torch.cuda.synchronize()
    ref, lse = oracle.local_attention(ch["q"], ch["k_sink"], ch["v_sink"], ch["k_loc"], ch["v_loc"])
    got = f64(out["out"])
    assert np.max(np.abs(got - ref)) <= ATT_MAXABS
    assert rel_fro(got, ref) <= ATT_RELFRO
    assert np.max(np.abs(f64(out["lse"]) - lse)) <= LSE_ABS


def test_dual_attention_full_size_sampled_rows(lib):
    """1.3B single chunk at full size (Nq 4680, keys 1560 + 4680 + 14040,
    12 heads x 128): every output row is produced by the launch the benchmark
    times; 96 sampled rows are checked against the oracle."""
    st = layer_streams(C1, 0, seed=0)
    ch = st.chunk(0)
    out = run_dual(lib, to_dev(ch))
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    rows = np.sort(np.random.default_rng(0).choice(C1.chunk_tokens, 96, replace=False))
    rows = np.concatenate([rows, [0, 127, 128, 4679]])
    sub = dict(ch)
    sub["q"] = ch["q"][torch.from_numpy(rows)]
    ref = ref_dual(sub)
    got = {k: (v[torch.from_numpy(rows).cuda()] if k in ("a_loc", "d", "a_full") else
               v[:, torch.from_numpy(rows).cuda()]) for k, v in out.items()
           if k != "status"}
    check_attention(got, ref, "full-size sample")


def _full_size_sample(lib, cfg, chunk, n_rows, seed):
    st = layer_streams(cfg, 0, seed=0)
    ch = st.chunk(chunk)
    out = run_dual(lib, to_dev(ch))
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    rows = np.sort(np.random.default_rng(seed).choice(cfg.chunk_tokens, n_rows, replace=False))
    rows = np.concatenate([rows, [0, cfg.chunk_tokens - 1]])
    sub = dict(ch)
    sub["q"] = ch["q"][torch.from_numpy(rows)]
    ref = ref_dual(sub)
    idx = torch.from_numpy(rows).cuda()
    got = {k: (v[idx] if k in ("a_loc", "d", "a_full") else v[:, idx]) for k, v in out.items()
           if k != "status"}
    check_attention(got, ref, f"{cfg.name} chunk {chunk}")


def test_dual_attention_full_size_14B_sampled_rows(lib):
    """14B width at full size (40 heads x 128, Nq 4680, keys 1560 + 4680 +
    14040: the last warmup chunk), 30 sampled rows against the oracle."""
    from ispa_synth import C3
    _full_size_sample(lib, C3, C3.n_chunks - 1, 30, seed=3)


def test_dual_attention_full_size_first_warmup_chunk(lib):
    """1.3B warmup chunk 0 at full size: no history (the local units write
    the final outputs directly, D = 0, LSE_hist = -inf)."""
    from ispa_synth import C2
    _full_size_sample(lib, C2, 0, 48, seed=4)


def test_gram_full_size_14B_sampled_tiles(lib):
    """The Gram of 4680 rows at the 14B width (d = 5120, stream-K over 1640
    output tiles): 8 sampled 128 x 128 tiles of G, R and S against float64."""
    rows, dim = 4680, 5120
    a = attention_like(rows, dim, seed=51)
    dm = 0.3 * attention_like(rows, dim, seed=52)
    M = lib.ispa_gram_accumulate(a.cuda(), dm.cuda())
    torch.cuda.synchronize()
    a64, d64 = f64(a), f64(dm)
    r = np.random.default_rng(5)
    for _ in range(8):
        I, J = sorted(r.integers(0, dim // 128, size=2))
        i, j = I * 128, J * 128
        for name, X, Y, oi, oj in (("G", a64, a64, 0, 0), ("R", a64, d64, 0, dim),
                                   ("S", d64, d64, dim, dim)):
            ref = X[:, i:i + 128].T @ Y[:, j:j + 128]
            got = f64(M[oi + i:oi + i + 128, oj + j:oj + j + 128])
            assert rel_fro(got, ref) <= GR_RELFRO, (name, I, J)


# ---------------------------------------------------------------- Gram

def upper_tile_mask(dim):
    I = np.arange(dim)[:, None] // 128
    J = np.arange(dim)[None, :] // 128
    return I <= J


@pytest.mark.parametrize("rows,dim", [(1000, 256), (777, 384), (64, 128), (700, 1536)])
def test_gram_accumulate_two_calls(lib, rows, dim):
    """Every output tile against float64; at d = 1536 there are 156 tiles, so
    the kernel runs one wave of whole tiles and splits the remaining tiles'
    row blocks over all CTAs (stream-K)."""
    a1 = attention_like(rows, dim, seed=1)
    d1 = 0.3 * attention_like(rows, dim, seed=2)
    a2 = attention_like(rows + 40, dim, seed=3)
    d2 = 0.3 * attention_like(rows + 40, dim, seed=4)
    status = lib.new_status("cuda")
    M = lib.ispa_gram_accumulate(a1.cuda(), d1.cuda(), status=status)
    M = lib.ispa_gram_accumulate(a2.cuda(), d2.cuda(), M=M, accumulate=True, status=status)
    torch.cuda.synchronize()
    assert lib.read_status(status) == 0     # no pipeline wait gave up
    G, R, S = oracle.gram(np.concatenate([f64(a1), f64(a2)]), np.concatenate([f64(d1), f64(d2)]))
    Mg = f64(M)
    up = upper_tile_mask(dim)
    assert rel_fro(Mg[:dim, :dim][up], G[up]) <= GR_RELFRO
    assert rel_fro(Mg[:dim, dim:], R) <= GR_RELFRO
    assert rel_fro(Mg[dim:, dim:][up], S[up]) <= GR_RELFRO


def test_gram_overwrite_and_empty(lib):
    dim = 256
    a = attention_like(300, dim, seed=5).cuda()
    M = torch.full((2 * dim, 2 * dim), 7.0, device="cuda")
    lib.ispa_gram_accumulate(a[:0], a[:0], M=M, accumulate=False)
    torch.cuda.synchronize()
    assert torch.all(M[:dim] == 0) and torch.all(M[dim:, dim:] == 0)
    assert torch.all(M[dim:, :dim] == 7.0)   # the unused block is not touched


# ---------------------------------------------------------------- solve / error / rank

def synthetic_layer(rows, dim, seed):
    a = attention_like(rows, dim, seed=seed)
    f = a + 0.4 * attention_like(rows, dim, seed=seed + 1, rho=0.5, common=0.1)
    W = gaussian((dim, dim), seed, 0, "W") / math.sqrt(dim)
    return f64(a), f64(f), W


def product_tol(X, Y, ref):
    """Relative Frobenius bound for an fp32-accurate product X @ Y (3xTF32
    operands keep about 21 mantissa bits; fp32 accumulation over K terms
    adds about sqrt(K) 2^-24), scaled by the cancellation ratio
    || |X| |Y| || / || X Y || and a safety factor of 8."""
    K = X.shape[1]
    mag = np.linalg.norm(np.abs(X) @ np.abs(Y)) / np.linalg.norm(ref)
    return 8.0 * (2.0 ** -21 + math.sqrt(K) * 2.0 ** -24) * mag


def pack_M(G, R, S):
    d = G.shape[0]
    M = np.zeros((2 * d, 2 * d), np.float32)
    M[:d, :d], M[:d, d:], M[d:, d:] = G, R, S
    return torch.from_numpy(M)


@pytest.mark.parametrize("dim", [128, 256, 512])
def test_absorb_solve_isolated(lib, dim):
    a, f, W = synthetic_layer(4 * dim + 100, dim, seed=dim)
    G, R, S = oracle.gram(a, f - a)
    M = pack_M(G, R, S)
    out = lib.ispa_absorb_solve(M.cuda(), W.cuda())
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    Gf, Rf = f64(M[:dim, :dim]), f64(M[:dim, dim:])
    lam = oracle.default_lambda(Gf)
    assert abs(out["lam"].item() - lam) <= 1e-6 * lam
    dW, B = oracle.absorb(Gf, Rf, f64(W), lam)
    assert rel_fro(f64(out["B"]), B) <= product_tol(Rf, f64(W), B)
    assert rel_fro(f64(out["dW"]), dW) <= DW_RELFRO


def test_absorb_solve_deterministic(lib):
    """Two solves of the same layer give bit-identical B and Delta W: the
    single-layer sweep runs on two streams and Delta W sums two K halves
    into a zeroed output, whose fp32 addition does not depend on the order."""
    dim = 512
    a, f, W = synthetic_layer(4 * dim + 100, dim, seed=77)
    G, R, S = oracle.gram(a, f - a)
    M = pack_M(G, R, S).cuda()
    Wd = W.cuda()
    first = lib.ispa_absorb_solve(M, Wd)
    second = lib.ispa_absorb_solve(M, Wd)
    torch.cuda.synchronize()
    assert lib.read_status(first["status"]) == 0 and lib.read_status(second["status"]) == 0
    assert torch.equal(first["dW"], second["dW"])
    assert torch.equal(first["B"], second["B"])


# Full-size solve inputs: rows = iid N(0, 1) plus one common mean mode m. The
# row count sets the bottom of the spectrum (Marchenko-Pastur) and |m|^2 the
# top, chosen so that kappa(G + lambda I) and lambda_max / lambda_mean are at
# least those of layer 0's warmup statistics at 1.3B width (4.5e3, 548) and
# 14B width (4.1e4, 1814); this construction gives 6.7e3 / 554 and
# 5.7e4 / 1815.
FULL_SIZE = {1536: (3472, 548.0), 5120: (7680, 1814.0)}


@pytest.mark.parametrize("dim", [1536, 5120])
def test_absorb_solve_full_size(lib, dim):
    """The solve at the 1.3B (d = 1536) and 14B (d = 5120) layer width: G and
    R formed on the host in fp32 and passed as-is to both sides; the oracle
    solves in float64."""
    rows, ratio = FULL_SIZE[dim]
    m2 = (ratio - 1.0) / (1.0 - ratio / dim)
    a = gaussian((rows, dim), dim, 0, "X") + gaussian((1, dim), dim + 1, 0, "X") * math.sqrt(m2 / dim)
    dm = 0.4 * (gaussian((rows, dim), dim + 2, 0, "X") + gaussian((1, dim), dim + 3, 0, "X"))
    G, R = a.T @ a, a.T @ dm
    M = torch.zeros(2 * dim, 2 * dim)
    M[:dim, :dim], M[:dim, dim:] = G, R
    W = gaussian((dim, dim), dim, 0, "W") / math.sqrt(dim)
    out = lib.ispa_absorb_solve(M.cuda(), W.cuda())
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    lam = oracle.default_lambda(f64(G))
    dW, B = oracle.absorb(f64(G), f64(R), f64(W), lam)
    assert rel_fro(f64(out["dW"]), dW) <= DW_RELFRO
    assert rel_fro(f64(out["B"]), B) <= product_tol(f64(R), f64(W), B)


def full_size_inputs(dim, seed):
    rows, ratio = FULL_SIZE[dim]
    m2 = (ratio - 1.0) / (1.0 - ratio / dim)
    a = gaussian((rows, dim), seed, 0, "X") + gaussian((1, dim), seed + 1, 0, "X") * math.sqrt(m2 / dim)
    dm = 0.4 * (gaussian((rows, dim), seed + 2, 0, "X") + gaussian((1, dim), seed + 3, 0, "X"))
    return a.T @ a, a.T @ dm, gaussian((dim, dim), seed, 0, "W") / math.sqrt(dim)


def test_absorb_solve_batched_full_size(lib):
    """Two layers at the 1.3B layer width in one batched call (the
    left-looking sweep with chunked accumulation) against the oracle."""
    dim, L = 1536, 2
    Ms, Ws, refs = [], [], []
    for l in range(L):
        G, R, W = full_size_inputs(dim, 500 + 10 * l)
        M = torch.zeros(2 * dim, 2 * dim)
        M[:dim, :dim], M[:dim, dim:] = G, R
        Ms.append(M)
        Ws.append(W)
        refs.append(oracle.absorb(f64(G), f64(R), f64(W), oracle.default_lambda(f64(G)))[0])
    out = lib.ispa_absorb_solve_batched(torch.stack(Ms).cuda(), torch.stack(Ws).cuda())
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    for l in range(L):
        assert rel_fro(f64(out["dW"][l]), refs[l]) <= DW_RELFRO


def test_absorb_solve_explicit_lambda_and_not_spd(lib):
    dim = 128
    a, f, W = synthetic_layer(600, dim, seed=9)
    G, R, S = oracle.gram(a, f - a)
    M = pack_M(G, R, S)
    out = lib.ispa_absorb_solve(M.cuda(), W.cuda(), lam=2.5)
    torch.cuda.synchronize()
    assert out["lam"].item() == 2.5
    dW, _ = oracle.absorb(f64(M[:dim, :dim]), f64(M[:dim, dim:]), f64(W), 2.5)
    assert rel_fro(f64(out["dW"]), dW) <= DW_RELFRO
    # a negative ridge weight larger than the smallest eigenvalue of G
    bad = lib.ispa_absorb_solve(M.cuda(), W.cuda(), lam=-1e6)
    torch.cuda.synchronize()
    assert bad["lam"].item() > 0  # lam <= 0 selects the default
    M0 = torch.zeros_like(M)
    bad = lib.ispa_absorb_solve(M0.cuda(), W.cuda())   # G = 0 and lambda = 0
    torch.cuda.synchronize()
    assert lib.read_status(bad["status"]) & lib.ISPA_STATUS_NOT_SPD
    # a NaN in G reaches a pivot: reported as a non-finite input, not as G + lambda I
    # failing to be positive definite
    Mn = M.clone()
    Mn[5, 5] = float("nan")
    bad = lib.ispa_absorb_solve(Mn.cuda(), W.cuda(), lam=2.5)
    torch.cuda.synchronize()
    assert lib.read_status(bad["status"]) & lib.ISPA_STATUS_NONFINITE


@pytest.mark.parametrize("dim", [128, 384])
def test_layer_error_isolated(lib, dim):
    a, f, W = synthetic_layer(3 * dim + 50, dim, seed=dim + 1)
    G, R, S = oracle.gram(a, f - a)
    M = pack_M(G, R, S)
    G32, R32 = f64(M[:dim, :dim]), f64(M[:dim, dim:])
    lam = oracle.default_lambda(G32)
    dW, B = oracle.absorb(G32, R32, f64(W), lam)
    err = lib.ispa_layer_error(M.cuda(), W.cuda(), torch.from_numpy(dW).float().cuda(),
                               torch.from_numpy(B).float().cuda(),
                               torch.tensor([lam], dtype=torch.float32).cuda())
    torch.cuda.synchronize()
    e2, eps = oracle.reconstruction_error(a, f, f64(W), dW)
    got = err.cpu().numpy()
    assert abs(got[0] - e2) <= 2e-3 * e2
    assert abs(got[1] - eps) <= 2e-3 * eps


def test_rank_layers_bit_exact(lib):
    r = np.random.default_rng(4)
    eps = r.integers(0, 9, size=37) / 10.0
    err = torch.from_numpy(np.stack([eps * 3, eps], 1)).cuda()
    perm, sel = lib.ispa_rank_layers(err, 18)
    torch.cuda.synchronize()
    ref_perm, ref_sel = oracle.rank_layers(eps, 18)
    assert perm.cpu().numpy().tolist() == ref_perm.tolist()
    assert sel.cpu().numpy().astype(bool).tolist() == ref_sel.tolist()


# ---------------------------------------------------------------- end to end

def test_warmup_tiny_end_to_end(lib):
    from kv_cache_absorption_b200.warmup import LayerWarmup, run_warmup
    st = layer_streams(C0, 0, seed=0)
    chunks = [st.chunk(c) for c in range(C0.n_chunks)]
    ref = oracle.warmup_layer(chunks, st.w)
    runner = LayerWarmup(C0.heads, C0.head_dim, C0.chunk_tokens, C0.sink_tokens,
                         C0.chunk_tokens, 256)
    err, perm, sel = run_warmup([[to_dev(c) for c in chunks]], st.w.cuda()[None], 1, runner)
    torch.cuda.synchronize()
    assert lib.read_status(runner.status) == 0
    d = C0.d
    Mg = f64(runner.M[0])
    up = upper_tile_mask(d)
    assert rel_fro(Mg[:d, :d][up], ref["G"][up]) <= GR_RELFRO
    assert rel_fro(Mg[:d, d:], ref["R"]) <= GR_RELFRO
    assert rel_fro(f64(runner.dW[0]), ref["dW"]) <= DW_RELFRO
    assert abs(err[0, 1].item() - ref["eps"]) <= 5e-3 * ref["eps"]


def test_warmup_grouped_layers_equal_per_layer_path(lib):
    """The warmup driver's grouped path (the same chunk of two layers per
    attention launch, groups of 2, 2 and 1 layers on two streams) gives the
    per-layer path's statistics, Delta W, errors and ranking. With the
    per-layer key-range split forced on both, M and Delta W agree bit for
    bit; with each launch's own split, to the fp32 rounding of the merge."""
    import dataclasses
    from kv_cache_absorption_b200.warmup import LayerWarmup, run_warmup
    cfg = dataclasses.replace(C0, layers=5)
    sts, qkv = stacked_layer_streams(cfg, list(range(cfg.layers)), seed=3, device="cuda")
    per_layer = [[st.chunk(c) for c in range(cfg.n_chunks)] for st in sts]
    stacked = [stacked_chunk(cfg, qkv, c) for c in range(cfg.n_chunks)]
    W_all = torch.stack([st.w for st in sts]).cuda()
    max_hist = max(len(cfg.history_frames_of(c)) for c in range(cfg.n_chunks)) * cfg.tokens_per_frame
    streams = [torch.cuda.current_stream(), torch.cuda.Stream()]

    def run(group):
        r = LayerWarmup(cfg.heads, cfg.head_dim, cfg.chunk_tokens, cfg.sink_tokens,
                        cfg.chunk_tokens, max_hist, n_layers=cfg.layers, n_slots=2, group=group)
        out = run_warmup(per_layer if group == 1 else None, W_all, 2, r, streams=streams,
                         stacked_chunks=stacked if group > 1 else None)
        torch.cuda.synchronize()
        assert lib.read_status(r.status) == 0
        return r, out

    rel = lambda a, b: float((a - b).norm() / b.norm())
    # the per-layer split forced on both paths: bit for bit (epsilon's fp64
    # sums are added across CTAs by atomics: equal up to their order)
    lib.ispa_attention_set_splits(1, 1)
    try:
        (r1, (e1, p1, s1)), (r2, (e2, p2, s2)) = run(1), run(2)
    finally:
        lib.ispa_attention_set_splits(0, 0)
    assert r2.layer_groups() == [(0, 2), (2, 2), (4, 1)]
    assert torch.equal(r1.M, r2.M)
    assert torch.equal(r1.dW, r2.dW)
    assert torch.allclose(e1, e2, rtol=1e-12, atol=0.0)
    assert torch.equal(p1, p2) and torch.equal(s1, s2)
    # each launch's own split
    (r1, (e1, p1, s1)), (r2, (e2, p2, s2)) = run(1), run(2)
    assert rel(r2.M, r1.M) <= 1e-6
    assert rel(r2.dW, r1.dW) <= 1e-4
    assert torch.allclose(e1, e2, rtol=1e-5, atol=0.0)
    assert torch.equal(p1, p2) and torch.equal(s1, s2)


def test_warmup_multilayer_ranking(lib):
    """Six layers of a reduced 1.3B geometry (frames of 64 tokens, 2 heads x
    64, 4 chunks with a growing history); the per-layer AR(1) correlation is
    spread so that the errors separate."""
    from kv_cache_absorption_b200.warmup import LayerWarmup, run_warmup
    L = 6
    chunks_dev, Ws, eps_ref = [], [], []
    for l in range(L):
        cfg = scaled(C0, tokens_per_frame=64, sink_tokens=64, chunk_frames=3, first_chunk_frame=1,
                     n_chunks=4, history_window=None, rho=0.5 + 0.08 * l)
        st = layer_streams(cfg, l, seed=1)
        chunks = [st.chunk(c) for c in range(4)]
        eps_ref.append(oracle.warmup_layer(chunks, st.w)["eps"])
        chunks_dev.append([to_dev(c) for c in chunks])
        Ws.append(st.w)
    ref_perm, ref_sel = oracle.rank_layers(eps_ref, 3)
    # one stream, then layers alternating over two streams (two buffer slots)
    for n_slots in (1, 2):
        runner = LayerWarmup(2, 64, 192, 64, 192, 9 * 64, n_layers=L, n_slots=n_slots)
        streams = [torch.cuda.current_stream()] + [torch.cuda.Stream()] * (n_slots - 1)
        err, perm, sel = run_warmup(chunks_dev, torch.stack(Ws).cuda(), 3, runner,
                                    streams=streams)
        torch.cuda.synchronize()
        got_eps = err[:, 1].cpu().numpy()
        assert np.max(np.abs(got_eps - eps_ref) / np.asarray(eps_ref)) <= 5e-3, n_slots
        assert perm.cpu().numpy().tolist() == ref_perm.tolist(), n_slots
        assert sel.cpu().numpy().astype(bool).tolist() == ref_sel.tolist(), n_slots


def test_nonfinite_query_flag(lib):
    """An infinite query value makes that row's scores and log-sum-exp
    non-finite: the call reports it in the status word; other rows are
    unaffected."""
    ch = random_chunk(40, 8, 32, 300, 2, 64, seed=6)
    ch["q"] = ch["q"].clone()
    ch["q"][7, 1, 3] = float("inf")
    out = run_dual(lib, to_dev(ch))
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == lib.ISPA_STATUS_NONFINITE
    ok = run_dual(lib, to_dev(random_chunk(40, 8, 32, 300, 2, 64, seed=6)))
    torch.cuda.synchronize()
    assert lib.read_status(ok["status"]) == 0
    assert torch.equal(out["a_loc"][8:], ok["a_loc"][8:])


def tf32_rn(x):
    """fp32 -> tf32, nearest, ties away from zero (how the attention epilogue
    stores A_loc and D for the Gram): add half an ulp of the 10-bit mantissa to
    the magnitude bits, clear the low 13 bits."""
    b = x.contiguous().view(torch.int32)
    return ((b + 0x1000) & ~0x1FFF).view(torch.float32)


def test_error_identity_when_the_absorption_explains_almost_everything(lib):
    """The GPU forms epsilon from the Gram blocks, ||E||^2 = <S, W W^T> -
    <Delta W, B> - lambda ||Delta W||^2, a difference of terms ~||D W||^2.
    Here D = A_loc M + small noise, so Delta W absorbs all but a few tenths of
    a percent of ||D W||^2 and the subtraction cancels ~300-fold; two layers'
    errors differ by ~3%. Against the oracle's directly materialised
    row-wise error on the same (tf32-valued) rows: the ranking is identical
    and epsilon stays within the end-to-end tolerance."""
    from kv_cache_absorption_b200.warmup import LayerWarmup, rank
    dim, rows, L = 256, 4096, 4
    lam = 0.04                                  # ~1e-4 tr(G) / d: little ridge bias
    noise = (1.0, 1.015, 1.1, 1.6)
    A = tf32_rn(attention_like(rows, dim, seed=31))
    runner = LayerWarmup(2, 128, rows, 1, 1, 0, n_layers=L)
    Ws, eps_ref, ratio = [], [], []
    for l in range(L):
        Mx = 0.05 * gaussian((dim, dim), 40 + l, 0, "X") / math.sqrt(dim)
        Z = gaussian((rows, dim), 60 + l, 0, "X")
        D = tf32_rn(A @ Mx + 8.7e-4 * noise[l] * Z)
        W = gaussian((dim, dim), 80 + l, 0, "W") / math.sqrt(dim)
        Ws.append(W)
        a64, d64 = f64(A), f64(D)
        G, R, S = oracle.gram(a64, d64)
        dW, _ = oracle.absorb(G, R, f64(W), lam)
        e2, eps = oracle.reconstruction_error(a64, a64 + d64, f64(W), dW)
        eps_ref.append(eps)
        ratio.append(e2 / float(np.sum((d64 @ f64(W)) ** 2)))
        lib.ispa_gram_accumulate(A.cuda(), D.cuda(), M=runner.M[l], status=runner.status)
    W_all = torch.stack(Ws).cuda()
    runner.solve_all(W_all, lam)
    runner.weight_gram(W_all)
    err = torch.empty(L, 2, dtype=torch.float64, device="cuda")
    runner.error_all(W_all, err)
    perm = torch.empty(L, dtype=torch.int32, device="cuda")
    sel = torch.empty(L, dtype=torch.uint8, device="cuda")
    rank(err, 2, perm, sel)
    torch.cuda.synchronize()
    assert lib.read_status(runner.status) == 0
    assert max(ratio) < 1e-2                     # the regime this test is about
    got = err[:, 1].cpu().numpy()
    rel_eps = np.abs(got - eps_ref) / np.asarray(eps_ref)
    assert perm.cpu().numpy().tolist() == np.argsort(eps_ref, kind="stable").tolist(), \
        (got, eps_ref)
    assert np.max(rel_eps) <= 5e-3, (rel_eps, ratio)


def test_fp16_range_flag(lib):
    ch = random_chunk(32, 8, 32, 16, 1, 64, seed=5)
    ch["v_hist"] = ch["v_hist"].clone()
    ch["v_hist"][3, 0, 5] = 1.0e5
    out = run_dual(lib, to_dev(ch))
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) & lib.ISPA_STATUS_FP16_RANGE


def test_absorb_and_error_batched_over_layers(lib):
    """Three layers solved and scored in single calls: each layer matches the
    oracle and the single-layer entry point."""
    dim, L = 256, 3
    Ms, Ws, refs = [], [], []
    for l in range(L):
        a, f, W = synthetic_layer(3 * dim + 17 * l, dim, seed=40 + l)
        G, R, S = oracle.gram(a, f - a)
        M = pack_M(G, R, S)
        G32, R32 = f64(M[:dim, :dim]), f64(M[:dim, dim:])
        lam = oracle.default_lambda(G32)
        dW, B = oracle.absorb(G32, R32, f64(W), lam)
        refs.append((dW, oracle.reconstruction_error(a, f, f64(W), dW)))
        Ms.append(M)
        Ws.append(W)
    M = torch.stack(Ms).cuda()
    W = torch.stack(Ws).contiguous().cuda()
    out = lib.ispa_absorb_solve_batched(M, W)
    err = lib.ispa_layer_error_batched(M, W, out["dW"], out["B"], out["lam"])
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    for l in range(L):
        dW_ref, (e2, eps) = refs[l]
        assert rel_fro(f64(out["dW"][l]), dW_ref) <= DW_RELFRO
        # one layer alone takes the right-looking sweep, several the left-looking one
        single = lib.ispa_absorb_solve(M[l].contiguous(), W[l].contiguous())
        torch.cuda.synchronize()
        assert rel_fro(f64(single["dW"]), f64(out["dW"][l])) <= DW_RELFRO
        got = err[l].cpu().numpy()
        assert abs(got[0] - e2) <= 2e-3 * e2 and abs(got[1] - eps) <= 2e-3 * eps


def test_weight_gram_and_error_from_wwt(lib):
    """W W^T formed once per layer, then the error as one reduction pass:
    same per-layer result as the path that forms W W^T inside the error."""
    dim, L = 384, 2
    Ms, Ws, refs = [], [], []
    for l in range(L):
        a, f, W = synthetic_layer(3 * dim + 31 * l, dim, seed=70 + l)
        G, R, S = oracle.gram(a, f - a)
        M = pack_M(G, R, S)
        G32, R32 = f64(M[:dim, :dim]), f64(M[:dim, dim:])
        lam = oracle.default_lambda(G32)
        dW, _ = oracle.absorb(G32, R32, f64(W), lam)
        refs.append(oracle.reconstruction_error(a, f, f64(W), dW))
        Ms.append(M)
        Ws.append(W)
    M = torch.stack(Ms).cuda()
    W = torch.stack(Ws).contiguous().cuda()
    P = lib.ispa_weight_gram_batched(W)
    out = lib.ispa_absorb_solve_batched(M, W)
    err_p = lib.ispa_layer_error_wwt_batched(M, P, out["dW"], out["B"], out["lam"])
    err_w = lib.ispa_layer_error_batched(M, W, out["dW"], out["B"], out["lam"])
    torch.cuda.synchronize()
    for l in range(L):
        Wl = f64(W[l])
        P_ref = Wl @ Wl.T
        assert rel_fro(f64(P[l]), P_ref) <= product_tol(Wl, Wl.T, P_ref)
        e2, eps = refs[l]
        got = err_p[l].cpu().numpy()
        assert abs(got[0] - e2) <= 2e-3 * e2 and abs(got[1] - eps) <= 2e-3 * eps
        # both paths reduce the same fp32 W W^T entries in fp64
        assert np.allclose(got, err_w[l].cpu().numpy(), rtol=1e-9, atol=0)


# ---------------------------------------------------------------- split history, streaming layers

@pytest.mark.parametrize("nq,sink,loc,hist,H,hd", [
    (300, 16, 100, 2000, 2, 128),    # 2 local tiles, 16 history tiles: 4 key ranges
    (129, 0, 64, 3100, 3, 64),       # 1 local tile, 25 history tiles: 13 ranges, ragged
])
def test_dual_attention_split_history(lib, nq, sink, loc, hist, H, hd):
    """Histories longer than three local branches are cut into key ranges
    (split-KV) and merged by their log-sum-exps: same results as the oracle's
    undecomposed pass."""
    ch = random_chunk(nq, sink, loc, hist, H, hd, seed=hist)
    out = run_dual(lib, to_dev(ch))
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    check_attention(out, ref_dual(ch), "split history")


@pytest.mark.parametrize("hist", [0, 700, 2000])
def test_full_attention_vs_oracle(lib, hist):
    """F-Layer attention (A_full and its LSE only), with and without split
    history."""
    ch = random_chunk(260, 16, 100, hist, 2, 128, seed=7 + hist)
    d = to_dev(ch)
    out = lib.ispa_full_attention(d["q"], d["k_sink"], d["v_sink"], d["k_loc"], d["v_loc"],
                                  d["k_hist"], d["v_hist"], want_lse=True)
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    ref = ref_dual(ch)
    got = f64(out["out"])
    assert np.max(np.abs(got - ref["a_full"])) <= ATT_MAXABS
    assert rel_fro(got, ref["a_full"]) <= ATT_RELFRO
    assert np.max(np.abs(f64(out["lse"]) - ref["lse_full"])) <= LSE_ABS


def test_project_and_absorbed_weight(lib):
    """out = A W' on the bf16 tensor cores (ragged rows): fp32 output within
    fp32 accumulation of the exact bf16 products, bf16 output within its own
    rounding; W' = bf16(W + Delta W) bit-exact against torch's rounding."""
    rows, dim = 333, 256
    a = gaussian((rows, dim), 3, 0, "X").to(torch.bfloat16)
    W = gaussian((dim, dim), 4, 0, "W") / math.sqrt(dim)
    dW = 0.1 * gaussian((dim, dim), 5, 0, "W") / math.sqrt(dim)
    w_bf = lib.ispa_absorbed_weight(W.cuda(), dW.cuda())
    torch.cuda.synchronize()
    assert torch.equal(w_bf.cpu(), (W + dW).to(torch.bfloat16))
    ref = f64(a) @ f64(w_bf)
    out32 = lib.ispa_project(a.cuda(), w_bf, out_dtype=torch.float32)
    out16 = lib.ispa_project(a.cuda(), w_bf)
    torch.cuda.synchronize()
    assert rel_fro(f64(out32), ref) <= product_tol(f64(a), f64(w_bf), ref)
    assert rel_fro(f64(out16), ref) <= 2.0 ** -8
    assert lib.ispa_project(a[:0].cuda(), w_bf).shape == (0, dim)


@pytest.mark.parametrize("local", [False, True])
def test_streaming_layer_vs_oracle(lib, local):
    """A post-transition chunk through one layer: F-Layer = full attention
    (split history) then W; L-Layer = local attention then W + Delta W. Both
    operands of the projection are bf16, so the tolerance is two bf16
    roundings (2 x 2^-9 relative) on top of the attention's."""
    ch = random_chunk(200, 16, 100, 1800, 2, 128, seed=11)
    dim = 256
    W = gaussian((dim, dim), 12, 0, "W") / math.sqrt(dim)
    dW = 0.2 * gaussian((dim, dim), 13, 0, "W") / math.sqrt(dim)
    d = to_dev(ch)
    if local:
        att = lib.ispa_local_attention(d["q"], d["k_sink"], d["v_sink"], d["k_loc"], d["v_loc"])
        w_bf = lib.ispa_absorbed_weight(W.cuda(), dW.cuda())
    else:
        att = lib.ispa_full_attention(d["q"], d["k_sink"], d["v_sink"], d["k_loc"], d["v_loc"],
                                      d["k_hist"], d["v_hist"])
        w_bf = lib.ispa_absorbed_weight(W.cuda())
    out = lib.ispa_project(att["out"], w_bf)
    torch.cuda.synchronize()
    assert lib.read_status(att["status"]) == 0
    ref = oracle.streaming_layer(ch["q"], ch["k_sink"], ch["v_sink"], ch["k_loc"], ch["v_loc"],
                                 ch["k_hist"], ch["v_hist"], f64(W), f64(dW) if local else None,
                                 local=local)
    assert rel_fro(f64(out), ref) <= ATT_RELFRO + 2 * 2.0 ** -9


@pytest.mark.parametrize("c", [4, 20])
def test_streaming_full_size_sampled_rows(lib, c):
    """1.3B streaming at full size: the first (history 12 frames) and last
    (history 60 frames = 93600 tokens, split into key ranges) post-transition
    chunks through an F-Layer and an L-Layer, the launches the streaming
    benchmark times, on 8 sampled rows against the oracle."""
    from ispa_synth import C4
    from kv_cache_absorption_b200.streaming import StreamingLayers
    st = layer_streams(C4, 0, seed=0)
    ch = st.chunk(c)
    dim = C4.d
    dW = 0.05 * gaussian((dim, dim), 21, 0, "W") / math.sqrt(dim)
    max_hist = len(C4.history_frames_of(C4.n_chunks + C4.stream_chunks - 1)) * C4.tokens_per_frame
    s = StreamingLayers(C4.heads, C4.head_dim, C4.chunk_tokens, C4.sink_tokens, C4.chunk_tokens,
                        max_hist, n_layers=2)
    W2 = torch.stack([st.w, st.w]).cuda()
    s.transition(W2, torch.stack([dW, dW]).cuda(), [False, True])
    d = to_dev(ch)
    rows = np.linspace(0, C4.chunk_tokens - 1, 8).astype(int)
    sub = dict(ch)
    sub["q"] = ch["q"][rows]
    for layer, local in ((0, False), (1, True)):
        out = f64(s.layer(layer, d))[rows]
        torch.cuda.synchronize()
        assert lib.read_status(s.status) == 0
        ref = oracle.streaming_layer(sub["q"], ch["k_sink"], ch["v_sink"], ch["k_loc"], ch["v_loc"],
                                     ch["k_hist"], ch["v_hist"], f64(st.w),
                                     f64(dW) if local else None, local=local)
        assert rel_fro(out, ref) <= ATT_RELFRO + 2 * 2.0 ** -9, (c, local, rel_fro(out, ref))



def test_streaming_through_kv_caches(lib):
    """A stream of post-transition chunks through an F-Layer and an L-Layer
    whose keys and values come from KV caches the chunks are appended to
    (the F-Layer's growing over the stream, the L-Layer's holding the sink and
    one chunk): every chunk's output against the oracle, which takes each
    chunk's keys straight from the synthetic frame streams. Ragged sizes: 200
    tokens per frame, a 72-token sink, histories of 600 to 1200 tokens."""
    from ispa_synth import Config
    from kv_cache_absorption_b200.streaming import KVCache, StreamingLayers
    cfg = Config("kv-cache-stream", layers=1, heads=2, head_dim=128, tokens_per_frame=200,
                 sink_tokens=72, chunk_frames=1, first_chunk_frame=1, n_chunks=3,
                 history_window=None, stream_chunks=4)
    st = layer_streams(cfg, 0, seed=5)
    dim = cfg.d
    dW = 0.1 * gaussian((dim, dim), 22, 0, "W") / math.sqrt(dim)
    c_first, c_last = cfg.n_chunks, cfg.n_chunks + cfg.stream_chunks - 1
    hist_last = len(cfg.history_frames_of(c_last)) * cfg.tokens_per_frame
    s = StreamingLayers(cfg.heads, cfg.head_dim, cfg.chunk_tokens, cfg.sink_tokens,
                        cfg.chunk_tokens, hist_last, n_layers=2)
    s.transition(torch.stack([st.w, st.w]).cuda(), torch.stack([dW, dW]).cuda(), [False, True])
    first = to_dev(st.chunk(c_first))
    caches = []
    for full in (True, False):
        kc = KVCache(cfg.heads, cfg.head_dim, cfg.sink_tokens, cfg.chunk_tokens, hist_last, full)
        kc.set_sink(first["k_sink"], first["v_sink"])
        if full:
            kc.set_history(first["k_hist"], first["v_hist"])
        caches.append(kc)
    for c in range(c_first, c_last + 1):
        ch = st.chunk(c)
        d = to_dev(ch)
        for layer, kc in enumerate(caches):
            kc.append(d["k_loc"], d["v_loc"])
            out = f64(s.layer(layer, kc.chunk_inputs(d["q"])))
            torch.cuda.synchronize()
            assert lib.read_status(s.status) == 0
            local = layer == 1
            ref = oracle.streaming_layer(ch["q"], ch["k_sink"], ch["v_sink"], ch["k_loc"],
                                         ch["v_loc"], ch["k_hist"], ch["v_hist"], f64(st.w),
                                         f64(dW) if local else None, local=local)
            assert rel_fro(out, ref) <= ATT_RELFRO + 2 * 2.0 ** -9, (c, local, rel_fro(out, ref))
    # at the last chunk the F-Layer's cache holds its whole history, the L-Layer's none
    assert (caches[0].hist, caches[0].cur) == (hist_last, cfg.chunk_tokens)
    assert (caches[1].hist, caches[1].cur) == (0, cfg.chunk_tokens)


def test_w8a8_projection_vs_oracle(lib):
    """W8A8 projection: the integer codes and scales bit-exact against the
    oracle's (the same fp32 divisions and rounding decide them), the output
    within fp32 scaling of the exact int32 sums; ragged rows."""
    rows, dim = 333, 256
    a = gaussian((rows, dim), 31, 0, "X").to(torch.bfloat16)
    a[5] = 0                                        # an all-zero row: scale 1, codes 0
    W = gaussian((dim, dim), 32, 0, "W") / math.sqrt(dim)
    dW = 0.1 * gaussian((dim, dim), 33, 0, "W") / math.sqrt(dim)
    wq_t, w_scale = lib.ispa_quantize_weight_int8(W.cuda(), dW.cuda())
    ws = torch.empty(lib.ispa_project_w8a8_workspace_size(rows, dim), dtype=torch.uint8,
                     device="cuda")
    out32 = lib.ispa_project_w8a8(a.cuda(), wq_t, w_scale, out_dtype=torch.float32, workspace=ws)
    out16 = lib.ispa_project_w8a8(a.cuda(), wq_t, w_scale)
    torch.cuda.synchronize()
    ref, qa, sa, qwt, sw = oracle.project_w8a8(a, W.numpy(), dW.numpy())
    assert np.array_equal(wq_t.cpu().numpy(), qwt)
    assert np.array_equal(w_scale.cpu().numpy(), sw)
    aq = ws[:rows * dim].view(torch.int8).view(rows, dim).cpu().numpy()
    assert np.array_equal(aq, qa)
    assert rel_fro(f64(out32), ref) <= 1e-6
    assert rel_fro(f64(out16), ref) <= 2.0 ** -8
    assert lib.ispa_project_w8a8(a[:0].cuda(), wq_t, w_scale).shape == (0, dim)


def test_w8a8_full_size_streaming_chunk(lib):
    """The 1.3B chunk shape (4680 rows, d = 1536) on an L-Layer's absorbed
    weight: against the oracle's W8A8 definition on sampled rows, and within
    the quantisation error of the bf16 projection."""
    rows, dim = 4680, 1536
    a = (0.1 * gaussian((rows, dim), 41, 0, "X")).to(torch.bfloat16)
    W = gaussian((dim, dim), 42, 0, "W") / math.sqrt(dim)
    dW = 0.05 * gaussian((dim, dim), 43, 0, "W") / math.sqrt(dim)
    wq_t, w_scale = lib.ispa_quantize_weight_int8(W.cuda(), dW.cuda())
    out = lib.ispa_project_w8a8(a.cuda(), wq_t, w_scale, out_dtype=torch.float32)
    full = lib.ispa_project(a.cuda(), lib.ispa_absorbed_weight(W.cuda(), dW.cuda()),
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    sel = np.linspace(0, rows - 1, 16).astype(int)
    ref = oracle.project_w8a8(a[sel], W.numpy(), dW.numpy())[0]
    assert rel_fro(f64(out)[sel], ref) <= 1e-6
    assert rel_fro(f64(out), f64(full)) <= 2e-2


def test_streaming_resumes_from_a_transition_checkpoint(lib, tmp_path):
    """A small warmup of 4 layers, its transition state written to a file
    (Delta W, lambda, errors, ranking, selection, sinks, the F-Layers'
    history) and read back into fresh streaming buffers: the resumed stream's
    outputs are bit-identical to those of the stream run straight after the
    warmup, and match the oracle's streaming layers."""
    from ispa_synth import Config
    from kv_cache_absorption_b200.checkpoint import (load_transition, resume_streaming,
                                                     save_transition)
    from kv_cache_absorption_b200.streaming import KVCache, StreamingLayers
    from kv_cache_absorption_b200.warmup import LayerWarmup, run_warmup
    cfg = Config("resume", layers=4, heads=2, head_dim=64, tokens_per_frame=96, sink_tokens=40,
                 chunk_frames=1, first_chunk_frame=1, n_chunks=3, history_window=None,
                 select_k=2, stream_chunks=2)
    sts = [layer_streams(scaled(cfg, rho=0.6 + 0.1 * l), l, seed=9) for l in range(cfg.layers)]
    max_hist = (cfg.n_chunks - 1) * cfg.tokens_per_frame
    runner = LayerWarmup(cfg.heads, cfg.head_dim, cfg.chunk_tokens, cfg.sink_tokens,
                         cfg.chunk_tokens, max_hist, n_layers=cfg.layers)
    W_all = torch.stack([st.w for st in sts]).cuda()
    chunks = [[to_dev(st.chunk(c)) for c in range(cfg.n_chunks)] for st in sts]
    err, perm, sel = run_warmup(chunks, W_all, cfg.select_k, runner)
    torch.cuda.synchronize()
    c_first, c_last = cfg.n_chunks, cfg.n_chunks + cfg.stream_chunks - 1
    hist_last = len(cfg.history_frames_of(c_last)) * cfg.tokens_per_frame
    selected = sel.cpu().bool()
    firsts = [to_dev(st.chunk(c_first)) for st in sts]

    def streaming(layers_state, caches):
        outs = []
        for c in range(c_first, c_last + 1):
            for l, st in enumerate(sts):
                d = to_dev(st.chunk(c))
                caches[l].append(d["k_loc"], d["v_loc"])
                outs.append(layers_state.layer(l, caches[l].chunk_inputs(d["q"])).clone())
        torch.cuda.synchronize()
        return outs

    def new_buffers():
        s = StreamingLayers(cfg.heads, cfg.head_dim, cfg.chunk_tokens, cfg.sink_tokens,
                            cfg.chunk_tokens, hist_last, n_layers=cfg.layers)
        kcs = [KVCache(cfg.heads, cfg.head_dim, cfg.sink_tokens, cfg.chunk_tokens, hist_last,
                       not bool(selected[l])) for l in range(cfg.layers)]
        return s, kcs

    # straight after the warmup
    s, kcs = new_buffers()
    s.transition(W_all, runner.dW, selected)
    for l, kc in enumerate(kcs):
        kc.set_sink(firsts[l]["k_sink"], firsts[l]["v_sink"])
        if not bool(selected[l]):
            kc.set_history(firsts[l]["k_hist"], firsts[l]["v_hist"])
    direct = streaming(s, kcs)
    # through the file
    path = str(tmp_path / "transition.pt")
    save_transition(path, runner.dW, runner.lam, err, perm, sel,
                    [f["k_sink"] for f in firsts], [f["v_sink"] for f in firsts],
                    [None if bool(selected[l]) else firsts[l]["k_hist"] for l in range(cfg.layers)],
                    [None if bool(selected[l]) else firsts[l]["v_hist"] for l in range(cfg.layers)])
    del s, kcs
    state = load_transition(path, d=cfg.d, layers=cfg.layers)
    assert torch.equal(state["dW"], runner.dW) and torch.equal(state["err"], err)
    s2, kcs2 = new_buffers()
    resume_streaming(state, W_all, s2, kcs2)
    resumed = streaming(s2, kcs2)
    assert lib.read_status(s2.status) == 0
    for a, b in zip(direct, resumed):
        assert torch.equal(a, b)
    # and the oracle's streaming layers with the GPU's Delta W
    i = 0
    for c in range(c_first, c_last + 1):
        for l, st in enumerate(sts):
            ch = st.chunk(c)
            local = bool(selected[l])
            ref = oracle.streaming_layer(ch["q"], ch["k_sink"], ch["v_sink"], ch["k_loc"],
                                         ch["v_loc"], ch["k_hist"], ch["v_hist"], f64(st.w),
                                         f64(runner.dW[l]) if local else None, local=local)
            assert rel_fro(f64(resumed[i]), ref) <= ATT_RELFRO + 2 * 2.0 ** -9, (c, l)
            i += 1
