"""Pins for the float64 oracle: each checks it against something other than
itself -- closed forms, a library routine, brute force, invariants -- so that
a dropped term, a wrong sign, a wrong index or a transposed operand anywhere
in it fails at least one test. CPU only."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import (absorb, branch_attention, default_lambda, dual_attention, gram,
                    local_attention, rank_layers, reconstruction_error, warmup_layer)

RNG = np.random.default_rng(1234)


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


# ---------------------------------------------------------------- attention

def sdpa(q, k, v, scale):
    """torch's own attention (CPU, float64) as an independent library routine."""
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]   # [1, H, nq, hd]
    kt = torch.from_numpy(k).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2)[None]
    out = F.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return out[0].permute(1, 0, 2).numpy()


def test_branch_matches_library_attention():
    q, k, v = rand(7, 3, 8), rand(19, 3, 8), rand(19, 3, 8)
    out, _ = branch_attention(q, k, v, 0.37)
    np.testing.assert_allclose(out, sdpa(q, k, v, 0.37), rtol=0, atol=1e-12)


def test_dual_matches_library_on_both_streams():
    H, hd = 2, 16
    q = rand(9, H, hd)
    ks, vs = rand(3, H, hd), rand(3, H, hd)
    kl, vl = rand(5, H, hd), rand(5, H, hd)
    kh, vh = rand(11, H, hd), rand(11, H, hd)
    o = dual_attention(q, ks, vs, kl, vl, kh, vh)
    sc = 1 / math.sqrt(hd)
    ref_loc = sdpa(q, np.concatenate([ks, kl]), np.concatenate([vs, vl]), sc).reshape(9, -1)
    ref_full = sdpa(q, np.concatenate([ks, kl, kh]), np.concatenate([vs, vl, vh]), sc).reshape(9, -1)
    np.testing.assert_allclose(o["a_loc"], ref_loc, atol=1e-12, rtol=0)
    np.testing.assert_allclose(o["a_full"], ref_full, atol=1e-12, rtol=0)
    np.testing.assert_allclose(o["d"], ref_full - ref_loc, atol=1e-12, rtol=0)


def test_zero_query_gives_mean_and_log_n():
    k, v = rand(13, 2, 4), rand(13, 2, 4)
    out, lse = branch_attention(np.zeros((3, 2, 4)), k, v, 0.5)
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(0), out.shape), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(13), atol=1e-14)


def test_single_key_returns_its_value_and_score():
    q, k, v = rand(4, 1, 6), rand(1, 1, 6), rand(1, 1, 6)
    out, lse = branch_attention(q, k, v, 0.3)
    np.testing.assert_allclose(out, np.broadcast_to(v[0], out.shape), atol=1e-14)
    np.testing.assert_allclose(lse[0], 0.3 * (q[:, 0] @ k[0, 0]), atol=1e-14)


def test_two_keys_closed_form():
    # softmax over two scores is the logistic function; worked with Python floats
    q, k, v = rand(1, 1, 3), rand(2, 1, 3), rand(2, 1, 3)
    s1 = float(q[0, 0] @ k[0, 0]) * 0.8
    s2 = float(q[0, 0] @ k[1, 0]) * 0.8
    w1 = 1.0 / (1.0 + math.exp(s2 - s1))
    out, lse = branch_attention(q, k, v, 0.8)
    np.testing.assert_allclose(out[0, 0], w1 * v[0, 0] + (1 - w1) * v[1, 0], atol=1e-14)
    assert abs(lse[0, 0] - (max(s1, s2) + math.log1p(math.exp(-abs(s1 - s2))))) < 1e-13


def test_hand_worked_example():
    # scale 1, one head of width 1: q = 1, keys 0 and log 3 -> weights 1/4, 3/4;
    # values 4 and 8 -> output 7; log-sum-exp = log(1 + 3) = log 4.
    q = np.array([[[1.0]]])
    k = np.array([[[0.0]], [[math.log(3.0)]]])
    v = np.array([[[4.0]], [[8.0]]])
    out, lse = branch_attention(q, k, v, 1.0)
    assert abs(out[0, 0, 0] - 7.0) < 1e-14
    assert abs(lse[0, 0] - math.log(4.0)) < 1e-14


def test_permuting_keys_changes_nothing():
    q = rand(5, 2, 8)
    ks, vs, kl, vl, kh, vh = (rand(n, 2, 8) for n in (4, 4, 6, 6, 9, 9))
    a = dual_attention(q, ks, vs, kl, vl, kh, vh)
    pl, ph = RNG.permutation(6), RNG.permutation(9)
    b = dual_attention(q, ks, vs, kl[pl], vl[pl], kh[ph], vh[ph])
    for key in ("a_loc", "a_full", "lse_loc", "lse_hist", "lse_full"):
        np.testing.assert_allclose(a[key], b[key], atol=1e-13)


def test_lse_merge_equals_undecomposed_pass():
    """Decomposable attention (Dutch summary section 2 step 1): the local and
    history branches, merged by their LSE weights, give the full output."""
    q = rand(6, 3, 16, scale=1.5)
    ks, vs, kl, vl, kh, vh = (rand(n, 3, 16) for n in (5, 5, 7, 7, 20, 20))
    o = dual_attention(q, ks, vs, kl, vl, kh, vh)
    a_hist, lse_hist = branch_attention(q, kh, vh, 0.25)
    np.testing.assert_allclose(lse_hist, o["lse_hist"], atol=1e-13)
    lse_full = np.logaddexp(o["lse_loc"], o["lse_hist"])            # [H, nq]
    np.testing.assert_allclose(lse_full, o["lse_full"], atol=1e-12)
    w_loc = np.exp(o["lse_loc"] - lse_full).T[:, :, None]          # [nq, H, 1]
    w_hist = np.exp(o["lse_hist"] - lse_full).T[:, :, None]
    merged = w_loc * o["a_loc"].reshape(6, 3, 16) + w_hist * a_hist
    np.testing.assert_allclose(merged.reshape(6, -1), o["a_full"], atol=1e-12, rtol=0)


def test_empty_history_and_empty_sink():
    q = rand(4, 2, 8)
    kl, vl = rand(5, 2, 8), rand(5, 2, 8)
    e = np.zeros((0, 2, 8))
    o = dual_attention(q, e, e, kl, vl, e, e)
    assert np.all(np.isneginf(o["lse_hist"]))
    assert np.all(np.isfinite(o["a_full"])) and np.all(np.isfinite(o["lse_full"]))
    np.testing.assert_array_equal(o["a_full"], o["a_loc"])
    np.testing.assert_array_equal(o["d"], 0.0)
    np.testing.assert_array_equal(o["lse_full"], o["lse_loc"])


def test_large_scores_do_not_overflow():
    q = rand(3, 1, 8, scale=300.0)
    k, v = rand(10, 1, 8), rand(10, 1, 8)
    out, lse = branch_attention(q, k, v, 1.0)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    # the output is a convex combination of the values
    assert np.all(out <= v.max(0) + 1e-12) and np.all(out >= v.min(0) - 1e-12)


def test_local_attention_equals_dual_local_stream():
    q = rand(5, 2, 8)
    ks, vs, kl, vl, kh, vh = (rand(n, 2, 8) for n in (3, 3, 4, 4, 6, 6))
    a, lse = local_attention(q, ks, vs, kl, vl)
    o = dual_attention(q, ks, vs, kl, vl, kh, vh)
    np.testing.assert_array_equal(a, o["a_loc"])
    np.testing.assert_array_equal(lse, o["lse_loc"])


# ---------------------------------------------------------------- absorption

def ridge_problem(n=40, d=6, seed=0):
    r = np.random.default_rng(seed)
    a_loc = r.standard_normal((n, d)) + 0.5
    a_full = a_loc + 0.3 * r.standard_normal((n, d))
    W = r.standard_normal((d, d)) / math.sqrt(d)
    return a_loc, a_full, W


def objective(a_loc, a_full, W, dW, lam):
    """The ridge objective exactly as the pages write it (Frobenius norms)."""
    E = a_loc @ (W + dW) - a_full @ W
    return float(np.sum(E * E) + lam * np.sum(dW * dW))


def test_gram_blocks_by_definition():
    a, f, _ = ridge_problem()
    G, R, S = gram(a, f - a)
    n, d = a.shape
    for i, j in [(0, 0), (1, 4), (5, 2)]:
        assert abs(G[i, j] - sum(a[t, i] * a[t, j] for t in range(n))) < 1e-10
        assert abs(R[i, j] - sum(a[t, i] * (f[t, j] - a[t, j]) for t in range(n))) < 1e-10
        assert abs(S[i, j] - sum((f[t, i] - a[t, i]) * (f[t, j] - a[t, j]) for t in range(n))) < 1e-10


def test_normal_equations_hold():
    a, f, W = ridge_problem(200, 16)
    G, R, _ = gram(a, f - a)
    lam = default_lambda(G)
    dW, B = absorb(G, R, W, lam)
    res = (G + lam * np.eye(16)) @ dW - R @ W
    assert np.linalg.norm(res) / np.linalg.norm(R @ W) < 1e-10
    np.testing.assert_allclose(B, R @ W, atol=1e-12)


def test_default_lambda_is_one_percent_of_mean_diagonal():
    G = np.diag([1.0, 2.0, 3.0, 6.0])
    assert abs(default_lambda(G) - 0.03) < 1e-15


def test_no_discrepancy_gives_zero_update():
    a, _, W = ridge_problem()
    G, R, _ = gram(a, np.zeros_like(a))
    dW, _ = absorb(G, R, W, 0.1)
    assert np.max(np.abs(dW)) == 0.0


def test_large_lambda_limit():
    a, f, W = ridge_problem()
    G, R, _ = gram(a, f - a)
    for lam in (1e6, 1e8):
        dW, _ = absorb(G, R, W, lam)
        rel = np.linalg.norm(lam * dW - R @ W) / np.linalg.norm(R @ W)
        assert rel < 10 * np.linalg.norm(G, 2) / lam


def test_matches_stacked_least_squares():
    """A different algorithm (SVD least squares on the augmented system
    [A_loc; sqrt(lambda) I] dW = [(A_full - A_loc) W; 0])."""
    a, f, W = ridge_problem(60, 8)
    lam = 0.7
    G, R, _ = gram(a, f - a)
    dW, _ = absorb(G, R, W, lam)
    lhs = np.vstack([a, math.sqrt(lam) * np.eye(8)])
    rhs = np.vstack([(f - a) @ W, np.zeros((8, 8))])
    ref = np.linalg.lstsq(lhs, rhs, rcond=None)[0]
    np.testing.assert_allclose(dW, ref, atol=1e-9, rtol=0)


def test_brute_force_minimum_tiny():
    """d = 3, N = 8: a derivative-free search over the objective the pages
    print reaches the closed-form minimiser; no perturbation beats it."""
    from scipy.optimize import minimize
    a, f, W = ridge_problem(8, 3, seed=5)
    lam = 0.2
    G, R, _ = gram(a, f - a)
    dW, _ = absorb(G, R, W, lam)
    fun = lambda x: objective(a, f, W, x.reshape(3, 3), lam)
    best = minimize(fun, np.zeros(9), method="Nelder-Mead",
                    options={"xatol": 1e-11, "fatol": 1e-14, "maxiter": 40000, "maxfev": 40000})
    np.testing.assert_allclose(best.x.reshape(3, 3), dW, atol=1e-6)
    f0 = fun(dW.ravel())
    r = np.random.default_rng(3)
    for _ in range(200):
        assert fun(dW.ravel() + 1e-3 * r.standard_normal(9)) > f0


def test_planted_solution_is_recovered():
    r = np.random.default_rng(9)
    a = r.standard_normal((100, 5))
    M = 0.2 * r.standard_normal((5, 5))
    f = a @ (np.eye(5) + M)
    W = r.standard_normal((5, 5))
    G, R, S = gram(a, f - a)
    lam = 1e-12 * np.trace(G) / 5
    dW, _ = absorb(G, R, W, lam)
    np.testing.assert_allclose(dW, M @ W, atol=1e-8)
    _, eps = reconstruction_error(a, f, W, dW)
    assert eps < 1e-16


# ---------------------------------------------------------------- epsilon

def test_error_identity_form_matches_direct():
    """||E||^2 = tr(W^T S W) - <dW, B> - lambda ||dW||^2 and
    ||A_full W||^2 = <G + R + R^T + S, W W^T>, both from (G + lambda I) dW = B."""
    a, f, W = ridge_problem(300, 12, seed=2)
    G, R, S = gram(a, f - a)
    lam = default_lambda(G)
    dW, B = absorb(G, R, W, lam)
    e2, eps = reconstruction_error(a, f, W, dW)
    e2_id = np.trace(W.T @ S @ W) - np.sum(dW * B) - lam * np.sum(dW * dW)
    den_id = np.sum((G + R + R.T + S) * (W @ W.T))
    assert abs(e2_id - e2) / e2 < 1e-10
    assert abs(e2 / den_id - eps) / eps < 1e-10


def test_error_bounded_by_no_absorb_case():
    a, f, W = ridge_problem(120, 10, seed=4)
    G, R, _ = gram(a, f - a)
    lam = default_lambda(G)
    dW, _ = absorb(G, R, W, lam)
    _, eps = reconstruction_error(a, f, W, dW)
    _, eps0 = reconstruction_error(a, f, W, np.zeros_like(dW))
    assert 0.0 <= eps < eps0
    assert abs(eps0 - np.sum(((f - a) @ W) ** 2) / np.sum((f @ W) ** 2)) < 1e-14


# ---------------------------------------------------------------- ranking

def test_rank_hand_example_with_ties():
    perm, sel = rank_layers([0.3, 0.1, 0.3, 0.1, 0.2], 2)
    assert list(perm) == [1, 3, 4, 0, 2]
    assert list(np.flatnonzero(sel)) == [1, 3]


def test_rank_is_a_stable_ascending_order():
    r = np.random.default_rng(7)
    eps = r.integers(0, 6, size=40) / 7.0
    perm, sel = rank_layers(eps, 20)
    assert list(perm) == sorted(range(40), key=lambda i: (eps[i], i))
    assert sel.sum() == 20 and all(sel[i] for i in perm[:20])


# ---------------------------------------------------------------- composition

def test_tiny_warmup_layer_end_to_end():
    from ispa_synth import C0, layer_streams
    st = layer_streams(C0, 0, seed=0)
    chunks = [st.chunk(c) for c in range(C0.n_chunks)]
    out = warmup_layer(chunks, st.w)
    assert out["a_loc"].shape == (512, 128)
    G = out["G"]
    res = (G + out["lam"] * np.eye(128)) @ out["dW"] - out["B"]
    assert np.linalg.norm(res) / np.linalg.norm(out["B"]) < 1e-10
    _, eps0 = reconstruction_error(out["a_loc"], out["a_full"], oracle.as_f64(st.w),
                                   np.zeros((128, 128)))
    assert 0 < out["eps"] < eps0
    for o in out["chunks"]:
        assert np.all(o["lse_full"] >= np.maximum(o["lse_loc"], o["lse_hist"]) - 1e-12)


# ---------------------------------------------------------------- planted mistakes

def _absorb_pins_pass(absorb_fn):
    """The absorb pins above, as one predicate over a candidate solver."""
    a, f, W = ridge_problem(8, 3, seed=5)
    lam = 0.2
    G, R, _ = gram(a, f - a)
    dW = absorb_fn(G, R, W, lam)
    f0 = objective(a, f, W, dW, lam)
    r = np.random.default_rng(3)
    never_beaten = all(objective(a, f, W, dW + 1e-3 * r.standard_normal((3, 3)), lam) > f0
                       for _ in range(200))
    lhs = np.vstack([a, math.sqrt(lam) * np.eye(3)])
    rhs = np.vstack([(f - a) @ W, np.zeros((3, 3))])
    ref = np.linalg.lstsq(lhs, rhs, rcond=None)[0]
    return never_beaten and np.allclose(dW, ref, atol=1e-9, rtol=0)


@pytest.mark.parametrize("mutant", [
    lambda G, R, W, lam: np.linalg.solve(G + lam * np.eye(len(G)), R.T @ W),   # R transposed
    lambda G, R, W, lam: np.linalg.solve(G + lam * np.eye(len(G)), R @ W.T),   # W transposed
    lambda G, R, W, lam: np.linalg.solve(G, R @ W),                            # lambda dropped
    lambda G, R, W, lam: np.linalg.solve(G - lam * np.eye(len(G)), R @ W),     # sign of lambda
    lambda G, R, W, lam: np.linalg.solve(G + lam * np.eye(len(G)), -R @ W),    # sign of D
])
def test_absorb_pins_catch_planted_mistakes(mutant):
    assert _absorb_pins_pass(lambda G, R, W, lam: absorb(G, R, W, lam)[0])
    assert not _absorb_pins_pass(mutant)


def test_attention_pins_catch_planted_mistakes():
    q, k, v = rand(7, 3, 8), rand(19, 3, 8), rand(19, 3, 8)
    ref = sdpa(q, k, v, 0.37)
    good, _ = branch_attention(q, k, v, 0.37)
    assert np.allclose(good, ref, atol=1e-12)
    # wrong scale, keys of another head, values not permuted with keys
    bad1, _ = branch_attention(q, k, v, 0.37 * 1.01)
    bad2, _ = branch_attention(q, k[:, ::-1], v, 0.37)
    bad3, _ = branch_attention(q, k, v[::-1], 0.37)
    for bad in (bad1, bad2, bad3):
        assert not np.allclose(bad, ref, atol=1e-12)


# ---------------------------------------------------------------- streaming layers

def test_streaming_f_layer_is_library_attention_times_w():
    """An F-Layer's output is softmax attention over every key (here torch's
    own attention on the concatenated keys) projected with W."""
    q = rand(6, 2, 8)
    ks, vs, kl, vl, kh, vh = (rand(n, 2, 8) for n in (3, 3, 5, 5, 9, 9))
    W, dW = rand(16, 16), rand(16, 16)
    got = oracle.streaming_layer(q, ks, vs, kl, vl, kh, vh, W, dW, local=False)
    ref = sdpa(q, np.concatenate([ks, kl, kh]), np.concatenate([vs, vl, vh]), 8 ** -0.5)
    np.testing.assert_allclose(got, ref.reshape(6, 16) @ W, rtol=0, atol=1e-12)


def test_streaming_l_layer_drops_history_and_uses_absorbed_weight():
    q = rand(6, 2, 8)
    ks, vs, kl, vl, kh, vh = (rand(n, 2, 8) for n in (3, 3, 5, 5, 9, 9))
    W, dW = rand(16, 16), rand(16, 16)
    got = oracle.streaming_layer(q, ks, vs, kl, vl, kh, vh, W, dW, local=True)
    ref = sdpa(q, np.concatenate([ks, kl]), np.concatenate([vs, vl]), 8 ** -0.5)
    np.testing.assert_allclose(got, ref.reshape(6, 16) @ (W + dW), rtol=0, atol=1e-12)
    # the history does not enter an L-Layer
    got2 = oracle.streaming_layer(q, ks, vs, kl, vl, 3 * kh, vh + 1, W, dW, local=True)
    np.testing.assert_array_equal(got, got2)
    # with no history and no absorption both layer kinds coincide
    f = oracle.streaming_layer(q, ks, vs, kl, vl, kh[:0], vh[:0], W, None, local=False)
    l0 = oracle.streaming_layer(q, ks, vs, kl, vl, kh[:0], vh[:0], W, None, local=True)
    np.testing.assert_allclose(f, l0, rtol=0, atol=1e-13)


def test_streaming_l_layer_with_absorbed_weight_tracks_full_layer():
    """Delta W absorbed on a chunk's own rows brings the L-Layer's output on
    that chunk closer to the F-Layer's than Delta W = 0 does (the ridge
    objective includes Delta W = 0)."""
    q = rand(40, 2, 8)
    ks, vs, kl, vl, kh, vh = (rand(n, 2, 8) for n in (3, 3, 6, 6, 30, 30))
    W = rand(16, 16, scale=0.25)
    o = dual_attention(q, ks, vs, kl, vl, kh, vh)
    G, R, _ = gram(o["a_loc"], o["d"])
    dW, _ = absorb(G, R, W, default_lambda(G))
    full = oracle.streaming_layer(q, ks, vs, kl, vl, kh, vh, W, local=False)
    l_abs = oracle.streaming_layer(q, ks, vs, kl, vl, kh, vh, W, dW, local=True)
    l_raw = oracle.streaming_layer(q, ks, vs, kl, vl, kh, vh, W, None, local=True)
    assert np.sum((l_abs - full) ** 2) < np.sum((l_raw - full) ** 2)


# ---------------------------------------------------------------- W8A8 projection

def test_int8_codes_scale_and_rounding():
    X = np.array([[0.0, 0.0, 0.0], [1.0, -2.0, 0.5], [127.0, 0.5, 1.5]], dtype=np.float32)
    q, s = oracle.quantize_rows_int8(X)
    assert s[0] == 1.0 and not q[0].any()                       # zero row
    assert s[1] == np.float32(2.0) / np.float32(127.0)
    assert list(q[1]) == [64, -127, 32]                            # 63.5 -> 64 (half to even), 31.75 -> 32
    assert s[2] == 1.0 and list(q[2]) == [127, 0, 2]              # 0.5 -> 0 and 1.5 -> 2: half to even
    r = np.random.default_rng(3).standard_normal((50, 64)).astype(np.float32)
    q, s = oracle.quantize_rows_int8(r)
    assert np.all(np.abs(q) <= 127) and np.all(np.abs(q).max(axis=1) == 127)
    # dequantisation error at most half a step per element
    assert np.all(np.abs(q * s[:, None] - r) <= 0.5 * s[:, None] * (1 + 1e-6))


def test_w8a8_exact_on_integer_grids():
    """Rows whose largest magnitude is 127 and whose entries are integers get
    scale 1 and exact codes: the W8A8 product is then the exact product."""
    r = np.random.default_rng(5)
    a = r.integers(-127, 128, size=(20, 32)).astype(np.float32)
    a[:, 0] = 127
    W = r.integers(-127, 128, size=(32, 16)).astype(np.float32)
    W[0, :] = -127
    out, qa, sa, qwt, sw = oracle.project_w8a8(a, W)
    assert np.all(sa == 1) and np.all(sw == 1)
    np.testing.assert_array_equal(out, a.astype(np.float64) @ W.astype(np.float64))


def test_w8a8_close_to_full_precision_product():
    r = np.random.default_rng(6)
    a = r.standard_normal((200, 256)).astype(np.float32)
    W = (r.standard_normal((256, 256)) / 16).astype(np.float32)
    dW = (0.1 * r.standard_normal((256, 256)) / 16).astype(np.float32)
    out = oracle.project_w8a8(a, W, dW)[0]
    ref = a.astype(np.float64) @ (W + dW).astype(np.float64)
    err = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    # per-element rounding of both operands: about (max/127)/sqrt(12) each
    assert 1e-4 < err < 2e-2
    # the sum of W and Delta W is taken before quantising
    out_w = oracle.project_w8a8(a, W + dW)[0]
    np.testing.assert_array_equal(out, out_w)
