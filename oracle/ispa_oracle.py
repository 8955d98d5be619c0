"""Plain, slow, float64 restatement of the ISPA warmup path.

TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and the
benchmark's CPU-baseline leg; never by the library.

Source: "Towards Memory-Efficient Autoregressive Video Generation via
Instance-Specific Parametric Absorption" -- the technical summary (Dutch
page, section 2 "Methodologie", steps 1-3 and "Dynamische Laagselectie";
the Portuguese page repeats it). Step 3 also defines the post-transition
streaming layers (streaming_layer). Notation follows the pages: A_loc,
A_full, W, Delta W, lambda, epsilon, K layers.

Readings where the pages are silent (each also listed in the design notes):
* attention outputs are the per-head softmax(q k^T / sqrt(hd)) v,
  concatenated head-major into rows of d = heads * head_dim;
* "local context" = sink tokens + current chunk; "full" adds the history;
* the matrix norm in the ridge objective is the squared Frobenius norm;
* lambda defaults to 1e-2 * trace(A_loc^T A_loc) / d;
* epsilon is the objective's data term at the optimum, divided by
  ||A_full W||_F^2 so that layers of different scale compare;
* selection: stable ascending sort by epsilon, first K layers.
"""
from __future__ import annotations

import numpy as np


def as_f64(x) -> np.ndarray:
    """Widen a tensor or array (bf16/fp32 included) exactly to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _scores(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """Per-head scaled scores [H, nq, nk] from q [nq, H, hd], k [nk, H, hd]."""
    return np.matmul(q.transpose(1, 0, 2), k.transpose(1, 2, 0)) * scale


def branch_attention(q, k, v, scale):
    """Softmax attention of queries over ONE key set, one head at a time.

    Dutch summary section 2 step 1: each stream is an ordinary attention
    output over its own context. Returns (out [nq, H, hd], lse [H, nq]),
    lse = natural-log log-sum-exp of the scaled scores (-inf for an empty
    key set, whose output is defined as 0).
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    nq, H, hd = q.shape
    if k.shape[0] == 0:
        return np.zeros((nq, H, hd)), np.full((H, nq), -np.inf)
    s = _scores(q, k, scale)                       # [H, nq, nk]
    m = s.max(axis=2, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=2, keepdims=True)
    p = e / z
    out = np.matmul(p, v.transpose(1, 0, 2)).transpose(1, 0, 2)   # [nq, H, hd]
    lse = (m + np.log(z))[:, :, 0]
    return out, lse


def dual_attention(q, k_sink, v_sink, k_loc, v_loc, k_hist, v_hist, scale=None):
    """The two warmup streams of one chunk (Dutch summary section 2 step 1).

    A_loc: attention over sink + current chunk ("lokale context").
    A_full: attention over sink + current chunk + history, computed as a
    SECOND, undecomposed pass over the concatenated keys -- the definition,
    not the pages' LSE-merged shortcut, which the tests check against it.
    Returns a dict with a_loc, a_full, d (= a_full - a_loc), all [nq, d],
    and lse_loc, lse_hist, lse_full [H, nq].
    """
    q = as_f64(q)
    nq, H, hd = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(hd)
    ks, vs = as_f64(k_sink), as_f64(v_sink)
    kl, vl = as_f64(k_loc), as_f64(v_loc)
    kh, vh = as_f64(k_hist), as_f64(v_hist)
    k_l = np.concatenate([ks, kl], axis=0)
    v_l = np.concatenate([vs, vl], axis=0)
    a_loc, lse_loc = branch_attention(q, k_l, v_l, scale)
    a_full, lse_full = branch_attention(q, np.concatenate([k_l, kh], axis=0),
                                        np.concatenate([v_l, vh], axis=0), scale)
    _, lse_hist = branch_attention(q, kh, vh, scale)
    a_loc = a_loc.reshape(nq, H * hd)
    a_full = a_full.reshape(nq, H * hd)
    return {"a_loc": a_loc, "a_full": a_full, "d": a_full - a_loc,
            "lse_loc": lse_loc, "lse_hist": lse_hist, "lse_full": lse_full}


def local_attention(q, k_sink, v_sink, k_loc, v_loc, scale=None):
    """L-Layer attention after the transition (Dutch summary section 2
    step 3): the history is dropped, only sink + current chunk remain."""
    q = as_f64(q)
    nq, H, hd = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(hd)
    out, lse = branch_attention(q, np.concatenate([as_f64(k_sink), as_f64(k_loc)]),
                                np.concatenate([as_f64(v_sink), as_f64(v_loc)]), scale)
    return out.reshape(nq, H * hd), lse


def gram(a_loc, d):
    """Second-moment matrices that the closed form needs (Dutch summary
    section 2 step 2): G = A_loc^T A_loc, R = A_loc^T (A_full - A_loc), and
    S = D^T D for the reconstruction error. Rows are all warmup query rows."""
    a_loc, d = as_f64(a_loc), as_f64(d)
    return a_loc.T @ a_loc, a_loc.T @ d, d.T @ d


def default_lambda(G) -> float:
    """Ridge weight: the pages leave lambda open; 1e-2 * trace(G) / d."""
    G = as_f64(G)
    return 1e-2 * float(np.trace(G)) / G.shape[0]


def absorb(G, R, W, lam):
    """Closed-form weight modulation (Dutch summary section 2 step 2):
    Delta W = (A_loc^T A_loc + lambda I)^-1 A_loc^T (A_full - A_loc) W,
    i.e. the normal equations (G + lambda I) Delta W = R W, solved densely
    (LU via numpy.linalg.solve). Returns (Delta W, B = R W)."""
    G, R, W = as_f64(G), as_f64(R), as_f64(W)
    B = R @ W
    dW = np.linalg.solve(G + lam * np.eye(G.shape[0]), B)
    return dW, B


def reconstruction_error(a_loc, a_full, W, dW):
    """Reconstruction error of a layer (Dutch summary, "Dynamische
    Laagselectie"), materialised directly: E = A_loc (W + dW) - A_full W.
    Returns (||E||_F^2, ||E||_F^2 / ||A_full W||_F^2)."""
    a_loc, a_full, W, dW = as_f64(a_loc), as_f64(a_full), as_f64(W), as_f64(dW)
    target = a_full @ W
    E = a_loc @ (W + dW) - target
    e2 = float(np.sum(E * E))
    return e2, e2 / float(np.sum(target * target))


def rank_layers(eps, K):
    """Instance-specific selection (Dutch summary, "Dynamische
    Laagselectie"): layers ordered by ascending error, ties to the lower
    index; the first K become L-Layers. Returns (perm, selected mask)."""
    eps = np.asarray(eps, dtype=np.float64)
    perm = np.argsort(eps, kind="stable")
    sel = np.zeros(eps.shape[0], dtype=bool)
    sel[perm[:K]] = True
    return perm, sel


def warmup_layer(chunks, W, lam=None):
    """One layer's whole warmup: dual attention on every chunk, stacked rows,
    Gram, lambda, Delta W and epsilon. ``chunks`` is a list of dicts with the
    seven per-chunk tensors of ``dual_attention``."""
    outs = [dual_attention(c["q"], c["k_sink"], c["v_sink"], c["k_loc"], c["v_loc"],
                           c["k_hist"], c["v_hist"]) for c in chunks]
    a_loc = np.concatenate([o["a_loc"] for o in outs], axis=0)
    a_full = np.concatenate([o["a_full"] for o in outs], axis=0)
    G, R, S = gram(a_loc, a_full - a_loc)
    if lam is None:
        lam = default_lambda(G)
    dW, B = absorb(G, R, W, lam)
    e2, eps = reconstruction_error(a_loc, a_full, W, dW)
    return {"chunks": outs, "a_loc": a_loc, "a_full": a_full, "G": G, "R": R, "S": S,
            "lam": lam, "dW": dW, "B": B, "err2": e2, "eps": eps}


def streaming_layer(q, k_sink, v_sink, k_loc, v_loc, k_hist, v_hist, W, dW=None, local=False,
                    scale=None):
    """One layer's output for a chunk after the transition (technical
    summary, section 2, step 3). An L-Layer (``local=True``) keeps only the
    sink and the current chunk and projects with the absorbed weight
    W + Delta W; an F-Layer attends over sink, chunk and history and projects
    with W. Returns the projected rows [nq, d] in float64."""
    W = as_f64(W)
    if local:
        a, _ = local_attention(q, k_sink, v_sink, k_loc, v_loc, scale)
        return a @ (W + (as_f64(dW) if dW is not None else 0.0))
    a = dual_attention(q, k_sink, v_sink, k_loc, v_loc, k_hist, v_hist, scale)["a_full"]
    return a @ W


def quantize_rows_int8(X):
    """Symmetric 8-bit codes per row of a float32 matrix (the W8A8 reading:
    technical summary, results, post-training quantisation): s = max|x| / 127
    (fp32 division; an all-zero row gets s = 1), q = round-half-even(x / s)
    in fp32, clamped to [-127, 127]. Returns (codes int8, scales float32)."""
    X = np.asarray(X, dtype=np.float32)
    mx = np.max(np.abs(X), axis=1)
    s = np.where(mx > 0, mx / np.float32(127.0), np.float32(1.0)).astype(np.float32)
    q = np.rint(X / s[:, None]).clip(-127, 127).astype(np.int8)
    return q, s


def project_w8a8(a, W, dW=None):
    """W8A8 projection of a streaming layer: activations a [rows, d] (bf16
    values) quantised per row, W' = W (+ Delta W, summed in fp32) quantised
    per output column; out = s_a s_w sum_k q_a q_w, in float64. Returns
    (out, q_a, s_a, q_w^T, s_w)."""
    A32 = as_f64(a).astype(np.float32)
    Wp = np.asarray(as_f64(W), dtype=np.float32)
    if dW is not None:
        Wp = Wp + np.asarray(as_f64(dW), dtype=np.float32)
    qa, sa = quantize_rows_int8(A32)
    qwt, sw = quantize_rows_int8(Wp.T)          # columns of W' = rows of its transpose
    acc = qa.astype(np.int64) @ qwt.astype(np.int64).T
    out = acc.astype(np.float64) * sa.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :]
    return out, qa, sa, qwt, sw
