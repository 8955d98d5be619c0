"""Writes the float64 oracle's digest of the full warmups:
``c2_warmup_oracle.npz`` (1.3B: 30 layers, d = 1536), ``c2r_warmup_oracle.npz``
(the same with per-layer correlations spread over [0.5, 0.95], a
ranking-stress addition) and ``c3_warmup_oracle.npz`` (14B: 40 layers,
d = 5120). Four warmup chunks of 4680 query rows per layer, seed 0.

Every number in these files comes from ``oracle`` on inputs from
``ispa_synth``; nothing here calls the CUDA library. The oracle computes each
layer as the technical summary states it (section 2, steps 1-2 and
"Dynamische Laagselectie"): two separate softmax passes per chunk (local keys;
all keys), the stacked rows' Gram matrices, lambda, the dense normal-equation
solve for Delta W, the directly materialised reconstruction error, and the
stable ranking. Heads are independent, so each head of a chunk is passed to
the oracle on its own (the all-heads score tensor of the 14B chunk would not
fit in host memory) and the outputs are concatenated head-major.

A layer's full results are too large to store, so the file keeps:
  eps, err2, tgt2 (= ||A_full W||^2), eps0 (error with Delta W = 0), lam,
  dW_fro, G_fro, R_fro, S_fro  -- one value per layer;
  perm, sel                    -- the oracle's ranking and selected layers;
  sk_G, sk_R, sk_S, sk_dW      -- two-sided sketches L^T X R, [k, k];
  sk_aloc, sk_afull            -- sketches P^T X L of the stacked attention
                                  rows (P over the rows, L over channels);
  dW_rows                      -- rows ``DW_ROWS`` of Delta W, float32;
with (P, L, R) = ``ispa_synth.sketch_matrices(rows, d)``.

Run from the repository root (hours of CPU for the 14B warmup; per-layer
results are cached, so an interrupted run resumes):
    python tests/golden/make_warmup_golden.py --configs c2,c2r,c3 --workers 3
"""
import argparse
import json
import multiprocessing as mp
import os
import sys
import tempfile
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

KEYS = ("q", "k_sink", "v_sink", "k_loc", "v_loc", "k_hist", "v_hist")
SEED = 0


def dw_rows(d):
    return [5, d // 2 + 3, d - 2]


def layer_digest(name, layer, cache, threads):
    """One layer's oracle results, reduced to the digest above (cached)."""
    path = os.path.join(cache, f"{name}_l{layer:02d}.npz")
    if os.path.exists(path):
        return path
    import threadpoolctl
    import torch
    torch.set_num_threads(1)
    import oracle
    from ispa_synth import CONFIGS, layer_streams, sketch_matrices
    cfg = CONFIGS[name]
    t0 = time.time()
    with threadpoolctl.threadpool_limits(threads):
        st = layer_streams(cfg, layer, seed=SEED)
        a_loc, a_full = [], []
        for c in range(cfg.n_chunks):
            ch = st.chunk(c)
            heads = [oracle.dual_attention(*(ch[k][:, h:h + 1] for k in KEYS))
                     for h in range(cfg.heads)]
            a_loc.append(np.concatenate([o["a_loc"] for o in heads], axis=1))
            a_full.append(np.concatenate([o["a_full"] for o in heads], axis=1))
            del heads
        a_loc = np.concatenate(a_loc, axis=0)
        a_full = np.concatenate(a_full, axis=0)
        W = oracle.as_f64(st.w)
        del st
        G, R, S = oracle.gram(a_loc, a_full - a_loc)
        lam = oracle.default_lambda(G)
        dW, B = oracle.absorb(G, R, W, lam)
        err2, eps = oracle.reconstruction_error(a_loc, a_full, W, dW)
        err0, eps0 = oracle.reconstruction_error(a_loc, a_full, W, np.zeros_like(W))
        P, Lm, Rm = (oracle.as_f64(x) for x in sketch_matrices(a_loc.shape[0], cfg.d))
        two = lambda X: Lm.T @ X @ Rm
        out = dict(
            eps=eps, err2=err2, tgt2=err2 / eps, eps0=eps0, lam=lam,
            dW_fro=np.linalg.norm(dW), G_fro=np.linalg.norm(G), R_fro=np.linalg.norm(R),
            S_fro=np.linalg.norm(S),
            sk_G=two(G), sk_R=two(R), sk_S=two(S), sk_dW=two(dW),
            sk_aloc=P.T @ a_loc @ Lm, sk_afull=P.T @ a_full @ Lm,
            dW_rows=dW[dw_rows(cfg.d)].astype(np.float32))
    np.savez(path + ".tmp.npz", **out)
    os.replace(path + ".tmp.npz", path)
    print(f"{name} layer {layer}: eps {eps:.6f} ({time.time() - t0:.0f} s)", flush=True)
    return path


def assemble(name, cache):
    from ispa_synth import CONFIGS
    import oracle
    cfg = CONFIGS[name]
    per = [dict(np.load(os.path.join(cache, f"{name}_l{l:02d}.npz"))) for l in range(cfg.layers)]
    out = {k: np.stack([p[k] for p in per]) for k in per[0]}
    perm, sel = oracle.rank_layers(out["eps"], cfg.select_k)
    out["perm"], out["sel"] = perm.astype(np.int32), sel
    out["meta"] = np.array(json.dumps({
        "workload": f"{cfg.name}: {cfg.layers} layers, {cfg.heads} heads x {cfg.head_dim}, "
                    f"{cfg.n_chunks} chunks x {cfg.chunk_tokens} rows, sink {cfg.sink_tokens}, "
                    f"seed {SEED}",
        "rho": [cfg.rho_of(l) for l in range(cfg.layers)],
        "K": cfg.select_k, "dw_rows": dw_rows(cfg.d)}))
    dst = os.path.join(HERE, f"{name}_warmup_oracle.npz")
    np.savez_compressed(dst, **out)
    print("wrote", dst)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--configs", default="c2,c2r,c3")
    ap.add_argument("--workers", type=int, default=3)
    ap.add_argument("--threads", type=int, default=2)
    ap.add_argument("--cache", default=os.path.join(tempfile.gettempdir(), "ispa_warmup_golden"))
    a = ap.parse_args()
    os.makedirs(a.cache, exist_ok=True)
    # Large temporaries: keep freed memory in the process instead of handing
    # it back to the OS and faulting it in again for every head.
    os.environ.setdefault("MALLOC_MMAP_MAX_", "0")
    os.environ.setdefault("MALLOC_TRIM_THRESHOLD_", str(1 << 40))
    from ispa_synth import CONFIGS
    names = a.configs.split(",")
    jobs = [(n, l, a.cache, a.threads) for n in names for l in range(CONFIGS[n].layers)]
    with mp.get_context("spawn").Pool(a.workers, maxtasksperchild=None) as pool:
        pool.starmap(layer_digest, jobs, chunksize=1)
    for n in names:
        assemble(n, a.cache)


if __name__ == "__main__":
    main()
