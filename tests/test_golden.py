"""The oracle still reproduces its frozen tiny-workload digest (see
tests/golden/make_golden.py for how and why it was written)."""
import json
import os

import numpy as np

from tests.golden.make_golden import digest

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_frozen_digest():
    with open(os.path.join(HERE, "c0_oracle.json")) as f:
        ref = json.load(f)
    now = digest()
    for key, val in ref.items():
        if key == "workload":
            continue
        np.testing.assert_allclose(np.asarray(now[key]), np.asarray(val), rtol=1e-9, atol=1e-12,
                                   err_msg=key)


WARMUPS = ("c2", "c2r", "c3")


def test_warmup_digests_are_consistent():
    """The stored oracle digests of the full warmups (written by
    tests/golden/make_warmup_golden.py) satisfy what the method fixes: the
    ranking is the stable ascending order of epsilon and selects its first K
    layers; epsilon = ||E||^2 / ||A_full W||^2; 0 <= epsilon <= epsilon with
    Delta W = 0 (Delta W minimises a convex objective that includes the
    choice Delta W = 0); lambda > 0; the workload's correlations as the input
    generator states them."""
    from ispa_synth import CONFIGS
    for name in WARMUPS:
        path = os.path.join(HERE, f"{name}_warmup_oracle.npz")
        z = np.load(path)
        cfg = CONFIGS[name]
        L, K = cfg.layers, cfg.select_k
        meta = json.loads(str(z["meta"]))
        assert meta["K"] == K and len(meta["rho"]) == L
        np.testing.assert_allclose(meta["rho"], [cfg.rho_of(l) for l in range(L)])
        eps = z["eps"]
        assert eps.shape == (L,)
        assert z["perm"].tolist() == np.argsort(eps, kind="stable").tolist()
        assert z["sel"].tolist() == [l in set(z["perm"][:K].tolist()) for l in range(L)]
        np.testing.assert_allclose(eps, z["err2"] / z["tgt2"], rtol=1e-12)
        assert np.all(eps > 0) and np.all(eps <= z["eps0"])
        assert np.all(z["lam"] > 0) and np.all(z["dW_fro"] > 0)
        for key in ("sk_G", "sk_R", "sk_S", "sk_dW", "sk_aloc", "sk_afull"):
            assert z[key].shape == (L, 16, 16) and np.all(np.isfinite(z[key]))
        assert z["dW_rows"].shape == (L, 3, cfg.d)
