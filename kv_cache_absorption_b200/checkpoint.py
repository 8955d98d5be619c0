"""Checkpoint of the transition state, so that streaming resumes without
redoing the warmup.

"Towards Memory-Efficient Autoregressive Video Generation via
Instance-Specific Parametric Absorption", technical summary section 2,
step 3: at the end of the warmup every layer has its Delta W and its
reconstruction error, and the K lowest-error layers become L-Layers, which
keep only the sink and the current chunk. What the stream needs from the
warmup is therefore: per layer Delta W (fp32), lambda and the error pair
{||E||^2, epsilon}; the ranking and the selected layers; every layer's sink
keys and values. An F-Layer also attends over its history, so the
checkpoint may carry the F-Layers' history keys and values as well (without
them a caller re-supplies the history from its own KV store). The model
weights W are not part of it: they belong to the model, not the instance.

Format: one ``torch.save`` file of CPU tensors with a format tag and the
geometry; ``load_transition`` checks both before anything is used.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

FORMAT = "ispa-transition-v1"


def save_transition(path: str, dW: torch.Tensor, lam: torch.Tensor, err: torch.Tensor,
                    perm: torch.Tensor, selected: torch.Tensor, sink_k: Sequence[torch.Tensor],
                    sink_v: Sequence[torch.Tensor],
                    hist_k: Optional[Sequence[Optional[torch.Tensor]]] = None,
                    hist_v: Optional[Sequence[Optional[torch.Tensor]]] = None,
                    meta: Optional[dict] = None) -> None:
    """Writes the transition state. dW [L, d, d] fp32; lam [L] fp32; err
    [L, 2] fp64; perm [L] int32; selected [L] (bool or uint8); sink_k/sink_v:
    L tensors [sink, heads, head_dim] bf16; hist_k/hist_v (optional): L
    entries, an F-Layer's history [n, heads, head_dim] bf16 or None (for an
    L-Layer, which keeps none)."""
    L, d, d2 = dW.shape
    if d != d2 or lam.shape != (L,) or err.shape != (L, 2) or perm.shape != (L,) \
            or selected.shape != (L,) or len(sink_k) != L or len(sink_v) != L:
        raise ValueError("inconsistent transition state")
    sel = selected.detach().to("cpu").bool()
    state = {
        "format": FORMAT, "layers": L, "d": d,
        "dW": dW.detach().to("cpu", torch.float32),
        "lambda": lam.detach().to("cpu", torch.float32),
        "err": err.detach().to("cpu", torch.float64),
        "perm": perm.detach().to("cpu", torch.int32),
        "selected": sel,
        "sink_k": [k.detach().to("cpu") for k in sink_k],
        "sink_v": [v.detach().to("cpu") for v in sink_v],
        "meta": dict(meta or {}),
    }
    if hist_k is not None:
        if hist_v is None or len(hist_k) != L or len(hist_v) != L:
            raise ValueError("history keys and values must be given for every layer")
        for l in range(L):
            if bool(sel[l]) and (hist_k[l] is not None or hist_v[l] is not None):
                raise ValueError(f"layer {l} is an L-Layer: it keeps no history")
        state["hist_k"] = [None if k is None else k.detach().to("cpu") for k in hist_k]
        state["hist_v"] = [None if v is None else v.detach().to("cpu") for v in hist_v]
    torch.save(state, path)


def load_transition(path: str, device="cuda", d: Optional[int] = None,
                    layers: Optional[int] = None) -> dict:
    """Reads a transition state written by ``save_transition``; tensors go to
    ``device``. Raises ValueError on another format or on a geometry other
    than the given ``d`` / ``layers``."""
    state = torch.load(path, map_location="cpu", weights_only=False)
    if not isinstance(state, dict) or state.get("format") != FORMAT:
        raise ValueError(f"{path}: not an ISPA transition state ({FORMAT})")
    L, dd = state["layers"], state["d"]
    if (d is not None and dd != d) or (layers is not None and L != layers):
        raise ValueError(f"{path}: state for {L} layers of d = {dd}, expected "
                         f"{layers} layers of d = {d}")
    if state["dW"].shape != (L, dd, dd) or state["selected"].shape != (L,):
        raise ValueError(f"{path}: corrupt transition state")
    out = dict(state)
    for key in ("dW", "lambda", "err", "perm"):
        out[key] = state[key].to(device)
    for key in ("sink_k", "sink_v", "hist_k", "hist_v"):
        if key in state:
            out[key] = [None if t is None else t.to(device) for t in state[key]]
    return out


def resume_streaming(state: dict, W_all: torch.Tensor, layers, caches=None):
    """Applies a loaded transition state: the streaming weights of ``layers``
    (a StreamingLayers) from W and Delta W with the stored selection, and, when
    ``caches`` (one KVCache per layer) is given, every cache's sink and, where
    the state has it, an F-Layer's history."""
    layers.transition(W_all, state["dW"], state["selected"])
    if caches is not None:
        if len(caches) != state["layers"]:
            raise ValueError("one KV cache per layer is needed")
        for l, kc in enumerate(caches):
            kc.set_sink(state["sink_k"][l], state["sink_v"][l])
            hk = state.get("hist_k")
            if hk is not None and hk[l] is not None:
                kc.set_history(hk[l], state["hist_v"][l])
    return layers
