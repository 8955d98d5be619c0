"""Layer-level driver of the ISPA warmup path on one GPU.

"Towards Memory-Efficient Autoregressive Video Generation via
Instance-Specific Parametric Absorption", technical summary section 2:
during the warmup every layer runs the dual-stream attention on each chunk
and accumulates the statistics of the closed form; at the transition each
layer's Delta W is solved, every layer's reconstruction error is formed and
the layers are ranked; the K lowest-error layers become L-Layers.

Orchestration only: buffers and workspaces are allocated once (through
torch) and every step is a call into the C ABI, so a warmup issues no
allocation and no host synchronisation.
"""
from __future__ import annotations

import torch

from . import ispa


class LayerWarmup:
    """Buffers for one layer geometry, reused across chunks and layers."""

    def __init__(self, heads: int, head_dim: int, chunk_rows: int, max_sink: int,
                 max_local: int, max_hist: int, device="cuda"):
        self.heads, self.head_dim = heads, head_dim
        self.d = d = heads * head_dim
        self.device = device
        f32 = dict(dtype=torch.float32, device=device)
        self.a_loc = torch.empty(chunk_rows, d, **f32)
        self.d_out = torch.empty(chunk_rows, d, **f32)
        self.a_full = torch.empty(chunk_rows, d, dtype=torch.bfloat16, device=device)
        self.lse = [torch.empty(heads, chunk_rows, **f32) for _ in range(3)]
        self.attn_ws = torch.empty(ispa.ispa_dual_attention_workspace_size(
            chunk_rows, max_sink, max_local, max_hist, heads, head_dim), dtype=torch.uint8,
            device=device)
        self.M = torch.zeros(2 * d, 2 * d, **f32)
        self.solve_ws = torch.empty(ispa.ispa_absorb_workspace_size(d), dtype=torch.uint8,
                                    device=device)
        self.err_ws = torch.empty(ispa.ispa_layer_error_workspace_size(d), dtype=torch.uint8,
                                  device=device)
        self.status = ispa.new_status(device)
        self.dW = torch.empty(d, d, **f32)
        self.B = torch.empty(d, d, **f32)
        self.lam = torch.empty(1, **f32)
        self._rows = 0

    def attention(self, ch: dict, stream=None):
        """Dual-stream attention of one chunk into a_loc, d_out, a_full, LSEs."""
        q = ch["q"]
        self._rows = nq = q.shape[0]
        kv = [ispa._kv(ch["k_sink"], ch["v_sink"], self.heads, self.head_dim, "sink"),
              ispa._kv(ch["k_loc"], ch["v_loc"], self.heads, self.head_dim, "local"),
              ispa._kv(ch.get("k_hist"), ch.get("v_hist"), self.heads, self.head_dim, "history")]
        rc = ispa._load().ispa_dual_attention(
            ispa._ptr(q), nq, self.heads, self.head_dim, kv[0], kv[1], kv[2],
            float(self.head_dim ** -0.5), ispa._ptr(self.a_loc), ispa._ptr(self.d_out),
            ispa._ptr(self.a_full), ispa._ptr(self.lse[0]), ispa._ptr(self.lse[1]),
            ispa._ptr(self.lse[2]), ispa._ptr(self.attn_ws), self.attn_ws.numel(),
            ispa._ptr(self.status), ispa._stream(stream))
        ispa._check(rc, "ispa_dual_attention")

    def gram(self, first: bool, stream=None):
        """Fold the last chunk's rows into G, R, S (first chunk overwrites)."""
        rc = ispa._load().ispa_gram_accumulate(
            ispa._ptr(self.a_loc), ispa._ptr(self.d_out), self._rows, self.d, ispa._ptr(self.M),
            0 if first else 1, 1, ispa._stream(stream))
        ispa._check(rc, "ispa_gram_accumulate")

    def chunk(self, ch: dict, first: bool, stream=None):
        self.attention(ch, stream)
        self.gram(first, stream)

    def solve(self, W: torch.Tensor, lam: float = 0.0, stream=None):
        """Delta W of the layer (and B = R W, lambda)."""
        rc = ispa._load().ispa_absorb_solve(
            ispa._ptr(self.M), ispa._ptr(W), self.d, float(lam), ispa._ptr(self.dW),
            ispa._ptr(self.B), ispa._ptr(self.lam), ispa._ptr(self.solve_ws),
            self.solve_ws.numel(), ispa._ptr(self.status), ispa._stream(stream))
        ispa._check(rc, "ispa_absorb_solve")

    def error(self, W: torch.Tensor, err_slot: torch.Tensor, stream=None):
        """The layer's {||E||^2, relative error} into err_slot (device double[2])."""
        rc = ispa._load().ispa_layer_error(
            ispa._ptr(self.M), ispa._ptr(W), ispa._ptr(self.dW), ispa._ptr(self.B),
            ispa._ptr(self.lam), self.d, ispa._ptr(err_slot), ispa._ptr(self.err_ws),
            self.err_ws.numel(), ispa._stream(stream))
        ispa._check(rc, "ispa_layer_error")

    def absorb(self, W: torch.Tensor, err_slot: torch.Tensor, lam: float = 0.0, stream=None):
        self.solve(W, lam, stream)
        self.error(W, err_slot, stream)


def rank(err: torch.Tensor, K: int, perm: torch.Tensor, selected: torch.Tensor, stream=None):
    """Stable ascending ranking of err [L, 2] (relative error in column 1)."""
    rc = ispa._load().ispa_rank_layers(ispa._ptr(err), err.shape[0], int(K), ispa._ptr(perm),
                                       ispa._ptr(selected), ispa._stream(stream))
    ispa._check(rc, "ispa_rank_layers")


def run_warmup(layers, K: int, runner: LayerWarmup, keep_dw: bool = False, stream=None):
    """Whole warmup over ``layers``: a list of (chunks, W) per layer, chunks a
    list of dicts of device tensors. Returns (err [L, 2] fp64, perm, selected,
    list of Delta W if keep_dw)."""
    n = len(layers)
    err = torch.empty(n, 2, dtype=torch.float64, device=runner.device)
    perm = torch.empty(n, dtype=torch.int32, device=runner.device)
    sel = torch.empty(n, dtype=torch.uint8, device=runner.device)
    dws = []
    for li, (chunks, W) in enumerate(layers):
        for c, ch in enumerate(chunks):
            runner.chunk(ch, first=(c == 0), stream=stream)
        runner.absorb(W, err[li], stream=stream)
        if keep_dw:
            dws.append(runner.dW.clone())
    rank(err, K, perm, sel, stream)
    return err, perm, sel, dws
