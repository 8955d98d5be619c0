"""Post-transition streaming on one GPU: F-Layers and L-Layers.

"Towards Memory-Efficient Autoregressive Video Generation via
Instance-Specific Parametric Absorption", technical summary section 2,
step 3: after the warmup's transition the K lowest-error layers become
L-Layers. They keep only the sink and the current chunk in their KV cache,
attend locally and project with the absorbed weight W + Delta W. The other
layers (F-Layers) keep their whole cache, attend over every earlier frame and
project with W. The memory saving is the dropped history of the L-Layers.

Orchestration only: every step is a call into the C ABI (full or local
attention, then the projection); buffers and workspaces are allocated once.
"""
from __future__ import annotations

import torch

from . import ispa


def kv_cache_bytes(n_full: int, n_local: int, sink: int, history: int, chunk: int, d: int,
                   bytes_per_elem: int = 2) -> int:
    """KV-cache bytes of one model at a chunk: an F-Layer holds keys and values
    of the sink, the history and the current chunk; an L-Layer only of the
    sink and the current chunk."""
    per_token = 2 * d * bytes_per_elem            # K and V
    return n_full * (sink + history + chunk) * per_token + n_local * (sink + chunk) * per_token


class KVCache:
    """One layer's KV cache after the transition, laid out [sink | history |
    current chunk] along the token axis. An F-Layer's cache has room for the
    whole stream and keeps every chunk (the current chunk becomes history
    when the next one arrives); an L-Layer's holds the sink and one chunk,
    which each new chunk overwrites."""

    def __init__(self, heads: int, head_dim: int, sink: int, chunk: int, max_hist: int,
                 full: bool, device="cuda"):
        cap = sink + chunk + (max_hist if full else 0)
        self.k = torch.empty(cap, heads, head_dim, dtype=torch.bfloat16, device=device)
        self.v = torch.empty_like(self.k)
        self.sink, self.chunk, self.full = sink, chunk, full
        self.hist = 0            # history tokens held
        self.cur = 0             # tokens of the current chunk
        self.hist0 = 0           # history preloaded at the transition

    @property
    def nbytes(self) -> int:
        return self.k.numel() * self.k.element_size() + self.v.numel() * self.v.element_size()

    def set_sink(self, k: torch.Tensor, v: torch.Tensor):
        self.k[:self.sink].copy_(k)
        self.v[:self.sink].copy_(v)

    def set_history(self, k: torch.Tensor, v: torch.Tensor):
        """Preload the history an F-Layer holds at the transition."""
        if not self.full:
            raise ValueError("an L-Layer keeps no history")
        n = k.shape[0]
        if self.sink + n + self.chunk > self.k.shape[0]:
            raise ValueError("history exceeds the cache")
        self.k[self.sink:self.sink + n].copy_(k)
        self.v[self.sink:self.sink + n].copy_(v)
        self.hist, self.cur, self.hist0 = n, 0, n

    def rewind(self):
        """Back to the state right after the transition (the preloaded history,
        no current chunk); the stored tokens are not touched."""
        self.hist, self.cur = self.hist0, 0

    def append(self, k: torch.Tensor, v: torch.Tensor):
        """A new chunk's keys and values: an F-Layer moves its previous chunk
        into the history, an L-Layer drops it."""
        n = k.shape[0]
        if self.full:
            self.hist += self.cur
        base = self.sink + self.hist
        if base + n > self.k.shape[0]:
            raise ValueError("the cache is full")
        self.k[base:base + n].copy_(k)
        self.v[base:base + n].copy_(v)
        self.cur = n

    def chunk_inputs(self, q: torch.Tensor) -> dict:
        """Attention inputs for the current chunk: views into the cache."""
        s, h, c = self.sink, self.hist, self.cur
        return {"q": q, "k_sink": self.k[:s], "v_sink": self.v[:s],
                "k_loc": self.k[s + h:s + h + c], "v_loc": self.v[s + h:s + h + c],
                "k_hist": self.k[s:s + h], "v_hist": self.v[s:s + h]}


class StreamingLayers:
    """Layer weights after the transition and the buffers of one chunk."""

    def __init__(self, heads: int, head_dim: int, chunk_rows: int, max_sink: int, max_local: int,
                 max_hist: int, n_layers: int, device="cuda"):
        self.heads, self.head_dim = heads, head_dim
        self.d = d = heads * head_dim
        self.n_layers = n_layers
        self.device = device
        bf16 = dict(dtype=torch.bfloat16, device=device)
        self.att = torch.empty(chunk_rows, d, **bf16)
        self.out = torch.empty(chunk_rows, d, **bf16)
        full_ws = ispa.ispa_full_attention_workspace_size(chunk_rows, max_sink, max_local, max_hist,
                                                          heads, head_dim)
        local_ws = ispa.ispa_dual_attention_workspace_size(chunk_rows, max_sink, max_local, 0,
                                                           heads, head_dim)
        self.ws = torch.empty(max(full_ws, local_ws), dtype=torch.uint8, device=device)
        self.status = ispa.new_status(device)
        self.Wp = torch.empty(n_layers, d, d, **bf16)
        self.local = torch.zeros(n_layers, dtype=torch.bool)
        self.wq = None           # int8 codes and scales of W' once quantize_weights has run
        self.wq_scale = None
        self.q_ws = torch.empty(ispa.ispa_project_w8a8_workspace_size(chunk_rows, d),
                                dtype=torch.uint8, device=device)

    def transition(self, W_all: torch.Tensor, dW_all: torch.Tensor, selected, stream=None):
        """Weights for streaming: bf16(W + Delta W) for the selected layers
        (L-Layers), bf16(W) for the others (F-Layers)."""
        sel = torch.as_tensor(selected).to("cpu", torch.bool)
        if sel.numel() != self.n_layers:
            raise ValueError(f"selected must have {self.n_layers} entries")
        self.local = sel.clone()
        for l in range(self.n_layers):
            ispa.ispa_absorbed_weight(W_all[l], dW_all[l] if bool(sel[l]) else None,
                                      out=self.Wp[l], stream=stream)

    def quantize_weights(self, W_all: torch.Tensor, dW_all: torch.Tensor, stream=None):
        """W8A8: 8-bit codes of every layer's projection weight (W + Delta W for
        the L-Layers, W for the F-Layers), per output column."""
        n, d = self.n_layers, self.d
        self.wq = torch.empty(n, d, d, dtype=torch.int8, device=self.device)
        self.wq_scale = torch.empty(n, d, dtype=torch.float32, device=self.device)
        for l in range(n):
            ispa.ispa_quantize_weight_int8(W_all[l], dW_all[l] if bool(self.local[l]) else None,
                                           wq_t=self.wq[l], w_scale=self.wq_scale[l], stream=stream)

    def layer(self, l: int, ch: dict, local=None, w8a8: bool = False, stream=None) -> torch.Tensor:
        # ``ch`` holds the chunk's query rows and the layer's keys/values (e.g.
        # KVCache.chunk_inputs); an L-Layer reads only the sink and the chunk.
        """One chunk through layer l (its kind from the transition unless
        ``local`` overrides it; with ``w8a8`` the projection runs on 8-bit
        weights and activations). Returns the projected rows (bf16, reused)."""
        is_local = bool(self.local[l]) if local is None else bool(local)
        q = ch["q"]
        nq = q.shape[0]
        kv_sink = ispa._kv(ch["k_sink"], ch["v_sink"], self.heads, self.head_dim, "sink")
        kv_loc = ispa._kv(ch["k_loc"], ch["v_loc"], self.heads, self.head_dim, "local")
        att = self.att[:nq]
        lib = ispa._load()
        scale = float(self.head_dim ** -0.5)
        if is_local:
            rc = lib.ispa_local_attention(
                ispa._ptr(q), nq, self.heads, self.head_dim, kv_sink, kv_loc, scale, None,
                ispa._ptr(att), None, ispa._ptr(self.ws), self.ws.numel(), ispa._ptr(self.status),
                ispa._stream(stream))
            ispa._check(rc, "ispa_local_attention")
        else:
            kv_hist = ispa._kv(ch.get("k_hist"), ch.get("v_hist"), self.heads, self.head_dim,
                               "history")
            rc = lib.ispa_full_attention(
                ispa._ptr(q), nq, self.heads, self.head_dim, kv_sink, kv_loc, kv_hist, scale,
                ispa._ptr(att), None, ispa._ptr(self.ws), self.ws.numel(), ispa._ptr(self.status),
                ispa._stream(stream))
            ispa._check(rc, "ispa_full_attention")
        out = self.out[:nq]
        if w8a8:
            rc = lib.ispa_project_w8a8(ispa._ptr(att), nq, self.d, ispa._ptr(self.wq[l]),
                                       ispa._ptr(self.wq_scale[l]), ispa._ptr(out), 0,
                                       ispa._ptr(self.q_ws), self.q_ws.numel(),
                                       ispa._ptr(self.status), ispa._stream(stream))
            ispa._check(rc, "ispa_project_w8a8")
            return out
        rc = lib.ispa_project(ispa._ptr(att), nq, self.d, ispa._ptr(self.Wp[l]), ispa._ptr(out), 0,
                              ispa._ptr(self.status), ispa._stream(stream))
        ispa._check(rc, "ispa_project")
        return out
