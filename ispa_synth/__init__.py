"""Seeded synthetic workloads for the ISPA warmup path.

This module only draws random numbers and lays out which frames play which
role (sink, history, local chunk). It holds none of the method's arithmetic:
no softmax, no Gram, no solve. Both the float64 oracle and the CUDA path are
fed from here, so that the two see bit-identical inputs.

Workload recipe (the pages run trained video models on real prompts, which
are not available; these AR(1) streams stand in for their activations):

* Every layer draws three independent streams, one each for Q, K and V.
  A stream is a sequence of latent frames of ``tokens_per_frame`` tokens and
  ``d = heads * head_dim`` channels. Frame 0 is N(0, 1); frame f is
  ``rho * frame(f-1) + sqrt(1 - rho^2) * Z`` with fresh Z ~ N(0, 1), so every
  frame is N(0, 1) marginally and neighbouring frames correlate with rho.
  The stream is then rounded to bf16 (round to nearest even).
* The output projection W of a layer is N(0, 1/d) in fp32.
* Seeds: layer l, tensor t in {Q, K, V, W, X} draws from a generator seeded
  with ``seed * 1_000_003 + l * 101 + t``.

Frame roles ("Towards Memory-Efficient Autoregressive Video Generation via
Instance-Specific Parametric Absorption", Dutch summary, section 2, step 1:
the local stream sees the current frame plus the sink tokens, the full
stream also sees the history):

* 1.3B / 14B geometry: frame 0 is the sink frame. Warmup chunk c (0-based)
  generates frames 3c+1 .. 3c+3 (its queries and its local keys); its
  history is frames 1 .. 3c. Chunk 0 therefore has an empty history.
* Tiny geometry: the sink is the first 16 tokens of frame 0; frames are 64
  tokens; warmup chunks are frames 5..12, one frame each, with a sliding
  history of the 4 frames before the current one (256 tokens).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Tuple

import torch

TENSOR_IDS = {"Q": 0, "K": 1, "V": 2, "W": 3, "X": 4}


@dataclasses.dataclass(frozen=True)
class Config:
    """Geometry of one workload. Sizes follow the 1.3B/14B video models the
    pages evaluate (1560 tokens per latent frame, 3-frame chunks, a 12-frame
    warmup) and a tiny case small enough for a float64 CPU check."""

    name: str
    layers: int
    heads: int
    head_dim: int
    tokens_per_frame: int
    sink_tokens: int          # tokens of frame 0 used as the sink
    chunk_frames: int         # frames generated per chunk
    first_chunk_frame: int    # first frame of warmup chunk 0
    n_chunks: int             # warmup chunks
    history_window: Optional[int]  # frames of history (None: all since frame 1)
    rho: float = 0.9
    select_k: Optional[int] = None  # layers turned local (lowest error)
    stream_chunks: int = 0    # post-transition chunks (streaming workload)
    # Ranking-stress variant: layer l draws with its own correlation, spread
    # evenly over [lo, hi] in the scrambled order (7 l mod L), so that the
    # layers' errors separate and the ranking is not the layer order.
    rho_spread: Optional[Tuple[float, float]] = None

    def rho_of(self, layer: int) -> float:
        if self.rho_spread is None or self.layers < 2:
            return self.rho
        lo, hi = self.rho_spread
        return lo + (hi - lo) * ((7 * layer) % self.layers) / (self.layers - 1)

    @property
    def d(self) -> int:
        return self.heads * self.head_dim

    @property
    def chunk_tokens(self) -> int:
        return self.chunk_frames * self.tokens_per_frame

    @property
    def warmup_rows(self) -> int:
        return self.n_chunks * self.chunk_tokens

    def chunk_frames_of(self, c: int) -> List[int]:
        f0 = self.first_chunk_frame + c * self.chunk_frames
        return list(range(f0, f0 + self.chunk_frames))

    def history_frames_of(self, c: int) -> List[int]:
        f0 = self.first_chunk_frame + c * self.chunk_frames
        lo = 1 if self.history_window is None else max(1, f0 - self.history_window)
        return list(range(lo, f0))

    @property
    def n_frames(self) -> int:
        return self.first_chunk_frame + (self.n_chunks + self.stream_chunks) * self.chunk_frames


# The five workloads, in the order the benchmark description lists them.
C0 = Config("tiny", layers=1, heads=2, head_dim=64, tokens_per_frame=64, sink_tokens=16,
            chunk_frames=1, first_chunk_frame=5, n_chunks=8, history_window=4)
C1 = Config("1.3B-chunk", layers=1, heads=12, head_dim=128, tokens_per_frame=1560,
            sink_tokens=1560, chunk_frames=3, first_chunk_frame=10, n_chunks=1,
            history_window=None)
C2 = Config("1.3B-warmup", layers=30, heads=12, head_dim=128, tokens_per_frame=1560,
            sink_tokens=1560, chunk_frames=3, first_chunk_frame=1, n_chunks=4,
            history_window=None, select_k=15)
C3 = Config("14B-warmup", layers=40, heads=40, head_dim=128, tokens_per_frame=1560,
            sink_tokens=1560, chunk_frames=3, first_chunk_frame=1, n_chunks=4,
            history_window=None, select_k=20)
C4 = Config("1.3B-stream", layers=30, heads=12, head_dim=128, tokens_per_frame=1560,
            sink_tokens=1560, chunk_frames=3, first_chunk_frame=1, n_chunks=4,
            history_window=None, select_k=15, stream_chunks=17)
# Addition to the five: the 1.3B warmup with per-layer correlations spread
# over [0.5, 0.95] (ranking-stress variant; not one of the five workloads).
C2R = Config("1.3B-warmup-rho-spread", layers=30, heads=12, head_dim=128, tokens_per_frame=1560,
             sink_tokens=1560, chunk_frames=3, first_chunk_frame=1, n_chunks=4,
             history_window=None, select_k=15, rho_spread=(0.5, 0.95))
CONFIGS = {"c0": C0, "c1": C1, "c2": C2, "c3": C3, "c4": C4, "c2r": C2R}


def scaled(cfg: Config, **kw) -> Config:
    """A copy of ``cfg`` with some fields replaced (smaller test geometries)."""
    return dataclasses.replace(cfg, **kw)


def _generator(seed: int, layer: int, tensor: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + layer * 101 + TENSOR_IDS[tensor])
    return g


def ar1_stream(n_frames: int, tokens: int, dim: int, rho: float, seed: int, layer: int,
               tensor: str, device="cpu") -> torch.Tensor:
    """AR(1)-over-frames stream [n_frames, tokens, dim], rounded to bf16."""
    g = _generator(seed, layer, tensor, device)
    out = torch.empty(n_frames, tokens, dim, dtype=torch.bfloat16, device=device)
    innov = math.sqrt(1.0 - rho * rho)
    prev = torch.randn(tokens, dim, generator=g, device=device, dtype=torch.float32)
    out[0] = prev.to(torch.bfloat16)
    for f in range(1, n_frames):
        z = torch.randn(tokens, dim, generator=g, device=device, dtype=torch.float32)
        prev = rho * prev + innov * z
        out[f] = prev.to(torch.bfloat16)
    return out


def projection(dim: int, seed: int, layer: int, device="cpu") -> torch.Tensor:
    """Output projection W ~ N(0, 1/d), fp32 [d, d]."""
    g = _generator(seed, layer, "W", device)
    return torch.randn(dim, dim, generator=g, device=device, dtype=torch.float32) / math.sqrt(dim)


@dataclasses.dataclass
class LayerStreams:
    """Q/K/V streams of one layer, [n_frames, tokens_per_frame, heads, head_dim] bf16."""
    cfg: Config
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    w: torch.Tensor

    def _rows(self, x: torch.Tensor, frames: List[int]) -> torch.Tensor:
        if not frames:
            return x.new_zeros(0, self.cfg.heads, self.cfg.head_dim)
        return x[frames[0]:frames[-1] + 1].reshape(-1, self.cfg.heads, self.cfg.head_dim)

    def chunk(self, c: int) -> dict:
        """Inputs of warmup (or streaming) chunk c: tensors of shape
        [tokens, heads, head_dim], bf16, contiguous."""
        cfg = self.cfg
        cur = cfg.chunk_frames_of(c)
        hist = cfg.history_frames_of(c)
        sink_k = self.k[0, :cfg.sink_tokens]
        sink_v = self.v[0, :cfg.sink_tokens]
        return {
            "q": self._rows(self.q, cur).contiguous(),
            "k_sink": sink_k.contiguous(), "v_sink": sink_v.contiguous(),
            "k_loc": self._rows(self.k, cur).contiguous(), "v_loc": self._rows(self.v, cur).contiguous(),
            "k_hist": self._rows(self.k, hist).contiguous(), "v_hist": self._rows(self.v, hist).contiguous(),
        }


def layer_streams(cfg: Config, layer: int, seed: int = 0, device="cpu",
                  n_frames: Optional[int] = None) -> LayerStreams:
    nf = cfg.n_frames if n_frames is None else n_frames
    shape = (nf, cfg.tokens_per_frame, cfg.heads, cfg.head_dim)
    rho = cfg.rho_of(layer)
    mk = lambda t: ar1_stream(nf, cfg.tokens_per_frame, cfg.d, rho, seed, layer, t,
                              device).reshape(shape)
    return LayerStreams(cfg, mk("Q"), mk("K"), mk("V"), projection(cfg.d, seed, layer, device))


def stacked_layer_streams(cfg: Config, layers: List[int], seed: int = 0, device="cpu",
                          n_frames: Optional[int] = None, gen_device=None):
    """layer_streams of several layers with their Q, K and V each in one
    [L, n_frames, tokens_per_frame, heads, head_dim] tensor on ``device``:
    stream i's q, k and v are views of entry i (layer ``layers[i]``), so
    that one chunk of every layer is one strided tensor (``stacked_chunk``).
    Each layer is drawn on ``gen_device`` (default: ``device``; the draws
    depend on the device the generator runs on) and copied in. Returns the
    streams and the (Q, K, V) storage."""
    gen_device = device if gen_device is None else gen_device
    nf = cfg.n_frames if n_frames is None else n_frames
    shape = (len(layers), nf, cfg.tokens_per_frame, cfg.heads, cfg.head_dim)
    Q, K, V = (torch.empty(shape, dtype=torch.bfloat16, device=device) for _ in range(3))
    streams = []
    for i, l in enumerate(layers):
        st = layer_streams(cfg, l, seed, gen_device, n_frames=nf)
        Q[i].copy_(st.q)
        K[i].copy_(st.k)
        V[i].copy_(st.v)
        streams.append(LayerStreams(cfg, Q[i], K[i], V[i], st.w.to(device)))
        del st
    return streams, (Q, K, V)


def stacked_chunk(cfg: Config, qkv, c: int) -> dict:
    """Chunk c of every layer of a ``stacked_layer_streams`` storage: the
    inputs of LayerStreams.chunk(c) as [L, tokens, heads, head_dim] views
    (each layer's rows contiguous, the layers one stream apart)."""
    Q, K, V = qkv
    L, H, hd = Q.shape[0], cfg.heads, cfg.head_dim

    def rows(x, frames):
        if not frames:
            return x.new_zeros(L, 0, H, hd)
        return x[:, frames[0]:frames[-1] + 1].reshape(L, -1, H, hd)

    cur, hist = cfg.chunk_frames_of(c), cfg.history_frames_of(c)
    return {"q": rows(Q, cur), "k_sink": K[:, 0, :cfg.sink_tokens], "v_sink": V[:, 0, :cfg.sink_tokens],
            "k_loc": rows(K, cur), "v_loc": rows(V, cur),
            "k_hist": rows(K, hist), "v_hist": rows(V, hist)}


def gaussian(shape, seed: int, layer: int = 0, tensor: str = "X", device="cpu",
             dtype=torch.float32) -> torch.Tensor:
    """Plain seeded N(0, 1) draws for kernel-level tests that feed a stage
    with synthetic inputs of its own (e.g. attention outputs for the Gram)."""
    g = _generator(seed, layer, tensor, device)
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(dtype)


def attention_like(rows: int, dim: int, seed: int, rho: float = 0.9, common: float = 0.3,
                   device="cpu") -> torch.Tensor:
    """Synthetic stand-in for attention outputs [rows, dim], fp32: a shared
    per-channel mean (softmax averages of V share one) plus AR(1)-correlated
    rows. Used to feed the Gram and solve stages on their own."""
    g = _generator(seed, 7, "X", device)
    mean = common * torch.randn(dim, generator=g, device=device)
    z = torch.randn(rows, dim, generator=g, device=device)
    out = torch.empty_like(z)
    out[0] = z[0]
    innov = math.sqrt(1 - rho * rho)
    # correlate neighbouring rows in blocks of 64 rows, vectorised over blocks
    blk = z.view(-1, 64, dim) if rows % 64 == 0 else None
    if blk is not None:
        acc = blk[:, 0].clone()
        out.view(-1, 64, dim)[:, 0] = acc
        for i in range(1, 64):
            acc = rho * acc + innov * blk[:, i]
            out.view(-1, 64, dim)[:, i] = acc
    else:
        for i in range(1, rows):
            out[i] = rho * out[i - 1] + innov * z[i]
    return (out * 0.1 + mean).contiguous()


SKETCH_SEED = 977


def sketch_matrices(n_rows: int, dim: int, k: int = 16):
    """Fixed Gaussian test matrices for comparing large results through small
    two-sided sketches X -> L^T X R (E ||L^T X R||_F^2 = k^2 ||X||_F^2 for
    N(0, 1) entries). Returns (rows [n_rows, k], left [dim, k], right [dim, k])
    in float32, identical on every machine (CPU generator)."""
    return (gaussian((n_rows, k), SKETCH_SEED, 0, "X"),
            gaussian((dim, k), SKETCH_SEED, 1, "X"),
            gaussian((dim, k), SKETCH_SEED, 2, "X"))
