"""Layer-level driver of the ISPA warmup path on one GPU.

"Towards Memory-Efficient Autoregressive Video Generation via
Instance-Specific Parametric Absorption", technical summary section 2:
during the warmup every layer runs the dual-stream attention on each chunk
and accumulates the statistics of the closed form; at the transition each
layer's Delta W is solved, every layer's reconstruction error is formed and
the layers are ranked; the K lowest-error layers become L-Layers.

Every layer keeps its own statistics block M = [[G, R], [., S]], so the
transition runs as two batched calls over all layers (solve, then error)
instead of one pair of calls per layer. The error uses W only through
W W^T, a property of the model weights: ``weight_gram`` forms it once per
layer when the weights are loaded, after which the error is one reduction
pass per layer.

Orchestration only: buffers and workspaces are allocated once (through
torch) and every step is a call into the C ABI, so a warmup issues no
allocation and no host synchronisation.
"""
from __future__ import annotations

import torch

from . import ispa


class _Slot:
    """Attention outputs and workspace of one chunk in flight."""

    def __init__(self, heads, head_dim, chunk_rows, max_sink, max_local, max_hist, device):
        d = heads * head_dim
        f32 = dict(dtype=torch.float32, device=device)
        self.a_loc = torch.empty(chunk_rows, d, **f32)
        self.d_out = torch.empty(chunk_rows, d, **f32)
        self.a_full = torch.empty(chunk_rows, d, dtype=torch.bfloat16, device=device)
        self.lse = [torch.empty(heads, chunk_rows, **f32) for _ in range(3)]
        self.ws = torch.empty(ispa.ispa_dual_attention_workspace_size(
            chunk_rows, max_sink, max_local, max_hist, heads, head_dim), dtype=torch.uint8,
            device=device)
        self.rows = 0


class _GroupSlot:
    """Attention outputs and workspace of one chunk of up to ``group`` layers
    in flight ([group, rows, d] outputs, one launch over the layers)."""

    def __init__(self, group, heads, head_dim, chunk_rows, max_sink, max_local, max_hist, device):
        d = heads * head_dim
        f32 = dict(dtype=torch.float32, device=device)
        self.a_loc = torch.empty(group, chunk_rows, d, **f32)
        self.d_out = torch.empty(group, chunk_rows, d, **f32)
        self.a_full = torch.empty(group, chunk_rows, d, dtype=torch.bfloat16, device=device)
        self.lse = [torch.empty(group, heads * chunk_rows, **f32) for _ in range(3)]
        self.heads = heads
        self.ws = torch.empty(ispa.ispa_dual_attention_layers_workspace_size(
            group, chunk_rows, max_sink, max_local, max_hist, heads, head_dim), dtype=torch.uint8,
            device=device)
        self.rows = 0


class LayerWarmup:
    """Buffers for ``n_layers`` layers of one geometry. The attention outputs
    are reused across chunks and layers; ``n_slots`` sets of them let that
    many layers run their chunks at once on separate streams (layers are
    independent until the transition), which fills the SMs the tail of one
    layer's launches leaves idle. With ``group`` > 1 there are also
    ``n_slots`` sets of outputs for ``group`` layers each, for
    ``layers_chunks_stacked``: the same chunk of ``group`` layers in one
    attention launch, whose units fill whole waves of the SMs."""

    def __init__(self, heads: int, head_dim: int, chunk_rows: int, max_sink: int,
                 max_local: int, max_hist: int, n_layers: int = 1, device="cuda",
                 n_slots: int = 1, group: int = 1):
        self.heads, self.head_dim = heads, head_dim
        self.d = d = heads * head_dim
        self.n_layers = n_layers
        self.device = device
        f32 = dict(dtype=torch.float32, device=device)
        self.slots = [_Slot(heads, head_dim, chunk_rows, max_sink, max_local, max_hist, device)
                      for _ in range(max(1, n_slots))]
        self.group = max(1, min(group, n_layers))
        self.group_slots = [] if self.group == 1 else [
            _GroupSlot(self.group, heads, head_dim, chunk_rows, max_sink, max_local, max_hist,
                       device) for _ in range(max(1, n_slots))]
        s0 = self.slots[0]
        self.a_loc, self.d_out, self.a_full, self.lse = s0.a_loc, s0.d_out, s0.a_full, s0.lse
        self.M = torch.zeros(n_layers, 2 * d, 2 * d, **f32)
        self.solve_ws = torch.empty(n_layers * ispa.ispa_absorb_workspace_size(d),
                                    dtype=torch.uint8, device=device)
        self.err_ws = torch.empty(n_layers * ispa.ispa_layer_error_workspace_size(d),
                                  dtype=torch.uint8, device=device)
        self.status = ispa.new_status(device)
        self.dW = torch.empty(n_layers, d, d, **f32)
        self.B = torch.empty(n_layers, d, d, **f32)
        self.lam = torch.empty(n_layers, **f32)
        self.P = None            # W W^T per layer, once weight_gram has run

    @property
    def n_slots(self) -> int:
        return len(self.slots)

    def attention(self, ch: dict, stream=None, slot: int = 0):
        """Dual-stream attention of one chunk into the slot's a_loc, d_out,
        a_full and LSEs."""
        sl = self.slots[slot]
        q = ch["q"]
        sl.rows = nq = q.shape[0]
        kv = [ispa._kv(ch["k_sink"], ch["v_sink"], self.heads, self.head_dim, "sink"),
              ispa._kv(ch["k_loc"], ch["v_loc"], self.heads, self.head_dim, "local"),
              ispa._kv(ch.get("k_hist"), ch.get("v_hist"), self.heads, self.head_dim, "history")]
        rc = ispa._load().ispa_dual_attention(
            ispa._ptr(q), nq, self.heads, self.head_dim, kv[0], kv[1], kv[2],
            float(self.head_dim ** -0.5), ispa._ptr(sl.a_loc), ispa._ptr(sl.d_out),
            ispa._ptr(sl.a_full), ispa._ptr(sl.lse[0]), ispa._ptr(sl.lse[1]),
            ispa._ptr(sl.lse[2]), ispa._ptr(sl.ws), sl.ws.numel(),
            ispa._ptr(self.status), ispa._stream(stream))
        ispa._check(rc, "ispa_dual_attention")

    def gram(self, first: bool, layer: int = 0, stream=None, slot: int = 0):
        """Fold the slot's last chunk into the layer's G, R, S (first chunk
        overwrites)."""
        sl = self.slots[slot]
        rc = ispa._load().ispa_gram_accumulate(
            ispa._ptr(sl.a_loc), ispa._ptr(sl.d_out), sl.rows, self.d,
            ispa._ptr(self.M[layer]), 0 if first else 1, 1, ispa._ptr(self.status),
            ispa._stream(stream))
        ispa._check(rc, "ispa_gram_accumulate")

    def chunk(self, ch: dict, first: bool, layer: int = 0, stream=None, slot: int = 0):
        self.attention(ch, stream, slot)
        self.gram(first, layer, stream, slot)

    def layers_chunks(self, chunks_per_layer, streams=None):
        """Every chunk of every layer into the layers' statistics. With
        ``streams`` (one per slot, the first the caller's current stream),
        layer l runs on streams[l mod n_slots]; the others fork from and join
        back into the first."""
        if not streams or len(streams) == 1 or self.n_slots == 1:
            s = streams[0] if streams else None
            for li, chunks in enumerate(chunks_per_layer):
                for c, ch in enumerate(chunks):
                    self.chunk(ch, first=(c == 0), layer=li, stream=s)
            return
        n = min(len(streams), self.n_slots)
        fork = torch.cuda.Event()
        fork.record(streams[0])
        for s in streams[1:n]:
            s.wait_event(fork)
        for li, chunks in enumerate(chunks_per_layer):
            slot = li % n
            for c, ch in enumerate(chunks):
                self.chunk(ch, first=(c == 0), layer=li, stream=streams[slot], slot=slot)
        for s in streams[1:n]:
            join = torch.cuda.Event()
            join.record(s)
            streams[0].wait_event(join)

    def attention_layers(self, sch: dict, l0: int, n: int, stream=None, slot: int = 0):
        """Dual-stream attention of one chunk of layers l0 .. l0 + n - 1 in
        one launch, into the group slot. ``sch``: the chunk's inputs as
        [L, rows, heads, head_dim] tensors (``ispa_synth.stacked_chunk``)."""
        gs = self.group_slots[slot]
        if n > self.group:
            raise ValueError(f"{n} layers exceed the group size {self.group}")
        take = lambda key: None if sch.get(key) is None else sch[key][l0:l0 + n]
        q = take("q")
        gs.rows = nq = q.shape[1]
        if nq > gs.a_loc.shape[1]:
            raise ValueError(f"{nq} query rows exceed the slot's {gs.a_loc.shape[1]}")
        ispa.ispa_dual_attention_layers(
            q, take("k_sink"), take("v_sink"), take("k_loc"), take("v_loc"), take("k_hist"),
            take("v_hist"), a_loc=gs.a_loc[:n, :nq], d_out=gs.d_out[:n, :nq],
            a_full=gs.a_full[:n, :nq],
            lse=[x[:n, :gs.heads * nq].view(n, gs.heads, nq) for x in gs.lse], workspace=gs.ws,
            status=self.status, stream=stream)

    def gram_group(self, first: bool, j: int, layer: int, stream=None, slot: int = 0):
        """Fold layer j of the group slot's last chunk into the statistics of
        ``layer`` (first chunk overwrites)."""
        gs = self.group_slots[slot]
        rc = ispa._load().ispa_gram_accumulate(
            ispa._ptr(gs.a_loc[j]), ispa._ptr(gs.d_out[j]), gs.rows, self.d,
            ispa._ptr(self.M[layer]), 0 if first else 1, 1, ispa._ptr(self.status),
            ispa._stream(stream))
        ispa._check(rc, "ispa_gram_accumulate")

    def layer_groups(self):
        """(first layer, layers) of each group, in order."""
        return [(l0, min(self.group, self.n_layers - l0))
                for l0 in range(0, self.n_layers, self.group)]

    def layers_chunks_stacked(self, stacked_chunks, streams=None):
        """Every chunk of every layer into the layers' statistics, ``group``
        layers per attention launch: ``stacked_chunks[c]`` holds chunk c of
        all layers (``ispa_synth.stacked_chunk``). Group g runs on
        streams[g mod n_slots]; the others fork from and join back into the
        first."""
        if not self.group_slots:
            raise ValueError("this runner was built with group = 1")
        streams = streams or [None]
        n = min(len(streams), len(self.group_slots))
        if n > 1:
            fork = torch.cuda.Event()
            fork.record(streams[0])
            for s in streams[1:n]:
                s.wait_event(fork)
        for g, (l0, cnt) in enumerate(self.layer_groups()):
            slot = g % n
            s = streams[slot]
            for c, sch in enumerate(stacked_chunks):
                self.attention_layers(sch, l0, cnt, stream=s, slot=slot)
                for j in range(cnt):
                    self.gram_group(c == 0, j, l0 + j, stream=s, slot=slot)
        if n > 1:
            for s in streams[1:n]:
                join = torch.cuda.Event()
                join.record(s)
                streams[0].wait_event(join)

    def solve(self, W: torch.Tensor, lam: float = 0.0, layer: int = 0, stream=None):
        """Delta W (and B = R W, lambda) of one layer into its slot."""
        rc = ispa._load().ispa_absorb_solve(
            ispa._ptr(self.M[layer]), ispa._ptr(W), self.d, float(lam),
            ispa._ptr(self.dW[layer]), ispa._ptr(self.B[layer]), ispa._ptr(self.lam[layer:]),
            ispa._ptr(self.solve_ws), self.solve_ws.numel(), ispa._ptr(self.status),
            ispa._stream(stream))
        ispa._check(rc, "ispa_absorb_solve")

    def error(self, W: torch.Tensor, err_slot: torch.Tensor, layer: int = 0, stream=None):
        """One layer's {||E||^2, relative error} into err_slot (device double[2])."""
        rc = ispa._load().ispa_layer_error(
            ispa._ptr(self.M[layer]), ispa._ptr(W), ispa._ptr(self.dW[layer]),
            ispa._ptr(self.B[layer]), ispa._ptr(self.lam[layer:]), self.d, ispa._ptr(err_slot),
            ispa._ptr(self.err_ws), self.err_ws.numel(), ispa._stream(stream))
        ispa._check(rc, "ispa_layer_error")

    def solve_all(self, W_all: torch.Tensor, lam: float = 0.0, stream=None):
        """Delta W of every layer in one batched call; W_all is [n_layers, d, d]."""
        n, d = self.n_layers, self.d
        _check_stack(W_all, n, d)
        rc = ispa._load().ispa_absorb_solve_batched(
            n, ispa._ptr(self.M), 4 * d * d, ispa._ptr(W_all), W_all.stride(0), d, float(lam),
            ispa._ptr(self.dW), d * d, ispa._ptr(self.B), d * d, ispa._ptr(self.lam),
            ispa._ptr(self.solve_ws), self.solve_ws.numel(), ispa._ptr(self.status),
            ispa._stream(stream))
        ispa._check(rc, "ispa_absorb_solve_batched")

    def weight_gram(self, W_all: torch.Tensor, stream=None):
        """P[l] = W[l] W[l]^T, formed once per set of weights."""
        n, d = self.n_layers, self.d
        _check_stack(W_all, n, d)
        if self.P is None:
            self.P = torch.empty(n, d, d, dtype=torch.float32, device=self.device)
        rc = ispa._load().ispa_weight_gram_batched(
            n, ispa._ptr(W_all), W_all.stride(0), d, ispa._ptr(self.P), d * d,
            ispa._ptr(self.status), ispa._stream(stream))
        ispa._check(rc, "ispa_weight_gram_batched")

    def error_all(self, W_all: torch.Tensor, err: torch.Tensor, stream=None):
        """Every layer's {||E||^2, relative error} into err [n_layers, 2] fp64
        (from W W^T when weight_gram has run, else from W)."""
        n, d = self.n_layers, self.d
        _check_stack(W_all, n, d)
        if err.dtype != torch.float64 or err.shape != (n, 2) or not err.is_contiguous():
            raise ValueError("err must be a contiguous float64 [n_layers, 2] tensor")
        if self.P is not None:
            rc = ispa._load().ispa_layer_error_wwt_batched(
                n, ispa._ptr(self.M), 4 * d * d, ispa._ptr(self.P), d * d, ispa._ptr(self.dW),
                d * d, ispa._ptr(self.B), d * d, ispa._ptr(self.lam), d, ispa._ptr(err),
                ispa._ptr(self.err_ws), self.err_ws.numel(), ispa._stream(stream))
            ispa._check(rc, "ispa_layer_error_wwt_batched")
            return
        rc = ispa._load().ispa_layer_error_batched(
            n, ispa._ptr(self.M), 4 * d * d, ispa._ptr(W_all), W_all.stride(0),
            ispa._ptr(self.dW), d * d, ispa._ptr(self.B), d * d, ispa._ptr(self.lam), d,
            ispa._ptr(err), ispa._ptr(self.err_ws), self.err_ws.numel(), ispa._stream(stream))
        ispa._check(rc, "ispa_layer_error_batched")

    def absorb_all(self, W_all: torch.Tensor, err: torch.Tensor, lam: float = 0.0, stream=None):
        self.solve_all(W_all, lam, stream)
        self.error_all(W_all, err, stream)


def _check_stack(W_all: torch.Tensor, n: int, d: int):
    if (W_all.dtype != torch.float32 or W_all.shape != (n, d, d) or W_all.stride(2) != 1
            or W_all.stride(1) != d):
        raise ValueError(f"W_all must be float32 [{n}, {d}, {d}] with contiguous rows")


def rank(err: torch.Tensor, K: int, perm: torch.Tensor, selected: torch.Tensor, stream=None):
    """Stable ascending ranking of err [L, 2] (relative error in column 1)."""
    rc = ispa._load().ispa_rank_layers(ispa._ptr(err), err.shape[0], int(K), ispa._ptr(perm),
                                       ispa._ptr(selected), ispa._stream(stream))
    ispa._check(rc, "ispa_rank_layers")


def run_warmup(chunks_per_layer, W_all: torch.Tensor, K: int, runner: LayerWarmup,
               stream=None, streams=None, stacked_chunks=None):
    """Whole warmup: ``chunks_per_layer[l]`` is layer l's list of chunk dicts
    (device tensors), ``W_all`` the [L, d, d] projections. Accumulates every
    layer's statistics (layers spread over ``streams`` when given; with
    ``stacked_chunks``, chunk c of all layers as [L, ...] tensors, and a
    runner built with group > 1, that many layers per attention launch),
    solves and scores all layers in two batched calls and ranks them. Returns
    (err [L, 2] fp64, perm, selected); Delta W of layer l is ``runner.dW[l]``."""
    n = len(chunks_per_layer) if stacked_chunks is None else stacked_chunks[0]["q"].shape[0]
    if n != runner.n_layers:
        raise ValueError(f"runner holds {runner.n_layers} layers, got {n}")
    err = torch.empty(n, 2, dtype=torch.float64, device=runner.device)
    perm = torch.empty(n, dtype=torch.int32, device=runner.device)
    sel = torch.empty(n, dtype=torch.uint8, device=runner.device)
    sts = streams if streams else ([stream] if stream else None)
    if stacked_chunks is not None:
        runner.layers_chunks_stacked(stacked_chunks, sts)
    else:
        runner.layers_chunks(chunks_per_layer, sts)
    runner.absorb_all(W_all, err, stream=stream)
    rank(err, K, perm, sel, stream)
    return err, perm, sel
