"""Canary guard regions around what the library's calls write.

compute-sanitizer cannot run on the GPUs used here, so each call below
writes into outputs and workspaces that sit inside larger buffers filled
with a canary byte: padding rows between the layers of a batched output and
a guard before and after every buffer (``tests/guards.py``). A call passes
when it leaves every canary byte as it was and overwrites every element of
its outputs; the results are also checked against the oracle or the
unguarded call. Shapes are ragged (partial query, key and row tiles) so that
the tile edges, where an out-of-range write would happen, are exercised.

The first test checks the guard logic itself on the CPU.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from ispa_synth import attention_like, gaussian
from tests.guards import CANARY, GUARD_BYTES, Guarded
from tests.test_gpu_parity import (DW_RELFRO, GR_RELFRO, _stack_layers, check_attention, f64,
                                   pack_M, random_chunk, ref_dual, rel_fro, synthetic_layer,
                                   upper_tile_mask)

gpu = pytest.mark.gpu


def test_guard_logic_on_the_cpu():
    """A write inside the tensor keeps the guards intact; one element past a
    layer's rows, a byte before or after the buffer, or an element left
    unwritten is reported."""
    g = Guarded((2, 5, 8), torch.float32, pad=3, device="cpu")
    assert g.intact() and not g.written()
    g.t.fill_(1.5)
    assert g.intact() and g.written()
    assert g.t.data_ptr() % GUARD_BYTES == g.buf.data_ptr() % GUARD_BYTES
    g.store[1, 5, 0] = 2.0                     # first padding row of layer 1
    assert not g.intact()
    g.store[1, 5, 0] = g.store[1, 6, 0]        # restore the canary bytes
    assert g.intact()
    g.buf[GUARD_BYTES - 1] = 0                 # the byte before the buffer
    assert not g.intact()
    g.buf[GUARD_BYTES - 1] = CANARY
    g.buf[-1] = 0                              # the last byte after it
    assert not g.intact()
    g.buf[-1] = CANARY
    g.t[0, 4, 7] = g.store[0, 6, 7]            # one element left with the canary pattern
    assert g.intact() and not g.written()
    for dtype, shape, pad in ((torch.float64, (3, 2), 0), (torch.bfloat16, (7,), 2),
                              (torch.uint8, (4, 4), 1)):
        h = Guarded(shape, dtype, pad=pad, device="cpu")
        h.t.fill_(1)
        assert h.intact() and h.written() and tuple(h.t.shape) == shape
        h.store.view(-1)[-1] = 0 if pad else h.store.view(-1)[-1]
        assert h.intact() == (pad == 0)


# ---------------------------------------------------------------- attention

@gpu
@pytest.mark.parametrize("nq,sink,loc,hist,H,hd,splits", [
    (700, 300, 600, 2000, 4, 128, None),     # the launch's own plan over two layers
    (700, 300, 600, 2000, 4, 128, (1, -1)),  # joint units
    (700, 300, 600, 2000, 4, 128, (3, 2)),   # several local and history ranges, merged
    (129, 16, 100, 3100, 3, 64, None),       # one query row past a tile, long history
    (1, 1, 0, 0, 1, 64, None),               # one query, one key, no history
])
def test_dual_attention_writes_stay_in_bounds(lib, nq, sink, loc, hist, H, hd, splits):
    L, d = 2, H * hd
    chunks = [random_chunk(nq, sink, loc, hist, H, hd, seed=90 + 3 * l) for l in range(L)]
    q = _stack_layers(chunks, "q")
    kv = [_stack_layers(chunks, k) if chunks[0][k].shape[0] else None
          for k in ("k_sink", "v_sink", "k_loc", "v_loc", "k_hist", "v_hist")]
    outs = [Guarded((L, nq, d), dt, pad=3) for dt in (torch.float32, torch.float32, torch.bfloat16)]
    lses = [Guarded((L, H, nq), torch.float32, pad=1) for _ in range(3)]
    if splits:
        lib.ispa_attention_set_splits(*splits)
    try:
        need = lib.ispa_dual_attention_layers_workspace_size(L, nq, sink, loc, hist, H, hd)
        ws = Guarded((need,), torch.uint8)
        got = lib.ispa_dual_attention_layers(q, *kv, a_loc=outs[0].t, d_out=outs[1].t,
                                             a_full=outs[2].t, lse=[g.t for g in lses],
                                             workspace=ws.t)
        torch.cuda.synchronize()
    finally:
        lib.ispa_attention_set_splits(0, 0)
    assert lib.read_status(got["status"]) == 0
    for name, g in zip(("a_loc", "d", "a_full", "lse_loc", "lse_hist", "lse_full"), outs + lses):
        assert g.intact(), name
        assert g.written(), name
    assert ws.intact(), "workspace"
    for l in range(L):
        check_attention({k: v[l] for k, v in got.items() if k != "status"}, ref_dual(chunks[l]),
                        f"layer {l}")


# ---------------------------------------------------------------- Gram

@gpu
@pytest.mark.parametrize("rows,dim", [(777, 384), (70, 128), (300, 1536)])
def test_gram_writes_only_its_blocks(lib, rows, dim):
    """G, R and S (ragged rows) into a guarded M: the guards and the block
    below the diagonal that M leaves unused (R^T's place) keep the canary."""
    a = attention_like(rows, dim, seed=11)
    dd = 0.3 * attention_like(rows, dim, seed=12)
    M = Guarded((2 * dim, 2 * dim), torch.float32)
    status = lib.new_status("cuda")
    lib.ispa_gram_accumulate(a.cuda(), dd.cuda(), M=M.t, status=status)
    torch.cuda.synchronize()
    assert lib.read_status(status) == 0
    assert M.intact()
    lower_left = M.t[dim:, :dim].contiguous().view(torch.uint8)
    assert bool((lower_left == CANARY).all())
    G, R, S = oracle.gram(f64(a), f64(dd))
    Mg = f64(M.t)
    up = upper_tile_mask(dim)
    assert rel_fro(Mg[:dim, :dim][up], G[up]) <= GR_RELFRO
    assert rel_fro(Mg[:dim, dim:], R) <= GR_RELFRO
    assert rel_fro(Mg[dim:, dim:][up], S[up]) <= GR_RELFRO


# ---------------------------------------------------------------- solve and error

@gpu
@pytest.mark.parametrize("dim", [128, 384])
def test_one_layer_solve_stays_in_its_workspace(lib, dim):
    """The one-layer sweep (step kernels, side streams) in a workspace of
    exactly ispa_absorb_workspace_size(d) bytes with guards around it."""
    a, f, W = synthetic_layer(4 * dim + 37, dim, seed=300 + dim)
    G, R, S = oracle.gram(a, f - a)
    M = pack_M(G, R, S).cuda()
    ws = Guarded((lib.ispa_absorb_workspace_size(dim),), torch.uint8)
    out = lib.ispa_absorb_solve(M, W.cuda(), workspace=ws.t)
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    assert ws.intact()
    Gf, Rf = f64(M[:dim, :dim]), f64(M[:dim, dim:])
    dW, _ = oracle.absorb(Gf, Rf, f64(W), oracle.default_lambda(Gf))
    assert rel_fro(f64(out["dW"]), dW) <= DW_RELFRO


@gpu
@pytest.mark.parametrize("L", [1, 3])
def test_batched_solve_and_error_write_in_bounds(lib, L):
    """Batched solve into layer-strided Delta W and B (padding rows between
    the layers), the lambdas, the workspace; then W W^T and the errors, each
    inside guards. One layer takes the one-layer sweep, three the
    left-looking one."""
    dim = 256
    Ms, Ws = [], []
    for l in range(L):
        a, f, W = synthetic_layer(3 * dim + 29 * l, dim, seed=400 + l)
        G, R, S = oracle.gram(a, f - a)
        Ms.append(pack_M(G, R, S))
        Ws.append(W)
    M = torch.stack(Ms).cuda()
    W = torch.stack(Ws).contiguous().cuda()
    dW, B = Guarded((L, dim, dim), torch.float32, pad=5), Guarded((L, dim, dim), torch.float32, pad=5)
    lam = Guarded((L,), torch.float32, pad=3)
    ws = Guarded((L * lib.ispa_absorb_workspace_size(dim),), torch.uint8)
    out = lib.ispa_absorb_solve_batched(M, W, dW=dW.t, B=B.t, lam_out=lam.t, workspace=ws.t)
    P = Guarded((L, dim, dim), torch.float32)
    lib.ispa_weight_gram_batched(W, P=P.t)
    err = Guarded((L, 2), torch.float64)
    ews = Guarded((L * lib.ispa_layer_error_workspace_size(dim),), torch.uint8)
    dWc, Bc = dW.t.contiguous(), B.t.contiguous()
    lib.ispa_layer_error_wwt_batched(M, P.t, dWc, Bc, lam.t, err=err.t, workspace=ews.t)
    torch.cuda.synchronize()
    assert lib.read_status(out["status"]) == 0
    for name, g in (("dW", dW), ("B", B), ("lambda", lam), ("W W^T", P), ("err", err)):
        assert g.intact(), name
        assert g.written(), name
    assert ws.intact() and ews.intact()
    # the same calls into unguarded buffers
    ref = lib.ispa_absorb_solve_batched(M, W)
    ref_err = lib.ispa_layer_error_wwt_batched(M, P.t, dWc, Bc, lam.t)
    torch.cuda.synchronize()
    for l in range(L):
        assert rel_fro(f64(dW.t[l]), f64(ref["dW"][l])) <= DW_RELFRO
    # the same inputs: equal up to the order of the fp64 atomic additions
    assert np.allclose(err.t.cpu().numpy(), ref_err.cpu().numpy(), rtol=1e-9, atol=0)


# ---------------------------------------------------------------- projections

@gpu
def test_projections_write_in_bounds(lib):
    """bf16 and fp32 projection outputs, the absorbed weight, the int8 weight
    codes and scales, the W8A8 output and its workspace, ragged rows."""
    rows, dim = 333, 256
    a = gaussian((rows, dim), 21, 0, "X").to(torch.bfloat16).cuda()
    W = (gaussian((dim, dim), 22, 0, "W") / math.sqrt(dim)).cuda()
    dW = (0.1 * gaussian((dim, dim), 23, 0, "W") / math.sqrt(dim)).cuda()
    wb = Guarded((dim, dim), torch.bfloat16, pad=2)
    lib.ispa_absorbed_weight(W, dW, out=wb.t)
    o16, o32 = Guarded((rows, dim), torch.bfloat16, pad=7), Guarded((rows, dim), torch.float32, pad=7)
    lib.ispa_project(a, wb.t, out=o16.t)
    lib.ispa_project(a, wb.t, out=o32.t)
    wq, sc = Guarded((dim, dim), torch.int8, pad=2), Guarded((dim,), torch.float32, pad=4)
    lib.ispa_quantize_weight_int8(W, dW, wq_t=wq.t, w_scale=sc.t)
    o8 = Guarded((rows, dim), torch.float32, pad=7)
    ws = Guarded((lib.ispa_project_w8a8_workspace_size(rows, dim),), torch.uint8)
    lib.ispa_project_w8a8(a, wq.t, sc.t, out=o8.t, workspace=ws.t)
    torch.cuda.synchronize()
    for name, g in (("absorbed weight", wb), ("bf16 out", o16), ("fp32 out", o32),
                    ("int8 codes", wq), ("scales", sc), ("w8a8 out", o8), ("w8a8 workspace", ws)):
        assert g.intact(), name
    for name, g in (("absorbed weight", wb), ("bf16 out", o16), ("fp32 out", o32),
                    ("scales", sc), ("w8a8 out", o8)):
        assert g.written(), name
    assert torch.equal(wb.t.cpu(), (W + dW).to(torch.bfloat16).cpu())
    ref = lib.ispa_project(a, wb.t.contiguous(), out_dtype=torch.float32)
    ref8 = lib.ispa_project_w8a8(a, wq.t.contiguous(), sc.t.contiguous(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o32.t, ref) and torch.equal(o8.t, ref8)
