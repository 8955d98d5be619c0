"""The kernels' bounded waits, made to run out.

Every pipeline wait in the tensor-core kernels is bounded; when one gives up
the kernel records ISPA_STATUS_TIMEOUT in the call's status word, lets the
copies and tensor-core operations it already issued finish (those waits keep
the full 2 s limit), frees its tensor memory and returns. Here the limit is
set to 1 ns (``ispa_set_wait_limit_ns``), so a wait that is not satisfied at
once gives up: each pipelined kernel must report the timeout and leave the
context usable, and the next call on the same stream with the default limit
must match the oracle. Nothing here faults or hangs a GPU: the waits end by
themselves, and the kernels unwind.
"""
import numpy as np
import pytest
import torch

import oracle
from ispa_synth import attention_like, gaussian
from tests.test_gpu_parity import (check_attention, f64, random_chunk, ref_dual, rel_fro,
                                   run_dual, synthetic_layer, pack_M, to_dev, DW_RELFRO,
                                   GR_RELFRO)

pytestmark = pytest.mark.gpu


class short_waits:
    """Pipeline waits of the launches inside the block give up after 1 ns."""

    def __init__(self, lib):
        self.lib = lib

    def __enter__(self):
        torch.cuda.synchronize()
        self.lib.ispa_set_wait_limit_ns(1)

    def __exit__(self, *exc):
        torch.cuda.synchronize()
        self.lib.ispa_set_wait_limit_ns(0)
        return False


def test_attention_wait_gives_up_then_recovers(lib):
    ch = random_chunk(700, 300, 600, 2000, 4, 128, seed=21)
    dc = to_dev(ch)
    with short_waits(lib):
        out = run_dual(lib, dc)
    assert lib.read_status(out["status"]) & lib.ISPA_STATUS_TIMEOUT
    again = run_dual(lib, dc)
    torch.cuda.synchronize()
    assert lib.read_status(again["status"]) == 0
    check_attention(again, ref_dual(ch), "after a timed-out call")


def test_gram_wait_gives_up_then_recovers(lib):
    rows, dim = 3000, 512
    a = attention_like(rows, dim, seed=22)
    dm = 0.3 * attention_like(rows, dim, seed=23)
    st = lib.new_status("cuda")
    with short_waits(lib):
        lib.ispa_gram_accumulate(a.cuda(), dm.cuda(), status=st)
    assert lib.read_status(st) & lib.ISPA_STATUS_TIMEOUT
    st2 = lib.new_status("cuda")
    M = lib.ispa_gram_accumulate(a.cuda(), dm.cuda(), status=st2)
    torch.cuda.synchronize()
    assert lib.read_status(st2) == 0
    G, R, _ = oracle.gram(f64(a), f64(dm))
    up = np.arange(dim)[:, None] // 128 <= np.arange(dim)[None, :] // 128
    assert rel_fro(f64(M)[:dim, :dim][up], G[up]) <= GR_RELFRO
    assert rel_fro(f64(M)[:dim, dim:], R) <= GR_RELFRO


def test_solve_gemm_wait_gives_up_then_recovers(lib):
    """The absorb solve's 3xTF32 tensor-core GEMMs (and the weight Gram, one
    such GEMM)."""
    dim = 384
    a, f, W = synthetic_layer(3 * dim, dim, seed=24)
    G, R, S = oracle.gram(a, f - a)
    M = pack_M(G, R, S).cuda()
    Wd = W.cuda()
    with short_waits(lib):
        bad = lib.ispa_absorb_solve(M, Wd)
        st = lib.new_status("cuda")
        lib.ispa_weight_gram_batched(Wd[None], status=st)
    assert lib.read_status(bad["status"]) & lib.ISPA_STATUS_TIMEOUT
    assert lib.read_status(st) & lib.ISPA_STATUS_TIMEOUT
    good = lib.ispa_absorb_solve(M, Wd)
    P = lib.ispa_weight_gram_batched(Wd[None])
    torch.cuda.synchronize()
    assert lib.read_status(good["status"]) == 0
    dW_ref, _ = oracle.absorb(G, R, f64(W), oracle.default_lambda(G))
    assert rel_fro(f64(good["dW"]), dW_ref) <= DW_RELFRO
    assert rel_fro(f64(P[0]), f64(W) @ f64(W).T) <= 1e-5


def test_projection_waits_give_up_then_recover(lib):
    """The streaming projections: bf16 and int8 tensor-core GEMMs."""
    rows, dim = 700, 256
    a = gaussian((rows, dim), 25, 0, "X").to(torch.bfloat16).cuda()
    W = (gaussian((dim, dim), 26, 0, "W") / 16.0).cuda()
    wb = lib.ispa_absorbed_weight(W)
    wq, ws = lib.ispa_quantize_weight_int8(W)
    st1, st2 = lib.new_status("cuda"), lib.new_status("cuda")
    with short_waits(lib):
        lib.ispa_project(a, wb, out_dtype=torch.float32, status=st1)
        lib.ispa_project_w8a8(a, wq, ws, out_dtype=torch.float32, status=st2)
    assert lib.read_status(st1) & lib.ISPA_STATUS_TIMEOUT
    assert lib.read_status(st2) & lib.ISPA_STATUS_TIMEOUT
    ref = f64(a) @ f64(wb)
    out = lib.ispa_project(a, wb, out_dtype=torch.float32)
    out8 = lib.ispa_project_w8a8(a, wq, ws, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert rel_fro(f64(out), ref) <= 1e-5
    ref8, *_ = oracle.project_w8a8(a, W)
    assert rel_fro(f64(out8), ref8) <= 1e-6
