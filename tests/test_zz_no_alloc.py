"""The allocation-free absorb solve (ispa_absorb_solve_noalloc).

For callers that cannot allocate device memory when they need a solve (a
host program that owns every device buffer and has no allocator at hand, or
a loop that must never enter an allocator), the library keeps this solve's
scratch in a device array of its own. This checks, through the C ABI, that
two calls in a row -- the second one smaller, over the first one's leftover
scratch contents, then a larger one again -- give the workspace-based
solve's results within the Delta W tolerance of the other tests; that a call
after the first one's set-up leaves the device's allocated and free memory
unchanged; and that sizes beyond the array are refused. It runs last so that
a failure here leaves every other test run.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from ispa_synth import attention_like, gaussian

pytestmark = pytest.mark.gpu

DW_RELFRO = 2e-3


def make_problem(rows, dim, seed):
    a = attention_like(rows, dim, seed=seed).double().numpy()
    f = a + 0.4 * attention_like(rows, dim, seed=seed + 1, rho=0.5, common=0.1).double().numpy()
    G, R, S = oracle.gram(a, f - a)
    M = np.zeros((2 * dim, 2 * dim), np.float32)
    M[:dim, :dim], M[:dim, dim:], M[dim:, dim:] = G, R, S
    W = gaussian((dim, dim), seed, 0, "W") / math.sqrt(dim)
    return torch.from_numpy(M).cuda(), W.contiguous().cuda()


def rel_fro(a, b):
    return (torch.linalg.norm((a - b).double()) / torch.linalg.norm(b.double())).item()


def outputs(dim):
    return (torch.empty(dim, dim, dtype=torch.float32, device="cuda"),
            torch.empty(dim, dim, dtype=torch.float32, device="cuda"),
            torch.empty(1, dtype=torch.float32, device="cuda"),
            torch.zeros(1, dtype=torch.int32, device="cuda"))


def noalloc_call(lib, M, W, dim, out=None):
    dW, B, lam, status = outputs(dim) if out is None else out
    rc = lib._load().ispa_absorb_solve_noalloc(
        ctypes.c_void_p(M.data_ptr()), ctypes.c_void_p(W.data_ptr()), dim, 0.0,
        ctypes.c_void_p(dW.data_ptr()), ctypes.c_void_p(B.data_ptr()),
        ctypes.c_void_p(lam.data_ptr()), ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == lib.ISPA_OK, lib.ispa_status_string(rc)
    return dW, B, lam, status


def test_noalloc_solve_matches_workspace_solve_on_two_calls(lib):
    # the second call is smaller (stale scratch above it), the third larger
    # again (over the second call's leftovers)
    for dim, seed in ((512, 3), (256, 4), (512, 5)):
        M, W = make_problem(3 * dim, dim, seed)
        dW, B, lam, status = noalloc_call(lib, M, W, dim)
        ref = lib.ispa_absorb_solve(M, W)            # the workspace-based entry point
        torch.cuda.synchronize()
        assert int(status.item()) == 0 and int(ref["status"].item()) == 0
        assert lam.item() == ref["lam"].item()
        assert rel_fro(B, ref["B"]) <= 1e-6
        assert rel_fro(dW, ref["dW"]) <= DW_RELFRO


def test_noalloc_solve_refuses_sizes_beyond_its_array(lib):
    dim = 640
    M = torch.zeros(2 * dim, 2 * dim, device="cuda")
    W = torch.zeros(dim, dim, device="cuda")
    out = torch.zeros(dim, dim, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib._load().ispa_absorb_solve_noalloc(
        ctypes.c_void_p(M.data_ptr()), ctypes.c_void_p(W.data_ptr()), dim, 0.0,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(out.data_ptr()), None,
        ctypes.c_void_p(st.data_ptr()), None)
    assert rc == lib.ISPA_ERR_UNSUPPORTED


def test_noalloc_solve_allocates_nothing(lib):
    """After the first call on the device has looked up the array's address,
    a call changes neither torch's allocated bytes nor the device's free
    memory: every byte it touches is the caller's or the library's array."""
    dim = 384
    M, W = make_problem(3 * dim, dim, 7)
    noalloc_call(lib, M, W, dim)                      # set-up on this device
    torch.cuda.synchronize()
    out = outputs(dim)
    torch.cuda.synchronize()
    alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
    dW, _, _, status = noalloc_call(lib, M, W, dim, out)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0
    assert int(status.item()) == 0
    ref = lib.ispa_absorb_solve(M, W)
    torch.cuda.synchronize()
    assert rel_fro(dW, ref["dW"]) <= DW_RELFRO
