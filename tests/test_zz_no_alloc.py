"""quip_ldlq_quantize_static: the LDLQ entry point that allocates nothing.

Some callers cannot call cudaMalloc (device memory owned by their own fixed
pool, a hard memory cap, or no tolerance for the synchronisation cudaMalloc /
cudaFree can cause); this entry point keeps its workspace in a fixed array of
the library's device memory instead.  Called through the C ABI directly, it
must give the same codes and grid as quip_ldlq_quantize with a
caller-allocated workspace, on two calls in a row (the second one finds the
first one's leftovers in the shared array), and reject layers whose
workspace does not fit the array."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_09_b200 as Q
from post_weight_quantization_09_b200 import _lib as L

pytestmark = pytest.mark.gpu

STATIC_BYTES = 16 << 20


def _inputs(m, n, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((2 * n, n))
    X[:, rng.choice(n, max(1, n // 50), replace=False)] *= 20
    U, _ = O.udu(O.damp(O.hessian(X), 0.01))
    W = rng.standard_normal((m, n)) * 0.02
    return (torch.tensor(W, dtype=torch.float32, device="cuda"),
            torch.tensor(U, dtype=torch.float32, device="cuda"))


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_static_workspace_matches_allocating_entry_point():
    lib = Q.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [(512, 1024, 2, 128, 3), (64, 128, 3, 32, 4)]        # two calls in a row
    for m, n, bits, block, seed in cases:
        W, U = _inputs(m, n, seed)
        ref = [torch.empty(m, n, dtype=torch.uint8, device="cuda"),
               torch.empty(m, device="cuda"), torch.empty(m, device="cuda")]
        Q.quip_ldlq_quantize(W, U, bits, block, *ref)
        out = [torch.full((m, n), 255, dtype=torch.uint8, device="cuda"),
               torch.full((m,), float("nan"), device="cuda"), torch.full((m,), float("nan"), device="cuda")]
        st = lib.quip_ldlq_quantize_static(_p(W), _p(U), U.stride(0), m, n, bits, block,
                                           _p(out[0]), _p(out[1]), _p(out[2]), stream)
        assert st == L.QUIP_OK, L.status_string(st)
        assert Q.quip_sync_status() == L.QUIP_OK
        assert torch.equal(out[0], ref[0])
        assert torch.equal(out[1], ref[1]) and torch.equal(out[2], ref[2])


def test_static_workspace_rejects_layers_that_do_not_fit():
    lib = Q.load()
    # A 4096 x 4096 layer needs m*n*4 (accumulator) + 3*m*n*2 (error pieces)
    # + 3*n*n*2 (factor pieces) + n*n*4 (fp32 factor) bytes, each rounded up
    # to 256, far more than the 16 MiB array: rejected before any launch.
    # The pointers are NULL, so should the size check ever regress, the call
    # stops at the argument check (QUIP_ERR_ARG) instead of launching.
    st = lib.quip_ldlq_quantize_static(None, None, 4096, 4096, 4096, 2, 128, None, None, None, None)
    assert st == L.QUIP_ERR_WORKSPACE
    need = Q.quip_workspace_size(L.QUIP_OP_LDLQ, None, 1024, 4096, 128)
    assert need > STATIC_BYTES
    assert Q.quip_workspace_size(L.QUIP_OP_LDLQ, None, 512, 1024, 128) <= STATIC_BYTES
