"""The proxy Hessian streamed over many calibration batches at the QuIP
paper's calibration size (Experiments, "Setup.": 128 segments of 2048
tokens = 262 144 tokens): quip_hessian_accumulate with accumulate = 1 over
16 384-token chunks, then quip_hessian_finalize with the total count,
against the FP64 oracle's X^T X / N accumulated over the same chunks."""
import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_09_b200 as Q
from post_weight_quantization_09_b200 import _lib as L
from quip_synth import calibration_chunks
from parity_util import host, rel_fro

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,N,chunk", [(4096, 262144, 16384)])
def test_streamed_hessian_at_calibration_size(n, N, chunk):
    Q.load()
    Q.quip_sync_status()
    H = torch.empty(n, n, device="cuda")
    acc = np.zeros((n, n))
    for a, X, xb in calibration_chunks(n, N, chunk, seed=5):
        Xd = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
        Q.quip_hessian_accumulate(Xd, H, accumulate=a > 0)
        acc += O.hessian(X) * X.shape[0]          # X^T X of the chunk, FP64
    Q.quip_hessian_finalize(H, N, 0.01)
    assert Q.quip_sync_status() == L.QUIP_OK
    ref = O.damp(acc / N, 0.01)
    err = rel_fro(host(H), ref)
    print(f"\nstreamed Hessian, n {n}, {N} tokens in chunks of {chunk}: rel-Fro {err:.3e}")
    assert err <= 1e-4
    # the finalized H is symmetric to the last bit
    Hh = host(H)
    assert np.array_equal(Hh, Hh.T)
