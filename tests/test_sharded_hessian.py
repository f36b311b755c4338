"""The token-sharded proxy Hessian.  H is the second moment of the
calibration inputs (QuIP, adaptive-rounding section), a sum over tokens, so
ranks that each sum X^T X over their own tokens and add the partial sums
(one all-reduce) before finalizing with the total token count get the H of
all tokens.

On CPU (gloo ranks): token_range's split, and quip_hessian_sharded's
sequence (local sum -> allreduce_hessian -> finalize with N_total) with the
two device steps stood in for by host arithmetic that keeps their contract
(the strict upper triangle of the partial sum is left unspecified, here
NaN).  On the GPU: the same sequence on one rank, and two shards summed on
one device, against the oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import post_weight_quantization_09_b200 as Q
from quip_synth import random_layer
from parity_util import host, rel_fro

DAMP = 0.01


@pytest.mark.parametrize("N,world", [(0, 1), (5, 1), (5, 2), (7, 3), (2, 4), (1001, 2),
                                     (1000, 8), (3, 8)])
def test_token_range_partitions_the_tokens(N, world):
    spans = [Q.token_range(N, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == N
    for (_, a1), (b0, _) in zip(spans, spans[1:]):
        assert a1 == b0                                   # contiguous, no gap or overlap
    sizes = [b - a for a, b in spans]
    assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1
    assert sum(sizes) == N


def test_token_range_rejects_bad_arguments():
    for args in ((10, 0, 0), (10, 2, 2), (10, 2, -1), (-1, 2, 0)):
        with pytest.raises(ValueError):
            Q.token_range(*args)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _accumulate_on_host(X, H_acc, accumulate=False, stream=None):
    """quip_hessian_accumulate's contract on the host: the lower triangle
    holds X^T X of these tokens (zero for none), the strict upper triangle
    is unspecified."""
    Xd = X.numpy().astype(np.float64)
    S = np.tril(Xd.T @ Xd)
    S[np.triu_indices_from(S, 1)] = np.nan
    H_acc.copy_(torch.from_numpy(S))


def _finalize_on_host(H, N_total, damp, stream=None):
    """quip_hessian_finalize's contract on the host: reads the lower
    triangle only, H = sym / N_total + damping."""
    Lw = np.tril(H.numpy().astype(np.float64))
    S = Lw + np.tril(Lw, -1).T
    H.copy_(torch.from_numpy(O.damp(S / N_total, damp)))


def _rank_main(rank, world, port, N, n, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X = random_layer(8, n, N, seed=11)["X"]
        t0, t1 = Q.token_range(N, world, rank)
        Q.quip_hessian_accumulate = _accumulate_on_host
        Q.quip_hessian_finalize = _finalize_on_host
        H = torch.empty(n, n, dtype=torch.float32)
        Q.quip_hessian_sharded(torch.from_numpy(np.ascontiguousarray(X[t0:t1])), H, N, DAMP)
        out[rank] = H.numpy().copy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N", [(2, 1001), (3, 2)])
def test_gloo_ranks_finalize_the_hessian_of_all_tokens(world, N):
    n = 48
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, N, n, out), nprocs=world, join=True)
    X = random_layer(8, n, N, seed=11)["X"]
    ref = O.damp(O.hessian(X), DAMP)
    for r in range(world):
        assert np.all(np.isfinite(out[r]))
        assert np.array_equal(out[r], out[0])             # every rank holds the same H
        assert rel_fro(out[r], ref) <= 1e-6
    if world == 2:
        # one rank's tokens alone give a different H: the exchange is needed
        t0, t1 = Q.token_range(N, world, 0)
        alone = O.damp(O.hessian(X[t0:t1]), DAMP)
        assert rel_fro(alone, ref) > 1e-3


@pytest.mark.gpu
def test_sharded_hessian_on_the_device():
    n, N = 192, 1001
    d = random_layer(8, n, N, seed=11, dtype="bf16")
    X = torch.from_numpy(d["X_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
    ref = O.damp(O.hessian(d["X"]), DAMP)
    Q.load()
    # one rank, no process group: the plain accumulate + finalize, to the bit
    H1 = torch.empty(n, n, device="cuda")
    Q.quip_hessian_sharded(X, H1, N, DAMP)
    H0 = torch.empty(n, n, device="cuda")
    Q.quip_hessian_accumulate(X, H0)
    Q.quip_hessian_finalize(H0, N, DAMP)
    assert torch.equal(H1, H0)
    # the bound of the streamed Hessian tests; one token of 1001 left out or
    # counted twice moves H by about 1e-3
    tol = 1e-4
    assert rel_fro(host(H1), ref) <= tol
    # two shards of token_range summed on one device (the all-reduce's sum)
    parts = []
    for r in range(2):
        t0, t1 = Q.token_range(N, 2, r)
        P = torch.empty(n, n, device="cuda")
        Q.quip_hessian_accumulate(X[t0:t1], P)
        parts.append(P)
    H2 = parts[0] + parts[1]
    Q.quip_hessian_finalize(H2, N, DAMP)
    torch.cuda.synchronize()
    assert rel_fro(host(H2), ref) <= tol
