"""Layers that read the same input (q / k / v; up / gate) share one proxy
Hessian, one incoherence transform of it and one LDL; LDLQ runs on their
stacked rows.  Each layer's results must be exactly those of quantising it
alone with the same calibration inputs, and the FP64 oracle must agree."""
import numpy as np
import pytest

import oracle as O
import post_weight_quantization_09_b200 as Q
from post_weight_quantization_09_b200 import _lib as L
from quip_synth import Side, random_layer
from parity_util import dev, host, ldlq_trajectory_check

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G,m,n,mk,nk,bits", [
    (3, 256, 512, Side("hadamard"), Side("hadamard"), 2),
    (2, 96, 384, Side("kronecker", 12, 8), Side("kronecker", 3, 128), 3),
])
def test_layer_group_equals_single_layers_and_oracle(G, m, n, mk, nk, bits):
    Q.load()
    Q.quip_sync_status()
    seed, damp, block = 11, 0.01, 128
    layers = [random_layer(m, n, 1024, seed=100 + g) for g in range(G)]
    X = layers[0]["X"]                                # the shared calibration input
    grp = Q.LayerGroupQuantizer(G, m, n, mk, nk, bits, block, damp, seed)
    rg = grp.run([dev(d["W"]) for d in layers], dev(X))
    codes_g, lo_g, s_g, what_g = (t.cpu() for t in (rg.codes, rg.lo, rg.scale, rg.W_hat))
    assert Q.quip_sync_status() == L.QUIP_OK
    for g, d in enumerate(layers):
        one = Q.LayerQuantizer(m, n, mk, nk, bits, block, damp, seed)
        r1 = one.run(dev(d["W"]), dev(X))
        rows = slice(g * m, (g + 1) * m)
        # the same kernels on the same rows with the same factor: bit for bit
        assert (codes_g[rows] == r1.codes.cpu()).all()
        assert (lo_g[rows] == r1.lo.cpu()).all() and (s_g[rows] == r1.scale.cpu()).all()
        assert (what_g[rows] == r1.W_hat.cpu()).all()
    # the FP64 oracle on layer G - 1 with the shared X
    P = O.run_pipeline(layers[-1]["W"], X, seed, mk, nk, bits, damp)
    rows = slice((G - 1) * m, G * m)
    C = host(codes_g[rows])
    assert (C == P.codes).mean() >= 0.999
    lo, s = host(lo_g[rows]), host(s_g[rows])
    loss = O.proxy_loss(O.dequantize(C, lo, s), P.Wt, P.Ht)
    assert abs(loss - P.loss) / P.loss <= 1e-3
    bad, not_near = ldlq_trajectory_check(C, P.Wt, P.Uf, lo, s, bits, tau=1e-3)
    assert not_near == 0.0
    assert Q.quip_sync_status() == L.QUIP_OK
