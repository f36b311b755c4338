"""GPU parity at the full sizes of the Llama-shaped layers, in the launch
configuration bench.py times (LayerQuantizer.run).  The FP64 oracle runs the
same seeded layer on the host; where the whole oracle would take too long it
runs on sampled rows (rows are independent once H~ and the transforms are
fixed)."""
import os
import time

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_09_b200 as Q
from post_weight_quantization_09_b200 import _lib as L
from quip_synth import CONFIGS, make_layer
from parity_util import dev, host, ldlq_trajectory_check, rel_fro, row_scaled_err

pytestmark = pytest.mark.gpu


def _run_device(cfg, d):
    q = Q.LayerQuantizer(cfg.m, cfg.n, cfg.m_side, cfg.n_side, cfg.bits, cfg.block, cfg.damp, cfg.seed)
    Wd = torch.from_numpy(d["W_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
    Xd = torch.from_numpy(d["X_bf16"].view(np.int16)).cuda().view(torch.bfloat16)
    # H before LDL overwrites it: run the first stages separately to keep a copy
    q.new_transform()
    Q.quip_hessian_accumulate(Xd, q.H)
    Q.quip_hessian_finalize(q.H, cfg.N, cfg.damp)
    H_dev = host(q.H)
    r = q.run(Wd, Xd)
    assert Q.quip_sync_status() == L.QUIP_OK
    return q, r, H_dev


def test_attn7b_full_layer():
    cfg = CONFIGS["attn7b"]
    d = make_layer(cfg)
    q, r, H_dev = _run_device(cfg, d)
    t0 = time.time()
    H = O.damp(O.hessian(d["X"]), cfg.damp)
    h_err = rel_fro(H_dev, H)
    assert h_err <= 1e-4, h_err
    U = O.make_side(cfg.seed, "m", "hadamard", cfg.m)
    V = O.make_side(cfg.seed, "n", "hadamard", cfg.n)
    Wt, Ht = O.incoherence_forward(d["W"], H, U, V)
    Uf, D = O.udu(Ht)
    lo, s = O.row_grid(Wt, cfg.bits)
    codes, Wt_hat, _ = O.ldlq(Wt, Uf, lo, s, cfg.bits)
    loss = O.proxy_loss(Wt_hat, Wt, Ht)
    C = host(r.codes)
    lo_d, s_d = host(r.lo), host(r.scale)
    agree = float((C == codes).mean())
    Wt_hat_d = O.dequantize(C, lo_d, s_d)
    loss_d = O.proxy_loss(Wt_hat_d, Wt, Ht)
    w_err = row_scaled_err(Wt_hat_d, Wt_hat, s, C == codes)
    bad, not_near = ldlq_trajectory_check(C, Wt, Uf, lo_d, s_d, cfg.bits, tau=1e-3)
    print(f"\nattn7b: H rel-Fro {h_err:.3e}  codes agree {agree:.6f}  loss {loss:.6g} vs {loss_d:.6g} "
          f"(rel {abs(loss_d - loss) / loss:.2e})  W^ err/s {w_err:.2e}  trajectory mismatch {bad:.2e} "
          f"(not near-tie {not_near:.2e})  oracle {time.time() - t0:.0f}s")
    assert abs(loss_d - loss) / loss <= 1e-3
    assert w_err <= 1e-4
    assert not_near == 0.0
    assert agree >= 0.999
    # sampled rows of the inverse transform: W^ = U^T W~^ V
    rows = np.random.default_rng(0).choice(cfg.m, 16, replace=False)
    Um, Vm = U.matrix(), V.matrix()
    W_hat_d = host(r.W_hat)
    for i in rows:
        ref_row = (Um[:, i] @ Wt_hat_d) @ Vm          # row i of U^T W~^ V
        assert np.abs(W_hat_d[i] - ref_row).max() <= 1e-4 * s_d.max()


def _sampled_layer_check(name, nrows=256):
    """Whole layer on the device vs the FP64 oracle on `nrows` sampled rows
    (the oracle forms H, H~ and its LDL in full; W~ and LDLQ only for the
    sampled rows, which is exact because rows are independent)."""
    cfg = CONFIGS[name]
    d = make_layer(cfg)
    q, r, H_dev = _run_device(cfg, d)
    Wt_dev = host(q.W_t)
    t0 = time.time()
    H = O.damp(O.hessian(d["X"]), cfg.damp)
    h_err = rel_fro(H_dev, H)
    U = O.make_side(cfg.seed, "m", cfg.m_side.kind, cfg.m, cfg.m_side.p, cfg.m_side.q)
    V = O.make_side(cfg.seed, "n", cfg.n_side.kind, cfg.n, cfg.n_side.p, cfg.n_side.q)
    Ht = O.incoherence_hessian(H, V)
    del H
    Uf, D = O.udu(Ht)
    rows = np.sort(np.random.default_rng(1).choice(cfg.m, nrows, replace=False))
    Wt = O.incoherence_rows(d["W"], U, V, rows)
    w_scale = np.abs(Wt).max()
    wt_err = np.abs(Wt_dev[rows] - Wt).max() / w_scale
    lo, s = O.row_grid(Wt, cfg.bits)
    codes, Wt_hat, _ = O.ldlq(Wt, Uf, lo, s, cfg.bits)
    C = host(r.codes)[rows]
    lo_d, s_d = host(r.lo)[rows], host(r.scale)[rows]
    agree = float((C == codes).mean())
    Wt_hat_d = O.dequantize(C, lo_d, s_d)
    loss = O.proxy_loss(Wt_hat, Wt, Ht)
    loss_d = O.proxy_loss(Wt_hat_d, Wt, Ht)
    w_err = row_scaled_err(Wt_hat_d, Wt_hat, s, C == codes)
    bad, not_near = ldlq_trajectory_check(C, Wt, Uf, lo_d, s_d, cfg.bits, tau=1e-3)
    print(f"\n{name}: H rel-Fro {h_err:.3e}  W~ err {wt_err:.2e}  codes agree {agree:.6f} on {nrows} rows  "
          f"loss {loss:.6g} vs {loss_d:.6g} (rel {abs(loss_d - loss) / loss:.2e})  W^ err/s {w_err:.2e}  "
          f"trajectory mismatch {bad:.2e} (not near-tie {not_near:.2e})  oracle {time.time() - t0:.0f}s")
    assert h_err <= 1e-4
    assert wt_err <= 1e-5
    assert abs(loss_d - loss) / loss <= 1e-3
    assert w_err <= 1e-4
    assert not_near == 0.0
    assert agree >= 0.999
    return q, r


@pytest.mark.parametrize("name", ["up7b", "down7b", "gate70b"])
def test_llama_layers_sampled_rows(name):
    _sampled_layer_check(name)
