"""GPU parity, stage by stage: each CUDA stage, called through the C ABI on
seeded inputs, against the FP64 oracle on the same inputs.  Sizes span
several tiles with ragged tails; edge cases included."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_09_b200 as Q
from post_weight_quantization_09_b200 import _lib as L
from quip_synth import CONFIGS, Side, make_layer, random_layer, round_to_bf16
from parity_util import dev, host, ldlq_trajectory_check, rel_fro, row_scaled_err

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    Q.load()
    Q.quip_sync_status()
    yield
    # no stage may leave a device-side error behind
    assert Q.quip_sync_status() == L.QUIP_OK


# ---------------------------------------------------------------- transforms


@pytest.mark.parametrize("m,n,mk,nk", [
    (64, 128, Side("hadamard"), Side("hadamard")),
    (8, 2048, Side("hadamard"), Side("hadamard")),
    (48, 86 * 3, Side("kronecker", 6, 8), Side("kronecker", 86, 3)),
    (224, 32, Side("kronecker", 224, 1), Side("identity")),
    (64, 128, Side("hadamard", permute=True), Side("hadamard", permute=True)),
    (28672, 48, Side("kronecker", 224, 128, True), Side("identity", permute=True)),
])
def test_transform_factors_match_oracle(m, n, mk, nk):
    tf = Q.Transform(1234, m, n, mk, nk)
    for side, spec, dim in ((0, mk, m), (1, nk, n)):
        f = tf.factors(side)
        ref = O.make_side(1234, "m" if side == 0 else "n", spec.kind, dim, spec.p, spec.q,
                          spec.permute)
        if spec.permute:
            np.testing.assert_array_equal(f["perm"].cpu().numpy(), ref.perm)
        else:
            assert "perm" not in f
        if spec.kind == "hadamard":
            np.testing.assert_array_equal(host(f["signs"]), ref.signs)
        elif spec.kind == "kronecker":
            np.testing.assert_allclose(host(f["A"]), ref.A, atol=2e-7)
            np.testing.assert_allclose(host(f["B"]), ref.B, atol=2e-7)
    tf.close()


def test_transform_redraw_in_place():
    tf = Q.Transform(1, 96, 64, Side("kronecker", 12, 8), Side("hadamard"))
    tf.draw(99)
    ref_m = O.make_side(99, "m", "kronecker", 96, 12, 8)
    ref_n = O.make_side(99, "n", "hadamard", 64)
    np.testing.assert_allclose(host(tf.factors(0)["A"]), ref_m.A, atol=2e-7)
    np.testing.assert_array_equal(host(tf.factors(1)["signs"]), ref_n.signs)
    tf.close()


@pytest.mark.parametrize("m,n,mk,nk,dtype", [
    (64, 128, Side("hadamard"), Side("hadamard"), "f32"),
    (512, 1024, Side("hadamard"), Side("hadamard"), "bf16"),
    (4096, 64, Side("hadamard"), Side("hadamard"), "bf16"),     # 2 column passes
    (8, 8192, Side("hadamard"), Side("hadamard"), "f32"),       # largest row FWHT
    (4, 8, Side("hadamard"), Side("hadamard"), "f32"),          # register-only paths
    (96, 86 * 2, Side("kronecker", 12, 8), Side("kronecker", 86, 2), "bf16"),
    (30, 64, Side("identity"), Side("hadamard"), "bf16"),
    # random permutation within the fast orthogonal multiplication
    (64, 128, Side("hadamard", permute=True), Side("hadamard", permute=True), "bf16"),
    (512, 1024, Side("identity"), Side("hadamard", permute=True), "f32"),
    (96, 86 * 2, Side("kronecker", 12, 8, True), Side("kronecker", 86, 2, True), "f32"),
    (30, 64, Side("identity", permute=True), Side("identity", permute=True), "bf16"),
    # m-side Kronecker factors on the tensor cores: K = 86 (not a multiple of
    # the 64-row K block) with 128-row slabs; two 128-row output tiles (p = 200)
    # and a ragged 72-column tile; an fp32 source split into bf16 pieces
    (11008, 64, Side("kronecker", 86, 128), Side("hadamard"), "bf16"),
    (3200, 72, Side("kronecker", 200, 16), Side("identity"), "bf16"),
    (96, 64, Side("kronecker", 12, 8), Side("hadamard"), "f32"),
])
def test_incoherence_forward_inverse(m, n, mk, nk, dtype):
    d = random_layer(m, n, min(4 * n, 2048), seed=m + n, dtype=dtype)
    W, X = d["W"], d["X"]
    H = O.damp(O.hessian(X), 0.01)
    U = O.make_side(7, "m", mk.kind, m, mk.p, mk.q, mk.permute)
    V = O.make_side(7, "n", nk.kind, n, nk.p, nk.q, nk.permute)
    with_h = n <= 4096          # the explicit FP64 V H V^T is slow beyond that
    Wt_ref, Ht_ref = O.incoherence_forward(W, H if with_h else np.eye(1), U, V) if with_h else \
        (U.matrix() @ W @ V.matrix().T, None)
    tf = Q.Transform(7, m, n, mk, nk)
    Wd = dev(W, torch.bfloat16 if dtype == "bf16" else torch.float32)
    Wt = torch.empty(m, n, device="cuda")
    Hd = dev(H) if with_h else None
    Q.quip_incoherence_forward(tf, Wd, Wt, Hd)
    scale_w = np.abs(Wt_ref).max()
    assert np.abs(host(Wt) - Wt_ref).max() <= 2e-6 * scale_w
    if with_h:
        assert rel_fro(host(Hd), Ht_ref) <= 2e-6
    back = torch.empty_like(Wt)
    Q.quip_incoherence_inverse(tf, Wt, back)
    assert np.abs(host(back) - W).max() <= 4e-6 * np.abs(W).max()
    Q.quip_incoherence_inverse(tf, Wt, Wt)                       # in place
    assert np.abs(host(Wt) - W).max() <= 4e-6 * np.abs(W).max()
    tf.close()


# ---------------------------------------------------------------- Hessian


@pytest.mark.parametrize("N,n,dtype", [
    (1024, 128, "f32"), (1000, 320, "bf16"), (777, 576, "bf16"), (4096, 256, "bf16"),
    (64, 64, "bf16"), (130, 40, "bf16"), (33, 7, "f32"),
])
def test_hessian_accumulate_and_finalize(N, n, dtype):
    d = random_layer(4, n, N, seed=N + n, dtype=dtype, x_outlier_frac=0.05, lognormal=False)
    X = d["X"]
    ref = O.damp(O.hessian(X), 0.01)
    Xd = dev(X, torch.bfloat16 if dtype == "bf16" else torch.float32)
    H = torch.full((n, n), float("nan"), device="cuda")
    Q.quip_hessian_accumulate(Xd, H)
    # bf16 products are exact; the tensor cores' fp32 sums lose about one ulp
    # per 16-token MMA step, bounded by the kernel's 2048-token chunks
    tol = 2e-5 if dtype == "bf16" else 1e-5
    lower = np.tril(host(H))
    assert rel_fro(lower, np.tril(X.astype(np.float64).T @ X)) <= tol
    Q.quip_hessian_finalize(H, N, 0.01)
    Hh = host(H)
    np.testing.assert_array_equal(Hh, Hh.T)
    assert rel_fro(Hh, ref) <= tol


def test_hessian_streams_token_chunks():
    d = random_layer(4, 320, 1500, seed=5, dtype="bf16", x_outlier_frac=0.02, lognormal=False)
    X = d["X"]
    Xd = dev(X, torch.bfloat16)
    H = torch.empty(320, 320, device="cuda")
    Q.quip_hessian_accumulate(Xd[:700], H, accumulate=False)
    Q.quip_hessian_accumulate(Xd[700:1200], H, accumulate=True)
    Q.quip_hessian_accumulate(Xd[1200:], H, accumulate=True)
    Q.quip_hessian_finalize(H, 1500, 0.01)
    assert rel_fro(host(H), O.damp(O.hessian(X), 0.01)) <= 1e-4


def test_hessian_zero_tokens_and_strided_x():
    H = torch.full((64, 64), 3.0, device="cuda")
    Q.quip_hessian_accumulate(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"), H)
    assert torch.all(torch.tril(H) == 0)
    d = random_layer(4, 64, 256, seed=2, dtype="bf16")
    big = torch.zeros(256, 128, dtype=torch.bfloat16, device="cuda")
    big[:, :64] = dev(d["X"], torch.bfloat16)
    Q.quip_hessian_accumulate(big[:, :64], H)                   # row stride 128
    assert rel_fro(np.tril(host(H)), np.tril(d["X"].astype(np.float64).T @ d["X"])) <= 1e-4


# ---------------------------------------------------------------- LDL


@pytest.mark.parametrize("n", [16, 128, 200, 516])
def test_ldl_matches_oracle(n):
    rng = np.random.default_rng(n)
    X = rng.standard_normal((3 * n, n)) * np.exp(rng.standard_normal(n))
    H = O.damp(O.hessian(X), 0.01).astype(np.float32).astype(np.float64)
    U_ref, D_ref = O.udu(H)
    Hd = dev(H)
    D = torch.empty(n, device="cuda")
    Q.quip_ldl(Hd, D)
    U = np.triu(host(Hd), 1)
    # forward error within 10x of what an fp32 LAPACK factorisation reaches
    J = np.arange(n)[::-1]
    L32 = np.linalg.cholesky(H[np.ix_(J, J)].astype(np.float32)).astype(np.float64)
    R32 = L32[np.ix_(J, J)]
    U32 = np.triu(R32 / np.diag(R32)[None, :], 1)
    err32 = np.abs(U32 - U_ref).max()
    assert np.abs(U - U_ref).max() <= 10 * err32 + 1e-6
    assert rel_fro(host(D), D_ref) <= 10 * rel_fro(np.diag(R32) ** 2, D_ref) + 1e-6
    # backward error of the device factor, in FP64
    R = (np.eye(n) + U) @ np.diag(host(D)) @ (np.eye(n) + U).T
    assert rel_fro(R, H) <= 2e-6


def test_ldl_panel_grid_beyond_one_wave():
    # n = 9728: the first panel's solve runs on 150 CTAs (more than one per SM),
    # so CTAs of a later wave must still see the unfactored diagonal block.
    n = 9728
    rng = np.random.default_rng(5)
    G = rng.standard_normal((n, 64))
    H = (np.eye(n) * 0.5 + G @ G.T / 64).astype(np.float32).astype(np.float64)
    U_ref, D_ref = O.udu(H)
    Hd = dev(H)
    D = torch.empty(n, device="cuda")
    Q.quip_ldl(Hd, D)
    assert Q.quip_sync_status() == L.QUIP_OK
    U = host(Hd)
    rows = rng.choice(n, 64, replace=False)
    for i in rows:
        np.testing.assert_allclose(U[i, i + 1:], U_ref[i, i + 1:], atol=5e-4)
    np.testing.assert_allclose(host(D), D_ref, rtol=5e-4)


def test_ldl_rejects_unaligned_order():
    with pytest.raises(Q.QuipError) as e:
        Q.quip_ldl(torch.eye(513, device="cuda"), torch.empty(513, device="cuda"))
    assert e.value.status == L.QUIP_ERR_SHAPE


def test_ldl_diagonal_and_not_pd():
    d = np.array([3.0, 1.0, 2.0, 5.0] * 20, dtype=np.float32)
    Hd = dev(np.diag(d))
    D = torch.empty(80, device="cuda")
    Q.quip_ldl(Hd, D)
    assert np.all(np.triu(host(Hd), 1) == 0)
    np.testing.assert_allclose(host(D), d, rtol=1e-6)
    bad = np.eye(72, dtype=np.float32)
    bad[3, 5] = bad[5, 3] = 2.0                                  # indefinite
    Q.quip_ldl(dev(bad), torch.empty(72, device="cuda"))
    assert Q.quip_sync_status() == L.QUIP_ERR_NOT_PD


# ---------------------------------------------------------------- LDLQ


def _ldlq_inputs(m, n, seed, const_rows=()):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((2 * n, n))
    X[:, rng.choice(n, max(1, n // 50), replace=False)] *= 20
    H = O.damp(O.hessian(X), 0.01)
    U, _ = O.udu(H)
    W = rng.standard_normal((m, n)) * 0.02
    for r in const_rows:
        W[r] = 0.37
    return W.astype(np.float32).astype(np.float64), U.astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("m,n,bits,block", [
    (64, 128, 2, 32), (100, 256, 3, 64), (33, 256, 4, 128), (256, 128, 2, 128), (1, 64, 8, 64),
    (70, 512, 2, 128), (40, 320, 3, 64), (129, 192, 2, 32),
    # more 32-row units than SMs: two units per CTA, the last CTA's second
    # unit partly past the last row
    (4800 + 17, 192, 2, 64),
])
def test_ldlq_stage_parity(m, n, bits, block):
    W, U = _ldlq_inputs(m, n, seed=m * n + bits, const_rows=(0,) if m > 1 else ())
    lo_ref, s_ref = O.row_grid(W, bits)
    c_ref, _, _ = O.ldlq(W, U, lo_ref, s_ref, bits)
    codes = torch.empty(m, n, dtype=torch.uint8, device="cuda")
    lo = torch.empty(m, device="cuda")
    sc = torch.empty(m, device="cuda")
    Ud = dev(U)
    Q.quip_ldlq_quantize(dev(W), Ud, bits, block, codes, lo, sc)
    C = host(codes)
    np.testing.assert_array_equal(host(lo), lo_ref)              # min is exact
    np.testing.assert_allclose(host(sc), s_ref, rtol=3e-7)
    agree = (C == c_ref).mean()
    assert agree >= 0.999, agree
    bad, not_near = ldlq_trajectory_check(C, W, U, host(lo), host(sc), bits, tau=1e-4)
    assert not_near == 0.0, (bad, not_near)
    if m > 1:
        assert np.all(C[0] == 0)                                 # constant row: s = 1, codes 0


def test_ldlq_identity_feedback_is_nearest():
    # Ů = 0: LDLQ reduces to nearest rounding (QuIP, Experiments, "Methods."),
    # compared with the FP64 oracle's nearest rounding on the device's grid;
    # the two may only differ where z sits within fp32 rounding of a .5 tie
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((50, 128)) * 0.02).astype(np.float32)
    codes = torch.empty(50, 128, dtype=torch.uint8, device="cuda")
    lo = torch.empty(50, device="cuda")
    sc = torch.empty(50, device="cuda")
    Q.quip_ldlq_quantize(dev(W), torch.zeros(128, 128, device="cuda"), 3, 64, codes, lo, sc)
    lo_h, s_h = host(lo), host(sc)
    want = O.nearest(W.astype(np.float64), lo_h, s_h, 3)
    got = host(codes)
    z = (W.astype(np.float64) - lo_h[:, None]) / s_h[:, None]
    near_tie = np.abs(z - np.floor(z) - 0.5) < 1e-5
    assert np.all((got == want) | near_tie)
    assert (got == want).mean() >= 0.999


def test_ldlq_block_invariance_on_device():
    W, U = _ldlq_inputs(128, 256, seed=11)
    out = []
    for block in (32, 64, 128):
        codes = torch.empty(128, 256, dtype=torch.uint8, device="cuda")
        lo, sc = torch.empty(128, device="cuda"), torch.empty(128, device="cuda")
        Q.quip_ldlq_quantize(dev(W), dev(U), 2, block, codes, lo, sc)
        out.append(host(codes))
    assert (out[0] == out[1]).mean() >= 0.999 and (out[0] == out[2]).mean() >= 0.999


def test_ldlq_nonfinite_weight_is_reported():
    W = np.zeros((32, 64), dtype=np.float32)
    W[5, 7] = np.nan
    codes = torch.empty(32, 64, dtype=torch.uint8, device="cuda")
    lo, sc = torch.empty(32, device="cuda"), torch.empty(32, device="cuda")
    Q.quip_ldlq_quantize(dev(W), torch.zeros(64, 64, device="cuda"), 2, 32, codes, lo, sc)
    assert Q.quip_sync_status() == L.QUIP_ERR_NONFINITE


def test_dequantize_exact():
    rng = np.random.default_rng(0)
    C = rng.integers(0, 16, size=(37, 64)).astype(np.uint8)
    lo = rng.standard_normal(37).astype(np.float32)
    s = rng.uniform(0.01, 0.1, 37).astype(np.float32)
    out = torch.empty(37, 64, device="cuda")
    Q.quip_dequantize(dev(C, torch.uint8), dev(lo), dev(s), out)
    want = O.dequantize(C, lo, s)
    assert np.abs(host(out) - want).max() <= 1e-6 * np.abs(want).max()


# ---------------------------------------------------------------- whole layer


def test_tiny_config_pipeline():
    cfg = CONFIGS["tiny"]
    d = make_layer(cfg)
    P = O.run_pipeline(d["W"], d["X"], cfg.seed, cfg.m_side, cfg.n_side, cfg.bits, cfg.damp)
    q = Q.LayerQuantizer(cfg.m, cfg.n, cfg.m_side, cfg.n_side, cfg.bits, cfg.block, cfg.damp, cfg.seed)
    r = q.run(dev(d["W"]), dev(d["X"]))
    assert Q.quip_sync_status() == L.QUIP_OK
    C = host(r.codes)
    assert (C == P.codes).mean() >= 0.999
    lo, s = host(r.lo), host(r.scale)
    Wt_hat = O.dequantize(C, lo, s)
    loss = O.proxy_loss(Wt_hat, P.Wt, P.Ht)
    assert abs(loss - P.loss) / P.loss <= 1e-3
    assert row_scaled_err(Wt_hat, P.Wt_hat, s, C == P.codes) <= 1e-4
    # device inverse transform vs the oracle's inverse of the device codes
    W_hat_ref = O.incoherence_inverse(Wt_hat, P.U, P.V)
    assert np.abs(host(r.W_hat) - W_hat_ref).max() <= 1e-4 * s.max()
    bad, not_near = ldlq_trajectory_check(C, P.Wt, P.Uf, lo, s, cfg.bits, tau=1e-3)
    assert not_near == 0.0


def test_incoherence_forward_h_only_then_w_only_equals_joint():
    m, n = 64, 256
    tf = Q.Transform(77, m, n, Side("hadamard"), Side("kronecker", 16, 16))
    d = random_layer(m, n, 512, seed=5)
    W = dev(d["W"])
    H0 = dev(d["X"].T.astype(np.float64) @ d["X"] / 512.0)
    Wt1, H1 = torch.empty(m, n, device="cuda"), H0.clone()
    Q.quip_incoherence_forward(tf, W, Wt1, H1)
    Wt2, H2 = torch.empty(m, n, device="cuda"), H0.clone()
    Q.quip_incoherence_forward(tf, None, None, H2)
    Q.quip_incoherence_forward(tf, W, Wt2, None)
    assert torch.equal(Wt1, Wt2) and torch.equal(H1, H2)
    with pytest.raises(Q.QuipError):
        Q.quip_incoherence_forward(tf, None, None, None)


def test_run_host_equals_device_run():
    cfg = CONFIGS["tiny"]
    d = make_layer(cfg)
    q = Q.LayerQuantizer(cfg.m, cfg.n, cfg.m_side, cfg.n_side, cfg.bits, cfg.block, cfg.damp, cfg.seed)
    r = q.run(dev(d["W"]), dev(d["X"]))
    codes, lo, sc = r.codes.cpu(), r.lo.cpu(), r.scale.cpu()
    q2 = Q.LayerQuantizer(cfg.m, cfg.n, cfg.m_side, cfg.n_side, cfg.bits, cfg.block, cfg.damp, cfg.seed)
    Wh = torch.from_numpy(d["W"]).pin_memory()
    Xh = torch.from_numpy(d["X"]).pin_memory()
    co = torch.empty(cfg.m, cfg.n, dtype=torch.uint8).pin_memory()
    lo_h = torch.empty(cfg.m).pin_memory()
    sc_h = torch.empty(cfg.m).pin_memory()
    for _ in range(2):                                 # twice: the buffers are reused
        co.zero_(), lo_h.zero_(), sc_h.zero_()
        q2.run_host(Wh, Xh, co, lo_h, sc_h)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(co, codes) and torch.equal(lo_h, lo) and torch.equal(sc_h, sc)


@pytest.mark.parametrize("n,nk,block", [
    (1088, Side("kronecker", 17, 64), 64),     # 9 column blocks, the last 64 wide: 5 chunks of 2
    (2048, Side("hadamard"), 128),             # 16 blocks: 8 chunks of 2
])
def test_host_call_streams_the_codes_back(n, nk, block):
    """quip_quantize_layer_host copies the codes back in column chunks while
    LDLQ runs (about eight, each after the block kernels that finish its
    columns): with one token chunk (the same Hessian) the host codes, grid and
    W^ are the device call's to the bit, including a last 64-wide block."""
    m, N, bits, seed = 256, 1024, 3, 5
    mk = Side("hadamard")
    d = random_layer(m, n, N, seed=17, dtype="bf16")
    q = Q.LayerQuantizer(m, n, mk, nk, bits, block, 0.01, seed)
    r = q.run(dev(d["W"], torch.bfloat16), dev(d["X"], torch.bfloat16))
    assert Q.quip_sync_status() == L.QUIP_OK
    codes, lo, sc = r.codes.cpu(), r.lo.cpu(), r.scale.cpu()
    W_hat = r.W_hat.cpu()
    Wh = torch.from_numpy(d["W_bf16"].view(np.int16)).view(torch.bfloat16).pin_memory()
    Xh = torch.from_numpy(d["X_bf16"].view(np.int16)).view(torch.bfloat16).pin_memory()
    co = torch.full((m, n), 255, dtype=torch.uint8).pin_memory()
    lo_h, sc_h = torch.empty(m).pin_memory(), torch.empty(m).pin_memory()
    wh = torch.empty(m, n).pin_memory()
    q2 = Q.LayerQuantizer(m, n, mk, nk, bits, block, 0.01, seed)
    ws = torch.empty(Q.quip_layer_workspace_size(q2.tf, N, L.QUIP_BF16, L.QUIP_BF16, block, True),
                     dtype=torch.uint8, device="cuda")
    Q.quip_quantize_layer_host(q2.tf, seed, Wh, Xh, bits, block, 0.01, co, lo_h, sc_h, wh, ws)
    torch.cuda.current_stream().synchronize()
    assert Q.quip_sync_status() == L.QUIP_OK
    assert torch.equal(co, codes) and torch.equal(lo_h, lo) and torch.equal(sc_h, sc)
    assert torch.equal(wh, W_hat)


def test_layer_call_equals_the_stages_and_the_oracle():
    """quip_quantize_layer (one library call) runs the same kernels in the
    same order as the stage-by-stage calls: identical codes, grid and W^;
    and both match the oracle on a layer with a Kronecker m side."""
    m, n, N, bits, block, seed = 1024, 512, 3000, 3, 128, 9
    mk, nk = Side("kronecker", 8, 128), Side("hadamard")
    d = random_layer(m, n, N, seed=13, dtype="bf16")
    W = dev(d["W"], torch.bfloat16)
    X = dev(d["X"], torch.bfloat16)
    staged = Q.LayerQuantizer(m, n, mk, nk, bits, block, 0.01, seed)
    staged.new_transform()
    Q.quip_hessian_accumulate(X, staged.H)
    Q.quip_hessian_finalize(staged.H, N, 0.01)
    Q.quip_incoherence_forward(staged.tf, None, None, staged.H, staged.ws)
    Q.quip_ldl(staged.H, staged.D, staged.ws)
    Q.quip_incoherence_forward(staged.tf, W, staged.W_t, None, staged.ws)
    Q.quip_ldlq_quantize(staged.W_t, staged.H, bits, block, staged.codes, staged.lo, staged.scale, staged.ws)
    Q.quip_dequantize(staged.codes, staged.lo, staged.scale, staged.W_hat)
    Q.quip_incoherence_inverse(staged.tf, staged.W_hat, staged.W_hat, staged.ws)
    q = Q.LayerQuantizer(m, n, mk, nk, bits, block, 0.01, seed)
    r = q.run(W, X)                                     # quip_quantize_layer
    assert Q.quip_sync_status() == L.QUIP_OK
    assert torch.equal(r.codes, staged.codes)
    assert torch.equal(r.lo, staged.lo) and torch.equal(r.scale, staged.scale)
    assert torch.equal(r.W_hat, staged.W_hat)
    assert torch.equal(q.W_t, staged.W_t) and torch.equal(q.D, staged.D)
    P = O.run_pipeline(d["W"], d["X"], seed, mk, nk, bits, 0.01)
    C = host(r.codes)
    assert (C == P.codes).mean() >= 0.999
    lo, s = host(r.lo), host(r.scale)
    assert abs(O.proxy_loss(O.dequantize(C, lo, s), P.Wt, P.Ht) - P.loss) / P.loss <= 1e-3
    bad, not_near = ldlq_trajectory_check(C, P.Wt, P.Uf, lo, s, bits, tau=1e-3)
    assert not_near == 0.0
    # host in, host out, with W^ copied back; X arrives in two token chunks
    Wh = torch.from_numpy(d["W_bf16"].view(np.int16)).view(torch.bfloat16).pin_memory()
    Xh = torch.from_numpy(d["X_bf16"].view(np.int16)).view(torch.bfloat16).pin_memory()
    co = torch.empty(m, n, dtype=torch.uint8).pin_memory()
    lo_h, sc_h = torch.empty(m).pin_memory(), torch.empty(m).pin_memory()
    wh = torch.empty(m, n).pin_memory()
    ws = torch.empty(Q.quip_layer_workspace_size(q.tf, N, L.QUIP_BF16, L.QUIP_BF16, block, True),
                     dtype=torch.uint8, device="cuda")
    for _ in range(2):                                  # twice: leftovers in the workspace
        co.zero_(), lo_h.zero_(), sc_h.zero_(), wh.zero_()
        Q.quip_quantize_layer_host(q.tf, seed, Wh, Xh, bits, block, 0.01, co, lo_h, sc_h, wh, ws)
        torch.cuda.current_stream().synchronize()
        assert Q.quip_sync_status() == L.QUIP_OK
        # the Hessian of two chunks differs from one pass by fp32 rounding only
        assert (co.numpy() == C).mean() >= 0.999
        np.testing.assert_array_equal(lo_h.numpy(), host(r.lo))
        np.testing.assert_allclose(wh.numpy(), host(r.W_hat), atol=1e-4 * s.max())


@pytest.mark.parametrize("n,mk", [
    (8192, Side("kronecker", 8, 128)), (8192, Side("hadamard")),
    (4096, Side("kronecker", 8, 128)), (4096, Side("identity")),
])
def test_layer_fused_row_kernels_equal_the_stages(n, mk):
    """The layer call's fused row kernels on 4096- and 8192-point Hadamard n
    sides: with a tensor-core Kronecker m side the forward row kernel also
    writes LDLQ's accumulator and the per-row grid, and the inverse row
    kernel reads the codes (the dequantisation folded in) and writes the
    bf16 pieces the Kronecker products take.  Codes, grid, W~ and W^ equal the
    stage calls' to the bit, and W^ the oracle's U^T W~^ V of those codes
    within 1e-4 of the row scale on sampled rows."""
    m, N, bits, block, seed = 1024, 256, 2, 128, 21
    nk = Side("hadamard")
    d = random_layer(m, n, N, seed=31, dtype="bf16")
    W, X = dev(d["W"], torch.bfloat16), dev(d["X"], torch.bfloat16)
    st = Q.LayerQuantizer(m, n, mk, nk, bits, block, 0.01, seed)
    st.new_transform()
    Q.quip_hessian_accumulate(X, st.H)
    Q.quip_hessian_finalize(st.H, N, 0.01)
    Q.quip_incoherence_forward(st.tf, None, None, st.H, st.ws)
    Q.quip_ldl(st.H, st.D, st.ws)
    Q.quip_incoherence_forward(st.tf, W, st.W_t, None, st.ws)
    Q.quip_ldlq_quantize(st.W_t, st.H, bits, block, st.codes, st.lo, st.scale, st.ws)
    Q.quip_dequantize(st.codes, st.lo, st.scale, st.W_hat)
    Q.quip_incoherence_inverse(st.tf, st.W_hat, st.W_hat, st.ws)
    q = Q.LayerQuantizer(m, n, mk, nk, bits, block, 0.01, seed)
    r = q.run(W, X)
    assert Q.quip_sync_status() == L.QUIP_OK
    assert torch.equal(q.W_t, st.W_t)
    assert torch.equal(r.lo, st.lo) and torch.equal(r.scale, st.scale)
    assert torch.equal(r.codes, st.codes)
    assert torch.equal(r.W_hat, st.W_hat)
    C, lo, s = host(r.codes), host(r.lo), host(r.scale)
    U = O.make_side(seed, "m", mk.kind, m, mk.p, mk.q)
    V = O.make_side(seed, "n", nk.kind, n)
    rows = np.random.default_rng(3).choice(m, 12, replace=False)
    ref = O.incoherence_inverse_rows(O.dequantize(C, lo, s), U, V, rows)
    assert np.abs(host(r.W_hat)[rows] - ref).max() <= 1e-4 * s.max()


@pytest.mark.parametrize("mk,nk", [
    (Side("hadamard", permute=True), Side("hadamard", permute=True)),
    (Side("kronecker", 8, 8, True), Side("hadamard", permute=True)),
])
def test_pipeline_with_random_permutations(mk, nk):
    m, n, bits, block, seed = 64, 256, 2, 128, 3
    d = random_layer(m, n, 1024, seed=41)
    P = O.run_pipeline(d["W"], d["X"], seed, mk, nk, bits, 0.01)
    q = Q.LayerQuantizer(m, n, mk, nk, bits, block, 0.01, seed)
    r = q.run(dev(d["W"]), dev(d["X"]))
    assert Q.quip_sync_status() == L.QUIP_OK
    C = host(r.codes)
    assert (C == P.codes).mean() >= 0.999
    lo, s = host(r.lo), host(r.scale)
    Wt_hat = O.dequantize(C, lo, s)
    assert abs(O.proxy_loss(Wt_hat, P.Wt, P.Ht) - P.loss) / P.loss <= 1e-3
    W_hat_ref = O.incoherence_inverse(Wt_hat, P.U, P.V)
    assert np.abs(host(r.W_hat) - W_hat_ref).max() <= 1e-4 * s.max()
    bad, not_near = ldlq_trajectory_check(C, P.Wt, P.Uf, lo, s, bits, tau=1e-3)
    assert not_near == 0.0


def test_timing_trace_lists_the_layer_launches():
    """quip_timing_trace: one record per launch of the layer call, in enqueue
    order, each with end >= start >= 0 on the stream it ran on; the Hessian
    path (SYRK, LDL) and the weight path run on different streams.  The same
    launches, aggregated, are what quip_timing_end reports."""
    m, n, N, bits, block, seed = 256, 256, 512, 2, 128, 3
    mk, nk = Side("kronecker", 2, 128), Side("hadamard")
    d = random_layer(m, n, N, seed=2, dtype="bf16")
    W, X = dev(d["W"], torch.bfloat16), dev(d["X"], torch.bfloat16)
    q = Q.LayerQuantizer(m, n, mk, nk, bits, block, 0.01, seed)
    q.run(W, X)
    torch.cuda.synchronize()
    Q.quip_timing_begin()
    q.run(W, X)
    torch.cuda.synchronize()
    tr = Q.quip_timing_trace()
    assert len(tr) > 10
    assert all(b >= a >= 0.0 for _, a, b, _ in tr)
    names = [k for k, _, _, _ in tr]
    assert "k_syrk_tc" in names and "k_ldlq_block" in names and "k_ldl_factor" in names
    sid = {k: s for k, _, _, s in tr}
    assert sid["k_syrk_tc"] != sid["k_ldlq_block"]
    Q.quip_timing_begin()
    q.run(W, X)
    torch.cuda.synchronize()
    agg = Q.quip_timing_end()
    assert sum(c for c, _ in agg.values()) == len(tr)
    assert agg["k_syrk_tc"][0] == names.count("k_syrk_tc")
