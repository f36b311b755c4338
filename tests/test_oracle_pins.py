"""Pins for the FP64 oracle: each test ties an oracle function to something
other than itself — a value fixed by the pages or by a published definition,
a closed form, an invariant, a library routine, or brute force on tiny
inputs.  All CPU-only."""
import itertools
import math

import numpy as np
import pytest
import scipy.linalg as sla

import oracle as O
from quip_synth import CONFIGS, make_layer, random_layer, Side
from conftest import golden_rows


def _spd(n, seed, N=None, outliers=True):
    rng = np.random.default_rng(seed)
    N = N or 3 * n
    X = rng.standard_normal((N, n)) * np.exp(rng.standard_normal(n))
    if outliers and n > 4:
        X[:, rng.choice(n, 2, replace=False)] *= 20
    return O.damp(O.hessian(X), 0.01)


# ---------------------------------------------------------------- Hessian


def test_hessian_equals_sum_of_outer_products():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((7, 5))
    brute = sum(np.outer(x, x) for x in X) / 7.0
    np.testing.assert_allclose(O.hessian(X), brute, rtol=0, atol=1e-14)


def test_hessian_hand_example():
    # two tokens x = (1, 2), (3, -1): second moment = [[5, -0.5], [-0.5, 2.5]]
    X = np.array([[1.0, 2.0], [3.0, -1.0]])
    np.testing.assert_array_equal(O.hessian(X), [[5.0, -0.5], [-0.5, 2.5]])


def test_damp_adds_alpha_mean_diag():
    H = np.array([[2.0, 1.0], [1.0, 4.0]])
    Hd = O.damp(H, 0.5)          # mean diag = 3 -> +1.5 on the diagonal
    np.testing.assert_array_equal(Hd, [[3.5, 1.0], [1.0, 5.5]])


def test_damping_commutes_with_orthogonal_transform():
    H = O.hessian(np.random.default_rng(1).standard_normal((50, 16)))
    V = O.make_side(3, "n", "hadamard", 16).matrix()
    np.testing.assert_allclose(V @ O.damp(H, 0.01) @ V.T, O.damp(V @ H @ V.T, 0.01), atol=1e-13)


# ---------------------------------------------------------------- RNG


def test_splitmix64_published_outputs():
    want = [int(x, 16) for x in golden_rows("splitmix64_seed0.txt")]
    got = [int(v) for v in O.splitmix64(0, 0, np.arange(3))]
    assert got == want


def test_splitmix64_streams_and_seed_shift():
    # stream t element i is output k = t*2^40 + i + 1 of the same sequence:
    # seed' = seed + gamma * t * 2^40 maps stream t to stream 0.
    gamma = 0x9E3779B97F4A7C15
    a = O.splitmix64(7, 3, np.arange(5))
    b = O.splitmix64((7 + gamma * 3 * (1 << 40)) % (1 << 64), 0, np.arange(5))
    np.testing.assert_array_equal(a, b)


def test_signs_and_gaussians_statistics():
    s = O.random_signs(0, 1, 1 << 16)
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert abs(s.mean()) < 0.02
    g = O.gaussian_matrix(0, 2, 256).ravel()
    assert abs(g.mean()) < 0.01 and abs(g.std() - 1) < 0.01
    # Box-Muller on the published draw: element 0 from outputs k=1 and k=2
    r = [int(x, 16) for x in golden_rows("splitmix64_seed0.txt")]
    u1 = ((r[0] >> 11) + 1) * 2.0 ** -53
    u2 = ((r[1] >> 11) + 1) * 2.0 ** -53
    assert O.gaussian_matrix(0, 0, 1)[0, 0] == pytest.approx(math.sqrt(-2 * math.log(u1)) * math.cos(2 * math.pi * u2), rel=1e-15)


# ---------------------------------------------------------------- transforms


def test_hadamard_textbook_and_library():
    rows = [list(map(float, r.split())) for r in golden_rows("hadamard_2_4.txt")]
    np.testing.assert_array_equal(O.sylvester_hadamard(2), rows[:2])
    np.testing.assert_array_equal(O.sylvester_hadamard(4), rows[2:])
    for n in (1, 8, 64, 256):
        Hn = O.sylvester_hadamard(n)
        np.testing.assert_array_equal(Hn, sla.hadamard(n))
        np.testing.assert_array_equal(Hn @ Hn.T, n * np.eye(n))
    Hn = sla.hadamard(128)
    for i in (0, 1, 77, 127):
        np.testing.assert_array_equal(O.hadamard_row(128, i), Hn[i])


def test_haar_qr_reproduces_g_and_is_orthogonal():
    G = O.gaussian_matrix(5, 4, 20)
    Q = O.haar_orthogonal(G)
    np.testing.assert_allclose(Q @ Q.T, np.eye(20), atol=1e-13)
    R = Q.T @ G
    np.testing.assert_allclose(np.tril(R, -1), 0, atol=1e-12)
    assert np.all(np.diag(R) > 0)
    # uniqueness: scipy's QR with the same sign convention gives the same Q
    Q2, R2 = sla.qr(G)
    Q2 = Q2 * np.sign(np.diag(R2))[None, :]
    np.testing.assert_allclose(Q, Q2, atol=1e-12)


@pytest.mark.parametrize("kind,dim,p,q", [("hadamard", 64, 0, 0), ("kronecker", 12, 3, 4),
                                          ("kronecker", 86 * 2, 86, 2)])
def test_side_orthogonal_and_rows(kind, dim, p, q):
    S = O.make_side(11, "m", kind, dim, p, q)
    M = S.matrix()
    np.testing.assert_allclose(M @ M.T, np.eye(dim), atol=1e-12)
    for i in (0, dim // 3, dim - 1):
        np.testing.assert_allclose(S.row(i), M[i], atol=1e-15)
    if kind == "kronecker":
        A, B = S.A, S.B
        a, b, a2, b2 = 1, 1 % q, 2, (q - 1)
        assert M[a * q + b, a2 * q + b2] == pytest.approx(A[a, a2] * B[b, b2], abs=1e-15)


def test_incoherence_preserves_proxy_and_inverts():
    # QuIP incoherence section: tr(W~ H~ W~^T) = tr(W H W^T); and for any
    # W^: tr((W~^ - W~) H~ (.)^T) = tr((U^T W~^ V - W) H (.)^T).
    rng = np.random.default_rng(2)
    W = rng.standard_normal((16, 32))
    H = _spd(32, 3)
    U = O.make_side(0, "m", "hadamard", 16)
    V = O.make_side(0, "n", "kronecker", 32, 4, 8)
    Wt, Ht = O.incoherence_forward(W, H, U, V)
    assert np.trace(Wt @ Ht @ Wt.T) == pytest.approx(np.trace(W @ H @ W.T), rel=1e-12)
    np.testing.assert_allclose(O.incoherence_inverse(Wt, U, V), W, atol=1e-13)
    Wh_t = Wt + 0.1 * rng.standard_normal(Wt.shape)
    assert O.proxy_loss(Wh_t, Wt, Ht) == pytest.approx(
        O.proxy_loss(O.incoherence_inverse(Wh_t, U, V), W, H), rel=1e-11)
    # incoherence spreads an outlier: max |W~| well below the spike
    Wsp = np.zeros((16, 32))
    Wsp[3, 5] = 1.0
    Wt2, _ = O.incoherence_forward(Wsp, H, U, V)
    assert np.abs(Wt2).max() < 0.5


def test_incoherence_rows_and_hessian_match_full_forward():
    rng = np.random.default_rng(12)
    W = rng.standard_normal((24, 16))
    H = _spd(16, 5)
    U = O.make_side(4, "m", "kronecker", 24, 6, 4)
    V = O.make_side(4, "n", "hadamard", 16)
    Wt, Ht = O.incoherence_forward(W, H, U, V)
    rows = [0, 7, 23]
    np.testing.assert_allclose(O.incoherence_rows(W, U, V, rows), Wt[rows], atol=1e-14)
    np.testing.assert_allclose(O.incoherence_hessian(H, V), Ht, atol=1e-13)
    np.testing.assert_allclose(O.incoherence_hessian_rows(H, V, [0, 9, 15]), Ht[[0, 9, 15]], atol=1e-13)
    # the inverse restricted to rows: rows of U^T W~ V, and the round trip
    Wi = O.incoherence_inverse(Wt, U, V)
    np.testing.assert_allclose(O.incoherence_inverse_rows(Wt, U, V, rows), Wi[rows], atol=1e-14)
    np.testing.assert_allclose(O.incoherence_inverse_rows(Wt, U, V, rows), W[rows], atol=1e-13)


@pytest.mark.parametrize("kind,dim,p,q,perm", [("hadamard", 32, 0, 0, False), ("kronecker", 12, 3, 4, False),
                                               ("hadamard", 16, 0, 0, True), ("kronecker", 12, 4, 3, True),
                                               ("identity", 8, 0, 0, True)])
def test_side_columns_are_the_matrix_columns(kind, dim, p, q, perm):
    S = O.make_side(5, "n", kind, dim, p, q, permute=perm)
    M = S.matrix()
    for i in range(dim):
        np.testing.assert_allclose(S.col(i), M[:, i], atol=1e-15)


def test_hadamard_sign_placement_hand_example():
    # V = H_4 diag(s) / 2 with s = (1, -1, 1, 1): V e_1 = s_1 * H_4[:, 1] / 2
    S = O.SideTransform("hadamard", 4, signs=np.array([1.0, -1.0, 1.0, 1.0]))
    np.testing.assert_array_equal(S.matrix() @ np.array([0.0, 1.0, 0.0, 0.0]), [-0.5, 0.5, -0.5, 0.5])
    # and W~ = W V^T transforms each row by V
    Wt, _ = O.incoherence_forward(np.array([[0.0, 1.0, 0.0, 0.0]]), np.eye(4),
                                  O.SideTransform("identity", 1), S)
    np.testing.assert_array_equal(Wt[0], [-0.5, 0.5, -0.5, 0.5])


def test_signs_from_published_draws():
    # top bits of the published seed-0 outputs e220..., 6e78..., 06c4... are 1, 0, 0
    np.testing.assert_array_equal(O.random_signs(0, 0, 3), [-1.0, 1.0, 1.0])


def test_identity_sides_are_identity():
    W = np.arange(12.0).reshape(3, 4)
    H = _spd(4, 0)
    I3, I4 = O.make_side(0, "m", "identity", 3), O.make_side(0, "n", "identity", 4)
    Wt, Ht = O.incoherence_forward(W, H, I3, I4)
    np.testing.assert_array_equal(Wt, W)
    np.testing.assert_allclose(Ht, H)


# ---------------------------------------------------------------- LDL


def test_udu_hand_2x2():
    rows = golden_rows("udu_2x2.txt")
    H = np.array([list(map(float, rows[0].split())), list(map(float, rows[1].split()))])
    u = float(rows[2])
    d = list(map(float, rows[3].split()))
    U, D = O.udu(H)
    assert U[0, 1] == pytest.approx(u, abs=1e-15) and U[1, 0] == 0 and U[0, 0] == 0
    np.testing.assert_allclose(D, d, atol=1e-14)


@pytest.mark.parametrize("n", [1, 2, 7, 64, 200])
def test_udu_reconstructs(n):
    H = _spd(n, n)
    U, D = O.udu(H)
    assert np.all(np.tril(U) == 0)
    assert np.all(D > 0)
    R = (np.eye(n) + U) @ np.diag(D) @ (np.eye(n) + U).T
    assert np.linalg.norm(R - H) / np.linalg.norm(H) < 1e-12


def test_udu_diagonal_and_not_pd():
    d = np.array([3.0, 1.0, 2.0, 5.0])
    U, D = O.udu(np.diag(d))
    np.testing.assert_array_equal(U, 0)
    np.testing.assert_allclose(D, d)
    with pytest.raises(np.linalg.LinAlgError):
        O.udu(np.array([[1.0, 2.0], [2.0, 1.0]]))


def test_udu_last_pivot_is_schur_complement_free():
    # D_{n-1} = H_{n-1,n-1} (nothing to its right); D_0 = 1 / (H^-1)_00
    H = _spd(9, 4)
    U, D = O.udu(H)
    assert D[-1] == pytest.approx(H[-1, -1], rel=1e-14)
    assert D[0] == pytest.approx(1.0 / np.linalg.inv(H)[0, 0], rel=1e-10)


# ---------------------------------------------------------------- grid / Q


def test_grid_and_quantize_basics():
    Wt = np.array([[0.0, 0.3, 0.9, 0.6], [1.0, 1.0, 1.0, 1.0], [-2.0, 2.0, 0.0, 0.7]])
    lo, s = O.row_grid(Wt, 2)
    np.testing.assert_allclose(lo, [0.0, 1.0, -2.0])
    np.testing.assert_allclose(s, [0.3, 1.0, 4.0 / 3.0])
    c = O.nearest(Wt, lo, s, 2)
    np.testing.assert_array_equal(c[0], [0, 1, 3, 2])
    np.testing.assert_array_equal(c[1], [0, 0, 0, 0])
    # min and max land exactly on the end levels
    assert c[2, 0] == 0 and c[2, 1] == 3
    # ties go to even; values beyond the grid clamp
    q = O.quantize(np.array([0.5, 1.5, 2.5, -3.0, 9.0]), np.zeros(5), np.ones(5), 2)
    np.testing.assert_array_equal(q, [0, 2, 2, 0, 3])


# ---------------------------------------------------------------- LDLQ


def test_ldlq_worked_examples():
    for row in golden_rows("ldlq_n2_example.txt"):
        w, c = row.split("|")
        W = np.array([list(map(float, w.split()))])
        lo, s = O.row_grid(W, 2)
        U = np.array([[0.0, 0.5], [0.0, 0.0]])
        codes, _, _ = O.ldlq(W, U, lo, s, 2)
        np.testing.assert_array_equal(codes[0], list(map(int, c.split())))
    r = golden_rows("ldlq_n3_example.txt")
    W = np.array([list(map(float, r[0].split()))])
    U = np.array([list(map(float, r[1].split())), list(map(float, r[2].split())), [0, 0, 0]])
    D = np.array(list(map(float, r[3].split())))
    lo, s = O.row_grid(W, 2)
    codes, What, eta = O.ldlq(W, U, lo, s, 2)
    np.testing.assert_array_equal(codes[0], list(map(int, r[4].split())))
    H = (np.eye(3) + U) @ np.diag(D) @ (np.eye(3) + U).T
    assert O.proxy_loss(What, W, H) == pytest.approx(float(r[5]), rel=1e-12)


def test_ldlq_with_diagonal_h_is_nearest():
    rng = np.random.default_rng(4)
    W = rng.standard_normal((20, 30))
    for H in (np.eye(30), np.diag(rng.uniform(0.5, 3, 30))):
        U, D = O.udu(H)
        lo, s = O.row_grid(W, 3)
        codes, _, _ = O.ldlq(W, U, lo, s, 3)
        np.testing.assert_array_equal(codes, O.nearest(W, lo, s, 3))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_ldlq_loss_equals_eta_D_eta(bits):
    rng = np.random.default_rng(bits)
    n = 48
    H = _spd(n, 10 + bits)
    W = rng.standard_normal((12, n)) * 0.02
    U, D = O.udu(H)
    lo, s = O.row_grid(W, bits)
    codes, What, eta = O.ldlq(W, U, lo, s, bits)
    assert O.proxy_loss(What, W, H) == pytest.approx(float(np.einsum("ij,j,ij->", eta, D, eta)), rel=1e-10)
    assert np.all((codes >= 0) & (codes <= 2 ** bits - 1))


@pytest.mark.parametrize("bits", [2, 3])
def test_ldlq_equals_optq_order(bits):
    rng = np.random.default_rng(20 + bits)
    n = 40
    H = _spd(n, 30 + bits)
    W = rng.standard_normal((25, n)) * 0.02
    U, _ = O.udu(H)
    lo, s = O.row_grid(W, bits)
    np.testing.assert_array_equal(O.ldlq(W, U, lo, s, bits)[0], O.optq(W, H, lo, s, bits))


@pytest.mark.parametrize("block", [1, 3, 8, 32, 64])
def test_ldlq_block_invariance(block):
    rng = np.random.default_rng(7)
    n = 64
    H = _spd(n, 8)
    W = rng.standard_normal((16, n)) * 0.02
    U, _ = O.udu(H)
    lo, s = O.row_grid(W, 2)
    c0, W0, _ = O.ldlq(W, U, lo, s, 2)
    c1, W1 = O.ldlq_blocked(W, U, lo, s, 2, block)
    np.testing.assert_array_equal(c0, c1)
    np.testing.assert_allclose(W0, W1, atol=1e-15)


def test_ldlq_rows_independent():
    # QuIP adaptive-rounding section: the per-layer objective decouples over
    # rows ("run in parallel across neurons").
    rng = np.random.default_rng(9)
    H = _spd(24, 9)
    W = rng.standard_normal((10, 24))
    U, _ = O.udu(H)
    perm = rng.permutation(10)
    lo, s = O.row_grid(W, 2)
    c = O.ldlq(W, U, lo, s, 2)[0]
    lo2, s2 = O.row_grid(W[perm], 2)
    np.testing.assert_array_equal(O.ldlq(W[perm], U, lo2, s2, 2)[0], c[perm])


@pytest.mark.parametrize("n,bits", [(3, 2), (4, 2), (5, 2), (6, 2), (3, 3), (4, 3)])
def test_ldlq_never_beats_brute_force(n, bits):
    rng = np.random.default_rng(100 * n + bits)
    H = _spd(n, n + bits, N=4 * n, outliers=False)
    U, _ = O.udu(H)
    W = rng.standard_normal((6, n))
    lo, s = O.row_grid(W, bits)
    codes, What, _ = O.ldlq(W, U, lo, s, bits)
    grid = np.array(list(itertools.product(range(2 ** bits), repeat=n)), dtype=np.float64)
    for i in range(W.shape[0]):
        cand = lo[i] + s[i] * grid - W[i]               # all (2^b)^n candidates
        best = np.min(np.einsum("kj,jl,kl->k", cand, H, cand))
        e = What[i] - W[i]
        l_ldlq = float(e @ H @ e)
        # exhaustive search finds the exact optimum; LDLQ may tie it, never beat it
        assert l_ldlq >= best - 1e-12


# ---------------------------------------------------------------- pipeline


def test_pipeline_tiny_config_invariants():
    cfg = CONFIGS["tiny"]
    d = make_layer(cfg)
    P = O.run_pipeline(d["W"], d["X"], cfg.seed, cfg.m_side, cfg.n_side, cfg.bits, cfg.damp)
    Pb = O.run_pipeline(d["W"], d["X"], cfg.seed, cfg.m_side, cfg.n_side, cfg.bits, cfg.damp, block=cfg.block)
    np.testing.assert_array_equal(P.codes, Pb.codes)
    # the loss in the incoherent domain is the loss in the original domain
    assert P.loss == pytest.approx(O.proxy_loss(P.W_hat, d["W"], P.H), rel=1e-10)
    # LDLQ beats nearest rounding on the proxy (QuIP Experiments)
    near = O.dequantize(O.nearest(P.Wt, P.lo, P.s, cfg.bits), P.lo, P.s)
    assert P.loss < O.proxy_loss(near, P.Wt, P.Ht)


def test_synth_recipe():
    cfg = CONFIGS["tiny"]
    d = make_layer(cfg)
    assert d["W"].shape == (64, 128) and d["X"].shape == (1024, 128)
    assert abs(d["W"].std() - 0.02) < 0.002
    d2 = random_layer(5, 7, 11, seed=3, dtype="bf16")
    # bf16 storage: low 16 bits of every float32 are zero
    assert np.all((d2["W"].view(np.uint32) & 0xFFFF) == 0)


# ---------------------------------------------------------------- random permutation (QuIP, Table 5)


def test_random_permutation_sorts_its_draws_brute_force():
    # tiny case by hand: pi must list the indices of the draws in increasing order
    for seed, n in ((0, 5), (9, 8)):
        keys = [int(k) for k in O.splitmix64(seed, O.STREAM_N_PERM, np.arange(n, dtype=np.uint64))]
        pi = O.random_permutation(seed, O.STREAM_N_PERM, n)
        assert sorted(pi.tolist()) == list(range(n))
        assert all(keys[pi[r]] < keys[pi[r + 1]] for r in range(n - 1))
        # brute force: the order of the draws, found by repeatedly taking the smallest
        rest, order = list(range(n)), []
        while rest:
            i = min(rest, key=lambda j: keys[j])
            order.append(i)
            rest.remove(i)
        assert pi.tolist() == order


def test_permutation_only_side_is_indexing():
    # identity structure with a permutation: W~ = P_m W P_n^T, i.e. W~[r, c] = W[pi_m[r], pi_n[c]],
    # and H~[a, b] = H[pi_n[a], pi_n[b]]; the inverse indexes back
    rng = np.random.default_rng(21)
    W = rng.standard_normal((6, 8))
    H = _spd(8, 4)
    U = O.make_side(5, "m", "identity", 6, permute=True)
    V = O.make_side(5, "n", "identity", 8, permute=True)
    pm, pn = U.perm, V.perm
    assert pm.tolist() != list(range(6)) and pn.tolist() != list(range(8))
    Wt, Ht = O.incoherence_forward(W, H, U, V)
    np.testing.assert_array_equal(Wt, W[pm][:, pn])
    np.testing.assert_allclose(Ht, H[pn][:, pn], atol=0)
    np.testing.assert_allclose(O.incoherence_inverse(Wt, U, V), W, atol=0)


@pytest.mark.parametrize("kind,dim,p,q", [("hadamard", 32, 0, 0), ("kronecker", 12, 3, 4)])
def test_permuted_side_orthogonal_rows_and_proxy(kind, dim, p, q):
    S = O.make_side(3, "n", kind, dim, p, q, permute=True)
    T = O.make_side(3, "n", kind, dim, p, q)
    M = S.matrix()
    np.testing.assert_allclose(M @ M.T, np.eye(dim), atol=1e-12)
    # S = T P: column pi[r] of S is column r of T
    np.testing.assert_allclose(M[:, S.perm], T.matrix(), atol=1e-15)
    for i in (0, dim - 1):
        np.testing.assert_allclose(S.row(i), M[i], atol=1e-15)
    rng = np.random.default_rng(8)
    W = rng.standard_normal((5, dim))
    H = _spd(dim, 9)
    Wt, Ht = O.incoherence_forward(W, H, O.make_side(0, "m", "identity", 5), S)
    assert np.trace(Wt @ Ht @ Wt.T) == pytest.approx(np.trace(W @ H @ W.T), rel=1e-12)


# ---------------------------------------------------------------- LDLQ-RG, Greedy


def _proxy_codes(W, H, lo, s, c):
    return O.proxy_loss(O.dequantize(c, lo, s), W, H)


def test_rounding_methods_worked_example():
    r = golden_rows("greedy_rg_n4_example.txt")
    W = np.array([list(map(float, r[0].split()))])
    H = np.array([list(map(float, r[i].split())) for i in range(1, 5)])
    lo, s = O.row_grid(W, 2)
    np.testing.assert_array_equal(O.diag_order(H), list(map(int, r[5].split())))
    losses = list(map(float, r[10].split()))
    for method, row, loss in zip(("nearest", "ldlq", "greedy", "ldlq_rg"), r[6:10], losses):
        c = O.quantize_layer(method, W, H, lo, s, 2, passes=1)
        np.testing.assert_array_equal(c[0], list(map(int, row.split())), err_msg=method)
        assert _proxy_codes(W, H, lo, s, c) == pytest.approx(loss, rel=1e-12), method


def test_diag_order_brute_force():
    # exactly one ordering lists the diagonal non-increasing with equal entries
    # by increasing index; find it among all n! orderings
    rng = np.random.default_rng(31)
    for n in (1, 2, 4, 5):
        for _ in range(10):
            d = rng.integers(0, 3, n).astype(float)
            ok = [p for p in itertools.permutations(range(n))
                  if all(d[p[r]] > d[p[r + 1]] or (d[p[r]] == d[p[r + 1]] and p[r] < p[r + 1])
                         for r in range(n - 1))]
            assert len(ok) == 1
            np.testing.assert_array_equal(O.diag_order(np.diag(d) + 0.01), ok[0])


def test_greedy_update_is_the_coordinate_minimiser():
    # one greedy update of column k: per row, no other code of that column (the
    # rest held) gives a lower proxy, found by trying all 2^b codes
    rng = np.random.default_rng(41)
    n, bits = 7, 2
    H = _spd(n, 41, outliers=False)
    W = rng.standard_normal((5, n))
    lo, s = O.row_grid(W, bits)
    c0 = rng.integers(0, 2 ** bits, W.shape)
    for k in range(n):
        c1 = O.greedy_pass(W, H, lo, s, bits, c0, order=[k])
        np.testing.assert_array_equal(np.delete(c1, k, 1), np.delete(c0, k, 1))
        for i in range(W.shape[0]):
            vals = []
            for v in range(2 ** bits):
                c = c0[i].astype(np.float64)
                c[k] = v
                e = lo[i] + s[i] * c - W[i]
                vals.append(float(e @ H @ e))
            assert vals[c1[i, k]] <= min(vals) + 1e-12


def test_greedy_with_diagonal_h_is_nearest():
    # with H diagonal the columns decouple: from any codes, one pass rounds
    # every column to nearest
    rng = np.random.default_rng(42)
    W = rng.standard_normal((9, 16))
    lo, s = O.row_grid(W, 3)
    c0 = rng.integers(0, 8, W.shape)
    for H in (np.eye(16), np.diag(rng.uniform(0.5, 3, 16))):
        np.testing.assert_array_equal(O.greedy_pass(W, H, lo, s, 3, c0), O.nearest(W, lo, s, 3))


@pytest.mark.parametrize("bits", [2, 3])
def test_greedy_passes_descend_to_a_coordinate_minimum(bits):
    rng = np.random.default_rng(43 + bits)
    n = 20
    H = _spd(n, 43 + bits)
    W = rng.standard_normal((6, n))
    lo, s = O.row_grid(W, bits)
    c = rng.integers(0, 2 ** bits, W.shape)
    loss = _proxy_codes(W, H, lo, s, c)
    for _ in range(100):
        c2 = O.greedy_pass(W, H, lo, s, bits, c)
        loss2 = _proxy_codes(W, H, lo, s, c2)
        assert loss2 <= loss + 1e-12                   # coordinate descent never climbs
        if np.array_equal(c2, c):
            break
        c, loss = c2, loss2
    else:
        pytest.fail("greedy passes did not settle")
    # at the fixed point no single code change lowers a row's proxy
    for i in range(W.shape[0]):
        e0 = lo[i] + s[i] * c[i] - W[i]
        l0 = float(e0 @ H @ e0)
        for k in range(n):
            for v in range(2 ** bits):
                e = e0.copy()
                e[k] = lo[i] + s[i] * v - W[i, k]
                assert float(e @ H @ e) >= l0 - 1e-12


def test_ldlq_rg_first_columns_and_equivariance():
    rng = np.random.default_rng(44)
    n, bits = 12, 2
    H = _spd(n, 44, outliers=False)
    W = rng.standard_normal((8, n))
    lo, s = O.row_grid(W, bits)
    order = O.diag_order(H)
    c = O.quantize_layer("ldlq_rg", W, H, lo, s, bits, passes=0)
    # the column quantised first (largest H_kk) has no feedback: nearest rounding
    np.testing.assert_array_equal(c[:, order[0]], O.nearest(W[:, order[:1]], lo, s, bits)[:, 0])
    # re-labelling the columns re-labels the codes (the order follows diag(H))
    sig = rng.permutation(n)
    c_sig = O.quantize_layer("ldlq_rg", W[:, sig], H[np.ix_(sig, sig)], lo, s, bits, passes=1)
    np.testing.assert_array_equal(c_sig, O.quantize_layer("ldlq_rg", W, H, lo, s, bits, passes=1)[:, sig])
    # with the diagonal already non-increasing, LDLQ-RG is LDLQ then greedy
    Hs, Ws = H[np.ix_(order, order)], W[:, order]
    want = O.greedy_pass(Ws, Hs, lo, s, bits, O.quantize_layer("ldlq", Ws, Hs, lo, s, bits))
    np.testing.assert_array_equal(O.quantize_layer("ldlq_rg", Ws, Hs, lo, s, bits, passes=1), want)


@pytest.mark.parametrize("n,bits", [(3, 2), (4, 2), (5, 2), (3, 3)])
def test_rg_and_greedy_never_beat_brute_force(n, bits):
    rng = np.random.default_rng(200 * n + bits)
    H = _spd(n, 7 * n + bits, N=4 * n, outliers=False)
    W = rng.standard_normal((5, n))
    lo, s = O.row_grid(W, bits)
    grid = np.array(list(itertools.product(range(2 ** bits), repeat=n)), dtype=np.float64)
    for method in ("greedy", "ldlq_rg"):
        c = O.quantize_layer(method, W, H, lo, s, bits, passes=2)
        for i in range(W.shape[0]):
            cand = lo[i] + s[i] * grid - W[i]
            best = np.min(np.einsum("kj,jl,kl->k", cand, H, cand))
            e = lo[i] + s[i] * c[i] - W[i]
            assert float(e @ H @ e) >= best - 1e-12


# ---------------------------------------------------------------- quantized inference


def test_pack_codes_worked_example_and_roundtrip():
    r = golden_rows("qmatvec_example.txt")
    for line, bits in ((r[0], 2), (r[1], 3)):
        c, w = line.split("|")
        codes = np.array([list(map(int, c.split()))])
        np.testing.assert_array_equal(O.pack_codes(codes, bits)[0], list(map(int, w.split())))
    rng = np.random.default_rng(50)
    for bits in range(1, 9):
        for n in (1, 5, 64, 129, 300):
            c = rng.integers(0, 2 ** bits, (3, n))
            p = O.pack_codes(c, bits)
            assert p.shape == (3, O.packed_words(n, bits)) and p.shape[1] % 4 == 0
            assert p.shape[1] * (32 // O.code_slot_bits(bits)) >= n
            np.testing.assert_array_equal(O.unpack_codes(p, n, bits), c)
            # the packed words hold exactly the codes' bits: popcounts agree
            assert sum(bin(int(v)).count("1") for v in p.ravel()) == \
                sum(bin(int(v)).count("1") for v in c.ravel())


def test_quantized_matvec_worked_example():
    r = golden_rows("qmatvec_example.txt")
    codes = np.array(list(map(int, r[2].split()))).reshape(2, 2)
    lo = np.array(list(map(float, r[3].split())))
    s = np.array(list(map(float, r[4].split())))
    x = np.array([list(map(float, r[5].split()))])
    I = O.SideTransform("identity", 2)
    np.testing.assert_allclose(O.quantized_matvec(codes, lo, s, I, I, x)[0],
                               list(map(float, r[6].split())), atol=1e-15)
    U = O.SideTransform("hadamard", 2, signs=np.array([1.0, 1.0]))
    V = O.SideTransform("hadamard", 2, signs=np.array([1.0, -1.0]))
    np.testing.assert_allclose(O.quantized_matvec(codes, lo, s, U, V, x)[0],
                               list(map(float, r[7].split())), atol=1e-14)


def test_quantized_matvec_is_the_layer_applied_to_the_vector():
    # the product of the quantized layer with x equals quantising, then
    # running the original-domain layer: y = W^ x, with W^ from the pipeline;
    # and it is linear in x
    cfg = CONFIGS["tiny"]
    d = make_layer(cfg)
    P = O.run_pipeline(d["W"], d["X"], cfg.seed, cfg.m_side, cfg.n_side, cfg.bits, cfg.damp)
    rng = np.random.default_rng(51)
    x = rng.standard_normal((3, cfg.n))
    y = O.quantized_matvec(P.codes, P.lo, P.s, P.U, P.V, x)
    np.testing.assert_allclose(y, x @ P.W_hat.T, rtol=1e-12, atol=1e-12)
    y2 = O.quantized_matvec(P.codes, P.lo, P.s, P.U, P.V, 2 * x[:1] - x[1:2])
    np.testing.assert_allclose(y2[0], 2 * y[0] - y[1], atol=1e-12)
    # in the incoherent domain: U y = W~^ (V x)
    np.testing.assert_allclose(y @ P.U.matrix().T,
                               (x @ P.V.matrix().T) @ O.dequantize(P.codes, P.lo, P.s).T, atol=1e-12)
