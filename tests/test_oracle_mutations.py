"""Plant plausible mistakes in the oracle (CPU only) and check that at least
one pin in test_oracle_pins.py fails for each: a dropped term, a wrong sign,
a transposed operand, a wrong index or normalisation."""
import numpy as np
import pytest

import oracle as O
import oracle.quip_oracle as Q
import test_oracle_pins as P


def _fails(pins):
    for pin in pins:
        try:
            pin()
        except (AssertionError, ValueError, IndexError, np.linalg.LinAlgError):
            return True
    return False


def _ldlq_wrong_sign(Wt, U, lo, s, bits):
    Wt = np.asarray(Wt, dtype=np.float64)
    m, n = Wt.shape
    codes = np.zeros((m, n), dtype=np.int64)
    What = np.zeros((m, n))
    eta = np.zeros((m, n))
    errT = np.zeros((n, m))
    for k in range(n):
        a = Wt[:, k] - U[:k, k] @ errT[:k]            # planted: feedback sign
        c = Q.quantize(a, lo, s, bits)
        codes[:, k], What[:, k] = c, lo + s * c
        eta[:, k] = What[:, k] - a
        errT[k] = Wt[:, k] - What[:, k]
    return codes, What, eta


def _ldlq_transposed(Wt, U, lo, s, bits):
    return Q.__dict__["_ldlq_orig"](Wt, np.asarray(U).T, lo, s, bits)


def _ldlq_drop_feedback(Wt, U, lo, s, bits):
    return Q.__dict__["_ldlq_orig"](Wt, np.zeros_like(U), lo, s, bits)


def _udu_lower(H):
    U, D = Q.__dict__["_udu_orig"](H)
    return U.T, D


def _udu_no_sqrt(H):
    U, D = Q.__dict__["_udu_orig"](H)
    return U, np.sqrt(D)


def _hessian_no_norm(X):
    X = np.asarray(X, dtype=np.float64)
    return X.T @ X


def _damp_trace(H, alpha):
    H = np.array(H, dtype=np.float64, copy=True)
    H[np.diag_indices_from(H)] += alpha * float(np.trace(H))     # planted: sum, not mean
    return H


def _grid_bits(Wt, bits):
    lo, s = Q.__dict__["_row_grid_orig"](Wt, bits)
    return lo, s * (2 ** bits - 1) / 2 ** bits                   # planted: 2^b not 2^b - 1


def _rint_floor(a, lo, s, bits):
    return np.clip(np.floor((a - lo) / s), 0, 2 ** bits - 1)


def _signs_on_output(self):
    if self.kind == "hadamard":
        return self.signs[:, None] * O.sylvester_hadamard(self.dim) / np.sqrt(self.dim)
    return Q.__dict__["_matrix_orig"](self)


def _forward_no_transpose(W, H, U, V):
    Um, Vn = U.matrix(), V.matrix()
    Wt = Um @ W @ Vn                                              # planted: V not V^T
    Ht = Vn @ H @ Vn.T
    return Wt, 0.5 * (Ht + Ht.T)


def _box_muller_sin(seed, stream, p):
    e = np.arange(p * p, dtype=np.uint64)
    u1 = Q.uniform53(Q.splitmix64(seed, stream, 2 * e))
    u2 = Q.uniform53(Q.splitmix64(seed, stream, 2 * e + np.uint64(1)))
    return (np.sqrt(-2.0 * np.log(u1)) * np.sin(2.0 * np.pi * u2)).reshape(p, p)


LDLQ_PINS = [P.test_ldlq_worked_examples, lambda: P.test_ldlq_loss_equals_eta_D_eta(2),
             lambda: P.test_ldlq_equals_optq_order(2)]

MUTANTS = [
    ("ldlq", _ldlq_wrong_sign, LDLQ_PINS),
    ("ldlq", _ldlq_transposed, LDLQ_PINS),
    ("ldlq", _ldlq_drop_feedback, LDLQ_PINS),
    ("udu", _udu_lower, [P.test_udu_hand_2x2, lambda: P.test_udu_reconstructs(7)]),
    ("udu", _udu_no_sqrt, [P.test_udu_hand_2x2, lambda: P.test_udu_reconstructs(7)]),
    ("hessian", _hessian_no_norm, [P.test_hessian_hand_example, P.test_hessian_equals_sum_of_outer_products]),
    ("damp", _damp_trace, [P.test_damp_adds_alpha_mean_diag]),
    ("row_grid", _grid_bits, [P.test_grid_and_quantize_basics]),
    ("quantize", _rint_floor, [P.test_grid_and_quantize_basics, P.test_ldlq_worked_examples]),
    ("incoherence_forward", _forward_no_transpose, [P.test_incoherence_preserves_proxy_and_inverts]),
    ("gaussian_matrix", _box_muller_sin, [P.test_signs_and_gaussians_statistics]),
]


@pytest.mark.parametrize("name,mutant,pins", MUTANTS, ids=[f"{m[0]}:{m[1].__name__}" for m in MUTANTS])
def test_planted_mistake_is_caught(monkeypatch, name, mutant, pins):
    monkeypatch.setitem(Q.__dict__, f"_{name}_orig", getattr(Q, name))
    monkeypatch.setattr(Q, name, mutant)
    monkeypatch.setattr(O, name, mutant)
    assert _fails(pins), f"no pin caught the planted mistake in {name}"


def test_planted_sign_placement_is_caught(monkeypatch):
    monkeypatch.setitem(Q.__dict__, "_matrix_orig", Q.SideTransform.matrix)
    monkeypatch.setattr(Q.SideTransform, "matrix", _signs_on_output)
    assert _fails([P.test_hadamard_sign_placement_hand_example])


def _perm_matrix_transposed(self):
    return Q.__dict__["_perm_matrix_orig"](self).T             # planted: P^T (pi^-1) for P


def _permutation_descending(seed, stream, n):
    keys = Q.splitmix64(seed, stream, np.arange(n, dtype=np.uint64))
    return np.argsort(keys, kind="stable")[::-1]                # planted: descending order


def test_planted_permutation_direction_is_caught(monkeypatch):
    monkeypatch.setitem(Q.__dict__, "_perm_matrix_orig", Q.SideTransform.perm_matrix)
    monkeypatch.setattr(Q.SideTransform, "perm_matrix", _perm_matrix_transposed)
    assert _fails([P.test_permutation_only_side_is_indexing])


def test_planted_permutation_order_is_caught(monkeypatch):
    monkeypatch.setattr(Q, "random_permutation", _permutation_descending)
    monkeypatch.setattr(O, "random_permutation", _permutation_descending)
    assert _fails([P.test_random_permutation_sorts_its_draws_brute_force])


def _greedy_sign(Wt, H, lo, s, bits, codes, order=None):
    c = np.array(codes, dtype=np.int64, copy=True)
    E = (lo[:, None] + s[:, None] * c) - Wt
    for k in (range(Wt.shape[1]) if order is None else order):
        t = Wt[:, k] + (E @ H[:, k] - E[:, k] * H[k, k]) / H[k, k]      # planted: sign
        c[:, k] = Q.quantize(t, lo, s, bits)
        E[:, k] = lo + s * c[:, k] - Wt[:, k]
    return c


def _greedy_self_term(Wt, H, lo, s, bits, codes, order=None):
    c = np.array(codes, dtype=np.int64, copy=True)
    E = (lo[:, None] + s[:, None] * c) - Wt
    for k in (range(Wt.shape[1]) if order is None else order):
        t = Wt[:, k] - (E @ H[:, k]) / H[k, k]                          # planted: j = k kept
        c[:, k] = Q.quantize(t, lo, s, bits)
        E[:, k] = lo + s * c[:, k] - Wt[:, k]
    return c


def _greedy_unscaled(Wt, H, lo, s, bits, codes, order=None):
    c = np.array(codes, dtype=np.int64, copy=True)
    E = (lo[:, None] + s[:, None] * c) - Wt
    for k in (range(Wt.shape[1]) if order is None else order):
        t = Wt[:, k] - (E @ H[:, k] - E[:, k] * H[k, k])                 # planted: no 1/H_kk
        c[:, k] = Q.quantize(t, lo, s, bits)
        E[:, k] = lo + s * c[:, k] - Wt[:, k]
    return c


def _diag_order_ascending(H):
    return np.argsort(np.diag(np.asarray(H, dtype=np.float64)), kind="stable")


GREEDY_PINS = [P.test_rounding_methods_worked_example, P.test_greedy_update_is_the_coordinate_minimiser,
               P.test_greedy_with_diagonal_h_is_nearest]


@pytest.mark.parametrize("mutant", [_greedy_sign, _greedy_self_term, _greedy_unscaled])
def test_planted_greedy_mistake_is_caught(monkeypatch, mutant):
    monkeypatch.setattr(Q, "greedy_pass", mutant)
    monkeypatch.setattr(O, "greedy_pass", mutant)
    assert _fails(GREEDY_PINS)


def test_planted_diag_order_direction_is_caught(monkeypatch):
    monkeypatch.setattr(Q, "diag_order", _diag_order_ascending)
    monkeypatch.setattr(O, "diag_order", _diag_order_ascending)
    assert _fails([P.test_rounding_methods_worked_example, P.test_diag_order_brute_force])


@pytest.mark.parametrize("twice", [False, True])
def test_planted_rg_unpermute_mistake_is_caught(monkeypatch, twice):
    # codes left in the quantisation order (c_p = c[:, pi]), or moved back the
    # wrong way (c_p[:, pi] instead of c_p[:, pi^-1])
    orig = Q.quantize_layer

    def wrong(method, Wt, Ht, lo, s, bits, passes=1):
        c = orig(method, Wt, Ht, lo, s, bits, passes)
        if method != "ldlq_rg":
            return c
        order = Q.diag_order(Ht)
        cp = c[:, order]
        return cp[:, order] if twice else cp

    monkeypatch.setattr(Q, "quantize_layer", wrong)
    monkeypatch.setattr(O, "quantize_layer", wrong)
    assert _fails([P.test_rounding_methods_worked_example, P.test_ldlq_rg_first_columns_and_equivariance])


def _pack_contiguous(codes, bits):
    # planted: consecutive codes in one word (word j div per, slot j mod per)
    codes = np.asarray(codes, dtype=np.int64)
    m, n = codes.shape
    slot = Q.code_slot_bits(bits)
    per = 32 // slot
    out = np.zeros((m, Q.packed_words(n, bits)), dtype=np.uint64)
    for j in range(n):
        out[:, j // per] |= codes[:, j].astype(np.uint64) << np.uint64((j % per) * slot)
    return out.astype(np.uint32)


def _matvec_untransposed(codes, lo, s, U, V, x):
    W_hat = U.matrix() @ Q.dequantize(codes, lo, s) @ V.matrix()     # planted: U for U^T
    return np.asarray(x, dtype=np.float64) @ W_hat.T


def test_planted_pack_layout_is_caught(monkeypatch):
    monkeypatch.setattr(Q, "pack_codes", _pack_contiguous)
    monkeypatch.setattr(O, "pack_codes", _pack_contiguous)
    assert _fails([P.test_pack_codes_worked_example_and_roundtrip])


def test_planted_matvec_transpose_is_caught(monkeypatch):
    monkeypatch.setattr(Q, "quantized_matvec", _matvec_untransposed)
    monkeypatch.setattr(O, "quantized_matvec", _matvec_untransposed)
    assert _fails([P.test_quantized_matvec_worked_example,
                   P.test_quantized_matvec_is_the_layer_applied_to_the_vector])
