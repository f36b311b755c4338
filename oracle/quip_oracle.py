"""Plain FP64 oracle of the QuIP pipeline for one linear layer.

TEST INFRASTRUCTURE: imported only by tests/, __graft_entry__.smoke() and the
CPU legs of bench.py.  Nothing here is on the product path.

Sources (page title, then the section / equation each step follows):

[QuIP]  "QuIP: 2-Bit Quantization of Large Language Models With Guarantees"
        (Chee, Cai, Kuleshov, De Sa; arXiv 2307.13304), HTML body.
          - Introduction: proxy objective l(W^) = tr((W^ - W) H (W^ - W)^T)
            and the Kronecker product of random orthogonal matrices.
          - Adaptive-rounding section (Eq. (1), display lost in the page):
            H is the second moment of the calibration inputs; rows of W are
            independent ("run in parallel across neurons").
          - "OPTQ (Formerly known as GPTQ)." paragraph: nearest rounding,
            scaled error update of the remaining columns, repeat.
          - Incoherence-processing section: H~ <- V H V^T, W~ <- U W V^T and
            the trace identity tr(W~ H~ W~^T) = tr(W H W^T).
          - Experiments, "Methods.": damping H <- H + alpha*mean(diag(H)) I;
            nearest rounding and LDLQ as rounding methods; LDLQ = OPTQ;
            LDLQ-RG (re-order by diag(H), then greedy updates of the proxy)
            and "Greedy" (the greedy updates alone).
[QuIP#] "QuIP#: Even Better LLM Quantization with Hadamard Incoherence and
        Lattice Codebooks" (arXiv 2402.04396), abstract: incoherence by the
        randomized Hadamard transform.

The LDLQ display and its LDL factorisation were lost from the QuIP page; the
reading used here (and by the CUDA path) is the one the rest of the text
supports: H = (I + U)(D)(I + U)^T with U strictly upper triangular, and
W^_k = Q(W_k + (W - W^) U_k), column k using only columns j < k.

Readings where the pages are silent (the CUDA path takes the same ones):
  * grid: per-row asymmetric min/max grid of 2^b levels over the whole
    incoherent row, fixed before rounding; s = (hi - lo) / (2^b - 1); a
    constant row uses s = 1;
  * Q: round half to even (numpy.rint), then clamp to [0, 2^b - 1];
  * Hadamard: Sylvester order, V = H_n diag(s) / sqrt(n), s_i = +-1;
  * Kronecker: V = A (x) B with A, B Haar-distributed (QR of a Gaussian
    matrix with the sign of diag(R) folded into Q);
  * the random signs and Gaussians come from SplitMix64, counter-based (see
    ``splitmix64``); the CUDA library implements the same published
    generator independently;
  * the random permutation within the fast orthogonal multiplication (QuIP,
    Experiments, "Further Ablation", Table 5; the algorithm box that placed
    it was lost): optional per side, applied to the coordinates before the
    structured factor, S = T P with (P x)_r = x_{pi[r]}; pi sorts the draws
    of the side's permutation stream (``random_permutation``);
  * LDLQ-RG and Greedy ("Methods." names them in one sentence each): the
    re-ordering quantises columns by decreasing diag(H~) (ties by index);
    a greedy update sets one column to its exact coordinate minimiser on
    the grid, others held; a pass visits every column once, in the
    quantisation order; Greedy starts from nearest rounding; the number of
    passes is a parameter (the pages give none);
  * quantized inference: the pages give no storage format for the codes;
    ``pack_codes`` defines the library's (a column-strided layout, so that
    consecutive words hold consecutive columns).

Pinned by tests/test_oracle_*.py (CPU).  Functions with no pin: none.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np

__all__ = [
    "hessian", "damp", "splitmix64", "uniform53", "random_signs", "gaussian_matrix",
    "haar_orthogonal", "sylvester_hadamard", "hadamard_row", "SideTransform", "make_side",
    "incoherence_forward", "incoherence_inverse", "incoherence_rows", "incoherence_hessian", "incoherence_hessian_rows",
    "incoherence_inverse_rows", "udu", "row_grid", "quantize",
    "ldlq", "ldlq_blocked", "nearest", "optq", "dequantize", "proxy_loss", "Pipeline",
    "run_pipeline", "STREAM_M_SIGNS", "STREAM_N_SIGNS", "STREAM_M_A", "STREAM_M_B",
    "STREAM_N_A", "STREAM_N_B", "STREAM_M_PERM", "STREAM_N_PERM", "random_permutation",
    "diag_order", "greedy_pass", "quantize_layer", "code_slot_bits", "packed_words", "pack_codes",
    "unpack_codes", "quantized_matvec",
]

# ----------------------------------------------------------------------------
# O1/O2  Proxy Hessian and damping
# ----------------------------------------------------------------------------


def hessian(X: np.ndarray) -> np.ndarray:
    """H = X^T X / N: second moment of the calibration inputs x in R^n.

    [QuIP] adaptive-rounding section: "H is the second moment matrix of these
    vectors, interpreted as a proxy Hessian".  X is N x n (one token per row).
    """
    X = np.asarray(X, dtype=np.float64)
    return X.T @ X / X.shape[0]


def damp(H: np.ndarray, alpha: float) -> np.ndarray:
    """H + alpha * mean(diag(H)) * I  ([QuIP] Experiments, "Methods.")."""
    H = np.array(H, dtype=np.float64, copy=True)
    mu = float(np.mean(np.diag(H)))
    H[np.diag_indices_from(H)] += alpha * mu
    return H


# ----------------------------------------------------------------------------
# O3  Random orthogonal transforms
# ----------------------------------------------------------------------------
#
# Counter-based SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
# number generators", OOPSLA 2014): the k-th output (k >= 1) from seed s is
# mix(s + k * gamma) with gamma = 0x9E3779B97F4A7C15 and mix the published
# 64-bit finaliser below.  Stream t, element i uses k = t * 2^40 + i + 1.

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_M_SIGNS, STREAM_N_SIGNS = 0, 1
STREAM_M_A, STREAM_M_B, STREAM_N_A, STREAM_N_B = 2, 3, 4, 5
STREAM_M_PERM, STREAM_N_PERM = 6, 7


def splitmix64(seed: int, stream: int, index: np.ndarray) -> np.ndarray:
    """uint64 outputs of SplitMix64 for the given stream and element indices."""
    idx = np.asarray(index, dtype=np.uint64)
    k = np.uint64(stream) * np.uint64(1 << 40) + idx + np.uint64(1)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + k * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform53(r: np.ndarray) -> np.ndarray:
    """Map uint64 to (0, 1]: ((r >> 11) + 1) * 2^-53."""
    return ((r >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def random_signs(seed: int, stream: int, n: int) -> np.ndarray:
    """s_i = -1 if the top bit of the i-th draw is set, else +1."""
    r = splitmix64(seed, stream, np.arange(n, dtype=np.uint64))
    return np.where((r >> np.uint64(63)) == np.uint64(1), -1.0, 1.0)


def gaussian_matrix(seed: int, stream: int, p: int) -> np.ndarray:
    """p x p i.i.d. N(0,1), row-major element e from draws 2e and 2e+1 by
    Box-Muller: sqrt(-2 ln u1) * cos(2 pi u2)."""
    e = np.arange(p * p, dtype=np.uint64)
    u1 = uniform53(splitmix64(seed, stream, 2 * e))
    u2 = uniform53(splitmix64(seed, stream, 2 * e + np.uint64(1)))
    g = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    return g.reshape(p, p)


def haar_orthogonal(G: np.ndarray) -> np.ndarray:
    """Q of G = QR with diag(R) > 0, i.e. Q <- Q diag(sign(diag R)).

    This is the standard way to draw a uniformly (Haar) distributed orthogonal
    matrix; [QuIP] Introduction asks for "random orthogonal matrices".
    """
    Q, R = np.linalg.qr(np.asarray(G, dtype=np.float64))
    d = np.sign(np.diag(R))
    d[d == 0] = 1.0
    return Q * d[None, :]


def random_permutation(seed: int, stream: int, n: int) -> np.ndarray:
    """pi = the indices that sort the stream's first n draws (ascending).

    A uniformly random permutation: the draws are distinct (the SplitMix64
    finaliser is a bijection of 64-bit words), so every order is equally
    likely.  (P x)_r = x_{pi[r]}.
    """
    keys = splitmix64(seed, stream, np.arange(n, dtype=np.uint64))
    return np.argsort(keys, kind="stable")


def sylvester_hadamard(n: int) -> np.ndarray:
    """H_1 = [1], H_2k = [[H_k, H_k], [H_k, -H_k]] (Sylvester, natural order)."""
    if n < 1 or n & (n - 1):
        raise ValueError("Hadamard order must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def hadamard_row(n: int, i: int) -> np.ndarray:
    """Row i of the Sylvester H_n without forming it: (-1)^popcount(i & j)."""
    j = np.arange(n, dtype=np.int64)
    x = j & i
    par = np.zeros(n, dtype=np.int64)
    while np.any(x):
        par ^= x & 1
        x >>= 1
    return 1.0 - 2.0 * par


@dataclass
class SideTransform:
    """One random orthogonal matrix S (m-side U or n-side V).

    kind 'hadamard': T = H_d diag(s) / sqrt(d)          ([QuIP#] abstract)
    kind 'kronecker': T = A (x) B, A p x p, B q x q     ([QuIP] Introduction)
    kind 'identity':  T = I
    S = T P when perm is given ((P x)_r = x_{perm[r]}: the random permutation
    within the fast orthogonal multiplication, [QuIP] Experiments, "Further
    Ablation" / Table 5), else S = T.
    """
    kind: str
    dim: int
    signs: Optional[np.ndarray] = None
    A: Optional[np.ndarray] = None
    B: Optional[np.ndarray] = None
    perm: Optional[np.ndarray] = None

    def _structured(self) -> np.ndarray:
        d = self.dim
        if self.kind == "identity":
            return np.eye(d)
        if self.kind == "hadamard":
            return sylvester_hadamard(d) * self.signs[None, :] / math.sqrt(d)
        return np.kron(self.A, self.B)

    def perm_matrix(self) -> np.ndarray:
        """P with P[r, perm[r]] = 1 (the identity without a permutation)."""
        P = np.zeros((self.dim, self.dim))
        p = self.perm if self.perm is not None else np.arange(self.dim)
        P[np.arange(self.dim), p] = 1.0
        return P

    def matrix(self) -> np.ndarray:
        T = self._structured()
        return T if self.perm is None else T @ self.perm_matrix()

    def row(self, i: int) -> np.ndarray:
        d = self.dim
        if self.kind == "identity":
            r = np.zeros(d)
            r[i] = 1.0
        elif self.kind == "hadamard":
            r = hadamard_row(d, i) * self.signs / math.sqrt(d)
        else:
            q = self.B.shape[0]
            r = np.kron(self.A[i // q], self.B[i % q])
        return r if self.perm is None else r @ self.perm_matrix()

    def col(self, i: int) -> np.ndarray:
        """Column i of S (row i of S^T, what the inverse transform applies)."""
        d = self.dim
        j = i if self.perm is None else int(np.flatnonzero(self.perm == i)[0])
        if self.kind == "identity":
            c = np.zeros(d)
            c[j] = 1.0
        elif self.kind == "hadamard":
            c = hadamard_row(d, j) * (self.signs[j] / math.sqrt(d))   # H_d is symmetric
        else:
            q = self.B.shape[0]
            c = np.kron(self.A[:, j // q], self.B[:, j % q])
        return c


def make_side(seed: int, side: str, kind: str, dim: int, p: int = 0, q: int = 0,
              permute: bool = False) -> SideTransform:
    """Draw the transform for side 'm' (rows of W) or 'n' (columns of W)."""
    perm = None
    if permute:
        perm = random_permutation(seed, STREAM_M_PERM if side == "m" else STREAM_N_PERM, dim)
    if kind == "identity":
        return SideTransform("identity", dim, perm=perm)
    if kind == "hadamard":
        st = STREAM_M_SIGNS if side == "m" else STREAM_N_SIGNS
        return SideTransform("hadamard", dim, signs=random_signs(seed, st, dim), perm=perm)
    if kind == "kronecker":
        if p * q != dim:
            raise ValueError("Kronecker factors must multiply to the dimension")
        sa, sb = (STREAM_M_A, STREAM_M_B) if side == "m" else (STREAM_N_A, STREAM_N_B)
        A = haar_orthogonal(gaussian_matrix(seed, sa, p))
        B = haar_orthogonal(gaussian_matrix(seed, sb, q))
        return SideTransform("kronecker", dim, A=A, B=B, perm=perm)
    raise ValueError(kind)


def incoherence_forward(W: np.ndarray, H: np.ndarray, U: SideTransform, V: SideTransform
                        ) -> Tuple[np.ndarray, np.ndarray]:
    """W~ = U W V^T and H~ = V H V^T (symmetrised).

    [QuIP] incoherence-processing section ("random orthogonal
    multiplications H~ <- V H V^T and W~ <- U W V^T").
    """
    Um, Vn = U.matrix(), V.matrix()
    Wt = Um @ np.asarray(W, dtype=np.float64) @ Vn.T
    Ht = Vn @ np.asarray(H, dtype=np.float64) @ Vn.T
    return Wt, 0.5 * (Ht + Ht.T)


def incoherence_rows(W: np.ndarray, U: SideTransform, V: SideTransform, rows) -> np.ndarray:
    """Rows `rows` of W~ = U W V^T, row i being U[i, :] W V^T (same definition
    as incoherence_forward, restricted to some output rows; rows of W~ are
    what the row-independent LDLQ consumes)."""
    Vn = V.matrix()
    Ur = np.stack([U.row(int(i)) for i in rows])
    return (Ur @ np.asarray(W, dtype=np.float64)) @ Vn.T


def incoherence_hessian(H: np.ndarray, V: SideTransform) -> np.ndarray:
    """H~ = V H V^T (symmetrised), the Hessian half of incoherence_forward."""
    Vn = V.matrix()
    Ht = Vn @ np.asarray(H, dtype=np.float64) @ Vn.T
    return 0.5 * (Ht + Ht.T)


def incoherence_hessian_rows(H: np.ndarray, V: SideTransform, rows) -> np.ndarray:
    """Rows `rows` of V H V^T (before symmetrisation), row i being
    V[i, :] H V^T: the Hessian transform restricted to some rows."""
    Vr = np.stack([V.row(int(i)) for i in rows])
    return (Vr @ np.asarray(H, dtype=np.float64)) @ V.matrix().T


def incoherence_inverse_rows(Wt_hat: np.ndarray, U: SideTransform, V: SideTransform, rows
                             ) -> np.ndarray:
    """Rows `rows` of W^ = U^T W~^ V, row i being U[:, i]^T W~^ V: the
    inverse transform restricted to some output rows."""
    Uc = np.stack([U.col(int(i)) for i in rows])
    return (Uc @ np.asarray(Wt_hat, dtype=np.float64)) @ V.matrix()


def incoherence_inverse(Wt_hat: np.ndarray, U: SideTransform, V: SideTransform) -> np.ndarray:
    """W^ = U^T W~^ V: undo the transforms (QuIP post-processing)."""
    return U.matrix().T @ np.asarray(Wt_hat, dtype=np.float64) @ V.matrix()


# ----------------------------------------------------------------------------
# O4  LDL factorisation H = (I + U) D (I + U)^T, U strictly upper
# ----------------------------------------------------------------------------


def udu(H: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Return (U, D) with H = (I + U) diag(D) (I + U)^T, U strictly upper.

    The factor is unique for positive-definite H.  Written via the Cholesky
    factorisation of the index-reversed matrix J H J = L L^T (a library
    routine): R = J L J is upper triangular with H = R R^T, so D_k = R_kk^2
    and I + U = R diag(R)^-1.
    """
    H = np.asarray(H, dtype=np.float64)
    n = H.shape[0]
    if n == 0:
        return np.zeros((0, 0)), np.zeros(0)
    J = np.arange(n)[::-1]
    L = np.linalg.cholesky(H[np.ix_(J, J)])   # raises LinAlgError if not PD
    R = L[np.ix_(J, J)]
    d = np.diag(R).copy()
    Ufull = R / d[None, :]
    return np.triu(Ufull, 1), d * d


# ----------------------------------------------------------------------------
# O5/O6  Grid, rounding, LDLQ
# ----------------------------------------------------------------------------


def row_grid(Wt: np.ndarray, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row asymmetric 2^b-level grid: lo = min, s = (max - min)/(2^b - 1).

    A constant row (max == min) gets s = 1 so every code is 0.
    """
    Wt = np.asarray(Wt, dtype=np.float64)
    lo = Wt.min(axis=1)
    hi = Wt.max(axis=1)
    s = (hi - lo) / (2 ** bits - 1)
    s = np.where(hi > lo, s, 1.0)
    return lo, s


def quantize(a: np.ndarray, lo: np.ndarray, s: np.ndarray, bits: int) -> np.ndarray:
    """Q(a): nearest grid level, ties to even, clamped to [0, 2^b - 1]."""
    return np.clip(np.rint((a - lo) / s), 0, 2 ** bits - 1)


def ldlq(Wt: np.ndarray, U: np.ndarray, lo: np.ndarray, s: np.ndarray, bits: int
         ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """LDLQ, unblocked: for k = 0..n-1
         a_k  = W_k + sum_{j<k} (W_j - W^_j) U_jk
         c_k  = Q(a_k),   W^_k = lo + s c_k,   eta_k = W^_k - a_k.

    [QuIP] adaptive-rounding section (LDLQ; feedback matrix from the LDL
    factorisation of H).  Returns integer codes (m x n, int64), W^ and eta.
    Rows are independent.
    """
    Wt = np.asarray(Wt, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    m, n = Wt.shape
    codes = np.zeros((m, n), dtype=np.int64)
    What = np.zeros((m, n))
    eta = np.zeros((m, n))
    errT = np.zeros((n, m))                 # (W - W^)^T, filled column by column
    for k in range(n):
        a = Wt[:, k] + U[:k, k] @ errT[:k]
        c = quantize(a, lo, s, bits)
        codes[:, k] = c
        What[:, k] = lo + s * c
        eta[:, k] = What[:, k] - a
        errT[k] = Wt[:, k] - What[:, k]
    return codes, What, eta


def ldlq_blocked(Wt: np.ndarray, U: np.ndarray, lo: np.ndarray, s: np.ndarray, bits: int,
                 block: int) -> Tuple[np.ndarray, np.ndarray]:
    """LDLQ with the column sum split at block boundaries (lazy batch).

    Inside a block of ``block`` columns the feedback is applied column by
    column; when the block ends, every later column receives the block's
    error times the matching rows of U at once.  Same a_k as ``ldlq`` up to
    the order of additions.
    """
    Wt = np.asarray(Wt, dtype=np.float64)
    m, n = Wt.shape
    A = Wt.copy()
    codes = np.zeros((m, n), dtype=np.int64)
    What = np.zeros((m, n))
    for k0 in range(0, n, block):
        k1 = min(n, k0 + block)
        for k in range(k0, k1):
            c = quantize(A[:, k], lo, s, bits)
            codes[:, k] = c
            What[:, k] = lo + s * c
            A[:, k + 1:k1] += np.outer(Wt[:, k] - What[:, k], U[k, k + 1:k1])
        A[:, k1:] += (Wt[:, k0:k1] - What[:, k0:k1]) @ U[k0:k1, k1:]
    return codes, What


def nearest(Wt: np.ndarray, lo: np.ndarray, s: np.ndarray, bits: int) -> np.ndarray:
    """Nearest rounding ([QuIP] Experiments, "Methods."); lo, s are per row."""
    lo = np.asarray(lo, dtype=np.float64)[:, None]
    s = np.asarray(s, dtype=np.float64)[:, None]
    return quantize(np.asarray(Wt, dtype=np.float64), lo, s, bits).astype(np.int64)


def optq(Wt: np.ndarray, H: np.ndarray, lo: np.ndarray, s: np.ndarray, bits: int) -> np.ndarray:
    """OPTQ's update order ([QuIP] "OPTQ (Formerly known as GPTQ)."):
    quantize column k by nearest rounding, compute its error scaled by the
    pivot of the upper Cholesky factor R of H^-1 (H^-1 = R^T R), subtract it
    from the remaining columns along row k of R, repeat.  Returns codes."""
    w = np.array(Wt, dtype=np.float64, copy=True)
    Hinv = np.linalg.inv(np.asarray(H, dtype=np.float64))
    R = np.linalg.cholesky(Hinv).T              # upper, Hinv = R^T R
    m, n = w.shape
    codes = np.zeros((m, n), dtype=np.int64)
    for k in range(n):
        c = quantize(w[:, k], lo, s, bits)
        codes[:, k] = c
        e = (w[:, k] - (lo + s * c)) / R[k, k]
        w[:, k + 1:] -= np.outer(e, R[k, k + 1:])
    return codes


def diag_order(H: np.ndarray) -> np.ndarray:
    """LDLQ-RG's quantisation order ([QuIP] Experiments, "Methods.": LDLQ-RG
    re-orders the weights by diag(H)): the column indices sorted by
    decreasing H_kk, equal diagonal entries by increasing index.
    order[r] is the column quantised r-th."""
    d = np.diag(np.asarray(H, dtype=np.float64))
    return np.argsort(-d, kind="stable")


def greedy_pass(Wt: np.ndarray, H: np.ndarray, lo: np.ndarray, s: np.ndarray, bits: int,
                codes: np.ndarray, order=None) -> np.ndarray:
    """One pass of greedy updates to the proxy ([QuIP] Experiments,
    "Methods.": LDLQ-RG adds greedy updates to the proxy, "Greedy" performs
    them alone).  The columns are visited in ``order`` (default 0..n-1); at
    column k every other column is held at its current value and column k
    takes, per row, the grid point that minimises
    tr((W^ - W) H (W^ - W)^T) over that one column.  As a function of
    W^_k the proxy is H_kk (W^_k - t_k)^2 + const with
        t_k = W_k - sum_{j != k} (W^_j - W_j) H_jk / H_kk,
    so the minimiser on the grid is the grid point nearest t_k: Q(t_k).
    Returns the new codes."""
    Wt = np.asarray(Wt, dtype=np.float64)
    H = np.asarray(H, dtype=np.float64)
    lo = np.asarray(lo, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    c = np.array(codes, dtype=np.int64, copy=True)
    m, n = Wt.shape
    E = (lo[:, None] + s[:, None] * c) - Wt     # W^ - W, kept current
    for k in (range(n) if order is None else order):
        others = E @ H[:, k] - E[:, k] * H[k, k]
        t = Wt[:, k] - others / H[k, k]
        c[:, k] = quantize(t, lo, s, bits)
        E[:, k] = lo + s * c[:, k] - Wt[:, k]
    return c


def quantize_layer(method: str, Wt: np.ndarray, Ht: np.ndarray, lo: np.ndarray, s: np.ndarray,
                   bits: int, passes: int = 1) -> np.ndarray:
    """The rounding methods of [QuIP] Experiments, "Methods.", on the
    incoherent weights and Hessian, one per-row grid (lo, s):
      nearest : nearest rounding;
      ldlq    : LDLQ with the LDL factor of Ht;
      greedy  : nearest rounding, then ``passes`` greedy passes;
      ldlq_rg : columns re-ordered by decreasing diag(Ht), LDLQ in that
                order (the LDL factor of the re-ordered Ht), then ``passes``
                greedy passes visiting the columns in the same order.
    Returns the codes in the original column order."""
    Wt = np.asarray(Wt, dtype=np.float64)
    Ht = np.asarray(Ht, dtype=np.float64)
    if method == "nearest":
        return nearest(Wt, lo, s, bits)
    if method == "ldlq":
        return ldlq(Wt, udu(Ht)[0], lo, s, bits)[0]
    if method == "greedy":
        c = nearest(Wt, lo, s, bits)
        for _ in range(passes):
            c = greedy_pass(Wt, Ht, lo, s, bits, c)
        return c
    if method == "ldlq_rg":
        order = diag_order(Ht)
        Wp = Wt[:, order]
        Hp = Ht[np.ix_(order, order)]
        cp = ldlq(Wp, udu(Hp)[0], lo, s, bits)[0]
        for _ in range(passes):
            cp = greedy_pass(Wp, Hp, lo, s, bits, cp)
        c = np.empty_like(cp)
        c[:, order] = cp                        # column order[r] was quantised r-th
        return c
    raise ValueError(f"unknown rounding method {method!r}")


# ----------------------------------------------------------------------------
# O7/O8  Dequantisation, loss
# ----------------------------------------------------------------------------


def dequantize(codes: np.ndarray, lo: np.ndarray, s: np.ndarray) -> np.ndarray:
    """W~^ = lo + s * code, per row."""
    return np.asarray(lo, dtype=np.float64)[:, None] + np.asarray(s, dtype=np.float64)[:, None] * codes


def proxy_loss(What: np.ndarray, W: np.ndarray, H: np.ndarray) -> float:
    """l(W^) = tr((W^ - W) H (W^ - W)^T)  ([QuIP] Introduction)."""
    E = np.asarray(What, dtype=np.float64) - np.asarray(W, dtype=np.float64)
    return float(np.einsum("ij,ij->", E @ np.asarray(H, dtype=np.float64), E))


# ----------------------------------------------------------------------------
# Quantized inference: the layer's product with a full-precision vector
# ----------------------------------------------------------------------------


def code_slot_bits(bits: int) -> int:
    """Width of a code's slot in a packed 32-bit word: the code width when it
    divides 32 (1, 2, 4, 8), else the next of 4 and 8 (3 -> 4; 5, 6, 7 -> 8)."""
    if bits in (1, 2, 4, 8):
        return bits
    if 1 <= bits <= 8:
        return 4 if bits < 4 else 8
    raise ValueError("bits must be 1..8")


def packed_words(n: int, bits: int) -> int:
    """32-bit words per packed row: ceil(n / (32 / slot)), rounded up to a
    multiple of 4 (16 bytes)."""
    per = 32 // code_slot_bits(bits)
    w = -(-n // per)
    return -(-w // 4) * 4


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Packed codes for the quantized matrix-vector product.  The pages print
    no storage format (QuIP, Experiments, "Throughput Comparison." speaks of
    a quantized-matrix full-precision-vector product kernel); this one is the
    library's: row i has Wd = packed_words(n, bits) words, and code j of the
    row sits in word j mod Wd at bit (j div Wd) * slot.  Unused slots are 0.
    Returns (m, Wd) uint32."""
    codes = np.asarray(codes, dtype=np.int64)
    m, n = codes.shape
    slot = code_slot_bits(bits)
    Wd = packed_words(n, bits)
    out = np.zeros((m, Wd), dtype=np.uint64)
    for j in range(n):
        out[:, j % Wd] |= (codes[:, j].astype(np.uint64) << np.uint64((j // Wd) * slot))
    return out.astype(np.uint32)


def unpack_codes(packed: np.ndarray, n: int, bits: int) -> np.ndarray:
    """Inverse of pack_codes: (m, n) int64 codes."""
    packed = np.asarray(packed, dtype=np.uint64)
    slot = code_slot_bits(bits)
    Wd = packed.shape[1]
    mask = np.uint64((1 << slot) - 1)
    out = np.zeros((packed.shape[0], n), dtype=np.int64)
    for j in range(n):
        out[:, j] = ((packed[:, j % Wd] >> np.uint64((j // Wd) * slot)) & mask).astype(np.int64)
    return out


def quantized_matvec(codes: np.ndarray, lo: np.ndarray, s: np.ndarray, U: SideTransform,
                     V: SideTransform, x: np.ndarray) -> np.ndarray:
    """y = W^ x for the quantized layer W^ = U^T (lo + s codes) V (QuIP,
    incoherence-processing section: the post-processing that undoes the
    transforms; Experiments, "Throughput Comparison.": the quantized matrix
    times a full-precision vector at inference).  x: (B, n) vectors as rows;
    returns (B, m).  Written as the plain definition: the dequantised
    original-domain matrix times each vector."""
    W_hat = incoherence_inverse(dequantize(codes, lo, s), U, V)
    return np.asarray(x, dtype=np.float64) @ W_hat.T


# ----------------------------------------------------------------------------
# The whole layer
# ----------------------------------------------------------------------------


@dataclass
class Pipeline:
    H: np.ndarray           # damped proxy Hessian
    U: SideTransform
    V: SideTransform
    Wt: np.ndarray          # incoherent weights
    Ht: np.ndarray          # incoherent damped Hessian
    Uf: np.ndarray          # strictly upper LDL factor of Ht
    D: np.ndarray
    lo: np.ndarray
    s: np.ndarray
    codes: np.ndarray
    Wt_hat: np.ndarray      # dequantised, incoherent domain
    W_hat: np.ndarray       # dequantised, original domain
    loss: float             # tr((Wt_hat - Wt) Ht (Wt_hat - Wt)^T)


def run_pipeline(W: np.ndarray, X: np.ndarray, seed: int, m_side, n_side, bits: int,
                 alpha: float = 0.01, block: Optional[int] = None, method: str = "ldlq",
                 passes: int = 1) -> Pipeline:
    """Hessian -> damping -> incoherence -> LDL -> grid -> LDLQ -> dequant -> inverse.

    ``m_side`` / ``n_side`` are objects with attributes kind, p, q.
    ``method`` picks the rounding (``quantize_layer``); Uf and D stay the
    LDL of Ht in its original order.
    """
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    H = damp(hessian(X), alpha)
    U = make_side(seed, "m", m_side.kind, m, m_side.p, m_side.q, getattr(m_side, "permute", False))
    V = make_side(seed, "n", n_side.kind, n, n_side.p, n_side.q, getattr(n_side, "permute", False))
    Wt, Ht = incoherence_forward(W, H, U, V)
    Uf, D = udu(Ht)
    lo, s = row_grid(Wt, bits)
    if method != "ldlq":
        codes = quantize_layer(method, Wt, Ht, lo, s, bits, passes)
        Wt_hat = dequantize(codes, lo, s)
    elif block is None:
        codes, Wt_hat, _ = ldlq(Wt, Uf, lo, s, bits)
    else:
        codes, Wt_hat = ldlq_blocked(Wt, Uf, lo, s, bits, block)
    W_hat = incoherence_inverse(Wt_hat, U, V)
    return Pipeline(H, U, V, Wt, Ht, Uf, D, lo, s, codes, Wt_hat, W_hat,
                    proxy_loss(Wt_hat, Wt, Ht))
