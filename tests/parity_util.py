"""Helpers for the GPU parity tests: run CUDA stages through the C ABI on
oracle-made inputs and compare with the FP64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O


def dev(a, dtype=torch.float32):
    return torch.as_tensor(np.ascontiguousarray(a)).to(dtype).cuda()


def host(t):
    return t.detach().cpu().double().numpy()


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def ldlq_trajectory_check(codes, Wt, U, lo, s, bits, tau):
    """Every code must be the LDLQ decision given the codes before it.

    For the given codes (from the device), recompute in FP64
      a_k = W~_k + sum_{j<k} (W~_j - (lo + s c_j)) U_jk,  z_k = (a_k - lo)/s
    and return (mismatch fraction, fraction of mismatches that are NOT
    near-ties), where a near-tie has z_k within tau of a rounding boundary.
    """
    codes = np.asarray(codes, dtype=np.float64)
    lo = np.asarray(lo, dtype=np.float64)[:, None]
    s = np.asarray(s, dtype=np.float64)[:, None]
    Wt = np.asarray(Wt, dtype=np.float64)
    Err = Wt - (lo + s * codes)
    A = Wt + Err @ np.triu(np.asarray(U, dtype=np.float64), 1)
    z = (A - lo) / s
    want = np.clip(np.rint(z), 0, 2 ** bits - 1)
    bad = want != codes
    frac = np.abs(z - np.floor(z) - 0.5)          # distance to the nearest x.5
    near = frac < tau
    return float(bad.mean()), float((bad & ~near).mean())


def oracle_layer(cfg, d):
    """Full FP64 pipeline for a config's synthetic layer (small configs)."""
    return O.run_pipeline(d["W"], d["X"], cfg.seed, cfg.m_side, cfg.n_side, cfg.bits, cfg.damp)


def greedy_trajectory_check(C0, C1, Wt, H, lo, s, bits, tau):
    """Every code of C1 must be the greedy decision of one pass from C0.

    Column k is visited with columns j < k already updated (C1) and j > k
    not yet (C0): in FP64,
      t_k = W~_k - (sum_{j<k} E1_j H_jk + sum_{j>k} E0_j H_jk) / H_kk,
      z_k = (t_k - lo)/s, E = lo + s c - W~.
    Returns (mismatch fraction, fraction of mismatches that are NOT
    near-ties), a near-tie having z_k within tau of a rounding boundary.
    """
    lo = np.asarray(lo, dtype=np.float64)[:, None]
    s = np.asarray(s, dtype=np.float64)[:, None]
    Wt = np.asarray(Wt, dtype=np.float64)
    H = np.asarray(H, dtype=np.float64)
    E0 = lo + s * np.asarray(C0, dtype=np.float64) - Wt
    E1 = lo + s * np.asarray(C1, dtype=np.float64) - Wt
    others = E1 @ np.triu(H, 1) + E0 @ np.tril(H, -1)
    T = Wt - others / np.diag(H)[None, :]
    z = (T - lo) / s
    want = np.clip(np.rint(z), 0, 2 ** bits - 1)
    bad = want != np.asarray(C1, dtype=np.float64)
    frac = np.abs(z - np.floor(z) - 0.5)
    near = frac < tau
    return float(bad.mean()), float((bad & ~near).mean())


def row_scaled_err(A, B, s, same):
    """max |A - B| / s_i over the entries where the codes agree (mask
    ``same``), each entry measured against its own row's grid step s_i: the
    dequantised-weight tolerance is stated per row, so a row with a small
    step is not judged against a larger row's step."""
    s = np.asarray(s, dtype=np.float64)[:, None]
    e = np.abs(np.asarray(A, dtype=np.float64) - np.asarray(B, dtype=np.float64)) / s
    return float(e[np.asarray(same, dtype=bool)].max()) if np.any(same) else 0.0
