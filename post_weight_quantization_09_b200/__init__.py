"""Incoherence-processed LDLQ (QuIP / QuIP#) for one linear layer on a B200.

Thin PyTorch-facing binding of libquip (``include/quip.h``).  PyTorch only
owns device memory and supplies the CUDA stream; every step runs in the
library's sm_100a kernels.  The functions below carry the C entry points'
names and take torch tensors; ``LayerQuantizer`` strings them together for
one layer (Hessian -> damping -> incoherence -> LDL -> LDLQ -> dequantise ->
inverse transform) with buffers allocated once.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import _lib as L
from ._lib import QuipError, load, status_string  # noqa: F401

__all__ = [
    "Transform", "quip_hessian_accumulate", "quip_hessian_finalize", "quip_hessian_sharded",
    "token_range", "allreduce_hessian", "quip_incoherence_forward",
    "quip_incoherence_inverse", "quip_ldl", "quip_ldlq_quantize", "quip_dequantize",
    "quip_nearest_quantize", "quip_diag_order", "quip_permute", "quip_greedy_refine", "METHODS",
    "quip_packed_words", "quip_pack_codes", "quip_qmatvec", "QuantizedLinear",
    "quip_workspace_size", "quip_layer_workspace_size", "quip_quantize_layer", "quip_quantize_layer_host",
    "layer_views", "quip_sync_status", "quip_timing_begin", "quip_timing_end", "quip_timing_trace", "LayerQuantizer",
    "LayerGroupQuantizer", "quantize_layer", "QuipError",
    "KIND",
]

KIND = {"identity": L.QUIP_T_IDENTITY, "hadamard": L.QUIP_T_HADAMARD, "kronecker": L.QUIP_T_KRONECKER}

# Rounding methods of the QuIP paper, Experiments, "Methods.": nearest
# rounding; LDLQ; "Greedy" (nearest, then greedy passes over the proxy);
# LDLQ-RG (columns by decreasing diag(H~), LDLQ in that order, greedy passes).
METHODS = ("ldlq", "nearest", "greedy", "ldlq_rg")


def _kind(side) -> int:
    """quip_tkind of a side spec (kind, p, q[, permute]), with QUIP_T_PERMUTE when asked."""
    return KIND[side.kind] | (L.QUIP_T_PERMUTE if getattr(side, "permute", False) else 0)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return L.QUIP_BF16
    if t.dtype == torch.float32:
        return L.QUIP_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _cuda(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


_cudart = None


def _memcpy_d2d(dst_ptr: int, src_ptr: int, nbytes: int) -> None:
    """Device-to-device copy through the CUDA runtime torch already loaded."""
    global _cudart
    if _cudart is None:
        _cudart = ctypes.CDLL("libcudart.so.12")
        _cudart.cudaMemcpy.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int]
        _cudart.cudaMemcpy.restype = ctypes.c_int
    if _cudart.cudaMemcpy(ctypes.c_void_p(dst_ptr), ctypes.c_void_p(src_ptr), nbytes, 3) != 0:
        raise RuntimeError("cudaMemcpy failed")


class Transform:
    """The pair (U, V) of random orthogonal matrices for an m x n layer."""

    def __init__(self, seed: int, m: int, n: int, m_side, n_side, stream=None):
        lib = load()
        self.m, self.n = m, n
        self.m_side, self.n_side = m_side, n_side
        h = ctypes.c_void_p()
        L.check(lib.quip_transform_create(
            ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF), m, n, _kind(m_side), m_side.p, m_side.q,
            _kind(n_side), n_side.p, n_side.q, _s(stream), ctypes.byref(h)), "quip_transform_create")
        self.handle = h

    def draw(self, seed: int, stream=None) -> None:
        """Redraw the random signs / factors from `seed` in place (no allocation)."""
        L.check(load().quip_transform_draw(self.handle, ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF),
                                           _s(stream)), "quip_transform_draw")

    def close(self) -> None:
        if self.handle:
            load().quip_transform_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def factors(self, side: int) -> dict:
        """Copies of one side's data: {'kind', 'signs'} or {'kind', 'A', 'B'} (fp32, cuda),
        plus 'perm' (int32, cuda) when the side has a random permutation."""
        kind, p, q = ctypes.c_int(), ctypes.c_int64(), ctypes.c_int64()
        s, a, b = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
        L.check(load().quip_transform_info(self.handle, side, ctypes.byref(kind), ctypes.byref(p),
                                           ctypes.byref(q), ctypes.byref(s), ctypes.byref(a),
                                           ctypes.byref(b)), "quip_transform_info")
        torch.cuda.synchronize()
        dim = self.m if side == 0 else self.n
        out = {"kind": kind.value}
        if kind.value == L.QUIP_T_HADAMARD:
            t = torch.empty(dim, dtype=torch.float32, device="cuda")
            _memcpy_d2d(t.data_ptr(), s.value, dim * 4)
            out["signs"] = t
        elif kind.value == L.QUIP_T_KRONECKER:
            A = torch.empty(p.value, p.value, dtype=torch.float32, device="cuda")
            B = torch.empty(q.value, q.value, dtype=torch.float32, device="cuda")
            _memcpy_d2d(A.data_ptr(), a.value, A.numel() * 4)
            _memcpy_d2d(B.data_ptr(), b.value, B.numel() * 4)
            out["A"], out["B"] = A, B
        pp = ctypes.c_void_p()
        L.check(load().quip_transform_permutation(self.handle, side, ctypes.byref(pp)),
                "quip_transform_permutation")
        if pp.value:
            P = torch.empty(dim, dtype=torch.int32, device="cuda")
            _memcpy_d2d(P.data_ptr(), pp.value, dim * 4)
            out["perm"] = P
        return out


def quip_workspace_size(op: int, tf: Optional[Transform], m: int, n: int, block: int = 0) -> int:
    nb = ctypes.c_size_t()
    L.check(load().quip_workspace_size(op, tf.handle if tf else None, m, n, block, ctypes.byref(nb)),
            "quip_workspace_size")
    return nb.value


def _ws(nbytes: int, device) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def quip_hessian_accumulate(X: torch.Tensor, H_acc: torch.Tensor, accumulate: bool = False,
                            stream=None) -> None:
    _cuda(X, "X"), _cuda(H_acc, "H_acc")
    N, n = X.shape
    L.check(load().quip_hessian_accumulate(_p(X), _dtype(X), N, n, X.stride(0), _p(H_acc),
                                           int(accumulate), _s(stream)), "quip_hessian_accumulate")


def quip_hessian_finalize(H: torch.Tensor, N_total: int, damp: float, stream=None) -> None:
    _cuda(H, "H")
    L.check(load().quip_hessian_finalize(_p(H), H.shape[0], N_total, damp, _s(stream)),
            "quip_hessian_finalize")


def token_range(N_total: int, world: int, rank: int) -> Tuple[int, int]:
    """Tokens [t0, t1) of N_total that rank ``rank`` of ``world`` accumulates
    for a token-sharded Hessian: contiguous, sizes differ by at most one, the
    ranks together cover each token once (a rank may get none)."""
    if world < 1 or not 0 <= rank < world or N_total < 0:
        raise ValueError(f"token_range: N_total={N_total}, world={world}, rank={rank}")
    q, r = divmod(N_total, world)
    t0 = rank * q + min(rank, r)
    return t0, t0 + q + (1 if rank < r else 0)


def allreduce_hessian(H_acc: torch.Tensor, group=None, stream=None) -> None:
    """H_acc <- the sum of every rank's H_acc over ``group``: one all-reduce
    of the n x n fp32 buffer, ordered on ``stream`` (default: the current
    stream) for device buffers.  The strict upper triangle, which the
    accumulation leaves unspecified, is summed too; quip_hessian_finalize
    never reads it.  Without a process group of two or more ranks it does
    nothing."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return
    if H_acc.is_cuda:
        with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream()):
            dist.all_reduce(H_acc, op=dist.ReduceOp.SUM, group=group)
    else:
        dist.all_reduce(H_acc, op=dist.ReduceOp.SUM, group=group)


def quip_hessian_sharded(X_local: torch.Tensor, H: torch.Tensor, N_total: int, damp: float,
                         group=None, stream=None) -> None:
    """The proxy Hessian of calibration tokens spread over the ranks of
    ``group`` (QuIP, adaptive-rounding section: H is the inputs' second
    moment, a sum over tokens, so token shards add): each rank accumulates
    X_local^T X_local over its own tokens, one all-reduce sums the partial
    sums, and every rank finalizes the same H with the total count N_total
    (the sum of the ranks' token counts) and damping ``damp``.  The LDL and
    the rest of the layer then run on each rank from that H."""
    quip_hessian_accumulate(X_local, H, stream=stream)
    allreduce_hessian(H, group, stream)
    quip_hessian_finalize(H, N_total, damp, stream=stream)


def quip_incoherence_forward(tf: Transform, W: Optional[torch.Tensor], W_t: Optional[torch.Tensor],
                             H: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                             stream=None) -> None:
    """W_t = U W V^T (skipped when W is None) and H = V H V^T in place
    (skipped when H is None)."""
    if W is not None:
        _cuda(W, "W"), _cuda(W_t, "W_t")
    ref = W if W is not None else H
    need = quip_workspace_size(L.QUIP_OP_INCOHERENCE_FORWARD, tf, tf.m, tf.n)
    if ws is None:
        ws = _ws(need, ref.device if ref is not None else torch.device("cuda"))
    dt = _dtype(W) if W is not None else L.QUIP_F32
    ldw = W.stride(0) if W is not None else tf.n
    L.check(load().quip_incoherence_forward(tf.handle, _p(W), dt, ldw, _p(W_t), _p(H),
                                            _p(ws), 0 if ws is None else ws.numel(), _s(stream)),
            "quip_incoherence_forward")


def quip_incoherence_inverse(tf: Transform, W_hat_t: torch.Tensor, W_hat: torch.Tensor,
                             ws: Optional[torch.Tensor] = None, stream=None) -> None:
    need = quip_workspace_size(L.QUIP_OP_INCOHERENCE_INVERSE, tf, tf.m, tf.n)
    if ws is None:
        ws = _ws(need, W_hat.device)
    L.check(load().quip_incoherence_inverse(tf.handle, _p(W_hat_t), _p(W_hat), _p(ws),
                                            0 if ws is None else ws.numel(), _s(stream)),
            "quip_incoherence_inverse")


def quip_ldl(H_t: torch.Tensor, D: torch.Tensor, ws: Optional[torch.Tensor] = None, stream=None) -> None:
    _cuda(H_t, "H_t")
    n = H_t.shape[0]
    need = quip_workspace_size(L.QUIP_OP_LDL, None, n, n)
    if ws is None:
        ws = _ws(need, H_t.device)
    L.check(load().quip_ldl(_p(H_t), _p(D), n, _p(ws), 0 if ws is None else ws.numel(), _s(stream)),
            "quip_ldl")


def quip_ldlq_quantize(W_t: torch.Tensor, Uring: torch.Tensor, bits: int, block: int,
                       codes: torch.Tensor, lo: torch.Tensor, scale: torch.Tensor,
                       ws: Optional[torch.Tensor] = None, stream=None) -> None:
    m, n = W_t.shape
    need = quip_workspace_size(L.QUIP_OP_LDLQ, None, m, n, block)
    if ws is None:
        ws = _ws(need, W_t.device)
    L.check(load().quip_ldlq_quantize(_p(W_t), _p(Uring), Uring.stride(0), m, n, bits, block, _p(codes),
                                      _p(lo), _p(scale), _p(ws), 0 if ws is None else ws.numel(),
                                      _s(stream)), "quip_ldlq_quantize")


def quip_nearest_quantize(W_t: torch.Tensor, bits: int, codes: torch.Tensor, lo: torch.Tensor,
                          scale: torch.Tensor, stream=None) -> None:
    m, n = W_t.shape
    L.check(load().quip_nearest_quantize(_p(W_t), m, n, bits, _p(codes), _p(lo), _p(scale), _s(stream)),
            "quip_nearest_quantize")


def quip_diag_order(H: torch.Tensor, perm: torch.Tensor, iperm: Optional[torch.Tensor] = None,
                    stream=None) -> None:
    _cuda(H, "H")
    L.check(load().quip_diag_order(_p(H), H.stride(0), H.shape[0], _p(perm), _p(iperm), _s(stream)),
            "quip_diag_order")


_PERM_DTYPE = {torch.float32: L.QUIP_F32, torch.bfloat16: L.QUIP_BF16, torch.uint8: L.QUIP_U8}


def quip_permute(inp: torch.Tensor, out: torch.Tensor, row_perm: Optional[torch.Tensor] = None,
                 col_perm: Optional[torch.Tensor] = None, stream=None) -> None:
    """out[r, c] = inp[row_perm[r], col_perm[c]] (None: identity)."""
    if inp.dtype != out.dtype or inp.dtype not in _PERM_DTYPE:
        raise TypeError(f"unsupported dtypes {inp.dtype} -> {out.dtype}")
    rows, cols = inp.shape
    L.check(load().quip_permute(_p(inp), _PERM_DTYPE[inp.dtype], rows, cols, inp.stride(0), _p(row_perm),
                                _p(col_perm), _p(out), out.stride(0), _s(stream)), "quip_permute")


def quip_greedy_refine(W_t: torch.Tensor, H: torch.Tensor, bits: int, lo: torch.Tensor,
                       scale: torch.Tensor, codes: torch.Tensor, passes: int = 1,
                       ws: Optional[torch.Tensor] = None, stream=None) -> None:
    m, n = W_t.shape
    need = quip_workspace_size(L.QUIP_OP_GREEDY, None, m, n)
    if ws is None:
        ws = _ws(need, W_t.device)
    L.check(load().quip_greedy_refine(_p(W_t), _p(H), H.stride(0), m, n, bits, _p(lo), _p(scale),
                                      _p(codes), passes, _p(ws), 0 if ws is None else ws.numel(),
                                      _s(stream)), "quip_greedy_refine")


def quip_packed_words(n: int, bits: int) -> int:
    return int(load().quip_packed_words(n, bits))


def quip_pack_codes(codes: torch.Tensor, bits: int, packed: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """Packed codes (m x packed_words int32 words; see quip.h for the layout)."""
    m, n = codes.shape
    if packed is None:
        packed = torch.empty(m, quip_packed_words(n, bits), dtype=torch.int32, device=codes.device)
    L.check(load().quip_pack_codes(_p(codes), m, n, bits, _p(packed), packed.stride(0), _s(stream)),
            "quip_pack_codes")
    return packed


def quip_qmatvec(tf: Transform, packed: torch.Tensor, lo: torch.Tensor, scale: torch.Tensor, bits: int,
                 x: torch.Tensor, y: torch.Tensor, ws: Optional[torch.Tensor] = None, stream=None) -> None:
    """y[b] = U^T (lo + s codes) V x[b] for the rows b of x (B x n) into y (B x m)."""
    B = x.shape[0]
    if ws is None:
        ws = _ws(quip_workspace_size(L.QUIP_OP_QMATVEC, tf, tf.m, tf.n, B), x.device)
    L.check(load().quip_qmatvec(tf.handle, _p(packed), packed.stride(0), _p(lo), _p(scale), bits, _p(x),
                                _dtype(x), x.stride(0), B, _p(y), y.stride(0), _p(ws),
                                0 if ws is None else ws.numel(), _s(stream)), "quip_qmatvec")


class QuantizedLinear:
    """A quantized layer for inference: y = W^ x with W^ = U^T (lo + s codes) V
    kept as packed codes, the per-row grid and the layer's transform (QuIP,
    Experiments, "Throughput Comparison.").  ``max_batch`` sizes the
    workspace; ``__call__`` takes x (B x n, fp32 or bf16, B <= max_batch)."""

    def __init__(self, tf: Transform, codes: torch.Tensor, lo: torch.Tensor, scale: torch.Tensor,
                 bits: int, max_batch: int = 8, stream=None):
        self.tf, self.bits, self.stream = tf, bits, stream
        self.m, self.n = tf.m, tf.n
        self.packed = quip_pack_codes(codes, bits, stream=stream)
        self.lo, self.scale = lo, scale
        self.max_batch = max_batch
        self.ws = torch.empty(max(quip_workspace_size(L.QUIP_OP_QMATVEC, tf, tf.m, tf.n, max_batch), 256),
                              dtype=torch.uint8, device=codes.device)

    def __call__(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        if x.shape[0] > self.max_batch:
            raise ValueError(f"batch {x.shape[0]} > max_batch {self.max_batch}")
        if out is None:
            out = torch.empty(x.shape[0], self.m, dtype=torch.float32, device=x.device)
        quip_qmatvec(self.tf, self.packed, self.lo, self.scale, self.bits, x, out, self.ws, self.stream)
        return out


def quip_dequantize(codes: torch.Tensor, lo: torch.Tensor, scale: torch.Tensor, W_hat_t: torch.Tensor,
                    stream=None) -> None:
    m, n = codes.shape
    L.check(load().quip_dequantize(_p(codes), _p(lo), _p(scale), m, n, _p(W_hat_t), _s(stream)),
            "quip_dequantize")


def quip_layer_workspace_size(tf: Transform, N: int, w_dtype: int, x_dtype: int, block: int,
                              host: bool) -> int:
    nb = ctypes.c_size_t()
    L.check(load().quip_layer_workspace_size(tf.handle, N, w_dtype, x_dtype, block, int(host), ctypes.byref(nb)),
            "quip_layer_workspace_size")
    return nb.value


def quip_quantize_layer(tf: Transform, seed: int, W: torch.Tensor, X: torch.Tensor, bits: int, block: int,
                        damp: float, codes: torch.Tensor, lo: torch.Tensor, scale: torch.Tensor,
                        W_hat: Optional[torch.Tensor], ws: torch.Tensor, stream=None) -> None:
    """The whole layer on device tensors (include/quip.h)."""
    _cuda(W, "W"), _cuda(X, "X")
    L.check(load().quip_quantize_layer(
        tf.handle, ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF), _p(W), _dtype(W), W.stride(0), _p(X), _dtype(X),
        X.shape[0], X.stride(0), bits, block, damp, _p(codes), _p(lo), _p(scale), _p(W_hat), _p(ws), ws.numel(),
        _s(stream)), "quip_quantize_layer")


def quip_quantize_layer_host(tf: Transform, seed: int, W_host: torch.Tensor, X_host: torch.Tensor, bits: int,
                             block: int, damp: float, codes_host: torch.Tensor, lo_host: torch.Tensor,
                             scale_host: torch.Tensor, W_hat_host: Optional[torch.Tensor], ws: torch.Tensor,
                             stream=None) -> None:
    """The whole layer from host tensors to host tensors (include/quip.h);
    synchronise `stream` before reading the outputs."""
    for t, nm in ((W_host, "W_host"), (X_host, "X_host"), (codes_host, "codes_host")):
        if t.is_cuda:
            raise ValueError(f"{nm} must be a host tensor")
    L.check(load().quip_quantize_layer_host(
        tf.handle, ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF), _p(W_host), _dtype(W_host), W_host.stride(0),
        _p(X_host), _dtype(X_host), X_host.shape[0], X_host.stride(0), bits, block, damp, _p(codes_host),
        _p(lo_host), _p(scale_host), _p(W_hat_host), _p(ws), ws.numel(), _s(stream)), "quip_quantize_layer_host")


def _round256(b: int) -> int:
    return (b + 255) // 256 * 256


def layer_views(ws: torch.Tensor, m: int, n: int):
    """(H, D, W_t) inside a whole-layer workspace after the call: the n x n
    matrix holding U in its strict upper triangle, D and W~ (the offsets
    include/quip.h gives)."""
    d0 = _round256(4 * n * n)
    w0 = d0 + _round256(4 * n)
    f32 = lambda a, cnt: ws[a:a + 4 * cnt].view(torch.float32)
    return f32(0, n * n).view(n, n), f32(d0, n), f32(w0, m * n).view(m, n)


def quip_sync_status(stream=None) -> int:
    return load().quip_sync_status(_s(stream))


def quip_timing_begin() -> None:
    L.check(load().quip_timing_begin(), "quip_timing_begin")


def quip_timing_end(max_entries: int = 64) -> dict:
    """{kernel name: (launches, total ms)} of the launches since quip_timing_begin()."""
    lib = load()
    names = (ctypes.c_char_p * max_entries)()
    counts = (ctypes.c_uint64 * max_entries)()
    ms = (ctypes.c_double * max_entries)()
    n = ctypes.c_int(0)
    L.check(lib.quip_timing_end(names, counts, ms, max_entries, ctypes.byref(n)), "quip_timing_end")
    return {names[i].decode(): (int(counts[i]), float(ms[i])) for i in range(min(n.value, max_entries))}


def quip_timing_trace(max_entries: int = 8192) -> list:
    """[(kernel name, start ms, end ms, stream id)] of the launches since
    quip_timing_begin(), in enqueue order, times after the first launch's start."""
    lib = load()
    names = (ctypes.c_char_p * max_entries)()
    t0 = (ctypes.c_double * max_entries)()
    t1 = (ctypes.c_double * max_entries)()
    sid = (ctypes.c_int * max_entries)()
    n = ctypes.c_int(0)
    L.check(lib.quip_timing_trace(names, t0, t1, sid, max_entries, ctypes.byref(n)), "quip_timing_trace")
    return [(names[i].decode(), float(t0[i]), float(t1[i]), int(sid[i])) for i in range(min(n.value, max_entries))]


@dataclass
class LayerResult:
    codes: torch.Tensor      # m x n uint8
    lo: torch.Tensor         # m fp32
    scale: torch.Tensor      # m fp32
    W_hat: torch.Tensor      # m x n fp32, dequantised in the original basis


class LayerQuantizer:
    """Buffers and transform for quantising one m x n layer; ``run`` issues the
    whole pipeline on one stream through the C ABI.  ``method`` is one of
    METHODS; ``passes`` is the number of greedy passes of "greedy" and
    "ldlq_rg"."""

    X_CHUNKS = 4            # token chunks of X in run_host (copy / Hessian overlap)

    def __init__(self, m: int, n: int, m_side, n_side, bits: int, block: int, damp: float = 0.01,
                 seed: int = 0, device: str = "cuda", stream=None, method: str = "ldlq",
                 passes: int = 1):
        if method not in METHODS:
            raise ValueError(f"method must be one of {METHODS}")
        self.m, self.n, self.bits, self.block, self.damp, self.seed = m, n, bits, block, damp, seed
        self.m_side, self.n_side = m_side, n_side
        self.method, self.passes = method, passes
        self.stream = stream
        dev = torch.device(device)
        f32 = dict(dtype=torch.float32, device=dev)
        self.H = torch.empty(n, n, **f32)
        self.W_t = torch.empty(m, n, **f32)
        self.D = torch.empty(n, **f32)
        self.codes = torch.empty(m, n, dtype=torch.uint8, device=dev)
        self.lo = torch.empty(m, **f32)
        self.scale = torch.empty(m, **f32)
        self.W_hat = torch.empty(m, n, **f32)
        self.tf: Optional[Transform] = None
        if method == "ldlq_rg":
            # the re-ordered problem: H~ and W~ with columns (and H~'s rows) in
            # the quantisation order, the codes in that order, the order itself
            self.Hp = torch.empty(n, n, **f32)
            self.Wp = torch.empty(m, n, **f32)
            self.codes_p = torch.empty(m, n, dtype=torch.uint8, device=dev)
            self.perm = torch.empty(n, dtype=torch.int32, device=dev)
            self.iperm = torch.empty(n, dtype=torch.int32, device=dev)
        ws = 0
        probe = Transform(seed, m, n, m_side, n_side, stream)
        for op, blk in ((L.QUIP_OP_INCOHERENCE_FORWARD, 0), (L.QUIP_OP_INCOHERENCE_INVERSE, 0),
                        (L.QUIP_OP_LDL, 0), (L.QUIP_OP_LDLQ, block), (L.QUIP_OP_GREEDY, 0)):
            if op == L.QUIP_OP_GREEDY and method not in ("greedy", "ldlq_rg"):
                continue
            ws = max(ws, quip_workspace_size(op, probe, m, n, blk))
        self.tf = probe
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)

    def new_transform(self) -> None:
        """Draw (U, V) again from the seed on the device (part of a full pass)."""
        self.tf.draw(self.seed, self.stream)

    def _layer_ws(self, N: int, w_dtype: int, x_dtype: int, host: bool) -> torch.Tensor:
        """Workspace of the whole-layer calls for N tokens (kept per shape)."""
        cache = self.__dict__.setdefault("_lws", {})
        key = (N, w_dtype, x_dtype, host)
        if key not in cache:
            nb = quip_layer_workspace_size(self.tf, N, w_dtype, x_dtype, self.block, host)
            cache[key] = torch.empty(max(nb, 256), dtype=torch.uint8, device=self.H.device)
        return cache[key]

    def run(self, W: torch.Tensor, X: torch.Tensor, redraw_transform: bool = True,
            w_ready: Optional[torch.cuda.Event] = None, after_ldlq=None,
            x_ready=None) -> LayerResult:
        """The whole layer on one stream.  H's transform and the LDL come
        before W's transform (they do not need W): ``w_ready``, when given, is
        waited for just before W is read, so a copy of W can overlap them.
        ``x_ready``, when given, is a list of (first row, end row, event): the
        Hessian accumulates each token chunk of X once its event completes.
        ``after_ldlq`` (a callable) is invoked once codes and grid are final."""
        st = self.stream
        stream = st if st is not None else torch.cuda.current_stream()
        if self.method == "ldlq" and redraw_transform and not x_ready and w_ready is None \
                and after_ldlq is None:
            # the whole layer in one library call
            ws = self._layer_ws(X.shape[0], _dtype(W), _dtype(X), False)
            quip_quantize_layer(self.tf, self.seed, W, X, self.bits, self.block, self.damp, self.codes, self.lo,
                                self.scale, self.W_hat, ws, st)
            self.H, self.D, self.W_t = layer_views(ws, self.m, self.n)
            return LayerResult(self.codes, self.lo, self.scale, self.W_hat)
        if redraw_transform:
            self.new_transform()
        if x_ready:
            for i, (a, b, ev) in enumerate(x_ready):
                stream.wait_event(ev)
                quip_hessian_accumulate(X[a:b], self.H, i > 0, st)
        else:
            quip_hessian_accumulate(X, self.H, False, st)
        quip_hessian_finalize(self.H, X.shape[0], self.damp, st)
        quip_incoherence_forward(self.tf, None, None, self.H, self.ws, st)
        self.prepare_hessian()
        if w_ready is not None:
            stream.wait_event(w_ready)
        quip_incoherence_forward(self.tf, W, self.W_t, None, self.ws, st)
        self.round_weights()
        if after_ldlq is not None:
            after_ldlq()
        quip_dequantize(self.codes, self.lo, self.scale, self.W_hat, st)
        quip_incoherence_inverse(self.tf, self.W_hat, self.W_hat, self.ws, st)
        return LayerResult(self.codes, self.lo, self.scale, self.W_hat)

    def prepare_hessian(self) -> None:
        """What the method needs from H~ (in self.H) before W~ exists: the LDL
        for "ldlq"; for "ldlq_rg" the order by diag(H~) and the LDL of the
        re-ordered H~ (in self.Hp; self.H is left as it is)."""
        st = self.stream
        if self.method == "ldlq_rg":
            quip_diag_order(self.H, self.perm, self.iperm, st)
            quip_permute(self.H, self.Hp, self.perm, self.perm, st)
            quip_ldl(self.Hp, self.D, self.ws, st)
        elif self.method == "ldlq":
            quip_ldl(self.H, self.D, self.ws, st)

    def round_weights(self) -> None:
        """Codes and grid of W~ (in self.W_t) by the layer's method."""
        st, method = self.stream, self.method
        if method == "ldlq":
            quip_ldlq_quantize(self.W_t, self.H, self.bits, self.block, self.codes, self.lo,
                               self.scale, self.ws, st)
        elif method in ("nearest", "greedy"):
            quip_nearest_quantize(self.W_t, self.bits, self.codes, self.lo, self.scale, st)
            if method == "greedy":
                quip_greedy_refine(self.W_t, self.H, self.bits, self.lo, self.scale, self.codes,
                                   self.passes, self.ws, st)
        else:
            quip_permute(self.W_t, self.Wp, None, self.perm, st)
            quip_ldlq_quantize(self.Wp, self.Hp, self.bits, self.block, self.codes_p, self.lo,
                               self.scale, self.ws, st)
            if self.passes > 0:
                # the LDL overwrote Hp: gather the re-ordered H~ again
                quip_permute(self.H, self.Hp, self.perm, self.perm, st)
                quip_greedy_refine(self.Wp, self.Hp, self.bits, self.lo, self.scale, self.codes_p,
                                   self.passes, self.ws, st)
            quip_permute(self.codes_p, self.codes, None, self.iperm, st)

    def run_host(self, W_host: torch.Tensor, X_host: torch.Tensor, codes_out: torch.Tensor,
                 lo_out: torch.Tensor, scale_out: torch.Tensor) -> None:
        """Host in, host out: copy W and X (pinned host tensors) to the device,
        run the layer, copy codes / lo / scale back into the pinned outputs.
        Copies run on a second stream: X in X_CHUNKS token chunks, each
        accumulated into the Hessian as soon as it lands, then W, overlapping
        the Hessian, its transform and the LDL; the results go back on that
        stream while the dequantisation and inverse transform run.
        Everything is joined into the layer's stream; synchronise it to read.
        LDLQ runs as one library call (quip_quantize_layer_host), which does
        these copies and their overlap itself."""
        if self.method == "ldlq":
            ws = self._layer_ws(X_host.shape[0], _dtype(W_host), _dtype(X_host), True)
            quip_quantize_layer_host(self.tf, self.seed, W_host, X_host, self.bits, self.block, self.damp,
                                     codes_out, lo_out, scale_out, None, ws, self.stream)
            return
        if getattr(self, "_W_dev", None) is None or self._W_dev.shape != W_host.shape \
                or self._W_dev.dtype != W_host.dtype:
            self._W_dev = torch.empty_like(W_host, device="cuda")
        if getattr(self, "_X_dev", None) is None or self._X_dev.shape != X_host.shape \
                or self._X_dev.dtype != X_host.dtype:
            self._X_dev = torch.empty_like(X_host, device="cuda")
        if getattr(self, "_copy", None) is None:
            self._copy = torch.cuda.Stream()
        main = self.stream if self.stream is not None else torch.cuda.current_stream()
        cp = self._copy
        cp.wait_stream(main)                       # the previous call is done with the buffers
        N = X_host.shape[0]
        step = max(1, -(-N // self.X_CHUNKS))
        x_ready = []
        with torch.cuda.stream(cp):
            for a in range(0, N, step):
                b = min(N, a + step)
                self._X_dev[a:b].copy_(X_host[a:b], non_blocking=True)
                x_ready.append((a, b, cp.record_event()))
            self._W_dev.copy_(W_host, non_blocking=True)
        w_ready = cp.record_event()

        def results_out():
            cp.wait_stream(main)
            with torch.cuda.stream(cp):
                codes_out.copy_(self.codes, non_blocking=True)
                lo_out.copy_(self.lo, non_blocking=True)
                scale_out.copy_(self.scale, non_blocking=True)

        self.run(self._W_dev, self._X_dev, w_ready=w_ready, after_ldlq=results_out, x_ready=x_ready)
        main.wait_stream(cp)


class LayerGroupQuantizer:
    """Quantise G layers of the same shape that read the same input (the
    q, k and v projections of an attention block; up and gate of an MLP):
    the proxy Hessian H = X^T X / N, its incoherence transform and its LDL
    are computed once, and LDLQ runs once on the G incoherent weight
    matrices stacked by rows (rows are independent: each row's rounding
    only involves its own entries and the shared factor).  All layers use
    the same transform (U, V), as one seed draws it; ``run`` issues the whole
    group on one stream through the C ABI.  Each layer's codes, grid and
    dequantised weights are exactly those of ``LayerQuantizer`` on that layer
    with the same X."""

    def __init__(self, groups: int, m: int, n: int, m_side, n_side, bits: int, block: int,
                 damp: float = 0.01, seed: int = 0, device: str = "cuda", stream=None):
        if groups < 1:
            raise ValueError("groups must be >= 1")
        self.G, self.m, self.n = groups, m, n
        self.bits, self.block, self.damp, self.seed = bits, block, damp, seed
        self.stream = stream
        dev = torch.device(device)
        f32 = dict(dtype=torch.float32, device=dev)
        self.H = torch.empty(n, n, **f32)
        self.W_t = torch.empty(groups * m, n, **f32)
        self.D = torch.empty(n, **f32)
        self.codes = torch.empty(groups * m, n, dtype=torch.uint8, device=dev)
        self.lo = torch.empty(groups * m, **f32)
        self.scale = torch.empty(groups * m, **f32)
        self.W_hat = torch.empty(groups * m, n, **f32)
        self.tf = Transform(seed, m, n, m_side, n_side, stream)
        ws = 0
        for op, mm, blk in ((L.QUIP_OP_INCOHERENCE_FORWARD, m, 0), (L.QUIP_OP_INCOHERENCE_INVERSE, m, 0),
                            (L.QUIP_OP_LDL, m, 0), (L.QUIP_OP_LDLQ, groups * m, block)):
            ws = max(ws, quip_workspace_size(op, self.tf if op != L.QUIP_OP_LDLQ else None, mm, n, blk))
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)

    def run(self, Ws, X: torch.Tensor, redraw_transform: bool = True) -> "LayerResult":
        """Ws: G tensors m x n (or one G m x n tensor); X: N x n calibration
        inputs shared by the layers.  Returns the stacked results (layer g in
        rows [g m, (g + 1) m))."""
        Ws = list(Ws.split(self.m, dim=0)) if isinstance(Ws, torch.Tensor) else list(Ws)
        if len(Ws) != self.G:
            raise ValueError(f"expected {self.G} weight matrices, got {len(Ws)}")
        st, m = self.stream, self.m
        if redraw_transform:
            self.tf.draw(self.seed, st)
        quip_hessian_accumulate(X, self.H, False, st)
        quip_hessian_finalize(self.H, X.shape[0], self.damp, st)
        for g, W in enumerate(Ws):
            quip_incoherence_forward(self.tf, W, self.W_t[g * m:(g + 1) * m], self.H if g == 0 else None,
                                     self.ws, st)
        quip_ldl(self.H, self.D, self.ws, st)
        quip_ldlq_quantize(self.W_t, self.H, self.bits, self.block, self.codes, self.lo, self.scale,
                           self.ws, st)
        quip_dequantize(self.codes, self.lo, self.scale, self.W_hat, st)
        for g in range(self.G):
            rows = self.W_hat[g * m:(g + 1) * m]
            quip_incoherence_inverse(self.tf, rows, rows, self.ws, st)
        return LayerResult(self.codes, self.lo, self.scale, self.W_hat)


def quantize_layer(W: torch.Tensor, X: torch.Tensor, m_side, n_side, bits: int, block: int,
                   damp: float = 0.01, seed: int = 0, method: str = "ldlq", passes: int = 1) -> LayerResult:
    """Quantise one layer from host (or device) tensors; results come back to the host."""
    q = LayerQuantizer(W.shape[0], W.shape[1], m_side, n_side, bits, block, damp, seed,
                       method=method, passes=passes)
    Wd = W.to("cuda", non_blocking=True)
    Xd = X.to("cuda", non_blocking=True)
    r = q.run(Wd, Xd)
    st = quip_sync_status()
    if st != L.QUIP_OK:
        raise QuipError(st, "quantize_layer")
    return LayerResult(r.codes.cpu(), r.lo.cpu(), r.scale.cpu(), r.W_hat.cpu())
