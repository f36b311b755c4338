"""GPU parity of the quantized layer's product with full-precision vectors
(QuIP, Experiments, "Throughput Comparison."; the incoherence-processing
section's post-processing): the packed code layout exactly, and
y = U^T (lo + s codes) V x against the FP64 oracle on seeded inputs."""
import numpy as np
import pytest
import torch

import oracle as O
import post_weight_quantization_09_b200 as Q
from post_weight_quantization_09_b200 import _lib as L
from quip_synth import CONFIGS, Side, make_layer
from parity_util import dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    Q.load()
    Q.quip_sync_status()
    yield
    assert Q.quip_sync_status() == L.QUIP_OK


@pytest.mark.parametrize("bits", range(1, 9))
@pytest.mark.parametrize("m,n", [(1, 5), (3, 37), (17, 129), (64, 4096), (5, 11008)])
def test_pack_codes_matches_oracle(m, n, bits):
    rng = np.random.default_rng(m * n + bits)
    C = rng.integers(0, 2 ** bits, (m, n)).astype(np.uint8)
    packed = Q.quip_pack_codes(dev(C, torch.uint8), bits)
    assert packed.shape == (m, O.packed_words(n, bits))
    np.testing.assert_array_equal(packed.cpu().numpy().view(np.uint32), O.pack_codes(C, bits))


def test_pack_codes_strided_rows():
    C = np.random.default_rng(1).integers(0, 4, (6, 100)).astype(np.uint8)
    Wd = O.packed_words(100, 2)
    buf = torch.full((6, Wd + 8), -1, dtype=torch.int32, device="cuda")
    Q.quip_pack_codes(dev(C, torch.uint8), 2, buf[:, :Wd + 4])
    got = buf.cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(got[:, :Wd], O.pack_codes(C, 2))
    assert np.all(buf[:, Wd:].cpu().numpy() == -1)                   # padding words untouched


def _layer(m, n, bits, seed):
    rng = np.random.default_rng(seed)
    C = rng.integers(0, 2 ** bits, (m, n)).astype(np.uint8)
    lo = (rng.standard_normal(m) * 0.05).astype(np.float32).astype(np.float64)
    s = rng.uniform(0.005, 0.05, m).astype(np.float32).astype(np.float64)
    return C, lo, s


CASES = [
    (64, 128, Side("hadamard"), Side("hadamard"), 2, 1),
    (256, 4096, Side("hadamard"), Side("hadamard"), 2, 3),
    (4096, 512, Side("hadamard"), Side("hadamard"), 4, 8),
    (11008 // 8, 4096, Side("kronecker", 86, 16), Side("hadamard"), 3, 2),
    (512, 11008 // 4, Side("hadamard"), Side("kronecker", 43, 64), 2, 11),
    (128, 256, Side("hadamard", permute=True), Side("kronecker", 16, 16, True), 8, 4),
    (100, 64, Side("identity"), Side("identity"), 1, 5),
    (33, 192, Side("identity", permute=True), Side("identity"), 2, 9),
]


@pytest.mark.parametrize("m,n,mk,nk,bits,B", CASES)
def test_qmatvec_matches_oracle(m, n, mk, nk, bits, B):
    seed = 7 * m + n + bits
    C, lo, s = _layer(m, n, bits, seed)
    rng = np.random.default_rng(seed + 1)
    x = rng.standard_normal((B, n)).astype(np.float32).astype(np.float64)
    tf = Q.Transform(seed, m, n, mk, nk)
    ql = Q.QuantizedLinear(tf, dev(C, torch.uint8), dev(lo), dev(s), bits, max_batch=B)
    y = host(ql(dev(x)))
    U = O.make_side(seed, "m", mk.kind, m, mk.p, mk.q, mk.permute)
    V = O.make_side(seed, "n", nk.kind, n, nk.p, nk.q, nk.permute)
    y_ref = O.quantized_matvec(C, lo, s, U, V, x)
    # fp32 sums of n products and log-depth transforms: error ~ sqrt(n) u
    # times |W~^| |x'|, bounded by ||W~^||_F ||x|| (Cauchy-Schwarz)
    Wf = np.linalg.norm(O.dequantize(C, lo, s))
    for b in range(B):
        assert np.linalg.norm(y[b] - y_ref[b]) <= 2e-5 * Wf * np.linalg.norm(x[b]), b
    tf.close()


def test_qmatvec_exact_on_dyadic_inputs():
    # identity sides, small integer vectors, dyadic grids: every product and
    # partial sum is exact in fp32, so the device result equals the oracle's
    m, n, bits = 70, 1000, 3
    rng = np.random.default_rng(3)
    C = rng.integers(0, 8, (m, n)).astype(np.uint8)
    lo = rng.integers(-8, 8, m) / 4.0
    s = np.full(m, 0.5)
    x = rng.integers(-3, 4, (4, n)).astype(np.float64)
    tf = Q.Transform(0, m, n, Side("identity"), Side("identity"))
    ql = Q.QuantizedLinear(tf, dev(C, torch.uint8), dev(lo), dev(s), bits, max_batch=4)
    I_m, I_n = O.SideTransform("identity", m), O.SideTransform("identity", n)
    np.testing.assert_array_equal(host(ql(dev(x))), O.quantized_matvec(C, lo, s, I_m, I_n, x))


def test_qmatvec_bf16_and_strided_vectors():
    m, n, bits, B = 128, 256, 2, 3
    C, lo, s = _layer(m, n, bits, 5)
    tf = Q.Transform(5, m, n, Side("hadamard"), Side("hadamard"))
    ql = Q.QuantizedLinear(tf, dev(C, torch.uint8), dev(lo), dev(s), bits, max_batch=B)
    xb = torch.randn(B, n + 8, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16).cuda()
    out = torch.full((B, m + 4), 7.0, device="cuda")
    ql(xb[:, :n], out[:, :m])
    x64 = xb[:, :n].float().cpu().double().numpy()
    U = O.make_side(5, "m", "hadamard", m)
    V = O.make_side(5, "n", "hadamard", n)
    y_ref = O.quantized_matvec(C, lo, s, U, V, x64)
    Wf = np.linalg.norm(O.dequantize(C, lo, s))
    for b in range(B):
        assert np.linalg.norm(host(out[b, :m]) - y_ref[b]) <= 2e-5 * Wf * np.linalg.norm(x64[b])
    assert np.all(out[:, m:].cpu().numpy() == 7.0)


def test_quantized_linear_is_the_quantized_layer():
    # the inference product of a layer quantised on the device equals its
    # dequantised weights (the pipeline's W^) times x
    cfg = CONFIGS["tiny"]
    d = make_layer(cfg)
    q = Q.LayerQuantizer(cfg.m, cfg.n, cfg.m_side, cfg.n_side, cfg.bits, cfg.block, cfg.damp, cfg.seed)
    r = q.run(dev(d["W"]), dev(d["X"]))
    ql = Q.QuantizedLinear(q.tf, r.codes, r.lo, r.scale, cfg.bits, max_batch=4)
    x = np.random.default_rng(9).standard_normal((4, cfg.n))
    y = host(ql(dev(x)))
    W_hat = host(r.W_hat)
    np.testing.assert_allclose(y, x.astype(np.float32).astype(np.float64) @ W_hat.T,
                               atol=2e-5 * np.linalg.norm(W_hat) * np.linalg.norm(x, axis=1).max())
