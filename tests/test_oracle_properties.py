"""Randomised properties of the oracle's rounding and packing functions
(hypothesis; CPU only).  Each property follows from the definitions in the
QuIP paper's Experiments, "Methods." (the rounding methods) or from the
packed layout's own definition; none of them re-derives the function it
checks."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle as O

SETTINGS = settings(max_examples=25, deadline=None, suppress_health_check=[HealthCheck.too_slow])


def _spd(n, rng):
    X = rng.standard_normal((3 * n, n)) * np.exp(0.5 * rng.standard_normal(n))
    return O.damp(O.hessian(X), 0.01)


@SETTINGS
@given(bits=st.integers(1, 8), m=st.integers(1, 4), n=st.integers(1, 300), seed=st.integers(0, 2 ** 31))
def test_pack_roundtrip_and_width(bits, m, n, seed):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 2 ** bits, (m, n))
    p = O.pack_codes(c, bits)
    assert p.dtype == np.uint32 and p.shape[1] % 4 == 0
    assert (p.shape[1] - 4) * (32 // O.code_slot_bits(bits)) < n      # no spare group of words
    np.testing.assert_array_equal(O.unpack_codes(p, n, bits), c)


@SETTINGS
@given(n=st.integers(1, 40), seed=st.integers(0, 2 ** 31))
def test_diag_order_is_a_sorted_permutation(n, seed):
    rng = np.random.default_rng(seed)
    d = rng.integers(0, 4, n).astype(float)                # many ties
    order = O.diag_order(np.diag(d))
    np.testing.assert_array_equal(np.sort(order), np.arange(n))
    dd = d[order]
    assert np.all(dd[:-1] >= dd[1:])
    ties = dd[:-1] == dd[1:]
    assert np.all(order[:-1][ties] < order[1:][ties])


@SETTINGS
@given(n=st.integers(2, 12), m=st.integers(1, 4), bits=st.integers(1, 4), seed=st.integers(0, 2 ** 31))
def test_greedy_pass_never_raises_any_row_proxy(n, m, bits, seed):
    rng = np.random.default_rng(seed)
    H = _spd(n, rng)
    W = rng.standard_normal((m, n))
    lo, s = O.row_grid(W, bits)
    c0 = rng.integers(0, 2 ** bits, (m, n))
    c1 = O.greedy_pass(W, H, lo, s, bits, c0)
    for i in range(m):
        e0 = lo[i] + s[i] * c0[i] - W[i]
        e1 = lo[i] + s[i] * c1[i] - W[i]
        assert e1 @ H @ e1 <= e0 @ H @ e0 + 1e-12 * max(1.0, e0 @ H @ e0)


@SETTINGS
@given(n=st.integers(2, 16), m=st.integers(1, 5), bits=st.integers(1, 8), seed=st.integers(0, 2 ** 31),
       method=st.sampled_from(["nearest", "ldlq", "greedy", "ldlq_rg"]))
def test_every_method_returns_codes_on_the_grid(n, m, bits, seed, method):
    rng = np.random.default_rng(seed)
    H = _spd(n, rng)
    W = rng.standard_normal((m, n))
    lo, s = O.row_grid(W, bits)
    c = O.quantize_layer(method, W, H, lo, s, bits, passes=1)
    assert c.shape == (m, n) and c.dtype.kind == "i"
    assert np.all((c >= 0) & (c <= 2 ** bits - 1))


@SETTINGS
@given(seed=st.integers(0, 2 ** 31), B=st.integers(1, 3))
def test_quantized_matvec_is_linear(seed, B):
    rng = np.random.default_rng(seed)
    m, n, bits = 8, 16, 2
    c = rng.integers(0, 4, (m, n))
    lo, s = rng.standard_normal(m), rng.uniform(0.1, 1.0, m)
    U = O.make_side(seed % 1000, "m", "hadamard", m)
    V = O.make_side(seed % 1000, "n", "kronecker", n, 4, 4)
    x = rng.standard_normal((B, n))
    a = rng.standard_normal()
    y = O.quantized_matvec(c, lo, s, U, V, x)
    np.testing.assert_allclose(O.quantized_matvec(c, lo, s, U, V, a * x), a * y, rtol=1e-10, atol=1e-12)
    assert np.isclose(np.linalg.norm(y), np.linalg.norm(x @ (O.dequantize(c, lo, s) @ V.matrix()).T),
                      rtol=1e-10)                       # U is orthogonal
