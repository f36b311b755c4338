"""bench.py's host-side arithmetic (no GPU): the algorithmic work models
and the pipeline speed-of-light fraction."""
import importlib.util
import os

import pytest

from conftest import ROOT
from quip_synth import CONFIGS


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


PK = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1300.0, "source": "test"}


def test_pipeline_floor_attn7b(bench):
    cfg = CONFIGS["attn7b"]
    f = bench.pipeline_floor(cfg, PK)
    m, n, N = cfg.m, cfg.n, cfg.N
    assert f["hessian"] == pytest.approx(N * n * (n + 1) / 1500e12 * 1e3)
    assert f["ldl"] == pytest.approx(n ** 3 / 3 / (1500e12 / 6) * 1e3)
    assert f["ldlq"] == pytest.approx(m * n * n / (1500e12 / 6) * 1e3)
    assert f["dequant"] == pytest.approx((5.0 * m * n + 8.0 * m) / 6000e9 * 1e3)
    e = bench.pipeline_entry(cfg, PK, 3.0)
    assert e["floor_ms"] == pytest.approx(sum(f.values()), abs=1e-4)
    assert e["frac"] == pytest.approx(e["floor_ms"] / 3.0, abs=1e-4)
    assert 0.0 < e["frac"] < 1.0


def test_pipeline_floor_fp32_hessian_uses_ffma_peak(bench):
    cfg = CONFIGS["tiny"]
    f = bench.pipeline_floor(cfg, PK)
    assert f["hessian"] == pytest.approx(cfg.N * cfg.n * (cfg.n + 1) / (bench.FFMA_TFLOPS * 1e12) * 1e3)


@pytest.mark.parametrize("method,passes", [("ldlq", 1), ("nearest", 1), ("greedy", 2), ("ldlq_rg", 1)])
def test_kernel_work_by_method(bench, method, passes):
    cfg = CONFIGS["attn7b"]
    kw = bench.kernel_work(cfg, method, passes)
    m, n = cfg.m, cfg.n
    has_ldl = method in ("ldlq", "ldlq_rg")
    assert ("k_ldl_factor" in kw) == has_ldl
    runs = (1 if has_ldl else 0) + (passes if method in ("greedy", "ldlq_rg") else 0)
    if runs:
        assert kw["k_ldlq_block"][1] == pytest.approx(runs * m * n * 127)   # 32 blocks x 128 x 127 per row
    else:
        assert "k_ldlq_block" not in kw
    if method in ("greedy", "ldlq_rg"):
        assert kw["k_gemm_split_tc[greedy]"][1] == pytest.approx(passes * 2.0 * m * n * n)
    assert ("k_nearest" in kw) == (method in ("nearest", "greedy"))
