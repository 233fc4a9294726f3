"""Host-side logic of bench.py (no GPU): the roofline numerators, the guard
that drops ncu traffic taken on other kernel sources, and the token-sampled
oracle fit behind the CPU baseline."""
import json

import pytest

import bench


def test_algorithmic_work_of_the_prefill_step():
    T, K, N = 4096, 2560, 6912
    a = bench.algorithmic(T, K, N)
    assert a["fwd_gemm_ops"] == 2 * T * K * N == 144_955_146_240
    assert a["bwd_flops_each"] == a["fwd_gemm_ops"] and a["step_ops"] == 3 * a["fwd_gemm_ops"]
    # read the bf16 masters; write the 2:4 values (half the codes) and 4-bit metadata per group of 4
    assert a["prep_bytes"] == N * K * 2 + N * K // 2 + N * K // 8 == 46_448_640
    # read bf16 x; write int8 codes and one fp32 scale per token
    assert a["actq_bytes"] == T * K * 2 + T * K + T * 4 == 31_473_664
    # dX and dW each read dY, one bf16 operand and write one bf16 result
    assert a["dx_bytes"] == a["dw_bytes"] == 2 * (T * N + N * K + T * K)


def test_ncu_traffic_only_for_the_sources_it_was_taken_on(monkeypatch, tmp_path):
    rec = {"fwd_gemm": {"source_sha": "aaaa", "dram_bytes_per_launch": 123.0}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "aaaa")
    assert bench.ncu_traffic("fwd_gemm") == 123.0
    assert bench.ncu_traffic("prepare") is None
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "bbbb")
    assert bench.ncu_traffic("fwd_gemm") is None


def test_kernel_source_hash_covers_every_kernel_file(monkeypatch, tmp_path):
    csrc = tmp_path / "sparse_linear_layers_bitlinear_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("x")
    (csrc / "b.cuh").write_text("y")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha()
    (csrc / "b.cuh").write_text("z")
    h1 = bench.kernel_source_sha()
    (csrc / "c.h").write_text("")
    h2 = bench.kernel_source_sha()
    assert len({h0, h1, h2}) == 3


@pytest.mark.parametrize("intercept", [0.0, 0.5])
def test_oracle_fit_recovers_a_linear_cost(monkeypatch, intercept):
    """With an oracle whose token part costs intercept + 0.01 s per token
    (and 1 s for the full-batch prepare and act-quant), the fitted full step
    is exact."""
    calls = []

    def fake_sample(wb, xb, dyb, n, m, tokens):
        calls.append(tokens)
        return 1.0, intercept + 0.01 * tokens

    monkeypatch.setattr(bench, "oracle_sample", fake_sample)
    fit = bench.OracleFit(None, None, None, 4096, 2, 4, target_s=10.0)
    assert fit.lo == 8 and 8 < fit.tokens <= 4096
    assert fit.step_s == pytest.approx(1.0 + intercept + 4096 * 0.01)
    assert calls[0] == 8 and calls[-1] == fit.tokens
