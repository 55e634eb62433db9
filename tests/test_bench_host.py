"""Host logic of bench.py: the ncu traffic record the roofline line reads."""

import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture()
def bench(tmp_path, monkeypatch):
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    monkeypatch.setattr(mod, "TRAFFIC_FILE", str(tmp_path / "traffic.json"))
    return mod


def _csv(path, launches):
    """An `ncu --csv` metrics log: one row per (launch, metric)."""
    hdr = '"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n'
    rows = []
    for i, (name, rd, wr, ns) in enumerate(launches):
        rows.append(f'"{i}","{name}","dram__bytes_read.sum","byte","{rd}"\n')
        rows.append(f'"{i}","{name}","dram__bytes_write.sum","byte","{wr}"\n')
        rows.append(f'"{i}","{name}","gpu__time_duration.sum","nsecond","{ns}"\n')
    path.write_text("==PROF== noise line\n" + hdr + "".join(rows))


def test_traffic_is_recorded_per_workload_and_routing(bench, tmp_path):
    gu = "void gemm_tc_kernel<64, 6, 2, 2, PersistentGroupedSched<1>, EpiSwiGLU<64>>(...)"
    other = "void gemm_tc_kernel<64, 6, 1, 2, DenseSched, EpiResidualT<64>>(...)"
    a = tmp_path / "a.csv"
    _csv(a, [(gu, "100", "10", "5000"), (other, "999", "999", "1"), (gu, "300", "30", "7000")])
    bench.ingest_ncu(str(a), "w", "model", "bf16", "cmd a")
    b = tmp_path / "b.csv"
    _csv(b, [(gu, "1000", "0", "9000")])
    bench.ingest_ncu(str(b), "w", "uniform", "bf16", "cmd b")
    assert bench.recorded_traffic("w", "model", "bf16") == pytest.approx((110 + 330) / 2)
    assert bench.recorded_traffic("w", "uniform", "bf16") == pytest.approx(1000)
    assert bench.recorded_traffic("other", "model", "bf16") is None
    assert bench.recorded_traffic("w", "model", "fp8") is None   # another weight format
    rec = json.load(open(bench.TRAFFIC_FILE))
    assert rec["w|model|bf16"]["launches"] == 2 and rec["w|model|bf16"]["command"] == "cmd a"


def test_traffic_is_dropped_once_the_kernel_sources_change(bench, tmp_path, monkeypatch):
    gu = "gemm_tc_kernel<...EpiSwiGLU<128>>"
    a = tmp_path / "a.csv"
    _csv(a, [(gu, "5", "5", "1")])
    bench.ingest_ncu(str(a), "w", "model", "bf16", "")
    assert bench.recorded_traffic("w", "model", "bf16") == pytest.approx(10)
    monkeypatch.setattr(bench, "sources_sha256", lambda: "changed")
    assert bench.recorded_traffic("w", "model", "bf16") is None


def test_a_capture_without_the_gate_up_kernel_is_refused(bench, tmp_path):
    a = tmp_path / "a.csv"
    _csv(a, [("attn_tc_kernel<176>", "1", "1", "1")])
    with pytest.raises(SystemExit):
        bench.ingest_ncu(str(a), "w", "model", "bf16", "")


def test_design_point_routing_gives_every_expert_the_same_load(bench):
    from synth import WORKLOADS
    cfg = WORKLOADS["c3-moe26b-canvas"].model
    T = cfg.canvas
    idx = bench.uniform_routing(cfg, T)
    assert idx.shape == (cfg.n_layers, T, cfg.top_k)
    import numpy as np
    for l in (0, cfg.n_layers - 1):
        counts = np.bincount(idx[l].ravel(), minlength=cfg.n_experts)
        assert np.all(counts == T * cfg.top_k // cfg.n_experts)          # 16 each at one canvas
        assert all(len(set(row)) == cfg.top_k for row in idx[l].tolist())  # k distinct experts per token


def test_gate_up_bytes_and_pass_flops_follow_the_shapes(bench):
    from synth import WORKLOADS
    cfg = WORKLOADS["c3-moe26b-canvas"].model
    T, d, F, k = cfg.canvas, cfg.d_model, cfg.ffn_dim, cfg.top_k
    # all experts: 128 x (gate + up) x F x d bf16 + the gathered rows in + the SwiGLU rows out
    assert bench.gate_up_bytes(cfg, T) == cfg.n_experts * 2 * F * d * 2 + T * k * d * 2 + T * k * F * 2
    assert bench.gate_up_bytes(cfg, T, routed=14) - bench.gate_up_bytes(cfg, T, routed=13) == 2 * F * d * 2
    # one canvas pass with no LM-head rows: per layer QKV + O + experts + router + attention
    P = 4096
    per_layer = (2 * T * d * (cfg.q_dim + 2 * cfg.kv_dim) + 2 * T * cfg.q_dim * d + 2 * T * k * 3 * F * d
                 + 2 * T * d * cfg.n_experts + 4 * T * (P + T) * cfg.n_heads * cfg.head_dim)
    assert bench.pass_flops(cfg, T, P, 0) == cfg.n_layers * per_layer
    assert bench.pass_flops(cfg, T, P, T) - bench.pass_flops(cfg, T, P, 0) == 2 * T * d * cfg.vocab
