"""Host logic of bench.py that needs no GPU: the measured-traffic lookup, which
must go stale (None) as soon as the kernel source differs from the one the
ncu summary was captured on, and the algorithmic-work model."""
import hashlib
import os

import bench


def _tree(tmp_path, src_text, recorded_sha, traffic=12345):
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "learned_sparse_feature_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k_sinkhorn.cu").write_text(src_text)
    (tmp_path / "profiles" / "sinkhorn_pair2048.md").write_text(
        f"# summary\n\nsource_sha256: {recorded_sha} (k_sinkhorn.cu)\ntraffic_bytes_per_launch: {traffic}\n")


def test_traffic_is_read_when_the_source_matches(tmp_path, monkeypatch):
    text = "kernel v1"
    _tree(tmp_path, text, hashlib.sha256(text.encode()).hexdigest())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    traffic, src = bench.measured_traffic("sinkhorn", "pair2048")
    assert traffic == 12345
    assert src == os.path.join("profiles", "sinkhorn_pair2048.md")


def test_traffic_goes_stale_when_the_kernel_changes(tmp_path, monkeypatch):
    _tree(tmp_path, "kernel v2", hashlib.sha256(b"kernel v1").hexdigest())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    traffic, _ = bench.measured_traffic("sinkhorn", "pair2048")
    assert traffic is None


def test_traffic_absent_for_other_kernels_and_workloads(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("qkv_gemm", "pair2048") == (None, None)
    assert bench.measured_traffic("sinkhorn", "pair512") == (None, None)


def test_algorithmic_work_matches_the_pages_counts():
    # pair2048: the attention FLOPs of 18 stages and the streamed-byte model of
    # 100 Sinkhorn iterations (two fp32 passes over the augmented matrix each)
    w = bench.algorithmic_work(1, 2048, 2048)
    bound, flops = w["attention"]
    assert bound == "tensor"
    assert abs(flops * 18 - 36 * 256 * 4096 ** 2) / (36 * 256 * 4096 ** 2) < 1e-12
    bound, bytes_ = w["sinkhorn"]
    assert bound == "hbm"
    assert bytes_ == 2 * 100 * 4 * 2049 * 2049


def test_planted_exit_weights_make_the_oracle_exit_after_the_layer():
    # the classifiers bench.py plants for --exit-layer K: the oracle's adaptive
    # GNN stops after layer K (its confidences are 0 before K and 1 at K)
    import numpy as np
    from learned_sparse_feature_b200 import synth
    from oracle import superglue_oracle as O
    w = bench.planted_exit_weights(synth.make_weights(0), 1)
    rng = np.random.default_rng(3)
    xs0 = [rng.standard_normal((5, 256))]
    xs1 = [rng.standard_normal((4, 256))]
    assert O.attentional_gnn_adaptive(xs0, xs1, w, 4, 1e-5, bench.EXIT_DEPTH_CONFIDENCE, 6)[4] == 2
    c = bench._config(synth.WORKLOADS["pair2048"], 1, "sinkhorn", 1)
    assert c["adaptive_depth"]["exit_after_layer"] == 1
    assert "adaptive_depth" not in bench._config(synth.WORKLOADS["pair2048"], 1)


def test_fp32_path_is_bounded_by_the_alu_peak():
    w32 = bench.algorithmic_work(1, 64, 64, precision="fp32")
    w16 = bench.algorithmic_work(1, 64, 64)
    for k in ("qkv_gemm", "attention", "mlp1_gemm", "mlp2_gemm", "proj_gemm", "score_gemm"):
        assert w32[k][0] == "alu" and w16[k][0] == "tensor" and w32[k][1] == w16[k][1]
    # 148 SMs x 128 FP32 lanes x 2 FLOP at 1965 MHz
    assert abs(bench.fp32_alu_peak_tflops(1965.0) - 74.45) < 0.01


def _fake_classes(steps, sinkhorn_ms, gnn_ms):
    per_class = {"encoder": (0.06 * steps, steps), "qkv_gemm": (0.18 * steps, 18 * steps),
                 "attention": (0.41 * steps, 18 * steps), "mlp1_gemm": (0.22 * steps, 18 * steps),
                 "mlp2_gemm": (0.22 * steps, 18 * steps), "proj_gemm": (0.01 * steps, steps),
                 "score_gemm": (0.012 * steps, steps), "sinkhorn": (sinkhorn_ms * steps, steps),
                 "gnn": (0.0, 0)}
    per_seg = {"encoder": (0.06 * steps, steps), "gnn": (gnn_ms * steps, steps),
               "sinkhorn": (sinkhorn_ms * steps, steps)}
    return per_class, per_seg


def test_summarize_bf16_pair2048():
    from learned_sparse_feature_b200 import synth
    w = synth.WORKLOADS["pair2048"]
    per_class, per_seg = _fake_classes(20, 0.70, 0.65)
    roof, breakdown, gnn = bench.summarize(per_class, per_seg, w, 1, 2048, 2048, 20, {"sm_mhz": 1965.0},
                                           measured_traffic_fn=lambda k, n: (None, None))
    assert roof["kernel"] == "sinkhorn" and roof["bound"] == "hbm" and 0.5 < roof["frac"] < 1.0
    assert set(roof["other_bounds_ms"]) == {"mufu_ex2", "compulsory_bytes", "kernel"}
    assert "gnn" not in breakdown and breakdown["attention"]["launches_per_step"] == 18
    assert "frac_tensor" in breakdown["attention"] and "frac_alu" in breakdown["encoder"]
    assert abs(gnn["ms_per_step"] - 0.65) < 1e-12 and 0.1 < gnn["frac_tensor"] < 0.5


def test_summarize_fp32_reports_alu_fractions():
    from learned_sparse_feature_b200 import synth
    w = synth.WORKLOADS["pair64_fp32"]
    per_class, per_seg = _fake_classes(20, 0.34, 2.29)
    per_class["mlp2_gemm"] = (0.92 * 20, 18 * 20)       # the largest class on this path
    roof, breakdown, gnn = bench.summarize(per_class, per_seg, w, 1, 64, 64, 20, {"sm_mhz": None},
                                           measured_traffic_fn=lambda k, n: (None, None))
    assert roof["kernel"] == "mlp2_gemm" and roof["bound"] == "alu"
    assert roof["peak"] == bench.fp32_alu_peak_tflops(1965.0) and roof["peak_source"].startswith("derived")
    assert "frac_alu" in breakdown["mlp1_gemm"] and "frac_tensor" not in breakdown["mlp1_gemm"]
    assert "frac_alu" in gnn and "frac_tensor" not in gnn


def test_summarize_double_softmax_head_class():
    from learned_sparse_feature_b200 import synth
    w = synth.WORKLOADS["pair2048"]
    per_class, per_seg = _fake_classes(20, 0.70, 0.65)
    per_class["dsm_head"] = per_class.pop("sinkhorn")
    per_class["dsm_head"] = (0.115 * 20, 20 * 20)
    roof, breakdown, _ = bench.summarize(per_class, per_seg, w, 1, 2048, 2048, 20, {"sm_mhz": 1965.0},
                                         measured_traffic_fn=lambda k, n: (None, None))
    assert roof["kernel"] == "attention" and roof["bound"] == "tensor"
    assert "frac_hbm" in breakdown["dsm_head"]
