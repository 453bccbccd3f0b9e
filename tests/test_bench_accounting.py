"""Host-side bookkeeping of bench.py (no GPU): the algorithmic FLOPs and bytes, the tensor
peak of each path's MMA kind, the launch count and the profile-traffic lookup."""
import torch

import bench
import workloads as W


def _acc(cfg):
    inp = W.gen_inputs(cfg)
    g = torch.Generator().manual_seed(1)
    ids = torch.stack([torch.randperm(cfg.E, generator=g)[:cfg.topk] for _ in range(cfg.T)])
    nonempty, max_seg = bench.segment_stats(cfg, ids, inp.replica_src)
    return inp, bench.accounting(cfg, inp, nonempty, max_seg), nonempty


def test_flops_and_bytes_follow_the_definitions():
    cfg = W.MoEConfig("acc", T=40, H=256, I=384, E=8, topk=2)
    inp, a, nonempty = _acc(cfg)
    NvS = cfg.T * cfg.topk
    assert a["fc1_flops"] == 4.0 * NvS * cfg.H * cfg.I
    assert a["layer_flops"] == 6.0 * NvS * cfg.H * cfg.I
    wrow = cfg.I * cfg.H * 2                                   # one bf16 gate (or up) matrix
    assert a["fc1_bytes"] == nonempty * 2 * wrow + NvS * cfg.H * 2 + NvS * cfg.I * 2
    assert a["layer_bytes"] == nonempty * 3 * wrow + cfg.T * cfg.H * 4 + cfg.T * cfg.E * 4


def test_activation_operand_bytes_per_path():
    base = dict(T=8, H=256, I=256, E=4, topk=2)
    NvS = 16
    per_value = {}
    for name, kw in {"bf16": {}, "nvfp4": dict(wfmt="nvfp4", act_quant=1), "mx_hilo": dict(wfmt="mxfp4"),
                     "w4a8": dict(wfmt="mxfp4", act_quant=2)}.items():
        cfg = W.MoEConfig(name, **base, **kw)
        inp, a, nonempty = _acc(cfg)
        wbytes = nonempty * (bench.weight_bytes_per_row(inp.w_gate) + bench.weight_bytes_per_row(inp.w_up))
        # h leaves bf16 (BF16), fp32 (NVFP4, quantised by a row pass) or as the down GEMM's
        # records (MXFP4: the same bytes per value as the operand)
        act_out = {"bf16": 2, "nvfp4": 4, "mx_hilo": 2 + 1 / 32, "w4a8": 1 + 1 / 32}[name]
        per_value[name] = (a["fc1_bytes"] - wbytes - NvS * cfg.I * act_out) / (NvS * cfg.H)
    assert per_value == {"bf16": 2.0, "nvfp4": 9 / 16, "mx_hilo": 2 + 1 / 32, "w4a8": 1 + 1 / 32}


def test_tensor_peak_of_each_mma_kind():
    assert bench.tensor_peak_ratio(W.CONFIGS["mixtral_prefill"])[0] == 1.0
    assert bench.tensor_peak_ratio(W.CONFIGS["nvfp4"])[0] == 4.0          # kind::mxf4nvf4
    assert bench.tensor_peak_ratio(W.CONFIGS["mxfp4_w4a8_prefill"])[0] == 2.0   # kind::mxf8f6f4, fp8 rate
    assert bench.tensor_peak_ratio(W.CONFIGS["mxfp4_prefill"])[0] == 1.0  # two fp8 products per MAC


def test_tensor_peak_regime_follows_the_clock_record(tmp_path, monkeypatch):
    # sustained (power-capped) bf16 peak only when the timed region saw the power cap
    assert bench.tensor_peak_key({"reasons": ["sw_power_cap"]})[0] == "bf16_tflops_sustained"
    assert bench.tensor_peak_key({"reasons": []})[0] == "bf16_tflops"
    assert bench.tensor_peak_key({"error": "nvml unavailable"})[0] == "bf16_tflops"
    # a measured file without the sustained figure keeps its other numbers
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 7000.0, "bf16_tflops": 1700.0}')
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert peaks["hbm_gbs"] == 7000.0 and peaks["bf16_tflops"] == 1700.0
    assert peaks["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]
    assert src.startswith("measured") and "bf16_tflops_sustained" in src


def test_roofline_records_on_both_bounds():
    # the record the bench prints for the dominant kernel, built without a GPU
    for name, clocks, bound in (("deepseek_prefill", {"reasons": ["sw_power_cap"]}, "tensor"),
                                ("nvfp4", {"reasons": []}, "hbm")):
        cfg = W.CONFIGS[name]
        acc = {"fc1_flops": 4.0e12, "fc1_bytes": 5.0e9, "layer_flops": 6.0e12, "layer_bytes": 8.0e9}
        if bound == "hbm":
            acc = {"fc1_flops": 4.0e11, "fc1_bytes": 5.0e9, "layer_flops": 6.0e11, "layer_bytes": 8.0e9}
        roof, t_roof = bench.roofline_records(cfg, acc, 2.0, clocks, None)
        assert roof["bound"] == bound and roof["frac"] == roof["achieved"] / roof["peak"]
        assert "sustained" in roof["peak_source"] if clocks["reasons"] else "burst" in roof["peak_source"]
        assert t_roof > 0 and set(roof) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}


def test_launch_counts_and_dtype():
    assert bench.kernel_launches(W.CONFIGS["mixtral_prefill"]) == 8
    assert bench.kernel_launches(W.CONFIGS["nvfp4"]) == 9
    assert bench.kernel_launches(W.CONFIGS["mxfp4_decode"]) == 5
    assert bench.compute_dtype(W.CONFIGS["mixtral_prefill"]) == "bf16"
    assert bench.compute_dtype(W.CONFIGS["nvfp4"]).startswith("nvfp4")


def test_profile_traffic_only_for_the_current_source():
    # the committed summaries carry the hash of the GEMM sources they were taken on
    v = bench.profiled_traffic("mixtral_prefill")
    assert v is None or v > 0
    assert bench.profiled_traffic("no_such_workload") is None


def test_bias_and_swigluoai_accounting():
    # SWIGLUOAI and the biases run in the GEMM epilogues: the bias rows of the non-empty
    # experts are read there, the launches are those of the plain layer
    cfg = W.MoEConfig("fused", T=40, H=256, I=384, E=8, topk=2, act="swigluoai", bias=True)
    inp, a, nonempty = _acc(cfg)
    NvS = cfg.T * cfg.topk
    wrow = cfg.I * cfg.H * 2
    assert a["fc1_flops"] == 4.0 * NvS * cfg.H * cfg.I
    assert a["fc1_bytes"] == (nonempty * 2 * wrow + NvS * cfg.H * 2 + NvS * cfg.I * 2 + nonempty * 2 * cfg.I * 4)
    assert a["fc2_bytes"] == nonempty * wrow + NvS * cfg.I * 2 + NvS * cfg.H * 4 + nonempty * cfg.H * 4
    assert a["layer_bytes"] == (nonempty * 3 * wrow + nonempty * (2 * cfg.I + cfg.H) * 4
                                + cfg.T * cfg.H * 4 + cfg.T * cfg.E * 4)
    # (T <= 256: routing and permutation are one kernel)
    assert bench.kernel_launches(cfg) == 5
    assert bench.kernel_launches(cfg.with_(bias=False)) == 5
    assert bench.kernel_launches(cfg.with_(T=300)) == 8
    assert bench.kernel_launches(W.CONFIGS["mxfp4_swiglu_bias_decode"]) == 5
    assert bench.kernel_launches(W.CONFIGS["deepseek_decode_grouped"]) == 6
    # NVFP4 weights, bf16 activations, SITU: the epilogue stores f16 directly, with or without
    # biases (SITU bounds h either way)
    nv = W.MoEConfig("nv", T=8, H=256, I=256, E=4, topk=2, act="situ", wfmt="nvfp4")
    assert bench.kernel_launches(nv) == 5
    assert bench.kernel_launches(nv.with_(bias=True)) == 5
    assert bench.act_config(W.CONFIGS["mxfp4_swiglu_bias_decode"]) == dict(
        swiglu_alpha=1.702, swiglu_beta=1.0, swiglu_limit=7.0, gemm_biases=True)
    assert bench.act_config(W.CONFIGS["mixtral_prefill"]) == {}
