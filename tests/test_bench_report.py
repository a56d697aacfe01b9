"""bench.py's roofline report on CPU, from made-up call times: every workload
gets a bound per call from the two rooflines (decode's GEMM is HBM-bound, the
larger GEMMs tensor-bound), fractions are achieved / peak, the longest call is
the one reported, and long kernels are held to the sustained tensor peak."""
import bench
import workloads

NAMES = ["sq_calibrate", "sq_prepare_weight", "sq_quantize_act", "sq_linear"]
LAUNCHES = {"sq_calibrate": 2, "sq_prepare_weight": 1, "sq_quantize_act": 1, "sq_linear": 1}


def _report(name, ms):
    wl = workloads.get(name)
    per_call = dict(zip(NAMES, ms))
    return wl, bench.kernel_report(wl, NAMES, per_call, per_call, LAUNCHES)


def test_bounds_follow_the_rooflines():
    for name in ("tiny", "proj", "mlp", "prefill", "decode"):
        wl, (kernels, roof) = _report(name, [0.01, 0.012, 0.006, 0.02])
        for n in NAMES[:3]:
            assert kernels[n]["bound"] == "hbm"
        want = "hbm" if name in ("tiny", "decode") else "tensor"
        assert kernels["sq_linear"]["bound"] == want, name
        assert roof["kernel"] == "sq_linear"
        assert roof["bound"] == want


def test_fractions_are_achieved_over_peak():
    hbm, bf16, bf16_sus, _ = bench.peaks()
    wl, (kernels, roof) = _report("proj", [0.010, 0.012, 0.006, 0.0125])
    k = kernels["sq_linear"]
    assert abs(k["achieved_tops"] - 2 * 512 * 4096 * 4096 / 12.5e-6 / 1e12) < 1e-6
    assert abs(roof["frac"] - k["achieved_tops"] / (bf16 * 2)) < 1e-9
    c = kernels["sq_calibrate"]
    assert c["algorithmic_bytes"] == 2 * 512 * 4096 + 2 * 4096 * 4096 + 8 * 4096
    assert abs(c["frac_of_measured_hbm"] - c["algorithmic_bytes"] / 10e-6 / 1e9 / hbm) < 1e-9
    wl, (kernels, roof) = _report("decode", [0.030, 0.040, 0.010, 0.014])
    assert roof["kernel"] == "sq_prepare_weight" and roof["unit"] == "GB/s"
    assert kernels["sq_linear"]["algorithmic_bytes"] == 8 * 8192 + 8192 * 8192 + 2 * 8 * 8192 + 4 * 8 + 4 * 8192


def test_long_kernels_use_the_sustained_peak():
    hbm, bf16, bf16_sus, _ = bench.peaks()
    wl, (kernels, roof) = _report("prefill", [0.08, 0.14, 0.06, 1.5])
    if bf16_sus is not None:
        assert kernels["sq_linear"]["peak"] == "sustained"
        assert abs(roof["peak"] - bf16_sus * 2) < 1e-9
    wl, (kernels, roof) = _report("mlp", [0.02, 0.03, 0.01, 0.08])
    assert kernels["sq_linear"]["peak"] == "burst"


def test_other_paths_take_their_own_peaks():
    """The backward's products are bf16 (the measured bf16 peak, not x2); the
    weight-only product runs on the fp32 CUDA cores (the ALU peak)."""
    hbm, bf16, bf16_sus, _ = bench.peaks()
    wl = workloads.get("mlp")
    names = ["sq_linear", "sq_ste_backward"]
    per = {"sq_linear": 0.08, "sq_ste_backward": 0.30}
    kernels, roof = bench.kernel_report(wl, names, per, per, {"sq_linear": 1, "sq_ste_backward": 7})
    k = kernels["sq_ste_backward"]
    assert k["bound"] == "tensor" and k["operands"] == "bf16"
    assert abs(k["int8_peak_tops"] - bf16) < 1e-9
    assert abs(k["achieved_tops"] - 4 * 2048 * 11008 * 4096 / 300e-6 / 1e12) < 1e-6
    # at proj size the backward's bytes and products take about as long: the
    # bound is whichever roofline is the longer at the peaks in use
    wl = workloads.get("proj")
    kernels, roof = bench.kernel_report(wl, names, {"sq_linear": 0.0125, "sq_ste_backward": 0.1},
                                        {"sq_linear": 0.0125, "sq_ste_backward": 0.1},
                                        {"sq_linear": 1, "sq_ste_backward": 7})
    nb, ops, _ = bench.algorithmic_work(wl)["sq_ste_backward"]
    want = "hbm" if nb / (hbm * 1e9) >= ops / (bf16 * 1e12) else "tensor"
    assert roof["kernel"] == "sq_ste_backward" and roof["bound"] == want
    wl = workloads.get("decode")
    names = ["sq_prepare_weight", "sq_linear_weight_only"]
    per = {"sq_prepare_weight": 0.0115, "sq_linear_weight_only": 0.054}
    kernels, roof = bench.kernel_report(wl, names, per, per, {n: 1 for n in names})
    assert roof["bound"] == "alu" and roof["kernel"] == "sq_linear_weight_only"
    assert abs(roof["peak"] - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9
    assert abs(roof["frac"] - 2 * 8 * 8192 * 8192 / 54e-6 / 1e12 / roof["peak"]) < 1e-9


def test_headline_defaults():
    """With no flags the bench times the largest layer (prefill) on the whole
    path; the decode layer defaults to the per-call forward on prepared,
    rotated weights."""
    a = bench.parse_args([])
    assert a.workload == "prefill" and a.path == "smoothquant" and a.warmup >= 3
    assert bench.parse_args(["--workload", "decode"]).path == "forward"
    assert bench.parse_args(["--workload", "decode", "--path", "smoothquant"]).path == "smoothquant"
    wl = workloads.get("decode")
    r = bench.forward_rotation(wl)
    assert r >= 4 and r * wl.N * wl.K >= 256 << 20


def test_rotation_makes_inputs_exceed_l2():
    assert bench.rotation_count(600 << 20) == 1
    assert bench.rotation_count(128 << 20) == 2
    assert bench.rotation_count(36 << 20) * (36 << 20) >= 256 << 20
    assert bench.rotation_count(1) == bench.MAX_ROTATION


def test_oracle_sample_plan():
    """Smaller layers run whole oracle steps; the prefill layer is sampled
    (and the sample text says how it is extrapolated)."""
    for name in ("tiny", "proj", "mlp", "decode"):
        wl = workloads.get(name)
        assert bench.sample_plan(wl, "smoothquant") == (wl.M, wl.N)
        assert "whole" in bench.oracle_sample_text(wl, "smoothquant")
    wl = workloads.get("prefill")
    mx, mw = bench.sample_plan(wl, "smoothquant")
    assert mx < wl.M and mw < wl.N
    assert "extrapolated" in bench.oracle_sample_text(wl, "smoothquant")


def test_forward_work_counts_the_weight_stream():
    wl = workloads.get("decode")
    nb, ops, typ = bench.algorithmic_work(wl)["sq_forward"]
    assert nb >= wl.N * wl.K and ops == 2 * wl.M * wl.N * wl.K and typ == "int8"
    kernels, roof = bench.kernel_report(wl, ["sq_forward"], {"sq_forward": 0.012}, {"sq_forward": 0.018},
                                        {"sq_forward": 1})
    assert roof["bound"] == "hbm" and roof["kernel"] == "sq_forward"


def test_forward_paths_sample_the_prefill_oracle():
    """The per-call forward paths time the oracle's forward whole on the
    smaller layers and on a sampled block at prefill size; the sampled form
    runs through the same phases (checked on the tiny layer, whole)."""
    wl = workloads.get("prefill")
    for path in ("forward", "forward-prologue"):
        mx, mw = bench.sample_plan(wl, path)
        assert mx < wl.M and mw < wl.N
        assert "extrapolated" in bench.oracle_sample_text(wl, path)
    tiny = workloads.get("tiny")
    assert bench.sample_plan(tiny, "forward-prologue") == (tiny.M, tiny.N)
    inp = bench.oracle_inputs(tiny, "forward-prologue")
    assert inp["Wq"].shape == (tiny.N, tiny.K)
    assert bench.oracle_step_seconds(inp, tiny, "forward-prologue") > 0
    nb, ops, typ = bench.algorithmic_work(wl)["sq_forward_prologue"]
    assert nb == bench.algorithmic_work(wl)["sq_forward"][0] and ops == 2 * wl.M * wl.N * wl.K
