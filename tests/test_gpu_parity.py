"""CUDA path (through the C ABI) against the CPU oracle, stage by stage.

Each stage is fed the GPU's own outputs of the previous stage, so a mismatch
points at one kernel: s -> (Wq, w_scale) -> (Xq, x_scale) -> acc -> Y.  The
end-to-end test then runs the pure oracle from the same seeded bf16 inputs.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from oracle import smoothquant as O
from tests.helpers import (assert_codes, assert_scales_close, assert_y_close, dev, dev_bf16, host,
                           host_bf16_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import w8a8_smoothquant_int8_sq_b200 as m
    return m


def _stages(sq, C, W, X, bias, alpha, label, report):
    """Run every stage on the GPU and compare with the oracle; returns GPU tensors."""
    K = W.shape[1]
    Cd, Wd, Xd = dev_bf16(C), dev_bf16(W), dev_bf16(X)
    bd = dev_bf16(bias) if bias is not None else None
    # a1 calibration (running max starts from zeros, as the page's buffer does)
    mx = torch.zeros(K, dtype=torch.float32, device="cuda")
    s_g = sq.sq_calibrate(Cd, Wd, alpha, mx_inout=mx)
    s_o, mx_o = O.calibrate(C, W, alpha)
    s_h = host(s_g)
    assert np.array_equal(host(mx), mx_o), f"{label}: running max differs"
    report["s_ulp"] = assert_scales_close(s_h, s_o, f"{label}: s")
    # a2 fold + weight quantisation, from the GPU's s
    Wq_g, ws_g = sq.sq_prepare_weight(Wd, s_g)
    Wq_o, ws_o = O.fold_and_quantize_weight(W, s_h)
    _, _, vw = O.fold_and_quantize_weight_f64(W, s_h)
    report["w_scale_ulp"] = assert_scales_close(host(ws_g), ws_o, f"{label}: w_scale")
    report["w_code_ties"] = assert_codes(host(Wq_g), Wq_o, vw, f"{label}: Wq")
    # a3 activation quantisation
    Xq_g, xs_g = sq.sq_quantize_act(Xd, s_g)
    Xq_o, xs_o = O.quantize_activation(X, s_h)
    _, _, vx = O.quantize_activation_f64(X, s_h)
    report["x_scale_ulp"] = assert_scales_close(host(xs_g), xs_o, f"{label}: x_scale")
    report["x_code_ties"] = assert_codes(host(Xq_g), Xq_o, vx, f"{label}: Xq")
    # a4 int8 GEMM, raw accumulator
    acc_g = host(sq.sq_gemm_s32(Xq_g, Wq_g))
    acc_o = O.int8_gemm(host(Xq_g), host(Wq_g))
    assert np.array_equal(acc_g.astype(np.int64), acc_o), f"{label}: int32 accumulators differ"
    # a5 dequant epilogue
    Y_g = sq.sq_linear(Xq_g, xs_g, Wq_g, ws_g, bd)
    report["y_tol_ratio"] = assert_y_close(host_bf16_bits(Y_g), acc_o, host(xs_g), host(ws_g), bias, f"{label}: Y")
    # fused forward = the two kernels above, bit for bit
    Y_f = sq.sq_forward(Xd, s_g, Wq_g, ws_g, bd)
    assert torch.equal(Y_f.view(torch.int16), Y_g.view(torch.int16)), f"{label}: sq_forward != sq_linear(quantize_act)"
    # quantisation inside the GEMM: the same codes, so the same Y bit for bit,
    # and the pre-pass's x_scale (workspace offset 0) equal to sq_quantize_act's
    M = X.shape[0]
    wsp = torch.full((sq.sq_forward_prologue_workspace_bytes(M, K),), 0x7F, dtype=torch.uint8, device="cuda")
    Y_p = sq.sq_forward_prologue(Xd, s_g, Wq_g, ws_g, bd, workspace=wsp)
    assert torch.equal(Y_p.view(torch.int16), Y_g.view(torch.int16)), \
        f"{label}: sq_forward_prologue != sq_linear(quantize_act)"
    assert torch.equal(wsp[:4 * M].view(torch.float32), xs_g), f"{label}: pre-pass x_scale != sq_quantize_act's"
    torch.cuda.synchronize()
    return dict(s=s_g, Wq=Wq_g, ws=ws_g, Xq=Xq_g, xs=xs_g, Y=Y_g, Yf=Y_f)


@pytest.mark.parametrize("name", ["tiny", "proj", "mlp", "decode"])
def test_workload_stage_parity(sq, name):
    wl = workloads.get(name)
    inp = workloads.make_inputs(wl)
    report = {}
    g = _stages(sq, inp["C"], inp["W"], inp["X"], inp["bias"], wl.alpha_f32, name, report)
    # end to end: every element of the fused forward's Y against the pure
    # oracle run from the same bf16 inputs.  When the GPU's s is within the
    # allowed 2 ulp but not equal, the oracle continues from the GPU's s (the
    # only value the two sides may then share) and the test says so.
    s_o, _ = O.calibrate(inp["C"], inp["W"], wl.alpha_f32)
    s_from = s_o
    if not np.array_equal(host(g["s"]), s_o):
        s_from = host(g["s"])
        print(f"\n[parity] {name}: s differs from the oracle's within tolerance; "
              f"end-to-end oracle continued from the GPU's s")
    Wq_o, ws_o = O.fold_and_quantize_weight(inp["W"], s_from)
    Y_o, Xq_o, xs_o, acc_o = O.forward(inp["X"], s_from, Wq_o, ws_o, inp["bias"])
    report["end_to_end_y_tol_ratio"] = assert_y_close(host_bf16_bits(g["Yf"]), acc_o, xs_o, ws_o, inp["bias"],
                                                      f"{name}: end-to-end Y")
    yfp = O.reference_linear_f64(inp["X"], inp["W"], inp["bias"])
    report["rel_err_vs_fp"] = O.quantization_error(yfp, O.widen_bf16(host_bf16_bits(g["Yf"])).astype(np.float64))
    print(f"\n[parity] {name}: {report}")
    assert report["rel_err_vs_fp"] < 0.05


@pytest.mark.parametrize("M,N,K,with_bias", [
    (1, 256, 256, True),        # single token
    (100, 200, 48, False),      # K below one 128-byte stage, ragged M and N
    (130, 36, 16, True),        # K = 16 (smallest), N not a multiple of 8 (scalar stores)
    (257, 520, 4112, True),     # ragged K block (4112 = 32*128 + 16), M just past two tiles
    (3, 8, 4096, False),        # tiny N
    (384, 768, 1024, True),     # several full tiles in both dimensions
    (129, 4104, 512, False),    # N just past a 256-wide tile boundary
    (17, 520, 4112, True),      # few tokens, 32-wide token tile, one split-K rank with no k-blocks
    (32, 4104, 1024, False),    # largest few-token case, ragged last weight block
    (8, 4096, 4096, True),      # few tokens, four-way split-K cluster
    (33, 256, 512, True),       # just above the few-token path
    (40, 96, 16384, False),     # largest K: eight warps per row in the row quantisers
    (3, 64, 16384, True),       # largest K on the few-token path
    (2056, 8200, 4112, True),   # 256 x 256 tiles on CTA pairs: ragged M, N and K blocks
    (200, 19004, 1024, False),  # CTA pairs with one m-block (the odd CTA's rows partly past M), scalar stores
])
def test_ragged_shapes(sq, M, N, K, with_bias):
    rng = np.random.default_rng(M * 7919 + N * 31 + K)
    oc = rng.choice(K, size=max(1, K // 100), replace=False)
    X = workloads.random_bf16((M, K), seed=M + 1, outlier_cols=oc, outlier_scale=50.0)
    C = workloads.random_bf16((64, K), seed=M + 2, outlier_cols=oc, outlier_scale=50.0)
    W = workloads.random_bf16((N, K), seed=M + 3, scale=0.02)
    b = workloads.random_bf16((N,), seed=M + 4, scale=0.01) if with_bias else None
    report = {}
    _stages(sq, C, W, X, b, np.float32(0.5).item(), f"{M}x{N}x{K}", report)
    print(f"\n[parity] {M}x{N}x{K}: {report}")


def test_zero_rows_and_floor(sq):
    K, M, N = 64, 4, 32
    X = workloads.random_bf16((M, K), seed=5)
    X[1] = 0
    W = workloads.random_bf16((N, K), seed=6, scale=0.02)
    W[3] = 0
    s = dev(np.ones(K, np.float32))
    Xq, xs = sq.sq_quantize_act(dev_bf16(X), s)
    Wq, ws = sq.sq_prepare_weight(dev_bf16(W), s)
    floor_scale = np.float32(np.float32(1e-8) / np.float32(127))
    assert host(xs)[1] == floor_scale and not host(Xq)[1].any()
    assert host(ws)[3] == floor_scale and not host(Wq)[3].any()
    Xq_o, xs_o = O.quantize_activation(X, np.ones(K, np.float32))
    assert np.array_equal(host(Xq), Xq_o) and np.array_equal(host(xs), xs_o)


@pytest.mark.parametrize("K", [256, 4096])  # one and four warps per row in the row quantiser
def test_tiny_values_and_subnormal_quotients(sq, K):
    """Values near the bottom of the fp32 range: X / s and W * s below 2^-126
    (subnormal quotients and products), rows whose maximum sits on the 1e-8
    floor, and rows mixing normal values with subnormal quotients.  The
    correctly rounded division of the quantisers (Markstein's correction of a
    reciprocal product) is exact only in the normal range; there a subnormal
    quotient is below the smallest scale fl(1e-8 / 127) by more than 2^80, so
    its code is 0 whatever its last bit, and a row maximum on the floor is
    1e-8 exactly.  Codes and scales must equal the oracle's."""
    M = 8
    rng = np.random.default_rng(99)
    s = np.ones(K, np.float32)
    s[:64] = np.float32(2.0 ** 40)          # X / s of moderate X lands near 2^-126
    s[64:96] = np.float32(2.0 ** -40)       # W * s of small W lands below 2^-126
    vals = np.exp(rng.uniform(np.log(1e-38), np.log(1e-30), size=(M, K))).astype(np.float32)
    vals *= np.where(rng.random((M, K)) < 0.5, -1.0, 1.0).astype(np.float32)
    X = workloads.f32_to_bf16_bits(vals)                      # every row tiny: scale on the floor
    big = workloads.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    X[2, 64:] = big[2, 64:]                                   # normal values beside subnormal quotients
    # row maximum ~4000 (scale ~31): the codes' division of the subnormal
    # X / s by the scale is subnormal too
    X[3, 64:] = workloads.f32_to_bf16_bits(workloads.bf16_bits_to_f32(big[3, 64:]) * np.float32(1000))
    X[4, :64] = workloads.f32_to_bf16_bits(np.full(64, 1e-26, np.float32))   # quotients ~ 9e-39
    X[5, 100] = workloads.f32_to_bf16_bits(np.array([2e-8], np.float32))[0]  # maximum just above the floor
    X[6, :] = 0
    W = workloads.f32_to_bf16_bits(
        np.exp(rng.uniform(np.log(1e-38), np.log(1e-2), size=(M, K))).astype(np.float32))
    sd = dev(s)
    Xq, xs = sq.sq_quantize_act(dev_bf16(X), sd)
    Wq, ws = sq.sq_prepare_weight(dev_bf16(W), sd)
    torch.cuda.synchronize()
    Xq_o, xs_o = O.quantize_activation(X, s)
    Wq_o, ws_o = O.fold_and_quantize_weight(W, s)
    _, _, vx = O.quantize_activation_f64(X, s)
    _, _, vw = O.fold_and_quantize_weight_f64(W, s)
    assert_scales_close(host(xs), xs_o, "tiny X: x_scale", max_ulp=0)
    assert_scales_close(host(ws), ws_o, "tiny W: w_scale", max_ulp=0)
    assert_codes(host(Xq), Xq_o, vx, "tiny X: codes")
    assert_codes(host(Wq), Wq_o, vw, "tiny W: codes")
    floor_scale = np.float32(np.float32(1e-8) / np.float32(127))
    assert host(xs)[0] == floor_scale and host(xs)[6] == floor_scale
    # the GEMM that quantises X itself makes the same codes in this range:
    # its Y equals sq_linear on the row quantiser's codes, bit for bit
    Y_l = sq.sq_linear(Xq, xs, Wq, ws)
    Y_p = sq.sq_forward_prologue(dev_bf16(X), sd, Wq, ws)
    assert torch.equal(Y_p.view(torch.int16), Y_l.view(torch.int16))


def test_accumulator_extremes(sq):
    K = 8192
    Xq = np.full((3, K), 127, np.int8)
    Xq[1] = -127
    Xq[2, ::2] = -127
    Wq = np.full((5, K), 127, np.int8)
    acc = host(sq.sq_gemm_s32(dev(Xq), dev(Wq)))
    assert acc[0, 0] == 132128768 and acc[1, 0] == -132128768 and acc[2, 0] == 0
    assert np.array_equal(acc.astype(np.int64), O.int8_gemm(Xq, Wq))


def test_running_max_two_batches(sq):
    wl = workloads.get("tiny")
    inp = workloads.make_inputs(wl, ("C", "W"))
    C, W = inp["C"], inp["W"]
    mx = torch.zeros(wl.K, dtype=torch.float32, device="cuda")
    sq.sq_calibrate(dev_bf16(C[:20]), dev_bf16(W), wl.alpha_f32, mx_inout=mx)
    s2 = sq.sq_calibrate(dev_bf16(C[20:]), dev_bf16(W), wl.alpha_f32, mx_inout=mx)
    s_one = sq.sq_calibrate(dev_bf16(C), dev_bf16(W), wl.alpha_f32)
    assert torch.equal(s2, s_one)
    # R == 0: s from the running max alone
    s3 = sq.sq_calibrate(None, dev_bf16(W), wl.alpha_f32, mx_inout=mx)
    assert torch.equal(s3, s_one)


def test_recompute_after_alpha_change(sq):
    """SmoothQuantW8A8.recompute_smooth_scale: after freezing, a new alpha
    gives a new s from the stored running activation max and the weight's
    column max alone (no calibration rows: R == 0), and W is folded and
    quantised again with it -- the calibration and weight-prep kernels reused."""
    wl = workloads.get("proj")
    inp = workloads.make_inputs(wl, ("C", "W"))
    C, W = inp["C"], inp["W"]
    Cd, Wd = dev_bf16(C), dev_bf16(W)
    mx = torch.zeros(wl.K, dtype=torch.float32, device="cuda")
    sq.sq_calibrate(Cd[:200], Wd, 0.5, mx_inout=mx)   # two calibration batches,
    sq.sq_calibrate(Cd[200:], Wd, 0.5, mx_inout=mx)   # then frozen at alpha 0.5
    for alpha in (np.float32(0.35).item(), np.float32(0.8).item()):
        s_g = sq.sq_calibrate(None, Wd, alpha, mx_inout=mx)
        Wq_g, ws_g = sq.sq_prepare_weight(Wd, s_g)
        torch.cuda.synchronize()
        s_o, mx_o = O.calibrate(C[:0], W, alpha, mx_prev=host(mx))
        assert np.array_equal(host(mx), mx_o)
        assert_scales_close(host(s_g), s_o, f"recomputed s at alpha {alpha}")
        Wq_o, ws_o = O.fold_and_quantize_weight(W, host(s_g))
        _, _, vw = O.fold_and_quantize_weight_f64(W, host(s_g))
        assert_scales_close(host(ws_g), ws_o, f"re-quantised w_scale at alpha {alpha}")
        assert_codes(host(Wq_g), Wq_o, vw, f"re-quantised Wq at alpha {alpha}")
        # the same s as calibrating on all rows at once with the new alpha
        assert torch.equal(s_g, sq.sq_calibrate(Cd, Wd, alpha))


def test_calibrate_leaves_workspace_zero(sq):
    """Whatever the workspace holds on entry, a call ends with the words it
    reduced into -- mx[K], mw[K] and one counter per 256 columns -- zeroed (the
    last block of each column stripe clears them)."""
    wl = workloads.get("tiny")
    inp = workloads.make_inputs(wl, ("C", "W"))
    K = wl.K
    ws = torch.full((sq.sq_calibrate_workspace_bytes(K),), 0xA5, dtype=torch.uint8, device="cuda")
    s1 = sq.sq_calibrate(dev_bf16(inp["C"]), dev_bf16(inp["W"]), wl.alpha_f32, workspace=ws)
    torch.cuda.synchronize()
    used = 4 * (2 * K + (K + 255) // 256)
    assert int(ws[:used].count_nonzero()) == 0
    s_o, _ = O.calibrate(inp["C"], inp["W"], wl.alpha_f32)
    assert_scales_close(host(s1), s_o, "tiny: s with a dirty workspace on entry")


def test_alpha_special_cases(sq):
    wl = workloads.get("tiny")
    inp = workloads.make_inputs(wl, ("C", "W"))
    for a in (0.0, 1.0):
        s = host(sq.sq_calibrate(dev_bf16(inp["C"]), dev_bf16(inp["W"]), a))
        s_o, _ = O.calibrate(inp["C"], inp["W"], a)
        assert_scales_close(s, s_o, f"alpha={a}")


def test_status_codes(sq):
    lib = sq.lib
    X = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    s = torch.ones(64, dtype=torch.float32, device="cuda")
    Xq = torch.empty(4, 64, dtype=torch.int8, device="cuda")
    xs = torch.empty(4, dtype=torch.float32, device="cuda")
    p = lambda t, off=0: ctypes.c_void_p(t.data_ptr() + off)  # noqa: E731
    assert lib.sq_quantize_act(p(X, 2), 4, 64, p(s), p(Xq), p(xs), None) == 3      # misaligned
    assert lib.sq_quantize_act(p(X), 4, 40, p(s), p(Xq), p(xs), None) == 3         # K % 16
    assert lib.sq_quantize_act(p(X), 0, 64, p(s), p(Xq), p(xs), None) == 2         # M = 0
    assert lib.sq_quantize_act(None, 4, 64, p(s), p(Xq), p(xs), None) == 1
    W = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    assert lib.sq_calibrate(p(X), 4, 64, p(W), 8, ctypes.c_float(1.5), p(s), None, p(ws), 16, None) == 4
    assert lib.sq_calibrate(p(X), 4, 64, p(W), 8, ctypes.c_float(0.5), p(s), None, p(ws), 16, None) == 8
    Wq = torch.zeros(8, 64, dtype=torch.int8, device="cuda")
    w_scale = torch.ones(8, dtype=torch.float32, device="cuda")
    Y = torch.empty(4, 8, dtype=torch.bfloat16, device="cuda")
    assert lib.sq_forward(p(X), p(s), p(Wq), p(w_scale), None, 4, 8, 64, p(Y), p(ws), 16, None) == 8
    with pytest.raises(ValueError):
        sq.sq_forward(X, s, Wq, w_scale, workspace=ws)
    assert sq.sq_forward_prologue_workspace_bytes(4, 64) == 512
    assert lib.sq_forward_prologue(p(X), p(s), p(Wq), p(w_scale), None, 4, 8, 64, p(Y), p(ws), 16, None) == 8
    big = torch.empty(512, dtype=torch.uint8, device="cuda")
    assert lib.sq_forward_prologue(p(X), p(s, 4), p(Wq), p(w_scale), None, 4, 8, 64, p(Y), p(big), 512, None) == 3
    assert lib.sq_forward_prologue(p(X), p(s), p(Wq), p(w_scale), None, 4, 8, 40, p(Y), p(big), 512, None) == 3


def test_fault_injection(sq):
    X = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    s = torch.ones(64, dtype=torch.float32, device="cuda")
    try:
        sq.sq_debug_fail_after(1)
        sq.sq_quantize_act(X, s)                       # the one allowed launch
        with pytest.raises(sq.SqError) as ei:
            sq.sq_quantize_act(X, s)
        assert ei.value.status == 6 and "injected" in str(ei.value)
    finally:
        sq.sq_debug_fail_after(-1)
    sq.sq_quantize_act(X, s)


def test_device_status_clean(sq):
    assert sq.sq_device_status() == 0


def test_prefill_full_size_sampled(sq):
    """The largest layer (X[8192x8192], W[28672x8192]) on the GPU at full size;
    the oracle checks s over all channels and sampled rows of Wq / Xq and a
    sampled block of Y (each output depends only on its row of Xq and of Wq)."""
    wl = workloads.get("prefill")
    inp = workloads.make_inputs(wl)
    Cd, Wd, Xd = dev_bf16(inp["C"]), dev_bf16(inp["W"]), dev_bf16(inp["X"])
    s_g = sq.sq_calibrate(Cd, Wd, wl.alpha_f32)
    Wq_g, ws_g = sq.sq_prepare_weight(Wd, s_g)
    Y_g = sq.sq_forward(Xd, s_g, Wq_g, ws_g)
    # activation quantisation inside the GEMM: every element equal
    Y_p = sq.sq_forward_prologue(Xd, s_g, Wq_g, ws_g)
    assert torch.equal(Y_p.view(torch.int16), Y_g.view(torch.int16)), "prefill: sq_forward_prologue != sq_forward"
    del Y_p
    torch.cuda.synchronize()
    s_o, _ = O.calibrate(inp["C"], inp["W"], wl.alpha_f32)
    assert_scales_close(host(s_g), s_o, "prefill: s")
    rng = np.random.default_rng(4242)
    rows_w = np.sort(rng.choice(wl.N, 96, replace=False))
    rows_x = np.sort(np.concatenate([[0, wl.M - 1], rng.choice(wl.M, 62, replace=False)]))
    s_h = host(s_g)
    Wq_o, ws_o = O.fold_and_quantize_weight(inp["W"][rows_w], s_h)
    assert np.array_equal(host(Wq_g[torch.as_tensor(rows_w, device="cuda")]), Wq_o)
    assert np.array_equal(host(ws_g)[rows_w], ws_o)
    Xq_o, xs_o = O.quantize_activation(inp["X"][rows_x], s_h)
    acc_o = O.int8_gemm(Xq_o, Wq_o)
    y_g = host_bf16_bits(Y_g)[np.ix_(rows_x, rows_w)]
    ratio = assert_y_close(y_g, acc_o, xs_o, ws_o, None, "prefill: sampled Y")
    print(f"\n[parity] prefill sampled {len(rows_x)}x{len(rows_w)}: y_tol_ratio {ratio}")
