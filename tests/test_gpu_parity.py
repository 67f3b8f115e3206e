"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Bar (from the layer's contract): activation codes and scales bit-exact; Y within relative
Frobenius error 5e-3 and max|dY| <= 1e-2 * max|Y_ref|, where Y_ref is the oracle's fp64
forward over the library's exported operands (codes, scales, L1, L2, 1/lambda, bias).
"""
import numpy as np
import pytest

import synth
from oracle import svdq_oracle as O
from tbound import assert_t_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the marker selects these tests on a GPU machine only
    pytest.skip("needs a CUDA device", allow_module_level=True)

import w4a4_rank_corrected_smooth_b200 as S  # noqa: E402

REL_FRO_TOL = 5e-3
MAX_ABS_TOL = 1e-2


def to_dev_bf16(x_bits: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16).cuda()


def y_to_f64(Y) -> np.ndarray:
    return O.bf16_to_f32(Y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


def make_layer(spec, precision, rank=None, act_absmax=None, X=None):
    X = synth.activations_bf16(spec) if X is None else X
    W = synth.weight_bf16(spec)
    b = synth.bias_bf16(spec)
    a = synth.act_absmax(X) if act_absmax is None else act_absmax
    lin = S.SVDQLinear(W, b, a, precision, spec.rank if rank is None else rank)
    return X, W, b, lin


def run_quant_down(lin, X):
    M = X.shape[0]
    Xd = to_dev_bf16(X)
    ws = lin.new_workspace(M)
    lin.svdq_quant_down(Xd, M, Xd.stride(0), ws, ws.numel())
    S.svdq_get_device_error()
    return lin.svdq_export_activations(ws, M)


def run_forward(lin, X, ldy_pad=0):
    M = X.shape[0]
    Xd = to_dev_bf16(X)
    ws = lin.new_workspace(M)
    Y = torch.full((M, lin.N + ldy_pad), float("nan"), dtype=torch.bfloat16, device="cuda")
    lin.svdq_linear_forward(Xd, M, Xd.stride(0), Y, Y.stride(0), ws, ws.numel())
    S.svdq_get_device_error()
    return Y


def check_activations(lin, X, prec, ops=None):
    ops = lin.export_weights() if ops is None else ops
    act = run_quant_down(lin, X)
    xh, cx, sx = O.quantize_activations(X, ops["inv_lambda"], prec)
    assert np.array_equal(act["codes_x"], cx), "activation codes differ from the oracle"
    assert np.array_equal(act["scales_x"], sx), "activation scales differ from the oracle"
    if lin.rank:
        T_ref = O.bf16_to_f32(O.lowrank_down(xh, ops["L1"])).astype(np.float64)
        T_gpu = O.bf16_to_f32(act["T"]).astype(np.float64)
        # fp32 tensor-core accumulation vs the exact sum, both rounded to bf16: per-element bound
        assert_t_close(T_gpu, T_ref, O.bf16_to_f32(O.f32_to_bf16(xh)), O.bf16_to_f32(ops["L1"]))
    return act


def check_y(Y_gpu: np.ndarray, Y_ref: np.ndarray):
    assert np.all(np.isfinite(Y_gpu))
    rel = O.rel_fro(Y_gpu, Y_ref)
    mx = np.max(np.abs(Y_gpu - Y_ref))
    assert rel <= REL_FRO_TOL, rel
    assert mx <= MAX_ABS_TOL * np.max(np.abs(Y_ref)), (mx, np.max(np.abs(Y_ref)))
    return rel, mx


def test_device_is_supported():
    S.svdq_check_device(0)


def test_wrong_capability_is_refused_at_load_time(monkeypatch):
    """Load-time validation: a device that is not compute capability 10.0 gets a clear
    SVDQ_ERR_UNSUPPORTED_DEVICE from the prepare (the only way to meet one on a B200 is the
    library's capability override, read on every check)."""
    spec = synth.custom("fake_cc", M=8, K=256, N=128, rank=16, seed=3)
    X = synth.activations_bf16(spec)
    for cc in ("9.0", "8.9", "12.0", "10.3"):
        monkeypatch.setenv("SVDQ_TEST_FAKE_CC", cc)
        with pytest.raises(S.SVDQError) as ei:
            S.svdq_check_device(0)
        assert ei.value.status == 2 and "compute capability" in str(ei.value)
        with pytest.raises(S.SVDQError) as ei:
            S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "nvfp4", 16)
        assert ei.value.status == 2, str(ei.value)
    monkeypatch.setenv("SVDQ_TEST_FAKE_CC", "ten")
    with pytest.raises(S.SVDQError) as ei:
        S.svdq_check_device(0)
    assert ei.value.status == 1
    monkeypatch.delenv("SVDQ_TEST_FAKE_CC")
    S.svdq_check_device(0)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "nvfp4", 16)
    lin.close()


def test_bounded_wait_reports_timeout_and_context_survives():
    S.svdq_get_device_error()  # clear
    S.svdq_selftest_wait_timeout(2000)
    with pytest.raises(S.SVDQError) as ei:
        S.svdq_get_device_error()
    assert ei.value.status == 5  # SVDQ_ERR_TIMEOUT
    S.svdq_get_device_error()  # cleared by the read
    x = torch.ones(1024, device="cuda")
    assert float(x.sum().item()) == 1024.0


@pytest.mark.parametrize("prec", ["nvfp4", "int4"])
def test_quant_down_bitexact_tiny(prec):
    spec = synth.get("tiny_256x512x512_r16")
    X, W, b, lin = make_layer(spec, prec)
    check_activations(lin, X, prec)


def _boundary_rows(K: int, prec: str, rng) -> np.ndarray:
    """Rows whose groups put x/scale exactly on E2M1 ties (NVFP4) or x/s on half-integers (INT4)
    and amax/6 on UE4M3 ties, plus +-1 bf16 ulp neighbours and tiny negatives (sign of zero)."""
    rows = []
    if prec == "nvfp4":
        ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
        for sd_code in (0x08, 0x20, 0x33, 0x40, 0x4D, 0x60, 0x70):
            sd = float(O.ue4m3_value(np.array([sd_code]))[0])
            row = np.zeros(K, np.float64)
            for g in range(K // 16):
                vals = np.array([6.0] + ties + [-t for t in ties] + [-0.01], np.float64)[:16]
                rng.shuffle(vals)
                row[g * 16:(g + 1) * 16] = vals * sd
            rows.append(row)
        # amax / 6 exactly on the midpoint between two UE4M3 values (ties to even)
        for c in (0x10, 0x21, 0x3A, 0x47, 0x58):
            mid = (float(O.ue4m3_value(np.array([c]))[0]) + float(O.ue4m3_value(np.array([c + 1]))[0])) / 2
            row = rng.standard_normal(K) * mid
            for g in range(K // 16):
                blk = row[g * 16:(g + 1) * 16]
                blk[np.argmax(np.abs(blk))] = 6.0 * mid
            rows.append(row)
    else:
        for s in (2.0 ** -8, 0.5, 3.0, 40.0):
            row = np.zeros(K, np.float64)
            for g in range(K // 64):
                vals = rng.integers(-14, 15, 64) / 2.0  # half-integers: rint ties
                vals[0] = 7.0
                row[g * 64:(g + 1) * 64] = vals * s
            rows.append(row)
    X = np.stack(rows)
    b = O.f32_to_bf16(X.astype(np.float32))
    return b


@pytest.mark.parametrize("prec", ["nvfp4", "int4"])
def test_quant_down_codec_boundaries_bitexact(prec):
    rng = np.random.default_rng(11)
    spec = synth.custom("boundary", M=32, K=512, N=256, rank=16)
    Xb = _boundary_rows(spec.K, prec, rng)
    X = np.concatenate([Xb, synth.activations_bf16(spec.with_rows(128))], axis=0)[:128]
    W = synth.weight_bf16(spec)
    # a_k = w_k makes lambda exactly 1, so x_hat = x and the crafted ties survive smoothing
    a = np.max(np.abs(O.bf16_to_f32(W)), axis=0).astype(np.float32)
    _, _, _, lin = make_layer(spec, prec, act_absmax=a, X=X)
    ops = lin.export_weights()
    assert np.all(ops["inv_lambda"] == 1.0)
    check_activations(lin, X, prec, ops)


@pytest.mark.parametrize("prec", ["nvfp4", "int4"])
def test_forward_tiny(prec):
    spec = synth.get("tiny_256x512x512_r16")
    X, W, b, lin = make_layer(spec, prec)
    ops = lin.export_weights()
    Y = y_to_f64(run_forward(lin, X))
    ref = O.linear(X, ops, prec)["Y"]
    check_y(Y, ref)


@pytest.mark.parametrize("prec", ["nvfp4", "int4"])
@pytest.mark.parametrize("M,K,N,r", [(1, 256, 256, 16), (17, 512, 264, 0), (255, 768, 512, 48), (129, 256, 512, 128),
                                     (300, 1024, 768, 64), (128, 512, 1024, 32)])
def test_forward_edge_shapes(M, K, N, r, prec):
    spec = synth.custom(f"edge_{M}_{K}_{N}_{r}", M=M, K=K, N=N, rank=r, seed=M + K + N + r)
    X, W, b, lin = make_layer(spec, prec)
    ops = lin.export_weights()
    check_activations(lin, X, prec, ops)
    Yd = run_forward(lin, X, ldy_pad=8)
    assert torch.isnan(Yd[:, N:].float()).all()  # nothing written past column N
    Y = y_to_f64(Yd[:, :N].contiguous())
    check_y(Y, O.linear(X, ops, prec)["Y"])


@pytest.mark.parametrize("prec", ["nvfp4", "int4"])
def test_forward_padded_x_stride(prec):
    """X as rows of a wider buffer (row stride K + 64 elements, the padding filled with large
    values that must not leak in): Y bit-identical to the forward of the contiguous X."""
    spec = synth.custom("x_stride", M=300, K=512, N=512, rank=32, seed=33)
    X, W, b, lin = make_layer(spec, prec)
    Y_ref = run_forward(lin, X)
    buf = torch.full((spec.M, spec.K + 64), 1000.0, dtype=torch.bfloat16, device="cuda")
    buf[:, :spec.K] = to_dev_bf16(X)
    ws = lin.new_workspace(spec.M)
    Y = torch.full((spec.M, spec.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    lin.svdq_linear_forward(buf, spec.M, buf.stride(0), Y, Y.stride(0), ws, ws.numel())
    S.svdq_get_device_error()
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
    lin.close()


def test_forward_m_zero_is_noop():
    spec = synth.custom("m0", M=16, K=256, N=256, rank=16)
    X, W, b, lin = make_layer(spec, "nvfp4")
    lin.svdq_linear_forward(None, 0, 256, None, 256, None, 0)


def test_forward_deterministic():
    spec = synth.custom("det", M=1000, K=1024, N=1024, rank=32, seed=3)
    X, W, b, lin = make_layer(spec, "nvfp4")
    y1 = run_forward(lin, X)
    y2 = run_forward(lin, X)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("prec", ["nvfp4", "int4"])
def test_forward_flux_qkv_full_size_sampled_rows(prec):
    """4608 x 3072 -> 9216, rank 32, in the launch configuration the benchmark times:
    all codes and scales bit-exact; Y checked on a seeded sample of 192 full rows."""
    spec = synth.get("flux_qkv_4608x3072x9216_r32")
    X, W, b, lin = make_layer(spec, prec)
    ops = lin.export_weights()
    act = check_activations(lin, X, prec, ops)
    Yd = run_forward(lin, X)
    rows = np.sort(np.random.default_rng(5).choice(spec.M, 192, replace=False))
    Y = y_to_f64(Yd[torch.from_numpy(rows).cuda()])
    xh, cx, sx = O.quantize_activations(X[rows], ops["inv_lambda"], prec)
    T = O.lowrank_down(xh, ops["L1"])
    ref = O.forward(cx, sx, T, ops["codes_w"], ops["scales_w"], ops["L2"], ops["bias"], prec)
    check_y(Y, ref)
    assert act["codes_x"].shape == (spec.M, spec.K // 2)
