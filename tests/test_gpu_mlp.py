"""GPU parity of the fused MLP pair (up layer -> bf16 -> GELU -> bf16 -> down layer, the hidden
activation kept out of memory) through the C ABI, against the oracle's module sequence over the
library's exported operands of both layers.

Bar: Y within relative Frobenius 5e-3 and max|dY| <= 1e-2 max|Y_ref| of the oracle's pair; the
epilogue's bf16 GELU equal to the oracle's on every one of the 2^16 bf16 inputs; the down layer's
activation codes and scales bit-exact against the oracle's quantizer applied to GELU of the up
layer's own bf16 output (the up layer's output is where the GPU's fp32 accumulation and the
oracle's exact sum may round to neighbouring bf16 values, so both sides take the hidden value
from the same up-layer output); its T within the per-element bound of the fp32 accumulation;
two runs bit-identical.  The GELU-output forward (the lighter fusion: GELU in the up layer's
epilogue, the hidden activation through memory to the down layer's forward) equals the oracle's
exact GELU of the plain forward on every element.
"""
import numpy as np
import pytest

import synth
from oracle import svdq_oracle as O
from tbound import assert_t_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import w4a4_rank_corrected_smooth_b200 as S  # noqa: E402

REL_FRO_TOL = 5e-3
MAX_ABS_TOL = 1e-2


def _bf16_dev(x_bits):
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16).cuda()


def _y64(Y):
    return O.bf16_to_f32(Y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


def _layers(M, K, H, N, r_up, r_down, seed):
    up_spec = synth.custom(f"mlp_up_{seed}", M=M, K=K, N=H, rank=r_up, seed=seed)
    down_spec = synth.custom(f"mlp_down_{seed}", M=M, K=H, N=N, rank=r_down, seed=seed + 1, x_kind="gelu")
    X = synth.activations_bf16(up_spec)
    up = S.SVDQLinear(synth.weight_bf16(up_spec), synth.bias_bf16(up_spec), synth.act_absmax(X), "nvfp4", r_up)
    calib = synth.activations_bf16(down_spec.with_rows(min(M, 512)))  # GELU-shaped hidden activations
    down = S.SVDQLinear(synth.weight_bf16(down_spec), synth.bias_bf16(down_spec), synth.act_absmax(calib), "nvfp4",
                        r_down)
    return X, up, down


def _run(up, down, X):
    M = X.shape[0]
    Xd = _bf16_dev(X)
    ws_up = up.new_workspace(M)
    mid = torch.empty(max(S.svdq_mlp_workspace_size(up, down, M), 256), dtype=torch.uint8, device="cuda")
    Y = torch.full((M, down.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    S.svdq_mlp_forward(up, down, Xd, M, Xd.stride(0), Y, Y.stride(0), ws_up, ws_up.numel(), mid, mid.numel())
    S.svdq_get_device_error()
    return Y, mid


def _check(up, down, X, rows, Y, mid):
    ops_up, ops_down = up.export_weights(), down.export_weights()
    ref = O.mlp_pair(X[rows], ops_up, ops_down, "nvfp4")
    got = _y64(Y[torch.from_numpy(rows).cuda()])
    assert np.all(np.isfinite(got))
    assert O.rel_fro(got, ref["Y"]) <= REL_FRO_TOL
    assert np.max(np.abs(got - ref["Y"])) <= MAX_ABS_TOL * np.max(np.abs(ref["Y"]))
    act = down.svdq_export_activations(mid, X.shape[0])
    # The up layer alone (same kernels, same accumulation order per tile) gives the bf16 values the
    # fused epilogue starts from; GELU, smoothing and quantization of them are decided exactly.
    M = X.shape[0]
    Xd = _bf16_dev(X)
    Yup = torch.empty((M, up.N), dtype=torch.bfloat16, device="cuda")
    ws = up.new_workspace(M)
    up.svdq_linear_forward(Xd, M, Xd.stride(0), Yup, Yup.stride(0), ws, ws.numel())
    S.svdq_get_device_error()
    y_up = Yup[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    y_up_ref = O.f64_to_bf16(ref["Y_up"])  # the up layer itself is within the usual tolerance
    yu, yr = O.bf16_to_f32(y_up).astype(np.float64), O.bf16_to_f32(y_up_ref).astype(np.float64)
    assert O.rel_fro(yu, yr) <= REL_FRO_TOL and np.max(np.abs(yu - yr)) <= MAX_ABS_TOL * np.max(np.abs(yr))
    h = O.gelu_bf16(y_up)
    xh, cx, sx = O.quantize_activations(h, ops_down["inv_lambda"], "nvfp4")
    assert np.array_equal(act["codes_x"][rows], cx), "hidden codes differ from the oracle's"
    assert np.array_equal(act["scales_x"][rows], sx), "hidden scales differ from the oracle's"
    if down.rank > 0:
        t_got = O.bf16_to_f32(act["T"][rows]).astype(np.float64)
        t_ref = O.bf16_to_f32(O.lowrank_down(xh, ops_down["L1"])).astype(np.float64)
        assert_t_close(t_got, t_ref, O.bf16_to_f32(O.f32_to_bf16(xh)), O.bf16_to_f32(ops_down["L1"]))


def test_epilogue_gelu_on_every_bf16_input():
    """The fused epilogue's GELU (through its test hook) against the oracle's exact bf16 GELU on all
    65536 bf16 patterns (NaN and infinity patterns excluded from the comparison)."""
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = O.bf16_to_f32(pats)
    fin = np.isfinite(vals)
    inp = torch.from_numpy(pats.view(np.int16)).cuda()
    out = torch.empty_like(inp)
    S.svdq_selftest_gelu_bf16(inp, out, inp.numel())
    torch.cuda.synchronize()
    got = out.cpu().numpy().view(np.uint16)
    ref = O.gelu_bf16(pats[fin])
    bad = np.nonzero(got[fin] != ref)[0]
    assert bad.size == 0, [(float(vals[fin][i]), int(got[fin][i]), int(ref[i])) for i in bad[:8]]


@pytest.mark.parametrize("M,r_up,r_down", [(300, 32, 32), (256, 16, 16), (129, 32, 0), (1, 0, 32)])
def test_small_mlp_pair(M, r_up, r_down):
    X, up, down = _layers(M, 512, 768, 512, r_up, r_down, seed=50 + M)
    Y, mid = _run(up, down, X)
    Y2, _ = _run(up, down, X)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16)), "two runs differ"
    _check(up, down, X, np.arange(M), Y, mid)
    up.close()
    down.close()


def test_flux_mlp_pair_sampled_rows():
    """FLUX's MLP (4608 x 3072 -> 12288 -> 3072, rank 32 both), 64 seeded rows over all columns."""
    X, up, down = _layers(4608, 3072, 12288, 3072, 32, 32, seed=70)
    Y, mid = _run(up, down, X)
    rows = np.sort(np.random.default_rng(12).choice(4608, 64, replace=False))
    _check(up, down, X, rows, Y, mid)
    up.close()
    down.close()


def test_argument_checks():
    X, up, down = _layers(64, 512, 768, 512, 16, 16, seed=90)
    _, up_bad, _ = _layers(64, 512, 1024, 512, 16, 16, seed=91)  # up N 1024 != down K 768
    with pytest.raises(S.SVDQError) as ei:
        S.svdq_mlp_workspace_size(up_bad, down, 64)
    assert ei.value.status == 1
    spec = synth.custom("mlp_r64", M=64, K=768, N=512, rank=64, seed=92)
    down64 = S.SVDQLinear(synth.weight_bf16(spec), None, synth.act_absmax(synth.activations_bf16(spec)), "nvfp4", 64)
    with pytest.raises(S.SVDQError):
        S.svdq_mlp_workspace_size(up, down64, 64)
    down_i4 = S.SVDQLinear(synth.weight_bf16(spec), None, synth.act_absmax(synth.activations_bf16(spec)), "int4", 16)
    with pytest.raises(S.SVDQError):
        S.svdq_mlp_workspace_size(up, down_i4, 64)
    for lin in (up, down, up_bad, down64, down_i4):
        lin.close()


def _plain_and_gelu(lin, X):
    """The plain forward and the GELU-output forward of one layer on the same input."""
    M = X.shape[0]
    Xd = _bf16_dev(X)
    ws = lin.new_workspace(M)
    Yp = torch.full((M, lin.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    Yg = torch.full((M, lin.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    lin.svdq_linear_forward(Xd, M, Xd.stride(0), Yp, Yp.stride(0), ws, ws.numel())
    lin.svdq_linear_forward_gelu(Xd, M, Xd.stride(0), Yg, Yg.stride(0), ws, ws.numel())
    S.svdq_get_device_error()
    return Yp, Yg


@pytest.mark.parametrize("M,K,N,r", [(300, 512, 768, 16), (1, 256, 256, 0), (4608, 3072, 12288, 32)])
def test_gelu_forward_is_the_exact_gelu_of_the_plain_forward(M, K, N, r):
    """The GELU-output forward: every element equals the oracle's correctly rounded bf16 GELU of the
    plain forward's element (the same MMAs in the same order give the same bf16 output first)."""
    spec = synth.custom(f"gelu_fwd_{M}_{N}", M=M, K=K, N=N, rank=r, seed=60 + M)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "nvfp4", r)
    Yp, Yg = _plain_and_gelu(lin, X)
    rows = np.arange(M) if M <= 512 else np.sort(np.random.default_rng(M).choice(M, 48, replace=False))
    idx = torch.from_numpy(rows).cuda()
    yp = Yp[idx].view(torch.int16).cpu().numpy().view(np.uint16)
    yg = Yg[idx].view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(yg, O.gelu_bf16(yp))
    lin.close()


def test_mlp_pair_through_the_gelu_forward():
    """The lighter fusion of FLUX's MLP pair: the up layer's GELU-output forward, then the down
    layer's forward on that hidden activation; Y against the oracle's pair on sampled rows, and
    the down layer's codes and scales bit-exact against the oracle's quantizer of the hidden rows."""
    X, up, down = _layers(4608, 3072, 12288, 3072, 32, 32, seed=70)
    M = X.shape[0]
    _, H = _plain_and_gelu(up, X)
    ws = down.new_workspace(M)
    Y = torch.full((M, down.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    down.svdq_linear_forward(H, M, H.stride(0), Y, Y.stride(0), ws, ws.numel())
    S.svdq_get_device_error()
    rows = np.sort(np.random.default_rng(13).choice(M, 64, replace=False))
    ref = O.mlp_pair(X[rows], up.export_weights(), down.export_weights(), "nvfp4")
    got = _y64(Y[torch.from_numpy(rows).cuda()])
    assert O.rel_fro(got, ref["Y"]) <= REL_FRO_TOL
    assert np.max(np.abs(got - ref["Y"])) <= MAX_ABS_TOL * np.max(np.abs(ref["Y"]))
    h = H[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    _, cx, sx = O.quantize_activations(h, down.export_weights()["inv_lambda"], "nvfp4")
    act = down.svdq_export_activations(ws, M)
    assert np.array_equal(act["codes_x"][rows], cx) and np.array_equal(act["scales_x"][rows], sx)
    up.close()
    down.close()


def test_gelu_forward_refuses_int4():
    spec = synth.custom("gelu_i4", M=16, K=256, N=256, rank=16, seed=95)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), None, synth.act_absmax(X), "int4", 16)
    Xd = _bf16_dev(X)
    ws = lin.new_workspace(16)
    Y = torch.empty((16, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.SVDQError) as ei:
        lin.svdq_linear_forward_gelu(Xd, 16, 256, Y, 256, ws, ws.numel())
    assert ei.value.status == 1
    lin.close()
