"""GPU parity on every FLUX-shaped configuration, full size, in the launch configuration the
benchmark uses (through the C ABI).

- MLP pair (up 4608x3072->12288, down 4608x12288->3072 on GELU inputs), NVFP4 and INT4;
- DiT block (16896x3072->21504 and 16896x15360->3072), NVFP4;
- the M x rank sweep at K = N = 3072 (M = 256 ... 16384, rank 0 ... 128), NVFP4.

Rows are independent, so a seeded subset of rows checked across all N is an exact check of those
rows: activation codes and scales bit-exact and Y within the layer's tolerance (relative Frobenius
5e-3, max|dY| <= 1e-2 max|Y_ref|) against the oracle's fp64 forward over the library's exported
operands.  The sweep's smaller layers check every row's codes and scales.
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


def _forward(lin, X):
    M = X.shape[0]
    Xd = _bf16_dev(X)
    ws = lin.new_workspace(M)
    Y = torch.full((M, lin.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    lin.svdq_linear_forward(Xd, M, Xd.stride(0), Y, Y.stride(0), ws, ws.numel())
    S.svdq_get_device_error()
    act = lin.svdq_export_activations(ws, M)
    return Y, act


def _check_rows(lin, X, Y, act, rows, prec, ops):
    xh, cx, sx = O.quantize_activations(X[rows], ops["inv_lambda"], prec)
    assert np.array_equal(act["codes_x"][rows], cx), "activation codes differ from the oracle"
    assert np.array_equal(act["scales_x"][rows], sx), "activation scales differ from the oracle"
    T = O.lowrank_down(xh, ops["L1"])
    if lin.rank:
        assert_t_close(O.bf16_to_f32(act["T"][rows]).astype(np.float64), O.bf16_to_f32(T).astype(np.float64),
                       O.bf16_to_f32(O.f32_to_bf16(xh)), O.bf16_to_f32(ops["L1"]))
    ref = O.forward(cx, sx, T, ops["codes_w"], ops["scales_w"], ops["L2"], ops["bias"], prec)
    got = O.bf16_to_f32(Y[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    assert np.all(np.isfinite(got))
    assert O.rel_fro(got, ref) <= REL_FRO_TOL
    assert np.max(np.abs(got - ref)) <= MAX_ABS_TOL * np.max(np.abs(ref))


@pytest.mark.parametrize("name,prec", [
    ("flux_mlp_up_4608x3072x12288_r32", "nvfp4"),
    ("flux_mlp_up_4608x3072x12288_r32", "int4"),
    ("flux_mlp_down_4608x12288x3072_r32", "nvfp4"),
    ("flux_mlp_down_4608x12288x3072_r32", "int4"),
    ("dit_qkv_mlp_in_16896x3072x21504_r32", "nvfp4"),
    ("dit_out_16896x15360x3072_r32", "nvfp4"),
])
def test_full_size_layer_sampled_rows(name, prec):
    spec = synth.get(name)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), prec, spec.rank)
    ops = lin.export_weights()
    Y, act = _forward(lin, X)
    rows = np.sort(np.random.default_rng(len(name)).choice(spec.M, 128, replace=False))
    _check_rows(lin, X, Y, act, rows, prec, ops)
    lin.close()


@pytest.mark.parametrize("rank", [0, 16, 32, 64, 128])
def test_sweep_all_m_for_rank(rank):
    # The sweep's X of M rows is the first M rows of one counter-based matrix; W is shared by all
    # points of a rank.
    big = synth.get(f"sweep_16384x3072x3072_r{rank}")
    X_all = synth.activations_bf16(big)
    lin = S.SVDQLinear(synth.weight_bf16(big), synth.bias_bf16(big), synth.act_absmax(X_all[:4096]), "nvfp4", rank)
    ops = lin.export_weights()
    rng = np.random.default_rng(rank)
    for M in (256, 1024, 4096, 16384):
        X = X_all[:M]
        Y, act = _forward(lin, X)
        if M <= 4096:  # every row's codes and scales
            _, cx, sx = O.quantize_activations(X, ops["inv_lambda"], "nvfp4")
            assert np.array_equal(act["codes_x"], cx) and np.array_equal(act["scales_x"], sx), M
        rows = np.sort(rng.choice(M, min(M, 96), replace=False))
        _check_rows(lin, X, Y, act, rows, "nvfp4", ops)
    lin.close()
