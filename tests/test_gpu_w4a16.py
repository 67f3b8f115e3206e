"""GPU parity of the W4A16 layer (4-bit INT4 weights of the smoothed weight, 16-bit activations, no
low-rank branch) through the C ABI against the oracle's fp64 forward over the library's exported
operands.

Cases: FLUX's modulation projections (one token per image: M = 1 ... 5 rows, K = 3072,
N = 18432 and 9216) and M = 12, 16, 40 (the 16-row passes), a long K (several staged chunks), a
ragged small layer with padded row strides, and a tall input that the launcher splits over
several grids.  Bar as for the W4A4 layer: relative Frobenius error 5e-3 and
max|dY| <= 1e-2 max|Y_ref|.
"""
import numpy as np
import pytest

import synth
from oracle import svdq_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import w4a4_rank_corrected_smooth_b200 as S  # noqa: E402

REL_FRO_TOL = 5e-3
MAX_ABS_TOL = 1e-2


def _dev(x_bits, ld):
    M, K = x_bits.shape
    buf = torch.zeros((M, ld), dtype=torch.int16, device="cuda")
    buf[:, :K] = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda()
    return buf.view(torch.bfloat16)


def _run(lin, X, ldx_pad=0, ldy_pad=0):
    M, K = X.shape
    Xd = _dev(X, K + ldx_pad)
    Y = torch.full((M, lin.N + ldy_pad), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = lin.new_workspace(M)
    lin.svdq_linear_forward(Xd, M, Xd.stride(0), Y, Y.stride(0), ws, 0)
    S.svdq_get_device_error()
    return Y


def _y64(Y, rows=None, N=None):
    y = Y if rows is None else Y[torch.from_numpy(np.asarray(rows)).cuda()]
    y = O.bf16_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    return y if N is None else y[:, :N]


def _check(got, ref):
    assert np.all(np.isfinite(got))
    assert O.rel_fro(got, ref) <= REL_FRO_TOL
    assert np.max(np.abs(got - ref)) <= MAX_ABS_TOL * np.max(np.abs(ref))


@pytest.mark.parametrize("N", [18432, 9216])
@pytest.mark.parametrize("M", [1, 2, 3, 5])
def test_modulation_projection(M, N):
    spec = synth.custom(f"mod_{N}", M=8, K=3072, N=N, rank=0, seed=N)
    X8 = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X8), "w4a16", 0)
    assert lin.workspace_size(M) == 0
    ops = lin.export_weights()
    X = X8[:M]
    Y = _run(lin, X)
    _check(_y64(Y), O.linear_w4a16(X, ops)["Y"])
    lin.close()


@pytest.mark.parametrize("M", [12, 16, 40])
def test_sixteen_row_passes(M):
    spec = synth.custom("w4a16_m16", M=M, K=3072, N=1024, rank=0, seed=21)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "w4a16", 0)
    _check(_y64(_run(lin, X)), O.linear_w4a16(X, lin.export_weights())["Y"])
    lin.close()


def test_long_k_in_several_chunks():
    # K = 16384: 256 groups, more than one staging of the activation fragments holds
    spec = synth.custom("w4a16_longk", M=3, K=16384, N=512, rank=0, seed=22)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "w4a16", 0)
    _check(_y64(_run(lin, X)), O.linear_w4a16(X, lin.export_weights())["Y"])
    lin.close()


def test_ragged_with_padded_strides():
    # K = 768 (three 256-element passes per warp), N = 40, M = 9 (a partial tile of 4 rows), row
    # strides padded (X by 24 elements, Y by 8)
    spec = synth.custom("w4a16_ragged", M=9, K=768, N=40, rank=0, seed=5)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "w4a16", 0)
    ops = lin.export_weights()
    Y = _run(lin, X, ldx_pad=24, ldy_pad=8)
    assert torch.isnan(Y[:, lin.N:]).all(), "the row padding of Y was written"
    _check(_y64(Y, N=lin.N), O.linear_w4a16(X, ops)["Y"])
    lin.close()


def test_without_bias_and_zero_rows():
    spec = synth.custom("w4a16_nobias", M=4, K=256, N=64, rank=0, seed=6)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), None, synth.act_absmax(X), "w4a16", 0)
    ops = lin.export_weights()
    assert not np.any(ops["bias"])
    _check(_y64(_run(lin, X)), O.linear_w4a16(X, ops)["Y"])
    Y0 = torch.empty((0, lin.N), dtype=torch.bfloat16, device="cuda")
    lin.svdq_linear_forward(Y0, 0, 256, Y0, lin.N, None, 0)  # M = 0: nothing to do
    lin.close()


def test_tall_input_over_several_grids():
    # 16 * 65535 + 19 rows: more 16-row passes than one grid holds, so the launcher splits the rows;
    # rows are independent, so sampled rows (both sides of the split) are an exact check.
    spec = synth.custom("w4a16_tall", M=1024, K=256, N=24, rank=0, seed=8)
    Xs = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(Xs), "w4a16", 0)
    ops = lin.export_weights()
    M = 16 * 65535 + 19
    X = np.tile(Xs, (M // 1024 + 1, 1))[:M]
    Y = _run(lin, X)
    split = 16 * 65535
    rows = np.array([0, 1, 1023, 131072, split - 17, split - 1, split, split + 1, split + 8, M - 1])
    ref = O.linear_w4a16(Xs[rows % 1024], ops)["Y"]
    _check(_y64(Y, rows), ref)
    lin.close()


def test_split_entry_points_are_refused():
    spec = synth.custom("w4a16_refuse", M=4, K=256, N=16, rank=0, seed=9)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "w4a16", 0)
    Xd = _dev(X, 256)
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(S.SVDQError) as ei:
        lin.svdq_quant_down(Xd, 4, 256, ws, ws.numel())
    assert ei.value.status == 1
    lin.close()
