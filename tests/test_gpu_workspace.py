"""Kernel 1's workspace and determinism, for both of its forms.

Kernel 1 writes every byte of the activation codes, scales and T that kernel 2 reads.  Its
warp-level form (16-row blocks, rank <= 32, up to two waves of blocks) sums its warps' shares of T
in a fixed order, and on layers of fewer blocks than two per SM also splits K over CTAs; its
128-row-tile form always splits K when the grid has room.  A split writes an fp32 partial of T per
slice and counts itself in a counter (per 16-row block or 128-row tile) tagged with the launch,
and the last slice sums the partials in slice order.  These tests check that the result needs no initialised workspace (0xFF
everywhere: garbage counters), that reusing a workspace gives bit-identical results, and that a
CUDA-graph replay of the forward (the same launch tag every time) does too.
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


def _bf16_dev(x_bits):
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16).cuda()


# (rank, M): the warp-level form with K split over CTAs (M = 512: 32 blocks of 16 rows, 6 slices)
# and without (M = 4608: 288 blocks); the 128-row tiles (rank 64), K split in 8
FORMS = [(32, 512), (32, 4608), (64, 512)]


def _layer(M=512, K=3072, N=512, r=32, seed=41):
    spec = synth.custom("quant_down_ws", M=M, K=K, N=N, rank=r, seed=seed)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "nvfp4", r)
    return spec, X, lin


def _check_T(lin, X, act):
    ops = lin.export_weights()
    xh, cx, sx = O.quantize_activations(X, ops["inv_lambda"], "nvfp4")
    assert np.array_equal(act["codes_x"], cx) and np.array_equal(act["scales_x"], sx)
    T_ref = O.bf16_to_f32(O.lowrank_down(xh, ops["L1"])).astype(np.float64)
    T_gpu = O.bf16_to_f32(act["T"]).astype(np.float64)
    # fp32 accumulation vs the exact sum, both rounded to bf16: per-element bound
    assert_t_close(T_gpu, T_ref, O.bf16_to_f32(O.f32_to_bf16(xh)), O.bf16_to_f32(ops["L1"]))


@pytest.mark.parametrize("r,M", FORMS)
def test_quant_down_needs_no_initialised_workspace_and_repeats_bit_exactly(r, M):
    spec, X, lin = _layer(M=M, r=r)
    Xd = _bf16_dev(X)
    ws = lin.new_workspace(spec.M)
    ws.fill_(0xFF)  # garbage everywhere
    lin.svdq_quant_down(Xd, spec.M, spec.K, ws, ws.numel())
    S.svdq_get_device_error()
    first = lin.svdq_export_activations(ws, spec.M)
    _check_T(lin, X, first)
    for _ in range(2):  # the same workspace again
        lin.svdq_quant_down(Xd, spec.M, spec.K, ws, ws.numel())
        S.svdq_get_device_error()
        again = lin.svdq_export_activations(ws, spec.M)
        for k in first:
            assert np.array_equal(first[k], again[k]), k
    lin.close()


@pytest.mark.parametrize("r,M", [(r, 1000 if M == 512 else M) for r, M in FORMS])
def test_graph_replay_of_the_forward_is_bit_identical_to_eager(r, M):
    spec, X, lin = _layer(M=M, r=r, seed=43)
    Xd = _bf16_dev(X)
    ws = lin.new_workspace(spec.M)
    Y_eager = torch.empty((spec.M, spec.N), dtype=torch.bfloat16, device="cuda")
    lin.svdq_linear_forward(Xd, spec.M, spec.K, Y_eager, spec.N, ws, ws.numel())
    torch.cuda.synchronize()
    S.svdq_get_device_error()
    Y = torch.full((spec.M, spec.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm the launch path once outside the capture
        lin.svdq_linear_forward(Xd, spec.M, spec.K, Y, spec.N, ws, ws.numel(), side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lin.svdq_linear_forward(Xd, spec.M, spec.K, Y, spec.N, ws, ws.numel())
    for _ in range(3):
        Y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        S.svdq_get_device_error()
        assert torch.equal(Y.view(torch.int16), Y_eager.view(torch.int16))
    del g
    lin.close()
