"""GPU parity of the fused QKV + RMS normalization + rotary operator (the grouped QKV projection
with norm_q, norm_k and the rotary embedding in its epilogue) through the C ABI, against the
oracle's fp64 steps over the library's exported operands.

Bar: the V columns are bit-identical to the plain forward's (same accumulation, bias and
rounding); the Q/K columns within relative Frobenius 5e-3 and max|dY| <= 1e-2 max|ref| of the
oracle's normalization and rotation of the exact layer output; two runs are bit-identical.
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
D = 128
EPS = 1e-6


def _bf16_dev(x_bits):
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16).cuda()


def _y64(Y):
    return O.bf16_to_f32(Y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


def _pack(rope_d, M):
    packed = torch.empty(S.svdq_rope_packed_size(M, D) // 4, dtype=torch.float32, device="cuda")
    S.svdq_pack_rope(rope_d, M, D, packed, packed.numel() * 4)
    return packed


def _inputs(M, seed):
    cos, sin = synth.rope_tables(M, D, text_tokens=min(512, M // 4), grid_w=64)
    rope = np.stack([cos, sin], axis=-1).reshape(M, D).astype(np.float32)
    gq = synth.rms_norm_weight(D, seed)
    gk = synth.rms_norm_weight(D, seed + 1)
    rope_d = _pack(torch.from_numpy(rope).cuda(), M)
    return cos, sin, gq, gk, rope_d, torch.from_numpy(gq).cuda(), torch.from_numpy(gk).cuda()


@pytest.mark.parametrize("M", [1, 31, 32, 33, 300])
def test_rope_packing_layout(M):
    """svdq_pack_rope moves every value to its place: the 16-byte half hf of the 4-pair unit u of row
    m sits at float4 ((m // 32 * 16 + u) * 2 + hf) * 32 + m % 32; rows past M repeat row M - 1."""
    rope = np.random.default_rng(M).standard_normal((M, D)).astype(np.float32)
    packed = _pack(torch.from_numpy(rope).cuda(), M).cpu().numpy().reshape(-1, 4)
    rows = (M + 31) // 32 * 32
    assert packed.shape[0] == rows * D // 4
    src = np.concatenate([rope, np.repeat(rope[-1:], rows - M, axis=0)]).reshape(rows, D // 8, 2, 4)
    expect = src.reshape(rows // 32, 32, D // 8, 2, 4).transpose(0, 2, 3, 1, 4).reshape(-1, 4)
    assert np.array_equal(packed, expect)


def _run(lin, Xd, M, gq_d, gk_d, rope_d, eps=EPS):
    ws = lin.new_workspace(M)
    Y = torch.full((M, lin.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    lin.svdq_linear_forward_qkv_norm_rope(Xd, M, Xd.stride(0), Y, Y.stride(0), gq_d, gk_d, eps, rope_d, D, ws,
                                          ws.numel())
    S.svdq_get_device_error()
    return Y, ws


def _check(lin, X, rows, Y, Y_plain, ops, cos, sin, gq, gk, eps=EPS, prec="nvfp4"):
    N = lin.N
    qk = 2 * N // 3
    got = _y64(Y[torch.from_numpy(rows).cuda()])
    # V: bit-identical to the plain forward (the same MMAs in the same order)
    assert torch.equal(Y[:, qk:].view(torch.int16), Y_plain[:, qk:].view(torch.int16))
    exact = O.linear(X[rows], ops, prec)["Y"]
    ref = O.qkv_norm_rope(exact, D, gq, gk, cos[rows], sin[rows], eps)
    assert np.all(np.isfinite(got))
    g, r = got[:, :qk], ref[:, :qk]
    assert O.rel_fro(g, r) <= REL_FRO_TOL
    assert np.max(np.abs(g - r)) <= MAX_ABS_TOL * np.max(np.abs(r))
    # and the V part of the oracle agrees with the plain layer's tolerance
    assert O.rel_fro(got[:, qk:], ref[:, qk:]) <= REL_FRO_TOL


@pytest.mark.parametrize("prec", ["nvfp4", "int4"])
@pytest.mark.parametrize("M,rank", [(300, 16), (256, 0), (1, 32)])
def test_small_qkv_layer(M, rank, prec):
    spec = synth.custom(f"qkv_small_{M}", M=M, K=512, N=3 * 2 * D, rank=rank, seed=40 + M)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), prec, rank)
    ops = lin.export_weights()
    cos, sin, gq, gk, rope_d, gq_d, gk_d = _inputs(M, 5)
    Xd = _bf16_dev(X)
    Y, _ = _run(lin, Xd, M, gq_d, gk_d, rope_d)
    Y2, _ = _run(lin, Xd, M, gq_d, gk_d, rope_d)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16)), "two runs differ"
    Y_plain = lin.forward(Xd)
    _check(lin, X, np.arange(M), Y, Y_plain, ops, cos, sin, gq, gk, prec=prec)
    lin.close()


def test_flux_qkv_layer_sampled_rows():
    """FLUX's grouped QKV (4608 x 3072 -> 3 x 3072: 24 heads of 128 each), rank 32, in the launch
    configuration of the plain forward; 128 seeded rows checked over all columns."""
    spec = synth.get("flux_qkv_4608x3072x9216_r32")
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "nvfp4", spec.rank)
    ops = lin.export_weights()
    cos, sin, gq, gk, rope_d, gq_d, gk_d = _inputs(spec.M, 7)
    Xd = _bf16_dev(X)
    Y, _ = _run(lin, Xd, spec.M, gq_d, gk_d, rope_d)
    Y_plain = lin.forward(Xd)
    rows = np.sort(np.random.default_rng(11).choice(spec.M, 128, replace=False))
    _check(lin, X, rows, Y, Y_plain, ops, cos, sin, gq, gk)
    lin.close()


def test_eps_zero_and_large():
    spec = synth.custom("qkv_eps", M=64, K=256, N=3 * D, rank=16, seed=3)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "nvfp4", 16)
    ops = lin.export_weights()
    cos, sin, gq, gk, rope_d, gq_d, gk_d = _inputs(64, 9)
    Xd = _bf16_dev(X)
    Y_plain = lin.forward(Xd)
    for eps in (0.0, 1.0):  # 1.0 is of the order of the heads' mean square: eps visibly matters
        Y, _ = _run(lin, Xd, 64, gq_d, gk_d, rope_d, eps=eps)
        _check(lin, X, np.arange(64), Y, Y_plain, ops, cos, sin, gq, gk, eps=eps)
    lin.close()


def test_argument_checks():
    cos, sin, gq, gk, rope_d, gq_d, gk_d = _inputs(256, 1)
    spec = synth.get("tiny_256x512x512_r16")  # N = 512: not 3 x heads x 128
    X = synth.activations_bf16(spec)
    Xd = _bf16_dev(X)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "nvfp4", 16)
    ws = lin.new_workspace(256)
    Y = torch.empty((256, 512), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.SVDQError) as ei:
        lin.svdq_linear_forward_qkv_norm_rope(Xd, 256, 512, Y, 512, gq_d, gk_d, EPS, rope_d, D, ws, ws.numel())
    assert ei.value.status == 1
    lin.close()
    spec = synth.custom("qkv_args", M=256, K=512, N=3 * D, rank=16, seed=2)
    X = synth.activations_bf16(spec)
    Xd = _bf16_dev(X)
    Y = torch.empty((256, 3 * D), dtype=torch.bfloat16, device="cuda")
    for prec, hd, rp, eps in (("w4a16", D, rope_d, EPS), ("nvfp4", 64, rope_d, EPS),
                              ("nvfp4", D, rope_d[1:], EPS), ("nvfp4", D, rope_d, -1.0),
                              ("nvfp4", D, rope_d, float("nan"))):
        lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), prec,
                           0 if prec == "w4a16" else 16)
        ws = lin.new_workspace(256)
        with pytest.raises(S.SVDQError) as ei:
            lin.svdq_linear_forward_qkv_norm_rope(Xd, 256, 512, Y, 3 * D, gq_d, gk_d, eps, rp, hd, ws, ws.numel())
        assert ei.value.status == 1, (prec, hd, eps)
        lin.close()
