"""Host-side checks of the C-ABI library (no GPU needed).

The library loads and exports every symbol include/svdq.h declares; its host quantizer is
bit-exact against the oracle's; its offline prepare (smoothing, randomized SVD, residual,
quantization) agrees with the oracle's; argument errors come back as status codes with messages.
"""
import os
import re

import numpy as np
import pytest

import synth
from oracle import svdq_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

S = pytest.importorskip("w4a4_rank_corrected_smooth_b200")


def header_functions():
    text = open(os.path.join(ROOT, "include", "svdq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    declared = header_functions()
    assert len(declared) >= 18
    lib = S.lib()
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(S.DECLARED_SYMBOLS) == declared


def test_status_strings_and_no_gpu_error_path():
    assert S.lib().svdq_status_string(0) == b"SVDQ_OK"
    assert S.lib().svdq_status_string(5) == b"SVDQ_ERR_TIMEOUT"
    import torch

    if not torch.cuda.is_available():
        with pytest.raises(S.SVDQError) as ei:
            S.svdq_check_device(0)
        assert ei.value.status == 2 and "no CUDA device" in str(ei.value)


def _boundary_values(rng, rows, K, prec):
    """Rows with values on quantizer ties and rounding boundaries, plus random rows."""
    out = (rng.standard_normal((rows, K)) * np.exp2(rng.integers(-12, 12, (rows, 1)))).astype(np.float32)
    G = 16 if prec == "nvfp4" else 64
    for r in range(0, rows, 4):
        for g in range(K // G):
            blk = out[r, g * G:(g + 1) * G]
            if prec == "nvfp4":
                sd = float(O.ue4m3_value(np.array([rng.integers(1, 0x7E)]))[0])
                ties = np.array([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0, -0.01, 0.0, -1.75, 4.0, 1.0, -6.0])
                blk[:] = (ties * sd).astype(np.float32)
            else:
                s = float(rng.integers(1 << 10, 1 << 12)) * 2.0 ** -12
                vals = rng.integers(-14, 15, G) / 2.0
                vals[0] = 7.0
                blk[:] = (vals * s).astype(np.float32)
    out[rows - 1, :] = 0.0
    out[rows - 2, :16] = -1e-30
    return out


@pytest.mark.parametrize("prec", ["nvfp4", "int4"])
def test_host_packer_bitexact_against_oracle(prec):
    rng = np.random.default_rng(31)
    V = _boundary_values(rng, 64, 512, prec)
    codes, scales = S.svdq_quantize_rows_host(V, prec)
    oc, os_ = O.quantize_rows(V, prec)
    assert np.array_equal(codes, oc)
    assert np.array_equal(scales, os_)


@pytest.mark.parametrize("prec", ["nvfp4", "int4"])
def test_host_prepare_against_oracle(prec):
    spec = synth.get("tiny_256x512x512_r16")
    X = synth.activations_bf16(spec)
    W = synth.weight_bf16(spec)
    b = synth.bias_bf16(spec)
    a = synth.act_absmax(X)
    lib = S.svdq_prepare_host(W, b, a, prec, spec.rank)
    ref = O.prepare(W, b, a, prec, spec.rank)
    # smoothing factors: the same fp64 formula, rounded once to fp32
    assert np.array_equal(lib["inv_lambda"], ref["inv_lambda"])
    # the library's residual is quantized exactly as the oracle quantizes it
    oc, os_ = O.quantize_rows(lib["R"], prec)
    assert np.array_equal(lib["codes_w"], oc) and np.array_equal(lib["scales_w"], os_)
    # randomized SVD: well-separated singular values exact, residual Frobenius norm near optimal
    sig = ref["sigma"]
    r = spec.rank
    sep = np.where(sig[:r] / sig[1:r + 1] > 1.5)[0]
    assert len(sep) > 0
    assert np.allclose(lib["sigma"][:sep[-1] + 1], sig[:sep[-1] + 1], rtol=1e-6)
    opt = np.sqrt(np.sum(sig[r:] ** 2))
    assert np.linalg.norm(lib["R"].astype(np.float64)) <= (1 + 1e-3) * opt
    # W_hat = L1 L2 + R up to bf16 rounding of L1/L2
    lam = 1.0 / lib["inv_lambda"].astype(np.float64)
    Wh = O.bf16_to_f32(W).astype(np.float64) * lam[None, :]
    L1 = O.bf16_to_f32(lib["L1"]).astype(np.float64)
    L2 = O.bf16_to_f32(lib["L2"]).astype(np.float64)
    assert O.rel_fro((L1 @ L2).T + lib["R"], Wh) < 5e-3


def test_host_prepare_full_rank_leaves_no_residual():
    spec = synth.custom("fullrank", M=64, K=256, N=64, rank=64, seed=4)
    X = synth.activations_bf16(spec)
    W = synth.weight_bf16(spec)
    lib = S.svdq_prepare_host(W, None, synth.act_absmax(X), "nvfp4", 64, svd_iters=20)
    lam = 1.0 / lib["inv_lambda"].astype(np.float64)
    Wh = O.bf16_to_f32(W).astype(np.float64) * lam[None, :]
    assert np.linalg.norm(lib["R"]) <= 1e-6 * np.linalg.norm(Wh)


def test_host_prepare_is_deterministic():
    spec = synth.custom("det_host", M=64, K=512, N=256, rank=32, seed=5)
    X = synth.activations_bf16(spec)
    W = synth.weight_bf16(spec)
    a = synth.act_absmax(X)
    p1 = S.svdq_prepare_host(W, None, a, "nvfp4", 32, seed=9)
    p2 = S.svdq_prepare_host(W, None, a, "nvfp4", 32, seed=9)
    for k in p1:
        assert np.array_equal(p1[k], p2[k]), k


@pytest.mark.parametrize("N,K,rank,prec,msg", [
    (256, 300, 16, "nvfp4", "multiple of 256"),
    (250, 512, 16, "nvfp4", "multiple of 8"),
    (256, 512, 24, "nvfp4", "multiple of 16"),
    (256, 512, 144, "nvfp4", "multiple of 16 in [0, 128]"),
    (64, 512, 80, "nvfp4", "exceeds min(N, K)"),
    (256, 512, 16, 7, "precision"),
])
def test_prepare_rejects_bad_arguments(N, K, rank, prec, msg):
    W = np.zeros((N, K), np.uint16)
    a = np.ones(K, np.float32)
    with pytest.raises(S.SVDQError) as ei:
        S.svdq_prepare_host(W, None, a, prec, rank)
    assert ei.value.status == 1 and msg in str(ei.value)


def test_prepare_rejects_bad_alpha():
    with pytest.raises(S.SVDQError) as ei:
        S.svdq_prepare_host(np.zeros((256, 256), np.uint16), None, np.ones(256, np.float32), "nvfp4", 16, alpha=1.5)
    assert "alpha" in str(ei.value)


def test_host_prepare_w4a16_against_oracle():
    """W4A16 (rank 0, INT4 weights of the smoothed weight): smoothing exact, codes and scales of the
    library's own fp32 smoothed weight exactly as the oracle quantizes them."""
    spec = synth.custom("w4a16_host", M=64, K=512, N=256, rank=0, seed=31)
    X = synth.activations_bf16(spec)
    W = synth.weight_bf16(spec)
    a = synth.act_absmax(X)
    lib = S.svdq_prepare_host(W, None, a, "w4a16", 0)
    ref = O.prepare_w4a16(W, None, a)
    assert np.array_equal(lib["inv_lambda"], ref["inv_lambda"])
    oc, os_ = O.quantize_rows(lib["R"], O.INT4)
    assert np.array_equal(lib["codes_w"], oc) and np.array_equal(lib["scales_w"], os_)
    # the library's smoothed weight is the oracle's up to the last fp32 rounding
    assert np.max(np.abs(lib["R"].astype(np.float64) - ref["R"].astype(np.float64))) <= \
        1e-6 * np.max(np.abs(ref["R"]))
    with pytest.raises(S.SVDQError) as ei:
        S.svdq_prepare_host(W, None, a, "w4a16", 16)
    assert ei.value.status == 1 and "no low-rank branch" in str(ei.value)
