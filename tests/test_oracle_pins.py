"""Pins for the CPU oracle: closed forms, invariants, brute force and special cases.

Each test checks the oracle against something other than itself: the format
definitions of E2M1 / UE4M3 / INT4 written out from their bit layouts, the
algebraic identities that the SVDQuant model card's stages 1-3 fix, the
Eckart-Young optimality of a truncated SVD, brute-force loops in a different
order, and hand-computed tiny cases.  A plausible slip in the oracle (a wrong
tie rule, a dropped term, a transposed factor, an inverted smoothing
direction) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import svdq_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def _f32(x):
    return np.float32(x)


def _next_up(x):
    return np.nextafter(np.float32(x), np.float32(np.inf), dtype=np.float32)


def _next_down(x):
    return np.nextafter(np.float32(x), np.float32(-np.inf), dtype=np.float32)


# ---------------------------------------------------------------- formats


def e2m1_closed_form(code: int) -> float:
    """E2M1 from its bits: sign | 2-bit exponent (bias 1) | 1 mantissa bit."""
    s = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return s * mag


def ue4m3_closed_form(code: int) -> float:
    e = (code >> 3) & 0xF
    m = code & 7
    return m * 2.0 ** -9 if e == 0 else 2.0 ** (e - 7) * (1.0 + m / 8.0)


def test_e2m1_table_matches_bit_definition():
    for c in range(16):
        v = float(O.e2m1_value(np.array([c]))[0])
        assert v == e2m1_closed_form(c) or (v == 0 and e2m1_closed_form(c) == 0)
    assert float(O.e2m1_value(np.array([7]))[0]) == 6.0


def test_e2m1_encode_grid_midpoints_ties_saturation_sign():
    mags = [e2m1_closed_form(c) for c in range(8)]
    for c, v in enumerate(mags):
        assert int(O.e2m1_encode(np.array([v], np.float32))[0]) == c
        if v != 0:
            assert int(O.e2m1_encode(np.array([-v], np.float32))[0]) == c | 8
    for c in range(7):
        a, b = mags[c], mags[c + 1]
        mid = _f32((a + b) / 2)  # exact: a few significant bits
        assert int(O.e2m1_encode(np.array([_next_down(mid)]))[0]) == c
        assert int(O.e2m1_encode(np.array([_next_up(mid)]))[0]) == c + 1
        even = c if c % 2 == 0 else c + 1  # ties go to the even mantissa bit
        assert int(O.e2m1_encode(np.array([mid]))[0]) == even
    # hand-listed ties from the rounding rule
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, want in ties.items():
        got = float(O.e2m1_value(O.e2m1_encode(np.array([x], np.float32)))[0])
        assert got == want, (x, got, want)
    for big in (6.0001, 7.0, 1e30):
        assert int(O.e2m1_encode(np.array([big], np.float32))[0]) == 7
        assert int(O.e2m1_encode(np.array([-big], np.float32))[0]) == 15
    # negative values that round to zero keep the sign bit (reading R6)
    assert int(O.e2m1_encode(np.array([-0.1], np.float32))[0]) == 8
    assert int(O.e2m1_encode(np.array([0.1], np.float32))[0]) == 0


def test_ue4m3_table_roundtrip_midpoints_saturation_underflow():
    for c in range(0x7F):
        assert float(O.ue4m3_value(np.array([c]))[0]) == ue4m3_closed_form(c)
        assert int(O.ue4m3_encode(np.array([ue4m3_closed_form(c)], np.float32))[0]) == c
    assert ue4m3_closed_form(0x7E) == 448.0
    for c in range(0x7E):
        a, b = ue4m3_closed_form(c), ue4m3_closed_form(c + 1)
        mid = _f32((a + b) / 2)
        assert float(mid) == (a + b) / 2
        assert int(O.ue4m3_encode(np.array([_next_down(mid)]))[0]) == c
        assert int(O.ue4m3_encode(np.array([_next_up(mid)]))[0]) == c + 1
        assert int(O.ue4m3_encode(np.array([mid]))[0]) == (c if c % 2 == 0 else c + 1)
    for big in (448.0001, 464.0, 480.0, 1e9):
        assert int(O.ue4m3_encode(np.array([big], np.float32))[0]) == 0x7E
    # half the smallest subnormal is a tie between 0 and 2^-9: goes to 0 (even)
    assert int(O.ue4m3_encode(np.array([2.0 ** -10], np.float32))[0]) == 0
    assert int(O.ue4m3_encode(np.array([_next_up(2.0 ** -10)], np.float32))[0]) == 1
    assert int(O.ue4m3_encode(np.array([2.0 ** -11], np.float32))[0]) == 0


def test_int4_rounding_half_even_and_clamp():
    # one group of 64 with amax 7 -> scale exactly 1, so codes are rint(v)
    v = np.zeros((1, 64), np.float32)
    vals = [7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.49, -6.51, 0.0]
    v[0, :len(vals)] = vals
    codes, scales = O.quantize_rows(v, O.INT4)
    assert scales[0, 0] == np.float32(1.0)
    q = O.int4_value(O.unpack_nibbles(codes))[0, :len(vals)]
    assert list(q) == [7, 0, 2, 2, 0, -2, -2, 3, -7, 0]
    # clamp: an element above amax cannot occur; a direct rint beyond 7 is clipped
    assert np.clip(np.rint(7.6), -8, 7) == 7


def test_packing_low_nibble_first():
    nib = np.array([[1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 0]], np.uint8)
    p = O.pack_nibbles(nib)
    assert list(p[0]) == [0x21, 0x43, 0x65, 0x87, 0xA9, 0xCB, 0xED, 0x0F]
    assert np.array_equal(O.unpack_nibbles(p), nib)


def test_bf16_rounding_against_closed_form_and_torch():
    import torch

    one = 1.0
    cases = {one + 2.0 ** -8: one, one + 3 * 2.0 ** -8: one + 2.0 ** -6, one + 2.0 ** -8 + 2.0 ** -20: one + 2.0 ** -7,
             -(one + 2.0 ** -8): -one, 3.0: 3.0}
    for x, want in cases.items():
        got = O.bf16_to_f32(O.f32_to_bf16(np.array([x], np.float32)))[0]
        assert float(got) == want, (x, got, want)
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp2(rng.integers(-20, 20, 100000))).astype(np.float32)
    ours = O.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ---------------------------------------------------------------- quantizer


def _random_on_grid_nvfp4(rng, rows, K, lo=0x08, hi=0x7E):
    G = 16
    nblk = K // G
    scodes = rng.integers(lo, hi, size=(rows, nblk))  # normal UE4M3 scales
    nib = rng.integers(0, 16, size=(rows, nblk, G)).astype(np.uint8)
    pos = rng.integers(0, G, size=(rows, nblk))
    sign = rng.integers(0, 2, size=(rows, nblk)).astype(np.uint8) << 3
    nib[np.arange(rows)[:, None], np.arange(nblk)[None, :], pos] = 7 | sign  # a +-6 in every block
    vals = np.array([e2m1_closed_form(int(c)) for c in range(16)])[nib]
    sval = np.array([ue4m3_closed_form(int(c)) for c in range(0x7F)])[scodes]
    v = (vals * sval[:, :, None]).reshape(rows, K).astype(np.float32)
    return v, nib.reshape(rows, K), scodes.astype(np.uint8)


def test_nvfp4_values_on_grid_roundtrip_exactly():
    rng = np.random.default_rng(1)
    v, nib, scodes = _random_on_grid_nvfp4(rng, 32, 256)
    codes, scales = O.quantize_rows(v, O.NVFP4)
    assert np.array_equal(scales, scodes)
    got = O.unpack_nibbles(codes)
    # +-0 both decode to 0; the encoder keeps the sign of -0.0 inputs
    assert np.array_equal(got, nib)
    assert np.array_equal(O.dequantize_rows(codes, scales, O.NVFP4), v.astype(np.float64))


def test_int4_values_on_grid_roundtrip_exactly():
    rng = np.random.default_rng(2)
    rows, K, G = 16, 256, 64
    # scales with <= 20 significant bits so that 7 * s is exact in fp32
    s = (rng.integers(1 << 19, 1 << 20, size=(rows, K // G)) * 2.0 ** -25).astype(np.float32)
    q = rng.integers(-7, 8, size=(rows, K // G, G))
    q[:, :, 0] = 7 * np.where(rng.integers(0, 2, size=(rows, K // G)) > 0, 1, -1)
    v = (q * s[:, :, None].astype(np.float64)).reshape(rows, K).astype(np.float32)
    codes, scales = O.quantize_rows(v, O.INT4)
    assert np.array_equal(scales, s)
    assert np.array_equal(O.int4_value(O.unpack_nibbles(codes)).reshape(rows, K // G, G), q)


def test_quantize_dequantize_idempotent():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((64, 512)) * np.exp2(rng.integers(-6, 6, (64, 1)))).astype(np.float32)
    c1, s1 = O.quantize_rows(x, O.NVFP4)
    d1 = O.dequantize_rows(c1, s1, O.NVFP4).astype(np.float32)
    c2, s2 = O.quantize_rows(d1, O.NVFP4)
    nib1 = O.unpack_nibbles(c1).reshape(64, 32, 16)
    blk6 = np.max(nib1 & 7, axis=2) == 7
    assert blk6.mean() > 0.5
    assert np.array_equal(s1[blk6], s2[blk6])
    nib2 = O.unpack_nibbles(c2).reshape(64, 32, 16)
    assert np.array_equal(nib1[blk6], nib2[blk6])
    # INT4: codes equal, scale within one ulp (RN(RN(7s)/7) may move by an ulp)
    c1, s1 = O.quantize_rows(x, O.INT4)
    d1 = O.dequantize_rows(c1, s1, O.INT4).astype(np.float32)
    c2, s2 = O.quantize_rows(d1, O.INT4)
    assert np.array_equal(c1, c2)
    ulp = np.spacing(s1)
    assert np.all(np.abs(s2 - s1) <= ulp)


def test_zero_and_underflow_blocks():
    v = np.zeros((2, 32), np.float32)
    v[1, :16] = -1e-30  # amax/6 underflows UE4M3 -> zero block, all codes +0
    v[1, 16:] = 3.0
    codes, scales = O.quantize_rows(v, O.NVFP4)
    assert scales[0, 0] == 0 and scales[0, 1] == 0 and scales[1, 0] == 0
    assert np.all(O.unpack_nibbles(codes)[:, :16] == 0) and np.all(O.unpack_nibbles(codes)[0] == 0)
    assert float(O.ue4m3_value(scales[1, 1:2])[0]) == 0.5 and np.all(O.unpack_nibbles(codes)[1, 16:] == 7)
    ci, si = O.quantize_rows(np.zeros((1, 64), np.float32), O.INT4)
    assert si[0, 0] == 0 and np.all(ci == 0)


def test_nvfp4_quantizer_brute_force_scalar_loop():
    """Scalar restatement of one block with Python floats (fp32 via numpy scalars)."""
    rng = np.random.default_rng(4)
    v = (rng.standard_normal((3, 16)) * 3).astype(np.float32)
    codes, scales = O.quantize_rows(v, O.NVFP4)
    mags = [e2m1_closed_form(c) for c in range(8)]
    for r in range(3):
        amax = max(abs(float(t)) for t in v[r])
        s = np.float32(np.float32(amax) / np.float32(6.0))
        # nearest UE4M3, ties to even, by scanning every code
        best = min(range(0x7F), key=lambda c: (abs(ue4m3_closed_form(c) - float(s)), c % 2))
        assert scales[r, 0] == best
        sd = np.float32(ue4m3_closed_form(best))
        for k in range(16):
            q = float(np.float32(v[r, k] / sd))
            c = min(range(8), key=lambda i: (abs(mags[i] - abs(q)), i % 2))
            want = c | (8 if q < 0 else 0)
            got = int(O.unpack_nibbles(codes)[r, k])
            assert got == want


# ---------------------------------------------------------------- smoothing + SVD


def test_smoothing_closed_form_and_product_invariance():
    W = np.array([[1.0, -5.0, 0.0], [0.5, 2.0, 0.0]])
    a = np.array([4.0, 0.0, 9.0])
    lam = O.smoothing_factors(a, W)
    assert list(lam) == [2.0, 1.0, 1.0]  # sqrt(4/1); a=0 -> 1; w=0 -> 1
    rng = np.random.default_rng(5)
    X = rng.standard_normal((7, 12))
    X[:, 3] *= 40
    W = rng.standard_normal((5, 12)) * 0.02
    lam = O.smoothing_factors(np.max(np.abs(X), 0), W)
    assert np.all(lam > 0)
    Xh = X / lam[None, :]
    Wh = O.smooth_weight(W, lam)
    assert np.allclose(Xh @ Wh.T, X @ W.T, rtol=1e-13, atol=1e-15)
    # smoothing migrates the outlier: column 3 of X_hat is no longer an outlier
    assert np.max(np.abs(Xh[:, 3])) < np.max(np.abs(X[:, 3])) / 4
    # the fp32 activation path divides by lam (multiplies by 1/lam), not the reverse
    xb = O.f32_to_bf16(X.astype(np.float32))
    xs = O.smooth_activations(xb, O.inv_lambda_f32(lam)).astype(np.float64)
    assert np.allclose(xs, O.bf16_to_f32(xb) / lam[None, :], rtol=2e-7)


def _householder(rng, n):
    Q = np.eye(n)
    for _ in range(3):
        v = rng.standard_normal(n)
        v /= np.linalg.norm(v)
        Q = Q @ (np.eye(n) - 2.0 * np.outer(v, v))
    return Q


def test_svd_recovers_constructed_spectrum():
    rng = np.random.default_rng(6)
    K, N = 20, 14
    Q1 = _householder(rng, K)[:, :N]
    Q2 = _householder(rng, N)
    sig = np.linspace(10.0, 1.0, N) ** 2
    Wkn = Q1 @ np.diag(sig) @ Q2.T
    r = 5
    L1, L2, S, U_r, S_r, Vt_r = O.svd_split(Wkn.T, r)
    assert np.allclose(S, sig, rtol=1e-12)
    assert L1.shape == (K, r) and L2.shape == (r, N)
    trunc = Q1[:, :r] @ np.diag(sig[:r]) @ Q2[:, :r].T
    assert np.linalg.norm(L1 @ L2 - trunc) <= 1e-12 * np.linalg.norm(trunc)
    for i in range(r):
        j = int(np.argmax(np.abs(U_r[:, i])))
        assert U_r[j, i] > 0
    # balanced split: both factors carry sqrt(sigma)
    assert np.allclose(np.linalg.norm(L1, axis=0), np.sqrt(sig[:r]), rtol=1e-12)
    assert np.allclose(np.linalg.norm(L2, axis=1), np.sqrt(sig[:r]), rtol=1e-12)


def test_full_rank_residual_is_zero_and_eckart_young():
    rng = np.random.default_rng(7)
    N, K = 12, 16
    W = rng.standard_normal((N, K))
    L1, L2, S, U_r, S_r, Vt_r = O.svd_split(W, min(N, K))
    R = O.residual_f32(W, U_r, S_r, Vt_r)
    assert np.linalg.norm(R.astype(np.float64)) <= 1e-12 * np.linalg.norm(W) + 1e-6 * 0
    for r in (1, 4, 9):
        L1, L2, S, U_r, S_r, Vt_r = O.svd_split(W, r)
        Rr = W - ((U_r * S_r) @ Vt_r).T
        assert math.isclose(np.sum(Rr ** 2), np.sum(S[r:] ** 2), rel_tol=1e-10)
        # fp32 residual agrees with the fp64 residual to fp32 rounding
        assert np.allclose(O.residual_f32(W, U_r, S_r, Vt_r), Rr, rtol=1e-6, atol=1e-6)


# ---------------------------------------------------------------- GEMM + forward


def test_gemm_4bit_brute_force_grouped_loops():
    rng = np.random.default_rng(8)
    for prec, G in ((O.NVFP4, 16), (O.INT4, 64)):
        M, N, K = 3, 4, 2 * G
        x = rng.standard_normal((M, K)).astype(np.float32)
        w = rng.standard_normal((N, K)).astype(np.float32) * 0.1
        cx, sx = O.quantize_rows(x, prec)
        cw, sw = O.quantize_rows(w, prec)
        Y = O.gemm_4bit(cx, sx, cw, sw, prec)
        nx = O.unpack_nibbles(cx)
        nw = O.unpack_nibbles(cw)

        def code_val(n):
            if prec == O.NVFP4:
                return e2m1_closed_form(int(n))
            n = int(n)
            return float(n - 16 if n >= 8 else n)

        def scale_val(s):
            return ue4m3_closed_form(int(s)) if prec == O.NVFP4 else float(s)

        for m in range(M):
            for n in range(N):
                acc = 0.0
                for g in reversed(range(K // G)):  # a different order from the library matmul
                    part = 0.0
                    for k in range(g * G, (g + 1) * G):
                        part += code_val(nx[m, k]) * code_val(nw[n, k])
                    acc += scale_val(sx[m, g]) * scale_val(sw[n, g]) * part
                assert math.isclose(Y[m, n], acc, rel_tol=1e-12, abs_tol=1e-12)


def test_forward_lossless_on_grid_equals_exact_product():
    """lam = 1, r = 0, operands already on the 4-bit grid: quantization is lossless,
    so the forward equals X W^T + b exactly."""
    rng = np.random.default_rng(9)
    v, _, _ = _random_on_grid_nvfp4(rng, 8, 64, 0x20, 0x50)
    w, _, _ = _random_on_grid_nvfp4(rng, 6, 64, 0x20, 0x50)
    xb = O.f32_to_bf16(v)
    assert np.array_equal(O.bf16_to_f32(xb), v)  # on-grid values are bf16 exact
    inv = np.ones(64, np.float32)
    xh, cx, sx = O.quantize_activations(xb, inv, O.NVFP4)
    cw, sw = O.quantize_rows(w, O.NVFP4)
    bias = O.f32_to_bf16(rng.standard_normal(6).astype(np.float32))
    Y = O.forward(cx, sx, np.zeros((8, 0), np.uint16), cw, sw, np.zeros((0, 6), np.uint16), bias, O.NVFP4)
    exact = v.astype(np.float64) @ w.astype(np.float64).T + O.bf16_to_f32(bias)[None, :]
    assert np.array_equal(Y, exact)


def test_lowrank_branch_hand_computed():
    """x_hat = e_0, L1 row 0 = [1, 2], L2 = [[1,0,0,...],[0,1,0,...]], W = 0, b = 0.5:
    T = [1, 2], T L2 = [1, 2, 0, ...], Y = [1.5, 2.5, 0.5, ...]."""
    K, N, r = 16, 5, 2
    x = np.zeros((1, K), np.float32)
    x[0, 0] = 1.0
    L1 = np.zeros((K, r), np.float32)
    L1[0] = [1.0, 2.0]
    L2 = np.zeros((r, N), np.float32)
    L2[0, 0] = 1.0
    L2[1, 1] = 1.0
    T = O.lowrank_down(x, O.f32_to_bf16(L1))
    assert list(O.bf16_to_f32(T)[0]) == [1.0, 2.0]
    cx, sx = O.quantize_rows(x, O.NVFP4)
    cw, sw = O.quantize_rows(np.zeros((N, K), np.float32), O.NVFP4)
    bias = O.f32_to_bf16(np.full(N, 0.5, np.float32))
    Y = O.forward(cx, sx, T, cw, sw, O.f32_to_bf16(L2), bias, O.NVFP4)
    assert list(Y[0]) == [1.5, 2.5, 0.5, 0.5, 0.5]
    # r = 0: the branch is empty and Y is the 4-bit path plus bias
    T0 = O.lowrank_down(x, np.zeros((K, 0), np.uint16))
    assert T0.shape == (1, 0)


def test_lowrank_down_rounds_x_hat_to_bf16_before_the_product():
    """The 16-bit branch multiplies bf16(x_hat), not x_hat: with x_hat = [1 + d, -1] and L1 = [[1, 2],
    [1, 2]], T = [bf16(1 + d) - 1, 2 (bf16(1 + d) - 1)], worked out by hand on the bf16 grid (spacing
    2^-7 on [1, 2)).  A branch that skipped the rounding would give d itself; one that rounded ties
    away from zero would give 2^-7 for the tie d = 2^-8."""
    d = np.array([2.0 ** -9, 3 * 2.0 ** -9, 2.0 ** -8, 3 * 2.0 ** -8, 2.0 ** -7 + 2.0 ** -10], np.float64)
    # nearest bf16 of 1 + d: below / above the midpoint, a tie to the even neighbour 1.0, a tie to
    # the even neighbour 1 + 2^-6, exactly 1 + 2^-7 plus less than half a spacing
    t0 = np.array([0.0, 2.0 ** -7, 0.0, 2.0 ** -6, 2.0 ** -7])
    x = np.zeros((len(d), 16), np.float32)
    x[:, 0] = (1.0 + d).astype(np.float32)
    x[:, 1] = -1.0
    assert np.all(x[:, 0].astype(np.float64) == 1.0 + d)  # the inputs are exact in fp32
    L1 = np.zeros((16, 2), np.float32)
    L1[0] = L1[1] = [1.0, 2.0]
    T = O.bf16_to_f32(O.lowrank_down(x, O.f32_to_bf16(L1))).astype(np.float64)
    assert np.array_equal(T[:, 0], t0)
    assert np.array_equal(T[:, 1], 2 * t0)


def test_prepare_and_linear_reconstruct_exact_at_full_rank():
    """Full rank: L1 L2 reproduces W_hat, so the low-rank branch alone (with W's 4-bit
    part ~0) approximates X W^T to bf16 precision -- pins the orientation of L1/L2."""
    rng = np.random.default_rng(10)
    M, K, N = 4, 32, 16
    X = O.f32_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    W = O.f32_to_bf16((rng.standard_normal((N, K)) * 0.05).astype(np.float32))
    a = np.max(np.abs(O.bf16_to_f32(X)), axis=0)
    ops = O.prepare(W, None, a, O.NVFP4, rank=N)
    assert np.max(np.abs(ops["R"])) < 1e-6
    out = O.linear(X, ops, O.NVFP4)
    exact = O.exact_linear(X, W, None)
    assert O.rel_fro(out["Y"], exact) < 2e-2


def test_svdquant_error_ordering_on_outlier_data():
    """Model card stage 1-3 claim: smoothing helps 4-bit quantization of outlier
    activations, and the low-rank branch helps further."""
    import synth

    spec = synth.get("tiny_256x512x512_r16")
    X = synth.activations_bf16(spec)
    W = synth.weight_bf16(spec)
    b = synth.bias_bf16(spec)
    exact = O.exact_linear(X, W, b)
    a = np.max(np.abs(O.bf16_to_f32(X)), axis=0)
    for prec in (O.NVFP4, O.INT4):
        plain = O.prepare(W, b, np.zeros_like(a), prec, rank=0)  # a = 0 -> lam = 1
        smooth = O.prepare(W, b, a, prec, rank=0)
        svdq = O.prepare(W, b, a, prec, rank=16)
        e_plain = O.rel_fro(O.linear(X, plain, prec)["Y"], exact)
        e_smooth = O.rel_fro(O.linear(X, smooth, prec)["Y"], exact)
        e_svdq = O.rel_fro(O.linear(X, svdq, prec)["Y"], exact)
        assert e_svdq < e_smooth < e_plain, (prec, e_svdq, e_smooth, e_plain)


# ---------------------------------------------------------------- W4A16 (R9)


def test_w4a16_lossless_on_grid_equals_exact_product():
    """lam = 1 and weights already on the INT4 grid (groups of 64 values q * 2^e with a |q| = 7
    in every group): quantization is lossless, so the W4A16 forward equals X W^T + b."""
    rng = np.random.default_rng(21)
    M, K, N = 5, 128, 6
    q = rng.integers(-7, 8, (N, K)).astype(np.float64)
    q[:, ::64] = 7.0  # every group's maximum is 7, so its scale is exactly 2^e
    e = rng.integers(-8, -2, (N, K // 64)).astype(np.float64)
    W = (q * np.repeat(2.0 ** e, 64, axis=1)).astype(np.float32)
    Wb = O.f32_to_bf16(W)
    assert np.array_equal(O.bf16_to_f32(Wb), W)
    X = O.f32_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    b = O.f32_to_bf16(rng.standard_normal(N).astype(np.float32))
    ops = O.prepare_w4a16(Wb, b, np.zeros(K, np.float32))  # a = 0 -> lam = 1
    assert np.all(ops["inv_lambda"] == 1.0)
    Y = O.linear_w4a16(X, ops)["Y"]
    np.testing.assert_allclose(Y, O.exact_linear(X, Wb, b), rtol=1e-12, atol=1e-12)


def test_w4a16_brute_force_loops():
    """The forward restated as plain loops over (m, n, group, k) on the unpacked codes, in another
    order than the library matmul: bf16 activations times code times group scale, plus bias."""
    rng = np.random.default_rng(22)
    M, K, N = 3, 128, 4
    X = O.f32_to_bf16((rng.standard_normal((M, K)) * 3).astype(np.float32))
    W = O.f32_to_bf16((rng.standard_normal((N, K)) * 0.05).astype(np.float32))
    b = O.f32_to_bf16(rng.standard_normal(N).astype(np.float32))
    a = (np.abs(rng.standard_normal(K)) + 0.1).astype(np.float32)
    ops = O.prepare_w4a16(W, b, a)
    out = O.linear_w4a16(X, ops)
    nib = O.unpack_nibbles(ops["codes_w"])
    qv = np.where(nib >= 8, nib.astype(np.int64) - 16, nib.astype(np.int64))
    xb = O.bf16_to_f32(out["x_hat_bf16"])
    bias = O.bf16_to_f32(b)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for g in range(K // 64):
                part = 0.0
                for k in range(g * 64 + 63, g * 64 - 1, -1):
                    part += float(xb[m, k]) * float(qv[n, k])
                acc += float(ops["scales_w"][n, g]) * part
            acc += float(bias[n])
            assert abs(acc - out["Y"][m, n]) <= 1e-12 * max(1.0, abs(acc))
    # the 16-bit activations are bf16 of the fp32 smoothed activations
    assert np.array_equal(out["x_hat_bf16"], O.f32_to_bf16(O.smooth_activations(X, ops["inv_lambda"])))


def test_w4a16_smoothing_reduces_error_on_outlier_data():
    """The pages use the W4A16 family for precision-sensitive layers; with the reading's
    smoothing, the weight error that multiplies the outlier channels shrinks by lam, so on outlier
    data the smoothed layer is closer to X W^T + b than the plain one."""
    import synth

    spec = synth.get("tiny_256x512x512_r16")
    X = synth.activations_bf16(spec)
    W = synth.weight_bf16(spec)
    b = synth.bias_bf16(spec)
    exact = O.exact_linear(X, W, b)
    a = np.max(np.abs(O.bf16_to_f32(X)), axis=0)
    e_plain = O.rel_fro(O.linear_w4a16(X, O.prepare_w4a16(W, b, np.zeros_like(a)))["Y"], exact)
    e_smooth = O.rel_fro(O.linear_w4a16(X, O.prepare_w4a16(W, b, a))["Y"], exact)
    assert e_smooth < 0.75 * e_plain, (e_smooth, e_plain)


def test_pages_quantization_config_matches_oracle_groups():
    with open(os.path.join(HERE, "golden", "quantization_config.json")) as f:
        cfg = json.load(f)
    assert cfg["svdq_w4a4"]["precision"] == O.NVFP4
    assert O.GROUP[O.NVFP4] == cfg["svdq_w4a4"]["group_size"] == 16
    assert cfg["svdq_w4a4"]["rank"] == 32
    assert O.GROUP[O.INT4] == 64


# ---------------------------------------------------------------- fused QKV + RMS norm + rotary


def _qkv(M, H, D, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((M, 3 * H * D)) * rng.uniform(0.1, 10.0, size=(M, 1))


def _parts(Y, H, D):
    M = Y.shape[0]
    return [Y[:, i * H * D:(i + 1) * H * D].reshape(M, H, D) for i in range(3)]


def test_qkv_norm_unit_mean_square_and_v_untouched():
    """Weight 1, eps 0, no turn: every Q and K head has mean square exactly 1 and V is Y's."""
    M, H, D = 5, 3, 16
    Y = _qkv(M, H, D, 1)
    one = np.ones(D)
    z = np.zeros((M, D // 2))
    out = O.qkv_norm_rope(Y, D, one, one, np.ones((M, D // 2)), z, eps=0.0)
    q, k, v = _parts(out, H, D)
    assert np.allclose(np.mean(q * q, axis=-1), 1.0, rtol=0, atol=1e-13)
    assert np.allclose(np.mean(k * k, axis=-1), 1.0, rtol=0, atol=1e-13)
    assert np.array_equal(v, _parts(Y, H, D)[2])


def test_qkv_norm_scale_invariance():
    """With eps 0 the normalization forgets each head's scale; V keeps it."""
    M, H, D = 4, 2, 8
    Y = _qkv(M, H, D, 2)
    rng = np.random.default_rng(3)
    gq, gk = rng.uniform(0.5, 1.5, D), rng.uniform(0.5, 1.5, D)
    ang = rng.uniform(-np.pi, np.pi, (M, D // 2))
    a = O.qkv_norm_rope(Y, D, gq, gk, np.cos(ang), np.sin(ang), eps=0.0)
    b = O.qkv_norm_rope(7.5 * Y, D, gq, gk, np.cos(ang), np.sin(ang), eps=0.0)
    qa, ka, va = _parts(a, H, D)
    qb, kb, vb = _parts(b, H, D)
    assert np.allclose(qa, qb, rtol=1e-13, atol=0) and np.allclose(ka, kb, rtol=1e-13, atol=0)
    assert np.allclose(vb, 7.5 * va, rtol=1e-15, atol=0)


def test_qkv_norm_eps_closed_form():
    """A head of constant value c: mean square c^2, so each channel becomes c / sqrt(c^2 + eps);
    with c = 1e-3 and eps = 1e-6 that is 1/sqrt(2) (eps under the root, added to the mean)."""
    M, H, D = 1, 1, 8
    Y = np.full((M, 3 * D), 1e-3)
    out = O.qkv_norm_rope(Y, D, np.ones(D), np.ones(D), np.ones((M, D // 2)), np.zeros((M, D // 2)), eps=1e-6)
    assert np.allclose(out[:, :2 * D], 1.0 / math.sqrt(2.0), rtol=1e-14, atol=0)


def test_qkv_norm_weight_is_per_channel():
    """A one-hot norm weight keeps only its channel, at y_j / rms(y); Q and K use their own weights."""
    M, H, D = 3, 2, 8
    Y = _qkv(M, H, D, 4)
    eq, ek = np.zeros(D), np.zeros(D)
    eq[5], ek[2] = 1.0, 1.0
    out = O.qkv_norm_rope(Y, D, eq, ek, np.ones((M, D // 2)), np.zeros((M, D // 2)), eps=0.0)
    q, k, _ = _parts(out, H, D)
    yq, yk, _ = _parts(Y, H, D)
    for got, y, j in ((q, yq, 5), (k, yk, 2)):
        rms = np.sqrt(np.mean(y * y, axis=-1))
        assert np.count_nonzero(np.delete(got, j, axis=-1)) == 0
        assert np.allclose(got[..., j], y[..., j] / rms, rtol=1e-14, atol=0)


def test_rotary_quarter_turn_pairs_adjacent_channels():
    """Head = e_{2i}; a quarter turn of pair i (cos 0, sin 1) moves it to e_{2i+1}: the pairs are
    adjacent channels and the turn goes from the first channel of a pair towards the second."""
    D, i = 8, 2
    Y = np.zeros((1, 3 * D))
    Y[0, 2 * i] = 1.0          # Q head 0
    Y[0, D + 2 * i + 1] = 1.0  # K head 0: e_{2i+1} goes to -e_{2i}
    cos = np.ones((1, D // 2))
    sin = np.zeros((1, D // 2))
    cos[0, i], sin[0, i] = 0.0, 1.0
    out = O.qkv_norm_rope(Y, D, np.ones(D), np.ones(D), cos, sin, eps=0.0)
    s = math.sqrt(D)  # a one-hot head has mean square 1/D
    want_q = np.zeros(D)
    want_q[2 * i + 1] = s
    want_k = np.zeros(D)
    want_k[2 * i] = -s
    assert np.allclose(out[0, :D], want_q, rtol=0, atol=1e-15)
    assert np.allclose(out[0, D:2 * D], want_k, rtol=0, atol=1e-15)


def test_rotary_is_complex_multiplication():
    """Each pair (a, b) read as the complex number a + ib is multiplied by exp(i theta)."""
    M, H, D = 6, 2, 16
    Y = _qkv(M, H, D, 5)
    ang = np.random.default_rng(6).uniform(-np.pi, np.pi, (M, D // 2))
    one = np.ones(D)
    normed = O.qkv_norm_rope(Y, D, one, one, np.ones_like(ang), np.zeros_like(ang), eps=0.0)
    turned = O.qkv_norm_rope(Y, D, one, one, np.cos(ang), np.sin(ang), eps=0.0)
    for part in (0, 1):
        n = _parts(normed, H, D)[part]
        t = _parts(turned, H, D)[part]
        z = (n[..., 0::2] + 1j * n[..., 1::2]) * np.exp(1j * ang)[:, None, :]
        assert np.allclose(t[..., 0::2], z.real, rtol=0, atol=1e-13)
        assert np.allclose(t[..., 1::2], z.imag, rtol=0, atol=1e-13)


def test_rotary_turn_back_restores_the_normalized_heads():
    """Weight 1 and eps 0: the output heads already have mean square 1, so applying the operator
    again with the opposite angles gives the normalized input back."""
    M, H, D = 4, 3, 8
    Y = _qkv(M, H, D, 7)
    ang = np.random.default_rng(8).uniform(-np.pi, np.pi, (M, D // 2))
    one = np.ones(D)
    fwd = O.qkv_norm_rope(Y, D, one, one, np.cos(ang), np.sin(ang), eps=0.0)
    back = O.qkv_norm_rope(fwd, D, one, one, np.cos(ang), -np.sin(ang), eps=0.0)
    normed = O.qkv_norm_rope(Y, D, one, one, np.ones_like(ang), np.zeros_like(ang), eps=0.0)
    assert np.allclose(back, normed, rtol=0, atol=1e-13)


def test_rotary_scores_depend_on_relative_position_only():
    """With angles pos * omega_i, the dot product of a turned query at position m and a turned key
    at position n depends on m - n only (the property rotary embeddings are built for)."""
    D, H = 16, 1
    omega = 10000.0 ** (-np.arange(0, D, 2) / D)
    rng = np.random.default_rng(9)
    qk = rng.standard_normal((1, 3 * H * D))
    Y = np.repeat(qk, 4, axis=0)
    pos = np.array([3.0, 11.0, 3.0 + 5.0, 11.0 + 5.0])  # (m, n) and (m + 5, n + 5)
    ang = pos[:, None] * omega[None, :]
    g = rng.uniform(0.5, 1.5, D)
    out = O.qkv_norm_rope(Y, D, g, g, np.cos(ang), np.sin(ang))
    q = out[:, :D]
    k = out[:, D:2 * D]
    s1 = float(q[0] @ k[1])
    s2 = float(q[2] @ k[3])
    assert abs(s1 - s2) <= 1e-12 * max(1.0, abs(s1))
    assert abs(float(q[0] @ k[0]) - float(q[1] @ k[1])) <= 1e-12 * max(1.0, abs(float(q[0] @ k[0])))


# ---------------------------------------------------------------- fused GELU/MLP pair


def test_gelu_textbook_values():
    """GELU(x) = x Phi(x) at values of the standard normal distribution function from tables."""
    table = {1.0: 0.8413447460685429, 2.0: 0.9772498680518208, -0.5: 0.3085375387259869,
             -1.96: 0.024997895148220435, 0.0: 0.5}
    for x, phi in table.items():
        assert abs(float(O.gelu(np.array([x]))[0]) - x * phi) <= 1e-15 * max(1.0, abs(x))


def test_gelu_odd_part_is_the_identity():
    """Phi(x) + Phi(-x) = 1, so GELU(x) - GELU(-x) = x."""
    x = np.random.default_rng(12).standard_normal(1000) * 5
    assert np.allclose(O.gelu(x) - O.gelu(-x), x, rtol=0, atol=1e-14 * 20)


def test_gelu_against_integrated_density():
    """Phi(x) = 1/2 + the integral of the normal density from 0 to x (composite Simpson rule)."""
    for x in (-3.7, -1.2, -0.3, 0.4, 1.5, 3.1):
        n = 2000
        t = np.linspace(0.0, x, n + 1)
        f = np.exp(-0.5 * t * t) / math.sqrt(2 * math.pi)
        h = x / n
        integral = h / 3 * (f[0] + f[-1] + 4 * f[1:-1:2].sum() + 2 * f[2:-1:2].sum())
        assert abs(float(O.gelu(np.array([x]))[0]) - x * (0.5 + integral)) <= 1e-12


def test_gelu_minimum():
    """GELU has one minimum, where Phi(x) + x phi(x) = 0 (x ~ -0.7518); neighbours lie above it."""
    lo, hi = -1.0, -0.5
    for _ in range(80):  # bisection on the derivative, written with math.erf
        mid = 0.5 * (lo + hi)
        d = 0.5 * (1 + math.erf(mid / math.sqrt(2))) + mid * math.exp(-0.5 * mid * mid) / math.sqrt(2 * math.pi)
        lo, hi = (mid, hi) if d < 0 else (lo, mid)
    xs = 0.5 * (lo + hi)
    assert abs(xs + 0.7517915246935645) < 1e-12
    g = O.gelu(np.array([xs - 1e-3, xs, xs + 1e-3]))
    assert g[1] < g[0] and g[1] < g[2]


def _bf16_nearest_brute(x: float) -> int:
    """Nearest bf16 by search over every finite bf16 pattern (ties: even mantissa)."""
    pats = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        vals = (pats << np.uint32(16)).view(np.float32).astype(np.float64)
    ok = np.isfinite(vals)
    d = np.where(ok, np.abs(vals - x), np.inf)
    best = np.min(d)
    cands = pats[d == best]
    if x == 0 or np.all((cands & 0x7FFF) == 0):  # x itself, or its nearest, is zero: zero of x's sign
        return 0x8000 if math.copysign(1.0, x) < 0 else 0
    even = cands[(cands & 1) == 0]
    pick = even if len(even) else cands
    # the pattern with the sign of x
    pick = [int(c) for c in pick if ((c >> 15) & 1) == (1 if x < 0 else 0)] or [int(pick[0])]
    return pick[0]


def test_f64_to_bf16_single_rounding():
    rng = np.random.default_rng(13)
    x = np.concatenate([rng.standard_normal(40) * 10.0 ** rng.integers(-8, 8, 40),
                        [9.031250271464623, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 3.0, -0.0]])
    got = O.f64_to_bf16(x)
    for xi, g in zip(x, got):
        assert int(g) == _bf16_nearest_brute(float(xi)), xi
    # one step from fp64: 9.031250271... lies above the midpoint 9.03125 of (9.0, 9.0625), which an
    # fp32 intermediate would hit exactly and round to even (9.0)
    assert O.bf16_to_f32(O.f64_to_bf16(np.array([9.031250271464623])))[0] == np.float32(9.0625)
    # on fp32 inputs it agrees with the fp32 rule
    v = rng.standard_normal(5000).astype(np.float32) * 100
    assert np.array_equal(O.f64_to_bf16(v.astype(np.float64)), O.f32_to_bf16(v))


def test_gelu_bf16_every_input():
    """The bf16 GELU on all 65280 finite bf16 inputs.  (1) Wherever |y| >= 2^-125 it equals the fp64
    y Phi(y) = y erfc(-y / sqrt 2) / 2 (library erfc, relative error ~1e-15) rounded once to bf16:
    none of those exact values lies within 1e-12 (relative) of a bf16 rounding boundary, so fp64
    decides every one of them.  (2) Below that, y / 2 is exact and GELU(y) = y / 2 + y^2 / sqrt
    (2 pi) + O(y^4) lies just above it; y / 2 is a bf16 subnormal there (spacing 2^-133), so the
    result is y / 2 rounded with ties upward.  (3) The
    fp64 form 1 + erf(y / sqrt 2) cancels in the negative tail (it returns 0 below y ~ -8.3), and the
    bf16 GELU must not follow it there."""
    from scipy.special import erfc

    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    y = O.bf16_to_f32(pats).astype(np.float64)
    fin = np.isfinite(y)
    pats, y = pats[fin], y[fin]
    got = O.gelu_bf16(pats)
    g64 = 0.5 * y * erfc(-y / math.sqrt(2.0))
    normal = np.abs(y) >= 2.0 ** -125
    assert np.array_equal(got[normal], O.f64_to_bf16(g64[normal]))
    sub = ~normal & (y != 0)
    half = y[sub] / 2  # exact: a multiple of 2^-134
    k = half / 2.0 ** -133  # in units of the bf16 subnormal spacing
    expect = np.where(k - np.floor(k) == 0.5, np.ceil(k), np.round(k)) * 2.0 ** -133
    assert np.array_equal(O.bf16_to_f32(got[sub]).astype(np.float64), expect)
    assert np.all(O.bf16_to_f32(got[y == 0]) == 0)
    assert list(O.gelu_bf16(np.array([0x0000, 0x8000], np.uint16))) == [0x0000, 0x8000]  # sign of zero kept
    tail = (y < -8.5) & (y > -13.0)
    assert np.all(O.bf16_to_f32(got[tail]) < 0)  # small but not zero
    assert np.all(0.5 * y[tail] * (1.0 + np.array([math.erf(v / math.sqrt(2.0)) for v in y[tail]])) == 0)


def test_mlp_pair_is_the_module_sequence():
    """On layers quantized losslessly (lam = 1, r = 0, on-grid operands) the up layer's output is
    the exact product; the pair must then be: round to bf16, GELU, round to bf16, down layer."""
    rng = np.random.default_rng(14)
    M, K, H, N = 4, 64, 64, 48
    v, _, _ = _random_on_grid_nvfp4(rng, M, K, 0x20, 0x50)
    wu, _, _ = _random_on_grid_nvfp4(rng, H, K, 0x20, 0x50)
    wd, _, _ = _random_on_grid_nvfp4(rng, N, H, 0x20, 0x50)
    xb = O.f32_to_bf16(v)
    bu = O.f32_to_bf16(rng.standard_normal(H).astype(np.float32))
    bd = O.f32_to_bf16(rng.standard_normal(N).astype(np.float32))

    def ops(w, b, k):
        cw, sw = O.quantize_rows(w, O.NVFP4)
        return {"inv_lambda": np.ones(k, np.float32), "codes_w": cw, "scales_w": sw,
                "L1": np.zeros((k, 0), np.uint16), "L2": np.zeros((0, w.shape[0]), np.uint16), "bias": b}

    out = O.mlp_pair(xb, ops(wu, bu, K), ops(wd, bd, H), O.NVFP4)
    y_up = v.astype(np.float64) @ wu.astype(np.float64).T + O.bf16_to_f32(bu)[None, :]
    assert np.array_equal(out["Y_up"], y_up)
    h = np.zeros((M, H), np.uint16)
    for m in range(M):
        for j in range(H):
            a = float(O.bf16_to_f32(np.array([_bf16_nearest_brute(float(y_up[m, j]))], np.uint16))[0])
            g = a * 0.5 * math.erfc(-a / math.sqrt(2.0))  # Phi without 1 + erf's cancellation
            h[m, j] = _bf16_nearest_brute(g)
    assert np.array_equal(out["h_bf16"], h)
    down = O.linear(h, ops(wd, bd, H), O.NVFP4)
    assert np.array_equal(out["Y"], down["Y"]) and np.array_equal(out["codes_h"], down["codes_x"])
