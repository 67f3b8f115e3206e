"""CPU oracle for the SVDQuant W4A4 rank-corrected smoothed linear layer.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  The product path (the
C-ABI library and its kernels) never calls it, and the two share no code.

Plain, slow and obviously correct: numpy, fp64 wherever the method does not
fix a precision, fp32 where the quantizer's decisions are taken (so that the
4-bit codes are decided exactly as the kernels must decide them).

What is computed, and where it comes from
-----------------------------------------
SVDQuant model card (huggingface mit-han-lab/svdq-int4-flux.1-depth-dev),
section "Quantization Method -- SVDQuant", figure caption stages 1-3:
  stage 2  outliers migrate from activations into weights:
           X_hat = X diag(lam)^-1,   W_hat = diag(lam) W
  stage 3  W_hat = L1 L2 + R  (rank-r SVD; the low-rank branch stays 16-bit,
           the residual R is quantized to 4 bits)
Same card, section "Nunchaku Engine Design" (a)(b): the forward is
  Y = Q4(X_hat) (x) Q4(R) + (X_hat L1) L2 + b
computed as "Quantize"+"Down Projection" on the input and
"4-Bit Compute"+"Up Projection" on the output.
"Nunchaku in Diffusers" blog, section "Native loading in Diffusers",
``quantization_config``: svdq_w4a4 precision nvfp4, group_size 16, rank 32,
compute_dtype bfloat16; section "Introducing Nunchaku Lite": INT4 and NVFP4
variants of the svdq_w4a4 kernel family.

Readings where the pages are silent:
  R1 lam_k = a_k^alpha * w_k^(alpha-1) with alpha = 0.5, i.e. sqrt(a_k / w_k),
     a_k = max_m |X[m,k]|, w_k = max_n |W[n,k]|; lam_k = 1 if a_k or w_k is 0.
  R2 X_hat = fp32(x) * fp32(1/lam): one fp32 multiply by the fp32 reciprocal.
  R3 balanced SVD split L1 = U_r sqrt(S), L2 = sqrt(S) V_r^T; the largest-|.|
     entry of each column of U_r is positive (lowest index on ties).
  R4 R = W_hat - U_r S_r V_r^T with the fp64 factors, then fp32.
  R5 L1, L2 and the branch input bf16(X_hat) are bf16 (round to nearest even);
     T = bf16(X_hat) L1 is accumulated exactly then rounded to bf16.
  R6 groups run along K.  NVFP4: group 16, scale = UE4M3(amax / 6) (RNE,
     saturating at 448, subnormals kept), code = E2M1_RNE_sat(v / scale)
     with fp32 IEEE division; a negative value whose magnitude rounds to 0
     keeps its sign (code 0b1000).  INT4: group 64, scale = fp32(amax / 7),
     code = clamp(rint_half_even(v / scale), -8, 7).  A block whose scale is
     0 stores scale 0 and all codes +0.  Single-level scaling: no per-tensor
     global scale.
  R7 packing: element 2i in bits 3:0, element 2i+1 in bits 7:4 of byte i.
  R8 output Y is returned here in fp64; the device returns bf16.
  R9 W4A16 (the "awq_w4a16" family of "Introducing Nunchaku Lite" and the
     quantization_config of "Native loading in Diffusers": precision int4,
     group_size 64, 4-bit weights with 16-bit activations): the pages fix only
     the weight format.  Reading: the same smoothing as R1; the smoothed weight
     W_hat is quantized per row with R6's INT4 quantizer (no low-rank branch);
     the 16-bit activations are bf16(X_hat) with X_hat as in R2; the output is
     bf16(X_hat) dequant(Q4(W_hat))^T + b (exact here, fp32 on a device).
  R10 fused QKV + Q/K normalization + rotary embedding ("Bringing Nunchaku
     4-bit Diffusion Inference to Diffusers", section "Quantizing models with
     structural rewrites": one operator consumes the grouped QKV projection,
     norm_q, norm_k and the rotary embedding; Q, K and V are concatenated along
     the output dimension in that order).  The pages name the steps only.
     Reading: the layer output Y (before its rounding to bf16) splits into Q, K
     and V of H heads of D channels each; every head vector of Q and K is
     divided by sqrt(mean of its squares + eps) and multiplied by the norm's
     per-channel weight (RMS normalization; eps = 1e-6); then channels 2i and
     2i+1 of the head are turned as one pair by the angle of (row m, pair i),
     given as cos and sin tables (out_2i = a cos - b sin, out_2i+1 = a sin +
     b cos); V passes unchanged; one rounding to bf16 at the end.
  R11 fused GELU/MLP ("Introducing Nunchaku Lite": the engine's fused GELU/MLP
     kernels; the pages give no formula).  Reading: the fused pair computes what
     the unfused modules compute -- the up layer's output rounded to bf16, GELU
     of it (x Phi(x), Phi the standard normal distribution function) rounded to
     bf16, and that hidden activation as the down layer's input; fusing only
     removes the hidden tensor's round trip through memory.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Tuple

import numpy as np

NVFP4 = "nvfp4"
INT4 = "int4"
GROUP = {NVFP4: 16, INT4: 64}

# ---------------------------------------------------------------------------
# bf16 <-> fp32 (own helpers; the oracle imports nothing from the product)
# ---------------------------------------------------------------------------


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32 values (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (finite inputs).

    Written as the value-level rule rather than a bit trick: the two bf16
    neighbours of x are found by truncation, and the nearer one wins; a tie
    picks the one whose last mantissa bit is 0.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    lo = (bits >> np.uint32(16)).astype(np.uint32)  # truncation toward zero (magnitude)
    hi = lo + np.uint32(1)
    v_lo = (lo << np.uint32(16)).view(np.float32).astype(np.float64)
    v_hi = (hi << np.uint32(16)).view(np.float32).astype(np.float64)
    xv = x.astype(np.float64)
    d_lo = np.abs(xv - v_lo)
    d_hi = np.abs(v_hi - xv)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((lo & np.uint32(1)) == np.uint32(1)))
    return np.where(pick_hi, hi, lo).astype(np.uint16)


# ---------------------------------------------------------------------------
# 4-bit and 8-bit number formats (definitions, by value tables)
# ---------------------------------------------------------------------------

# E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit.  Code c (0..7) magnitude:
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def ue4m3_value(code: np.ndarray) -> np.ndarray:
    """Unsigned E4M3 (4 exponent bits, bias 7, 3 mantissa bits) -> value (fp64).

    exponent field 0 is subnormal: m/8 * 2^-6.  Code 0x7F is NaN (not used);
    the largest finite value is 0x7E = 1.75 * 2^8 = 448.
    """
    c = np.asarray(code, dtype=np.int64)
    e = (c >> 3) & 0xF
    m = c & 0x7
    sub = m / 8.0 * 2.0 ** -6
    nrm = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    return np.where(e == 0, sub, nrm)


_UE4M3_TABLE = ue4m3_value(np.arange(0x7F))  # finite codes 0..0x7E, increasing


def _nearest_even(x: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the table value nearest to x (table increasing, x >= 0),
    ties to the even index, x above the last entry saturates to it."""
    x = np.asarray(x, dtype=np.float64)
    idx_hi = np.searchsorted(table, x, side="left")  # first entry >= x
    idx_hi = np.minimum(idx_hi, len(table) - 1)
    idx_lo = np.maximum(idx_hi - 1, 0)
    d_lo = np.abs(x - table[idx_lo])
    d_hi = np.abs(table[idx_hi] - x)
    pick = np.where(d_lo < d_hi, idx_lo,
                    np.where(d_hi < d_lo, idx_hi, np.where(idx_lo % 2 == 0, idx_lo, idx_hi)))
    pick = np.where(x >= table[-1], len(table) - 1, pick)
    return pick.astype(np.int64)


def ue4m3_encode(s: np.ndarray) -> np.ndarray:
    """fp32 s >= 0 -> UE4M3 byte: round to nearest even, saturate to 448 (R6)."""
    s = np.asarray(s, dtype=np.float32)
    return _nearest_even(s.astype(np.float64), _UE4M3_TABLE).astype(np.uint8)


def e2m1_encode(q: np.ndarray) -> np.ndarray:
    """fp32 q -> E2M1 nibble (sign in bit 3): RNE on the magnitude grid,
    saturating at 6; the sign bit follows the sign of q (R6)."""
    q = np.asarray(q, dtype=np.float32)
    mag = _nearest_even(np.abs(q).astype(np.float64), E2M1_GRID)
    sign = np.signbit(q).astype(np.int64)
    return (mag | (sign << 3)).astype(np.uint8)


def e2m1_value(nib: np.ndarray) -> np.ndarray:
    n = np.asarray(nib, dtype=np.int64)
    v = E2M1_GRID[n & 7]
    return np.where((n & 8) != 0, -v, v)


def int4_value(nib: np.ndarray) -> np.ndarray:
    n = np.asarray(nib, dtype=np.int64) & 0xF
    return np.where(n >= 8, n - 16, n).astype(np.float64)


def pack_nibbles(nib: np.ndarray) -> np.ndarray:
    """[rows, K] nibbles -> [rows, K/2] bytes; element 2i low nibble (R7)."""
    nib = np.asarray(nib, dtype=np.uint8) & np.uint8(0xF)
    return (nib[:, 0::2] | (nib[:, 1::2] << np.uint8(4))).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & np.uint8(0xF)
    out[:, 1::2] = p >> np.uint8(4)
    return out


# ---------------------------------------------------------------------------
# Group quantizer Q (R6): identical for weight rows of R and activation rows.
# "Quantize" kernel of the engine design; 4-bit residual of stage 3.
# ---------------------------------------------------------------------------


def quantize_rows(v: np.ndarray, precision: str) -> Tuple[np.ndarray, np.ndarray]:
    """Quantize each row of ``v`` (fp32, [rows, K]) in groups along K.

    Returns (codes [rows, K/2] uint8 packed, scales): NVFP4 scales are UE4M3
    bytes [rows, K/16]; INT4 scales are fp32 [rows, K/64].
    """
    v = np.ascontiguousarray(v, dtype=np.float32)
    rows, K = v.shape
    G = GROUP[precision]
    assert K % G == 0
    blocks = v.reshape(rows, K // G, G)
    amax = np.max(np.abs(blocks), axis=2)  # exact in fp32
    if precision == NVFP4:
        s = (amax / np.float32(6.0)).astype(np.float32)  # fp32 IEEE divide
        sbyte = ue4m3_encode(s)
        s_d = ue4m3_value(sbyte).astype(np.float32)  # decoded scale, exact in fp32
        zero_blk = s_d == 0
        safe = np.where(zero_blk, np.float32(1.0), s_d).astype(np.float32)
        q = (blocks / safe[:, :, None]).astype(np.float32)  # fp32 IEEE divide
        nib = e2m1_encode(q)
        nib = np.where(zero_blk[:, :, None], np.uint8(0), nib)
        return pack_nibbles(nib.reshape(rows, K)), sbyte
    if precision == INT4:
        s = (amax / np.float32(7.0)).astype(np.float32)
        zero_blk = s == 0
        safe = np.where(zero_blk, np.float32(1.0), s).astype(np.float32)
        q = (blocks / safe[:, :, None]).astype(np.float32)
        qi = np.clip(np.rint(q), -8, 7).astype(np.int64)  # rint: half to even
        qi = np.where(zero_blk[:, :, None], 0, qi)
        nib = (qi & 0xF).astype(np.uint8)
        return pack_nibbles(nib.reshape(rows, K)), s
    raise ValueError(precision)


def dequantize_rows(codes: np.ndarray, scales: np.ndarray, precision: str) -> np.ndarray:
    """Exact fp64 value of each quantized element: code value x group scale."""
    nib = unpack_nibbles(codes)
    rows, K = nib.shape
    G = GROUP[precision]
    if precision == NVFP4:
        vals = e2m1_value(nib)
        sc = ue4m3_value(scales)
    else:
        vals = int4_value(nib)
        sc = np.asarray(scales, dtype=np.float32).astype(np.float64)
    return (vals.reshape(rows, K // G, G) * sc[:, :, None]).reshape(rows, K)


# ---------------------------------------------------------------------------
# Offline prepare: smoothing (stage 2) and SVD (stage 3)
# ---------------------------------------------------------------------------


def smoothing_factors(a: np.ndarray, W: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """lam_k from the activation channel maxima a_k and W's column maxima (R1).

    W is fp64 [N, K] (nn.Linear layout); returns fp64 lam [K].
    """
    a = np.asarray(a, dtype=np.float64)
    w = np.max(np.abs(np.asarray(W, dtype=np.float64)), axis=0)
    lam = np.ones_like(a)
    ok = (a > 0) & (w > 0)
    if alpha == 0.5:
        lam[ok] = np.sqrt(a[ok] / w[ok])
    else:
        lam[ok] = a[ok] ** alpha * w[ok] ** (alpha - 1.0)
    return lam


def inv_lambda_f32(lam: np.ndarray) -> np.ndarray:
    """fp32(1/lam) (R2)."""
    return (1.0 / np.asarray(lam, dtype=np.float64)).astype(np.float32)


def smooth_weight(W: np.ndarray, lam: np.ndarray) -> np.ndarray:
    """W_hat[n, k] = W[n, k] * lam_k in fp64 (stage 2: diag(lam) W in K x N form)."""
    return np.asarray(W, dtype=np.float64) * np.asarray(lam, dtype=np.float64)[None, :]


def svd_split(W_hat_nk: np.ndarray, r: int):
    """Top-r SVD of the smoothed weight (stage 3), balanced split (R3).

    Works on the K x N orientation of the formula: W_hat_kn = U S V^T,
    L1 = U_r sqrt(S_r) (K x r), L2 = sqrt(S_r) V_r^T (r x N).
    Returns (L1, L2, sigma_all, U_r, S_r, Vt_r), all fp64.
    """
    Wkn = np.asarray(W_hat_nk, dtype=np.float64).T
    U, S, Vt = np.linalg.svd(Wkn, full_matrices=False)  # library primitive
    K, N = Wkn.shape
    r = min(r, len(S))
    U_r = U[:, :r].copy()
    Vt_r = Vt[:r, :].copy()
    for i in range(r):
        j = int(np.argmax(np.abs(U_r[:, i])))  # lowest index among equal maxima
        if U_r[j, i] < 0:
            U_r[:, i] = -U_r[:, i]
            Vt_r[i, :] = -Vt_r[i, :]
    S_r = S[:r].copy()
    rs = np.sqrt(S_r)
    L1 = U_r * rs[None, :]
    L2 = rs[:, None] * Vt_r
    return L1, L2, S, U_r, S_r, Vt_r


def residual_f32(W_hat_nk: np.ndarray, U_r: np.ndarray, S_r: np.ndarray, Vt_r: np.ndarray) -> np.ndarray:
    """R (N x K, fp32) = W_hat - (U_r S_r V_r^T)^T with the fp64 factors (R4)."""
    low_kn = (U_r * S_r[None, :]) @ Vt_r if len(S_r) else 0.0
    R_nk = np.asarray(W_hat_nk, dtype=np.float64) - (np.asarray(low_kn).T if len(S_r) else 0.0)
    return np.asarray(R_nk, dtype=np.float64).astype(np.float32)


def prepare(W_bf16: np.ndarray, bias_bf16: Optional[np.ndarray], a: np.ndarray, precision: str,
            rank: int, alpha: float = 0.5) -> Dict[str, np.ndarray]:
    """Offline prepare: smoothing, SVD split, residual quantization.

    Returns the canonical operands: inv_lambda fp32 [K], codes_w [N, K/2],
    scales_w, L1 bf16 [K, r], L2 bf16 [r, N], bias bf16 [N], plus fp64
    diagnostics (lam, sigma, R).
    """
    W = bf16_to_f32(W_bf16).astype(np.float64)
    N, K = W.shape
    lam = smoothing_factors(a, W, alpha)
    W_hat = smooth_weight(W, lam)
    if rank > 0:
        L1, L2, sigma, U_r, S_r, Vt_r = svd_split(W_hat, rank)
        R = residual_f32(W_hat, U_r, S_r, Vt_r)
    else:
        sigma = np.zeros(0)
        L1 = np.zeros((K, 0))
        L2 = np.zeros((0, N))
        R = W_hat.astype(np.float32)
    codes_w, scales_w = quantize_rows(R, precision)
    bias = np.zeros(N, dtype=np.uint16) if bias_bf16 is None else np.asarray(bias_bf16, dtype=np.uint16)
    return {
        "lam": lam,
        "inv_lambda": inv_lambda_f32(lam),
        "sigma": sigma,
        "L1_f64": L1,
        "L2_f64": L2,
        "L1": f32_to_bf16(L1.astype(np.float32)),
        "L2": f32_to_bf16(L2.astype(np.float32)),
        "R": R,
        "codes_w": codes_w,
        "scales_w": scales_w,
        "bias": bias,
    }


# ---------------------------------------------------------------------------
# Forward: "Quantize"+"Down Projection", then "4-Bit Compute"+"Up Projection"
# ---------------------------------------------------------------------------


def smooth_activations(X_bf16: np.ndarray, inv_lambda: np.ndarray) -> np.ndarray:
    """X_hat = fp32(x) * inv_lambda_k, one fp32 multiply per element (R2)."""
    x = bf16_to_f32(X_bf16)
    return (x * np.asarray(inv_lambda, dtype=np.float32)[None, :]).astype(np.float32)


def quantize_activations(X_bf16: np.ndarray, inv_lambda: np.ndarray, precision: str):
    """Per-token, per-K-group activation quantization ("Quantize")."""
    xh = smooth_activations(X_bf16, inv_lambda)
    codes, scales = quantize_rows(xh, precision)
    return xh, codes, scales


def lowrank_down(x_hat_f32: np.ndarray, L1_bf16: np.ndarray) -> np.ndarray:
    """T = bf16(X_hat) L1, exact fp64 sum, rounded to bf16 (R5) ("Down Projection")."""
    r = L1_bf16.shape[1] if np.ndim(L1_bf16) == 2 else 0
    if r == 0:
        return np.zeros((x_hat_f32.shape[0], 0), dtype=np.uint16)
    xb = bf16_to_f32(f32_to_bf16(x_hat_f32)).astype(np.float64)
    T = xb @ bf16_to_f32(L1_bf16).astype(np.float64)
    return f32_to_bf16(T.astype(np.float32))


def gemm_4bit(codes_x, scales_x, codes_w, scales_w, precision: str) -> np.ndarray:
    """acc[m, n] = sum_g s_x[m,g] s_w[n,g] sum_{k in g} q_x[m,k] q_w[n,k]  ("4-Bit Compute").

    Every dequantized element (code value x scale) is exact in fp64, so the
    grouped sum equals the fp64 product of the dequantized operands; the
    product is taken with a library matmul.
    """
    A = dequantize_rows(codes_x, scales_x, precision)
    B = dequantize_rows(codes_w, scales_w, precision)
    return A @ B.T


def forward(codes_x, scales_x, T_bf16, codes_w, scales_w, L2_bf16, bias_bf16, precision: str) -> np.ndarray:
    """Y (fp64) = 4-bit GEMM + T L2 + b  ("4-Bit Compute" + "Up Projection")."""
    Y = gemm_4bit(codes_x, scales_x, codes_w, scales_w, precision)
    if np.ndim(T_bf16) == 2 and T_bf16.shape[1] > 0:
        Y = Y + bf16_to_f32(T_bf16).astype(np.float64) @ bf16_to_f32(L2_bf16).astype(np.float64)
    if bias_bf16 is not None:
        Y = Y + bf16_to_f32(bias_bf16).astype(np.float64)[None, :]
    return Y


def linear(X_bf16: np.ndarray, ops: Dict[str, np.ndarray], precision: str) -> Dict[str, np.ndarray]:
    """The whole hot path on prepared operands ``ops`` (keys as ``prepare`` returns)."""
    xh, cx, sx = quantize_activations(X_bf16, ops["inv_lambda"], precision)
    T = lowrank_down(xh, ops["L1"])
    Y = forward(cx, sx, T, ops["codes_w"], ops["scales_w"], ops["L2"], ops["bias"], precision)
    return {"x_hat": xh, "codes_x": cx, "scales_x": sx, "T": T, "Y": Y}


# ---------------------------------------------------------------------------
# W4A16 ("awq_w4a16", R9): 4-bit weights, 16-bit activations
# ---------------------------------------------------------------------------


def prepare_w4a16(W_bf16: np.ndarray, bias_bf16: Optional[np.ndarray], a: np.ndarray,
                  alpha: float = 0.5) -> Dict[str, np.ndarray]:
    """Offline prepare of a W4A16 layer: smoothing (R1), INT4 group-64 codes and fp32 scales of
    the smoothed weight (R6), no low-rank branch.  Keys as ``prepare`` returns them."""
    return prepare(W_bf16, bias_bf16, a, INT4, 0, alpha)


def linear_w4a16(X_bf16: np.ndarray, ops: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """Y (fp64) = bf16(X_hat) dequant(Q4(W_hat))^T + b, the sum taken exactly (R9).

    Every dequantized weight (int4 code x fp32 scale) and every bf16 activation is exact in fp64;
    the product is taken with a library matmul."""
    xh = smooth_activations(X_bf16, ops["inv_lambda"])
    xb16 = f32_to_bf16(xh)
    Wd = dequantize_rows(ops["codes_w"], ops["scales_w"], INT4)
    Y = bf16_to_f32(xb16).astype(np.float64) @ Wd.T
    if ops.get("bias") is not None:
        Y = Y + bf16_to_f32(ops["bias"]).astype(np.float64)[None, :]
    return {"x_hat_bf16": xb16, "Y": Y}


# ---------------------------------------------------------------------------
# Fused QKV + RMS normalization of Q and K + rotary embedding (R10)
# ---------------------------------------------------------------------------


def rms_norm_heads(heads: np.ndarray, weight: np.ndarray, eps: float) -> np.ndarray:
    """heads [M, H, D] (fp64): each head vector over its D channels divided by the square root of
    (its mean square + eps), then multiplied channel by channel by ``weight`` [D]."""
    ms = np.mean(heads * heads, axis=-1, keepdims=True)
    return heads / np.sqrt(ms + eps) * np.asarray(weight, np.float64)[None, None, :]


def rotate_pairs(heads: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """heads [M, H, D] (fp64); channels (2i, 2i+1) of every head of row m turned by the angle
    whose cosine and sine are cos[m, i] and sin[m, i] ([M, D/2])."""
    a = heads[..., 0::2]
    b = heads[..., 1::2]
    c = np.asarray(cos, np.float64)[:, None, :]
    s = np.asarray(sin, np.float64)[:, None, :]
    out = np.empty_like(heads)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def qkv_norm_rope(Y: np.ndarray, head_dim: int, gamma_q: np.ndarray, gamma_k: np.ndarray,
                  cos: np.ndarray, sin: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """The fused operator's steps after the projection (R10), in fp64: Y [M, 3 H D] = [Q | K | V];
    Q and K normalized per head and rotated, V unchanged."""
    Y = np.asarray(Y, np.float64)
    M, N = Y.shape
    assert N % (3 * head_dim) == 0 and head_dim % 2 == 0
    H = N // (3 * head_dim)
    out = Y.copy()
    for part, gamma in ((0, gamma_q), (1, gamma_k)):
        cols = slice(part * H * head_dim, (part + 1) * H * head_dim)
        heads = Y[:, cols].reshape(M, H, head_dim)
        out[:, cols] = rotate_pairs(rms_norm_heads(heads, gamma, eps), cos, sin).reshape(M, H * head_dim)
    return out


def linear_qkv_norm_rope(X_bf16: np.ndarray, ops: Dict[str, np.ndarray], precision: str, head_dim: int,
                         gamma_q: np.ndarray, gamma_k: np.ndarray, cos: np.ndarray, sin: np.ndarray,
                         eps: float = 1e-6) -> Dict[str, np.ndarray]:
    """The grouped QKV layer followed by R10: the layer's forward (as ``linear``) and the fused
    normalization and rotation of its exact output."""
    r = linear(X_bf16, ops, precision)
    r["Y_layer"] = r["Y"]
    r["Y"] = qkv_norm_rope(r["Y"], head_dim, gamma_q, gamma_k, cos, sin, eps)
    return r


# ---------------------------------------------------------------------------
# Fused GELU/MLP pair (R11)
# ---------------------------------------------------------------------------


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns, round to nearest, ties to even, in one step (no intermediate
    fp32 rounding).  Same value-level rule as ``f32_to_bf16``: the two bf16 neighbours of x are
    found by truncating its fp32-or-wider magnitude, and the nearer one wins."""
    x = np.asarray(x, dtype=np.float64)
    t = x.astype(np.float32)
    # the fp32 nearest to x can lie on the other side of x; step back so that t is a truncation
    over = np.abs(t.astype(np.float64)) > np.abs(x)
    t = np.where(over, np.nextafter(t, np.float32(0), dtype=np.float32), t).astype(np.float32)
    lo = (np.ascontiguousarray(t).view(np.uint32) >> np.uint32(16)).astype(np.uint32)
    hi = lo + np.uint32(1)
    v_lo = (lo << np.uint32(16)).view(np.float32).astype(np.float64)
    v_hi = (hi << np.uint32(16)).view(np.float32).astype(np.float64)
    d_lo = np.abs(x - v_lo)
    d_hi = np.abs(v_hi - x)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((lo & np.uint32(1)) == np.uint32(1)))
    return np.where(pick_hi, hi, lo).astype(np.uint16)


def gelu(y: np.ndarray) -> np.ndarray:
    """GELU in fp64: y Phi(y), with Phi(y) = (1 + erf(y / sqrt 2)) / 2 (R11)."""
    from scipy.special import erf  # a library primitive for the normal distribution function

    y = np.asarray(y, dtype=np.float64)
    return 0.5 * y * (1.0 + erf(y / np.sqrt(2.0)))


_GELU_BF16 = {}


def gelu_bf16(y_bf16: np.ndarray) -> np.ndarray:
    """bf16 GELU of bf16 inputs: y Phi(y) evaluated to 50 significant digits (mpmath, with
    Phi(y) = erfc(-y / sqrt 2) / 2, free of the cancellation of 1 + erf in the negative tail) and
    rounded once to the nearest bf16, ties to even (R11).  A bf16 input has 2^16 patterns, so the
    values are computed once per distinct pattern and cached."""
    import mpmath

    y_bf16 = np.asarray(y_bf16, dtype=np.uint16)
    uniq = np.unique(y_bf16)
    _GELU_BF16[0x8000] = 0x8000  # y Phi(y) of -0 is -0 (a product with a negative zero)
    todo = [int(u) for u in uniq if int(u) not in _GELU_BF16]
    if todo:
        with mpmath.workdps(50):
            two = mpmath.mpf(2)
            for u in todo:
                y = mpmath.mpf(float(bf16_to_f32(np.array([u], np.uint16))[0]))
                _GELU_BF16[u] = _mp_to_bf16(y * mpmath.erfc(-y / mpmath.sqrt(two)) / two)
    lut = np.array([_GELU_BF16[int(u)] for u in uniq], dtype=np.uint16)
    return lut[np.searchsorted(uniq, y_bf16)]


def _mp_to_bf16(g) -> int:
    """Nearest bf16 (ties to even) of a high-precision value: 8 significant bits for normal
    magnitudes, spacing 2^-133 below 2^-126 (subnormals)."""
    import mpmath

    if g == 0:
        return 0x8000 if mpmath.sign(g) < 0 else 0
    a = abs(g)
    q = max(int(mpmath.floor(mpmath.log(a, 2))), -126) - 7  # exponent of the bf16 spacing at a
    m = a / mpmath.mpf(2) ** q  # in [2^7, 2^8) for normal a
    n = int(mpmath.floor(m))
    frac = m - n
    if frac > 0.5 or (frac == 0.5 and n % 2 == 1):
        n += 1
    bits = int(np.array([np.float32(n * 2.0 ** q)], np.float32).view(np.uint32)[0] >> 16)
    return bits | (0x8000 if g < 0 else 0)


def mlp_pair(X_bf16: np.ndarray, ops_up: Dict[str, np.ndarray], ops_down: Dict[str, np.ndarray],
             precision: str) -> Dict[str, np.ndarray]:
    """up layer -> bf16 -> GELU -> bf16 -> down layer (R11).  Returns the up layer's exact output,
    the bf16 hidden activation, the down layer's 4-bit operands and T, and Y (fp64)."""
    up = linear(X_bf16, ops_up, precision)
    y_up_bf16 = f64_to_bf16(up["Y"])
    h = gelu_bf16(y_up_bf16)
    down = linear(h, ops_down, precision)
    return {"Y_up": up["Y"], "y_up_bf16": y_up_bf16, "h_bf16": h, "codes_h": down["codes_x"],
            "scales_h": down["scales_x"], "T_h": down["T"], "Y": down["Y"]}


def exact_linear(X_bf16: np.ndarray, W_bf16: np.ndarray, bias_bf16: Optional[np.ndarray]) -> np.ndarray:
    """Unquantized fp64 reference X W^T + b (used only for the informative error report)."""
    Y = bf16_to_f32(X_bf16).astype(np.float64) @ bf16_to_f32(W_bf16).astype(np.float64).T
    if bias_bf16 is not None:
        Y = Y + bf16_to_f32(bias_bf16).astype(np.float64)[None, :]
    return Y


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(np.asarray(a, np.float64) - np.asarray(b, np.float64)) /
                 max(np.linalg.norm(np.asarray(b, np.float64)), 1e-300))


def flops(M: int, K: int, N: int, r: int) -> int:
    return 2 * M * N * K + 2 * M * r * (K + N)


__all__ = [name for name in dir() if not name.startswith("_")]
del math
