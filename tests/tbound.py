"""Per-element tolerance for the low-rank down projection T = bf16(x_hat) L1 (bf16 output).

The GPU sums the K products in fp32 (tensor-core accumulation, then the K-split slices in a
fixed order); the oracle sums them exactly.  Any order of K - 1 fp32 additions, each off by at
most one fp32 ulp (2^-23 relative, which also covers an accumulator that truncates), is within
err = K * 2^-23 * sum_k |bf16(x_hat[m,k])| |L1[k,i]| of the exact sum.  Both sides then round to
bf16, so |T_gpu - T_ref| <= ulp_bf16(|T| + err) + err element by element.
"""
import numpy as np


def ulp_bf16(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at magnitude v (2^(e - 8) for v in [2^(e-1), 2^e)); subnormal floor."""
    v = np.abs(np.asarray(v, dtype=np.float64))
    _, e = np.frexp(v)
    return np.where(v > 0, np.ldexp(1.0, e - 8), 0.0) + 2.0 ** -133


def t_bound(xb: np.ndarray, L1: np.ndarray, T_ref: np.ndarray) -> np.ndarray:
    """Elementwise bound on |T_gpu - T_ref|: xb = bf16(x_hat) as float, L1 as float (K x r)."""
    K = xb.shape[1]
    err = K * 2.0 ** -23 * (np.abs(xb.astype(np.float64)) @ np.abs(L1.astype(np.float64)))
    return ulp_bf16(np.abs(T_ref) * (1 + 2.0 ** -8) + err) + err


def assert_t_close(T_gpu: np.ndarray, T_ref: np.ndarray, xb: np.ndarray, L1: np.ndarray):
    bound = t_bound(xb, L1, T_ref)
    diff = np.abs(T_gpu - T_ref)
    bad = diff > bound
    assert not bad.any(), (int(bad.sum()), float(diff[bad].max()), float(bound[bad].min()))
