"""Python binding of the SVDQuant W4A4 linear C ABI (``include/svdq.h``).

Argument marshalling only: every step of the layer runs in the C++/CUDA library
``lib/libsvdq_b200.so``.  PyTorch supplies device memory and streams.  If the library is
missing or cannot be loaded, importing this package raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "lib", "libsvdq_b200.so")

SVDQ_NVFP4 = 0
SVDQ_INT4 = 1
SVDQ_W4A16 = 2  # 4-bit weights, 16-bit activations, no low-rank branch (rank 0)
PRECISIONS = {"nvfp4": SVDQ_NVFP4, "int4": SVDQ_INT4, "w4a16": SVDQ_W4A16}
GROUP = {SVDQ_NVFP4: 16, SVDQ_INT4: 64, SVDQ_W4A16: 64}

SVDQ_OK = 0
STATUS_NAMES = {0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_UNSUPPORTED_DEVICE", 3: "SVDQ_ERR_CUDA",
                4: "SVDQ_ERR_OOM", 5: "SVDQ_ERR_TIMEOUT", 6: "SVDQ_ERR_INTERNAL"}


class SVDQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class PrepareParams(ctypes.Structure):
    _fields_ = [("precision", ctypes.c_int), ("rank", ctypes.c_int), ("alpha", ctypes.c_float),
                ("svd_iters", ctypes.c_int), ("seed", ctypes.c_uint64)]


class WeightsInfo(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int), ("K", ctypes.c_int), ("rank", ctypes.c_int), ("precision", ctypes.c_int),
                ("group", ctypes.c_int), ("device", ctypes.c_int)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python w4a4_rank_corrected_smooth_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    sig = {
        "svdq_status_string": ([i], ctypes.c_char_p),
        "svdq_last_error": ([], ctypes.c_char_p),
        "svdq_check_device": ([i], i),
        "svdq_get_device_error": ([vp], i),
        "svdq_prepare_weights": ([vp, i, i, vp, vp, ctypes.POINTER(PrepareParams), i, vp, ctypes.POINTER(vp)], i),
        "svdq_free_weights": ([vp], i),
        "svdq_clone_weights": ([vp, vp, ctypes.POINTER(vp)], i),
        "svdq_get_weights_info": ([vp, ctypes.POINTER(WeightsInfo)], i),
        "svdq_export_weights": ([vp, vp, vp, vp, vp, vp, vp, vp], i),
        "svdq_workspace_size": ([vp, i, ctypes.POINTER(sz)], i),
        "svdq_linear_forward": ([vp, vp, i, i, vp, i, vp, sz, vp], i),
        "svdq_linear_forward_noalloc": ([vp, vp, i, i, vp, i, vp], i),
        "svdq_linear_forward_gelu": ([vp, vp, i, i, vp, i, vp, sz, vp], i),
        "svdq_linear_forward_qkv_norm_rope": ([vp, vp, i, i, vp, i, vp, vp, ctypes.c_float, vp, i, vp, sz, vp], i),
        "svdq_mlp_workspace_size": ([vp, vp, i, ctypes.POINTER(sz)], i),
        "svdq_mlp_forward": ([vp, vp, vp, i, i, vp, i, vp, sz, vp, sz, vp], i),
        "svdq_quant_down": ([vp, vp, i, i, vp, sz, vp], i),
        "svdq_gemm_up": ([vp, i, vp, i, vp, sz, vp], i),
        "svdq_export_activations": ([vp, vp, sz, i, vp, vp, vp, vp], i),
        "svdq_quantize_rows_host": ([vp, i, i, i, vp, vp], i),
        "svdq_prepare_host": ([vp, i, i, vp, vp, ctypes.POINTER(PrepareParams), vp, vp, vp, vp, vp, vp, vp], i),
        "svdq_selftest_wait_timeout": ([i, vp], i),
        "svdq_selftest_gelu_bf16": ([vp, vp, i, vp], i),
        "svdq_rope_packed_size": ([i, i, ctypes.POINTER(sz)], i),
        "svdq_pack_rope": ([vp, i, i, vp, sz, vp], i),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()
DECLARED_SYMBOLS = tuple(sorted([
    "svdq_status_string", "svdq_last_error", "svdq_check_device", "svdq_get_device_error", "svdq_prepare_weights",
    "svdq_free_weights", "svdq_clone_weights", "svdq_get_weights_info", "svdq_export_weights", "svdq_workspace_size", "svdq_linear_forward", "svdq_linear_forward_noalloc", "svdq_linear_forward_gelu",
    "svdq_linear_forward_qkv_norm_rope", "svdq_mlp_workspace_size", "svdq_mlp_forward",
    "svdq_quant_down", "svdq_gemm_up", "svdq_export_activations", "svdq_quantize_rows_host", "svdq_prepare_host",
    "svdq_selftest_wait_timeout", "svdq_selftest_gelu_bf16", "svdq_rope_packed_size", "svdq_pack_rope"]))


def lib() -> ctypes.CDLL:
    return _lib


def _check(status: int) -> None:
    if status != SVDQ_OK:
        raise SVDQError(status, _lib.svdq_last_error().decode())


def _ptr(a) -> Optional[int]:
    """Address of a numpy array or torch tensor (None passes NULL)."""
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        assert a.flags["C_CONTIGUOUS"]
        return a.ctypes.data
    return a.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _prec(precision) -> int:
    return PRECISIONS[precision] if isinstance(precision, str) else int(precision)


# ------------------------------------------------------------------ C entry points, same names


def svdq_check_device(device: int = 0) -> None:
    _check(_lib.svdq_check_device(device))


def svdq_get_device_error(stream=None) -> None:
    _check(_lib.svdq_get_device_error(_stream(stream)))


def svdq_selftest_wait_timeout(spin_limit: int, stream=None) -> None:
    _check(_lib.svdq_selftest_wait_timeout(spin_limit, _stream(stream)))


def svdq_rope_packed_size(M: int, head_dim: int = 128) -> int:
    """Bytes of the packed rotary table of M tokens (see include/svdq.h)."""
    out = ctypes.c_size_t()
    _check(_lib.svdq_rope_packed_size(M, head_dim, ctypes.byref(out)))
    return out.value


def svdq_pack_rope(rope, M: int, head_dim: int, packed, packed_bytes: int, stream=None) -> None:
    """Packs a device rotary table (M rows of head_dim/2 (cos, sin) fp32 pairs) for the fused QKV
    operator into the caller's device buffer ``packed``."""
    _check(_lib.svdq_pack_rope(_ptr(rope), M, head_dim, _ptr(packed), packed_bytes, _stream(stream)))


def svdq_selftest_gelu_bf16(inp, out, n: int, stream=None) -> None:
    """The fused MLP epilogue's bf16 GELU on ``n`` bf16 patterns (device tensors of 16-bit ints)."""
    _check(_lib.svdq_selftest_gelu_bf16(_ptr(inp), _ptr(out), n, _stream(stream)))


def svdq_quantize_rows_host(V: np.ndarray, precision):
    p = _prec(precision)
    V = np.ascontiguousarray(V, dtype=np.float32)
    rows, K = V.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 16), np.uint8) if p == SVDQ_NVFP4 else np.zeros((rows, K // 64), np.float32)
    _check(_lib.svdq_quantize_rows_host(_ptr(V), rows, K, p, _ptr(codes), _ptr(scales)))
    return codes, scales


def _params(precision, rank, alpha=0.5, svd_iters=0, seed=0) -> PrepareParams:
    return PrepareParams(_prec(precision), int(rank), float(alpha), int(svd_iters), int(seed))


def svdq_prepare_host(W_bf16: np.ndarray, bias_bf16: Optional[np.ndarray], act_absmax: np.ndarray, precision, rank: int,
                      alpha: float = 0.5, svd_iters: int = 0, seed: int = 0) -> dict:
    p = _params(precision, rank, alpha, svd_iters, seed)
    W = np.ascontiguousarray(W_bf16, dtype=np.uint16)
    N, K = W.shape
    a = np.ascontiguousarray(act_absmax, dtype=np.float32)
    b = None if bias_bf16 is None else np.ascontiguousarray(bias_bf16, dtype=np.uint16)
    out = {
        "inv_lambda": np.zeros(K, np.float32),
        "codes_w": np.zeros((N, K // 2), np.uint8),
        "scales_w": np.zeros((N, K // 16), np.uint8) if p.precision == SVDQ_NVFP4 else np.zeros((N, K // 64), np.float32),
        "L1": np.zeros((K, rank), np.uint16),
        "L2": np.zeros((rank, N), np.uint16),
        "sigma": np.zeros(rank, np.float64),
        "R": np.zeros((N, K), np.float32),
    }
    _check(_lib.svdq_prepare_host(_ptr(W), N, K, _ptr(b), _ptr(a), ctypes.byref(p), _ptr(out["inv_lambda"]),
                                  _ptr(out["codes_w"]), _ptr(out["scales_w"]), _ptr(out["L1"]), _ptr(out["L2"]),
                                  _ptr(out["sigma"]), _ptr(out["R"])))
    return out


class SVDQLinear:
    """A prepared SVDQuant W4A4 layer on one device (owns the library handle)."""

    def __init__(self, W_bf16: np.ndarray, bias_bf16: Optional[np.ndarray], act_absmax: np.ndarray, precision="nvfp4",
                 rank: int = 32, alpha: float = 0.5, svd_iters: int = 0, seed: int = 0, device: int = 0, stream=None):
        p = _params(precision, rank, alpha, svd_iters, seed)
        W = np.ascontiguousarray(W_bf16, dtype=np.uint16)
        self.N, self.K = W.shape
        self.rank = int(rank)
        self.precision = p.precision
        self.device = device
        a = np.ascontiguousarray(act_absmax, dtype=np.float32)
        b = None if bias_bf16 is None else np.ascontiguousarray(bias_bf16, dtype=np.uint16)
        h = ctypes.c_void_p()
        self._h = None
        _check(_lib.svdq_prepare_weights(_ptr(W), self.N, self.K, _ptr(b), _ptr(a), ctypes.byref(p), device,
                                         _stream(stream), ctypes.byref(h)))
        self._h = h

    def clone(self, stream=None) -> "SVDQLinear":
        """An independent copy of this prepared layer (device buffers duplicated, no re-prepare)."""
        h = ctypes.c_void_p()
        _check(_lib.svdq_clone_weights(self._h, _stream(stream), ctypes.byref(h)))
        other = object.__new__(SVDQLinear)
        other.N, other.K, other.rank, other.precision, other.device = self.N, self.K, self.rank, self.precision, self.device
        other._h = h
        return other

    def close(self) -> None:
        if self._h is not None:
            _lib.svdq_free_weights(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def info(self) -> WeightsInfo:
        out = WeightsInfo()
        _check(_lib.svdq_get_weights_info(self._h, ctypes.byref(out)))
        return out

    def workspace_size(self, M: int) -> int:
        out = ctypes.c_size_t()
        _check(_lib.svdq_workspace_size(self._h, M, ctypes.byref(out)))
        return out.value

    def export_weights(self) -> dict:
        N, K, r = self.N, self.K, self.rank
        out = {
            "inv_lambda": np.zeros(K, np.float32),
            "codes_w": np.zeros((N, K // 2), np.uint8),
            "scales_w": np.zeros((N, K // 16), np.uint8) if self.precision == SVDQ_NVFP4 else np.zeros((N, K // 64), np.float32),
            "L1": np.zeros((K, r), np.uint16),
            "L2": np.zeros((r, N), np.uint16),
            "bias": np.zeros(N, np.uint16),
            "sigma": np.zeros(r, np.float64),
        }
        _check(_lib.svdq_export_weights(self._h, _ptr(out["inv_lambda"]), _ptr(out["codes_w"]), _ptr(out["scales_w"]),
                                        _ptr(out["L1"]), _ptr(out["L2"]), _ptr(out["bias"]), _ptr(out["sigma"])))
        return out

    # -------------------------------------------------------------- hot path (device pointers)

    def svdq_linear_forward(self, X, M: int, ldx: int, Y, ldy: int, workspace, workspace_bytes: int, stream=None):
        _check(_lib.svdq_linear_forward(self._h, _ptr(X), M, ldx, _ptr(Y), ldy, _ptr(workspace), workspace_bytes,
                                        _stream(stream)))

    def svdq_linear_forward_gelu(self, X, M: int, ldx: int, Y, ldy: int, workspace, workspace_bytes: int,
                                 stream=None):
        """The forward with GELU on its output, Y = bf16(GELU(bf16(acc + bias))) (NVFP4 layers)."""
        _check(_lib.svdq_linear_forward_gelu(self._h, _ptr(X), M, ldx, _ptr(Y), ldy, _ptr(workspace),
                                             workspace_bytes, _stream(stream)))

    def svdq_linear_forward_noalloc(self, X, M: int, ldx: int, Y, ldy: int, stream=None):
        """The forward using the library's fixed device scratch instead of a caller workspace
        (for callers that cannot allocate device memory; see include/svdq.h)."""
        _check(_lib.svdq_linear_forward_noalloc(self._h, _ptr(X), M, ldx, _ptr(Y), ldy, _stream(stream)))

    def svdq_linear_forward_qkv_norm_rope(self, X, M: int, ldx: int, Y, ldy: int, gamma_q, gamma_k, eps: float,
                                          rope, head_dim: int, workspace, workspace_bytes: int, stream=None):
        """The grouped QKV layer with RMS normalization of the Q and K heads and the rotary
        embedding fused into its epilogue (device pointers; see include/svdq.h)."""
        _check(_lib.svdq_linear_forward_qkv_norm_rope(self._h, _ptr(X), M, ldx, _ptr(Y), ldy, _ptr(gamma_q),
                                                      _ptr(gamma_k), float(eps), _ptr(rope), head_dim,
                                                      _ptr(workspace), workspace_bytes, _stream(stream)))

    def svdq_quant_down(self, X, M: int, ldx: int, workspace, workspace_bytes: int, stream=None):
        _check(_lib.svdq_quant_down(self._h, _ptr(X), M, ldx, _ptr(workspace), workspace_bytes, _stream(stream)))

    def svdq_gemm_up(self, M: int, Y, ldy: int, workspace, workspace_bytes: int, stream=None):
        _check(_lib.svdq_gemm_up(self._h, M, _ptr(Y), ldy, _ptr(workspace), workspace_bytes, _stream(stream)))

    def svdq_export_activations(self, workspace, M: int, stream=None) -> dict:
        K, r = self.K, self.rank
        out = {
            "codes_x": np.zeros((M, K // 2), np.uint8),
            "scales_x": np.zeros((M, K // 16), np.uint8) if self.precision == SVDQ_NVFP4 else np.zeros((M, K // 64), np.float32),
            "T": np.zeros((M, r), np.uint16),
        }
        _check(_lib.svdq_export_activations(self._h, _ptr(workspace), self.workspace_size(M), M, _ptr(out["codes_x"]),
                                            _ptr(out["scales_x"]), _ptr(out["T"]), _stream(stream)))
        return out

    # -------------------------------------------------------------- torch convenience

    def new_workspace(self, M: int):
        import torch

        return torch.empty(max(self.workspace_size(M), 256), dtype=torch.uint8, device=f"cuda:{self.device}")

    def forward(self, X, workspace=None, Y=None, stream=None):
        """Y = layer(X) for a bf16 CUDA tensor X of shape (M, K) (row stride = X.stride(0))."""
        import torch

        assert X.dtype == torch.bfloat16 and X.is_cuda and X.dim() == 2 and X.stride(1) == 1
        M = X.shape[0]
        if workspace is None:
            workspace = self.new_workspace(M)
        if Y is None:
            Y = torch.empty((M, self.N), dtype=torch.bfloat16, device=X.device)
        self.svdq_linear_forward(X, M, X.stride(0), Y, Y.stride(0), workspace, workspace.numel(), stream)
        return Y

    __call__ = forward


def svdq_mlp_workspace_size(up: "SVDQLinear", down: "SVDQLinear", M: int) -> int:
    """Bytes of the fused MLP pair's middle workspace for M rows (see include/svdq.h)."""
    out = ctypes.c_size_t()
    _check(_lib.svdq_mlp_workspace_size(up.handle, down.handle, M, ctypes.byref(out)))
    return out.value


def svdq_mlp_forward(up: "SVDQLinear", down: "SVDQLinear", X, M: int, ldx: int, Y, ldy: int, ws_up, ws_up_bytes: int,
                     ws_mid, ws_mid_bytes: int, stream=None) -> None:
    """Y = down(bf16(GELU(bf16(up(X))))) with the hidden activation kept out of memory (device
    pointers; see include/svdq.h)."""
    _check(_lib.svdq_mlp_forward(up.handle, down.handle, _ptr(X), M, ldx, _ptr(Y), ldy, _ptr(ws_up), ws_up_bytes,
                                 _ptr(ws_mid), ws_mid_bytes, _stream(stream)))


__all__ = ["SVDQLinear", "SVDQError", "svdq_check_device", "svdq_get_device_error", "svdq_selftest_wait_timeout",
           "svdq_selftest_gelu_bf16", "svdq_rope_packed_size", "svdq_pack_rope",
           "svdq_quantize_rows_host", "svdq_prepare_host", "svdq_mlp_workspace_size", "svdq_mlp_forward", "SVDQ_NVFP4",
           "SVDQ_INT4", "SVDQ_W4A16", "LIB_PATH", "lib", "DECLARED_SYMBOLS"]
