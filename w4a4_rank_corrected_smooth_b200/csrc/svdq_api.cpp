// C ABI of the library (declarations and contracts in include/svdq.h).
#include "../../include/svdq.h"

#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "host_prepare.h"
#include "kernels.h"
#include "layout.h"

struct svdq_weights {
  int N = 0, K = 0, rank = 0, precision = 0, device = 0, num_sms = 0;
  svdq::CanonicalLayer canon;
  float* d_inv_lambda = nullptr;
  uint8_t* d_codes = nullptr;
  uint8_t* d_sf = nullptr;
  uint8_t* d_l1 = nullptr;
  uint8_t* d_l2 = nullptr;
  float* d_bias = nullptr;
};

namespace {

thread_local std::string g_last_error;

svdq_status fail(svdq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

svdq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(e == cudaErrorMemoryAllocation ? SVDQ_ERR_OOM : SVDQ_ERR_CUDA, "%s: %s (%s)", what,
              cudaGetErrorString(e), cudaGetErrorName(e));
}

// Restores the caller's current device on scope exit.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess) ok = true;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The W4A16 layer quantizes its weights with the INT4 quantizer (group 64, fp32 scales).
int quantizer_precision(int precision) { return precision == SVDQ_W4A16 ? SVDQ_INT4 : precision; }

svdq_status check_shape(int N, int K, const svdq_prepare_params* p) {
  if (!p) return fail(SVDQ_ERR_INVALID_ARG, "params is NULL");
  if (p->precision != SVDQ_NVFP4 && p->precision != SVDQ_INT4 && p->precision != SVDQ_W4A16)
    return fail(SVDQ_ERR_INVALID_ARG, "precision %d is not SVDQ_NVFP4 (0), SVDQ_INT4 (1) or SVDQ_W4A16 (2)",
                p->precision);
  if (p->precision == SVDQ_W4A16 && p->rank != 0)
    return fail(SVDQ_ERR_INVALID_ARG, "rank=%d: the W4A16 layer has no low-rank branch (rank must be 0)", p->rank);
  if (p->precision == SVDQ_W4A16 && K > svdq::kW4A16MaxK)
    return fail(SVDQ_ERR_INVALID_ARG, "K=%d exceeds %d for the W4A16 layer", K, svdq::kW4A16MaxK);
  if (N <= 0 || K <= 0) return fail(SVDQ_ERR_INVALID_ARG, "N=%d and K=%d must be positive", N, K);
  if (K % svdq::kBK != 0) return fail(SVDQ_ERR_INVALID_ARG, "K=%d must be a multiple of %d", K, svdq::kBK);
  if (N % 8 != 0) return fail(SVDQ_ERR_INVALID_ARG, "N=%d must be a multiple of 8", N);
  if (p->rank < 0 || p->rank > svdq::kMaxRank || p->rank % 16 != 0)
    return fail(SVDQ_ERR_INVALID_ARG, "rank=%d must be a multiple of 16 in [0, %d]", p->rank, svdq::kMaxRank);
  if (p->rank > N || p->rank > K) return fail(SVDQ_ERR_INVALID_ARG, "rank=%d exceeds min(N, K)", p->rank);
  if (!(p->alpha > 0.0f && p->alpha < 1.0f)) return fail(SVDQ_ERR_INVALID_ARG, "alpha=%g must be in (0, 1)", p->alpha);
  return SVDQ_OK;
}

template <class T>
svdq_status upload(T** dst, const std::vector<T>& src, cudaStream_t stream) {
  const size_t bytes = src.size() * sizeof(T);
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(dst), bytes > 0 ? bytes : 16);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc of prepared weights");
  if (bytes > 0) {
    e = cudaMemcpyAsync(*dst, src.data(), bytes, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_fail(e, "upload of prepared weights");
  }
  return SVDQ_OK;
}

void free_device(svdq_weights* w) {
  cudaFree(w->d_inv_lambda);
  cudaFree(w->d_codes);
  cudaFree(w->d_sf);
  cudaFree(w->d_l1);
  cudaFree(w->d_l2);
  cudaFree(w->d_bias);
  w->d_inv_lambda = nullptr;
  w->d_codes = w->d_sf = w->d_l1 = w->d_l2 = nullptr;
  w->d_bias = nullptr;
}

// Workspace bytes of a forward (kernel 1's region: codes, scales, T and its K-split partials).
size_t forward_workspace_bytes(const svdq_weights* w, int M) {
  if (w->precision == SVDQ_W4A16 || M <= 0) return 0;
  return svdq::workspace_layout(M, w->K, w->rank).total;
}

svdq_status check_forward_common(const svdq_weights* w, int M, const void* ws, size_t ws_bytes) {
  if (!w) return fail(SVDQ_ERR_INVALID_ARG, "weights handle is NULL");
  if (M < 0) return fail(SVDQ_ERR_INVALID_ARG, "M=%d is negative", M);
  if (M == 0) return SVDQ_OK;
  if (w->precision == SVDQ_W4A16) return SVDQ_OK;  // no workspace: one kernel, nothing in between
  const size_t need = forward_workspace_bytes(w, M);
  if (!ws) return fail(SVDQ_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(ws, 256)) return fail(SVDQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < need)
    return fail(SVDQ_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu bytes needed for M=%d", ws_bytes,
                need, M);
  return SVDQ_OK;
}

svdq_status do_quant_down(const svdq_weights* w, const void* X, int M, int ldx, void* ws, cudaStream_t stream) {
  if (!X) return fail(SVDQ_ERR_INVALID_ARG, "X is NULL");
  if (ldx < w->K || ldx % 8 != 0) return fail(SVDQ_ERR_INVALID_ARG, "ldx=%d must be >= K=%d and a multiple of 8", ldx, w->K);
  if (!aligned(X, 16)) return fail(SVDQ_ERR_INVALID_ARG, "X must be 16-byte aligned");
  const svdq::WorkspaceLayout L = svdq::workspace_layout(M, w->K, w->rank);
  uint8_t* base = static_cast<uint8_t*>(ws);
  svdq::QuantDownArgs a;
  a.X = static_cast<const uint16_t*>(X);
  a.M = M;
  a.K = w->K;
  a.ldx = ldx;
  a.rank = w->rank;
  a.precision = w->precision;
  a.inv_lambda = w->d_inv_lambda;
  a.l1 = w->d_l1;
  a.codes = base + L.codes;
  a.sf = base + L.sf;
  a.t = base + L.t;
  a.part = L.part ? reinterpret_cast<float*>(base + L.part) : nullptr;
  a.cnt = L.cnt ? reinterpret_cast<unsigned long long*>(base + L.cnt) : nullptr;
  a.split_cap = L.split_cap;  // with rank 0 no partials are needed
  cudaError_t e = svdq::launch_quant_down(a, w->num_sms, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launch of the quantize/down-projection kernel");
  return SVDQ_OK;
}

// The fused MLP pair's epilogue of the up layer's kernel 2: the down layer's operands.
struct MlpEpilogue {
  const svdq_weights* down;
  uint8_t* mid;  // the down layer's workspace, then the T partials
  size_t part_offset;
  int smax, pairs;
};

// The fused MLP's schedule of the up layer's kernel 2: CTA pairs (as the launch picks them) and the
// T-partial slots one 256-row block can receive (pairs whose contiguous tile ranges meet it).
struct MlpSchedule {
  int tiles, nt, pairs, smax;
};
MlpSchedule mlp_schedule(const svdq_weights* up, int M) {
  MlpSchedule s;
  const int mt2 = (M + 2 * svdq::kBM - 1) / (2 * svdq::kBM);
  s.nt = (up->N + svdq::kBN - 1) / svdq::kBN;
  s.tiles = mt2 * s.nt;
  s.pairs = up->num_sms / 2 < s.tiles ? up->num_sms / 2 : s.tiles;
  if (s.pairs < 1) s.pairs = 1;
  s.smax = s.nt / (s.tiles / s.pairs) + 2;
  return s;
}

// The fused Q/K normalization and rotary embedding of kernel 2's epilogue.
struct QkvEpilogue {
  int qk_cols;
  const float* gamma_q;
  const float* gamma_k;
  const float* rope;
  float eps;
};

svdq_status do_gemm(const svdq_weights* w, int M, void* Y, int ldy, const void* ws, cudaStream_t stream,
                    const QkvEpilogue* qkv = nullptr, const MlpEpilogue* mlp = nullptr, bool gelu = false) {
  if (!Y) return fail(SVDQ_ERR_INVALID_ARG, "Y is NULL");
  if (ldy < w->N || ldy % 8 != 0) return fail(SVDQ_ERR_INVALID_ARG, "ldy=%d must be >= N=%d and a multiple of 8", ldy, w->N);
  if (!aligned(Y, 16)) return fail(SVDQ_ERR_INVALID_ARG, "Y must be 16-byte aligned");
  const svdq::WorkspaceLayout L = svdq::workspace_layout(M, w->K, w->rank);
  const uint8_t* base = static_cast<const uint8_t*>(ws);
  svdq::GemmArgs a;
  a.M = M;
  a.N = w->N;
  a.K = w->K;
  a.rank = w->rank;
  a.precision = w->precision;
  a.ldy = ldy;
  a.a_codes = base + L.codes;
  a.a_sf = base + L.sf;
  a.t = base + L.t;
  a.b_codes = w->d_codes;
  a.b_sf = w->d_sf;
  a.l2 = w->d_l2;
  a.bias = w->d_bias;
  a.Y = static_cast<uint16_t*>(Y);
  a.gelu = gelu;
  if (qkv) {
    a.qk_cols = qkv->qk_cols;
    a.gamma_q = qkv->gamma_q;
    a.gamma_k = qkv->gamma_k;
    a.rope = qkv->rope;
    a.eps = qkv->eps;
  }
  if (mlp) {
    const svdq::WorkspaceLayout Ld = svdq::workspace_layout(M, mlp->down->K, mlp->down->rank);
    a.mlp = true;
    a.il_down = mlp->down->d_inv_lambda;
    a.codes_down = mlp->mid + Ld.codes;
    a.sf_down = mlp->mid + Ld.sf;
    a.l1_down = mlp->down->d_l1;
    a.r_down = mlp->down->rank;
    a.tpart = reinterpret_cast<float*>(mlp->mid + mlp->part_offset);
    a.mlp_smax = mlp->smax;
    a.mlp_pairs = mlp->pairs;
  }
  cudaError_t e = svdq::launch_gemm(a, w->num_sms, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launch of the 4-bit GEMM/up-projection kernel");
  return SVDQ_OK;
}

svdq_status do_w4a16(const svdq_weights* w, const void* X, int M, int ldx, void* Y, int ldy, cudaStream_t stream) {
  if (!X) return fail(SVDQ_ERR_INVALID_ARG, "X is NULL");
  if (ldx < w->K || ldx % 8 != 0) return fail(SVDQ_ERR_INVALID_ARG, "ldx=%d must be >= K=%d and a multiple of 8", ldx, w->K);
  if (!aligned(X, 16)) return fail(SVDQ_ERR_INVALID_ARG, "X must be 16-byte aligned");
  svdq::W4A16Args a;
  a.X = static_cast<const uint16_t*>(X);
  a.M = M;
  a.K = w->K;
  a.ldx = ldx;
  a.N = w->N;
  a.ldy = ldy;
  a.inv_lambda = w->d_inv_lambda;
  a.codes = w->d_codes;
  a.scales = reinterpret_cast<const float*>(w->d_sf);
  a.bias = w->d_bias;
  a.Y = static_cast<uint16_t*>(Y);
  cudaError_t e = svdq::launch_w4a16(a, w->num_sms, stream);
  if (e != cudaSuccess) return cuda_fail(e, "launch of the W4A16 kernel");
  return SVDQ_OK;
}

}  // namespace

extern "C" {

const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "SVDQ_OK";
    case SVDQ_ERR_INVALID_ARG: return "SVDQ_ERR_INVALID_ARG";
    case SVDQ_ERR_UNSUPPORTED_DEVICE: return "SVDQ_ERR_UNSUPPORTED_DEVICE";
    case SVDQ_ERR_CUDA: return "SVDQ_ERR_CUDA";
    case SVDQ_ERR_OOM: return "SVDQ_ERR_OOM";
    case SVDQ_ERR_TIMEOUT: return "SVDQ_ERR_TIMEOUT";
    case SVDQ_ERR_INTERNAL: return "SVDQ_ERR_INTERNAL";
  }
  return "SVDQ_ERR_UNKNOWN";
}

const char* svdq_last_error(void) { return g_last_error.c_str(); }

svdq_status svdq_check_device(int device) {
  int count = 0;
  cudaError_t e = cudaGetDeviceCount(&count);
  if (e != cudaSuccess || count == 0)
    return fail(SVDQ_ERR_UNSUPPORTED_DEVICE, "no CUDA device is available (%s)", cudaGetErrorString(e));
  if (device < 0 || device >= count) return fail(SVDQ_ERR_INVALID_ARG, "device %d out of range [0, %d)", device, count);
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, device);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  int major = prop.major, minor = prop.minor;
  // Test hook: pretend the device has another capability ("MAJOR.MINOR") to exercise the error path.
  if (const char* fake = std::getenv("SVDQ_TEST_FAKE_CC")) {
    if (std::sscanf(fake, "%d.%d", &major, &minor) != 2) return fail(SVDQ_ERR_INVALID_ARG, "bad SVDQ_TEST_FAKE_CC");
  }
  if (major != 10 || minor != 0)
    return fail(SVDQ_ERR_UNSUPPORTED_DEVICE,
                "device %d (%s) has compute capability %d.%d; these kernels are built for sm_100a (10.0) only", device,
                prop.name, major, minor);
  return SVDQ_OK;
}

svdq_status svdq_get_device_error(void* stream) {
  unsigned int v = 0, vw = 0;
  cudaError_t e = svdq::read_and_clear_device_error(&v, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  e = svdq::read_and_clear_w4a16_error(&vw, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "reading the W4A16 kernel's device error word");
  v |= vw;
  if (v != 0) return fail(SVDQ_ERR_TIMEOUT, "a kernel's bounded wait gave up (device error bits 0x%x)", v);
  return SVDQ_OK;
}

svdq_status svdq_quantize_rows_host(const float* V, int rows, int K, int precision, uint8_t* codes, void* scales) {
  if (!V || !codes || !scales) return fail(SVDQ_ERR_INVALID_ARG, "NULL argument");
  if (rows < 0 || K <= 0) return fail(SVDQ_ERR_INVALID_ARG, "bad rows/K");
  if (precision != SVDQ_NVFP4 && precision != SVDQ_INT4) return fail(SVDQ_ERR_INVALID_ARG, "bad precision");
  if (K % (precision == SVDQ_NVFP4 ? 16 : 64) != 0) return fail(SVDQ_ERR_INVALID_ARG, "K not a multiple of the group");
  svdq::quantize_rows_host(V, rows, K, precision, codes, scales);
  return SVDQ_OK;
}

svdq_status svdq_prepare_host(const uint16_t* W_bf16, int N, int K, const uint16_t* bias_bf16, const float* act_absmax,
                              const svdq_prepare_params* params, float* inv_lambda, uint8_t* codes_w, void* scales_w,
                              uint16_t* L1, uint16_t* L2, double* sigma, float* R_out) {
  svdq_status s = check_shape(N, K, params);
  if (s != SVDQ_OK) return s;
  if (!W_bf16 || !act_absmax) return fail(SVDQ_ERR_INVALID_ARG, "W or act_absmax is NULL");
  svdq::CanonicalLayer c;
  try {
    svdq::prepare_canonical(W_bf16, N, K, bias_bf16, act_absmax, quantizer_precision(params->precision), params->rank,
                            params->alpha, params->svd_iters > 0 ? params->svd_iters : 12, params->seed, c);
  } catch (const std::bad_alloc&) {
    return fail(SVDQ_ERR_OOM, "host allocation failed in prepare");
  }
  const size_t NK = static_cast<size_t>(N) * K;
  if (inv_lambda) std::memcpy(inv_lambda, c.inv_lambda.data(), sizeof(float) * K);
  if (codes_w) std::memcpy(codes_w, c.codes_w.data(), NK / 2);
  if (scales_w) {
    if (params->precision == SVDQ_NVFP4) std::memcpy(scales_w, c.scales_nvfp4.data(), NK / 16);
    else std::memcpy(scales_w, c.scales_int4.data(), sizeof(float) * NK / 64);
  }
  if (L1 && params->rank) std::memcpy(L1, c.L1.data(), sizeof(uint16_t) * K * params->rank);
  if (L2 && params->rank) std::memcpy(L2, c.L2.data(), sizeof(uint16_t) * N * params->rank);
  if (sigma && params->rank) std::memcpy(sigma, c.sigma.data(), sizeof(double) * params->rank);
  if (R_out) std::memcpy(R_out, c.R.data(), sizeof(float) * NK);
  return SVDQ_OK;
}

svdq_status svdq_prepare_weights(const uint16_t* W_bf16, int N, int K, const uint16_t* bias_bf16,
                                 const float* act_absmax, const svdq_prepare_params* params, int device, void* stream,
                                 svdq_weights** out) {
  if (!out) return fail(SVDQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  svdq_status s = check_shape(N, K, params);
  if (s != SVDQ_OK) return s;
  if (!W_bf16 || !act_absmax) return fail(SVDQ_ERR_INVALID_ARG, "W or act_absmax is NULL");
  s = svdq_check_device(device);
  if (s != SVDQ_OK) return s;
  DeviceGuard guard(device);
  if (!guard.ok) return fail(SVDQ_ERR_CUDA, "cudaSetDevice(%d) failed", device);
  svdq_weights* w = new (std::nothrow) svdq_weights();
  if (!w) return fail(SVDQ_ERR_OOM, "host allocation of the handle failed");
  w->N = N;
  w->K = K;
  w->rank = params->rank;
  w->precision = params->precision;
  w->device = device;
  cudaDeviceGetAttribute(&w->num_sms, cudaDevAttrMultiProcessorCount, device);
  svdq::DeviceImages img;
  try {
    svdq::prepare_canonical(W_bf16, N, K, bias_bf16, act_absmax, quantizer_precision(params->precision), params->rank,
                            params->alpha, params->svd_iters > 0 ? params->svd_iters : 12, params->seed, w->canon);
    svdq::pack_device_layouts(w->canon, img);
    // W4A16: codes and scales in the warp-level MMA's fragment order (same sizes as above).
    if (params->precision == SVDQ_W4A16) svdq::pack_w4a16_fragments(w->canon, img);
  } catch (const std::bad_alloc&) {
    delete w;
    return fail(SVDQ_ERR_OOM, "host allocation failed in prepare");
  }
  w->canon.R.clear();
  w->canon.R.shrink_to_fit();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = upload(&w->d_inv_lambda, w->canon.inv_lambda, st)) != SVDQ_OK ||
      (s = upload(&w->d_codes, img.codes, st)) != SVDQ_OK || (s = upload(&w->d_sf, img.sf, st)) != SVDQ_OK ||
      (s = upload(&w->d_l1, img.l1, st)) != SVDQ_OK || (s = upload(&w->d_l2, img.l2, st)) != SVDQ_OK ||
      (s = upload(&w->d_bias, img.bias, st)) != SVDQ_OK) {
    free_device(w);
    delete w;
    return s;
  }
  cudaError_t e = cudaStreamSynchronize(st);  // host images die with this scope
  if (e != cudaSuccess) {
    free_device(w);
    delete w;
    return cuda_fail(e, "uploading prepared weights");
  }
  *out = w;
  return SVDQ_OK;
}

svdq_status svdq_free_weights(svdq_weights* w) {
  if (!w) return SVDQ_OK;
  DeviceGuard guard(w->device);
  free_device(w);
  delete w;
  return SVDQ_OK;
}

svdq_status svdq_clone_weights(const svdq_weights* src, void* stream, svdq_weights** out) {
  if (!src || !out) return fail(SVDQ_ERR_INVALID_ARG, "NULL argument");
  *out = nullptr;
  DeviceGuard guard(src->device);
  if (!guard.ok) return fail(SVDQ_ERR_CUDA, "cudaSetDevice(%d) failed", src->device);
  svdq_weights* w = new (std::nothrow) svdq_weights();
  if (!w) return fail(SVDQ_ERR_OOM, "host allocation of the handle failed");
  try {
    w->canon = src->canon;
  } catch (const std::bad_alloc&) {
    delete w;
    return fail(SVDQ_ERR_OOM, "host allocation failed while cloning");
  }
  w->N = src->N;
  w->K = src->K;
  w->rank = src->rank;
  w->precision = src->precision;
  w->device = src->device;
  w->num_sms = src->num_sms;
  const size_t npad = static_cast<size_t>((src->N + svdq::kBN - 1) / svdq::kBN) * svdq::kBN;
  const size_t K = static_cast<size_t>(src->K), r = static_cast<size_t>(src->rank);
  struct Buf { void** dst; const void* src; size_t bytes; };
  const Buf bufs[] = {
      {reinterpret_cast<void**>(&w->d_inv_lambda), src->d_inv_lambda, K * sizeof(float)},
      {reinterpret_cast<void**>(&w->d_codes), src->d_codes, npad * K / 2},
      {reinterpret_cast<void**>(&w->d_sf), src->d_sf, npad * K / svdq::kBK * svdq::kSfBytesPerRowKb},
      {reinterpret_cast<void**>(&w->d_l1), src->d_l1, K * r * 2},
      {reinterpret_cast<void**>(&w->d_l2), src->d_l2, npad * r * 2},
      {reinterpret_cast<void**>(&w->d_bias), src->d_bias, npad * sizeof(float)},
  };
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (const Buf& b : bufs) {
    cudaError_t e = cudaMalloc(b.dst, b.bytes > 0 ? b.bytes : 16);
    if (e == cudaSuccess && b.bytes > 0) e = cudaMemcpyAsync(*b.dst, b.src, b.bytes, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) {
      free_device(w);
      delete w;
      return cuda_fail(e, "cloning prepared weights");
    }
  }
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    free_device(w);
    delete w;
    return cuda_fail(e, "cloning prepared weights");
  }
  *out = w;
  return SVDQ_OK;
}

svdq_status svdq_get_weights_info(const svdq_weights* w, svdq_weights_info* info) {
  if (!w || !info) return fail(SVDQ_ERR_INVALID_ARG, "NULL argument");
  info->N = w->N;
  info->K = w->K;
  info->rank = w->rank;
  info->precision = w->precision;
  info->group = w->precision == SVDQ_NVFP4 ? 16 : 64;
  info->device = w->device;
  return SVDQ_OK;
}

svdq_status svdq_export_weights(const svdq_weights* w, float* inv_lambda, uint8_t* codes_w, void* scales_w,
                                uint16_t* L1, uint16_t* L2, uint16_t* bias, double* sigma) {
  if (!w) return fail(SVDQ_ERR_INVALID_ARG, "weights handle is NULL");
  const svdq::CanonicalLayer& c = w->canon;
  const size_t NK = static_cast<size_t>(w->N) * w->K;
  if (inv_lambda) std::memcpy(inv_lambda, c.inv_lambda.data(), sizeof(float) * w->K);
  if (codes_w) std::memcpy(codes_w, c.codes_w.data(), NK / 2);
  if (scales_w) {
    if (w->precision == SVDQ_NVFP4) std::memcpy(scales_w, c.scales_nvfp4.data(), NK / 16);
    else std::memcpy(scales_w, c.scales_int4.data(), sizeof(float) * NK / 64);
  }
  if (L1 && w->rank) std::memcpy(L1, c.L1.data(), sizeof(uint16_t) * w->K * w->rank);
  if (L2 && w->rank) std::memcpy(L2, c.L2.data(), sizeof(uint16_t) * w->N * w->rank);
  if (bias) std::memcpy(bias, c.bias.data(), sizeof(uint16_t) * w->N);
  if (sigma && w->rank) std::memcpy(sigma, c.sigma.data(), sizeof(double) * w->rank);
  return SVDQ_OK;
}

svdq_status svdq_workspace_size(const svdq_weights* w, int M, size_t* bytes) {
  if (!w || !bytes) return fail(SVDQ_ERR_INVALID_ARG, "NULL argument");
  if (M < 0) return fail(SVDQ_ERR_INVALID_ARG, "M=%d is negative", M);
  *bytes = forward_workspace_bytes(w, M);
  return SVDQ_OK;
}

svdq_status svdq_linear_forward_noalloc(const svdq_weights* w, const void* X, int M, int ldx, void* Y, int ldy,
                                        void* stream) {
  if (!w) return fail(SVDQ_ERR_INVALID_ARG, "weights handle is NULL");
  if (M < 0) return fail(SVDQ_ERR_INVALID_ARG, "M=%d is negative", M);
  if (M == 0) return SVDQ_OK;
  const size_t need = forward_workspace_bytes(w, M);
  const size_t have = svdq::noalloc_scratch_bytes();
  if (need > have)
    return fail(SVDQ_ERR_INVALID_ARG,
                "svdq_linear_forward_noalloc: M=%d (K=%d, rank=%d) needs %zu bytes of scratch, more than the %zu bytes "
                "of the library's fixed scratch; use svdq_linear_forward with a caller workspace",
                M, w->K, w->rank, need, have);
  DeviceGuard guard(w->device);
  if (!guard.ok) return fail(SVDQ_ERR_CUDA, "cudaSetDevice(%d) failed", w->device);
  void* scratch = nullptr;
  cudaError_t e = svdq::noalloc_scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "looking up the fixed scratch (cudaGetSymbolAddress)");
  return svdq_linear_forward(w, X, M, ldx, Y, ldy, scratch, have, stream);
}

svdq_status svdq_rope_packed_size(int M, int head_dim, size_t* bytes) {
  if (!bytes) return fail(SVDQ_ERR_INVALID_ARG, "NULL argument");
  if (M < 0) return fail(SVDQ_ERR_INVALID_ARG, "M=%d is negative", M);
  if (head_dim != svdq::kQkvHeadDim)
    return fail(SVDQ_ERR_INVALID_ARG, "head_dim=%d: the fused QKV operator supports %d", head_dim, svdq::kQkvHeadDim);
  *bytes = svdq::rope_packed_bytes(M);
  return SVDQ_OK;
}

svdq_status svdq_pack_rope(const float* rope, int M, int head_dim, float* packed, size_t packed_bytes, void* stream) {
  size_t need = 0;
  svdq_status s = svdq_rope_packed_size(M, head_dim, &need);
  if (s != SVDQ_OK || M == 0) return s;
  if (!rope || !packed) return fail(SVDQ_ERR_INVALID_ARG, "rope and packed must not be NULL");
  if (!aligned(rope, 16) || !aligned(packed, 16))
    return fail(SVDQ_ERR_INVALID_ARG, "rope and packed must be 16-byte aligned");
  if (packed_bytes < need)
    return fail(SVDQ_ERR_INVALID_ARG, "packed buffer of %zu bytes is smaller than the %zu bytes needed for M=%d",
                packed_bytes, need, M);
  cudaError_t e = svdq::launch_rope_pack(rope, M, packed, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "launch of the rotary-table packing kernel");
  return SVDQ_OK;
}

svdq_status svdq_linear_forward_qkv_norm_rope(const svdq_weights* w, const void* X, int M, int ldx, void* Y,
                                              int ldy, const float* gamma_q, const float* gamma_k, float eps,
                                              const float* rope, int head_dim, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  if (w && w->precision == SVDQ_W4A16)
    return fail(SVDQ_ERR_INVALID_ARG, "the fused QKV operator runs on a W4A4 layer (NVFP4 or INT4), not W4A16");
  if (head_dim != svdq::kQkvHeadDim)
    return fail(SVDQ_ERR_INVALID_ARG, "head_dim=%d: the fused QKV operator supports %d", head_dim,
                svdq::kQkvHeadDim);
  if (w && w->N % (3 * head_dim) != 0)
    return fail(SVDQ_ERR_INVALID_ARG, "N=%d is not 3 x heads x head_dim (head_dim=%d)", w->N, head_dim);
  if (!(eps >= 0.0f && eps <= 3.4e38f)) return fail(SVDQ_ERR_INVALID_ARG, "eps=%g must be >= 0 and finite", eps);
  svdq_status s = check_forward_common(w, M, workspace, workspace_bytes);
  if (s != SVDQ_OK || M == 0) return s;
  if (!gamma_q || !gamma_k || !rope) return fail(SVDQ_ERR_INVALID_ARG, "gamma_q, gamma_k and rope must not be NULL");
  if (!aligned(gamma_q, 16) || !aligned(gamma_k, 16) || !aligned(rope, 16))
    return fail(SVDQ_ERR_INVALID_ARG, "gamma_q, gamma_k and rope must be 16-byte aligned");
  if (!Y) return fail(SVDQ_ERR_INVALID_ARG, "Y is NULL");
  if (ldy < w->N || ldy % 8 != 0 || !aligned(Y, 16))
    return fail(SVDQ_ERR_INVALID_ARG, "Y must be 16-byte aligned with ldy >= N and a multiple of 8");
  DeviceGuard guard(w->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = do_quant_down(w, X, M, ldx, workspace, st);
  if (s != SVDQ_OK) return s;
  QkvEpilogue q;
  q.qk_cols = 2 * (w->N / 3);
  q.gamma_q = gamma_q;
  q.gamma_k = gamma_k;
  q.rope = rope;
  q.eps = eps;
  return do_gemm(w, M, Y, ldy, workspace, st, &q);
}

namespace {

svdq_status mlp_check(const svdq_weights* up, const svdq_weights* down) {
  if (!up || !down) return fail(SVDQ_ERR_INVALID_ARG, "weights handle is NULL");
  if (up->precision != SVDQ_NVFP4 || down->precision != SVDQ_NVFP4)
    return fail(SVDQ_ERR_INVALID_ARG, "the fused MLP pair runs on NVFP4 layers only");
  if (up->N != down->K)
    return fail(SVDQ_ERR_INVALID_ARG, "the up layer's N=%d is not the down layer's K=%d", up->N, down->K);
  if (down->rank != 0 && down->rank != 16 && down->rank != 32)
    return fail(SVDQ_ERR_INVALID_ARG, "the fused MLP pair supports a down-layer rank of 0, 16 or 32 (got %d)",
                down->rank);
  if (up->device != down->device) return fail(SVDQ_ERR_INVALID_ARG, "the two layers live on different devices");
  return SVDQ_OK;
}

// The middle workspace: the down layer's workspace for M rows, then [M padded][2 N_up/256][r]
// fp32 partials of its T.
size_t mlp_part_offset(const svdq_weights* down, int M) {
  return svdq::align_up(svdq::workspace_layout(M, down->K, down->rank).total, 1024);
}
size_t mlp_part_bytes(const svdq_weights* up, const svdq_weights* down, int M) {
  const svdq::WorkspaceLayout L = svdq::workspace_layout(M, down->K, down->rank);
  const MlpSchedule sc = mlp_schedule(up, M);
  return static_cast<size_t>(L.m_tiles) * svdq::kBM * 2 * sc.smax * down->rank * sizeof(float);
}

}  // namespace

svdq_status svdq_mlp_workspace_size(const svdq_weights* up, const svdq_weights* down, int M, size_t* bytes) {
  if (!bytes) return fail(SVDQ_ERR_INVALID_ARG, "bytes is NULL");
  svdq_status s = mlp_check(up, down);
  if (s != SVDQ_OK) return s;
  if (M < 0) return fail(SVDQ_ERR_INVALID_ARG, "M=%d is negative", M);
  *bytes = M == 0 ? 0 : mlp_part_offset(down, M) + mlp_part_bytes(up, down, M);
  return SVDQ_OK;
}

svdq_status svdq_mlp_forward(const svdq_weights* up, const svdq_weights* down, const void* X, int M, int ldx,
                             void* Y, int ldy, void* ws_up, size_t ws_up_bytes, void* ws_mid, size_t ws_mid_bytes,
                             void* stream) {
  svdq_status s = mlp_check(up, down);
  if (s != SVDQ_OK) return s;
  s = check_forward_common(up, M, ws_up, ws_up_bytes);
  if (s != SVDQ_OK || M == 0) return s;
  const size_t need = mlp_part_offset(down, M) + mlp_part_bytes(up, down, M);
  if (!ws_mid) return fail(SVDQ_ERR_INVALID_ARG, "the middle workspace is NULL");
  if (!aligned(ws_mid, 256)) return fail(SVDQ_ERR_INVALID_ARG, "the middle workspace must be 256-byte aligned");
  if (ws_mid_bytes < need)
    return fail(SVDQ_ERR_INVALID_ARG, "middle workspace of %zu bytes is smaller than the %zu bytes needed for M=%d",
                ws_mid_bytes, need, M);
  if (!Y) return fail(SVDQ_ERR_INVALID_ARG, "Y is NULL");
  if (ldy < down->N || ldy % 8 != 0 || !aligned(Y, 16))
    return fail(SVDQ_ERR_INVALID_ARG, "Y must be 16-byte aligned with ldy >= N and a multiple of 8");
  DeviceGuard guard(up->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = do_quant_down(up, X, M, ldx, ws_up, st);
  if (s != SVDQ_OK) return s;
  MlpEpilogue m;
  m.down = down;
  m.mid = static_cast<uint8_t*>(ws_mid);
  m.part_offset = mlp_part_offset(down, M);
  const MlpSchedule sc = mlp_schedule(up, M);
  m.smax = sc.smax;
  m.pairs = sc.pairs;
  // the up layer's Y is not written: its tensor map (unused) points at the middle workspace
  s = do_gemm(up, M, ws_mid, up->N, ws_up, st, nullptr, &m);
  if (s != SVDQ_OK) return s;
  if (down->rank > 0) {
    const svdq::WorkspaceLayout Ld = svdq::workspace_layout(M, down->K, down->rank);
    cudaError_t e = svdq::launch_mlp_t_reduce(reinterpret_cast<const float*>(m.mid + m.part_offset),
                                              Ld.m_tiles * svdq::kBM, sc.smax, down->rank, sc.nt, sc.pairs, sc.tiles,
                                              m.mid + Ld.t, st);
    if (e != cudaSuccess) return cuda_fail(e, "launch of the fused MLP's T reduction");
  }
  return do_gemm(down, M, Y, ldy, ws_mid, st);
}

svdq_status svdq_quant_down(const svdq_weights* w, const void* X, int M, int ldx, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (w && w->precision == SVDQ_W4A16)
    return fail(SVDQ_ERR_INVALID_ARG, "the W4A16 layer runs as one kernel: use svdq_linear_forward");
  svdq_status s = check_forward_common(w, M, workspace, workspace_bytes);
  if (s != SVDQ_OK || M == 0) return s;
  DeviceGuard guard(w->device);
  return do_quant_down(w, X, M, ldx, workspace, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_gemm_up(const svdq_weights* w, int M, void* Y, int ldy, const void* workspace, size_t workspace_bytes,
                         void* stream) {
  if (w && w->precision == SVDQ_W4A16)
    return fail(SVDQ_ERR_INVALID_ARG, "the W4A16 layer runs as one kernel: use svdq_linear_forward");
  svdq_status s = check_forward_common(w, M, workspace, workspace_bytes);
  if (s != SVDQ_OK || M == 0) return s;
  DeviceGuard guard(w->device);
  return do_gemm(w, M, Y, ldy, workspace, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_linear_forward(const svdq_weights* w, const void* X, int M, int ldx, void* Y, int ldy,
                                void* workspace, size_t workspace_bytes, void* stream) {
  svdq_status s = check_forward_common(w, M, workspace, workspace_bytes);
  if (s != SVDQ_OK || M == 0) return s;
  if (!Y) return fail(SVDQ_ERR_INVALID_ARG, "Y is NULL");
  if (ldy < w->N || ldy % 8 != 0 || !aligned(Y, 16))
    return fail(SVDQ_ERR_INVALID_ARG, "Y must be 16-byte aligned with ldy >= N and a multiple of 8");
  DeviceGuard guard(w->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (w->precision == SVDQ_W4A16) return do_w4a16(w, X, M, ldx, Y, ldy, st);
  s = do_quant_down(w, X, M, ldx, workspace, st);
  if (s != SVDQ_OK) return s;
  return do_gemm(w, M, Y, ldy, workspace, st);
}

svdq_status svdq_linear_forward_gelu(const svdq_weights* w, const void* X, int M, int ldx, void* Y, int ldy,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  if (w && w->precision != SVDQ_NVFP4)
    return fail(SVDQ_ERR_INVALID_ARG, "the GELU-output forward runs on an NVFP4 layer (precision %d)", w->precision);
  svdq_status s = check_forward_common(w, M, workspace, workspace_bytes);
  if (s != SVDQ_OK || M == 0) return s;
  if (!Y) return fail(SVDQ_ERR_INVALID_ARG, "Y is NULL");
  if (ldy < w->N || ldy % 8 != 0 || !aligned(Y, 16))
    return fail(SVDQ_ERR_INVALID_ARG, "Y must be 16-byte aligned with ldy >= N and a multiple of 8");
  DeviceGuard guard(w->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = do_quant_down(w, X, M, ldx, workspace, st);
  if (s != SVDQ_OK) return s;
  return do_gemm(w, M, Y, ldy, workspace, st, nullptr, nullptr, true);
}

svdq_status svdq_export_activations(const svdq_weights* w, const void* workspace, size_t workspace_bytes, int M,
                                    uint8_t* codes_x, void* scales_x, uint16_t* T, void* stream) {
  if (w && w->precision == SVDQ_W4A16)
    return fail(SVDQ_ERR_INVALID_ARG, "the W4A16 layer runs as one kernel: use svdq_linear_forward");
  svdq_status s = check_forward_common(w, M, workspace, workspace_bytes);
  if (s != SVDQ_OK || M == 0) return s;
  DeviceGuard guard(w->device);
  const svdq::WorkspaceLayout L = svdq::workspace_layout(M, w->K, w->rank);
  std::vector<uint8_t> host(L.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(host.data(), workspace, L.total, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "copying the workspace to the host");
  const int K = w->K, KB = K / svdq::kBK, r = w->rank;
  for (int m = 0; m < M; ++m) {
    const int mt = m / svdq::kBM, row = m % svdq::kBM;
    if (codes_x) {
      for (int b = 0; b < K / 2; ++b) {
        const int kb = b / svdq::kRowBytes;
        codes_x[static_cast<size_t>(m) * (K / 2) + b] =
            host[L.codes + svdq::codes_chunk_offset(mt, kb, KB, svdq::kBM) + svdq::swz128(row, b % svdq::kRowBytes)];
      }
    }
    if (scales_x) {
      if (w->precision == SVDQ_NVFP4) {
        uint8_t* sx = static_cast<uint8_t*>(scales_x);
        for (int j = 0; j < K / 16; ++j) {
          const int kb = j / 16;
          sx[static_cast<size_t>(m) * (K / 16) + j] =
              host[L.sf + svdq::sf_chunk_offset(mt, kb, KB, svdq::kBM) + svdq::sf_nvfp4_offset(row, j % 16, svdq::kBM)];
        }
      } else {
        float* sx = static_cast<float*>(scales_x);
        for (int g = 0; g < K / 64; ++g) {
          const int kb = g / 4;
          std::memcpy(&sx[static_cast<size_t>(m) * (K / 64) + g],
                      &host[L.sf + svdq::sf_chunk_offset(mt, kb, KB, svdq::kBM) + 4 * svdq::sf_int4_a_index(row, g % 4)],
                      4);
        }
      }
    }
    if (T) {
      for (int i = 0; i < r; ++i)
        std::memcpy(&T[static_cast<size_t>(m) * r + i],
                    &host[L.t + static_cast<size_t>(mt) * svdq::kBM * r * 2 + svdq::lr_offset(row, i, svdq::kBM, r)], 2);
    }
  }
  return SVDQ_OK;
}

svdq_status svdq_selftest_wait_timeout(int spin_limit, void* stream) {
  if (spin_limit < 0) return fail(SVDQ_ERR_INVALID_ARG, "spin_limit must be >= 0");
  cudaError_t e = svdq::launch_selftest_wait(spin_limit, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "launch of the wait self-test kernel");
  return SVDQ_OK;
}

svdq_status svdq_selftest_gelu_bf16(const uint16_t* in, uint16_t* out, int n, void* stream) {
  if (n < 0) return fail(SVDQ_ERR_INVALID_ARG, "n=%d is negative", n);
  if (n > 0 && (!in || !out)) return fail(SVDQ_ERR_INVALID_ARG, "NULL buffer");
  cudaError_t e = svdq::launch_selftest_gelu(in, out, n, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "launch of the GELU self-test kernel");
  return SVDQ_OK;
}

}  // extern "C"
