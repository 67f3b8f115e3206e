// The W4A16 layer's forward for sm_100a: 4-bit weights with 16-bit activations, the "awq_w4a16"
// layer family ("Introducing Nunchaku Lite"; the quantization_config of "Native loading in
// Diffusers": int4, group size 64).  The pages fix only the weight format; this library reads it
// as the W4A4 layer's smoothing with the INT4 group-64 quantizer applied to the smoothed weight,
// no low-rank branch, activations bf16(x * (1/lambda)), fp32 accumulation, bias, bf16 output.

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels.h"

namespace svdq {

// ============================================================================ W4A16
//
// The "awq_w4a16" layer family: 4-bit weights (INT4, one fp32 scale per 64 elements along K, the
// smoothed weight's codes in canonical row-major layout), 16-bit activations, for small M (the
// modulation projections run on one token per image).  Memory bound: the weights are read once.
// A block stages MT rows of bf16(x_hat) = bf16(fp32(x) * (1/lambda)) in shared memory as fp32;
// each warp then computes one output row n at a time: lane l takes 8 consecutive elements of every
// 256 (a coalesced 4-byte word of codes), converts the codes exactly to fp32, dots them with x_hat,
// scales the partial by the group scale and accumulates in fp32; a warp reduction and the bias
// finish the row.

struct W4A16Params {
  const uint16_t* X;
  int M, K, ldx, N, ldy;
  const float* inv_lambda;
  const uint8_t* codes;
  const float* scales;
  const float* bias;
  uint16_t* Y;
};

template <int MT>
__global__ void __launch_bounds__(256) w4a16_kernel(const W4A16Params p) {
  extern __shared__ __align__(16) float xs[];  // MT x K
  const int m0 = blockIdx.y * MT;
  const int k8n = p.K / 8;
  for (int i = threadIdx.x; i < MT * k8n; i += blockDim.x) {
    const int mi = i / k8n, k8 = (i - mi * k8n) * 8;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0.0f;
    if (m0 + mi < p.M) {
      const uint4 x = *reinterpret_cast<const uint4*>(p.X + static_cast<size_t>(m0 + mi) * p.ldx + k8);
      const float4 i0 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + k8));
      const float4 i1 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + k8 + 4));
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
      const float il[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        // x_hat = fp32(x) * (1/lambda) (one rounding), then the 16-bit activation bf16(x_hat)
        v[2 * t] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(__uint_as_float(w[t] << 16), il[2 * t])));
        v[2 * t + 1] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(__uint_as_float(w[t] & 0xFFFF0000u), il[2 * t + 1])));
      }
    }
    float4* dst = reinterpret_cast<float4*>(xs + static_cast<size_t>(mi) * p.K + k8);
    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int n = blockIdx.x * 8 + warp; n < p.N; n += gridDim.x * 8) {
    const uint32_t* crow = reinterpret_cast<const uint32_t*>(p.codes + static_cast<size_t>(n) * (p.K / 2));
    const float* srow = p.scales + static_cast<size_t>(n) * (p.K / 64);
    float acc[MT];
#pragma unroll
    for (int mi = 0; mi < MT; ++mi) acc[mi] = 0.0f;
#pragma unroll 4
    for (int k0 = lane * 8; k0 < p.K; k0 += 256) {
      const uint32_t c = __ldg(crow + k0 / 8);  // elements k0 .. k0 + 7, element j in nibble j
      const float s = __ldg(srow + k0 / 64);
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // code nibble -> its signed value exactly: (nibble ^ 8) is value + 8 in [0, 15]; placed in
        // the low mantissa bits of 2^23 and 2^23 + 8 subtracted
        q[j] = __uint_as_float(((c >> (4 * j)) & 0xFu) ^ 0x4B000008u) - 8388616.0f;
      }
#pragma unroll
      for (int mi = 0; mi < MT; ++mi) {
        const float4 xa = *reinterpret_cast<const float4*>(xs + static_cast<size_t>(mi) * p.K + k0);
        const float4 xb = *reinterpret_cast<const float4*>(xs + static_cast<size_t>(mi) * p.K + k0 + 4);
        float part = q[0] * xa.x;
        part = fmaf(q[1], xa.y, part);
        part = fmaf(q[2], xa.z, part);
        part = fmaf(q[3], xa.w, part);
        part = fmaf(q[4], xb.x, part);
        part = fmaf(q[5], xb.y, part);
        part = fmaf(q[6], xb.z, part);
        part = fmaf(q[7], xb.w, part);
        acc[mi] = fmaf(part, s, acc[mi]);
      }
    }
#pragma unroll
    for (int mi = 0; mi < MT; ++mi)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[mi] += __shfl_xor_sync(0xffffffffu, acc[mi], o);
    if (lane == 0) {
      const float b = p.bias[n];
#pragma unroll
      for (int mi = 0; mi < MT; ++mi)
        if (m0 + mi < p.M) {
          const __nv_bfloat16 y = __float2bfloat16_rn(acc[mi] + b);
          p.Y[static_cast<size_t>(m0 + mi) * p.ldy + n] = *reinterpret_cast<const uint16_t*>(&y);
        }
    }
  }
}

template <int MT>
static cudaError_t launch_w4a16_mt(const W4A16Params& p, int num_sms, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(MT) * p.K * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(w4a16_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // Rows in launches of at most 65535 row tiles (the grid's y limit).
  constexpr int kRowsPerLaunch = 65535 * MT;
  for (int m = 0; m < p.M; m += kRowsPerLaunch) {
    W4A16Params q = p;
    q.M = p.M - m < kRowsPerLaunch ? p.M - m : kRowsPerLaunch;
    q.X = p.X + static_cast<size_t>(m) * p.ldx;
    q.Y = p.Y + static_cast<size_t>(m) * p.ldy;
    const int mtiles = (q.M + MT - 1) / MT;
    int bx = (q.N + 7) / 8;
    const int cap = num_sms * 4 / (mtiles < 4 ? mtiles : 4);
    if (bx > cap) bx = cap > 0 ? cap : 1;
    w4a16_kernel<MT><<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(mtiles)), 256, smem, stream>>>(q);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_w4a16(const W4A16Args& a, int num_sms, cudaStream_t stream) {
  W4A16Params p;
  p.X = a.X;
  p.M = a.M;
  p.K = a.K;
  p.ldx = a.ldx;
  p.N = a.N;
  p.ldy = a.ldy;
  p.inv_lambda = a.inv_lambda;
  p.codes = a.codes;
  p.scales = a.scales;
  p.bias = a.bias;
  p.Y = a.Y;
  // Rows of x_hat staged per block: as many as the M x K fp32 tile allows in ~192 KB, up to 4.
  const size_t budget = 192 * 1024;
  if (a.M >= 4 && 4 * static_cast<size_t>(a.K) * 4 <= budget) return launch_w4a16_mt<4>(p, num_sms, stream);
  if (a.M >= 2 && 2 * static_cast<size_t>(a.K) * 4 <= budget) return launch_w4a16_mt<2>(p, num_sms, stream);
  return launch_w4a16_mt<1>(p, num_sms, stream);
}

}  // namespace svdq
