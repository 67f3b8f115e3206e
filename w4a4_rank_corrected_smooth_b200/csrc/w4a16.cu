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
// The "awq_w4a16" layer family: 4-bit weights with one fp32 scale per 64 elements along K, 16-bit
// activations, used where M is small (FLUX's modulation projections run on one token per image).
// HBM bound by the weights (half a byte an element), and at that rate a weight can afford about
// three instructions on the CUDA cores -- less than a convert-and-FMA chain needs.  So the
// contraction runs on the warp-level bf16 tensor-core MMA (m16n8k16, fp32 accumulation) with A
// from registers: a lane turns one 32-bit word of codes into four bf16x2 fragment registers with
// one LOP3 each (the code, sign-flipped, into the mantissa of 128: 136 + q exactly) and one
// bf16x2 subtract of 136 (exact); the group's four k-steps accumulate from zero and the group
// scale multiplies the result into the fp32 accumulator.  B (the activations) is staged once per
// CTA in shared memory in fragment order: bf16(fp32(x) * (1/lambda)).
//
// Work split: a CTA owns R blocks of 16 weight rows and all of K; its 8 warps take the 64-wide
// groups in turn (split K), each keeping the codes and scales of its next kWAhead groups in flight
// while it computes the current one; the warps' partial sums are added in warp order in shared
// memory (deterministic), the bias added, and Y written.  grid.y runs over passes of 8 MB rows of X.

constexpr int kWThreads = 256;
constexpr int kWWarps = kWThreads / 32;
constexpr int kWStageBytes = 96 * 1024;  // activation fragments staged per pass over K
constexpr int kWAhead = 3;               // groups of codes and scales in flight per warp

struct W4A16Params {
  const uint16_t* X;
  int M, K, ldx, N, ldy;
  const float* inv_lambda;
  const uint4* codes;    // [N/16][K/64][32] x 16 B, fragment order
  const float2* scales;  // [N/16][K/64][8] pairs (rows i, i + 8)
  const float* bias;
  uint16_t* Y;
  int G;        // K / 64
  int chunk_g;  // groups whose activation fragments are staged at a time
};

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Two codes (nibbles at bits 0-3 and 16-19 of w) -> bf16x2 of their signed values, exactly.
__device__ __forceinline__ uint32_t codes_to_bf16x2(uint32_t w) {
  uint32_t t;
  // (w & 0x000F000F) ^ 0x43084308: each half becomes bf16 128 + (v ^ 8) = 136 + q
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(t) : "r"(w), "r"(0x000F000Fu), "r"(0x43084308u));
  uint32_t q;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(t), "r"(0x43084308u));
  return q;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int R, int MB>
__global__ void __launch_bounds__(kWThreads) w4a16_kernel(const W4A16Params p) {
  extern __shared__ __align__(16) uint8_t smem_w[];
  uint4* xs = reinterpret_cast<uint4*>(smem_w);  // [MB][chunk_g][2 halves][32 lanes]
  float* red = reinterpret_cast<float*>(smem_w + static_cast<size_t>(MB) * p.chunk_g * 1024);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2;
  const int m0 = blockIdx.y * 8 * MB;
  const int nsets = (p.N + 16 * R - 1) / (16 * R);
  const bool one_chunk = p.G <= p.chunk_g;

  // Stage B for groups [gc, gc + ng): entry (mb, group gl, half h, lane l) holds, for X row
  // m0 + 8 mb + l / 4 and the group's k-steps 2h and 2h + 1, the registers b0, b1 of each step
  // (element pairs at k = 16 s + 2 (l % 4) + {0, 1} and that + 8).  Filled from 16-byte loads of
  // 8 consecutive elements of a row (item = row, 8-element unit; consecutive threads take
  // consecutive units): their four pairs are register j = 2 (s % 2) + (k % 16 >= 8) of the four
  // lanes 4 (m % 8) + t, t = 0..3.
  uint32_t* const xw = reinterpret_cast<uint32_t*>(xs);
  auto stage = [&](int gc, int ng) {
    const int units = ng * 8;  // 8-element units of the chunk per row
    const int items = MB * 8 * units;
#pragma unroll 4
    for (int e = threadIdx.x; e < items; e += kWThreads) {
      const int ml = e / units, u = e - ml * units;  // row of the pass, unit of the chunk
      const int m = m0 + ml;
      const int k0 = gc * 64 + 8 * u;
      uint32_t v[4] = {0u, 0u, 0u, 0u};
      if (m < p.M) {
        const uint4 xx = *reinterpret_cast<const uint4*>(p.X + static_cast<size_t>(m) * p.ldx + k0);
        const float4 i0 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + k0));
        const float4 i1 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + k0 + 4));
        v[0] = bf16x2_bits(__fmul_rn(__uint_as_float(xx.x << 16), i0.x), __fmul_rn(__uint_as_float(xx.x & 0xFFFF0000u), i0.y));
        v[1] = bf16x2_bits(__fmul_rn(__uint_as_float(xx.y << 16), i0.z), __fmul_rn(__uint_as_float(xx.y & 0xFFFF0000u), i0.w));
        v[2] = bf16x2_bits(__fmul_rn(__uint_as_float(xx.z << 16), i1.x), __fmul_rn(__uint_as_float(xx.z & 0xFFFF0000u), i1.y));
        v[3] = bf16x2_bits(__fmul_rn(__uint_as_float(xx.w << 16), i1.z), __fmul_rn(__uint_as_float(xx.w & 0xFFFF0000u), i1.w));
      }
      const int kk = 8 * u;                 // element offset inside the chunk
      const int gl = kk >> 6, s16 = (kk >> 4) & 3, hi8 = (kk >> 3) & 1;
      const int mb = ml >> 3, gid = ml & 7;
      const int j = 2 * (s16 & 1) + hi8;
      uint32_t* dst = xw + ((((mb * ng + gl) * 2 + (s16 >> 1)) * 32 + 4 * gid) * 4 + j);
#pragma unroll
      for (int t = 0; t < 4; ++t) dst[4 * t] = v[t];  // lane 4 gid + t: entries of 4 words
    }
  };
  if (one_chunk) {
    stage(0, p.G);
    __syncthreads();
  }

  for (int set = blockIdx.x; set < nsets; set += gridDim.x) {
    const int b0 = set * R;
    float acc[R][MB][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[r][mb][j] = 0.0f;

    for (int gc = 0; gc < p.G; gc += p.chunk_g) {
      const int ng = p.G - gc < p.chunk_g ? p.G - gc : p.chunk_g;
      if (!one_chunk) {
        __syncthreads();  // the previous chunk's fragments are no longer read
        stage(gc, ng);
        __syncthreads();
      }
      // The warp's groups gl = warp, warp + 8, ...: the codes and scales of its next kWAhead groups
      // are in flight while one group's math runs.  Slot q holds the groups gb + q * 8 of the block
      // gb; a slot is refilled with the group kWAhead steps later as soon as its math is done.
      uint4 c[kWAhead][R];
      float2 s[kWAhead][R];
      auto fetch = [&](int q, int g) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          c[q][r] = make_uint4(0u, 0u, 0u, 0u);
          s[q][r] = make_float2(0.0f, 0.0f);
          if (g < ng) {
            const size_t cb = static_cast<size_t>(b0 + r) * p.G + gc + g;
            c[q][r] = __ldg(p.codes + cb * 32 + lane);
            s[q][r] = __ldg(p.scales + cb * 8 + gid);
          }
        }
      };
#pragma unroll
      for (int q = 0; q < kWAhead; ++q) fetch(q, warp + q * kWWarps);
      for (int gb = warp; gb < ng; gb += kWAhead * kWWarps) {
#pragma unroll
        for (int q = 0; q < kWAhead; ++q) {
          const int gl = gb + q * kWWarps;
          if (gl < ng) {
            uint4 bq[MB][2];
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
#pragma unroll
              for (int h = 0; h < 2; ++h) bq[mb][h] = xs[((mb * ng + gl) * 2 + h) * 32 + lane];
#pragma unroll
            for (int r = 0; r < R; ++r) {
              const uint32_t w[4] = {c[q][r].x, c[q][r].y, c[q][r].z, c[q][r].w};
              float d[MB][4];
#pragma unroll
              for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                for (int j = 0; j < 4; ++j) d[mb][j] = 0.0f;
#pragma unroll
              for (int st = 0; st < 4; ++st) {
                uint32_t a[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) a[j] = codes_to_bf16x2(w[st] >> (4 * j));
#pragma unroll
                for (int mb = 0; mb < MB; ++mb) {
                  const uint4& hb = bq[mb][st >> 1];
                  const uint32_t bb0 = (st & 1) ? hb.z : hb.x;
                  const uint32_t bb1 = (st & 1) ? hb.w : hb.y;
                  mma_bf16_16816(d[mb], a, bb0, bb1);
                }
              }
#pragma unroll
              for (int mb = 0; mb < MB; ++mb) {
                acc[r][mb][0] = fmaf(s[q][r].x, d[mb][0], acc[r][mb][0]);
                acc[r][mb][1] = fmaf(s[q][r].x, d[mb][1], acc[r][mb][1]);
                acc[r][mb][2] = fmaf(s[q][r].y, d[mb][2], acc[r][mb][2]);
                acc[r][mb][3] = fmaf(s[q][r].y, d[mb][3], acc[r][mb][3]);
              }
            }
            fetch(q, gl + kWAhead * kWWarps);
          }
        }
      }
    }

    // Split-K sum over the warps in warp order, bias, bf16, store.  Accumulator j of lane l is
    // weight row 16 b + l / 4 + 8 (j / 2) and X row 8 mb + 2 (l % 4) + j % 2.
    constexpr int kPer = R * MB * 4 * 32;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[warp * kPer + ((r * MB + mb) * 4 + j) * 32 + lane] = acc[r][mb][j];
    __syncthreads();
    for (int e = threadIdx.x; e < kPer; e += kWThreads) {
      float sum = 0.0f;
#pragma unroll
      for (int w = 0; w < kWWarps; ++w) sum += red[w * kPer + e];
      const int l = e & 31, j = (e >> 5) & 3, rm = e >> 7;
      const int mb = rm % MB, r = rm / MB;
      const int n = (b0 + r) * 16 + (l >> 2) + 8 * (j >> 1);
      const int m = m0 + 8 * mb + 2 * (l & 3) + (j & 1);
      if (n < p.N && m < p.M) {
        const __nv_bfloat16 y = __float2bfloat16_rn(sum + p.bias[n]);
        p.Y[static_cast<size_t>(m) * p.ldy + n] = *reinterpret_cast<const uint16_t*>(&y);
      }
    }
    __syncthreads();  // red is rewritten by the next set
  }
}

template <int R, int MB>
static cudaError_t launch_w4a16_rm(const W4A16Params& p0, int num_sms, cudaStream_t stream) {
  W4A16Params p = p0;
  const int chunk_max = kWStageBytes / (1024 * MB);
  p.chunk_g = p.G < chunk_max ? p.G : chunk_max;
  const size_t smem = static_cast<size_t>(MB) * p.chunk_g * 1024 + sizeof(float) * kWWarps * R * MB * 4 * 32;
  cudaError_t e = cudaFuncSetAttribute(w4a16_kernel<R, MB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, w4a16_kernel<R, MB>, kWThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int nsets = (p.N + 16 * R - 1) / (16 * R);
  const int ctas = nsets < per_sm * num_sms ? nsets : per_sm * num_sms;
  const int rows_per_pass = 8 * MB;
  // grid.y is limited to 65535 passes: larger M runs in several launches
  constexpr int kPassesPerLaunch = 65535;
  const int passes = (p.M + rows_per_pass - 1) / rows_per_pass;
  for (int q0 = 0; q0 < passes; q0 += kPassesPerLaunch) {
    W4A16Params pq = p;
    const int np = passes - q0 < kPassesPerLaunch ? passes - q0 : kPassesPerLaunch;
    pq.X = p.X + static_cast<size_t>(q0) * rows_per_pass * p.ldx;
    pq.Y = p.Y + static_cast<size_t>(q0) * rows_per_pass * p.ldy;
    pq.M = p.M - q0 * rows_per_pass;
    w4a16_kernel<R, MB><<<dim3(static_cast<unsigned>(ctas), static_cast<unsigned>(np)), kWThreads, smem, stream>>>(pq);
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
  p.codes = reinterpret_cast<const uint4*>(a.codes);
  p.scales = reinterpret_cast<const float2*>(a.scales);
  p.bias = a.bias;
  p.Y = a.Y;
  p.G = a.K / 64;
  p.chunk_g = 0;
  // Rows of X per pass: 16 (two 8-column MMA tiles share each converted A fragment) once M > 8.
  // Weight rows per task: 64 while that still gives two tasks per SM, else 32, else 16.
  const bool two = a.M > 8;
  const int blocks16 = (a.N + 15) / 16;
  if (blocks16 >= 4 * 2 * num_sms * 9 / 10)
    return two ? launch_w4a16_rm<4, 2>(p, num_sms, stream) : launch_w4a16_rm<4, 1>(p, num_sms, stream);
  if (blocks16 >= 2 * 2 * num_sms * 9 / 10)
    return two ? launch_w4a16_rm<2, 2>(p, num_sms, stream) : launch_w4a16_rm<2, 1>(p, num_sms, stream);
  return two ? launch_w4a16_rm<1, 2>(p, num_sms, stream) : launch_w4a16_rm<1, 1>(p, num_sms, stream);
}

}  // namespace svdq
