// The W4A16 layer's forward for sm_100a: 4-bit weights with 16-bit activations, the "awq_w4a16"
// layer family ("Introducing Nunchaku Lite"; the quantization_config of "Native loading in
// Diffusers": int4, group size 64).  The pages fix only the weight format; this library reads it
// as the W4A4 layer's smoothing with the INT4 group-64 quantizer applied to the smoothed weight,
// no low-rank branch, activations bf16(x * (1/lambda)), fp32 accumulation, bias, bf16 output.

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels.h"

// This translation unit keeps a device error word of its own (read_and_clear_w4a16_error).
#define SVDQ_DEVICE_ERROR_DEFINED
namespace svdq {
static __device__ unsigned int g_device_error = 0;
}
#include "ptx.cuh"

namespace svdq {

// ============================================================================ W4A16
//
// Weight-only 4-bit layers run where M is small (FLUX's modulation projections: one token per
// image), so they are bound by reading the weights (half a byte an element) from HBM.  The weights
// are streamed, not fetched into registers: one producer thread per CTA keeps a ring of stages in
// flight with 1-D bulk copies (each stage: 16 groups of 64 along K of the CTA's R blocks of 16
// weight rows, codes and scales, 36 KB at R = 4), so an SM has ~100-150 KB of weights in flight
// without a register spent on them.  Sixteen consumer warps (four per scheduler, so that one
// warp's chain of dependent MMAs hides behind the others') take one group each per stage.
// The contraction runs on the warp-level bf16 tensor-core MMA (m16n8k16, fp32 accumulation) with A
// from registers: a lane turns one 32-bit word of codes into four bf16x2 fragment registers with one
// LOP3 each (the code, sign-flipped, into the mantissa of 128: 136 + q exactly) and one bf16x2
// subtract of 136 (exact); the group's four k-steps accumulate from zero and the group scale
// multiplies the result into the fp32 accumulator.  B (the activations) is staged once per CTA (per
// chunk of K) in shared memory in fragment order: bf16(fp32(x) * (1/lambda)).  The warps' partial
// sums are added in warp order in shared memory (deterministic), the bias added, and Y written.
// Codes are stored in fragment order, [N/16 blocks][K/64 groups][32 lanes][16 B], and scales as
// [blocks][groups][8 pairs (rows i, i + 8)] of fp32, so one (block, group) is 512 + 64 contiguous
// bytes and a stage's share of one block is one copy of each.

constexpr int kWWarps = 16;                     // consumer warps
constexpr int kWProducerWarp = kWWarps;         // one more warp: the producer (one thread)
constexpr int kWThreads = (kWWarps + 1) * 32;
constexpr int kWConsumers = kWWarps * 32;
constexpr int kWGs = kWWarps;                   // groups per stage: one per consumer warp
constexpr uint32_t kWCodeBytes = 512;           // one (block, group) of codes
constexpr uint32_t kWScaleBytes = 64;           // one (block, group) of scales
constexpr int kWMaxStages = 8;
constexpr size_t kWSmemBudget = 226 * 1024;
constexpr int kWBarrier = 1;                    // named barrier of the consumer warps

struct W4A16Params {
  const uint16_t* X;
  int M, K, ldx, N, ldy;
  const float* inv_lambda;
  const uint8_t* codes;   // [blocks][G][512 B]
  const uint8_t* scales;  // [blocks][G][64 B]
  const float* bias;
  uint16_t* Y;
  int G;        // K / 64
  int nsets;    // sets of R blocks
  int chunk_g;  // groups of x_hat fragments staged at a time: G, or a multiple of kWGs
  int stages;   // ring stages
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

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync %0, %1;" ::"n"(kWBarrier), "n"(kWConsumers) : "memory");
}

// Bytes of one ring stage for R blocks.
__host__ __device__ constexpr uint32_t w4a16_stage_bytes(int R) {
  return static_cast<uint32_t>(R) * kWGs * (kWCodeBytes + kWScaleBytes);
}

template <int R, int MB>
__global__ void __launch_bounds__(kWThreads, 1) w4a16_kernel(const W4A16Params p) {
  extern __shared__ __align__(128) uint8_t smem_w[];
  constexpr uint32_t kStage = w4a16_stage_bytes(R);
  constexpr uint32_t kStageScales = static_cast<uint32_t>(R) * kWGs * kWCodeBytes;  // scales after the codes
  constexpr int kPer = R * MB * 4 * 32;  // accumulators of one warp
  const int NS = p.stages;
  uint8_t* ring = smem_w;                                            // NS x kStage
  uint4* xs = reinterpret_cast<uint4*>(ring + static_cast<size_t>(NS) * kStage);  // [MB][chunk_g][2][32]
  float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(xs) + static_cast<size_t>(MB) * p.chunk_g * 1024);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + kWWarps * kPer);
  uint64_t* empty = full + kWMaxStages;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2;
  const int m0 = blockIdx.y * 8 * MB;
  const int nst = (p.G + kWGs - 1) / kWGs;  // stages per set
  const bool one_chunk = p.G <= p.chunk_g;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kWProducerWarp) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int slot = 0;
      uint32_t ph = 0;
      bool ok = true;
      long long issued = 0;
      for (int set = blockIdx.x; set < p.nsets; set += gridDim.x) {
        for (int st = 0; st < nst; ++st) {
          if (ok && !wait_parity_bounded(&empty[slot], ph ^ 1u, kErrWaitW4A16)) ok = false;
          if (ok) {
            const int g0 = st * kWGs;
            const int ng = p.G - g0 < kWGs ? p.G - g0 : kWGs;
            uint8_t* sb = ring + static_cast<size_t>(slot) * kStage;
            mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(R * ng) * (kWCodeBytes + kWScaleBytes));
#pragma unroll
            for (int r = 0; r < R; ++r) {
              const size_t bg = static_cast<size_t>(set * R + r) * p.G + g0;  // (block, first group)
              bulk_g2s(sb + static_cast<uint32_t>(r * kWGs) * kWCodeBytes, p.codes + bg * kWCodeBytes,
                       static_cast<uint32_t>(ng) * kWCodeBytes, &full[slot]);
              bulk_g2s(sb + kStageScales + static_cast<uint32_t>(r * kWGs) * kWScaleBytes, p.scales + bg * kWScaleBytes,
                       static_cast<uint32_t>(ng) * kWScaleBytes, &full[slot]);
            }
            ++issued;
          }
          if (++slot == NS) {
            slot = 0;
            ph ^= 1u;
          }
        }
      }
      // Before the CTA exits, every copy it issued has landed (the consumers saw most of them; after
      // a timeout they stop looking).
      const long long first = issued > NS ? issued - NS : 0;
      for (long long i = first; i < issued; ++i)
        if (!wait_parity_bounded(&full[i % NS], static_cast<uint32_t>((i / NS) & 1), kErrWaitW4A16)) break;
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  // Stage x_hat for groups [gc, gc + ng): entry (mb, group gl, half h, lane l) holds, for X row
  // m0 + 8 mb + l / 4 and the group's k-steps 2h and 2h + 1, the registers b0, b1 of each step
  // (element pairs at k = 16 s + 2 (l % 4) + {0, 1} and that + 8).  Filled from 16-byte loads of
  // 8 consecutive elements of a row (item = row, 8-element unit; consecutive threads take
  // consecutive units): their four pairs are register j = 2 (s % 2) + (k % 16 >= 8) of the four
  // lanes 4 (m % 8) + t, t = 0..3.  Only the pass's rows below M are staged (a single token per
  // image is the common case); the lanes of the rows past M take zero fragments instead of reading.
  uint32_t* const xw = reinterpret_cast<uint32_t*>(xs);
  const int rows_live = p.M - m0 < 8 * MB ? p.M - m0 : 8 * MB;
  auto stage_x = [&](int gc, int ng) {
    const int units = ng * 8;  // 8-element units of the chunk per row
    const int items = rows_live * units;
#pragma unroll 4
    for (int e = threadIdx.x; e < items; e += kWConsumers) {
      const int ml = e / units, u = e - ml * units;  // row of the pass, unit of the chunk
      const int m = m0 + ml;
      const int k0 = gc * 64 + 8 * u;
      uint32_t v[4];
      {
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
      const int mb = ml >> 3, gr = ml & 7;
      const int j = 2 * (s16 & 1) + hi8;
      uint32_t* dst = xw + ((((mb * ng + gl) * 2 + (s16 >> 1)) * 32 + 4 * gr) * 4 + j);
#pragma unroll
      for (int t = 0; t < 4; ++t) dst[4 * t] = v[t];  // lane 4 gr + t: entries of 4 words
    }
  };
  if (one_chunk) {
    stage_x(0, p.G);
    consumers_sync();
  }

  int slot = 0;
  uint32_t ph = 0;
  bool ok = true;
  for (int set = blockIdx.x; set < p.nsets; set += gridDim.x) {
    const int b0 = set * R;
    float acc[R][MB][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[r][mb][j] = 0.0f;
    int cg0 = 0, cng = p.G;  // the staged chunk: first group, groups
    for (int st = 0; st < nst; ++st) {
      const int g0 = st * kWGs;
      const int ng = p.G - g0 < kWGs ? p.G - g0 : kWGs;
      if (!one_chunk && g0 % p.chunk_g == 0) {
        cg0 = g0;
        cng = p.G - g0 < p.chunk_g ? p.G - g0 : p.chunk_g;
        consumers_sync();  // the previous chunk's fragments are no longer read
        stage_x(cg0, cng);
        consumers_sync();
      }
      if (ok) {
        bool w = true;
        if (lane == 0) w = wait_parity_bounded(&full[slot], ph, kErrWaitW4A16);
        ok = __shfl_sync(0xffffffffu, w, 0);
      }
      if (ok && warp < ng) {
        const int gl = g0 - cg0 + warp;  // the warp's group in the staged chunk
        uint4 bq[MB][2];
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            bq[mb][h] = 8 * mb + gid < rows_live ? xs[((mb * cng + gl) * 2 + h) * 32 + lane] : make_uint4(0u, 0u, 0u, 0u);
        const uint8_t* sb = ring + static_cast<size_t>(slot) * kStage;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint4 c = *reinterpret_cast<const uint4*>(sb + static_cast<uint32_t>(r * kWGs + warp) * kWCodeBytes + 16u * lane);
          const float2 s = *reinterpret_cast<const float2*>(sb + kStageScales +
                                                            static_cast<uint32_t>(r * kWGs + warp) * kWScaleBytes + 8u * gid);
          const uint32_t w[4] = {c.x, c.y, c.z, c.w};
          float d[MB][4];
#pragma unroll
          for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int j = 0; j < 4; ++j) d[mb][j] = 0.0f;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            uint32_t a[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) a[j] = codes_to_bf16x2(w[ks] >> (4 * j));
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) {
              const uint4& hb = bq[mb][ks >> 1];
              const uint32_t bb0 = (ks & 1) ? hb.z : hb.x;
              const uint32_t bb1 = (ks & 1) ? hb.w : hb.y;
              mma_bf16_16816(d[mb], a, bb0, bb1);
            }
          }
#pragma unroll
          for (int mb = 0; mb < MB; ++mb) {
            acc[r][mb][0] = fmaf(s.x, d[mb][0], acc[r][mb][0]);
            acc[r][mb][1] = fmaf(s.x, d[mb][1], acc[r][mb][1]);
            acc[r][mb][2] = fmaf(s.y, d[mb][2], acc[r][mb][2]);
            acc[r][mb][3] = fmaf(s.y, d[mb][3], acc[r][mb][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);  // this warp no longer reads the stage
      if (++slot == NS) {
        slot = 0;
        ph ^= 1u;
      }
    }

    // Split-K sum over the warps in warp order, bias, bf16, store.  Accumulator j of lane l is
    // weight row 16 b + l / 4 + 8 (j / 2) and X row 8 mb + 2 (l % 4) + j % 2.
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[warp * kPer + ((r * MB + mb) * 4 + j) * 32 + lane] = acc[r][mb][j];
    consumers_sync();
    for (int e = threadIdx.x; e < kPer; e += kWConsumers) {
      float sum = 0.0f;
#pragma unroll
      for (int w = 0; w < kWWarps; ++w) sum += red[w * kPer + e];
      const int l = e & 31, j = (e >> 5) & 3, rm = e >> 7;
      const int mb = rm % MB, r = rm / MB;
      const int n = (b0 + r) * 16 + (l >> 2) + 8 * (j >> 1);
      const int m = m0 + 8 * mb + 2 * (l & 3) + (j & 1);
      if (n < p.N && m < p.M && ok) {
        const __nv_bfloat16 y = __float2bfloat16_rn(sum + p.bias[n]);
        p.Y[static_cast<size_t>(m) * p.ldy + n] = *reinterpret_cast<const uint16_t*>(&y);
      }
    }
    consumers_sync();  // red is rewritten by the next set
  }
}

// Shared memory of one CTA: the ring, the staged x_hat chunk, the warps' partial sums, the barriers.
static size_t w4a16_smem(int R, int MB, int chunk_g, int stages) {
  return static_cast<size_t>(stages) * w4a16_stage_bytes(R) + static_cast<size_t>(MB) * chunk_g * 1024 +
         sizeof(float) * kWWarps * R * MB * 4 * 32 + 2 * kWMaxStages * sizeof(uint64_t);
}

template <int R, int MB>
static cudaError_t launch_w4a16_rm(const W4A16Params& p0, int num_sms, cudaStream_t stream) {
  W4A16Params p = p0;
  const int nblocks = (p.N + kBN - 1) / kBN * (kBN / 16);  // the packed weights are padded to 256 rows
  p.nsets = nblocks / R;
  // x_hat of all of K with as many stages as fit (at least three), else chunks of K with two
  p.chunk_g = p.G;
  int stages = kWMaxStages;
  while (stages > 3 && w4a16_smem(R, MB, p.chunk_g, stages) > kWSmemBudget) --stages;
  if (w4a16_smem(R, MB, p.chunk_g, stages) > kWSmemBudget) {
    stages = 2;
    const size_t fixed = w4a16_smem(R, MB, 0, stages);
    if (fixed >= kWSmemBudget) return cudaErrorInvalidConfiguration;
    p.chunk_g = static_cast<int>((kWSmemBudget - fixed) / (static_cast<size_t>(MB) * 1024)) / kWGs * kWGs;
    if (p.chunk_g < kWGs) return cudaErrorInvalidConfiguration;
  }
  p.stages = stages;
  const size_t smem = w4a16_smem(R, MB, p.chunk_g, stages);
  cudaError_t e = cudaFuncSetAttribute(w4a16_kernel<R, MB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int ctas = p.nsets < num_sms ? p.nsets : num_sms;  // one CTA per SM (shared memory)
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
  p.codes = a.codes;
  p.scales = reinterpret_cast<const uint8_t*>(a.scales);
  p.bias = a.bias;
  p.Y = a.Y;
  p.G = a.K / 64;
  p.nsets = 0;
  p.chunk_g = 0;
  p.stages = 0;
  // Rows of X per pass: 16 (two 8-column MMA tiles share each converted A fragment) once M > 8.
  // Blocks of 16 weight rows per set: 4 while that still gives about a set per SM, else 2, else 1.
  const bool two = a.M > 8;
  const int nblocks = (a.N + kBN - 1) / kBN * (kBN / 16);
  if (nblocks / 4 >= num_sms * 9 / 10)
    return two ? launch_w4a16_rm<4, 2>(p, num_sms, stream) : launch_w4a16_rm<4, 1>(p, num_sms, stream);
  if (nblocks / 2 >= num_sms * 9 / 10)
    return two ? launch_w4a16_rm<2, 2>(p, num_sms, stream) : launch_w4a16_rm<2, 1>(p, num_sms, stream);
  return two ? launch_w4a16_rm<1, 2>(p, num_sms, stream) : launch_w4a16_rm<1, 1>(p, num_sms, stream);
}

cudaError_t read_and_clear_w4a16_error(unsigned int* value, cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace svdq
