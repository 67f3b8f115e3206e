// The two fused kernels of the SVDQuant W4A4 linear (SVDQuant model card, "Nunchaku Engine
// Design" (b): Down Projection fused with Quantize because they read the same input; Up
// Projection fused with 4-Bit Compute because they write the same output), for sm_100a.
//
// Kernel 1, quant_down: one CTA per (128-row M tile, K slice); the K slices of one M tile form
// a thread-block cluster.  Eight worker warps stream X from HBM once, apply the smoothing
// factor, quantize every K-group (NVFP4: UE4M3 scale per 16; INT4: fp32 scale per 64) into the
// tiled layouts kernel 2 copies verbatim, and stage bf16(x_hat) in shared memory; one warp feeds
// it with L1 to tcgen05 bf16 MMAs that accumulate T = x_hat L1 in tensor memory.  The cluster
// reduces its fp32 partials of T through distributed shared memory in a fixed order (so the
// result is deterministic) and writes bf16 T once.
//
// Kernel 2, gemm: persistent, warp specialised.  Warp 0 streams each (k-block) stage with 1-D
// bulk copies (the operands are stored as shared-memory images); warp 1 issues the tcgen05 MMAs:
// first the bf16 up projection T L2 (kind::f16) and then the block-scaled 4-bit GEMM
// (kind::mxf4nvf4 with UE4M3 scales copied into tensor memory by tcgen05.cp) into the same fp32
// accumulator in tensor memory; eight epilogue warps drain the accumulator, add the bias and
// write bf16 Y once.
#include <cuda_bf16.h>

#include "kernels.h"
#include "layout.h"
#include "ptx.cuh"

namespace svdq {

// ============================================================================ kernel 1

constexpr int kQdStages = 4;
constexpr int kQdWorkerWarps = 8;
constexpr int kQdThreads = (kQdWorkerWarps + 1) * 32;
constexpr int kXsBytes = kBM * 128;  // bf16 x_hat: 128 rows x 64 columns, 128-byte swizzle

struct QdParams {
  const uint16_t* X;
  int M, K, ldx, rank, KB, splits;
  const float* inv_lambda;
  const uint8_t* l1;
  uint8_t* codes;
  uint8_t* sf;
  uint8_t* t;
};

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Quantizes this lane's 8 smoothed values (a 16-group spans a lane pair; a 64-group spans the 8
// lanes of a row).  Returns the packed codes (element 2i in the low nibble of byte i) and, in
// `scale_bits`, the group scale (UE4M3 byte or fp32 bits).
template <int PREC>
__device__ __forceinline__ uint32_t quantize8(const float (&xh)[8], uint32_t& scale_bits) {
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(xh[j]));
  uint32_t codes = 0;
  if (PREC == 0) {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    const float s = __fdiv_rn(amax, 6.0f);
    const uint32_t sc = cvt_e4m3(s);
    const float sd = e4m3_to_f32(sc);
    scale_bits = sc;
    if (sd != 0.0f) {
#pragma unroll
      for (int t = 0; t < 4; ++t)
        codes |= cvt_e2m1x2(__fdiv_rn(xh[2 * t], sd), __fdiv_rn(xh[2 * t + 1], sd)) << (8 * t);
    }
  } else {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    const float s = __fdiv_rn(amax, 7.0f);
    scale_bits = __float_as_uint(s);
    if (s != 0.0f) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        int q = __float2int_rn(__fdiv_rn(xh[j], s));
        q = max(-8, min(7, q));
        codes |= (static_cast<uint32_t>(q) & 0xFu) << (4 * j);
      }
    }
  }
  return codes;
}

template <int PREC>
__global__ void __launch_bounds__(kQdThreads, 1) quant_down_kernel(const QdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int r = p.rank;
  const bool has_lr = r > 0;
  const uint32_t l1_stage_bytes = static_cast<uint32_t>(r) * 128u;
  uint8_t* xs = smem;                                              // kQdStages x 16 KB
  uint8_t* l1s = smem + kQdStages * kXsBytes;                      // kQdStages x r*128
  uint64_t* bars = reinterpret_cast<uint64_t*>(l1s + kQdStages * align_up(l1_stage_bytes, 1024));
  uint64_t* xfull = bars;                   // workers -> MMA (count 8)
  uint64_t* l1full = bars + kQdStages;      // L1 copy landed (count 1 + tx)
  uint64_t* empty = bars + 2 * kQdStages;   // MMA done reading the stage (tcgen05.commit)
  uint64_t* done = bars + 3 * kQdStages;    // all MMAs of this CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;  // == rank in the cluster (clusters are consecutive blocks)
  const int kb0 = split * p.KB / p.splits, kb1 = (split + 1) * p.KB / p.splits;
  const int c0 = kb0 * 4, nch = (kb1 - kb0) * 4;
  const uint32_t tmem_cols = r <= 32 ? 32u : (r <= 64 ? 64u : 128u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQdStages; ++s) {
      mbar_init(&xfull[s], kQdWorkerWarps);
      mbar_init(&l1full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (has_lr && warp == kQdWorkerWarps) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = has_lr ? *tmem_slot : 0u;

  if (warp < kQdWorkerWarps) {
    // ------------------------------------------------------------ workers
    const int sub = lane >> 3, kg = lane & 7;
    const uint8_t* xrow[4];
    bool rvalid[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = mt * kBM + warp * 16 + i * 4 + sub;
      rvalid[i] = row < p.M;
      xrow[i] = reinterpret_cast<const uint8_t*>(p.X + static_cast<size_t>(rvalid[i] ? row : 0) * p.ldx);
    }
    uint4 cur[4], nxt[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int col = c0 * 64 + kg * 8;
      cur[i] = rvalid[i] ? ld_stream_v4(xrow[i] + static_cast<size_t>(col) * 2) : make_uint4(0, 0, 0, 0);
    }
    for (int c = 0; c < nch; ++c) {
      const int gc = c0 + c;
      if (c + 1 < nch) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int col = (gc + 1) * 64 + kg * 8;
          nxt[i] = rvalid[i] ? ld_stream_v4(xrow[i] + static_cast<size_t>(col) * 2) : make_uint4(0, 0, 0, 0);
        }
      }
      const int col = gc * 64 + kg * 8;
      const float4 il0 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + col));
      const float4 il1 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + col + 4));
      const float il[8] = {il0.x, il0.y, il0.z, il0.w, il1.x, il1.y, il1.z, il1.w};
      const int kb = gc >> 2, cc = gc & 3;
      const int st = c % kQdStages;
      if (has_lr && c >= kQdStages) {
        if (!wait_parity_bounded(&empty[st], ((c / kQdStages) - 1) & 1, kErrWaitQuantDown)) {
          *abort_flag = 1;
          break;
        }
      }
      uint8_t* codes_chunk = p.codes + codes_chunk_offset(mt, kb, p.KB, kBM);
      uint8_t* sf_chunk = p.sf + sf_chunk_offset(mt, kb, p.KB, kBM);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = warp * 16 + i * 4 + sub;  // row inside the tile
        const uint32_t w[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w};
        float xh[8];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          xh[2 * t] = __fmul_rn(__uint_as_float(w[t] << 16), il[2 * t]);
          xh[2 * t + 1] = __fmul_rn(__uint_as_float(w[t] & 0xFFFF0000u), il[2 * t + 1]);
        }
        uint32_t sbits;
        const uint32_t codes = quantize8<PREC>(xh, sbits);
        *reinterpret_cast<uint32_t*>(codes_chunk + swz128(row, cc * 32 + kg * 4)) = codes;
        if (PREC == 0) {
          const uint32_t s1 = __shfl_down_sync(0xffffffffu, sbits, 2);
          const uint32_t s2 = __shfl_down_sync(0xffffffffu, sbits, 4);
          const uint32_t s3 = __shfl_down_sync(0xffffffffu, sbits, 6);
          if (kg == 0)
            *reinterpret_cast<uint32_t*>(sf_chunk + cc * 512 + (row & 31) * 16 + (row >> 5) * 4) =
                sbits | (s1 << 8) | (s2 << 16) | (s3 << 24);
        } else {
          if (kg == 0) reinterpret_cast<uint32_t*>(sf_chunk)[sf_int4_a_index(row, cc)] = sbits;
        }
        if (has_lr) {
          uint4 hv;
          hv.x = pack_bf16x2(xh[0], xh[1]);
          hv.y = pack_bf16x2(xh[2], xh[3]);
          hv.z = pack_bf16x2(xh[4], xh[5]);
          hv.w = pack_bf16x2(xh[6], xh[7]);
          *reinterpret_cast<uint4*>(xs + st * kXsBytes + swz128(row, kg * 16)) = hv;
        }
      }
      if (has_lr) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&xfull[st]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
    }
  } else if (has_lr && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16(128, r);
    int pcount = 0;  // L1 chunks whose copy has been issued
    bool ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      while (pcount < nch && pcount < c + kQdStages) {
        const int sp = pcount % kQdStages;
        if (pcount >= kQdStages && !wait_parity_bounded(&empty[sp], ((pcount / kQdStages) - 1) & 1, kErrWaitQuantDown)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&l1full[sp], l1_stage_bytes);
        bulk_g2s(l1s + sp * align_up(l1_stage_bytes, 1024), p.l1 + static_cast<size_t>(c0 + pcount) * l1_stage_bytes,
                 l1_stage_bytes, &l1full[sp]);
        ++pcount;
      }
      if (!ok) break;
      const int st = c % kQdStages;
      const uint32_t par = (c / kQdStages) & 1;
      if (!wait_parity_bounded(&l1full[st], par, kErrWaitQuantDown) ||
          !wait_parity_bounded(&xfull[st], par, kErrWaitQuantDown)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t ad = smem_desc(smem_u32(xs + st * kXsBytes), 16, 1024, kLayoutSw128);
      const uint64_t bd = smem_desc(smem_u32(l1s + st * align_up(l1_stage_bytes, 1024)), 16, 1024, kLayoutSw128);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16(tmem_base, ad + 2 * ks, bd + 2 * ks, idesc, (c | ks) != 0 ? 1u : 0u);
      tc_commit(&empty[st]);
    }
    tc_commit(done);
    if (!ok) {
      *abort_flag = 1;
      // Let every issued L1 copy land before the CTA can retire.
      for (int q = 0; q < pcount; ++q)
        wait_parity_bounded(&l1full[q % kQdStages], (q / kQdStages) & 1, kErrWaitQuantDown);
    }
  }

  // ---------------------------------------------------------------- T epilogue
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  float* part = reinterpret_cast<float*>(xs);  // 128 x r fp32 partial (reuses the x_hat stages)
  if (has_lr && warp < 4) {
    bool ok = !aborted && wait_parity_bounded(done, 0, kErrWaitQuantDown);
    ok = __all_sync(0xffffffffu, ok);  // the TMEM loads below are warp-collective
    tc_fence_after();
    if (ok) {
      const int row = warp * 32 + lane;
      for (int j = 0; j < r; j += 16) {
        uint32_t v[16];
        tmem_ld16(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + j, v);
        tmem_wait_ld();
        if (p.splits == 1) {
          uint8_t* tt = p.t + static_cast<size_t>(mt) * kBM * r * 2;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[8 * h + 0]), __uint_as_float(v[8 * h + 1]));
            o.y = pack_bf16x2(__uint_as_float(v[8 * h + 2]), __uint_as_float(v[8 * h + 3]));
            o.z = pack_bf16x2(__uint_as_float(v[8 * h + 4]), __uint_as_float(v[8 * h + 5]));
            o.w = pack_bf16x2(__uint_as_float(v[8 * h + 6]), __uint_as_float(v[8 * h + 7]));
            *reinterpret_cast<uint4*>(tt + lr_offset(row, j + 8 * h, kBM, r)) = o;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 16; q += 4)
            *reinterpret_cast<float4*>(part + row * r + j + q) =
                make_float4(__uint_as_float(v[q]), __uint_as_float(v[q + 1]), __uint_as_float(v[q + 2]),
                            __uint_as_float(v[q + 3]));
        }
      }
    }
  }
  if (has_lr && p.splits > 1) {
    // Fixed-order reduction of the cluster's partials: rank s sums rows [s*128/S, (s+1)*128/S).
    // Every thread of every CTA passes both cluster barriers, whatever happened before.
    cluster_sync();
    if (warp < kQdWorkerWarps && !aborted) {
      const int rlo = split * kBM / p.splits, rhi = (split + 1) * kBM / p.splits;
      const int units = (rhi - rlo) * r / 4;
      const uint32_t part_addr = smem_u32(part);
      uint8_t* tt = p.t + static_cast<size_t>(mt) * kBM * r * 2;
      for (int u = threadIdx.x; u < units; u += kQdWorkerWarps * 32) {
        const int row = rlo + (u * 4) / r, col = (u * 4) % r;
        const uint32_t off = static_cast<uint32_t>((row * r + col) * 4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int q = 0; q < p.splits; ++q) {
          const float4 x = ld_shared_cluster_f4(mapa_shared(part_addr + off, static_cast<uint32_t>(q)));
          acc.x += x.x;
          acc.y += x.y;
          acc.z += x.z;
          acc.w += x.w;
        }
        uint2 o;
        o.x = pack_bf16x2(acc.x, acc.y);
        o.y = pack_bf16x2(acc.z, acc.w);
        *reinterpret_cast<uint2*>(tt + lr_offset(row, col, kBM, r)) = o;
      }
    }
    cluster_sync();
  }
  tc_fence_before();
  __syncthreads();
  if (has_lr && warp == kQdWorkerWarps) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

int quant_down_splits(int M, int K, int num_sms) {
  const int mt = (M + kBM - 1) / kBM;
  const int KB = K / kBK;
  int s = 1;
  // Enough CTAs to keep every SM streaming; the K slices of a tile form one cluster (<= 8).
  while (s < 8 && s * 2 <= KB && mt * s < num_sms) s *= 2;
  return s;
}

static size_t quant_down_smem_bytes(int r) {
  return 1024 + kQdStages * kXsBytes + kQdStages * align_up(static_cast<size_t>(r) * 128, 1024) + 256;
}

cudaError_t launch_quant_down(const QuantDownArgs& a, int num_sms, cudaStream_t stream) {
  QdParams p;
  p.X = a.X;
  p.M = a.M;
  p.K = a.K;
  p.ldx = a.ldx;
  p.rank = a.rank;
  p.KB = a.K / kBK;
  p.splits = quant_down_splits(a.M, a.K, num_sms);
  p.inv_lambda = a.inv_lambda;
  p.l1 = a.l1;
  p.codes = a.codes;
  p.sf = a.sf;
  p.t = a.t;
  const int mt = (a.M + kBM - 1) / kBM;
  const size_t smem = quant_down_smem_bytes(a.rank);
  void (*kern)(const QdParams) = a.precision == 0 ? quant_down_kernel<0> : quant_down_kernel<1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(mt * p.splits));
  cfg.blockDim = dim3(kQdThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(p.splits);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

// ============================================================================ kernel 2

constexpr int kGStages = 4;
constexpr int kGEpiWarps = 8;
constexpr int kGThreads = (2 + kGEpiWarps) * 32;
constexpr uint32_t kGA = kBM * kRowBytes;                     // 16 KB
constexpr uint32_t kGB = kBN * kRowBytes;                     // 32 KB
constexpr uint32_t kGSfa = kBM * kSfBytesPerRowKb;            // 2 KB
constexpr uint32_t kGSfb = kBN * kSfBytesPerRowKb;            // 4 KB
constexpr uint32_t kGStage = kGA + kGB + kGSfa + kGSfb;       // 54 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemSfa = 256, kTmemSfb = 272;

struct GemmParams {
  int M, N, K, rank, KB, MT, NT, ldy;
  const uint8_t* a_codes;
  const uint8_t* a_sf;
  const uint8_t* t;
  const uint8_t* b_codes;
  const uint8_t* b_sf;
  const uint8_t* l2;
  const float* bias;
  uint16_t* Y;
};

__global__ void __launch_bounds__(kGThreads, 1) gemm_nvfp4_kernel(const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kGStage);
  uint64_t* empty = full + kGStages;
  uint64_t* acc_full = empty + kGStages;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = p.rank;
  const int nlr = (r + kLrChunk - 1) / kLrChunk;
  const int tiles = p.MT * p.NT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kGEpiWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int st = 0;
      uint32_t ph = 0;
      int issued_phase[kGStages];
      for (int s = 0; s < kGStages; ++s) issued_phase[s] = -1;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int mt = tile / p.NT, nt = tile % p.NT;
        const int nstages = nlr + p.KB;
        for (int j = 0; j < nstages; ++j) {
          if (*abort_flag || !wait_parity_bounded(&empty[st], ph ^ 1u, kErrWaitGemm)) {
            ok = false;
            break;
          }
          uint8_t* sbase = smem + st * kGStage;
          if (j < nlr) {
            const uint32_t cw = lr_chunk_width(r, j);
            const uint32_t tb = kBM * cw * 2, lb = kBN * cw * 2;
            mbar_arrive_expect_tx(&full[st], tb + lb);
            bulk_g2s(sbase, p.t + static_cast<size_t>(mt) * kBM * r * 2 + static_cast<size_t>(kBM) * kLrChunk * 2 * j, tb,
                     &full[st]);
            bulk_g2s(sbase + kGA, p.l2 + static_cast<size_t>(nt) * kBN * r * 2 + static_cast<size_t>(kBN) * kLrChunk * 2 * j,
                     lb, &full[st]);
          } else {
            const int kb = j - nlr;
            mbar_arrive_expect_tx(&full[st], kGStage);
            bulk_g2s(sbase, p.a_codes + codes_chunk_offset(mt, kb, p.KB, kBM), kGA, &full[st]);
            bulk_g2s(sbase + kGA, p.b_codes + codes_chunk_offset(nt, kb, p.KB, kBN), kGB, &full[st]);
            bulk_g2s(sbase + kGA + kGB, p.a_sf + sf_chunk_offset(mt, kb, p.KB, kBM), kGSfa, &full[st]);
            bulk_g2s(sbase + kGA + kGB + kGSfa, p.b_sf + sf_chunk_offset(nt, kb, p.KB, kBN), kGSfb, &full[st]);
          }
          issued_phase[st] = static_cast<int>(ph);
          if (++st == kGStages) {
            st = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        for (int s = 0; s < kGStages; ++s)
          if (issued_phase[s] >= 0) wait_parity_bounded(&full[s], static_cast<uint32_t>(issued_phase[s]), kErrWaitGemm);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t id_lr = idesc_bf16(128, 256);
      const uint32_t id_fp4 = idesc_nvfp4(128, 256);
      int st = 0;
      uint32_t ph = 0;
      bool ok = true;
      int local = 0;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++local) {
        if (*abort_flag || !wait_parity_bounded(acc_empty, (static_cast<uint32_t>(local) & 1u) ^ 1u, kErrWaitGemm)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t accum = 0;
        const int nstages = nlr + p.KB;
        for (int j = 0; j < nstages; ++j) {
          if (*abort_flag || !wait_parity_bounded(&full[st], ph, kErrWaitGemm)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + st * kGStage);
          if (j < nlr) {
            const uint32_t cw = lr_chunk_width(r, j);
            const uint64_t ad = smem_desc(sb, 128, cw * 16, kLayoutNone);
            const uint64_t bd = smem_desc(sb + kGA, 128, cw * 16, kLayoutNone);
            for (uint32_t ks = 0; ks < cw / 16; ++ks) {
              mma_bf16(tmem, ad + 16 * ks, bd + 16 * ks, id_lr, accum);
              accum = 1;
            }
          } else {
            const uint32_t sfa = sb + kGA + kGB, sfb = sfa + kGSfa;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              tmem_cp_32x128_warpx4(tmem + kTmemSfa + 4 * kk, smem_desc(sfa + 512 * kk, 0, 128, kLayoutNone));
              tmem_cp_32x128_warpx4(tmem + kTmemSfb + 8 * kk, smem_desc(sfb + 1024 * kk, 0, 128, kLayoutNone));
              tmem_cp_32x128_warpx4(tmem + kTmemSfb + 8 * kk + 4, smem_desc(sfb + 1024 * kk + 512, 0, 128, kLayoutNone));
            }
            const uint64_t ad = smem_desc(sb, 16, 1024, kLayoutSw128);
            const uint64_t bd = smem_desc(sb + kGA, 16, 1024, kLayoutSw128);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_nvfp4(tmem, ad + 2 * kk, bd + 2 * kk, id_fp4, tmem + kTmemSfa + 4 * kk, tmem + kTmemSfb + 8 * kk,
                        accum);
              accum = 1;
            }
          }
          tc_commit(&empty[st]);
          if (++st == kGStages) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      if (!ok) {
        *abort_flag = 1;
        // Make sure no issued tcgen05 operation is still running when TMEM is released.
        tc_commit(acc_full);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (8 warps)
    const int q = warp & 3, h = (warp - 2) >> 2;
    int local = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++local) {
      bool ok = !*abort_flag && wait_parity_bounded(acc_full, static_cast<uint32_t>(local) & 1u, kErrWaitGemm);
      if (!__all_sync(0xffffffffu, ok)) {  // the TMEM loads below are warp-collective
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int mt = tile / p.NT, nt = tile % p.NT;
      uint32_t v[4][32];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(h * 128 + i * 32), v[i]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      const int row = mt * kBM + q * 32 + lane;
      const int n0 = nt * kBN + h * 128;
      if (row < p.M) {
        uint16_t* yrow = p.Y + static_cast<size_t>(row) * p.ldy;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int n = n0 + i * 32 + g * 8;
            if (n < p.N) {
              const float4 b0 = __ldg(reinterpret_cast<const float4*>(p.bias + n));
              const float4 b1 = __ldg(reinterpret_cast<const float4*>(p.bias + n + 4));
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(v[i][g * 8 + 0]) + b0.x, __uint_as_float(v[i][g * 8 + 1]) + b0.y);
              o.y = pack_bf16x2(__uint_as_float(v[i][g * 8 + 2]) + b0.z, __uint_as_float(v[i][g * 8 + 3]) + b0.w);
              o.z = pack_bf16x2(__uint_as_float(v[i][g * 8 + 4]) + b1.x, __uint_as_float(v[i][g * 8 + 5]) + b1.y);
              o.w = pack_bf16x2(__uint_as_float(v[i][g * 8 + 6]) + b1.z, __uint_as_float(v[i][g * 8 + 7]) + b1.w);
              *reinterpret_cast<uint4*>(yrow + n) = o;
            }
          }
        }
      }
    }
  }

  // The MMA issuer's last commit (normal or abort) tells when no tcgen05 op is in flight.
  __syncthreads();
  if (warp == 1) {
    if (*abort_flag && lane == 0) {
      // acc_full received one extra commit in the abort path; wait for all of them to land.
      const unsigned long long t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 2000000ull) {
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

static size_t gemm_smem_bytes() { return 1024 + kGStages * kGStage + 256; }

cudaError_t launch_gemm(const GemmArgs& a, int num_sms, cudaStream_t stream) {
  GemmParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.rank = a.rank;
  p.KB = a.K / kBK;
  p.MT = (a.M + kBM - 1) / kBM;
  p.NT = (a.N + kBN - 1) / kBN;
  p.ldy = a.ldy;
  p.a_codes = a.a_codes;
  p.a_sf = a.a_sf;
  p.t = a.t;
  p.b_codes = a.b_codes;
  p.b_sf = a.b_sf;
  p.l2 = a.l2;
  p.bias = a.bias;
  p.Y = a.Y;
  if (a.precision != 0) return cudaErrorNotSupported;
  const size_t smem = gemm_smem_bytes();
  cudaError_t e =
      cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = p.MT * p.NT;
  const int grid = tiles < num_sms ? tiles : num_sms;
  gemm_nvfp4_kernel<<<grid, kGThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

// ============================================================================ failure detection

__global__ void selftest_wait_kernel(int spin_limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = false;
    for (int i = 0; i < spin_limit && !ok; ++i) ok = mbar_try_wait(&bar, 0);  // nothing ever arrives
    if (!ok) atomicOr(&g_device_error, kErrWaitSelftest);
  }
}

cudaError_t launch_selftest_wait(int spin_limit, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(spin_limit);
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(unsigned int* value, cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace svdq
