// The two fused kernels of the SVDQuant W4A4 linear (SVDQuant model card, "Nunchaku Engine
// Design" (b): Down Projection fused with Quantize because they read the same input; Up
// Projection fused with 4-Bit Compute because they write the same output), for sm_100a.
//
// Kernel 1, quant_down, in two forms.  Both apply the smoothing factor, quantize every K-group
// (NVFP4: UE4M3 scale per 16; INT4: fp32 scale per 64) with the same exact rounding into the tiled
// layouts kernel 2 copies verbatim, and compute T = bf16(x_hat) L1 deterministically.
// quant_down_kernel: one CTA of eight warps per 16 rows, each warp streaming its share of the rows'
// 64-column chunks into registers and feeding bf16(x_hat) from them to warp-level bf16 MMAs; the
// warps' shares of T are added through shared memory (layers of up to two waves of 16-row blocks,
// rank <= 32).  quant_down_tile_kernel: one CTA per (128-row tile, K slice), X by TMA, T by
// tcgen05 MMAs in tensor memory, K slices reduced by the last to arrive (larger layers and ranks).
//
// Kernel 2, gemm (NVFP4): persistent, warp specialised, on pairs of CTAs (cta_group::2 MMAs on
// 256 x 256 tiles).  Two producer threads stream each k-block stage (operand tiles and scale
// tiles) by TMA; four scale warps write the stage's UE4M3 scales into tensor memory with
// tcgen05.st; the MMA thread of the leader CTA issues the block-scaled 4-bit MMAs
// (kind::mxf4nvf4) and the bf16 up projection T L2 (kind::f16) into one fp32 accumulator in
// tensor memory; eight epilogue warps drain it, add the bias and write bf16 Y once by TMA.
// Kernel 2, gemm (INT4): as described at its own section below.
#include <cuda.h>
#include <atomic>
#include <mutex>
#include <cuda_bf16.h>

#include "kernels.h"
#include "layout.h"
#include "ptx.cuh"

namespace svdq {

// ============================================================================ kernel 1
//
// Smoothing, 4-bit activation quantization and the bf16 down projection T = bf16(x_hat) L1, with
// X read from HBM once.  One CTA of kQdWarps warps per block of 16 rows; warp w takes the 64-column
// chunks w, w + kQdWarps, ... of K, so the CTA sweeps its rows front to back.  Lane l (g = l / 4,
// j = l % 4) holds rows g and g + 8 of the block and, of every chunk, the columns 8j .. 8j + 7 and
// 32 + 8j .. 32 + 8j + 7: four 16-byte copies (each row of a warp's chunk is read by 4 lanes as 64
// contiguous bytes twice).  The copies run kQdAhead chunks ahead of their use, asynchronously into
// a per-warp ring in shared memory (so that a whole SM keeps ~100 KB of X in flight, which HBM's
// latency under load needs), and each lane reads back only what it copied itself.
//
// NVFP4: the 16-element group 2h + j / 2 of half h of a chunk lies in lanes j and j ^ 1 (one
// shuffle for its maximum); INT4: the 64-element group is the whole chunk row (two shuffles).
// The codes come from the same exactly bracketed quantizer as before (see quant_rows below).
//
// Down projection on warp-level bf16 MMAs (m16n8k16) straight from the registers that hold x_hat:
// the MMA's sum over k does not depend on the order of k, as long as A and B share it, so MMA s of
// half h reads, in lane j, the physical columns 32h + 8j + 4s .. + 3 where the fragment layout
// names the logical columns 2j, 2j + 1, 2j + 8, 2j + 9.  The matching B fragment of rank column n is
// then 8 contiguous bytes of L1's K-major layout: one 16-byte load serves both MMAs of a half.
// Each warp accumulates its chunks' share of T for its 16 rows in fp32; at the end the warps' shares
// are summed through shared memory in warp order (deterministic) and rounded to bf16 once.

constexpr int kQdWarps = 8;
constexpr int kQdThreads = kQdWarps * 32;
constexpr int kQdRows = 16;  // rows per CTA (the MMA's M)
constexpr int kQdAhead = 4;  // chunks of X in flight per warp
// Per-warp ring: kQdAhead + 1 slots of 4 x 32 lanes x 16 bytes; a slot is refilled one iteration
// after its contents were read, so the read has long completed.
constexpr uint32_t kQdSlotBytes = 4 * 32 * 16;
constexpr uint32_t kQdRingBytes = kQdWarps * (kQdAhead + 1) * kQdSlotBytes;
// Relative nudges that bracket a correctly rounded quotient (see quant_rows).
constexpr float kNudgeLo = 1.0f - 0x1p-20f;
constexpr float kNudgeHi = 1.0f + 0x1p-20f;

struct QdParams {
  const uint16_t* X;
  int ldx, M, K, KB, rank;
  const float* inv_lambda;
  const uint8_t* l1;
  uint8_t* codes;
  uint8_t* sf;
  uint8_t* t;
  int splits;               // K slices per 16-row block (layers of fewer blocks than SMs)
  float* part;              // [block][slice][16][rank] fp32 partials of T (splits > 1, rank > 0)
  unsigned long long* cnt;  // per 16-row block: (launch epoch << 8) | slices arrived
  unsigned long long epoch; // distinct per launch, never 0
};

// Counts this CTA's slice in the counter of its rows and returns whether it was the last of
// `splits`.  The counter holds (epoch << 8) | count; a value from another launch (or uninitialised
// memory) restarts the count, and the last CTA resets it to 0, so a replay of the same launch also
// starts from 0.  Lock-free (a failed CAS means another slice succeeded); bounded all the same.
__device__ __forceinline__ bool arrive_slice_counter(unsigned long long* cnt, unsigned long long epoch, int splits,
                                                     bool* ok) {
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(cnt);
  for (int it = 0; it < (1 << 20); ++it) {
    const unsigned long long nxt = (cur >> 8) == epoch ? cur + 1 : ((epoch << 8) | 1ull);
    const unsigned long long prev = atomicCAS(cnt, cur, nxt);
    if (prev == cur) return static_cast<int>(nxt & 0xFFull) == splits;
    cur = prev;
  }
  atomicOr(&g_device_error, kErrWaitQuantDown);
  *ok = false;
  return false;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Two fp32 lanes in one 64-bit register for the packed (f32x2) FP pipe of sm_100.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// Element-wise round-to-nearest product of two fp32 pairs.
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Element-wise round-to-nearest a - b and a * b + c of fp32 pairs.
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// E2M1 codes (RNE, saturating) of the 8 values held as 4 fp32 pairs; element 2i in the low nibble.
__device__ __forceinline__ uint32_t e2m1x8_pairs(const uint64_t (&v)[4]) {
  float a[8];
#pragma unroll
  for (int t = 0; t < 4; ++t) f2unpack(v[t], a[2 * t], a[2 * t + 1]);
  uint32_t c;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(c)
      : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7]));
  return c;
}

// E2M1 codes of x[j] * mul (each product rounded to nearest), element 2i in the low nibble of byte i.
__device__ __forceinline__ uint32_t e2m1x8_scaled(const uint64_t (&x)[4], float mul) {
  const uint64_t m = f2pack(mul, mul);
  uint64_t q[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) q[t] = f2mul(x[t], m);
  return e2m1x8_pairs(q);
}

// The exact codes E2M1_rne(RN(x / sd)) with IEEE divisions (rare path).
__device__ __forceinline__ uint32_t e2m1x8_div(const float (&v)[8], float sd) {
  uint32_t c = 0;
#pragma unroll
  for (int t = 0; t < 4; ++t) c |= cvt_e2m1x2(__fdiv_rn(v[2 * t], sd), __fdiv_rn(v[2 * t + 1], sd)) << (8 * t);
  return c;
}

__device__ __forceinline__ uint32_t int4x8(const float (&v)[8], float mul) {
  uint32_t c = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float q = fminf(7.0f, fmaxf(-8.0f, rintf(__fmul_rn(v[j], mul))));
    c |= (static_cast<uint32_t>(static_cast<int>(q)) & 0xFu) << (4 * j);
  }
  return c;
}

__device__ __forceinline__ uint32_t int4x8_div(const float (&v)[8], float s) {
  uint32_t c = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int q = max(-8, min(7, __float2int_rn(__fdiv_rn(v[j], s))));
    c |= (static_cast<uint32_t>(q) & 0xFu) << (4 * j);
  }
  return c;
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 16-byte asynchronous copy global -> shared (L2 only); zero-filled when src_bytes is 0.
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* gptr, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(gptr), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
  return v;
}

// fp32 (>= 0) -> E4M3 byte, round to nearest even, saturating at 448 (no ordering constraint).
__device__ __forceinline__ uint32_t cvt_e4m3_rn(float x) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(x));
  return static_cast<uint32_t>(out) & 0xFFu;
}

// Warp-level D += A B (m16n8k16, bf16 inputs, fp32 accumulation), free to be scheduled.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// x_hat = fp32(x) * (1/lambda) of 8 bf16 values (one rounding each), as 4 fp32 pairs.
__device__ __forceinline__ void smooth8(const uint4& w, const float4& i0, const float4& i1, uint64_t (&xp)[4]) {
  xp[0] = f2mul(f2pack(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u)), f2pack(i0.x, i0.y));
  xp[1] = f2mul(f2pack(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u)), f2pack(i0.z, i0.w));
  xp[2] = f2mul(f2pack(__uint_as_float(w.z << 16), __uint_as_float(w.z & 0xFFFF0000u)), f2pack(i1.x, i1.y));
  xp[3] = f2mul(f2pack(__uint_as_float(w.w << 16), __uint_as_float(w.w & 0xFFFF0000u)), f2pack(i1.z, i1.w));
}

__device__ __forceinline__ float absmax8(const uint64_t (&xp)[4]) {
  float v[8];
#pragma unroll
  for (int t = 0; t < 4; ++t) f2unpack(xp[t], v[2 * t], v[2 * t + 1]);
  return fmaxf(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))),
               fmaxf(fmaxf(fabsf(v[4]), fabsf(v[5])), fmaxf(fabsf(v[6]), fabsf(v[7]))));
}

template <int PREC, int NTM>
__global__ void __launch_bounds__(kQdThreads, 2) quant_down_kernel(const QdParams p) {
  // Dynamic shared memory: the warps' rings of X, later (after every chunk) reused for
  // [kQdWarps][16][rank] fp32: each warp's share of T.
  extern __shared__ __align__(16) float shares[];
  __shared__ float rcp_tbl[128];     // NVFP4: 1 / value of each UE4M3 code (0 for code 0)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, j = lane & 3;
  const int r = p.rank, nt = r >> 3;
  if (PREC == 0 && threadIdx.x < 128) rcp_tbl[threadIdx.x] = threadIdx.x == 0 ? 0.0f : __frcp_rn(e4m3_to_f32(threadIdx.x));
  __syncthreads();
  // Kernel 2 may be scheduled now (it waits for this grid's completion before reading anything).
  pdl_launch_dependents();

  const int blk = blockIdx.x / p.splits, split = blockIdx.x % p.splits;
  const int m0 = blk * kQdRows;
  int row[2], rin[2];
  bool live[2];
  const uint16_t* xrow[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    row[i] = m0 + g + 8 * i;
    rin[i] = row[i] & (kBM - 1);
    live[i] = row[i] < p.M;  // rows past M (up to the workspace's padded end) quantize zeros
    xrow[i] = p.X + static_cast<size_t>(live[i] ? row[i] : 0) * p.ldx + 8 * j;
  }
  const int mt = m0 / kBM;
  const int nch = p.K >> 6;
  const int c0 = split * nch / p.splits, c1 = (split + 1) * nch / p.splits;  // this CTA's chunks of K
  uint8_t* const codes_t = p.codes + codes_chunk_offset(mt, 0, p.KB, kBM);
  uint8_t* const sf_t = p.sf + sf_chunk_offset(mt, 0, p.KB, kBM);
  const float kInv6 = __frcp_rn(6.0f);

  float d[NTM > 0 ? NTM : 1][4];
#pragma unroll
  for (int ni = 0; ni < (NTM > 0 ? NTM : 1); ++ni) d[ni][0] = d[ni][1] = d[ni][2] = d[ni][3] = 0.0f;

  const uint32_t ring = smem_u32(shares) + static_cast<uint32_t>(warp) * (kQdAhead + 1) * kQdSlotBytes +
                        static_cast<uint32_t>(lane) * 16u;
  // Chunk c into ring slot `slot` (one commit group per call, empty past the end, so that the
  // group count stays in step with the chunks).
  auto issue = [&](int c, int slot) {
    if (c < c1) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          cp_async16(ring + static_cast<uint32_t>(slot) * kQdSlotBytes + (2 * i + h) * 512u, xrow[i] + 64 * c + 32 * h,
                     live[i] ? 16u : 0u);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int q = 0; q < kQdAhead; ++q) issue(c0 + warp + q * kQdWarps, q);
  int slot = 0;
  for (int c = c0 + warp; c < c1; c += kQdWarps) {
    cp_async_wait<kQdAhead - 1>();  // this chunk's copies have landed
    uint4 cur[2][2];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) cur[i][h] = lds_v4(ring + static_cast<uint32_t>(slot) * kQdSlotBytes + (2 * i + h) * 512u);
    // the slot read in the previous iteration takes the chunk kQdAhead ahead
    issue(c + kQdAhead * kQdWarps, slot == 0 ? kQdAhead : slot - 1);
    slot = slot == kQdAhead ? 0 : slot + 1;
    const int k0 = c << 6;
    const int kb = k0 >> 8, kin = k0 & 255;
    uint64_t xp[2][2][4];  // x_hat of [row][half] as fp32 pairs
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float4 i0 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + k0 + 32 * h + 8 * j));
      const float4 i1 = __ldg(reinterpret_cast<const float4*>(p.inv_lambda + k0 + 32 * h + 8 * j + 4));
#pragma unroll
      for (int i = 0; i < 2; ++i) smooth8(cur[i][h], i0, i1, xp[i][h]);
    }
    uint8_t* const codes_kb = codes_t + static_cast<size_t>(kb) * (kBM * kRowBytes);
    uint8_t* const sf_kb = sf_t + static_cast<size_t>(kb) * (kBM * kSfBytesPerRowKb);
    if (PREC == 0) {
      // NVFP4: the 16-element group of half h held by lanes j and j ^ 1
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float amax = absmax8(xp[i][h]);
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
          // scale code UE4M3_rne(RN(amax / 6)) and codes E2M1_rne(RN(x / s)), each bracketed
          // between two products whose codes agree exactly when the quotient is not within ~2^-20
          // of a rounding threshold; otherwise the IEEE divisions decide
          const float s_est = __fmul_rn(amax, kInv6);
          uint32_t sbits = cvt_e4m3_rn(__fmul_rn(s_est, kNudgeLo));
          bool slow = sbits != cvt_e4m3_rn(__fmul_rn(s_est, kNudgeHi));
          uint32_t code = 0u;
          if (!slow && sbits != 0u) {
            const float rr = rcp_tbl[sbits];
            code = e2m1x8_scaled(xp[i][h], __fmul_rn(rr, kNudgeLo));
            slow = code != e2m1x8_scaled(xp[i][h], __fmul_rn(rr, kNudgeHi));
          }
          if (slow) {
            float v[8];
#pragma unroll
            for (int t = 0; t < 4; ++t) f2unpack(xp[i][h][t], v[2 * t], v[2 * t + 1]);
            sbits = cvt_e4m3_rn(__fdiv_rn(amax, 6.0f));
            const float sd = e4m3_to_f32(sbits);
            code = sd != 0.0f ? e2m1x8_div(v, sd) : 0u;
          }
          *reinterpret_cast<uint32_t*>(codes_kb + swz128(rin[i], (kin + 32 * h + 8 * j) >> 1)) = code;
          if ((j & 1) == 0) sf_kb[sf_nvfp4_offset(rin[i], ((kin + 32 * h) >> 4) + (j >> 1), kBM)] = static_cast<uint8_t>(sbits);
        }
    } else {
      // INT4: the 64-element group is the chunk row, spread over the four lanes j
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float amax = fmaxf(absmax8(xp[i][0]), absmax8(xp[i][1]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const float sc = __fdiv_rn(amax, 7.0f);
        float v[2][8];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int t = 0; t < 4; ++t) f2unpack(xp[i][h][t], v[h][2 * t], v[h][2 * t + 1]);
        uint32_t code[2] = {0u, 0u};
        bool slow = false;
        if (sc != 0.0f) {
          const float rr = __frcp_rn(sc);
          if (rr < 1e30f) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              code[h] = int4x8(v[h], __fmul_rn(rr, kNudgeLo));
              slow |= code[h] != int4x8(v[h], __fmul_rn(rr, kNudgeHi));
            }
          } else {
            slow = true;  // tiny scale: its reciprocal is out of range
          }
        }
        if (slow) {
#pragma unroll
          for (int h = 0; h < 2; ++h) code[h] = int4x8_div(v[h], sc);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h)
          *reinterpret_cast<uint32_t*>(codes_kb + swz128(rin[i], (kin + 32 * h + 8 * j) >> 1)) = code[h];
        if (j == 0) reinterpret_cast<float*>(sf_kb)[sf_int4_a_index(rin[i], kin >> 6)] = sc;
      }
    }
    if (NTM > 0) {
      __syncwarp();  // the slow paths above are divergent; the MMAs are warp-collective
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a[2][4];
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          float v0[4], v1[4];
          f2unpack(xp[0][h][2 * s], v0[0], v0[1]);
          f2unpack(xp[0][h][2 * s + 1], v0[2], v0[3]);
          f2unpack(xp[1][h][2 * s], v1[0], v1[1]);
          f2unpack(xp[1][h][2 * s + 1], v1[2], v1[3]);
          a[s][0] = pack_bf16x2(v0[0], v0[1]);  // row g, logical k 2j, 2j + 1
          a[s][1] = pack_bf16x2(v1[0], v1[1]);  // row g + 8
          a[s][2] = pack_bf16x2(v0[2], v0[3]);  // row g, logical k 2j + 8, 2j + 9
          a[s][3] = pack_bf16x2(v1[2], v1[3]);  // row g + 8
        }
#pragma unroll
        for (int ni = 0; ni < NTM; ++ni)
          if (ni < nt) {
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(
                p.l1 + l1_offset(static_cast<uint32_t>(k0 + 32 * h + 8 * j), static_cast<uint32_t>(8 * ni + g), r)));
            mma_16816(d[ni], a[0], b.x, b.y);
            mma_16816(d[ni], a[1], b.z, b.w);
          }
      }
    }
  }
  cp_async_wait<0>();

  if (NTM > 0) {
    // Each warp's share of T, then the sum over warps in warp order, rounded to bf16 once.
    __syncthreads();  // every warp is done with its ring, which the shares overwrite
#pragma unroll
    for (int ni = 0; ni < NTM; ++ni)
      if (ni < nt) {
        float* s0 = shares + (warp * kQdRows + g) * r + 8 * ni + 2 * j;
        *reinterpret_cast<float2*>(s0) = make_float2(d[ni][0], d[ni][1]);
        *reinterpret_cast<float2*>(s0 + 8 * r) = make_float2(d[ni][2], d[ni][3]);
      }
    __syncthreads();
    uint8_t* const tt = p.t + static_cast<size_t>(mt) * kBM * r * 2;
    float* const pb = p.part + static_cast<size_t>(blk) * p.splits * kQdRows * r;  // this block's partials
    for (int e = threadIdx.x; e < kQdRows * r / 2; e += kQdThreads) {
      const int rw = (2 * e) / r, col = (2 * e) % r;
      float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
      for (int w = 0; w < kQdWarps; ++w) {
        const float2 v = *reinterpret_cast<const float2*>(shares + (w * kQdRows + rw) * r + col);
        a0 += v.x;
        a1 += v.y;
      }
      if (p.splits == 1)
        *reinterpret_cast<uint32_t*>(tt + lr_offset(static_cast<uint32_t>((m0 + rw) & (kBM - 1)), col, kBM, r)) =
            pack_bf16x2(a0, a1);
      else
        *reinterpret_cast<float2*>(pb + (static_cast<size_t>(split) * kQdRows + rw) * r + col) = make_float2(a0, a1);
    }
    if (p.splits > 1) {
      // The last slice of the block to finish adds all slices' partials in slice order
      // (deterministic) and writes bf16 T.  Publication: the CTA barrier orders every thread's
      // partial stores before thread 0's GPU-scope fence, which is cumulative, and that fence
      // before the counter update; the last slice fences again before reading.
      __shared__ int s_last;
      __syncthreads();
      if (threadIdx.x == 0) {
        bool ok = true;
        __threadfence();
        const bool last = arrive_slice_counter(p.cnt + blk, p.epoch, p.splits, &ok);
        if (last) __threadfence();
        if (!ok) atomicExch(p.cnt + blk, 0ull);  // a replay of this launch starts the count afresh
        s_last = last ? 1 : 0;
      }
      __syncthreads();
      if (s_last) {
        for (int e = threadIdx.x; e < kQdRows * r / 2; e += kQdThreads) {
          const int rw = (2 * e) / r, col = (2 * e) % r;
          float2 a = __ldcg(reinterpret_cast<const float2*>(pb + static_cast<size_t>(rw) * r + col));
          for (int q = 1; q < p.splits; ++q) {
            const float2 v = __ldcg(reinterpret_cast<const float2*>(pb + (static_cast<size_t>(q) * kQdRows + rw) * r + col));
            a.x += v.x;
            a.y += v.y;
          }
          *reinterpret_cast<uint32_t*>(tt + lr_offset(static_cast<uint32_t>((m0 + rw) & (kBM - 1)), col, kBM, r)) =
              pack_bf16x2(a.x, a.y);
        }
        if (threadIdx.x == 0) atomicExch(p.cnt + blk, 0ull);
      }
    }
  }
}


// ---------------------------------------------------------------------------- kernel 1, large layers
//
// The same three steps on 128-row tiles, for layers whose rows exceed one wave of the warp-level
// kernel or whose rank exceeds 32 (there its 16-row blocks re-read L1 r/16 times the bytes of X
// from L2).  One CTA per (128-row tile, K slice): a TMA warp streams X (and the stage's 1/lambda
// and L1 chunk) into a ring of shared-memory stages; sixteen worker warps apply the smoothing
// factor and quantize (NVFP4: one 16-element group per thread; INT4: 8 lanes share a 64-element
// group) with the same exact bracketed rounding, and write bf16(x_hat) back into the stage; one
// warp feeds it with L1 to tcgen05 bf16 MMAs that accumulate T in tensor memory.  When K is split
// over several CTAs, each writes its fp32 partial of T and counts itself in the tile's counter;
// the last to arrive adds the partials in slice order (deterministic) and writes bf16 T once.

constexpr int kQtMaxStages = 8;
constexpr int kQtWorkerWarps = 16;
constexpr int kQtMmaWarp = kQtWorkerWarps;        // tcgen05 MMA issuer (+ TMEM owner)
constexpr int kQtTmaWarp = kQtWorkerWarps + 1;    // TMA producer
constexpr int kQtThreads = (kQtWorkerWarps + 2) * 32;
constexpr uint32_t kQtXsBytes = kBM * 128;  // one stage of X: 128 rows x 64 bf16, 128-byte swizzle
constexpr uint32_t kQtIlBytes = 64 * 4;     // the stage's 64 values of 1/lambda
constexpr size_t kQtSmemBudget = 220 * 1024;

struct QtParams {
  int M, K, rank, KB, splits, stages;
  const float* inv_lambda;
  const uint8_t* l1;
  uint8_t* codes;
  uint8_t* sf;
  uint8_t* t;
  float* part;              // [m-tile][split][128][rank] fp32 partials of T (splits > 1)
  unsigned long long* cnt;  // per m-tile: (launch epoch << 8) | slices arrived
  unsigned long long epoch; // distinct per launch, never 0
};


template <int PREC>
__global__ void __launch_bounds__(kQtThreads, 1)
    quant_down_tile_kernel(const __grid_constant__ CUtensorMap tmap_x, const QtParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ float rcp_tbl[128];  // RN(1 / UE4M3 value) for every finite scale code
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int r = p.rank;
  const int NS = p.stages;
  const bool has_lr = r > 0;
  const uint32_t l1_bytes = static_cast<uint32_t>(r) * 128u;
  const uint32_t l1_stride = static_cast<uint32_t>(align_up(l1_bytes, 1024));
  uint8_t* xs = smem;                       // NS x 16 KB (X, then bf16 x_hat in place)
  uint8_t* l1s = smem + NS * kQtXsBytes;      // NS x r*128 (L1 chunk)
  const float* ils = reinterpret_cast<const float*>(l1s + NS * l1_stride);  // NS x 64 fp32 (1/lambda chunk)
  uint64_t* bars = reinterpret_cast<uint64_t*>(l1s + NS * l1_stride + NS * kQtIlBytes);
  uint64_t* full = bars;                    // TMA landed: X tile (+ L1 chunk)
  uint64_t* xready = bars + NS;             // workers wrote x_hat (one arrive per worker warp)
  uint64_t* empty = bars + 2 * NS;          // stage free again
  uint64_t* done = bars + 3 * NS;           // all MMAs of this CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;
  const int kb0 = split * p.KB / p.splits, kb1 = (split + 1) * p.KB / p.splits;
  const int c0 = kb0 * 4, nch = (kb1 - kb0) * 4;
  const uint32_t tmem_cols = r <= 32 ? 32u : (r <= 64 ? 64u : 128u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&xready[s], kQtWorkerWarps);
      mbar_init(&empty[s], has_lr ? 1 : kQtWorkerWarps);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (PREC == 0 && threadIdx.x < 128) rcp_tbl[threadIdx.x] = threadIdx.x == 0 ? 0.0f : __frcp_rn(e4m3_to_f32(threadIdx.x));
  if (has_lr && warp == kQtMmaWarp) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = has_lr ? *tmem_slot : 0u;
  // Kernel 2 may be scheduled once every block of this grid has got here (it waits for this
  // grid's completion before reading anything this kernel writes).
  pdl_launch_dependents();

  if (warp < kQtWorkerWarps) {
    // ------------------------------------------------------------ workers
    // Quantization is exact (codes = E2M1_rne(RN(x / s)), resp. rint(RN(x / s)) for INT4): the
    // quotient is bracketed between x * RN(RN(1/s)(1 -+ 2^-20)); both roundings are monotonic, so
    // when the two bracketing codes agree they are the exact codes, and otherwise (x/s within
    // ~2^-20 of a threshold) the IEEE division decides.
    if (PREC == 0) {
      // NVFP4: thread t of the 512 handles one 16-element group per 64-column chunk: row t / 4,
      // group t % 4 (two swizzled 16-byte units; the quarter-warps' loads hit distinct banks).
      const int row = warp * 8 + (lane >> 2), g = lane & 3;
      const float kInv6 = __frcp_rn(6.0f);
      // Per-thread constants: the two swizzled 16-byte units of the group inside a stage, and
      // this row's code/scale positions inside a (tile, k-block) chunk.
      const uint32_t off0 = swz128(row, g * 32), off1 = swz128(row, g * 32 + 16);
      uint8_t* const codes_tile = p.codes + codes_chunk_offset(mt, 0, p.KB, kBM);
      uint8_t* const sf_tile = p.sf + sf_chunk_offset(mt, 0, p.KB, kBM) + (row & 31) * 16 + (row >> 5) * 4 + g;
      int st = 0;
      uint32_t ph = 0;
      for (int c = 0; c < nch; ++c) {
        const bool ok = !*abort_flag && wait_parity_bounded(&full[st], ph, kErrWaitQuantDown);
        if (!__all_sync(0xffffffffu, ok)) {
          *abort_flag = 1;
          break;
        }
        const int gc = c0 + c;
        const int kb = gc >> 2, cc = gc & 3;
        const float4* ilv = reinterpret_cast<const float4*>(ils + st * 64 + g * 16);
        uint8_t* xt = xs + st * kQtXsBytes;
        uint4* cell0 = reinterpret_cast<uint4*>(xt + off0);
        uint4* cell1 = reinterpret_cast<uint4*>(xt + off1);
        const uint4 xa = *cell0, xb = *cell1;
        const uint32_t w[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
        uint64_t xp[2][4];  // x_hat as fp32 pairs: element 2t, 2t + 1 of half h in xp[h][t]
        float pm[8];        // per-pair maxima of |x_hat|, reduced as a tree (max is exact)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float4 i0 = ilv[2 * h], i1 = ilv[2 * h + 1];
          const float il[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            // bf16 -> fp32 is exact; x_hat = fp32(x) * (1/lambda), one rounding per element
            const uint32_t ww = w[4 * h + t];
            xp[h][t] = f2mul(f2pack(__uint_as_float(ww << 16), __uint_as_float(ww & 0xFFFF0000u)),
                             f2pack(il[2 * t], il[2 * t + 1]));
            float lo, hi;
            f2unpack(xp[h][t], lo, hi);
            pm[4 * h + t] = fmaxf(fabsf(lo), fabsf(hi));
          }
        }
        const float amax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                 fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        // scale code: UE4M3_rne(RN(amax / 6)), bracketed the same way
        const float s_est = __fmul_rn(amax, kInv6);
        uint32_t sbits = cvt_e4m3(__fmul_rn(s_est, kNudgeLo));
        const uint32_t sc_hi = cvt_e4m3(__fmul_rn(s_est, kNudgeHi));
        uint2 code = make_uint2(0u, 0u);
        bool slow = sbits != sc_hi;
        if (!slow && sbits != 0) {
          const float rr = rcp_tbl[sbits];
          const float mlo = __fmul_rn(rr, kNudgeLo), mhi = __fmul_rn(rr, kNudgeHi);
          code.x = e2m1x8_scaled(xp[0], mlo);
          code.y = e2m1x8_scaled(xp[1], mlo);
          slow = (code.x != e2m1x8_scaled(xp[0], mhi)) | (code.y != e2m1x8_scaled(xp[1], mhi));
        }
        if (slow) {  // rare: the exact quotients decide
          float xh[2][8];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int t = 0; t < 4; ++t) f2unpack(xp[h][t], xh[h][2 * t], xh[h][2 * t + 1]);
          sbits = cvt_e4m3(__fdiv_rn(amax, 6.0f));
          const float sd = e4m3_to_f32(sbits);
          code.x = sd != 0.0f ? e2m1x8_div(xh[0], sd) : 0u;
          code.y = sd != 0.0f ? e2m1x8_div(xh[1], sd) : 0u;
        }
        *reinterpret_cast<uint2*>(codes_tile + static_cast<size_t>(kb) * (kBM * kRowBytes) + swz128(row, cc * 32 + g * 8)) = code;
        sf_tile[static_cast<size_t>(kb) * (kBM * kSfBytesPerRowKb) + cc * 512] = static_cast<uint8_t>(sbits);
        if (has_lr) {
          uint32_t hv[8];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              float lo, hi;
              f2unpack(xp[h][t], lo, hi);
              hv[4 * h + t] = pack_bf16x2(lo, hi);
            }
          *cell0 = make_uint4(hv[0], hv[1], hv[2], hv[3]);  // bf16(x_hat) in place: the MMA's A operand
          *cell1 = make_uint4(hv[4], hv[5], hv[6], hv[7]);
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(has_lr ? &xready[st] : &empty[st]);
        if (++st == NS) {
          st = 0;
          ph ^= 1u;
        }
      }
    } else {
      // INT4: lane (sub, kg) of warp w handles 8 consecutive columns (16-byte unit kg) of rows
      // 8w + sub and 8w + 4 + sub; the 64-element group spans the 8 lanes of a row.
      const int sub = lane >> 3, kg = lane & 7;
      for (int c = 0; c < nch; ++c) {
        const int st = c % NS;
        const bool ok = !*abort_flag && wait_parity_bounded(&full[st], (c / NS) & 1, kErrWaitQuantDown);
        if (!__all_sync(0xffffffffu, ok)) {
          *abort_flag = 1;
          break;
        }
        const int gc = c0 + c;
        const float4 il0 = *reinterpret_cast<const float4*>(ils + st * 64 + kg * 8);
        const float4 il1 = *reinterpret_cast<const float4*>(ils + st * 64 + kg * 8 + 4);
        const float il[8] = {il0.x, il0.y, il0.z, il0.w, il1.x, il1.y, il1.z, il1.w};
        const int kb = gc >> 2, cc = gc & 3;
        uint8_t* codes_chunk = p.codes + codes_chunk_offset(mt, kb, p.KB, kBM);
        uint8_t* sf_chunk = p.sf + sf_chunk_offset(mt, kb, p.KB, kBM);
        uint8_t* xt = xs + st * kQtXsBytes;
        int row[2];
        uint4* cell[2];
        float xh[2][8];
        float amax[2];
        uint64_t ilp[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) ilp[t] = f2pack(il[2 * t], il[2 * t + 1]);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          row[i] = warp * 8 + i * 4 + sub;
          cell[i] = reinterpret_cast<uint4*>(xt + swz128(row[i], kg * 16));
          const uint4 xv = *cell[i];
          const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const uint64_t xp = f2mul(f2pack(__uint_as_float(w[t] << 16), __uint_as_float(w[t] & 0xFFFF0000u)), ilp[t]);
            f2unpack(xp, xh[i][2 * t], xh[i][2 * t + 1]);
          }
          amax[i] = fmaxf(fmaxf(fmaxf(fabsf(xh[i][0]), fabsf(xh[i][1])), fmaxf(fabsf(xh[i][2]), fabsf(xh[i][3]))),
                          fmaxf(fmaxf(fabsf(xh[i][4]), fabsf(xh[i][5])), fmaxf(fabsf(xh[i][6]), fabsf(xh[i][7]))));
          amax[i] = fmaxf(amax[i], __shfl_xor_sync(0xffffffffu, amax[i], 1));
          amax[i] = fmaxf(amax[i], __shfl_xor_sync(0xffffffffu, amax[i], 2));
          amax[i] = fmaxf(amax[i], __shfl_xor_sync(0xffffffffu, amax[i], 4));
        }
        uint32_t codes[2], sbits[2];
        bool slow = false;
        float sc[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          sc[i] = __fdiv_rn(amax[i], 7.0f);
          sbits[i] = __float_as_uint(sc[i]);
          codes[i] = 0;
          if (sc[i] != 0.0f) {
            const float rr = __frcp_rn(sc[i]);
            if (rr < 1e30f) {
              const uint32_t lo = int4x8(xh[i], __fmul_rn(rr, kNudgeLo));
              const uint32_t hi = int4x8(xh[i], __fmul_rn(rr, kNudgeHi));
              codes[i] = lo;
              slow |= lo != hi;
            } else {
              slow = true;  // tiny scale: reciprocal out of range
            }
          }
        }
        if (slow) {
#pragma unroll
          for (int i = 0; i < 2; ++i) codes[i] = sc[i] != 0.0f ? int4x8_div(xh[i], sc[i]) : 0u;
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          *reinterpret_cast<uint32_t*>(codes_chunk + swz128(row[i], cc * 32 + kg * 4)) = codes[i];
          if (kg == 0) reinterpret_cast<uint32_t*>(sf_chunk)[sf_int4_a_index(row[i], cc)] = sbits[i];
          if (has_lr) {
            uint4 hv;
            hv.x = pack_bf16x2(xh[i][0], xh[i][1]);
            hv.y = pack_bf16x2(xh[i][2], xh[i][3]);
            hv.z = pack_bf16x2(xh[i][4], xh[i][5]);
            hv.w = pack_bf16x2(xh[i][6], xh[i][7]);
            *cell[i] = hv;  // bf16(x_hat) in place: the tile becomes the MMA's A operand
          }
        }
        if (has_lr) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(has_lr ? &xready[st] : &empty[st]);
      }
    }
  } else if (warp == kQtTmaWarp) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int issued = 0;
      for (int c = 0; c < nch; ++c) {
        const int st = c % NS;
        if (c >= NS && (*abort_flag || !wait_parity_bounded(&empty[st], ((c / NS) - 1) & 1, kErrWaitQuantDown))) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[st], kQtXsBytes + kQtIlBytes + (has_lr ? l1_bytes : 0u));
        tma_load_2d(xs + st * kQtXsBytes, &tmap_x, (c0 + c) * 64, mt * kBM, &full[st]);
        bulk_g2s(const_cast<float*>(ils) + st * 64, p.inv_lambda + static_cast<size_t>(c0 + c) * 64, kQtIlBytes, &full[st]);
        if (has_lr)
          bulk_g2s(l1s + st * l1_stride, p.l1 + static_cast<size_t>(c0 + c) * l1_bytes, l1_bytes, &full[st]);
        ++issued;
      }
      if (*abort_flag) {
        // Let every issued copy land before the CTA can retire.
        for (int q = (issued > NS ? issued - NS : 0); q < issued; ++q)
          wait_parity_bounded(&full[q % NS], (q / NS) & 1, kErrWaitQuantDown);
      }
    }
  } else if (has_lr && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16(128, r);
    for (int c = 0; c < nch; ++c) {
      const int st = c % NS;
      const uint32_t par = (c / NS) & 1;
      if (*abort_flag || !wait_parity_bounded(&full[st], par, kErrWaitQuantDown) ||
          !wait_parity_bounded(&xready[st], par, kErrWaitQuantDown)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint64_t ad = smem_desc(smem_u32(xs + st * kQtXsBytes), 16, 1024, kLayoutSw128);
      const uint64_t bd = smem_desc(smem_u32(l1s + st * l1_stride), 16, 1024, kLayoutSw128);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) mma_bf16(tmem_base, ad + 2 * ks, bd + 2 * ks, idesc, (c | ks) != 0 ? 1u : 0u);
      tc_commit(&empty[st]);
    }
    tc_commit(done);
  }

  // ---------------------------------------------------------------- T epilogue
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  if (has_lr && warp < 4) {
    bool ok = !aborted && wait_parity_bounded(done, 0, kErrWaitQuantDown);
    ok = __all_sync(0xffffffffu, ok);  // the TMEM loads below are warp-collective
    tc_fence_after();
    if (ok) {
      const int row = warp * 32 + lane;
      float* prow = p.splits > 1 ? p.part + ((static_cast<size_t>(mt) * p.splits + split) * kBM + row) * r : nullptr;
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
            *reinterpret_cast<float4*>(prow + j + q) = make_float4(__uint_as_float(v[q]), __uint_as_float(v[q + 1]),
                                                                   __uint_as_float(v[q + 2]), __uint_as_float(v[q + 3]));
        }
      }
    }
  }
  if (has_lr && p.splits > 1) {
    // The last slice of the tile to finish sums all slices' partials in slice order
    // (deterministic) and writes bf16 T.  Publication: the CTA barrier orders every thread's
    // partial stores before thread 0's GPU-scope fence, which is cumulative, and that fence
    // before the counter update; the last slice fences again before reading.
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
      bool ok = !aborted;
      __threadfence();
      const bool last = ok && arrive_slice_counter(p.cnt + mt, p.epoch, p.splits, &ok);
      if (last) __threadfence();
      if (!ok) {
        // A slice that gave up resets the tile's count, so that a replay of this launch (a CUDA
        // graph keeps its launch tag) does not resume a count this launch left incomplete.
        *abort_flag = 1;
        atomicExch(p.cnt + mt, 0ull);
      }
      s_last = last ? 1 : 0;
    }
    __syncthreads();
    if (s_last) {
      uint8_t* tt = p.t + static_cast<size_t>(mt) * kBM * r * 2;
      const float* pt = p.part + static_cast<size_t>(mt) * p.splits * kBM * r;
      const size_t slice = static_cast<size_t>(kBM) * r;
      const int units = kBM * r / 4;
      // Two 4-column units per thread per round, all of a round's loads issued before the sums.
      for (int u0 = threadIdx.x; u0 < units; u0 += 2 * blockDim.x) {
        const int u1 = u0 + blockDim.x;
        const bool has1 = u1 < units;
        const int o0 = u0 * 4, o1 = (has1 ? u1 : u0) * 4;
        float4 a0 = __ldcg(reinterpret_cast<const float4*>(pt + o0));
        float4 a1 = __ldcg(reinterpret_cast<const float4*>(pt + o1));
        float4 x0[7], x1[7];
#pragma unroll
        for (int q = 1; q < 8; ++q)
          if (q < p.splits) {
            x0[q - 1] = __ldcg(reinterpret_cast<const float4*>(pt + q * slice + o0));
            x1[q - 1] = __ldcg(reinterpret_cast<const float4*>(pt + q * slice + o1));
          }
#pragma unroll
        for (int q = 1; q < 8; ++q)
          if (q < p.splits) {
            a0.x += x0[q - 1].x; a0.y += x0[q - 1].y; a0.z += x0[q - 1].z; a0.w += x0[q - 1].w;
            a1.x += x1[q - 1].x; a1.y += x1[q - 1].y; a1.z += x1[q - 1].z; a1.w += x1[q - 1].w;
          }
        *reinterpret_cast<uint2*>(tt + lr_offset(o0 / r, o0 % r, kBM, r)) =
            make_uint2(pack_bf16x2(a0.x, a0.y), pack_bf16x2(a0.z, a0.w));
        if (has1)
          *reinterpret_cast<uint2*>(tt + lr_offset(o1 / r, o1 % r, kBM, r)) =
              make_uint2(pack_bf16x2(a1.x, a1.y), pack_bf16x2(a1.z, a1.w));
      }
      if (threadIdx.x == 0) atomicExch(p.cnt + mt, 0ull);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (has_lr && warp == kQtMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

static int quant_down_tile_stages(int r) {
  const size_t per = kQtXsBytes + align_up(static_cast<size_t>(r) * 128, 1024) + kQtIlBytes;
  const int ns = static_cast<int>((kQtSmemBudget - 2048) / per);
  return ns < kQtMaxStages ? ns : kQtMaxStages;
}

static size_t quant_down_tile_smem_bytes(int r) {
  const int ns = quant_down_tile_stages(r);
  return 1024 + ns * (kQtXsBytes + align_up(static_cast<size_t>(r) * 128, 1024) + kQtIlBytes) + 256;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link dependency).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// A tag that differs between launches (56 bits, never 0) for the K-split arrival counters.
static unsigned long long next_launch_epoch() {
  static std::atomic<unsigned long long> counter{0};
  const unsigned long long e = (counter.fetch_add(1) + 1) & ((1ull << 56) - 1);
  return e == 0 ? 1 : e;
}

static cudaError_t launch_quant_down_tile(const QuantDownArgs& a, int num_sms, cudaStream_t stream) {
  QtParams p;
  p.M = a.M;
  p.K = a.K;
  p.rank = a.rank;
  p.KB = a.K / kBK;
  p.stages = quant_down_tile_stages(a.rank);
  p.inv_lambda = a.inv_lambda;
  p.l1 = a.l1;
  p.codes = a.codes;
  p.sf = a.sf;
  p.t = a.t;
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.ldx) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kBM)};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.X), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int mt = 2 * ((a.M + 2 * kBM - 1) / (2 * kBM));  // pairs of 128-row tiles (kernel 2 works on 256 rows)
  const size_t smem = quant_down_tile_smem_bytes(a.rank);
  void (*kern)(const CUtensorMap, const QtParams) = a.precision == 0 ? quant_down_tile_kernel<0> : quant_down_tile_kernel<1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // One CTA per SM (shared memory), one wave: as many K slices per tile as the SMs allow, within
  // what the workspace's partials have room for.
  int splits = num_sms / mt;
  if (splits > a.split_cap) splits = a.split_cap;
  if (splits < 1) splits = 1;
  if (a.rank > 0 && splits > 1 && (!a.part || !a.cnt)) splits = 1;
  p.splits = splits;
  p.part = a.part;
  p.cnt = a.cnt;
  p.epoch = next_launch_epoch();
  if (a.precision == 0)
    quant_down_tile_kernel<0><<<mt * splits, kQtThreads, smem, stream>>>(tmap, p);
  else
    quant_down_tile_kernel<1><<<mt * splits, kQtThreads, smem, stream>>>(tmap, p);
  return cudaGetLastError();
}


static cudaError_t launch_quant_down_warps(const QuantDownArgs& a, int num_sms, cudaStream_t stream) {
  QdParams p;
  p.X = a.X;
  p.ldx = a.ldx;
  p.M = a.M;
  p.K = a.K;
  p.KB = a.K / kBK;
  p.rank = a.rank;
  p.inv_lambda = a.inv_lambda;
  p.l1 = a.l1;
  p.codes = a.codes;
  p.sf = a.sf;
  p.t = a.t;
  // Every row of the workspace's padded tiles (kernel 2 consumes rows in pairs of 128-row tiles).
  const int mpad = 2 * kBM * ((a.M + 2 * kBM - 1) / (2 * kBM));
  const int blocks = mpad / kQdRows;
  // Layers of fewer 16-row blocks than two per SM split K over up to 8 CTAs per block (each warp
  // keeping at least one chunk), within what the workspace's partials of T have room for.
  int splits = (2 * num_sms) / blocks;
  const int by_chunks = (a.K / 64) / kQdWarps;
  if (splits > by_chunks) splits = by_chunks;
  if (splits > 8) splits = 8;
  if (a.rank > 0 && splits > a.split_cap) splits = a.split_cap;
  if (a.rank > 0 && (!a.part || !a.cnt)) splits = 1;
  if (splits < 1) splits = 1;
  p.splits = splits;
  p.part = a.part;
  p.cnt = a.cnt;
  p.epoch = next_launch_epoch();
  const unsigned grid = static_cast<unsigned>(blocks * splits);
  const size_t shares = static_cast<size_t>(kQdWarps) * kQdRows * a.rank * sizeof(float);
  const size_t smem = shares > kQdRingBytes ? shares : kQdRingBytes;
  // rank 0 or at most 32 (the caller dispatches larger ranks to the 128-row tiles)
  void (*kern)(const QdParams) = a.precision == 0 ? (a.rank == 0 ? quant_down_kernel<0, 0> : quant_down_kernel<0, 4>)
                                                  : (a.rank == 0 ? quant_down_kernel<1, 0> : quant_down_kernel<1, 4>);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  kern<<<grid, kQdThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

// The warp-level kernel when its 16-row blocks fit in one wave (two per SM), the rank is at most 32
// and K at most 4096 (the FLUX QKV and MLP-up layers: X streamed with the most parallelism); the
// 128-row tiles otherwise.  Past K = 4096 the tiles win even at rank 0 (FLUX MLP-down, K = 12288:
// 40 us against 50 us at rank 0, 54 us against 66 us at rank 32), since each warp-level CTA
// walks all of K for its 16 rows and, with rank > 0, reads all of L1 from L2.
cudaError_t launch_quant_down(const QuantDownArgs& a, int num_sms, cudaStream_t stream) {
  const int mpad = 2 * kBM * ((a.M + 2 * kBM - 1) / (2 * kBM));
  if (a.rank <= 32 && mpad / kQdRows <= 2 * num_sms && a.K <= 4096) return launch_quant_down_warps(a, num_sms, stream);
  return launch_quant_down_tile(a, num_sms, stream);
}



// A byte buffer seen as a 2-D tensor of 256-byte rows, copied in boxes of `box_rows` rows (the
// operands are stored as shared-memory images, so a box is a contiguous chunk of the buffer).
static cudaError_t make_rows_map(CUtensorMap* map, const void* base, uint64_t bytes, uint32_t box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {256, bytes / 256};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {256, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  return cudaSuccess;
}

// ============================================================================ kernel 2
//
// A cluster of two CTAs computes 256 x 256 output tiles with cta_group::2 MMAs: each CTA holds its
// own 128 rows of A and half (128 rows) of B in shared memory, the scale factors its half of the
// accumulator needs (its SFA, all 256 rows of SFB) in TMEM, and accumulates its 128 rows x 256
// columns in TMEM.  The leader CTA alone issues the MMAs.
//
// Every per-stage chain is kept short because each runs on one thread (or warp) whose
// synchronisation and issue instructions have long latencies:
//   producers (2 threads per CTA): wait empty[s]; one copies the A and B tiles of this CTA by
//     TMA onto its full[s] (arming it with the stage's bytes), the other the two scale tiles;
//   scale warps (4 per CTA, one per TMEM lane quadrant): wait full[s], copy the stage's scale
//     bytes from shared memory into the stage's TMEM scale buffer with tcgen05.st (instead of
//     tcgen05.cp in the MMA issuer's instruction stream), then arrive on the leader's ready[s] --
//     which thereby also tells the leader that this CTA's operand tiles have landed;
//   MMA issuer (leader, 1 thread): wait ready[s] (8 arrivals: both CTAs' scale warps); 4 MMAs;
//     one commit multicast to empty[s] of both CTAs;
//   epilogue (8 warps per CTA): drain the accumulator, add the bias, round to bf16 into a 128-byte
//     swizzled staging box and write it with a TMA tensor store, twice per warp.
// The up projection T L2 (r/16 bf16 MMAs into the same accumulator): up to rank 64 its operands are
// loaded into the staging buffer, which the epilogue does not use during a tile's k-loop, once the
// previous tile's stores have read it, and their MMAs close the tile; larger ranks take ring
// stages before the k-blocks.  Kernel 2 is launched as a programmatic dependent of kernel 1.

constexpr int kGStages = 5;
// The epilogues with GELU (fused MLP pair, GELU output) run four stages: the fifth stage's shared
// memory holds the GELU table (the fused MLP epilogue outlasts the k-loop anyway).
__host__ __device__ constexpr int gemm_stages(int epi) { return epi >= 2 ? 4 : kGStages; }
// Warp roles, four warpgroups: 0 = the scale warps (warp w writes TMEM lane quadrant w); 1 = the
// operand producer, the MMA issuer, the scale producer and one idle warp; 2 and 3 = the epilogue.
constexpr int kGSfWarps = 4;
constexpr int kGProducerWarp = 4;
constexpr int kGMmaWarp = 5;
constexpr int kGScaleProducerWarp = 6;
constexpr int kGEpiWarps = 8;
constexpr int kGFirstEpiWarp = 8;
constexpr int kGThreads = (kGFirstEpiWarp + kGEpiWarps) * 32;
// Register split: the block is launched with kGRegsLaunch registers a thread (512 x 128 = the
// SM's 65536); warpgroup 0 then gives back down to kGRegsSf, warpgroup 1 to kGRegsLow, and the
// two epilogue warpgroups take kGRegsEpi (one thread holds a row's 128 accumulator columns).
constexpr int kGRegsLaunch = 128, kGRegsSf = 72, kGRegsLow = 72, kGRegsEpi = 184;
static_assert(128 * kGRegsSf + 128 * kGRegsLow + 2 * 128 * kGRegsEpi <= kGThreads * kGRegsLaunch,
              "register split exceeds the block's");
static_assert(kGRegsSf % 8 == 0 && kGRegsLow % 8 == 0 && kGRegsEpi % 8 == 0 && kGRegsLow >= 24 && kGRegsEpi <= 256,
              "setmaxnreg range");
static_assert(kGThreads * kGRegsLaunch <= 65536, "launch registers");
constexpr uint32_t kGA = kBM * kRowBytes;                   // 16 KB: own 128 rows of A
constexpr uint32_t kGB = (kBN / 2) * kRowBytes;             // 16 KB: own half of B
constexpr uint32_t kGSfa = kBM * kSfBytesPerRowKb;          // 2 KB of A scales per (m-tile, k-block)
constexpr uint32_t kGSfb = kBN * kSfBytesPerRowKb;          // 4 KB of B scales per (n-tile, k-block)
constexpr uint32_t kGStage = kGA + kGB + kGSfa + kGSfb;     // 38 KB
constexpr uint32_t kGOutBox = 32 * 128;                     // staging box: 32 rows x 64 bf16, 128-byte swizzle
constexpr uint32_t kGStaging = kGEpiWarps * kGOutBox;       // 32 KB: one box per epilogue warp
constexpr uint32_t kGLrL2Offset = 16384;                    // L2 half in staging (T before it; rank <= 64)
constexpr uint32_t kTmemCols = 512;
constexpr int kRopeAhead = 4;  // fused Q/K epilogue: rotary-table units in flight per thread
// Per-stage scale buffer: 12 blocks of 4 columns (SFA k-steps 0..3, then SFB k-steps 0..3 with
// two 128-row blocks each), in the order of the 12 blocks of 512 B of the global scale layout.
constexpr uint32_t kTmemSf = 256, kTmemSfCols = 48;
static_assert(kTmemSf + kGStages * kTmemSfCols <= kTmemCols, "TMEM columns");

struct GemmParams {
  int M, N, K, rank, KB, MT2, NT, ldy;
  const float* bias;
  int qk_cols;  // fused Q/K normalization and rotary embedding on columns [0, qk_cols)
  const float* gamma_q;
  const float* gamma_k;
  const float* rope;
  float eps;
  // fused MLP pair (see GemmArgs)
  const float* il_down;
  uint8_t* codes_down;
  uint8_t* sf_down;
  const uint8_t* l1_down;
  int r_down;
  float* tpart;
  int mlp_smax;  // slots per (row, column half) of tpart
};

// Box heights (256-byte rows) of the operand maps.
constexpr uint32_t kBoxA = kGA / 256, kBoxB = kGB / 256, kBoxSfa = kGSfa / 256, kBoxSfb = kGSfb / 256, kBoxLr = 16;

struct alignas(64) GemmMaps {
  CUtensorMap a, b, sfa, sfb, t, l2, y;
};

__device__ __forceinline__ void tmem_alloc2(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Arrive on the barrier at offset `bar` of both CTAs of the pair once all prior tcgen05 ops of
// this thread complete.
__device__ __forceinline__ void tc_commit2_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}
__device__ __forceinline__ void mma2_bf16(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma2_nvfp4(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t sfa,
                                           uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(sfa), "r"(sfb), "r"(acc)
      : "memory");
}
// 2-D tensor copy of this CTA's box into its own shared memory; completion is counted on the
// barrier at cluster address `bar` (the leader CTA's barrier for both CTAs of the pair).
__device__ __forceinline__ void tma_rows_cg2(void* smem_dst, const CUtensorMap* map, int row, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(row), "r"(bar)
      : "memory");
}

// Arrive on a barrier given by cluster address (possibly the peer CTA's).  Default (CTA-scope
// release) semantics: what the arrival publishes is TMEM state, ordered by the tcgen05 wait and
// fence that precede it, so no cluster-scope memory fence is needed (and it would stall the
// warp behind every memory operation the SM has in flight).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr) : "memory");
}
// 2-D tensor store of a box from this CTA's shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t ssrc, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(ssrc)
               : "memory");
}
__device__ __forceinline__ void bulk_s2g(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Lane 0 waits (bounded) and the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = !*abort_flag && wait_parity_bounded(bar, parity, kErrWaitGemm);
  return __shfl_sync(0xffffffffu, ok, 0);
}

// Read-only 16-byte load kept in program order (volatile asm), so the compiler does not hoist
// the epilogue's bias loads above the accumulator loads and run out of registers.
__device__ __forceinline__ float4 ldg_f4_in_order(const float* ptr) {
  float4 r;
  asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(ptr));
  return r;
}

// ---------------------------------------------------------------------------- bf16 GELU
// GELU(y) = y Phi(y) of a bf16 input y, rounded once to the nearest bf16 (ties to even), as the
// exact definition gives it.  Phi(y) = erfc(-y / sqrt 2) / 2 keeps full relative accuracy in the
// negative tail, where 1 + erf(y / sqrt 2) cancels.
//
// Nearest bf16 (as fp32) of a double, ties to even: the two bf16 neighbours of g come from
// truncating g toward zero to fp32 and then to bf16; both differences to g are exact in double.
__device__ __noinline__ float bf16_nearest_of_double(double g) {
  const uint32_t tb = __float_as_uint(__double2float_rz(g));
  const uint32_t lo = tb & 0xFFFF0000u, hi = lo + 0x10000u;
  const double dlo = fabs(g - static_cast<double>(__uint_as_float(lo)));
  const double dhi = fabs(static_cast<double>(__uint_as_float(hi)) - g);
  const bool up = dhi < dlo || (dhi == dlo && (lo & 0x10000u));
  return __uint_as_float(up ? hi : lo);
}

// The rare inputs whose fp32 evaluation does not decide the rounding.
__device__ __noinline__ float gelu_bf16_slow(float y) {
  const double yd = static_cast<double>(y);
  return bf16_nearest_of_double(0.5 * yd * erfc(-yd * 0.70710678118654752440));
}

// |y| < 2^-125, +-0 included: GELU(y) = y / 2 + y^2 / sqrt(2 pi) + O(y^4).  y / 2 is exact and a
// bf16 subnormal (spacing 2^-133) or zero here, and the correction, positive and far below half a
// spacing, only breaks ties, toward +infinity.  The bf16 magnitude bits of such a y are y in units
// of 2^-133, so this is integer arithmetic on the bits (no subnormal floating-point step); a zero
// keeps its sign, as y Phi(y) does.
__device__ __forceinline__ float gelu_bf16_tiny(uint32_t yb) {
  const uint32_t u = (yb >> 16) & 0x7FFFu;
  const uint32_t neg = yb & 0x80000000u;
  const uint32_t half = neg ? (u >> 1) : ((u + 1u) >> 1);
  return __uint_as_float(neg | (half << 16));
}

__device__ __forceinline__ float gelu_bf16(float y) {
  if ((__float_as_uint(y) & 0x7FFFFFFFu) < 0x01000000u) return gelu_bf16_tiny(__float_as_uint(y));
  const float z = __fmul_rn(y, -0.70710678118654752f);
  const float g = __fmul_rn(__fmul_rn(0.5f, y), erfcf(z));
  // Relative error of g: erfcf's documented 4 ulp, two roundings of the argument amplified by
  // |d ln erfc(z) / d ln z| <= 2 z^2 + 1 where z > 0 (the tail; for z <= 0 erfc lies in [1, 2] and
  // barely moves), and the last product; (16 + 2 z^2) 2^-23 covers them with room for the roundings
  // of the bracket itself.  Past z = 16 the value is far below fp32's normal range, where the
  // absolute term, |y| times a few units of erfcf's last place (2^-149), takes over; the floor
  // 2^-140 lies far below half a bf16 spacing anywhere (>= 2^-134).
  const float zp = fminf(fmaxf(z, 0.0f), 16.0f);
  const float rel = __fmul_rn(__fmaf_rn(__fmul_rn(2.0f, zp), zp, 16.0f), 0x1p-23f);
  const float d = __fmaf_rn(fabsf(g), rel, __fmaf_rn(fabsf(y), 0x1p-146f, 0x1p-140f));
  const float lo = __bfloat162float(__float2bfloat16_rn(__fsub_rn(g, d)));
  const float hi = __bfloat162float(__float2bfloat16_rn(__fadd_rn(g, d)));
  return __float_as_uint(lo) == __float_as_uint(hi) ? lo : gelu_bf16_slow(y);
}

// The fused MLP epilogue evaluates GELU for every hidden value, so the range that holds nearly all
// of them goes through a table in shared memory: the exact bf16 GELU of every bf16 input with |y|
// in [2^-10, 16) (both signs, 14 binades of 128 values, 7 KB), filled by gelu_bf16 itself at kernel
// start.  Outside that range the rounded value has a closed form (gelu_bf16_outside_table).
constexpr int kGeluTblE0 = 117;      // bf16 exponent field of 2^-10
constexpr int kGeluTblBinades = 14;  // 2^-10 .. 2^3
constexpr int kGeluTblSize = 2 * kGeluTblBinades * 128;

__device__ __noinline__ void fill_gelu_table(uint16_t* tbl, int tid, int nthreads) {
  for (int i = tid; i < kGeluTblSize; i += nthreads) {
    const uint32_t sign = static_cast<uint32_t>(i / (kGeluTblBinades * 128));
    const uint32_t rest = static_cast<uint32_t>(i % (kGeluTblBinades * 128));
    const uint32_t b = (sign << 15) | ((kGeluTblE0 + rest / 128) << 7) | (rest % 128);
    tbl[i] = static_cast<uint16_t>(__float_as_uint(gelu_bf16(__uint_as_float(b << 16))) >> 16);
  }
}

// The bf16 inputs outside the table, where GELU(y) = y/2 + y^2/sqrt(2 pi) + O(y^4) near zero and
// y (1 - Q(|y|)) or |y| Q(|y|) in the tails (Q the normal upper tail):
// - |y| < 2^-125: the tiny-input integer path (y/2 may be a bf16 subnormal with a tie);
// - 2^-125 <= |y| < 2^-10: y/2, a normal bf16 number; the correction, below 0.8 |y| |y/2| <
//   2^-10 |y/2|, stays under half the bf16 spacing next to y/2 on either side (at least 2^-9 |y/2|,
//   the side toward zero of a power of two included), so it cannot move the rounding;
// - y >= 16: y, since Q(16) < 1e-57;
// - y <= -16: -0, since |y| Q(|y|) < 1e-56 is below half the smallest bf16 subnormal (2^-134) and
//   the exact value is negative;
// - NaN: itself.
__device__ __forceinline__ float gelu_bf16_outside_table(float y) {
  const uint32_t a = __float_as_uint(y) & 0x7FFFFFFFu;
  if (a < 0x01000000u) return gelu_bf16_tiny(__float_as_uint(y));
  if (a < 0x3A800000u) return __fmul_rn(0.5f, y);
  if (y <= -16.0f) return -0.0f;
  return y;
}

// The correctly rounded bf16 GELU of a bf16 y (as fp32), with the table `tbl` in shared memory.
__device__ __forceinline__ float gelu_bf16_tab(float y, const uint16_t* tbl) {
  const uint32_t b = __float_as_uint(y) >> 16;
  const uint32_t e = ((b >> 7) & 0xFFu) - static_cast<uint32_t>(kGeluTblE0);
  if (e < static_cast<uint32_t>(kGeluTblBinades))
    return __uint_as_float(static_cast<uint32_t>(tbl[((b >> 15) * kGeluTblBinades + e) * 128u + (b & 127u)]) << 16);
  return gelu_bf16_outside_table(y);
}

// The same for the two bf16 values of a packed pair (low half first).
__device__ __forceinline__ uint32_t gelu_bf16x2_tab(uint32_t w, const uint16_t* tbl) {
  const float lo = gelu_bf16_tab(__uint_as_float(w << 16), tbl);
  const float hi = gelu_bf16_tab(__uint_as_float(w & 0xFFFF0000u), tbl);
  return (__float_as_uint(lo) >> 16) | (__float_as_uint(hi) & 0xFFFF0000u);
}

// The rare branch of gelu_bf16x8_warp, out of line so that the epilogues' unrolled loops stay small
// (their instruction fetch is a bottleneck of its own).
__device__ __noinline__ uint32_t gelu_bf16x2_rare(uint32_t w, const uint16_t* tbl) { return gelu_bf16x2_tab(w, tbl); }

// The same for the eight bf16 values packed in w[0..3], in place; warp-collective (all 32 lanes call
// it together).  When every value of every lane lies in the table's range (nearly always) each takes
// one table load and no branch of its own; otherwise every value goes through gelu_bf16_tab.
__device__ __forceinline__ void gelu_bf16x8_warp(uint32_t (&w)[4], const uint16_t* tbl) {
  constexpr uint32_t kN = kGeluTblBinades * 128, kBase = static_cast<uint32_t>(kGeluTblE0) << 7;
  uint32_t idx[8];
  bool in = true;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const uint32_t b = (t & 1) ? (w[t >> 1] >> 16) : (w[t >> 1] & 0xFFFFu);
    const uint32_t i = (b & 0x7FFFu) - kBase;  // wraps below the table
    in &= i < kN;
    idx[t] = (i < kN ? i : kN - 1) + (b >> 15) * kN;
  }
  if (__all_sync(0xffffffffu, in)) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      w[q] = static_cast<uint32_t>(tbl[idx[2 * q]]) | (static_cast<uint32_t>(tbl[idx[2 * q + 1]]) << 16);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = gelu_bf16x2_rare(w[q], tbl);
  }
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Staging box layout: 32 rows of 128 bytes (64 bf16); 16-byte unit u of row l sits at
// u ^ (l % 8), the tensor map's 128-byte swizzle, so lanes 8i..8i+7 hit distinct bank groups.
// kEpi: 0 = bias and bf16 Y; 1 = fused Q/K normalization and rotary embedding; 2 = fused MLP pair;
// 3 = bias, bf16, then GELU (Y = GELU(bf16(acc + bias)), each rounded to bf16).
template <int kEpi>
__global__ void __launch_bounds__(kGThreads, 1) gemm_nvfp4_kernel(const __grid_constant__ GemmMaps maps,
                                                                    const GemmParams p) {
  constexpr int kNS = gemm_stages(kEpi);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + kNS * kGStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + kGStaging);  // (both) this CTA's tiles landed
  uint64_t* empty = full + kNS;        // (both) MMAs done with the stage
  uint64_t* ready = empty + kNS;       // (leader) both CTAs' tiles landed and scales written
  uint64_t* acc_full = ready + kNS;    // (both) accumulator ready
  uint64_t* acc_empty = acc_full + 1;       // (leader) both CTAs drained the accumulator
  uint64_t* lr_full = acc_empty + 1;        // (leader) both CTAs' low-rank operands landed in staging
  uint64_t* stg_free = lr_full + 1;         // (both) the epilogue's stores finished reading staging
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stg_free + 1);
  float* gamma_sm = reinterpret_cast<float*>(staging + kGStaging + 256);  // fused Q/K: gamma_q, gamma_k
  uint16_t* gelu_tbl = reinterpret_cast<uint16_t*>(staging + kGStaging + 256);  // modes 2, 3: GELU table
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int r = p.rank;
  const int nlr = (r + kLrChunk - 1) / kLrChunk;
  const int tiles = p.MT2 * p.NT;
  // Up to rank 64 the low-rank operands (T and this CTA's half of L2: 512 r bytes) fit in the
  // epilogue's staging, which is idle during a tile's k-loop: they are loaded there once the
  // previous tile's stores have read it, and their MMAs close the tile.  Larger ranks, and the
  // fused epilogues (which can outlast a k-loop: the MMAs would wait for them), take ring stages
  // after the k-blocks; either way the tile's MMAs run in the same order (k-blocks, then the up
  // projection), so every epilogue mode sees the same accumulator.
  const bool lr_in_staging = kEpi == 0 && r > 0 && r <= 64;
  const int nlr_ring = lr_in_staging ? 0 : nlr;
  const int nstages_tile = p.KB + nlr_ring;  // k-blocks, then (ring) low-rank chunks
  // Tiles of this pair: interleaved (pair, pair + npairs, ...), except in the fused MLP mode, which
  // walks a contiguous m-major range so that consecutive tiles share rows and their partials of the
  // down layer's T accumulate in one slot.
  const int t_first = kEpi == 2 ? static_cast<int>(static_cast<long long>(pair) * tiles / npairs) : pair;
  const int t_end = kEpi == 2 ? static_cast<int>(static_cast<long long>(pair + 1) * tiles / npairs) : tiles;
  const int t_step = kEpi == 2 ? 1 : npairs;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready[s], 2 * kGSfWarps);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kGEpiWarps);
    mbar_init(lr_full, 1);
    mbar_init(stg_free, kGEpiWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kGMmaWarp) {
    tmem_alloc2(tmem_slot, kTmemCols);
    tmem_relinquish2();
  }
  if constexpr (kEpi >= 2) fill_gelu_table(gelu_tbl, threadIdx.x, kGThreads);  // (before kernel 1 ends)
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Launched as a programmatic dependent of kernel 1: everything above overlapped its tail; the
  // activation codes, scales and T are read only after it has completed.
  pdl_wait_primary();
  if (warp >= kGFirstEpiWarp) {
    setmaxnreg_inc<kGRegsEpi>();
    if constexpr (kEpi == 1) {  // the normalization weights, read by every row, into shared memory
      const int et = threadIdx.x - kGFirstEpiWarp * 32;
      gamma_sm[et] = et < kQkvHeadDim ? p.gamma_q[et] : p.gamma_k[et - kQkvHeadDim];
      asm volatile("bar.sync 1, %0;" ::"n"(kGEpiWarps * 32) : "memory");
    }
    // ------------------------------------------------------------ epilogue (8 warps per CTA)
    // Warp (q, h): rows 32 q .. 32 q + 31 of this CTA's 128, columns 128 h .. 128 h + 127 of the
    // tile; lane l holds row 32 q + l.  One staging box of 32 rows x 64 columns (128-byte rows,
    // 16-byte units swizzled by row % 8), filled and stored by TMA twice per tile.
    const int q = warp & 3, h = (warp - kGFirstEpiWarp) >> 2;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    uint8_t* box = staging + (warp - kGFirstEpiWarp) * kGOutBox;
    const uint32_t lrow = static_cast<uint32_t>(lane) * 128u;
    const bool lr_issuer = lr_in_staging && warp == kGFirstEpiWarp && lane == 0;
    const uint32_t lr_full_leader = mapa_shared(smem_u32(lr_full), 0);
    // This CTA's T rows and half of L2 for `tile`, into staging (T at 0, L2 at kGLrL2Offset),
    // completing on the leader's lr_full, which the leader arms with both CTAs' bytes.
    auto issue_lr = [&](int tile) {
      const int m2 = tile / p.NT, nt = tile % p.NT;
      const int mt = 2 * m2 + static_cast<int>(rank);
      const uint32_t tb = kBM * static_cast<uint32_t>(r) * 2, lb = (kBN / 2) * static_cast<uint32_t>(r) * 2;
      if (leader) mbar_arrive_expect_tx(lr_full, 2 * (tb + lb));
      const int trow = static_cast<int>(static_cast<size_t>(mt) * kBM * r * 2 / 256);
      const int lrow = static_cast<int>((static_cast<size_t>(nt) * kBN * r * 2 + rank * lb) / 256);
      for (uint32_t q = 0; q < tb / 4096; ++q) tma_rows_cg2(staging + 4096 * q, &maps.t, trow + 16 * q, lr_full_leader);
      for (uint32_t q = 0; q < lb / 4096; ++q)
        tma_rows_cg2(staging + kGLrL2Offset + 4096 * q, &maps.l2, lrow + 16 * q, lr_full_leader);
    };
    if (lr_issuer && t_first < t_end) issue_lr(t_first);
    int local = 0;
    for (int tile = t_first; tile < t_end; tile += t_step, ++local) {
      const int m2 = tile / p.NT, nt = tile % p.NT;
      const int row0 = (2 * m2 + static_cast<int>(rank)) * kBM + q * 32;
      const int n0 = nt * kBN + h * 128;
      // Fused Q/K: this row's rotary table goes in flight before the wait for the accumulator.  The
      // packed table (rope_packed_index) puts the 32 rows of a warp side by side, so each load reads
      // 512 contiguous bytes; the loads run kRopeAhead units ahead of their use.  Rows past M (never
      // stored) read the last row's angles.
      const float* rp = nullptr;
      float4 rq[kRopeAhead][2];
      if constexpr (kEpi == 1) {
        if (n0 < p.qk_cols) {
          const int m = row0 + lane < p.M ? row0 + lane : p.M - 1;
          rp = p.rope + rope_packed_index(m, 0, 0);
#pragma unroll
          for (int k = 0; k < kRopeAhead; ++k) {
            rq[k][0] = __ldg(reinterpret_cast<const float4*>(rp + rope_packed_index(0, k, 0)));
            rq[k][1] = __ldg(reinterpret_cast<const float4*>(rp + rope_packed_index(0, k, 1)));
          }
        }
      }
      if (!warp_wait(acc_full, static_cast<uint32_t>(local) & 1u, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tacc = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(h * 128);
      // All 128 columns are read before the accumulator is released (the next tile's MMAs wait
      // for it), then biased, rounded and staged.
      uint32_t v[2][2][32];
      tmem_ld32(tacc, v[0][0]);
      tmem_ld32(tacc + 32, v[0][1]);
      tmem_ld32(tacc + 64, v[1][0]);
      tmem_ld32(tacc + 96, v[1][1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty_leader);  // the accumulator may be overwritten now
      // Row l of the box starts at a multiple of 128 B, so unit u's address (row + ((u ^ l % 8) << 4))
      // is (row ^ ((l % 8) << 4)) ^ (u << 4): one XOR per store.
      const uint32_t srow_swz = smem_u32(box) + lrow ^ ((static_cast<uint32_t>(lane) & 7u) << 4);
      if constexpr (kEpi == 2) {
        // Fused MLP pair: the biased output rounded to bf16, GELU of it rounded to bf16, times the
        // down layer's 1/lambda: the down layer's x_hat.  It is quantized here into the down
        // layer's workspace (codes and UE4M3 scales of the 8 groups of 16 this thread holds, the
        // same exact rounding as kernel 1), and this half-tile's fp32 partial of the down layer's
        // T = bf16(x_hat) L1 comes from warp-level bf16 MMAs on a copy staged in the box.  Rows
        // past M hold zeros.
        const int grow = row0 + lane;
        const bool live = grow < p.M;
        const int gmt = grow >> 7, rin = grow & 127;
        uint8_t* const cdst = p.codes_down + codes_chunk_offset(gmt, nt, p.N / kBK, kBM);
        uint8_t* const sdst = p.sf_down + sf_chunk_offset(gmt, nt, p.N / kBK, kBM);
        const float kInv6 = __frcp_rn(6.0f);
        // D (mi, ni) of the T partial: rows 16 mi .. 16 mi + 15 of the warp's 32, T columns 8 ni ..
        // 8 ni + 7 (rank <= 32)
        const int nti = p.r_down >> 3, g8 = lane >> 2, t4 = lane & 3;
        float d[2][4][4];
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
          for (int ni = 0; ni < 4; ++ni)
#pragma unroll
            for (int e = 0; e < 4; ++e) d[mi][ni][e] = 0.0f;
#pragma unroll
        for (int bx = 0; bx < 2; ++bx) {  // 64 columns at a time through the box
          // the biased output rounded to bf16, into this thread's row of the box
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int hh = u >> 2, c = 8 * (u & 3);
            const float4 b0 = ldg_f4_in_order(p.bias + n0 + 64 * bx + 8 * u);
            const float4 b1 = ldg_f4_in_order(p.bias + n0 + 64 * bx + 8 * u + 4);
            st_shared_v4(srow_swz ^ (static_cast<uint32_t>(u) << 4),
                         make_uint4(pack_bf16x2(__uint_as_float(v[bx][hh][c]) + b0.x, __uint_as_float(v[bx][hh][c + 1]) + b0.y),
                                    pack_bf16x2(__uint_as_float(v[bx][hh][c + 2]) + b0.z, __uint_as_float(v[bx][hh][c + 3]) + b0.w),
                                    pack_bf16x2(__uint_as_float(v[bx][hh][c + 4]) + b1.x, __uint_as_float(v[bx][hh][c + 5]) + b1.y),
                                    pack_bf16x2(__uint_as_float(v[bx][hh][c + 6]) + b1.z, __uint_as_float(v[bx][hh][c + 7]) + b1.w)));
          }
          // Per 16-column group: GELU rounded to bf16, times the down layer's 1/lambda (its x_hat),
          // quantized with kernel 1's exact rounding into the down layer's workspace; bf16(x_hat)
          // goes back into the box for the T partial.  The loop is not unrolled, so that the GELU's
          // temporaries stay few (only the other half's accumulator columns remain in registers).
#pragma unroll 1
          for (int jg = 0; jg < 4; ++jg) {
            const uint32_t a0 = srow_swz ^ (static_cast<uint32_t>(2 * jg) << 4);
            const uint32_t a1 = srow_swz ^ (static_cast<uint32_t>(2 * jg + 1) << 4);
            const uint4 w0 = ld_shared_v4(a0), w1 = ld_shared_v4(a1);
            uint32_t g0[4] = {w0.x, w0.y, w0.z, w0.w}, g1[4] = {w1.x, w1.y, w1.z, w1.w};
            gelu_bf16x8_warp(g0, gelu_tbl);  // GELU of the 16 bf16 values, each rounded to bf16
            gelu_bf16x8_warp(g1, gelu_tbl);
            const uint32_t wy[8] = {g0[0], g0[1], g0[2], g0[3], g1[0], g1[1], g1[2], g1[3]};
            const float* ilp = p.il_down + n0 + 64 * bx + 16 * jg;
            float il[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const float4 t = __ldg(reinterpret_cast<const float4*>(ilp + 4 * q4));
              il[4 * q4] = t.x;
              il[4 * q4 + 1] = t.y;
              il[4 * q4 + 2] = t.z;
              il[4 * q4 + 3] = t.w;
            }
            uint64_t xp[2][4];
            float pm[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              const float lo = live ? __fmul_rn(__uint_as_float(wy[t] << 16), il[2 * t]) : 0.0f;
              const float hi = live ? __fmul_rn(__uint_as_float(wy[t] & 0xFFFF0000u), il[2 * t + 1]) : 0.0f;
              xp[t >> 2][t & 3] = f2pack(lo, hi);
              pm[t] = fmaxf(fabsf(lo), fabsf(hi));
            }
            const float amax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                     fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
            const float s_est = __fmul_rn(amax, kInv6);
            uint32_t sbits = cvt_e4m3(__fmul_rn(s_est, kNudgeLo));
            const uint32_t sc_hi = cvt_e4m3(__fmul_rn(s_est, kNudgeHi));
            uint2 code = make_uint2(0u, 0u);
            bool slow = sbits != sc_hi;
            if (!slow && sbits != 0) {
              const float rr = __frcp_rn(e4m3_to_f32(sbits));
              const float mlo = __fmul_rn(rr, kNudgeLo), mhi = __fmul_rn(rr, kNudgeHi);
              code.x = e2m1x8_scaled(xp[0], mlo);
              code.y = e2m1x8_scaled(xp[1], mlo);
              slow = (code.x != e2m1x8_scaled(xp[0], mhi)) | (code.y != e2m1x8_scaled(xp[1], mhi));
            }
            float xh[2][8];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
              for (int t = 0; t < 4; ++t) f2unpack(xp[hf][t], xh[hf][2 * t], xh[hf][2 * t + 1]);
            if (slow) {  // rare: the exact quotients decide
              sbits = cvt_e4m3(__fdiv_rn(amax, 6.0f));
              const float sd = e4m3_to_f32(sbits);
              code.x = sd != 0.0f ? e2m1x8_div(xh[0], sd) : 0u;
              code.y = sd != 0.0f ? e2m1x8_div(xh[1], sd) : 0u;
            }
            const int j = 4 * bx + jg;  // group j of the thread's 128 columns
            *reinterpret_cast<uint2*>(cdst + swz128(rin, 64 * h + 8 * j)) = code;
            sdst[sf_nvfp4_offset(rin, 8 * h + j, kBM)] = static_cast<uint8_t>(sbits);
            st_shared_v4(a0, make_uint4(pack_bf16x2(xh[0][0], xh[0][1]), pack_bf16x2(xh[0][2], xh[0][3]),
                                        pack_bf16x2(xh[0][4], xh[0][5]), pack_bf16x2(xh[0][6], xh[0][7])));
            st_shared_v4(a1, make_uint4(pack_bf16x2(xh[1][0], xh[1][1]), pack_bf16x2(xh[1][2], xh[1][3]),
                                        pack_bf16x2(xh[1][4], xh[1][5]), pack_bf16x2(xh[1][6], xh[1][7])));
          }
          if (p.r_down > 0) {
            __syncwarp();  // every row of the box holds bf16(x_hat)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              uint32_t a[2][4];
#pragma unroll
              for (int mi = 0; mi < 2; ++mi) {
                const uint32_t rr = 16u * mi + (lane & 7) + 8u * ((lane >> 3) & 1);
                const uint32_t un = 2u * ks + (lane >> 4);
                ldmatrix_x4(a[mi], smem_u32(box) + rr * 128u + ((un ^ (rr & 7u)) << 4));
              }
              const int kcol = n0 + 64 * bx + 16 * ks + 2 * t4;  // the down layer's k of b0
#pragma unroll
              for (int ni = 0; ni < 4; ++ni) {
                if (ni < nti) {
                  const uint32_t b0 = __ldg(reinterpret_cast<const uint32_t*>(
                      p.l1_down + l1_offset(static_cast<uint32_t>(kcol), 8u * ni + g8, p.r_down)));
                  const uint32_t b1 = __ldg(reinterpret_cast<const uint32_t*>(
                      p.l1_down + l1_offset(static_cast<uint32_t>(kcol + 8), 8u * ni + g8, p.r_down)));
                  mma_sync_bf16_16816(d[0][ni], a[0], b0, b1);
                  mma_sync_bf16_16816(d[1][ni], a[1], b0, b1);
                }
              }
            }
          }
          __syncwarp();  // the box is rewritten by the next half
        }
        if (p.r_down > 0) {
          // This pair's slot among the pairs whose tile ranges meet these rows (it owns the slot):
          // the first tile of the pair's run on these rows stores, the later ones add in tile order.
          const int p_first = static_cast<int>((static_cast<long long>(m2 * p.NT + 1) * npairs - 1) / tiles);
          const int slot = pair - p_first;
          const bool seg_start = tile == t_first || (tile - 1) / p.NT != m2;
          const int nslots = 2 * p.mlp_smax;
          float* const tp = p.tpart + static_cast<size_t>(row0) * nslots * p.r_down + (h * p.mlp_smax + slot) * p.r_down;
#pragma unroll
          for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int ni = 0; ni < 4; ++ni)
              if (ni < nti)
#pragma unroll
                for (int jh = 0; jh < 2; ++jh) {
                  const int rl = 16 * mi + g8 + 8 * jh;
                  float2* dst = reinterpret_cast<float2*>(tp + static_cast<size_t>(rl) * nslots * p.r_down + 8 * ni + 2 * t4);
                  float2 pv = make_float2(d[mi][ni][2 * jh], d[mi][ni][2 * jh + 1]);
                  if (!seg_start) {
                    const float2 o = *dst;
                    pv = make_float2(o.x + pv.x, o.y + pv.y);
                  }
                  *dst = pv;
                }
        }
        fence_proxy_async_smem();  // the box's generic accesses precede the next tile's bulk copies into staging
      } else {
        // Fused Q/K path: the thread's 128 columns are one head of its row.  Bias first, and the
        // head's mean square.
        bool qk = false;
        float nrm = 0.0f;
        const float* gam = nullptr;
        if constexpr (kEpi == 1) {
          qk = n0 < p.qk_cols;
          if (qk) {
            float ss = 0.0f;
#pragma unroll
            for (int bx = 0; bx < 2; ++bx)
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int hh = u >> 2, c = 8 * (u & 3);
                const float4 b0 = ldg_f4_in_order(p.bias + n0 + 64 * bx + 8 * u);
                const float4 b1 = ldg_f4_in_order(p.bias + n0 + 64 * bx + 8 * u + 4);
                const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const float x = __uint_as_float(v[bx][hh][c + j]) + bb[j];
                  v[bx][hh][c + j] = __float_as_uint(x);
                  ss = fmaf(x, x, ss);
                }
              }
            nrm = rsqrtf(fmaf(ss, 1.0f / kQkvHeadDim, p.eps));
            gam = gamma_sm + (n0 < p.qk_cols / 2 ? 0 : kQkvHeadDim);
          }
        }
#pragma unroll
        for (int bx = 0; bx < 2; ++bx) {
          bulk_wait_read0();  // (lane 0's groups) the box's previous store has finished reading it
          __syncwarp();
#pragma unroll
          for (int u = 0; u < 8; ++u) {  // 16-byte unit u: columns 8u .. 8u + 7 of the box
            const int hh = u >> 2, c = 8 * (u & 3);
            uint4 o;
            if (kEpi == 1 && qk) {
              // normalize (x / rms * gamma), then turn pairs (2i, 2i + 1) by the row's angle i
              const int k = 8 * bx + u, slot = k % kRopeAhead;
              const float4 g0 = *reinterpret_cast<const float4*>(gam + 8 * k);
              const float4 g1 = *reinterpret_cast<const float4*>(gam + 8 * k + 4);
              const float4 r0 = rq[slot][0];  // (cos, sin) of pairs 0, 1
              const float4 r1 = rq[slot][1];  // pairs 2, 3
              if (k + kRopeAhead < 16) {
                rq[slot][0] = __ldg(reinterpret_cast<const float4*>(rp + rope_packed_index(0, k + kRopeAhead, 0)));
                rq[slot][1] = __ldg(reinterpret_cast<const float4*>(rp + rope_packed_index(0, k + kRopeAhead, 1)));
              }
              const float x0 = __uint_as_float(v[bx][hh][c + 0]) * nrm * g0.x;
              const float x1 = __uint_as_float(v[bx][hh][c + 1]) * nrm * g0.y;
              const float x2 = __uint_as_float(v[bx][hh][c + 2]) * nrm * g0.z;
              const float x3 = __uint_as_float(v[bx][hh][c + 3]) * nrm * g0.w;
              const float x4 = __uint_as_float(v[bx][hh][c + 4]) * nrm * g1.x;
              const float x5 = __uint_as_float(v[bx][hh][c + 5]) * nrm * g1.y;
              const float x6 = __uint_as_float(v[bx][hh][c + 6]) * nrm * g1.z;
              const float x7 = __uint_as_float(v[bx][hh][c + 7]) * nrm * g1.w;
              o.x = pack_bf16x2(x0 * r0.x - x1 * r0.y, x0 * r0.y + x1 * r0.x);
              o.y = pack_bf16x2(x2 * r0.z - x3 * r0.w, x2 * r0.w + x3 * r0.z);
              o.z = pack_bf16x2(x4 * r1.x - x5 * r1.y, x4 * r1.y + x5 * r1.x);
              o.w = pack_bf16x2(x6 * r1.z - x7 * r1.w, x6 * r1.w + x7 * r1.z);
            } else {
              const float4 b0 = ldg_f4_in_order(p.bias + n0 + 64 * bx + 8 * u);
              const float4 b1 = ldg_f4_in_order(p.bias + n0 + 64 * bx + 8 * u + 4);
              o.x = pack_bf16x2(__uint_as_float(v[bx][hh][c + 0]) + b0.x, __uint_as_float(v[bx][hh][c + 1]) + b0.y);
              o.y = pack_bf16x2(__uint_as_float(v[bx][hh][c + 2]) + b0.z, __uint_as_float(v[bx][hh][c + 3]) + b0.w);
              o.z = pack_bf16x2(__uint_as_float(v[bx][hh][c + 4]) + b1.x, __uint_as_float(v[bx][hh][c + 5]) + b1.y);
              o.w = pack_bf16x2(__uint_as_float(v[bx][hh][c + 6]) + b1.z, __uint_as_float(v[bx][hh][c + 7]) + b1.w);
              if constexpr (kEpi == 3) {  // GELU of each bf16 output, rounded to bf16 once more
                uint32_t g4[4] = {o.x, o.y, o.z, o.w};
                gelu_bf16x8_warp(g4, gelu_tbl);
                o = make_uint4(g4[0], g4[1], g4[2], g4[3]);
              }
            }
            st_shared_v4(srow_swz ^ (static_cast<uint32_t>(u) << 4), o);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (row0 < p.M && n0 + 64 * bx < p.N) tma_store_2d(&maps.y, smem_u32(box), n0 + 64 * bx, row0);
            bulk_commit();
          }
        }
      }
      if (lr_in_staging && tile + t_step < t_end) {
        // staging is about to receive the next tile's low-rank operands
        bulk_wait_read0();  // (lane 0's groups)
        __syncwarp();
        if (lane == 0) mbar_arrive(stg_free);
        if (lr_issuer) {
          if (*abort_flag || !wait_parity_bounded(stg_free, static_cast<uint32_t>(local) & 1u, kErrWaitGemm)) {
            *abort_flag = 1;
            break;
          }
          issue_lr(tile + t_step);
        }
      }
    }
    if (lane == 0) bulk_wait0();
  } else if (warp < kGSfWarps) {
    setmaxnreg_dec<kGRegsSf>();
    // ------------------------------------------------------------ scale warps (both CTAs)
    // Warp of lane quadrant q: lane l copies, for each of the stage's 12 scale blocks of 512 B in
    // shared memory, bytes [16 l, 16 l + 16) into TMEM lane 32 q + l, four columns per block (the
    // same contents in every quadrant, as the MMA's scale layout wants).
    const int q = warp & 3;
    const uint32_t ready_leader = mapa_shared(smem_u32(ready), 0);
    const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16) + kTmemSf;
    int st = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int tile = t_first; tile < t_end && ok; tile += t_step) {
      for (int j = 0; j < nstages_tile; ++j) {
        if (!warp_wait(&full[st], ph, abort_flag)) {
          ok = false;
          break;
        }
        if (j < p.KB) {
          tc_fence_after();  // the MMAs that last read this buffer completed before the stage refilled
          const uint8_t* src = smem + st * kGStage + kGA + kGB + 16 * lane;
          uint32_t v[3][16];
#pragma unroll
          for (int b = 0; b < 12; ++b) {
            const uint4 w = *reinterpret_cast<const uint4*>(src + 512 * b);
            v[b >> 2][4 * (b & 3) + 0] = w.x;
            v[b >> 2][4 * (b & 3) + 1] = w.y;
            v[b >> 2][4 * (b & 3) + 2] = w.z;
            v[b >> 2][4 * (b & 3) + 3] = w.w;
          }
          const uint32_t dst = tq + kTmemSfCols * static_cast<uint32_t>(st);
          tmem_st16(dst, v[0]);
          tmem_st16(dst + 16, v[1]);
          tmem_st16(dst + 32, v[2]);
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(ready_leader + 8u * st);
        if (++st == kNS) {
          st = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok) *abort_flag = 1;
  } else {
    setmaxnreg_dec<kGRegsLow>();
    if (warp == kGProducerWarp) {
      if (lane == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        int st = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int tile = t_first; tile < t_end && ok; tile += t_step) {
          const int m2 = tile / p.NT, nt = tile % p.NT;
          const int mt = 2 * m2 + static_cast<int>(rank);  // this CTA's 128-row tile
          for (int j = 0; j < nstages_tile; ++j) {
            if (*abort_flag || !wait_parity_bounded(&empty[st], ph ^ 1u, kErrWaitGemm)) {
              ok = false;
              break;
            }
            uint8_t* sb = smem + st * kGStage;
            if (j >= p.KB) {  // low-rank chunk j - KB
              const int lc = j - p.KB;
              const uint32_t cw = lr_chunk_width(r, lc);
              const uint32_t tb = kBM * cw * 2, lb = (kBN / 2) * cw * 2;
              mbar_arrive_expect_tx(&full[st], tb + lb);
              const int trow = static_cast<int>((static_cast<size_t>(mt) * kBM * r * 2 + static_cast<size_t>(kBM) * kLrChunk * 2 * lc) / 256);
              const int lrow = static_cast<int>((static_cast<size_t>(nt) * kBN * r * 2 + static_cast<size_t>(kBN) * kLrChunk * 2 * lc + rank * lb) / 256);
              for (uint32_t q = 0; q < tb / 4096; ++q) tma_load_2d(sb + 4096 * q, &maps.t, 0, trow + 16 * q, &full[st]);
              for (uint32_t q = 0; q < lb / 4096; ++q) tma_load_2d(sb + kGA + 4096 * q, &maps.l2, 0, lrow + 16 * q, &full[st]);
            } else {
              const int kb = j;
              mbar_arrive_expect_tx(&full[st], kGStage);
              tma_load_2d(sb, &maps.a, 0, static_cast<int>(codes_chunk_offset(mt, kb, p.KB, kBM) / 256), &full[st]);
              tma_load_2d(sb + kGA, &maps.b, 0, static_cast<int>((codes_chunk_offset(nt, kb, p.KB, kBN) + rank * kGB) / 256),
                          &full[st]);
            }
            if (++st == kNS) {
              st = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) *abort_flag = 1;
      }
    } else if (warp == kGScaleProducerWarp) {
      if (lane == 0) {
        // ------------------------------------------------------------ scale producer (both CTAs)
        // Copies each k-block stage's two scale tiles onto full[s], which the operand producer arms
        // with the whole stage's bytes (a copy may complete before that arrival; the phase cannot).
        int st = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int tile = t_first; tile < t_end && ok; tile += t_step) {
          const int m2 = tile / p.NT, nt = tile % p.NT;
          const int mt = 2 * m2 + static_cast<int>(rank);
          for (int j = 0; j < nstages_tile; ++j) {
            if (j < p.KB) {
              if (*abort_flag || !wait_parity_bounded(&empty[st], ph ^ 1u, kErrWaitGemm)) {
                ok = false;
                break;
              }
              const int kb = j;
              uint8_t* sb = smem + st * kGStage;
              tma_load_2d(sb + kGA + kGB, &maps.sfa, 0, static_cast<int>(sf_chunk_offset(mt, kb, p.KB, kBM) / 256), &full[st]);
              tma_load_2d(sb + kGA + kGB + kGSfa, &maps.sfb, 0, static_cast<int>(sf_chunk_offset(nt, kb, p.KB, kBN) / 256),
                          &full[st]);
            }
            if (++st == kNS) {
              st = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) *abort_flag = 1;
      }
    } else if (warp == kGMmaWarp) {
      if (lane == 0 && leader) {
        // ------------------------------------------------------------ MMA issuer (leader CTA)
        const uint32_t id_lr = idesc_bf16(256, 256);
        const uint32_t id_fp4 = idesc_nvfp4(256, 256);
        int st = 0;
        uint32_t ph = 0;
        bool ok = true;
        int local = 0;
        for (int tile = t_first; tile < t_end && ok; tile += t_step, ++local) {
          if (*abort_flag || !wait_parity_bounded(acc_empty, (static_cast<uint32_t>(local) & 1u) ^ 1u, kErrWaitGemm)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t accum = 0;
          for (int j = 0; j < nstages_tile; ++j) {
            if (*abort_flag || !wait_parity_bounded(&ready[st], ph, kErrWaitGemm)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sb = smem_u32(smem + st * kGStage);
            if (j >= p.KB) {  // low-rank chunk j - KB
              const uint32_t cw = lr_chunk_width(r, j - p.KB);
              const uint64_t ad = smem_desc(sb, 128, cw * 16, kLayoutNone);
              const uint64_t bd = smem_desc(sb + kGA, 128, cw * 16, kLayoutNone);
              for (uint32_t ks = 0; ks < cw / 16; ++ks) {
                mma2_bf16(tmem, ad + 16 * ks, bd + 16 * ks, id_lr, accum);
                accum = 1;
              }
            } else {
              const uint32_t sf = tmem + kTmemSf + kTmemSfCols * static_cast<uint32_t>(st);
              const uint64_t ad = smem_desc(sb, 16, 1024, kLayoutSw128);
              const uint64_t bd = smem_desc(sb + kGA, 16, 1024, kLayoutSw128);
  #pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                mma2_nvfp4(tmem, ad + 2 * kk, bd + 2 * kk, id_fp4, sf + 4 * kk, sf + 16 + 8 * kk, accum);
                accum = 1;
              }
            }
            tc_commit2_both(smem_u32(&empty[st]));
            if (++st == kNS) {
              st = 0;
              ph ^= 1u;
            }
          }
          if (!ok) break;
          if (lr_in_staging) {
            if (*abort_flag || !wait_parity_bounded(lr_full, static_cast<uint32_t>(local) & 1u, kErrWaitGemm)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sg = smem_u32(staging);
            const uint64_t ad = smem_desc(sg, 128, static_cast<uint32_t>(r) * 16, kLayoutNone);
            const uint64_t bd = smem_desc(sg + kGLrL2Offset, 128, static_cast<uint32_t>(r) * 16, kLayoutNone);
            for (int ks = 0; ks < r / 16; ++ks) mma2_bf16(tmem, ad + 16 * ks, bd + 16 * ks, id_lr, 1u);
          }
          tc_commit2_both(smem_u32(acc_full));
        }
        if (!ok) {
          *abort_flag = 1;
          tc_commit2_both(smem_u32(acc_full));  // completes once every issued tcgen05 op has
        }
      }
    }
  }

  __syncthreads();
  if (warp == kGMmaWarp && leader && *abort_flag && lane == 0) {
    const unsigned long long t0 = globaltimer_ns();  // the abort-path commits land within microseconds
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  tc_fence_before();
  cluster_sync();  // neither CTA releases TMEM or exits while its peer may still address it
  if (warp == kGMmaWarp) {
    tc_fence_after();
    tmem_dealloc2(tmem, kTmemCols);
  }
}

// ============================================================================ kernel 2, INT4
//
// INT4 codes with one fp32 scale per 64 elements cannot use block-scaled MMAs.  Converter warps
// therefore dequantize each 64-element group into bf16 operand tiles in shared memory: one LOP3
// puts two sign-flipped codes into the mantissas of 128, a bf16x2 subtract of 136 leaves the
// signed values (exact), and a bf16x2 multiply by the group's scale gives bf16(q s) -- the scale
// taken to bf16 first.  bf16 MMAs (kind::f16) then accumulate the whole tile, the up projection
// T L2 included, in one fp32 accumulator in tensor memory, double buffered so that the next tile's
// MMAs run while the epilogue drains this one; the epilogue only adds the bias (and applies the
// fused Q/K normalization and rotary turn).  Within a group, the MMA's k order is free as long as
// A and B share it: a 32-bit word of codes (elements e0..e7) becomes the bf16 pairs (e0, e4),
// (e1, e5), (e2, e6), (e3, e7) on both sides, with no byte shuffles.  Rounding each operand to
// bf16 keeps Y within about 1e-3 (relative Frobenius) of the exact grouped sum.
// Warp roles, four warpgroups: 0 = converters, 1 = producer, MMA issuer and two idle warps, 2 and 3
// = epilogue; the converters and warpgroup 1 give registers to the epilogue (setmaxnreg).

constexpr int kIStages = 3;                                   // packed stages
constexpr int kIGroups = 2;                                   // bf16 group buffers
constexpr int kIAcc = 2;                                      // TMEM accumulators (128 columns each)
constexpr int kISfStages = 4;                                 // scale stages (one k-block each)
constexpr uint32_t kISfA = kBM * 4 * 4;                       // 2 KB: fp32 [128 rows][4 groups]
constexpr uint32_t kISfB = 4 * kBN * 4;                       // 4 KB: fp32 [4 groups][256 rows]
constexpr int kIBN = 128;                                     // output columns per tile
constexpr int kIConvWarps = 4;                                // warps 0-3
constexpr int kIProducerWarp = 4;
constexpr int kIMmaWarp = 5;
constexpr int kIFirstEpiWarp = 8;
constexpr int kIEpiWarps = 8;                                 // warps 8-15
constexpr int kIEpiCols = kIBN / (kIEpiWarps / 4);             // 64 accumulator columns per epilogue thread
constexpr int kIThreads = (kIFirstEpiWarp + kIEpiWarps) * 32;
constexpr int kIRegsLaunch = 128, kIRegsConv = 64, kIRegsLow = 40, kIRegsEpi = 200;
static_assert(128 * kIRegsConv + 128 * kIRegsLow + 2 * 128 * kIRegsEpi <= kIThreads * kIRegsLaunch,
              "register split exceeds the block's");
static_assert(kIThreads * kIRegsLaunch <= 65536, "launch registers");
constexpr uint32_t kIPackA = kBM * kRowBytes;                 // 16 KB
constexpr uint32_t kIPackB = kIBN * kRowBytes;                // 16 KB
constexpr uint32_t kIPack = kIPackA + kIPackB;
constexpr uint32_t kIGrpA = kBM * 128;                        // 16 KB: 128 rows x 64 f16
constexpr uint32_t kIGrpB = kIBN * 128;
constexpr uint32_t kIGrp = kIGrpA + kIGrpB;
constexpr uint32_t kIStagePitch = kIBN * 2 + 16;              // bf16 output row + 16 B
constexpr uint32_t kIStaging = kBM * kIStagePitch;

struct GemmI4Params {
  int M, N, K, rank, KB, MT, NT, ldy;
  const uint8_t* a_codes;
  const float* a_sf;
  const uint8_t* t;
  const uint8_t* b_codes;
  const float* b_sf;
  const uint8_t* l2;
  const float* bias;
  uint16_t* Y;
  int qk_cols;  // fused Q/K normalization and rotary embedding on columns [0, qk_cols)
  const float* gamma_q;
  const float* gamma_k;
  const float* rope;
  float eps;
};

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}


// Eight packed int4 codes (element j in bits 4j..4j+3) -> four bf16x2 registers holding the pairs
// (e0, e4), (e1, e5), (e2, e6), (e3, e7) times the bf16 pair s2: (w >> 4s) & 0x000F000F puts e_s and
// e_s+4 in the low mantissa bits of two bf16 halves; XOR 0x4308 makes each half 128 + (v ^ 8) =
// 136 + q, the subtract of 136 leaves q exactly, and the multiply rounds q s once.
__device__ __forceinline__ uint4 int4x8_to_bf16_scaled(uint32_t w, uint32_t s2) {
  uint32_t r[4];
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    uint32_t t, q;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(t) : "r"(w >> (4 * s)), "r"(0x000F000Fu), "r"(0x43084308u));
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(q) : "r"(t), "r"(0x43084308u));
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r[s]) : "r"(q), "r"(s2));
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

__global__ void __launch_bounds__(kIThreads, 1) gemm_int4_kernel(const GemmI4Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* packed = smem;                                  // kIStages x 32 KB
  uint8_t* groups = packed + kIStages * kIPack;            // kIGroups x 32 KB (bf16 A, B)
  uint8_t* sfring = groups + kIGroups * kIGrp;              // kISfStages x 6 KB
  uint8_t* staging = sfring + kISfStages * (kISfA + kISfB);
  uint64_t* pfull = reinterpret_cast<uint64_t*>(staging + kIStaging);
  uint64_t* pempty = pfull + kIStages;
  uint64_t* gfull = pempty + kIStages;
  uint64_t* gempty = gfull + kIGroups;
  uint64_t* tfull = gempty + kIGroups;
  uint64_t* tempty = tfull + kIAcc;
  uint64_t* sfull = tempty + kIAcc;
  uint64_t* sempty = sfull + kISfStages;
  uint64_t* sspair = sempty + kISfStages;  // (fused Q/K) both column halves' sums of squares written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sspair + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = p.rank;
  const int nlr = (r + kLrChunk - 1) / kLrChunk;
  const int tiles = p.MT * p.NT;
  const int nst = nlr + p.KB;         // packed stages per tile
  const int ngrp = p.KB * 4;          // 64-element groups per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < kIStages; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], 1);
    }
    for (int s = 0; s < kIGroups; ++s) {
      mbar_init(&gfull[s], kIConvWarps);
      mbar_init(&gempty[s], 1);
    }
    for (int b = 0; b < kIAcc; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kIEpiWarps);
    }
    for (int b = 0; b < kISfStages; ++b) {
      mbar_init(&sfull[b], 1);
      mbar_init(&sempty[b], kIConvWarps);
    }
    for (int q = 0; q < 4; ++q) mbar_init(&sspair[q], 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kIMmaWarp) {
    tmem_alloc(tmem_slot, kIAcc * kIBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kIFirstEpiWarp) {
    setmaxnreg_inc<kIRegsEpi>();
    // ------------------------------------------------------------ epilogue (8 warps)
    const int ew = warp - kIFirstEpiWarp;
    const int q = warp & 3, cg = ew >> 2;  // TMEM lane quadrant this warp may access (warp % 4), column group
    const int rloc = q * 32 + lane;
    uint8_t* srow = staging + rloc * kIStagePitch + cg * kIEpiCols * 2;
    int local = 0, qkn = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++local) {
      const int mt = tile / p.NT, n128 = tile % p.NT;
      const uint32_t b = static_cast<uint32_t>(local) & 1u;  // accumulator of this tile
      bool w = true;
      if (lane == 0)
        w = !*abort_flag && wait_parity_bounded(&tfull[b], (static_cast<uint32_t>(local) >> 1) & 1u, kErrWaitGemm);
      if (!__shfl_sync(0xffffffffu, w, 0)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // this thread's 64 accumulator columns of its row; then the accumulator goes back to the MMA
      uint64_t acc[kIEpiCols / 2];  // fp32 pairs
      {
        uint32_t v0[32], v1[32];
        const uint32_t ta = tmem + b * kIBN + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(cg * kIEpiCols);
        tmem_ld32(ta, v0);
        tmem_ld32(ta + 32, v1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[b]);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          acc[c] = f2pack(__uint_as_float(v0[2 * c]), __uint_as_float(v0[2 * c + 1]));
          acc[16 + c] = f2pack(__uint_as_float(v1[2 * c]), __uint_as_float(v1[2 * c + 1]));
        }
      }
      // bias, bf16, stage, one bulk store per row segment
      const int row = mt * kBM + rloc;
      const int n0 = n128 * kIBN + cg * kIEpiCols;
      // Fused Q/K path: the tile's 128 columns are one head; this thread holds half of its row, so
      // the two column halves exchange their sums of squares (double-buffered slots, one barrier
      // phase per such tile, bounded wait) and add them in column order.
      const bool qk = p.qk_cols > 0 && n128 * kIBN < p.qk_cols;
      float nrm = 0.0f;
      if (qk) {
        float ssq = 0.0f;
#pragma unroll
        for (int u = 0; u < kIEpiCols / 8; ++u) {
          const float4 b0 = __ldg(reinterpret_cast<const float4*>(p.bias + n0 + u * 8));
          const float4 b1 = __ldg(reinterpret_cast<const float4*>(p.bias + n0 + u * 8 + 4));
          const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float x0, x1;
            f2unpack(acc[u * 4 + k], x0, x1);
            x0 += bb[2 * k];
            x1 += bb[2 * k + 1];
            acc[u * 4 + k] = f2pack(x0, x1);
            ssq = fmaf(x0, x0, ssq);
            ssq = fmaf(x1, x1, ssq);
          }
        }
        float* slots = reinterpret_cast<float*>(staging + kIStaging + 1024);  // [2 parities][2 halves][128 rows]
        const int par = qkn & 1;
        slots[(par * 2 + cg) * kBM + rloc] = ssq;
        __syncwarp();
        bool w = true;
        if (lane == 0) {
          mbar_arrive(&sspair[q]);
          w = !*abort_flag && wait_parity_bounded(&sspair[q], static_cast<uint32_t>(par), kErrWaitGemm);
        }
        if (!__shfl_sync(0xffffffffu, w, 0)) {
          ok = false;
          break;
        }
        const float other = slots[(par * 2 + (cg ^ 1)) * kBM + rloc];
        nrm = rsqrtf(fmaf(cg == 0 ? ssq + other : other + ssq, 1.0f / 128.0f, p.eps));
        ++qkn;
      }
      bulk_wait_read0();
      const float* gam = n128 * kIBN < p.qk_cols / 2 ? p.gamma_q : p.gamma_k;
      const int mrope = row < p.M ? row : p.M - 1;
#pragma unroll
      for (int u = 0; u < kIEpiCols / 8; ++u) {
        uint4 o;
        float a[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) f2unpack(acc[u * 4 + k], a[2 * k], a[2 * k + 1]);
        if (qk) {
          // normalize, then turn pairs (2i, 2i + 1) of the head by the row's angle i
          const int hc = cg * kIEpiCols + u * 8;  // the head's channel of a[0]
          const float4 g0 = __ldg(reinterpret_cast<const float4*>(gam + hc));
          const float4 g1 = __ldg(reinterpret_cast<const float4*>(gam + hc + 4));
          const float4 r0 = __ldg(reinterpret_cast<const float4*>(p.rope + rope_packed_index(mrope, hc >> 3, 0)));
          const float4 r1 = __ldg(reinterpret_cast<const float4*>(p.rope + rope_packed_index(mrope, hc >> 3, 1)));
          const float x0 = a[0] * nrm * g0.x, x1 = a[1] * nrm * g0.y, x2 = a[2] * nrm * g0.z, x3 = a[3] * nrm * g0.w;
          const float x4 = a[4] * nrm * g1.x, x5 = a[5] * nrm * g1.y, x6 = a[6] * nrm * g1.z, x7 = a[7] * nrm * g1.w;
          o.x = pack_bf16x2(x0 * r0.x - x1 * r0.y, x0 * r0.y + x1 * r0.x);
          o.y = pack_bf16x2(x2 * r0.z - x3 * r0.w, x2 * r0.w + x3 * r0.z);
          o.z = pack_bf16x2(x4 * r1.x - x5 * r1.y, x4 * r1.y + x5 * r1.x);
          o.w = pack_bf16x2(x6 * r1.z - x7 * r1.w, x6 * r1.w + x7 * r1.z);
        } else {
          const float4 b0 = __ldg(reinterpret_cast<const float4*>(p.bias + n0 + u * 8));
          const float4 b1 = __ldg(reinterpret_cast<const float4*>(p.bias + n0 + u * 8 + 4));
          o.x = pack_bf16x2(a[0] + b0.x, a[1] + b0.y);
          o.y = pack_bf16x2(a[2] + b0.z, a[3] + b0.w);
          o.z = pack_bf16x2(a[4] + b1.x, a[5] + b1.y);
          o.w = pack_bf16x2(a[6] + b1.z, a[7] + b1.w);
        }
        *reinterpret_cast<uint4*>(srow + 16 * u) = o;
      }
      fence_proxy_async_smem();
      if (row < p.M && n0 < p.N) {
        const int ncols = (p.N - n0) < kIEpiCols ? (p.N - n0) : kIEpiCols;
        bulk_s2g(p.Y + static_cast<size_t>(row) * p.ldy + n0, smem_u32(srow), static_cast<uint32_t>(ncols) * 2u);
      }
      bulk_commit();
    }
    bulk_wait0();
    if (!ok) *abort_flag = 1;
  } else if (warp < kIConvWarps) {
    setmaxnreg_dec<kIRegsConv>();
    // ------------------------------------------------------------ converters (4 warps)
    // After an abort a warp skips its work but still passes every named barrier, so the four
    // converter warps always execute the same barrier sequence.
    const int t = threadIdx.x;  // 0..127: one row of A and one of B
    int st = 0, gs = 0, ss = 0;
    uint32_t ph = 0, gph = 0, sph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
      const int nh = (tile % p.NT) & 1;  // this CTA's half of the 256-row weight tile
      for (int j = 0; j < nst; ++j) {
        if (j < nlr) {  // low-rank stages go straight to the MMA
          if (++st == kIStages) {
            st = 0;
            ph ^= 1u;
          }
          continue;
        }
        bool w = ok;
        if (lane == 0 && w) {
          w = !*abort_flag && wait_parity_bounded(&pfull[st], ph, kErrWaitGemm);
          if (w) w = wait_parity_bounded(&sfull[ss], sph, kErrWaitGemm);  // the k-block's scales
        }
        ok = __shfl_sync(0xffffffffu, w, 0);
        const uint8_t* pk = packed + st * kIPack;
        const float* sfa = reinterpret_cast<const float*>(sfring + ss * (kISfA + kISfB));
        const float* sfb = sfa + kISfA / 4;
        for (int gi = 0; gi < 4; ++gi) {
          bool e = ok;
          if (lane == 0 && e) e = !*abort_flag && wait_parity_bounded(&gempty[gs], gph ^ 1u, kErrWaitGemm);
          ok = __shfl_sync(0xffffffffu, e, 0);
          if (ok) {
            uint8_t* gb = groups + gs * kIGrp;
#pragma unroll
            for (int op = 0; op < 2; ++op) {  // A then B: row t of each
              const uint8_t* src = pk + op * kIPackA;
              uint8_t* dst = gb + op * kIGrpA;
              const float sc = op == 0 ? sfa[sf_int4_a_index(t, gi)] : sfb[sf_int4_b_index(nh * kIBN + t, gi)];
              const uint32_t s2 = pack_bf16x2(sc, sc);
              // row t of the group: eight 16-byte bf16 units (one per packed 32-bit word), unit u
              // at core matrix (t / 8, u) of the no-swizzle K-major layout (128 bytes between core
              // matrices along K, 1024 bytes per 8-row block)
              const uint32_t base = (t >> 3) * 1024u + (t & 7) * 16u;
#pragma unroll
              for (int jj = 0; jj < 2; ++jj) {  // two packed 16-byte units = 64 codes of the group
                const uint4 v = *reinterpret_cast<const uint4*>(src + swz128(t, (2 * gi + jj) * 16));
                *reinterpret_cast<uint4*>(dst + base + (4 * jj + 0) * 128u) = int4x8_to_bf16_scaled(v.x, s2);
                *reinterpret_cast<uint4*>(dst + base + (4 * jj + 1) * 128u) = int4x8_to_bf16_scaled(v.y, s2);
                *reinterpret_cast<uint4*>(dst + base + (4 * jj + 2) * 128u) = int4x8_to_bf16_scaled(v.z, s2);
                *reinterpret_cast<uint4*>(dst + base + (4 * jj + 3) * 128u) = int4x8_to_bf16_scaled(v.w, s2);
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&gfull[gs]);
          }
          if (++gs == kIGroups) {
            gs = 0;
            gph ^= 1u;
          }
        }
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&sempty[ss]);  // this warp has read the k-block's scales
        if (++ss == kISfStages) {
          ss = 0;
          sph ^= 1u;
        }
        named_bar(1, kIConvWarps * 32);  // every converter finished reading this packed stage
        if (t == 0 && ok) mbar_arrive(&pempty[st]);
        if (++st == kIStages) {
          st = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok) *abort_flag = 1;
  } else {
    setmaxnreg_dec<kIRegsLow>();
    if (warp == kIProducerWarp) {
      if (lane == 0) {
        // ------------------------------------------------------------ producer
        int st = 0;
        uint32_t ph = 0;
        int issued_phase[kIStages], sf_issued_phase[kISfStages];
        for (int s = 0; s < kIStages; ++s) issued_phase[s] = -1;
        for (int s = 0; s < kISfStages; ++s) sf_issued_phase[s] = -1;
        int ss = 0;
        uint32_t sph = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
          const int mt = tile / p.NT, n128 = tile % p.NT, n256 = n128 >> 1, nh = n128 & 1;
          for (int j = 0; j < nst; ++j) {
            if (*abort_flag || !wait_parity_bounded(&pempty[st], ph ^ 1u, kErrWaitGemm)) {
              ok = false;
              break;
            }
            uint8_t* sb = packed + st * kIPack;
            if (j < nlr) {
              const uint32_t cw = lr_chunk_width(r, j);
              const uint32_t bytes = kBM * cw * 2;  // T rows and L2 rows alike (128 each)
              mbar_arrive_expect_tx(&pfull[st], 2 * bytes);
              bulk_g2s(sb, p.t + static_cast<size_t>(mt) * kBM * r * 2 + static_cast<size_t>(kBM) * kLrChunk * 2 * j, bytes,
                       &pfull[st]);
              bulk_g2s(sb + kIPackA,
                       p.l2 + static_cast<size_t>(n256) * kBN * r * 2 + static_cast<size_t>(kBN) * kLrChunk * 2 * j + nh * bytes,
                       bytes, &pfull[st]);
            } else {
              const int kb = j - nlr;
              // the k-block's scales: A [128 rows][4 groups], B [4 groups][256 rows] (both halves)
              if (*abort_flag || !wait_parity_bounded(&sempty[ss], sph ^ 1u, kErrWaitGemm)) {
                ok = false;
                break;
              }
              uint8_t* sfb = sfring + ss * (kISfA + kISfB);
              mbar_arrive_expect_tx(&sfull[ss], kISfA + kISfB);
              bulk_g2s(sfb, p.a_sf + (static_cast<size_t>(mt) * p.KB + kb) * (kBM * 4), kISfA, &sfull[ss]);
              bulk_g2s(sfb + kISfA, p.b_sf + (static_cast<size_t>(n256) * p.KB + kb) * (kBN * 4), kISfB, &sfull[ss]);
              sf_issued_phase[ss] = static_cast<int>(sph);
              if (++ss == kISfStages) {
                ss = 0;
                sph ^= 1u;
              }
              mbar_arrive_expect_tx(&pfull[st], kIPack);
              bulk_g2s(sb, p.a_codes + codes_chunk_offset(mt, kb, p.KB, kBM), kIPackA, &pfull[st]);
              bulk_g2s(sb + kIPackA, p.b_codes + codes_chunk_offset(n256, kb, p.KB, kBN) + nh * kIPackB, kIPackB, &pfull[st]);
            }
            issued_phase[st] = static_cast<int>(ph);
            if (++st == kIStages) {
              st = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) {
          *abort_flag = 1;
          for (int s = 0; s < kIStages; ++s)
            if (issued_phase[s] >= 0) wait_parity_bounded(&pfull[s], static_cast<uint32_t>(issued_phase[s]), kErrWaitGemm);
          for (int s = 0; s < kISfStages; ++s)
            if (sf_issued_phase[s] >= 0)
              wait_parity_bounded(&sfull[s], static_cast<uint32_t>(sf_issued_phase[s]), kErrWaitGemm);
        }
      }
    } else if (warp == kIMmaWarp) {
      if (lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t id_bf16 = idesc_bf16(128, kIBN);
        int st = 0, gs = 0, local = 0;
        uint32_t ph = 0, gph = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++local) {
          const uint32_t b = static_cast<uint32_t>(local) & 1u;
          const uint32_t acc_t = tmem + b * kIBN;
          if (*abort_flag ||
              !wait_parity_bounded(&tempty[b], ((static_cast<uint32_t>(local) >> 1) & 1u) ^ 1u, kErrWaitGemm)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t accum = 0;
          // the up projection T L2 first, then every 64-element group, all into this accumulator
          for (int j = 0; j < nlr && ok; ++j) {
            if (*abort_flag || !wait_parity_bounded(&pfull[st], ph, kErrWaitGemm)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t cw = lr_chunk_width(r, j);
            const uint32_t sb = smem_u32(packed + st * kIPack);
            const uint64_t ad = smem_desc(sb, 128, cw * 16, kLayoutNone);
            const uint64_t bd = smem_desc(sb + kIPackA, 128, cw * 16, kLayoutNone);
            for (uint32_t ks = 0; ks < cw / 16; ++ks) {
              mma_bf16(acc_t, ad + 16 * ks, bd + 16 * ks, id_bf16, accum);
              accum = 1;
            }
            tc_commit(&pempty[st]);
            if (++st == kIStages) {
              st = 0;
              ph ^= 1u;
            }
          }
          for (int g = 0; g < ngrp && ok; ++g) {
            if (*abort_flag || !wait_parity_bounded(&gfull[gs], gph, kErrWaitGemm)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t gb = smem_u32(groups + gs * kIGrp);
            const uint64_t ad = smem_desc(gb, 128, 1024, kLayoutNone);
            const uint64_t bd = smem_desc(gb + kIGrpA, 128, 1024, kLayoutNone);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {  // 16 bf16 of K per MMA: 2 core matrices (256 bytes) on
              mma_bf16(acc_t, ad + 16 * ks, bd + 16 * ks, id_bf16, accum);
              accum = 1;
            }
            tc_commit(&gempty[gs]);
            if (++gs == kIGroups) {
              gs = 0;
              gph ^= 1u;
            }
          }
          if (ok) tc_commit(&tfull[b]);
        }
        if (!ok) {
          *abort_flag = 1;
          tc_commit(&tfull[0]);
        }
      }
    }
  }

  __syncthreads();
  if (warp == kIMmaWarp) {
    if (*abort_flag && lane == 0) {
      const unsigned long long t0 = globaltimer_ns();  // the abort-path commit lands within microseconds
      while (globaltimer_ns() - t0 < 2000000ull) {
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kIAcc * kIBN);
  }
}

static size_t gemm_int4_smem_bytes() {
  // ... staging, then 1 KB of barriers and flags, then the fused Q/K sum-of-squares slots (2 KB)
  return 1024 + kIStages * kIPack + kIGroups * kIGrp + kISfStages * (kISfA + kISfB) + kIStaging + 1024 + 2048;
}

static cudaError_t launch_gemm_int4(const GemmArgs& a, int num_sms, cudaStream_t stream) {
  GemmI4Params p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.rank = a.rank;
  p.KB = a.K / kBK;
  p.MT = 2 * ((a.M + 2 * kBM - 1) / (2 * kBM));
  p.NT = 2 * ((a.N + kBN - 1) / kBN);
  p.ldy = a.ldy;
  p.a_codes = a.a_codes;
  p.a_sf = reinterpret_cast<const float*>(a.a_sf);
  p.t = a.t;
  p.b_codes = a.b_codes;
  p.b_sf = reinterpret_cast<const float*>(a.b_sf);
  p.l2 = a.l2;
  p.bias = a.bias;
  p.Y = a.Y;
  p.qk_cols = a.qk_cols;
  p.gamma_q = a.gamma_q;
  p.gamma_k = a.gamma_k;
  p.rope = a.rope;
  p.eps = a.eps;
  const size_t smem = gemm_int4_smem_bytes();
  // setmaxnreg.inc waits until the block's pool (launch registers x threads) holds the epilogue's
  // share: refuse a build whose launch register count differs from the one the split assumes.
  static const cudaError_t regs_ok = [] {
    cudaFuncAttributes fa;
    const cudaError_t err = cudaFuncGetAttributes(&fa, gemm_int4_kernel);
    if (err != cudaSuccess) return err;
    return fa.numRegs == kIRegsLaunch && fa.maxThreadsPerBlock >= kIThreads ? cudaSuccess
                                                                            : cudaErrorInvalidConfiguration;
  }();
  if (regs_ok != cudaSuccess) return regs_ok;
  cudaError_t e = cudaFuncSetAttribute(gemm_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = p.MT * p.NT;
  const int grid = tiles < num_sms ? tiles : num_sms;
  gemm_int4_kernel<<<grid, kIThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

static size_t gemm_smem_bytes(int mode) {
  const size_t extra = mode >= 2 ? kGeluTblSize * 2 : (mode == 1 ? 2 * kQkvHeadDim * 4 : 0);
  return 1024 + static_cast<size_t>(gemm_stages(mode)) * kGStage + kGStaging + 256 + extra;
}

cudaError_t launch_gemm(const GemmArgs& a, int num_sms, cudaStream_t stream) {
  if (a.precision != 0) return launch_gemm_int4(a, num_sms, stream);
  GemmParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.rank = a.rank;
  p.KB = a.K / kBK;
  p.MT2 = (a.M + 2 * kBM - 1) / (2 * kBM);
  p.NT = (a.N + kBN - 1) / kBN;
  p.ldy = a.ldy;
  p.bias = a.bias;
  p.qk_cols = a.qk_cols;
  p.gamma_q = a.gamma_q;
  p.gamma_k = a.gamma_k;
  p.rope = a.rope;
  p.eps = a.eps;
  p.il_down = a.il_down;
  p.codes_down = a.codes_down;
  p.sf_down = a.sf_down;
  p.l1_down = a.l1_down;
  p.r_down = a.r_down;
  p.tpart = a.tpart;
  p.mlp_smax = a.mlp_smax;
  const size_t mt = static_cast<size_t>(p.MT2) * 2, nt = static_cast<size_t>(p.NT), KB = static_cast<size_t>(p.KB);
  const size_t rr = static_cast<size_t>(a.rank);
  GemmMaps maps;
  cudaError_t me;
  if ((me = make_rows_map(&maps.a, a.a_codes, mt * KB * kGA, kBoxA)) != cudaSuccess ||
      (me = make_rows_map(&maps.b, a.b_codes, nt * KB * kBN * kRowBytes, kBoxB)) != cudaSuccess ||
      (me = make_rows_map(&maps.sfa, a.a_sf, mt * KB * kGSfa, kBoxSfa)) != cudaSuccess ||
      (me = make_rows_map(&maps.sfb, a.b_sf, nt * KB * kGSfb, kBoxSfb)) != cudaSuccess ||
      (me = make_rows_map(&maps.t, a.t, rr ? mt * kBM * rr * 2 : 4096, kBoxLr)) != cudaSuccess ||
      (me = make_rows_map(&maps.l2, a.l2, rr ? nt * kBN * rr * 2 : 4096, kBoxLr)) != cudaSuccess)
    return me;
  {
    // Y: M rows of N bf16 (row stride ldy), written in boxes of 32 rows x 64 columns, 128-byte swizzle.
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return cudaErrorInitializationError;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.N), static_cast<cuuint64_t>(a.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.ldy) * 2};
    const cuuint32_t box[2] = {64, 32};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.Y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int mode = a.mlp ? 2 : (a.qk_cols > 0 ? 1 : (a.gelu ? 3 : 0));
  const size_t smem = gemm_smem_bytes(mode);
  auto kernel = mode == 3   ? gemm_nvfp4_kernel<3>
                : mode == 2 ? gemm_nvfp4_kernel<2>
                            : (mode == 1 ? gemm_nvfp4_kernel<1> : gemm_nvfp4_kernel<0>);
  // The epilogue warpgroups' setmaxnreg.inc waits until the block's pool holds their share, and
  // the pool is the launch's registers a thread x threads: refuse to launch a build whose count
  // differs from the one the split was sized for (the wait would never end).
  auto check_regs = [](const void* k) {
    cudaFuncAttributes fa;
    const cudaError_t err = cudaFuncGetAttributes(&fa, k);
    if (err != cudaSuccess) return err;
    return fa.numRegs == kGRegsLaunch && fa.maxThreadsPerBlock >= kGThreads ? cudaSuccess
                                                                            : cudaErrorInvalidConfiguration;
  };
  static const cudaError_t regs_plain = check_regs(reinterpret_cast<const void*>(gemm_nvfp4_kernel<0>));
  static const cudaError_t regs_qkv = check_regs(reinterpret_cast<const void*>(gemm_nvfp4_kernel<1>));
  static const cudaError_t regs_mlp = check_regs(reinterpret_cast<const void*>(gemm_nvfp4_kernel<2>));
  static const cudaError_t regs_gelu = check_regs(reinterpret_cast<const void*>(gemm_nvfp4_kernel<3>));
  cudaError_t e = mode == 3 ? regs_gelu : (mode == 2 ? regs_mlp : (mode == 1 ? regs_qkv : regs_plain));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = p.MT2 * p.NT;
  int pairs = num_sms / 2;
  if (pairs > tiles) pairs = tiles;
  if (mode == 2 && a.mlp_pairs != pairs) return cudaErrorInvalidValue;  // the T slots were sized for it
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, maps, p);
}

// ============================================================================ fused MLP: T of the down layer

// One thread per (row, T column): the partials of the pairs whose tile ranges met the row's 256-row
// block, both column halves, added in a fixed order (deterministic), rounded to bf16 once, stored
// in kernel 2's T layout.  A pair's range is [p tiles / npairs, (p + 1) tiles / npairs).
__global__ void __launch_bounds__(256) mlp_t_reduce_kernel(const float* part, int mpad, int smax, int r, int nt_up,
                                                           int npairs, int tiles, uint8_t* t) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= mpad * r) return;
  const int m = idx / r, i = idx - (idx / r) * r;
  const int m2 = m / (2 * kBM);
  auto pair_of = [&](long long tile) { return static_cast<int>(((tile + 1) * npairs - 1) / tiles); };
  const int p0 = pair_of(static_cast<long long>(m2) * nt_up), p1 = pair_of(static_cast<long long>(m2) * nt_up + nt_up - 1);
  const float* src = part + static_cast<size_t>(m) * 2 * smax * r + i;
  float sum = 0.0f;
  for (int h = 0; h < 2; ++h)
    for (int sl = 0; sl <= p1 - p0; ++sl) sum += src[static_cast<size_t>(h * smax + sl) * r];
  const __nv_bfloat16 b = __float2bfloat16_rn(sum);
  *reinterpret_cast<__nv_bfloat16*>(t + static_cast<size_t>(m >> 7) * kBM * r * 2 +
                                    lr_offset(static_cast<uint32_t>(m & 127), static_cast<uint32_t>(i), kBM, r)) = b;
}

cudaError_t launch_mlp_t_reduce(const float* part, int mpad, int smax, int r, int nt_up, int npairs, int tiles,
                                uint8_t* t, cudaStream_t stream) {
  const long long n = static_cast<long long>(mpad) * r;
  if (n <= 0) return cudaSuccess;
  mlp_t_reduce_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(part, mpad, smax, r, nt_up, npairs,
                                                                                  tiles, t);
  return cudaGetLastError();
}

// ============================================================================ fixed scratch

// Scratch of svdq_linear_forward_noalloc: a fixed array in the module's global memory, so that
// the forward can run without any device allocation.  Every device that loads the library holds
// it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(20) << 20;  // 20 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of the fixed scratch on the current device.  The host-side name of the array is
// only a stand-in, so the address is looked up (with the device current) once per device and
// context, and cached: a new context on the device (after cudaDeviceReset, say) loads the module
// again at another address, so a change of the current context triggers a fresh lookup.
using CtxGetCurrentFn = int (*)(void**);  // cuCtxGetCurrent(CUcontext*), reached through the runtime

static CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return static_cast<CtxGetCurrentFn>(nullptr);
  }();
  return fn;
}

cudaError_t noalloc_scratch_address(void** ptr) {
  static std::mutex mu;
  static void* addr[128] = {};
  static void* ctx_of[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  void* ctx = nullptr;
  CtxGetCurrentFn get_ctx = ctx_get_current();
  if (!get_ctx || get_ctx(&ctx) != 0) return cudaErrorInitializationError;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev] || ctx_of[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
    ctx_of[dev] = ctx;
  }
  *ptr = addr[dev];
  return cudaSuccess;
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

// The rotary table into the fused QKV epilogue's layout (rope_packed_index); rows past M, up to the
// next multiple of 32, repeat row M - 1.
__global__ void rope_pack_kernel(const float4* rope, int M, int rows, float4* packed) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;  // one float4 of the packed table
  if (i >= rows * (kQkvHeadDim / 4)) return;
  const int lane = i & 31, hf = (i >> 5) & 1, unit = (i >> 6) & (kQkvHeadDim / 8 - 1);
  const int row = (i / (32 * kQkvHeadDim / 4)) * 32 + lane;
  const int src = row < M ? row : M - 1;
  packed[i] = rope[static_cast<size_t>(src) * (kQkvHeadDim / 4) + 2 * unit + hf];
}

cudaError_t launch_rope_pack(const float* rope, int M, float* packed, cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  const int rows = (M + 31) / 32 * 32;
  const int n = rows * (kQkvHeadDim / 4);
  rope_pack_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(rope), M, rows, reinterpret_cast<float4*>(packed));
  return cudaGetLastError();
}

// The fused MLP epilogue's bf16 GELU on a list of bf16 inputs (a test hook).
// Eight values per thread through the epilogues' warp-collective path (every lane calls it).
__global__ void selftest_gelu_kernel(const uint16_t* in, uint16_t* out, int n) {
  __shared__ uint16_t tbl[kGeluTblSize];
  fill_gelu_table(tbl, threadIdx.x, blockDim.x);
  __syncthreads();
  const long long i0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t lo = i0 + 2 * q < n ? in[i0 + 2 * q] : 0u;
    const uint32_t hi = i0 + 2 * q + 1 < n ? in[i0 + 2 * q + 1] : 0u;
    w[q] = lo | (hi << 16);
  }
  gelu_bf16x8_warp(w, tbl);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (i0 + 2 * q < n) out[i0 + 2 * q] = static_cast<uint16_t>(w[q] & 0xFFFFu);
    if (i0 + 2 * q + 1 < n) out[i0 + 2 * q + 1] = static_cast<uint16_t>(w[q] >> 16);
  }
}

cudaError_t launch_selftest_gelu(const uint16_t* in, uint16_t* out, int n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  selftest_gelu_kernel<<<static_cast<unsigned>((n + 2047) / 2048), 256, 0, stream>>>(in, out, n);
  return cudaGetLastError();
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
