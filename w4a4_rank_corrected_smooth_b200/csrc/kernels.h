// Host launchers of the device kernels (defined in kernels.cu).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "layout.h"

namespace svdq {

struct QuantDownArgs {
  const uint16_t* X;       // M x K bf16, row stride ldx
  int M, K, ldx, rank, precision;
  const float* inv_lambda; // K
  const uint8_t* l1;       // tiled L1 (layout.h l1_offset)
  uint8_t* codes;          // workspace: tiled activation codes
  uint8_t* sf;             // workspace: tiled activation scales
  uint8_t* t;              // workspace: tiled bf16 T
  // 128-row-tile kernel only (when it splits K and rank > 0):
  float* part;             // workspace: fp32 partials of T per K slice
  unsigned long long* cnt; // workspace: one arrival counter per 128-row tile
  int split_cap;           // largest K split the partials have room for
};

struct GemmArgs {
  int M, N, K, rank, precision, ldy;
  const uint8_t* a_codes;
  const uint8_t* a_sf;
  const uint8_t* t;
  const uint8_t* b_codes;
  const uint8_t* b_sf;
  const uint8_t* l2;
  const float* bias;  // N (padded to a multiple of 256)
  uint16_t* Y;
  // Fused RMS normalization of Q and K and rotary embedding (NVFP4 only; qk_cols = 0: off).
  // Columns [0, qk_cols) are the Q heads then the K heads, kQkvHeadDim channels each.
  int qk_cols = 0;
  const float* gamma_q = nullptr;  // kQkvHeadDim
  const float* gamma_k = nullptr;  // kQkvHeadDim
  const float* rope = nullptr;     // M rows of kQkvHeadDim / 2 (cos, sin) pairs
  float eps = 0.0f;
  // Fused MLP pair (NVFP4 only; mlp = false: off): instead of Y, the epilogue writes the down
  // layer's activation codes and scales of GELU(Y) and the fp32 partials of its T.
  bool mlp = false;
  const float* il_down = nullptr;  // N (= the down layer's K): the down layer's 1/lambda
  uint8_t* codes_down = nullptr;   // the down layer's workspace: codes, scales
  uint8_t* sf_down = nullptr;
  const uint8_t* l1_down = nullptr;  // the down layer's L1 (kernel 1's B-operand layout)
  int r_down = 0;                  // 0, 16 or 32
  float* tpart = nullptr;          // [M padded][2 column halves][mlp_smax][r_down] fp32 partials of T
  int mlp_smax = 0;                // slots per (row, column half): pairs meeting one 256-row block
  int mlp_pairs = 0;               // CTA pairs of the up layer's kernel 2 (the slots assume it)
  // GELU output (NVFP4 only): Y = GELU(bf16(acc + bias)), rounded to bf16 (the first half of an MLP
  // whose hidden activation goes through HBM to the next layer's forward).
  bool gelu = false;
};

// The down layer's T from the fused MLP epilogue's partials (see the kernel), written in kernel 2's
// T layout.
cudaError_t launch_mlp_t_reduce(const float* part, int mpad, int smax, int r, int nt_up, int npairs, int tiles,
                                uint8_t* t, cudaStream_t stream);

// Head size of the fused QKV operator: one epilogue thread holds one row of one head.
constexpr int kQkvHeadDim = 128;

// The fused QKV operator's rotary table: for each block of 32 rows, each 16-byte half (hf) of each
// group of 4 (cos, sin) pairs (unit) of the 32 rows side by side, so that a warp whose lanes hold
// the block's rows reads 512 contiguous bytes per unit half.  Index of the float4 in floats:
SVDQ_HD constexpr size_t rope_packed_index(int row, int unit, int hf) {
  return ((static_cast<size_t>(row >> 5) * (kQkvHeadDim / 8) + static_cast<size_t>(unit)) * 2 + hf) * 128 +
         static_cast<size_t>(row & 31) * 4;
}
// Bytes of the packed table for M rows (rounded up to a multiple of 32).
constexpr size_t rope_packed_bytes(int M) { return static_cast<size_t>((M + 31) / 32 * 32) * kQkvHeadDim * 4; }
cudaError_t launch_rope_pack(const float* rope, int M, float* packed, cudaStream_t stream);

// W4A16 layer (4-bit weights in canonical row-major layout, 16-bit activations).
struct W4A16Args {
  const uint16_t* X;        // M x K bf16, row stride ldx
  int M, K, ldx, N, ldy;
  const float* inv_lambda;  // K
  const uint8_t* codes;     // N x K/2 (element 2i in the low nibble of byte i)
  const float* scales;      // N x K/64 fp32
  const float* bias;        // N (fp32)
  uint16_t* Y;              // M x N bf16, row stride ldy
};

// Returns a cudaError_t of the launch (cudaSuccess when the launch was queued).
cudaError_t launch_quant_down(const QuantDownArgs& a, int num_sms, cudaStream_t stream);
cudaError_t launch_gemm(const GemmArgs& a, int num_sms, cudaStream_t stream);
cudaError_t launch_w4a16(const W4A16Args& a, int num_sms, cudaStream_t stream);
// Largest K the W4A16 kernel accepts (x_hat rows are staged in shared memory).
constexpr int kW4A16MaxK = 49152;
cudaError_t launch_selftest_wait(int spin_limit, cudaStream_t stream);
cudaError_t launch_selftest_gelu(const uint16_t* in, uint16_t* out, int n, cudaStream_t stream);
cudaError_t read_and_clear_device_error(unsigned int* value, cudaStream_t stream);
cudaError_t read_and_clear_w4a16_error(unsigned int* value, cudaStream_t stream);

// Fixed-size scratch in the library's device module (for the allocation-free forward).
size_t noalloc_scratch_bytes();
cudaError_t noalloc_scratch_address(void** ptr);

}  // namespace svdq
