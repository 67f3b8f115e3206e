// Host launchers of the device kernels (defined in kernels.cu).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace svdq {

struct QuantDownArgs {
  const uint16_t* X;       // M x K bf16, row stride ldx
  int M, K, ldx, rank, precision;
  const float* inv_lambda; // K
  const uint8_t* l1;       // tiled L1 (layout.h l1_offset)
  uint8_t* codes;          // workspace: tiled activation codes
  uint8_t* sf;             // workspace: tiled activation scales
  uint8_t* t;              // workspace: tiled bf16 T
  float* part;             // workspace: fp32 partials of T per K slice (split_cap > 1 and rank > 0)
  unsigned long long* cnt; // workspace: one arrival counter per 128-row tile (same condition)
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
};

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
cudaError_t read_and_clear_device_error(unsigned int* value, cudaStream_t stream);

// Fixed-size scratch in the library's device module (for the allocation-free forward).
size_t noalloc_scratch_bytes();
cudaError_t noalloc_scratch_address(void** ptr);

}  // namespace svdq
