// Host-side prepare of an SVDQuant layer: canonical operands and their tiled device images.
#pragma once
#include <cstdint>
#include <vector>

namespace svdq {

struct CanonicalLayer {
  int N = 0, K = 0, rank = 0, precision = 0;
  std::vector<float> inv_lambda;        // K
  std::vector<uint8_t> codes_w;         // N x K/2
  std::vector<uint8_t> scales_nvfp4;    // N x K/16
  std::vector<float> scales_int4;       // N x K/64
  std::vector<uint16_t> L1;             // K x r bf16
  std::vector<uint16_t> L2;             // r x N bf16
  std::vector<uint16_t> bias;           // N bf16
  std::vector<double> sigma;            // r
  std::vector<float> R;                 // N x K residual (fp32)
};

struct DeviceImages {
  int n_tiles = 0;
  std::vector<uint8_t> codes, sf, l1, l2;
  std::vector<float> bias;
};

float bf16_bits_to_float(uint16_t b);
uint16_t float_to_bf16_bits(float f);
uint8_t encode_ue4m3(float s);
float decode_ue4m3(uint8_t c);
uint8_t encode_e2m1(float q);

void quantize_rows_host(const float* V, int rows, int K, int precision, uint8_t* codes, void* scales);

void randomized_svd(const double* B, int N, int K, int r, int iters, uint64_t seed, std::vector<double>& U,
                    std::vector<double>& sigma, std::vector<double>& V);

int prepare_canonical(const uint16_t* W_bf16, int N, int K, const uint16_t* bias_bf16, const float* act_absmax,
                      int precision, int rank, float alpha, int iters, uint64_t seed, CanonicalLayer& out);

void pack_device_layouts(const CanonicalLayer& c, DeviceImages& d);

// W4A16: codes and scales in the warp-level MMA's fragment order (see host_prepare.cpp).
void pack_w4a16_fragments(const CanonicalLayer& c, DeviceImages& d);

}  // namespace svdq
