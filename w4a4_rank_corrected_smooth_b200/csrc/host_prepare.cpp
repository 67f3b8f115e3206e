// Offline prepare of an SVDQuant layer on the host (SVDQuant model card, "Quantization
// Method -- SVDQuant", stages 2-3): smoothing factors, smoothed weight, rank-r SVD split by
// randomized subspace iteration, fp32 residual, and the residual's 4-bit group quantizer.
// Also the packers that turn canonical operands into the tiled device layouts of layout.h.
#include "host_prepare.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <random>
#include <thread>
#include <vector>

#include "layout.h"

namespace svdq {

// ------------------------------------------------------------------ bf16

float bf16_bits_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint16_t float_to_bf16_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint32_t lsb = (u >> 16) & 1u;
  return static_cast<uint16_t>((u + 0x7FFFu + lsb) >> 16);  // round to nearest even (finite inputs)
}

// ------------------------------------------------------------------ codecs

// UE4M3 code of s >= 0: round to nearest even, saturate at 448 (code 0x7E).
uint8_t encode_ue4m3(float s) {
  if (!(s > 0.0f)) return 0;
  if (s >= 448.0f) return 0x7E;
  if (s < 0.015625f) {  // below 2^-6: subnormal, step 2^-9
    const float m = std::nearbyint(s * 512.0f);  // exact scaling, ties to even
    return static_cast<uint8_t>(m);           // m == 8 is code 0x08 = 2^-6
  }
  int e2;
  const float f = std::frexp(s, &e2);  // s = f * 2^e2, f in [0.5, 1)
  int ebias = (e2 - 1) + 7;
  float mant = std::nearbyint((2.0f * f - 1.0f) * 8.0f);  // exact, ties to even
  if (mant >= 8.0f) {
    mant = 0.0f;
    ebias += 1;
  }
  const int code = (ebias << 3) | static_cast<int>(mant);
  return static_cast<uint8_t>(code > 0x7E ? 0x7E : code);
}

float decode_ue4m3(uint8_t c) {
  const int e = (c >> 3) & 0xF, m = c & 7;
  if (e == 0) return std::ldexp(static_cast<float>(m), -9);
  return std::ldexp(1.0f + static_cast<float>(m) / 8.0f, e - 7);
}

// E2M1 nibble of q: the magnitude code counts the rounding thresholds that |q| passes; a
// threshold exactly hit rounds toward the even code (0.25->0, 0.75->1.0, 1.25->1.0,
// 1.75->2.0, 2.5->2.0, 3.5->4.0, 5->4.0); above 5 saturates to 6.  Sign from the sign bit.
uint8_t encode_e2m1(float q) {
  const float a = std::fabs(q);
  const int mag = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
  return static_cast<uint8_t>(mag | (std::signbit(q) ? 8 : 0));
}

static void quantize_row_nvfp4(const float* v, int K, uint8_t* codes, uint8_t* scales) {
  for (int g = 0; g < K / 16; ++g) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) amax = std::max(amax, std::fabs(v[g * 16 + i]));
    const float s = amax / 6.0f;
    const uint8_t sc = encode_ue4m3(s);
    const float sd = decode_ue4m3(sc);
    scales[g] = sc;
    for (int i = 0; i < 16; i += 2) {
      uint8_t lo = 0, hi = 0;
      if (sd != 0.0f) {
        lo = encode_e2m1(v[g * 16 + i] / sd);
        hi = encode_e2m1(v[g * 16 + i + 1] / sd);
      }
      codes[(g * 16 + i) / 2] = static_cast<uint8_t>(lo | (hi << 4));
    }
  }
}

static void quantize_row_int4(const float* v, int K, uint8_t* codes, float* scales) {
  for (int g = 0; g < K / 64; ++g) {
    float amax = 0.0f;
    for (int i = 0; i < 64; ++i) amax = std::max(amax, std::fabs(v[g * 64 + i]));
    const float s = amax / 7.0f;
    scales[g] = s;
    for (int i = 0; i < 64; i += 2) {
      int q[2] = {0, 0};
      if (s != 0.0f) {
        for (int t = 0; t < 2; ++t) {
          float x = std::nearbyint(v[g * 64 + i + t] / s);
          x = std::min(7.0f, std::max(-8.0f, x));
          q[t] = static_cast<int>(x);
        }
      }
      codes[(g * 64 + i) / 2] = static_cast<uint8_t>((q[0] & 0xF) | ((q[1] & 0xF) << 4));
    }
  }
}

template <class F>
static void parallel_for(int n, F&& f) {
  int nt = static_cast<int>(std::thread::hardware_concurrency());
  nt = std::max(1, std::min(nt, 64));
  nt = std::min(nt, std::max(1, n));
  if (nt == 1) {
    for (int i = 0; i < n; ++i) f(i, 0);
    return;
  }
  std::vector<std::thread> th;
  th.reserve(nt);
  for (int t = 0; t < nt; ++t) {
    th.emplace_back([&, t] {
      const int a = static_cast<int>(static_cast<long long>(n) * t / nt);
      const int b = static_cast<int>(static_cast<long long>(n) * (t + 1) / nt);
      for (int i = a; i < b; ++i) f(i, t);
    });
  }
  for (auto& x : th) x.join();
}

static int num_threads_for(int n) {
  int nt = static_cast<int>(std::thread::hardware_concurrency());
  nt = std::max(1, std::min(nt, 64));
  return std::min(nt, std::max(1, n));
}

void quantize_rows_host(const float* V, int rows, int K, int precision, uint8_t* codes, void* scales) {
  parallel_for(rows, [&](int r, int) {
    const float* v = V + static_cast<size_t>(r) * K;
    uint8_t* c = codes + static_cast<size_t>(r) * (K / 2);
    if (precision == 0) {
      quantize_row_nvfp4(v, K, c, static_cast<uint8_t*>(scales) + static_cast<size_t>(r) * (K / 16));
    } else {
      quantize_row_int4(v, K, c, static_cast<float*>(scales) + static_cast<size_t>(r) * (K / 64));
    }
  });
}

// ------------------------------------------------------------------ dense helpers (fp64)

// Y[N x l] = B[N x K] * Z[K x l]   (all row-major)
static void mul_B_Z(const double* B, int N, int K, const double* Z, int l, double* Y) {
  parallel_for(N, [&](int n, int) {
    const double* b = B + static_cast<size_t>(n) * K;
    double* y = Y + static_cast<size_t>(n) * l;
    for (int j = 0; j < l; ++j) y[j] = 0.0;
    for (int k = 0; k < K; ++k) {
      const double bk = b[k];
      const double* z = Z + static_cast<size_t>(k) * l;
      for (int j = 0; j < l; ++j) y[j] += bk * z[j];
    }
  });
}

// Z[K x l] = B^T[K x N] * Q[N x l]: per-thread partial sums over row ranges, then a fixed-order reduction.
static void mul_Bt_Q(const double* B, int N, int K, const double* Q, int l, double* Z) {
  const int nt = std::min(16, num_threads_for(N / 64 + 1));
  std::vector<std::vector<double>> part(nt, std::vector<double>(static_cast<size_t>(K) * l, 0.0));
  std::vector<std::thread> th;
  for (int t = 0; t < nt; ++t) {
    th.emplace_back([&, t] {
      const int a = static_cast<int>(static_cast<long long>(N) * t / nt);
      const int b = static_cast<int>(static_cast<long long>(N) * (t + 1) / nt);
      double* z = part[t].data();
      for (int n = a; n < b; ++n) {
        const double* brow = B + static_cast<size_t>(n) * K;
        const double* q = Q + static_cast<size_t>(n) * l;
        for (int k = 0; k < K; ++k) {
          const double bk = brow[k];
          double* zk = z + static_cast<size_t>(k) * l;
          for (int j = 0; j < l; ++j) zk[j] += bk * q[j];
        }
      }
    });
  }
  for (auto& x : th) x.join();
  parallel_for(K, [&](int k, int) {
    double* zk = Z + static_cast<size_t>(k) * l;
    for (int j = 0; j < l; ++j) {
      double s = 0.0;
      for (int t = 0; t < nt; ++t) s += part[t][static_cast<size_t>(k) * l + j];
      zk[j] = s;
    }
  });
}

// Orthonormalise the l columns of Y (n x l, row-major) in place: modified Gram-Schmidt, twice.
static void orthonormalize_columns(double* Y, int n, int l) {
  for (int pass = 0; pass < 2; ++pass) {
    for (int j = 0; j < l; ++j) {
      for (int i = 0; i < j; ++i) {
        double d = 0.0;
        for (int r = 0; r < n; ++r) d += Y[static_cast<size_t>(r) * l + i] * Y[static_cast<size_t>(r) * l + j];
        for (int r = 0; r < n; ++r) Y[static_cast<size_t>(r) * l + j] -= d * Y[static_cast<size_t>(r) * l + i];
      }
      double nrm = 0.0;
      for (int r = 0; r < n; ++r) nrm += Y[static_cast<size_t>(r) * l + j] * Y[static_cast<size_t>(r) * l + j];
      nrm = std::sqrt(nrm);
      const double inv = nrm > 0 ? 1.0 / nrm : 0.0;
      for (int r = 0; r < n; ++r) Y[static_cast<size_t>(r) * l + j] *= inv;
    }
  }
}

// One-sided (Hestenes) Jacobi SVD of a tall G (m x l) stored column by column (column j at
// G + j*m): on return the columns of G are U*Sigma (mutually orthogonal) and V (l x l,
// row-major) holds the accumulated rotations, G0 = (U Sigma) V^T.
static void one_sided_jacobi(double* G, int m, int l, double* V) {
  for (int i = 0; i < l; ++i)
    for (int j = 0; j < l; ++j) V[i * l + j] = (i == j) ? 1.0 : 0.0;
  for (int sweep = 0; sweep < 60; ++sweep) {
    bool rotated = false;
    for (int p = 0; p < l - 1; ++p) {
      for (int q = p + 1; q < l; ++q) {
        double* gp = G + static_cast<size_t>(p) * m;
        double* gq = G + static_cast<size_t>(q) * m;
        double a = 0.0, b = 0.0, c = 0.0;
        for (int r = 0; r < m; ++r) {
          a += gp[r] * gp[r];
          b += gq[r] * gq[r];
          c += gp[r] * gq[r];
        }
        if (c == 0.0 || std::fabs(c) <= 1e-15 * std::sqrt(a * b)) continue;
        rotated = true;
        const double zeta = (b - a) / (2.0 * c);
        const double t = (zeta >= 0 ? 1.0 : -1.0) / (std::fabs(zeta) + std::sqrt(1.0 + zeta * zeta));
        const double cs = 1.0 / std::sqrt(1.0 + t * t), sn = cs * t;
        for (int r = 0; r < m; ++r) {
          const double x = gp[r], y = gq[r];
          gp[r] = cs * x - sn * y;
          gq[r] = sn * x + cs * y;
        }
        for (int r = 0; r < l; ++r) {
          double& vp = V[r * l + p];
          double& vq = V[r * l + q];
          const double x = vp, y = vq;
          vp = cs * x - sn * y;
          vq = sn * x + cs * y;
        }
      }
    }
    if (!rotated) break;
  }
}

// Top-r SVD of B (N x K, row-major, B = W_hat in nn.Linear layout) by randomized subspace
// iteration (Halko, Martinsson and Tropp 2011, Alg. 4.4) with a one-sided Jacobi SVD of the
// projected matrix.  Outputs, in the K x N orientation of the formula W_hat = U S V^T:
// U (K x r), sigma (r), V (N x r), all row-major fp64.
void randomized_svd(const double* B, int N, int K, int r, int iters, uint64_t seed, std::vector<double>& U,
                    std::vector<double>& sigma, std::vector<double>& V) {
  const int l = std::min(std::min(N, K), r + 16);
  std::vector<double> Om(static_cast<size_t>(K) * l);
  {
    std::mt19937_64 gen(seed);
    std::normal_distribution<double> nd(0.0, 1.0);
    for (auto& x : Om) x = nd(gen);
  }
  std::vector<double> Y(static_cast<size_t>(N) * l), Z(static_cast<size_t>(K) * l);
  mul_B_Z(B, N, K, Om.data(), l, Y.data());
  orthonormalize_columns(Y.data(), N, l);
  for (int it = 0; it < iters; ++it) {
    mul_Bt_Q(B, N, K, Y.data(), l, Z.data());
    orthonormalize_columns(Z.data(), K, l);
    mul_B_Z(B, N, K, Z.data(), l, Y.data());
    orthonormalize_columns(Y.data(), N, l);
  }
  // C^T = B^T Q  (K x l); C = Q^T B is the projection of B onto span(Q).
  mul_Bt_Q(B, N, K, Y.data(), l, Z.data());
  std::vector<double> Gc(static_cast<size_t>(K) * l);  // column-major copy of C^T
  for (int k = 0; k < K; ++k)
    for (int j = 0; j < l; ++j) Gc[static_cast<size_t>(j) * K + k] = Z[static_cast<size_t>(k) * l + j];
  std::vector<double> Vg(static_cast<size_t>(l) * l);
  one_sided_jacobi(Gc.data(), K, l, Vg.data());
  // Gc = U_c Sigma (columns), C^T = U_c Sigma Vg^T  =>  B ~= Q C = (Q Vg) Sigma U_c^T.
  std::vector<double> norms(l);
  for (int j = 0; j < l; ++j) {
    double s = 0.0;
    for (int k = 0; k < K; ++k) s += Gc[static_cast<size_t>(j) * K + k] * Gc[static_cast<size_t>(j) * K + k];
    norms[j] = std::sqrt(s);
  }
  std::vector<int> order(l);
  for (int j = 0; j < l; ++j) order[j] = j;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return norms[a] > norms[b]; });
  U.assign(static_cast<size_t>(K) * r, 0.0);
  V.assign(static_cast<size_t>(N) * r, 0.0);
  sigma.assign(r, 0.0);
  for (int i = 0; i < r; ++i) {
    const int j = order[i];
    const double s = norms[j];
    sigma[i] = s;
    const double inv = s > 0 ? 1.0 / s : 0.0;
    for (int k = 0; k < K; ++k) U[static_cast<size_t>(k) * r + i] = Gc[static_cast<size_t>(j) * K + k] * inv;
    for (int n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int t = 0; t < l; ++t) acc += Y[static_cast<size_t>(n) * l + t] * Vg[static_cast<size_t>(t) * l + j];
      V[static_cast<size_t>(n) * r + i] = acc;
    }
    // Sign convention: the largest-magnitude entry of each U column is positive (first on ties).
    int arg = 0;
    double best = -1.0;
    for (int k = 0; k < K; ++k) {
      const double a = std::fabs(U[static_cast<size_t>(k) * r + i]);
      if (a > best) {
        best = a;
        arg = k;
      }
    }
    if (U[static_cast<size_t>(arg) * r + i] < 0) {
      for (int k = 0; k < K; ++k) U[static_cast<size_t>(k) * r + i] = -U[static_cast<size_t>(k) * r + i];
      for (int n = 0; n < N; ++n) V[static_cast<size_t>(n) * r + i] = -V[static_cast<size_t>(n) * r + i];
    }
  }
}

// ------------------------------------------------------------------ prepare

int prepare_canonical(const uint16_t* W_bf16, int N, int K, const uint16_t* bias_bf16, const float* act_absmax,
                      int precision, int rank, float alpha, int iters, uint64_t seed, CanonicalLayer& out) {
  out.N = N;
  out.K = K;
  out.rank = rank;
  out.precision = precision;
  const size_t NK = static_cast<size_t>(N) * K;
  // Smoothing factors (stage 2): lam_k = a_k^alpha w_k^(alpha-1); 1 when a_k or w_k is 0.
  std::vector<double> wmax(K, 0.0);
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k)
      wmax[k] = std::max(wmax[k], std::fabs(static_cast<double>(bf16_bits_to_float(W_bf16[static_cast<size_t>(n) * K + k]))));
  std::vector<double> lam(K, 1.0);
  out.inv_lambda.resize(K);
  for (int k = 0; k < K; ++k) {
    const double a = static_cast<double>(act_absmax[k]);
    if (a > 0 && wmax[k] > 0) {
      lam[k] = (alpha == 0.5f) ? std::sqrt(a / wmax[k])
                               : std::pow(a, static_cast<double>(alpha)) * std::pow(wmax[k], static_cast<double>(alpha) - 1.0);
    }
    out.inv_lambda[k] = static_cast<float>(1.0 / lam[k]);
  }
  // Smoothed weight W_hat = W diag(lam) (nn.Linear layout N x K), fp64.
  std::vector<double> Wh(NK);
  parallel_for(N, [&](int n, int) {
    for (int k = 0; k < K; ++k)
      Wh[static_cast<size_t>(n) * K + k] =
          static_cast<double>(bf16_bits_to_float(W_bf16[static_cast<size_t>(n) * K + k])) * lam[k];
  });
  out.R.assign(NK, 0.0f);
  out.L1.assign(static_cast<size_t>(K) * rank, 0);
  out.L2.assign(static_cast<size_t>(rank) * N, 0);
  out.sigma.assign(rank, 0.0);
  if (rank > 0) {
    std::vector<double> U, sig, V;
    randomized_svd(Wh.data(), N, K, rank, iters, seed, U, sig, V);
    out.sigma = sig;
    // L1 = U sqrt(S) (K x r); L2 = sqrt(S) V^T (r x N), bf16.
    for (int k = 0; k < K; ++k)
      for (int i = 0; i < rank; ++i)
        out.L1[static_cast<size_t>(k) * rank + i] =
            float_to_bf16_bits(static_cast<float>(U[static_cast<size_t>(k) * rank + i] * std::sqrt(sig[i])));
    for (int i = 0; i < rank; ++i)
      for (int n = 0; n < N; ++n)
        out.L2[static_cast<size_t>(i) * N + n] =
            float_to_bf16_bits(static_cast<float>(std::sqrt(sig[i]) * V[static_cast<size_t>(n) * rank + i]));
    // Residual R = W_hat - U S V^T with the fp64 factors, stored fp32 (N x K).
    parallel_for(N, [&](int n, int) {
      for (int k = 0; k < K; ++k) {
        double low = 0.0;
        for (int i = 0; i < rank; ++i)
          low += U[static_cast<size_t>(k) * rank + i] * sig[i] * V[static_cast<size_t>(n) * rank + i];
        out.R[static_cast<size_t>(n) * K + k] = static_cast<float>(Wh[static_cast<size_t>(n) * K + k] - low);
      }
    });
  } else {
    for (size_t i = 0; i < NK; ++i) out.R[i] = static_cast<float>(Wh[i]);
  }
  out.codes_w.assign(NK / 2, 0);
  if (precision == 0) {
    out.scales_nvfp4.assign(NK / 16, 0);
    quantize_rows_host(out.R.data(), N, K, 0, out.codes_w.data(), out.scales_nvfp4.data());
  } else {
    out.scales_int4.assign(NK / 64, 0.0f);
    quantize_rows_host(out.R.data(), N, K, 1, out.codes_w.data(), out.scales_int4.data());
  }
  out.bias.assign(N, 0);
  if (bias_bf16) std::memcpy(out.bias.data(), bias_bf16, sizeof(uint16_t) * N);
  return 0;
}

// ------------------------------------------------------------------ device layouts

void pack_device_layouts(const CanonicalLayer& c, DeviceImages& d) {
  const int N = c.N, K = c.K, r = c.rank;
  const int KB = K / kBK;
  const int NT = (N + kBN - 1) / kBN;
  const size_t npad = static_cast<size_t>(NT) * kBN;
  d.n_tiles = NT;
  // Weight codes: per (n-tile, k-block) a 256-row x 128-byte swizzled chunk; padded rows are 0.
  d.codes.assign(npad * K / 2, 0);
  parallel_for(N, [&](int n, int) {
    const int nt = n / kBN, row = n % kBN;
    for (int kb = 0; kb < KB; ++kb) {
      uint8_t* chunk = d.codes.data() + codes_chunk_offset(nt, kb, KB, kBN);
      const uint8_t* src = c.codes_w.data() + static_cast<size_t>(n) * (K / 2) + static_cast<size_t>(kb) * kRowBytes;
      for (int b = 0; b < kRowBytes; ++b) chunk[swz128(row, b)] = src[b];
    }
  });
  // Weight scales.
  d.sf.assign(npad * K / kBK * kSfBytesPerRowKb, 0);
  parallel_for(N, [&](int n, int) {
    const int nt = n / kBN, row = n % kBN;
    for (int kb = 0; kb < KB; ++kb) {
      uint8_t* chunk = d.sf.data() + sf_chunk_offset(nt, kb, KB, kBN);
      if (c.precision == 0) {
        for (int j = 0; j < 16; ++j)
          chunk[sf_nvfp4_offset(row, j, kBN)] = c.scales_nvfp4[static_cast<size_t>(n) * (K / 16) + kb * 16 + j];
      } else {
        float* f = reinterpret_cast<float*>(chunk);
        for (int g = 0; g < 4; ++g) f[sf_int4_b_index(row, g)] = c.scales_int4[static_cast<size_t>(n) * (K / 64) + kb * 4 + g];
      }
    }
  });
  // L1 for the down projection (per 64-k chunk: r rows x 128 bytes, swizzled).
  d.l1.assign(static_cast<size_t>(K) * r * 2, 0);
  for (int k = 0; k < K; ++k)
    for (int i = 0; i < r; ++i) {
      const uint16_t v = c.L1[static_cast<size_t>(k) * r + i];
      std::memcpy(d.l1.data() + l1_offset(k, i, r), &v, 2);
    }
  // L2 for the up projection: per n-tile, 256 rows (n) x r columns, core-matrix layout.
  d.l2.assign(npad * r * 2, 0);
  for (int n = 0; n < N; ++n) {
    const int nt = n / kBN, row = n % kBN;
    uint8_t* tile = d.l2.data() + static_cast<size_t>(nt) * kBN * r * 2;
    for (int i = 0; i < r; ++i) {
      const uint16_t v = c.L2[static_cast<size_t>(i) * N + n];
      std::memcpy(tile + lr_offset(row, i, kBN, r), &v, 2);
    }
  }
  d.bias.assign(npad, 0.0f);
  for (int n = 0; n < N; ++n) d.bias[n] = bf16_bits_to_float(c.bias[n]);
}

// W4A16 weights in the order the warp-level bf16 MMA (m16n8k16) takes its A operand from
// registers: per block b of 16 rows and group g of 64 elements along K, 32 lanes x 16 bytes.
// Lane l (row i = l / 4, pair t = l % 4) holds four 32-bit words, one per 16-deep k-step s;
// nibble j of word s (j = 0..3) and nibble j + 4 are the two elements of fragment register j:
//   j = 0: row i,     k = 64 g + 16 s + 2 t + {0, 1}
//   j = 1: row i + 8, k = 64 g + 16 s + 2 t + {0, 1}
//   j = 2: row i,     k = 64 g + 16 s + 8 + 2 t + {0, 1}
//   j = 3: row i + 8, k = 64 g + 16 s + 8 + 2 t + {0, 1}
// (the element with the lower k in nibble j, the other in nibble j + 4).  Scales: per (b, g)
// eight pairs (s[16 b + i], s[16 b + i + 8]) as fp32.  Rows past N stay 0 up to the padded N.
void pack_w4a16_fragments(const CanonicalLayer& c, DeviceImages& d) {
  const int N = c.N, K = c.K, G = K / 64;
  const size_t npad = static_cast<size_t>((N + kBN - 1) / kBN) * kBN;
  const int NB = static_cast<int>(npad / 16);
  d.codes.assign(npad * K / 2, 0);
  d.sf.assign(npad * static_cast<size_t>(G) * sizeof(float), 0);
  auto nib = [&](int n, int k) -> uint32_t {
    if (n >= N) return 0;
    const uint8_t byte = c.codes_w[static_cast<size_t>(n) * (K / 2) + k / 2];
    return (k & 1) ? (byte >> 4) : (byte & 0xFu);
  };
  parallel_for(NB, [&](int b, int) {
    for (int g = 0; g < G; ++g) {
      uint8_t* dst = d.codes.data() + ((static_cast<size_t>(b) * G + g) * 32) * 16;
      for (int l = 0; l < 32; ++l) {
        const int i = l / 4, t = l % 4;
        for (int s = 0; s < 4; ++s) {
          uint32_t word = 0;
          for (int j = 0; j < 4; ++j) {
            const int n = 16 * b + i + 8 * (j & 1);
            const int k = 64 * g + 16 * s + 8 * (j >> 1) + 2 * t;
            word |= nib(n, k) << (4 * j);
            word |= nib(n, k + 1) << (4 * (j + 4));
          }
          std::memcpy(dst + 16 * l + 4 * s, &word, 4);
        }
      }
      float* sdst = reinterpret_cast<float*>(d.sf.data()) + (static_cast<size_t>(b) * G + g) * 16;
      for (int i = 0; i < 8; ++i)
        for (int h = 0; h < 2; ++h) {
          const int n = 16 * b + i + 8 * h;
          sdst[2 * i + h] = n < N ? c.scales_int4[static_cast<size_t>(n) * G + g] : 0.0f;
        }
    }
  });
}

}  // namespace svdq
