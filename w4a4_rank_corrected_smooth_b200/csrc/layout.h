// Tiled device layouts shared by the host packer and the two kernels.
//
// All 4-bit operands are stored so that one k-block (256 elements along K = 128 bytes per row)
// of one tile is a contiguous chunk whose bytes are exactly the shared-memory image the
// tcgen05 MMA reads: K-major, 128-byte swizzle (16-byte unit u of row r sits at unit
// u ^ (r % 8)), 8-row atoms of 1024 bytes.  A whole stage is then one 1-D bulk copy.
#pragma once
#include <cstddef>
#include <cstdint>

#if defined(__CUDACC__)
#define SVDQ_HD __host__ __device__
#else
#define SVDQ_HD
#endif

namespace svdq {

constexpr int kBM = 128;          // rows of an activation (M) tile
constexpr int kBN = 256;          // rows of a weight (N) tile
constexpr int kBK = 256;          // elements of one k-block along K
constexpr int kRowBytes = 128;    // bytes of one row of one k-block of 4-bit codes
constexpr int kLrChunk = 64;      // low-rank columns per pipeline stage
constexpr int kMaxRank = 128;
constexpr int kSfBytesPerRowKb = 16;  // scale bytes per row per k-block (NVFP4: 16 x UE4M3; INT4: 4 x fp32)

SVDQ_HD constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Byte offset of (row, byte) inside a swizzled 128-byte-row chunk.
SVDQ_HD constexpr uint32_t swz128(uint32_t row, uint32_t byte) {
  return row * 128u + ((((byte >> 4) ^ (row & 7u)) << 4) | (byte & 15u));
}

// Codes chunk of (tile, kb): rows_per_tile x 128 bytes.
SVDQ_HD constexpr size_t codes_chunk_offset(size_t tile, size_t kb, size_t KB, size_t rows_per_tile) {
  return (tile * KB + kb) * rows_per_tile * kRowBytes;
}

// NVFP4 scale factors of one (tile, kb): for each of the 4 MMAs of the k-block (kk), one
// 512-byte block per 128 rows laid out for tcgen05.cp 32x128b.warpx4: row r, scale j (0..3)
// of that MMA at (r % 32) * 16 + ((r % 128) / 32) * 4 + j.
SVDQ_HD constexpr uint32_t sf_nvfp4_offset(uint32_t row, uint32_t j16, uint32_t rows_per_tile) {
  return (j16 >> 2) * (rows_per_tile / 128u) * 512u + (row >> 7) * 512u + (row & 31u) * 16u +
         ((row & 127u) >> 5) * 4u + (j16 & 3u);
}

SVDQ_HD constexpr size_t sf_chunk_offset(size_t tile, size_t kb, size_t KB, size_t rows_per_tile) {
  return (tile * KB + kb) * rows_per_tile * kSfBytesPerRowKb;
}

// INT4 scales of one (tile, kb): activations [128 rows][4 groups] fp32; weights [4 groups][256 rows] fp32.
SVDQ_HD constexpr uint32_t sf_int4_a_index(uint32_t row, uint32_t g) { return row * 4u + g; }
SVDQ_HD constexpr uint32_t sf_int4_b_index(uint32_t row, uint32_t g) { return g * 256u + row; }

// Low-rank operands (T tiles of 128 rows, L2 tiles of 256 rows) in the no-swizzle K-major
// core-matrix layout: chunk c covers columns [64c, 64c + cw); inside a chunk, 8x8 core
// matrices of 128 bytes, adjacent along K (LBO = 128 B), 8-row groups SBO = cw * 16 B apart.
SVDQ_HD constexpr uint32_t lr_chunk_width(int r, int c) {
  return static_cast<uint32_t>((r - kLrChunk * c) < kLrChunk ? (r - kLrChunk * c) : kLrChunk);
}
SVDQ_HD constexpr uint32_t lr_offset(uint32_t row, uint32_t col, uint32_t rows_per_tile, int r) {
  const uint32_t c = col / kLrChunk;
  const uint32_t cw = lr_chunk_width(r, static_cast<int>(c));
  const uint32_t cc = col % kLrChunk;
  return rows_per_tile * kLrChunk * 2u * c + (row >> 3) * (cw * 16u) + (cc >> 3) * 128u + (row & 7u) * 16u +
         (cc & 7u) * 2u;
}

// L1 (K x r), K-major per rank column: per 64-element chunk of K, r rows (one per rank column) x
// 128 bytes, swizzled like the codes.  Eight consecutive k of one column form a 16-byte unit, which
// the warp-level MMAs of kernel 1 and of the fused MLP epilogue load as B fragments.
SVDQ_HD constexpr size_t l1_offset(uint32_t k, uint32_t i, int r) {
  return static_cast<size_t>(k / 64u) * static_cast<size_t>(r) * 128u + swz128(i, (k % 64u) * 2u);
}

// Kernel 1's 128-row-tile form splits K into at most this many slices per tile: at most 8, at most
// one per k-block, and at most 160 CTAs in all (one wave on a GPU of up to 160 SMs).
SVDQ_HD constexpr int quant_down_split_cap(int m_tiles, int KB) {
  const int by_grid = m_tiles > 0 ? 160 / m_tiles : 1;
  const int cap = by_grid < 8 ? by_grid : 8;
  return cap < 1 ? 1 : (cap < KB ? cap : KB);
}

struct WorkspaceLayout {
  size_t codes = 0, sf = 0, t = 0, part = 0, cnt = 0, total = 0;
  int m_tiles = 0, split_cap = 1;
};

// Workspace: activation codes, scales and T (bf16) of every row of the padded tiles and, for kernel 1
// when it splits K (rank > 0), the fp32 partials of T of every slice plus one arrival counter per
// 16-row block (the 128-row-tile form uses the first one per 128-row tile).
inline WorkspaceLayout workspace_layout(int M, int K, int r) {
  WorkspaceLayout w;
  w.m_tiles = 2 * ((M + 2 * kBM - 1) / (2 * kBM));  // kernel 2 consumes rows in pairs of 128-row tiles
  w.split_cap = quant_down_split_cap(w.m_tiles, K / kBK);
  const size_t mpad = static_cast<size_t>(w.m_tiles) * kBM;
  w.codes = 0;
  size_t end = mpad * static_cast<size_t>(K) / 2;
  w.sf = align_up(end, 1024);
  end = w.sf + mpad * static_cast<size_t>(K) / kBK * kSfBytesPerRowKb;
  w.t = align_up(end, 1024);
  end = w.t + mpad * static_cast<size_t>(r) * 2;
  if (r > 0 && w.split_cap > 1) {
    w.part = align_up(end, 1024);
    end = w.part + mpad * static_cast<size_t>(w.split_cap) * static_cast<size_t>(r) * 4;
    w.cnt = align_up(end, 256);
    end = w.cnt + mpad / 16 * 8;
  }
  w.total = M > 0 ? align_up(end, 1024) : 0;
  return w;
}

}  // namespace svdq
