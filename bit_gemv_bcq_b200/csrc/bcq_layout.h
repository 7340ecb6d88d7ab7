// bcq_layout.h -- data layouts and launch parameters shared by the host code
// and the kernels of libbcq.
//
// Blocking
// --------
// Rows are grouped in row-blocks of 32 (one row per lane of a warp), columns
// in K-blocks of 256 (two scale groups: A = first 128 columns, B = last 128).
// RB = ceil(N / 32), KB = ceil(K / 256).  A "unit" is one (K-block,
// row-block) pair; units are numbered kb-major: u = kb * RB + rb.
//
// Packed planes (written by bcq_pack_planes, read by the GEMV kernel)
// ------------------------------------------------------------------
// One plane of one unit is 1 KiB: 32 rows x 32 bytes, each byte an 8-column
// "chunk" of bits (bit j = column 8c + j).  Row-blocks are grouped by 8
// (RG = ceil(RB / 8) row groups); words are ordered K-block, row group,
// plane, row-block in the group:
//
//   word = (((((kb * RG + rg) * p_H + i) * 8 + r) * 2 + pass) * 32 + lane) * 4 + u
//
// for row-block rb = 8 rg + r, so the first p planes of a row group are one
// contiguous span of 8p KiB (a ring stage is one bulk copy) and a p-bit call
// never touches planes >= p.
// The four bytes j of word (pass, lane, u) hold, for row 32 rb + lane, chunk
// c = (4u + j + lane) mod 16 of group h = (lane / 16) xor pass.  In pass 0
// lanes 0-15 walk group A and lanes 16-31 group B; in pass 1 they swap.  At
// every step the 32 lanes touch 32 different (group, chunk) columns of the
// lookup table, one per shared-memory bank, whatever the bit values.
// Inside a byte the chunk's 8 bits are rotated right by one: bit j of the
// stored byte is column 8c + ((j + 1) mod 8), i.e. stored = rotr8(canonical,
// 1).  The one-row kernel then forms the address b * 128 + column * 4 of a
// dense 32 KiB table directly from the stored byte (see below).
// Row-blocks past N and columns past K are zero.
//
// Packed scales (written by bcq_pack_scales, read by the GEMV kernel)
// ------------------------------------------------------------------
// A per-(row, group) array with q values per entry (alpha^(q): q = 1..4; the
// offsets z: q = 1):
//
//   half = (((kb * RB + rb) * 32 + lane) * 2 + pass) * q + i
//
// holding entry (row 32 rb + lane, group 2 kb + ((lane / 16) xor pass)),
// value i: one lane reads its 2q values of a unit with one or a few vector
// loads.  Zero outside the matrix.
//
// Lookup table in shared memory
// -----------------------------
// The table of one K-block sits at the start of the dynamic shared memory.
// For the stored byte s of a chunk (s = rotr8(b, 1) for the canonical byte
// b) and column col = h * 16 + c, the entry sum_j (2 bit_j(b) - 1) x[8c + j]
// is at
//   M = 1 (gemv_m1_kernel):  b * 128 + col * 4    (fp32, dense 32 KiB)
//   M = 2, 4 (pair tables):  s * 256 + col * 8    (fp32 pair: row 0, row 1)
// Pair tables: one prmt forms s * 256 + (column byte) from a plane word and
// a per-lane register holding the column bytes.  M = 1: with a = s & 0x7F
// and e = (s & 0x80) | (column byte), one prmt forms a * 256 + e =
// rotl8(s, 1) * 128 + col * 4 = b * 128 + col * 4 (two lop3 per word make
// a and e for its four bytes).  The table's shared address is the immediate
// offset of the load, so the table needs no alignment.
//
// One-row kernel (gemv_m1_kernel) ring stage: the P planes of a row group
// (plane i at i * 8 KiB, row-block w at w KiB), then its packed alpha^(P)
// (row-block w at w * 128 P bytes), then its packed offsets (w * 128
// bytes): three bulk copies of the packed arrays, 16-byte aligned.
#pragma once

#include <cstdint>

namespace bcq {

constexpr int kRowBlock = 32;            // rows per row-block (one per lane)
constexpr int kKBlock = 256;             // columns per K-block (2 groups)
constexpr int kGroup = 128;              // columns per scale group
constexpr int kWordsPerUnitPlane = 256;  // 1 KiB per (kb, plane, rb)
constexpr int kUnitPlaneBytes = 1024;
constexpr int kTeamWarps = 8;            // a team reads a stage: one row-block each
constexpr int kConsumerWarps = 16;       // two teams, alternate groups
constexpr int kRowGroup = 8;             // row-blocks per row group = per ring stage
constexpr int kPlaneGroupBytes = kRowGroup * kUnitPlaneBytes;  // one plane of a row group
constexpr uint32_t kLutBytes = 65536;
constexpr int kMaxStages = 20;
constexpr int kMaxProducerWarps = 4;
constexpr int kMaxMPerLaunch = 2;        // activation rows per GEMV launch
// Shared-window address of the dynamic shared memory of a CTA launched
// without clusters and without static shared memory (checked at run time).
constexpr uint32_t kDynBase = 0x400;

// Dynamic shared memory of a lookup launch of M rows with D ring stages of
// P planes: the table (two pair tables for M = 4), the ring, the barriers.
__host__ __device__ constexpr uint32_t gemv_stage_bytes(int P) {
  return (uint32_t)P * kPlaneGroupBytes;
}
__host__ __device__ constexpr uint32_t gemv_lut_bytes(int M) {
  return M == 4 ? 2u * kLutBytes : kLutBytes;
}
__host__ __device__ constexpr uint32_t gemv_off_bar(int D, int P, int M = 1) {
  return gemv_lut_bytes(M) + (uint32_t)D * gemv_stage_bytes(P);
}
__host__ __device__ constexpr uint32_t gemv_off_misc(int D, int P, int M = 1) {
  return gemv_off_bar(D, P, M) + 16u * (uint32_t)D;
}
__host__ __device__ constexpr uint32_t gemv_dyn_bytes(int D, int P, int M = 1) {
  return gemv_off_misc(D, P, M) + 16u;
}

// The one-row kernel: 16 consumer warps in two teams of 8 (team t takes
// stages t, t + 2, ...; warp w of a team takes row-block w of the stage)
// and NP producer warps; a dense 32 KiB table; ring stages of planes +
// scales + offsets; then the full / empty barriers and the abort flag.
constexpr int kM1Warps = 16;
constexpr int kM1TeamWarps = 8;
// Producer warps of the one-row kernel for P planes, one part of every stage
// each (measured: splitting the planes between two warps pays at four planes
// only).
__host__ __device__ constexpr int m1_producers(int P) { return P >= 4 ? 4 : 3; }
constexpr uint32_t kLut1Bytes = 32768;
__host__ __device__ constexpr uint32_t m1_alpha_off(int P) {
  return (uint32_t)P * kPlaneGroupBytes;
}
__host__ __device__ constexpr uint32_t m1_z_off(int P) {
  return m1_alpha_off(P) + (uint32_t)kRowGroup * 128u * (uint32_t)P;
}
__host__ __device__ constexpr uint32_t m1_stage_bytes(int P) {
  return m1_z_off(P) + (uint32_t)kRowGroup * 128u;
}
__host__ __device__ constexpr uint32_t m1_off_bar(int D, int P) {
  return kLut1Bytes + (uint32_t)D * m1_stage_bytes(P);
}
__host__ __device__ constexpr uint32_t m1_off_misc(int D, int P) {
  return m1_off_bar(D, P) + 16u * (uint32_t)D;
}
__host__ __device__ constexpr uint32_t m1_dyn_bytes(int D, int P) {
  return m1_off_misc(D, P) + 16u;
}

// Units of one CTA, computed on the host: [u0, u1), its group count and
// first and last K-blocks (no integer division on the device).
struct CtaWork {
  int u0, u1, ng, kb;  // kb: first K-block (bits 0-15), last K-block (16-31)
};
constexpr int kMaxCtas = 256;

// The tensor-core GEMV (bcq_mma.cuh): activations of the current K-block
// (two slots of 16 rows x 256 columns, stored in the order of the MMA's B
// fragments: xtile_offset) and their group sums, then per-warp double
// buffers of scales and offsets, then the ring.
constexpr int kMmaRows = 16;                 // activation rows per tensor-core launch (max)
constexpr uint32_t kXTileBytes = kMmaRows * kKBlock * 2;             // 8192
constexpr uint32_t kMmaGsumOff = 2 * kXTileBytes;                    // 16384
constexpr uint32_t kMmaScaleOff = kMmaGsumOff + 2 * kMmaRows * 2 * 4; // 16640
// Scales staged per warp and unit: 32 lanes x 2P halves of alpha^(P), then
// the offsets (2 halves a lane).  Mixed launches (rows of several
// precisions) stage alpha^(q) of every precision q = 1..4 present, each in
// its own block of 32 x 2q halves at byte 64 q (q - 1), and the offsets of
// each precision q present at byte 1280 + 128 (q - 1).
__host__ __device__ constexpr uint32_t mma_scale_buf_bytes(int P, bool mixed = false) {
  return mixed ? 1280u + 4u * 128u : (uint32_t)32 * (2 * P + 2) * 2;
}
__host__ __device__ constexpr uint32_t mma_z_off(int P, bool mixed = false, int q = 1) {
  return mixed ? 1280u + 128u * (uint32_t)(q - 1) : 128u * (uint32_t)P;
}
__host__ __device__ constexpr uint32_t mma_alpha_block(int q) { return 64u * (uint32_t)q * (uint32_t)(q - 1); }
__host__ __device__ constexpr uint32_t mma_ring_off(int P, bool mixed = false) {
  return (kMmaScaleOff + 16u * 2u * mma_scale_buf_bytes(P, mixed) + 1023u) & ~1023u;
}
__host__ __device__ constexpr uint32_t mma_off_bar(int D, int P, bool mixed = false) {
  return mma_ring_off(P, mixed) + (uint32_t)D * gemv_stage_bytes(P);
}
__host__ __device__ constexpr uint32_t mma_dyn_bytes(int D, int P, bool mixed = false) {
  return mma_off_bar(D, P, mixed) + 16u * (uint32_t)D + 16u;
}

// The tcgen05 GEMV (bcq_umma.cuh), for NN = 16 or 64 activation rows per
// launch (the MMA's N).  Shared memory: the activation tiles of two K-blocks
// in the canonical K-major layout of the MMA's B operand (NN rows x 256
// columns), their group sums, per-warp scale buffers (as above), the ring,
// then the barriers.  Tensor memory (512 columns, lane = weight row): four
// MMA groups (team x half of a team's row group) of 128 columns each: fp32
// accumulators of NN columns (column = activation row; two, alternating by
// unit, for NN = 16, one for NN = 64) and 32-column A-operand buffers (64
// K-columns of +-alpha; three for NN = 16, two for NN = 64).
constexpr int kUmmaGroups = 4;                  // = MMA-issuing warps
constexpr int kUmmaGroupWarps = 4;              // expanding warps of an MMA group
constexpr uint32_t kUmmaGroupCols = 128;
constexpr uint32_t kUmmaABufCols = 32;
constexpr uint32_t kUmmaTmemCols = 512;
constexpr int kMaxLaunchRows = 64;              // activation rows of one launch (any kernel)

template <int NN>
struct UmmaShape {
  static_assert(NN == 16 || NN == 64, "16 or 64 activation rows");
  static constexpr int kN = NN;
  static constexpr uint32_t kXTileBytes = (uint32_t)NN * 512u;  // NN rows x 256 fp16
  static constexpr uint32_t kGsumOff = 2u * kXTileBytes;
  static constexpr uint32_t kScaleOff = kGsumOff + 2u * NN * 2u * 4u;
  static constexpr int kAccBufs = NN == 16 ? 2 : 1;
  static constexpr int kABufs = NN == 16 ? 3 : 2;
  static constexpr uint32_t kACol = (uint32_t)kAccBufs * NN;  // first A column of a group
  static constexpr int kBarsPerGroup = 2 * kABufs + 2 * kAccBufs;
  static_assert(kACol + kABufs * kUmmaABufCols <= kUmmaGroupCols, "tensor memory budget");
};
template <int NN>
__host__ __device__ constexpr uint32_t umma_ring_off(int P) {
  return (UmmaShape<NN>::kScaleOff + 16u * 2u * mma_scale_buf_bytes(P) + 1023u) & ~1023u;
}
template <int NN>
__host__ __device__ constexpr uint32_t umma_off_bar(int D, int P) {
  return umma_ring_off<NN>(P) + (uint32_t)D * gemv_stage_bytes(P);
}
// full[D], empty[D], then per MMA group: A full[kABufs], A empty[kABufs],
// accumulator full[kAccBufs], accumulator empty[kAccBufs]; then the
// tensor-memory address and the abort flag.
template <int NN>
__host__ __device__ constexpr uint32_t umma_off_misc(int D, int P) {
  return umma_off_bar<NN>(D, P) + 16u * (uint32_t)D +
         8u * (kUmmaGroups * UmmaShape<NN>::kBarsPerGroup);
}
template <int NN>
__host__ __device__ constexpr uint32_t umma_dyn_bytes(int D, int P) {
  return umma_off_misc<NN>(D, P) + 16u;
}

struct GemvParams {
  const uint16_t* x;         // fp16 [M][K] (rows of this launch)
  const uint32_t* planes;    // packed planes
  const uint16_t* alpha[2];  // packed scales of row 0 and row 1 (q[m] per entry)
  const uint16_t* z;         // packed offsets of the launch (of row 0 in a mixed lookup launch), or nullptr
  const uint16_t* z1;        // packed offsets of row 1 in a mixed lookup launch (per-precision offsets)
  uint16_t* y;               // fp16 [M][N] (rows of this launch)
  float* part;               // tagged fp32 partial sums [KB][M][RB * 32] (KB > 1), zero between calls
  int M, N, K, KB, RB, RG, p_H;
  int q[2];                  // precision of each row (<= planes streamed)
  int U;                     // units (< 2^31)
  int C;                     // CTAs
  int D, NP;                 // ring stages, producer warps
  int MW;                    // MMA-issuing warps (tcgen05 kernel), else 0
  int early_weights;         // with PDL: stream weights before the grid wait
  unsigned long long timeout_ns;
  int rows[kMaxLaunchRows];  // tensor-core launches: x / y row of launch row m
  // mixed tensor-core launches: precision of launch row m, packed scales and
  // offsets of each precision q (alpha_q[q - 1], z_q[q - 1]) and the
  // precisions present (bit q)
  int qrow[kMaxLaunchRows];
  const uint16_t* alpha_q[4];
  const uint16_t* z_q[4];    // their offsets (or nullptr: none)
  int qmask;
  CtaWork work[kMaxCtas];    // per CTA (C entries)
};

struct LutParams {
  const uint16_t* x;   // fp16 [M][K] (M = 1 or 2)
  float* lut;          // fp32 [M][K/8][256]
  float* gsum;         // fp32 [M][K/128] or nullptr
  int M, K, KB, G;
};

}  // namespace bcq
