// bcq_layout.h -- data layouts and launch parameters shared by the host code
// and the kernels of libbcq.
//
// Packed planes (written by bcq_pack_planes, read by the GEMV kernel)
// ------------------------------------------------------------------
// Rows are grouped in row-blocks of 32 (one row per lane of a warp) and
// columns in K-blocks of 256 (two scale groups A = first 128 columns,
// B = last 128).  One plane of one (row-block, K-block) is 1 KiB: 32 rows x
// 32 bytes, each byte an 8-column "chunk" of bits (bit j = column 8c + j).
//
//   word index = ((((rb * p_H + i) * KB + kb) * 2 + pass) * 32 + lane) * 4 + u
//
// The four bytes j of word (pass, lane, u) hold, for row 32 rb + lane, the
// chunk c = (4u + j + lane) mod 16 of group h = (lane / 16) xor pass.  In pass
// 0 lanes 0-15 walk group A and lanes 16-31 group B; in pass 1 they swap.  At
// every step the 32 lanes therefore touch 32 different (group, chunk) columns
// of the lookup table, one per shared-memory bank, whatever the bit values.
// Plane i of a row-block is contiguous per K range, so a p-bit call streams
// planes 0..p-1 and never touches the others.
//
// Lookup table in shared memory
// -----------------------------
// The table of a K-block kb (phase-local) and activation row m is "slot"
// s = m * NKB + kb.  Slot s lives at absolute shared address
//   kLutAbs + (s / 2) * 65536 + (s % 2) * 128
// and entry (byte value b, column h*16 + c) at + b * 256 + (h*16 + c) * 4.
// A 256-byte stride per byte value lets one prmt build the address
// b * 256 + column * 4 from a plane word and a per-lane column register.
#pragma once

#include <cstdint>

namespace bcq {

constexpr int kRowBlock = 32;           // rows per row-block (one per lane)
constexpr int kKBlock = 256;            // columns per K-block (2 groups)
constexpr int kGroup = 128;             // columns per scale group
constexpr int kWordsPerPlaneBlock = 256;  // 1 KiB per (rb, plane, kb)
constexpr int kUnitBytesPerPlane = 512;   // one pass of one plane: 32 lanes x 16 B
constexpr uint32_t kLutAbs = 65536;     // absolute shared address of the LUT
constexpr uint32_t kLutTableBytes = 65536;
constexpr int kMaxMPerLaunch = 4;       // activation rows per GEMV launch
constexpr int kLowReserve = 4096;       // room for the shared window's own base

struct GemvParams {
  const uint16_t* x;        // fp16 [M][K] (rows of this launch)
  const uint32_t* planes;   // packed planes
  const uint16_t* alpha[4]; // alpha^(q) fp16 [N][G][q], q = 1..4
  const uint16_t* z;        // fp16 [N][G] or nullptr
  uint16_t* y;              // fp16 [M][N] (rows of this launch)
  int M, N, K, G, KB, RB, p_H;
  int p_load;               // planes streamed: max over rows of p_m
  int p_m[4];               // precision of each activation row
  int S;                    // CTAs per cluster = K splits
  int rb_base, rb_rem;      // row-blocks per cluster: base (+1 for the first rem)
  int D;                    // ring stages per warp
  int part_rows;            // row stride of the partial-sum arrays
  uint32_t off_part;        // low-region offsets, from the dynamic smem base
  uint32_t off_gsum;
  uint32_t off_bar;
  uint32_t off_flag;
  uint32_t low_bytes;       // bytes used in the low region
  uint32_t ring_abs;        // absolute shared address of the ring region
  unsigned long long timeout_ns;
};

struct LutParams {
  const uint16_t* x;   // fp16 [M][K]
  float* lut;          // fp32 [M][K/8][256]
  float* gsum;         // fp32 [M][K/128] or nullptr
  int M, K, KB, G;
  uint32_t off_gsum;
};

}  // namespace bcq
