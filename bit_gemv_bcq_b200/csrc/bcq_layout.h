// bcq_layout.h -- data layouts and launch parameters shared by the host code
// and the kernels of libbcq.
//
// Packed planes (written by bcq_pack_planes, read by the GEMV kernel)
// ------------------------------------------------------------------
// Rows are grouped in row-blocks of 32 (one row per lane of a warp) and
// row-blocks in row groups of 4; columns in K-blocks of 256 (two scale groups
// A = first 128 columns, B = last 128) and K-blocks in chunks of 2 (512
// columns).  One plane of one (row-block, K-block) is 1 KiB: 32 rows x 32
// bytes, each byte an 8-column "chunk" of bits (bit j = column 8c + j).
// Words are ordered chunk-major, then row group, then plane, then row-block:
//
//   word = ((((((chunk * RBG + rg) * p_H + i) * 4 + r) * 2 + kbi) * 2 + pass) * 32 + lane) * 4 + u
//
// (row-block 4 rg + r, K-block 2 chunk + kbi), so the first p planes of one
// (chunk, row group) are one contiguous span of 8 p KiB: a GEMV task streams
// all its planes with one bulk copy, and a p-bit call never touches planes
// >= p.  Row-blocks past the matrix are zero.
// The four bytes j of word (pass, lane, u) hold, for row 32 rb + lane, the
// 8-column chunk c = (4u + j + lane) mod 16 of group h = (lane / 16) xor pass.
// In pass 0 lanes 0-15 walk group A and lanes 16-31 group B; in pass 1 they
// swap.  At every step the 32 lanes touch 32 different (group, chunk) columns
// of the lookup table, one per shared-memory bank, whatever the bit values.
//
// Packed scales (written by bcq_pack_scales, read by the GEMV kernel)
// ------------------------------------------------------------------
// A per-(row, group) array with q values per entry (alpha^(q): q = 1..4; the
// offsets z: q = 1) in the same order (RBP = 4 RBG row-blocks):
//
//   half = (((((chunk * RBP + rb) * 2 + kbi) * 2 + pass) * 32 + lane) * q + i
//
// holding entry (row 32 rb + lane, group 2 (2 chunk + kbi) + ((lane / 16) xor
// pass)), value i; zero outside the matrix.  1 KiB q per (chunk, row group).
//
// Lookup table in shared memory
// -----------------------------
// The LUT starts at lut_base, the first 64 KiB boundary of the shared window
// above the CTA's low region (the window address of a CTA in a cluster
// carries its rank in bits 24 and up, so the base is computed at run time).
// The table of K-block kbi (of the current chunk) and activation row m is
// "slot" s = m * 2 + kbi, at lut_base + (s / 2) * 65536 + (s % 2) * 128, and
// entry (byte value b, column h*16 + c) at + b * 256 + (h*16 + c) * 4.  A
// 256-byte stride per byte value lets one prmt form lut_base + b * 256 +
// column * 4 from a plane word and a per-lane register holding two column
// offsets and the upper half of lut_base; the slot offset is an immediate.
#pragma once

#include <cstdint>

namespace bcq {

constexpr int kRowBlock = 32;           // rows per row-block (one per lane)
constexpr int kKBlock = 256;            // columns per K-block (2 groups)
constexpr int kChunkBlocks = 2;         // K-blocks per chunk
constexpr int kRowGroup = 4;            // row-blocks per row group (= per task)
constexpr int kGroup = 128;             // columns per scale group
constexpr int kWordsPerPlaneBlock = 256;  // 1 KiB per (rb, plane, kb)
constexpr int kPlaneChunkBytes = 2048;    // one plane of one (chunk, row-block)
constexpr int kUnitBytesPerPlane = 512;   // one pass of one K-block: 32 lanes x 16 B
constexpr uint32_t kLutAlign = 65536;   // the LUT starts on this boundary
constexpr uint32_t kLutTableBytes = 65536;
constexpr int kMaxMPerLaunch = 2;       // activation rows per GEMV launch
constexpr int kLowReserve = 4096;       // room for the shared window's own base
constexpr int kMaxStages = 8;
constexpr int kMaxConsumerWarps = 12;
constexpr int kMaxProducerWarps = 4;    // bulk-copy issue is per-warp latency bound

struct GemvParams {
  const uint16_t* x;        // fp16 [M][K] (rows of this launch)
  const uint32_t* planes;   // packed planes
  const uint16_t* scale[3]; // packed alpha^(q) of the distinct precisions
                            // ([0], [1]), packed offsets ([2], or nullptr)
  uint16_t* y;              // fp16 [M][N] (rows of this launch)
  int M, N, K, G, KB, KC, RBG, p_H;
  int p_load;               // planes streamed: max over rows of p_m
  int p_m[2];               // precision of each activation row
  int nq;                   // distinct precisions among the rows
  int q_of[2];              // precision of distinct entry d
  int d_of[2];              // distinct entry of activation row m
  int has_z;                // offsets present
  int S;                    // CTAs per cluster = K splits (in chunks)
  int rg_base, rg_rem;      // row groups per cluster: base (+1 for the first rem)
  int W;                    // consumer warps (a multiple of 4); then NP producers
  int NP;                   // producer warps
  int D;                    // ring stages (a multiple of W / 4 and of NP)
  int part_rows;            // row stride of the running row sums
  uint32_t stage_off[kMaxStages];  // stage offsets from the dynamic smem base
  uint32_t stage_bytes;     // bytes of one stage
  uint32_t st_scale[3];     // offsets in a stage of the scale and offset spans
  uint32_t off_acc;         // low-region offsets from the dynamic smem base:
  uint32_t off_recv;        //   running row sums [M][part_rows], receive
  uint32_t off_gsum;        //   buffer [S][M][own_rows], group sums,
  uint32_t off_bar;         //   full/empty/receive barriers, abort flag
  uint32_t off_flag;
  int own_rows;             // rows of the cluster's rows each rank finishes
  uint32_t low_bytes;       // end of the low region's fixed part
  uint32_t lut_bytes;       // LUT bytes
  uint32_t dyn_bytes;       // dynamic shared memory of the launch
  int early_weights;        // with PDL: stream weights before the grid wait
  unsigned long long timeout_ns;
};

struct LutParams {
  const uint16_t* x;   // fp16 [M][K]
  float* lut;          // fp32 [M][K/8][256]
  float* gsum;         // fp32 [M][K/128] or nullptr
  int M, K, KB, G;
  uint32_t dyn_bytes;
};

}  // namespace bcq
