// bcq_umma.cuh -- the tcgen05 (5th-generation tensor core) BCQ GEMV for
// batches of activation rows (included by bcq_kernels.cu only, after
// bcq_mma.cuh, whose scale staging and bit helpers it shares).
//
// The same sum as the other paths (AnyBCQ Paper-Notes page, 关键设计 /
// 直接bit-plane运算的CUDA内核: plane-by-plane contraction with alpha_i; the
// offsets of 训练策略 per 128-column group):
//   y[m][n] = sum_i sum_k (+-alpha_i[n][g(k)]) x[m][k] + sum_g z[n][g] S[m][g]
// with each plane term formed from the bits and alpha only.  Here the 16
// consumer warps expand every plane of their row-blocks into fp16 +-alpha
// (shift the bit to the fp16 sign position, xor it into alpha: exact) and
// store them into tensor memory as the A operand of tcgen05.mma (M = 128
// weight rows = four row-blocks, K = 16), the activation tile is the B
// operand in shared memory (N = 16 activation rows), and the fp32
// accumulator stays in tensor memory until the unit's last plane.  Every
// warp of an MMA group issues one of each chunk's four MMAs into an
// accumulator of its own (one thread issues an MMA every ~55 cycles; a
// dozen issuing threads keep the tensor core at ~9 cycles per MMA), and the
// tensor core works while the warps expand the next chunk.
//
// K order.  Inside a 256-column K-block the A operand holds the columns in
// the order the expansion produces them: tensor-memory column
// c = 64 h + 16 U + s (group h, 32-column word U of the group, shift s)
// holds the columns of bits 15 - s (low half) and 31 - s (high half) of the
// group's natural word U, where bit t is column 128 h + 32 U + 8 (t / 8) +
// ((t + 1) mod 8) (the packed bytes are rotated by one bit).  The activation
// tile is stored with the same permutation.
#pragma once

#include <cstdint>

#include "bcq_device.cuh"
#include "bcq_layout.h"
#include "bcq_pipeline.cuh"

namespace bcq {

// ---------------------------------------------------------------- tcgen05

__device__ __forceinline__ void umma_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void umma_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Whole warp: allocate ncols tensor-memory columns, address to smem dst.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Arrive once on the mbarrier when every MMA this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// D (tensor memory, fp32) (+)= A (tensor memory, fp16) x B (shared memory, fp16).
__device__ __forceinline__ void umma_f16_ts(uint32_t d, uint32_t a, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Generic-proxy shared-memory writes become visible to the tensor core.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Instruction descriptor of kind::f16: fp16 A and B, fp32 D, both K-major,
// M = 128, N = NN (bits 4-5 D format, 7-9 / 10-12 A / B format, 15 / 16
// A / B major, 17-22 N / 8, 24-28 M / 16).
template <int NN>
__host__ __device__ constexpr uint32_t umma_idesc() {
  return (1u << 4) | ((uint32_t)(NN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// Shared-memory descriptor of an NN-row B operand slice in the canonical
// K-major layout without swizzle: 8-row x 16-byte core matrices, K-adjacent
// ones NN * 16 bytes apart (leading byte offset), row-adjacent ones 128 bytes
// apart (stride byte offset); bits 46-47 = 1 (descriptor version).
template <int NN>
__device__ __forceinline__ uint64_t umma_bdesc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((NN * 16u) >> 4) << 16) |
         ((uint64_t)(128u >> 4) << 32) | (1ull << 46);
}

// ------------------------------------------------------- activation tile

// Tile positions of one lane's columns.  Column 8l + e8 of a K-block sits at
// its permuted K position (see above) j of the canonical layout: row n,
// position j at (j / 8) * NN * 16 + (n / 8) * 128 + (n % 8) * 16 + (j % 8) * 2.
// In closed form: with r = (e8 + 7) mod 8 the column's
// shift is s = (l odd ? 7 : 15) - r, its position j = 2 (64 h + 16 U + s) + e
// (e = (l / 2) mod 2) and its byte offset in the row's slice
//   (16 h + 4 U) NN * 16 + 2e - 32 NN (l mod 2) + ((15 - r) / 4) NN * 16 + ((15 - r) mod 4) * 4,
// a per-lane base plus a compile-time constant per column (checked against
// the definition above for every row, lane and column).
template <int NN>
__host__ __device__ constexpr uint32_t umma_xtile_col_off(int e8) {
  return (uint32_t)(((15 - ((e8 + 7) & 7)) >> 2) * NN * 16 + ((15 - ((e8 + 7) & 7)) & 3) * 4);
}
template <int NN, int E8>
struct UmmaXTileCols {
  static __device__ __forceinline__ void run(uint32_t base, const uint32_t (&w)[4]) {
    sts_u16_at<umma_xtile_col_off<NN>(E8)>(base, (w[E8 >> 1] >> (16 * (E8 & 1))) & 0xFFFFu);
    UmmaXTileCols<NN, E8 + 1>::run(base, w);
  }
};
template <int NN>
struct UmmaXTileCols<NN, 8> {
  static __device__ __forceinline__ void run(uint32_t, const uint32_t (&)[4]) {}
};

// Launch row n of K-block kb's activation tile into slot kb & 1: lane l
// holds columns 8l .. 8l + 7 (v, from load_x_tile), stored at their
// positions (above).  Also the row's group sums, and the fence that shows
// the tile to the MMAs.
template <int NN>
__device__ __forceinline__ void umma_store_x_tile(uint32_t sbase, int kb, int n, int lane,
                                                  const uint4& v) {
  using S = UmmaShape<NN>;
  const uint32_t slot = (uint32_t)(kb & 1);
  const uint32_t tile = sbase + slot * S::kXTileBytes +
                        (uint32_t)((n >> 3) * 128 + (n & 7) * 16);
  const int h = lane >> 4, U = (lane >> 2) & 3, e = (lane >> 1) & 1;
  const uint32_t base = tile + (uint32_t)((16 * h + 4 * U) * NN * 16 + e * 2) -
                        (uint32_t)(lane & 1) * (32u * NN);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  UmmaXTileCols<NN, 0>::run(base, w);
  float f[8];
  unpack8(v, f);
  float sum = ((f[0] + f[1]) + (f[2] + f[3])) + ((f[4] + f[5]) + (f[6] + f[7]));
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  if ((lane & 15) == 0)  // lane 0: group A, lane 16: group B
    sts_f32(sbase + S::kGsumOff + ((slot * NN + n) * 2 + (lane >> 4)) * 4u, sum);
  fence_proxy_async_smem();
}

// --------------------------------------------------------------- expansion

// The 32 columns of natural word `wd` (bit b = column 32 U + b of the group)
// as 16 registers of fp16 pairs: register s holds bits 15 - s and 31 - s,
// each +alpha for bit 1 and -alpha for bit 0 (alpha2: alpha in both halves).
__device__ __forceinline__ void expand_word(uint32_t wd, uint32_t alpha2, uint32_t (&r)[16]) {
#pragma unroll
  for (int s = 0; s < 16; ++s) r[s] = xor_andnot(alpha2, wd << s, 0x80008000u);
}

// --------------------------------------------------------------- the kernel

// Barriers of MMA group G (each an 8-byte mbarrier), after the ring's.
struct UmmaBars {
  uint32_t afull, aempty, accfull, accempty;  // first of kABufs / kAccBufs each
};
template <int NN>
__device__ __forceinline__ UmmaBars umma_bars(uint32_t bar0, int G) {
  using S = UmmaShape<NN>;
  const uint32_t b = bar0 + 8u * (uint32_t)(G * S::kBarsPerGroup);
  return {b, b + 8u * S::kABufs, b + 16u * S::kABufs, b + 16u * S::kABufs + 8u * S::kAccBufs};
}

// Warp-specialised, one CTA per SM, with the units, groups, ring, producer
// warps and teams of the other GEMV kernels.
//   warps 0..15   expand: team w / 8 takes alternate groups; team warp tw
//                 expands row-block rb0 + tw into tensor-memory lanes
//                 32 (tw % 4) .. + 31 of MMA group (team, tw / 4): per plane
//                 and 64-column chunk, wait for a free A buffer of the
//                 group's three, store +-alpha, signal the buffer full.  A
//                 unit's accumulator is read one chunk into the next unit
//                 (by then its MMAs are done): offsets added, partial sums
//                 stored, accumulator signalled free.
//   warps 16..19  issue: one per MMA group, lane 0 issues each full
//                 buffer's four MMAs (K = 16 each) into the unit's
//                 accumulator (two, alternating by unit) and commits them to
//                 the buffer's empty barrier, and each unit's last to the
//                 accumulator's full barrier.
//   warps 20..    produce: bulk copies of the planes into the ring.
//   P  planes streamed (one precision for every row of the launch)
template <int P, int NN>
__global__ void __launch_bounds__(32 * (kConsumerWarps + kUmmaGroups + 2), 1)
    gemv_umma_kernel(const __grid_constant__ GemvParams prm) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int D = prm.D, NP = prm.NP, RB = prm.RB;
  constexpr uint32_t kStage = gemv_stage_bytes(P);
  constexpr int kMmaWarp0 = kConsumerWarps;
  constexpr int kProducerWarp0 = kConsumerWarps + kUmmaGroups;
  using S = UmmaShape<NN>;
  constexpr int XR = NN / 16;  // activation tile rows per expanding warp
  const uint32_t ring = sbase + umma_ring_off<NN>(P);
  const uint32_t full0 = sbase + umma_off_bar<NN>(D, P);
  const uint32_t empty0 = full0 + 8u * (uint32_t)D;
  const uint32_t gbar0 = empty0 + 8u * (uint32_t)D;
  const uint32_t misc = umma_off_misc<NN>(D, P);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + misc + 4u);
  constexpr int kConsumers = kConsumerWarps * 32;

  const bool cfg_ok = D >= 2 && D <= kMaxStages && NP >= 1 && NP <= 2 && (D & 1) == 0 &&
                      prm.M >= 1 && prm.M <= NN && prm.MW == kUmmaGroups &&
                      (int)blockDim.x == 32 * (kConsumerWarps + kUmmaGroups + NP);
  CtaRange R;
  make_range(prm, R);
  uint4 xv[XR];  // expanding warps: the first activation tile's rows, first of all
  if (warp < kConsumerWarps) {
    grid_dependency_wait();
#pragma unroll
    for (int r = 0; r < XR; ++r) load_x_tile(prm, R.kb0, warp + 16 * r, lane, xv[r]);
  }
  if (warp == 0) {
    if (cfg_ok && lane < D) {
      mbar_init(full0 + 8u * lane, 1);
      mbar_init(empty0 + 8u * lane, kTeamWarps);
    }
    if (cfg_ok) {
      for (int b = lane; b < kUmmaGroups * S::kBarsPerGroup; b += 32) {
        const int k = b % S::kBarsPerGroup;  // A full, A empty, acc full, acc empty
        const bool by_warps = k < S::kABufs || k >= 2 * S::kABufs + S::kAccBufs;
        mbar_init(gbar0 + 8u * b, by_warps ? kUmmaGroupWarps : 1);
      }
    }
    if (lane == 0) {
      *abort_flag = cfg_ok ? 0 : 1;
      if (!cfg_ok) record_error(&g_device_error, BCQ_ERR_UNSUPPORTED);
    }
    if (cfg_ok) fence_mbar_init();
    __syncwarp();
    if (cfg_ok) tmem_alloc(sbase + misc, kUmmaTmemCols);
  }
  umma_fence_before();
  __syncthreads();
  umma_fence_after();
  launch_dependents();
  if (*abort_flag) return;  // set before the barrier: uniform (no tensor memory held)
  const uint32_t tmem = *tmem_slot;

  if (warp >= kProducerWarp0) {
    produce_stages<P>(prm, R, warp - kProducerWarp0, lane, ring, full0, empty0, abort_flag);
    return;
  }

  auto give_up = [&]() {
    if (lane == 0 && *abort_flag == 0) {
      record_error(&g_device_error, BCQ_ERR_TIMEOUT);
      *abort_flag = 1;
    }
  };

  if (warp >= kMmaWarp0) {
    // ------------------------------------------------------------ issuers
    const int G = warp - kMmaWarp0;
    const int team = G >> 1, hf = G & 1;
    const uint32_t tg = tmem + (uint32_t)G * kUmmaGroupCols;
    const UmmaBars bars = umma_bars<NN>(gbar0, G);
    GroupCursor gc;
    cursor_init(gc, R.u0, R.u1, R.kb0, RB);
    if (team) cursor_next(gc, R.u1, RB);
    int ab = 0, accb = 0;
    uint32_t a_round = 0, acc_round = 0;
    for (int gg = team; gg < R.NG; gg += 2) {
      if (hf * 4 < gc.n) {  // the same test as the group's expanding warps
        const uint32_t xt = sbase + (uint32_t)(gc.kb & 1) * S::kXTileBytes;
        // descriptor of the tile's first K-slice; slice j is NN * 32 bytes on,
        // i.e. NN * 2 in the descriptor's start-address field (address / 16,
        // 14 bits: shared addresses stay below 2^18, so the add never carries
        // out of the field)
        const uint64_t bd0 = umma_bdesc<NN>(xt);
        const uint32_t tacc = tg + (uint32_t)accb * (uint32_t)NN;
        // the accumulator's previous unit has been read
        if (acc_round > 0 &&
            !mbar_wait_bounded(bars.accempty + 8u * accb, (acc_round - 1u) & 1u, prm.timeout_ns))
          give_up();
#pragma unroll 1
        for (int i = 0; i < P; ++i) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            if (!mbar_wait_bounded(bars.afull + 8u * ab, a_round & 1u, prm.timeout_ns)) give_up();
            __syncwarp();
            umma_fence_after();
            if (lane == 0) {
              if (*abort_flag == 0) {
                const uint32_t acol = tg + S::kACol + (uint32_t)ab * kUmmaABufCols;
                const uint64_t bdc = bd0 + (uint64_t)(4 * c) * (NN * 2u);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  umma_f16_ts(tacc, acol + 8u * (uint32_t)j, bdc + (uint64_t)j * (NN * 2u),
                              umma_idesc<NN>(), j != 0 || (i | c) != 0 ? 1u : 0u);
              }
              umma_commit(bars.aempty + 8u * ab);
            }
            if (++ab == S::kABufs) {
              ab = 0;
              ++a_round;
            }
          }
        }
        if (lane == 0) umma_commit(bars.accfull + 8u * accb);
        if (++accb == S::kAccBufs) {
          accb = 0;
          ++acc_round;
        }
      }
      cursor_next(gc, R.u1, RB);
      cursor_next(gc, R.u1, RB);
    }
    __syncwarp();
    named_barrier_sync(6, kConsumers + 32 * kUmmaGroups);  // before the tensor memory is freed
    return;
  }

  // -------------------------------------------------------- expanding warps
  const int team = warp / kTeamWarps;
  const int tw = warp % kTeamWarps;
  const int hf = tw >> 2, qd = tw & 3;  // qd = warp % 4: the warp's tensor-memory lane quarter
  const int G = team * 2 + hf;          // MMA group
  const uint32_t tg = tmem + (uint32_t)G * kUmmaGroupCols;
  const uint32_t tl = tg + ((uint32_t)(qd * 32) << 16);  // this warp's lanes
  const UmmaBars bars = umma_bars<NN>(gbar0, G);
  // rotation of this lane's row (bcq_layout.h): natural word v of a pass is
  // the funnel shift of rotated words (v - ra) mod 4 and (v - ra + 1) mod 4
  const int rho = lane & 15;
  const uint32_t ra = (uint32_t)(((rho + 3) >> 2) & 3);
  const uint32_t dsh = (uint32_t)((-rho) & 3) * 8u;
  const uint32_t sbuf0 = sbase + S::kScaleOff + (uint32_t)warp * 2u * mma_scale_buf_bytes(P);
  const size_t part_stride = (size_t)RB * kRowBlock;
  int cur_kb = -1;

  // The unit whose accumulator is still to be read (deferred epilogue).
  bool pending = false, p_store = false;
  int p_kb = 0, p_row = 0, p_accb = 0;
  uint32_t p_use = 0;
  float p_z0 = 0.f, p_z1 = 0.f;
  auto epilogue = [&]() {
    if (!mbar_wait_bounded(bars.accfull + 8u * p_accb, p_use & 1u, prm.timeout_ns)) give_up();
    __syncwarp();
    umma_fence_after();
    const uint32_t gsl = sbase + S::kGsumOff + (uint32_t)(p_kb & 1) * NN * 8u;
#pragma unroll 1
    for (int m0 = 0; m0 < NN; m0 += 8) {
      uint32_t d[8];
      tmem_ld8(tl + (uint32_t)p_accb * (uint32_t)NN + (uint32_t)m0, d);
      tmem_wait_ld();
      if (p_store && *abort_flag == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int m = m0 + e;
          if (m < prm.M) {
            // offsets: z[row][group] * S[m][group]
            const float sA = lds_f32_dyn(gsl + (uint32_t)(m * 2) * 4u);
            const float sB = lds_f32_dyn(gsl + (uint32_t)(m * 2 + 1) * 4u);
            const float v = fmaf(p_z0, sA, fmaf(p_z1, sB, __uint_as_float(d[e])));
            if (prm.KB > 1)
              st_partial(prm.part + ((size_t)p_kb * prm.M + m) * part_stride + (size_t)p_row, v);
            else if (p_row < prm.N)
              prm.y[(size_t)prm.rows[m] * prm.N + p_row] = f2h_rn(v);
          }
        }
      }
    }
    umma_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cta(bars.accempty + 8u * p_accb);
    pending = false;
  };

  // tiles of every K-block up to kbt, in order, by all 16 warps; every
  // earlier unit's MMAs are complete before a slot is rebuilt (both teams
  // read their last accumulator first)
  auto advance_tiles = [&](int kbt) {
    if (cur_kb >= kbt) return;
    if (pending) epilogue();
    while (cur_kb < kbt) {
      const int kbn = cur_kb < 0 ? R.kb0 : cur_kb + 1;
#pragma unroll
      for (int r = 0; r < XR; ++r) {  // rows warp, warp + 16, ... of the tile
        if (cur_kb >= 0) load_x_tile(prm, kbn, warp + 16 * r, lane, xv[r]);
        umma_store_x_tile<NN>(sbase, kbn, warp + 16 * r, lane, xv[r]);
      }
      named_barrier_sync(1, kConsumers);
      cur_kb = kbn;
    }
  };

  GroupCursor gc;  // this team's next group
  cursor_init(gc, R.u0, R.u1, R.kb0, RB);
  int gg = team;
  if (team) cursor_next(gc, R.u1, RB);
  int s = team;
  uint32_t ph = 0;
  GroupCursor pc = gc;
  int buf = 0;
  if (gg < R.NG && tw < pc.n) stage_scales<P>(prm, pc.kb, pc.rb0 + tw, lane, sbuf0);
  cp_async_commit();
  cursor_next(pc, R.u1, RB);
  cursor_next(pc, R.u1, RB);
  int ab = 0, accb = 0;
  uint32_t a_round = 0, acc_round = 0;

  while (gg < R.NG) {
    advance_tiles(gc.kb);
    const bool active = tw < gc.n;
    const bool group_active = hf * 4 < gc.n;  // uniform over the MMA group's warps
    const uint32_t sbuf = sbuf0 + (uint32_t)buf * mma_scale_buf_bytes(P);
    if (gg + 2 < R.NG && tw < pc.n)
      stage_scales<P>(prm, pc.kb, pc.rb0 + tw, lane,
                      sbuf0 + (uint32_t)(buf ^ 1) * mma_scale_buf_bytes(P));
    cp_async_commit();
    cp_async_wait<1>();
    __syncwarp();
    // warp-uniform: the tensor-memory stores below are .sync.aligned
    const bool ok =
        __all_sync(0xFFFFFFFFu, wait_stage(full0 + 8u * s, ph, abort_flag, prm.timeout_ns));
    if (!ok) give_up();
    const bool work = ok && active;
    if (group_active) {
      const uint32_t st = ring + (uint32_t)s * kStage + (uint32_t)tw * kUnitPlaneBytes;
#pragma unroll 1
      for (int i = 0; i < P; ++i) {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          const int pass = h ^ (lane >> 4);  // rows >= 16 hold group A in pass 1
          uint32_t nw[4] = {0u, 0u, 0u, 0u};
          uint32_t al2 = 0u;
          if (work) {
            const uint32_t base =
                st + (uint32_t)i * kPlaneGroupBytes + (uint32_t)pass * 512u + (uint32_t)lane * 16u;
            uint32_t w[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) w[v] = lds_u32(base + (((uint32_t)v - ra) & 3u) * 4u);
#pragma unroll
            for (int v = 0; v < 4; ++v) nw[v] = funnel_r(w[v], w[(v + 1) & 3], dsh);
            const uint32_t ah =
                lds_u16(sbuf + ((uint32_t)lane * 2u * P + (uint32_t)pass * P + i) * 2u);
            al2 = ah | (ah << 16);
          }
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            if (a_round > 0 &&
                !mbar_wait_bounded(bars.aempty + 8u * ab, (a_round - 1u) & 1u, prm.timeout_ns))
              give_up();
            __syncwarp();
            umma_fence_after();
            const uint32_t acol = S::kACol + (uint32_t)ab * kUmmaABufCols;
            if (work) {
#pragma unroll
              for (int t = 0; t < 2; ++t) {
                uint32_t r[16];
                expand_word(nw[2 * cc + t], al2, r);
                tmem_st16(tl + acol + 16u * (uint32_t)t, r);
              }
            }
            tmem_wait_st();
            umma_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(bars.afull + 8u * ab);
            if (++ab == S::kABufs) {
              ab = 0;
              ++a_round;
            }
            // the previous unit's MMAs are done by now, or nearly
            if (pending && (i | h | cc) == 0) epilogue();
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive_cta(empty0 + 8u * s);  // the stage's planes are read
    if (group_active) {
      if (pending) epilogue();
      pending = true;
      p_store = work;
      p_kb = gc.kb;
      p_row = (gc.rb0 + tw) * kRowBlock + lane;
      p_accb = accb;
      p_use = acc_round;
      p_z0 = p_z1 = 0.f;
      if (work && prm.z) {
        p_z0 = h2f((uint16_t)lds_u16(sbuf + 128u * P + (uint32_t)(lane * 2 + (lane >> 4)) * 2u));
        p_z1 = h2f((uint16_t)lds_u16(sbuf + 128u * P + (uint32_t)(lane * 2 + ((lane >> 4) ^ 1)) * 2u));
      }
      if (++accb == S::kAccBufs) {
        accb = 0;
        ++acc_round;
      }
    }
    buf ^= 1;
    cursor_next(pc, R.u1, RB);
    cursor_next(pc, R.u1, RB);
    cursor_next(gc, R.u1, RB);
    cursor_next(gc, R.u1, RB);
    s += 2;
    if (s >= D) {
      s -= D;
      ph ^= 1u;
    }
    gg += 2;
  }
  cp_async_wait<0>();
  if (pending) epilogue();
  advance_tiles(R.kb_last);  // the same barriers in both teams

  // every MMA of the CTA completed (each group read its last accumulator)
  // and every partial is stored: free the tensor memory, then reduce
  umma_fence_before();
  named_barrier_sync(6, kConsumers + 32 * kUmmaGroups);
  if (warp == 0) {
    umma_fence_after();
    tmem_dealloc(tmem, kUmmaTmemCols);
  }
  // (no barrier: a warp starts its reduction tasks as soon as it is done;
  // the partials it waits for are polled, not counted)
  if (prm.KB > 1) {
    splitk_tail<8>(prm, R, prm.M, prm.rows, tid, kConsumers, abort_flag);
  }
}

}  // namespace bcq
