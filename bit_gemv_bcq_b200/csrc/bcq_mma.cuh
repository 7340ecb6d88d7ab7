// bcq_mma.cuh -- the tensor-core BCQ GEMV (included by bcq_kernels.cu only).
//
// For a batch of up to 16 activation rows the lookup table costs grow with
// the batch; here each plane is instead expanded in registers into fp16
// matrix fragments holding +-alpha (alpha^(p)[n][g][i] with the sign of the
// plane bit: bit 1 -> +alpha, 0 -> -alpha, exact in fp16) and multiplied with
// the activations on the tensor cores (mma.sync m16n8k16, fp32 accumulate):
//   y[m][n] = sum_g sum_i sum_{k in g} (+-alpha) x[m][k]  +  sum_g z[n][g] S[m][g]
// which is the same sum as the lookup path (AnyBCQ Paper-Notes page, 关键设计
// / 直接bit-plane运算的CUDA内核: plane-by-plane contraction with alpha_i,
// offsets per group from 训练策略), with no dequantised weight matrix: each
// plane term is formed from the bits and alpha only, in registers.
//
// The planes are read from the same packed layout as the lookup path (one
// bulk copy per row group and K-block into the ring); the producer warps,
// the CTA's unit ranges and the split-K reduction are shared with it
// (bcq_pipeline.cuh).
#pragma once

#include <cstdint>

#include "bcq_device.cuh"
#include "bcq_layout.h"
#include "bcq_pipeline.cuh"

namespace bcq {

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t funnel_r(uint32_t lo, uint32_t hi, uint32_t sh) {
  uint32_t d;
  asm("shf.r.clamp.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(lo), "r"(hi), "r"(sh));
  return d;
}

// a ^ (~b & c) in one instruction.
__device__ __forceinline__ uint32_t xor_andnot(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xD2;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Lane l of a warp copies row l's scales (2P halves: pass 0 then pass 1) and
// offsets (2 halves) of unit (kb, rb) into buf: alpha at l * 4P bytes, z at
// 128P + 4l.  Packed layouts: bcq_layout.h.
// (MIXED: the scales of every precision q present, each into its own block
// of the buffer, see mma_scale_buf_bytes.)
template <int Q>
__device__ __forceinline__ void stage_alpha_q(const uint16_t* a, uint32_t da) {
  if (Q == 1) {
    cp_async4(da, a);
  } else if (Q == 2) {
    cp_async8(da, a);
  } else if (Q == 3) {
    cp_async4(da, a);
    cp_async4(da + 4u, a + 2);
    cp_async4(da + 8u, a + 4);
  } else {
    cp_async16(da, a);
  }
}

template <int P, bool MIXED = false>
__device__ __forceinline__ void stage_scales(const GemvParams& prm, int kb, int rb, int lane,
                                             uint32_t buf) {
  const size_t e = ((size_t)kb * prm.RB + rb) * kRowBlock + lane;
  if constexpr (MIXED) {
    if (prm.qmask & 2) stage_alpha_q<1>(prm.alpha_q[0] + e * 2, buf + mma_alpha_block(1) + 4u * lane);
    if (prm.qmask & 4) stage_alpha_q<2>(prm.alpha_q[1] + e * 4, buf + mma_alpha_block(2) + 8u * lane);
    if (prm.qmask & 8) stage_alpha_q<3>(prm.alpha_q[2] + e * 6, buf + mma_alpha_block(3) + 12u * lane);
    if (prm.qmask & 16) stage_alpha_q<4>(prm.alpha_q[3] + e * 8, buf + mma_alpha_block(4) + 16u * lane);
#pragma unroll
    for (int q = 1; q <= 4; ++q)
      if (((prm.qmask >> q) & 1) && prm.z_q[q - 1])
        cp_async4(buf + mma_z_off(P, true, q) + 4u * lane, prm.z_q[q - 1] + e * 2);
    return;
  }
  const uint16_t* a = prm.alpha[0] + e * (2 * P);
  const uint32_t da = buf + (uint32_t)lane * (4u * P);
  if (P == 1) {
    cp_async4(da, a);
  } else if (P == 2) {
    cp_async8(da, a);
  } else if (P == 3) {
    cp_async4(da, a);
    cp_async4(da + 4u, a + 2);
    cp_async4(da + 8u, a + 4);
  } else {
    cp_async16(da, a);
  }
  if (prm.z) cp_async4(buf + 128u * P + 4u * lane, prm.z + e * 2);
}

// The 16-row activation tile of K-block kb into slot (kb & 1), rows beyond
// the launch's M zero, and its group sums gs[slot][m][h].  All 16 consumer
// warps: warp w loads row w (lane l: columns 8l .. 8l + 7).
__device__ __forceinline__ void load_x_tile(const GemvParams& prm, int kb, int warp, int lane,
                                            uint4& v) {
  const int k = kb * kKBlock + lane * 8;
  v = make_uint4(0u, 0u, 0u, 0u);
  if (warp < prm.M && k < prm.K) {
    const uint16_t* p = prm.x + (size_t)prm.rows[warp] * prm.K + k;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
  }
}

// The same row's columns of K-block kb, prefetched into L2 only.
__device__ __forceinline__ void prefetch_x_tile(const GemvParams& prm, int kb, int warp, int lane) {
  const int k = kb * kKBlock + lane * 8;
  if (warp < prm.M && k < prm.K)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(prm.x + (size_t)prm.rows[warp] * prm.K + k));
}

// Position of column c (0..255) of a K-block in the tile's K order: inside
// each 32-column word U of group h, the natural word of a weight row holds
// column c at stored bit b (bytes rotated: b = 8 (c / 8) + (c + 7) mod 8),
// and fragment register s = 8 t + i (k-step 2 U + t, k-pair i) holds bits
// 15 - s (its low half, k = 2i) and 31 - s (high half, k = 2i + 1).
__host__ __device__ __forceinline__ int mma_k_position(int c) {
  const int h = c >> 7, U = (c >> 5) & 3, cw = c & 31;
  const int b = (cw & ~7) | ((cw + 7) & 7);
  const int e = b >> 4;
  const int s = (e ? 31 : 15) - b;
  return h * 128 + (2 * U + (s >> 3)) * 16 + 2 * (s & 7) + e;
}


// Byte offset of tile K position kpos (mma_k_position) of launch row n in the
// fragment-ordered activation tile.  For group h, natural word v of the group
// (its k-steps 2v and 2v + 1), n-tile n / 8 and lane 4 (n % 8) + q, 16 bytes
// hold that thread's B fragments of k-step 2v and then of k-step 2v + 1 (b0:
// k-pair q of the k-step, b1: k-pair q + 4), so one 16-byte load, free of
// bank conflicts across the warp, gives a thread the fragments of two k-steps.
__host__ __device__ __forceinline__ uint32_t xtile_offset(int n, int kpos) {
  const int h = kpos >> 7, s8 = (kpos >> 4) & 7, kk = kpos & 15;
  const int v = s8 >> 1, odd = s8 & 1;
  const int q = (kk >> 1) & 3, reg = kk >> 3, half = kk & 1;
  return (uint32_t)((((h * 4 + v) * 2 + (n >> 3)) * 32 + (n & 7) * 4 + q) * 16 +
                    (odd * 2 + reg) * 4 + half * 2);
}

// Where column 8l + e8 of a K-block goes in the fragment-ordered tile
// (xtile_offset of its mma_k_position), written out for a lane: with j = l % 4
// the column's stored bit is b = 8j + (e8 + 7) mod 8, its register index
// s = (j odd ? 7 : 15) - (e8 + 7) mod 8, and its byte offset is
//   base(n, l) + (s mod 4) * 16 + (s / 8) * 8 + ((s / 4) mod 2) * 4
// with base(n, l) = ((((l / 16) * 4 + (l / 4) % 4) * 2 + n / 8) * 32 + (n % 8) * 4) * 16
// + 2 ((l / 2) % 2).  For odd j every such offset is 8 bytes below the even
// one, so the lane's base takes - 8 (l % 2) and the eight offsets are
// compile-time constants (checked against xtile_offset for every n, l, e8).
__host__ __device__ constexpr uint32_t xtile_col_off(int e8) {
  return (uint32_t)(((15 - ((e8 + 7) & 7)) & 3) * 16 + ((15 - ((e8 + 7) & 7)) >> 3) * 8 +
                    (((15 - ((e8 + 7) & 7)) >> 2) & 1) * 4);
}
template <uint32_t OFF>
__device__ __forceinline__ void sts_u16_at(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u16 [%0+%1], %2;" ::"r"(addr), "n"(OFF), "h"((unsigned short)v)
               : "memory");
}
template <int E8>
struct XTileCols {
  static __device__ __forceinline__ void run(uint32_t base, const uint32_t (&w)[4]) {
    sts_u16_at<xtile_col_off(E8)>(base, (w[E8 >> 1] >> (16 * (E8 & 1))) & 0xFFFFu);
    XTileCols<E8 + 1>::run(base, w);
  }
};
template <>
struct XTileCols<8> {
  static __device__ __forceinline__ void run(uint32_t, const uint32_t (&)[4]) {}
};

// Launch row `warp` of K-block kb's activation tile into slot kb & 1: lane l
// holds columns 8l .. 8l + 7 (v), each stored at its place in the fragment
// order (xtile_offset of its tile K position, in the closed form above);
// also the row's group sums.
__device__ __forceinline__ void store_x_tile(uint32_t sbase, int kb, int warp, int lane,
                                             const uint4& v) {
  const uint32_t slot = (uint32_t)(kb & 1);
  const uint32_t t = sbase + slot * kXTileBytes;
  const int h = lane >> 4, U = (lane >> 2) & 3, e = (lane >> 1) & 1;
  const uint32_t base = t + (uint32_t)(((((h * 4 + U) * 2 + (warp >> 3)) * 32 + (warp & 7) * 4) * 16) + e * 2) -
                        8u * (uint32_t)(lane & 1);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  XTileCols<0>::run(base, w);
  float f[8];
  unpack8(v, f);
  float s = ((f[0] + f[1]) + (f[2] + f[3])) + ((f[4] + f[5]) + (f[6] + f[7]));
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if ((lane & 15) == 0)  // lane 0: group A, lane 16: group B
    sts_f32(sbase + kMmaGsumOff + ((slot * kMmaRows + warp) * 2 + (lane >> 4)) * 4u, s);
}

// x * y, asked for as an integer multiply (the FMA pipe) rather than a
// shift (the ALU pipe, which the fragment lop3s keep busy).
__device__ __forceinline__ uint32_t mul_lo(uint32_t x, uint32_t y) {
  uint32_t d;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(d) : "r"(x), "r"(y));
  return d;
}

// Tagged partial store (see st_partial) when pred is set, as one predicated
// instruction rather than a branch.
__device__ __forceinline__ void st_partial_if(float* p, float v, int pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t"
      "@q st.relaxed.gpu.global.u32 [%0], %1;\n\t}" ::"l"(p),
      "r"(~__float_as_uint(v)), "r"(pred)
      : "memory");
}

// A shared-memory load at byte offset `off` of the dynamic shared memory, as
// a plain load (the compiler folds constant parts of the offset into the
// instruction).  The callers read ring stages only after waiting on their
// barriers, which are compiler memory barriers too.
template <typename T>
__device__ __forceinline__ T sld(const unsigned char* sm, uint32_t off) {
  return *reinterpret_cast<const T*>(sm + off);
}

// One plane i of one group h of this warp's row-block: both 16-row tiles, the
// group's 8 k-steps, every n-tile.  Thread (g = lane / 4, q = lane % 4) holds
// weight rows g, g + 8, g + 16, g + 24.
//
// Offsets (bytes, from the dynamic shared memory base sm): wa[e][v] of the
// stored word that begins natural word v of row g (e = 0) or g + 8 (e = 1) in
// plane i, pass 0; bx of this lane's B fragments in the K-block's tile; sa of
// the alpha of row g in the warp's scale buffer sbuf.  The packed bytes of row
// r are rotated by r mod 16 (bcq_layout.h): natural 4-byte word v of a pass
// (chunks 4v .. 4v + 3) is the funnel shift, by dsh bits, of the stored words
// (v - R) mod 4 and (v - R + 1) mod 4, R and dsh constants of the thread's
// rows (rows g + 16 and g + 24 rotate as g and g + 8; passes are 512 bytes
// apart, rows 16 apart).  In the tile's K order (mma_k_position) fragment
// register s = 8 t + k-pair of a row and word v (k-step 2v + t) holds the
// word's bits 15 - s and 31 - s: (word << s) with every other bit masked,
// turned into +-alpha by xoring the fp16 sign bits of alpha2 (one lop3).
// Thread q needs k-pairs q and q + 4 of each k-step.
// MIXED: the rows of the launch have precisions of their own (qm[nt][c]:
// activation row nt * 8 + 2q + c, 0 past the launch's rows).  The fragments
// then hold +-1 (exact), the (plane, group) product is accumulated apart and
// folded into acc with alpha^(qm)[row][group][i] of each activation row
// (zero for a plane i >= qm): the same sum, with each row's own scales.
template <int NT, int P, bool MIXED>
__device__ __forceinline__ void mma_group_plane(const unsigned char* sm, const uint32_t (&wa)[2][4],
                                                uint32_t bx, uint32_t sbuf, uint32_t sa, int i, int h,
                                                int g, int q, uint32_t dsh, float (&acc)[2][NT][4],
                                                const int (&qm)[NT][2]) {
  const uint32_t mq0 = 1u << q, mq4 = 1u << (q + 4), mq8 = 1u << (q + 8), mq12 = 1u << (q + 12);
  uint32_t nw[4][4];
  uint32_t al[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int pass = (j >> 1) ^ h;  // rows >= 16 hold group A in pass 1
    const uint32_t o = (uint32_t)(pass * 512 + (j >> 1) * 256);
    uint32_t w[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) w[v] = sld<uint32_t>(sm, wa[j & 1][v] + o);
#pragma unroll
    for (int v = 0; v < 4; ++v) nw[j][v] = funnel_r(w[v], w[(v + 1) & 3], dsh);
    if constexpr (MIXED) {
      al[j] = 0x3C003C00u;
    } else {  // alpha of (row g + 8 j, group h, plane i) in both halves
      const uint32_t ah = sld<uint16_t>(sm, sa + (uint32_t)(8 * j * 4 * P + pass * 2 * P) + 2u * (uint32_t)i);
      al[j] = prmt(ah, 0u, 0x1010u);
    }
  }
  float tmp[2][NT][4];  // MIXED: this (plane, group) alone
  if constexpr (MIXED) {
#pragma unroll
    for (int f = 0; f < 2; ++f)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) tmp[f][nt][e] = 0.f;
  }
#pragma unroll
  for (int v = 0; v < 4; ++v) {  // word v of group h: k-steps 2v, 2v + 1
    uint4 bq[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) bq[nt] = sld<uint4>(sm, bx + (uint32_t)(((h * 4 + v) * 2 + nt) * 512));
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      uint32_t a[4][2];  // row j: k-pairs q (register 8t + q) and q + 4
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        a[j][0] = xor_andnot(al[j], mul_lo(nw[j][v], t ? mq8 : mq0), 0x80008000u);
        a[j][1] = xor_andnot(al[j], mul_lo(nw[j][v], t ? mq12 : mq4), 0x80008000u);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t b0 = t ? bq[nt].z : bq[nt].x, b1 = t ? bq[nt].w : bq[nt].y;
        // tile f: rows 16 f + g (j = 2f) and 16 f + g + 8 (j = 2f + 1)
        mma_16816(MIXED ? tmp[0][nt] : acc[0][nt], a[0][0], a[1][0], a[0][1], a[1][1], b0, b1);
        mma_16816(MIXED ? tmp[1][nt] : acc[1][nt], a[2][0], a[3][0], a[2][1], a[3][1], b0, b1);
      }
    }
  }
  if constexpr (MIXED) {
    // fold: element e of tile f is weight row 16 f + g + 8 (e / 2) and
    // activation row nt * 8 + 2q + (e % 2)
#pragma unroll
    for (int f = 0; f < 2; ++f)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = 16 * f + g + 8 * hr;
        const int pass = (r >> 4) ^ h;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int qv = qm[nt][c];
            float al2 = 0.f;
            if (i < qv)
              al2 = h2f(sld<uint16_t>(sm, sbuf + mma_alpha_block(qv) +
                                      ((uint32_t)r * 2u * qv + (uint32_t)pass * qv + i) * 2u));
            acc[f][nt][2 * hr + c] = fmaf(al2, tmp[f][nt][2 * hr + c], acc[f][nt][2 * hr + c]);
          }
      }
  }
}

// One CTA per SM, the same units, groups, ring and teams as the lookup
// kernel: warps 0..15 consume in two teams of 8 that take alternate groups
// (team warp w: row-block rb0 + w of the stage), NP producer warps stream
// the planes.  Each K-block's activation tile is loaded by all 16 warps
// (slot kb & 1) between the same kind of barriers as the table build.
//   NT  n-tiles of 8 activation rows (M <= 8 NT), P  planes (one precision)
//   MIXED  the rows have precisions of their own (P: the largest)
template <int NT, int P, bool MIXED = false>
__global__ void __launch_bounds__(32 * (kConsumerWarps + 2), 1)
    gemv_mma_kernel(const __grid_constant__ GemvParams prm) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int D = prm.D, NP = prm.NP, RB = prm.RB;
  constexpr uint32_t kStage = gemv_stage_bytes(P);
  const uint32_t ring = sbase + mma_ring_off(P, MIXED);
  const uint32_t full0 = sbase + mma_off_bar(D, P, MIXED);
  const uint32_t empty0 = full0 + 8u * (uint32_t)D;
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(smem + mma_off_bar(D, P, MIXED) + 16u * D);
  constexpr int kConsumers = kConsumerWarps * 32;

  const bool cfg_ok = D >= 2 && D <= kMaxStages && NP >= 1 && NP <= 2 && (D & 1) == 0 &&
                      prm.M >= 1 && prm.M <= 8 * NT &&
                      (int)blockDim.x == 32 * (kConsumerWarps + NP);
  CtaRange R;
  make_range(prm, R);
  uint4 xv;  // consumers: the first activation tile's row, first of all
  if (warp < kConsumerWarps) {
    grid_dependency_wait();
    load_x_tile(prm, R.kb0, warp, lane, xv);
  }
  if (warp == 0) {
    if (cfg_ok && lane < D) {
      mbar_init(full0 + 8u * lane, 1);
      mbar_init(empty0 + 8u * lane, kTeamWarps);
    }
    if (lane == 0) {
      *abort_flag = cfg_ok ? 0 : 1;
      if (!cfg_ok) record_error(&g_device_error, BCQ_ERR_UNSUPPORTED);
    }
    if (cfg_ok) fence_mbar_init();
  }
  __syncthreads();
  launch_dependents();
  if (*abort_flag) return;  // set before the barrier: uniform

  if (warp >= kConsumerWarps) {
    produce_stages<P>(prm, R, warp - kConsumerWarps, lane, ring, full0, empty0, abort_flag);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int team = warp / kTeamWarps;
  const int tw = warp % kTeamWarps;
  const int g = lane >> 2, q = lane & 3;
  // rotation of this thread's rows g and g + 8 (mod 16; see mma_group_plane)
  const uint32_t ra0 = (uint32_t)(((g + 3) >> 2) & 3), ra1 = (uint32_t)(((g + 11) >> 2) & 3);
  const uint32_t dsh = (uint32_t)((-g) & 3) * 8u;
  uint32_t woff[2][4];  // stored word that begins natural word v of row g / g + 8, pass 0
#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int v = 0; v < 4; ++v)
      woff[e][v] = (uint32_t)(g + 8 * e) * 16u + (((uint32_t)v - (e ? ra1 : ra0)) & 3u) * 4u;
  constexpr uint32_t kSbuf = mma_scale_buf_bytes(P, MIXED);
  const uint32_t sbuf0 = sbase + kMmaScaleOff + (uint32_t)warp * 2u * kSbuf;
  const size_t part_stride = (size_t)RB * kRowBlock;
  int qm[NT][2];  // MIXED: precision of this thread's activation rows
  uint32_t mok = 0;  // bit 2 nt + c: activation row nt * 8 + 2q + c is a row of the launch
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int m = nt * 8 + 2 * q + c;
      if (m < prm.M) mok |= 1u << (2 * nt + c);
      qm[nt][c] = MIXED && m < prm.M ? prm.qrow[m] : 0;
    }
  int cur_kb = -1;

  // tiles of every K-block up to kbt, in order, by all 16 warps; the next
  // K-block's activations are prefetched into L2 (no registers held over
  // the main loop)
  auto advance_tiles = [&](int kbt) {
    while (cur_kb < kbt) {
      const int kbn = cur_kb < 0 ? R.kb0 : cur_kb + 1;
      if (cur_kb >= 0) load_x_tile(prm, kbn, warp, lane, xv);
      if (kbn < R.kb_last) prefetch_x_tile(prm, kbn + 1, warp, lane);
      // the slot rebuilt was last read two K-blocks ago, before the previous
      // build's barrier
      store_x_tile(sbase, kbn, warp, lane, xv);
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
  // scales of the team's groups, staged one group ahead (cp.async, two
  // buffers per warp)
  int buf = 0;
  if (gg < R.NG && tw < gc.n) stage_scales<P, MIXED>(prm, gc.kb, gc.rb0 + tw, lane, sbuf0);
  cp_async_commit();

  while (gg < R.NG) {
    advance_tiles(gc.kb);
    const bool active = tw < gc.n;
    const uint32_t sbuf = sbuf0 + (uint32_t)buf * kSbuf;
    // stage the next group's scales into the other buffer, then make sure
    // this group's have landed
    if (gg + 2 < R.NG) {
      GroupCursor pc = gc;
      cursor_next(pc, R.u1, RB);
      cursor_next(pc, R.u1, RB);
      if (tw < pc.n)
        stage_scales<P, MIXED>(prm, pc.kb, pc.rb0 + tw, lane, sbuf0 + (uint32_t)(buf ^ 1) * kSbuf);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncwarp();
    const bool ok = wait_stage(full0 + 8u * s, ph, abort_flag, prm.timeout_ns);
    if (!ok && lane == 0 && *abort_flag == 0) {
      record_error(&g_device_error, BCQ_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    float acc[2][NT][4];  // [16-row tile][n-tile]: both groups, every plane
#pragma unroll
    for (int f = 0; f < 2; ++f)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[f][nt][e] = 0.f;
    if (ok && active) {
      // (offsets from the shared memory base)
      const uint32_t st = ring - sbase + (uint32_t)s * kStage + (uint32_t)tw * kUnitPlaneBytes;
      const uint32_t bx = (uint32_t)(gc.kb & 1) * kXTileBytes + (uint32_t)lane * 16u;
      const uint32_t so = sbuf - sbase;
      const uint32_t sa = so + (uint32_t)g * (4u * P);  // alpha of row g
#pragma unroll 1
      for (int i = 0; i < P; ++i) {
        const uint32_t sp = st + (uint32_t)i * kPlaneGroupBytes;
        uint32_t wa[2][4];
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
          for (int v = 0; v < 4; ++v) wa[e][v] = sp + woff[e][v];
#pragma unroll
        for (int h = 0; h < 2; ++h)
          mma_group_plane<NT, P, MIXED>(smem, wa, bx, so, sa, i, h, g, q, dsh, acc, qm);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive_cta(empty0 + 8u * s);
    if (ok && active && *abort_flag == 0) {
      // offsets: z[row][group] * S[m][group]; then the unit's partial sums
      const uint32_t gsl = kMmaGsumOff + (uint32_t)(gc.kb & 1) * kMmaRows * 8u;
      const uint32_t so = sbuf - sbase;
      float2 sg[NT][2];  // S[m][group 0 / 1] of this thread's activation rows m
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c)
          sg[nt][c] = sld<float2>(smem, gsl + (uint32_t)(nt * 8 + 2 * q + c) * 8u);
      const int row0 = (gc.rb0 + tw) * kRowBlock + g;  // weight row of f = hr = 0
      float* pm[NT][2];
      if (prm.KB > 1) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int c = 0; c < 2; ++c)
            pm[nt][c] = prm.part + ((size_t)gc.kb * prm.M + (nt * 8 + 2 * q + c)) * part_stride +
                        (size_t)row0;
      }
#pragma unroll
      for (int f = 0; f < 2; ++f) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int r = 16 * f + g + 8 * hr;
          // offsets of groups 0 and 1: group h sits in pass (r / 16) ^ h
          float z0 = 0.f, z1 = 0.f;
          if (!MIXED && prm.z) {
            const uint32_t zw = sld<uint32_t>(smem, so + mma_z_off(P) + (uint32_t)r * 4u);
            z0 = h2f((uint16_t)(f ? zw >> 16 : zw & 0xFFFFu));
            z1 = h2f((uint16_t)(f ? zw & 0xFFFFu : zw >> 16));
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if constexpr (MIXED) {  // the offsets of this activation row's precision
                const int qv = qm[nt][c];
                z0 = z1 = 0.f;
                if (qv > 0 && prm.z_q[qv - 1]) {
                  const uint32_t zw = sld<uint32_t>(smem, so + mma_z_off(P, true, qv) + (uint32_t)r * 4u);
                  z0 = h2f((uint16_t)(f ? zw >> 16 : zw & 0xFFFFu));
                  z1 = h2f((uint16_t)(f ? zw & 0xFFFFu : zw >> 16));
                }
              }
              acc[f][nt][2 * hr + c] =
                  fmaf(z0, sg[nt][c].x, fmaf(z1, sg[nt][c].y, acc[f][nt][2 * hr + c]));
            }
          }
        }
      }
      // (one uniform branch around all the stores)
      if (prm.KB > 1) {
#pragma unroll
        for (int f = 0; f < 2; ++f)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int c = 0; c < 2; ++c)
                st_partial_if(pm[nt][c] + (16 * f + 8 * hr), acc[f][nt][2 * hr + c],
                              (int)((mok >> (2 * nt + c)) & 1u));
      } else {
#pragma unroll
        for (int f = 0; f < 2; ++f)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                const int m = nt * 8 + 2 * q + c;
                const int row = row0 + 16 * f + 8 * hr;
                if (((mok >> (2 * nt + c)) & 1u) && row < prm.N)
                  prm.y[(size_t)prm.rows[m] * prm.N + row] = f2h_rn(acc[f][nt][2 * hr + c]);
              }
      }
    }
    buf ^= 1;
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
  advance_tiles(R.kb_last);  // the same barriers in both teams

  // (no barrier: a warp starts its reduction tasks as soon as it is done;
  // the partials it waits for are polled, not counted)
  if (prm.KB > 1) {
    splitk_tail<8>(prm, R, prm.M, prm.rows, tid, kConsumers, abort_flag);
  }
}

}  // namespace bcq
