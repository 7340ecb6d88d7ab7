// bcq_m1.cuh -- the one-row lookup GEMV (included by bcq_kernels.cu only,
// after the table-build helpers it shares with the pair-table kernel).
//
// Method (page title, section): "AnyBCQ: Hardware Efficient Flexible
// Binary-Coded Quantization for Multi-Precision LLMs" (Paper-Notes page),
// "关键设计 / 直接bit-plane运算的CUDA内核": a p-bit call streams only the first p
// bit-planes; each plane's product with x is additions and subtractions of
// cached +-x partial sums (a table per 8-column chunk), scaled by alpha_i and
// accumulated; "训练策略": groups of 128 columns with an asymmetric offset.
//
// Shape of the kernel, for one activation row (decode), one CTA per SM:
//   * producer warps bulk-copy (TMA, 1-D, no multicast, L2 evict-first) the
//     P planes, the scales and the offsets of 8 row-blocks of one K-block
//     into each ring stage (three copies per stage);
//   * 16 consumer warps build the K-block's dense 32 KiB table (entry b of
//     column col at b * 128 + col * 4), then work in two teams of 8 that
//     take alternate stages, one row-block per warp: per plane 32 lookups a
//     lane (prmt-formed addresses), alpha and offset fused in fp32;
//   * split-K over K-blocks: each unit's fp32 partial sums go to the
//     caller's workspace as tagged words; after its main loop each CTA sums
//     the partials of the row-blocks designated to it (splitk_tail: polled,
//     added in K order, fp16 y, cleared), its 16 consumer warps in parallel.
#pragma once

#include <cstdint>

#include "bcq_device.cuh"
#include "bcq_layout.h"
#include "bcq_pipeline.cuh"

namespace bcq {

// ------------------------------------------------------------ table build

// Entries lo = LO..15 of high nibble hi0 (and, HH = 2, hi0 + 1) of one
// column, at compile-time offsets from tb = lut + hi0 * 16 * 128 + col * 4.
template <int LO, int HH>
struct LutRows1c {
  static __device__ __forceinline__ void run(uint32_t tb, const float (&L)[16], float H0,
                                             float H1) {
    sts_f32_at<(uint32_t)LO * 128u>(tb, L[LO] + H0);
    if (HH > 1) sts_f32_at<(uint32_t)(16 + LO) * 128u>(tb, L[LO] + H1);
    LutRows1c<LO + 1, HH>::run(tb, L, H0, H1);
  }
};
template <int HH>
struct LutRows1c<16, HH> {
  static __device__ __forceinline__ void run(uint32_t, const float (&)[16], float, float) {}
};

// The dense table of one K-block (entry b of column col at lut + b * 128 +
// col * 4, b the canonical byte: bit j = column 8c + j), built by 16 / HH
// warps: warp w writes high nibbles HH * w .. HH * w + HH - 1 of all 32
// columns (lane = column, whose 8 activations xv holds).  Also the group
// sums of this lane's pass-0 group (gs[0]) and of the other group (gs[1]).
// The caller synchronises.
template <int HH>
__device__ __forceinline__ void build_lut1c(const uint4& xv, uint32_t lut, int warp, int lane,
                                            float (&gs)[2]) {
  float v[8];
  unpack8(xv, v);
  float L[16];
  low_sums(v, L);
  const int hi0 = HH * warp;
  const uint32_t tb = lut + (uint32_t)(hi0 * 16) * 128u + (uint32_t)lane * 4u;
  LutRows1c<0, HH>::run(tb, L, high_sum(v, hi0), high_sum(v, HH > 1 ? hi0 + 1 : hi0));
  float s = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  gs[0] = s;
  gs[1] = __shfl_xor_sync(0xFFFFFFFFu, s, 16);
}

// ---------------------------------------------------------------- lookups

// prmt selector for byte j: result byte 0 <- byte j of e (sign bit of the
// stored byte and the column byte), byte 1 <- byte j of a (its low 7 bits),
// bytes 2-3 <- the sign of that byte of a (zero).
__device__ __forceinline__ constexpr uint32_t sel1c(int j) {
  return (uint32_t)j | ((uint32_t)(4 + j) << 4) | ((uint32_t)(12 + j) << 8) |
         ((uint32_t)(12 + j) << 12);
}

// (a & b) | c in one instruction.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Column registers: cr[pass][u] holds, in byte j, 4 x the table column of
// byte j of word u in that pass (group (lane / 16) xor pass, chunk
// (4u + j + lane) mod 16): below 128, so bit 7 is free for the sign bit.
__device__ __forceinline__ void m1_column_regs(int lane, uint32_t (&cr)[2][4]) {
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const uint32_t h = (uint32_t)((lane >> 4) ^ pass);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t r = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t c = (uint32_t)((4 * u + j + lane) & 15);
        r |= ((h * 16u + c) * 4u) << (8 * j);
      }
      cr[pass][u] = r;
    }
  }
}

// Sum of the 16 table entries a lane's 16 stored plane bytes select: for
// each word, a = w & 0x7F7F7F7F and e = (w & 0x80808080) | columns; one prmt
// per byte gives (s & 0x7F) * 256 + (s & 0x80) + 4 col = 128 b + 4 col.
__device__ __forceinline__ float plane_sum1c(const uint4& w, const uint32_t (&cr)[4]) {
  const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t a = wd[u] & 0x7F7F7F7Fu;
    const uint32_t e = and_or(wd[u], 0x80808080u, cr[u]);
#pragma unroll
    for (int j = 0; j < 4; ++j) s[j] += lds_f32<kDynBase>(prmt(e, a, sel1c(j)));
  }
  return (s[0] + s[1]) + (s[2] + s[3]);
}

// ------------------------------------------------------------- producers

// The four producer warps stream every stage k of the CTA (stage k = group
// k: at most 8 row-blocks of one K-block in one row group), each its own
// part: warps 0 and 1 the first half of the planes and the rest at P = 4,
// warp 0 all of them below (one bulk copy for a whole row group, one per
// plane otherwise), warp 2 the packed scales alpha^(P), warp 3 the packed
// offsets (a warp with nothing to copy only arrives).  Each arrives on the stage's full barrier with the bytes it
// copies (four arrivals a phase), so a stage's copies go out at once instead
// of one after another.  A producer cannot run a ring ahead of the others:
// slot s is refilled only after the stage before it was consumed, which
// needed every part.
// Planes, scales and offsets are read once per call: evict-first in L2, so x
// and the workspace stay there.  Lane 0 issues; the warp returns when every
// stage of the last ring has landed (or the CTA gave up).
template <int P>
__device__ __forceinline__ void produce_m1_stages(const GemvParams& prm, const CtaRange& R,
                                                  int pw, int lane, uint32_t ring,
                                                  uint32_t full0, uint32_t empty0,
                                                  volatile int* abort_flag) {
  constexpr uint32_t kStage = m1_stage_bytes(P);
  const int D = prm.D, RB = prm.RB;
  if (!prm.early_weights) grid_dependency_wait();
  // role: 0 / 1 the two halves of the planes (1 unused below four planes),
  // 2 the scales, 3 the offsets
  const int role = m1_producers(P) == 3 && pw >= 1 ? pw + 1 : pw;
  if (lane == 0) {
    const uint64_t pol = evict_first_policy();
    int issued = 0;
    GroupCursor gc;
    cursor_init(gc, R.u0, R.u1, R.kb0, RB);
    int s = 0;
    uint32_t eph = 1;
    for (int k = 0; k < R.NG; ++k) {
      if (k >= D && !mbar_wait_bounded(empty0 + 8u * s, eph, prm.timeout_ns)) {
        record_error(&g_device_error, BCQ_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      if (*abort_flag) break;
      const uint32_t bar = full0 + 8u * s;
      const uint32_t dst = ring + (uint32_t)s * kStage;
      const uint32_t n = (uint32_t)gc.n;
      const size_t unit = (size_t)gc.kb * RB + gc.rb0;  // packed scale unit of row-block rb0
      if (role < 2) {  // planes [i0, i1): the first half of them, or the rest
        constexpr int kHalf = m1_producers(P) == 4 ? P / 2 : P;
        const int i0 = role ? kHalf : 0, i1 = role ? P : kHalf;
        const int rg = gc.rb0 / kRowGroup, r0 = gc.rb0 - rg * kRowGroup;
        const uint32_t* src =
            prm.planes + ((size_t)gc.kb * prm.RG + rg) * prm.p_H * (kRowGroup * kWordsPerUnitPlane);
        mbar_arrive_expect_tx(bar, n * (uint32_t)(i1 - i0) * kUnitPlaneBytes);
        if (i1 > i0 && gc.n == kRowGroup) {
          bulk_g2s_hint(dst + (uint32_t)i0 * kPlaneGroupBytes,
                        src + (size_t)i0 * kRowGroup * kWordsPerUnitPlane,
                        (uint32_t)(i1 - i0) * kPlaneGroupBytes, bar, pol);
        } else {
          for (int i = i0; i < i1; ++i)
            bulk_g2s_hint(dst + (uint32_t)i * kPlaneGroupBytes,
                          src + (size_t)(i * kRowGroup + r0) * kWordsPerUnitPlane,
                          n * kUnitPlaneBytes, bar, pol);
        }
      } else if (role == 2) {
        mbar_arrive_expect_tx(bar, n * 128u * P);
        bulk_g2s_hint(dst + m1_alpha_off(P), prm.alpha[0] + unit * (64u * P), n * 128u * P, bar,
                      pol);
      } else if (prm.z) {
        mbar_arrive_expect_tx(bar, n * 128u);
        bulk_g2s_hint(dst + m1_z_off(P), prm.z + unit * 64u, n * 128u, bar, pol);
      } else {
        mbar_arrive_cta(bar);
      }
      issued = k + 1;
      cursor_next(gc, R.u1, RB);
      if (++s == D) {
        s = 0;
        eph ^= 1u;
      }
    }
    // every copy this warp issued lands before the CTA may exit (the full
    // barriers of the last ring's stages complete only when all parts have)
    for (int s2 = 0; s2 < D && s2 < issued; ++s2) {
      const int klast = issued - 1 - ((issued - 1 - s2) % D);
      (void)mbar_wait_bounded(full0 + 8u * s2, (uint32_t)((klast / D) & 1), prm.timeout_ns);
    }
  }
  __syncwarp();
}

// ----------------------------------------------------------------- kernel

// One CTA per SM over units [u0, u1) (kb-major, host-planned): warps 0..15
// consume in two teams of 8 that take alternate stages (team warp w:
// row-block rb0 + w of the stage), warps 16.. produce (planes, scales,
// offsets of every stage).  P: the precision (planes streamed, scales
// alpha^(P)).
template <int P>
__global__ void __launch_bounds__(32 * (kM1Warps + m1_producers(P)), 1)
    gemv_m1_kernel(const __grid_constant__ GemvParams prm) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int D = prm.D, NP = prm.NP, RB = prm.RB;
  constexpr uint32_t kStage = m1_stage_bytes(P);
  constexpr int kConsumers = kM1Warps * 32;
  const uint32_t ring = sbase + kLut1Bytes;
  const uint32_t full0 = sbase + m1_off_bar(D, P);
  const uint32_t empty0 = full0 + 8u * (uint32_t)D;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + m1_off_misc(D, P));

  // The table is addressed through load immediates: the dynamic shared
  // memory must start where they assume.  A stage's team consumed the stage
  // D earlier (D even: teams alternate); three producers (one part of every
  // stage each).
  const bool cfg_ok = sbase == kDynBase && D >= 2 && D <= kMaxStages && NP == m1_producers(P) &&
                      (D & 1) == 0 && (int)blockDim.x == 32 * (kM1Warps + NP);
  CtaRange R;
  make_range(prm, R);
  if (warp == kM1Warps) {
    if (cfg_ok && lane < D) {  // one lane per ring slot
      mbar_init(full0 + 8u * lane, m1_producers(P));
      mbar_init(empty0 + 8u * lane, kM1TeamWarps);
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

  if (warp >= kM1Warps) {
    produce_m1_stages<P>(prm, R, warp - kM1Warps, lane, ring, full0, empty0, abort_flag);
    return;
  }
  // x, y and the workspace may belong to the preceding grid: wait for it.
  grid_dependency_wait();

  // -------------------------------------------------------------- consumers
  const int team = warp / kM1TeamWarps;
  const int tw = warp % kM1TeamWarps;  // row-block of a stage
  uint4 xv[1], xn[1];
  load_x<1>(prm.x, prm.K, R.kb0, lane, xv);
  int xn_kb = -1;
  if (R.kb0 < R.kb_last) {  // the next K-block's x, a table ahead
    load_x<1>(prm.x, prm.K, R.kb0 + 1, lane, xn);
    xn_kb = R.kb0 + 1;
  }
  uint32_t cr[2][4];
  m1_column_regs(lane, cr);
  float gs[2];
  build_lut1c<1>(xv[0], sbase, warp, lane, gs);
  named_barrier_sync(1, kConsumers);
  int cur_kb = R.kb0;

  // Tables of every K-block up to kbt, in order, built by all 16 consumer
  // warps (one high nibble each) between two barriers; both teams take
  // part in each, so they meet at the same barriers even when one has no
  // stage in some K-block.
  auto advance_tables = [&](int kbt) {
    while (cur_kb < kbt) {
      const int kbn = cur_kb + 1;
      named_barrier_sync(1, kConsumers);  // every warp is done with the old table
      if (xn_kb == kbn) {
        xv[0] = xn[0];
      } else {
        load_x<1>(prm.x, prm.K, kbn, lane, xv);
      }
      if (kbn < R.kb_last) {
        load_x<1>(prm.x, prm.K, kbn + 1, lane, xn);
        xn_kb = kbn + 1;
      }
      build_lut1c<1>(xv[0], sbase, warp, lane, gs);
      named_barrier_sync(1, kConsumers);
      cur_kb = kbn;
    }
  };

  const size_t part_stride = (size_t)RB * kRowBlock;
  const uint16_t* zp = prm.z;
  GroupCursor gc;  // this team's next stage
  cursor_init(gc, R.u0, R.u1, R.kb0, RB);
  if (team) cursor_next(gc, R.u1, RB);
  int s = team;  // ring slot of the team's next stage
  uint32_t ph = 0;

#pragma unroll 1
  for (int g = team; g < R.NG; g += 2) {
    advance_tables(gc.kb);
    const bool active = tw < gc.n;
    const bool ok = __all_sync(0xFFFFFFFFu, wait_stage(full0 + 8u * s, ph, abort_flag, prm.timeout_ns));
    if (!ok && lane == 0 && *abort_flag == 0) {
      record_error(&g_device_error, BCQ_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    const bool live = ok && active;
    const uint32_t st = ring + (uint32_t)s * kStage;
    // the stage's words, scales and offsets of this warp's row-block into
    // registers; then the slot is free for the producer
    uint4 w[P][2];
    uint32_t a[P];
    uint32_t zz = 0u;
    if (live) {
      const uint32_t pw0 = st + (uint32_t)tw * kUnitPlaneBytes + (uint32_t)lane * 16u;
#pragma unroll
      for (int i = 0; i < P; ++i) {
        w[i][0] = lds_v4(pw0 + (uint32_t)i * kPlaneGroupBytes);
        w[i][1] = lds_v4(pw0 + (uint32_t)i * kPlaneGroupBytes + 512u);
      }
      const uint32_t sa = st + m1_alpha_off(P) + (uint32_t)(tw * 32 + lane) * (4u * P);
      if (P == 1) {
        a[0] = lds_u32v(sa);
      } else if (P == 2) {
        const uint2 r = lds_v2u(sa);
        a[0] = r.x;
        a[P > 1 ? 1 : 0] = r.y;
      } else if (P == 3) {
#pragma unroll
        for (int r = 0; r < P; ++r) a[r] = lds_u32v(sa + 4u * r);
      } else {
        const uint4 r = lds_v4(sa);
        a[0] = r.x;
        a[P > 1 ? 1 : 0] = r.y;
        a[P > 2 ? 2 : 0] = r.z;
        a[P > 3 ? 3 : 0] = r.w;
      }
      if (zp) zz = lds_u32v(st + m1_z_off(P) + (uint32_t)(tw * 32 + lane) * 4u);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive_cta(empty0 + 8u * s);
    if (live) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < P; ++i) {
        const float p0 = plane_sum1c(w[i][0], cr[0]);
        const float p1 = plane_sum1c(w[i][1], cr[1]);
        acc = fmaf(half_at(a[i >> 1], i & 1), p0, acc);
        acc = fmaf(half_at(a[(P + i) >> 1], (P + i) & 1), p1, acc);
      }
      acc = fmaf(half_at(zz, 0), gs[0], fmaf(half_at(zz, 1), gs[1], acc));
      const int rb = gc.rb0 + tw;
      const int row = rb * kRowBlock + lane;
      if (prm.KB > 1) {
        st_partial(prm.part + (size_t)gc.kb * part_stride + (size_t)row, acc);
      } else if (row < prm.N) {
        prm.y[row] = f2h_rn(acc);
      }
    }
    cursor_next(gc, R.u1, RB);
    cursor_next(gc, R.u1, RB);
    s += 2;
    if (s >= D) {
      s -= D;
      ph ^= 1u;
    }
  }
  advance_tables(R.kb_last);  // the same barriers in both teams
  // split-K reduction over all 16 consumer warps (a no-op with one K-block)
  if (prm.KB > 1) splitk_tail<16>(prm, R, 1, nullptr, tid, kConsumers, abort_flag);
}

}  // namespace bcq
