// bcq_kernels.cu -- sm_100a kernels of libbcq and their launch wrappers.
//
//   pack_planes_kernel   canonical planes -> streaming layout (offline)
//   pack_scales_kernel   per-(row, group) scales/offsets -> streaming order
//   gemv_lut_kernel      producer warps stream plane stages by bulk copy;
//                        consumer warps build the K-block's lookup table,
//                        look up and accumulate, fuse alpha and z, and write
//                        split-K partial sums; the CTA that computed a
//                        row-block's unit in K-block rb mod KB sums its
//                        partials in K order -> fp16 y
//   gemv_m1_kernel       the one-row GEMV (bcq_m1.cuh)
//   lut_dump_kernel      the same table build, written out for inspection
//   wait_probe_kernel    exercises the bounded mbarrier wait
//
// Method (page title, section): "AnyBCQ: Hardware Efficient Flexible
// Binary-Coded Quantization for Multi-Precision LLMs" (Paper-Notes page),
// "关键设计 / 直接bit-plane运算的CUDA内核": load one bit-plane at a time; since
// B_i is +-1 the product with x is additions and subtractions, served from a
// table of cached partial sums; scale by alpha_i, accumulate; output after
// p planes; a p-bit call loads only p planes.  Group size 128, asymmetric
// offset: same page, "训练策略".
#include <cuda_runtime.h>

#include <cstdint>

#include "bcq_device.cuh"
#include "bcq_launch.h"
#include "bcq_layout.h"
#include "bcq_pipeline.cuh"

namespace bcq {


// ============================================================ pack planes

// One thread per packed word; see bcq_layout.h for the layout.
__global__ void pack_planes_kernel(const uint32_t* __restrict__ canon,
                                   uint32_t* __restrict__ packed, int p_H, int N, int K,
                                   int RG, size_t total_words) {
  const int KW = K / 32;
  for (size_t w = blockIdx.x * (size_t)blockDim.x + threadIdx.x; w < total_words;
       w += (size_t)gridDim.x * blockDim.x) {
    const int u = (int)(w & 3);
    const int lane = (int)((w >> 2) & 31);
    const int pass = (int)((w >> 7) & 1);
    size_t rest = w >> 8;
    const int r = (int)(rest % kRowGroup);
    rest /= kRowGroup;
    const int i = (int)(rest % p_H);
    rest /= p_H;
    const size_t rg = rest % RG;
    const size_t kb = rest / RG;
    const size_t rb = rg * kRowGroup + r;
    const size_t n = rb * kRowBlock + lane;
    const int h = (lane >> 4) ^ pass;
    uint32_t out = 0;
    if (n < (size_t)N) {
      const uint32_t* row = canon + ((size_t)i * N + n) * KW;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = (4 * u + j + lane) & 15;
        const size_t cb = kb * 32 + h * 16 + c;  // canonical byte index in the row
        if (cb * 8 < (size_t)K) {
          const uint32_t byte = (row[cb >> 2] >> (8 * (cb & 3))) & 0xFFu;
          out |= (((byte >> 1) | (byte << 7)) & 0xFFu) << (8 * j);  // rotr8(byte, 1)
        }
      }
    }
    packed[w] = out;
  }
}

// ============================================================ pack scales

// One thread per packed half; see bcq_layout.h for the layout.
__global__ void pack_scales_kernel(const uint16_t* __restrict__ src,
                                   uint16_t* __restrict__ dst, int q, int N, int G,
                                   int RB, size_t total) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(e % q);
    const size_t slot = e / q;
    const int pass = (int)(slot & 1);
    const int lane = (int)((slot >> 1) & 31);
    const size_t rest = slot >> 6;
    const size_t rb = rest % RB;
    const size_t kb = rest / RB;
    const size_t n = rb * kRowBlock + lane;
    const size_t g = 2 * kb + ((lane >> 4) ^ pass);
    uint16_t v = 0;
    if (n < (size_t)N && g < (size_t)G) v = src[(n * G + g) * q + i];
    dst[e] = v;
  }
}

// ============================================================ LUT build

// Loads this lane's 8 activations of K-block kb for rows 0..M-1: the chunk
// c = lane % 16 of group h = lane / 16 (zero past K).  x was written before
// this grid started (or by a grid it waited for), so it is read through L2.
// Rows m >= nrows are zero; rowmap (or nullptr: row m) gives the row of x.
template <int M>
__device__ __forceinline__ void load_x(const uint16_t* x, int K, int kb, int lane,
                                       uint4 (&xv)[M], int nrows = M,
                                       const int* rowmap = nullptr) {
  const int k = kb * kKBlock + (lane >> 4) * kGroup + (lane & 15) * 8;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    if (k < K && m < nrows) {
      const uint16_t* p = x + (size_t)(rowmap ? rowmap[m] : m) * K + k;
      asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(xv[m].x), "=r"(xv[m].y), "=r"(xv[m].z), "=r"(xv[m].w)
                   : "l"(p));
    } else {
      xv[m] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

__device__ __forceinline__ void unpack8(const uint4& r, float (&v)[8]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[2 * e] = h2f((uint16_t)(w[e] & 0xFFFFu));
    v[2 * e + 1] = h2f((uint16_t)(w[e] >> 16));
  }
}

// Signed sums of the low nibble: L[lo] = sum_{j<4} (bit_j(lo) ? +v_j : -v_j).
__device__ __forceinline__ void low_sums(const float (&v)[8], float (&L)[16]) {
  const float a3 = v[0] + v[1], a1 = v[0] - v[1];
  const float b3 = v[2] + v[3], b1 = v[2] - v[3];
  const float a[4] = {-a3, a1, -a1, a3};
  const float b[4] = {-b3, b1, -b1, b3};
#pragma unroll
  for (int lo = 0; lo < 16; ++lo) L[lo] = a[lo & 3] + b[lo >> 2];
}

// Signed sum of the high nibble hi over v4..v7.
__device__ __forceinline__ float high_sum(const float (&v)[8], int hi) {
  return (((hi & 1) ? v[4] : -v[4]) + ((hi & 2) ? v[5] : -v[5])) +
         (((hi & 4) ? v[6] : -v[6]) + ((hi & 8) ? v[7] : -v[7]));
}

// Stores entries (hi0 * 16 + lo) (and, with HH = 2, (hi0 * 16 + 16 + lo)),
// lo = LO..15, of one column: offsets are compile-time immediates.
template <int LO, int HH>
struct LutRows1 {
  static __device__ __forceinline__ void run(uint32_t tb, const float (&L)[16], float H0,
                                             float H1) {
    sts_f32_at<(uint32_t)LO * 256u>(tb, L[LO] + H0);
    if (HH > 1) sts_f32_at<(uint32_t)(16 + LO) * 256u>(tb, L[LO] + H1);
    LutRows1<LO + 1, HH>::run(tb, L, H0, H1);
  }
};
template <int HH>
struct LutRows1<16, HH> {
  static __device__ __forceinline__ void run(uint32_t, const float (&)[16], float, float) {}
};

// The same for entry pairs (two activation rows).
template <int LO, int HH>
struct LutRows2 {
  static __device__ __forceinline__ void run(uint32_t tb, const float (&L0)[16],
                                             const float (&L1)[16], float H00, float H01,
                                             float H10, float H11) {
    sts_f32x2_at<(uint32_t)LO * 256u>(tb, L0[LO] + H00, L1[LO] + H10);
    if (HH > 1) sts_f32x2_at<(uint32_t)(16 + LO) * 256u>(tb, L0[LO] + H01, L1[LO] + H11);
    LutRows2<LO + 1, HH>::run(tb, L0, L1, H00, H01, H10, H11);
  }
};
template <int HH>
struct LutRows2<16, HH> {
  static __device__ __forceinline__ void run(uint32_t, const float (&)[16], const float (&)[16],
                                             float, float, float, float) {}
};

// Activations of one chunk in the bit order of a stored plane byte: bit j of
// the stored byte is column (j + 1) mod 8 of the chunk (bcq_layout.h).
__device__ __forceinline__ void unpack8_stored(const uint4& r, float (&v)[8]) {
  float c[8];
  unpack8(r, c);
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = c[(j + 1) & 7];
}

// Builds the pair-layout table of one K-block at shared address lut (layout
// in bcq_layout.h), indexed by the stored byte s: 16 / HH warps of the
// caller each write the entries of high nibbles HH * warp .. HH * warp +
// HH - 1 for all 32 columns (lane = column).  Entry s of a column with
// activations v0..v7 (in stored bit order) is sum_j (2 bit_j(s) - 1) v_j,
// formed as L[s & 15] + H[s >> 4].  Also returns the group sums of this
// lane's pass-0 group (gs[m][0]) and of the other group (gs[m][1]).  The
// caller synchronises before the table is read.
template <int M, int HH>
__device__ __forceinline__ void build_lut(const uint4 (&xv)[M], int slot, uint32_t lut,
                                          int warp, int lane, float (&gs)[M][2]) {
  float v[M][8];
#pragma unroll
  for (int m = 0; m < M; ++m) unpack8_stored(xv[m], v[m]);
  float L[M][16];
#pragma unroll
  for (int m = 0; m < M; ++m) low_sums(v[m], L[m]);
  const int hi0 = warp * HH;
  const int hi1 = HH > 1 ? hi0 + 1 : hi0;
  if (M == 1) {
    const uint32_t tb = lut + (uint32_t)(hi0 * 16) * 256u + (uint32_t)slot * 128u +
                        (uint32_t)lane * 4u;
    LutRows1<0, HH>::run(tb, L[0], high_sum(v[0], hi0), high_sum(v[0], hi1));
  } else {
    const uint32_t tb = lut + (uint32_t)(hi0 * 16) * 256u + (uint32_t)lane * 8u;
    LutRows2<0, HH>::run(tb, L[0], L[M - 1], high_sum(v[0], hi0), high_sum(v[0], hi1),
                         high_sum(v[M - 1], hi0), high_sum(v[M - 1], hi1));
  }
  // group sums: lanes 0-15 hold group A, 16-31 group B
#pragma unroll
  for (int m = 0; m < M; ++m) {
    float s = ((v[m][0] + v[m][1]) + (v[m][2] + v[m][3])) +
              ((v[m][4] + v[m][5]) + (v[m][6] + v[m][7]));
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    gs[m][0] = s;
    gs[m][1] = __shfl_xor_sync(0xFFFFFFFFu, s, 16);
  }
}

// ============================================================ GEMV

// prmt selectors for byte j of a plane word: result byte 0 <- column byte
// (byte j & 1 of the column register), byte 1 <- plane byte j, bytes 2-3 <-
// bytes 2-3 of the column register (zero).  The result is b * 256 + column
// byte, the table offset of entry b of that column.
__device__ __forceinline__ constexpr uint32_t sel_of(int j) {
  return (4u + (uint32_t)(j & 1)) | ((uint32_t)j << 4) | 0x7600u;
}

// Column registers of this lane: cr0[u][q] holds the column bytes of bytes
// 2q and 2q + 1 of word u in pass 0; cr1 the same for pass 1 (other group).
template <int M>
__device__ __forceinline__ void column_regs(int lane, uint32_t (&cr0)[4][2],
                                            uint32_t (&cr1)[4][2]) {
  const uint32_t h0 = (uint32_t)(lane >> 4);
  const uint32_t flip = M == 1 ? 0x4040u : 0x8080u;  // group bit of each byte
#pragma unroll
  for (int u = 0; u < 4; ++u) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t r = 0;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t c = (uint32_t)((4 * u + 2 * q + e + lane) & 15);
        const uint32_t col = h0 * 16u + c;
        r |= (M == 1 ? col * 4u : col * 8u) << (8 * e);
      }
      cr0[u][q] = r;
      cr1[u][q] = r ^ flip;
    }
  }
}

// Sum of the 16 table entries one lane's 16 plane bytes select (M = 1).
__device__ __forceinline__ float plane_sum1(const uint4& w, const uint32_t (&cr)[4][2]) {
  const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      s[j] += lds_f32<kDynBase>(prmt(wd[u], cr[u][j >> 1], sel_of(j)));
  }
  return (s[0] + s[1]) + (s[2] + s[3]);
}

// The same for two activation rows (entries are pairs).
template <uint32_t kBase = kDynBase>
__device__ __forceinline__ void plane_sum2(const uint4& w, const uint32_t (&cr)[4][2],
                                           float& r0, float& r1) {
  const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
  float s0[2] = {0.f, 0.f}, s1[2] = {0.f, 0.f};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 e = lds_f32x2<kBase>(prmt(wd[u], cr[u][j >> 1], sel_of(j)));
      s0[j & 1] += e.x;
      s1[j & 1] += e.y;
    }
  }
  r0 = s0[0] + s0[1];
  r1 = s1[0] + s1[1];
}

// Scales and offsets of one unit for this lane: a[m][r] holds halves
// 2r, 2r + 1 of the lane's 2P values (pass 0: planes 0..P-1, then pass 1);
// z holds the offsets of the pass-0 and pass-1 groups (z1: those of row 1
// when the two rows of a mixed launch take their own offsets).
template <int M, int P>
struct ScaleSet {
  uint32_t a[M][P];
  uint32_t z, z1;
};

template <int M, int P, bool MIXED>
__device__ __forceinline__ void load_scales(const GemvParams& prm, int kb, int rb, int lane,
                                            ScaleSet<M, P>& s) {
  const size_t e = ((size_t)kb * prm.RB + rb) * kRowBlock + lane;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    if (!MIXED) {
      if (m > 0) {
#pragma unroll
        for (int r = 0; r < P; ++r) s.a[m][r] = s.a[0][r];  // same precision, same scales
        continue;
      }
      const uint16_t* a = prm.alpha[0] + e * (2 * P);
      if (P == 1) {
        s.a[m][0] = ldg_nc_u32(a);
      } else if (P == 2) {
        const uint2 r = ldg_nc_v2(a);
        s.a[m][0] = r.x;
        s.a[m][P > 1 ? 1 : 0] = r.y;
      } else if (P == 3) {
#pragma unroll
        for (int r = 0; r < P; ++r) s.a[m][r] = ldg_nc_u32(a + 2 * r);
      } else {
        const uint4 r = ldg_nc_v4(a);
        s.a[m][0] = r.x;
        s.a[m][P > 1 ? 1 : 0] = r.y;
        s.a[m][P > 2 ? 2 : 0] = r.z;
        s.a[m][P > 3 ? 3 : 0] = r.w;
      }
    } else {
      const int q = prm.q[m];
      const uint16_t* a = prm.alpha[m] + e * (size_t)(2 * q);
#pragma unroll
      for (int r = 0; r < P; ++r) s.a[m][r] = 0u;
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
        for (int i = 0; i < P; ++i) {
          const int hidx = pass * P + i;
          const uint32_t v = i < q ? (uint32_t)ldg_nc_u16(a + pass * q + i) : 0u;
          s.a[m][hidx >> 1] |= v << (16 * (hidx & 1));
        }
      }
    }
  }
  s.z = prm.z ? ldg_nc_u32(prm.z + e * 2) : 0u;
  if (MIXED && M == 2) s.z1 = prm.z1 == prm.z ? s.z : (prm.z1 ? ldg_nc_u32(prm.z1 + e * 2) : 0u);
}

template <int M, int P>
__device__ __forceinline__ void zero_scales(ScaleSet<M, P>& s) {
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int r = 0; r < P; ++r) s.a[m][r] = 0u;
  s.z = s.z1 = 0u;
}

__device__ __forceinline__ float half_at(uint32_t r, int hi) {
  return h2f((uint16_t)(hi ? (r >> 16) : (r & 0xFFFFu)));
}


// One CTA per SM: units [u0, u1) of the launch in kb-major order.  Warps
// 0..15 consume, in two teams of 8 that take alternate groups; the NP warps
// after them produce.  Stage g of the CTA holds the P planes of group g
// (plane i at i * 8 KiB, row-block rb0 + w at w KiB); it lands in ring slot
// g mod D and is read by the team of its group (team warp w takes
// row-block rb0 + w).  The teams share the lookup table: each K-block's
// table is built by all 16 warps together.
//   M      activation rows of the launch (1 or 2)
//   P      planes streamed (the largest precision among the rows)
//   MIXED  rows may use precisions below P (scales loaded per row)
template <int M, int P, bool MIXED>
__global__ void __launch_bounds__(32 * (kConsumerWarps + 2), 1)
    gemv_lut_kernel(const __grid_constant__ GemvParams prm) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int D = prm.D, NP = prm.NP, RB = prm.RB;
  constexpr uint32_t kStage = gemv_stage_bytes(P);
  const uint32_t full0 = sbase + gemv_off_bar(D, P, M);
  const uint32_t empty0 = full0 + 8u * (uint32_t)D;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + gemv_off_misc(D, P, M));
  constexpr int kConsumers = kConsumerWarps * 32;

  // The table is addressed through load immediates: the dynamic shared
  // memory must start where they assume.  A stage's team must have consumed
  // the stage D earlier (D even: teams alternate), and each producer refills
  // only its own slots (D a multiple of NP).
  const bool cfg_ok = sbase == kDynBase && D >= 2 && D <= kMaxStages && NP >= 1 && NP <= 2 &&
                      (D & 1) == 0 && (int)blockDim.x == 32 * (kConsumerWarps + NP);
  CtaRange R;
  make_range(prm, R);
  // consumers: activations of the first table first of all (x may come
  // from the preceding grid: wait for it)
  uint4 xv[M];
  if (warp < kConsumerWarps) {
    grid_dependency_wait();
    load_x<M>(prm.x, prm.K, R.kb0, lane, xv, M == 4 ? prm.M : M, M >= 2 ? prm.rows : nullptr);
  }
  if (warp == 0) {
    if (cfg_ok && lane < D) {  // one lane per ring slot
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
    produce_stages<P>(prm, R, warp - kConsumerWarps, lane, sbase + gemv_lut_bytes(M), full0, empty0,
                      abort_flag);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int team = warp / kTeamWarps;
  const int tw = warp % kTeamWarps;  // row-block of a stage
  GroupCursor gc;                    // this team's next group
  cursor_init(gc, R.u0, R.u1, R.kb0, RB);
  uint32_t cr0[4][2], cr1[4][2];
  column_regs<M>(lane, cr0, cr1);
  int cr_slot = 0;
  int cur_kb = -1, xn_kb = -1;
  uint4 xn[M];
  float gs[M][2];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    xn[m] = make_uint4(0u, 0u, 0u, 0u);
    gs[m][0] = gs[m][1] = 0.f;
  }
  int g = team;  // team t takes groups t, t + 2, ...
  if (team) cursor_next(gc, R.u1, RB);
  // ring position of the team's next stage (stage = group; D >= 2)
  int s = team;
  uint32_t ph = 0;
  // Scales and offsets are loaded PF team-groups ahead into pf[j mod PF];
  // the loop is unrolled by PF so no register with a load in flight is
  // ever copied.
  constexpr int PF = 2;
  ScaleSet<M, P> pf[PF];
  GroupCursor pc = gc;
  int gp = g;
#pragma unroll
  for (int j = 0; j < PF; ++j) {
    zero_scales(pf[j]);
    if (gp < R.NG && tw < pc.n) load_scales<M, P, MIXED>(prm, pc.kb, pc.rb0 + tw, lane, pf[j]);
    cursor_next(pc, R.u1, RB);
    cursor_next(pc, R.u1, RB);
    gp += 2;
  }
  const size_t part_stride = (size_t)RB * kRowBlock;
  // Results of a group are used (offset term, store) only after the team's
  // next group has issued its first lookups, so no warp stalls on its own
  // loads: acc[J] / pend*[J] hold the group in slot J until then.
  float acc[PF][M];
  bool pend[PF];
  int pend_row[PF] = {0, 0}, pend_kb[PF] = {0, 0};
  uint32_t pend_z[PF] = {0u, 0u}, pend_z1[PF] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < PF; ++j) pend[j] = false;

  auto finish = [&](auto slot_tag) {
    constexpr int J = decltype(slot_tag)::value;
    if (!pend[J]) return;
    pend[J] = false;
    if (*abort_flag) return;
    float r[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const uint32_t zr = (MIXED && m == 1) ? pend_z1[J] : pend_z[J];
      r[m] = fmaf(half_at(zr, 0), gs[m][0], fmaf(half_at(zr, 1), gs[m][1], acc[J][m]));
    }
    const int row = pend_row[J];
    if (prm.KB > 1) {
#pragma unroll
      for (int m = 0; m < M; ++m)
        if (M < 4 || m < prm.M)
          st_partial(prm.part + ((size_t)pend_kb[J] * (M == 4 ? prm.M : M) + m) * part_stride +
                         (size_t)row,
                     r[m]);
    } else if (row < prm.N) {
#pragma unroll
      for (int m = 0; m < M; ++m)
        if (M < 4 || m < prm.M)
          prm.y[(size_t)(M >= 2 ? prm.rows[m] : m) * prm.N + row] = f2h_rn(r[m]);
    }
  };

  // Tables of every K-block up to kbt, in order; all 16 consumer warps take
  // part in each (the teams meet at the barriers), so both teams go through
  // the same K-blocks even when one has no group in some of them.
  auto advance_tables = [&](int kbt) {
    if (cur_kb >= kbt) return;
    finish(Slot<0>{});  // group sums change with the table
    finish(Slot<1>{});
    while (cur_kb < kbt) {
      const int kbn = cur_kb < 0 ? R.kb0 : cur_kb + 1;
      if (cur_kb >= 0) {
        if (xn_kb == kbn) {
#pragma unroll
          for (int m = 0; m < M; ++m) xv[m] = xn[m];
        } else {
          load_x<M>(prm.x, prm.K, kbn, lane, xv, M == 4 ? prm.M : M, M >= 2 ? prm.rows : nullptr);
        }
      }
      // the next K-block's x is fetched a table ahead (four-row launches
      // load it when needed: its registers would spill in the main loop)
      if (M != 4 && kbn < R.kb_last) {
        load_x<M>(prm.x, prm.K, kbn + 1, lane, xn, M, M >= 2 ? prm.rows : nullptr);
        xn_kb = kbn + 1;
      }
      // M = 2 has one table: every warp must be done with the old one.
      // M = 1 alternates two slots; the one rebuilt was last read two
      // K-blocks ago, before the previous build's barrier.
      if (M >= 2 && cur_kb >= 0) named_barrier_sync(1, kConsumers);
      const int slot = M == 1 ? (kbn & 1) : 0;
      if constexpr (M == 4) {
        // two pair tables: rows 0-1 at the start, rows 2-3 kLutBytes on
        uint4 xa[2] = {xv[0], xv[1]}, xb[2] = {xv[2], xv[3]};
        float ga[2][2], gb[2][2];
        build_lut<2, 1>(xa, 0, sbase, warp, lane, ga);
        build_lut<2, 1>(xb, 0, sbase + kLutBytes, warp, lane, gb);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          gs[0][h] = ga[0][h];
          gs[1][h] = ga[1][h];
          gs[2][h] = gb[0][h];
          gs[3][h] = gb[1][h];
        }
      } else {
        build_lut<M, 1>(xv, slot, sbase, warp, lane, gs);
      }
      if (M == 1 && slot != cr_slot) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            cr0[u][q] ^= 0x8080u;
            cr1[u][q] ^= 0x8080u;
          }
        cr_slot = slot;
      }
      named_barrier_sync(1, kConsumers);
      cur_kb = kbn;
    }
  };

  auto group = [&](auto slot_tag) {
    constexpr int J = decltype(slot_tag)::value;
    constexpr int JP = (J + PF - 1) % PF;  // slot of the team's previous group
    advance_tables(gc.kb);
    const bool active = tw < gc.n;
    const ScaleSet<M, P>& sc = pf[J];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[J][m] = 0.f;
    const bool ok = wait_stage(full0 + 8u * s, ph, abort_flag, prm.timeout_ns);
    if (!ok && lane == 0 && *abort_flag == 0) {
      record_error(&g_device_error, BCQ_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    const bool live = ok && active;
    const uint32_t st = sbase + gemv_lut_bytes(M) + (uint32_t)s * kStage +
                        (uint32_t)tw * kUnitPlaneBytes + (uint32_t)lane * 16u;
    // planes in batches of two: their plane words, then the lookups of both;
    // the stage is released once all its words are in registers
#pragma unroll
    for (int i0 = 0; i0 < P; i0 += 2) {
      constexpr int kB = 2;
      uint4 w[kB][2];
#pragma unroll
      for (int t = 0; t < kB; ++t) {
        if (i0 + t < P && live) {
          w[t][0] = lds_v4(st + (uint32_t)(i0 + t) * kPlaneGroupBytes);
          w[t][1] = lds_v4(st + (uint32_t)(i0 + t) * kPlaneGroupBytes + 512u);
        } else {
          w[t][0] = w[t][1] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (i0 + kB >= P) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cta(empty0 + 8u * s);
      }
#pragma unroll
      for (int t = 0; t < kB; ++t) {
        const int i = i0 + t;
        if (i < P && live) {
          // half (pass * P + i) of the lane's scales of row m
          if constexpr (M == 1) {
            const float p0 = plane_sum1(w[t][0], cr0);
            const float p1 = plane_sum1(w[t][1], cr1);
            acc[J][0] = fmaf(half_at(sc.a[0][i >> 1], i & 1), p0, acc[J][0]);
            acc[J][0] = fmaf(half_at(sc.a[0][(P + i) >> 1], (P + i) & 1), p1, acc[J][0]);
          } else if constexpr (M == 4) {
            // one precision: the scales of row 0 serve every row
            float a0, a1, b0, b1, c0, c1, d0, d1;
            plane_sum2(w[t][0], cr0, a0, a1);
            plane_sum2<kDynBase + kLutBytes>(w[t][0], cr0, c0, c1);
            plane_sum2(w[t][1], cr1, b0, b1);
            plane_sum2<kDynBase + kLutBytes>(w[t][1], cr1, d0, d1);
            const float s0 = half_at(sc.a[0][i >> 1], i & 1);
            const float s1 = half_at(sc.a[0][(P + i) >> 1], (P + i) & 1);
            acc[J][0] = fmaf(s1, b0, fmaf(s0, a0, acc[J][0]));
            acc[J][1] = fmaf(s1, b1, fmaf(s0, a1, acc[J][1]));
            acc[J][2] = fmaf(s1, d0, fmaf(s0, c0, acc[J][2]));
            acc[J][3] = fmaf(s1, d1, fmaf(s0, c1, acc[J][3]));
          } else {
            float a0, a1, b0, b1;
            plane_sum2(w[t][0], cr0, a0, a1);
            plane_sum2(w[t][1], cr1, b0, b1);
            acc[J][0] = fmaf(half_at(sc.a[0][i >> 1], i & 1), a0, acc[J][0]);
            acc[J][0] = fmaf(half_at(sc.a[0][(P + i) >> 1], (P + i) & 1), b0, acc[J][0]);
            acc[J][M - 1] = fmaf(half_at(sc.a[M - 1][i >> 1], i & 1), a1, acc[J][M - 1]);
            acc[J][M - 1] =
                fmaf(half_at(sc.a[M - 1][(P + i) >> 1], (P + i) & 1), b1, acc[J][M - 1]);
          }
        }
      }
      if (i0 == 0) finish(Slot<JP>{});  // the previous group's loads are long done
    }
    pend[J] = active;
    pend_row[J] = (gc.rb0 + tw) * kRowBlock + lane;
    pend_kb[J] = gc.kb;
    pend_z[J] = sc.z;
    if (MIXED) pend_z1[J] = sc.z1;
    // this slot's scales now take the team's group PF ahead
    zero_scales(pf[J]);
    if (gp < R.NG && tw < pc.n) load_scales<M, P, MIXED>(prm, pc.kb, pc.rb0 + tw, lane, pf[J]);
    cursor_next(pc, R.u1, RB);
    cursor_next(pc, R.u1, RB);
    gp += 2;
    // the team's next group is two stages on (D even: no slot is skipped)
    cursor_next(gc, R.u1, RB);
    cursor_next(gc, R.u1, RB);
    s += 2;
    if (s >= D) {
      s -= D;
      ph ^= 1u;
    }
    g += 2;
  };

  while (g < R.NG) {
    group(Slot<0>{});
    if (g < R.NG) group(Slot<1>{});
  }
  finish(Slot<0>{});
  finish(Slot<1>{});
  advance_tables(R.kb_last);  // the same barriers in both teams

  // split-K reduction (a no-op when the launch has one K-block)
  // (no barrier: a warp starts its reduction tasks as soon as it is done;
  // the partials it waits for are polled, not counted)
  if (prm.KB > 1) {
    // (rows: compile-time for one- and two-row launches, so the tail keeps
    // only the loads it needs in registers)
    splitk_tail<M == 1 ? 16 : 8>(prm, R, M == 4 ? prm.M : M, M >= 2 ? prm.rows : nullptr, tid,
                                 kConsumers, abort_flag);
  }
}

}  // namespace bcq

#include "bcq_m1.cuh"
#include "bcq_mma.cuh"
#include "bcq_umma.cuh"

namespace bcq {

// ============================================================ LUT dump

// One CTA per K-block: the table exactly as the GEMV kernels build it (M = 1:
// the one-row kernel's dense table, indexed by the canonical byte; M = 2:
// the pair table, indexed by the stored byte rotr8(b, 1)), read back to
// global memory in the canonical [M][K/8][256] order.
template <int M>
__global__ void __launch_bounds__(256) lut_dump_kernel(const __grid_constant__ LutParams P) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int kb = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint4 xv[M];
  load_x<M>(P.x, P.K, kb, lane, xv);
  float gs[M][2];
  if constexpr (M == 1) {
    build_lut1c<2>(xv[0], sbase, warp, lane, gs[0]);  // 8 warps
  } else {
    build_lut<M, 2>(xv, 0, sbase, warp, lane, gs);
  }
  __syncthreads();
  const int C8 = P.K / 8;
  for (int e = threadIdx.x; e < M * 32 * 256; e += blockDim.x) {
    const int col = e & 31;
    const int b = (e >> 5) & 255;
    const int m = e >> 13;
    const int k = kb * kKBlock + (col >> 4) * kGroup + (col & 15) * 8;
    if (k >= P.K) continue;
    const uint32_t sb = ((uint32_t)b >> 1) | (((uint32_t)b & 1u) << 7);  // stored byte
    const uint32_t a = M == 1 ? sbase + (uint32_t)b * 128u + (uint32_t)col * 4u
                              : sbase + sb * 256u + (uint32_t)col * 8u + (uint32_t)m * 4u;
    P.lut[((size_t)m * C8 + k / 8) * 256 + b] = lds_f32_dyn(a);
  }
  if (P.gsum && warp == 0 && (lane & 15) == 0) {
    const int g = 2 * kb + (lane >> 4);  // lane 0: group A, lane 16: group B
    if (g < P.G) {
#pragma unroll
      for (int m = 0; m < M; ++m) P.gsum[(size_t)m * P.G + g] = gs[m][0];
    }
  }
}

// ============================================================ wait probe

__global__ void wait_probe_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t a = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(a, 1);  // one arrival expected; nothing ever arrives
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(a, 0, limit_ns))
    record_error(&g_device_error, BCQ_ERR_TIMEOUT);
}

// ============================================================ launchers

cudaError_t launch_pack(const uint32_t* canon, uint32_t* packed, int p_H, int N, int K,
                        cudaStream_t st) {
  const size_t KB = ((size_t)K + kKBlock - 1) / kKBlock;
  const int RB = (N + kRowBlock - 1) / kRowBlock;
  const int RG = (RB + kRowGroup - 1) / kRowGroup;
  const size_t total = KB * (size_t)RG * p_H * kRowGroup * kWordsPerUnitPlane;
  const int threads = 256;
  size_t blocks = (total + threads - 1) / threads;
  if (blocks > 148u * 64u) blocks = 148u * 64u;
  pack_planes_kernel<<<(unsigned)blocks, threads, 0, st>>>(canon, packed, p_H, N, K, RG, total);
  return cudaGetLastError();
}

cudaError_t launch_pack_scales(const uint16_t* src, uint16_t* dst, int q, int N, int K,
                               cudaStream_t st) {
  const size_t KB = ((size_t)K + kKBlock - 1) / kKBlock;
  const int G = K / kGroup;
  const int RB = (N + kRowBlock - 1) / kRowBlock;
  const size_t total = KB * (size_t)RB * kRowBlock * 2 * q;
  const int threads = 256;
  size_t blocks = (total + threads - 1) / threads;
  if (blocks > 148u * 64u) blocks = 148u * 64u;
  pack_scales_kernel<<<(unsigned)blocks, threads, 0, st>>>(src, dst, q, N, G, RB, total);
  return cudaGetLastError();
}

GemvKernel gemv_kernel_for(int M, int P, bool mixed) {
  if (M == 1) {
    switch (P) {
      case 1: return gemv_lut_kernel<1, 1, false>;
      case 2: return gemv_lut_kernel<1, 2, false>;
      case 3: return gemv_lut_kernel<1, 3, false>;
      case 4: return gemv_lut_kernel<1, 4, false>;
      default: return nullptr;
    }
  }
  if (M == 4 && !mixed) {
    switch (P) {
      case 1: return gemv_lut_kernel<4, 1, false>;
      case 2: return gemv_lut_kernel<4, 2, false>;
      case 3: return gemv_lut_kernel<4, 3, false>;
      case 4: return gemv_lut_kernel<4, 4, false>;
      default: return nullptr;
    }
  }
  if (M == 2 && !mixed) {
    switch (P) {
      case 1: return gemv_lut_kernel<2, 1, false>;
      case 2: return gemv_lut_kernel<2, 2, false>;
      case 3: return gemv_lut_kernel<2, 3, false>;
      case 4: return gemv_lut_kernel<2, 4, false>;
      default: return nullptr;
    }
  }
  if (M == 2) {
    switch (P) {
      case 2: return gemv_lut_kernel<2, 2, true>;
      case 3: return gemv_lut_kernel<2, 3, true>;
      case 4: return gemv_lut_kernel<2, 4, true>;
      default: return nullptr;
    }
  }
  return nullptr;
}

GemvKernel gemv_m1_kernel_for(int P) {
  switch (P) {
    case 1: return gemv_m1_kernel<1>;
    case 2: return gemv_m1_kernel<2>;
    case 3: return gemv_m1_kernel<3>;
    case 4: return gemv_m1_kernel<4>;
    default: return nullptr;
  }
}

GemvKernel gemv_mma_kernel_for(int NT, int P, bool mixed) {
  if (mixed) {
    if (NT == 1) {
      switch (P) {
        case 2: return gemv_mma_kernel<1, 2, true>;
        case 3: return gemv_mma_kernel<1, 3, true>;
        case 4: return gemv_mma_kernel<1, 4, true>;
        default: return nullptr;
      }
    }
    if (NT == 2) {
      switch (P) {
        case 2: return gemv_mma_kernel<2, 2, true>;
        case 3: return gemv_mma_kernel<2, 3, true>;
        case 4: return gemv_mma_kernel<2, 4, true>;
        default: return nullptr;
      }
    }
    return nullptr;
  }
  if (NT == 1) {
    switch (P) {
      case 1: return gemv_mma_kernel<1, 1>;
      case 2: return gemv_mma_kernel<1, 2>;
      case 3: return gemv_mma_kernel<1, 3>;
      case 4: return gemv_mma_kernel<1, 4>;
      default: return nullptr;
    }
  }
  if (NT == 2) {
    switch (P) {
      case 1: return gemv_mma_kernel<2, 1>;
      case 2: return gemv_mma_kernel<2, 2>;
      case 3: return gemv_mma_kernel<2, 3>;
      case 4: return gemv_mma_kernel<2, 4>;
      default: return nullptr;
    }
  }
  return nullptr;
}

GemvKernel gemv_umma_kernel_for(int P, int NN) {
  if (NN == 16) {
    switch (P) {
      case 1: return gemv_umma_kernel<1, 16>;
      case 2: return gemv_umma_kernel<2, 16>;
      case 3: return gemv_umma_kernel<3, 16>;
      case 4: return gemv_umma_kernel<4, 16>;
      default: return nullptr;
    }
  }
  if (NN == 64) {
    switch (P) {
      case 1: return gemv_umma_kernel<1, 64>;
      case 2: return gemv_umma_kernel<2, 64>;
      case 3: return gemv_umma_kernel<3, 64>;
      case 4: return gemv_umma_kernel<4, 64>;
      default: return nullptr;
    }
  }
  return nullptr;
}

cudaError_t launch_gemv(GemvKernel fn, const GemvParams& p, size_t dyn, bool pdl,
                        cudaStream_t st, int consumer_warps, bool cooperative) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.C, 1, 1);
  cfg.blockDim = dim3((unsigned)(32 * (consumer_warps + p.MW + p.NP)), 1, 1);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cooperative) {  // every CTA resident at once: the split-K tail polls other CTAs
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na].val.cooperative = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, fn, p);
}

cudaError_t blocks_per_sm(GemvKernel fn, int nthreads, size_t dyn, int* out) {
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, fn, nthreads, dyn);
}

cudaError_t launch_lut_dump(const uint16_t* x, int M, int K, float* lut, float* gsum,
                            cudaStream_t st) {
  LutParams p{};
  p.x = x;
  p.lut = lut;
  p.gsum = gsum;
  p.M = M;
  p.K = K;
  p.KB = (K + kKBlock - 1) / kKBlock;
  p.G = K / kGroup;
  const size_t dyn = kLutBytes;
  void (*fn)(LutParams) = nullptr;
  switch (M) {
    case 1: fn = lut_dump_kernel<1>; break;
    case 2: fn = lut_dump_kernel<2>; break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
  if (e != cudaSuccess) return e;
  fn<<<(unsigned)p.KB, 256, dyn, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_wait_probe(unsigned long long limit_ns, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(limit_ns);
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(cudaStream_t st, int* code) {
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return e;
  }
  *code = v;
  return cudaSuccess;
}

}  // namespace bcq
