// bcq_kernels.cu -- sm_100a kernels of libbcq and their launch wrappers.
//
//   pack_planes_kernel   canonical planes -> streaming layout (offline)
//   gemv_lut_kernel      LUT build + plane streaming + lookup-accumulate +
//                        alpha/z fusion + cluster split-K reduction + fp16 out
//   lut_dump_kernel      the same LUT build, written out for inspection
//   wait_probe_kernel    exercises the bounded mbarrier wait
//
// Method (page title, section): "AnyBCQ: Hardware Efficient Flexible
// Binary-Coded Quantization for Multi-Precision LLMs" (Paper-Notes page),
// "关键设计 / 直接bit-plane运算的CUDA内核": load one bit-plane at a time; since
// B_i is +-1 the product with x is additions and subtractions, served from a
// table of cached partial sums; scale by alpha_i, accumulate; output after
// p planes; a p-bit call loads only p planes.  Group size 128, asymmetric
// offset: same page, "训练策略".
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bcq_device.cuh"
#include "bcq_launch.h"
#include "bcq_layout.h"

namespace cg = cooperative_groups;

namespace bcq {

// Device error word of this library (one per device): kernels record the
// first problem they hit; bcq_device_error() reads and clears it.
__device__ int g_device_error = 0;

// ============================================================ pack planes

// One thread per packed word; see bcq_layout.h for the layout.
__global__ void pack_planes_kernel(const uint32_t* __restrict__ canon,
                                   uint32_t* __restrict__ packed, int p_H,
                                   int N, int K, int KB, size_t total_words) {
  const int KW = K / 32;
  for (size_t w = blockIdx.x * (size_t)blockDim.x + threadIdx.x; w < total_words;
       w += (size_t)gridDim.x * blockDim.x) {
    const int u = (int)(w & 3);
    const int lane = (int)((w >> 2) & 31);
    const int pass = (int)((w >> 7) & 1);
    size_t rest = w >> 8;
    const int kb = (int)(rest % KB);
    rest /= KB;
    const int i = (int)(rest % p_H);
    const size_t rb = rest / p_H;
    const size_t n = rb * kRowBlock + lane;
    const int h = (lane >> 4) ^ pass;
    uint32_t out = 0;
    if (n < (size_t)N) {
      const uint32_t* row = canon + ((size_t)i * N + n) * KW;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = (4 * u + j + lane) & 15;
        const int cb = kb * 32 + h * 16 + c;  // canonical byte index in the row
        if (cb * 8 < K) {
          const uint32_t byte = (row[cb >> 2] >> (8 * (cb & 3))) & 0xFFu;
          out |= byte << (8 * j);
        }
      }
    }
    packed[w] = out;
  }
}

// ============================================================ LUT build

// Shared address of the table of slot s (= m * NKB + kb).
template <int NKB>
__device__ __forceinline__ uint32_t lut_table_addr(int m, int kbp) {
  const int s = m * NKB + kbp;
  return kLutAbs + (uint32_t)(s >> 1) * kLutTableBytes + (uint32_t)(s & 1) * 128u;
}

// Builds the tables of K-blocks [kb_first, kb_first + nkb) for the M rows of
// x (fp16 [M][K]) into the LUT region, and the group sums into
// gsum[m * 2 * NKB + g_local].  Columns beyond K read as zero.  All threads
// of the CTA take part; the caller synchronises afterwards.
//
// Entry b of a chunk with values x0..x7 is sum_j (2 bit_j(b) - 1) x_j,
// formed as L[b & 15] + H[b >> 4], L from x0..x3 and H from x4..x7.
template <int M, int NKB>
__device__ void build_lut_phase(const uint16_t* __restrict__ x, int K, int KB,
                                int kb_first, int nkb, float* gsum) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int h = lane >> 4, c = lane & 15;
  const int ntask = M * nkb * 4;  // (m, kb, quarter of the high nibbles)
  for (int t = warp; t < ntask; t += nwarps) {
    const int q4 = t & 3;
    const int mk = t >> 2;
    const int m = mk / nkb;
    const int kbp = mk % nkb;
    const int kbg = kb_first + kbp;
    const int k = kbg * kKBlock + h * kGroup + c * 8;
    float v[8];
    if (kbg < KB && k < K) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x + (size_t)m * K + k));
      const uint32_t r[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = h2f((uint16_t)(r[e] & 0xFFFFu));
        v[2 * e + 1] = h2f((uint16_t)(r[e] >> 16));
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
    }
    // signed sums of pairs: index bit 0 -> sign of the first, bit 1 -> second
    const float a3 = v[0] + v[1], a1 = v[0] - v[1];
    const float a[4] = {-a3, a1, -a1, a3};
    const float b3 = v[2] + v[3], b1 = v[2] - v[3];
    const float bb[4] = {-b3, b1, -b1, b3};
    const float c3 = v[4] + v[5], c1 = v[4] - v[5];
    const float cc[4] = {-c3, c1, -c1, c3};
    const float d3 = v[6] + v[7], d1 = v[6] - v[7];
    const float dd[4] = {-d3, d1, -d1, d3};
    float L[16];
#pragma unroll
    for (int lo = 0; lo < 16; ++lo) L[lo] = a[lo & 3] + bb[lo >> 2];
    const uint32_t tab = lut_table_addr<NKB>(m, kbp) + (uint32_t)lane * 4u;
#pragma unroll
    for (int hh = 0; hh < 4; ++hh) {
      const int hi = q4 * 4 + hh;
      const float H = cc[hi & 3] + dd[hi >> 2];
#pragma unroll
      for (int lo = 0; lo < 16; ++lo)
        sts_f32(tab + (uint32_t)(hi * 16 + lo) * 256u, L[lo] + H);
    }
  }
  // group sums: one warp per (m, kb, group half)
  const int ngs = M * nkb * 2;
  for (int t = warp; t < ngs; t += nwarps) {
    const int hh = t & 1;
    const int m = (t >> 1) / nkb;
    const int kbp = (t >> 1) % nkb;
    const int kbg = kb_first + kbp;
    const int k = kbg * kKBlock + hh * kGroup + lane * 4;
    float s = 0.f;
    if (kbg < KB && k < K) {
      const uint2 raw = __ldg(reinterpret_cast<const uint2*>(x + (size_t)m * K + k));
      s = (h2f((uint16_t)(raw.x & 0xFFFFu)) + h2f((uint16_t)(raw.x >> 16))) +
          (h2f((uint16_t)(raw.y & 0xFFFFu)) + h2f((uint16_t)(raw.y >> 16)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if (lane == 0) gsum[m * 2 * NKB + kbp * 2 + hh] = s;
  }
}

// ============================================================ GEMV

// prmt selectors: result byte 0 <- column byte j of the per-lane column
// register, byte 1 <- plane byte j, bytes 2-3 <- sign of the column byte (0).
// The result is the table offset b * 256 + column * 4.  Selectors for
// j = 0..3: 0xCC04, 0xDD15, 0xEE26, 0xFF37.
__device__ __forceinline__ constexpr uint32_t sel_of(int j) { return 0xCC04u + 0x1111u * (uint32_t)j; }

template <int M, int NKB, int KBP, int MM>
struct LutAcc {
  static __device__ __forceinline__ void run(uint32_t a, float (&p)[M]) {
    constexpr int s = MM * NKB + KBP;
    constexpr uint32_t off = kLutAbs + (uint32_t)(s / 2) * kLutTableBytes + (uint32_t)(s % 2) * 128u;
    p[MM] += lds_f32<off>(a);
    LutAcc<M, NKB, KBP, MM + 1>::run(a, p);
  }
};
template <int M, int NKB, int KBP>
struct LutAcc<M, NKB, KBP, M> {
  static __device__ __forceinline__ void run(uint32_t, float (&)[M]) {}
};

// Lookup-accumulate of one unit (one pass of one K-block of 32 rows) for
// K-block KBP of the current phase.  acc[m] receives
//   sum_{i < p_load} ae[m][i] * P_i[m]  +  zv * S[m][group]
template <int M, int NKB, int KBP>
__device__ __forceinline__ void unit_body(uint32_t stage, int p_load,
                                          const uint32_t (&cr)[4],
                                          const float (&ae)[M][4], float zv,
                                          const float (&gs)[M], float (&acc)[M]) {
#pragma unroll
  for (int m = 0; m < M; ++m) acc[m] = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (i < p_load) {
      const uint4 wv = lds_v4(stage + (uint32_t)i * kUnitBytesPerPlane);
      const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
      float pa[M], pb[M];
#pragma unroll
      for (int m = 0; m < M; ++m) pa[m] = pb[m] = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
          const uint32_t a0 = prmt(wd[u], cr[u], sel_of(j));
          const uint32_t a1 = prmt(wd[u], cr[u], sel_of(j + 1));
          LutAcc<M, NKB, KBP, 0>::run(a0, pa);
          LutAcc<M, NKB, KBP, 0>::run(a1, pb);
        }
      }
#pragma unroll
      for (int m = 0; m < M; ++m) acc[m] = fmaf(ae[m][i], pa[m] + pb[m], acc[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < M; ++m) acc[m] = fmaf(zv, gs[m], acc[m]);
}

__device__ __forceinline__ void load_alpha(const uint16_t* __restrict__ p, int q,
                                           float (&a)[4]) {
  a[0] = a[1] = a[2] = a[3] = 0.f;
  if (q == 2) {
    const uint32_t v = __ldg(reinterpret_cast<const unsigned int*>(p));
    a[0] = h2f((uint16_t)(v & 0xFFFFu));
    a[1] = h2f((uint16_t)(v >> 16));
  } else if (q == 4) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    a[0] = h2f((uint16_t)(v.x & 0xFFFFu));
    a[1] = h2f((uint16_t)(v.x >> 16));
    a[2] = h2f((uint16_t)(v.y & 0xFFFFu));
    a[3] = h2f((uint16_t)(v.y >> 16));
  } else {
    const unsigned short* ps = reinterpret_cast<const unsigned short*>(p);
    a[0] = h2f(__ldg(ps));
    if (q == 3) {
      a[1] = h2f(__ldg(ps + 1));
      a[2] = h2f(__ldg(ps + 2));
    }
  }
}

// Position of a warp in its sequence of units.  In phase ph a warp takes the
// units u = warp, warp + W, ...; unit u = (rb_local * nkb_ph + kbp) * 2 + pass.
struct UnitIter {
  int ph, u;
};

struct CtaGeom {
  int nrb, range, nphase, nkb_full, W, warp;
  __device__ __forceinline__ int nkb(int ph) const {
    const int r = range - ph * nkb_full;
    return r < nkb_full ? r : nkb_full;
  }
  __device__ __forceinline__ int units(int ph) const { return nrb * nkb(ph) * 2; }
  __device__ __forceinline__ void normalise(UnitIter& it) const {
    while (it.ph < nphase && it.u >= units(it.ph)) {
      ++it.ph;
      it.u = warp;
    }
  }
  __device__ __forceinline__ UnitIter first() const {
    UnitIter it{0, warp};
    normalise(it);
    return it;
  }
  __device__ __forceinline__ void next(UnitIter& it) const {
    it.u += W;
    normalise(it);
  }
  __device__ __forceinline__ bool valid(const UnitIter& it) const { return it.ph < nphase; }
};

template <int M, int NKB>
__global__ void __launch_bounds__(256, 1) gemv_lut_kernel(const __grid_constant__ GemvParams P) {
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int W = blockDim.x >> 5;

  const int S = P.S;
  const int rank = (int)(blockIdx.x % (unsigned)S);
  const int cl = (int)(blockIdx.x / (unsigned)S);
  const int rb0 = cl * P.rb_base + (cl < P.rb_rem ? cl : P.rb_rem);
  const int nrb = P.rb_base + (cl < P.rb_rem ? 1 : 0);
  const int kb0 = (int)(((long long)rank * P.KB) / S);
  const int kb1 = (int)(((long long)(rank + 1) * P.KB) / S);

  CtaGeom geo;
  geo.nrb = nrb;
  geo.range = kb1 - kb0;
  geo.nkb_full = NKB;
  geo.nphase = (geo.range + NKB - 1) / NKB;
  geo.W = W;
  geo.warp = warp;

  float* part = reinterpret_cast<float*>(smem + P.off_part);
  float* gsum = reinterpret_cast<float*>(smem + P.off_gsum);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + P.off_flag);
  const uint32_t stage_bytes = (uint32_t)P.p_load * kUnitBytesPerPlane;
  const uint32_t ring_w = P.ring_abs + (uint32_t)(warp * P.D) * stage_bytes;
  const uint32_t bar_w = sbase + P.off_bar + (uint32_t)(warp * P.D) * 8u;

  // The LUT sits at a fixed shared address above the low region.
  const bool layout_ok = sbase + P.low_bytes <= kLutAbs;
  if (tid == 0) {
    *abort_flag = layout_ok ? 0 : 1;
    if (!layout_ok) record_error(&g_device_error, BCQ_ERR_UNSUPPORTED);
  }
  if (layout_ok && lane == 0) {
    for (int s = 0; s < P.D; ++s) mbar_init(bar_w + 8u * s, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // per-lane column registers for the two passes (see bcq_layout.h)
  uint32_t cr0[4], cr1[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t r0 = 0, r1 = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t c = (uint32_t)((4 * u + j + lane) & 15);
      const uint32_t h0 = (uint32_t)(lane >> 4), h1 = h0 ^ 1u;
      r0 |= ((h0 * 16u + c) * 4u) << (8 * j);
      r1 |= ((h1 * 16u + c) * 4u) << (8 * j);
    }
    cr0[u] = r0;
    cr1[u] = r1;
  }

  auto issue = [&](const UnitIter& it, int s) {
    const int nk = geo.nkb(it.ph);
    const int rbl = it.u / (2 * nk);
    const int r = it.u % (2 * nk);
    const int kbg = kb0 + it.ph * NKB + (r >> 1);
    const int pass = r & 1;
    const size_t rbg = (size_t)(rb0 + rbl);
    if (lane == 0) {
      const uint32_t bar = bar_w + 8u * s;
      mbar_arrive_expect_tx(bar, stage_bytes);
      const uint32_t dst = ring_w + (uint32_t)s * stage_bytes;
      for (int i = 0; i < P.p_load; ++i) {
        const uint32_t* src = P.planes +
            (((rbg * P.p_H + i) * P.KB + kbg) * kWordsPerPlaneBlock + (size_t)pass * 128);
        bulk_g2s(dst + (uint32_t)i * kUnitBytesPerPlane, src, kUnitBytesPerPlane, bar);
      }
    }
  };

  UnitIter it_issue = geo.first();
  UnitIter it = it_issue;
  int issued = 0, consumed = 0;
  if (layout_ok) {
    for (int s = 0; s < P.D && geo.valid(it_issue); ++s) {
      issue(it_issue, s);
      geo.next(it_issue);
      ++issued;
    }
  }

  for (int ph = 0; ph < geo.nphase; ++ph) {
    if (layout_ok)
      build_lut_phase<M, NKB>(P.x, P.K, P.KB, kb0 + ph * NKB, geo.nkb(ph), gsum);
    __syncthreads();
    while (layout_ok && geo.valid(it) && it.ph == ph) {
      if (*abort_flag) break;
      const int s = consumed % P.D;
      const uint32_t parity = (uint32_t)((consumed / P.D) & 1);
      const int nk = geo.nkb(ph);
      const int rbl = it.u / (2 * nk);
      const int r = it.u % (2 * nk);
      const int kbp = r >> 1;
      const int pass = r & 1;
      const int kbg = kb0 + ph * NKB + kbp;
      const int h = (lane >> 4) ^ pass;
      const int n = (rb0 + rbl) * kRowBlock + lane;
      const int g = 2 * kbg + h;

      // scales and offset of this lane's (row, group); zero outside the matrix
      float ae[M][4];
      float zv = 0.f;
      if (n < P.N && g < P.G) {
        const size_t ng = (size_t)n * P.G + g;
        if (P.z) zv = h2f(__ldg(reinterpret_cast<const unsigned short*>(P.z + ng)));
#pragma unroll
        for (int m = 0; m < M; ++m) {
          if (m > 0 && P.p_m[m] == P.p_m[m - 1]) {
#pragma unroll
            for (int i = 0; i < 4; ++i) ae[m][i] = ae[m - 1][i];
          } else {
            const int q = P.p_m[m];
            load_alpha(P.alpha[q - 1] + ng * q, q, ae[m]);
          }
        }
      } else {
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
          for (int i = 0; i < 4; ++i) ae[m][i] = 0.f;
      }
      float gs[M];
#pragma unroll
      for (int m = 0; m < M; ++m) gs[m] = gsum[m * 2 * NKB + kbp * 2 + h];
      // rows with fewer planes than p_load ignore the extra planes
#pragma unroll
      for (int m = 0; m < M; ++m)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (i >= P.p_m[m]) ae[m][i] = 0.f;

      if (!mbar_wait_bounded(bar_w + 8u * s, parity, P.timeout_ns)) {
        if (lane == 0) {
          record_error(&g_device_error, BCQ_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        __syncwarp();
        break;
      }
      uint32_t cr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) cr[u] = pass ? cr1[u] : cr0[u];
      const uint32_t stage = ring_w + (uint32_t)s * stage_bytes + (uint32_t)lane * 16u;
      float acc[M];
      switch (kbp) {
        case 0: unit_body<M, NKB, 0>(stage, P.p_load, cr, ae, zv, gs, acc); break;
        case 1: if constexpr (NKB > 1) unit_body<M, NKB, 1>(stage, P.p_load, cr, ae, zv, gs, acc); break;
        case 2: if constexpr (NKB > 2) unit_body<M, NKB, 2>(stage, P.p_load, cr, ae, zv, gs, acc); break;
        default: if constexpr (NKB > 3) unit_body<M, NKB, 3>(stage, P.p_load, cr, ae, zv, gs, acc); break;
      }
      const int slot = (ph * NKB + kbp) * 2 + pass;
#pragma unroll
      for (int m = 0; m < M; ++m)
        part[(size_t)(slot * M + m) * P.part_rows + rbl * kRowBlock + lane] = acc[m];
      ++consumed;
      __syncwarp();
      if (geo.valid(it_issue)) {
        fence_proxy_async_smem();
        issue(it_issue, s);
        geo.next(it_issue);
        ++issued;
      }
      geo.next(it);
    }
    __syncthreads();
  }

  // Drain: after an abort, wait (bounded) for copies still in flight before
  // the shared memory is released.
  if (layout_ok) {
    for (int k = consumed; k < issued; ++k)
      (void)mbar_wait_bounded(bar_w + 8u * (k % P.D), (uint32_t)((k / P.D) & 1), P.timeout_ns);
  }

  // Split-K reduction over the CTAs of the cluster (distributed shared
  // memory), then one fp16 rounding per output.
  cg::cluster_group cluster = cg::this_cluster();
  if (S > 1) cluster.sync(); else __syncthreads();
  {
    const int rows_c = nrb * kRowBlock;
    const int chunk = (rows_c + S - 1) / S;
    const int r0 = rank * chunk;
    const int r1 = min(rows_c, r0 + chunk);
    const int nr = r1 - r0;
    for (int e = tid; e < M * nr; e += blockDim.x) {
      const int m = e / nr;
      const int rl = r0 + e % nr;
      const int n = rb0 * kRowBlock + rl;
      if (n >= P.N) continue;
      float sum = 0.f;
      for (int rk = 0; rk < S; ++rk) {
        const float* pr = S > 1 ? cluster.map_shared_rank(part, rk) : part;
        const int a0 = (int)(((long long)rk * P.KB) / S);
        const int a1 = (int)(((long long)(rk + 1) * P.KB) / S);
        const int slots = 2 * (a1 - a0);
        for (int sl = 0; sl < slots; ++sl) sum += pr[(size_t)(sl * M + m) * P.part_rows + rl];
      }
      P.y[(size_t)m * P.N + n] = f2h_rn(sum);
    }
  }
  if (S > 1) cluster.sync();
}

// ============================================================ LUT dump

template <int M, int NKB>
__global__ void __launch_bounds__(256, 1) lut_dump_kernel(const __grid_constant__ LutParams P) {
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  float* gsum = reinterpret_cast<float*>(smem + P.off_gsum);
  if (sbase + P.off_gsum + 64 > kLutAbs) {
    if (threadIdx.x == 0) record_error(&g_device_error, BCQ_ERR_UNSUPPORTED);
    return;
  }
  const int kb_first = blockIdx.x * NKB;
  const int nkb = min(NKB, P.KB - kb_first);
  build_lut_phase<M, NKB>(P.x, P.K, P.KB, kb_first, nkb, gsum);
  __syncthreads();
  const int C = P.K / 8;
  const int total = M * nkb * 32 * 256;
  for (int e = threadIdx.x; e < total; e += blockDim.x) {
    const int col = e & 31;
    const int b = (e >> 5) & 255;
    const int mk = e >> 13;
    const int m = mk / nkb, kbp = mk % nkb;
    const int k = (kb_first + kbp) * kKBlock + (col >> 4) * kGroup + (col & 15) * 8;
    if (k >= P.K) continue;
    const float v = lds_f32_dyn(lut_table_addr<NKB>(m, kbp) + (uint32_t)b * 256u + (uint32_t)col * 4u);
    P.lut[((size_t)m * C + k / 8) * 256 + b] = v;
  }
  if (P.gsum) {
    for (int e = threadIdx.x; e < M * nkb * 2; e += blockDim.x) {
      const int m = e / (nkb * 2);
      const int gl = e % (nkb * 2);
      const int g = (kb_first) * 2 + gl;
      if (g < P.G) P.gsum[(size_t)m * P.G + g] = gsum[m * 2 * NKB + gl];
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
  if (threadIdx.x == 0 && !mbar_wait_bounded(a, 0, limit_ns)) record_error(&g_device_error, BCQ_ERR_TIMEOUT);
}

// ============================================================ launchers

cudaError_t launch_pack(const uint32_t* canon, uint32_t* packed, int p_H, int N,
                        int K, cudaStream_t st) {
  const int KB = (K + kKBlock - 1) / kKBlock;
  const size_t RB = ((size_t)N + kRowBlock - 1) / kRowBlock;
  const size_t total = RB * p_H * KB * kWordsPerPlaneBlock;
  const int threads = 256;
  size_t blocks = (total + threads - 1) / threads;
  if (blocks > 148u * 64u) blocks = 148u * 64u;
  pack_planes_kernel<<<(unsigned)blocks, threads, 0, st>>>(canon, packed, p_H, N, K, KB, total);
  return cudaGetLastError();
}

GemvKernel gemv_kernel_for(int M, int NKB) {
  switch (M * 8 + NKB) {
    case 1 * 8 + 1: return gemv_lut_kernel<1, 1>;
    case 1 * 8 + 2: return gemv_lut_kernel<1, 2>;
    case 1 * 8 + 3: return gemv_lut_kernel<1, 3>;
    case 1 * 8 + 4: return gemv_lut_kernel<1, 4>;
    case 2 * 8 + 1: return gemv_lut_kernel<2, 1>;
    case 2 * 8 + 2: return gemv_lut_kernel<2, 2>;
    case 3 * 8 + 1: return gemv_lut_kernel<3, 1>;
    case 4 * 8 + 1: return gemv_lut_kernel<4, 1>;
    default: return nullptr;
  }
}

cudaError_t launch_gemv(GemvKernel fn, const GemvParams& p, int C, int W,
                        size_t dyn, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(C * p.S), 1, 1);
  cfg.blockDim = dim3((unsigned)(32 * W), 1, 1);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (p.S > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p.S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    na = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, fn, p);
}

cudaError_t max_active_clusters(GemvKernel fn, int S, int W, size_t dyn, int* out) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)S, 1, 1);
  cfg.blockDim = dim3((unsigned)(32 * W), 1, 1);
  cfg.dynamicSmemBytes = dyn;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaOccupancyMaxActiveClusters(out, fn, &cfg);
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
  p.off_gsum = 0;
  const int NKB = 4 / M;  // M * NKB <= 4 -> at most 2 tables of 64 KiB
  const size_t dyn = kLutAbs + 2u * kLutTableBytes;
  const unsigned blocks = (unsigned)((p.KB + NKB - 1) / NKB);
  void (*fn)(LutParams) = nullptr;
  switch (M) {
    case 1: fn = lut_dump_kernel<1, 4>; break;
    case 2: fn = lut_dump_kernel<2, 2>; break;
    case 3: fn = lut_dump_kernel<3, 1>; break;
    case 4: fn = lut_dump_kernel<4, 1>; break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
  if (e != cudaSuccess) return e;
  fn<<<blocks, 256, dyn, st>>>(p);
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
