// bcq_kernels.cu -- sm_100a kernels of libbcq and their launch wrappers.
//
//   pack_planes_kernel   canonical planes -> streaming layout (offline)
//   pack_scales_kernel   per-(row, group) scales/offsets -> streaming order
//   gemv_lut_kernel      LUT build + plane/scale streaming (producer warp,
//                        bulk copies) + lookup-accumulate + alpha/z fusion +
//                        cluster split-K reduction + fp16 out
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
                                   int N, int K, int RBG, size_t total_words) {
  const int KW = K / 32;
  for (size_t w = blockIdx.x * (size_t)blockDim.x + threadIdx.x; w < total_words;
       w += (size_t)gridDim.x * blockDim.x) {
    const int u = (int)(w & 3);
    const int lane = (int)((w >> 2) & 31);
    const int pass = (int)((w >> 7) & 1);
    const int kbi = (int)((w >> 8) & 1);
    size_t rest = w >> 9;
    const int r = (int)(rest % kRowGroup);
    rest /= kRowGroup;
    const int i = (int)(rest % p_H);
    rest /= p_H;
    const size_t rg = rest % RBG;
    const size_t chunk = rest / RBG;
    const size_t rb = rg * kRowGroup + r;
    const size_t kb = chunk * kChunkBlocks + kbi;
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
          out |= byte << (8 * j);
        }
      }
    }
    packed[w] = out;
  }
}

// ============================================================ pack scales

// One thread per packed half; see bcq_layout.h for the layout.
__global__ void pack_scales_kernel(const uint16_t* __restrict__ src,
                                   uint16_t* __restrict__ dst, int q, int N,
                                   int G, int RBP, size_t total) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(e % q);
    const size_t slot = e / q;
    const int lane = (int)(slot & 31);
    const int pass = (int)((slot >> 5) & 1);
    const int kbi = (int)((slot >> 6) & 1);
    const size_t rest = slot >> 7;
    const size_t rb = rest % RBP;
    const size_t chunk = rest / RBP;
    const size_t n = rb * kRowBlock + lane;
    const size_t g = 2 * (chunk * kChunkBlocks + kbi) + ((lane >> 4) ^ pass);
    uint16_t v = 0;
    if (n < (size_t)N && g < (size_t)G) v = src[(n * G + g) * q + i];
    dst[e] = v;
  }
}

// ============================================================ LUT build

// First 64 KiB boundary of the shared window above the CTA's low region.
__device__ __forceinline__ uint32_t lut_base_of(uint32_t sbase) {
  return (sbase & ~(kLutAlign - 1u)) + kLutAlign;
}

// Shared address of the table of slot s (= m * NKB + kb).
template <int NKB>
__device__ __forceinline__ uint32_t lut_table_addr(uint32_t lut_base, int m, int kbp) {
  const int s = m * NKB + kbp;
  return lut_base + (uint32_t)(s >> 1) * kLutTableBytes + (uint32_t)(s & 1) * 128u;
}

// Builds the tables of K-blocks [kb_first, kb_first + nkb) for the M rows of
// x (fp16 [M][K]) into the LUT at lut_base, and the group sums into
// gsum[m * 2 * NKB + g_local].  Columns beyond K read as zero.  All threads
// of the first nwarps warps take part; the caller synchronises afterwards.
//
// Entry b of a chunk with values x0..x7 is sum_j (2 bit_j(b) - 1) x_j,
// formed as L[b & 15] + H[b >> 4], L from x0..x3 and H from x4..x7.
template <int M, int NKB>
__device__ void build_lut_phase(const uint16_t* __restrict__ x, int K, int KB,
                                int kb_first, int nkb, uint32_t lut_base, float* gsum,
                                int nwarps) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int h = lane >> 4, c = lane & 15;
  const int ntask = M * nkb * 8;  // (m, kb, eighth of the high nibbles)
  for (int t = warp; t < ntask; t += nwarps) {
    const int q8 = t & 7;
    const int mk = t >> 3;
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
    // signed sum of x4..x7 for high nibble hi (computed per hi below)
    const float x4 = v[4], x5 = v[5], x6 = v[6], x7 = v[7];
    float L[16];
#pragma unroll
    for (int lo = 0; lo < 16; ++lo) L[lo] = a[lo & 3] + bb[lo >> 2];
    const uint32_t tab = lut_table_addr<NKB>(lut_base, m, kbp) + (uint32_t)lane * 4u;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int hi = q8 * 2 + hh;
      const float H = ((hi & 1) ? x4 : -x4) + ((hi & 2) ? x5 : -x5) +
                      (((hi & 4) ? x6 : -x6) + ((hi & 8) ? x7 : -x7));
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

// prmt selectors for byte j of a plane word: result byte 0 <- column offset
// (byte j & 1 of the column register), byte 1 <- plane byte j, bytes 2-3 <-
// bytes 2-3 of the column register (the upper half of lut_base).  The result
// is lut_base + b * 256 + column * 4.
__device__ __forceinline__ constexpr uint32_t sel_of(int j) {
  return (4u + (uint32_t)(j & 1)) | ((uint32_t)j << 4) | 0x7600u;
}

template <int M, int KBI, int MM>
struct LutAcc {
  static __device__ __forceinline__ void run(uint32_t a, float (&p)[M]) {
    constexpr int s = MM * kChunkBlocks + KBI;
    constexpr uint32_t off = (uint32_t)(s / 2) * kLutTableBytes + (uint32_t)(s % 2) * 128u;
    p[MM] += lds_f32<off>(a);
    LutAcc<M, KBI, MM + 1>::run(a, p);
  }
};
template <int M, int KBI>
struct LutAcc<M, KBI, M> {
  static __device__ __forceinline__ void run(uint32_t, float (&)[M]) {}
};

// Lookup-accumulate of one pass of one K-block of 32 rows.  planes_at is
// this lane's 16 bytes of plane 0; plane i is plane_stride bytes further.
//   acc[m] += sum_{i < p_load} ae[m][i] * P_i[m]  +  zv * gs[m]
template <int M, int KBI>
__device__ __forceinline__ void unit_body(uint32_t planes_at, uint32_t plane_stride,
                                          int p_load, const uint32_t (&cr)[4][2],
                                          const float (&ae)[M][4], float zv,
                                          const float (&gs)[M], float (&acc)[M]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (i < p_load) {
      const uint4 wv = lds_v4(planes_at + (uint32_t)i * plane_stride);
      const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
      float pa[M], pb[M];
#pragma unroll
      for (int m = 0; m < M; ++m) pa[m] = pb[m] = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
          const uint32_t a0 = prmt(wd[u], cr[u][j >> 1], sel_of(j));
          const uint32_t a1 = prmt(wd[u], cr[u][j >> 1], sel_of(j + 1));
          LutAcc<M, KBI, 0>::run(a0, pa);
          LutAcc<M, KBI, 0>::run(a1, pb);
        }
      }
#pragma unroll
      for (int m = 0; m < M; ++m) acc[m] = fmaf(ae[m][i], pa[m] + pb[m], acc[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < M; ++m) acc[m] = fmaf(zv, gs[m], acc[m]);
}

// Reads q scale values of this lane from a staged span of packed scales.
__device__ __forceinline__ void read_scales(uint32_t at, int q, float (&a)[4]) {
  a[0] = a[1] = a[2] = a[3] = 0.f;
  if (q == 4) {
    uint32_t v0, v1;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v0), "=r"(v1) : "r"(at));
    a[0] = h2f((uint16_t)(v0 & 0xFFFFu));
    a[1] = h2f((uint16_t)(v0 >> 16));
    a[2] = h2f((uint16_t)(v1 & 0xFFFFu));
    a[3] = h2f((uint16_t)(v1 >> 16));
  } else if (q == 2) {
    uint32_t v0;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v0) : "r"(at));
    a[0] = h2f((uint16_t)(v0 & 0xFFFFu));
    a[1] = h2f((uint16_t)(v0 >> 16));
  } else {
    uint16_t h0, h1 = 0, h2 = 0;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h0) : "r"(at));
    if (q == 3) {
      asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h1) : "r"(at + 2u));
      asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h2) : "r"(at + 4u));
    }
    a[0] = h2f(h0);
    a[1] = h2f(h1);
    a[2] = h2f(h2);
  }
}

// Both passes of K-block KBI of the chunk for this warp's row-block j of
// the task staged at st.
template <int M, int KBI>
__device__ __forceinline__ void task_kbi(const GemvParams& P, uint32_t st, int j, int lane,
                                         uint32_t plane_stride, const uint32_t (&cr0)[4][2],
                                         const uint32_t (&cr1)[4][2], const float* gsum,
                                         float (&acc)[M]) {
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int sub = (KBI * 2 + pass) * 32 + lane;
    float ae[M][4];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const int d = P.d_of[m];
      const int q = P.q_of[d];
      read_scales(st + P.st_scale[d] + (uint32_t)(j * 256 * q + sub * q * 2), q, ae[m]);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (i >= P.p_m[m]) ae[m][i] = 0.f;
    }
    float zv = 0.f;
    if (P.has_z) {
      uint16_t zh;
      asm volatile("ld.shared.u16 %0, [%1];"
                   : "=h"(zh)
                   : "r"(st + P.st_scale[2] + (uint32_t)(j * 256 + sub * 2)));
      zv = h2f(zh);
    }
    const int h = (lane >> 4) ^ pass;
    float gs[M];
#pragma unroll
    for (int m = 0; m < M; ++m) gs[m] = gsum[m * 4 + KBI * 2 + h];
    uint32_t cr[4][2];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      cr[u][0] = pass ? cr1[u][0] : cr0[u][0];
      cr[u][1] = pass ? cr1[u][1] : cr0[u][1];
    }
    const uint32_t at = st + (uint32_t)(j * kPlaneChunkBytes + KBI * 1024 +
                                        pass * kUnitBytesPerPlane + lane * 16);
    unit_body<M, KBI>(at, plane_stride, P.p_load, cr, ae, zv, gs, acc);
  }
}

__device__ __forceinline__ void consumer_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Stage s address: offsets with bit 31 set count from the end of the LUT,
// the others from the dynamic shared memory base.
__device__ __forceinline__ uint32_t stage_addr(const GemvParams& P, int s, uint32_t sbase,
                                               uint32_t lut_end) {
  const uint32_t o = P.stage_off[s];
  return (o & 0x80000000u) ? lut_end + (o & 0x7FFFFFFFu) : sbase + o;
}

// One CTA: K-range [c0, c1) in chunks of 512 columns (one LUT phase per chunk)
// times the row-blocks of its cluster.  Warps 0..W-1 consume, warp W produces.
// A task is T consecutive row-blocks of one chunk; its planes, scales and
// offsets arrive by bulk copy in one ring stage; consumer group (task mod G)
// takes it, one row-block per warp.
template <int M>
__global__ void __launch_bounds__(32 * (kMaxConsumerWarps + kMaxProducerWarps), 1)
    gemv_lut_kernel(const __grid_constant__ GemvParams P) {
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int W = P.W, D = P.D, NP = P.NP;
  constexpr int T = kRowGroup;  // row-blocks per task: one per warp of a group
  const int G = W / T;

  const int S = P.S;
  const int rank = (int)(blockIdx.x % (unsigned)S);
  const int cl = (int)(blockIdx.x / (unsigned)S);
  const int rg0 = cl * P.rg_base + (cl < P.rg_rem ? cl : P.rg_rem);
  const int nrg = P.rg_base + (cl < P.rg_rem ? 1 : 0);
  const int rb0 = rg0 * kRowGroup;
  const int nrb = nrg * kRowGroup;
  const int c0 = (int)(((long long)rank * P.KC) / S);
  const int c1 = (int)(((long long)(rank + 1) * P.KC) / S);
  const int nphase = c1 - c0;
  const int ntask = nrg;
  const int ktot = nphase * ntask;

  float* accr = reinterpret_cast<float*>(smem + P.off_acc);    // [M][part_rows]
  float* gsum = reinterpret_cast<float*>(smem + P.off_gsum);   // [M][4]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + P.off_flag);
  const uint32_t full0 = sbase + P.off_bar;                    // D full barriers
  const uint32_t empty0 = full0 + 8u * kMaxStages;             // D empty barriers
  const uint32_t lut_base = lut_base_of(sbase);
  const uint32_t lut_end = lut_base + P.lut_bytes;

  // The LUT and the stages must lie inside this CTA's dynamic shared memory
  // (and a ring depth that is a multiple of the consumer groups: see the
  // stage rule in the planner).
  const uint32_t pad = lut_base - sbase;
  const bool layout_ok = pad >= P.low_bytes && pad + P.lut_bytes <= P.dyn_bytes &&
                         D >= 1 && D <= kMaxStages && NP >= 1 && NP <= kMaxProducerWarps &&
                         D % G == 0 && D % NP == 0 && W % T == 0 && W <= kMaxConsumerWarps;
  const uint32_t recv_bar = full0 + 16u * kMaxStages;
  const int rows_c = nrb * kRowBlock;
  const int own0 = rank * P.own_rows;
  const int own_n = max(0, min(rows_c, own0 + P.own_rows) - own0);
  const int nthreads = (W + NP) * 32;
  if (warp >= W) {
    // ------------------------------------------------------------ producers
    // Producer pw issues tasks k = pw, pw + NP, ... (their stages
    // s = k mod D are its own).  Barrier set-up (one barrier per lane of
    // producer 0) overlaps the consumers' LUT build; everyone waits for it
    // (named barrier 2) before the first barrier access.
    const int pw = warp - W;
    if (pw == 0) {
      if (lane == 0) {
        *abort_flag = layout_ok ? 0 : 1;
        if (!layout_ok) record_error(&g_device_error, BCQ_ERR_UNSUPPORTED);
      }
      if (layout_ok) {
        if (lane < D) {
          mbar_init(full0 + 8u * lane, 1);
          mbar_init(empty0 + 8u * lane, (uint32_t)T);
        }
        if (lane == 31) {
          mbar_init(recv_bar, 1);
          mbar_arrive_expect_tx(recv_bar, (uint32_t)((S - 1) * M * own_n * 4));
        }
        fence_mbar_init();
      }
      __syncwarp();
      asm volatile("bar.arrive 2, %0;" ::"r"(nthreads) : "memory");
    } else {
      asm volatile("bar.sync 2, %0;" ::"r"(nthreads) : "memory");
    }
    if (!P.early_weights) grid_dependency_wait();
    const int nreq = 1 + P.nq + P.has_z;
    const uint32_t stage_bytes = P.stage_bytes;
    int issued = 0;  // one past the last task this producer issued
    for (int k = pw; layout_ok && k < ktot; k += NP) {
      const int s = k % D;
      bool ok = true;
      if (k >= D && lane == 0)
        ok = mbar_wait_bounded(empty0 + 8u * s, (uint32_t)(((k / D) - 1) & 1), P.timeout_ns);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) {
        if (lane == 0) {
          record_error(&g_device_error, BCQ_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      if (*abort_flag) break;
      const int ph = k / ntask;
      const int t = k % ntask;
      const size_t chunk = (size_t)(c0 + ph);
      const size_t rg = (size_t)(rg0 + t);
      const uint32_t dst = stage_addr(P, s, sbase, lut_end);
      if (lane == 0) mbar_arrive_expect_tx(full0 + 8u * s, stage_bytes);
      __syncwarp();
      // one bulk copy per lane, all issued by one instruction: the first
      // p_load planes of the row group (contiguous), the scales of each
      // distinct precision, the offsets
      if (lane < nreq) {
        const void* src;
        uint32_t to, bytes;
        if (lane == 0) {
          src = P.planes + ((chunk * P.RBG + rg) * P.p_H) * (kRowGroup * kPlaneChunkBytes / 4);
          to = 0;
          bytes = (uint32_t)P.p_load * kRowGroup * kPlaneChunkBytes;
        } else if (lane <= P.nq) {
          const int d = lane - 1;
          const int q = P.q_of[d];
          src = P.scale[d] + (chunk * P.RBG + rg) * (512 * q);
          to = P.st_scale[d];
          bytes = 1024u * q;
        } else {
          src = P.scale[2] + (chunk * P.RBG + rg) * 512;
          to = P.st_scale[2];
          bytes = 1024u;
        }
        bulk_g2s(dst + to, src, bytes, full0 + 8u * s);
      }
      issued = k + 1;
    }
    if (P.early_weights) grid_dependency_wait();
    launch_dependents();
    if (S > 1) cluster_arrive_relaxed();  // off the path to the first copies
    // copies still in flight must land before the CTA releases its memory
    if (lane == 0) {
      for (int s = pw; s < D; s += NP) {
        if (s >= issued) break;
        const int klast = issued - 1 - ((issued - 1 - s) % D);
        (void)mbar_wait_bounded(full0 + 8u * s, (uint32_t)((klast / D) & 1), P.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ consumers
    grid_dependency_wait();
    const int grp = warp / T;
    const int j = warp % T;
    // per-lane column registers for the two passes: [u][j/2] holds the column
    // offsets of bytes 2*(j/2), 2*(j/2)+1 and lut_base >> 16
    uint32_t cr0[4][2], cr1[4][2];
    {
      const uint32_t hi = lut_base & 0xFFFF0000u;
      const uint32_t h0 = (uint32_t)(lane >> 4), h1 = h0 ^ 1u;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t r0 = hi, r1 = hi;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const uint32_t c = (uint32_t)((4 * u + 2 * q + e + lane) & 15);
            r0 |= ((h0 * 16u + c) * 4u) << (8 * e);
            r1 |= ((h1 * 16u + c) * 4u) << (8 * e);
          }
          cr0[u][q] = r0;
          cr1[u][q] = r1;
        }
      }
    }
    const uint32_t plane_stride = (uint32_t)T * kPlaneChunkBytes;
    if (nphase == 0) {
      asm volatile("bar.sync 2, %0;" ::"r"(nthreads) : "memory");
      if (S > 1) cluster_arrive_relaxed();
    }
    for (int ph = 0; ph < nphase; ++ph) {
      if (layout_ok)
        build_lut_phase<M, kChunkBlocks>(P.x, P.K, P.KB, (c0 + ph) * kChunkBlocks,
                                         kChunkBlocks, lut_base, gsum, W);
      if (ph == 0) {
        asm volatile("bar.sync 2, %0;" ::"r"(nthreads) : "memory");  // barriers ready
        if (S > 1) cluster_arrive_relaxed();
      }
      consumer_sync(W * 32);
      for (int t = grp; layout_ok && t < ntask; t += G) {
        if (*abort_flag) break;
        const int k = ph * ntask + t;
        const int s = k % D;
        const bool ok = mbar_wait_bounded(full0 + 8u * s, (uint32_t)((k / D) & 1), P.timeout_ns);
        if (!ok) {
          if (lane == 0) {
            record_error(&g_device_error, BCQ_ERR_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
        const int rbl = t * T + j;
        if (rbl < nrb) {
          const uint32_t st = stage_addr(P, s, sbase, lut_end);
          float acc[M];
#pragma unroll
          for (int m = 0; m < M; ++m) acc[m] = 0.f;
          task_kbi<M, 0>(P, st, j, lane, plane_stride, cr0, cr1, gsum, acc);
          task_kbi<M, 1>(P, st, j, lane, plane_stride, cr0, cr1, gsum, acc);
#pragma unroll
          for (int m = 0; m < M; ++m) {
            float* dstp = accr + (size_t)m * P.part_rows + rbl * kRowBlock + lane;
            *dstp = (ph == 0 ? 0.f : *dstp) + acc[m];
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cta(empty0 + 8u * s);
      }
      consumer_sync(W * 32);
    }
  }
  __syncthreads();

  // Split-K reduction over the CTAs of the cluster: rank r finishes rows
  // [r * own_rows, (r + 1) * own_rows) of the cluster.  Every other rank
  // stores its sums for those rows into r's receive buffer (distributed
  // shared memory, counted on r's receive barrier); r adds them in rank
  // order and rounds once to fp16.
  float* recv = reinterpret_cast<float*>(smem + P.off_recv);   // [S][M][own_rows]
  if (S > 1) cluster_wait();  // every CTA of the cluster has its receive barrier ready
  if (S > 1 && layout_ok) {
    for (int e = tid; e < M * rows_c; e += nthreads) {
      const int m = e / rows_c;
      const int rl = e % rows_c;
      const int owner = rl / P.own_rows;
      if (owner == rank) continue;
      const uint32_t slot = smem_u32(recv + ((size_t)rank * M + m) * P.own_rows + (rl - owner * P.own_rows));
      st_async_f32(mapa_shared(slot, (uint32_t)owner), accr[(size_t)m * P.part_rows + rl],
                   mapa_shared(recv_bar, (uint32_t)owner));
    }
    if (layout_ok && !mbar_wait_bounded(recv_bar, 0, P.timeout_ns)) {
      if (tid == 0) record_error(&g_device_error, BCQ_ERR_TIMEOUT);
    }
  }
  for (int e = tid; e < M * own_n; e += nthreads) {
    const int m = e / own_n;
    const int i = e % own_n;
    const int rl = own0 + i;
    const int n = rb0 * kRowBlock + rl;
    if (n >= P.N) continue;
    float sum = 0.f;
    for (int rk = 0; rk < S; ++rk)
      sum += rk == rank ? accr[(size_t)m * P.part_rows + rl]
                        : recv[((size_t)rk * M + m) * P.own_rows + i];
    P.y[(size_t)m * P.N + n] = f2h_rn(sum);
  }
}

// ============================================================ LUT dump

template <int M, int NKB>
__global__ void __launch_bounds__(256, 1) lut_dump_kernel(const __grid_constant__ LutParams P) {
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t sbase = smem_u32(smem);
  float* gsum = reinterpret_cast<float*>(smem);
  const uint32_t lut_base = lut_base_of(sbase);
  if (lut_base - sbase < 64 || lut_base - sbase + 2u * kLutTableBytes > P.dyn_bytes) {
    if (threadIdx.x == 0) record_error(&g_device_error, BCQ_ERR_UNSUPPORTED);
    return;
  }
  const int kb_first = blockIdx.x * NKB;
  const int nkb = min(NKB, P.KB - kb_first);
  build_lut_phase<M, NKB>(P.x, P.K, P.KB, kb_first, nkb, lut_base, gsum,
                          (int)(blockDim.x >> 5));
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
    const float v = lds_f32_dyn(lut_table_addr<NKB>(lut_base, m, kbp) + (uint32_t)b * 256u +
                                (uint32_t)col * 4u);
    P.lut[((size_t)m * C + k / 8) * 256 + b] = v;
  }
  if (P.gsum) {
    for (int e = threadIdx.x; e < M * nkb * 2; e += blockDim.x) {
      const int m = e / (nkb * 2);
      const int gl = e % (nkb * 2);
      const int g = kb_first * 2 + gl;
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
  const size_t KC = ((size_t)KB + kChunkBlocks - 1) / kChunkBlocks;
  const int RB = (N + kRowBlock - 1) / kRowBlock;
  const int RBG = (RB + kRowGroup - 1) / kRowGroup;
  const size_t total = KC * (size_t)RBG * p_H * kRowGroup * kChunkBlocks * kWordsPerPlaneBlock;
  const int threads = 256;
  size_t blocks = (total + threads - 1) / threads;
  if (blocks > 148u * 64u) blocks = 148u * 64u;
  pack_planes_kernel<<<(unsigned)blocks, threads, 0, st>>>(canon, packed, p_H, N, K, RBG, total);
  return cudaGetLastError();
}

cudaError_t launch_pack_scales(const uint16_t* src, uint16_t* dst, int q, int N,
                               int K, cudaStream_t st) {
  const int KB = (K + kKBlock - 1) / kKBlock;
  const size_t KC = ((size_t)KB + kChunkBlocks - 1) / kChunkBlocks;
  const int G = K / kGroup;
  const int RB = (N + kRowBlock - 1) / kRowBlock;
  const int RBP = (RB + kRowGroup - 1) / kRowGroup * kRowGroup;
  const size_t total = KC * (size_t)RBP * 128 * q;
  const int threads = 256;
  size_t blocks = (total + threads - 1) / threads;
  if (blocks > 148u * 64u) blocks = 148u * 64u;
  pack_scales_kernel<<<(unsigned)blocks, threads, 0, st>>>(src, dst, q, N, G, RBP, total);
  return cudaGetLastError();
}

GemvKernel gemv_kernel_for(int M) {
  switch (M) {
    case 1: return gemv_lut_kernel<1>;
    case 2: return gemv_lut_kernel<2>;
    default: return nullptr;
  }
}

cudaError_t launch_gemv(GemvKernel fn, const GemvParams& p, int C, int W,
                        size_t dyn, bool pdl, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(C * p.S), 1, 1);
  cfg.blockDim = dim3((unsigned)(32 * (W + p.NP)), 1, 1);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (p.S > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)p.S;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, fn, p);
}

cudaError_t max_active_clusters(GemvKernel fn, int S, int nthreads, size_t dyn, int* out) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)S, 1, 1);
  cfg.blockDim = dim3((unsigned)nthreads, 1, 1);
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
  const int NKB = 4 / M;  // M * NKB <= 4 -> at most 2 tables of 64 KiB
  const size_t dyn = kLutAlign + 2u * kLutTableBytes;
  p.dyn_bytes = (uint32_t)dyn;
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
