// bcq_api.cu -- the C ABI of libbcq (include/bcq.h): argument validation,
// launch planning and dispatch.  No device memory is allocated here.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include "bcq.h"
#include "bcq_launch.h"
#include "bcq_layout.h"

namespace bcq {
namespace {

constexpr int kVersion = 100;                // 0.1.0
constexpr size_t kMaxDynSmem = 232448;       // 227 KiB per CTA on sm_100
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int env_int(const char* name, int dflt) {
  const char* v = std::getenv(name);
  if (!v || !*v) return dflt;
  return std::atoi(v);
}

// Per-device facts and per-launch-shape occupancy, cached after the first
// query (callers hold g_mu).
struct OccEntry {
  GemvKernel fn;
  int S, W;
  size_t dyn;
  int clusters;
};
struct DeviceCache {
  bool init = false;
  int sm_count = 0;
  OccEntry occ[64];
  int n_occ = 0;
  GemvKernel attr_done[8] = {};
};
std::mutex g_mu;
DeviceCache g_cache[16];

struct Plan {
  GemvKernel fn = nullptr;
  int M = 0, S = 1, C = 1, W = 8, NP = 2, D = 2;
  size_t dyn = 0;
  GemvParams p{};
  double cost = 1e300;
};

size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

// Shared-memory layout of one candidate (cluster count already chosen);
// false if it does not fit.  Low region (from the dynamic base): running row
// sums [M][rows], group sums, full/empty barriers, abort flag, then as many
// ring stages as fit below the first 64 KiB boundary; then the LUT; then the
// remaining stages.
bool layout(Plan& pl, uint32_t per_rb_bytes, uint32_t scale_q0, uint32_t scale_q1,
            bool has_z, int p_load, int d_max) {
  const int part_rows = kRowBlock * kRowGroup * (pl.p.rg_base + (pl.p.rg_rem > 0 ? 1 : 0));
  const int own_rows = (part_rows + pl.S - 1) / pl.S;
  pl.p.own_rows = own_rows;
  size_t off = 0;
  pl.p.off_acc = (uint32_t)off;
  off = align16(off + (size_t)pl.M * part_rows * sizeof(float));
  pl.p.off_recv = (uint32_t)off;
  off = align16(off + (pl.S > 1 ? (size_t)pl.S * pl.M * own_rows * sizeof(float) : 0));
  pl.p.off_gsum = (uint32_t)off;
  off = align16(off + (size_t)pl.M * 4 * sizeof(float));
  pl.p.off_bar = (uint32_t)off;
  off = align16(off + (2 * kMaxStages + 1) * 8);
  pl.p.off_flag = (uint32_t)off;
  off = align16(off + 16);
  const size_t low_cap = kLutAlign - kLowReserve;
  if (off > low_cap) return false;
  pl.p.part_rows = part_rows;
  const size_t stage = (size_t)kRowGroup * per_rb_bytes;
  pl.p.stage_bytes = (uint32_t)stage;
  // stage sub-spans: planes [p_load][T * 2 KiB], scales of each distinct
  // precision [T * 256 q], offsets [T * 256]
  size_t so = (size_t)p_load * kRowGroup * kPlaneChunkBytes;
  pl.p.st_scale[0] = (uint32_t)so;
  so += (size_t)kRowGroup * 256 * scale_q0;
  pl.p.st_scale[1] = (uint32_t)so;
  so += (size_t)kRowGroup * 256 * scale_q1;
  pl.p.st_scale[2] = (uint32_t)so;
  (void)has_z;
  const size_t lut_bytes = (size_t)((pl.M * kChunkBlocks + 1) / 2) * kLutTableBytes;
  pl.p.lut_bytes = (uint32_t)lut_bytes;
  int D = 0;
  while (D < d_max && off + stage <= low_cap) {
    pl.p.stage_off[D++] = (uint32_t)off;
    off = align16(off + stage);
  }
  pl.p.low_bytes = (uint32_t)off;
  size_t high = 0;
  while (D < d_max && kLutAlign + lut_bytes + high + stage <= kMaxDynSmem) {
    pl.p.stage_off[D++] = 0x80000000u | (uint32_t)high;
    high = align16(high + stage);
  }
  // Task k uses stage k % D and consumer group k % G.  With D a multiple of
  // G the previous task on a stage (k - D) belongs to the same group, which
  // has consumed it before waiting for task k; otherwise a group could test
  // a stage's barrier two phases ahead and read the parity of an old phase.
  // The same holds per producer warp (task k is issued by producer
  // k mod kProducerWarps, which must own stage k mod D).
  const int G = pl.W / kRowGroup;
  int step = G;
  while (step % pl.NP) step += G;  // lcm(G, NP)
  D -= D % step;
  if (D < step || D < 2) return false;
  // stages past D are not used: recompute the high part of the layout
  high = 0;
  size_t low_end = pl.p.off_flag + 16;
  low_end = align16(low_end);
  for (int s = 0; s < D; ++s) {
    if (!(pl.p.stage_off[s] & 0x80000000u)) {
      low_end = std::max<size_t>(low_end, align16(pl.p.stage_off[s] + stage));
    } else {
      high = std::max<size_t>(high, align16((pl.p.stage_off[s] & 0x7FFFFFFFu) + stage));
    }
  }
  pl.p.low_bytes = (uint32_t)low_end;
  pl.D = D;
  pl.dyn = kLutAlign + lut_bytes + high;
  pl.p.dyn_bytes = (uint32_t)pl.dyn;
  return pl.dyn <= kMaxDynSmem;
}

// Plans can be queried without a GPU (bcq_plan_query): they are then made
// for a nominal B200 (148 SMs, one CTA per SM).
DeviceCache g_virtual;
thread_local bool t_virtual = false;

bcq_status get_device(DeviceCache** dc) {
  if (t_virtual) {
    if (!g_virtual.init) {
      g_virtual.sm_count = 148;
      g_virtual.init = true;
    }
    *dc = &g_virtual;
    return BCQ_OK;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BCQ_ERR_CUDA;
  if (dev < 0 || dev >= 16) return BCQ_ERR_UNSUPPORTED;
  DeviceCache& c = g_cache[dev];
  if (!c.init) {
    if (cudaDeviceGetAttribute(&c.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BCQ_ERR_CUDA;
    c.init = true;
  }
  *dc = &c;
  return BCQ_OK;
}

// Clusters of S CTAs (S = 1: single CTAs) of this shape that fit at once.
bcq_status active_clusters(DeviceCache& dc, int ki, GemvKernel fn, int S, int nthreads,
                           size_t dyn, int* out) {
  if (t_virtual) {  // one CTA per SM; clusters of S never straddle
    *out = dyn <= kMaxDynSmem && nthreads <= 1024 ? dc.sm_count / S : 0;
    return BCQ_OK;
  }
  if (dc.attr_done[ki] != fn) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kMaxDynSmem) != cudaSuccess)
      return BCQ_ERR_CUDA;
    dc.attr_done[ki] = fn;
  }
  for (int i = 0; i < dc.n_occ; ++i) {
    const OccEntry& e = dc.occ[i];
    if (e.fn == fn && e.S == S && e.W == nthreads && e.dyn == dyn) {
      *out = e.clusters;
      return BCQ_OK;
    }
  }
  int n = 0;
  if (S == 1) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, nthreads, dyn) != cudaSuccess)
      return BCQ_ERR_CUDA;
    n = per_sm * dc.sm_count;
  } else if (max_active_clusters(fn, S, nthreads, dyn, &n) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  if (dc.n_occ < 64) dc.occ[dc.n_occ++] = OccEntry{fn, S, nthreads, dyn, n};
  *out = n;
  return BCQ_OK;
}

// Chooses the split-K factor S (cluster size, in 512-column chunks), the
// cluster count C, the task size T (row-blocks per task) and the ring depth D
// for one launch of M (1 or 2) activation rows.  The cost model counts
// shared-memory wavefronts per CTA (LUT build: M per column; lookups: M per
// 32 plane bytes; staging: 2 per 128 plane bytes) against the HBM time of the
// whole call, plus a fixed cost per cluster reduction and per chunk.
bcq_status plan_gemv(int M, int N, int K, int p_load, uint32_t per_rb_bytes,
                     uint32_t scale_q0, uint32_t scale_q1, bool has_z, Plan* out) {
  DeviceCache* dc = nullptr;
  bcq_status st = get_device(&dc);
  if (st != BCQ_OK) return st;
  const int KB = (K + kKBlock - 1) / kKBlock;
  const int KC = (KB + kChunkBlocks - 1) / kChunkBlocks;
  const int RB = (N + kRowBlock - 1) / kRowBlock;
  const int RBG = (RB + kRowGroup - 1) / kRowGroup;
  const int force_S = env_int("BCQ_FORCE_S", 0);
  const int force_W = env_int("BCQ_FORCE_W", 0);
  const int force_NP = env_int("BCQ_FORCE_NP", 0);
  const int force_D = env_int("BCQ_FORCE_D", 0);
  const double hbm_bytes_per_clk = 3300.0;  // ~6.5 TB/s at ~1.95 GHz
  const double total_bytes = (double)N * K * p_load / 8.0;  // planes
  GemvKernel fn = gemv_kernel_for(M);
  if (!fn) return BCQ_ERR_UNSUPPORTED;
  const int ki = M - 1;
  Plan best;
  const int S_list[4] = {1, 2, 4, 8};
  // (consumer warps W, producer warps NP); fewer warps only when nothing
  // larger fits
  const int WN_list[6][2] = {{12, 3}, {12, 4}, {8, 2}, {8, 4}, {4, 1}, {4, 2}};
  for (int si = 0; si < 4; ++si) {
    const int S = S_list[si];
    if (force_S && S != force_S) continue;
    if (S > KC) continue;
    const int range_max = (KC + S - 1) / S;  // chunks per CTA
    for (int wi = 0; wi < 6; ++wi) {
      Plan pl;
      pl.M = M;
      pl.S = S;
      pl.fn = fn;
      pl.W = WN_list[wi][0];
      pl.NP = WN_list[wi][1];
      if (force_W && pl.W != force_W) continue;
      if (force_NP && pl.NP != force_NP) continue;
      if (pl.W < 8 && best.fn && best.W >= 8) continue;
      const int nthreads = 32 * (pl.W + pl.NP);
      const int d_max = std::min(kMaxStages, force_D ? force_D : kMaxStages);
      // occupancy with the largest layout this candidate can take
      pl.p.rg_base = std::max(1, RBG / std::max(1, dc->sm_count / S));
      pl.p.rg_rem = 0;
      if (!layout(pl, per_rb_bytes, scale_q0, scale_q1, has_z, p_load, d_max)) continue;
      int C = 0;
      st = active_clusters(*dc, ki, fn, S, nthreads, pl.dyn, &C);
      if (st != BCQ_OK) return st;
      if (C <= 0) continue;
      C = std::min(C, RBG);
      pl.C = C;
      pl.p.rg_base = RBG / C;
      pl.p.rg_rem = RBG % C;
      if (!layout(pl, per_rb_bytes, scale_q0, scale_q1, has_z, p_load, d_max)) continue;
      int C2 = 0;
      st = active_clusters(*dc, ki, fn, S, nthreads, pl.dyn, &C2);
      if (st != BCQ_OK) return st;
      if (C2 < C) continue;
      const int nrg = pl.p.rg_base + (pl.p.rg_rem > 0 ? 1 : 0);
      const int G = pl.W / kRowGroup;
      const double balance = (double)((nrg + G - 1) / G) * G / std::max(1, nrg);
      const double rows_cta = (double)nrg * kRowGroup * kRowBlock * balance;
      const double k_cta = (double)range_max * kChunkBlocks * kKBlock;
      const double stream_bytes = rows_cta * k_cta * p_load / 8.0;
      const double build_wf = (double)M * k_cta;
      const double stream_wf = stream_bytes * (M / 32.0 + 2.0 / 128.0);
      const int per_sm = (C * S + dc->sm_count - 1) / dc->sm_count;  // CTAs sharing an SM
      const double t_smem = (build_wf + stream_wf) * per_sm;
      const double t_hbm = total_bytes / hbm_bytes_per_clk;
      const double tail = (S > 1 ? 800.0 : 200.0) + 400.0 * range_max;
      const double issue = 12.0 / pl.W;  // consumer warps share the lookups
      pl.cost = std::max(t_smem * issue, t_hbm) + tail;
      if (pl.cost < best.cost) best = pl;
    }
  }
  if (!best.fn) return BCQ_ERR_UNSUPPORTED;
  *out = best;
  return BCQ_OK;
}

bcq_status validate_gemm(const uint16_t* x, const uint32_t* planes,
                         const uint16_t* const alpha[4], const uint16_t* z,
                         int p, const int32_t* p_row, int M, int N, int K,
                         int p_H, int group, const uint16_t* y) {
  if (!alpha) return BCQ_ERR_NULL;
  if (M < 0 || M > BCQ_MAX_M) return BCQ_ERR_SHAPE;
  if (M > 0 && (!x || !planes || !y)) return BCQ_ERR_NULL;
  if (p_H < 1 || p_H > BCQ_MAX_PLANES) return BCQ_ERR_PRECISION;
  if (group != BCQ_GROUP) return BCQ_ERR_UNSUPPORTED;
  if (N < 1 || N > (1 << 26) || K < BCQ_GROUP || K % BCQ_GROUP || K > (1 << 22))
    return BCQ_ERR_SHAPE;
  if (p < 0 || p > p_H) return BCQ_ERR_PRECISION;
  if (p == 0 && M > 0 && !p_row) return BCQ_ERR_PRECISION;
  bool used[5] = {false, false, false, false, false};
  for (int m = 0; m < M; ++m) {
    const int q = p > 0 ? p : p_row[m];
    if (q < 1 || q > p_H) return BCQ_ERR_PRECISION;
    used[q] = true;
  }
  for (int q = 1; q <= 4; ++q) {
    if (!used[q]) continue;
    if (!alpha[q - 1]) return BCQ_ERR_PRECISION;
    if (!aligned(alpha[q - 1], 16)) return BCQ_ERR_ALIGN;
  }
  if (M > 0) {
    if (!aligned(x, 16) || !aligned(planes, 16) || !aligned(y, 2)) return BCQ_ERR_ALIGN;
    if (z && !aligned(z, 16)) return BCQ_ERR_ALIGN;
  }
  return BCQ_OK;
}

std::atomic<int> g_pdl_mode{0};  // 0 off, 1 PDL, 2 PDL + early weight prefetch

bcq_status run_gemm(const uint16_t* x, const uint32_t* planes,
                    const uint16_t* const alpha[4], const uint16_t* z, int p,
                    const int32_t* p_row, int M, int N, int K, int p_H,
                    uint16_t* y, cudaStream_t st) {
  const int G = K / kGroup;
  const int KB = (K + kKBlock - 1) / kKBlock;
  const int KC = (KB + kChunkBlocks - 1) / kChunkBlocks;
  const int RB = (N + kRowBlock - 1) / kRowBlock;
  const int RBG = (RB + kRowGroup - 1) / kRowGroup;
  const int nchunk = (M + kMaxMPerLaunch - 1) / kMaxMPerLaunch;
  const int pdl_mode = g_pdl_mode.load();
  const int wait_us = env_int("BCQ_WAIT_LIMIT_US", 0);
  (void)nchunk;
  int m0 = 0;
  int single = 0;  // launches left to run one row at a time
  while (m0 < M) {
    // balanced launches of at most kMaxMPerLaunch rows (one row at a time
    // when a two-row launch has no layout that fits)
    const int rem = M - m0;
    const int nch = (rem + kMaxMPerLaunch - 1) / kMaxMPerLaunch;
    const int rows = single > 0 ? 1 : (rem + nch - 1) / nch;
    GemvParams gp{};
    int p_load = 0;
    gp.nq = 0;
    for (int r = 0; r < rows; ++r) {
      const int q = p > 0 ? p : p_row[m0 + r];
      gp.p_m[r] = q;
      p_load = std::max(p_load, q);
      int d = 0;
      while (d < gp.nq && gp.q_of[d] != q) ++d;
      if (d == gp.nq) gp.q_of[gp.nq++] = q;
      gp.d_of[r] = d;
    }
    for (int r = rows; r < kMaxMPerLaunch; ++r) {
      gp.p_m[r] = gp.p_m[0];
      gp.d_of[r] = gp.d_of[0];
    }
    const uint32_t q0 = (uint32_t)gp.q_of[0];
    const uint32_t q1 = gp.nq > 1 ? (uint32_t)gp.q_of[1] : 0u;
    const uint32_t per_rb = (uint32_t)p_load * kPlaneChunkBytes + 256u * (q0 + q1) +
                            (z ? 256u : 0u);
    Plan pl;
    bcq_status s = plan_gemv(rows, N, K, p_load, per_rb, q0, q1, z != nullptr, &pl);
    if (s == BCQ_ERR_UNSUPPORTED && rows > 1) {
      single = rows;
      continue;
    }
    if (s != BCQ_OK) return s;
    if (single > 0) --single;
    GemvParams& q = pl.p;
    q.x = x + (size_t)m0 * K;
    q.planes = planes;
    q.scale[0] = alpha[gp.q_of[0] - 1];
    q.scale[1] = gp.nq > 1 ? alpha[gp.q_of[1] - 1] : nullptr;
    q.scale[2] = z;
    q.y = y + (size_t)m0 * N;
    q.M = rows;
    q.N = N;
    q.K = K;
    q.G = G;
    q.KB = KB;
    q.KC = KC;
    q.RBG = RBG;
    q.p_H = p_H;
    q.p_load = p_load;
    for (int r = 0; r < kMaxMPerLaunch; ++r) {
      q.p_m[r] = gp.p_m[r];
      q.d_of[r] = gp.d_of[r];
      q.q_of[r] = gp.q_of[r];
    }
    q.nq = gp.nq;
    q.has_z = z != nullptr;
    q.S = pl.S;
    q.W = pl.W;
    q.NP = pl.NP;
    q.D = pl.D;
    q.early_weights = pdl_mode == 2 ? 1 : 0;
    q.timeout_ns = wait_us > 0 ? (unsigned long long)wait_us * 1000ull : kDefaultWaitNs;
    if (launch_gemv(pl.fn, q, pl.C, pl.W, pl.dyn, pdl_mode != 0, st) != cudaSuccess)
      return BCQ_ERR_CUDA;
    m0 += rows;
  }
  return BCQ_OK;
}

}  // namespace
}  // namespace bcq

using namespace bcq;

extern "C" {

const char* bcq_status_string(int status) {
  switch (status) {
    case BCQ_OK: return "BCQ_OK";
    case BCQ_ERR_NULL: return "BCQ_ERR_NULL: a required pointer is NULL";
    case BCQ_ERR_SHAPE: return "BCQ_ERR_SHAPE: M, N or K out of range";
    case BCQ_ERR_PRECISION: return "BCQ_ERR_PRECISION: precision out of range or its scales missing";
    case BCQ_ERR_ALIGN: return "BCQ_ERR_ALIGN: pointer alignment";
    case BCQ_ERR_CUDA: return "BCQ_ERR_CUDA: CUDA runtime or launch failure";
    case BCQ_ERR_TIMEOUT: return "BCQ_ERR_TIMEOUT: a bounded wait in a kernel ran out";
    case BCQ_ERR_UNSUPPORTED: return "BCQ_ERR_UNSUPPORTED: request not handled by this build";
    default: return "BCQ_ERR_UNKNOWN";
  }
}

int bcq_version(void) { return kVersion; }

size_t bcq_packed_planes_bytes(int p_H, int N, int K) {
  if (p_H < 1 || p_H > BCQ_MAX_PLANES || N < 1 || N > (1 << 26) || K < BCQ_GROUP ||
      K % BCQ_GROUP || K > (1 << 22))
    return 0;
  const size_t RB = ((size_t)N + kRowBlock - 1) / kRowBlock;
  const size_t RBG = (RB + kRowGroup - 1) / kRowGroup;
  const size_t KB = ((size_t)K + kKBlock - 1) / kKBlock;
  const size_t KC = (KB + kChunkBlocks - 1) / kChunkBlocks;
  return KC * RBG * (size_t)p_H * kRowGroup * kChunkBlocks * kWordsPerPlaneBlock *
         sizeof(uint32_t);
}

bcq_status bcq_pack_planes(const uint32_t* planes_canon, uint32_t* planes_packed,
                           int p_H, int N, int K, void* stream) {
  if (!planes_canon || !planes_packed) return BCQ_ERR_NULL;
  if (p_H < 1 || p_H > BCQ_MAX_PLANES) return BCQ_ERR_PRECISION;
  if (N < 1 || N > (1 << 26) || K < BCQ_GROUP || K % BCQ_GROUP || K > (1 << 22))
    return BCQ_ERR_SHAPE;
  if (!aligned(planes_canon, 4) || !aligned(planes_packed, 16)) return BCQ_ERR_ALIGN;
  return launch_pack(planes_canon, planes_packed, p_H, N, K, (cudaStream_t)stream) == cudaSuccess
             ? BCQ_OK
             : BCQ_ERR_CUDA;
}

size_t bcq_packed_scales_bytes(int q, int N, int K) {
  if (q < 1 || q > BCQ_MAX_PLANES || N < 1 || N > (1 << 26) || K < BCQ_GROUP ||
      K % BCQ_GROUP || K > (1 << 22))
    return 0;
  const size_t RB = ((size_t)N + kRowBlock - 1) / kRowBlock;
  const size_t RBP = (RB + kRowGroup - 1) / kRowGroup * kRowGroup;
  const size_t KB = ((size_t)K + kKBlock - 1) / kKBlock;
  const size_t KC = (KB + kChunkBlocks - 1) / kChunkBlocks;
  return KC * RBP * kChunkBlocks * 2 * 32 * (size_t)q * sizeof(uint16_t);
}

bcq_status bcq_pack_scales(const uint16_t* src, int q, int N, int K, uint16_t* dst,
                           void* stream) {
  if (!src || !dst) return BCQ_ERR_NULL;
  if (q < 1 || q > BCQ_MAX_PLANES) return BCQ_ERR_PRECISION;
  if (N < 1 || N > (1 << 26) || K < BCQ_GROUP || K % BCQ_GROUP || K > (1 << 22))
    return BCQ_ERR_SHAPE;
  if (!aligned(src, 2) || !aligned(dst, 16)) return BCQ_ERR_ALIGN;
  return launch_pack_scales(src, dst, q, N, K, (cudaStream_t)stream) == cudaSuccess
             ? BCQ_OK
             : BCQ_ERR_CUDA;
}

int bcq_plan_query(int M, int N, int K, int p_load, int q0, int q1, int has_z,
                   int use_device, int* out) {
  if (!out) return BCQ_ERR_NULL;
  if (M < 1 || M > kMaxMPerLaunch || N < 1 || K < BCQ_GROUP || K % BCQ_GROUP) return BCQ_ERR_SHAPE;
  if (p_load < 1 || p_load > 4 || q0 < 1 || q0 > 4 || q1 < 0 || q1 > 4) return BCQ_ERR_PRECISION;
  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  t_virtual = !use_device || cudaGetDevice(&dev) != cudaSuccess;
  if (t_virtual) (void)cudaGetLastError();
  const uint32_t per_rb = (uint32_t)p_load * kPlaneChunkBytes + 256u * (uint32_t)(q0 + q1) +
                          (has_z ? 256u : 0u);
  Plan pl;
  bcq_status st = plan_gemv(M, N, K, p_load, per_rb, (uint32_t)q0, (uint32_t)q1, has_z != 0, &pl);
  t_virtual = false;
  if (st != BCQ_OK) return st;
  out[0] = pl.S;
  out[1] = pl.C;
  out[2] = pl.W;
  out[3] = pl.NP;
  out[4] = pl.D;
  out[5] = (int)pl.dyn;
  out[6] = (int)pl.p.stage_bytes;
  out[7] = pl.p.rg_base;
  return BCQ_OK;
}

int bcq_set_pdl(int mode) {
  if (mode < 0 || mode > 2) return BCQ_ERR_UNSUPPORTED;
  g_pdl_mode.store(mode);
  return BCQ_OK;
}

bcq_status bcq_gemm(const uint16_t* x, const uint32_t* planes,
                    const uint16_t* const alpha[4], const uint16_t* z, int p,
                    const int32_t* p_row, int M, int N, int K, int p_H, int group,
                    uint16_t* y, void* stream) {
  bcq_status s = validate_gemm(x, planes, alpha, z, p, p_row, M, N, K, p_H, group, y);
  if (s != BCQ_OK || M == 0) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  return run_gemm(x, planes, alpha, z, p, p_row, M, N, K, p_H, y, (cudaStream_t)stream);
}

bcq_status bcq_gemm_host(const uint16_t* x_host, const uint32_t* planes,
                         const uint16_t* const alpha[4], const uint16_t* z, int p,
                         const int32_t* p_row, int M, int N, int K, int p_H, int group,
                         uint16_t* y_host, uint16_t* x_dev, uint16_t* y_dev, void* stream) {
  if (M > 0 && (!x_host || !y_host)) return BCQ_ERR_NULL;
  bcq_status s = validate_gemm(x_dev, planes, alpha, z, p, p_row, M, N, K, p_H, group, y_dev);
  if (s != BCQ_OK || M == 0) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(x_dev, x_host, (size_t)M * K * 2, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return BCQ_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    s = run_gemm(x_dev, planes, alpha, z, p, p_row, M, N, K, p_H, y_dev, st);
  }
  if (s != BCQ_OK) return s;
  if (cudaMemcpyAsync(y_host, y_dev, (size_t)M * N * 2, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return BCQ_ERR_CUDA;
  return BCQ_OK;
}

bcq_status bcq_build_lut(const uint16_t* x, int M, int K, float* lut, float* group_sums,
                         void* stream) {
  if (!x || !lut) return BCQ_ERR_NULL;
  if (M < 1 || M > 4 || K < BCQ_GROUP || K % BCQ_GROUP || K > (1 << 22))
    return BCQ_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(lut, 4) || (group_sums && !aligned(group_sums, 4)))
    return BCQ_ERR_ALIGN;
  return launch_lut_dump(x, M, K, lut, group_sums, (cudaStream_t)stream) == cudaSuccess
             ? BCQ_OK
             : BCQ_ERR_CUDA;
}

bcq_status bcq_device_error(void* stream) {
  int code = 0;
  if (read_and_clear_device_error((cudaStream_t)stream, &code) != cudaSuccess) return BCQ_ERR_CUDA;
  return (bcq_status)code;
}

bcq_status bcq_debug_wait_timeout(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return BCQ_ERR_SHAPE;
  return launch_wait_probe((unsigned long long)limit_us * 1000ull, (cudaStream_t)stream) ==
                 cudaSuccess
             ? BCQ_OK
             : BCQ_ERR_CUDA;
}

}  // extern "C"
