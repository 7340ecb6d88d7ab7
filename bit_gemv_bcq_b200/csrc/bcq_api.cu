// bcq_api.cu -- the C ABI of libbcq (include/bcq.h): argument validation,
// launch planning and dispatch.  No device memory is allocated here.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
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
  int M = 0, NKB = 0, S = 1, C = 1, W = 8, D = 2;
  size_t dyn = 0;
  GemvParams p{};
  double cost = 1e300;
};

size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

// Shared-memory layout of one candidate (cluster count already chosen);
// false if the low region or the whole CTA does not fit.
bool layout(Plan& pl, int KB, int p_load) {
  const int range_max = (KB + pl.S - 1) / pl.S;
  const int slots = 2 * range_max;
  const int part_rows = kRowBlock * (pl.p.rb_base + (pl.p.rb_rem > 0 ? 1 : 0));
  size_t off = 0;
  pl.p.off_part = (uint32_t)off;
  off = align16(off + (size_t)slots * pl.M * part_rows * sizeof(float));
  pl.p.off_gsum = (uint32_t)off;
  off = align16(off + (size_t)pl.M * 2 * pl.NKB * sizeof(float));
  pl.p.off_bar = (uint32_t)off;
  off = align16(off + (size_t)pl.W * pl.D * 8);
  pl.p.off_flag = (uint32_t)off;
  off = align16(off + 16);
  if (off + kLowReserve > kLutAbs) return false;
  pl.p.low_bytes = (uint32_t)off;
  pl.p.part_rows = part_rows;
  const size_t lut_bytes = (size_t)((pl.M * pl.NKB + 1) / 2) * kLutTableBytes;
  pl.p.ring_abs = (uint32_t)(kLutAbs + lut_bytes);
  pl.dyn = pl.p.ring_abs + (size_t)pl.W * pl.D * p_load * kUnitBytesPerPlane;
  return pl.dyn <= kMaxDynSmem;
}

bcq_status get_device(DeviceCache** dc) {
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
bcq_status active_clusters(DeviceCache& dc, int ki, GemvKernel fn, int S, int W,
                           size_t dyn, int* out) {
  if (dc.attr_done[ki] != fn) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kMaxDynSmem) != cudaSuccess)
      return BCQ_ERR_CUDA;
    dc.attr_done[ki] = fn;
  }
  for (int i = 0; i < dc.n_occ; ++i) {
    const OccEntry& e = dc.occ[i];
    if (e.fn == fn && e.S == S && e.W == W && e.dyn == dyn) {
      *out = e.clusters;
      return BCQ_OK;
    }
  }
  int n = 0;
  if (S == 1) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, 32 * W, dyn) != cudaSuccess)
      return BCQ_ERR_CUDA;
    n = per_sm * dc.sm_count;
  } else if (max_active_clusters(fn, S, W, dyn, &n) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  if (dc.n_occ < 64) dc.occ[dc.n_occ++] = OccEntry{fn, S, W, dyn, n};
  *out = n;
  return BCQ_OK;
}

int kernel_index(int M, int NKB) {
  switch (M * 8 + NKB) {
    case 9: return 0;
    case 10: return 1;
    case 11: return 2;
    case 12: return 3;
    case 17: return 4;
    case 18: return 5;
    case 25: return 6;
    case 33: return 7;
    default: return -1;
  }
}

// Chooses the split-K factor S (cluster size), cluster count C, warps W and
// ring depth D for one launch of M (1..4) activation rows.  The cost model
// counts shared-memory wavefronts per CTA (LUT build: M per column; lookups:
// M per 32 plane bytes; staging: 2 per 128 plane bytes) against the HBM time
// of the whole call, plus a fixed cost per cluster reduction and per phase.
bcq_status plan_gemv(int M, int N, int K, int p_load, Plan* out) {
  DeviceCache* dc = nullptr;
  bcq_status st = get_device(&dc);
  if (st != BCQ_OK) return st;
  const int KB = (K + kKBlock - 1) / kKBlock;
  const int RB = (N + kRowBlock - 1) / kRowBlock;
  const int nkb_max = M == 1 ? 4 : M == 2 ? 2 : 1;
  const int force_S = env_int("BCQ_FORCE_S", 0);
  const int force_W = env_int("BCQ_FORCE_W", 0);
  const int force_D = env_int("BCQ_FORCE_D", 0);
  const double hbm_bytes_per_clk = 3300.0;  // ~6.5 TB/s at ~1.95 GHz
  const double total_bytes = (double)N * K * p_load / 8.0;
  Plan best;
  const int S_list[4] = {1, 2, 4, 8};
  for (int si = 0; si < 4; ++si) {
    const int S = S_list[si];
    if (force_S && S != force_S) continue;
    if (S > KB) continue;
    const int range_max = (KB + S - 1) / S;
    Plan pl;
    pl.M = M;
    pl.S = S;
    pl.NKB = std::min(nkb_max, range_max);
    pl.fn = gemv_kernel_for(M, pl.NKB);
    const int ki = kernel_index(M, pl.NKB);
    if (!pl.fn || ki < 0) continue;
    pl.W = force_W ? force_W : 8;
    if (pl.W != 8 && pl.W != 4) continue;
    const size_t lut_bytes = (size_t)((M * pl.NKB + 1) / 2) * kLutTableBytes;
    const size_t ring_room = kMaxDynSmem - (kLutAbs + lut_bytes);
    const size_t stage = (size_t)p_load * kUnitBytesPerPlane;
    int D = (int)std::min<size_t>(8, ring_room / (pl.W * stage));
    if (force_D) D = std::min(D, force_D);
    if (D < 1) continue;
    pl.D = D;
    const size_t dyn = kLutAbs + lut_bytes + (size_t)pl.W * D * stage;
    int C = 0;
    st = active_clusters(*dc, ki, pl.fn, S, pl.W, dyn, &C);
    if (st != BCQ_OK) return st;
    if (C <= 0) continue;
    C = std::min(C, RB);
    pl.C = C;
    pl.p.rb_base = RB / C;
    pl.p.rb_rem = RB % C;
    if (!layout(pl, KB, p_load)) continue;
    const double rows_cta = (double)pl.p.part_rows;
    const double k_cta = (double)range_max * kKBlock;
    const double stream_bytes = rows_cta * k_cta * p_load / 8.0;
    const double build_wf = (double)M * k_cta;
    const double stream_wf = stream_bytes * (M / 32.0 + 2.0 / 128.0);
    const int per_sm = (C * S + dc->sm_count - 1) / dc->sm_count;  // CTAs sharing an SM
    const double t_smem = (build_wf + stream_wf) * per_sm;
    const double t_hbm = total_bytes / hbm_bytes_per_clk;
    const int nphase = (range_max + pl.NKB - 1) / pl.NKB;
    const double tail = (S > 1 ? 800.0 : 200.0) + 300.0 * nphase;
    pl.cost = std::max(t_smem, t_hbm) + tail;
    if (pl.cost < best.cost) best = pl;
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
    const size_t need = q == 2 ? 4 : q == 4 ? 8 : 2;
    if (!aligned(alpha[q - 1], need)) return BCQ_ERR_ALIGN;
  }
  if (M > 0) {
    if (!aligned(x, 16) || !aligned(planes, 16) || !aligned(y, 2)) return BCQ_ERR_ALIGN;
    if (z && !aligned(z, 2)) return BCQ_ERR_ALIGN;
  }
  return BCQ_OK;
}

bcq_status run_gemm(const uint16_t* x, const uint32_t* planes,
                    const uint16_t* const alpha[4], const uint16_t* z, int p,
                    const int32_t* p_row, int M, int N, int K, int p_H,
                    uint16_t* y, cudaStream_t st) {
  const int G = K / kGroup;
  const int KB = (K + kKBlock - 1) / kKBlock;
  const int RB = (N + kRowBlock - 1) / kRowBlock;
  const int nchunk = (M + kMaxMPerLaunch - 1) / kMaxMPerLaunch;
  int m0 = 0;
  for (int c = 0; c < nchunk; ++c) {
    // balanced chunks of at most four rows
    const int rows = (M - m0) / (nchunk - c) + (((M - m0) % (nchunk - c)) ? 1 : 0);
    int pm[4] = {0, 0, 0, 0};
    int p_load = 0;
    for (int r = 0; r < rows; ++r) {
      pm[r] = p > 0 ? p : p_row[m0 + r];
      p_load = std::max(p_load, pm[r]);
    }
    Plan pl;
    bcq_status s = plan_gemv(rows, N, K, p_load, &pl);
    if (s != BCQ_OK) return s;
    GemvParams& gp = pl.p;
    gp.x = x + (size_t)m0 * K;
    gp.planes = planes;
    for (int q = 0; q < 4; ++q) gp.alpha[q] = alpha[q];
    gp.z = z;
    gp.y = y + (size_t)m0 * N;
    gp.M = rows;
    gp.N = N;
    gp.K = K;
    gp.G = G;
    gp.KB = KB;
    gp.RB = RB;
    gp.p_H = p_H;
    gp.p_load = p_load;
    for (int r = 0; r < 4; ++r) gp.p_m[r] = r < rows ? pm[r] : pm[0];
    gp.S = pl.S;
    gp.D = pl.D;
    const int wait_us = env_int("BCQ_WAIT_LIMIT_US", 0);
    gp.timeout_ns = wait_us > 0 ? (unsigned long long)wait_us * 1000ull : kDefaultWaitNs;
    if (launch_gemv(pl.fn, gp, pl.C, pl.W, pl.dyn, st) != cudaSuccess) return BCQ_ERR_CUDA;
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
  const size_t KB = ((size_t)K + kKBlock - 1) / kKBlock;
  return RB * (size_t)p_H * KB * kWordsPerPlaneBlock * sizeof(uint32_t);
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
  if (M < 1 || M > kMaxMPerLaunch || K < BCQ_GROUP || K % BCQ_GROUP || K > (1 << 22))
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
