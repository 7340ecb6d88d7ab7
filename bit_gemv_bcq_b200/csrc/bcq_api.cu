// bcq_api.cu -- the C ABI of libbcq (include/bcq.h): argument validation,
// launch planning and dispatch.  No device memory is allocated here; split-K
// partial sums go to a caller-owned workspace.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bcq.h"
#include "bcq_launch.h"
#include "bcq_layout.h"

namespace bcq {
namespace {

constexpr int kVersion = 200;                // 0.2.0
constexpr size_t kMaxDynSmem = 232448;       // 227 KiB per CTA on sm_100
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s
constexpr int kDefaultProducers = 2;
// Calls with at least this many rows take the tensor-core path.
constexpr int kDefaultMmaMinRows = 3;

// Kernels: the lookup-table kernel (one or two rows), and for batches a
// tensor-core kernel: mma.sync (default) or tcgen05 (BCQ_MMA_KIND=tcgen05).
enum GemvPath { kPathLut = 0, kPathMmaSync = 1, kPathUmma = 2, kPathLut4 = 3, kPathM1 = 4 };

// One-row launches: the dense-table kernel (bcq_m1.cuh) unless
// BCQ_M1_KIND=pair asks for the pair-table kernel with one row.
bool use_m1_kernel(int /*K*/) {
  const char* v = std::getenv("BCQ_M1_KIND");
  return !(v && std::strcmp(v, "pair") == 0);
}

int batch_path() {
  const char* v = std::getenv("BCQ_MMA_KIND");
  return (v && std::strcmp(v, "tcgen05") == 0) ? kPathUmma : kPathMmaSync;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int env_int(const char* name, int dflt) {
  const char* v = std::getenv(name);
  if (!v || !*v) return dflt;
  return std::atoi(v);
}

bool shape_ok(int N, int K) {
  return N >= 1 && N <= (1 << 26) && K >= BCQ_GROUP && K % BCQ_GROUP == 0 && K <= (1 << 22);
}

size_t row_blocks(int N) { return ((size_t)N + kRowBlock - 1) / kRowBlock; }
size_t k_blocks(int K) { return ((size_t)K + kKBlock - 1) / kKBlock; }

// Workspace: the tagged fp32 partial sums [KB][min(M, 64)][RB * 32] (the
// rows of the largest launch); zero = not written yet.
size_t workspace_bytes(int M, int N, int K) {
  const size_t KB = k_blocks(K);
  if (M < 1 || KB <= 1) return 0;
  const size_t ml = (size_t)std::min(M, kMaxLaunchRows);
  return KB * ml * row_blocks(N) * kRowBlock * sizeof(float);
}

// Per-device facts, cached after the first query (callers hold g_mu).
struct DeviceCache {
  bool init = false;
  int sm_count = 0;
  GemvKernel attr_done[16] = {};
  int n_attr = 0;
};
std::mutex g_mu;
DeviceCache g_cache[16];

// Plans can be queried without a GPU (bcq_plan_query): they are then made
// for a nominal B200 (148 SMs).
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

struct Plan {
  GemvKernel fn = nullptr;
  int C = 0, D = 0, NP = 0, MW = 0, CW = kConsumerWarps;
  size_t dyn = 0;
  long long units_max = 0;
  int KB = 0;
};

// One launch of M (1 or 2) rows streaming P planes.  Grid: at most one CTA
// per SM and one per unit; each CTA takes an equal share of the units in
// kb-major order.  Ring: D stages of 8P KiB (the P planes of one row group
// of one K-block) fed by NP producer warps, as deep as shared memory allows
// beside the 64 KiB table; D is even (a stage's team consumed the stage D
// earlier) and a multiple of NP (a producer refills only its own slots).
bcq_status plan_gemv(int M, int N, int K, int P, bool mixed, int path, Plan* out) {
  DeviceCache* dc = nullptr;
  bcq_status st = get_device(&dc);
  if (st != BCQ_OK) return st;
  Plan pl;
  const int NN = M > kMmaRows ? kMaxLaunchRows : kMmaRows;  // tcgen05: 16 or 64 rows
  pl.fn = path == kPathUmma      ? gemv_umma_kernel_for(P, NN)
          : path == kPathMmaSync ? gemv_mma_kernel_for(M > 8 ? 2 : 1, P, mixed)
          : path == kPathM1      ? gemv_m1_kernel_for(P)
                                 : gemv_kernel_for(M, P, mixed);
  if (!pl.fn) return BCQ_ERR_UNSUPPORTED;
  auto dyn_of = [&](int d) {
    return path == kPathUmma      ? (NN == kMmaRows ? umma_dyn_bytes<16>(d, P)
                                                     : umma_dyn_bytes<64>(d, P))
           : path == kPathMmaSync ? mma_dyn_bytes(d, P, mixed)
           : path == kPathM1      ? m1_dyn_bytes(d, P)
                                  : gemv_dyn_bytes(d, P, M);
  };
  const long long RB = (long long)row_blocks(N);
  const long long KB = (long long)k_blocks(K);
  const long long U = RB * KB;
  pl.KB = (int)KB;
  // (the one-row kernel: m1_producers(P) producers, one part of every stage each)
  pl.NP = path == kPathM1 ? m1_producers(P) : std::max(1, std::min(2, env_int("BCQ_FORCE_NP", kDefaultProducers)));
  // ring stages: even (the two teams alternate) and a multiple of NP
  const int step = 2;
  const size_t dyn_cap = kMaxDynSmem;
  int D = env_int("BCQ_FORCE_D", kMaxStages);
  D = std::min(kMaxStages, D) / step * step;
  if (D < step) D = step;
  while (D > step && dyn_of(D) > dyn_cap) D -= step;
  pl.MW = path == kPathUmma ? kUmmaGroups : 0;
  pl.CW = path == kPathM1 ? kM1Warps : kConsumerWarps;
  const int nthreads = 32 * (pl.CW + pl.MW + pl.NP);
  while (true) {
    pl.dyn = dyn_of(D);
    int per_sm = 0;
    if (pl.dyn <= kMaxDynSmem) {
      if (t_virtual) {
        per_sm = 1;
      } else {
        bool done = false;
        for (int i = 0; i < dc->n_attr; ++i) done = done || dc->attr_done[i] == pl.fn;
        if (blocks_per_sm(pl.fn, nthreads, pl.dyn, &per_sm) != cudaSuccess) return BCQ_ERR_CUDA;
        if (!done && dc->n_attr < 16) dc->attr_done[dc->n_attr++] = pl.fn;
      }
    }
    if (per_sm >= 1) break;
    if (D - step < step) return BCQ_ERR_UNSUPPORTED;
    D -= step;
  }
  pl.D = D;
  // With no more K-blocks than SMs, every K-block gets the same number of
  // CTAs and no CTA spans two K-blocks (a second table build would make it
  // the slowest CTA, and the last to arrive for all of its row-blocks).  The
  // one-row kernel keeps that split only while it leaves at most a tenth of
  // the SMs idle; otherwise every SM takes an equal share of the units and
  // some CTAs rebuild the table once (4096 x 14336: 148 CTAs, not 112).
  long long C = std::min<long long>(U, std::min(dc->sm_count, kMaxCtas));
  if (KB <= C) {
    const long long even = std::min<long long>(U, KB * std::min<long long>(RB, C / KB));
    if (path != kPathM1 || even * 10 >= C * 9) C = even;
  }
  const int force_C = env_int("BCQ_FORCE_C", 0);
  if (force_C > 0) C = std::min<long long>(U, std::min(force_C, kMaxCtas));
  pl.C = (int)C;
  pl.units_max = (U + C - 1) / C;
  if (U >= (1ll << 31)) return BCQ_ERR_UNSUPPORTED;  // units are counted in 32 bits
  *out = pl;
  return BCQ_OK;
}

bcq_status validate_gemm(const uint16_t* x, const uint32_t* planes,
                         const uint16_t* const alpha[4], const uint16_t* const zq[4], int p,
                         const int32_t* p_row, int M, int N, int K, int p_H, int group,
                         const uint16_t* y, const void* ws, size_t ws_bytes) {
  if (!alpha) return BCQ_ERR_NULL;
  if (M < 0 || M > BCQ_MAX_M) return BCQ_ERR_SHAPE;
  if (M > 0 && (!x || !planes || !y)) return BCQ_ERR_NULL;
  if (p_H < 1 || p_H > BCQ_MAX_PLANES) return BCQ_ERR_PRECISION;
  if (group != BCQ_GROUP) return BCQ_ERR_UNSUPPORTED;
  if (!shape_ok(N, K)) return BCQ_ERR_SHAPE;
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
    for (int q = 1; q <= 4; ++q)
      if (used[q] && zq[q - 1] && !aligned(zq[q - 1], 16)) return BCQ_ERR_ALIGN;
    const size_t need = workspace_bytes(M, N, K);
    if (need > 0) {
      if (!ws || ws_bytes < need) return BCQ_ERR_NULL;
      if (!aligned(ws, 16)) return BCQ_ERR_ALIGN;
    }
  }
  return BCQ_OK;
}

std::atomic<int> g_pdl_mode{0};  // 0 off, 1 PDL, 2 PDL + early plane streaming

// Splits the U = RB * KB units (kb-major) over C CTAs: when the CTAs divide
// evenly among the K-blocks, C / KB CTAs share the row-blocks of each
// K-block and no CTA builds two tables; otherwise every CTA takes an equal
// share (the first U mod C one unit more).  Groups: per K-block, the row
// groups of 8 row-blocks the CTA touches.
void plan_units(int RB, int KB, int C, CtaWork* work) {
  const long long U = (long long)RB * KB;
  for (int c = 0; c < C; ++c) {
    long long u0, u1;
    if (C >= KB && C % KB == 0) {
      const int cpk = C / KB, kb = c / cpk, j = c - kb * cpk;
      const int q = RB / cpk, r = RB % cpk;
      u0 = (long long)kb * RB + (long long)j * q + std::min(j, r);
      u1 = u0 + q + (j < r ? 1 : 0);
    } else {
      const long long q = U / C, r = U % C;
      u0 = c * q + std::min<long long>(c, r);
      u1 = u0 + q + (c < r ? 1 : 0);
    }
    int ng = 0;
    for (long long u = u0; u < u1;) {
      const long long kb = u / RB;
      const long long end = std::min(u1, (kb + 1) * RB);
      const long long a = u - kb * RB, b = end - kb * RB;
      ng += (int)((b + kRowGroup - 1) / kRowGroup - a / kRowGroup);
      u = end;
    }
    const int kb0 = (int)(u0 / RB);
    const int kb1 = u1 > u0 ? (int)((u1 - 1) / RB) : kb0;
    work[c] = CtaWork{(int)u0, (int)u1, ng, kb0 | (kb1 << 16)};
  }
}

// Fills the fields every launch shares.
void fill_common(GemvParams& g, const Plan& pl, const uint32_t* planes, int N, int K, int p_H,
                 void* ws, int pdl_mode, int wait_us) {
  const int RB = (int)row_blocks(N);
  const int KB = (int)k_blocks(K);
  g.planes = planes;
  g.part = KB > 1 ? static_cast<float*>(ws) : nullptr;
  g.N = N;
  g.K = K;
  g.KB = KB;
  g.RB = RB;
  g.RG = (RB + kRowGroup - 1) / kRowGroup;
  g.p_H = p_H;
  g.U = (int)((long long)RB * KB);
  g.C = pl.C;
  plan_units(RB, KB, pl.C, g.work);
  g.D = pl.D;
  g.NP = pl.NP;
  g.MW = pl.MW;
  g.early_weights = pdl_mode == 2 ? 1 : 0;
  g.timeout_ns = wait_us > 0 ? (unsigned long long)wait_us * 1000ull : kDefaultWaitNs;
}

// Cooperative launches (all CTAs of a grid resident at once, which the
// split-K tail's polling relies on); BCQ_COOPERATIVE=0 turns the attribute
// off (for comparison only: the tail then assumes the grid fits at once).
bool cooperative_launch() { return env_int("BCQ_COOPERATIVE", 1) != 0; }

// One launch of a call: the kernel, the rows of x and y it takes (in launch
// order) and their precisions.
struct Launch {
  int path = kPathLut;  // kPathLut (pair tables, 1-2 rows), kPathM1, kPathLut4, kPathMmaSync, kPathUmma
  bool mixed = false;   // rows of several precisions
  int n = 0;            // rows
  int P = 0;            // planes streamed: the largest precision
  int row[kMaxLaunchRows];
  int q[kMaxLaunchRows];
};

// The launches of one call (no device work; bcq_gemm and the queries share
// it).  Rows of one precision, M >= BCQ_MMA_MIN_ROWS (3): tcgen05 launches
// of up to 64 rows while at least 32 are left, 33 at one or two bits
// (measured on 14336 x 4096: 64 rows in one launch cost 0.6 of four 16-row
// launches; exactly 32 rows at p = 2 take 54.5 us as one launch and 46.7 us
// as two 16-row launches, at p = 4 70.0 against 75.2 us), a four-row
// lookup launch for a group of 3-4 rows (measured on 14336 x 4096: p = 2 /
// 3 / 4 in 17.2 / 23.6 / 26.2 us against 22.9 / 29.6 / 36.6 us on the
// tensor-core kernel;
// BCQ_LUT4_MAX_ROWS=0 turns it off, BCQ_LUT4_MIN_BITS sets a precision
// threshold), tensor-core launches of up to 16 rows, lookup launches for a
// remainder of 1-2 rows.  Rows of several precisions (per-request
// precision): up to 16 rows are one mixed tensor-core launch that streams
// the planes once, up to the largest precision, each row applying its own
// scales and offsets; larger batches are grouped by precision as above and
// the rows left over in every group share mixed launches (16 rows at most
// each).  Fewer than BCQ_MMA_MIN_ROWS rows: lookup launches of two rows,
// mixed or not.  One-row lookup launches use the dense-table kernel.
int route_call(int M, int p, const int32_t* p_row, int K, Launch* out) {
  const int mma_min = std::max(1, env_int("BCQ_MMA_MIN_ROWS", kDefaultMmaMinRows));
  const int lut4_max = std::min(4, env_int("BCQ_LUT4_MAX_ROWS", 4));
  const int lut4_bits = env_int("BCQ_LUT4_MIN_BITS", 1);
  const int tc = batch_path();
  auto qof = [&](int m) { return p > 0 ? p : p_row[m]; };
  int n = 0;
  auto add = [&](int path, const int* rows, int cnt) {
    Launch& L = out[n++];
    L.path = path;
    L.n = cnt;
    L.P = 0;
    bool mixed = false;
    for (int j = 0; j < cnt; ++j) {
      L.row[j] = rows[j];
      L.q[j] = qof(rows[j]);
      L.P = std::max(L.P, L.q[j]);
      mixed = mixed || L.q[j] != L.q[0];
    }
    L.mixed = mixed;
    if (path == kPathLut && cnt == 1 && use_m1_kernel(K)) L.path = kPathM1;
  };
  auto pairs = [&](const int* rows, int cnt) {
    for (int j = 0; j < cnt; j += kMaxMPerLaunch) add(kPathLut, rows + j, std::min(kMaxMPerLaunch, cnt - j));
  };
  int all[BCQ_MAX_M];
  bool uniform = true;
  for (int m = 0; m < M; ++m) {
    all[m] = m;
    uniform = uniform && qof(m) == qof(0);
  }
  if (M < mma_min) {
    pairs(all, M);
    return n;
  }
  // (BCQ_MIXED_LAUNCH=0: mixed batches grouped by precision, for comparison)
  const bool mixed_launch = env_int("BCQ_MIXED_LAUNCH", 1) != 0;
  if (!uniform && mixed_launch && M <= kMmaRows) {
    add(kPathMmaSync, all, M);
    return n;
  }
  int left_rows[BCQ_MAX_M];
  int nleft = 0;
  for (int q = 1; q <= 4; ++q) {
    int rows[BCQ_MAX_M];
    int cnt = 0;
    for (int m = 0; m < M; ++m)
      if (qof(m) == q) rows[cnt++] = m;
    for (int r0 = 0; r0 < cnt;) {
      const int left = cnt - r0;
      if (left > 2 * kMmaRows || (left == 2 * kMmaRows && q > 2)) {
        const int c = std::min(kMaxLaunchRows, left);
        add(kPathUmma, rows + r0, c);
        r0 += c;
      } else if (left >= mma_min && left <= lut4_max && q >= lut4_bits) {
        add(kPathLut4, rows + r0, left);
        r0 += left;
      } else if (left >= mma_min) {
        const int c = std::min(kMmaRows, left);
        add(tc, rows + r0, c);
        r0 += c;
      } else {
        for (int j = r0; j < cnt; ++j) left_rows[nleft++] = rows[j];
        r0 = cnt;
      }
    }
  }
  // rows left over in every precision group
  if (mixed_launch) {
    int r0 = 0;
    while (nleft - r0 >= mma_min) {
      const int c = std::min(kMmaRows, nleft - r0);
      add(kPathMmaSync, left_rows + r0, c);
      r0 += c;
    }
    pairs(left_rows + r0, nleft - r0);
  } else {
    pairs(left_rows, nleft);
  }
  return n;
}

bcq_status run_gemm(const uint16_t* x, const uint32_t* planes, const uint16_t* const alpha[4],
                    const uint16_t* const zq[4], int p, const int32_t* p_row, int M, int N, int K,
                    int p_H, uint16_t* y, void* ws, cudaStream_t st) {
  const int pdl_mode = g_pdl_mode.load();
  const int wait_us = env_int("BCQ_WAIT_LIMIT_US", 0);
  static thread_local Launch launches[BCQ_MAX_M];
  const int n = route_call(M, p, p_row, K, launches);
  for (int li = 0; li < n; ++li) {
    const Launch& L = launches[li];
    Plan pl;
    const int plan_rows = L.path == kPathLut4 ? 4 : L.n;
    const int plan_path = L.path == kPathLut4 ? kPathLut : L.path;
    bcq_status s = plan_gemv(plan_rows, N, K, L.P, L.mixed, plan_path, &pl);
    if (s != BCQ_OK) return s;
    GemvParams g{};
    fill_common(g, pl, planes, N, K, p_H, ws, pdl_mode, wait_us);
    g.M = L.n;
    g.q[0] = L.q[0];
    g.q[1] = L.q[L.n > 1 ? 1 : 0];
    g.alpha[0] = alpha[g.q[0] - 1];
    g.alpha[1] = alpha[g.q[1] - 1];
    g.z = zq[g.q[0] - 1];
    g.z1 = zq[g.q[1] - 1];
    if (L.path == kPathM1 || (L.path == kPathLut && L.n == 1)) {  // one row, addressed directly
      g.x = x + (size_t)L.row[0] * K;
      g.y = y + (size_t)L.row[0] * N;
    } else {
      g.x = x;
      g.y = y;
      for (int j = 0; j < L.n; ++j) {
        g.rows[j] = L.row[j];
        g.qrow[j] = L.q[j];
      }
    }
    if (L.mixed && L.path == kPathMmaSync) {
      for (int q = 1; q <= 4; ++q) {
        g.alpha_q[q - 1] = alpha[q - 1];
        g.z_q[q - 1] = zq[q - 1];
      }
      for (int j = 0; j < L.n; ++j) g.qmask |= 1 << L.q[j];
    }
    if (launch_gemv(pl.fn, g, pl.dyn, pdl_mode != 0, st, pl.CW, cooperative_launch()) !=
        cudaSuccess)
      return BCQ_ERR_CUDA;
  }
  return BCQ_OK;
}

}  // namespace
bcq_status check_gemm_args(const uint16_t* x, const uint32_t* planes,
                           const uint16_t* const alpha[4], const uint16_t* z, int p,
                           const int32_t* p_row, int M, int N, int K, int p_H, int group,
                           const uint16_t* y, const void* ws, size_t ws_bytes) {
  const uint16_t* const zq[4] = {z, z, z, z};
  return validate_gemm(x, planes, alpha, zq, p, p_row, M, N, K, p_H, group, y, ws, ws_bytes);
}

}  // namespace bcq

using namespace bcq;

extern "C" {

const char* bcq_status_string(int status) {
  switch (status) {
    case BCQ_OK: return "BCQ_OK";
    case BCQ_ERR_NULL: return "BCQ_ERR_NULL: a required pointer is NULL (or a buffer too small)";
    case BCQ_ERR_SHAPE: return "BCQ_ERR_SHAPE: M, N or K out of range";
    case BCQ_ERR_PRECISION: return "BCQ_ERR_PRECISION: precision out of range or its scales missing";
    case BCQ_ERR_ALIGN: return "BCQ_ERR_ALIGN: pointer alignment";
    case BCQ_ERR_CUDA: return "BCQ_ERR_CUDA: CUDA runtime or launch failure";
    case BCQ_ERR_TIMEOUT: return "BCQ_ERR_TIMEOUT: a bounded wait in a kernel ran out";
    case BCQ_ERR_UNSUPPORTED: return "BCQ_ERR_UNSUPPORTED: request not handled by this build";
    case BCQ_ERR_SCRATCH: return "BCQ_ERR_SCRATCH: the call needs more than the built-in scratch";
    default: return "BCQ_ERR_UNKNOWN";
  }
}

int bcq_version(void) { return kVersion; }

size_t bcq_packed_planes_bytes(int p_H, int N, int K) {
  if (p_H < 1 || p_H > BCQ_MAX_PLANES || !shape_ok(N, K)) return 0;
  const size_t RG = (row_blocks(N) + kRowGroup - 1) / kRowGroup;
  return k_blocks(K) * RG * (size_t)p_H * kPlaneGroupBytes;
}

bcq_status bcq_pack_planes(const uint32_t* planes_canon, uint32_t* planes_packed, int p_H,
                           int N, int K, void* stream) {
  if (!planes_canon || !planes_packed) return BCQ_ERR_NULL;
  if (p_H < 1 || p_H > BCQ_MAX_PLANES) return BCQ_ERR_PRECISION;
  if (!shape_ok(N, K)) return BCQ_ERR_SHAPE;
  if (!aligned(planes_canon, 4) || !aligned(planes_packed, 16)) return BCQ_ERR_ALIGN;
  return launch_pack(planes_canon, planes_packed, p_H, N, K, (cudaStream_t)stream) == cudaSuccess
             ? BCQ_OK
             : BCQ_ERR_CUDA;
}

size_t bcq_packed_scales_bytes(int q, int N, int K) {
  if (q < 1 || q > BCQ_MAX_PLANES || !shape_ok(N, K)) return 0;
  return k_blocks(K) * row_blocks(N) * kRowBlock * 2 * (size_t)q * sizeof(uint16_t);
}

bcq_status bcq_pack_scales(const uint16_t* src, int q, int N, int K, uint16_t* dst,
                           void* stream) {
  if (!src || !dst) return BCQ_ERR_NULL;
  if (q < 1 || q > BCQ_MAX_PLANES) return BCQ_ERR_PRECISION;
  if (!shape_ok(N, K)) return BCQ_ERR_SHAPE;
  if (!aligned(src, 2) || !aligned(dst, 16)) return BCQ_ERR_ALIGN;
  return launch_pack_scales(src, dst, q, N, K, (cudaStream_t)stream) == cudaSuccess
             ? BCQ_OK
             : BCQ_ERR_CUDA;
}

size_t bcq_workspace_bytes(int M, int N, int K) {
  if (M < 0 || M > BCQ_MAX_M || !shape_ok(N, K)) return 0;
  return workspace_bytes(M, N, K);
}

int bcq_plan_query(int M, int N, int K, int p_load, int mixed, int use_device, int* out) {
  if (!out) return BCQ_ERR_NULL;
  if (M < 1 || M > kMaxLaunchRows || !shape_ok(N, K)) return BCQ_ERR_SHAPE;
  if (p_load < 1 || p_load > 4) return BCQ_ERR_PRECISION;
  if (mixed && (M < 2 || M > kMmaRows || p_load < 2)) return BCQ_ERR_PRECISION;
  // the kernel bcq_gemm gives a launch of M rows (route_call's rules)
  const int mma_min = std::max(1, env_int("BCQ_MMA_MIN_ROWS", kDefaultMmaMinRows));
  const bool lut4 = !mixed && M > kMaxMPerLaunch && M >= mma_min &&
                    M <= std::min(4, env_int("BCQ_LUT4_MAX_ROWS", 4)) &&
                    p_load >= env_int("BCQ_LUT4_MIN_BITS", 1);
  int path;
  if (M <= kMaxMPerLaunch) path = M == 1 && !mixed && use_m1_kernel(K) ? kPathM1 : kPathLut;
  else if (mixed) path = kPathMmaSync;
  else if (lut4) path = kPathLut;
  else if (M > kMmaRows) path = kPathUmma;
  else path = batch_path();
  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  t_virtual = !use_device || cudaGetDevice(&dev) != cudaSuccess;
  if (t_virtual) (void)cudaGetLastError();
  Plan pl;
  bcq_status st = plan_gemv(lut4 ? 4 : M, N, K, p_load, mixed != 0, path, &pl);
  t_virtual = false;
  if (st != BCQ_OK) return st;
  out[0] = pl.C;
  out[1] = pl.CW;
  out[2] = pl.NP;
  out[3] = pl.D;
  out[4] = (int)pl.dyn;
  out[5] = (int)(path == kPathM1 ? m1_stage_bytes(p_load) : gemv_stage_bytes(p_load));
  out[6] = (int)pl.units_max;
  out[7] = pl.KB;
  return BCQ_OK;
}

int bcq_route_query(int M, int p, const int32_t* p_row, int N, int K, int* out,
                    int max_launches) {
  if (!out || max_launches < 0) return BCQ_ERR_NULL;
  if (M < 1 || M > BCQ_MAX_M || !shape_ok(N, K)) return BCQ_ERR_SHAPE;
  if (p < 0 || p > 4 || (p == 0 && !p_row)) return BCQ_ERR_PRECISION;
  for (int m = 0; m < M && p == 0; ++m)
    if (p_row[m] < 1 || p_row[m] > 4) return BCQ_ERR_PRECISION;
  static thread_local Launch launches[BCQ_MAX_M];
  const int n = route_call(M, p, p_row, K, launches);
  out[0] = n;
  for (int i = 0; i < n && i < max_launches; ++i) {
    const Launch& L = launches[i];
    int kind = BCQ_KERNEL_LUT_PAIR;
    if (L.path == kPathM1) kind = BCQ_KERNEL_LUT_ONE;
    else if (L.path == kPathLut4) kind = BCQ_KERNEL_LUT_FOUR;
    else if (L.path == kPathMmaSync) kind = L.mixed ? BCQ_KERNEL_MMA_MIXED : BCQ_KERNEL_MMA;
    else if (L.path == kPathUmma) kind = BCQ_KERNEL_TCGEN05;
    out[1 + 3 * i] = kind;
    out[2 + 3 * i] = L.n;
    out[3 + 3 * i] = L.P;
  }
  return BCQ_OK;
}

int bcq_set_pdl(int mode) {
  if (mode < 0 || mode > 2) return BCQ_ERR_UNSUPPORTED;
  g_pdl_mode.store(mode);
  return BCQ_OK;
}

bcq_status bcq_gemm(const uint16_t* x, const uint32_t* planes, const uint16_t* const alpha[4],
                    const uint16_t* z, int p, const int32_t* p_row, int M, int N, int K,
                    int p_H, int group, uint16_t* y, void* workspace, size_t workspace_bytes,
                    void* stream) {
  const uint16_t* const zq[4] = {z, z, z, z};
  return bcq_gemm_zp(x, planes, alpha, zq, p, p_row, M, N, K, p_H, group, y, workspace,
                     workspace_bytes, stream);
}

bcq_status bcq_gemm_zp(const uint16_t* x, const uint32_t* planes, const uint16_t* const alpha[4],
                       const uint16_t* const z[4], int p, const int32_t* p_row, int M, int N,
                       int K, int p_H, int group, uint16_t* y, void* workspace,
                       size_t workspace_bytes, void* stream) {
  static const uint16_t* const kNoOffsets[4] = {nullptr, nullptr, nullptr, nullptr};
  const uint16_t* const* zq = z ? z : kNoOffsets;
  bcq_status s = validate_gemm(x, planes, alpha, zq, p, p_row, M, N, K, p_H, group, y, workspace,
                               workspace_bytes);
  if (s != BCQ_OK || M == 0) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  return run_gemm(x, planes, alpha, zq, p, p_row, M, N, K, p_H, y, workspace,
                  (cudaStream_t)stream);
}

bcq_status bcq_gemm_host(const uint16_t* x_host, const uint32_t* planes,
                         const uint16_t* const alpha[4], const uint16_t* z, int p,
                         const int32_t* p_row, int M, int N, int K, int p_H, int group,
                         uint16_t* y_host, uint16_t* x_dev, uint16_t* y_dev, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (M > 0 && (!x_host || !y_host)) return BCQ_ERR_NULL;
  const uint16_t* const zq[4] = {z, z, z, z};
  bcq_status s = validate_gemm(x_dev, planes, alpha, zq, p, p_row, M, N, K, p_H, group, y_dev,
                               workspace, workspace_bytes);
  if (s != BCQ_OK || M == 0) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(x_dev, x_host, (size_t)M * K * 2, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return BCQ_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    s = run_gemm(x_dev, planes, alpha, zq, p, p_row, M, N, K, p_H, y_dev, workspace, st);
  }
  if (s != BCQ_OK) return s;
  if (cudaMemcpyAsync(y_host, y_dev, (size_t)M * N * 2, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return BCQ_ERR_CUDA;
  return BCQ_OK;
}

bcq_status bcq_build_lut(const uint16_t* x, int M, int K, float* lut, float* group_sums,
                         void* stream) {
  if (!x || !lut) return BCQ_ERR_NULL;
  if (M < 1 || M > 4 || K < BCQ_GROUP || K % BCQ_GROUP || K > (1 << 22)) return BCQ_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(lut, 4) || (group_sums && !aligned(group_sums, 4)))
    return BCQ_ERR_ALIGN;
  const int G = K / BCQ_GROUP;
  for (int m0 = 0; m0 < M; m0 += kMaxMPerLaunch) {
    const int rows = std::min(kMaxMPerLaunch, M - m0);
    if (launch_lut_dump(x + (size_t)m0 * K, rows, K, lut + (size_t)m0 * (K / 8) * 256,
                        group_sums ? group_sums + (size_t)m0 * G : nullptr,
                        (cudaStream_t)stream) != cudaSuccess)
      return BCQ_ERR_CUDA;
  }
  return BCQ_OK;
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
