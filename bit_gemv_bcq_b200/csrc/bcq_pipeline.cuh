// bcq_pipeline.cuh -- pieces shared by the GEMV kernels of libbcq (included
// by bcq_kernels.cu only): the CTA's share of the (K-block, row-block) units
// and its groups, the stage wait, the producer warps' bulk-copy ring and the
// split-K reduction through the caller's workspace.
#pragma once

#include <cstdint>

#include "bcq_device.cuh"
#include "bcq_layout.h"

namespace bcq {

// Device error word of this library (one per device): kernels record the
// first problem they hit; bcq_device_error() reads and clears it.  (This
// header belongs to the single translation unit bcq_kernels.cu.)
__device__ int g_device_error = 0;

// The units of one CTA: [u0, u1) in kb-major order (the host's split: see
// plan_units), cut into groups: the row-blocks of one K-block inside one row
// group (at most kRowGroup).
struct CtaRange {
  int u0, u1, NG, kb0, kb_last;
};

__device__ __forceinline__ void make_range(const GemvParams& p, CtaRange& R) {
  const CtaWork w = p.work[blockIdx.x];
  R.u0 = w.u0;
  R.u1 = w.u1;
  R.NG = w.ng;
  R.kb0 = w.kb & 0xFFFF;
  R.kb_last = w.kb >> 16;
}

// Walks the groups of a CTA in order: K-block kb, first row-block rb0, n
// row-blocks (all in row group rb0 / kRowGroup); seg_end bounds the
// row-blocks of kb inside the CTA's range.
struct GroupCursor {
  int kb, rb0, n, seg_end;
};

__device__ __forceinline__ void cursor_init(GroupCursor& c, int u0, int u1, int kb0, int RB) {
  c.kb = kb0;
  c.rb0 = u0 - c.kb * RB;
  c.seg_end = min(RB, u1 - c.kb * RB);
  c.n = min(kRowGroup - (c.rb0 & (kRowGroup - 1)), c.seg_end - c.rb0);
}

__device__ __forceinline__ void cursor_next(GroupCursor& c, int u1, int RB) {
  c.rb0 += c.n;
  if (c.rb0 >= c.seg_end) {
    ++c.kb;
    c.rb0 = 0;
    c.seg_end = min(RB, u1 - c.kb * RB);
  }
  c.n = min(kRowGroup - (c.rb0 & (kRowGroup - 1)), c.seg_end - c.rb0);
}

// Waits for phase `parity` of a stage barrier: a non-blocking test first
// (the common case: the stage has landed), then bounded waiting that gives
// up when the CTA aborts.
__device__ __forceinline__ bool wait_stage(uint32_t bar, uint32_t parity,
                                           volatile int* abort_flag,
                                           unsigned long long limit_ns) {
  if (mbar_test(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
#pragma unroll 1
  while (true) {
    if (*abort_flag) return false;
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

template <int J>
struct Slot {
  static constexpr int value = J;
};

// Producer warp pw of NP: issues stages (groups) k = pw, pw + NP, ...; with D
// a multiple of NP it alone refills its ring slots, so the empty-barrier
// phase it waits for is never two phases behind.  Stage g holds the first P
// planes of group g (plane i at i * 8 KiB, row-block rb0 + w at w KiB): a
// whole row group is one bulk copy, a partial one (at the ends of the CTA's
// range) one copy per plane.  Lane 0 issues; the warp returns when every
// copy it issued has landed (or the CTA gave up).
template <int P>
__device__ __forceinline__ void produce_stages(const GemvParams& prm, const CtaRange& R, int pw,
                                               int lane, uint32_t ring, uint32_t full0,
                                               uint32_t empty0, volatile int* abort_flag) {
  constexpr uint32_t kStage = gemv_stage_bytes(P);
  const int D = prm.D, NP = prm.NP, RB = prm.RB;
  if (!prm.early_weights) grid_dependency_wait();
  if (lane == 0) {
    const uint64_t pol = evict_first_policy();  // planes are read once per call
    int issued = 0;
    GroupCursor gc;
    cursor_init(gc, R.u0, R.u1, R.kb0, RB);
    if (pw) cursor_next(gc, R.u1, RB);
    int s = pw;        // ring slot of stage k (incremental: no division)
    uint32_t eph = 1;  // parity of the empty phase that frees slot s (stage k - D)
    for (int k = pw; k < R.NG; k += NP) {
      if (k >= D && !mbar_wait_bounded(empty0 + 8u * s, eph, prm.timeout_ns)) {
        record_error(&g_device_error, BCQ_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      if (*abort_flag) break;
      const uint32_t bar = full0 + 8u * s;
      const uint32_t dst = ring + (uint32_t)s * kStage;
      const int rg = gc.rb0 / kRowGroup, r0 = gc.rb0 - rg * kRowGroup;
      const uint32_t* src =
          prm.planes + ((size_t)gc.kb * prm.RG + rg) * prm.p_H * (kRowGroup * kWordsPerUnitPlane);
      mbar_arrive_expect_tx(bar, (uint32_t)(P * gc.n) * kUnitPlaneBytes);
      if (gc.n == kRowGroup) {
        bulk_g2s_hint(dst, src, kStage, bar, pol);
      } else {
#pragma unroll
        for (int i = 0; i < P; ++i)
          bulk_g2s_hint(dst + (uint32_t)i * kPlaneGroupBytes,
                        src + (size_t)(i * kRowGroup + r0) * kWordsPerUnitPlane,
                        (uint32_t)gc.n * kUnitPlaneBytes, bar, pol);
      }
      issued = k + 1;
      for (int t = 0; t < NP; ++t) cursor_next(gc, R.u1, RB);
      s += NP;
      if (s >= D) {
        s -= D;
        eph ^= 1u;
      }
    }
    // every copy this warp issued lands before the CTA may exit
    for (int s2 = pw; s2 < D && s2 < issued; s2 += NP) {
      const int klast = issued - 1 - ((issued - 1 - s2) % D);
      (void)mbar_wait_bounded(full0 + 8u * s2, (uint32_t)((klast / D) & 1), prm.timeout_ns);
    }
  }
  __syncwarp();
}

// One reduction task of splitk_tail: the lane's row of launch rows m0 ..
// m0 + NM - 1 (pp: its first partial), all KB K-blocks, kC at a time; sums
// them in K-block order into sum[] and zeroes them.  FULL: KB is a multiple
// of kC (no guard on the loads).  False when a wait ran out (warp-uniform).
template <int kC, int NM, bool FULL>
__device__ __forceinline__ bool reduce_task(const GemvParams& prm, float* pp, size_t part_stride,
                                            size_t kstride, int KB, float (&sum)[2],
                                            volatile int* abort_flag) {
  for (int k0 = 0; k0 < KB; k0 += kC) {
    float* pk = pp + (size_t)k0 * kstride;
    uint32_t v[NM][kC];  // every load of the chunk in flight at once
#pragma unroll
    for (int mm = 0; mm < NM; ++mm) {
      const float* pl = pk + (size_t)mm * part_stride;
#pragma unroll
      for (int j = 0; j < kC; ++j) {
        v[mm][j] = (FULL || k0 + j < KB) ? ld_partial_tag(pl) : 1u;
        pl += kstride;
      }
    }
    bool have = true;
#pragma unroll
    for (int mm = 0; mm < NM; ++mm)
#pragma unroll
      for (int j = 0; j < kC; ++j) have = have && v[mm][j] != 0u;
    if (!__all_sync(0xFFFFFFFFu, have)) {
      // some partials are still on their way: re-load the missing ones
      const unsigned long long t0 = globaltimer_ns();
#pragma unroll 1
      while (true) {
        __nanosleep(32);
        have = true;
#pragma unroll
        for (int mm = 0; mm < NM; ++mm)
#pragma unroll
          for (int j = 0; j < kC; ++j) {
            if (v[mm][j] == 0u)
              v[mm][j] = ld_partial_tag(pk + (size_t)mm * part_stride + (size_t)j * kstride);
            have = have && v[mm][j] != 0u;
          }
        if (__all_sync(0xFFFFFFFFu, have)) break;
        // (warp-uniform: every lane leaves the loop together)
        if (__any_sync(0xFFFFFFFFu, *abort_flag != 0 || globaltimer_ns() - t0 > prm.timeout_ns))
          return false;
      }
    }
#pragma unroll
    for (int mm = 0; mm < NM; ++mm) {
      float* pz = pk + (size_t)mm * part_stride;
#pragma unroll
      for (int j = 0; j < kC; ++j) {
        if (FULL || k0 + j < KB) {
          sum[mm] += partial_value(v[mm][j]);
          // the workspace is left zero-filled for any later shape
          stg_cg_zero(pz);
        }
        pz += kstride;
      }
    }
  }
  return true;
}

// Split-K reduction, run by each of the CTA's nthreads consumer threads once
// its warp has stored its own partial sums (no barrier).  Every unit's fp32
// partials [kb][m][row] go to the workspace as tagged words (st_partial: zero
// = not written yet), so no fence or arrival counter is needed: a reducer
// polls the partials themselves.  The polling needs every CTA of the grid
// to run: the GEMV kernels are launched cooperatively (one CTA per SM at
// most, cudaLaunchAttributeCooperative), so the launch makes all of them
// resident at once, whatever else holds the GPU.  Row-block rb is reduced by the CTA that
// computed its unit in K-block rb mod KB, so the work is spread evenly
// whatever the order in which CTAs finish.  The (row-block, two launch rows)
// tasks of the CTA are dealt to its warps in turn; a warp loads all KB
// partials of its task kC K-blocks at a time (one round trip each), re-loads
// (bounded) those still zero, adds them in K-block order (the result does not
// depend on scheduling), writes y (row m of the launch goes to y row ymap[m],
// or m without a map) and zeroes those partials, so the workspace is zero
// again for the next call.
template <int kC>
__device__ __forceinline__ void splitk_tail(const GemvParams& prm, const CtaRange& R, int Mrows,
                                            const int* ymap, int tid, int nthreads,
                                            volatile int* abort_flag) {
  const int RB = prm.RB, KB = prm.KB;
  const int lane = tid & 31, warp = tid >> 5, nwarps = nthreads >> 5;
  const size_t part_stride = (size_t)RB * kRowBlock;
  const size_t kstride = (size_t)Mrows * part_stride;  // one K-block of partials
  const bool live = *abort_flag == 0;
  const bool full = KB % kC == 0;
  // Tasks are dealt round-robin (no division), starting at the first warp of
  // the second team: the first team takes the odd group out of an odd
  // number, so the second team is done first and polls earlier (measured:
  // M = 1 calls 1-3 % faster than dealing from warp 0).
  int task = 0, mine = warp ^ (nwarps >> 1);
  for (int kb = R.kb0; kb <= R.kb_last && live; ++kb) {
    const int a = kb == R.kb0 ? R.u0 - kb * RB : 0;
    const int b = kb == R.kb_last ? R.u1 - kb * RB : RB;
    int first = kb;  // designated row-blocks: kb, kb + KB, ...
    if (first < a) first += (a - first + KB - 1) / KB * KB;
    const int mp = (Mrows + 1) >> 1;  // tasks per row-block: two launch rows each
    for (int rbx = first; rbx < b; rbx += KB) {
      if (mine >= task + mp) {  // none of this row-block's tasks is this warp's
        task += mp;
        continue;
      }
      for (int m0 = 0; m0 < Mrows; m0 += 2, ++task) {
        if (task != mine) continue;
        mine += nwarps;
        const int row = rbx * kRowBlock + lane;
        const int nm = Mrows - m0 < 2 ? Mrows - m0 : 2;
        float* pp = prm.part + (size_t)m0 * part_stride + (size_t)row;
        float sum[2] = {0.f, 0.f};
        const bool ok =
            nm == 2 ? (full ? reduce_task<kC, 2, true>(prm, pp, part_stride, kstride, KB, sum, abort_flag)
                            : reduce_task<kC, 2, false>(prm, pp, part_stride, kstride, KB, sum, abort_flag))
                    : (full ? reduce_task<kC, 1, true>(prm, pp, part_stride, kstride, KB, sum, abort_flag)
                            : reduce_task<kC, 1, false>(prm, pp, part_stride, kstride, KB, sum, abort_flag));
        if (!ok) {
          if (lane == 0 && *abort_flag == 0) {
            record_error(&g_device_error, BCQ_ERR_TIMEOUT);
            *abort_flag = 1;
          }
          continue;
        }
        if (row < prm.N) {
          prm.y[(size_t)(ymap ? ymap[m0] : m0) * prm.N + row] = f2h_rn(sum[0]);
          if (nm == 2) prm.y[(size_t)(ymap ? ymap[m0 + 1] : m0 + 1) * prm.N + row] = f2h_rn(sum[1]);
        }
      }
    }
  }
}

}  // namespace bcq
