// bcq_launch.h -- host-side entry points into the kernels of bcq_kernels.cu.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "bcq.h"
#include "bcq_layout.h"

namespace bcq {

using GemvKernel = void (*)(GemvParams);

cudaError_t launch_pack(const uint32_t* canon, uint32_t* packed, int p_H, int N, int K,
                        cudaStream_t st);

cudaError_t launch_pack_scales(const uint16_t* src, uint16_t* dst, int q, int N, int K,
                               cudaStream_t st);

// The GEMV kernel for M activation rows (1 or 2) streaming P planes; mixed:
// the rows use different precisions.  nullptr if there is none.
GemvKernel gemv_kernel_for(int M, int P, bool mixed);

// The one-row lookup GEMV kernel (bcq_m1.cuh) for precision P; nullptr if
// there is none.
GemvKernel gemv_m1_kernel_for(int P);

// The tensor-core GEMV kernel for NT n-tiles of 8 activation rows (1 or 2)
// streaming P planes (one precision, or mixed: rows of precisions up to P);
// nullptr if there is none.
GemvKernel gemv_mma_kernel_for(int NT, int P, bool mixed);

// The tcgen05 GEMV kernel for up to NN (16 or 64) activation rows streaming
// P planes (one precision); nullptr if there is none.
GemvKernel gemv_umma_kernel_for(int P, int NN);

// p.C CTAs of 32 * (consumer_warps + p.MW + p.NP) threads; cooperative: all
// CTAs resident at once (the launch fails rather than run fewer).
cudaError_t launch_gemv(GemvKernel fn, const GemvParams& p, size_t dyn, bool pdl,
                        cudaStream_t st, int consumer_warps, bool cooperative);

// CTAs of this shape that fit on one SM (also raises the kernel's dynamic
// shared-memory limit to dyn).
cudaError_t blocks_per_sm(GemvKernel fn, int nthreads, size_t dyn, int* out);

cudaError_t launch_lut_dump(const uint16_t* x, int M, int K, float* lut, float* gsum,
                            cudaStream_t st);

cudaError_t launch_wait_probe(unsigned long long limit_ns, cudaStream_t st);

// Synchronises st, returns the device error word in *code and clears it.
cudaError_t read_and_clear_device_error(cudaStream_t st, int* code);

// The argument checks of bcq_gemm (defined in bcq_api.cu).
bcq_status check_gemm_args(const uint16_t* x, const uint32_t* planes,
                           const uint16_t* const alpha[4], const uint16_t* z, int p,
                           const int32_t* p_row, int M, int N, int K, int p_H, int group,
                           const uint16_t* y, const void* ws, size_t ws_bytes);

}  // namespace bcq
