// bcq_launch.h -- host-side entry points into the kernels of bcq_kernels.cu.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "bcq_layout.h"

namespace bcq {

using GemvKernel = void (*)(GemvParams);

cudaError_t launch_pack(const uint32_t* canon, uint32_t* packed, int p_H, int N,
                        int K, cudaStream_t st);

// The GEMV kernel for M activation rows (1 or 2); nullptr otherwise.
GemvKernel gemv_kernel_for(int M);

cudaError_t launch_pack_scales(const uint16_t* src, uint16_t* dst, int q, int N,
                               int K, cudaStream_t st);

// p.W consumer warps + p.NP producer warps per CTA.
cudaError_t launch_gemv(GemvKernel fn, const GemvParams& p, int C, int W,
                        size_t dyn, bool pdl, cudaStream_t st);

cudaError_t max_active_clusters(GemvKernel fn, int S, int nthreads, size_t dyn, int* out);

cudaError_t launch_lut_dump(const uint16_t* x, int M, int K, float* lut,
                            float* gsum, cudaStream_t st);

cudaError_t launch_wait_probe(unsigned long long limit_ns, cudaStream_t st);

// Synchronises st, returns the device error word in *code and clears it.
cudaError_t read_and_clear_device_error(cudaStream_t st, int* code);

}  // namespace bcq
