/*
 * bcq.h -- C ABI of libbcq, the B200 (sm_100a) multi-precision
 * binary-coded-quantization (BCQ) matmul.
 *
 *   y[m][n] = sum_k x[m][k] * W_hat[n][k]
 *   W_hat[n][k] = sum_{i=1..p_m} alpha^(p_m)[n][g][i-1] * B_i[n][k] + z[n][g],
 *   g = k / 128,  B_i[n][k] in {-1, +1}
 *
 * Sources (page title, section):
 *   "AnyBCQ: Hardware Efficient Flexible Binary-Coded Quantization for
 *   Multi-Precision LLMs" (Paper-Notes page):
 *     - "研究背景与动机 / 切入角度": weights are a sum of scaled binary
 *       bit-planes; p-bit inference touches p planes;
 *     - "关键设计 / 渐进式精度扩展": planes are shared by every precision and
 *       each precision p has its own scales alpha^(p);
 *     - "关键设计 / 直接bit-plane运算的CUDA内核": the kernel loads one plane at
 *       a time, turns the contraction into additions and subtractions of
 *       cached +-x partial sums (a LUT), scales by alpha_i and accumulates;
 *       a p-bit call loads only the first p planes;
 *     - "训练策略": asymmetric, group-wise with group size 128;
 *     - "吞吐量" and the arXiv abstract: per-request precision selection.
 *
 * Conventions shared by every entry point
 *   - Every buffer is owned by the caller.  Device pointers must point to
 *     memory of the current CUDA device; "host" pointers to host memory.
 *   - fp16 data is passed as its IEEE binary16 bit pattern (uint16_t).
 *   - Canonical bit-planes: uint32 [p_H][N][K/32]; bit j of word w of row n is
 *     column 32w + j (LSB first); bit value 1 means +1, 0 means -1.
 *   - `stream` is a cudaStream_t of the current device passed as void* (NULL =
 *     legacy default stream).
 *     Work is enqueued asynchronously on it; the call returns after the launch.
 *   - Every argument is validated before anything is launched.  A call that
 *     returns an error status has launched nothing and touched no buffer.
 *   - BCQ_ERR_CUDA reports a failed launch or copy (cudaGetLastError); the
 *     CUDA error itself can be read with cudaGetLastError() by the caller.
 *   - Kernels never wait without a limit.  A wait that runs out sets a device
 *     error word (read with bcq_device_error) and the kernel returns early;
 *     its outputs are then unspecified.
 *   - The library allocates no device memory.  Calls whose split-K partial
 *     sums need room take a caller-owned workspace (bcq_workspace_bytes).
 */
#ifndef BCQ_H_
#define BCQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bcq_status {
  BCQ_OK = 0,
  BCQ_ERR_NULL = 1,         /* a required pointer is NULL                      */
  BCQ_ERR_SHAPE = 2,        /* M, N or K out of range, or K not a multiple of 128 */
  BCQ_ERR_PRECISION = 3,    /* p / p_row / p_H out of range, or a needed alpha is NULL */
  BCQ_ERR_ALIGN = 4,        /* a device pointer breaks its alignment rule      */
  BCQ_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed            */
  BCQ_ERR_TIMEOUT = 6,      /* a bounded wait inside a kernel ran out          */
  BCQ_ERR_UNSUPPORTED = 7,  /* valid request this build does not handle (e.g. group != 128) */
  BCQ_ERR_SCRATCH = 8       /* bcq_gemm_noalloc: the call needs more scratch than it has */
} bcq_status;

#define BCQ_GROUP 128       /* columns per scale group                          */
#define BCQ_MAX_PLANES 4    /* p_H <= 4                                         */
#define BCQ_MAX_M 64        /* rows of x per call                               */
#define BCQ_NOALLOC_SCRATCH_BYTES (16u << 20)  /* bcq_gemm_noalloc's built-in scratch */

/* Human-readable name of a status code.  Never NULL. */
const char* bcq_status_string(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
int bcq_version(void);

/*
 * Size in bytes of the packed plane buffer for p_H planes of an N x K weight
 * (rows padded to a multiple of 32, columns to a multiple of 256): exactly
 * 1 KiB per (plane, 32 rows, 256 columns).  Returns 0
 * for invalid shapes (p_H outside 1..4, N < 1, K < 128 or K % 128 != 0).
 */
size_t bcq_packed_planes_bytes(int p_H, int N, int K);

/*
 * Repack canonical bit-planes into the streaming layout bcq_gemm reads.
 * Offline, once per weight matrix (the format of the stored planes is shared
 * by every precision: AnyBCQ page, "渐进式精度扩展").
 *
 *   planes_canon   device, uint32 [p_H][N][K/32], 4-byte aligned, read only.
 *   planes_packed  device, bcq_packed_planes_bytes(p_H, N, K) bytes, 16-byte
 *                  aligned, written entirely (padding included).  Its layout
 *                  is private to the library; plane i occupies its own
 *                  sub-blocks so that a p-bit call reads planes 0..p-1 only.
 * Errors: NULL pointers -> BCQ_ERR_NULL; p_H outside 1..4 -> BCQ_ERR_PRECISION;
 * N < 1, K < 128, K % 128 != 0 -> BCQ_ERR_SHAPE; misaligned -> BCQ_ERR_ALIGN.
 */
bcq_status bcq_pack_planes(const uint32_t* planes_canon, uint32_t* planes_packed,
                           int p_H, int N, int K, void* stream);

/*
 * Size in bytes of a packed per-(row, group) array with q values per entry
 * (q = 1..4; rows padded to a multiple of 32, groups to an even count), or 0
 * for invalid arguments (same shape rules as above).
 */
size_t bcq_packed_scales_bytes(int q, int N, int K);

/*
 * Repack a per-(row, group) fp16 array into the streaming order bcq_gemm
 * reads, next to the planes of the same rows and groups.  Offline, once per
 * weight matrix.  Used for the scales of each precision (AnyBCQ page,
 * "渐进式精度扩展": every precision p has its own alpha^(p)) with q = p, and
 * for the asymmetric offsets z ("训练策略") with q = 1.
 *
 *   src   device, fp16 [N][K/128][q] (entry (n, g) holds q values), 2-byte
 *         aligned, read only.
 *   dst   device, bcq_packed_scales_bytes(q, N, K) bytes, 16-byte aligned,
 *         written entirely (zero padding outside the matrix).
 * Errors: NULL -> BCQ_ERR_NULL; q outside 1..4 -> BCQ_ERR_PRECISION; shape ->
 * BCQ_ERR_SHAPE; misaligned -> BCQ_ERR_ALIGN.
 */
bcq_status bcq_pack_scales(const uint16_t* src, int q, int N, int K,
                           uint16_t* dst, void* stream);

/*
 * Bytes of workspace bcq_gemm needs for M rows of x and an N x K weight: 0
 * when K <= 256 (no split over K), else room for the fp32 partial sums of
 * every (256-column K-block, row) for the rows of the largest launch
 * (min(M, 64)), rows padded to a multiple of 32:
 * ceil(K / 256) * min(M, 64) * ceil(N / 32) * 32 * 4 bytes.  0 for invalid
 * shapes as well.
 */
size_t bcq_workspace_bytes(int M, int N, int K);

/*
 * y = x . W_hat^T for M rows of x, each row at its own precision.
 *
 *   x        device, fp16 [M][K] row-major, 16-byte aligned.
 *   planes   device, packed planes from bcq_pack_planes (p_H, N, K).
 *   alpha    PACKED scales only: canonical [N][K/128][q] arrays are not
 *            accepted (they would be read in the wrong order, with no error);
 *            pass each through bcq_pack_scales(.., q, ..) first.  HOST array
 *            of 4 device pointers; alpha[q-1] -> the packed scales of
 *            precision q (alpha^(q)[n][g][i], i = plane).  It must be
 *            non-NULL for every precision used by the call; the others may be
 *            NULL.  16-byte aligned.
 *   z        PACKED offsets only (canonical [N][K/128] arrays go through
 *            bcq_pack_scales(.., 1, ..) first), or NULL (= 0).  16-byte
 *            aligned.
 *   p        uniform precision 1..p_H for every row, or 0 to use p_row.
 *   p_row    HOST array int32 [M] of precisions 1..p_H (read during the call
 *            only), or NULL when p > 0.
 *   M        rows of x, 0..BCQ_MAX_M (0 = nothing to do, returns BCQ_OK).
 *   N, K     weight shape; K % 128 == 0, K >= 128, N >= 1.
 *   p_H      planes stored in `planes` (1..4).
 *   group    must be 128 (other sizes -> BCQ_ERR_UNSUPPORTED).
 *   y        device, fp16 [M][N] row-major, overwritten; 2-byte aligned.
 *   workspace, workspace_bytes
 *            device scratch of at least bcq_workspace_bytes(M, N, K) bytes,
 *            16-byte aligned (NULL allowed when that is 0).  Zero-fill it once
 *            before its first use; every call that completes without a device
 *            error leaves it zero-filled again (zero it again after
 *            BCQ_ERR_TIMEOUT).  Calls that may run at the same time (other
 *            streams) need workspaces of their own; calls in one stream may
 *            share one.
 * Launches: one GEMV kernel per group of rows, each a cooperative launch of
 * at most one CTA per SM: all its CTAs are resident at once, so the split-K
 * reduction at its end (a CTA polls the partial sums other CTAs of the grid
 * store) completes whatever else runs on the GPU.
 * The call reads planes 0..max_m(p_m)-1 only.  Accumulation is fp32; each
 * output is rounded once to fp16 (round to nearest even).  Partial sums over
 * 256-column K-blocks are added in a fixed order, so for a given device and
 * shape the result does not depend on scheduling: results are reproducible.
 * Errors: as listed above; workspace too small or NULL -> BCQ_ERR_NULL;
 * misaligned workspace -> BCQ_ERR_ALIGN.
 */
bcq_status bcq_gemm(const uint16_t* x, const uint32_t* planes,
                    const uint16_t* const alpha[4], const uint16_t* z,
                    int p, const int32_t* p_row, int M, int N, int K, int p_H,
                    int group, uint16_t* y, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * bcq_gemm with offsets per precision: row m uses z^(p_m) with its scales
 * alpha^(p_m), i.e. W_hat^(p)[n][k] = sum_{i<p} alpha^(p)[n][g][i] B_i[n][k]
 * + z^(p)[n][g].  The pages write the offset without a precision index
 * (AnyBCQ page, "训练策略": asymmetric quantisation); this entry point is the
 * variant in which every precision keeps its own offsets, as the expansion
 * in "渐进式精度扩展" keeps its own scales.
 *
 *   z   HOST array of 4 device pointers, or NULL (no offsets); z[q-1] -> the
 *       offsets of precision q (canonically fp16 [N][K/128]) packed by
 *       bcq_pack_scales(.., 1, ..), or NULL (= 0 for that precision).  Only
 *       the precisions used by the call are read; 16-byte aligned.
 * Every other argument, the result and the errors are those of bcq_gemm;
 * bcq_gemm(.., z, ..) is bcq_gemm_zp with z[0..3] all equal to z.
 */
bcq_status bcq_gemm_zp(const uint16_t* x, const uint32_t* planes,
                       const uint16_t* const alpha[4], const uint16_t* const z[4],
                       int p, const int32_t* p_row, int M, int N, int K, int p_H,
                       int group, uint16_t* y, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * The launch plan bcq_gemm would use for one launch of M (1..64) activation
 * rows streaming p_load planes (mixed = 1: rows of different precisions, at
 * most 16).  M = 1 plans the one-row lookup kernel (K > 256; else the
 * pair-table kernel), M = 2 the pair-table kernel, mixed M >= 3 the mixed
 * tensor-core kernel, 3 <= M <= 4 of one precision the four-row lookup
 * launch (two pair tables), 5 <= M <= 16 the tensor-core kernel that
 * bcq_gemm would use for a batch (BCQ_MMA_KIND), and M >= 17 the 64-row
 * tcgen05 launch; the same switches as bcq_gemm apply.  use_device = 1
 * plans for the current device; 0 (or no usable device) plans for a nominal
 * 148-SM B200 without touching CUDA.  out[8] receives: CTAs, consumer warps,
 * producer warps, ring stages, dynamic shared memory bytes, bytes per ring
 * stage, largest number of units (K-block x row-block pairs) of one CTA,
 * K-blocks (partial sums per output).  For inspection and tests.
 */
int bcq_plan_query(int M, int N, int K, int p_load, int mixed, int use_device, int* out);

/* Kernels of a launch, as bcq_route_query reports them. */
enum {
  BCQ_KERNEL_LUT_PAIR = 1,   /* lookup table, 1-2 rows (pair tables; mixed pairs) */
  BCQ_KERNEL_LUT_ONE = 2,    /* lookup table, one row, dense table (K > 256) */
  BCQ_KERNEL_LUT_FOUR = 3,   /* lookup table, 3-4 rows of one precision */
  BCQ_KERNEL_MMA = 4,        /* tensor cores (mma.sync), up to 16 rows of one precision */
  BCQ_KERNEL_MMA_MIXED = 5,  /* tensor cores (mma.sync), up to 16 rows of several precisions */
  BCQ_KERNEL_TCGEN05 = 6     /* tensor cores (tcgen05), up to 64 rows of one precision */
};

/*
 * The launches bcq_gemm (or bcq_gemm_zp) makes for M rows at precision p (or
 * p_row, HOST [M], when p = 0) on an N x K weight, without launching
 * anything (the same routing code): out[0] = number of launches L; for
 * launch i < max_launches,
 * out[1 + 3i], out[2 + 3i], out[3 + 3i] = kernel (BCQ_KERNEL_*), rows, planes
 * streamed.  out needs 1 + 3 * max_launches ints.  A mixed batch of up to 16
 * rows is one launch that streams the planes once, up to its largest
 * precision (AnyBCQ page, "吞吐量": each request at its own precision).
 * Errors: out NULL -> BCQ_ERR_NULL; M, N, K -> BCQ_ERR_SHAPE; p / p_row
 * outside 1..4 -> BCQ_ERR_PRECISION.
 */
int bcq_route_query(int M, int p, const int32_t* p_row, int N, int K, int* out,
                    int max_launches);

/*
 * Launch option for the GEMV kernels of this process (all devices):
 *   0  plain stream order (default);
 *   1  programmatic dependent launch: a GEMV kernel may be scheduled while the
 *      preceding kernel in its stream finishes; it touches no global memory
 *      before that kernel has completed;
 *   2  as 1, but the kernel may start streaming its weights (planes, and in
 *      the one-row kernel also the packed scales and offsets) before the
 *      preceding kernel has completed (x, y and the workspace still wait).
 *      Only valid when no kernel immediately before it in the stream writes
 *      the planes, scales or offsets it reads.
 * Returns BCQ_OK, or BCQ_ERR_UNSUPPORTED for another mode.
 */
int bcq_set_pdl(int mode);

/*
 * bcq_gemm with x and y in HOST memory: enqueues the copy of x_host into
 * x_dev, the matmul, and the copy of y_dev back into y_host, all on `stream`
 * (pinned host buffers make the copies asynchronous).  x_dev (fp16 [M][K],
 * 16-byte aligned) and y_dev (fp16 [M][N]) are caller-owned device staging
 * buffers; workspace as for bcq_gemm.  The caller synchronises `stream`
 * before reading y_host.
 * Errors as bcq_gemm, plus BCQ_ERR_NULL for missing host or staging buffers.
 */
bcq_status bcq_gemm_host(const uint16_t* x_host, const uint32_t* planes,
                         const uint16_t* const alpha[4], const uint16_t* z,
                         int p, const int32_t* p_row, int M, int N, int K,
                         int p_H, int group, uint16_t* y_host,
                         uint16_t* x_dev, uint16_t* y_dev, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * bcq_gemm without a caller workspace, for callers that cannot allocate
 * device memory: code that runs where cudaMalloc is not allowed (inside a
 * memory pool or allocator that must not recurse into itself, a plug-in whose
 * host framework owns every allocation, or a real-time loop that must not
 * block on the driver's allocator) still needs the split-K scratch that
 * bcq_gemm takes as `workspace`.  This entry point uses a scratch array that
 * is part of the library itself instead.  The paper has no counterpart: it
 * is a packaging choice of this library, not part of the method.
 *
 * Arguments, results and errors are those of bcq_gemm, without workspace and
 * workspace_bytes.  In addition:
 *   - The scratch is one static device array of BCQ_NOALLOC_SCRATCH_BYTES
 *     (16 MiB), held on every GPU that loads the library until the process
 *     exits.  A call whose bcq_workspace_bytes(M, N, K) exceeds it returns
 *     BCQ_ERR_SCRATCH and launches nothing; use bcq_gemm for such shapes.
 *   - Each call looks up the array's device address (cudaGetSymbolAddress,
 *     with the call's device current) unless `stream` is capturing a CUDA
 *     graph, when the address found by the last such lookup on that device
 *     is used: make one call on a device before any stream capture on it.
 *     (Looking it up again on every call keeps it right after a device or
 *     context reset, which loads the library's device code anew.)
 *   - Each call clears the part of the scratch it uses (cudaMemsetAsync on
 *     `stream`) before its kernels.  Nothing is allocated, by this call or
 *     by any routine it calls.
 *   - Every call on a device shares the one array.  Calls that may overlap on
 *     the GPU (different streams, or other threads' streams) race on it and
 *     their results are undefined; serialise them, or use bcq_gemm with a
 *     workspace per stream.
 */
bcq_status bcq_gemm_noalloc(const uint16_t* x, const uint32_t* planes,
                            const uint16_t* const alpha[4], const uint16_t* z,
                            int p, const int32_t* p_row, int M, int N, int K,
                            int p_H, int group, uint16_t* y, void* stream);

/*
 * Offline quantiser: fp16 weights -> shared bit-planes, per-precision scales
 * alpha^(p) for p = p_L..p_H and one offset per group, in the canonical
 * layouts that bcq_pack_planes / bcq_pack_scales take.
 *
 * Source: AnyBCQ (Paper-Notes page), "关键设计 / 渐进式精度扩展" (greedy start
 * and alternating refinement -- least squares for the scales, nearest code
 * for every weight -- at the base precision p_L; each expansion p -> p + 1
 * keeps B_1..B_p, appends B_{p+1} = sign(R_p), the sign of the residual, and
 * refits all p + 1 scales by least squares) and "训练策略" (asymmetric,
 * group size 128, 20 refinement rounds).  Each 128-column group of each row
 * is an independent problem, computed in fp64:
 *   - greedy start: z = mean(w); for i = 1..p_L: b_i = sign(r) (sign(0) = +1),
 *     alpha_i = <b_i, r> / 128, r -= alpha_i b_i, from r = w - z;
 *   - `rounds` times: (z, alpha) = joint least squares for the current codes;
 *     then every weight takes the code whose value
 *     z + (((alpha_1 b_1) + alpha_2 b_2) + ...) is nearest (ties: the code with
 *     the smallest index c, b_i = +1 where bit i of c is set); then a final
 *     least-squares refit.  z is kept from here on;
 *   - in a least-squares fit, a column (the all-ones column of z first, then
 *     planes 1..p) that is an exact linear combination of the columns before
 *     it gets scale 0;
 *   - scales and offsets are rounded to fp16 (nearest even) when stored.
 *
 *   w       device, fp16 [N][K] row-major, 2-byte aligned, read only.
 *   N, K    N >= 0, K >= 0, K % 128 == 0 (N == 0 or K == 0: nothing to do).
 *   p_L, p_H  1 <= p_L <= p_H <= 4.
 *   rounds  refinement rounds at p_L, 0..1000 (the page uses 20).
 *   planes  device, uint32 [p_H][N][K/32], 4-byte aligned, overwritten
 *           (bit j of word w of row n = column 32w + j, 1 = +1).
 *   alpha   HOST array of 4 device pointers; alpha[p-1] for p = p_L..p_H
 *           receives fp16 [N][K/128][p] (2-byte aligned); the others are
 *           ignored and may be NULL.
 *   z       device, fp16 [N][K/128], 2-byte aligned, overwritten.
 *   sse     device, fp64 [p_H - p_L + 1][N][K/128], 8-byte aligned, or NULL:
 *           the squared error of every group at precision p_L + j with the
 *           unrounded scales.
 * Errors: NULL pointers -> BCQ_ERR_NULL; p_L / p_H out of range or a needed
 * alpha NULL -> BCQ_ERR_PRECISION; bad N, K or rounds -> BCQ_ERR_SHAPE;
 * misaligned pointers -> BCQ_ERR_ALIGN; launch failure -> BCQ_ERR_CUDA.
 */
bcq_status bcq_quantize(const uint16_t* w, int N, int K, int p_L, int p_H, int rounds,
                        uint32_t* planes, uint16_t* const alpha[4], uint16_t* z,
                        double* sse, void* stream);

/*
 * bcq_quantize for the per-precision offsets of bcq_gemm_zp: the same steps,
 * except that each expansion p -> p + 1 refits the offset z^(p+1) jointly
 * with the p + 1 scales (least squares with the all-ones column first, as at
 * the base precision) and the residual of precision p uses z^(p).
 *
 *   z   HOST array of 4 device pointers; z[p-1] for p = p_L..p_H receives
 *       fp16 [N][K/128] (2-byte aligned), the others are ignored; z^(p_L) is
 *       the offset bcq_quantize would write.
 * Every other argument and error is that of bcq_quantize (a NULL z or a
 * NULL z[p-1] in p_L..p_H -> BCQ_ERR_NULL).
 */
bcq_status bcq_quantize_zp(const uint16_t* w, int N, int K, int p_L, int p_H, int rounds,
                           uint32_t* planes, uint16_t* const alpha[4], uint16_t* const z[4],
                           double* sse, void* stream);

/*
 * The lookup table and group sums exactly as the GEMV kernel builds them in
 * shared memory (AnyBCQ page, "直接bit-plane运算的CUDA内核": cached signed
 * partial sums of x).  For test and inspection.
 *
 *   x           device, fp16 [M][K], 16-byte aligned; 1 <= M <= 4.
 *   lut         device, fp32 [M][K/8][256]:
 *               lut[m][c][b] = sum_{j<8} (2*bit_j(b) - 1) * x[m][8c + j].
 *   group_sums  device, fp32 [M][K/128]: sum of x[m] over each group; may be NULL.
 */
bcq_status bcq_build_lut(const uint16_t* x, int M, int K, float* lut,
                         float* group_sums, void* stream);

/*
 * Synchronises `stream`, then returns and clears the device error word of
 * the current device: BCQ_OK when no kernel reported a problem, otherwise
 * the status a kernel recorded (BCQ_ERR_TIMEOUT for a wait that ran out).
 * Returns BCQ_ERR_CUDA if the synchronisation or the read fails.
 */
bcq_status bcq_device_error(void* stream);

/*
 * Test hook for the bounded waits: launches one CTA that waits on a
 * shared-memory barrier nothing will complete, using the same bounded-wait
 * routine as the GEMV kernel, with a limit of `limit_us` microseconds
 * (1..1000000).  The kernel records BCQ_ERR_TIMEOUT in the device error word
 * and returns; read it with bcq_device_error().  Faults nothing.
 */
bcq_status bcq_debug_wait_timeout(int limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BCQ_H_ */
