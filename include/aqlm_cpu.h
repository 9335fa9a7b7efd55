/*
 * aqlm_cpu.h -- C ABI of libaqlm_cpu.so: the AQLM weight-only linear layer on the
 * host CPU (multithreaded; AVX2/FMA/F16C and AVX-512 where the CPU has them).
 *
 * The AQLM repo summary ("Additive quantization that actually survives one-bit
 * weights", section "Key highlights") lists CPU inference among the format's
 * options, and the inference-research record "AQLM (additive / multi-codebook
 * quantization)", section "Kernels", names the lookup route used here for B = 8
 * codebooks: per group of g inputs and codebook m, a table of x . codeword for all
 * 256 entries, after which every weight group costs M table reads instead of g
 * multiply-adds.
 *
 * This library is separate from libaqlm.so (the GPU path).  Neither calls the
 * other: a GPU call never falls back to this code, and this code never touches a
 * GPU.  It computes the same definition as aqlm_matmul:
 *
 *   y = x . W^T . diag(scales) + bias,   W[n, j*g + t] = sum_m C_m[codes[n, j, m]][t]
 *
 * Layouts (row-major, caller-owned HOST memory):
 *   x          fp16   [batch, K]
 *   codes      uint8 (B = 8) / uint16 (B = 16)   [N, K/g, M]
 *   codebooks  fp16   [M, 2^B, g]
 *   scales     fp16   [N]
 *   bias       fp16   [N] or NULL
 *   y          fp16   [batch, N]  (written; must not overlap the inputs)
 * Supported schemes: those of aqlm.h (B = 8 with M = 1..4, B = 16 with M = 1..2,
 * g = 8 or 16).  Accumulation is fp32; y is rounded to fp16 (round to nearest
 * even).  Tolerance against the fp64 reference of the decoded fp16 weights:
 * max|y - y_ref| / max|y_ref| <= 5e-3.
 *
 * Methods: lookup tables, built per K slice of 16 groups and read for every output
 * row (threads take slices and keep per-thread partial sums, added in thread order
 * at the end); decode + dot, where each thread decodes its output rows to fp32 one at
 * a time and takes dot products with every batch row; and, with AVX-512, fused decode
 * + dot, where 16 weights at a time are decoded in registers and multiplied into
 * accumulators of up to 8 batch rows, nothing decoded being stored.  At SIMD level 2
 * B = 8 at batch 1 uses the lookup tables and everything else the fused method; at
 * levels 0 and 1 B = 8 at batch <= 8 uses the lookup tables and everything else
 * decode + dot.  The result is deterministic for a given nthreads and SIMD level (the
 * fused method's does not depend on nthreads).
 *
 * nthreads: 0 = the OpenMP default, else that many threads.  The call allocates
 * host scratch (tables, partial sums; released before it returns).
 *
 * Errors (aqlm_status from aqlm.h): AQLM_ERR_INVALID_ARG for NULL pointers,
 * K % g != 0, non-positive sizes, batch > 65535, nthreads < 0 or outputs that
 * overlap inputs; AQLM_ERR_UNSUPPORTED for other schemes; AQLM_ERR_MISALIGNED if a
 * pointer is not aligned to its element (2 bytes for fp16 and uint16).  No
 * alignment beyond that is needed.  Never aborts.
 */
#ifndef AQLM_CPU_H_
#define AQLM_CPU_H_

#include "aqlm.h"

#ifdef __cplusplus
extern "C" {
#endif

aqlm_status aqlm_cpu_matmul(const void* x, const void* codes, const void* codebooks,
                            const void* scales, const void* bias, void* y,
                            int M, int B, int g, int K, int N, int batch, int nthreads);

/* SIMD level the kernels run with on this CPU: 0 = portable scalar code,
 * 1 = AVX2 + FMA + F16C, 2 = AVX-512 F, BW and VL as well.  At most the cap set
 * below. */
int aqlm_cpu_simd_level(void);

/* Caps the SIMD level (clamped to 0..2) for every later call in the process, so
 * that the lower levels can be run and tested on a CPU that has the higher ones; the
 * default cap is 2.
 * Returns the previous cap.  Not meant to be changed while another thread is inside
 * aqlm_cpu_matmul. */
int aqlm_cpu_set_max_simd_level(int level);

/* ABI version of this header. */
int aqlm_cpu_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AQLM_CPU_H_ */
