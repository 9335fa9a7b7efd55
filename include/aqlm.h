/*
 * aqlm.h -- C ABI of libaqlm.so, the B200 (sm_100a) AQLM weight-only linear layer.
 *
 * The layer (AQLM, "Extreme Compression of Large Language Models via Additive
 * Quantization"; paper record, method paragraph; AQLM repo summary "What it
 * does"; inference-research record "AQLM (additive / multi-codebook
 * quantization)", sections "Bits", "Activation scheme", "Kernels", "notes"):
 *
 *     y = x . W^T . diag(s) + bias
 *
 * where every g-wide group of a weight row is the SUM of M fp16 codewords, one
 * picked from each of M codebooks of 2^B entries, and the activations x stay
 * fp16 (w2a16).  Weights never exist in HBM in dense form: the kernels decode
 * them on chip ("fast lookup, no per-element dequantization" for token
 * generation; "dequantize-to-FP16 then an FP16 tensor-core GEMM" for larger
 * batches).
 *
 * Data layout (all row-major, C order, caller-owned DEVICE memory):
 *   x          fp16   [batch, K]
 *   codes      uint8  [N, K/g, M] when B == 8, uint16 [N, K/g, M] when B == 16;
 *              unsigned, no offset, codebook index m varies fastest
 *   codebooks  fp16   [M, 2^B, g]
 *   scales     fp16   [N]            (one scale per output channel)
 *   bias       fp16   [N] or NULL
 *   y          fp16   [batch, N]
 *   W_out      fp16   [N, K]         (aqlm_dequantize only)
 *
 * Supported schemes (M, B, g): B = 8 (256-entry codebooks) with M = 1..4, and
 * B = 16 (65536-entry codebooks) with M = 1..2, each with g = 8 or 16 -- among them
 * the published (1, 16, 8) "1x16 g8", (2, 8, 8) "2x8 g8", (1, 16, 16) "1x16 g16" and
 * the 4-bit (2, 16, 8) and (4, 8, 8).  Other shapes return AQLM_ERR_UNSUPPORTED.
 * K must be a multiple of g; N >= 1; 1 <= batch <= 65535.  Every pointer must be
 * 16-byte aligned (AQLM_ERR_MISALIGNED otherwise); bias may be NULL.
 *
 * Ownership and state: the library never allocates or frees device memory on
 * a call and keeps no per-call state.  It holds one 32-bit device status word
 * per device (a static device variable) where kernels record a bounded wait
 * that gave up, and the static scratch of aqlm_matmul_group_static.  All compute calls are asynchronous on `stream`
 * (NULL = the legacy default stream) and may be captured in CUDA graphs.
 *
 * Stream ordering: kernels are launched with programmatic dependent launch.  A
 * call may start reading the weight buffers (codes, codebooks, scales, bias)
 * while the kernel launched just before it on the same stream is still running;
 * it reads x and writes y only after that kernel has completed.  Weight buffers
 * must therefore not be written by the kernel immediately preceding a call on
 * the same stream (they are constant during inference).
 *
 * Errors: every function returns a status and never aborts, throws or exits.
 * Argument errors are detected on the host before any launch.  A failed
 * launch returns AQLM_ERR_CUDA (the CUDA error is cleared and can be read with
 * aqlm_last_cuda_error).  Device-side failures (a wait that ran out) surface
 * through aqlm_check_device_status.
 */
#ifndef AQLM_H_
#define AQLM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; NULL means the legacy default stream. */
typedef struct CUstream_st* aqlm_stream_t;

typedef enum {
  AQLM_OK = 0,
  AQLM_ERR_INVALID_ARG = 1,   /* NULL pointer, K % g != 0, non-positive size, ... */
  AQLM_ERR_UNSUPPORTED = 2,   /* (M, B, g) or forced path not implemented        */
  AQLM_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned               */
  AQLM_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed     */
  AQLM_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up              */
} aqlm_status;

/* Work schedule of the tensor-core kernel (aqlm_matmul_ws, aqlm_input_grad_ws). */
typedef enum {
  AQLM_SCHEDULE_AUTO = 0,     /* the plan's cost model picks                              */
  AQLM_SCHEDULE_TILES = 1,    /* one CTA per (row tile, batch tile, K split): no workspace */
  AQLM_SCHEDULE_STREAMK = 2   /* stream-K over the SMs; needs the workspace, and a shape   *
                               * with a nonzero workspace size (else                       *
                               * AQLM_ERR_UNSUPPORTED)                                     */
} aqlm_schedule;

/* Kernel families aqlm_matmul can route to. */
typedef enum {
  AQLM_PATH_AUTO = 0,         /* pick by (M, B, g, batch)                               */
  AQLM_PATH_GEMV = 1,         /* codeword-gather GEMV, any supported scheme, batch <= 8 */
  AQLM_PATH_GEMV_LUT = 2,     /* x.codeword lookup-table GEMV, B = 8, batch 1; code     *
                               * rows (K/g * M bytes) a multiple of 16 and <= 8192       */
  AQLM_PATH_TENSOR_CORE = 3   /* on-chip decode -> tcgen05 fp16 MMA, any batch          */
} aqlm_path;

/*
 * y = x . W^T . diag(scales) + bias, with W decoded on chip from codes and
 * codebooks.  Defined by the AQLM pages as follows.  A weight group is the sum of
 * the codewords its codes pick: repo summary "Additive quantization that actually
 * survives one-bit weights", section "What it does"; paper record "Extreme
 * Compression of Large Language Models via Additive Quantization", method
 * paragraph.  Activations stay fp16 (w2a16): inference-research record "AQLM
 * (additive / multi-codebook quantization)", sections "Bits" and "Activation
 * scheme".  One scale per output channel, none shared over a group: the same
 * record, "notes".  Token generation looks the products up ("Kernels"); larger
 * batches decode to fp16 and run an fp16 tensor-core GEMM ("notes").
 *   x          fp16 [batch, K], read          codes      [N, K/g, M] u8/u16, read
 *   codebooks  fp16 [M, 2^B, g], read         scales     fp16 [N], read
 *   bias       fp16 [N] or NULL, read         y          fp16 [batch, N], written
 * All are caller-owned device memory (layout, alignment and ownership as in the file
 * header); y must not overlap an input (AQLM_ERR_INVALID_ARG).  Accumulation is
 * fp32 (or better); y is
 * rounded to fp16 (RNE).  Result tolerance against the fp64 reference of the
 * decoded fp16 weights: max|y - y_ref| / max|y_ref| <= 5e-3.
 * Returns AQLM_OK after enqueueing the work on `stream`; AQLM_ERR_INVALID_ARG,
 * AQLM_ERR_UNSUPPORTED or AQLM_ERR_MISALIGNED (nothing launched) for bad arguments;
 * AQLM_ERR_CUDA if the launch failed.
 */
aqlm_status aqlm_matmul(const void* x, const void* codes, const void* codebooks,
                        const void* scales, const void* bias, void* y,
                        int M, int B, int g, int K, int N, int batch,
                        aqlm_stream_t stream);

/* aqlm_matmul with the kernel family chosen by the caller (tests, benchmarks).
 * AQLM_ERR_UNSUPPORTED if that family cannot run this (scheme, batch). */
aqlm_status aqlm_matmul_path(const void* x, const void* codes, const void* codebooks,
                             const void* scales, const void* bias, void* y,
                             int M, int B, int g, int K, int N, int batch,
                             aqlm_path path, aqlm_stream_t stream);

/*
 * Bytes of workspace aqlm_matmul_ws can use for this shape, for either of:
 *  - the tensor-core kernel's stream-K schedule: every SM takes an equal share of the
 *    (weight-row tile, batch tile, 64-wide K stage) space, and a tile cut between SMs
 *    is finished by the piece that ends last, from fp32 partials in the workspace,
 *    summed in K order (so results do not depend on timing).  It needs the decoded
 *    weight stages in shared memory (a batch tile above 128 for schemes other than
 *    1x16 g8) and K a whole number of code tiles;
 *  - batch 1 with 256-entry codebooks, at least 10 MiB of codes and code rows of at
 *    least 1536 bytes: AUTO then runs the grouped lookup kernel of aqlm_matmul_group
 *    on this one layer (faster there than the single-layer lookup kernel), its fp32
 *    partial sums in the workspace.
 * The same y = x . W^T . diag(s) + bias as aqlm_matmul either way.  0 when the shape
 * uses neither, or for invalid arguments.  Pure host logic, the same for every
 * device: needs no GPU.
 */
size_t aqlm_matmul_workspace_size(int M, int B, int g, int K, int N, int batch);

/* A workspace that can carry the stream-K schedule starts with this many bytes of
 * counters (one uint32 per CTA and TMEM lane quadrant, at most 160 CTAs), the same
 * for every shape; fp32 partial slots follow. */
#define AQLM_WORKSPACE_COUNTER_BYTES 2560u

/*
 * aqlm_matmul_path with a caller workspace and a schedule for the tensor-core kernel
 * (other paths ignore both).  For this call AUTO is the tile plan: on B200 the stream-K
 * schedule measured slower for every layer shape tried (it pays a fix-up, a four-warp
 * final epilogue and a slower stage loop), so it runs only when asked for
 * (AQLM_SCHEDULE_STREAMK).  aqlm_input_grad_ws's AUTO takes it where its cost model
 * estimates it faster (a tile plan that would leave a nearly empty last wave of CTAs).
 * workspace: NULL with workspace_bytes 0
 * (then exactly aqlm_matmul_path), or caller-owned DEVICE memory, 256-byte aligned,
 * of at least aqlm_matmul_workspace_size(...) bytes (else AQLM_ERR_MISALIGNED /
 * AQLM_ERR_INVALID_ARG), overlapping none of the call's arrays (AQLM_ERR_INVALID_ARG).
 * Its first AQLM_WORKSPACE_COUNTER_BYTES are counters that must be zero when the
 * workspace is first used; every call whose kernels finish leaves them zero again,
 * so a workspace allocated zero-filled can be reused call after call, by any shape
 * (the counters sit at the same place for all).  After AQLM_ERR_TIMEOUT from
 * aqlm_check_device_status, zero them again.  Calls that may run concurrently
 * (different streams) must not share a workspace; calls on one stream may.
 * The library may also ignore the workspace (another path, or a faster plan).
 * AQLM_SCHEDULE_STREAMK without a workspace is AQLM_ERR_INVALID_ARG; an unknown
 * schedule is AQLM_ERR_INVALID_ARG.  AQLM_SCHEDULE_STREAMK on another kernel family,
 * or on a shape the stream-K schedule cannot take (including one whose workspace
 * serves only the grouped lookup route), is AQLM_ERR_UNSUPPORTED, before any launch.
 */
aqlm_status aqlm_matmul_ws(const void* x, const void* codes, const void* codebooks,
                           const void* scales, const void* bias, void* y,
                           int M, int B, int g, int K, int N, int batch, aqlm_path path,
                           aqlm_schedule schedule, void* workspace, size_t workspace_bytes,
                           aqlm_stream_t stream);

/*
 * The dense fp16 weight of the layer, the first half of the large-batch route
 * "dequantize-to-FP16 then an FP16 tensor-core GEMM" (inference-research record
 * "AQLM (additive / multi-codebook quantization)", notes), each group the sum of
 * the codewords its codes pick (repo summary "Additive quantization that actually
 * survives one-bit weights", section "What it does"):
 *
 *   W_out[n, j*g + t] = fp16_rne( fp32( C_0[c_0][t] + C_1[c_1][t] + ... ) * fp32(s_n) )
 *
 * with c_m = codes[n, j, m]; the codewords are added in fp32 in ascending m,
 * starting from C_0 itself, then one fp32 multiply by the channel scale and
 * one round-to-nearest-even to fp16.  Bit-exact by definition.
 *   codes, codebooks, scales  as for aqlm_matmul, read
 *   W_out                     fp16 [N, K], caller-owned device memory, written;
 *                             must not overlap an input (AQLM_ERR_INVALID_ARG)
 * Errors as for aqlm_matmul (no bias, no batch); returns after enqueueing.
 */
aqlm_status aqlm_dequantize(const void* codes, const void* codebooks, const void* scales,
                            void* W_out, int M, int B, int g, int K, int N,
                            aqlm_stream_t stream);

/*
 * Input gradient of the layer, for fine-tuning through a fixed quantised layer
 * (AQLM repo summary "Additive quantization that actually survives one-bit
 * weights": PV-Tuning after quantisation, section "What it does"; PEFT
 * fine-tuning, section "Key highlights").  The weights do not change, so the
 * backward pass of y = x . W^T . diag(s) + bias needs only
 *
 *   dx[b, k] = sum_n dy[b, n] * W16[n, k]        (dx = dy . diag(s) . W)
 *
 * with W16 exactly what aqlm_dequantize writes (the channel scale inside).
 *   dy   fp16 [batch, N]   row-major, read
 *   dx   fp16 [batch, K]   row-major, written; must not overlap dy or the weights
 * codes, codebooks, scales: as for aqlm_matmul.  Accumulation is fp32; dx is
 * rounded to fp16 (RNE).  Tolerance against the fp64 reference dy . W16:
 * max|dx - dx_ref| / max|dx_ref| <= 5e-3.
 * Supported: every scheme above, with N % 8 == 0 and code rows (K/g * M * B/8
 * bytes) a multiple of 16 bytes; other shapes return AQLM_ERR_UNSUPPORTED.
 * Alignment, ownership, stream ordering (dy plays x's part, dx y's) and errors
 * as for aqlm_matmul; overlapping dx and inputs is AQLM_ERR_INVALID_ARG.
 */
aqlm_status aqlm_input_grad(const void* dy, const void* codes, const void* codebooks,
                            const void* scales, void* dx, int M, int B, int g, int K, int N,
                            int batch, aqlm_stream_t stream);

/* Workspace bytes with which aqlm_input_grad_ws may use the stream-K schedule
 * (as for aqlm_matmul_workspace_size; the gradient kernel's rows are the K input
 * features).  0 when unused (B = 16 schemes) or for invalid arguments; needs no GPU. */
size_t aqlm_input_grad_workspace_size(int M, int B, int g, int K, int N, int batch);

/* aqlm_input_grad with a schedule and a caller workspace: the same result;
 * schedule and workspace as for aqlm_matmul_ws (it must not overlap dy, dx or the
 * weights). */
aqlm_status aqlm_input_grad_ws(const void* dy, const void* codes, const void* codebooks,
                               const void* scales, void* dx, int M, int B, int g, int K, int N,
                               int batch, aqlm_schedule schedule, void* workspace,
                               size_t workspace_bytes, aqlm_stream_t stream);

/* Validates aqlm_input_grad's arguments exactly as it does, without launching
 * anything.  Pure host logic: needs no GPU. */
aqlm_status aqlm_validate_input_grad(const void* dy, const void* codes, const void* codebooks,
                                     const void* scales, const void* dx, int M, int B, int g,
                                     int K, int N, int batch);

/* One layer of a group call: the arguments of aqlm_matmul, same meaning and
 * layout. */
typedef struct {
  const void* x;
  const void* codes;
  const void* codebooks;
  const void* scales;
  const void* bias;   /* may be NULL */
  void* y;
  int M, B, g, K, N, batch;
} aqlm_problem;

/*
 * Grouped launch of independent layers (a decoder block's linears, or a set of
 * experts).  The AQLM pages give no such call; it serves the token-generation case
 * where one layer is too small to fill the GPU (inference-research record "AQLM
 * (additive / multi-codebook quantization)": batch-1 decoding is dominated by
 * per-layer overheads, which CUDA graphs and fused launches remove).
 *
 * Computes y_i for every problems[i] exactly as aqlm_matmul would (same
 * definition and tolerance).  The problems must be independent: no y_i may
 * overlap another problem's x, y, codes, codebooks, scales or bias (overlapping
 * outputs and inputs are rejected with AQLM_ERR_INVALID_ARG as far as the
 * pointer ranges show).  Batch-1 problems with 256-entry codebooks (B = 8, any M
 * and g above) whose code rows (K / g * M bytes) are whole 16-byte units are
 * computed together, up to 32 per launch pair (a partial-sum kernel and a
 * reduction); the others are launched one after another as by aqlm_matmul.  Both kernels of a
 * pair keep the stream-ordering contract above.
 *
 * workspace: caller-owned DEVICE memory of at least
 * aqlm_group_workspace_size(problems, count) bytes, 256-byte aligned (NULL allowed
 * when that size is 0).  Layout: AQLM_WORKSPACE_COUNTER_BYTES left untouched (the
 * counters of aqlm_matmul_ws sit there, so one buffer may serve both kinds of call on
 * a stream), then the fp32 partial sums between the two kernels of a pair, which
 * need no initialisation.  It must not overlap any problem's buffers
 * (AQLM_ERR_INVALID_ARG).  Calls that may run concurrently (different streams) must
 * not share a workspace.
 * count == 0 is a no-op; count < 0 or problems == NULL (with count > 0) is
 * AQLM_ERR_INVALID_ARG.  Every problem is validated as aqlm_validate does before
 * anything is launched.
 */
aqlm_status aqlm_matmul_group(const aqlm_problem* problems, int count, void* workspace,
                              size_t workspace_bytes, aqlm_stream_t stream);

/*
 * aqlm_matmul_group without a caller workspace, for callers that cannot
 * allocate device memory.  The AQLM pages have no counterpart: this is a library
 * convenience.  The partial sums live in a static device buffer of
 * AQLM_STATIC_GROUP_SCRATCH_BYTES inside the library (one per device; the address
 * is taken with cudaGetSymbolAddress on a device's first call and again whenever
 * the device's CUDA context has changed, e.g. after cudaDeviceReset); the call
 * allocates nothing.  Problems whose aqlm_group_workspace_size exceeds that size
 * are rejected with AQLM_ERR_INVALID_ARG before anything is launched (16 MiB
 * covers, for example, a Llama-2-7B decoder layer set, 1.6 MB, or the 24
 * Mixtral-8x7B expert linears of one layer, 11 MB).  The buffer needs no clearing:
 * the reduction reads only partials written by the same call.
 * Calls that overlap in time (different streams or host threads on one device)
 * share the buffer and RACE: the caller must serialise them.  Calls on one
 * stream are ordered and safe.  Otherwise identical to aqlm_matmul_group.
 */
#define AQLM_STATIC_GROUP_SCRATCH_BYTES (16u << 20)
/* The library's value of AQLM_STATIC_GROUP_SCRATCH_BYTES (a caller compiled
 * against another header can read the real limit here).  Pure host logic. */
size_t aqlm_static_group_scratch_bytes(void);
aqlm_status aqlm_matmul_group_static(const aqlm_problem* problems, int count, aqlm_stream_t stream);

/*
 * aqlm_matmul_group with the activations in HOST memory: on `stream`, copies
 * x_host into the problems' device x buffers, runs the group, and copies every
 * problem's y back into y_host.
 *   x_host  fp16, the problems' x one after another in problem order
 *           (problem i: batch_i * K_i values), read
 *   y_host  fp16, the problems' y one after another (batch_i * N_i values), written
 * When the device buffers of consecutive problems are contiguous (problem i + 1's x
 * starts where problem i's ends, likewise y), one copy moves all of them; otherwise
 * there is one copy per problem (cudaMemcpyAsync; pinned host buffers make the
 * copies asynchronous).  The call returns after enqueueing: y_host is valid, and
 * x_host may be modified, once `stream` has passed the call (synchronise before).  The pages have
 * no counterpart: this is the token-generation step of a serving loop, from host
 * activations to host outputs.  Validation, workspace and errors as for
 * aqlm_matmul_group, all checked before the first copy (a rejected call changes no
 * device buffer); NULL x_host or y_host (with count > 0) is AQLM_ERR_INVALID_ARG.
 */
aqlm_status aqlm_matmul_group_host(const aqlm_problem* problems, int count, const void* x_host, void* y_host,
                                   void* workspace, size_t workspace_bytes, aqlm_stream_t stream);

/* Workspace bytes aqlm_matmul_group needs for these problems: 0 if no problem is
 * grouped; else AQLM_WORKSPACE_COUNTER_BYTES plus, for every run of up to 32 grouped
 * problems, the sum over them of ceil(K / g * M / 128) * N * 4 bytes (one fp32
 * partial per row and 128 code bytes) rounded up to 256, the maximum over runs.  The
 * problems launched one by one need none.  Pure host logic. */
size_t aqlm_group_workspace_size(const aqlm_problem* problems, int count);

/* The kernel family AQLM_PATH_AUTO picks for this problem, or -1 if unsupported.
 * Pure host logic: needs no GPU. */
int aqlm_select_path(int M, int B, int g, int K, int N, int batch);

/* Validates arguments exactly as aqlm_matmul_path does, without launching
 * anything.  Pure host logic: needs no GPU. */
aqlm_status aqlm_validate(const void* x, const void* codes, const void* codebooks,
                          const void* scales, const void* bias, const void* y,
                          int M, int B, int g, int K, int N, int batch, aqlm_path path);

/* Human-readable name of a status code (static string, never NULL). */
const char* aqlm_status_string(aqlm_status status);

/* Synchronises `stream`, then reads and clears the current device's status
 * word.  Returns AQLM_ERR_TIMEOUT if a kernel recorded a wait that gave up
 * (`detail`, if not NULL, receives the recorded site code), AQLM_ERR_CUDA if the
 * synchronisation failed, AQLM_OK otherwise. */
aqlm_status aqlm_check_device_status(aqlm_stream_t stream, uint32_t* detail);

/* Exercises the device-side failure path without faulting the GPU: launches a
 * one-thread kernel that waits, through the same bounded wait the matmul kernels
 * use, on an mbarrier nothing arrives on.  The wait gives up after timeout_us
 * microseconds (1..1000000, else AQLM_ERR_INVALID_ARG) and records site code
 * AQLM_SITE_SELFTEST in the status word; the kernel returns normally.  A following
 * aqlm_check_device_status reports AQLM_ERR_TIMEOUT with that detail.  For tests;
 * the pages have no counterpart. */
#define AQLM_SITE_SELFTEST 0x501u
aqlm_status aqlm_selftest_bounded_wait(unsigned timeout_us, aqlm_stream_t stream);

/* The cudaError_t value of the last CUDA failure this thread saw in the library
 * (0 if none). */
int aqlm_last_cuda_error(void);

/* ABI version of this header (incremented on any signature change). */
int aqlm_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AQLM_H_ */
