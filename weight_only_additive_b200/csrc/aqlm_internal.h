// Internal interface between the C-ABI layer (aqlm_api.cu) and the kernels.
// Host code only calls these after aqlm_validate-style checks have passed.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace aqlm {

// Bounded device waits give up after this much wall time (1 s) and record a
// site code in the library's device status word.
constexpr uint64_t kWaitTimeoutNs = 1000000000ull;

// Site codes written to the device status word.
enum : uint32_t {
  kSiteTcMmaDone = 0x101,   // tensor-core kernel: waiting for an MMA commit
  kSiteLutMma = 0x201,      // lookup-table GEMV: waiting for the table-building MMA
  kSiteLutCodes = 0x202,    // lookup-table GEMV: code-tile pipeline (TMA landing / slot release)
  kSitePipeFull = 0x301,    // pipelined tensor-core kernel: waiting for a decoded/loaded stage
  kSitePipeEmpty = 0x302,   // pipelined tensor-core kernel: waiting for a stage to be released
  kSitePipeCodes = 0x303,   // pipelined tensor-core kernel: code-tile ring
  kSitePipeAcc = 0x304,     // pipelined tensor-core kernel: waiting for the accumulator
  kSiteGroupRing = 0x401,   // grouped lookup-table kernel: code-tile ring (landing / slot release)
  kSiteGroupMma = 0x402,    // grouped lookup-table kernel: waiting for the table-building MMA
  kSiteSelftest = 0x501,    // aqlm_selftest_bounded_wait: the wait that nothing completes
};

// Self-test of the bounded-wait path: one thread waits on an mbarrier that nothing
// arrives on, gives up after timeout_ns and records kSiteSelftest.
cudaError_t launch_selftest_wait(uint32_t* status, uint64_t timeout_ns, cudaStream_t stream);

struct Problem {
  const void* x;
  const void* codes;
  const void* codebooks;
  const void* scales;
  const void* bias;  // may be null
  void* y;
  int M, B, g, K, N, batch;
  // the tensor-core kernel's stream-K schedule: its counters (kStreamKCounterBytes,
  // zero between calls) and partial slots, or null
  uint32_t* sk_count = nullptr;
  float* sk_part = nullptr;
  size_t sk_part_bytes = 0;
  int schedule = 0;  // aqlm_schedule: 0 auto, 1 tiles, 2 stream-K (forced)
};

// Each launcher enqueues its kernel(s) on `stream` and returns the launch error.
cudaError_t launch_dequantize(const void* codes, const void* codebooks, const void* scales,
                              void* W_out, int M, int B, int g, int K, int N,
                              cudaStream_t stream);
cudaError_t launch_gemv(const Problem& p, cudaStream_t stream);
cudaError_t launch_gemv_lut(const Problem& p, uint32_t* status, cudaStream_t stream);
// True if the lookup-table GEMV handles this problem (2x8 g8, batch 1, K % 64 == 0).
bool gemv_lut_supported(int M, int B, int g, int K, int batch);
cudaError_t launch_tc(const Problem& p, uint32_t* status, cudaStream_t stream);

// cuTensorMapEncodeTiled from the driver (through the runtime's entry-point
// query, so the library does not link libcuda); nullptr if unavailable.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled();

// A process-unique id (never 0) of the calling thread's current CUDA context, or 0 when
// there is none or the driver cannot say.  Per-device host caches of things that live
// in a context (symbol addresses, kernel attributes) compare it to notice a context
// created after cudaDeviceReset.
uint64_t current_context_id();

// Pipelined decode -> tcgen05 kernel; cudaErrorNotSupported when the shape is
// outside what it handles (the caller then uses the single-stage kernel).  With a
// workspace of tc_pipe_workspace_bytes (> 0) it may run the stream-K schedule.
cudaError_t launch_tc_pipelined(const Problem& p, uint32_t* status, cudaStream_t stream);
// Stream-K counters: one uint32 per (CTA, TMEM lane quadrant), at most 160 CTAs;
// the first bytes of every workspace that can carry the schedule.
constexpr size_t kStreamKCounterBytes = 160 * 4 * sizeof(uint32_t);
// fp32 partial-slot bytes the stream-K schedule of the pipelined kernel needs on any
// device; 0 when the shape never uses it.
size_t tc_pipe_partial_bytes(int M, int B, int g, int K, int N, int batch);
// Shape test of the pipelined kernel: K % 64 == 0 and code rows a multiple of 16 bytes.
inline bool tc_pipelined_shape(int M, int B, int g, int K) {
  const long long row_bytes = static_cast<long long>(K / g) * M * (B <= 8 ? 1 : 2);
  return K % 64 == 0 && row_bytes % 16 == 0;
}

// Input gradient dx = dy . W16 (W16 the dequantised weight, scale included) on the
// pipelined tensor-core kernel run transposed: dy [batch, N], dx [batch, K].
struct GradProblem {
  const void* dy;
  const void* codes;
  const void* codebooks;
  const void* scales;
  void* dx;
  int M, B, g, K, N, batch;
  uint32_t* sk_count = nullptr;  // as in Problem
  float* sk_part = nullptr;
  size_t sk_part_bytes = 0;
  int schedule = 0;
};
cudaError_t launch_input_grad(const GradProblem& p, uint32_t* status, cudaStream_t stream);
size_t input_grad_partial_bytes(int M, int B, int g, int K, int N, int batch);
// Shape test of the gradient kernel: dy rows and code rows are TMA tensors, so
// N % 8 == 0 (16-byte dy rows) and code rows a multiple of 16 bytes.
inline bool grad_shape_supported(int M, int B, int g, int K, int N) {
  const long long row_bytes = static_cast<long long>(K / g) * M * (B <= 8 ? 1 : 2);
  return N % 8 == 0 && row_bytes % 16 == 0;
}

// Grouped lookup-table GEMV over independent 2x8 g8 batch-1 layers (one launch
// of the partial-sum kernel, one of the reduction), at most kMaxGroupLayers per
// launch.  The workspace holds every layer's fp32 partials, [ceil(G/64)][N] each,
// 256-byte aligned.
constexpr int kMaxGroupLayers = 32;
bool lut_group_supported(const Problem& p);
size_t lut_group_workspace_bytes(const Problem* probs, int count);
cudaError_t launch_lut_group(const Problem* probs, int count, void* workspace, uint32_t* status,
                             cudaStream_t stream);

// True if the scheme is one the kernels are instantiated for: B = 8 codebooks
// (256 entries) with M = 1..4, B = 16 codebooks (65536 entries) with M = 1..2, each
// with codewords of g = 8 or 16 weights.
inline bool scheme_supported(int M, int B, int g) {
  if (g != 8 && g != 16) return false;
  if (B == 8) return M >= 1 && M <= 4;
  if (B == 16) return M == 1 || M == 2;
  return false;
}

// Calls F::template run<M, B, G>(args...) for the supported scheme (M, B, g), or
// returns `fallback`.  Every launcher instantiates its kernels through this list.
template <typename F, typename R, typename... Args>
inline R dispatch_scheme(int M, int B, int g, R fallback, Args&&... args) {
#define AQLM_SCHEME(m, b, gg) \
  if (M == m && B == b && g == gg) return F::template run<m, b, gg>(args...);
  AQLM_SCHEME(1, 8, 8) AQLM_SCHEME(2, 8, 8) AQLM_SCHEME(3, 8, 8) AQLM_SCHEME(4, 8, 8)
  AQLM_SCHEME(1, 8, 16) AQLM_SCHEME(2, 8, 16) AQLM_SCHEME(3, 8, 16) AQLM_SCHEME(4, 8, 16)
  AQLM_SCHEME(1, 16, 8) AQLM_SCHEME(2, 16, 8) AQLM_SCHEME(1, 16, 16) AQLM_SCHEME(2, 16, 16)
#undef AQLM_SCHEME
  return fallback;
}

}  // namespace aqlm
