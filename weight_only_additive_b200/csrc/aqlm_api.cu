// C ABI of libaqlm.so: argument validation, kernel-family dispatch and the
// device status word.  Declarations and the contract live in include/aqlm.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <utility>

#include "aqlm.h"
#include "aqlm_internal.h"

namespace {

// One status word per device (the array lives in every device's copy of this
// module).  Kernels record the site of a bounded wait that gave up here.
__device__ uint32_t g_device_status;

// Scratch of aqlm_matmul_group_static: fp32 partial sums between its two
// kernels, one buffer per device (every device's copy of this module has one).
__device__ __align__(256) uint8_t g_group_scratch[AQLM_STATIC_GROUP_SCRATCH_BYTES];

thread_local int t_last_cuda_error = 0;

constexpr int kMaxDevices = 64;

// Device address of a file-scope __device__ variable on the current device, looked up
// with cudaGetSymbolAddress once per device and context: a cudaDeviceReset ends the
// context and the next one may place the module's variables elsewhere, so an address
// is reused only while the context that it came from is still current.
struct SymbolCache {
  std::mutex mu;
  uint64_t ctx[kMaxDevices] = {};
  void* ptr[kMaxDevices] = {};
};

void* symbol_address(const void* symbol, SymbolCache& cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(cache.mu);
  const uint64_t ctx = aqlm::current_context_id();
  if (cache.ptr[dev] && ctx != 0 && cache.ctx[dev] == ctx) return cache.ptr[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  cache.ptr[dev] = p;
  // read after the lookup, which creates the device's context when there is none yet
  cache.ctx[dev] = aqlm::current_context_id();
  return p;
}

SymbolCache g_status_cache;
SymbolCache g_scratch_cache;

// Device address of g_device_status for the current device (nullptr on failure).
uint32_t* device_status_ptr() {
  return static_cast<uint32_t*>(symbol_address(reinterpret_cast<const void*>(&g_device_status), g_status_cache));
}

// Device address of g_group_scratch for the current device (nullptr on failure).
void* static_scratch_ptr() {
  return symbol_address(reinterpret_cast<const void*>(&g_group_scratch), g_scratch_cache);
}

aqlm_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return AQLM_OK;
  t_last_cuda_error = static_cast<int>(e);
  cudaGetLastError();  // clear the sticky-free error so later calls start clean
  return AQLM_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool path_accepts(aqlm_path path, int M, int B, int g, int K, int batch) {
  switch (path) {
    case AQLM_PATH_GEMV: return batch <= 8;
    case AQLM_PATH_GEMV_LUT: return aqlm::gemv_lut_supported(M, B, g, K, batch);
    case AQLM_PATH_TENSOR_CORE: return true;
    default: return false;
  }
}

aqlm_status launch_matmul(const aqlm::Problem& p, aqlm_path path, cudaStream_t s);

// Batch-1 layers that the grouped lookup kernel, as a one-problem group, runs faster
// than the single-layer lookup kernel: measured on B200 for every B = 8 scheme at the
// published shapes, the single-layer kernel's clusters fall behind once a layer has
// at least 10 MiB of codes in code rows of at least 1536 bytes (3x8 g8 11008 x 4096:
// 13.3 -> 11.1 us; 4x8 g8 4096 x 14336: 26.6 -> 15.6 us; 2x8 g8 4096 x 11008: 10.2 ->
// 9.4 us), and is as fast or faster below (4x8 g8 4096 x 4096: 7.7 against 8.7 us;
// 2x8 g8 11008 x 4096 with 1024-byte rows: 7.6 us).
bool group_route_pays(const aqlm::Problem& p) {
  if (p.batch != 1 || !aqlm::lut_group_supported(p)) return false;
  const long long row_bytes = static_cast<long long>(p.K / p.g) * p.M * (p.B <= 8 ? 1 : 2);
  return row_bytes >= 1536 && row_bytes * p.N >= (10ll << 20);
}

// A schedule request against the shape's workspace need (`need` 0: no stream-K).
aqlm_status check_schedule(aqlm_schedule schedule, const void* workspace, size_t need) {
  if (schedule < AQLM_SCHEDULE_AUTO || schedule > AQLM_SCHEDULE_STREAMK) return AQLM_ERR_INVALID_ARG;
  if (schedule != AQLM_SCHEDULE_STREAMK) return AQLM_OK;
  if (need == 0) return AQLM_ERR_UNSUPPORTED;
  return workspace ? AQLM_OK : AQLM_ERR_INVALID_ARG;
}

aqlm_status validate_shape(int M, int B, int g, int K, int N, int batch) {
  if (M < 1 || B < 1 || g < 1 || K < 1 || N < 1 || batch < 1) return AQLM_ERR_INVALID_ARG;
  if (K % g != 0) return AQLM_ERR_INVALID_ARG;
  if (batch > 65535) return AQLM_ERR_INVALID_ARG;
  if (!aqlm::scheme_supported(M, B, g)) return AQLM_ERR_UNSUPPORTED;
  return AQLM_OK;
}

// Checks a caller workspace of aqlm_matmul_ws / aqlm_input_grad_ws: NULL with 0 bytes
// means none; otherwise 256-byte aligned, at least `need` bytes, and no overlap with
// the call's arrays (ptrs[i], sizes[i]; NULL entries skipped).
aqlm_status check_workspace(const void* ws, size_t ws_bytes, size_t need, const void* const* ptrs,
                            const size_t* sizes, int count) {
  if (ws == nullptr) return ws_bytes == 0 ? AQLM_OK : AQLM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return AQLM_ERR_MISALIGNED;
  if (ws_bytes < need || ws_bytes == 0) return AQLM_ERR_INVALID_ARG;
  const uintptr_t lo = reinterpret_cast<uintptr_t>(ws), hi = lo + ws_bytes;
  for (int i = 0; i < count; ++i) {
    if (!ptrs[i]) continue;
    const uintptr_t a = reinterpret_cast<uintptr_t>(ptrs[i]);
    if (a < hi && lo < a + sizes[i]) return AQLM_ERR_INVALID_ARG;
  }
  return AQLM_OK;
}

}  // namespace

namespace aqlm {
uint64_t current_context_id() {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(f);
    cudaGetLastError();
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return static_cast<uint64_t>(id) + 1u;  // 0 stays "unknown"
}

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
    cudaGetLastError();
  });
  return fn;
}
}  // namespace aqlm

extern "C" {

int aqlm_abi_version(void) { return 8; }

const char* aqlm_status_string(aqlm_status status) {
  switch (status) {
    case AQLM_OK: return "AQLM_OK";
    case AQLM_ERR_INVALID_ARG: return "AQLM_ERR_INVALID_ARG: invalid argument";
    case AQLM_ERR_UNSUPPORTED: return "AQLM_ERR_UNSUPPORTED: scheme or path not supported";
    case AQLM_ERR_MISALIGNED: return "AQLM_ERR_MISALIGNED: pointer not 16-byte aligned";
    case AQLM_ERR_CUDA: return "AQLM_ERR_CUDA: CUDA call or kernel launch failed";
    case AQLM_ERR_TIMEOUT: return "AQLM_ERR_TIMEOUT: device-side bounded wait gave up";
  }
  return "AQLM: unknown status";
}

int aqlm_last_cuda_error(void) { return t_last_cuda_error; }

int aqlm_select_path(int M, int B, int g, int K, int N, int batch) {
  if (validate_shape(M, B, g, K, N, batch) != AQLM_OK) return -1;
  if (aqlm::gemv_lut_supported(M, B, g, K, batch)) return AQLM_PATH_GEMV_LUT;
  // The pipelined tensor-core kernel decodes a weight tile once for the whole batch
  // and gathers codewords faster than the GEMV, so it wins from batch 1 on whenever
  // its shape test holds; the GEMV covers the remaining small-batch shapes.
  if (aqlm::tc_pipelined_shape(M, B, g, K)) return AQLM_PATH_TENSOR_CORE;
  if (batch <= 8) return AQLM_PATH_GEMV;
  return AQLM_PATH_TENSOR_CORE;
}

aqlm_status aqlm_validate(const void* x, const void* codes, const void* codebooks,
                          const void* scales, const void* bias, const void* y,
                          int M, int B, int g, int K, int N, int batch, aqlm_path path) {
  if (!x || !codes || !codebooks || !scales || !y) return AQLM_ERR_INVALID_ARG;
  const aqlm_status st = validate_shape(M, B, g, K, N, batch);
  if (st != AQLM_OK) return st;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(codebooks) || !aligned16(scales) ||
      !aligned16(y) || (bias && !aligned16(bias)))
    return AQLM_ERR_MISALIGNED;
  if (path != AQLM_PATH_AUTO && !path_accepts(path, M, B, g, K, batch)) {
    if (path < AQLM_PATH_AUTO || path > AQLM_PATH_TENSOR_CORE) return AQLM_ERR_INVALID_ARG;
    return AQLM_ERR_UNSUPPORTED;
  }
  // y is written while x, the weights and the bias are read
  const auto at = [](const void* p, size_t n) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return std::make_pair(a, a + n);
  };
  const auto yr = at(y, static_cast<size_t>(batch) * N * 2);
  const size_t code_bytes = static_cast<size_t>(N) * (K / g) * M * (B <= 8 ? 1 : 2);
  const std::pair<uintptr_t, uintptr_t> inputs[5] = {
      at(x, static_cast<size_t>(batch) * K * 2), at(codes, code_bytes),
      at(codebooks, static_cast<size_t>(M) * (size_t(1) << B) * g * 2), at(scales, static_cast<size_t>(N) * 2),
      at(bias, bias ? static_cast<size_t>(N) * 2 : 0)};
  for (const auto& r : inputs)
    if (r.first != r.second && yr.first < r.second && r.first < yr.second) return AQLM_ERR_INVALID_ARG;
  return AQLM_OK;
}

size_t aqlm_matmul_workspace_size(int M, int B, int g, int K, int N, int batch) {
  if (validate_shape(M, B, g, K, N, batch) != AQLM_OK) return 0;
  size_t part = aqlm::tc_pipe_partial_bytes(M, B, g, K, N, batch);
  const aqlm::Problem p{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, M, B, g, K, N, batch};
  if (group_route_pays(p)) part = std::max(part, aqlm::lut_group_workspace_bytes(&p, 1));
  return part > 0 ? AQLM_WORKSPACE_COUNTER_BYTES + part : 0;
}

aqlm_status aqlm_matmul_ws(const void* x, const void* codes, const void* codebooks,
                           const void* scales, const void* bias, void* y,
                           int M, int B, int g, int K, int N, int batch, aqlm_path path,
                           aqlm_schedule schedule, void* workspace, size_t workspace_bytes,
                           aqlm_stream_t stream) {
  aqlm_status st = aqlm_validate(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch, path);
  if (st != AQLM_OK) return st;
  // stream-K is possible only where the tensor-core kernel has partial slots for it
  // (the workspace may be sized for the grouped route alone)
  st = check_schedule(schedule, workspace, aqlm::tc_pipe_partial_bytes(M, B, g, K, N, batch));
  if (st != AQLM_OK) return st;
  if (schedule == AQLM_SCHEDULE_STREAMK) {
    // a forced stream-K schedule is the tensor-core kernel's
    if (path != AQLM_PATH_AUTO && path != AQLM_PATH_TENSOR_CORE) return AQLM_ERR_UNSUPPORTED;
    path = AQLM_PATH_TENSOR_CORE;
  }
  const size_t code_bytes = static_cast<size_t>(N) * (K / g) * M * (B <= 8 ? 1 : 2);
  const void* ptrs[6] = {x, codes, codebooks, scales, bias, y};
  const size_t sizes[6] = {static_cast<size_t>(batch) * K * 2, code_bytes,
                           static_cast<size_t>(M) * (size_t(1) << B) * g * 2, static_cast<size_t>(N) * 2,
                           static_cast<size_t>(N) * 2, static_cast<size_t>(batch) * N * 2};
  st = check_workspace(workspace, workspace_bytes, aqlm_matmul_workspace_size(M, B, g, K, N, batch), ptrs, sizes, 6);
  if (st != AQLM_OK) return st;
  aqlm::Problem p{x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch};
  if (workspace) {  // [counters][partial slots]
    p.sk_count = static_cast<uint32_t*>(workspace);
    p.sk_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + AQLM_WORKSPACE_COUNTER_BYTES);
    p.sk_part_bytes = workspace_bytes - AQLM_WORKSPACE_COUNTER_BYTES;
  }
  p.schedule = static_cast<int>(schedule);
  if (path == AQLM_PATH_AUTO && workspace && group_route_pays(p)) {
    // a batch-1 layer the grouped lookup kernel runs faster than the single-layer one:
    // a one-problem group, its partial sums after the workspace's counters
    uint32_t* status = device_status_ptr();
    if (!status) return from_cuda(cudaErrorInvalidDevice);
    return from_cuda(aqlm::launch_lut_group(&p, 1, static_cast<uint8_t*>(workspace) + AQLM_WORKSPACE_COUNTER_BYTES,
                                            status, reinterpret_cast<cudaStream_t>(stream)));
  }
  return launch_matmul(p, path, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// Launches one validated problem on `path` (AUTO resolved here).
aqlm_status launch_matmul(const aqlm::Problem& p, aqlm_path path, cudaStream_t s) {
  if (path == AQLM_PATH_AUTO) path = static_cast<aqlm_path>(aqlm_select_path(p.M, p.B, p.g, p.K, p.N, p.batch));
  switch (path) {
    case AQLM_PATH_GEMV: return from_cuda(aqlm::launch_gemv(p, s));
    case AQLM_PATH_GEMV_LUT: {
      uint32_t* status = device_status_ptr();
      if (!status) return from_cuda(cudaErrorInvalidDevice);
      return from_cuda(aqlm::launch_gemv_lut(p, status, s));
    }
    case AQLM_PATH_TENSOR_CORE: {
      uint32_t* status = device_status_ptr();
      if (!status) return from_cuda(cudaErrorInvalidDevice);
      return from_cuda(aqlm::launch_tc(p, status, s));
    }
    default: return AQLM_ERR_UNSUPPORTED;
  }
}

}  // namespace

extern "C" {

aqlm_status aqlm_matmul_path(const void* x, const void* codes, const void* codebooks,
                             const void* scales, const void* bias, void* y,
                             int M, int B, int g, int K, int N, int batch,
                             aqlm_path path, aqlm_stream_t stream) {
  return aqlm_matmul_ws(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch, path, AQLM_SCHEDULE_AUTO, nullptr,
                        0, stream);
}

aqlm_status aqlm_matmul(const void* x, const void* codes, const void* codebooks,
                        const void* scales, const void* bias, void* y,
                        int M, int B, int g, int K, int N, int batch, aqlm_stream_t stream) {
  return aqlm_matmul_path(x, codes, codebooks, scales, bias, y, M, B, g, K, N, batch,
                          AQLM_PATH_AUTO, stream);
}

aqlm_status aqlm_validate_input_grad(const void* dy, const void* codes, const void* codebooks,
                                     const void* scales, const void* dx, int M, int B, int g,
                                     int K, int N, int batch) {
  if (!dy || !codes || !codebooks || !scales || !dx) return AQLM_ERR_INVALID_ARG;
  const aqlm_status st = validate_shape(M, B, g, K, N, batch);
  if (st != AQLM_OK) return st;
  if (!aligned16(dy) || !aligned16(codes) || !aligned16(codebooks) || !aligned16(scales) || !aligned16(dx))
    return AQLM_ERR_MISALIGNED;
  if (!aqlm::grad_shape_supported(M, B, g, K, N)) return AQLM_ERR_UNSUPPORTED;
  // dx is written while dy and the weights are read
  const auto at = [](const void* p, size_t n) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return std::make_pair(a, a + n);
  };
  const auto dxr = at(dx, static_cast<size_t>(batch) * K * 2);
  const size_t code_bytes = static_cast<size_t>(N) * (K / g) * M * (B <= 8 ? 1 : 2);
  const std::pair<uintptr_t, uintptr_t> inputs[4] = {
      at(dy, static_cast<size_t>(batch) * N * 2), at(codes, code_bytes),
      at(codebooks, static_cast<size_t>(M) * (size_t(1) << B) * g * 2), at(scales, static_cast<size_t>(N) * 2)};
  for (const auto& r : inputs)
    if (dxr.first < r.second && r.first < dxr.second) return AQLM_ERR_INVALID_ARG;
  return AQLM_OK;
}

size_t aqlm_input_grad_workspace_size(int M, int B, int g, int K, int N, int batch) {
  if (validate_shape(M, B, g, K, N, batch) != AQLM_OK) return 0;
  const size_t part = aqlm::input_grad_partial_bytes(M, B, g, K, N, batch);
  return part > 0 ? AQLM_WORKSPACE_COUNTER_BYTES + part : 0;
}

aqlm_status aqlm_input_grad_ws(const void* dy, const void* codes, const void* codebooks,
                               const void* scales, void* dx, int M, int B, int g, int K, int N,
                               int batch, aqlm_schedule schedule, void* workspace, size_t workspace_bytes,
                               aqlm_stream_t stream) {
  aqlm_status st = aqlm_validate_input_grad(dy, codes, codebooks, scales, dx, M, B, g, K, N, batch);
  if (st != AQLM_OK) return st;
  st = check_schedule(schedule, workspace, aqlm_input_grad_workspace_size(M, B, g, K, N, batch));
  if (st != AQLM_OK) return st;
  const size_t code_bytes = static_cast<size_t>(N) * (K / g) * M * (B <= 8 ? 1 : 2);
  const void* ptrs[5] = {dy, codes, codebooks, scales, dx};
  const size_t sizes[5] = {static_cast<size_t>(batch) * N * 2, code_bytes,
                           static_cast<size_t>(M) * (size_t(1) << B) * g * 2, static_cast<size_t>(N) * 2,
                           static_cast<size_t>(batch) * K * 2};
  st = check_workspace(workspace, workspace_bytes, aqlm_input_grad_workspace_size(M, B, g, K, N, batch), ptrs,
                       sizes, 5);
  if (st != AQLM_OK) return st;
  uint32_t* status = device_status_ptr();
  if (!status) return from_cuda(cudaErrorInvalidDevice);
  aqlm::GradProblem p{dy, codes, codebooks, scales, dx, M, B, g, K, N, batch};
  if (workspace) {  // [counters][partial slots]
    p.sk_count = static_cast<uint32_t*>(workspace);
    p.sk_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + AQLM_WORKSPACE_COUNTER_BYTES);
    p.sk_part_bytes = workspace_bytes - AQLM_WORKSPACE_COUNTER_BYTES;
  }
  p.schedule = static_cast<int>(schedule);
  return from_cuda(aqlm::launch_input_grad(p, status, reinterpret_cast<cudaStream_t>(stream)));
}

aqlm_status aqlm_input_grad(const void* dy, const void* codes, const void* codebooks,
                            const void* scales, void* dx, int M, int B, int g, int K, int N,
                            int batch, aqlm_stream_t stream) {
  return aqlm_input_grad_ws(dy, codes, codebooks, scales, dx, M, B, g, K, N, batch, AQLM_SCHEDULE_AUTO, nullptr, 0,
                            stream);
}

namespace {

struct ByteRange {
  uintptr_t lo, hi;  // [lo, hi)
};

ByteRange range_of(const void* p, size_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return ByteRange{a, a + bytes};
}

bool overlaps(ByteRange a, ByteRange b) { return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi; }

// Every buffer of a (validated) problem, y last.
int problem_ranges(const aqlm_problem& q, ByteRange (&r)[6]) {
  const size_t code_bytes = static_cast<size_t>(q.N) * (q.K / q.g) * q.M * (q.B <= 8 ? 1 : 2);
  r[0] = range_of(q.x, static_cast<size_t>(q.batch) * q.K * 2);
  r[1] = range_of(q.codes, code_bytes);
  r[2] = range_of(q.codebooks, static_cast<size_t>(q.M) * (size_t{1} << q.B) * q.g * 2);
  r[3] = range_of(q.scales, static_cast<size_t>(q.N) * 2);
  r[4] = range_of(q.bias, q.bias ? static_cast<size_t>(q.N) * 2 : 0);
  r[5] = range_of(q.y, static_cast<size_t>(q.batch) * q.N * 2);
  return 6;
}

aqlm::Problem to_problem(const aqlm_problem& q) {
  return aqlm::Problem{q.x, q.codes, q.codebooks, q.scales, q.bias, q.y, q.M, q.B, q.g, q.K, q.N, q.batch};
}

// Workspace of the grouped runs: the largest run of up to kMaxGroupLayers
// grouped problems (in call order).
size_t group_workspace(const aqlm_problem* problems, int count) {
  size_t best = 0, cur = 0;
  int in_run = 0;
  for (int i = 0; i < count; ++i) {
    const aqlm::Problem p = to_problem(problems[i]);
    if (!aqlm::lut_group_supported(p)) continue;
    if (in_run == aqlm::kMaxGroupLayers) {
      cur = 0;
      in_run = 0;
    }
    cur += aqlm::lut_group_workspace_bytes(&p, 1);
    ++in_run;
    if (cur > best) best = cur;
  }
  return best;
}

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

// Bytes a group workspace needs: the counters of the stream-K layout (kept first in
// every workspace of this library, so a buffer shared with aqlm_matmul_ws calls never
// has partials written over them), then the grouped partial sums; 0 when nothing is
// grouped.  The problems launched one by one run the tile plans, which need none.
size_t group_need(const aqlm_problem* problems, int count) {
  const size_t grouped = group_workspace(problems, count);
  return grouped > 0 ? AQLM_WORKSPACE_COUNTER_BYTES + round256(grouped) : 0;
}

// The argument checks of a group call, made before any copy or launch: every problem
// valid, no output overlapping another problem's buffers, and (when anything is
// grouped) a workspace of the needed size and alignment that overlaps none of them.
aqlm_status validate_group(const aqlm_problem* problems, int count, const void* workspace,
                           size_t workspace_bytes, size_t* need_out) {
  for (int i = 0; i < count; ++i) {
    const aqlm_problem& q = problems[i];
    const aqlm_status st = aqlm_validate(q.x, q.codes, q.codebooks, q.scales, q.bias, q.y, q.M, q.B, q.g, q.K,
                                         q.N, q.batch, AQLM_PATH_AUTO);
    if (st != AQLM_OK) return st;
  }
  // independence: no output may overlap another problem's buffers
  for (int i = 0; i < count; ++i) {
    ByteRange ri[6];
    problem_ranges(problems[i], ri);
    for (int j = 0; j < count; ++j) {
      if (j == i) continue;
      ByteRange rj[6];
      problem_ranges(problems[j], rj);
      for (int k = 0; k < 6; ++k)
        if (overlaps(ri[5], rj[k])) return AQLM_ERR_INVALID_ARG;
    }
  }
  const size_t need = group_need(problems, count);
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return AQLM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return AQLM_ERR_MISALIGNED;
    const ByteRange wr = range_of(workspace, need);
    for (int i = 0; i < count; ++i) {
      ByteRange ri[6];
      problem_ranges(problems[i], ri);
      for (int k = 0; k < 6; ++k)
        if (overlaps(wr, ri[k])) return AQLM_ERR_INVALID_ARG;
    }
  }
  *need_out = need;
  return AQLM_OK;
}

// Launches a validated group (`need` from validate_group): runs of up to
// kMaxGroupLayers grouped problems in the grouped kernel, the others one by one.
aqlm_status run_group(const aqlm_problem* problems, int count, void* workspace, size_t need, cudaStream_t s) {
  uint8_t* const ws = static_cast<uint8_t*>(workspace);
  aqlm::Problem run[aqlm::kMaxGroupLayers];
  int n_run = 0;
  uint32_t* status = nullptr;
  if (need > 0) {
    status = device_status_ptr();
    if (!status) return from_cuda(cudaErrorInvalidDevice);
  }
  for (int i = 0; i <= count; ++i) {
    const bool flush = (i == count) || n_run == aqlm::kMaxGroupLayers;
    if (flush && n_run > 0) {
      const aqlm_status st =
          from_cuda(aqlm::launch_lut_group(run, n_run, ws + AQLM_WORKSPACE_COUNTER_BYTES, status, s));
      if (st != AQLM_OK) return st;
      n_run = 0;
    }
    if (i == count) break;
    const aqlm::Problem p = to_problem(problems[i]);
    if (aqlm::lut_group_supported(p)) {
      run[n_run++] = p;
    } else {
      const aqlm_status st = launch_matmul(p, AQLM_PATH_AUTO, s);
      if (st != AQLM_OK) return st;
    }
  }
  return AQLM_OK;
}

}  // namespace

size_t aqlm_group_workspace_size(const aqlm_problem* problems, int count) {
  if (!problems || count <= 0) return 0;
  for (int i = 0; i < count; ++i) {
    const aqlm_problem& q = problems[i];
    if (validate_shape(q.M, q.B, q.g, q.K, q.N, q.batch) != AQLM_OK) return 0;
  }
  return group_need(problems, count);
}

aqlm_status aqlm_matmul_group(const aqlm_problem* problems, int count, void* workspace,
                              size_t workspace_bytes, aqlm_stream_t stream) {
  if (count == 0) return AQLM_OK;
  if (count < 0 || !problems) return AQLM_ERR_INVALID_ARG;
  size_t need = 0;
  const aqlm_status vst = validate_group(problems, count, workspace, workspace_bytes, &need);
  if (vst != AQLM_OK) return vst;
  return run_group(problems, count, workspace, need, reinterpret_cast<cudaStream_t>(stream));
}

aqlm_status aqlm_matmul_group_host(const aqlm_problem* problems, int count, const void* x_host, void* y_host,
                                   void* workspace, size_t workspace_bytes, aqlm_stream_t stream) {
  if (count == 0) return AQLM_OK;
  if (count < 0 || !problems || !x_host || !y_host) return AQLM_ERR_INVALID_ARG;
  // every argument check of the group call before the first copy
  size_t need = 0;
  const aqlm_status vst = validate_group(problems, count, workspace, workspace_bytes, &need);
  if (vst != AQLM_OK) return vst;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const auto xbytes = [&](int i) { return static_cast<size_t>(problems[i].batch) * problems[i].K * 2; };
  const auto ybytes = [&](int i) { return static_cast<size_t>(problems[i].batch) * problems[i].N * 2; };
  // one copy per maximal run of problems whose device buffers are contiguous
  const auto copy_runs = [&](bool in) -> aqlm_status {
    size_t off = 0;
    for (int i = 0; i < count;) {
      const auto bytes = [&](int k) { return in ? xbytes(k) : ybytes(k); };
      const auto dptr = [&](int k) {
        return in ? static_cast<uint8_t*>(const_cast<void*>(problems[k].x)) : static_cast<uint8_t*>(problems[k].y);
      };
      int j = i;
      size_t run = bytes(i);
      while (j + 1 < count && dptr(j + 1) == dptr(i) + run) {
        ++j;
        run += bytes(j);
      }
      const aqlm_status st = from_cuda(
          in ? cudaMemcpyAsync(dptr(i), static_cast<const uint8_t*>(x_host) + off, run, cudaMemcpyHostToDevice, s)
             : cudaMemcpyAsync(static_cast<uint8_t*>(y_host) + off, dptr(i), run, cudaMemcpyDeviceToHost, s));
      if (st != AQLM_OK) return st;
      off += run;
      i = j + 1;
    }
    return AQLM_OK;
  };
  aqlm_status st = copy_runs(true);
  if (st != AQLM_OK) return st;
  st = run_group(problems, count, workspace, need, s);
  if (st != AQLM_OK) return st;
  return copy_runs(false);
}

size_t aqlm_static_group_scratch_bytes(void) { return AQLM_STATIC_GROUP_SCRATCH_BYTES; }

aqlm_status aqlm_matmul_group_static(const aqlm_problem* problems, int count, aqlm_stream_t stream) {
  if (count == 0) return AQLM_OK;
  if (count < 0 || !problems) return AQLM_ERR_INVALID_ARG;
  const size_t need = aqlm_group_workspace_size(problems, count);
  if (need > AQLM_STATIC_GROUP_SCRATCH_BYTES) return AQLM_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (need > 0) {
    // validate before touching the device, as every entry point does
    for (int i = 0; i < count; ++i) {
      const aqlm_problem& q = problems[i];
      const aqlm_status st = aqlm_validate(q.x, q.codes, q.codebooks, q.scales, q.bias, q.y, q.M, q.B, q.g, q.K,
                                           q.N, q.batch, AQLM_PATH_AUTO);
      if (st != AQLM_OK) return st;
    }
    scratch = static_scratch_ptr();
    if (!scratch) return from_cuda(cudaErrorInvalidDevice);
  }
  return aqlm_matmul_group(problems, count, scratch, scratch ? AQLM_STATIC_GROUP_SCRATCH_BYTES : 0, stream);
}

aqlm_status aqlm_selftest_bounded_wait(unsigned timeout_us, aqlm_stream_t stream) {
  if (timeout_us == 0 || timeout_us > 1000000u) return AQLM_ERR_INVALID_ARG;
  uint32_t* status = device_status_ptr();
  if (!status) return from_cuda(cudaErrorInvalidDevice);
  return from_cuda(aqlm::launch_selftest_wait(status, static_cast<uint64_t>(timeout_us) * 1000u,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

aqlm_status aqlm_dequantize(const void* codes, const void* codebooks, const void* scales,
                            void* W_out, int M, int B, int g, int K, int N,
                            aqlm_stream_t stream) {
  if (!codes || !codebooks || !scales || !W_out) return AQLM_ERR_INVALID_ARG;
  const aqlm_status st = validate_shape(M, B, g, K, N, 1);
  if (st != AQLM_OK) return st;
  if (!aligned16(codes) || !aligned16(codebooks) || !aligned16(scales) || !aligned16(W_out))
    return AQLM_ERR_MISALIGNED;
  // W_out is written while the codes, codebooks and scales are read
  const uintptr_t w0 = reinterpret_cast<uintptr_t>(W_out), w1 = w0 + static_cast<size_t>(N) * K * 2;
  const size_t code_bytes = static_cast<size_t>(N) * (K / g) * M * (B <= 8 ? 1 : 2);
  const std::pair<const void*, size_t> inputs[3] = {
      {codes, code_bytes}, {codebooks, static_cast<size_t>(M) * (size_t(1) << B) * g * 2}, {scales, size_t(N) * 2}};
  for (const auto& in : inputs) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(in.first);
    if (w0 < a + in.second && a < w1) return AQLM_ERR_INVALID_ARG;
  }
  return from_cuda(aqlm::launch_dequantize(codes, codebooks, scales, W_out, M, B, g, K, N,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

aqlm_status aqlm_check_device_status(aqlm_stream_t stream, uint32_t* detail) {
  if (detail) *detail = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return from_cuda(e);
  uint32_t* dev_status = device_status_ptr();
  if (!dev_status) return from_cuda(cudaErrorInvalidDevice);
  uint32_t value = 0;
  e = cudaMemcpy(&value, dev_status, sizeof value, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return from_cuda(e);
  if (value != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpy(dev_status, &zero, sizeof zero, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return from_cuda(e);
    if (detail) *detail = value;
    return AQLM_ERR_TIMEOUT;
  }
  return AQLM_OK;
}

}  // extern "C"
