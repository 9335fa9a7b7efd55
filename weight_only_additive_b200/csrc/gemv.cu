// Codeword-gather GEMV for token generation (batch 1..8), any supported scheme.
//
// y[b, n] = s_n * sum_j sum_t x[b, j*g + t] * (sum_m C_m[codes[n,j,m]][t]) + bias_n
//
// The decoded weights never leave registers: each group's M codewords are
// gathered (16 or 32 bytes each; the 1 MiB 1x16 codebook lives in L2, the
// 8 KiB 2x8 codebooks in L1), summed in fp32 and dotted with the fp16
// activations (inference-research record "Kernels": lookup instead of
// per-element dequantisation of W in memory).  One warp per output row; each
// lane streams 16-byte code vectors (8 groups) with no L1 allocation; fp32
// accumulation; warp-shuffle reduction; the channel scale and bias are fused
// into the store.
#include <type_traits>

#include "aqlm_device.cuh"

namespace aqlm {
namespace {

template <int M, int B, int G, int BATCH>
__device__ __forceinline__ void accumulate_group(const __half* __restrict__ x, int K, int j,
                                                 const uint32_t (&code)[M],
                                                 const __half* __restrict__ codebooks, uint64_t cb_pol,
                                                 float (&acc)[BATCH]) {
  constexpr int kVec = G / 8;
  float w[G];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const __half* cw = codebooks + (static_cast<size_t>(m) * (1u << B) + code[m]) * G;
#pragma unroll
    for (int v = 0; v < kVec; ++v) {
      const uint4 q = ldg_nc_v4_hint(cw + 8 * v, cb_pol);
      const uint32_t h[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = h2_to_f2(h[i]);
        const int t = 8 * v + 2 * i;
        w[t] = (m == 0) ? f.x : w[t] + f.x;
        w[t + 1] = (m == 0) ? f.y : w[t + 1] + f.y;
      }
    }
  }
#pragma unroll
  for (int b = 0; b < BATCH; ++b) {
    const __half* xr = x + static_cast<size_t>(b) * K + static_cast<size_t>(j) * G;
#pragma unroll
    for (int v = 0; v < kVec; ++v) {
      const uint4 q = ldg_nc_v4(xr + 8 * v);
      const uint32_t h[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = h2_to_f2(h[i]);
        acc[b] = fmaf(f.x, w[8 * v + 2 * i], acc[b]);
        acc[b] = fmaf(f.y, w[8 * v + 2 * i + 1], acc[b]);
      }
    }
  }
}

template <int M, int B, int G, int BATCH>
__global__ void __launch_bounds__(128) gemv_gather_kernel(
    const __half* __restrict__ x, const void* __restrict__ codes,
    const __half* __restrict__ codebooks, const __half* __restrict__ scales,
    const __half* __restrict__ bias, __half* __restrict__ y, int K, int N) {
  using code_t = typename std::conditional<(B <= 8), uint8_t, uint16_t>::type;
  constexpr int kCodeBytes = sizeof(code_t);
  constexpr int kGroupsPerVec = 16 / (M * kCodeBytes);
  grid_dependents_launch();
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (n >= N) return;  // never the block's first warp: every block reaches the wait below
  const int groups = K / G;
  const size_t row_bytes = static_cast<size_t>(groups) * M * kCodeBytes;
  const uint8_t* row = static_cast<const uint8_t*>(codes) + static_cast<size_t>(n) * row_bytes;

  const uint64_t stream_pol = l2_policy_evict_first();
  // codebook lines are gathered all kernel long: keep them in L2
  const uint64_t cb_pol = l2_policy_evict_last();
  float acc[BATCH];
#pragma unroll
  for (int b = 0; b < BATCH; ++b) acc[b] = 0.f;
  // x may be the previous kernel's output (and y its input): wait for it
  grid_dependency_wait();

  // 16-byte code vectors when every row starts 16-byte aligned.
  // (when M codes of a group do not tile 16 bytes, e.g. M = 3, every group takes the
  // scalar path below)
  constexpr bool kVecOk = (16 % (M * kCodeBytes)) == 0;
  const int nvec = (kVecOk && row_bytes % 16 == 0) ? groups / kGroupsPerVec : 0;
  for (int v = lane; v < nvec; v += 32) {
    const uint4 q = ldg_stream_v4(row + static_cast<size_t>(v) * 16, stream_pol);
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int gi = 0; gi < kGroupsPerVec; ++gi) {
      uint32_t code[M];
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const int byte = (gi * M + m) * kCodeBytes;  // little-endian position in the vector
        code[m] = (words[byte / 4] >> (8 * (byte % 4))) & ((1u << (8 * kCodeBytes)) - 1u);
      }
      accumulate_group<M, B, G, BATCH>(x, K, v * kGroupsPerVec + gi, code, codebooks, cb_pol, acc);
    }
  }
  // Remaining groups (ragged tail, or rows that are not 16-byte aligned).
  const code_t* rc = reinterpret_cast<const code_t*>(row);
  for (int j = nvec * kGroupsPerVec + lane; j < groups; j += 32) {
    uint32_t code[M];
#pragma unroll
    for (int m = 0; m < M; ++m) code[m] = rc[static_cast<size_t>(j) * M + m];
    accumulate_group<M, B, G, BATCH>(x, K, j, code, codebooks, cb_pol, acc);
  }

#pragma unroll
  for (int b = 0; b < BATCH; ++b) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[b] += __shfl_xor_sync(0xffffffffu, acc[b], off);
  }
  if (lane == 0) {
    const float s = __half2float(scales[n]);
    const float bi = bias ? __half2float(bias[n]) : 0.f;
#pragma unroll
    for (int b = 0; b < BATCH; ++b) y[static_cast<size_t>(b) * N + n] = __float2half_rn(acc[b] * s + bi);
  }
}

template <int M, int B, int G, int BATCH>
cudaError_t launch_fixed(const Problem& p, cudaStream_t stream) {
  const int warps_per_block = 4;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(static_cast<unsigned>((p.N + warps_per_block - 1) / warps_per_block), 1, 1);
  cfg.blockDim = dim3(32 * warps_per_block, 1, 1);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_gather_kernel<M, B, G, BATCH>, static_cast<const __half*>(p.x), p.codes,
                            static_cast<const __half*>(p.codebooks), static_cast<const __half*>(p.scales),
                            static_cast<const __half*>(p.bias), static_cast<__half*>(p.y), p.K, p.N);
}

template <int M, int B, int G>
cudaError_t launch_scheme(const Problem& p, cudaStream_t stream) {
  switch (p.batch) {
    case 1: return launch_fixed<M, B, G, 1>(p, stream);
    case 2: return launch_fixed<M, B, G, 2>(p, stream);
    case 3: return launch_fixed<M, B, G, 3>(p, stream);
    case 4: return launch_fixed<M, B, G, 4>(p, stream);
    case 5: return launch_fixed<M, B, G, 5>(p, stream);
    case 6: return launch_fixed<M, B, G, 6>(p, stream);
    case 7: return launch_fixed<M, B, G, 7>(p, stream);
    case 8: return launch_fixed<M, B, G, 8>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

namespace {
struct GemvLauncher {
  template <int M, int B, int G>
  static cudaError_t run(const Problem& p, cudaStream_t stream) {
    return launch_scheme<M, B, G>(p, stream);
  }
};
}  // namespace

cudaError_t launch_gemv(const Problem& p, cudaStream_t stream) {
  return dispatch_scheme<GemvLauncher>(p.M, p.B, p.g, cudaErrorInvalidValue, p, stream);
}

}  // namespace aqlm
