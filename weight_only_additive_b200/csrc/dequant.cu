// aqlm_dequantize: rebuild the fp16 weight matrix from codes and codebooks.
//
// W[n, j*g + t] = fp16_rne( fp32( C_0[c_0][t] + C_1[c_1][t] + ... ) * fp32(s_n) ),
// codewords added in fp32 in ascending codebook order starting from C_0
// (weights as sums of codebook vectors: AQLM repo summary "What it does";
// inference-research record, "Activation scheme").  One thread per
// (row, group): it reads M codes, gathers M codewords of g fp16 values (16 or
// 32 bytes each), and writes g fp16 values with 16-byte stores.  The kernel is
// bound by the HBM write of W (2*N*K bytes).
#include <type_traits>

#include "aqlm_device.cuh"

namespace aqlm {
namespace {

template <int M, int B, int G>
__global__ void __launch_bounds__(256) dequant_kernel(const void* __restrict__ codes,
                                                      const __half* __restrict__ codebooks,
                                                      const __half* __restrict__ scales,
                                                      __half* __restrict__ W, int groups_per_row,
                                                      long long total_groups) {
  using code_t = typename std::conditional<(B <= 8), uint8_t, uint16_t>::type;
  constexpr int kVec = G / 8;  // 16-byte vectors per codeword
  const code_t* c = static_cast<const code_t*>(codes);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
       idx < total_groups; idx += stride) {
    const long long n = idx / groups_per_row;
    float acc[G];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const uint32_t code = c[idx * M + m];
      const __half* cw = codebooks + (static_cast<size_t>(m) * (1u << B) + code) * G;
#pragma unroll
      for (int v = 0; v < kVec; ++v) {
        const uint4 q = ldg_nc_v4(cw + 8 * v);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 f = h2_to_f2(w[h]);
          const int t = 8 * v + 2 * h;
          if (m == 0) {
            acc[t] = f.x;
            acc[t + 1] = f.y;
          } else {
            acc[t] = __fadd_rn(acc[t], f.x);
            acc[t + 1] = __fadd_rn(acc[t + 1], f.y);
          }
        }
      }
    }
    const float s = __half2float(scales[n]);
    uint4* out = reinterpret_cast<uint4*>(W + idx * G);
#pragma unroll
    for (int v = 0; v < kVec; ++v) {
      uint4 q;
      q.x = f2_to_h2_rn(__fmul_rn(acc[8 * v + 0], s), __fmul_rn(acc[8 * v + 1], s));
      q.y = f2_to_h2_rn(__fmul_rn(acc[8 * v + 2], s), __fmul_rn(acc[8 * v + 3], s));
      q.z = f2_to_h2_rn(__fmul_rn(acc[8 * v + 4], s), __fmul_rn(acc[8 * v + 5], s));
      q.w = f2_to_h2_rn(__fmul_rn(acc[8 * v + 6], s), __fmul_rn(acc[8 * v + 7], s));
      out[v] = q;
    }
  }
}

template <int M, int B, int G>
cudaError_t launch(const void* codes, const void* codebooks, const void* scales, void* W,
                   int K, int N, cudaStream_t stream) {
  const int groups = K / G;
  const long long total = static_cast<long long>(groups) * N;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  const long long cap = 148LL * 32;  // grid-stride beyond 32 CTAs per SM
  if (blocks > cap) blocks = cap;
  dequant_kernel<M, B, G><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      codes, static_cast<const __half*>(codebooks), static_cast<const __half*>(scales),
      static_cast<__half*>(W), groups, total);
  return cudaGetLastError();
}

}  // namespace

namespace {
struct DequantLauncher {
  template <int M, int B, int G>
  static cudaError_t run(const void* codes, const void* codebooks, const void* scales, void* W_out, int K, int N,
                         cudaStream_t stream) {
    return launch<M, B, G>(codes, codebooks, scales, W_out, K, N, stream);
  }
};
}  // namespace

cudaError_t launch_dequantize(const void* codes, const void* codebooks, const void* scales,
                              void* W_out, int M, int B, int g, int K, int N,
                              cudaStream_t stream) {
  return dispatch_scheme<DequantLauncher>(M, B, g, cudaErrorInvalidValue, codes, codebooks, scales, W_out, K, N,
                                          stream);
}

}  // namespace aqlm
