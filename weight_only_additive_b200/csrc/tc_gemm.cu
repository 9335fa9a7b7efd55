// Batch >= 16 path: on-chip decode of W tiles into shared memory feeding the
// 5th-generation tensor cores (tcgen05.mma kind::f16, fp32 accumulator in TMEM).
//
// "Dequantize-to-FP16 then an FP16 tensor-core GEMM" (inference-research record
// "AQLM (additive / multi-codebook quantization)", notes) -- fused: the fp16
// weights exist only as 128 x 64 tiles in shared memory, never in HBM.
//
// Swap-AB: the MMA's M dimension is 128 weight rows, its N dimension is a tile
// of BN batch rows (16..256), so D[n, b] = sum_k W[n, k] * x[b, k] lands in TMEM
// with one weight row per TMEM lane.  Per 64-wide K block:
//   * each of the 128 threads decodes its weight row's 64 values (M codeword
//     gathers per group, fp32 sum, one fp16 rounding; the scale is applied to
//     the fp32 accumulator in the epilogue) into the 128-byte-swizzled K-major
//     A tile;
//   * the threads copy the x tile (BN x 64 fp16) into the same layout;
//   * one thread issues four 128 x BN x 16 MMAs and commits them to an
//     mbarrier, which every thread waits on (bounded) before the tiles are
//     rewritten.
// Epilogue: tcgen05.ld of 16 columns at a time, y = s_n * D + bias_n -> fp16.
#include <type_traits>

#include "aqlm_device.cuh"

namespace aqlm {
namespace {

constexpr int kTileN = 128;     // weight rows per CTA (MMA M)
constexpr int kTileK = 64;      // K per stage: one 128-byte swizzle row of fp16
constexpr int kMaxBN = 256;     // batch rows per CTA (MMA N)
constexpr int kThreads = 128;

__device__ __forceinline__ uint32_t swizzle128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int M, int B, int G>
__global__ void __launch_bounds__(kThreads, 1) tc_decode_mma_kernel(
    const __half* __restrict__ x, const void* __restrict__ codes,
    const __half* __restrict__ codebooks, const __half* __restrict__ scales,
    const __half* __restrict__ bias, __half* __restrict__ y, int K, int N, int batch, int BN,
    uint32_t tmem_cols, uint32_t* status) {
  using code_t = typename std::conditional<(B <= 8), uint8_t, uint16_t>::type;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;                                   // 128 x 128 B
  uint8_t* sB = smem + kTileN * 128;                    // BN x 128 B
  uint64_t* bar = reinterpret_cast<uint64_t*>(sB + kMaxBN * 128);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n0 = blockIdx.x * kTileN;
  const int b0 = blockIdx.y * BN;
  const int groups = K / G;
  const code_t* code_base = static_cast<const code_t*>(codes);

  if (warp == 0) tmem_alloc(tmem_slot, tmem_cols);
  if (tid == 0) {
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_d = *tmem_slot;

  const uint32_t idesc = umma_idesc_f16_f32(kTileN, static_cast<uint32_t>(BN));
  const int nkb = (K + kTileK - 1) / kTileK;
  const int row = n0 + tid;  // the weight row this thread decodes
  uint32_t phase = 0;
  bool ok = true;

  for (int kb = 0; kb < nkb; ++kb) {
    // ---- A tile: decode 64 weights of this thread's row -------------------
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int k = kb * kTileK + c * 8;
      uint4 packed = make_uint4(0u, 0u, 0u, 0u);
      if (row < N && k < K) {
        const int j = k / G;
        const int t0 = k - j * G;
        float w[8];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const uint32_t code = code_base[(static_cast<size_t>(row) * groups + j) * M + m];
          const uint4 q = ldg_nc_v4(codebooks + (static_cast<size_t>(m) * (1u << B) + code) * G + t0);
          const uint32_t h[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = h2_to_f2(h[i]);
            w[2 * i] = (m == 0) ? f.x : w[2 * i] + f.x;
            w[2 * i + 1] = (m == 0) ? f.y : w[2 * i + 1] + f.y;
          }
        }
        packed.x = f2_to_h2_rn(w[0], w[1]);
        packed.y = f2_to_h2_rn(w[2], w[3]);
        packed.z = f2_to_h2_rn(w[4], w[5]);
        packed.w = f2_to_h2_rn(w[6], w[7]);
      }
      *reinterpret_cast<uint4*>(sA + swizzle128(tid, c)) = packed;
    }
    // ---- B tile: x rows b0 .. b0+BN-1 ---------------------------------------
    for (int i = tid; i < BN * 8; i += kThreads) {
      const int r = i >> 3;
      const int c = i & 7;
      const int b = b0 + r;
      const int k = kb * kTileK + c * 8;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (b < batch && k < K) v = ldg_nc_v4(x + static_cast<size_t>(b) * K + k);
      *reinterpret_cast<uint4*>(sB + swizzle128(r, c)) = v;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after_sync();
      const uint64_t adesc = umma_desc_sw128_kmajor(smem_addr(sA));
      const uint64_t bdesc = umma_desc_sw128_kmajor(smem_addr(sB));
#pragma unroll
      for (int ks = 0; ks < kTileK / 16; ++ks) {
        // +32 bytes along K per 16-wide step inside the swizzle row
        umma_f16_ss(tmem_d, adesc + 2 * ks, bdesc + 2 * ks, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
      }
      umma_commit(bar);
    }
    const bool done = mbar_wait_bounded(bar, phase, status, kSiteTcMmaDone);
    if (!__syncthreads_and(done ? 1 : 0)) {
      // Give the MMAs in flight one more bounded wait before TMEM is freed.
      mbar_wait_bounded(bar, phase, status, kSiteTcMmaDone);
      ok = false;
      break;
    }
    phase ^= 1u;
  }

  if (ok) {
    tc_fence_after_sync();
    const int n = n0 + warp * 32 + lane;
    const float s = (n < N) ? __half2float(scales[n]) : 0.f;
    const float bi = (bias != nullptr && n < N) ? __half2float(bias[n]) : 0.f;
    for (int c0 = 0; c0 < BN; c0 += 16) {
      float v[16];
      tmem_ld_32x32b_x16(tmem_d + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c0), v);
      if (n < N) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int b = b0 + c0 + i;
          if (b < batch) y[static_cast<size_t>(b) * N + n] = __float2half_rn(v[i] * s + bi);
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_d, tmem_cols);
  }
}

template <int M, int B, int G>
cudaError_t launch_scheme(const Problem& p, uint32_t* status, cudaStream_t stream) {
  int BN = ((p.batch + 15) / 16) * 16;
  if (BN > kMaxBN) BN = kMaxBN;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(BN)) cols <<= 1;
  // Shared memory: alignment slack + A + B + barrier/slot.  Also large enough
  // that the CTAs resident on one SM never ask for more than 512 TMEM columns.
  size_t smem = 1024 + kTileN * 128 + kMaxBN * 128 + 64;
  const size_t per_sm = 227 * 1024;
  const size_t max_ctas = 512 / cols;
  const size_t min_smem = per_sm / max_ctas + 1;
  if (smem < min_smem) smem = min_smem;
  auto kern = tc_decode_mma_kernel<M, B, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((p.N + kTileN - 1) / kTileN),
            static_cast<unsigned>((p.batch + BN - 1) / BN));
  kern<<<grid, kThreads, smem, stream>>>(
      static_cast<const __half*>(p.x), p.codes, static_cast<const __half*>(p.codebooks),
      static_cast<const __half*>(p.scales), static_cast<const __half*>(p.bias),
      static_cast<__half*>(p.y), p.K, p.N, p.batch, BN, cols, status);
  return cudaGetLastError();
}

}  // namespace

namespace {
struct TcLauncher {
  template <int M, int B, int G>
  static cudaError_t run(const Problem& p, uint32_t* status, cudaStream_t stream) {
    return launch_scheme<M, B, G>(p, status, stream);
  }
};
}  // namespace

cudaError_t launch_tc(const Problem& p, uint32_t* status, cudaStream_t stream) {
  // the pipelined kernel takes every shape with K % 64 == 0 and 16-byte code rows
  const cudaError_t e = launch_tc_pipelined(p, status, stream);
  if (e != cudaErrorNotSupported) return e;
  return dispatch_scheme<TcLauncher>(p.M, p.B, p.g, cudaErrorInvalidValue, p, status, stream);
}

}  // namespace aqlm
