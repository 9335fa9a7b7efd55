// Lookup-table GEMV for 2x8 codebooks (two codebooks of 256 fp16 codewords of
// 8 weights), batch 1: "fast lookup, no per-element dequantization"
// (inference-research record "AQLM (additive / multi-codebook quantization)",
// section "Kernels").
//
//   T_m[j][i] = sum_t x[8j + t] * C_m[i][t]            (per group j, codebook m, entry i)
//   y[n]      = s_n * sum_j (T_0[j][codes[n,j,0]] + T_1[j][codes[n,j,1]]) + bias_n
//
// Work split.  A cluster of C CTAs owns a block of output rows; CTA c of the
// cluster owns a K slice of P passes x 64 groups.  Per pass the CTA
//   1. builds the lookup table of its 64 groups with two tcgen05.mma
//      (M = 128 rows of x groups, N = 256 codebook entries, K = 16 with the
//      upper 8 zero), accumulator in TMEM;
//   2. moves it TMEM -> registers -> shared memory as fp16 pairs
//      (T_0, T_1) per (entry, group): 256 entries x 64 groups x 4 B = 64 KB;
//   3. streams the codes of its rows (cp.async, double-buffered, 32 rows x
//      128 B per warp chunk) and sums lookups.
// The row partials of the C CTAs are exchanged with bulk shared-memory copies
// inside the cluster and summed in a fixed order (deterministic), then the
// channel scale and bias are applied.
//
// Bank-conflict-free lookups.  Lane l of a warp owns row l of a 32-row chunk.
// At step s it reads code word w = (l + s) mod 32 of its row (4 codes: groups
// 2w and 2w+1, codebooks 0 and 1).  The table stores group 2w in word column
// w and group 2w+1 in column 32 + w of each entry's 64-word row, so the 32
// lanes of a lookup touch 32 different banks whatever the codes are.  The
// table is written from TMEM lane rho = word column, which is conflict-free
// too: A row rho holds group 2*(rho mod 32) + rho/32.
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "aqlm_device.cuh"

namespace aqlm {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kGroupsPerPass = 64;
constexpr uint32_t kLutBytes = 256u * 64u * 4u;   // 64 KB
constexpr uint32_t kAOpBytes = 128u * 32u;         // 4 KB
constexpr uint32_t kBOpBytes = 256u * 32u;         // 8 KB per codebook
constexpr uint32_t kChunkBytes = 32u * 128u;       // 32 rows x 128 B of codes
constexpr uint32_t kTmemCols = 512;                // D_0 at [0,256), D_1 at [256,512)

struct LutParams {
  const __half* x;
  const uint8_t* codes;
  const __half* codebooks;
  const __half* scales;
  const __half* bias;
  __half* y;
  int K, N, G;
  int C;      // CTAs per cluster (K slices)
  int P;      // passes of 64 groups per CTA
  int RB;     // output rows per cluster
  int RBc;    // rows each CTA reduces (multiple of 4)
  int nchunk; // ceil(RB / 32)
  uint32_t* status;
};

struct SmemLayout {
  uint32_t lut, aop, bop, codebuf, part, recv, bars, total;
};

__host__ __device__ inline SmemLayout smem_layout(int C, int RBc, int nchunk) {
  SmemLayout L;
  L.lut = 0;                                   // must stay at offset 0 (see lookup addressing)
  L.aop = L.lut + kLutBytes;                   // 1024-aligned
  L.bop = L.aop + kAOpBytes;
  L.codebuf = L.bop + 2 * kBOpBytes;
  L.part = L.codebuf + kWarps * 2 * kChunkBytes;
  const int part_count = nchunk * 32 > C * RBc ? nchunk * 32 : C * RBc;
  const uint32_t part_floats = static_cast<uint32_t>(part_count);
  L.recv = L.part + ((part_floats * 4 + 15) & ~15u);
  L.bars = L.recv + static_cast<uint32_t>(C * RBc * 4);
  L.total = L.bars + 64;
  return L;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;"
               ::"r"(dst), "l"(src), "r"(src_bytes), "l"(pol) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// acc + (low or high fp16 half of w), exact conversion and one fp32 rounding.
__device__ __forceinline__ float add_lo(float acc, uint32_t w) {
  float r;
  asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tadd.rn.f32.f16 %0, lo, %2;\n\t}" : "=f"(r) : "r"(w), "f"(acc));
  return r;
}
__device__ __forceinline__ float add_hi(float acc, uint32_t w) {
  float r;
  asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tadd.rn.f32.f16 %0, hi, %2;\n\t}" : "=f"(r) : "r"(w), "f"(acc));
  return r;
}

// Descriptor of a K-major operand in the no-swizzle canonical layout: 8-row x
// 16-byte core matrices, the two K halves 128 bytes apart (leading byte
// offset), consecutive 8-row groups 256 bytes apart (stride byte offset).
__device__ __forceinline__ uint64_t umma_desc_kmajor_noswizzle(uint32_t smem_byte_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_byte_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;
  d |= static_cast<uint64_t>(256u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;  // layout type 0 (no swizzle), base offset 0
}
__device__ __forceinline__ uint32_t kmajor_noswizzle_offset(int row, int khalf) {
  return static_cast<uint32_t>((row >> 3) * 256 + khalf * 128 + (row & 7) * 16);
}

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Issue the cp.async copies of one 32-row code chunk (rows row0.., groups
// gbeg..gbeg+gcnt) into `buf`; bytes outside the rows or groups are zero-filled.
__device__ __forceinline__ void load_code_chunk(const LutParams& p, uint32_t buf, int row0, int row_end,
                                                int gbeg, int gcnt, int lane, uint64_t pol) {
  const size_t row_bytes = static_cast<size_t>(p.G) * 2;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int id = it * 32 + lane;
    const int r = id >> 3;
    const int part = id & 7;
    const int row = row0 + r;
    const int valid_groups = gcnt - part * 8;
    uint32_t bytes = 0;
    const uint8_t* src = p.codes;
    if (row < row_end && valid_groups > 0) {
      bytes = static_cast<uint32_t>(valid_groups >= 8 ? 16 : valid_groups * 2);
      src = p.codes + static_cast<size_t>(row) * row_bytes + static_cast<size_t>(gbeg) * 2 + part * 16;
    }
    cp_async_16(buf + static_cast<uint32_t>(r * 128 + part * 16), src, bytes, pol);
  }
  cp_async_commit();
}

__global__ void __launch_bounds__(kThreads, 1) gemv_lut_2x8_kernel(const LutParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int C = p.C;
  const SmemLayout L = smem_layout(C, p.RBc, p.nchunk);
  const uint32_t sbase = smem_addr(smem);
  float* part = reinterpret_cast<float*>(smem + L.part);
  float* recv = reinterpret_cast<float*>(smem + L.recv);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* red_bar = mma_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_bar + 2);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t crank = cluster_ctarank();
  const int cluster = blockIdx.x / C;
  const int rb0 = cluster * p.RB;
  const int rb1 = min(p.N, rb0 + p.RB);
  const int nrows = max(0, rb1 - rb0);
  const int nch = (nrows + 31) >> 5;
  const uint64_t pol = l2_policy_evict_first();

  // ---- set-up: TMEM, barriers, B operands (both codebooks, K padded to 16) ----
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  if (tid == 0) {
    mbar_init(mma_bar, 1);
    mbar_init(red_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < 2 * 256; i += kThreads) {
    const int m = i >> 8, idx = i & 255;
    const uint4 v = ldg_nc_v4(p.codebooks + (static_cast<size_t>(m) * 256 + idx) * 8);
    uint8_t* b = smem + L.bop + m * kBOpBytes;
    *reinterpret_cast<uint4*>(b + kmajor_noswizzle_offset(idx, 0)) = v;
    *reinterpret_cast<uint4*>(b + kmajor_noswizzle_offset(idx, 1)) = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int i = tid; i < p.nchunk * 32; i += kThreads) part[i] = 0.f;
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = umma_idesc_f16_f32(128, 256);
  uint32_t mma_phase = 0;
  bool ok = true;

  const uint32_t code_buf0 = sbase + L.codebuf + static_cast<uint32_t>(warp) * 2 * kChunkBytes;

  for (int pass = 0; pass < p.P; ++pass) {
    const int gbeg = (static_cast<int>(crank) * p.P + pass) * kGroupsPerPass;
    const int gcnt = min(kGroupsPerPass, p.G - gbeg);
    if (gcnt <= 0) break;  // uniform across the CTA

    // prefetch this warp's first code chunk while the table is being built
    if (warp < nch) load_code_chunk(p, code_buf0, rb0 + warp * 32, rb1, gbeg, gcnt, lane, pol);

    // ---- A operand: row rho holds x of group gbeg + 2*(rho % 32) + rho / 32 ----
    if (tid < 128) {
      const int rho = tid;
      const int gg = 2 * (rho & 31) + (rho >> 5);
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (rho < 64 && gg < gcnt) v = ldg_nc_v4(p.x + static_cast<size_t>(gbeg + gg) * 8);
      *reinterpret_cast<uint4*>(smem + L.aop + kmajor_noswizzle_offset(rho, 0)) = v;
      *reinterpret_cast<uint4*>(smem + L.aop + kmajor_noswizzle_offset(rho, 1)) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {
      tc_fence_after_sync();
      const uint64_t adesc = umma_desc_kmajor_noswizzle(sbase + L.aop);
      umma_f16_ss(tmem, adesc, umma_desc_kmajor_noswizzle(sbase + L.bop), idesc, 0u);
      umma_f16_ss(tmem + 256, adesc, umma_desc_kmajor_noswizzle(sbase + L.bop + kBOpBytes), idesc, 0u);
      umma_commit(mma_bar);
    }
    bool done = ok ? mbar_wait_bounded(mma_bar, mma_phase, p.status, kSiteLutMma) : false;
    mma_phase ^= 1u;
    ok = __syncthreads_and(done ? 1 : 0) != 0;
    tc_fence_after_sync();

    // ---- table: TMEM lanes 0..63 (warps 0,1,4,5) -> fp16 pairs in shared memory ----
    if (ok && (warp & 3) < 2) {
      const int rho = 32 * (warp & 3) + lane;  // word column of this thread
      const int idx0 = (warp >> 2) * 128;
      uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L.lut);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const int i0 = idx0 + 32 * c;
        uint32_t r0[32], r1[32];
        const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        tmem_ld_32x32b_x32(tmem + lane_off + static_cast<uint32_t>(i0), r0);
        tmem_ld_32x32b_x32(tmem + lane_off + 256u + static_cast<uint32_t>(i0), r1);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          lut[(i0 + j) * 64 + rho] = f2_to_h2_rn(__uint_as_float(r0[j]), __uint_as_float(r1[j]));
      }
    }
    tc_fence_before_sync();
    __syncthreads();

    // ---- lookups: lane = row of a 32-row chunk, rotated code words ----
    if (ok) {
      int it = 0;
      for (int ch = warp; ch < nch; ch += kWarps, ++it) {
        const uint32_t buf = code_buf0 + static_cast<uint32_t>(it & 1) * kChunkBytes;
        const int next = ch + kWarps;
        if (next < nch) {
          load_code_chunk(p, code_buf0 + static_cast<uint32_t>((it + 1) & 1) * kChunkBytes,
                          rb0 + next * 32, rb1, gbeg, gcnt, lane, pol);
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
        __syncwarp();
        const uint32_t row_buf = buf + static_cast<uint32_t>(lane) * 128u;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
        for (int s = 0; s < 32; ++s) {
          const uint32_t wv = static_cast<uint32_t>(((lane + s) & 31) << 2);   // 4 * code word
          const uint32_t cw = lds32(row_buf + wv);
          // byte offsets into the table (it starts at shared offset 0): entry * 256 + column * 4
          const uint32_t o0 = __byte_perm(cw, wv, 0x5504);
          const uint32_t o1 = __byte_perm(cw, wv, 0x5514);
          const uint32_t o2 = __byte_perm(cw, wv, 0x5524);
          const uint32_t o3 = __byte_perm(cw, wv, 0x5534);
          a0 = add_lo(a0, lds32(sbase + o0));
          a1 = add_hi(a1, lds32(sbase + o1));
          a2 = add_lo(a2, lds32(sbase + o2 + 128u));
          a3 = add_hi(a3, lds32(sbase + o3 + 128u));
        }
        part[ch * 32 + lane] += (a0 + a1) + (a2 + a3);
        __syncwarp();
      }
    }
    // the next pass rebuilds the table: every warp must be done reading it
    __syncthreads();
  }

  cp_async_wait<0>();  // no copy may still be in flight when the CTA moves on

  // ---- cluster reduction of the row partials ----------------------------------
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
  const uint32_t slice_bytes = static_cast<uint32_t>(p.RBc) * 4u;
  if (tid == 0) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_addr(red_bar)), "r"(slice_bytes * static_cast<uint32_t>(C)) : "memory");
  }
  fence_proxy_async_smem();
  cluster_sync_all();  // partials final everywhere, every receive barrier armed
  if (tid < C) {
    const uint32_t dst_rank = static_cast<uint32_t>(tid);
    const uint32_t src = sbase + L.part + dst_rank * slice_bytes;
    const uint32_t dst = mapa_shared(sbase + L.recv + crank * slice_bytes, dst_rank);
    const uint32_t bar = mapa_shared(smem_addr(red_bar), dst_rank);
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "r"(src), "r"(slice_bytes), "r"(bar) : "memory");
  }
  const bool got = mbar_wait_bounded(red_bar, 0, p.status, kSiteLutReduce);
  if (got && ok) {
    for (int r = tid; r < p.RBc; r += kThreads) {
      const int row = rb0 + static_cast<int>(crank) * p.RBc + r;
      if (row >= rb1) break;
      float s = 0.f;
      for (int c = 0; c < C; ++c) s += recv[c * p.RBc + r];
      const float bi = p.bias ? __half2float(p.bias[row]) : 0.f;
      p.y[row] = __float2half_rn(s * __half2float(p.scales[row]) + bi);
    }
  }
  cluster_sync_all();  // no CTA leaves while a peer's copy may still read its memory
}

struct Plan {
  int C, P, Q;
};

// The cost model picks (cluster size C, passes P) for a layer: P passes of 64
// groups per CTA, C = ceil(G / 64P) <= 16 CTAs per cluster, Q clusters resident.
// Cost per CTA (cycles): rows * 128P lookups at ~24 per cycle plus ~600 per pass
// to build and store the table.
int plan_cost(int N, int C, int P, int Q) {
  const int rows = (N + Q - 1) / Q;
  return rows * 128 * P / 24 + 600 * P;
}

// Chooses (C, P, Q) for a layer on the current device; cached per (device, N, K).
cudaError_t lut_plan(int dev, int N, int G, Plan* out) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int>, Plan> cache;
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(std::make_tuple(dev, N, G));
    if (it != cache.end()) {
      *out = it->second;
      return cudaSuccess;
    }
  }
  auto kern = gemv_lut_2x8_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  const int cmax = (e == cudaSuccess) ? 16 : 8;
  cudaGetLastError();
  Plan best{0, 0, 0};
  int best_cost = 0;
  for (int P = 1; P <= 64; ++P) {
    const int C = (G + 64 * P - 1) / (64 * P);
    if (C > cmax) continue;
    const int RB_guess = (N + 7) / 8;
    const int RBc_guess = (((RB_guess + C - 1) / C) + 3) & ~3;
    const SmemLayout Lg = smem_layout(C, RBc_guess, (RB_guess + 31) / 32);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(Lg.total));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(C);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(C), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = Lg.total;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int q = 0;
    e = cudaOccupancyMaxActiveClusters(&q, kern, &cfg);
    if (e != cudaSuccess || q <= 0) {
      cudaGetLastError();
      if (C == 1) break;
      continue;
    }
    const int cost = plan_cost(N, C, P, q);
    if (best.C == 0 || cost < best_cost) {
      best = Plan{C, P, q};
      best_cost = cost;
    }
    if (C == 1) break;
  }
  if (best.C == 0) return cudaErrorInvalidConfiguration;
  std::lock_guard<std::mutex> lock(mu);
  cache[std::make_tuple(dev, N, G)] = best;
  *out = best;
  return cudaSuccess;
}

}  // namespace

bool gemv_lut_supported(int M, int B, int g, int K, int batch) {
  return M == 2 && B == 8 && g == 8 && batch == 1 && K % 64 == 0;
}

cudaError_t launch_gemv_lut(const Problem& pr, uint32_t* status, cudaStream_t stream) {
  const int G = pr.K / 8;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  Plan best;
  e = lut_plan(dev, pr.N, G, &best);
  if (e != cudaSuccess) return e;
  auto kern = gemv_lut_2x8_kernel;

  LutParams p{};
  p.x = static_cast<const __half*>(pr.x);
  p.codes = static_cast<const uint8_t*>(pr.codes);
  p.codebooks = static_cast<const __half*>(pr.codebooks);
  p.scales = static_cast<const __half*>(pr.scales);
  p.bias = static_cast<const __half*>(pr.bias);
  p.y = static_cast<__half*>(pr.y);
  p.K = pr.K;
  p.N = pr.N;
  p.G = G;
  p.C = best.C;
  p.P = best.P;
  const int Q = std::max(1, std::min(best.Q, (pr.N + 31) / 32));
  p.RB = (pr.N + Q - 1) / Q;
  p.RBc = (((p.RB + p.C - 1) / p.C) + 3) & ~3;
  p.nchunk = (p.RB + 31) / 32;
  p.status = status;
  const SmemLayout L = smem_layout(p.C, p.RBc, p.nchunk);
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
  if (e != cudaSuccess) return e;
  const int clusters = (pr.N + p.RB - 1) / p.RB;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(p.C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(clusters * p.C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace aqlm
