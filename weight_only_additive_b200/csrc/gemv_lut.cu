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
#include <cuda.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "aqlm_device.cuh"

namespace aqlm {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kGroupsPerPass = 64;
constexpr int kMaxPasses = 4;                      // K <= 16 CTAs x 4 passes x 64 groups x 8
constexpr int kTileRows = 64;                      // rows per code tile (one TMA box)
constexpr uint32_t kLutBytes = 256u * 64u * 4u;   // 64 KB
constexpr uint32_t kAOpBytes = 128u * 32u;         // 4 KB per pass
constexpr uint32_t kBOpBytes = 256u * 32u;         // 8 KB per codebook
constexpr uint32_t kTileBytes = 64u * 128u;        // 64 rows x 128 B of codes (one TMA box)
constexpr uint32_t kTmemCols = 512;                // D_0 at [0,256), D_1 at [256,512)
constexpr uint32_t kSmemLimit = 227u * 1024u;

struct LutParams {
  const __half* x;
  const __half* codebooks;
  const __half* scales;
  const __half* bias;
  __half* y;
  int K, N, G;
  int C;      // CTAs per cluster (K slices)
  int P;      // passes of 64 groups per CTA
  int RB;     // output rows per cluster
  int RBc;    // rows each CTA reduces (multiple of 4)
  int ntask;  // ceil(RB / 8): 8-row tasks per pass
  int ntile;  // ceil(RB / 64): code tiles per pass
  uint32_t* status;
};

struct SmemLayout {
  uint32_t lut, aop, bop, tiles, part, recv, bars, total;
};

// All code tiles of the CTA's passes stay resident: P * ntile tiles of 8 KB.
__host__ __device__ inline SmemLayout smem_layout(int C, int P, int RBc, int ntask, int ntile) {
  SmemLayout L;
  L.lut = 0;
  L.aop = L.lut + kLutBytes;                                        // 1024-aligned
  L.bop = L.aop + kAOpBytes * static_cast<uint32_t>(P);
  L.tiles = L.bop + 2 * kBOpBytes;
  L.part = L.tiles + static_cast<uint32_t>(P * ntile) * kTileBytes;
  const int part_count = ntask * 8 > C * RBc ? ntask * 8 : C * RBc;
  L.recv = L.part + ((static_cast<uint32_t>(part_count) * 4u + 15u) & ~15u);
  L.bars = L.recv + static_cast<uint32_t>(C * RBc * 4);
  L.total = L.bars + 8u * static_cast<uint32_t>(P * ntile + 2);
  return L;
}

// Rows per cluster for a layer: as even a split over Q resident clusters as the
// shared memory allows (all code tiles of a CTA resident); 0 if not even 64 fit.
__host__ __device__ inline int rows_per_cluster(int N, int Q, int C, int P) {
  int RB = (N + Q - 1) / Q;
  RB = (RB + 7) & ~7;
  while (RB >= 8) {
    const int RBc = (((RB + C - 1) / C) + 3) & ~3;
    if (smem_layout(C, P, RBc, (RB + 7) / 8, (RB + kTileRows - 1) / kTileRows).total <= kSmemLimit) return RB;
    RB = RB > 64 ? RB - 64 : RB - 8;
  }
  return 0;
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

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
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
__host__ __device__ inline uint32_t kmajor_noswizzle_offset(int row, int khalf) {
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

__global__ void __launch_bounds__(kThreads, 1) gemv_lut_2x8_kernel(const __grid_constant__ CUtensorMap code_map,
                                                                    const LutParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int C = p.C;
  const SmemLayout L = smem_layout(C, p.P, p.RBc, p.ntask, p.ntile);
  const uint32_t sbase = smem_addr(smem);
  float* part = reinterpret_cast<float*>(smem + L.part);
  float* recv = reinterpret_cast<float*>(smem + L.recv);
  uint64_t* tile_bar = reinterpret_cast<uint64_t*>(smem + L.bars);   // [P * ntile] tile landed
  uint64_t* mma_bar = tile_bar + p.P * p.ntile;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_bar + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t crank = cluster_ctarank();
  const int cluster = blockIdx.x / C;
  const int rb0 = cluster * p.RB;
  const int rb1 = min(p.N, rb0 + p.RB);
  const int nrows = max(0, rb1 - rb0);
  const int nt = (nrows + 7) >> 3;                          // 8-row tasks of this row block
  const int ntl = (nrows + kTileRows - 1) / kTileRows;      // 64-row tiles of this row block

  // passes this CTA runs (gcnt > 0); uniform across the CTA
  int npass = 0;
  while (npass < p.P && (static_cast<int>(crank) * p.P + npass) * kGroupsPerPass < p.G) ++npass;

  // The next kernel in the stream may start its own weight-only set-up now.
  grid_dependents_launch();

  // ---- 1. barriers; one thread starts the whole code stream (a TMA box per tile) --------
  if (tid == 0) {
    for (int i = 0; i < p.P * p.ntile; ++i) mbar_init(&tile_bar[i], 1);
    mbar_init(mma_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (tid == 32 * (kWarps - 1)) {
    const uint64_t pol = l2_policy_evict_first();
    for (int ps = 0; ps < npass; ++ps) {
      const int gbeg = (static_cast<int>(crank) * p.P + ps) * kGroupsPerPass;
      for (int tl = 0; tl < ntl; ++tl) {
        const int i = ps * p.ntile + tl;
        mbar_arrive_expect_tx(&tile_bar[i], kTileBytes);
        tma_load_2d(sbase + L.tiles + static_cast<uint32_t>(i) * kTileBytes, &code_map, gbeg * 2,
                           rb0 + tl * kTileRows, &tile_bar[i], pol);
      }
    }
  }

  // scale and bias of the rows this CTA reduces at the end (read now, used last)
  float row_scale = 0.f, row_bias = 0.f;
  {
    const int row = rb0 + static_cast<int>(crank) * p.RBc + tid;
    if (tid < p.RBc && row < rb1) {
      row_scale = __half2float(p.scales[row]);
      row_bias = p.bias ? __half2float(p.bias[row]) : 0.f;
    }
  }

  // ---- 2. operands (both codebooks, x of every pass) and TMEM ------------------------------
  {
    for (int i = tid; i < 2 * 256; i += kThreads) {
      const int m = i >> 8, idx = i & 255;
      const uint32_t bo = L.bop + static_cast<uint32_t>(m) * kBOpBytes;
      cp_async_16_zfill(sbase + bo + kmajor_noswizzle_offset(idx, 0), p.codebooks + (static_cast<size_t>(m) * 256 + idx) * 8, 16);
      *reinterpret_cast<uint4*>(smem + bo + kmajor_noswizzle_offset(idx, 1)) = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = tid; i < p.ntask * 8; i += kThreads) part[i] = 0.f;
    // Everything above reads only weights.  x may be the output of the kernel just
    // before this one in the stream (programmatic dependent launch): wait for it.
    grid_dependency_wait();
    for (int i = tid; i < npass * 128; i += kThreads) {  // A row rho (and rho+64) = one group of x
      const int ps = i >> 7, rho = i & 127;
      const int gbeg = (static_cast<int>(crank) * p.P + ps) * kGroupsPerPass;
      const int gg = 2 * (rho & 31) + ((rho >> 5) & 1);
      const uint32_t ao = L.aop + static_cast<uint32_t>(ps) * kAOpBytes;
      const bool valid = gbeg + gg < p.G;
      cp_async_16_zfill(sbase + ao + kmajor_noswizzle_offset(rho, 0),
                       valid ? static_cast<const void*>(p.x + static_cast<size_t>(gbeg + gg) * 8)
                             : static_cast<const void*>(p.x),
                       valid ? 16u : 0u);
      *reinterpret_cast<uint4*>(smem + ao + kmajor_noswizzle_offset(rho, 1)) = make_uint4(0u, 0u, 0u, 0u);
    }
    cp_async_commit();
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  asm volatile("cp.async.wait_all;" ::: "memory");
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = umma_idesc_f16_f32(128, 256);
  uint32_t mma_phase = 0;
  bool ok = true;
  const int r8 = lane >> 2;  // row of the 8-row task
  const int q4 = lane & 3;   // quarter of the row's 32 code words

  for (int ps = 0; ps < npass; ++ps) {
    // ---- 3. table of this pass: two MMAs into TMEM ---------------------------------------
    if (tid == 0 && ok) {
      tc_fence_after_sync();
      const uint64_t adesc = umma_desc_kmajor_noswizzle(sbase + L.aop + static_cast<uint32_t>(ps) * kAOpBytes);
      umma_f16_ss(tmem, adesc, umma_desc_kmajor_noswizzle(sbase + L.bop), idesc, 0u);
      umma_f16_ss(tmem + 256, adesc, umma_desc_kmajor_noswizzle(sbase + L.bop + kBOpBytes), idesc, 0u);
      umma_commit(mma_bar);
    }
    const bool done = ok ? mbar_wait_bounded(mma_bar, mma_phase, p.status, kSiteLutMma) : false;
    mma_phase ^= 1u;
    ok = __syncthreads_and(done ? 1 : 0) != 0;
    tc_fence_after_sync();

    // ---- 4. TMEM -> shared-memory table, all 16 warps (A rows rho and rho+64 agree) --------
    if (ok) {
      const int qd = warp & 3;
      const int col = 32 * (qd & 1) + lane;                 // word column = rho mod 64
      const int i0 = 32 * (2 * (warp >> 2) + (qd >> 1));    // 32 table entries per warp
      const uint32_t lane_off = static_cast<uint32_t>(32 * qd) << 16;
      uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L.lut);
      uint32_t r0[32], r1[32];
      tmem_ld_32x32b_x32(tmem + lane_off + static_cast<uint32_t>(i0), r0);
      tmem_ld_32x32b_x32(tmem + lane_off + 256u + static_cast<uint32_t>(i0), r1);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        lut[(i0 + j) * 64 + col] = f2_to_h2_rn(__uint_as_float(r0[j]), __uint_as_float(r1[j]));
    }
    tc_fence_before_sync();
    __syncthreads();

    {
      // ---- 5. lookups: a task is 8 rows; 4 lanes per row, 8 code words each -------------------
      // Lane (r8, q4) reads code word w = 8*q4 + ((r8 + s) mod 8) at step s: the 32 lanes
      // always touch 32 distinct words, so both the code reads and the table reads are
      // free of bank conflicts.  Pairs of looked-up fp16 values are added as half2 and
      // the task's 16 pair sums are accumulated in half2, then widened to fp32.
      for (int t = warp; t < nt; t += kWarps) {
        const int i = ps * p.ntile + t / 8;  // tile holding rows 8t .. 8t+7
        const bool landed = mbar_wait_bounded(&tile_bar[i], 0u, p.status, kSiteLutCodes);
        if (ok && landed) {
          const uint32_t* cw_row = reinterpret_cast<const uint32_t*>(
              smem + L.tiles + i * kTileBytes + ((t & 7) * 8 + r8) * 128);
          uint32_t cw[8];
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8) cw[s8] = cw_row[8 * q4 + ((r8 + s8) & 7)];
          __half2 hacc = __float2half2_rn(0.f);
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8) {
            const uint32_t wv = static_cast<uint32_t>((8 * q4 + ((r8 + s8) & 7)) << 2);  // 4 * code word
            // table byte offsets: entry * 256 + column * 4 (column w, or 32 + w at +128)
            const uint32_t t0 = *reinterpret_cast<const uint32_t*>(smem + __byte_perm(cw[s8], wv, 0x5504));
            const uint32_t t1 = *reinterpret_cast<const uint32_t*>(smem + __byte_perm(cw[s8], wv, 0x5514));
            const uint32_t t2 = *reinterpret_cast<const uint32_t*>(smem + __byte_perm(cw[s8], wv, 0x5524) + 128u);
            const uint32_t t3 = *reinterpret_cast<const uint32_t*>(smem + __byte_perm(cw[s8], wv, 0x5534) + 128u);
            // (codebook-0 value of t0, codebook-1 value of t1) and likewise for t2, t3
            const uint32_t p01 = __byte_perm(t0, t1, 0x7610);
            const uint32_t p23 = __byte_perm(t2, t3, 0x7610);
            hacc = __hadd2(hacc, __hadd2(*reinterpret_cast<const __half2*>(&p01),
                                         *reinterpret_cast<const __half2*>(&p23)));
          }
          const float2 f = __half22float2(hacc);
          float v = f.x + f.y;
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          if (q4 == 0) part[t * 8 + r8] += v;
        } else if (!landed) {
          ok = false;
        }
      }
    }
    // the next pass rebuilds the table: every warp must be done reading it
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
  }

  // ---- 6. partials -> their owner CTA (remote shared-memory stores), one cluster barrier ----
  // Row r of the block is reduced by CTA r / RBc; this CTA's partial of it lands in
  // the owner's recv[crank][r mod RBc].  After the barrier every owner holds all C
  // partials of its rows and no CTA touches another CTA's memory any more.
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
  for (int v4 = tid; v4 * 4 < p.RBc * C; v4 += kThreads) {
    const int r = v4 * 4;  // 4 consecutive rows, never split between owners (RBc % 4 == 0)
    const uint32_t owner = static_cast<uint32_t>(r / p.RBc);
    const float4 val = *reinterpret_cast<const float4*>(part + r);
    const uint32_t dst = mapa_shared(sbase + L.recv + (crank * static_cast<uint32_t>(p.RBc) +
                                                       static_cast<uint32_t>(r - static_cast<int>(owner) * p.RBc)) * 4u,
                                     owner);
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};"
                 ::"r"(dst), "f"(val.x), "f"(val.y), "f"(val.z), "f"(val.w) : "memory");
  }
  cluster_sync_all();
  if (ok) {
    for (int r = tid; r < p.RBc; r += kThreads) {
      const int row = rb0 + static_cast<int>(crank) * p.RBc + r;
      if (row >= rb1) break;
      float s = 0.f;
      for (int c = 0; c < C; ++c) s += recv[c * p.RBc + r];
      const float sc = (r == tid) ? row_scale : __half2float(p.scales[row]);
      const float bi = (r == tid) ? row_bias : (p.bias ? __half2float(p.bias[row]) : 0.f);
      p.y[row] = __float2half_rn(s * sc + bi);
    }
  }
}

struct Plan {
  int C, P, Q, RB;
};

// The cost model picks (cluster size C, passes P) for a layer: P passes of 64
// groups per CTA, C = ceil(G / 64P) <= 16 CTAs per cluster, Q clusters resident,
// RB rows per cluster (fewer than N / Q when the code tiles would not fit, which
// costs extra waves).  Cycles per CTA: rows * 128P lookups at ~24 per cycle plus
// ~600 per pass to build and store the table.
int plan_cost(int N, int P, int Q, int RB) {
  const int clusters = (N + RB - 1) / RB;
  const int waves = (clusters + Q - 1) / Q;
  return waves * (RB * 128 * P / 24 + 600 * P);
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
  Plan best{0, 0, 0, 0};
  int best_cost = 0;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemLimit));
  if (e != cudaSuccess) return e;
  for (int P = 1; P <= kMaxPasses; ++P) {
    const int C = (G + 64 * P - 1) / (64 * P);
    if (C > cmax) continue;
    // one CTA per SM (its TMEM and shared memory), so residency is set by cluster placement
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(C);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(C), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemLimit;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int q = 0;
    e = cudaOccupancyMaxActiveClusters(&q, kern, &cfg);
    if (e != cudaSuccess || q <= 0) {
      cudaGetLastError();
      if (C == 1) break;
      continue;
    }
    q = std::min(q, std::max(1, (N + 31) / 32));
    const int RB = rows_per_cluster(N, q, C, P);
    if (RB == 0) {
      if (C == 1) break;
      continue;
    }
    const int cost = plan_cost(N, P, q, RB);
    if (best.C == 0 || cost < best_cost) {
      best = Plan{C, P, q, RB};
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
  return M == 2 && B == 8 && g == 8 && batch == 1 && K % 64 == 0 && K <= 16 * kMaxPasses * kGroupsPerPass * 8;
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

  // Codes as a 2D byte tensor [N rows][2G bytes]; a box is 64 rows x 128 bytes
  // (one 64-group pass of 64 rows).  Out-of-range rows and bytes read as zero.
  EncodeTiledFn encode = encode_tiled();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(G) * 2, static_cast<cuuint64_t>(pr.N)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(G) * 2};
  const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(kTileRows)};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(pr.codes), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  LutParams p{};
  p.x = static_cast<const __half*>(pr.x);
  p.codebooks = static_cast<const __half*>(pr.codebooks);
  p.scales = static_cast<const __half*>(pr.scales);
  p.bias = static_cast<const __half*>(pr.bias);
  p.y = static_cast<__half*>(pr.y);
  p.K = pr.K;
  p.N = pr.N;
  p.G = G;
  p.C = best.C;
  p.P = best.P;
  p.RB = best.RB;
  p.RBc = (((p.RB + p.C - 1) / p.C) + 3) & ~3;
  p.ntask = (p.RB + 7) / 8;
  p.ntile = (p.RB + kTileRows - 1) / kTileRows;
  p.status = status;
  const SmemLayout L = smem_layout(p.C, p.P, p.RBc, p.ntask, p.ntile);
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
  if (e != cudaSuccess) return e;
  const int clusters = (pr.N + p.RB - 1) / p.RB;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(p.C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(clusters * p.C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cfg.attrs = attr;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, map, p);
}

}  // namespace aqlm
