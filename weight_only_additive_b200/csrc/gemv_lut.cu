// Lookup-table GEMV for codebooks of 256 entries (B = 8), batch 1: "fast lookup,
// no per-element dequantization" (inference-research record "AQLM (additive /
// multi-codebook quantization)", section "Kernels").
//
//   T_m[j][i] = sum_t x[g j + t] * C_m[i][t]            (per group j, codebook m, entry i)
//   y[n]      = s_n * sum_j sum_m T_m[j][codes[n,j,m]] + bias_n
//
// A code row is G M bytes (byte b = code of codebook b mod M in group b / M), cut
// into slices of 128 bytes; the table of a slice holds the 128 x 256 entries of
// its bytes, and a row's partial over the slice is the sum of its 128 lookups.
//
// Work split.  A cluster of C CTAs owns a block of output rows; CTA c of the
// cluster owns P consecutive slices (passes).  Per pass the CTA
//   1. builds the slice's table with tcgen05.mma (M = 128 rows, N = 256 codebook
//      entries, K = 16 per step), accumulator in TMEM;
//   2. moves it TMEM -> registers -> shared memory as fp16 entries,
//      256 entries x 128 bytes x 2 B = 64 KB;
//   3. sums the lookups of its rows from code tiles (64 rows x 128 bytes, one TMA
//      box each).  The CTA's tiles are issued at the start into R shared-memory
//      slots; when they do not all fit (long rows), a slot is reloaded with a later
//      pass's tile as soon as the pass that read it ends.
// The row partials of the C CTAs are exchanged through distributed shared memory
// inside the cluster and summed in a fixed order (deterministic), then the channel
// scale and bias are applied.
//
// 2x8 g8 (two codebooks of 8-wide codewords, a slice = 64 groups) has its own tuned
// instantiation: one MMA per codebook, whose two results pack into one word per
// (entry, group).  Every other scheme uses the stacked build of lut_table.cuh (the
// M codebooks side by side along K, one TMEM lane per code byte), with its x slices
// double-buffered.
//
// Bank-conflict-free lookups.  A task is 8 rows, 4 lanes per row; lane (r8, q4)
// reads code word w = 8 q4 + ((r8 + s) mod 8) of its row at step s (4 code bytes,
// pairs 2w and 2w + 1).  The table stores pair 2w in word column w and pair 2w + 1
// in column 32 + w of each entry's 64-word row, so the 32 lanes of a lookup touch 32
// different banks whatever the codes are.
#include <cuda.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "aqlm_device.cuh"
#include "lut_table.cuh"

namespace aqlm {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxPasses = 4;                      // code rows <= 16 CTAs x 4 passes x 128 bytes
constexpr int kTileRows = 64;                      // rows per code tile (one TMA box)
constexpr uint32_t kLutBytes = lut::kTableBytes;   // 64 KB
constexpr uint32_t kAOpBytes = lut::kAOpBytes;     // 4 KB per pass and K step
constexpr uint32_t kBOpBytes = lut::kBOpBytes;     // 8 KB per codebook (tuned) or K step (stacked)
constexpr uint32_t kTileBytes = 64u * 128u;        // 64 rows x 128 B of codes (one TMA box)
constexpr uint32_t kTmemCols = 512;                // D_0 at [0,256), D_1 at [256,512)
constexpr uint32_t kSmemLimit = 227u * 1024u;

struct LutParams {
  const __half* x;
  const __half* codebooks;
  const __half* scales;
  const __half* bias;
  __half* y;
  int N, G, M, g;
  int S;      // 128-byte slices of a code row
  int C;      // CTAs per cluster
  int P;      // passes (slices) per CTA
  int RB;     // output rows per cluster
  int RBc;    // rows each CTA reduces (multiple of 4)
  int ntask;  // ceil(RB / 8): 8-row tasks per pass
  int ntile;  // ceil(RB / 64): code tiles per pass
  int R;      // code-tile slots, >= ntile: tile i = ps ntile + tl of the CTA goes to slot i mod R
  uint32_t* status;
};

struct SmemLayout {
  uint32_t lut, aop, bop, tiles, part, recv, bars, total;
};

// Table operands: the tuned build keeps the A operands of all P passes (one K step
// each) and two one-step codebooks; the stacked build has ks K steps
// (lut::stacked_ksteps) and two A buffers that take the passes in turn.
struct OperandBytes {
  uint32_t a, b;
};
__host__ __device__ inline OperandBytes operand_bytes(bool generic, int P, int M, int g) {
  if (!generic) return OperandBytes{kAOpBytes * static_cast<uint32_t>(P), 2u * kBOpBytes};
  const uint32_t ks = static_cast<uint32_t>(lut::stacked_ksteps(M, g));
  return OperandBytes{kAOpBytes * ks * static_cast<uint32_t>(P < 2 ? P : 2), kBOpBytes * ks};
}

// R code-tile slots of 8 KB (all P * ntile tiles of the CTA when they fit, else at
// least one pass's ntile, reused pass after pass); one mbarrier per tile.
__host__ __device__ inline SmemLayout smem_layout(int C, int P, int RBc, int ntask, int ntile, int R, OperandBytes ob) {
  SmemLayout L;
  L.lut = 0;
  L.aop = L.lut + kLutBytes;                                        // 1024-aligned
  L.bop = L.aop + ob.a;
  L.tiles = L.bop + ob.b;
  L.part = L.tiles + static_cast<uint32_t>(R) * kTileBytes;
  const int part_count = ntask * 8 > C * RBc ? ntask * 8 : C * RBc;
  L.recv = L.part + ((static_cast<uint32_t>(part_count) * 4u + 15u) & ~15u);
  L.bars = L.recv + static_cast<uint32_t>(C * RBc * 4);
  L.total = L.bars + 8u * static_cast<uint32_t>(P * ntile + 2);
  return L;
}

// Rows per cluster RB and code-tile slots R for a layer: as even a split over Q
// resident clusters as the shared memory allows.  R = P ntile (every tile of the CTA
// resident) when that fits, else the slots that fit, as long as one pass's ntile tiles
// do; {0, 0} if not even 8 rows fit.
struct RowSplit {
  int RB, R;
};
inline RowSplit rows_per_cluster(int N, int Q, int C, int P, OperandBytes ob) {
  int RB = (N + Q - 1) / Q;
  RB = (RB + 7) & ~7;
  while (RB >= 8) {
    const int RBc = (((RB + C - 1) / C) + 3) & ~3;
    const int ntile = (RB + kTileRows - 1) / kTileRows;
    const SmemLayout full = smem_layout(C, P, RBc, (RB + 7) / 8, ntile, P * ntile, ob);
    if (full.total <= kSmemLimit) return RowSplit{RB, P * ntile};
    const int drop = static_cast<int>((full.total - kSmemLimit + kTileBytes - 1) / kTileBytes);
    if (P * ntile - drop >= ntile) return RowSplit{RB, P * ntile - drop};
    RB = RB > 64 ? RB - 64 : RB - 8;
  }
  return RowSplit{0, 0};
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
using lut::kmajor_desc;
using lut::kmajor_offset;

// Issues the CTA's code tiles i_begin .. i_end - 1 (one thread): tile i is row tile
// i mod ntile (skipped from ntl on, past this cluster's rows) of pass i / ntile, a
// 64-row x 128-byte TMA box into slot i mod R.  Out of line: it runs a few times per
// launch and its registers would otherwise weigh on the lookup loop.
__device__ __noinline__ void issue_code_tiles(const CUtensorMap* map, uint32_t tiles, uint64_t* tile_bar, int i_begin,
                                              int i_end, int ntile, int ntl, int R, int slice0, int rb0) {
  const uint64_t pol = l2_policy_evict_first();
  for (int i = i_begin; i < i_end; ++i) {
    const int ps = i / ntile, tl = i - ps * ntile;
    if (tl >= ntl) continue;
    mbar_arrive_expect_tx(&tile_bar[i], kTileBytes);
    // bytes past the row end and rows past N are zero-filled
    tma_load_2d(tiles + static_cast<uint32_t>(i % R) * kTileBytes, map, (slice0 + ps) * 128, rb0 + tl * kTileRows,
                &tile_bar[i], pol);
  }
}

// kGeneric = false: 2x8 g8 (the tuned table build); true: any B = 8 scheme.
// kRecycle = false: all P ntile code tiles of a CTA are resident (R = P ntile);
// true: fewer slots, reloaded pass after pass.  Separate instantiations, since the
// reload bookkeeping cost the resident case 3-20 % when it was one kernel (its lookup
// loop's code changes).
template <bool kGeneric, bool kRecycle>
__global__ void __launch_bounds__(kThreads, 1) gemv_lut_kernel(const __grid_constant__ CUtensorMap code_map,
                                                                const LutParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int C = p.C;
  const SmemLayout L = smem_layout(C, p.P, p.RBc, p.ntask, p.ntile, p.R, operand_bytes(kGeneric, p.P, p.M, p.g));
  const int ks = lut::stacked_ksteps(p.M, p.g);                      // stacked build only
  const uint32_t abuf = kAOpBytes * static_cast<uint32_t>(ks);       // one A buffer of it
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

  // passes this CTA runs (slices crank P .. crank P + npass - 1 of the row); uniform
  const int slice0 = static_cast<int>(crank) * p.P;
  const int npass = max(0, min(p.P, p.S - slice0));

  // The next kernel in the stream may start its own weight-only set-up now.
  grid_dependents_launch();

  // ---- 1. barriers; one thread starts the code stream (a TMA box per tile) ---------------
  if (tid == 0) {
    for (int i = 0; i < p.P * p.ntile; ++i) mbar_init(&tile_bar[i], 1);
    mbar_init(mma_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // Tile i = ps ntile + tl (pass ps, rows rb0 + 64 tl ..) lands in slot i mod R.  The
  // tiles i < R start now; tile i >= R starts at the end of the pass that consumed
  // tile i - R (an earlier pass, since R >= ntile).
  const bool issuer = tid == 32 * (kWarps - 1);
  if constexpr (kRecycle) {
    if (issuer)
      issue_code_tiles(&code_map, sbase + L.tiles, tile_bar, 0, min(npass * p.ntile, p.R), p.ntile, ntl, p.R, slice0,
                       rb0);
  } else {
    if (issuer) {
      const uint64_t pol = l2_policy_evict_first();
      for (int ps = 0; ps < npass; ++ps) {
        for (int tl = 0; tl < ntl; ++tl) {
          const int i = ps * p.ntile + tl;
          mbar_arrive_expect_tx(&tile_bar[i], kTileBytes);
          // bytes past the row end and rows past N are zero-filled
          tma_load_2d(sbase + L.tiles + static_cast<uint32_t>(i) * kTileBytes, &code_map, (slice0 + ps) * 128,
                      rb0 + tl * kTileRows, &tile_bar[i], pol);
        }
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

  // ---- 2. operands (the codebooks, x of every pass) and TMEM -------------------------------
  {
    if constexpr (kGeneric) {
      lut::load_codebooks_stacked<kThreads>(p.codebooks, p.M, p.g, sbase + L.bop, tid);
    } else {
      for (int i = tid; i < 2 * 256; i += kThreads) {
        const int m = i >> 8, idx = i & 255;
        const uint32_t bo = L.bop + static_cast<uint32_t>(m) * kBOpBytes;
        cp_async_16_zfill(sbase + bo + kmajor_offset(idx, 0), p.codebooks + (static_cast<size_t>(m) * 256 + idx) * 8, 16);
        *reinterpret_cast<uint4*>(smem + bo + kmajor_offset(idx, 1)) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    for (int i = tid; i < p.ntask * 8; i += kThreads) part[i] = 0.f;
    // Everything above reads only weights.  x may be the output of the kernel just
    // before this one in the stream (programmatic dependent launch): wait for it.
    grid_dependency_wait();
    if constexpr (kGeneric) {
      // passes 0 and 1; pass ps + 2 follows once the MMAs of pass ps have read its buffer
      for (int ps = 0; ps < npass && ps < 2; ++ps)
        lut::load_x_stacked<kThreads>(p.x, p.G, p.M, p.g, slice0 + ps, sbase + L.aop + static_cast<uint32_t>(ps) * abuf,
                                      tid);
    } else {
      for (int i = tid; i < npass * 128; i += kThreads) {  // A row rho (and rho+64) = one group of x
        const int ps = i >> 7, rho = i & 127;
        const int gbeg = (slice0 + ps) * 64;
        const int gg = 2 * (rho & 31) + ((rho >> 5) & 1);
        const uint32_t ao = L.aop + static_cast<uint32_t>(ps) * kAOpBytes;
        const bool valid = gbeg + gg < p.G;
        cp_async_16_zfill(sbase + ao + kmajor_offset(rho, 0),
                          valid ? static_cast<const void*>(p.x + static_cast<size_t>(gbeg + gg) * 8)
                                : static_cast<const void*>(p.x),
                          valid ? 16u : 0u);
        *reinterpret_cast<uint4*>(smem + ao + kmajor_offset(rho, 1)) = make_uint4(0u, 0u, 0u, 0u);
      }
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
    // ---- 3.-4. table of this pass: MMAs into TMEM, then TMEM -> shared memory --------------
    const uint64_t adesc = kmajor_desc(sbase + L.aop + static_cast<uint32_t>(ps) * kAOpBytes);
    if constexpr (!kGeneric) {
      if (tid == 0 && ok) {
        tc_fence_after_sync();
        umma_f16_ss(tmem, adesc, kmajor_desc(sbase + L.bop), idesc, 0u);
        umma_f16_ss(tmem + 256, adesc, kmajor_desc(sbase + L.bop + kBOpBytes), idesc, 0u);
        umma_commit(mma_bar);
      }
      const bool done = ok ? mbar_wait_bounded(mma_bar, mma_phase, p.status, kSiteLutMma) : false;
      mma_phase ^= 1u;
      ok = __syncthreads_and(done ? 1 : 0) != 0;
      tc_fence_after_sync();
      // all 16 warps: A rows rho and rho + 64 hold the same group
      if (ok) lut::store_table_2x8(tmem, warp, lane, smem + L.lut);
      tc_fence_before_sync();
      __syncthreads();
    } else {
      // the stacked build: one MMA chain, one TMEM lane per code byte of the slice
      if (tid == 0 && ok) {
        tc_fence_after_sync();
        lut::mma_stacked(tmem, sbase + L.aop + static_cast<uint32_t>(ps & 1) * abuf, sbase + L.bop, ks, idesc);
        umma_commit(mma_bar);
      }
      const bool done = ok ? mbar_wait_bounded(mma_bar, mma_phase, p.status, kSiteLutMma) : false;
      mma_phase ^= 1u;
      // A buffer ps mod 2 has been read: start the x slice of pass ps + 2 there
      if (done && ps + 2 < npass)
        lut::load_x_stacked<kThreads>(p.x, p.G, p.M, p.g, slice0 + ps + 2,
                                      sbase + L.aop + static_cast<uint32_t>(ps & 1) * abuf, tid);
      cp_async_commit();
      ok = __syncthreads_and(done ? 1 : 0) != 0;
      tc_fence_after_sync();
      if (ok) lut::store_table_stacked(tmem, warp, lane, smem + L.lut);
      tc_fence_before_sync();
      __syncthreads();
    }

    {
      // ---- 5. lookups: a task is 8 rows; 4 lanes per row, 8 code words each -------------------
      // Lane (r8, q4) reads code word w = 8*q4 + ((r8 + s) mod 8) at step s: the 32 lanes
      // always touch 32 distinct words, so both the code reads and the table reads are
      // free of bank conflicts.  Every looked-up fp16 value is added to an fp32
      // accumulator (two per lane, one per half of the table word).
      const int slot0 = kRecycle ? (ps * p.ntile) % p.R : 0;  // slot of the pass's first tile
      for (int t = warp; t < nt; t += kWarps) {
        const int i = ps * p.ntile + t / 8;  // tile holding rows 8t .. 8t+7
        int slot = i;                        // its slot, i mod R
        if constexpr (kRecycle) {
          slot = slot0 + t / 8;
          if (slot >= p.R) slot -= p.R;
        }
        const bool landed = mbar_wait_bounded(&tile_bar[i], 0u, p.status, kSiteLutCodes);
        if (ok && landed) {
          const uint32_t* cw_row = reinterpret_cast<const uint32_t*>(
              smem + L.tiles + slot * kTileBytes + ((t & 7) * 8 + r8) * 128);
          uint32_t cw[8];
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8) cw[s8] = cw_row[8 * q4 + ((r8 + s8) & 7)];
          // fp32 accumulators: even code bytes (low halves of their table words) and odd
          // code bytes (high halves)
          float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8) {
            const uint32_t wv = static_cast<uint32_t>((8 * q4 + ((r8 + s8) & 7)) << 2);  // 4 * code word
            // table byte offsets: entry * 256 + column * 4 (column w, or 32 + w at +128)
            const uint32_t t0 = *reinterpret_cast<const uint32_t*>(smem + __byte_perm(cw[s8], wv, 0x5504));
            const uint32_t t1 = *reinterpret_cast<const uint32_t*>(smem + __byte_perm(cw[s8], wv, 0x5514));
            const uint32_t t2 = *reinterpret_cast<const uint32_t*>(smem + __byte_perm(cw[s8], wv, 0x5524) + 128u);
            const uint32_t t3 = *reinterpret_cast<const uint32_t*>(smem + __byte_perm(cw[s8], wv, 0x5534) + 128u);
            acc0 = add_f32_lo_f16(t0, acc0);
            acc1 = add_f32_hi_f16(t1, acc1);
            acc0 = add_f32_lo_f16(t2, acc0);
            acc1 = add_f32_hi_f16(t3, acc1);
          }
          float v = acc0 + acc1;
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          if (q4 == 0) part[t * 8 + r8] += v;
        } else if (!landed) {
          ok = false;
        }
      }
    }
    if constexpr (kGeneric) {
      // the next pass's A operand (committed one group before the newest) has landed
      asm volatile("cp.async.wait_group 1;" ::: "memory");
      fence_proxy_async_smem();
    }
    // the next pass rebuilds the table: every warp must be done reading it
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    // the slots of pass ps are free: start the tiles R + ps ntile .. that take them
    if (kRecycle && issuer && ok && p.R + ps * p.ntile < npass * p.ntile)
      issue_code_tiles(&code_map, sbase + L.tiles, tile_bar, p.R + ps * p.ntile,
                       min(npass * p.ntile, p.R + (ps + 1) * p.ntile), p.ntile, ntl, p.R, slice0, rb0);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");

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
  int C, P, Q, RB, R;
};

// The cost model picks (cluster size C, passes P) for a layer: P slices of 128 code
// bytes per CTA, C = ceil(S / P) <= 16 CTAs per cluster, Q clusters resident, RB
// rows per cluster (fewer than N / Q when not even one pass of code tiles fits,
// which costs extra waves).  Cycles per CTA: rows * 128P lookups at ~24 per cycle,
// ~600 per pass to build and store the table, and ~800 per pass whose tiles wait for
// recycled slots (their loads start only when the previous pass ends).
int plan_cost(int N, int P, int Q, int RB, int R) {
  const int clusters = (N + RB - 1) / RB;
  const int waves = (clusters + Q - 1) / Q;
  const int ntile = (RB + kTileRows - 1) / kTileRows;
  const int late_passes = (P * ntile - R + ntile - 1) / ntile;
  return waves * (RB * 128 * P / 24 + 600 * P + 800 * late_passes);
}

// Chooses (C, P, Q) for a layer on the current device; cached per (device, N, S, M,
// g, instantiation).
template <bool kGeneric>
cudaError_t lut_plan(int dev, int N, int S, int M, int g, Plan* out) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int>, Plan> cache;
  static bool wide_clusters[64] = {};
  static uint64_t attrs_ctx[64] = {};  // context the kernels' attributes were set in (0: not yet)
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(std::make_tuple(dev, N, S, M, g));
  if (it != cache.end()) {
    *out = it->second;
    return cudaSuccess;
  }
  const uint64_t ctx = current_context_id();
  if (ctx == 0 || attrs_ctx[dev] != ctx) {
    // clusters of up to 16 CTAs where the device allows them, else the portable 8
    wide_clusters[dev] = cudaFuncSetAttribute(gemv_lut_kernel<kGeneric, false>,
                                              cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
                         cudaFuncSetAttribute(gemv_lut_kernel<kGeneric, true>,
                                              cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    cudaGetLastError();
    cudaError_t e = cudaFuncSetAttribute(gemv_lut_kernel<kGeneric, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemLimit));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemv_lut_kernel<kGeneric, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSmemLimit));
    if (e != cudaSuccess) return e;
    attrs_ctx[dev] = ctx;
  }
  const int cmax = wide_clusters[dev] ? 16 : 8;
  Plan best{0, 0, 0, 0, 0};
  int best_cost = 0;
  for (int P = 1; P <= kMaxPasses; ++P) {
    const int C = (S + P - 1) / P;
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
    // both instantiations: one CTA per SM, the same shared memory and TMEM
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&q, gemv_lut_kernel<kGeneric, false>, &cfg);
    if (e != cudaSuccess || q <= 0) {
      cudaGetLastError();
      if (C == 1) break;
      continue;
    }
    q = std::min(q, std::max(1, (N + 31) / 32));
    const RowSplit split = rows_per_cluster(N, q, C, P, operand_bytes(kGeneric, P, M, g));
    const int RB = split.RB;
    if (RB == 0) {
      if (C == 1) break;
      continue;
    }
    const int cost = plan_cost(N, P, q, RB, split.R);
    if (best.C == 0 || cost < best_cost) {
      best = Plan{C, P, q, RB, split.R};
      best_cost = cost;
    }
    if (C == 1) break;
  }
  if (best.C == 0) return cudaErrorInvalidConfiguration;
  cache[std::make_tuple(dev, N, S, M, g)] = best;
  *out = best;
  return cudaSuccess;
}

template <bool kGeneric>
cudaError_t launch_lut(const Problem& pr, uint32_t* status, cudaStream_t stream) {
  const int G = pr.K / pr.g;
  const int row_bytes = G * pr.M;
  const int S = (row_bytes + 127) / 128;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  Plan best;
  e = lut_plan<kGeneric>(dev, pr.N, S, pr.M, pr.g, &best);
  if (e != cudaSuccess) return e;

  // Codes as a 2D byte tensor [N rows][G M bytes]; a box is 64 rows x 128 bytes
  // (one slice of 64 rows).  Out-of-range rows and bytes read as zero.
  EncodeTiledFn encode = encode_tiled();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(pr.N)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
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
  p.N = pr.N;
  p.G = G;
  p.M = pr.M;
  p.g = pr.g;
  p.S = S;
  p.C = best.C;
  p.P = best.P;
  p.RB = best.RB;
  p.RBc = (((p.RB + p.C - 1) / p.C) + 3) & ~3;
  p.ntask = (p.RB + 7) / 8;
  p.ntile = (p.RB + kTileRows - 1) / kTileRows;
  p.R = best.R;
  p.status = status;
  const SmemLayout L = smem_layout(p.C, p.P, p.RBc, p.ntask, p.ntile, p.R, operand_bytes(kGeneric, p.P, p.M, p.g));
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
  if (p.R < p.P * p.ntile) return cudaLaunchKernelEx(&cfg, gemv_lut_kernel<kGeneric, true>, map, p);
  return cudaLaunchKernelEx(&cfg, gemv_lut_kernel<kGeneric, false>, map, p);
}

}  // namespace

// Batch-1 layers with 256-entry codebooks (B = 8), M = 1..4, g = 8 or 16, whose code
// rows are whole 16-byte units (the TMA tensor's row stride) and at most 16 CTAs x 4
// passes x 128 bytes long.
bool gemv_lut_supported(int M, int B, int g, int K, int batch) {
  if (B != 8 || batch != 1 || M < 1 || M > 4 || (g != 8 && g != 16) || K <= 0 || K % g != 0) return false;
  const long long row_bytes = static_cast<long long>(K / g) * M;
  return row_bytes % 16 == 0 && row_bytes <= 16LL * kMaxPasses * 128;
}

cudaError_t launch_gemv_lut(const Problem& pr, uint32_t* status, cudaStream_t stream) {
  if (pr.M == 2 && pr.g == 8) return launch_lut<false>(pr, status, stream);
  return launch_lut<true>(pr, status, stream);
}

}  // namespace aqlm
