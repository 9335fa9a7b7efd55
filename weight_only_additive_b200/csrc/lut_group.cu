// Grouped lookup-table GEMV: one launch computes a set of independent batch-1 layers
// with 256-entry codebooks (a decoder block's linears), the "fast lookup, no per-element
// dequantization" path of the inference-research record "AQLM (additive /
// multi-codebook quantization)", section "Kernels", applied to a whole layer set
// so that no layer pays its own launch, set-up and tail.
//
//   T_m[j][i] = sum_t x[8j + t] * C_m[i][t]                 (group j, codebook m, entry i)
//   part[s][n] = sum_{j in slice s} (T_0[j][codes[n,j,0]] + T_1[j][codes[n,j,1]])
//   y[n]       = s_n * sum_s part[s][n] + bias_n             (second kernel, s ascending)
// (written for 2x8 g8, where a slice of 128 code bytes is 64 groups; for any M, g a
// slice is 128 code bytes and part sums the table entries of its bytes).
//
// Work items.  Item (p, s, t) is layer p's 128-code-byte slice s on its 64-row tile
// t; a layer has ceil(G M / 128) x ceil(N / 64) items.  Items are numbered layer by
// layer, slice-major, and every CTA (one per SM, persistent) takes a contiguous
// range of them, so consecutive items mostly share (p, s) and therefore the
// lookup table: a CTA rebuilds it only when (p, s) changes.  The ranges have equal
// estimated cost (items plus the table builds they start), not equal item counts.
//
// Per CTA:
//   warp 16     TMA producer: streams the code tile (64 rows x 128 bytes) of every
//               item of the range into a ring of shared-memory slots, running as
//               far ahead as the ring allows; codes are read exactly once.
//   warps 0-15  table builders and lookup workers.  On a new (p, s) they wait for
//               the prefetched operands (x slice, both codebooks), issue two
//               tcgen05.mma (M = 128 rows of x groups, N = 256 entries, K = 16 with
//               the upper 8 zero) into TMEM and move the table to shared memory as
//               fp16 pairs (T_0, T_1) per (entry, group).  Then the warps of tile
//               group j take the tiles k = j (mod kTileGroups), kTasks interleaved
//               8-row tasks per warp, and write each row's fp32 partial to the
//               workspace.
// Generic instantiations (any B = 8 scheme) build each slice's table with the stacked
// build of lut_table.cuh (the M codebooks side by side along K, one TMEM lane per code
// byte); launches of 2x8 g8 layers only keep the tuned build described above.
//
// The partials of a row are summed over the slices in ascending order by a second
// small kernel (programmatic dependent launch; one thread per row, its loads issued
// eight slices at a time), which applies the channel scale and bias: the result does
// not depend on which CTA ran which item.
//
// Bank-conflict-free lookups: as in the single-layer lookup-table kernel, lane
// (r8, q4) reads code word 8 q4 + ((r8 + s) mod 8) at step s, and the table keeps
// group 2w in word column w and group 2w + 1 in column 32 + w of each entry's
// 64-word row, so the 32 lanes of every table read hit 32 different banks.
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "aqlm_device.cuh"
#include "lut_table.cuh"

namespace aqlm {
namespace {

#ifndef AQLM_GROUP_WORKER_WARPS
#define AQLM_GROUP_WORKER_WARPS 16
#endif
constexpr int kWorkerWarps = AQLM_GROUP_WORKER_WARPS;  // table builders (the first 16) and lookup workers
constexpr int kWorkers = 32 * kWorkerWarps;
constexpr int kThreads = kWorkers + 32;            // + TMA producer warp
constexpr int kProducerWarp = kWorkers / 32;
constexpr int kTileRows = 64;
constexpr uint32_t kTileBytes = 64u * 128u;        // 64 rows x 64 groups x 2 codes
constexpr uint32_t kLutBytes = lut::kTableBytes;   // 64 KB
constexpr uint32_t kAOpBytes = lut::kAOpBytes;     // 4 KB
constexpr uint32_t kBOpBytes = lut::kBOpBytes;     // 8 KB per codebook
#ifndef AQLM_GROUP_TASKS
#define AQLM_GROUP_TASKS 2
#endif
constexpr int kTasks = AQLM_GROUP_TASKS;           // 8-row tasks per warp and tile (interleaved)
constexpr int kWarpsPerTile = 8 / kTasks;          // a 64-row tile is 8 tasks
constexpr int kTileGroups = kWorkerWarps / kWarpsPerTile;  // warps of group j take tiles k = j (mod kTileGroups)
static_assert(kTasks * kWarpsPerTile == 8 && kTileGroups * kWarpsPerTile == kWorkerWarps && kWorkerWarps >= 16,
              "tile split");
constexpr uint32_t kTmemCols = 512;                // D_0 at [0, 256), D_1 at [256, 512)

constexpr uint32_t kOffLut = 0;
constexpr uint32_t kOffA = kOffLut + kLutBytes;    // 2 A buffers

// Shared-memory layout of an instantiation.  The tuned one (2x8 g8 layers only) has
// A buffers of one K step and B = two codebooks of one K step each (kBSteps = 2); the
// generic ones (stacked build) have A buffers and a B operand of kBSteps K steps,
// enough for layers whose M g is at most 16 kBSteps.  The code-tile ring takes what is
// left: 16 slots (128 KB in flight) for kBSteps = 2, 12 for kBSteps = 4.
template <int kBSteps, bool kGeneric>
struct GroupLayout {
  static constexpr uint32_t kABytes = (kGeneric ? kBSteps : 1) * kAOpBytes;
  static constexpr uint32_t kOffB = kOffA + 2 * kABytes;
  static constexpr uint32_t kOffRing = kOffB + kBSteps * kBOpBytes;   // 1024-aligned
  static constexpr int kSlots = kBSteps <= 2 ? 16 : 12;
  static constexpr uint32_t kOffBars = kOffRing + kSlots * kTileBytes;
  static constexpr uint32_t kSmemBytes = kOffBars + 8u * (2 * kSlots + 1) + 16u;
  static_assert(kOffRing % 1024 == 0, "ring slots must stay 1024-byte aligned");
  static_assert(kSmemBytes + 1024u <= 227u * 1024u, "shared memory budget");
};
using TunedLayout = GroupLayout<2, false>;

struct GroupLayerDev {
  const __half* x;
  const __half* codebooks;
  const __half* scales;
  const __half* bias;
  __half* y;
  float* part;   // [S][N] fp32 partials in the workspace
  int N, G, S, T;  // rows, groups (K / g), 128-code-byte slices, 64-row tiles
  int M, g;        // codebooks per group, group width
  long long item0; // first item of this layer
  long long row0;  // first output row of this layer in the reduction grid
};

// CTAs of one launch: one per SM (the host clamps the grid to this).
constexpr int kMaxGroupCtas = 160;

struct GroupParams {
  GroupLayerDev layer[kMaxGroupLayers];
  int count;
  long long items;
  long long rows;
  uint32_t* status;
  // CTA c takes items [cta_item0[c], cta_item0[c + 1]): contiguous ranges of equal
  // estimated cost (items plus the table builds they start, see build_group_launch)
  long long cta_item0[kMaxGroupCtas + 1];
};

struct GroupMaps {
  CUtensorMap map[kMaxGroupLayers];
};

// Named barrier over the worker warps that also ANDs a flag across them.
__device__ __forceinline__ bool workers_sync_and(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(v ? 1u : 0u), "n"(kWorkers)
      : "memory");
  return out != 0;
}

// Bounded wait that gives up at once when another role has aborted.
__device__ __forceinline__ bool group_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                           uint32_t* status, uint32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitTimeoutNs) {
      record_failure(status, site);
      *abort_flag = 1u;
      return false;
    }
  }
  return true;
}

// Layer of a global item index (layers are few; a linear scan is cheapest).
__device__ __forceinline__ int layer_of(const GroupParams& p, long long item) {
  int l = 0;
  while (l + 1 < p.count && p.layer[l + 1].item0 <= item) ++l;
  return l;
}

// Position of an item as (layer, slice, tile); advanced one item at a time so the
// loops need no division (items are numbered layer by layer, slice-major).
struct ItemCursor {
  int l, s, t;
  __device__ __forceinline__ void seek(const GroupParams& p, long long item) {
    l = layer_of(p, item);
    const long long local = item - p.layer[l].item0;
    s = static_cast<int>(local / p.layer[l].T);
    t = static_cast<int>(local - static_cast<long long>(s) * p.layer[l].T);
  }
  __device__ __forceinline__ void next(const GroupParams& p) {
    if (++t == p.layer[l].T) {
      t = 0;
      if (++s == p.layer[l].S) {
        s = 0;
        ++l;
      }
    }
  }
};

using lut::kmajor_offset;
using lut::kmajor_desc;

// Table operands of the tuned instantiation (cp.async, caller commits): A row rho holds
// x group 2 (rho mod 32) + (rho / 32 mod 2) of slice s (rows 64-127 repeat rows 0-63),
// zero past the layer's last group, so that every TMEM lane quadrant holds the groups
// its conversion warps pack; B holds the two codebooks.  The upper K halves are zeroed
// once at start-up and the loaders write only the lower halves.
__device__ __forceinline__ void load_x_slice_tuned(const GroupLayerDev& L, int s, uint32_t sbase, int buf, int wtid) {
  const uint32_t ao = kOffA + static_cast<uint32_t>(buf) * TunedLayout::kABytes;
  for (int rho = wtid; rho < 128; rho += kWorkers) {
    const int gg = s * 64 + 2 * (rho & 31) + ((rho >> 5) & 1);
    const bool valid = gg < L.G;
    cp_async_16_zfill(sbase + ao + kmajor_offset(rho, 0),
                      valid ? static_cast<const void*>(L.x + static_cast<size_t>(gg) * 8) : static_cast<const void*>(L.x),
                      valid ? 16u : 0u);
  }
}
__device__ __forceinline__ void load_codebooks_tuned(const GroupLayerDev& L, uint32_t sbase, int wtid) {
  for (int e = wtid; e < 512; e += kWorkers)  // codebook m = e / 256, entry e % 256
    cp_async_16_zfill(sbase + TunedLayout::kOffB + static_cast<uint32_t>(e >> 8) * kBOpBytes + kmajor_offset(e & 255, 0),
                      L.codebooks + static_cast<size_t>(e) * 8, 16u);
}
// Generic instantiations: the stacked build's operands (A buffer buf of slice s; B, one
// buffer, reloaded only when the layer changes).
template <int kBSteps>
__device__ __forceinline__ void load_x_slice_stacked(const GroupLayerDev& L, int s, uint32_t sbase, int buf, int wtid) {
  using LY = GroupLayout<kBSteps, true>;
  lut::load_x_stacked<kWorkers>(L.x, L.G, L.M, L.g, s, sbase + kOffA + static_cast<uint32_t>(buf) * LY::kABytes, wtid);
}
template <int kBSteps>
__device__ __forceinline__ void load_codebooks_stacked(const GroupLayerDev& L, uint32_t sbase, int wtid) {
  lut::load_codebooks_stacked<kWorkers>(L.codebooks, L.M, L.g, sbase + GroupLayout<kBSteps, true>::kOffB, wtid);
}

// kGeneric = false: every layer of the launch is 2x8 g8 (the tuned code);
// kGeneric = true: any B = 8 scheme with M g <= 16 kBSteps (the stacked build).
template <int kBSteps, bool kGeneric>
__global__ void __launch_bounds__(kThreads, 1) lut_group_kernel(const __grid_constant__ GroupMaps maps,
                                                                const __grid_constant__ GroupParams p) {
  static_assert(kGeneric || kBSteps == 2, "the tuned instantiation holds two one-step codebooks");
  using LY = GroupLayout<kBSteps, kGeneric>;
  constexpr int kSlots = LY::kSlots;
  constexpr uint32_t kOffRing = LY::kOffRing, kOffBars = LY::kOffBars;
  extern __shared__ uint8_t smem_raw[];
  // the ring slots are TMA destinations: keep the layout 1024-byte aligned
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBars);  // tile landed
  uint64_t* empty = full + kSlots;                                  // tile read by its 8 warps
  uint64_t* mma_bar = empty + kSlots;                               // table MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_bar + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const long long it0 = p.cta_item0[blockIdx.x];
  const long long it1 = p.cta_item0[blockIdx.x + 1];

  // The next kernel in the stream (the reduction) may be scheduled now; it waits
  // for this grid to complete before it reads the partials.
  grid_dependents_launch();
  if (tid == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kWarpsPerTile);
    }
    mbar_init(mma_bar, 1);
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if constexpr (!kGeneric) {
    // zero upper K halves of the operand buffers (never written again)
    for (int i = tid; i < 2 * 128 + 512; i += kThreads) {
      const uint32_t off = i < 256 ? kOffA + static_cast<uint32_t>(i >> 7) * LY::kABytes + kmajor_offset(i & 127, 1)
                                   : LY::kOffB + static_cast<uint32_t>((i - 256) >> 8) * kBOpBytes +
                                         kmajor_offset((i - 256) & 255, 1);
      *reinterpret_cast<uint4*>(smem + off) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    // ---- code tiles of every item of the range (weights: no dependency wait) ----
    // Tile k of the range goes to slot k mod kSlots and is read by warp group
    // k mod kTileGroups, so each group owns every kTileGroups-th slot.  Producer lane j
    // streams group j's tiles in order, waiting only for that group's slots: a group
    // that falls behind holds back its own loads, not every group's.
    static_assert(kSlots % kTileGroups == 0 && kTileGroups <= 32, "slots per warp group");
    if (lane < kTileGroups) {
      const uint64_t pol = l2_policy_evict_first();
      ItemCursor c;
      c.seek(p, it0 + lane);
      for (long long k = lane; it0 + k < it1; k += kTileGroups) {
        const int slot = static_cast<int>(k % kSlots);
        const uint32_t use = static_cast<uint32_t>(k / kSlots);
        if (use > 0 && !group_wait(&empty[slot], (use - 1u) & 1u, abort_flag, p.status, kSiteGroupRing)) break;
        mbar_arrive_expect_tx(&full[slot], kTileBytes);
        // bytes past the row end and rows past N are zero-filled
        tma_load_2d(sbase + kOffRing + static_cast<uint32_t>(slot) * kTileBytes, &maps.map[c.l], c.s * 128,
                    c.t * kTileRows, &full[slot], pol);
        if (it0 + k + kTileGroups < it1)
          for (int i = 0; i < kTileGroups; ++i) c.next(p);
      }
    }
  } else {
    // ---- workers ------------------------------------------------------------------------
    // x is read (table operands) and the workspace written only after the previous
    // kernel in the stream has completed.
    grid_dependency_wait();
    const int wtid = tid;
    const int wg = warp / kWarpsPerTile;    // tiles k = wg (mod kTileGroups) are this warp's
    const int task = warp % kWarpsPerTile;  // its tasks of such a tile: task + kWarpsPerTile * u
    const int r8 = lane >> 2;    // row of the task
    const int q4 = lane & 3;     // quarter of the row's 32 code words
    const uint32_t idesc = umma_idesc_f16_f32(128, 256);
    // byte offset (4 x word column) of the code word lane (r8, q4) reads at step s8
    uint32_t wv[8];
#pragma unroll
    for (int s8 = 0; s8 < 8; ++s8) wv[s8] = static_cast<uint32_t>((8 * q4 + ((r8 + s8) & 7)) << 2);
    uint32_t mma_phase = 0;
    bool ok = true;
    if (it0 < it1) {
      const int l = layer_of(p, it0);
      const int s0 = static_cast<int>((it0 - p.layer[l].item0) / p.layer[l].T);
      if constexpr (kGeneric) {
        load_codebooks_stacked<kBSteps>(p.layer[l], sbase, wtid);
        load_x_slice_stacked<kBSteps>(p.layer[l], s0, sbase, 0, wtid);
      } else {
        load_codebooks_tuned(p.layer[l], sbase, wtid);
        load_x_slice_tuned(p.layer[l], s0, sbase, 0, wtid);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");

    // Items come in runs of equal (layer, slice): the table is rebuilt at the start of
    // every run, then each warp visits only its own tiles of the run (item index
    // k = wg mod kTileGroups), so no warp walks the items of other warps.
    ItemCursor c;
    c.seek(p, it0);
    const int nitems = static_cast<int>(it1 - it0);  // < 2^31 items per CTA
    int run = 0;
    for (int kbase = 0; kbase < nitems;) {
      const int l = c.l, s = c.s, t0 = c.t;
      const GroupLayerDev& L = p.layer[l];
      const int run_len = (nitems - kbase < L.T - t0) ? nitems - kbase : L.T - t0;
      {
        // ---- new (layer, slice): table from the prefetched operands in buffer run & 1 ----
        const int buf = run & 1;
        asm volatile("cp.async.wait_all;" ::: "memory");
        fence_proxy_async_smem();
        tc_fence_before_sync();
        ok = workers_sync_and(ok);  // old table no longer read; operands in place
        tc_fence_after_sync();
        if constexpr (!kGeneric) {
          if (ok && wtid == 0) {
            const uint64_t adesc = kmajor_desc(sbase + kOffA + static_cast<uint32_t>(buf) * LY::kABytes);
            const uint32_t bo = sbase + LY::kOffB;
            umma_f16_ss(tmem, adesc, kmajor_desc(bo), idesc, 0u);
            umma_f16_ss(tmem + 256u, adesc, kmajor_desc(bo + kBOpBytes), idesc, 0u);
            umma_commit(mma_bar);
          }
          // prefetch the x slice of the range's next (layer, slice) into the other A
          // buffer, whose MMAs completed before the previous table was stored
          const bool more = kbase + run_len < nitems;
          const int nl = (s + 1 < L.S) ? l : l + 1;
          if (ok && more) load_x_slice_tuned(p.layer[nl], (s + 1 < L.S) ? s + 1 : 0, sbase, buf ^ 1, wtid);
          const bool done = ok && group_wait(mma_bar, mma_phase, abort_flag, p.status, kSiteGroupMma);
          mma_phase ^= 1u;
          // the MMAs have read B: a new layer's codebooks may replace it now
          if (done && more && nl != l) load_codebooks_tuned(p.layer[nl], sbase, wtid);
          asm volatile("cp.async.commit_group;" ::: "memory");
          ok = workers_sync_and(done);
          tc_fence_after_sync();
          if (ok && warp < 16) lut::store_table_2x8(tmem, warp, lane, smem + kOffLut);
          tc_fence_before_sync();
          ok = workers_sync_and(ok);  // table complete
        } else {
          // the stacked build: one MMA chain gives the whole slice's table, one TMEM
          // lane per code byte
          if (ok && wtid == 0) {
            lut::mma_stacked(tmem, sbase + kOffA + static_cast<uint32_t>(buf) * LY::kABytes, sbase + LY::kOffB,
                             lut::stacked_ksteps(L.M, L.g), idesc);
            umma_commit(mma_bar);
          }
          // prefetch the x slice of the range's next (layer, slice) into the other A
          // buffer, whose MMAs completed before the previous table was stored
          const bool more = kbase + run_len < nitems;
          const int nl = (s + 1 < L.S) ? l : l + 1;
          if (ok && more) load_x_slice_stacked<kBSteps>(p.layer[nl], (s + 1 < L.S) ? s + 1 : 0, sbase, buf ^ 1, wtid);
          const bool done = ok && group_wait(mma_bar, mma_phase, abort_flag, p.status, kSiteGroupMma);
          mma_phase ^= 1u;
          // the MMAs have read B: a new layer's codebooks may replace it now
          if (done && more && nl != l) load_codebooks_stacked<kBSteps>(p.layer[nl], sbase, wtid);
          asm volatile("cp.async.commit_group;" ::: "memory");
          ok = workers_sync_and(done);
          tc_fence_after_sync();
          if (ok && warp < 16) lut::store_table_stacked(tmem, warp, lane, smem + kOffLut);
          tc_fence_before_sync();
          ok = workers_sync_and(ok);  // table complete
        }
        ++run;
      }
      for (int i = ((wg - kbase) % kTileGroups + kTileGroups) % kTileGroups; i < run_len; i += kTileGroups) {
        const int k = kbase + i;
        const int my_slot = k % kSlots;
        const uint32_t my_ph = static_cast<uint32_t>((k / kSlots) & 1);
        const int t = t0 + i;
        // ---- lookups of this item's tile: rows 8 (task + kWarpsPerTile u) + r8 ----
        const bool landed =
            __all_sync(0xffffffffu, ok && group_wait(&full[my_slot], my_ph, abort_flag, p.status, kSiteGroupRing));
        if (landed) {
          const uint32_t* row0 = reinterpret_cast<const uint32_t*>(
              smem + kOffRing + static_cast<uint32_t>(my_slot) * kTileBytes + static_cast<uint32_t>(task * 8 + r8) * 128u);
          uint32_t cw[kTasks][8];
#pragma unroll
          for (int u = 0; u < kTasks; ++u)
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) cw[u][s8] = row0[u * kWarpsPerTile * 8 * 32 + (wv[s8] >> 2)];
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[my_slot]);  // the tile's codes are in registers
          // fp32 accumulators: even code bytes (the low halves of their words) into
          // acc0, odd code bytes (high halves) into acc1
          float acc0[kTasks], acc1[kTasks];
#pragma unroll
          for (int u = 0; u < kTasks; ++u) acc0[u] = acc1[u] = 0.f;
          const uint8_t* lut = smem + kOffLut;
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8) {
#pragma unroll
            for (int u = 0; u < kTasks; ++u) {
              // table byte offsets: entry * 256 + column * 4 (column w, or 32 + w at +128);
              // a byte's value is half (byte mod 2) of the word its pair reads
              const uint32_t a0 = *reinterpret_cast<const uint32_t*>(lut + __byte_perm(cw[u][s8], wv[s8], 0x5504));
              const uint32_t a1 = *reinterpret_cast<const uint32_t*>(lut + __byte_perm(cw[u][s8], wv[s8], 0x5514));
              const uint32_t a2 =
                  *reinterpret_cast<const uint32_t*>(lut + __byte_perm(cw[u][s8], wv[s8], 0x5524) + 128u);
              const uint32_t a3 =
                  *reinterpret_cast<const uint32_t*>(lut + __byte_perm(cw[u][s8], wv[s8], 0x5534) + 128u);
              acc0[u] = add_f32_lo_f16(a0, acc0[u]);
              acc1[u] = add_f32_hi_f16(a1, acc1[u]);
              acc0[u] = add_f32_lo_f16(a2, acc0[u]);
              acc1[u] = add_f32_hi_f16(a3, acc1[u]);
            }
          }
          float v[kTasks];
#pragma unroll
          for (int u = 0; u < kTasks; ++u) v[u] = acc0[u] + acc1[u];
#pragma unroll
          for (int u = 0; u < kTasks; ++u) v[u] += __shfl_xor_sync(0xffffffffu, v[u], 1);
#pragma unroll
          for (int u = 0; u < kTasks; ++u) v[u] += __shfl_xor_sync(0xffffffffu, v[u], 2);
          if (q4 == 0) {
            float* dst = L.part + static_cast<size_t>(s) * L.N;
#pragma unroll
            for (int u = 0; u < kTasks; ++u) {
              const int row = t * kTileRows + (task + kWarpsPerTile * u) * 8 + r8;
              if (row < L.N) dst[row] = v[u];
            }
          }
        } else {
          ok = false;
          if (lane == 0) mbar_arrive(&empty[my_slot]);
        }
      }
      kbase += run_len;
      c.t = 0;  // the next run starts the next slice (or the next layer's first)
      if (++c.s == L.S) {
        c.s = 0;
        ++c.l;
      }
    }
  }

  if (*abort_flag) {
    // a wait gave up: let copies already in flight land before the CTA leaves
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 50000ull) {
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// y[n] = fp16(s_n * sum_s part[s][n] + bias_n).  A block takes kReduceRows consecutive
// rows of the launch's concatenated row space; thread t owns rows t, t + kReduceThreads,
// ... of it (consecutive threads read consecutive rows of a slice: coalesced), issues
// its loads eight slices at a time for all its rows and adds every row's slices in
// ascending order.  The order is fixed, so the result does not depend on
// timing or on which CTA produced which partial.
#ifndef AQLM_REDUCE_THREADS
#define AQLM_REDUCE_THREADS 128
#endif
#ifndef AQLM_REDUCE_ROWS_PER_THREAD
#define AQLM_REDUCE_ROWS_PER_THREAD 1
#endif
constexpr int kReduceThreads = AQLM_REDUCE_THREADS;
constexpr int kReduceRowsPerThread = AQLM_REDUCE_ROWS_PER_THREAD;
constexpr int kReduceRows = kReduceThreads * kReduceRowsPerThread;
// At most 48 registers a thread: a block then fits beside a partial-sum CTA (17 warps
// of 96 registers), so the reduction's blocks are resident and waiting when that grid
// completes, and the next call's CTAs are not held back by them.
constexpr int kReduceMinBlocks = 65536 / (kReduceThreads * 48);
__global__ void __launch_bounds__(kReduceThreads, kReduceMinBlocks) lut_group_reduce_kernel(
    const __grid_constant__ GroupParams p) {
  grid_dependents_launch();
  const float* col[kReduceRowsPerThread];
  int S[kReduceRowsPerThread], N[kReduceRowsPerThread], lay[kReduceRowsPerThread], nn[kReduceRowsPerThread];
  int smax = 0;
  int l = 0;
#pragma unroll
  for (int k = 0; k < kReduceRowsPerThread; ++k) {
    const long long row = static_cast<long long>(blockIdx.x) * kReduceRows + k * kReduceThreads + threadIdx.x;
    while (l + 1 < p.count && p.layer[l + 1].row0 <= row) ++l;
    const GroupLayerDev& L = p.layer[l];
    const bool valid = row < p.rows;
    lay[k] = l;
    nn[k] = static_cast<int>(row - L.row0);
    N[k] = L.N;
    S[k] = valid ? L.S : 0;
    col[k] = L.part + (valid ? nn[k] : 0);
    smax = max(smax, S[k]);
  }
  // the partials are the previous kernel's output
  grid_dependency_wait();
  float acc[kReduceRowsPerThread];
#pragma unroll
  for (int k = 0; k < kReduceRowsPerThread; ++k) acc[k] = 0.f;
  for (int s0 = 0; s0 < smax; s0 += 8) {
    float v[kReduceRowsPerThread][8];
#pragma unroll
    for (int k = 0; k < kReduceRowsPerThread; ++k)
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[k][u] = s0 + u < S[k] ? col[k][static_cast<size_t>(s0 + u) * N[k]] : 0.f;
#pragma unroll
    for (int k = 0; k < kReduceRowsPerThread; ++k)
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[k] += v[k][u];
  }
#pragma unroll
  for (int k = 0; k < kReduceRowsPerThread; ++k) {
    if (S[k] == 0) continue;
    const GroupLayerDev& L = p.layer[lay[k]];
    const int n = nn[k];
    const float bi = L.bias ? __half2float(L.bias[n]) : 0.f;
    L.y[n] = __float2half_rn(acc[k] * __half2float(L.scales[n]) + bi);
  }
}

}  // namespace
}  // namespace aqlm

namespace aqlm {

// Batch-1 layers with 256-entry codebooks (B = 8), M = 1..4, g = 8 or 16, whose code
// rows are whole 16-byte units (the TMA tensor's row stride).
bool lut_group_supported(const Problem& p) {
  if (p.B != 8 || p.batch != 1 || p.M < 1 || p.M > 4 || (p.g != 8 && p.g != 16) || p.K % p.g != 0) return false;
  const long long row_bytes = static_cast<long long>(p.K / p.g) * p.M;
  return row_bytes % 16 == 0;
}

namespace {
// One fp32 partial per row and 128-code-byte slice.
inline size_t part_bytes(const Problem& p) {
  const size_t row_bytes = static_cast<size_t>(p.K / p.g) * p.M;
  const size_t slices = (row_bytes + 127) / 128;
  return (slices * static_cast<size_t>(p.N) * sizeof(float) + 255u) & ~static_cast<size_t>(255u);
}
}  // namespace

size_t lut_group_workspace_bytes(const Problem* probs, int count) {
  size_t bytes = 0;
  for (int i = 0; i < count; ++i)
    if (lut_group_supported(probs[i])) bytes += part_bytes(probs[i]);
  return bytes;
}

namespace {

// Everything a launch pair needs besides the stream: built once per distinct call
// (problem list, workspace, status word, device) and kept in a small cache, so a
// call repeated every token (the usual case: the same layer set with new x and y
// contents) skips the tensor-map encoding and the per-layer bookkeeping.
struct GroupLaunch {
  GroupParams p;
  GroupMaps maps;
  unsigned grid = 0, rgrid = 0;
  int max_ksteps = 0;     // the most stacked-build K steps of a layer: selects the instantiation
  bool generic = false;   // some layer is not 2x8 g8
};

struct GroupKey {
  int dev = -1, count = 0;
  const void* workspace = nullptr;
  const uint32_t* status = nullptr;
  Problem probs[kMaxGroupLayers];
};

bool same_problem(const Problem& a, const Problem& b) {
  return a.x == b.x && a.codes == b.codes && a.codebooks == b.codebooks && a.scales == b.scales &&
         a.bias == b.bias && a.y == b.y && a.M == b.M && a.B == b.B && a.g == b.g && a.K == b.K && a.N == b.N &&
         a.batch == b.batch;
}

bool same_key(const GroupKey& k, int dev, const Problem* probs, int count, const void* ws, const uint32_t* status) {
  if (k.dev != dev || k.count != count || k.workspace != ws || k.status != status) return false;
  for (int i = 0; i < count; ++i)
    if (!same_problem(k.probs[i], probs[i])) return false;
  return true;
}

constexpr int kLaunchCacheEntries = 8;
constexpr int kMaxDevices = 64;
std::mutex g_launch_mu;
GroupKey g_launch_key[kLaunchCacheEntries];
GroupLaunch g_launch_val[kLaunchCacheEntries];
int g_launch_next = 0;
int g_sms[kMaxDevices] = {};  // 0 = not queried yet (also means "attribute not set")
uint64_t g_attr_ctx[kMaxDevices] = {};  // context the kernels' attributes were set in

// Tensor maps and parameters of one launch pair (host work only, no CUDA calls but
// the driver's tensor-map encoder).
cudaError_t build_group_launch(const Problem* probs, int count, void* workspace, uint32_t* status, int sms,
                               GroupLaunch* out) {
  EncodeTiledFn encode = encode_tiled();
  if (!encode) return cudaErrorNotSupported;
  GroupParams& p = out->p;
  GroupMaps& maps = out->maps;
  p = GroupParams{};
  maps = GroupMaps{};
  out->max_ksteps = 0;
  out->generic = false;
  long long items = 0, rows = 0;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  for (int i = 0; i < count; ++i) {
    const Problem& pr = probs[i];
    if (!lut_group_supported(pr)) return cudaErrorInvalidValue;
    GroupLayerDev& L = p.layer[i];
    L.x = static_cast<const __half*>(pr.x);
    L.codebooks = static_cast<const __half*>(pr.codebooks);
    L.scales = static_cast<const __half*>(pr.scales);
    L.bias = static_cast<const __half*>(pr.bias);
    L.y = static_cast<__half*>(pr.y);
    L.part = reinterpret_cast<float*>(ws);
    ws += part_bytes(pr);
    L.N = pr.N;
    L.M = pr.M;
    L.g = pr.g;
    L.G = pr.K / pr.g;
    const int row_bytes = L.G * pr.M;
    L.S = (row_bytes + 127) / 128;
    L.T = (pr.N + kTileRows - 1) / kTileRows;
    out->max_ksteps = std::max(out->max_ksteps, lut::stacked_ksteps(pr.M, pr.g));
    if (pr.M != 2 || pr.g != 8) out->generic = true;
    L.item0 = items;
    L.row0 = rows;
    items += static_cast<long long>(L.S) * L.T;
    rows += pr.N;
    // codes as a 2D byte tensor [N rows][G M bytes]; a box is 64 rows x 128 bytes
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(pr.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
    const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(kTileRows)};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&maps.map[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(pr.codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  p.count = count;
  p.items = items;
  p.rows = rows;
  p.status = status;
  const int grid = static_cast<int>(std::min<long long>(std::min(items, static_cast<long long>(sms)), kMaxGroupCtas));
  out->grid = static_cast<unsigned>(grid);
  // Contiguous item ranges of equal estimated cost: an item (one 64-row code tile)
  // costs 1, and every run of equal (layer, slice) costs kTableCost more for its
  // lookup-table build (a build stalls a CTA's lookups for a few tile times; 3 timed
  // best on B200 among 3, 5 and 8).  Layers with few rows have short runs, so a CTA
  // whose range falls on them takes fewer items.
#ifndef AQLM_GROUP_TABLE_COST
#define AQLM_GROUP_TABLE_COST 3
#endif
  constexpr long long kTableCost = AQLM_GROUP_TABLE_COST;
  long long total = 0;
  for (int i = 0; i < count; ++i) total += static_cast<long long>(p.layer[i].S) * (p.layer[i].T + kTableCost);
  p.cta_item0[0] = 0;
  int next = 1;
  long long cost = 0;  // cost of the items before the current run
  for (int i = 0; i < count && next < grid; ++i) {
    const GroupLayerDev& L = p.layer[i];
    for (int sl = 0; sl < L.S && next < grid; ++sl) {
      const long long run0 = L.item0 + static_cast<long long>(sl) * L.T;
      const long long run_cost = L.T + kTableCost;
      // boundaries whose target cost falls inside this run: target = next * total / grid
      while (next < grid && static_cast<long long>(next) * total < (cost + run_cost) * grid) {
        const long long target = (static_cast<long long>(next) * total + grid - 1) / grid;  // ceil
        long long off = target - cost - kTableCost;  // items of the run before the boundary
        off = std::max(0LL, std::min(off, static_cast<long long>(L.T)));
        p.cta_item0[next] = std::max(p.cta_item0[next - 1], run0 + off);
        ++next;
      }
      cost += run_cost;
    }
  }
  for (; next <= grid; ++next) p.cta_item0[next] = items;
  out->rgrid = static_cast<unsigned>((rows + kReduceRows - 1) / kReduceRows);
  return cudaSuccess;
}

}  // namespace

// All problems must satisfy lut_group_supported; count <= kMaxGroupLayers; the
// workspace holds lut_group_workspace_bytes(probs, count) bytes, 256-byte aligned.
cudaError_t launch_lut_group(const Problem* probs, int count, void* workspace, uint32_t* status,
                             cudaStream_t stream) {
  if (count <= 0 || count > kMaxGroupLayers) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  GroupLaunch launch;
  {
    std::lock_guard<std::mutex> lock(g_launch_mu);
    const uint64_t ctx = current_context_id();
    if (g_sms[dev] == 0 || ctx == 0 || g_attr_ctx[dev] != ctx) {
      // once per device and context: the SM count and the kernels' shared-memory limits
      int sms = 0;
      e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(lut_group_kernel<2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(GroupLayout<2, false>::kSmemBytes + 1024u));
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(lut_group_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(GroupLayout<2, true>::kSmemBytes + 1024u));
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(lut_group_kernel<4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(GroupLayout<4, true>::kSmemBytes + 1024u));
      if (e != cudaSuccess) return e;
      g_sms[dev] = std::max(1, sms);
      g_attr_ctx[dev] = ctx;
    }
    int hit = -1;
    for (int c = 0; c < kLaunchCacheEntries && hit < 0; ++c)
      if (same_key(g_launch_key[c], dev, probs, count, workspace, status)) hit = c;
    if (hit < 0) {
      hit = g_launch_next;
      g_launch_next = (g_launch_next + 1) % kLaunchCacheEntries;
      g_launch_key[hit].dev = -1;  // invalid until built
      e = build_group_launch(probs, count, workspace, status, g_sms[dev], &g_launch_val[hit]);
      if (e != cudaSuccess) return e;
      GroupKey& k = g_launch_key[hit];
      k.dev = dev;
      k.count = count;
      k.workspace = workspace;
      k.status = status;
      for (int i = 0; i < count; ++i) k.probs[i] = probs[i];
    }
    launch = g_launch_val[hit];
  }

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const bool wide = launch.max_ksteps > 2;  // M g above 32: the kBSteps = 4 layout
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(launch.grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (wide ? GroupLayout<4, true>::kSmemBytes
                               : launch.generic ? GroupLayout<2, true>::kSmemBytes
                                                : GroupLayout<2, false>::kSmemBytes) +
                         1024u;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (wide)
    e = cudaLaunchKernelEx(&cfg, lut_group_kernel<4, true>, launch.maps, launch.p);
  else if (launch.generic)
    e = cudaLaunchKernelEx(&cfg, lut_group_kernel<2, true>, launch.maps, launch.p);
  else
    e = cudaLaunchKernelEx(&cfg, lut_group_kernel<2, false>, launch.maps, launch.p);
  if (e != cudaSuccess) return e;

  cudaLaunchConfig_t rcfg = {};
  rcfg.gridDim = dim3(launch.rgrid, 1, 1);
  rcfg.blockDim = dim3(kReduceThreads, 1, 1);
  rcfg.stream = stream;
  rcfg.attrs = attr;
  rcfg.numAttrs = 1;
  return cudaLaunchKernelEx(&rcfg, lut_group_reduce_kernel, launch.p);
}

}  // namespace aqlm
