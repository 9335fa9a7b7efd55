// Pipelined decode -> tensor-core path (every batch size when K % 64 == 0): codeword
// decode into shared memory overlapped with 5th-generation tensor-core MMAs
// (tcgen05.mma kind::f16, fp32 accumulator in TMEM).
//
// "Dequantize-to-FP16 then an FP16 tensor-core GEMM" (inference-research record
// "AQLM (additive / multi-codebook quantization)", notes), fused so the fp16
// weights exist only as 128 x 64 shared-memory tiles.  Swap-AB: the MMA's M is
// 128 weight rows, its N is the batch tile (16..256), so D[n, b] lands in TMEM
// with one weight row per lane.  Because the weight tile is decoded once for the
// whole batch tile, the same kernel also serves token generation (batch 1..8):
// its decoders gather codewords faster than the GEMV's lanes do.
//
// Warp roles (352 threads with one decoder group; a second group of 8 decoder warps
// takes every other stage in the 608-thread kernels):
//   warps 0-7  decoders, then epilogue.  Threads r and r + 128 own weight row
//              n0 + r (16-byte chunks 0-3 and 4-7 of each 64-wide K stage).  Per
//              stage a thread reads its codes from the code tile and writes its
//              64 bytes of the A stage in the 128-byte-swizzled K-major layout:
//                1x16: the codeword is the fp16 data, so each 16-byte piece is one
//                      cp.async gather from the (L2-resident) codebook straight into
//                      its swizzled slot, tracked by cp.async.mbarrier.arrive;
//                2x8:  the two codewords come from the codebooks staged in shared
//                      memory, are added as half2 and stored.
//   warp 8     TMA producer of x tiles (B operand, 128-byte swizzle, zero-filled
//              past the batch and K edges).
//   warp 9     MMA issuer: 4 x (128 x BN x 16) per stage, commit releases the stage.
//   warp 10    TMA producer of code tiles (128 rows x 64 bytes = 4 or 8 stages).
// Split K: SK CTAs of a (1, 1, SK) cluster take consecutive K ranges of the same
// weight rows and exchange fp32 partials through distributed shared memory.
// Epilogue: tcgen05.ld of 16 columns at a time, y = s_n * D + bias_n -> fp16.
// Stream-K (a separate instantiation, kStreamK): one CTA per SM over the (row tile,
// batch tile, K stage) space, two TMEM accumulators, and four more warps that finish
// each tile piece from fp32 partials in a caller workspace (see the epilogue).
#include <cuda.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>

#include "aqlm_device.cuh"

namespace aqlm {
namespace {

constexpr int kRows = 128;            // MMA M: weight rows per CTA
constexpr int kStageK = 64;           // K per stage (one 128-byte swizzle row of fp16)
constexpr int kGroupThreads = 256;    // a decoder group: 8 warps, two threads per weight row of a stage
constexpr int kMaxDecoderGroups = 2;

// Decoder groups per CTA.  With two, group g decodes the stages i = g mod 2 of the
// CTA's range, so two stages are decoded at once (latency hiding: measured 1.1-1.2x
// on the B = 8 layer kernels and 1.55x on the input gradient at large batch).  The
// codeword-gather decoders of the B = 16 layer kernels already keep L1TEX busy with
// one group (a second made them 2-7 % slower), and 4x8 g8 ran faster with one.
// Block: the decoder warps, then the x producer, the MMA issuer and the code producer.
// Stream-K kernels (kStreamK) add four epilogue warps, one per TMEM lane quadrant.
template <int M, int B, int G, bool kGrad, bool kStreamK = false>
struct PipeShape {
  static constexpr int kGroups = (!kGrad && (B == 16 || (M == 4 && G == 8))) ? 1 : kMaxDecoderGroups;
  static constexpr int kDecoders = kGroups * kGroupThreads;
  static constexpr int kThreads = kDecoders + 96 + (kStreamK ? 128 : 0);
};
constexpr uint32_t kABytes = kRows * 128u;   // 16 KB per A stage (in shared memory)
// A stages kept in tensor memory: the accumulator takes columns [0, 256) of a 512-column
// allocation and A stage s columns [kATmemCol + 32 s, + 32) (128 rows x 64 fp16).
constexpr uint32_t kATmemCol = 256;
constexpr int kMaxATmemStages = 8;
constexpr int kCodeSlots = 4;          // code-tile slots at most (the plan may use 2: PipeParams::cs_log)
constexpr uint32_t kSmemLimit = 227u * 1024u;

struct PipeParams {
  const __half* codebooks;
  const __half* scales;
  const __half* bias;
  __half* y;       // [batch, rows]
  int K, N, batch;
  int rows;        // output rows = the MMA's M extent: N (layer) or K (input gradient)
  int BN;          // batch tile (multiple of 16, <= 256)
  int nk;          // K / 64 stages (whole K)
  int S;           // A/B stage ring depth
  int SK;          // CTAs splitting K (cluster size along z): 1..16
  int ks_per;      // K stages per split (the last split may have fewer)
  int red_rows;    // split-K reduction: weight rows each CTA of the cluster owns
  uint32_t tmem_cols;
  int cb32;        // codebooks 32-byte aligned: g = 16 codewords in one 256-bit load
  int cb_sh;       // 2x8 g8 codebook copies in shared memory: 8 >> cb_sh of them (cb_layout_offset)
  int cs_log;      // code-tile ring of 1 << cs_log slots (2 or 4)
  uint32_t* status;
  // Stream-K schedule (kStreamK kernels).  The work is the tiles x nk stages of
  // (row tile, batch tile, K stage), tile t being row tile t / batch_tiles and batch
  // tile t mod batch_tiles, cut into sk_units units of sk_unit stages; CTA c takes
  // units [c U / C, (c + 1) U / C) with C = sk_ctas (SkRange).  A tile cut between
  // CTAs is finished by whichever of its pieces ends last (see the epilogue).
  int sk_ctas, sk_units, sk_unit, batch_tiles;
  int acc_cols;         // TMEM columns of one accumulator (two, alternating by piece)
  float* sk_part;       // 2 sk_ctas slots of 128 x BN fp32 partials ([4][BN / 4][32][4])
  // per (CTA holding a cut tile's first piece, lane quadrant): pieces stored so far;
  // zero between launches.  A CTA's range holds the first piece of at most one cut
  // tile (only the last tile it reaches can continue past it), so the counters have
  // a fixed size whatever the shape, and callers can share one workspace between shapes.
  uint32_t* sk_count;
};

// Stream-K partition of a CTA range, in stages.
struct SkRange {
  int C, U, unit;
  __host__ __device__ int begin(int c) const {
    return static_cast<int>(static_cast<long long>(c) * U / C) * unit;
  }
  // the CTA whose range holds stage w: the largest c with begin(c) <= w
  __host__ __device__ int cta_of(int w) const {
    return static_cast<int>(((static_cast<long long>(w / unit) + 1) * C - 1) / U);
  }
};

// Per-scheme constants.  A stage is 64 weights of a row: kStageCodeBytes of codes.
// Code tiles are TMA boxes of 128 rows x kTileRowBytes (64 bytes when stages tile 64
// bytes, loaded with the 64-byte swizzle; 48 bytes for M = 3, unswizzled).  B = 8
// codebooks live in shared memory; B = 16 codebooks (1-2 MiB) are gathered from L2.
constexpr int gcd_int(int a, int b) { return b == 0 ? a : gcd_int(b, a % b); }
template <int M, int B, int G>
struct PipeScheme {
  static constexpr int kCodeBytes = B <= 8 ? 1 : 2;
  static constexpr int kStageCodeBytes = (kStageK / G) * M * kCodeBytes;
  static constexpr int kTileRowBytes = (64 % kStageCodeBytes == 0) ? 64 : 48;
  static constexpr int kStagesPerTile = kTileRowBytes / kStageCodeBytes;
  static constexpr uint32_t kCodeTileBytes = static_cast<uint32_t>(kRows * kTileRowBytes);
  static constexpr bool kSwizzle64 = kTileRowBytes == 64;
  static constexpr bool kSmemCb = B == 8;
  // Decoded A stages may live in tensor memory (tcgen05.st, the MMA reading A from TMEM)
  // for every scheme decoded through registers; 1x16 g8 copies codewords into shared
  // memory by cp.async, so its A stages stay there.  The host picks the kATmem
  // instantiation per launch (pipe_kernel).
  // 1x16 g8 decodes by cp.async copies of codewords into the A stage; measured faster
  // than the register-staged gathers for this scheme, with A in shared memory or in
  // tensor memory (4096 x 4096 batch 1: 14.5 against 15.5 us; 11008 x 4096 batch 256:
  // 51.5 against 74.1 us)
  static constexpr bool kCpAsyncDecode = B == 16 && M == 1 && G == 8;
  static constexpr bool kATmemOk = !kCpAsyncDecode;
  // 2x8 g8: up to eight copies of each codebook in shared memory (cb_layout_offset), so
  // that the eight lanes of a quarter-warp phase read random codewords with few or no
  // bank conflicts; the host picks the count that still leaves room for three stages
  static constexpr int kCbMaxReplicas = (B == 8 && M == 2 && G == 8) ? 8 : 1;
  static constexpr uint32_t kCbBytes = kSmemCb ? static_cast<uint32_t>(M * 256 * G * 2) : 0u;  // one copy
  static constexpr int kSplitAlign = 16 / gcd_int(16, kStageCodeBytes);  // split starts: 16-byte code offsets
  static_assert(kTileRowBytes % kStageCodeBytes == 0 && kTileRowBytes % 16 == 0, "code tile rows");
  // every full code tile holds stages of both decoder groups
  static_assert(kStagesPerTile % kMaxDecoderGroups == 0, "stages per code tile");
  // a decoder thread reads half a stage of codes: inside one 16-byte chunk when swizzled
  static_assert(kStageCodeBytes % 2 == 0 && (!kSwizzle64 || 16 % (kStageCodeBytes / 2) == 0), "code halves");
};

// Input gradient dx = dy . W16 (kGrad kernels).  The MMA's M is 128 input features
// k, its K is the reduction over output rows n, 64 per stage.  The A stage holds
// W16[n][k] for 64 rows n x 128 features k in the MN-major 128-byte-swizzled
// layout (k contiguous), which is the order a decoded codeword comes in.  A code
// tile is one stage: 64 rows x the (128 / g) groups of the CTA's 128 features,
// loaded as a TMA box of kBoxBytes (rounded up to 16 bytes, starting at the
// 16-byte boundary at or below the tile's first code byte).
template <int M, int B, int G>
struct GradScheme {
  static constexpr int kCodeBytes = B <= 8 ? 1 : 2;
  static constexpr int kTileCodeBytes = (kRows / G) * M * kCodeBytes;   // codes of 128 features
  static constexpr int kBoxBytes = kTileCodeBytes % 16 == 0 ? kTileCodeBytes : (kTileCodeBytes + 8 + 15) / 16 * 16;
  static constexpr int kStagesPerTile = 1;
  static constexpr int kStageCodeBytes = kTileCodeBytes;   // one code tile per stage
  static constexpr uint32_t kCodeTileBytes = static_cast<uint32_t>(kStageK * kBoxBytes);
  static constexpr bool kSmemCb = B == 8;
  static constexpr bool kATmemOk = false;  // the MN-major A stage stays in shared memory
  // 2x8 g8: codebook copies as in the layer kernel (decode_grad_b8)
  static constexpr int kCbMaxReplicas = (B == 8 && M == 2 && G == 8) ? 8 : 1;
  static constexpr uint32_t kCbBytes = kSmemCb ? static_cast<uint32_t>(M * 256 * G * 2) : 0u;  // one copy
  static constexpr int kSplitAlign = 1;
  // a decoder thread reads the codes of a quarter of the tile's features
  static_assert(kTileCodeBytes % 8 == 0 && kBoxBytes <= 64, "gradient code tiles");
};

struct PipeLayout {
  uint32_t a, b, codes, cb, bars, total;
};

// a_stage_bytes: kABytes, or 0 when the A stages live in tensor memory.  acc_bars: 1,
// or 8 for stream-K (accumulator full / empty for two accumulators, and one bulk-copy
// barrier per epilogue warp).
__host__ __device__ inline PipeLayout pipe_layout(int S, int BN, uint32_t code_tile_bytes, uint32_t cb_bytes,
                                                  int code_slots, uint32_t a_stage_bytes, int acc_bars = 1) {
  PipeLayout L;
  L.a = 0;                                                          // 1024-aligned stages
  L.b = L.a + static_cast<uint32_t>(S) * a_stage_bytes;
  L.codes = L.b + static_cast<uint32_t>(S) * static_cast<uint32_t>(BN) * 128u;
  L.cb = L.codes + static_cast<uint32_t>(code_slots) * code_tile_bytes;
  L.bars = L.cb + cb_bytes;
  // full[S], empty[S], code_full[kCodeSlots], code_empty[kCodeSlots], acc bars, tmem slot, abort flag
  L.total = L.bars + 8u * static_cast<uint32_t>(2 * S + 2 * kCodeSlots + acc_bars) + 16u;
  return L;
}

__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hadd2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t mapa_shared_cluster(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ uint32_t swz128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Shared-memory offset, within one codebook's region, of 16-byte codeword e in copy j
// of R = 8 >> sh copies.  A codebook region is 256 / (8 / R) rows of 128 bytes; copy j
// owns the 16-byte columns j (8 / R) .. j (8 / R) + 8 / R - 1 of every row, and entry e
// sits in row e / (8 / R), column j (8 / R) + e mod (8 / R).  Lane l of a warp reads
// copy l mod R, so the eight lanes of a quarter-warp phase share each column group
// with 8 / R - 1 others only (R = 8: none, conflict-free; R = 1: the plain [256][16 B]
// layout, which this formula reduces to).
__device__ __forceinline__ uint32_t cb_layout_offset(uint32_t e, uint32_t j, int sh) {
  return ((e >> sh) << 7) | (((j << sh) | (e & ((1u << sh) - 1u))) << 4);
}

// MN-major 128-byte-swizzled A stage of the input-gradient kernel: feature k
// (0..127) is the contiguous (MN) index, row n (0..63) the reduction (K) index.
// Swizzle atoms are 8 rows x 64 features (1 KB, rows 128 bytes apart); atoms along
// n are kGradSbo apart, the two 64-feature halves kGradLbo apart.  Offset of the
// 16-byte chunk holding features 8 kc .. 8 kc + 7 of row n.
constexpr uint32_t kGradSbo = 1024u;
constexpr uint32_t kGradLbo = 8192u;
__device__ __forceinline__ uint32_t grad_a_offset(int n, int kc) {
  return static_cast<uint32_t>(kc >> 3) * kGradLbo + static_cast<uint32_t>(n >> 3) * kGradSbo +
         static_cast<uint32_t>((n & 7) * 128 + (((kc & 7) ^ (n & 7)) << 4));
}

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle:
// leading byte offset = stride between swizzle atoms along M/N, stride byte
// offset = stride between 8-row groups along K.
__device__ __forceinline__ uint64_t umma_desc_sw128_mnmajor(uint32_t smem_byte_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_byte_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Byte `off` of row `row` of a code tile.  With the 64-byte TMA swizzle the 16-byte
// chunk index is XORed with bits 7-8 of the byte offset (row / 2 mod 4), so the 32
// rows a warp reads at one chunk spread over all banks instead of two.
template <int kTileRowBytes, bool kSwizzle64>
__device__ __forceinline__ uint32_t code_tile_offset(int row, int off) {
  if constexpr (kSwizzle64)
    return static_cast<uint32_t>(row * 64 + ((((off >> 4) ^ (row >> 1)) & 3) << 4) + (off & 15));
  else
    return static_cast<uint32_t>(row * kTileRowBytes + off);
}

// pipe_wait for warps with nothing else to do (the stream-K epilogue): they sleep
// between polls, so their waiting takes no issue slots or shared-memory bandwidth
// from the decoders.
__device__ __forceinline__ bool pipe_wait_sleepy(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                                 uint32_t* status, uint32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    __nanosleep(256);
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitTimeoutNs) {
      record_failure(status, site);
      *abort_flag = 1u;
      return false;
    }
  }
  return true;
}

// Bounded wait that also gives up at once when another role has aborted.
__device__ __forceinline__ bool pipe_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
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

// B = 16 with register staging: the 16-byte pieces of the thread's 4 chunks of one
// stage (chunks 4 hf .. 4 hf + 3), for each of the M codebooks, gathered from the
// L2-resident codebooks into registers.  g = 16: one 256-bit load per 32-byte
// codeword (two chunks) when the codebooks are 32-byte aligned, else two 128-bit
// loads; g = 8: one 128-bit load per codeword.  `cw` points at the codes of the
// thread's half of the stage ([group][m], 2 bytes each).  v[m][i] receives chunk
// (i + rot) mod 4 (rot = 0 or 2).
template <int M, int G>
__device__ __forceinline__ void gather_stage_b16(uint4 (&v)[M][4], const uint8_t* cw, bool row_valid,
                                                 const __half* __restrict__ codebooks, bool cb32, uint64_t cb_pol,
                                                 int rot = 0) {
  const uint16_t* c16 = reinterpret_cast<const uint16_t*>(cw);
  if (!row_valid) {
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) v[m][cc] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const __half* cb = codebooks + static_cast<size_t>(m) * 65536u * G;
    if constexpr (G == 8) {
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
        v[m][cc] = ldg_nc_v4_hint(cb + static_cast<size_t>(c16[((cc + rot) & 3) * M + m]) * 8, cb_pol);
    } else if (cb32) {
#pragma unroll
      for (int q = 0; q < 2; ++q)
        ldg_nc_v8_hint(cb + static_cast<size_t>(c16[(q ^ (rot >> 1)) * M + m]) * 16, v[m][2 * q], v[m][2 * q + 1],
                       cb_pol);
    } else {
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int ch = (cc + rot) & 3;
        v[m][cc] = ldg_nc_v4_hint(cb + static_cast<size_t>(c16[(ch >> 1) * M + m]) * 16 + 8 * (ch & 1), cb_pol);
      }
    }
  }
}

// fp32 sum of the M 16-byte pieces (8 fp16 each) in codebook order, one rounding.
template <int M>
__device__ __forceinline__ uint4 sum_pieces(const uint4 (&q)[M]) {
  if constexpr (M == 1) {
    return q[0];
  } else if constexpr (M == 2) {
    // two fp16 values: their half2 sum is their exact sum rounded once
    return make_uint4(hadd2_u32(q[0].x, q[1].x), hadd2_u32(q[0].y, q[1].y), hadd2_u32(q[0].z, q[1].z),
                      hadd2_u32(q[0].w, q[1].w));
  } else {
    float f[8];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const uint32_t w[4] = {q[m].x, q[m].y, q[m].z, q[m].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 t = h2_to_f2(w[h]);
        f[2 * h] = (m == 0) ? t.x : f[2 * h] + t.x;
        f[2 * h + 1] = (m == 0) ? t.y : f[2 * h + 1] + t.y;
      }
    }
    return make_uint4(f2_to_h2_rn(f[0], f[1]), f2_to_h2_rn(f[2], f[3]), f2_to_h2_rn(f[4], f[5]),
                      f2_to_h2_rn(f[6], f[7]));
  }
}

// W16 for 8 features of one row from the M 16-byte codeword pieces: the pieces
// summed in fp32 in codebook order, times the row's scale, rounded once to fp16 --
// the dequantisation definition, so the gradient kernel's A operand is W16 bit for
// bit.  For M = 1 a half2 multiply gives the same bits: the product of two fp16
// values is exact in fp32, so both round the exact product once.
template <int M>
__device__ __forceinline__ uint4 scaled_sum_pieces(const uint4 (&q)[M], float s) {
  if constexpr (M == 1) {
    const __half2 s2 = __float2half2_rn(s);
    const uint32_t w[4] = {q[0].x, q[0].y, q[0].z, q[0].w};
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&w[h]), s2);
      o[h] = *reinterpret_cast<const uint32_t*>(&r);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
  } else {
    float f[8];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const uint32_t w[4] = {q[m].x, q[m].y, q[m].z, q[m].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 t = h2_to_f2(w[h]);
        f[2 * h] = (m == 0) ? t.x : f[2 * h] + t.x;
        f[2 * h + 1] = (m == 0) ? t.y : f[2 * h + 1] + t.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = f[e] * s;
    return make_uint4(f2_to_h2_rn(f[0], f[1]), f2_to_h2_rn(f[2], f[3]), f2_to_h2_rn(f[4], f[5]),
                      f2_to_h2_rn(f[6], f[7]));
  }
}

// The chunk (of the thread's 4) that quarter `qq` stores at step `step`.  The 8
// lanes of a quarter-warp (2 rows x 4 quarters) then write 8 different 16-byte bank
// groups of the MN-major stage: quarters 0 and 2 (and 1 and 3) differ only in the
// 64-feature half, which the swizzle does not separate, so they start 2 chunks apart.
__device__ __forceinline__ int grad_chunk_at(int step, int qq) { return (step + 2 * (qq >> 1)) & 3; }

// Input gradient, B = 8: decode the 4 chunks (32 features) of row `n` that thread
// quarter `qq` owns into the MN-major A stage at shared offset `a_off`.  `cw`
// points at the quarter's codes ([group][m], 1 byte each); `smem_cb` holds the M
// codebooks [M][256][G], or for 2x8 g8 the 8 >> cb_sh copies of cb_layout_offset (the
// thread reads copy `lane` mod R).
template <int M, int G>
__device__ __forceinline__ void decode_grad_b8(uint8_t* smem, uint32_t a_off, int n, int qq, bool row_valid,
                                               const uint8_t* cw, const uint8_t* smem_cb, float s, int cb_sh,
                                               int lane) {
  constexpr uint32_t kCbStride = 256u * G * 2u;
#pragma unroll
  for (int step = 0; step < 4; ++step) {
    const int cc = grad_chunk_at(step, qq);
    const int j = cc / (G / 8), h = cc % (G / 8);  // group within the quarter, 16-byte piece
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    if (row_valid) {
      uint4 pieces[M];
      if constexpr (M == 2 && G == 8) {
        const uint32_t cj = static_cast<uint32_t>(lane) & ((8u >> cb_sh) - 1u);
#pragma unroll
        for (int m = 0; m < M; ++m)
          pieces[m] = *reinterpret_cast<const uint4*>(smem_cb + static_cast<uint32_t>(m) * (32768u >> cb_sh) +
                                                      cb_layout_offset(cw[j * M + m], cj, cb_sh));
      } else {
#pragma unroll
        for (int m = 0; m < M; ++m)
          pieces[m] = *reinterpret_cast<const uint4*>(smem_cb + static_cast<uint32_t>(m) * kCbStride +
                                                      static_cast<uint32_t>(cw[j * M + m]) * (G * 2u) +
                                                      16u * static_cast<uint32_t>(h));
      }
      out = scaled_sum_pieces<M>(pieces, s);
    }
    *reinterpret_cast<uint4*>(smem + a_off + grad_a_offset(n, 4 * qq + cc)) = out;
  }
}

// The thread's 4 decoded 16-byte chunks of weight row r (chunks 4 hf .. 4 hf + 3 of a
// 64-wide stage) into the A stage: shared memory (128-byte swizzled K-major layout at
// a_off), or tensor memory (to_tmem: lane r, columns 16 hf .. 16 hf + 15 of the stage at
// a_tmem, which carries the warp's lane quadrant; warp-collective, waits for the stores).
__device__ __forceinline__ void store_a_half(bool to_tmem, uint8_t* smem, uint32_t a_off, uint32_t a_tmem, int r,
                                             int hf, const uint4 (&out)[4]) {
  if (to_tmem) {
    uint32_t v[16];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      v[4 * cc] = out[cc].x;
      v[4 * cc + 1] = out[cc].y;
      v[4 * cc + 2] = out[cc].z;
      v[4 * cc + 3] = out[cc].w;
    }
    tmem_st_32x32b_x16_wait(a_tmem + 16u * static_cast<uint32_t>(hf), v);
  } else {
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) *reinterpret_cast<uint4*>(smem + a_off + swz128(r, 4 * hf + cc)) = out[cc];
  }
}

// Decode half (`hf` = 0: chunks 0-3, 1: chunks 4-7) of one 64-wide K stage of
// weight row `r` into the swizzled A stage at shared offset `a_off`.  `cw` points at
// the codes of this half of the stage (half the stage's code bytes, never crossing a
// 16-byte chunk of a swizzled code tile).
//   B = 16, M = 1, g = 8: each 16-byte chunk is one codeword, copied from the
//     L2-resident codebook straight into its slot by cp.async (one 2-byte code load
//     per gather, so each gather issues as soon as its own code has arrived).
//   B = 8: the codebooks are staged in shared memory ([M][256][G]); a chunk is the
//     sum of the matching 16-byte pieces of the group's M codewords.
template <int M, int B, int G>
__device__ __forceinline__ void decode_half_stage(bool to_tmem, uint8_t* smem, uint32_t sbase, uint32_t a_off,
                                                  uint32_t a_tmem, int r, int hf, bool row_valid, const uint8_t* cw,
                                                  const __half* __restrict__ codebooks, const uint8_t* smem_cb,
                                                  uint64_t cb_pol, int cb_sh) {
  if constexpr (B == 16) {
    static_assert(M == 1 && G == 8, "other B = 16 shapes use the register-staged decoder");
    const uint16_t* c16 = reinterpret_cast<const uint16_t*>(cw);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int chunk = 4 * hf + cc;
      const uint32_t code = c16[cc];
      const __half* src = codebooks + static_cast<size_t>(code) * 8;
      cp_async_16_zfill_hint(sbase + a_off + swz128(r, chunk),
                             row_valid ? static_cast<const void*>(src) : static_cast<const void*>(codebooks),
                             row_valid ? 16u : 0u, cb_pol);
    }
  } else if constexpr (M == 2 && G == 8) {
    // 2x8: the thread's 8 code bytes (c0, c1 per group) of this stage in one load
    const uint2 q = *reinterpret_cast<const uint2*>(cw);
    const uint32_t cwords[2] = {q.x, q.y};
    uint4 out[4];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      out[cc] = make_uint4(0u, 0u, 0u, 0u);
      if (row_valid) {
        const uint32_t c0 = (cwords[cc >> 1] >> (16 * (cc & 1))) & 0xFFu;
        const uint32_t c1 = (cwords[cc >> 1] >> (16 * (cc & 1) + 8)) & 0xFFu;
        // the thread reads copy r mod R of each codebook (r mod 32 is its lane); the
        // second codebook's region follows the first's (4 KB per copy)
        const uint32_t j = static_cast<uint32_t>(r) & ((8u >> cb_sh) - 1u);
        const uint4 pieces[2] = {
            *reinterpret_cast<const uint4*>(smem_cb + cb_layout_offset(c0, j, cb_sh)),
            *reinterpret_cast<const uint4*>(smem_cb + (32768u >> cb_sh) + cb_layout_offset(c1, j, cb_sh))};
        out[cc] = sum_pieces<2>(pieces);
      }
      // shared-memory A: each chunk stored as soon as it is decoded (measured faster than
      // one store burst at the end)
      if (!to_tmem) *reinterpret_cast<uint4*>(smem + a_off + swz128(r, 4 * hf + cc)) = out[cc];
    }
    if (to_tmem) store_a_half(true, smem, a_off, a_tmem, r, hf, out);
  } else {
    constexpr uint32_t kCbStride = 256u * G * 2u;  // bytes per codebook
    uint4 out[4];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int j = cc / (G / 8), h = cc % (G / 8);  // group within the half, 16-byte piece
      out[cc] = make_uint4(0u, 0u, 0u, 0u);
      if (row_valid) {
        uint4 pieces[M];
#pragma unroll
        for (int m = 0; m < M; ++m)
          pieces[m] = *reinterpret_cast<const uint4*>(smem_cb + static_cast<uint32_t>(m) * kCbStride +
                                                      static_cast<uint32_t>(cw[j * M + m]) * (G * 2u) +
                                                      16u * static_cast<uint32_t>(h));
        out[cc] = sum_pieces<M>(pieces);
      }
      if (!to_tmem) *reinterpret_cast<uint4*>(smem + a_off + swz128(r, 4 * hf + cc)) = out[cc];
    }
    if (to_tmem) store_a_half(true, smem, a_off, a_tmem, r, hf, out);
  }
}

__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}


// kGrad = false: y = x . W16^T . diag(s) + bias (rows = N, reduction over K).
// kGrad = true:  dx = dy . W16 (rows = K input features, reduction over the N
//                output rows; x_map then describes dy [batch, N]).
// kATmem: the decoded A stages live in tensor memory (schemes with kATmemOk); a separate
// instantiation, since the same loops with a runtime switch compiled measurably slower.
// kStreamK: the CTA takes a range of the (tile, K stage) space that may cross tiles
// (PipeParams), and four epilogue warps finish each tile piece while the decoders
// go on with the next (see the epilogue below).
template <int M, int B, int G, bool kGrad, bool kATmem, bool kStreamK>
__global__ void __launch_bounds__(PipeShape<M, B, G, kGrad, kStreamK>::kThreads, 1)
    tc_pipe_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap code_map,
                   const PipeParams p) {
  constexpr int kDecoderGroups = PipeShape<M, B, G, kGrad>::kGroups;
  constexpr int kDecoders = PipeShape<M, B, G, kGrad>::kDecoders;
  constexpr int kThreads = PipeShape<M, B, G, kGrad, kStreamK>::kThreads;
  constexpr int kWarpX = kDecoders / 32, kWarpMma = kWarpX + 1, kWarpCodes = kWarpX + 2;
  constexpr int kWarpEpi = kWarpX + 3;  // stream-K: warps kWarpEpi .. + 3, lane quadrants 3, 0, 1, 2
  static_assert(!(kATmem && kStreamK), "stream-K keeps A in shared memory");
  extern __shared__ uint8_t smem_raw[];
  // stages must be 1024-byte aligned for the 128-byte swizzle
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  using SC = std::conditional_t<kGrad, GradScheme<M, B, G>, PipeScheme<M, B, G>>;
  constexpr int kStageCodeBytes = SC::kStageCodeBytes;
  constexpr int kStagesPerTile = SC::kStagesPerTile;
  constexpr uint32_t kCodeTileBytes = SC::kCodeTileBytes;
  const int S = p.S;
  static_assert(!kATmem || SC::kATmemOk, "A in tensor memory needs a register-decoded scheme");
  constexpr bool a_in_tmem = kATmem;
  const PipeLayout L = pipe_layout(S, p.BN, kCodeTileBytes, SC::kCbBytes * (8u >> p.cb_sh), 1 << p.cs_log,
                                   a_in_tmem ? 0u : kABytes, kStreamK ? 8 : 1);
  const int cs_log = p.cs_log;          // code-tile slots: 1 << cs_log
  const int cs_mask = (1 << cs_log) - 1;
  const uint32_t sbase = smem_addr(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);   // stage s decoded and x landed
  uint64_t* empty = full + S;                                     // stage s consumed by the MMAs
  uint64_t* cfull = empty + S;                                    // code tile landed
  uint64_t* cempty = cfull + kCodeSlots;                          // code tile read by the 8 decoder warps
  uint64_t* acc_bar = cempty + kCodeSlots;                        // accumulator complete
  // stream-K: acc_bar[a] = accumulator a complete, acc_bar[2 + a] = accumulator a
  // drained, acc_bar[4 + q] = epilogue warp q's bulk copies landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_bar + (kStreamK ? 8 : 1));
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n0 = kStreamK ? 0 : blockIdx.x * kRows;
  const int b0 = kStreamK ? 0 : blockIdx.y * p.BN;
  const int split = blockIdx.z;  // == rank in the (1, 1, SK) cluster
  // this CTA's K range: stages [ks0, ks1), read as nct code tiles of kStagesPerTile
  // stages starting at stage ks0 (the host keeps ks0's code offset 16-byte aligned).
  // Stream-K: stages [w0, w0 + nks) of the (tile, K stage) space; units are whole
  // code tiles and nk a multiple of them, so no code tile straddles two tiles.
  const SkRange skr{p.sk_ctas, p.sk_units, p.sk_unit};
  const int w0 = kStreamK ? skr.begin(blockIdx.x) : 0;
  const int ks0 = kStreamK ? 0 : split * p.ks_per;
  const int ks1 = kStreamK ? 0 : min(p.nk, ks0 + p.ks_per);
  const int nks = kStreamK ? skr.begin(blockIdx.x + 1) - w0 : max(0, ks1 - ks0);  // host guarantees >= 1
  const int nct = (nks + kStagesPerTile - 1) / kStagesPerTile;
  // row-tile origin, batch-tile origin and K stage of the CTA's stage i
  auto stage_at = [&](int i, int& n0_, int& b0_, int& k_) {
    if constexpr (kStreamK) {
      const int w = w0 + i;
      const int t = w / p.nk;
      k_ = w - t * p.nk;
      n0_ = (t / p.batch_tiles) * kRows;
      b0_ = (t % p.batch_tiles) * p.BN;
    } else {
      n0_ = n0;
      b0_ = b0;
      k_ = ks0 + i;
    }
  };

  // the next kernel on the stream may start its own set-up now; x is read (and
  // y written) only after this grid's dependency wait in the x producer below
  grid_dependents_launch();
  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], kGroupThreads + 1);  // the group that decodes the stage + the x tile
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kCodeSlots; ++i) {
      mbar_init(&cfull[i], 1);
      // every decoder warp that reads the tile: both groups when a tile holds several
      // stages (the final, partial tile may see one group only: its slot is not reused)
      mbar_init(&cempty[i], (kStagesPerTile >= kDecoderGroups ? kDecoders : kGroupThreads) / 32);
    }
    mbar_init(acc_bar, 1);
    if constexpr (kStreamK) {
      mbar_init(acc_bar + 1, 1);
      mbar_init(acc_bar + 2, 4);  // the four epilogue warps
      mbar_init(acc_bar + 3, 4);
      for (int i = 4; i < 8; ++i) mbar_init(acc_bar + i, 1);
    }
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if constexpr (SC::kSmemCb) {
    if constexpr (SC::kCbMaxReplicas == 1) {
      // the M codebooks, [M][256][G] fp16, copied as they are
      for (int i = tid; i < static_cast<int>(SC::kCbBytes / 16u); i += kThreads)
        *reinterpret_cast<uint4*>(smem + L.cb + 16u * static_cast<uint32_t>(i)) = ldg_nc_v4(p.codebooks + 8 * i);
    } else {
      // 2x8 g8: every copy of codeword e of codebook m (cb_layout_offset)
      const int reps = 8 >> p.cb_sh;
      for (int i = tid; i < M * 256 * reps; i += kThreads) {
        const int j = i % reps, me = i / reps;  // copy, codeword m * 256 + e
        const uint32_t m = static_cast<uint32_t>(me >> 8), e = static_cast<uint32_t>(me & 255);
        *reinterpret_cast<uint4*>(smem + L.cb + m * (32768u >> p.cb_sh) +
                                  cb_layout_offset(e, static_cast<uint32_t>(j), p.cb_sh)) = ldg_nc_v4(p.codebooks + 8 * me);
      }
    }
  }
  if (warp == 0) tmem_alloc(tmem_slot, p.tmem_cols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWarpX) {
    // ---- x tiles (B operand): reused by every CTA, keep them in L2 ----
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();
      // x may be the previous kernel's output.  Every y store of this CTA
      // follows the MMAs, which follow these x tiles, so it is ordered too.
      grid_dependency_wait();
      for (int i = 0; i < nks; ++i) {
        const int s = i % S, u = i / S;
        if (u > 0 && !pipe_wait(&empty[s], static_cast<uint32_t>((u - 1) & 1), abort_flag, p.status, kSitePipeEmpty))
          break;
        int n0_, b0_, k_;
        stage_at(i, n0_, b0_, k_);
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(p.BN) * 128u);
        tma_load_2d(sbase + L.b + static_cast<uint32_t>(s * p.BN) * 128u, &x_map, k_ * kStageK, b0_, &full[s], pol);
      }
    }
  } else if (warp == kWarpCodes) {
    // ---- code tiles: 128 rows x 64 bytes, read once ----
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      for (int t = 0; t < nct; ++t) {
        const int c = t & cs_mask, u = t >> cs_log;
        if (u > 0 && !pipe_wait(&cempty[c], static_cast<uint32_t>((u - 1) & 1), abort_flag, p.status, kSitePipeCodes))
          break;
        int n0_, b0_, k_;  // the tile's first stage
        stage_at(t * kStagesPerTile, n0_, b0_, k_);
        mbar_arrive_expect_tx(&cfull[c], kCodeTileBytes);
        if constexpr (kGrad) {
          // rows k_ 64 .. + 63 of the feature columns of row tile n0_; rows past N and
          // bytes past the row end are zero-filled
          tma_load_2d(sbase + L.codes + static_cast<uint32_t>(c) * kCodeTileBytes, &code_map,
                      (n0_ * SC::kTileCodeBytes / kRows) & ~15, k_ * kStageK, &cfull[c], pol);
        } else {
          // bytes past the row end (K edge) are zero-filled; stages past ks1 are not decoded
          tma_load_2d(sbase + L.codes + static_cast<uint32_t>(c) * kCodeTileBytes, &code_map, k_ * kStageCodeBytes,
                      n0_, &cfull[c], pol);
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ---- one thread issues the MMAs; each stage's commit releases it ----
    if (lane == 0) {
      // the gradient's A stage is MN-major (bit 15 of the instruction descriptor)
      const uint32_t idesc = umma_idesc_f16_f32(kRows, static_cast<uint32_t>(p.BN)) | (kGrad ? (1u << 15) : 0u);
      int piece = 0;  // stream-K: tile pieces begun so far; piece q accumulates into accumulator q mod 2
      for (int i = 0; i < nks; ++i) {
        const int s = i % S;
        bool first = i == 0, last = i == nks - 1;  // the first / last stage of a tile piece
        uint32_t d_tmem = tmem;
        if constexpr (kStreamK) {
          const int k_ = (w0 + i) % p.nk;
          if (k_ == 0 && i > 0) ++piece;
          first = first || k_ == 0;
          last = last || k_ == p.nk - 1;
          const int a = piece & 1;
          d_tmem = tmem + static_cast<uint32_t>(a * p.acc_cols);
          // the epilogue has drained what piece - 2 left in this accumulator
          if (first && piece >= 2 &&
              !pipe_wait(acc_bar + 2 + a, static_cast<uint32_t>(((piece - 2) >> 1) & 1), abort_flag, p.status,
                         kSitePipeAcc))
            break;
        }
        if (!pipe_wait(&full[s], static_cast<uint32_t>((i / S) & 1), abort_flag, p.status, kSitePipeFull)) break;
        fence_proxy_async_smem();  // decoder writes (cp.async / st.shared) -> tensor-core reads
        tc_fence_after_sync();
        const uint64_t bdesc = umma_desc_sw128_kmajor(sbase + L.b + static_cast<uint32_t>(s * p.BN) * 128u);
        if (a_in_tmem) {
          // A stage s at TMEM columns kATmemCol + 32 s: 8 columns (16 fp16) per K = 16 step
          const uint32_t a_tmem = tmem + kATmemCol + 32u * static_cast<uint32_t>(s);
#pragma unroll
          for (int kk = 0; kk < kStageK / 16; ++kk)
            umma_f16_ts(d_tmem, a_tmem + 8u * kk, bdesc + 2 * kk, idesc, (!first || kk > 0) ? 1u : 0u);
        } else {
          const uint32_t a_addr = sbase + L.a + static_cast<uint32_t>(s) * kABytes;
#pragma unroll
          for (int kk = 0; kk < kStageK / 16; ++kk) {
            // K = 16 per MMA: 32 bytes along a K-major row, or two 8-row atoms (2 x SBO) MN-major
            const uint64_t adesc = kGrad ? umma_desc_sw128_mnmajor(a_addr + 2u * kGradSbo * kk, kGradLbo, kGradSbo)
                                         : umma_desc_sw128_kmajor(a_addr) + 2 * kk;
            umma_f16_ss(d_tmem, adesc, bdesc + 2 * kk, idesc, (!first || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
        if (kStreamK && last) umma_commit(acc_bar + (piece & 1));
      }
      if (!kStreamK) umma_commit(acc_bar);
    }
  } else if (kStreamK && warp >= kWarpEpi) {
    if constexpr (kStreamK) {
      // ---- stream-K epilogue.  Warp q = warp mod 4 owns TMEM lanes 32 q .. 32 q + 31,
      // rows 32 q + lane of every tile piece of the CTA, taken in order as the MMAs
      // complete them.  A tile done whole by this CTA goes straight to y.  A tile cut
      // into P pieces (CTAs cf .. cf + P - 1, in K order) is finished by one of them:
      // each piece stores its fp32 partial in its slot and counts itself in the
      // counter of (cf, q); the piece that finds the other P - 1 counted (before
      // storing, or from what its own increment returns) adds all P in K order (its own
      // from TMEM), writes y and clears the counter.  No piece waits for another, the
      // sum order does not depend on which piece finishes, and the warps of a CTA do
      // not wait for each other.
      //   A slot is [quadrant][BN / 4][32 rows][4] fp32, so the 32 rows of a warp form
      // one contiguous run.  When the finishing piece is the CTA's last, every stage,
      // code and codebook byte of shared memory is free (all MMAs are done), and each
      // warp brings the other pieces' runs into its quarter of it with bulk copies
      // before adding: the partial reads then cost one copy per piece instead of a
      // chain of dependent L2 round trips per 16 columns.
      const int q = warp & 3;
      grid_dependency_wait();  // y and the workspace may be in use by the previous grid
      const int cta = static_cast<int>(blockIdx.x);
      const int w_end = w0 + nks;
      const int BN = p.BN;
      const uint32_t tq = tmem + (static_cast<uint32_t>(32 * q) << 16);
      const size_t slot_floats = static_cast<size_t>(kRows) * BN;
      const size_t quad_float4s = static_cast<size_t>(BN / 4) * 32;  // this warp's run in a slot
      const uint32_t quad_smem = ((L.bars - L.a) / 4u) & ~15u;        // this warp's share of the free memory
      const uint32_t region = sbase + L.a + static_cast<uint32_t>(q) * quad_smem;
      uint64_t* bulk_bar = acc_bar + 4 + q;
      uint32_t bulk_phase = 0;
      int piece = 0;
      for (int w = w0; w < w_end; ++piece) {
        const int t = w / p.nk;
        const int w_next = min(w_end, (t + 1) * p.nk);
        const int a = piece & 1;
        if (!__all_sync(0xffffffffu,
                        pipe_wait_sleepy(acc_bar + a, static_cast<uint32_t>((piece >> 1) & 1), abort_flag, p.status,
                                         kSitePipeAcc) && !*abort_flag)) {
          *abort_flag = 1u;
          break;
        }
        tc_fence_after_sync();
        const uint32_t acc = tq + static_cast<uint32_t>(a * p.acc_cols);
        const int n0_ = (t / p.batch_tiles) * kRows, b0_ = (t % p.batch_tiles) * BN;
        const int n = n0_ + 32 * q + lane;
        const bool n_valid = n < p.rows;
        // the gradient's scale is inside its A operand and it has no bias
        const float sc = kGrad ? 1.f : (n_valid ? __half2float(p.scales[n]) : 0.f);
        const float bi = (!kGrad && n_valid && p.bias != nullptr) ? __half2float(p.bias[n]) : 0.f;
        const int cf = skr.cta_of(t * p.nk), cl = skr.cta_of((t + 1) * p.nk - 1);
        const int P = cl - cf + 1;
        // this warp's run of CTA cc's slot for tile t: slot 2 cc holds a CTA's first
        // piece, 2 cc + 1 its last (middle pieces are whole tiles)
        auto run_of = [&](int cc) {
          return reinterpret_cast<float4*>(p.sk_part + static_cast<size_t>(2 * cc + (skr.begin(cc) < t * p.nk ? 1 : 0)) *
                                                           slot_floats) +
                 static_cast<size_t>(q) * quad_float4s;
        };
        auto store_y = [&](int c0, const float (&v)[16]) {
          if (n_valid) {
    #pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int b = b0_ + c0 + i;
              if (b < p.batch) p.y[static_cast<size_t>(b) * p.rows + n] = __float2half_rn(v[i] * sc + bi);
            }
          }
        };
        uint32_t* cnt = p.sk_count + 4 * cf + q;
        bool finish = P == 1;
        if (!finish) {
          uint32_t seen = lane == 0 ? ld_acquire_gpu_u32(cnt) : 0u;
          seen = __shfl_sync(0xffffffffu, seen, 0);
          if (seen == static_cast<uint32_t>(P - 1)) {
            finish = true;  // every other piece is stored: no need to store this one
          } else {
            float4* mine = run_of(cta);
            for (int c0 = 0; c0 < BN; c0 += 16) {
              float v[16];
              tmem_ld_32x32b_x16(acc + static_cast<uint32_t>(c0), v);
    #pragma unroll
              for (int u = 0; u < 4; ++u)
                __stcg(mine + (c0 / 4 + u) * 32 + lane, make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]));
            }
            __threadfence();
            __syncwarp();
            uint32_t old = lane == 0 ? atomicAdd(cnt, 1u) : 0u;
            old = __shfl_sync(0xffffffffu, old, 0);
            finish = old == static_cast<uint32_t>(P - 1);
          }
          if (finish) (void)ld_acquire_gpu_u32(cnt);  // every lane: the other pieces' stores are visible
        }
        if (finish && P == 1) {
          for (int c0 = 0; c0 < BN; c0 += 16) {
            float v[16];
            tmem_ld_32x32b_x16(acc + static_cast<uint32_t>(c0), v);
            store_y(c0, v);
          }
        } else if (finish && w_next == w_end && static_cast<uint32_t>(16 * ((P - 1) * 32 * 4 + 64)) <= quad_smem) {
          // the CTA's last piece: the other pieces' runs come into shared memory by bulk
          // copies, W columns of each per pass, and y leaves through a staged fp16 tile
          // (32 rows x W columns, row index fastest) as 16-byte stores of 8 rows when
          // the row count keeps them aligned
          const int W = min(BN, static_cast<int>(quad_smem / static_cast<uint32_t>((P - 1) * 32 * 4 + 64)) / 16 * 16);
          const bool vec_y = (p.rows & 7) == 0;
          for (int c_lo = 0; c_lo < BN; c_lo += W) {
            const int wcols = min(W, BN - c_lo);
            const uint32_t run_bytes = static_cast<uint32_t>(wcols) * 32u * 4u;
            __half* ystage = reinterpret_cast<__half*>(smem + (region - sbase) + static_cast<uint32_t>(P - 1) * run_bytes);
            if (lane == 0) {
              fence_proxy_async_global();  // the acquired partials, then the async-proxy copies
              fence_proxy_async_smem();    // this warp's reads of the previous pass, then the copies
              mbar_arrive_expect_tx(bulk_bar, static_cast<uint32_t>(P - 1) * run_bytes);
              int k = 0;
              for (int cc = cf; cc <= cl; ++cc) {
                if (cc == cta) continue;
                bulk_load(region + static_cast<uint32_t>(k) * run_bytes, run_of(cc) + (c_lo / 4) * 32, run_bytes,
                          bulk_bar);
                ++k;
              }
            }
            __syncwarp();
            if (!__all_sync(0xffffffffu, pipe_wait(bulk_bar, bulk_phase, abort_flag, p.status, kSitePipeAcc))) {
              *abort_flag = 1u;
              break;
            }
            bulk_phase ^= 1u;
            for (int c0 = c_lo; c0 < c_lo + wcols; c0 += 16) {
              float v[16];
              tmem_ld_32x32b_x16(acc + static_cast<uint32_t>(c0), v);
              float sum[16];
    #pragma unroll
              for (int i = 0; i < 16; ++i) sum[i] = 0.f;
              int k = 0;
              for (int cc = cf; cc <= cl; ++cc) {
                if (cc == cta) {
    #pragma unroll
                  for (int i = 0; i < 16; ++i) sum[i] += v[i];
                } else {
                  const float4* src = reinterpret_cast<const float4*>(smem + (region - sbase)) +
                                      static_cast<size_t>(k) * (run_bytes / 16u);
    #pragma unroll
                  for (int u = 0; u < 4; ++u) {
                    const float4 f = src[((c0 - c_lo) / 4 + u) * 32 + lane];
                    sum[4 * u] += f.x;
                    sum[4 * u + 1] += f.y;
                    sum[4 * u + 2] += f.z;
                    sum[4 * u + 3] += f.w;
                  }
                  ++k;
                }
              }
              if (vec_y) {
    #pragma unroll
                for (int i = 0; i < 16; ++i) ystage[(c0 - c_lo + i) * 32 + lane] = __float2half_rn(sum[i] * sc + bi);
              } else {
                store_y(c0, sum);
              }
            }
            if (vec_y) {
              __syncwarp();  // the staged tile is complete
              // lane l writes 8 rows of one column per step: 8 columns x 64 bytes per warp store
              for (int u = lane; u < wcols * 4; u += 32) {
                const int col = u >> 2, part = u & 3;
                const int b = b0_ + c_lo + col;
                const int nn = n0_ + 32 * q + 8 * part;
                if (b < p.batch && nn < p.rows)
                  *reinterpret_cast<uint4*>(p.y + static_cast<size_t>(b) * p.rows + nn) =
                      *reinterpret_cast<const uint4*>(ystage + col * 32 + 8 * part);
              }
            }
            __syncwarp();  // every lane has read this pass before the next one's copies
          }
        } else if (finish) {
          // a piece before the CTA's last: the pipeline still uses shared memory, so the
          // partials are read from L2 directly
          for (int c0 = 0; c0 < BN; c0 += 16) {
            float v[16];
            tmem_ld_32x32b_x16(acc + static_cast<uint32_t>(c0), v);
            float sum[16];
    #pragma unroll
            for (int i = 0; i < 16; ++i) sum[i] = 0.f;
            for (int cc = cf; cc <= cl; ++cc) {
              if (cc == cta) {
    #pragma unroll
                for (int i = 0; i < 16; ++i) sum[i] += v[i];
              } else {
                const float4* src = run_of(cc);
    #pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const float4 f = __ldcg(src + (c0 / 4 + u) * 32 + lane);
                  sum[4 * u] += f.x;
                  sum[4 * u + 1] += f.y;
                  sum[4 * u + 2] += f.z;
                  sum[4 * u + 3] += f.w;
                }
              }
            }
            store_y(c0, sum);
          }
        }
        if (finish && P > 1) {
          __syncwarp();
          if (lane == 0) *reinterpret_cast<volatile uint32_t*>(cnt) = 0u;  // ready for the next launch
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_bar + 2 + a);  // accumulator a may be overwritten
        w = w_next;
      }
    }
  } else {
    // the 65536-entry codebooks of the B = 16 schemes are gathered from L2 all kernel
    // long: keep their lines there while the code stream (evict_first) passes by
    const uint64_t cb_pol = l2_policy_evict_last();
    if constexpr (kGrad) {
    // ---- decoders (input gradient): thread (row nl = 8 w + lane / 4, quarter qq =
    // lane % 4) decodes features 32 qq .. 32 qq + 31 of row (ks0 + i) 64 + nl at
    // stage i, scaled by that row's s_n.  A warp reads 8 rows x 4 quarters of codes
    // (contiguous bytes) and its 32 chunk stores cover every bank group 4 times.
    const int grp = warp / (kGroupThreads / 32);
    const int nl = 8 * (warp % (kGroupThreads / 32)) + (lane >> 2);
    const int qq = lane & 3;
    // this thread's codes in a code tile of row tile n0_ (whose first byte sits at
    // offset (n0_ g-groups) mod 16 of the 16-byte-aligned box)
    auto code_off_at = [&](int n0_) {
      return static_cast<uint32_t>(nl * SC::kBoxBytes + ((n0_ * SC::kTileCodeBytes / kRows) & 15) +
                                   qq * (SC::kTileCodeBytes / 4));
    };
    // output row n0_ and reduction row (over N) of stage i
    auto grad_stage = [&](int i, int& n0_, int& n_) {
      int b0_, k_;
      stage_at(i, n0_, b0_, k_);
      n_ = k_ * kStageK + nl;
    };
    if constexpr (B == 16) {
      // codewords gathered from L2 into registers kLook stages ahead, as in the layer kernel
      constexpr int kLook = (M == 1) ? 3 : 1;
      uint4 st[kLook + 1][M][4];
      float sv[kLook + 1];
      bool alive = true;
      const int nmine = (nks - grp + kDecoderGroups - 1) / kDecoderGroups;  // this group's stages
      for (int base = 0; alive && base < nmine + kLook; base += kLook + 1) {
#pragma unroll
        for (int u = 0; u <= kLook; ++u) {
          const int ki = base + u, kj = ki - kLook;   // this group's stage numbers
          const int i = grp + kDecoderGroups * ki;    // stage gathered now
          const int j = grp + kDecoderGroups * kj;    // stage stored now
          const bool issue = ki < nmine, store = kj >= 0 && kj < nmine;
          const int c = i & cs_mask;
          const int sj = j >= 0 ? j % S : 0, uj = j >= 0 ? j / S : 0;
          bool ready = true;
          if (issue)
            ready = pipe_wait(&cfull[c], static_cast<uint32_t>((i >> cs_log) & 1), abort_flag, p.status,
                              kSitePipeCodes);
          if (ready && store && uj > 0)
            ready = pipe_wait(&empty[sj], static_cast<uint32_t>((uj - 1) & 1), abort_flag, p.status, kSitePipeEmpty);
          if (!__all_sync(0xffffffffu, ready)) {
            *abort_flag = 1u;
            alive = false;
            break;
          }
          if (issue) {
            int n0_, n;
            grad_stage(i, n0_, n);
            const bool valid = n < p.N;
            sv[u] = valid ? __half2float(p.scales[n]) : 0.f;
            gather_stage_b16<M, G>(st[u], smem + L.codes + static_cast<uint32_t>(c) * kCodeTileBytes + code_off_at(n0_),
                                   valid,
                                   p.codebooks, p.cb32 != 0, cb_pol, 2 * (qq >> 1));
            __syncwarp();  // every lane has read its codes of this tile
            if (lane == 0) mbar_arrive(&cempty[c]);
          }
          if (store) {
            const int slot = (u + 1) % (kLook + 1);
            int n0_, nj;
            grad_stage(j, n0_, nj);
            const bool valid = nj < p.N;
            const uint32_t a_off = L.a + static_cast<uint32_t>(sj) * kABytes;
#pragma unroll
            for (int step = 0; step < 4; ++step) {
              // register slot `step` holds chunk grad_chunk_at(step, qq) (gathered rotated)
              uint4 pieces[M];
#pragma unroll
              for (int m = 0; m < M; ++m) pieces[m] = st[slot][m][step];
              const uint4 out = valid ? scaled_sum_pieces<M>(pieces, sv[slot]) : make_uint4(0u, 0u, 0u, 0u);
              *reinterpret_cast<uint4*>(smem + a_off + grad_a_offset(nl, 4 * qq + grad_chunk_at(step, qq))) = out;
            }
            fence_proxy_async_smem();
            mbar_arrive(&full[sj]);
          }
        }
      }
    } else {
      // B = 8: codebooks in shared memory; the next stage's scale is loaded one stage ahead.
      // The (tile, K stage) of this group's stage is tracked by stepping, not divided out
      // per stage (the decoders are issue-bound).
      int ct = 0, ck = ks0 + grp;
      if constexpr (kStreamK) {
        const int w = w0 + grp;
        ct = w / p.nk;
        ck = w - ct * p.nk;
      }
      int cached_t = -1, cached_n0 = n0;
      auto n0_of = [&](int t) {
        if constexpr (kStreamK) {
          if (t != cached_t) {
            cached_t = t;
            cached_n0 = (t / p.batch_tiles) * kRows;
          }
        }
        return cached_n0;
      };
      auto step = [&](int& t, int& k) {
        k += kDecoderGroups;
        if constexpr (kStreamK) {
          while (k >= p.nk) {
            k -= p.nk;
            ++t;
          }
        }
      };
      float s_next = (grp < nks && ck * kStageK + nl < p.N) ? __half2float(p.scales[ck * kStageK + nl]) : 0.f;
      for (int i = grp; i < nks; i += kDecoderGroups) {
        const int c = i & cs_mask;
        bool ready = pipe_wait(&cfull[c], static_cast<uint32_t>((i >> cs_log) & 1), abort_flag, p.status,
                               kSitePipeCodes);
        const int s = i % S, u = i / S;
        if (ready && u > 0)
          ready = pipe_wait(&empty[s], static_cast<uint32_t>((u - 1) & 1), abort_flag, p.status, kSitePipeEmpty);
        if (!__all_sync(0xffffffffu, ready)) {
          *abort_flag = 1u;
          break;
        }
        const int n = ck * kStageK + nl;
        const int n0_ = n0_of(ct);
        const float sc = s_next;
        int nt = ct, nkk = ck;
        step(nt, nkk);
        if (i + kDecoderGroups < nks) {
          const int n_next = nkk * kStageK + nl;
          s_next = n_next < p.N ? __half2float(p.scales[n_next]) : 0.f;
        }
        decode_grad_b8<M, G>(smem, L.a + static_cast<uint32_t>(s) * kABytes, nl, qq, n < p.N,
                             smem + L.codes + static_cast<uint32_t>(c) * kCodeTileBytes + code_off_at(n0_), smem + L.cb, sc,
                             p.cb_sh, lane);
        fence_proxy_async_smem();
        mbar_arrive(&full[s]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&cempty[c]);
        ct = nt;
        ck = nkk;
      }
    }
    } else {
    // ---- decoders: threads r and r + 128 share weight row n0 + r (chunks 0-3 / 4-7) ----
    const int r = tid & (kRows - 1);
    // A stages in tensor memory: the warp's lane quadrant (rows 32 (warp mod 4) ..) at
    // the A columns (stage s adds 32 s)
    const uint32_t a_tmem_q = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + kATmemCol;
    const int hf = kDecoderGroups == 1 ? tid >> 7 : (tid >> 7) & 1;
    const int grp = kDecoderGroups == 1 ? 0 : tid / kGroupThreads;
    const bool row_valid = n0 + r < p.N;
    // stream-K: whether row r of stage i's row tile exists
    const bool all_rows = p.N % kRows == 0;  // every row tile full: no per-stage row test
    auto row_valid_at = [&](int i) {
      if constexpr (kStreamK) {
        if (all_rows) return true;
        int n0_, b0_, k_;
        stage_at(i, n0_, b0_, k_);
        return n0_ + r < p.N;
      } else {
        return row_valid;
      }
    };
    if constexpr (B == 16 && !PipeScheme<M, B, G>::kCpAsyncDecode) {
      // B = 16 except 1x16 g8: register-staged gathers, kLook stages ahead.  At step i
      // the thread issues the gathers of stage i (g = 16: one 256-bit load per 32-byte
      // codeword, one L1TEX request instead of two cp.async) and stores stage i - kLook,
      // gathered kLook steps earlier and summed over the M codebooks, into its A slot.
      // Measured faster than cp.async for g = 16 and slower for 1x16 g8, which keeps
      // the cp.async path below.
      constexpr int kLook = (M == 1) ? 3 : 1;
      uint4 st[kLook + 1][M][4];
      bool alive = true;
      const int nmine = (nks - grp + kDecoderGroups - 1) / kDecoderGroups;  // this group's stages
      for (int base = 0; alive && base < nmine + kLook; base += kLook + 1) {
#pragma unroll
        for (int u = 0; u <= kLook; ++u) {
          const int ki = base + u, kj = ki - kLook;   // this group's stage numbers
          const int i = grp + kDecoderGroups * ki;    // stage gathered now
          const int j = grp + kDecoderGroups * kj;    // stage stored now
          const bool issue = ki < nmine, store = kj >= 0 && kj < nmine;
          const int t = i / kStagesPerTile, within = i % kStagesPerTile, c = t & cs_mask;
          const int sj = j >= 0 ? j % S : 0, uj = j >= 0 ? j / S : 0;
          // wait decisions are made warp-uniform: a warp either goes on or leaves as a whole
          bool ready = true;
          if (issue && within < kDecoderGroups)  // this group's first stage of the tile
            ready = pipe_wait(&cfull[c], static_cast<uint32_t>((t >> cs_log) & 1), abort_flag, p.status,
                              kSitePipeCodes);
          if (ready && store && uj > 0)
            ready = pipe_wait(&empty[sj], static_cast<uint32_t>((uj - 1) & 1), abort_flag, p.status, kSitePipeEmpty);
          if (!__all_sync(0xffffffffu, ready)) {
            *abort_flag = 1u;
            alive = false;
            break;
          }
          if (issue) {
            const uint8_t* cw = smem + L.codes + static_cast<uint32_t>(c) * kCodeTileBytes +
                                code_tile_offset<SC::kTileRowBytes, SC::kSwizzle64>(
                                    r, within * kStageCodeBytes + hf * (kStageCodeBytes / 2));
            gather_stage_b16<M, G>(st[u], cw, row_valid_at(i), p.codebooks, p.cb32 != 0, cb_pol);
            if (within + kDecoderGroups >= kStagesPerTile || i + kDecoderGroups >= nks) {  // its last one
              __syncwarp();  // every lane has read its codes of this tile
              if (lane == 0) mbar_arrive(&cempty[c]);
            }
          }
          if (store) {
            uint4 out[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              uint4 pieces[M];
#pragma unroll
              for (int m = 0; m < M; ++m) pieces[m] = st[(u + 1) % (kLook + 1)][m][cc];
              out[cc] = sum_pieces<M>(pieces);
            }
            if (a_in_tmem) tc_fence_after_sync();  // the stage's release (MMA commit) -> these tcgen05.st
            store_a_half(a_in_tmem, smem, L.a + static_cast<uint32_t>(sj) * (a_in_tmem ? 0u : kABytes),
                                 a_tmem_q + 32u * static_cast<uint32_t>(sj), r, hf, out);
            if (a_in_tmem) {
              tc_fence_before_sync();  // tcgen05.st -> the MMA issuer's reads, through the barrier
            } else {
              fence_proxy_async_smem();
            }
            mbar_arrive(&full[sj]);
          }
        }
      }
    } else {
    if constexpr (kDecoderGroups == 1) {
      // one group: every stage in order (written without the group arithmetic:
      // the compiler schedules this form measurably better for 4x8 g8)
      for (int i = 0; i < nks; ++i) {
        const int t = i / kStagesPerTile, within = i % kStagesPerTile, c = t & cs_mask;
        // wait decisions are made warp-uniform: a warp either goes on or leaves as a whole
        bool ready = true;
        if (within == 0)
          ready = pipe_wait(&cfull[c], static_cast<uint32_t>((t >> cs_log) & 1), abort_flag, p.status,
                            kSitePipeCodes);
        const int s = i % S, u = i / S;
        if (ready && u > 0)
          ready = pipe_wait(&empty[s], static_cast<uint32_t>((u - 1) & 1), abort_flag, p.status, kSitePipeEmpty);
        if (!__all_sync(0xffffffffu, ready)) {
          *abort_flag = 1u;
          break;
        }
        const uint8_t* cw = smem + L.codes + static_cast<uint32_t>(c) * kCodeTileBytes +
                            code_tile_offset<SC::kTileRowBytes, SC::kSwizzle64>(
                                r, within * kStageCodeBytes + hf * (kStageCodeBytes / 2));
        if (a_in_tmem) tc_fence_after_sync();  // the stage's release (MMA commit) -> these tcgen05.st
        decode_half_stage<M, B, G>(a_in_tmem, smem, sbase, L.a + static_cast<uint32_t>(s) * (a_in_tmem ? 0u : kABytes),
                                           a_tmem_q + 32u * static_cast<uint32_t>(s), r, hf, row_valid_at(i), cw,
                                           p.codebooks, smem + L.cb, cb_pol, p.cb_sh);
        if constexpr (B == 16) {
          cp_async_arrive_noinc(&full[s]);  // 1x16 g8: the stage lands by cp.async
        } else if (a_in_tmem) {
          tc_fence_before_sync();  // tcgen05.st -> the MMA issuer's reads, through the barrier
          mbar_arrive(&full[s]);
        } else {
          fence_proxy_async_smem();
          mbar_arrive(&full[s]);
        }
        if (within == kStagesPerTile - 1 || i == nks - 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&cempty[c]);
        }
      }
    } else {
      for (int i = grp; i < nks; i += kDecoderGroups) {
        const int t = i / kStagesPerTile, within = i % kStagesPerTile, c = t & cs_mask;
        // wait decisions are made warp-uniform: a warp either goes on or leaves as a whole
        bool ready = true;
        if (within < kDecoderGroups)  // this group's first stage of the tile
          ready = pipe_wait(&cfull[c], static_cast<uint32_t>((t >> cs_log) & 1), abort_flag, p.status,
                            kSitePipeCodes);
        const int s = i % S, u = i / S;
        if (ready && u > 0)
          ready = pipe_wait(&empty[s], static_cast<uint32_t>((u - 1) & 1), abort_flag, p.status, kSitePipeEmpty);
        if (!__all_sync(0xffffffffu, ready)) {
          *abort_flag = 1u;
          break;
        }
        const uint8_t* cw = smem + L.codes + static_cast<uint32_t>(c) * kCodeTileBytes +
                            code_tile_offset<SC::kTileRowBytes, SC::kSwizzle64>(
                                r, within * kStageCodeBytes + hf * (kStageCodeBytes / 2));
        if (a_in_tmem) tc_fence_after_sync();  // the stage's release (MMA commit) -> these tcgen05.st
        decode_half_stage<M, B, G>(a_in_tmem, smem, sbase, L.a + static_cast<uint32_t>(s) * (a_in_tmem ? 0u : kABytes),
                                           a_tmem_q + 32u * static_cast<uint32_t>(s), r, hf, row_valid_at(i), cw,
                                           p.codebooks, smem + L.cb, cb_pol, p.cb_sh);
        if constexpr (B == 16) {
          cp_async_arrive_noinc(&full[s]);  // 1x16 g8: the stage lands by cp.async
        } else if (a_in_tmem) {
          tc_fence_before_sync();  // tcgen05.st -> the MMA issuer's reads, through the barrier
          mbar_arrive(&full[s]);
        } else {
          fence_proxy_async_smem();
          mbar_arrive(&full[s]);
        }
        if (within + kDecoderGroups >= kStagesPerTile || i + kDecoderGroups >= nks) {  // its last one
          __syncwarp();
          if (lane == 0) mbar_arrive(&cempty[c]);
        }
      }
    }
    }
    }  // kGrad
    asm volatile("cp.async.wait_all;" ::: "memory");
  }

  // ---- epilogue (stream-K kernels finish their pieces above) ------------------------
  if constexpr (!kStreamK) {
  // Decoder warp w reads TMEM lanes 32*(w % 4).. (weight rows) and, with the other
  // warps of its lane quadrant, every (kDecoders / 128)-th 16-column chunk of the batch tile.
  const bool decoder = warp < kDecoders / 32;
  const int q = warp & 3;        // TMEM lane quadrant
  const int cpar = warp >> 2;    // which 16-column chunks
  bool acc_ok = true;
  if (decoder) {
    acc_ok = __all_sync(0xffffffffu, pipe_wait(acc_bar, 0u, abort_flag, p.status, kSitePipeAcc) && !*abort_flag);
    tc_fence_after_sync();
  }
  const int n = n0 + 32 * q + lane;   // output row (input feature k for the gradient)
  const bool n_valid = n < p.rows;
  if (p.SK == 1) {
    if (decoder && acc_ok) {
      // the gradient's scale is inside its A operand and it has no bias
      const float sc = kGrad ? 1.f : (n_valid ? __half2float(p.scales[n]) : 0.f);
      const float bi = (!kGrad && n_valid && p.bias != nullptr) ? __half2float(p.bias[n]) : 0.f;
      for (int c0 = 16 * cpar; c0 < p.BN; c0 += 16 * (kDecoders / 128)) {
        float v[16];
        tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(c0), v);
        if (n_valid) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int b = b0 + c0 + i;
            if (b < p.batch) p.y[static_cast<size_t>(b) * p.rows + n] = __float2half_rn(v[i] * sc + bi);
          }
        }
      }
    }
  } else {
    // Split K: the CTA of rank k owns weight rows [k R, (k + 1) R) of the tile
    // (R = red_rows).  Every CTA stores its fp32 partial of row r into slot
    // (split, r - k R) of the owner's receive buffer (over the stages, which every
    // CTA has stopped using at the first cluster barrier; pitch BN + 4 floats); the
    // owner then sums the SK partials in split order.
    const int SK = p.SK;
    const int R = p.red_rows;
    const int pitch = p.BN + 4;
    tc_fence_before_sync();
    cluster_barrier();  // every CTA's MMAs are done: its stage memory may be overwritten
    if (decoder && acc_ok) {
      const int r = 32 * q + lane;
      const uint32_t owner = static_cast<uint32_t>(r / R);
      const uint32_t slot_row = static_cast<uint32_t>(split * R + (r - static_cast<int>(owner) * R));
      const uint32_t remote_base =
          mapa_shared_cluster(sbase + L.a + slot_row * static_cast<uint32_t>(pitch) * 4u, owner);
      for (int c0 = 16 * cpar; c0 < p.BN; c0 += 16 * (kDecoders / 128)) {
        float v[16];
        tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(c0), v);
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};"
                       ::"r"(remote_base + static_cast<uint32_t>(c0 + i) * 4u), "f"(v[i]), "f"(v[i + 1]),
                       "f"(v[i + 2]), "f"(v[i + 3]) : "memory");
      }
    }
    if (!acc_ok) *abort_flag = 1u;
    cluster_barrier();  // every partial has landed
    if (!*abort_flag) {
      const float* recv = reinterpret_cast<const float*>(smem + L.a);
      const int r_begin = split * R;
      const int rows_owned = max(0, min(kRows, r_begin + R) - r_begin);
      for (int idx = tid; idx < rows_owned * p.BN; idx += kThreads) {
        const int rl = idx % rows_owned;  // owned row (fast index: coalesced y stores)
        const int col = idx / rows_owned;
        const int nn = n0 + r_begin + rl;
        const int b = b0 + col;
        if (nn >= p.rows || b >= p.batch) continue;
        float acc = 0.f;
        for (int j = 0; j < SK; ++j) acc += recv[(j * R + rl) * pitch + col];
        if constexpr (kGrad) {
          p.y[static_cast<size_t>(b) * p.rows + nn] = __float2half_rn(acc);
        } else {
          const float bi = p.bias != nullptr ? __half2float(p.bias[nn]) : 0.f;
          p.y[static_cast<size_t>(b) * p.rows + nn] = __float2half_rn(acc * __half2float(p.scales[nn]) + bi);
        }
      }
    }
  }
  }  // !kStreamK

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
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

// Launch plan: ring depth S and the K split SK (cluster size).  The kernel is bound by
// the decode rate of the SMs it occupies, so the plan spreads row tiles x K splits
// over the SMs: estimated time = waves x (stages per CTA + fixed cost per CTA) + the
// split-K exchange, with the number of co-resident clusters taken from the occupancy
// calculator.  A CTA that allocates tensor memory runs alone on its SM (the
// calculator reports one CTA per SM for such kernels whatever their shared memory),
// so the deepest ring that fits is taken.  The exchange moves 128 x BN fp32 partials
// per CTA through distributed shared memory; measured on B200 it costs about two
// stage times per 16 batch columns, which makes SK = 1 the choice for wide batches.
struct TcPlan {
  int S = 0, SK = 1, ks_per = 0, red_rows = 128, cb_sh = 3, cs_log = 2;
  bool a_tmem = false;
  bool streamk = false;  // stream-K schedule (needs the caller's workspace)
  int sk_ctas = 0, sk_units = 0, sk_unit = 0;
};

constexpr int kPlanFixedStages = 3;     // set-up, pipeline fill and epilogue, in stage times
constexpr int kPlanExchangePer16 = 2;   // split-K exchange, stage times per 16 batch columns
constexpr int kMaxSplit = 16;
// Stream-K: at most this many CTAs (one per SM; B200 has 148), so the workspace size is
// known without a device.  Its overhead over a tile plan, in stage times: the fix-up of
// cut tiles, the four-warp epilogue of every CTA's last piece, the spread of CTA
// finish times that the next launch waits for, and a slower stage loop (measured: 0.85
// to 0.9 us per stage against 0.57 to 0.75 for the same decode in tile plans, with 4x
// the long-scoreboard stalls).  Measured on B200, one launch after another: about
// 45-50 stage times at batch tile 256, about 5 at tile 16, so 8 + BN / 6.  Only the
// input-gradient kernel gains, where its tile plan leaves a mostly empty last wave
// (4096 x 14336 at batch 1024: 448 tiles on 148 SMs, 191-194 -> 177-184 us); the layer
// kernel lost in every measured shape (2x8 11008 x 4096 at batch 256: 37.7 us as 86
// tiles, 50.6 as stream-K; 14336 x 4096 at batch 1024: 147 against 163 us), so the
// cost model offers stream-K to the gradient kernel only, and the layer kernel runs
// it when a caller asks for it (AQLM_SCHEDULE_STREAMK).
constexpr int kMaxSkCtas = 160;
constexpr int kSkOverheadStages = 8;

// Schemes with a stream-K kernel: all but the B = 16 gradient kernels, whose
// register-staged gathers do not fit the 80 registers a thread has with the four
// epilogue warps added (they spilled).
template <int M, int B, int G, bool kGrad>
constexpr bool kStreamKOk = !(kGrad && B == 16);

// Stream-K work units: code tiles of the layer kernel (so no code tile straddles two
// tiles), single stages for the gradient.  0 when the shape cannot use stream-K: the
// A stages would live in tensor memory (its columns hold the second accumulator), or
// nk is not a whole number of units.
template <int M, int B, int G, bool kGrad>
inline int streamk_unit(int nk, int BN) {
  using SC = std::conditional_t<kGrad, GradScheme<M, B, G>, PipeScheme<M, B, G>>;
  if (!kStreamKOk<M, B, G, kGrad>) return 0;
  if (SC::kATmemOk && BN <= 128) return 0;
  return nk % SC::kStagesPerTile == 0 ? SC::kStagesPerTile : 0;
}

// fp32 partial slots of the stream-K schedule with C CTAs: 2 C slots of 128 x BN.
// (The counters live apart, in the kStreamKCounterBytes at the start of a workspace.)
inline size_t streamk_partial_bytes(int C, int BN) {
  return static_cast<size_t>(2 * C) * kRows * static_cast<size_t>(BN) * sizeof(float);
}
static_assert(kStreamKCounterBytes == static_cast<size_t>(kMaxSkCtas) * 4 * sizeof(uint32_t),
              "one counter per (CTA, lane quadrant)");

template <int M, int B, int G, bool kGrad>
using PipeSchemeOf = std::conditional_t<kGrad, GradScheme<M, B, G>, PipeScheme<M, B, G>>;

template <int M, int B, int G, bool kGrad>
inline uint32_t pipe_smem_bytes(int S, int BN, int cb_sh, int cs_log, bool a_tmem, bool streamk = false) {
  using SC = PipeSchemeOf<M, B, G, kGrad>;
  const uint32_t bytes = pipe_layout(S, BN, SC::kCodeTileBytes, SC::kCbBytes * (8u >> cb_sh), 1 << cs_log,
                                     a_tmem ? 0u : kABytes, streamk ? 8 : 1)
                             .total +
                         1024;
  // With A in tensor memory a CTA allocates all 512 columns.  Two such CTAs on one SM
  // (from consecutive launches, or if the layout were small enough) would make the
  // second one's tcgen05.alloc wait for the first, and with split-K clusters two
  // clusters could then wait on each other.  Asking for more than half an SM's shared
  // memory keeps every such CTA alone on its SM.  Stream-K CTAs stay alone too: the
  // schedule spreads the work over one CTA per SM.
  return (a_tmem || streamk) ? std::max(bytes, kSmemLimit / 2 + 1024u) : bytes;
}

// The instantiation a launch runs: A stages in tensor memory or in shared memory, or
// the stream-K kernel.
using PipeKernelFn = void (*)(CUtensorMap, CUtensorMap, PipeParams);
template <int M, int B, int G, bool kGrad>
PipeKernelFn pipe_kernel(bool a_tmem, bool streamk = false) {
  if constexpr (kStreamKOk<M, B, G, kGrad>) {
    if (streamk) return tc_pipe_kernel<M, B, G, kGrad, false, true>;
  }
  if constexpr (PipeSchemeOf<M, B, G, kGrad>::kATmemOk) {
    if (a_tmem) return tc_pipe_kernel<M, B, G, kGrad, true, false>;
  }
  return tc_pipe_kernel<M, B, G, kGrad, false, false>;
}

// rows: output rows (the MMA's M extent); nk: 64-wide reduction stages.
// ws_ok: the caller gave a workspace for the stream-K schedule.  schedule: 0 = the cost
// model picks, 1 = tile plan, 2 = stream-K (cudaErrorInvalidConfiguration if it cannot run).
template <int M, int B, int G, bool kGrad>
cudaError_t plan_pipe(int dev, int rows, int nk, int batch, int BN, bool ws_ok, int schedule, TcPlan* out) {
  constexpr int kSplitAlign = PipeSchemeOf<M, B, G, kGrad>::kSplitAlign;  // split starts keep 16-byte code offsets
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, bool, int>, TcPlan> cache;
  const auto key = std::make_tuple(dev, rows, nk, batch, ws_ok, schedule);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *out = it->second;
      return cudaSuccess;
    }
  }
  // A stages in tensor memory up to batch tile 128.  At 256 the decoders' tcgen05.st
  // competed with the 256-column accumulator (2x8 11008 x 4096 at batch 256: 36.9 ->
  // 58.7 us); below it they save the shared-memory A stores and the MMA's A reads.
  const bool a_tmem = PipeSchemeOf<M, B, G, kGrad>::kATmemOk && BN <= 128;
  auto kern = pipe_kernel<M, B, G, kGrad>(a_tmem);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemLimit));
  if (e != cudaSuccess) return e;
  const int cmax = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess
                       ? kMaxSplit : 8;
  cudaGetLastError();

  const int row_tiles = (rows + kRows - 1) / kRows;
  const int batch_tiles = (batch + BN - 1) / BN;
  const long long clusters = static_cast<long long>(row_tiles) * batch_tiles;
  // codebook copies (2x8 g8) and code-tile slots: the most copies that still leave
  // room for three stages, with four code slots if they fit, else two (a code tile
  // holds four 2x8 stages, so two slots still keep the decoders fed).  Measured on
  // 11008 x 4096: 8 copies made batch 4-64 11 % faster, but at batch 256 with four
  // code slots they left room for two stages only and the kernel ran 1.8x slower.
  int cb_sh = 3, cs_log = 2;
  if constexpr (PipeSchemeOf<M, B, G, kGrad>::kCbMaxReplicas > 1) {
    bool found = false;
    for (int sh = 0; sh < 3 && !found; ++sh)
      for (int cs = 2; cs >= 1 && !found; --cs)
        if (pipe_smem_bytes<M, B, G, kGrad>(3, BN, sh, cs, a_tmem) <= kSmemLimit) {
          cb_sh = sh;
          cs_log = cs;
          found = true;
        }
  }
  TcPlan best;
  best.cb_sh = cb_sh;
  best.cs_log = cs_log;
  best.a_tmem = a_tmem;
  long long best_cost = -1;
  for (int S = 6; S >= 2; --S) {
    static_assert(6 <= kMaxATmemStages, "A stages in tensor memory");
    const uint32_t smem = pipe_smem_bytes<M, B, G, kGrad>(S, BN, cb_sh, cs_log, a_tmem);
    if (smem > kSmemLimit) continue;
    // shared stage memory (the split-K exchange reuses it): B tiles, plus A when A is in
    // shared memory
    const uint32_t kAStage = a_tmem ? 0u : kABytes;
    const uint32_t stage_bytes = static_cast<uint32_t>(S) * (kAStage + static_cast<uint32_t>(BN) * 128u);
    for (int SK = 1; SK <= cmax; ++SK) {
      int per = (nk + SK - 1) / SK;
      per = (per + kSplitAlign - 1) / kSplitAlign * kSplitAlign;
      if (static_cast<long long>(SK - 1) * per >= nk) continue;  // a split would be empty
      const int R = (kRows + SK - 1) / SK;
      if (SK > 1 && static_cast<uint32_t>(SK * R * (BN + 4)) * 4u > stage_bytes) continue;
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 1;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = static_cast<unsigned>(SK);
      cfg.gridDim = dim3(1, 1, static_cast<unsigned>(SK));
      cfg.blockDim = dim3(PipeShape<M, B, G, kGrad>::kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int active = 0;
      if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess || active <= 0) {
        cudaGetLastError();
        continue;
      }
      const long long waves = (clusters + active - 1) / active;
      const long long exchange = SK > 1 ? 16 * (1 + kPlanExchangePer16 * (BN / 16)) + SK : 0;
      const long long cost = waves * 16 * (per + kPlanFixedStages) + exchange;
      if (best_cost < 0 || cost < best_cost) {
        best_cost = cost;
        best.S = S;
        best.SK = SK;
        best.ks_per = per;
        best.red_rows = R;
      }
    }
  }
  if (best_cost < 0) return cudaErrorNotSupported;
  // Stream-K: one CTA per SM over (tile, stage) units, so no SM idles when the tiles do
  // not divide evenly over the SMs.  Taken when its estimate, overhead included
  // (kSkOverheadStages), beats the tile plan's.
  const int unit = streamk_unit<M, B, G, kGrad>(nk, BN);
  if (ws_ok && unit > 0 && (schedule == 2 || (schedule == 0 && kGrad))) {
    auto kern_sk = pipe_kernel<M, B, G, kGrad>(false, true);
    int sms = 0;
    if (cudaFuncSetAttribute(kern_sk, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemLimit)) ==
            cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) {
      const long long units = clusters * (nk / unit);
      const int C = static_cast<int>(std::min<long long>({static_cast<long long>(sms), units, kMaxSkCtas}));
      for (int S = 6; S >= 2 && C > 0; --S) {
        const uint32_t smem = pipe_smem_bytes<M, B, G, kGrad>(S, BN, cb_sh, cs_log, false, true);
        if (smem > kSmemLimit) continue;
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern_sk, PipeShape<M, B, G, kGrad, true>::kThreads,
                                                          smem) != cudaSuccess ||
            per_sm < 1)
          continue;
        const long long per = (units + C - 1) / C * unit;
        const long long cost = 16 * (per + kPlanFixedStages + kSkOverheadStages + BN / 6);
        if (cost < best_cost || schedule == 2) {
          best.streamk = true;
          best.S = S;
          best.SK = 1;
          best.ks_per = 0;
          best.red_rows = kRows;
          best.a_tmem = false;
          best.sk_ctas = C;
          best.sk_units = static_cast<int>(units);
          best.sk_unit = unit;
        }
        break;  // the deepest ring that fits
      }
    }
    cudaGetLastError();
  }
  if (schedule == 2 && !best.streamk) return cudaErrorInvalidConfiguration;
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = best;
  *out = best;
  return cudaSuccess;
}

// Encodes the two tensor maps and launches one (row tile, batch tile, split) grid.
//   x_src  [batch, red] fp16: x (layer, red = K) or dy (gradient, red = N)
//   codes  [N, row_bytes] bytes; box {box_x, box_rows}
template <int M, int B, int G, bool kGrad>
cudaError_t launch_pipe_kernel(const void* x_src, int red, const void* codes, size_t row_bytes, int N,
                               uint32_t box_x, uint32_t box_rows, PipeParams p, const TcPlan& plan,
                               uint32_t* sk_count, float* sk_part, cudaStream_t stream) {
  EncodeTiledFn encode = encode_tiled();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap x_map, code_map;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(red), static_cast<cuuint64_t>(p.batch)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(red) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kStageK), static_cast<cuuint32_t>(p.BN)};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&x_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(x_src), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
    const cuuint32_t box[2] = {box_x, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    // layer kernel: the 64-byte swizzle on 64-byte tile rows, so the decoders' reads
    // of one chunk of 32 consecutive rows spread over the banks (48-byte rows, M = 3,
    // are not swizzled).  Gradient kernel: unswizzled (a warp reads contiguous bytes).
    const bool swz = !kGrad && box_x == 64;
    if (encode(&code_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swz ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(p.BN)) cols <<= 1;
  p.acc_cols = static_cast<int>(cols);
  // A stages in tensor memory: the accumulator's 256 columns, then 32 a stage
  if (plan.a_tmem) cols = 512;
  // stream-K: two accumulators
  if (plan.streamk) cols *= 2;
  p.tmem_cols = cols;
  const int row_tiles = (p.rows + kRows - 1) / kRows;
  const int batch_tiles = (p.batch + p.BN - 1) / p.BN;
  p.batch_tiles = batch_tiles;
  if (plan.streamk) {
    p.sk_ctas = plan.sk_ctas;
    p.sk_units = plan.sk_units;
    p.sk_unit = plan.sk_unit;
    p.sk_count = sk_count;
    p.sk_part = sk_part;
  }
  p.S = plan.S;
  p.SK = plan.SK;
  p.ks_per = plan.ks_per;
  p.red_rows = plan.red_rows;
  p.cb_sh = plan.cb_sh;
  p.cs_log = plan.cs_log;
  p.cb32 = (reinterpret_cast<uintptr_t>(p.codebooks) & 31u) == 0 ? 1 : 0;
  const uint32_t smem =
      pipe_smem_bytes<M, B, G, kGrad>(plan.S, p.BN, plan.cb_sh, plan.cs_log, plan.a_tmem, plan.streamk);
  auto kern = pipe_kernel<M, B, G, kGrad>(plan.a_tmem, plan.streamk);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemLimit));
  if (e != cudaSuccess) return e;
  if (plan.SK > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = static_cast<unsigned>(plan.SK);
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = plan.streamk ? dim3(static_cast<unsigned>(plan.sk_ctas), 1, 1)
                             : dim3(static_cast<unsigned>(row_tiles), static_cast<unsigned>(batch_tiles),
                                    static_cast<unsigned>(plan.SK));
  cfg.blockDim = dim3(plan.streamk ? PipeShape<M, B, G, kGrad, true>::kThreads : PipeShape<M, B, G, kGrad>::kThreads,
                      1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, x_map, code_map, p);
}

// Batch tile: the batch rounded up to a multiple of 16, at most 256 (the MMA's N).
inline int pipe_batch_tile(int batch) { return std::min(256, (batch + 15) / 16 * 16); }

// Partial-slot bytes the stream-K schedule needs for (rows, nk, batch) on any device
// (at most kMaxSkCtas CTAs); 0 when the shape cannot use it.
template <int M, int B, int G, bool kGrad>
size_t pipe_partial_bytes(int rows, int nk, int batch) {
  const int BN = pipe_batch_tile(batch);
  const int unit = streamk_unit<M, B, G, kGrad>(nk, BN);
  if (unit == 0) return 0;
  const long long tiles = static_cast<long long>((rows + kRows - 1) / kRows) * ((batch + BN - 1) / BN);
  const long long units = tiles * (nk / unit);
  return streamk_partial_bytes(static_cast<int>(std::min<long long>(units, kMaxSkCtas)), BN);
}

template <int M, int B, int G>
cudaError_t launch_pipe(const Problem& pr, uint32_t* status, cudaStream_t stream) {
  using SC = PipeScheme<M, B, G>;
  if (!tc_pipelined_shape(M, B, G, pr.K)) return cudaErrorNotSupported;
  if (!encode_tiled()) return cudaErrorNotSupported;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int BN = pipe_batch_tile(pr.batch);
  const size_t part_need = pipe_partial_bytes<M, B, G, false>(pr.N, pr.K / kStageK, pr.batch);
  const bool ws_ok = part_need > 0 && pr.sk_count != nullptr && pr.sk_part != nullptr && pr.sk_part_bytes >= part_need;
  TcPlan plan;
  e = plan_pipe<M, B, G, false>(dev, pr.N, pr.K / kStageK, pr.batch, BN, ws_ok, pr.schedule, &plan);
  if (e != cudaSuccess) return e;
  PipeParams p{};
  p.codebooks = static_cast<const __half*>(pr.codebooks);
  p.scales = static_cast<const __half*>(pr.scales);
  p.bias = static_cast<const __half*>(pr.bias);
  p.y = static_cast<__half*>(pr.y);
  p.K = pr.K;
  p.N = pr.N;
  p.batch = pr.batch;
  p.rows = pr.N;
  p.BN = BN;
  p.nk = pr.K / kStageK;
  p.status = status;
  const size_t row_bytes = static_cast<size_t>(pr.K / G) * M * SC::kCodeBytes;
  return launch_pipe_kernel<M, B, G, false>(pr.x, pr.K, pr.codes, row_bytes, pr.N,
                                            static_cast<uint32_t>(SC::kTileRowBytes), static_cast<uint32_t>(kRows), p,
                                            plan, pr.sk_count, pr.sk_part, stream);
}

template <int M, int B, int G>
cudaError_t launch_grad(const GradProblem& pr, uint32_t* status, cudaStream_t stream) {
  using SC = GradScheme<M, B, G>;
  if (!grad_shape_supported(M, B, G, pr.K, pr.N)) return cudaErrorNotSupported;
  if (!encode_tiled()) return cudaErrorNotSupported;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int BN = pipe_batch_tile(pr.batch);
  const int nk = (pr.N + kStageK - 1) / kStageK;
  const size_t part_need = pipe_partial_bytes<M, B, G, true>(pr.K, nk, pr.batch);
  const bool ws_ok = part_need > 0 && pr.sk_count != nullptr && pr.sk_part != nullptr && pr.sk_part_bytes >= part_need;
  TcPlan plan;
  e = plan_pipe<M, B, G, true>(dev, pr.K, nk, pr.batch, BN, ws_ok, pr.schedule, &plan);
  if (e != cudaSuccess) return e;
  PipeParams p{};
  p.codebooks = static_cast<const __half*>(pr.codebooks);
  p.scales = static_cast<const __half*>(pr.scales);
  p.bias = nullptr;
  p.y = static_cast<__half*>(pr.dx);
  p.K = pr.K;
  p.N = pr.N;
  p.batch = pr.batch;
  p.rows = pr.K;
  p.BN = BN;
  p.nk = nk;
  p.status = status;
  const size_t row_bytes = static_cast<size_t>(pr.K / G) * M * SC::kCodeBytes;
  return launch_pipe_kernel<M, B, G, true>(pr.dy, pr.N, pr.codes, row_bytes, pr.N,
                                           static_cast<uint32_t>(SC::kBoxBytes), static_cast<uint32_t>(kStageK), p,
                                           plan, pr.sk_count, pr.sk_part, stream);
}

struct PipeLauncher {
  template <int M, int B, int G>
  static cudaError_t run(const Problem& p, uint32_t* status, cudaStream_t stream) {
    return launch_pipe<M, B, G>(p, status, stream);
  }
};

struct GradLauncher {
  template <int M, int B, int G>
  static cudaError_t run(const GradProblem& p, uint32_t* status, cudaStream_t stream) {
    return launch_grad<M, B, G>(p, status, stream);
  }
};

struct PipeWorkspace {
  template <int M, int B, int G>
  static size_t run(int K, int N, int batch) {
    if (!tc_pipelined_shape(M, B, G, K)) return 0;
    return pipe_partial_bytes<M, B, G, false>(N, K / kStageK, batch);
  }
};

struct GradWorkspace {
  template <int M, int B, int G>
  static size_t run(int K, int N, int batch) {
    if (!grad_shape_supported(M, B, G, K, N)) return 0;
    return pipe_partial_bytes<M, B, G, true>(K, (N + kStageK - 1) / kStageK, batch);
  }
};

}  // namespace

cudaError_t launch_tc_pipelined(const Problem& p, uint32_t* status, cudaStream_t stream) {
  return dispatch_scheme<PipeLauncher>(p.M, p.B, p.g, cudaErrorNotSupported, p, status, stream);
}

cudaError_t launch_input_grad(const GradProblem& p, uint32_t* status, cudaStream_t stream) {
  return dispatch_scheme<GradLauncher>(p.M, p.B, p.g, cudaErrorNotSupported, p, status, stream);
}

size_t tc_pipe_partial_bytes(int M, int B, int g, int K, int N, int batch) {
  return dispatch_scheme<PipeWorkspace>(M, B, g, size_t{0}, K, N, batch);
}

size_t input_grad_partial_bytes(int M, int B, int g, int K, int N, int batch) {
  return dispatch_scheme<GradWorkspace>(M, B, g, size_t{0}, K, N, batch);
}

}  // namespace aqlm
