// Lookup-table construction shared by the two lookup-table GEMV kernels
// (single-layer and grouped) for codebooks of 256 entries (B = 8), any M = 1..4
// and g = 8 or 16: the "fast lookup, no per-element dequantization" route of the
// inference-research record "AQLM (additive / multi-codebook quantization)",
// section "Kernels".
//
// A code row of G groups x M codebooks is G M bytes, byte b being the code of
// codebook m = b mod M in group j = b / M.  The kernels cut it into slices of 128
// bytes (b0 = 128 s); the table of a slice holds, for every byte b of it and every
// entry i, T[b][i] = x_j . C_m[i], so that a row's partial over the slice is the plain
// sum over its 128 bytes of T[b][code byte b], whatever M is.
//
// Stacked build (every scheme).  One tcgen05.mma chain computes the whole table:
// the M codebooks sit side by side along K (B row i = C_0[i] | C_1[i] | ... , K = g M
// rounded up to 16 per MMA step), and A row rho holds x_j in codebook m's K slot for
// the byte b = b0 + beta(rho) (zeros elsewhere), so D[rho][i] = T[b][i]: one TMEM lane
// per byte of the slice.  beta puts the bytes b = q (mod 4) in lane quadrant q and the
// byte of code word l in lane l of it, so that all 16 warps convert (a warp reads only
// its own lane quadrant) and their 16-bit table stores hit 32 different banks.
//
// 2x8 g8 (the tuned build): A rows are x groups (two per code word), one MMA per
// codebook, and a lane packs both codebooks' entries of its group into one word.
//
// Table layout (what the lookups read): byte b goes to half b mod 2 of the word of
// pair p = b / 2, in word column p / 2 (p even) or 32 + p / 2 (p odd) of each
// entry's 64-word (256-byte) row.
#pragma once

#include "aqlm_device.cuh"

namespace aqlm {
namespace lut {

constexpr uint32_t kAOpBytes = 128u * 32u;  // 128 rows x (16 fp16): one K step of A
constexpr uint32_t kBOpBytes = 256u * 32u;  // 256 entries x (16 fp16): one K step of B
constexpr uint32_t kTableBytes = 256u * 64u * 4u;

// No-swizzle K-major operand layout: 8-row x 16-byte core matrices, the two K
// halves 128 bytes apart, consecutive 8-row groups 256 bytes apart.
__host__ __device__ inline uint32_t kmajor_offset(int row, int khalf) {
  return static_cast<uint32_t>((row >> 3) * 256 + khalf * 128 + (row & 7) * 16);
}
// Its UMMA shared-memory descriptor (leading byte offset 128, stride byte offset 256,
// layout type 0 = no swizzle, base offset 0).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t smem_byte_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_byte_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;
  d |= static_cast<uint64_t>(256u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

// MMA K steps (16 wide) of the stacked build: the M codebooks' g-wide codewords.
__host__ __device__ inline int stacked_ksteps(int M, int g) { return (M * g + 15) / 16; }

// K-major no-swizzle layout of ks K steps: 8-row x 16-byte core matrices, the 8-wide
// K chunks kc 128 bytes apart, consecutive 8-row groups 256 ks bytes apart.
__host__ __device__ inline uint32_t stacked_offset(int row, int kc, int ks) {
  return static_cast<uint32_t>((row >> 3) * (256 * ks) + kc * 128 + (row & 7) * 16);
}
// Descriptor of K step t of such an operand (leading byte offset 128, stride byte
// offset 256 ks; pass the operand base + 256 t).
__device__ __forceinline__ uint64_t stacked_desc(uint32_t smem_byte_addr, int ks) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_byte_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;
  d |= static_cast<uint64_t>((256u * static_cast<uint32_t>(ks)) >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

// Byte of the slice (0..127) held by A row / TMEM lane rho.
__host__ __device__ inline int stacked_row_byte(int rho) { return 4 * (rho & 31) + (rho >> 5); }

// A operand of slice s (cp.async, the caller commits): 128 rows x ks K steps.
template <int kNThreads>
__device__ __forceinline__ void load_x_stacked(const __half* x, int G, int M, int g, int s, uint32_t dst, int tid) {
  const int ks = stacked_ksteps(M, g);
  const int cpg = g >> 3;  // 8-wide chunks per codeword
  for (int idx = tid; idx < 128 * 2 * ks; idx += kNThreads) {
    const int rho = idx & 127, kc = idx >> 7;
    const int b = s * 128 + stacked_row_byte(rho);
    const int j = b / M, m = b - j * M;
    const int part = kc - m * cpg;
    const bool valid = j < G && part >= 0 && part < cpg;
    cp_async_16_zfill(dst + stacked_offset(rho, kc, ks),
                      valid ? static_cast<const void*>(x + static_cast<size_t>(j) * g + 8 * part)
                            : static_cast<const void*>(x),
                      valid ? 16u : 0u);
  }
}

// B operand (cp.async, the caller commits): 256 entry rows x ks K steps, entry i =
// C_0[i] | C_1[i] | ... | C_{M-1}[i] | zeros.
template <int kNThreads>
__device__ __forceinline__ void load_codebooks_stacked(const __half* codebooks, int M, int g, uint32_t dst, int tid) {
  const int ks = stacked_ksteps(M, g);
  const int cpg = g >> 3;
  for (int idx = tid; idx < 256 * 2 * ks; idx += kNThreads) {
    const int e = idx & 255, kc = idx >> 8;
    const int m = kc / cpg, part = kc - m * cpg;
    const bool valid = m < M;
    cp_async_16_zfill(dst + stacked_offset(e, kc, ks),
                      valid ? static_cast<const void*>(codebooks + (static_cast<size_t>(m) * 256 + e) * g + 8 * part)
                            : static_cast<const void*>(codebooks),
                      valid ? 16u : 0u);
  }
}

// The MMA chain of the stacked build (one thread): D[0, 256) = A . B^T over ks steps.
__device__ __forceinline__ void mma_stacked(uint32_t tmem, uint32_t a_addr, uint32_t b_addr, int ks, uint32_t idesc) {
  for (int t = 0; t < ks; ++t)
    umma_f16_ss(tmem, stacked_desc(a_addr + 256u * static_cast<uint32_t>(t), ks),
                stacked_desc(b_addr + 256u * static_cast<uint32_t>(t), ks), idesc, t > 0 ? 1u : 0u);
}

// TMEM -> shared-memory table of the stacked build, by 16 warps: warp w reads lane
// quadrant q = w mod 4 (bytes b = 4 l + q) for entries 64 (w / 4) .. + 63.  Byte b is
// half q mod 2 of the word of pair 2 l + q / 2, i.e. word column 32 (q / 2) + l.
// Every byte of the slice gets its entries, also the zero-filled bytes past the row
// end (their A rows are zero, so are their entries; a skipped entry would keep an
// older table's value).
__device__ __forceinline__ void store_table_stacked(uint32_t tmem, int warp, int lane, uint8_t* table) {
  const int qd = warp & 3, sub = warp >> 2;
  const int col = 32 * (qd >> 1) + lane;
  uint16_t* t16 = reinterpret_cast<uint16_t*>(table) + (qd & 1);
  const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    float v[16];
    tmem_ld_32x32b_x16(tmem + lane_base + static_cast<uint32_t>(64 * sub + 16 * h), v);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int i = 64 * sub + 16 * h + e;
      t16[(i * 64 + col) * 2] = __half_as_ushort(__float2half_rn(v[e]));
    }
  }
}

// TMEM -> shared-memory table of a 2x8 g8 slice (64 groups, codebook 0 at columns
// [0, 256), codebook 1 at [256, 512)), by 16 warps.  The A rows hold group
// 2 (rho mod 32) + (rho / 32 mod 2), rows 64-127 repeating rows 0-63, so TMEM lane
// rho carries both codebooks of the groups in word column rho mod 64: each lane packs
// the pair (T_0, T_1) of its group into one word, and warp w reads lane quadrant
// w mod 4 for 32 entries.
__device__ __forceinline__ void store_table_2x8(uint32_t tmem, int warp, int lane, uint8_t* table) {
  const int qd = warp & 3;
  const int col = 32 * (qd & 1) + lane;               // word column = rho mod 64
  const int i0 = 32 * (2 * (warp >> 2) + (qd >> 1));  // 32 table entries per warp
  const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
  uint32_t* t32 = reinterpret_cast<uint32_t*>(table);
  uint32_t r0[32], r1[32];
  tmem_ld_32x32b_x32(tmem + lane_base + static_cast<uint32_t>(i0), r0);
  tmem_ld_32x32b_x32(tmem + lane_base + 256u + static_cast<uint32_t>(i0), r1);
#pragma unroll
  for (int j = 0; j < 32; ++j) t32[(i0 + j) * 64 + col] = f2_to_h2_rn(__uint_as_float(r0[j]), __uint_as_float(r1[j]));
}

}  // namespace lut
}  // namespace aqlm
