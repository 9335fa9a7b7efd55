// AQLM weight-only linear layer on the host CPU (libaqlm_cpu.so; contract in
// include/aqlm_cpu.h).
//
//   y = x . W^T . diag(s) + bias,   W[n, j*g + t] = sum_m C_m[codes[n, j, m]][t]
//
// Three methods:
//   * lookup tables (B = 8): the route of the inference-research record "AQLM
//     (additive / multi-codebook quantization)", section "Kernels".  For a K slice of
//     kSlice groups, T[j][m][b][i] = x_b[j] . C_m[i] for all 256 entries i (g fused
//     multiply-adds per 8 or 16 entries); then every output row adds M table values
//     per group (16 of them per gather instruction with AVX-512).  Threads take
//     slices (static schedule) and keep a partial sum per output; the partials are
//     added in thread order at the end, so the table is built once per slice
//     whatever N is.
//   * decode + dot: each thread decodes blocks of 4 output rows to fp32 (codeword
//     pieces converted with F16C and added in codebook order) and takes the dot
//     products with every batch row (AVX2 FMA, 4 accumulators).
//   * fused decode + dot (AVX-512): 16 weights of a row are decoded in a register and
//     multiplied into register accumulators for up to 8 batch rows and 2 to 8 output
//     rows at once; nothing decoded is stored.
// Which runs: with AVX-512, the lookup tables for B = 8 at batch 1 and the fused
// method otherwise; without it, the lookup tables for B = 8 at batch <= 8 and decode
// + dot otherwise.  (On a Xeon host with AVX-512 the lookups' gathers beat the fused
// decode only at batch 1, where a table entry serves one product.)
// fp32 accumulation everywhere; y = fp16_rne(s_n * acc + bias_n).
//
// The SIMD functions carry target attributes and run only when the CPU reports the
// instruction sets they use; otherwise portable scalar versions of the lookup and
// decode + dot loops run.  A process-wide cap (aqlm_cpu_set_max_simd_level) selects
// a lower level on such a CPU too, for tests and comparisons.
#include <immintrin.h>
#include <omp.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <type_traits>
#include <vector>

#include "aqlm_cpu.h"

namespace {

constexpr int kSlice = 16;     // groups per lookup-table slice (tables of 16 KB per codebook fit L1)
constexpr int kLutMaxBatch = 8;
constexpr int kRowBlock = 4;    // rows decoded together in the decode + dot method
constexpr int kPrefetchRows = 32;  // lookup rows: codes requested this many rows ahead

// ---------------------------------------------------------------------------
// binary16 <-> binary32 for the scalar code (IEEE 754: 1 sign, 5 exponent bits
// with bias 15, 10 fraction bits).
// ---------------------------------------------------------------------------
float half_to_float(uint16_t h) {
  const uint32_t sign = static_cast<uint32_t>(h & 0x8000u) << 16;
  const uint32_t e = (h >> 10) & 31u, f = h & 1023u;
  uint32_t bits;
  if (e == 31) {
    bits = sign | 0x7F800000u | (f << 13);            // inf / nan
  } else if (e != 0) {
    bits = sign | ((e + 112u) << 23) | (f << 13);      // normal: rebias 15 -> 127
  } else if (f == 0) {
    bits = sign;                                       // +-0
  } else {
    int shift = 0;                                     // subnormal: normalise
    uint32_t m = f;
    while (!(m & 1024u)) {
      m <<= 1;
      ++shift;
    }
    bits = sign | (static_cast<uint32_t>(113 - shift) << 23) | ((m & 1023u) << 13);
  }
  float out;
  std::memcpy(&out, &bits, 4);
  return out;
}

uint16_t float_to_half(float v) {
  uint32_t x;
  std::memcpy(&x, &v, 4);
  const uint16_t sign = static_cast<uint16_t>((x >> 16) & 0x8000u);
  const uint32_t ax = x & 0x7FFFFFFFu;
  if (ax >= 0x7F800000u) return sign | 0x7C00u | (ax > 0x7F800000u ? 0x200u : 0u);
  const int e = static_cast<int>(ax >> 23) - 127;
  if (e > 15) return sign | 0x7C00u;                   // overflows to infinity
  // value = mant * 2^(e - 23) with the implicit bit; binary16 keeps 10 fraction
  // bits for e >= -14 and fewer below (subnormals)
  const uint32_t mant = (ax & 0x7FFFFFu) | (e > -127 ? 0x800000u : 0u);
  const int drop = (e >= -14) ? 13 : 13 + (-14 - e);
  if (drop > 24) return sign;                          // below half the smallest subnormal
  const uint32_t q = mant >> drop;
  const uint32_t rem = mant & ((1u << drop) - 1u), half = 1u << (drop - 1);
  uint32_t r = q + ((rem > half || (rem == half && (q & 1u))) ? 1u : 0u);
  if (e >= -14) {
    // normal: r holds 1.fraction (11 bits), a carry may bump the exponent
    const uint32_t he = static_cast<uint32_t>(e + 15);
    return static_cast<uint16_t>(sign | ((he << 10) + (r - 1024u)));
  }
  return static_cast<uint16_t>(sign | r);              // subnormal (r = 1024 means 2^-14)
}

bool cpu_has_avx2() {
  static const bool ok = __builtin_cpu_supports("avx2") && __builtin_cpu_supports("fma") &&
                         __builtin_cpu_supports("f16c");
  return ok;
}

bool cpu_has_avx512() {
  static const bool ok = cpu_has_avx2() && __builtin_cpu_supports("avx512f") &&
                         __builtin_cpu_supports("avx512bw") && __builtin_cpu_supports("avx512vl");
  return ok;
}

constexpr int kMaxSimd = 2;
std::atomic<int> g_max_simd{kMaxSimd};

// 0 = scalar, 1 = AVX2 + FMA + F16C, 2 = AVX-512 (F, BW, VL) as well: what the CPU
// has, capped by aqlm_cpu_set_max_simd_level.
int simd_level() {
  const int hw = cpu_has_avx512() ? 2 : cpu_has_avx2() ? 1 : 0;
  return std::min(hw, g_max_simd.load());
}

struct Layer {
  const uint16_t* x;
  const uint8_t* codes;   // raw bytes
  const uint16_t* cb;
  const uint16_t* scales;
  const uint16_t* bias;
  uint16_t* y;
  int M, B, g, K, N, batch, G, cbytes;
};

inline uint32_t code_of(const Layer& L, int64_t n, int64_t j, int m) {
  const int64_t idx = (n * L.G + j) * L.M + m;
  return L.cbytes == 1 ? L.codes[idx] : reinterpret_cast<const uint16_t*>(L.codes)[idx];
}

// ---------------------------------------------------------------------------
// lookup-table method
// ---------------------------------------------------------------------------
// ct: fp32 codebooks transposed to [m][t][256] (entries contiguous for the build).
void transpose_codebooks(const Layer& L, std::vector<float>& ct) {
  ct.assign(static_cast<size_t>(L.M) * L.g * 256, 0.f);
  for (int m = 0; m < L.M; ++m)
    for (int i = 0; i < 256; ++i)
      for (int t = 0; t < L.g; ++t)
        ct[(static_cast<size_t>(m) * L.g + t) * 256 + i] =
            half_to_float(L.cb[(static_cast<size_t>(m) * 256 + i) * L.g + t]);
}

// T[(jj * M + m) * batch + b][i] for the groups j0 .. j0 + nj - 1.
void build_tables_scalar(const Layer& L, const float* xf, const float* ct, int j0, int nj, float* T) {
  for (int jj = 0; jj < nj; ++jj)
    for (int m = 0; m < L.M; ++m)
      for (int b = 0; b < L.batch; ++b) {
        float* row = T + (static_cast<size_t>(jj * L.M + m) * L.batch + b) * 256;
        const float* xv = xf + static_cast<size_t>(b) * L.K + static_cast<size_t>(j0 + jj) * L.g;
        for (int i = 0; i < 256; ++i) {
          float acc = 0.f;
          for (int t = 0; t < L.g; ++t) acc += xv[t] * ct[(static_cast<size_t>(m) * L.g + t) * 256 + i];
          row[i] = acc;
        }
      }
}

__attribute__((target("avx2,fma,f16c")))
void build_tables_avx2(const Layer& L, const float* xf, const float* ct, int j0, int nj, float* T) {
  for (int jj = 0; jj < nj; ++jj)
    for (int m = 0; m < L.M; ++m)
      for (int b = 0; b < L.batch; ++b) {
        float* row = T + (static_cast<size_t>(jj * L.M + m) * L.batch + b) * 256;
        const float* xv = xf + static_cast<size_t>(b) * L.K + static_cast<size_t>(j0 + jj) * L.g;
        const float* cm = ct + static_cast<size_t>(m) * L.g * 256;
        for (int i = 0; i < 256; i += 16) {
          __m256 a0 = _mm256_setzero_ps(), a1 = _mm256_setzero_ps();
          for (int t = 0; t < L.g; ++t) {
            const __m256 xt = _mm256_set1_ps(xv[t]);
            a0 = _mm256_fmadd_ps(xt, _mm256_loadu_ps(cm + t * 256 + i), a0);
            a1 = _mm256_fmadd_ps(xt, _mm256_loadu_ps(cm + t * 256 + i + 8), a1);
          }
          _mm256_storeu_ps(row + i, a0);
          _mm256_storeu_ps(row + i + 8, a1);
        }
      }
}

// partial[b * N + n] += sum over the slice's groups and codebooks of the table values.
template <int MM>
void lookup_rows(const Layer& L, const float* T, int j0, int nj, float* partial) {
  const int M = MM > 0 ? MM : L.M;
  const int stride = M * nj;  // code bytes of the slice in a row
  const int64_t row_bytes = static_cast<int64_t>(L.G) * M;
  for (int64_t n = 0; n < L.N; ++n) {
    const uint8_t* c = L.codes + (n * L.G + j0) * M;
    if (n + kPrefetchRows < L.N) {  // the slice's codes kPrefetchRows rows ahead
      const char* ahead = reinterpret_cast<const char*>(c + kPrefetchRows * row_bytes);
      __builtin_prefetch(ahead);
      __builtin_prefetch(ahead + stride - 1);
    }
    for (int b = 0; b < L.batch; ++b) {
      const float* Tb = T + static_cast<size_t>(b) * 256;
      const size_t step = static_cast<size_t>(L.batch) * 256;  // next (group, codebook) table
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      int k = 0;
      for (; k + 4 <= stride; k += 4) {
        a0 += Tb[(k + 0) * step + c[k + 0]];
        a1 += Tb[(k + 1) * step + c[k + 1]];
        a2 += Tb[(k + 2) * step + c[k + 2]];
        a3 += Tb[(k + 3) * step + c[k + 3]];
      }
      for (; k < stride; ++k) a0 += Tb[k * step + c[k]];
      partial[static_cast<size_t>(b) * L.N + n] += (a0 + a1) + (a2 + a3);
    }
  }
}

// The same tables built 16 entries per instruction; per entry the same fused
// multiply-adds in the same order as build_tables_avx2, so the values agree.
__attribute__((target("avx512f,avx512bw,avx512vl,avx2,fma,f16c")))
void build_tables_avx512(const Layer& L, const float* xf, const float* ct, int j0, int nj, float* T) {
  for (int jj = 0; jj < nj; ++jj)
    for (int m = 0; m < L.M; ++m)
      for (int b = 0; b < L.batch; ++b) {
        float* row = T + (static_cast<size_t>(jj * L.M + m) * L.batch + b) * 256;
        const float* xv = xf + static_cast<size_t>(b) * L.K + static_cast<size_t>(j0 + jj) * L.g;
        const float* cm = ct + static_cast<size_t>(m) * L.g * 256;
        for (int i = 0; i < 256; i += 32) {
          __m512 a0 = _mm512_setzero_ps(), a1 = _mm512_setzero_ps();
          for (int t = 0; t < L.g; ++t) {
            const __m512 xt = _mm512_set1_ps(xv[t]);
            a0 = _mm512_fmadd_ps(xt, _mm512_loadu_ps(cm + t * 256 + i), a0);
            a1 = _mm512_fmadd_ps(xt, _mm512_loadu_ps(cm + t * 256 + i + 16), a1);
          }
          _mm512_storeu_ps(row + i, a0);
          _mm512_storeu_ps(row + i + 16, a1);
        }
      }
}

// lookup_rows with 16 table reads per gather instruction.  A row's codes of the
// slice are M * nj consecutive bytes (at most 64, NV vectors of 16); lane l of vector
// v reads table (16 v + l) at the entry its code names, so the index is
// (16 v + l) * batch * 256 + code and the base pointer selects the batch row.
template <int NV>
__attribute__((target("avx512f,avx512bw,avx512vl,avx2,fma,f16c")))
void lookup_rows_avx512(const Layer& L, const float* T, int j0, int nj, float* partial) {
  const int stride = L.M * nj;
  const int step = L.batch * 256;
  const __m512i lane = _mm512_set_epi32(15, 14, 13, 12, 11, 10, 9, 8, 7, 6, 5, 4, 3, 2, 1, 0);
  __m512i off[NV];
  __mmask16 msk[NV];
  for (int v = 0; v < NV; ++v) {
    const int rem = stride - 16 * v;
    msk[v] = static_cast<__mmask16>(rem >= 16 ? 0xFFFFu : (1u << rem) - 1u);
    off[v] = _mm512_mullo_epi32(_mm512_add_epi32(lane, _mm512_set1_epi32(16 * v)), _mm512_set1_epi32(step));
  }
  const int64_t row_bytes = static_cast<int64_t>(L.G) * L.M;
  for (int64_t n = 0; n < L.N; ++n) {
    const uint8_t* c = L.codes + (n * L.G + j0) * L.M;
    if (n + kPrefetchRows < L.N) {  // the slice's codes kPrefetchRows rows ahead
      const char* ahead = reinterpret_cast<const char*>(c + kPrefetchRows * row_bytes);
      _mm_prefetch(ahead, _MM_HINT_T0);
      _mm_prefetch(ahead + stride - 1, _MM_HINT_T0);
    }
    __m512i idx[NV];
    for (int v = 0; v < NV; ++v)
      idx[v] = _mm512_add_epi32(_mm512_cvtepu8_epi32(_mm_maskz_loadu_epi8(msk[v], c + 16 * v)), off[v]);
    for (int b = 0; b < L.batch; ++b) {
      const float* Tb = T + static_cast<size_t>(b) * 256;
      __m512 acc = _mm512_mask_i32gather_ps(_mm512_setzero_ps(), msk[0], idx[0], Tb, 4);
      for (int v = 1; v < NV; ++v)
        acc = _mm512_add_ps(acc, _mm512_mask_i32gather_ps(_mm512_setzero_ps(), msk[v], idx[v], Tb, 4));
      partial[static_cast<size_t>(b) * L.N + n] += _mm512_reduce_add_ps(acc);
    }
  }
}

void lookup_rows_level2(const Layer& L, const float* T, int j0, int nj, float* partial) {
  switch ((L.M * nj + 15) / 16) {
    case 1: lookup_rows_avx512<1>(L, T, j0, nj, partial); break;
    case 2: lookup_rows_avx512<2>(L, T, j0, nj, partial); break;
    case 3: lookup_rows_avx512<3>(L, T, j0, nj, partial); break;
    default: lookup_rows_avx512<4>(L, T, j0, nj, partial); break;
  }
}

void run_lut(const Layer& L, const float* xf, int nt) {
  std::vector<float> ct;
  transpose_codebooks(L, ct);
  const int S = (L.G + kSlice - 1) / kSlice;
  nt = std::max(1, std::min(nt, S));
  std::vector<std::vector<float>> partial(static_cast<size_t>(nt));
  const int level = simd_level();
#pragma omp parallel num_threads(nt)
  {
    const int tid = omp_get_thread_num();
    std::vector<float>& part = partial[static_cast<size_t>(tid)];
    std::vector<float> T(static_cast<size_t>(kSlice) * L.M * L.batch * 256);
#pragma omp for schedule(static)
    for (int s = 0; s < S; ++s) {
      if (part.empty()) part.assign(static_cast<size_t>(L.batch) * L.N, 0.f);
      const int j0 = s * kSlice, nj = std::min(kSlice, L.G - j0);
      if (level == 2) {
        build_tables_avx512(L, xf, ct.data(), j0, nj, T.data());
        lookup_rows_level2(L, T.data(), j0, nj, part.data());
        continue;
      }
      if (level == 1)
        build_tables_avx2(L, xf, ct.data(), j0, nj, T.data());
      else
        build_tables_scalar(L, xf, ct.data(), j0, nj, T.data());
      switch (L.M) {
        case 1: lookup_rows<1>(L, T.data(), j0, nj, part.data()); break;
        case 2: lookup_rows<2>(L, T.data(), j0, nj, part.data()); break;
        default: lookup_rows<0>(L, T.data(), j0, nj, part.data()); break;
      }
    }
  }
  // y = s * (sum of the thread partials, in thread order) + bias
#pragma omp parallel for schedule(static) num_threads(nt)
  for (int64_t n = 0; n < L.N; ++n) {
    const float sc = half_to_float(L.scales[n]);
    const float bi = L.bias ? half_to_float(L.bias[n]) : 0.f;
    for (int b = 0; b < L.batch; ++b) {
      float acc = 0.f;
      for (int t = 0; t < nt; ++t)
        if (!partial[static_cast<size_t>(t)].empty()) acc += partial[static_cast<size_t>(t)][static_cast<size_t>(b) * L.N + n];
      L.y[static_cast<size_t>(b) * L.N + n] = float_to_half(acc * sc + bi);
    }
  }
}

// ---------------------------------------------------------------------------
// decode + dot method
// ---------------------------------------------------------------------------
void decode_row_scalar(const Layer& L, int64_t n, float* w) {
  for (int64_t j = 0; j < L.G; ++j)
    for (int t = 0; t < L.g; ++t) {
      float a = 0.f;
      for (int m = 0; m < L.M; ++m)
        a += half_to_float(L.cb[((static_cast<size_t>(m) << L.B) + code_of(L, n, j, m)) * L.g + t]);
      w[j * L.g + t] = a;
    }
}

__attribute__((target("avx2,fma,f16c")))
void decode_row_avx2(const Layer& L, int64_t n, float* w) {
  for (int64_t j = 0; j < L.G; ++j)
    for (int t = 0; t < L.g; t += 8) {
      __m256 a = _mm256_setzero_ps();
      for (int m = 0; m < L.M; ++m) {
        const uint16_t* src = L.cb + ((static_cast<size_t>(m) << L.B) + code_of(L, n, j, m)) * L.g + t;
        a = _mm256_add_ps(a, _mm256_cvtph_ps(_mm_loadu_si128(reinterpret_cast<const __m128i*>(src))));
      }
      _mm256_storeu_ps(w + j * L.g + t, a);
    }
}

__attribute__((target("avx2,fma,f16c")))
inline float hsum_avx2(__m256 v) {
  const __m128 s = _mm_add_ps(_mm256_castps256_ps128(v), _mm256_extractf128_ps(v, 1));
  const __m128 t = _mm_add_ps(s, _mm_movehl_ps(s, s));
  return _mm_cvtss_f32(_mm_add_ss(t, _mm_shuffle_ps(t, t, 1)));
}

// dots[r] = x_b . w_r for the rows of a block (K a multiple of 8: g is 8 or 16)
__attribute__((target("avx2,fma,f16c")))
void dots_avx2(const float* xb, const float* w, int rows, int K, float* dots) {
  __m256 acc[kRowBlock];
  for (int r = 0; r < kRowBlock; ++r) acc[r] = _mm256_setzero_ps();
  for (int k = 0; k < K; k += 8) {
    const __m256 xv = _mm256_loadu_ps(xb + k);
    for (int r = 0; r < rows; ++r) acc[r] = _mm256_fmadd_ps(xv, _mm256_loadu_ps(w + static_cast<size_t>(r) * K + k), acc[r]);
  }
  for (int r = 0; r < rows; ++r) dots[r] = hsum_avx2(acc[r]);
}

void dots_scalar(const float* xb, const float* w, int rows, int K, float* dots) {
  for (int r = 0; r < rows; ++r) {
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < K; ++k) a[k & 7] += xb[k] * w[static_cast<size_t>(r) * K + k];
    dots[r] = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
  }
}

void run_decode_dot(const Layer& L, const float* xf, int nt) {
  const bool avx2 = simd_level() >= 1;
  const int64_t blocks = (L.N + kRowBlock - 1) / kRowBlock;
#pragma omp parallel num_threads(nt)
  {
    std::vector<float> w(static_cast<size_t>(kRowBlock) * L.K);
#pragma omp for schedule(static)
    for (int64_t blk = 0; blk < blocks; ++blk) {
      const int64_t n0 = blk * kRowBlock;
      const int rows = static_cast<int>(std::min<int64_t>(kRowBlock, L.N - n0));
      for (int r = 0; r < rows; ++r) {
        if (avx2)
          decode_row_avx2(L, n0 + r, w.data() + static_cast<size_t>(r) * L.K);
        else
          decode_row_scalar(L, n0 + r, w.data() + static_cast<size_t>(r) * L.K);
      }
      for (int b = 0; b < L.batch; ++b) {
        float d[kRowBlock];
        const float* xb = xf + static_cast<size_t>(b) * L.K;
        if (avx2)
          dots_avx2(xb, w.data(), rows, L.K, d);
        else
          dots_scalar(xb, w.data(), rows, L.K, d);
        for (int r = 0; r < rows; ++r) {
          const int64_t n = n0 + r;
          const float bi = L.bias ? half_to_float(L.bias[n]) : 0.f;
          L.y[static_cast<size_t>(b) * L.N + n] = float_to_half(d[r] * half_to_float(L.scales[n]) + bi);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// fused decode + dot (AVX-512): 16 weights of a row are decoded in a register and
// multiplied into per-(row, batch row) accumulators at once, so no decoded row is
// stored.  B = 8 codebooks are read from an fp32 copy ([M][256][g], 8 KB per codebook
// at g = 8, so L1-resident); B = 16 codebooks stay fp16 and are converted as they are
// read.  Per weight the pieces are added in codebook order in fp32 (as the decode
// defines), the products accumulate in fp32 lanes, and the lanes are added at the end
// of the row; every row is computed by one thread in one fixed order, so the result
// does not depend on the thread count.
// ---------------------------------------------------------------------------
// rows per block for BB batch rows: R * BB accumulators (at most 16 of the 32 zmm)
template <int BB>
constexpr int fused_rows() { return BB <= 2 ? 8 : BB <= 4 ? 4 : BB == 5 ? 3 : 2; }

// 16 decoded weights of one row from its codes at groups j (and j + 1 when g = 8):
// cr points at the row's codes of group j, cb at the codebooks (fp32 for B = 8, fp16
// for B = 16).  `two` = false decodes only group j (g = 8, last group of an odd G),
// leaving the upper 8 lanes zero.
template <int MM, int GG, bool kF32>
__attribute__((target("avx512f,avx512bw,avx512vl,avx2,fma,f16c"), always_inline))
inline __m512 decode16(const void* cr, const void* cb, int M, int g, bool two) {
  const int nm = MM > 0 ? MM : M;
  const int gg = GG > 0 ? GG : g;
  __m512 w = _mm512_setzero_ps();
  for (int m = 0; m < nm; ++m) {
    __m512 piece;
    if constexpr (kF32) {
      const uint8_t* c = static_cast<const uint8_t*>(cr);
      const float* cm = static_cast<const float*>(cb) + static_cast<size_t>(m) * 256 * gg;
      if (gg == 16) {
        piece = _mm512_loadu_ps(cm + static_cast<size_t>(c[m]) * 16);
      } else {
        const __m256 lo = _mm256_loadu_ps(cm + static_cast<size_t>(c[m]) * 8);
        const __m256 hi = two ? _mm256_loadu_ps(cm + static_cast<size_t>(c[nm + m]) * 8) : _mm256_setzero_ps();
        piece = _mm512_castpd_ps(_mm512_insertf64x4(_mm512_castps_pd(_mm512_castps256_ps512(lo)),
                                                    _mm256_castps_pd(hi), 1));
      }
    } else {
      const uint16_t* c = static_cast<const uint16_t*>(cr);
      const uint16_t* cm = static_cast<const uint16_t*>(cb) + (static_cast<size_t>(m) << 16) * gg;
      if (gg == 16) {
        piece = _mm512_cvtph_ps(_mm256_loadu_si256(reinterpret_cast<const __m256i*>(cm + static_cast<size_t>(c[m]) * 16)));
      } else {
        const __m128i lo = _mm_loadu_si128(reinterpret_cast<const __m128i*>(cm + static_cast<size_t>(c[m]) * 8));
        const __m128i hi = two ? _mm_loadu_si128(reinterpret_cast<const __m128i*>(cm + static_cast<size_t>(c[nm + m]) * 8))
                               : _mm_setzero_si128();
        piece = _mm512_cvtph_ps(_mm256_inserti128_si256(_mm256_castsi128_si256(lo), hi, 1));
      }
    }
    w = m == 0 ? piece : _mm512_add_ps(w, piece);
  }
  return w;
}

// y[b0 .. b0 + BB) x rows [n0, n0 + R) (rows past N repeat row N - 1 and are not stored).
template <int MM, int GG, bool kF32, int BB>
__attribute__((target("avx512f,avx512bw,avx512vl,avx2,fma,f16c")))
void fused_block_avx512(const Layer& L, const float* xf, const void* cb, int64_t n0, int b0) {
  constexpr int R = fused_rows<BB>();
  const int M = MM > 0 ? MM : L.M, g = GG > 0 ? GG : L.g;
  const int cbytes = kF32 ? 1 : 2;
  const int64_t rowc = static_cast<int64_t>(L.G) * M;  // codes per row
  const uint8_t* crow[R];
  for (int r = 0; r < R; ++r)
    crow[r] = L.codes + std::min<int64_t>(n0 + r, L.N - 1) * rowc * cbytes;
  const float* xb = xf + static_cast<size_t>(b0) * L.K;
  __m512 acc[R][BB];
  for (int r = 0; r < R; ++r)
    for (int b = 0; b < BB; ++b) acc[r][b] = _mm512_setzero_ps();
  const int K16 = L.K & ~15;
  for (int k = 0; k < K16; k += 16) {
    __m512 xk[BB];
    for (int b = 0; b < BB; ++b) xk[b] = _mm512_loadu_ps(xb + static_cast<size_t>(b) * L.K + k);
    const int64_t coff = static_cast<int64_t>(k / g) * M * cbytes;
    for (int r = 0; r < R; ++r) {
      const __m512 w = decode16<MM, GG, kF32>(crow[r] + coff, cb, M, g, true);
      for (int b = 0; b < BB; ++b) acc[r][b] = _mm512_fmadd_ps(w, xk[b], acc[r][b]);
    }
  }
  if (K16 < L.K) {  // g = 8 and G odd: the last group alone
    __m512 xk[BB];
    for (int b = 0; b < BB; ++b) xk[b] = _mm512_maskz_loadu_ps(0x00FF, xb + static_cast<size_t>(b) * L.K + K16);
    const int64_t coff = static_cast<int64_t>(K16 / g) * M * cbytes;
    for (int r = 0; r < R; ++r) {
      const __m512 w = decode16<MM, GG, kF32>(crow[r] + coff, cb, M, g, false);
      for (int b = 0; b < BB; ++b) acc[r][b] = _mm512_fmadd_ps(w, xk[b], acc[r][b]);
    }
  }
  for (int r = 0; r < R; ++r) {
    const int64_t n = n0 + r;
    if (n >= L.N) break;
    const float sc = half_to_float(L.scales[n]);
    const float bi = L.bias ? half_to_float(L.bias[n]) : 0.f;
    for (int b = 0; b < BB; ++b)
      L.y[static_cast<size_t>(b0 + b) * L.N + n] = float_to_half(_mm512_reduce_add_ps(acc[r][b]) * sc + bi);
  }
}

template <int MM, int GG, bool kF32>
void fused_rows_avx512(const Layer& L, const float* xf, const void* cb, int64_t n0, int rows_per_task) {
  // one task: rows [n0, n0 + rows_per_task) for every batch row, in chunks of 8
  for (int b0 = 0; b0 < L.batch; b0 += 8) {
    const int bb = std::min(8, L.batch - b0);
    auto run = [&](auto tag) {
      constexpr int BBc = decltype(tag)::value;
      constexpr int R = fused_rows<BBc>();
      for (int64_t n = n0; n < std::min<int64_t>(n0 + rows_per_task, L.N); n += R)
        fused_block_avx512<MM, GG, kF32, BBc>(L, xf, cb, n, b0);
    };
    switch (bb) {
      case 1: run(std::integral_constant<int, 1>()); break;
      case 2: run(std::integral_constant<int, 2>()); break;
      case 3: run(std::integral_constant<int, 3>()); break;
      case 4: run(std::integral_constant<int, 4>()); break;
      case 5: run(std::integral_constant<int, 5>()); break;
      case 6: run(std::integral_constant<int, 6>()); break;
      case 7: run(std::integral_constant<int, 7>()); break;
      default: run(std::integral_constant<int, 8>()); break;
    }
  }
}

// rows per task: a multiple of every fused_rows value (8, 4, 3, 2)
constexpr int kFusedTaskRows = 48;

void run_fused(const Layer& L, const float* xf, int nt) {
  std::vector<float> cbf;
  const void* cb = L.cb;
  if (L.B == 8) {  // fp32 copy, [M][256][g] as stored
    cbf.resize(static_cast<size_t>(L.M) * 256 * L.g);
    for (size_t i = 0; i < cbf.size(); ++i) cbf[i] = half_to_float(L.cb[i]);
    cb = cbf.data();
  }
  using Fn = void (*)(const Layer&, const float*, const void*, int64_t, int);
  Fn fn;
  if (L.B == 8) {
    static constexpr Fn g8[4] = {fused_rows_avx512<1, 8, true>, fused_rows_avx512<2, 8, true>,
                                 fused_rows_avx512<3, 8, true>, fused_rows_avx512<4, 8, true>};
    static constexpr Fn g16[4] = {fused_rows_avx512<1, 16, true>, fused_rows_avx512<2, 16, true>,
                                  fused_rows_avx512<3, 16, true>, fused_rows_avx512<4, 16, true>};
    fn = (L.g == 8 ? g8 : g16)[L.M - 1];
  } else {
    if (L.g == 8)
      fn = L.M == 1 ? fused_rows_avx512<1, 8, false> : fused_rows_avx512<2, 8, false>;
    else
      fn = L.M == 1 ? fused_rows_avx512<1, 16, false> : fused_rows_avx512<2, 16, false>;
  }
  const int64_t tasks = (L.N + kFusedTaskRows - 1) / kFusedTaskRows;
#pragma omp parallel for schedule(static) num_threads(nt)
  for (int64_t t = 0; t < tasks; ++t) fn(L, xf, cb, t * kFusedTaskRows, kFusedTaskRows);
}

bool scheme_ok(int M, int B, int g) {
  if (g != 8 && g != 16) return false;
  if (B == 8) return M >= 1 && M <= 4;
  if (B == 16) return M == 1 || M == 2;
  return false;
}

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na && nb && x < y + nb && y < x + na;
}

}  // namespace

extern "C" {

int aqlm_cpu_abi_version(void) { return 3; }

int aqlm_cpu_simd_level(void) { return simd_level(); }

int aqlm_cpu_set_max_simd_level(int level) {
  return g_max_simd.exchange(std::max(0, std::min(kMaxSimd, level)));
}

aqlm_status aqlm_cpu_matmul(const void* x, const void* codes, const void* codebooks,
                            const void* scales, const void* bias, void* y,
                            int M, int B, int g, int K, int N, int batch, int nthreads) {
  if (!x || !codes || !codebooks || !scales || !y) return AQLM_ERR_INVALID_ARG;
  if (M < 1 || B < 1 || g < 1 || K < 1 || N < 1 || batch < 1 || batch > 65535 || nthreads < 0)
    return AQLM_ERR_INVALID_ARG;
  if (K % g != 0) return AQLM_ERR_INVALID_ARG;
  if (!scheme_ok(M, B, g)) return AQLM_ERR_UNSUPPORTED;
  const auto a2 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 1u) == 0; };
  if (!a2(x) || !a2(codebooks) || !a2(scales) || !a2(y) || (bias && !a2(bias)) || (B > 8 && !a2(codes)))
    return AQLM_ERR_MISALIGNED;
  const int cbytes = B <= 8 ? 1 : 2;
  const size_t ybytes = static_cast<size_t>(batch) * N * 2;
  if (overlap(y, ybytes, x, static_cast<size_t>(batch) * K * 2) ||
      overlap(y, ybytes, codes, static_cast<size_t>(N) * (K / g) * M * cbytes) ||
      overlap(y, ybytes, codebooks, (static_cast<size_t>(M) << B) * g * 2) ||
      overlap(y, ybytes, scales, static_cast<size_t>(N) * 2) || (bias && overlap(y, ybytes, bias, static_cast<size_t>(N) * 2)))
    return AQLM_ERR_INVALID_ARG;

  Layer L{static_cast<const uint16_t*>(x), static_cast<const uint8_t*>(codes),
          static_cast<const uint16_t*>(codebooks), static_cast<const uint16_t*>(scales),
          static_cast<const uint16_t*>(bias), static_cast<uint16_t*>(y), M, B, g, K, N, batch, K / g, cbytes};
  const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
  std::vector<float> xf(static_cast<size_t>(batch) * K);
  for (size_t i = 0; i < xf.size(); ++i) xf[i] = half_to_float(L.x[i]);
  if (simd_level() == 2 && !(B == 8 && batch == 1))
    run_fused(L, xf.data(), nt);
  else if (B == 8 && batch <= kLutMaxBatch)
    run_lut(L, xf.data(), nt);
  else
    run_decode_dot(L, xf.data(), nt);
  return AQLM_OK;
}

}  // extern "C"
