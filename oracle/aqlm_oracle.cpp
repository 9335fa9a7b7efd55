// AQLM CPU oracle: a plain, slow, obviously correct statement of what the
// AQLM weight-only linear layer computes.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load, call or
// link this file: only the tests, the package's smoke check and the CPU
// baseline leg of the benchmark use it.  It shares no code, header, table or
// helper with the CUDA library (weight_only_additive_b200/csrc).
//
// What it computes (sources: the AQLM pages -- "Additive quantization that
// actually survives one-bit weights" (heatdrop.ai repo summary), section
// "What it does"; the inference-research record "AQLM (additive /
// multi-codebook quantization)", sections "Bits", "Activation scheme",
// "Kernels" and "notes"; the paper record "Extreme Compression of Large
// Language Models via Additive Quantization", method paragraph):
//
//   * a weight row is cut into groups of g consecutive inputs; each group is
//     stored as M codes, code m indexing codebook m (2^B entries of g fp16
//     values), and the group's weights are the SUM of the M selected
//     codewords ("What it does"; "Activation scheme"; paper-record method);
//   * activations stay fp16 (w2a16, "Bits");
//   * the layer is y = x . W^T . diag(s) + bias with one fp16 scale per output
//     channel -- the inference-research "notes" say no scale is shared across
//     a group, so the only scale is per output row;
//   * large batches dequantise to fp16 and run a dense fp16 GEMM ("notes"),
//     small batches use lookups instead of per-element dequantisation
//     ("Kernels") -- the LUT form below states that second route;
//   * fine-tuning through a quantised layer (PEFT fine-tuning, repo summary
//     "Key highlights"; PV-Tuning after quantisation, "What it does") keeps W
//     fixed and needs the gradient with respect to the layer input,
//     dx = dy . W16, the transpose of the same product (input-gradient form).
//
// Readings where the pages are silent (each also listed in the design notes):
//   * codes layout [N, K/g, M] (m fastest), unsigned, no offset; uint8 when
//     B <= 8, uint16 when 8 < B <= 16;  codebooks [M, 2^B, g];
//   * decode order: a = C_0[c_0][t]; a = a + C_m[c_m][t] for m = 1..M-1 in
//     fp32 round-to-nearest-even, then one fp32 multiply by s_n, then one
//     round-to-nearest-even to fp16.  The sum starts from C_0 itself (not
//     0 + C_0) so the sign of zero survives;
//   * reference outputs are accumulated in fp64 (exact products, k ascending).
//
// Build: g++ -O2 -ffp-contract=off -fopenmp -shared -fPIC (no -ffast-math:
// every float operation here must be a single IEEE-754 operation).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---------------------------------------------------------------------------
// IEEE 754 binary16 <-> binary32, written from the format's definition:
// binary16 = 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
//   e = 0       : (-1)^s * f * 2^-24             (zero / subnormal)
//   1 <= e < 31 : (-1)^s * (1024 + f) * 2^(e-25) (normal)
//   e = 31      : infinity (f = 0) or NaN (f != 0)
// ---------------------------------------------------------------------------
float half_bits_to_float(uint16_t h) {
  const uint32_t sign = h >> 15;
  const uint32_t e = (h >> 10) & 0x1fu;
  const uint32_t f = h & 0x3ffu;
  float mag;
  if (e == 0) {
    mag = std::ldexp(static_cast<float>(f), -24);
  } else if (e == 31) {
    mag = f ? NAN : INFINITY;
  } else {
    mag = std::ldexp(static_cast<float>(1024u + f), static_cast<int>(e) - 25);
  }
  return sign ? -mag : mag;
}

// Round a binary32 value to the nearest binary16 value, ties to even.
// Overflow (|v| >= 65520) gives infinity; NaN gives a quiet NaN.
uint16_t float_to_half_bits_rne(float v) {
  uint32_t u;
  std::memcpy(&u, &v, sizeof u);
  const uint16_t sign = static_cast<uint16_t>((u >> 16) & 0x8000u);
  const uint32_t e8 = (u >> 23) & 0xffu;
  const uint32_t frac = u & 0x7fffffu;
  if (e8 == 0xffu) return static_cast<uint16_t>(sign | (frac ? 0x7e00u : 0x7c00u));
  if (e8 == 0) return sign;  // |v| < 2^-126: far below half of 2^-24
  const int e = static_cast<int>(e8) - 127;  // v = m24 * 2^(e-23)
  if (e > 15) return static_cast<uint16_t>(sign | 0x7c00u);
  const uint32_t m24 = frac | 0x800000u;
  // Drop the bits below the binary16 unit in the last place:
  // 2^(e-10) for normal results (e >= -14), 2^-24 for subnormal results.
  const int shift = (e >= -14) ? 13 : (-1 - e);
  if (shift > 24) return sign;  // value < 2^-25: below half an ulp
  uint32_t q = m24 >> shift;
  const uint32_t rem = m24 & ((1u << shift) - 1u);
  const uint32_t halfway = 1u << (shift - 1);
  if (rem > halfway || (rem == halfway && (q & 1u))) ++q;
  uint32_t bits;
  if (e >= -14) {
    bits = (static_cast<uint32_t>(e + 15) << 10) + (q - 1024u);  // q in [1024, 2048]
  } else {
    bits = q;  // subnormal count; 1024 becomes the smallest normal
  }
  if (bits >= 0x7c00u) bits = 0x7c00u;
  return static_cast<uint16_t>(sign | bits);
}

struct Shape {
  int M, B, g, K, N, G;
  int64_t entries;  // 2^B
};

bool make_shape(int M, int B, int g, int K, int N, Shape* s) {
  if (M < 1 || M > 64 || B < 1 || B > 16 || g < 1 || K < 1 || N < 1) return false;
  if (K % g != 0) return false;
  s->M = M; s->B = B; s->g = g; s->K = K; s->N = N; s->G = K / g;
  s->entries = int64_t(1) << B;
  return true;
}

// Code for (row n, group j, codebook m), layout [N, G, M], m fastest.
inline uint32_t code_at(const void* codes, const Shape& s, int64_t n, int64_t j, int m) {
  const int64_t idx = (n * s.G + j) * s.M + m;
  if (s.B <= 8) return static_cast<const uint8_t*>(codes)[idx];
  return static_cast<const uint16_t*>(codes)[idx];
}

// Codebook entry C_m[i][t], layout [M, 2^B, g].
inline uint16_t codebook_at(const uint16_t* cb, const Shape& s, int m, int64_t i, int t) {
  return cb[(static_cast<int64_t>(m) * s.entries + i) * s.g + t];
}

bool codes_in_range(const void* codes, const Shape& s) {
  const int64_t total = int64_t(s.N) * s.G * s.M;
  for (int64_t i = 0; i < total; ++i) {
    const uint32_t c = s.B <= 8 ? static_cast<const uint8_t*>(codes)[i]
                                : static_cast<const uint16_t*>(codes)[i];
    if (c >= static_cast<uint32_t>(s.entries)) return false;
  }
  return true;
}

// Decode one weight row n into fp16 bits (the dequantisation definition).
void decode_row(const void* codes, const uint16_t* cb, const uint16_t* scales,
                const Shape& s, int64_t n, uint16_t* row_out) {
  const float scale = half_bits_to_float(scales[n]);
  for (int64_t j = 0; j < s.G; ++j) {
    for (int t = 0; t < s.g; ++t) {
      float a = half_bits_to_float(codebook_at(cb, s, 0, code_at(codes, s, n, j, 0), t));
      for (int m = 1; m < s.M; ++m) {
        a = a + half_bits_to_float(codebook_at(cb, s, m, code_at(codes, s, n, j, m), t));
      }
      const float w = a * scale;
      row_out[j * s.g + t] = float_to_half_bits_rne(w);
    }
  }
}

int pick_threads(int nthreads) {
#ifdef _OPENMP
  return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

}  // namespace

extern "C" {

// Status codes: 0 = ok, 1 = invalid shape/argument, 2 = code out of range,
// 3 = problem too large for this form.
int oracle_abi_version(void) { return 1; }

int oracle_max_threads(void) { return pick_threads(0); }

void oracle_half_to_float(const uint16_t* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = half_bits_to_float(in[i]);
}

void oracle_float_to_half(const float* in, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = float_to_half_bits_rne(in[i]);
}

// Same conversion, applied to raw 32-bit patterns [start, start + n): lets a
// test sweep every binary32 pattern without materialising them.
void oracle_float_bits_to_half_range(uint32_t start, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) {
    const uint32_t u = start + static_cast<uint32_t>(i);
    float v;
    std::memcpy(&v, &u, sizeof v);
    out[i] = float_to_half_bits_rne(v);
  }
}

// W_out[n, j*g + t] = f16_rne( (sum_m C_m[codes[n,j,m]][t]) * s_n ), fp32 sum.
int oracle_dequantize(const void* codes, const uint16_t* codebooks, const uint16_t* scales,
                      uint16_t* W_out, int M, int B, int g, int K, int N, int nthreads) {
  Shape s;
  if (!make_shape(M, B, g, K, N, &s) || !codes || !codebooks || !scales || !W_out) return 1;
  if (!codes_in_range(codes, s)) return 2;
  const int nt = pick_threads(nthreads);
#pragma omp parallel for schedule(static) num_threads(nt)
  for (int64_t n = 0; n < N; ++n) decode_row(codes, codebooks, scales, s, n, W_out + n * K);
  return 0;
}

// Reference output: decode each requested row to fp16 (the dequantisation
// definition), then the fp64 dot product with every batch row.
// rows == NULL means all N rows in order; y is [batch, nrows].
int oracle_linear_rows(const uint16_t* x, const void* codes, const uint16_t* codebooks,
                       const uint16_t* scales, const uint16_t* bias, double* y,
                       int M, int B, int g, int K, int N, int batch,
                       const int64_t* rows, int64_t nrows, int nthreads) {
  Shape s;
  if (!make_shape(M, B, g, K, N, &s) || !x || !codes || !codebooks || !scales || !y || batch < 1)
    return 1;
  if (!rows) nrows = N;
  for (int64_t r = 0; rows && r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= N) return 1;
  if (!codes_in_range(codes, s)) return 2;
  const int nt = pick_threads(nthreads);
#pragma omp parallel num_threads(nt)
  {
    std::vector<uint16_t> wrow(static_cast<size_t>(K));
#pragma omp for schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
      const int64_t n = rows ? rows[r] : r;
      decode_row(codes, codebooks, scales, s, n, wrow.data());
      for (int64_t b = 0; b < batch; ++b) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          acc += static_cast<double>(half_bits_to_float(x[b * K + k])) *
                 static_cast<double>(half_bits_to_float(wrow[k]));
        }
        if (bias) acc += static_cast<double>(half_bits_to_float(bias[n]));
        y[b * nrows + r] = acc;
      }
    }
  }
  return 0;
}

// Exact-codeword form, no fp16 rounding of W:
// y[b,n] = f64(s_n) * sum_j sum_m sum_t f64(x[b, j*g+t]) * f64(C_m[code][t]) + f64(bias_n)
int oracle_linear_exact(const uint16_t* x, const void* codes, const uint16_t* codebooks,
                        const uint16_t* scales, const uint16_t* bias, double* y,
                        int M, int B, int g, int K, int N, int batch, int nthreads) {
  Shape s;
  if (!make_shape(M, B, g, K, N, &s) || !x || !codes || !codebooks || !scales || !y || batch < 1)
    return 1;
  if (!codes_in_range(codes, s)) return 2;
  const int nt = pick_threads(nthreads);
#pragma omp parallel for schedule(static) num_threads(nt)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t b = 0; b < batch; ++b) {
      double acc = 0.0;
      for (int64_t j = 0; j < s.G; ++j)
        for (int m = 0; m < M; ++m) {
          const uint32_t c = code_at(codes, s, n, j, m);
          for (int t = 0; t < g; ++t)
            acc += static_cast<double>(half_bits_to_float(x[b * K + j * g + t])) *
                   static_cast<double>(half_bits_to_float(codebook_at(codebooks, s, m, c, t)));
        }
      double out = static_cast<double>(half_bits_to_float(scales[n])) * acc;
      if (bias) out += static_cast<double>(half_bits_to_float(bias[n]));
      y[b * N + n] = out;
    }
  }
  return 0;
}

// Lookup-table form (the "fast lookup, no per-element dequantization" route):
//   T[j][m][i] = sum_t f64(x[b, j*g+t]) * f64(C_m[i][t])     for every entry i
//   y[b,n]     = f64(s_n) * sum_j sum_m T[j][m][codes[n,j,m]] + f64(bias_n)
// The table has G*M*2^B entries per batch row; larger problems return 3.
int oracle_linear_lut(const uint16_t* x, const void* codes, const uint16_t* codebooks,
                      const uint16_t* scales, const uint16_t* bias, double* y,
                      int M, int B, int g, int K, int N, int batch, int nthreads) {
  Shape s;
  if (!make_shape(M, B, g, K, N, &s) || !x || !codes || !codebooks || !scales || !y || batch < 1)
    return 1;
  if (!codes_in_range(codes, s)) return 2;
  const int64_t table = int64_t(s.G) * M * s.entries;
  if (table > (int64_t(1) << 25)) return 3;
  std::vector<double> T(static_cast<size_t>(table));
  const int nt = pick_threads(nthreads);
  for (int64_t b = 0; b < batch; ++b) {
#pragma omp parallel for schedule(static) num_threads(nt)
    for (int64_t j = 0; j < s.G; ++j)
      for (int m = 0; m < M; ++m)
        for (int64_t i = 0; i < s.entries; ++i) {
          double dot = 0.0;
          for (int t = 0; t < g; ++t)
            dot += static_cast<double>(half_bits_to_float(x[b * K + j * g + t])) *
                   static_cast<double>(half_bits_to_float(codebook_at(codebooks, s, m, i, t)));
          T[(j * M + m) * s.entries + i] = dot;
        }
#pragma omp parallel for schedule(static) num_threads(nt)
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t j = 0; j < s.G; ++j)
        for (int m = 0; m < M; ++m)
          acc += T[(j * M + m) * s.entries + code_at(codes, s, n, j, m)];
      double out = static_cast<double>(half_bits_to_float(scales[n])) * acc;
      if (bias) out += static_cast<double>(half_bits_to_float(bias[n]));
      y[b * N + n] = out;
    }
  }
  return 0;
}

// Input gradient of y = x . W16^T + bias with respect to x:
//   dx[b, k] = sum_{n ascending} f64(dy[b, n]) * f64(W16[n, k])     (fp64)
// W16 is the dequantised weight of oracle_dequantize (scale included, rounded
// to fp16), so this is exactly the transpose of the product that
// oracle_linear_rows computes.  cols == NULL means all K columns in order; dx
// is [batch, ncols].
int oracle_input_grad_cols(const uint16_t* dy, const void* codes, const uint16_t* codebooks,
                           const uint16_t* scales, double* dx, int M, int B, int g, int K, int N,
                           int batch, const int64_t* cols, int64_t ncols, int nthreads) {
  Shape s;
  if (!make_shape(M, B, g, K, N, &s) || !dy || !codes || !codebooks || !scales || !dx || batch < 1)
    return 1;
  if (!cols) ncols = K;
  for (int64_t r = 0; cols && r < ncols; ++r)
    if (cols[r] < 0 || cols[r] >= K) return 1;
  if (!codes_in_range(codes, s)) return 2;
  const int nt = pick_threads(nthreads);
  std::vector<uint16_t> W(static_cast<size_t>(N) * static_cast<size_t>(K));
#pragma omp parallel for schedule(static) num_threads(nt)
  for (int64_t n = 0; n < N; ++n) decode_row(codes, codebooks, scales, s, n, W.data() + n * K);
#pragma omp parallel for schedule(static) num_threads(nt)
  for (int64_t r = 0; r < ncols; ++r) {
    const int64_t k = cols ? cols[r] : r;
    for (int64_t b = 0; b < batch; ++b) {
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        acc += static_cast<double>(half_bits_to_float(dy[b * N + n])) *
               static_cast<double>(half_bits_to_float(W[n * K + k]));
      }
      dx[b * ncols + r] = acc;
    }
  }
  return 0;
}

}  // extern "C"
