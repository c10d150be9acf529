// CPU oracle for the packed 1-bit / balanced-ternary matmul.
//
// TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
// definition that the CUDA path is checked against.  Only the tests, the smoke
// check and the bench's CPU-baseline leg load it; the product path never does.
// It shares no code, header, table or constant with the CUDA library.
//
// Style: one definition per function, written straight from the pages, with
// no blocking, fusion or reordering.  The binary path never counts bits: it
// unpacks every sign to an int8 +-1 and sums products in int64, so that the
// identity <x,w> = n - 2*popcount(x XOR w) that the CUDA path relies on is
// checked, not assumed.  Floating point is float64 except where the method
// fixes float32 (the alpha-scaled output, the TWN threshold and scale, which
// are float32 tensors).
//
// Sources (page title, section):
//   [BME]  "Binary Math Effectiveness -- why / how / when", section 1 "The core
//          identity" (encoding table, the identity, XNOR form, "Edge cases").
//   [ADR]  "Architecture Decision Record", section "Decision"
//          (binary_gemm_u64: packed XNOR+popcount matmul over uint64 words).
//   [BTE]  "BalancedTernaryEngine" README, sections "Features" (TWN threshold
//          0.7*mean|W|, least-squares per-channel scale, 10 trits per 16-bit
//          word in base 3) and ".tbin Format" (ternary record: scales, packed
//          trits 10 per 16-bit word); Layer.forward in "Module Overview".
//
// Readings where the pages are silent (each also listed in the design notes):
//   * bit order: element k of a row is bit (k mod 64) of word k/64 (LSB first);
//   * sign rule: bit = 1 exactly when !(x > 0): +-0, NaN and -inf give -1;
//   * TWN: one threshold per tensor, strict |w| > Delta, Delta = float32 of
//     0.7 * mean|W| computed in float64; scale per output row = mean |w| over
//     the row's non-zero trits (0 for a row with none);
//   * base 3: digit = trit + 1, trit 10j+i of a row has weight 3^i in word j;
//     rows are packed independently and padded with zero trits (digit 1).
#include "bnn_oracle.h"

#include <cmath>
#include <cstring>

namespace {

int64_t words64(int64_t k) { return (k + 63) / 64; }
int64_t words10(int64_t k) { return (k + 9) / 10; }

// [BME] encoding table: bit 0 means +1, bit 1 means -1.
int8_t sign_of_bit(uint64_t word, int64_t bit) {
  return ((word >> bit) & 1u) ? int8_t(-1) : int8_t(+1);
}

// bfloat16 is the top half of an IEEE float32; widening is exact.
double bf16_to_double(uint16_t h) {
  uint32_t bits = uint32_t(h) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return double(f);
}

}  // namespace

extern "C" {

// [BME] "Edge cases", last row: inputs <= 0 project to -1, > 0 to +1.  Bits at
// positions >= k in the last word stay 0 ("pad bits encode +1").
void oracle_pack_signs(const float* x, int64_t rows, int64_t k, uint64_t* out) {
  const int64_t kw = words64(k);
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t j = 0; j < kw; ++j) out[r * kw + j] = 0;
    for (int64_t e = 0; e < k; ++e) {
      const float v = x[r * k + e];
      const bool minus = !(v > 0.0f);
      if (minus) out[r * kw + e / 64] |= (uint64_t(1) << (e % 64));
    }
  }
}

// [BME] encoding table, read back: one int8 +-1 per logical element.
void oracle_unpack_signs(const uint64_t* p, int64_t rows, int64_t k, int8_t* out) {
  const int64_t kw = words64(k);
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t e = 0; e < k; ++e) out[r * k + e] = sign_of_bit(p[r * kw + e / 64], e % 64);
}

// Count of bits set at positions >= k ([BME] "Edge cases": pad bits must be 0).
int64_t oracle_count_pad_bits(const uint64_t* p, int64_t rows, int64_t k) {
  const int64_t kw = words64(k);
  int64_t count = 0;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = k; b < 64 * kw; ++b) count += (p[r * kw + b / 64] >> (b % 64)) & 1u;
  return count;
}

// One output of the binary matmul by its definition: <x,w> = sum_e x_e * w_e
// over the logical length k ([BME] section 1), then the per-output-channel
// scale ([BME] "Edge cases", channel scale alpha).  With |dot| <= k <= 2^24
// the product alpha * dot is exact in float64 (a 24-bit significand times an
// integer of at most 25 bits), so the single rounding to float32 below is the
// correctly rounded float32 product.
static void binary_one(const uint64_t* xrow, const uint64_t* wrow, int64_t k,
                       const float* alpha, int64_t col, int32_t* dot_out, float* out_out) {
  int64_t sum = 0;
  for (int64_t e = 0; e < k; ++e)
    sum += int64_t(sign_of_bit(xrow[e / 64], e % 64)) * int64_t(sign_of_bit(wrow[e / 64], e % 64));
  if (dot_out) *dot_out = int32_t(sum);
  if (out_out) *out_out = float(double(alpha[col]) * double(sum));
}

// [ADR] binary_gemm_u64 semantics over row-major X[m,k] and W[n,k] (both packed
// to ceil(k/64) words per row): dots[i,j] = <x_i, w_j>, out[i,j] = alpha_j * dots[i,j].
// Either output pointer may be null.
void oracle_binary_gemm(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                        int64_t m, int64_t n, int64_t k, int32_t* dots, float* out) {
  const int64_t kw = words64(k);
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j)
      binary_one(xp + i * kw, wp + j * kw, k, alpha, j,
                 dots ? dots + i * n + j : nullptr, out ? out + i * n + j : nullptr);
}

// The same, for `count` chosen (row, col) pairs only (large shapes).
void oracle_binary_gemm_sampled(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                                int64_t m, int64_t n, int64_t k, const int64_t* rows,
                                const int64_t* cols, int64_t count, int32_t* dots, float* out) {
  (void)m;
  (void)n;
  const int64_t kw = words64(k);
  for (int64_t s = 0; s < count; ++s)
    binary_one(xp + rows[s] * kw, wp + cols[s] * kw, k, alpha, cols[s],
               dots ? dots + s : nullptr, out ? out + s : nullptr);
}

// One binarised linear layer followed by the next layer's input packing
// ([BTE] ".tbin Format": a ternary/binary record carries a per-channel bias;
// "binary_nn" README, FFN stacks of BinaryLinear: binary activations from layer
// to layer).  In this order: the +-1 dot (as oracle_binary_gemm), the channel
// scale y = fl32(alpha_j * dot), the bias y = fl32(y + bias_j) (an IEEE float32
// addition, skipped when bias is null), then the sign pack of the row of y
// exactly as oracle_pack_signs (bit = !(y > 0), pad bits 0) into
// next[i, 0 .. ceil(n/64)).  Any output pointer may be null.
void oracle_binary_linear(const uint64_t* xp, const uint64_t* wp, const float* alpha, const float* bias,
                          int64_t m, int64_t n, int64_t k, int32_t* dots, float* y, uint64_t* next) {
  const int64_t kw = words64(k);
  const int64_t nw = words64(n);
  float* row = new float[n > 0 ? n : 1];
  for (int64_t i = 0; i < m; ++i) {
    for (int64_t j = 0; j < n; ++j) {
      int32_t d = 0;
      float v = 0.0f;
      binary_one(xp + i * kw, wp + j * kw, k, alpha, j, &d, &v);
      if (bias) {
        const float b = bias[j];
        v = v + b;  // binary32 addition, round to nearest even (built with -ffp-contract=off)
      }
      row[j] = v;
      if (dots) dots[i * n + j] = d;
      if (y) y[i * n + j] = v;
    }
    if (next) oracle_pack_signs(row, 1, n, next + i * nw);
  }
  delete[] row;
}

// [BTE] "Features": TWN threshold Delta = 0.7 * mean|W| over the whole tensor,
// the mean summed in float64 in element order and Delta rounded once to float32.
float oracle_twn_delta(const float* w, int64_t total) {
  double sum_abs = 0.0;
  for (int64_t e = 0; e < total; ++e) sum_abs += std::fabs(double(w[e]));
  const double mean_abs = total > 0 ? sum_abs / double(total) : 0.0;
  return float(0.7 * mean_abs);
}

// [BTE] "Features": trit = sign(w) where |w| > Delta else 0 (the comparison in
// float32), and a per-channel least-squares scale.  For fixed trits t the
// least-squares scale of row r minimises sum_e (w_e - s * t_e)^2, i.e.
// s = <w,t>/<t,t> = mean of |w| over t != 0 (0 for a row with no non-zero trit).
void oracle_twn_apply(const float* w, int64_t n, int64_t k, float d, int8_t* trits, float* scale) {
  for (int64_t r = 0; r < n; ++r) {
    double kept = 0.0;
    int64_t nonzero = 0;
    for (int64_t e = 0; e < k; ++e) {
      const float v = w[r * k + e];
      int8_t t = 0;
      if (std::fabs(v) > d) t = v > 0.0f ? int8_t(+1) : int8_t(-1);
      trits[r * k + e] = t;
      if (t != 0) {
        kept += std::fabs(double(v));
        ++nonzero;
      }
    }
    scale[r] = nonzero > 0 ? float(kept / double(nonzero)) : 0.0f;
  }
}

// The two steps above in order: Delta from the whole tensor, then trits and scales.
void oracle_twn_ternarize(const float* w, int64_t n, int64_t k, int8_t* trits,
                          float* scale, float* delta) {
  const float d = oracle_twn_delta(w, n * k);
  *delta = d;
  oracle_twn_apply(w, n, k, d, trits, scale);
}

// [BME] section 5 "Ternary math" (absmean scale gamma = mean|w|, BitNet
// b1.58) and [BTE] "Features" (mode absmean), the trit rule for a given gamma:
// q = w / gamma in float32, trit = RoundClip(q, -1, 1) = clamp(round-half-to-
// even(q), -1, 1); so |q| > 0.5 gives sign(q) and |q| <= 0.5 (ties included)
// gives 0.  gamma = 0 gives all zero trits.  Scales are the per-row
// least-squares scales of oracle_twn_apply ([BTE] "Features": per-channel
// least-squares scaling).
void oracle_absmean_apply(const float* w, int64_t n, int64_t k, float g, int8_t* trits, float* scale) {
  for (int64_t r = 0; r < n; ++r) {
    double kept = 0.0;
    int64_t nonzero = 0;
    for (int64_t e = 0; e < k; ++e) {
      const float v = w[r * k + e];
      int8_t t = 0;
      if (g > 0.0f) {
        const float q = v / g;
        const float rounded = std::nearbyint(q);  // default rounding mode: to nearest, ties to even
        t = rounded > 0.0f ? int8_t(+1) : (rounded < 0.0f ? int8_t(-1) : int8_t(0));
      }
      trits[r * k + e] = t;
      if (t != 0) {
        kept += std::fabs(double(v));
        ++nonzero;
      }
    }
    scale[r] = nonzero > 0 ? float(kept / double(nonzero)) : 0.0f;
  }
}

// The absmean mode in order: gamma = float32 of mean|W| over the whole tensor
// (float64 sum in element order, rounded once), then the trit rule above.
void oracle_absmean_ternarize(const float* w, int64_t n, int64_t k, int8_t* trits, float* scale,
                              float* gamma_out) {
  const int64_t total = n * k;
  double sum_abs = 0.0;
  for (int64_t e = 0; e < total; ++e) sum_abs += std::fabs(double(w[e]));
  const float g = float(total > 0 ? sum_abs / double(total) : 0.0);
  *gamma_out = g;
  oracle_absmean_apply(w, n, k, g, trits, scale);
}

// [BTE] "Features": 10 trits per 16-bit word, base 3.  Word j of a row holds
// trits 10j .. 10j+9; trit 10j+i contributes (trit + 1) * 3^i.  Missing trits
// past k count as 0 (digit 1).
void oracle_base3_pack(const int8_t* trits, int64_t n, int64_t k, uint16_t* packed) {
  const int64_t kt = words10(k);
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t j = 0; j < kt; ++j) {
      uint32_t word = 0, weight = 1;
      for (int64_t i = 0; i < 10; ++i) {
        const int64_t e = 10 * j + i;
        const int t = e < k ? int(trits[r * k + e]) : 0;
        word += uint32_t(t + 1) * weight;
        weight *= 3;
      }
      packed[r * kt + j] = uint16_t(word);
    }
  }
}

// Inverse of the above: digit i of word w is (w / 3^i) mod 3, trit = digit - 1.
// Returns the number of words >= 3^10 (not produced by the packer; such words
// are decoded digit by digit all the same, with the 10th digit taken mod 3).
int64_t oracle_base3_unpack(const uint16_t* packed, int64_t n, int64_t k, int8_t* trits) {
  const int64_t kt = words10(k);
  int64_t invalid = 0;
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t j = 0; j < kt; ++j) {
      const uint32_t word = packed[r * kt + j];
      if (word >= 59049u) ++invalid;
      uint32_t power = 1;
      for (int64_t i = 0; i < 10; ++i) {
        const int64_t e = 10 * j + i;
        const int digit = int((word / power) % 3u);
        if (e < k) trits[r * k + e] = int8_t(digit - 1);
        power *= 3;
      }
    }
  }
  return invalid;
}

// [BTE] Layer.forward: y[i,j] = scale_j * sum_e x[i,e] * t[j,e], with the
// activations given as bfloat16 (widened exactly) and everything summed in
// float64.  mag[i,j] = scale_j * sum_e |x[i,e] * t[j,e]| is the magnitude the
// tolerance of a float32-accumulating implementation is measured against.
static void ternary_one(const uint16_t* xrow, const int8_t* trow, int64_t k, float s,
                        double* y, double* mag) {
  double acc = 0.0, acc_abs = 0.0;
  for (int64_t e = 0; e < k; ++e) {
    const double p = bf16_to_double(xrow[e]) * double(trow[e]);
    acc += p;
    acc_abs += std::fabs(p);
  }
  *y = double(s) * acc;
  if (mag) *mag = std::fabs(double(s)) * acc_abs;
}

void oracle_ternary_gemm(const uint16_t* x_bf16, const uint16_t* packed, const float* scale,
                         int64_t m, int64_t n, int64_t k, double* out, double* mag) {
  const int64_t kt = words10(k);
  int8_t* t = new int8_t[k > 0 ? k : 1];
  for (int64_t j = 0; j < n; ++j) {
    oracle_base3_unpack(packed + j * kt, 1, k, t);
    for (int64_t i = 0; i < m; ++i)
      ternary_one(x_bf16 + i * k, t, k, scale[j], out + i * n + j, mag ? mag + i * n + j : nullptr);
  }
  delete[] t;
}

// The ternary layer with its per-channel bias ([BTE] ".tbin Format" biases,
// "Module Overview" Layer.forward): y = scale_j * sum + bias_j in float64, and
// mag = |scale_j| * sum |x t| + |bias_j| (the magnitude the tolerance scales with).
void oracle_ternary_linear(const uint16_t* x_bf16, const uint16_t* packed, const float* scale, const float* bias,
                           int64_t m, int64_t n, int64_t k, double* out, double* mag) {
  oracle_ternary_gemm(x_bf16, packed, scale, m, n, k, out, mag);
  if (!bias) return;
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j) {
      out[i * n + j] += double(bias[j]);
      if (mag) mag[i * n + j] += std::fabs(double(bias[j]));
    }
}

// [BTE] "Features" (sparse encoding: an index + sign format for high-sparsity
// layers) and "Module Overview" (Packer.pack_sparse).  Reading: for each weight
// row, the positions of its non-zero trits in increasing order, one 16-bit
// entry each -- the position in bits 0..14 (so k <= 32768) and bit 15 set when
// the trit is -1; row j's entries are entries[row_ptr[j] .. row_ptr[j+1]),
// row_ptr[0] = 0.
int64_t oracle_sparse_count(const int8_t* trits, int64_t n, int64_t k, int64_t* row_ptr) {
  row_ptr[0] = 0;
  for (int64_t j = 0; j < n; ++j) {
    int64_t c = 0;
    for (int64_t e = 0; e < k; ++e) c += trits[j * k + e] != 0 ? 1 : 0;
    row_ptr[j + 1] = row_ptr[j] + c;
  }
  return row_ptr[n];
}

void oracle_sparse_encode(const int8_t* trits, int64_t n, int64_t k, const int64_t* row_ptr, uint16_t* entries) {
  for (int64_t j = 0; j < n; ++j) {
    int64_t at = row_ptr[j];
    for (int64_t e = 0; e < k; ++e) {
      const int8_t t = trits[j * k + e];
      if (t != 0) entries[at++] = uint16_t(uint16_t(e) | (t < 0 ? 0x8000u : 0u));
    }
  }
}

// Inverse of oracle_sparse_encode; returns the number of malformed entries
// (position >= k, or positions not strictly increasing within a row).
int64_t oracle_sparse_decode(const int64_t* row_ptr, const uint16_t* entries, int64_t n, int64_t k, int8_t* trits) {
  int64_t bad = 0;
  for (int64_t e = 0; e < n * k; ++e) trits[e] = 0;
  for (int64_t j = 0; j < n; ++j) {
    int64_t prev = -1;
    for (int64_t q = row_ptr[j]; q < row_ptr[j + 1]; ++q) {
      const int64_t pos = entries[q] & 0x7FFF;
      if (pos >= k || pos <= prev) {
        ++bad;
        continue;
      }
      prev = pos;
      trits[j * k + pos] = (entries[q] & 0x8000) ? -1 : 1;
    }
  }
  return bad;
}

// The sparse layer: y[i,j] = scale_j * sum over row j's entries of (+-1) *
// x[i, position] (+ bias_j), in float64, with mag as in oracle_ternary_linear.
void oracle_sparse_gemm(const uint16_t* x_bf16, const int64_t* row_ptr, const uint16_t* entries, const float* scale,
                        const float* bias, int64_t m, int64_t n, int64_t k, double* out, double* mag) {
  (void)k;
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j) {
      double acc = 0.0, acc_abs = 0.0;
      for (int64_t q = row_ptr[j]; q < row_ptr[j + 1]; ++q) {
        const double v = bf16_to_double(x_bf16[i * k + (entries[q] & 0x7FFF)]);
        acc += (entries[q] & 0x8000) ? -v : v;
        acc_abs += std::fabs(v);
      }
      out[i * n + j] = double(scale[j]) * acc + (bias ? double(bias[j]) : 0.0);
      if (mag) mag[i * n + j] = std::fabs(double(scale[j])) * acc_abs + (bias ? std::fabs(double(bias[j])) : 0.0);
    }
}

void oracle_ternary_gemm_sampled(const uint16_t* x_bf16, const uint16_t* packed,
                                 const float* scale, int64_t m, int64_t n, int64_t k,
                                 const int64_t* rows, const int64_t* cols, int64_t count,
                                 double* out, double* mag) {
  (void)m;
  (void)n;
  const int64_t kt = words10(k);
  int8_t* t = new int8_t[k > 0 ? k : 1];
  for (int64_t s = 0; s < count; ++s) {
    oracle_base3_unpack(packed + cols[s] * kt, 1, k, t);
    ternary_one(x_bf16 + rows[s] * k, t, k, scale[cols[s]], out + s, mag ? mag + s : nullptr);
  }
  delete[] t;
}

}  // extern "C"
