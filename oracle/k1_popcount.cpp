// CPU BASELINE, not the oracle: the pages' own packed XOR + popcount matmul,
// restated in plain C++ so that the GPU can be timed against the method as
// the pages run it on a CPU.
//
// TEST AND BENCHMARK INFRASTRUCTURE ONLY: loaded by the tests (which check it
// against the oracle) and by the bench's CPU-baseline leg, never by the
// product path.  It shares nothing with the oracle (bnn_oracle.cpp never
// counts bits; this file does nothing else) or with the CUDA library.
//
// Source: "Architecture Decision Record", section "Decision": a native
// binary_gemm_u64 kernel, packed words XORed and counted with the 64-bit
// population count, row by row, single-threaded ("Accepted non-goals": no
// multithreading in that design).  "Binary Math Effectiveness", section 1:
// <x,w> = n - 2 * popcount(x XOR w) over the logical n; "Edge cases": the
// channel scale alpha multiplies the dot.
//
// Restatement: for every activation row i and weight row j, the XOR of each
// pair of words is population-counted (std::popcount, the hardware
// instruction with -mpopcnt) and summed; dot = k - 2 * sum; out = alpha_j *
// float(dot).  The loop nest is the plain one, rows of X outermost; `threads`
// > 1 splits the (row, column) pairs over OpenMP threads in contiguous
// blocks (static schedule), so a single-row GEMV spreads too -- the pages'
// setting is threads = 1.
#include <bit>
#include <cstdint>

#include <omp.h>

extern "C" {

void k1_binary_gemm(const uint64_t* xp, const uint64_t* wp, const float* alpha, int64_t m, int64_t n, int64_t k,
                    int threads, int32_t* dots, float* out) {
  const int64_t kw = (k + 63) / 64;
#pragma omp parallel for collapse(2) num_threads(threads) schedule(static)
  for (int64_t i = 0; i < m; ++i) {
    for (int64_t j = 0; j < n; ++j) {
      const uint64_t* x = xp + i * kw;
      const uint64_t* w = wp + j * kw;
      int64_t d = 0;
      for (int64_t t = 0; t < kw; ++t) d += std::popcount(x[t] ^ w[t]);
      const int32_t dot = static_cast<int32_t>(k - 2 * d);
      if (dots) dots[i * n + j] = dot;
      if (out) out[i * n + j] = alpha[j] * static_cast<float>(dot);
    }
  }
}

// Threads an OpenMP region of `threads` threads actually runs with.
int k1_threads_used(int threads) {
  int used = 0;
#pragma omp parallel num_threads(threads)
  {
#pragma omp single
    used = omp_get_num_threads();
  }
  return used;
}

}  // extern "C"
