// CPU oracle for the packed 1-bit / balanced-ternary matmul -- declarations.
// TEST INFRASTRUCTURE ONLY (see bnn_oracle.cpp): loaded by the tests, the
// smoke check and the bench's CPU-baseline leg, never by the product path.
// All pointers are host pointers; every matrix is row-major with the reduction
// dimension k contiguous.  Packed sign rows hold ceil(k/64) uint64 words, packed
// trit rows ceil(k/10) uint16 words.
#pragma once
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

void oracle_pack_signs(const float* x, int64_t rows, int64_t k, uint64_t* out);
void oracle_unpack_signs(const uint64_t* p, int64_t rows, int64_t k, int8_t* out);
int64_t oracle_count_pad_bits(const uint64_t* p, int64_t rows, int64_t k);
void oracle_binary_gemm(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                        int64_t m, int64_t n, int64_t k, int32_t* dots, float* out);
void oracle_binary_gemm_sampled(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                                int64_t m, int64_t n, int64_t k, const int64_t* rows,
                                const int64_t* cols, int64_t count, int32_t* dots, float* out);
void oracle_binary_linear(const uint64_t* xp, const uint64_t* wp, const float* alpha, const float* bias,
                          int64_t m, int64_t n, int64_t k, int32_t* dots, float* y, uint64_t* next);
float oracle_twn_delta(const float* w, int64_t total);
void oracle_twn_apply(const float* w, int64_t n, int64_t k, float delta, int8_t* trits, float* scale);
void oracle_twn_ternarize(const float* w, int64_t n, int64_t k, int8_t* trits,
                          float* scale, float* delta);
void oracle_absmean_apply(const float* w, int64_t n, int64_t k, float gamma, int8_t* trits, float* scale);
void oracle_absmean_ternarize(const float* w, int64_t n, int64_t k, int8_t* trits, float* scale,
                              float* gamma_out);
void oracle_base3_pack(const int8_t* trits, int64_t n, int64_t k, uint16_t* packed);
int64_t oracle_base3_unpack(const uint16_t* packed, int64_t n, int64_t k, int8_t* trits);
void oracle_ternary_gemm(const uint16_t* x_bf16, const uint16_t* packed, const float* scale,
                         int64_t m, int64_t n, int64_t k, double* out, double* mag);
void oracle_ternary_linear(const uint16_t* x_bf16, const uint16_t* packed, const float* scale, const float* bias,
                           int64_t m, int64_t n, int64_t k, double* out, double* mag);
int64_t oracle_sparse_count(const int8_t* trits, int64_t n, int64_t k, int64_t* row_ptr);
void oracle_sparse_encode(const int8_t* trits, int64_t n, int64_t k, const int64_t* row_ptr, uint16_t* entries);
int64_t oracle_sparse_decode(const int64_t* row_ptr, const uint16_t* entries, int64_t n, int64_t k, int8_t* trits);
void oracle_sparse_gemm(const uint16_t* x_bf16, const int64_t* row_ptr, const uint16_t* entries, const float* scale,
                        const float* bias, int64_t m, int64_t n, int64_t k, double* out, double* mag);
void oracle_ternary_gemm_sampled(const uint16_t* x_bf16, const uint16_t* packed,
                                 const float* scale, int64_t m, int64_t n, int64_t k,
                                 const int64_t* rows, const int64_t* cols, int64_t count,
                                 double* out, double* mag);

#ifdef __cplusplus
}
#endif
