// .tbin ternary model files: a host-side parser of the record table and a
// device-side loader of one ternary record into the buffers the ternary calls
// take (base-3 words, float32 scales and biases).
//
// "BalancedTernaryEngine" README, ".tbin Format" (version 2; version 1 has no
// record kind byte).  Every field is little-endian.  A ternary record holds
// out_feat float16 scales (one per output channel), then 0 or out_feat float16
// biases -- the record size decides which -- then out_feat x ceil(in_feat/10)
// base-3 words.  The loader reads the file's bytes where they already sit in
// device memory: one thread per output element assembles its little-endian
// 16-bit field from two byte loads (fields sit at any byte offset, since names
// have any length) and widens float16 to float32 (exact).
#include <cuda_fp16.h>

#include <cstring>

#include "bnn_internal.cuh"

namespace {

bool rd(const uint8_t* f, uint64_t len, uint64_t at, void* dst, uint64_t n) {
  if (at > len || n > len - at) return false;
  std::memcpy(dst, f + at, n);  // little-endian host: the bytes are the value
  return true;
}

template <typename T>
bool rdv(const uint8_t* f, uint64_t len, uint64_t at, T& v) {
  return rd(f, len, at, &v, sizeof(T));
}

__device__ __forceinline__ uint16_t le16(const uint8_t* p) {
  return static_cast<uint16_t>(p[0] | (static_cast<uint16_t>(p[1]) << 8));
}

__global__ void tbin_ternary_kernel(const uint8_t* __restrict__ file, uint64_t w_off, uint64_t s_off, uint64_t b_off,
                                    int64_t words, int64_t out_f, int has_bias, uint16_t* __restrict__ packed,
                                    float* __restrict__ scale, float* __restrict__ bias) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < words; i += stride)
    packed[i] = le16(file + w_off + 2 * i);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < out_f; i += stride) {
    if (scale) scale[i] = __half2float(__ushort_as_half(le16(file + s_off + 2 * i)));
    if (bias) bias[i] = has_bias ? __half2float(__ushort_as_half(le16(file + b_off + 2 * i))) : 0.0f;
  }
}

__global__ void tbin_raw_kernel(const uint8_t* __restrict__ file, uint64_t off, int64_t count, float* __restrict__ out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride)
    out[i] = __half2float(__ushort_as_half(le16(file + off + 2 * i)));
}

int grid_for(int64_t work) {
  const int64_t need = (work + 255) / 256;
  const int64_t cap = static_cast<int64_t>(bnn::sm_count()) * 8;
  return static_cast<int>(need < 1 ? 1 : (need < cap ? need : cap));
}

}  // namespace

extern "C" bnn_status bnn_tbin_parse(const uint8_t* file, uint64_t len, uint32_t* version, uint64_t* meta_offset,
                                     uint64_t* meta_len, bnn_tbin_record* records, int64_t capacity,
                                     int64_t* count) {
  if (!file || !count || capacity < 0 || (capacity > 0 && !records)) return BNN_ERR_INVALID_ARG;
  uint32_t ver = 0, num = 0, mlen = 0;
  if (len < 16 || std::memcmp(file, "TBN\0", 4) != 0 || !rdv(file, len, 4, ver) || !rdv(file, len, 8, num) ||
      !rdv(file, len, 12, mlen) || (ver != 1 && ver != 2) || mlen > len - 16)
    return BNN_ERR_INVALID_ARG;
  if (version) *version = ver;
  if (meta_offset) *meta_offset = 16;
  if (meta_len) *meta_len = mlen;
  uint64_t at = 16 + static_cast<uint64_t>(mlen);
  for (uint32_t r = 0; r < num; ++r) {
    bnn_tbin_record rec;
    std::memset(&rec, 0, sizeof(rec));
    uint8_t kind = 0;
    if (ver == 2 && !rdv(file, len, at++, kind)) return BNN_ERR_INVALID_ARG;
    uint32_t size = 0;
    if (!rdv(file, len, at, size)) return BNN_ERR_INVALID_ARG;
    at += 4;
    if (size > len - at) return BNN_ERR_INVALID_ARG;
    const uint64_t end = at + size;
    uint16_t name_len = 0;
    if (!rdv(file, end, at, name_len) || name_len > end - at - 2) return BNN_ERR_INVALID_ARG;
    rec.kind = kind;
    rec.name_offset = at + 2;
    rec.name_len = name_len;
    uint64_t q = at + 2 + name_len;
    if (kind == 0) {
      uint32_t out_f = 0, in_f = 0;
      if (!rdv(file, end, q, out_f) || !rdv(file, end, q + 4, in_f) || !rdv(file, end, q + 8, rec.delta) ||
          !rdv(file, end, q + 12, rec.sparsity))
        return BNN_ERR_INVALID_ARG;
      q += 16;
      const uint64_t words = static_cast<uint64_t>(out_f) * ((static_cast<uint64_t>(in_f) + 9) / 10);
      const uint64_t fixed = 2ull * out_f + 2ull * words;
      if (fixed > end - q) return BNN_ERR_INVALID_ARG;
      const uint64_t left = end - q - fixed;
      if (left != 0 && left != 2ull * out_f) return BNN_ERR_INVALID_ARG;
      rec.out_features = out_f;
      rec.in_features = in_f;
      rec.scales_offset = q;
      rec.num_biases = left ? out_f : 0;
      rec.biases_offset = left ? q + 2ull * out_f : 0;
      rec.weights_offset = q + 2ull * out_f + left;
      rec.weights_words = words;
    } else if (kind == 1) {
      uint8_t nd = 0;
      if (!rdv(file, end, q, nd) || nd > BNN_TBIN_MAX_DIMS) return BNN_ERR_INVALID_ARG;
      uint64_t elems = 1;
      for (uint8_t d = 0; d < nd; ++d) {
        if (!rdv(file, end, q + 1 + 4ull * d, rec.dims[d])) return BNN_ERR_INVALID_ARG;
        // the product never exceeds the file's length, so it cannot wrap
        if (rec.dims[d] != 0 && elems > len / rec.dims[d]) return BNN_ERR_INVALID_ARG;
        elems *= rec.dims[d];
      }
      q += 1 + 4ull * nd;
      if (end - q != 2 * elems) return BNN_ERR_INVALID_ARG;
      rec.ndims = nd;
      rec.data_offset = q;
      rec.data_elems = elems;
    } else {
      return BNN_ERR_INVALID_ARG;
    }
    if (static_cast<int64_t>(r) < capacity) records[r] = rec;
    at = end;
  }
  *count = num;
  return BNN_OK;
}

extern "C" bnn_status bnn_tbin_load_ternary(const uint8_t* file_dev, uint64_t len, const bnn_tbin_record* rec,
                                            uint16_t* packed, float* scale, float* bias, cudaStream_t s) {
  if (!file_dev || !rec || rec->kind != 0 || !packed) return BNN_ERR_INVALID_ARG;
  const uint64_t words = rec->weights_words, out_f = rec->out_features;
  // The record may come from the caller rather than from bnn_tbin_parse, so
  // nothing in it is trusted: the word count must be the documented output
  // size, and every byte the kernel reads must lie inside the file.  Counts
  // are compared against halved byte lengths (never doubled), so no product
  // can wrap.
  const uint64_t row_words = (static_cast<uint64_t>(rec->in_features) + 9) / 10;
  if (words != out_f * row_words) return BNN_ERR_INVALID_ARG;  // out_f, row_words < 2^32: no wrap
  if (rec->weights_offset > len || words > (len - rec->weights_offset) / 2 || rec->scales_offset > len ||
      out_f > (len - rec->scales_offset) / 2 ||
      (rec->num_biases && (rec->biases_offset > len || out_f > (len - rec->biases_offset) / 2)) ||
      (rec->num_biases != 0 && rec->num_biases != out_f))
    return BNN_ERR_INVALID_ARG;
  if (!bnn::aligned(packed, 2) || (scale && !bnn::aligned(scale, 4)) || (bias && !bnn::aligned(bias, 4)))
    return BNN_ERR_MISALIGNED;
  const int64_t work = static_cast<int64_t>(words > out_f ? words : out_f);
  if (work == 0) return BNN_OK;
  tbin_ternary_kernel<<<grid_for(work), 256, 0, s>>>(file_dev, rec->weights_offset, rec->scales_offset,
                                                     rec->biases_offset, static_cast<int64_t>(words),
                                                     static_cast<int64_t>(out_f), rec->num_biases ? 1 : 0, packed,
                                                     scale, bias);
  return bnn::check_launch();
}

extern "C" bnn_status bnn_tbin_load_raw(const uint8_t* file_dev, uint64_t len, const bnn_tbin_record* rec,
                                        float* out, cudaStream_t s) {
  if (!file_dev || !rec || rec->kind != 1 || !out) return BNN_ERR_INVALID_ARG;
  // a caller-supplied record is not trusted: halve the byte length instead of doubling the count
  if (rec->data_offset > len || rec->data_elems > (len - rec->data_offset) / 2) return BNN_ERR_INVALID_ARG;
  if (!bnn::aligned(out, 4)) return BNN_ERR_MISALIGNED;
  if (rec->data_elems == 0) return BNN_OK;
  tbin_raw_kernel<<<grid_for(static_cast<int64_t>(rec->data_elems)), 256, 0, s>>>(
      file_dev, rec->data_offset, static_cast<int64_t>(rec->data_elems), out);
  return bnn::check_launch();
}
