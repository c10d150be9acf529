/*
 * bnn.h -- C ABI of the packed 1-bit / balanced-ternary matmul for NVIDIA B200
 * (sm_100a).  Library: libbnn.so (built in-tree by ternary_neural_net_b200/build.py).
 *
 * Sources the operations are defined by (page title, section):
 *   [BME] "Binary Math Effectiveness -- why / how / when", section 1 "The core
 *         identity": bit 0 encodes +1 and bit 1 encodes -1; <x,w> = n - 2d with
 *         d = popcount(x XOR w) over the logical n; "Edge cases": pad bits
 *         encode +1 and do not count, n = 0 gives 0, a channel scale alpha = 0
 *         gives 0, inputs <= 0 project to -1 and > 0 to +1.
 *   [ADR] "Architecture Decision Record", section "Decision": binary_gemm_u64,
 *         the packed XNOR/XOR + popcount matmul over uint64 words.
 *   [BTE] "BalancedTernaryEngine" README, section "Features": TWN threshold
 *         Delta = 0.7 * mean|W|, least-squares per-channel scale, 10 trits per
 *         16-bit word in base 3; "Module Overview": Layer.forward.
 *
 * Conventions shared by every call:
 *   - Layout.  Every matrix is row-major with the reduction dimension k
 *     contiguous: activations X[m,k], weights W[n,k] (the nn.Linear weight
 *     layout), outputs [m,n].  A packed sign row is kw = ceil(k/64) uint64
 *     words; element e of the row is bit (e mod 64) of word e/64 (least
 *     significant bit first), bits at positions >= k are 0.  A packed trit row
 *     is kt = ceil(k/10) uint16 words; word j holds trits 10j..10j+9, trit
 *     10j+i contributing (trit + 1) * 3^i, trits past k being 0 (digit 1).
 *     Rows are stored back to back with no extra pitch.
 *   - Pointers are DEVICE pointers (memory the caller allocated with any CUDA
 *     allocator, e.g. PyTorch's).  The caller owns every buffer; the library
 *     keeps no pointer after a call returns.  Buffers must not overlap.
 *   - Every call is asynchronous and ordered on the stream `s` it is given
 *     (0 = the legacy default stream).  It returns after enqueueing its
 *     kernels; the status covers argument checks and the launch only.  It
 *     never synchronises the device or the stream.
 *   - Errors.  BNN_ERR_INVALID_ARG: a size is negative or too large, or a
 *     required pointer is NULL.  BNN_ERR_MISALIGNED: a pointer is not aligned
 *     to its element size (8 bytes for uint64, 4 for float/int32, 2 for
 *     uint16).  BNN_ERR_CUDA: a CUDA runtime call or a kernel launch failed
 *     (bnn_last_cuda_error() gives the cudaError_t of the calling thread's
 *     last failure).  Nothing is written when a call fails its argument
 *     checks.  Sizes of 0 are valid and return BNN_OK.
 *   - Threads.  Calls are re-entrant; concurrent calls on different streams
 *     are independent.
 *   - Weights are static data.  The matmul calls (bnn_binary_gemm*,
 *     bnn_binary_linear, bnn_ternary_gemm*, bnn_ternary_linear,
 *     bnn_ternary_sparse_gemm) are launched with programmatic dependent
 *     launch: they may start, and read their WEIGHT operands (packed sign or
 *     trit rows; the sparse row_ptr and entries), while the kernel before them
 *     on the stream is still running.  Activations, scales, biases and outputs
 *     keep plain stream order.  So a weight operand must be complete before
 *     the stream reaches the matmuls that read it: after preparing it (with
 *     bnn_pack_signs, bnn_ternary_pack*, bnn_ternary_sparse_encode,
 *     bnn_tbin_load_ternary or any other kernel), synchronise the stream or
 *     the device, or prepare it on another stream and make this one wait on
 *     an event recorded there.  Activations packed or produced right before a
 *     matmul on the same stream need nothing.
 */
#ifndef BNN_H
#define BNN_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BNN_OK = 0,
  BNN_ERR_INVALID_ARG = 1,
  BNN_ERR_MISALIGNED = 2,
  BNN_ERR_CUDA = 3,
  BNN_ERR_UNSUPPORTED = 4
} bnn_status;

/* Largest logical reduction length accepted by the binary matmul: with
 * |dot| <= k <= 2^24 every dot is exact in float32, so the alpha epilogue is a
 * single correctly rounded float32 multiply. */
#define BNN_MAX_K_BINARY (1 << 24)

/*
 * bnn_pack_signs -- sign-pack float32 rows into uint64 words.  [BME] section 1
 * encoding table and "Edge cases" (<= 0 -> -1, > 0 -> +1; pad bits +1).
 *
 *   x     float32 [rows, k], device, 4-byte aligned.
 *   rows  number of rows, >= 0.
 *   k     logical row length, >= 0.
 *   out   uint64 [rows, ceil(k/64)], device, 8-byte aligned.  Bit e of a row
 *         is 1 exactly when !(x[e] > 0), so +-0, NaN and -inf give -1 (bit 1)
 *         and denormals keep their sign (no flush to zero).  Pad bits are 0.
 */
bnn_status bnn_pack_signs(const float* x, int64_t rows, int64_t k, uint64_t* out,
                          cudaStream_t s);

/*
 * bnn_binary_gemm -- packed XOR + popcount matmul with a per-output-channel
 * scale.  [ADR] "Decision" (binary_gemm_u64); [BME] section 1 (identity and
 * "Edge cases").
 *
 *   xp     uint64 [m, ceil(k/64)] packed activations, device, 8-byte aligned.
 *   wp     uint64 [n, ceil(k/64)] packed weights, device, 8-byte aligned.
 *          Pad bits of xp and wp must be 0 (bnn_pack_signs guarantees it);
 *          they are not masked.
 *   alpha  float32 [n] per-output-channel scale, device; may be NULL only
 *          when out is NULL.
 *   m, n   output shape, >= 0.
 *   k      logical reduction length, 0 <= k <= BNN_MAX_K_BINARY.
 *   dots   int32 [m, n] or NULL: dots[i,j] = k - 2 * popcount(xp_i XOR wp_j),
 *          the exact +-1 dot product.
 *   out    float32 [m, n] or NULL: out[i,j] = alpha[j] * (float)dots[i,j], one
 *          IEEE float32 multiply, round to nearest even.
 *   At least one of dots and out must be non-NULL.  With k = 0 every dot is 0
 *   and out is alpha * 0.
 */
bnn_status bnn_binary_gemm(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                           int64_t m, int64_t n, int64_t k, int32_t* dots, float* out,
                           cudaStream_t s);

/* Kernel family for bnn_binary_gemm_algo.  All give bit-identical results. */
typedef enum {
  BNN_ALGO_AUTO = 0,   /* what bnn_binary_gemm uses: POPC GEMV for m <= 8, MMA_S8 for
                          9 <= m <= 63, TC for m >= 64 */
  BNN_ALGO_POPC = 1,   /* XOR + 64-bit popcount on the integer pipe (skinny GEMV for m <= 8,
                          register-tiled GEMM otherwise) */
  BNN_ALGO_MMA_S8 = 2, /* packed bits expanded in registers to 0/-1 int8 fragments of
                          m16n8k32 s8 mma.sync; popc(a AND b) summed exactly in int32 */
  BNN_ALGO_TC = 3      /* packed bits expanded to 4-bit floats (1.0 or 0) in shared memory;
                          tcgen05.mma kind::mxf4 with unit scale factors sums popc(a AND b)
                          exactly into a float32 tensor-memory accumulator (every count up
                          to k <= 2^24 is a float32), and k - 2 popc(a) - 2 popc(b) +
                          4 popc(a AND b) is the dot */
} bnn_binary_algo;

/*
 * bnn_binary_gemm_algo -- bnn_binary_gemm with an explicit kernel family
 * (same arguments, outputs and errors; BNN_ERR_INVALID_ARG for an unknown
 * algo).  The identity it evaluates is the same in every family: the MMA
 * family sums the +-1 products directly, which equals k - 2*popcount(x XOR w)
 * exactly.
 */
bnn_status bnn_binary_gemm_algo(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                                int64_t m, int64_t n, int64_t k, int32_t* dots, float* out,
                                bnn_binary_algo algo, cudaStream_t s);

/*
 * bnn_binary_linear -- one binarised linear layer with its epilogue fused:
 * the packed matmul of bnn_binary_gemm, the channel scale, an optional
 * per-channel bias ([BTE] ".tbin Format": records carry per-channel biases)
 * and the sign pack of the layer output as the next layer's packed input
 * (binary activations from layer to layer, as in the FFN stacks of
 * BinaryLinear layers of the "binary_nn" README).
 *
 *   xp, wp, m, n, k   as for bnn_binary_gemm.
 *   alpha  float32 [n], device; required when out or next is non-NULL.
 *   bias   float32 [n], device, or NULL for no bias.
 *   y[i,j] = fl32(alpha[j] * (float)dot[i,j]), then, with a bias,
 *            fl32(y[i,j] + bias[j]): two IEEE float32 operations, round to
 *            nearest even, never fused into one multiply-add.
 *   dots   int32 [m, n] or NULL: the exact dots (as bnn_binary_gemm).
 *   out    float32 [m, n] or NULL: y.
 *   next   uint64 [m, ceil(n/64)] or NULL, 8-byte aligned: row i is
 *          bnn_pack_signs of row i of y (bit j = !(y[i,j] > 0), pad bits 0).
 *   At least one of dots, out and next must be non-NULL.  Runs on the
 *   tensor-core kernel family (BNN_ALGO_TC) for every m.  Errors as for
 *   bnn_binary_gemm.
 */
bnn_status bnn_binary_linear(const uint64_t* xp, const uint64_t* wp, const float* alpha,
                             const float* bias, int64_t m, int64_t n, int64_t k, int32_t* dots,
                             float* out, uint64_t* next, cudaStream_t s);

/*
 * bnn_ternary_pack -- TWN ternarisation, least-squares per-row scale and base-3
 * packing of a float32 weight matrix.  [BTE] "Features".
 *
 *   w       float32 [n, k] weights, device, 4-byte aligned.
 *   n, k    shape, >= 0, n * k < 2^40.
 *   packed  uint16 [n, ceil(k/10)] base-3 words (see Layout), device, 2-byte aligned.
 *   scale   float32 [n], device: scale[r] = float32(mean of |w[r,e]| over the
 *           e with a non-zero trit), 0 for a row whose trits are all 0; the
 *           least-squares scale for the row's trits.
 *   delta   float32 [1], device: Delta = float32(0.7 * mean|W|), the mean
 *           taken over all n*k weights in float64 (0 when n*k = 0).
 *   Trit of w[r,e]: +1 if |w| > Delta and w > 0, -1 if |w| > Delta and w < 0,
 *   else 0 (a tie |w| == Delta gives 0; NaN gives 0).
 *   Scratch: the float64 partial sums of |W| (8 bytes per 65536 weights) are
 *   taken from the stream-ordered allocator (cudaMallocAsync / cudaFreeAsync
 *   on s); BNN_ERR_CUDA if that allocation fails.  The reduction order is
 *   fixed, so results are bitwise reproducible from run to run.
 */
bnn_status bnn_ternary_pack(const float* w, int64_t n, int64_t k, uint16_t* packed,
                            float* scale, float* delta, cudaStream_t s);

/* Ternarisation rules for bnn_ternary_pack_mode. */
typedef enum {
  BNN_TERNARY_TWN = 0,      /* Delta = float32(0.7 mean|W|); trit = sign(w) where |w| > Delta */
  BNN_TERNARY_ABSMEAN = 1,  /* gamma = float32(mean|W|); trit = clamp(round-half-even(w / gamma), -1, 1) */
  BNN_TERNARY_DELTA = 2     /* a given threshold F >= 0; trit = sign(w) where |w| > F */
} bnn_ternary_mode;

/*
 * bnn_ternary_pack_mode -- ternarise, scale and pack with one of the three
 * quantisation modes of [BTE] "Features" ("twn", "absmean" -- the BitNet
 * b1.58 absmean scale of "Binary Math Effectiveness", section 5 -- and
 * "delta", a fixed threshold with MSE-optimal scales).  Every mode writes
 * the per-row least-squares scale (mean |w| over the row's non-zero trits, 0
 * for none) and base-3 words exactly as bnn_ternary_pack does.
 *
 *   mode        a bnn_ternary_mode; BNN_ERR_INVALID_ARG otherwise.
 *   threshold   F for BNN_TERNARY_DELTA (must be >= 0, not NaN); ignored
 *               by the other modes.
 *   thresh_out  float32 [1], device: Delta (TWN), gamma (ABSMEAN) or F (DELTA).
 *   In ABSMEAN the quotient w / gamma is one IEEE float32 division and a
 *   quotient of exactly +-0.5 rounds to 0; gamma = 0 gives all-zero trits.
 *   TWN is bnn_ternary_pack itself; ABSMEAN takes its float64 partial sums
 *   from the stream-ordered allocator like bnn_ternary_pack; DELTA allocates
 *   nothing.  Other arguments, layouts and errors as bnn_ternary_pack.
 */
bnn_status bnn_ternary_pack_mode(const float* w, int64_t n, int64_t k, int mode, float threshold,
                                 uint16_t* packed, float* scale, float* thresh_out, cudaStream_t s);

/*
 * bnn_ternary_pack_noalloc -- bnn_ternary_pack for callers that must not
 * allocate device memory.  The pages have no counterpart to this call: it is
 * an interface choice of this library.
 *
 * Some callers cannot allocate when they pack weights: a serving runtime that
 * reserves all device memory up front under its own allocator and forbids
 * allocation on its request path, a process whose device or driver setup has
 * no stream-ordered memory pools (cudaMallocAsync unavailable), or a
 * latency-bound loop that cannot risk an allocator call blocking or failing.
 * This entry point computes exactly what bnn_ternary_pack computes (same
 * kernels, same reduction order, bitwise the same outputs) and takes the
 * same arguments, but keeps its float64 partial sums in a fixed 64 KiB array
 * compiled into libbnn.so instead of allocating them.  It calls no
 * cudaMalloc, cudaMallocAsync, cudaFree or other allocating routine.
 *
 *   Limit: n * k <= 2^29 (536,870,912 weights, one partial sum per 65536
 *   weights in an array of 8192); larger sizes return BNN_ERR_INVALID_ARG
 *   with nothing written.
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it for the
 *   device's current CUDA context; make that first call before any stream
 *   capture on the device.  After a device reset (a new context) the next
 *   call looks the address up again, so it too should come before any
 *   capture.
 *   Sharing: every GPU that loads the library holds the array until the
 *   process exits, and all calls on a device share it.  Each call writes
 *   every slot it reads before reading it, so nothing needs clearing between
 *   calls, but two calls that overlap on the GPU (e.g. on streams with no
 *   ordering between them) race on the array and may both produce wrong
 *   results: order such calls on one stream or with events.
 */
bnn_status bnn_ternary_pack_noalloc(const float* w, int64_t n, int64_t k, uint16_t* packed,
                                    float* scale, float* delta, cudaStream_t s);

/*
 * bnn_ternary_gemm -- ternary layer forward: base-3 unpack and accumulate.
 * [BTE] "Module Overview" (Layer.forward) with the "Features" encoding.
 *
 *   x_bf16  bfloat16 [m, k] activations as raw 16-bit patterns, device,
 *           2-byte aligned.
 *   packed  uint16 [n, ceil(k/10)] base-3 words, device, 2-byte aligned; every
 *           word must be < 3^10 = 59049 (not checked on the hot path).
 *   scale   float32 [n], device.
 *   m, n, k shape, >= 0.
 *   out     float32 [m, n], device: out[i,j] = scale[j] * sum_e x[i,e] * t[j,e],
 *           the products exact, the sum accumulated in float32 (in an order
 *           the library chooses), the scale applied once after the sum.
 */
bnn_status bnn_ternary_gemm(const uint16_t* x_bf16, const uint16_t* packed, const float* scale,
                            int64_t m, int64_t n, int64_t k, float* out, cudaStream_t s);

/* Number of bounded device-side waits that ran out since the last reset
 * (a kernel that gives up a wait leaves its outputs unspecified and counts it
 * here); reset != 0 clears the count.  Synchronous; -1 if the query fails.
 * No counterpart on the pages: a diagnostic of this library. */
int bnn_device_error_count(int reset);

/* Kernel family for bnn_ternary_gemm_algo.  Results agree within the
 * tolerance of bnn_ternary_gemm (float32 accumulation in different orders). */
typedef enum {
  BNN_TALGO_AUTO = 0,        /* what bnn_ternary_gemm uses: CUDA-core GEMV for m <= 8; TC for
                                m > 8 when k % 8 == 0 and x is 16-byte aligned; MMA otherwise */
  BNN_TALGO_CUDA_CORES = 1,  /* CUDA-core GEMV kernels (m <= 8 only; BNN_ERR_UNSUPPORTED beyond) */
  BNN_TALGO_MMA = 2,         /* trits decoded to bf16 tiles, bf16 mma.sync m16n8k16 */
  BNN_TALGO_TC = 3           /* trits decoded to bf16, tcgen05.mma kind::f16 accumulating in tensor
                                memory; activations by TMA when k % 8 == 0 and x is 16-byte aligned,
                                and then for m <= 64 (packed 4-byte aligned) the decoded trits are
                                stored to tensor memory and read from there by the MMA */
} bnn_ternary_algo;

/*
 * bnn_ternary_gemm_algo -- bnn_ternary_gemm with an explicit kernel family
 * (a bnn_ternary_algo; BNN_ERR_INVALID_ARG for an unknown one).  Same
 * arguments, outputs and errors as bnn_ternary_gemm.
 */
bnn_status bnn_ternary_gemm_algo(const uint16_t* x_bf16, const uint16_t* packed, const float* scale,
                                 int64_t m, int64_t n, int64_t k, float* out, int algo, cudaStream_t s);

/*
 * bnn_ternary_linear -- bnn_ternary_gemm with the layer's per-channel bias
 * added in the epilogue ([BTE] ".tbin Format": each record carries per-channel
 * biases; "Module Overview": Layer.forward).
 *
 *   bias   float32 [n], device, 4-byte aligned, or NULL (then identical to
 *          bnn_ternary_gemm).
 *   out[i,j] = scale[j] * sum_e x[i,e] t[j,e] + bias[j], fp32 accumulation;
 *          within 1e-3 of |scale[j]| * sum |x t| + |bias[j]| of the exact value.
 *   Other arguments, kernels (the AUTO family) and errors as for
 *   bnn_ternary_gemm.
 */
bnn_status bnn_ternary_linear(const uint16_t* x_bf16, const uint16_t* packed, const float* scale,
                              const float* bias, int64_t m, int64_t n, int64_t k, float* out,
                              cudaStream_t s);

/*
 * Index + sign sparse ternary layers.  [BTE] "Features" (sparse encoding:
 * index + sign format for high-sparsity layers), "Module Overview"
 * (Packer.pack_sparse).  Format: row j's non-zero trits are entries
 * [row_ptr[j], row_ptr[j+1]) of a uint16 array, in increasing position order,
 * each the position (bits 0..14) with bit 15 set for -1; row_ptr[0] = 0.
 * Positions need 15 bits, so k <= BNN_MAX_K_SPARSE.
 */
#define BNN_MAX_K_SPARSE 32768

/*
 * bnn_ternary_sparse_count -- row_ptr of the sparse form of base-3 packed
 * weights.
 *   packed   uint16 [n, ceil(k/10)] base-3 words (see Layout), device.
 *   row_ptr  int64 [n + 1], device, 8-byte aligned: row_ptr[j+1] - row_ptr[j]
 *            = number of non-zero trits of row j; row_ptr[n] = total entries
 *            (read it back to size `entries`).
 */
bnn_status bnn_ternary_sparse_count(const uint16_t* packed, int64_t n, int64_t k, int64_t* row_ptr,
                                    cudaStream_t s);

/*
 * bnn_ternary_sparse_encode -- write the entries of the sparse form.
 *   row_ptr  as produced by bnn_ternary_sparse_count for the same packed.
 *   entries  uint16 [row_ptr[n]], device, 2-byte aligned (may be NULL only
 *            when n or k is 0).
 */
bnn_status bnn_ternary_sparse_encode(const uint16_t* packed, int64_t n, int64_t k, const int64_t* row_ptr,
                                     uint16_t* entries, cudaStream_t s);

/*
 * bnn_ternary_sparse_gemm -- the ternary layer over the sparse form:
 *   out[i,j] = scale[j] * sum_{e in row j} (+-1) x[i, pos_e] (+ bias[j]),
 *   x bf16 [m, k], float32 accumulation; scale float32 [n]; bias float32 [n]
 *   or NULL; out float32 [m, n].  Same tolerance as bnn_ternary_gemm.
 */
bnn_status bnn_ternary_sparse_gemm(const uint16_t* x_bf16, const int64_t* row_ptr, const uint16_t* entries,
                                   const float* scale, const float* bias, int64_t m, int64_t n, int64_t k,
                                   float* out, cudaStream_t s);

/*
 * .tbin ternary model files.  [BTE] ".tbin Format": header (magic "TBN\0",
 * version 1 or 2, num_layers, meta_len, JSON metadata), then records (kind
 * byte in version 2: 0 ternary, 1 raw float16; size; payload).  All fields
 * little-endian.  A ternary record holds out_features float16 scales, then 0
 * or out_features float16 biases (the record size decides), then
 * out_features x ceil(in_features/10) base-3 words.
 */
#define BNN_TBIN_MAX_DIMS 8

typedef struct bnn_tbin_record {
  uint32_t kind;            /* 0 ternary, 1 raw float16 */
  uint32_t name_len;        /* UTF-8 name: name_len bytes at name_offset */
  uint64_t name_offset;
  /* kind 0 */
  uint32_t out_features, in_features;
  float delta, sparsity;
  uint32_t num_biases;      /* 0 or out_features */
  uint32_t reserved;
  uint64_t scales_offset;   /* out_features float16 */
  uint64_t biases_offset;   /* num_biases float16 (0 when there are none) */
  uint64_t weights_offset;  /* weights_words uint16 base-3 words */
  uint64_t weights_words;
  /* kind 1 */
  uint32_t ndims;
  uint32_t dims[BNN_TBIN_MAX_DIMS];
  uint64_t data_offset;     /* data_elems float16 */
  uint64_t data_elems;
} bnn_tbin_record;

/*
 * bnn_tbin_parse -- read the record table of a .tbin file held in HOST memory
 * (file, len bytes); nothing is copied and no CUDA call is made.  *count =
 * num_layers; the first min(capacity, num_layers) records are written to
 * records (all byte offsets are from the start of the file).  version,
 * meta_offset and meta_len may be NULL.  BNN_ERR_INVALID_ARG for a bad magic
 * or version, a truncated file or a record whose size does not fit its fields.
 */
bnn_status bnn_tbin_parse(const uint8_t* file, uint64_t len, uint32_t* version, uint64_t* meta_offset,
                          uint64_t* meta_len, bnn_tbin_record* records, int64_t capacity, int64_t* count);

/*
 * bnn_tbin_load_ternary -- copy one ternary record out of the file's bytes in
 * DEVICE memory (file_dev, len bytes, any alignment) into the buffers the
 * ternary calls take: packed uint16 [out_features, ceil(in_features/10)],
 * scale float32 [out_features] (may be NULL), bias float32 [out_features] (may
 * be NULL; zeros when the record has no biases).  float16 -> float32 is exact.
 */
bnn_status bnn_tbin_load_ternary(const uint8_t* file_dev, uint64_t len, const bnn_tbin_record* rec,
                                 uint16_t* packed, float* scale, float* bias, cudaStream_t s);

/* bnn_tbin_load_raw -- a raw float16 record's data as float32 [data_elems]. */
bnn_status bnn_tbin_load_raw(const uint8_t* file_dev, uint64_t len, const bnn_tbin_record* rec, float* out,
                             cudaStream_t s);

/* Human-readable name of a status code (static storage, never NULL). */
const char* bnn_status_string(bnn_status st);

/* cudaError_t (as int) of the calling thread's most recent BNN_ERR_CUDA, or 0. */
int bnn_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BNN_H */
