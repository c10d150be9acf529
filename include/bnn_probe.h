/*
 * bnn_probe.h -- measurement helpers exported by libbnn.so next to the matmul
 * calls of bnn.h.  They are not steps of the method; the bench uses them to
 * measure, on the same device, the roofline denominators the kernels are
 * bounded by: the integer-pipe rate of the XOR + popcount matmul and the
 * read-only HBM stream rate of the batch-1 GEMVs (which only read weights).
 */
#ifndef BNN_PROBE_H
#define BNN_PROBE_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#include "bnn.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * bnn_probe_popc -- enqueue one kernel of `blocks` x 256 threads in which
 * every thread runs `iters` rounds of 8 independent dependency chains.
 *   mode 0: each round of a chain is one 32-bit popcount and one add
 *           (counts 1 popcount per round);
 *   mode 1: each round is the matmul's inner step on a 64-bit word pair:
 *           XOR of both halves, two 32-bit popcounts, one 3-input add
 *           (counts 1 word-op = 64 bit-MACs per round).
 *   sink   int32 [blocks * 256] device buffer that receives the chains'
 *          final values (so the work cannot be optimised away).
 *   ops    host out: the number of counted operations the kernel performs
 *          (blocks * 256 * iters * 8).
 * Asynchronous on s; time it with events around the call.
 */
bnn_status bnn_probe_popc(int mode, int64_t blocks, int64_t iters, int32_t* sink, double* ops,
                          cudaStream_t s);

/*
 * bnn_probe_stream_read -- enqueue one kernel of `blocks` x 512 threads that
 * reads `bytes` bytes of `buf` once with 16-byte streaming loads (each warp a
 * contiguous 2 KiB block per step, four loads in flight per thread, blocks
 * strided across the grid) and writes nothing else.
 *   buf    device, 16-byte aligned; bytes a multiple of 16 (>= 0).
 *   sink   uint32 [1] device; written only when the fold of the data equals
 *          a fixed key (so the loads cannot be optimised away).
 * Time it with events around the call: bytes / time is the read-only HBM
 * bandwidth when bytes is well above the L2 size.  BNN_ERR_INVALID_ARG /
 * BNN_ERR_MISALIGNED for bad arguments.  A diagnostic of this library.
 */
bnn_status bnn_probe_stream_read(const void* buf, int64_t bytes, int64_t blocks, uint32_t* sink,
                                 cudaStream_t s);

/*
 * bnn_probe_wait_limit -- bound, in polls, the main mbarrier waits of the
 * tensor-core binary GEMM kernels (bnn_binary_gemm for m >= 64,
 * BNN_ALGO_TC, bnn_binary_linear) launched after this call; 0 restores the
 * normal bound (suspending polls for up to one second of wall time).  The
 * final waits for copies and MMAs already in flight keep the normal bound
 * whatever the setting.  A wait that runs out
 * makes its CTA skip every store, wait for its copies and MMAs, free its
 * tensor memory and return; bnn_device_error_count() counts it.  With a
 * small limit (a few polls) the first waits run out before the first copies
 * land, which is how a test exercises that path without any GPU fault.
 * Process-wide, host only; always BNN_OK.  A diagnostic of this library (no
 * counterpart on the pages).
 */
bnn_status bnn_probe_wait_limit(uint32_t polls);

/*
 * bnn_probe_ternary_plan -- the launch plan bnn_ternary_gemm uses for one
 * activation tile (1 <= m <= 64, k % 8 == 0, aligned operands: the kernel that
 * decodes into tensor memory), computed on the host from given occupancy:
 *   n, k    weight rows and logical reduction length (both >= 1);
 *   active  host int[4]: how many clusters of 1, 2, 3 and 4 CTAs of that
 *           kernel fit the GPU at once (0 excludes that cluster size); the
 *           library itself asks the CUDA occupancy API;
 *   rows    host out: weight rows per CTA (32, 64, 96 or 128);
 *   ks      host out: CTAs per cluster splitting the 256-trit stages (1..4).
 * Host only, no CUDA call; BNN_ERR_INVALID_ARG for bad arguments.  A
 * diagnostic of this library (no counterpart on the pages).
 */
bnn_status bnn_probe_ternary_plan(int64_t n, int64_t k, const int* active, int* rows, int* ks);

#ifdef __cplusplus
}
#endif

#endif /* BNN_PROBE_H */
