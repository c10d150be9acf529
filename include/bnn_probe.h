/*
 * bnn_probe.h -- measurement helper exported by libbnn.so next to the four
 * matmul calls of bnn.h.  It is not a step of the method; the bench uses it to
 * measure the integer-pipe rate that the XOR + popcount matmul is bounded by,
 * so the roofline denominator is a number taken on the same device.
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
