/*
 * fa_debug.h -- self-test entry points of libfa.so.  They exercise single hardware
 * primitives the attention kernels are built from, so that a fault in a descriptor
 * encoding or in the failure-detection path can be isolated on one tile.  They are not
 * part of the attention method and have no counterpart on the source pages.
 * Same conventions as fa.h: device pointers, asynchronous on `stream`, fa_status return,
 * nothing launched on a non-zero return.
 */
#ifndef FA_DEBUG_H_
#define FA_DEBUG_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* One CTA computes C = A * B with tcgen05.mma (bf16 in, fp32 accumulate in TMEM) and
 * reads the accumulator back with tcgen05.ld.  A is [128][k] bf16 row-major; C is
 * [128][n] fp32 row-major; n, k in {64, 128}.
 *   mode 0: B is [n][k] bf16 row-major (K-major; C = A B^T), A and B in shared memory.
 *   mode 1: B is [k][n] bf16 row-major (MN-major), A staged in TENSOR memory as packed
 *           bf16 pairs (the P operand layout of the forward kernel).
 *   mode 2: B is [k][n] bf16 row-major (MN-major), A in shared memory. */
int fa_debug_umma_tile(const void* a, const void* b, float* c, int n, int k, int mode,
                       void* stream);

/* Evaluates, for each of the n fp32 inputs x[i] (device pointers), the kernels' software
 * exp2 (range reduction to [-1/2, 1/2] + degree-3 minimax polynomial on the FMA pipe) into
 * y_poly[i] and the hardware ex2.approx into y_hw[i].  1 <= n <= 2^28. */
int fa_debug_exp2(const float* x, float* y_poly, float* y_hw, int n, void* stream);

/* Loads one box of 128 rows x 64 elements (rows row0 .. row0+127 of head h of batch b,
 * head-dim elements 64*chunk .. 64*chunk+63) of a [B][N][H][d] bf16 tensor x with a TMA
 * copy, through the same tensor-map encoding and 128-byte swizzle as the attention kernels,
 * and writes it unswizzled to y ([128][64] bf16, row-major).  Rows past N read as zero. */
int fa_debug_tma_tile(const void* x, void* y, int B, int N, int H, int d, int b, int h, int row0,
                      int chunk, void* stream);

/* One CTA: lane r (0..127) writes in[r][0..ncols) into tensor-memory columns [0, ncols)
 * with tcgen05.st and reads them back with tcgen05.ld into out[r][0..ncols).
 * ncols in {32, 64, 128, 256}; in, out: [128][ncols] 32-bit words. */
int fa_debug_tmem_roundtrip(const uint32_t* in, uint32_t* out, int ncols, void* stream);

/* Dumps the forward kernel's persistent schedule: for a launch of `grid` CTAs on a
 * (B, H, N, causal) problem, units[c][r] (c < grid, r < max_rounds) is the unit CTA c works
 * on in round r, encoded bh * num_pairs + pair (num_pairs = ceil(N / 256)), and -1 after the
 * last one. */
int fa_debug_fwd_schedule(int B, int H, int N, int causal, int grid, int* units, int max_rounds,
                          void* stream);

/* Launches one CTA whose only work is a bounded wait on an mbarrier that nothing ever
 * arrives at.  The wait gives up after `timeout_ns` nanoseconds (1e3 .. 1e10), records
 * FA_ERR_TIMEOUT in a status word and the CTA exits normally.  status_word_or_null: NULL
 * for the library-owned word, or a backward workspace (its first int is that call's word,
 * see fa_read_device_status), 4-byte aligned.  Read the result with
 * fa_read_device_status() on the same word. */
int fa_debug_wait_timeout(long long timeout_ns, void* status_word_or_null, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_DEBUG_H_ */
