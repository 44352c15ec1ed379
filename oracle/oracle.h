/*
 * oracle.h -- declarations of the CPU oracle for the emulated RCCLX collectives.
 *
 * TEST INFRASTRUCTURE ONLY.  The oracle is a plain, slow, single-threaded C
 * restatement of what the collectives compute.  Only the test-suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header, table or constant with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Layouts (all host memory, caller-allocated):
 *   a "rank buffer" array is [nranks][stride] elements of `dtype`, row r being
 *   the tensor that simulated rank r passes to the collective;
 *   fp8 payloads are uint8 codes (one per element) plus one fp32 scale per
 *   128-element block, blocks anchored at the first element of the segment
 *   being quantised.
 *
 * Every function returns 0 on success and a negative value when its contract
 * is broken (bad argument, non-finite input on an FP8 wire, no memory).
 */
#ifndef RLX_ORACLE_H
#define RLX_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1 };          /* element type of rank buffers   */
enum { ORC_NATIVE = 0, ORC_FP8 = 1 };        /* what crosses the emulated wire */

/* OCP FP8 E4M3 ("fn": no infinities, 0x7F/0xFF are NaN). */
float   orc_e4m3_value(uint8_t code);
uint8_t orc_e4m3_encode(float v);
/* Encode the fp32 values whose bit patterns are first, first+1, ... (n of them). */
void    orc_e4m3_encode_bits_range(uint32_t first, size_t n, uint8_t *out);

float    orc_bf16_to_f32(uint16_t h);
uint16_t orc_f32_to_bf16(float f);

/* Block quantisation of `rows` rows of n elements (row stride `stride`
 * elements for x and for codes); scales are [rows][ceil(n/128)]. */
int orc_quantize(int dtype, const void *x, size_t rows, size_t n, size_t stride,
                 uint8_t *codes, float *scales);
int orc_dequantize(const uint8_t *codes, const float *scales, size_t rows, size_t n,
                   size_t stride, int dtype, void *y);

/* SUM allreduce of [nranks][stride] rank buffers over `count` elements.
 * send == recv (in place) is allowed. */
int orc_allreduce_flat(int dtype, int wire, const void *send, void *recv,
                       size_t count, size_t stride, int nranks);
int orc_allreduce_tree(int dtype, int wire, const void *send, void *recv,
                       size_t count, size_t stride, int nranks);

/* reduce-scatter: send [nranks][send_stride >= nranks*m], recv [nranks][recv_stride >= m] */
int orc_reduce_scatter(int dtype, int wire, const void *send, size_t send_stride,
                       void *recv, size_t recv_stride, size_t m, int nranks);
/* all-gather: send [nranks][send_stride >= m], recv [nranks][recv_stride >= nranks*m] */
int orc_all_gather(int dtype, int wire, const void *send, size_t send_stride,
                   void *recv, size_t recv_stride, size_t m, int nranks);
/* all-to-all: send and recv [nranks][stride >= nranks*m] */
int orc_alltoall(int dtype, int wire, const void *send, size_t send_stride,
                 void *recv, size_t recv_stride, size_t m, int nranks);

/* Element count of one DDA-tree chunk for this count and rank count. */
size_t orc_tree_chunk(size_t count, int nranks);

#ifdef __cplusplus
}
#endif
#endif
