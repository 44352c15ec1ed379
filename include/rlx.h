/*
 * rlx.h -- C ABI of librlx.so: emulated RCCLX collectives on one B200 GPU.
 *
 * N simulated ranks live as the N rows of one device array [N][stride] in a
 * single GPU's memory (no peer access, no second GPU).  Each call computes, on
 * the caller's stream, what the RCCLX collective of that name leaves in every
 * rank's output buffer:
 *
 *   DDA-flat allreduce  -- every rank reads every rank's buffer and reduces it
 *     itself ("Meta open-sources RCCLX", dev.infolabhq.com/pt, section
 *     "Direct Data Access (DDA) — De O(N) para O(1) de Latência"; RCCLX post,
 *     Spanish copy, section "Ataque directo a datos (DDA)").
 *   DDA-tree allreduce  -- a reduce-scatter phase followed by an all-gather
 *     phase (same sections).
 *   Low-precision (LP) collectives -- AllReduce, AllGather, AlltoAll and
 *     ReduceScatter on FP32 or BF16 data with FP8 on the wire (up to 4:1) and
 *     all arithmetic in FP32; precision is lost only at the one or two
 *     quantisations of each collective (RCCLX post, Spanish copy, section
 *     "Colectivos de mengua precisión"; infolabhq summary, section
 *     "Coletivos de Baixa Precisão — Compressão FP8 com Precisão FP32").
 *
 * The pages name only "FP8".  This library fixes the format as follows, and
 * every FP8 result below is defined by it:
 *   - OCP FP8 E4M3 ("fn": max finite 448, no infinities);
 *   - one fp32 scale per 128 consecutive elements; blocks are anchored at the
 *     first element of the segment a sender quantises (the row, or the chunk
 *     of the row that one collective step sends);
 *   - scale s = fl32(amax / 448), amax = max |x| over the block;
 *   - code = E4M3 round-to-nearest-even of fl32(x / s), saturating at +-448,
 *     sign kept; s == 0 gives scale 0 and codes +-0;
 *   - dequantised value = fl32(e4m3(code) * s);
 *   - every emulated wire hop quantises, a rank's own contribution included,
 *     so all ranks' results are bit-identical;
 *   - sums run in fp32 in rank order 0, 1, ..., N-1 from the first term, with
 *     no fused multiply-add; a bf16 result is one round-to-nearest-even of the
 *     fp32 result;
 *   - with nranks == 1 nothing crosses a wire and every collective copies.
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers (cudaMalloc / torch CUDA memory) on the
 *     current device; the caller owns every buffer.  The library allocates
 *     nothing.  It keeps no state between calls, with one exception: the
 *     fixed device array of rlx_allreduce_tree_noalloc and the cache of its
 *     device address (one entry per device, see that entry point).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is only
 *     enqueued: the call returns before the GPU finishes.  Faults during the
 *     kernel surface at the caller's next synchronisation.
 *   - Arguments are checked before anything is launched; a call that returns
 *     an error launched nothing.  A count of 0 returns RLX_OK at once.
 *   - Element pointers must be aligned to their element size (4 B fp32, 2 B
 *     bf16) and scale pointers to 4 B (else RLX_ERR_ALIGNMENT).  Wider
 *     alignment (16 B rows and chunks) selects the vectorised kernels;
 *     anything else runs element-wise kernels with the same results.
 *   - nranks is 1..RLX_MAX_RANKS.  Row strides are in elements.
 *   - Size products that overflow size_t, and calls over RLX_MAX_ELEMENTS
 *     elements (all ranks together), are rejected (RLX_ERR_INVALID_ARG).
 *   - FP8-wire inputs must be finite; non-finite inputs give unspecified codes.
 */
#ifndef RLX_H
#define RLX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define RLX_API __attribute__((visibility("default")))
#else
#define RLX_API
#endif

#define RLX_BLOCK 128     /* elements per FP8 scale block           */
#define RLX_MAX_RANKS 16  /* largest simulated rank count supported */
/* Largest element count of one call, all ranks (rows) together: 2^36, more
 * than any B200 holds; larger requests return RLX_ERR_INVALID_ARG. */
#define RLX_MAX_ELEMENTS ((size_t)1 << 36)

typedef enum {
    RLX_OK = 0,
    RLX_ERR_INVALID_ARG = 1,  /* null pointer, bad enum, bad size/stride, overlap */
    RLX_ERR_ALIGNMENT = 2,    /* pointer not aligned to its element type          */
    RLX_ERR_UNSUPPORTED = 3,  /* reduction op other than SUM                      */
    RLX_ERR_WORKSPACE = 4,    /* workspace missing, too small or misaligned       */
    RLX_ERR_CUDA = 5,         /* a CUDA call failed (see rlx_last_cuda_error)     */
    RLX_ERR_TIMEOUT = 6       /* a bounded device-side wait ran out (written to a
                                 call's status word, see rlx_allreduce_tree_fused) */
} rlx_status;

typedef enum { RLX_F32 = 0, RLX_BF16 = 1 } rlx_dtype;
typedef enum { RLX_WIRE_NATIVE = 0, RLX_WIRE_FP8_E4M3 = 1 } rlx_wire;
typedef enum { RLX_SUM = 0 } rlx_op;
typedef enum {
    RLX_COLL_ALLREDUCE_FLAT = 0,
    RLX_COLL_ALLREDUCE_TREE = 1,
    RLX_COLL_REDUCE_SCATTER = 2,
    RLX_COLL_ALL_GATHER = 3,
    RLX_COLL_ALLTOALL = 4,
    RLX_COLL_ALLREDUCE_TREE_FUSED = 5
} rlx_coll;

/*
 * Block quantisation to FP8 E4M3 (the sender side of every LP collective).
 *   x       [rows][stride] elements of `dtype` (bf16 widens exactly to fp32);
 *           only the first n of each row are read.
 *   codes   [rows][stride] bytes; the first n of each row are written.
 *   scales  [rows][ceil(n/128)] fp32, contiguous.
 * Blocks are anchored at each row's first element; the last may be partial.
 * x must not overlap codes or scales.
 */
RLX_API rlx_status rlx_quantize_fp8(const void *x, rlx_dtype dtype, size_t rows, size_t n,
                            size_t stride, uint8_t *codes, float *scales, void *stream);

/*
 * Block dequantisation (the receiver side): y = fl32(e4m3(code) * scale),
 * written as `dtype` (bf16: one round-to-nearest-even).  Same layouts as
 * rlx_quantize_fp8, y in place of x.  y must not overlap codes or scales.
 */
RLX_API rlx_status rlx_dequantize_fp8(const uint8_t *codes, const float *scales, size_t rows,
                              size_t n, size_t stride, void *y, rlx_dtype dtype,
                              void *stream);

/*
 * DDA-flat SUM allreduce.  send and recv are [nranks][stride] of `dtype`;
 * afterwards recv[r][i] = SUM_s w(send[s][i]) for every rank r and i < count,
 * w the identity on the native wire and dequantise(quantise(.)) of the
 * sender's row on the FP8 wire (one quantisation).  send == recv (in place) is
 * allowed; any other overlap is rejected.  Elements past count are untouched.
 */
RLX_API rlx_status rlx_allreduce_flat(const void *send, void *recv, size_t count, size_t stride,
                              int nranks, rlx_dtype dtype, rlx_wire wire, rlx_op op,
                              void *stream);

/*
 * DDA-tree SUM allreduce: a reduce-scatter pass then an all-gather pass.
 * Chunk c (owned by rank c) is elements [c*C, min((c+1)*C, count)) with
 * C = 128 * ceil(ceil(count/128) / nranks).
 *   native wire: pass 1 writes the reduced chunk c into recv[c]; pass 2 copies
 *     it to every other rank.  Bit-identical to rlx_allreduce_flat.
 *   FP8 wire: pass 1 reduces the dequantised FP8 contributions and quantises
 *     the reduced chunk again (second quantisation) into `workspace`; pass 2
 *     dequantises it into every rank.
 * Small messages (up to a few waves of the GPU) run both passes in one kernel
 * launch over thread-block clusters: each cluster reduces a contiguous range
 * of the chunks, synchronises its CTAs with the cluster barrier and gathers
 * the same range; larger ones run the passes as two launches.  The results
 * are the same bytes either way.
 * workspace: device memory of at least rlx_workspace_bytes(RLX_COLL_ALLREDUCE_TREE,
 * ...) bytes, 16-byte aligned, not overlapping send/recv; may be NULL when that
 * size is 0.  Its contents on return are unspecified.  Same-stream calls may
 * reuse one workspace; concurrent calls need one each.  In place allowed.
 */
RLX_API rlx_status rlx_allreduce_tree(const void *send, void *recv, size_t count, size_t stride,
                              int nranks, rlx_dtype dtype, rlx_wire wire, rlx_op op,
                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * DDA-tree SUM allreduce in ONE kernel launch: the same results as
 * rlx_allreduce_tree, bit for bit, but the all-gather of chunk c starts as
 * soon as chunk c is reduced instead of after the whole reduce-scatter pass,
 * and there is no second launch (the pages credit the DDA-tree with
 * near-constant latency: "Meta open-sources RCCLX", infolabhq pt, section
 * "Direct Data Access (DDA) — De O(N) para O(1) de Latência").  Meant for
 * small and medium messages, where launch latency dominates.
 *
 * The kernel's CTAs coordinate through the workspace: the reduce-scatter
 * work of chunk c adds to a per-chunk count with release semantics, and the
 * all-gather work of chunk c waits, with acquire loads, until that count is
 * complete.  Every wait is bounded: it gives up after wait_limit_ns
 * nanoseconds of the GPU's global timer (0 = RLX_DEFAULT_WAIT_NS), or after a
 * fixed number of polls if the timer does not advance; the kernel then skips
 * the work that depended on the wait, returns, and reports RLX_ERR_TIMEOUT in
 * *status.  No wait can block forever on work that is never started: work is
 * handed out in order, all of the reduce-scatter work before any of the
 * all-gather work, and only to CTAs that are already running.
 *
 * workspace: device memory of at least
 *   rlx_workspace_bytes(RLX_COLL_ALLREDUCE_TREE_FUSED, count, nranks, dtype, wire)
 * bytes, 16-byte aligned, not overlapping send/recv.  Its first
 * RLX_TREE_SYNC_BYTES bytes are synchronisation words that must be ZERO
 * before the first call on a workspace (cudaMemset it once); every call
 * leaves them zero when its kernel ends, after a timeout too.  Word 4 + c
 * (32-bit) counts the reduce-scatter work finished on chunk c; chunk c is
 * ready when that count, read as a signed number, reaches the chunk's total
 * (so a count preset to INT_MIN never gets there).  The rest
 * (FP8 wire only) carries the reduced chunks' FP8 payload.  Calls that can
 * run at the same time need a workspace each.
 * status: NULL, or a device int the kernel sets to RLX_OK or RLX_ERR_TIMEOUT
 *   when it ends (read it after synchronising).  On RLX_ERR_TIMEOUT recv is
 *   unspecified.
 * The host return value covers argument checks and the launch only.
 * Everything else as rlx_allreduce_tree (in place allowed).
 */
#define RLX_TREE_SYNC_BYTES 256
#define RLX_DEFAULT_WAIT_NS 1000000000ull
RLX_API rlx_status rlx_allreduce_tree_fused(const void *send, void *recv, size_t count,
                                            size_t stride, int nranks, rlx_dtype dtype,
                                            rlx_wire wire, rlx_op op, void *workspace,
                                            size_t workspace_bytes, int *status,
                                            uint64_t wait_limit_ns, void *stream);

/*
 * ReduceScatter: send [nranks][send_stride >= nranks*m], recv
 * [nranks][recv_stride >= m]; recv[r][j] = SUM_s w(send[s][r*m + j]), j < m,
 * where on the FP8 wire each sender quantises the chunk it sends with blocks
 * anchored at the chunk start.  send and recv must not overlap.
 */
RLX_API rlx_status rlx_reduce_scatter(const void *send, size_t send_stride, void *recv,
                              size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                              rlx_wire wire, rlx_op op, void *stream);

/*
 * AllGather: send [nranks][send_stride >= m], recv [nranks][recv_stride >= nranks*m];
 * recv[r][s*m + j] = w(send[s][j]).  send and recv must not overlap.
 */
RLX_API rlx_status rlx_all_gather(const void *send, size_t send_stride, void *recv,
                          size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                          rlx_wire wire, void *stream);

/*
 * AlltoAll: send and recv [nranks][stride >= nranks*m];
 * recv[r][s*m + j] = w(send[s][r*m + j]) -- an N x N transpose of m-element
 * chunks.  send and recv must not overlap.
 */
RLX_API rlx_status rlx_alltoall(const void *send, size_t send_stride, void *recv,
                        size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                        rlx_wire wire, void *stream);

/*
 * DDA-tree SUM allreduce without a workspace argument, for callers that
 * cannot allocate device memory where they run the collective (a plug-in
 * handed only its input and output buffers, or a loop that must not call
 * cudaMalloc because it can synchronise the whole device).  The pages have
 * no counterpart: this is a convenience of this library.
 *
 * Same arguments and results as rlx_allreduce_tree, bit for bit.  On the FP8
 * wire the payload between the two passes lives in a fixed device array that
 * the library defines at file scope (16.5 MiB on every GPU that loads the
 * library, held until the process exits), so count may be at most
 * RLX_NOALLOC_MAX_COUNT elements per rank; larger counts return
 * RLX_ERR_WORKSPACE and launch nothing.  The native wire needs no payload
 * and has no such limit.  The library allocates nothing.
 *
 * The first call on each device looks up the array's device address with
 * that device current and caches it with the id of the device's CUDA
 * context; after the context is replaced (cudaDeviceReset) the next call
 * looks the address up again.  Make such a first call before any stream
 * capture.
 * All calls on a device share the one array: two calls whose kernels can
 * overlap on the GPU (different streams, no ordering between them) race on
 * it.  Calls ordered on one stream are safe; nothing in the array needs to
 * be cleared between calls.
 */
#define RLX_NOALLOC_MAX_COUNT 16777216u
RLX_API rlx_status rlx_allreduce_tree_noalloc(const void *send, void *recv, size_t count,
                                              size_t stride, int nranks, rlx_dtype dtype,
                                              rlx_wire wire, rlx_op op, void *stream);

/* Workspace bytes the collective needs for these arguments (0 = none). */
RLX_API size_t rlx_workspace_bytes(rlx_coll coll, size_t count, int nranks, rlx_dtype dtype,
                           rlx_wire wire);

/* Static English text for a status code. */
RLX_API const char *rlx_status_string(rlx_status status);

/* The cudaError_t of the last CUDA failure seen by this host thread (0 if none). */
RLX_API int rlx_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* RLX_H */
