// rlx_reduce.cu -- the reducing passes: DDA-flat allreduce, DDA-tree pass 1
// (reduce-scatter into chunk owners) and the standalone ReduceScatter, each on
// the native wire and on the FP8 wire.
//
// DDA-flat: every rank reads every rank's buffer and reduces locally
// ("Meta open-sources RCCLX", infolabhq pt, "Direct Data Access (DDA) — De
// O(N) para O(1) de Latência").  On one GPU the N identical local reductions
// are one reduction per element index whose result is stored into all N rows.
// DDA-tree pass 1: rank c reduces chunk c (same section).  LP collectives:
// each sender's contribution is quantised to FP8 and dequantised by the
// receiver, sums are FP32 (RCCLX post, es, "Colectivos de mengua precisión").
//
// Work mapping
//   native wire: one thread per 16-byte vector of each row (4 fp32 or 8 bf16);
//     the thread loads that vector from all N ranks before adding, so N
//     16-byte loads are in flight per thread;
//   FP8 wire: one warp per 128-element block (two adjacent blocks for bf16),
//     4 elements per lane per block, so a block amax is one warp reduction;
//     the warp loads its blocks from all N ranks, dequantises each rank's
//     quantised block and sums in rank order.
// Units of work are numbered in memory order (chunk-major for chunked
// passes) and handed out in CTA-sized runs by for_each_unit, so the CTAs in
// flight stream one compact stretch of every row.
#include "rlx_passes.cuh"

namespace rlx {
namespace {

// ------------------------------------------------------------------ kernels

// Units per warp (per CTA run) of each kernel.
#ifndef RLX_P_NATIVE
#define RLX_P_NATIVE 1
#endif
#ifndef RLX_P_FP8
#define RLX_P_FP8 2
#endif
#ifndef RLX_P_FP8_FLAT
#define RLX_P_FP8_FLAT 1
#endif
// FP8 tree / reduce-scatter passes with fewer blocks than this run one block
// per warp (shorter dependent chain per warp: small-message latency), larger
// ones RLX_P_FP8 (fewer CTA start-ups: bandwidth).
#ifndef RLX_FP8_SMALL_BLOCKS
#define RLX_FP8_SMALL_BLOCKS 32768
#endif
constexpr int kPn = RLX_P_NATIVE;
constexpr int kPf = RLX_P_FP8;
constexpr int kPfFlat = RLX_P_FP8_FLAT;

// Resident CTAs per SM requested from the compiler (caps registers per
// thread) for kernels with up to 8 ranks; the 16-rank forms hold twice the
// data and get the default.
#ifndef RLX_MINB_NATIVE
#define RLX_MINB_NATIVE 3
#endif
#ifndef RLX_MINB_FP8
#define RLX_MINB_FP8 4
#endif
#ifndef RLX_MINB_FP8_BF16
#define RLX_MINB_FP8_BF16 4
#endif
#ifndef RLX_MINB_FP8_FLAT
#define RLX_MINB_FP8_FLAT 4
#endif
template <int NR> constexpr int kMinBlocksNative = NR <= 8 ? RLX_MINB_NATIVE : 1;
template <typename T, int NR>
constexpr int kMinBlocksFp8 = NR > 8 ? 1 : sizeof(T) == 2 ? RLX_MINB_FP8_BF16 : RLX_MINB_FP8;
template <int NR> constexpr int kMinBlocksFp8Flat = NR <= 8 ? RLX_MINB_FP8_FLAT : 1;

// DDA-flat, native: unit g = 32 consecutive 16-byte vectors (lane l: 32g + l).
template <typename T, int NR, bool VEC, bool EXACT>
__global__ void __launch_bounds__(kThreads, kMinBlocksNative<NR>)
flat_native_kernel(const T *send, T *recv, size_t count, size_t stride, int n) {
    constexpr int V = VecN<T>::n;
    const size_t nvec = (count + V - 1) / V;
    const uint32_t units = static_cast<uint32_t>((nvec + 31) / 32);
    with_rank_count<NR, EXACT>(n, [&](auto nn) {
        for_each_unit<kPn>(units, [&](uint32_t g) {
            const size_t i0 = (static_cast<size_t>(g) * 32 + lane_id()) * V;
            with_full((static_cast<size_t>(g) + 1) * 32 * V <= count, [&](auto full) {
                const int valid = vec_valid_in<V>(i0, count, full);
                if (valid == 0) return;
                float acc[V];
                reduce_vec<T, NR, VEC>(send + i0, stride, nn, valid, full, acc);
                for (int r = 0; r < nn; ++r) storev<T, VEC>(recv + r * stride + i0, valid, acc);
            });
        });
    });
}

// DDA-flat, FP8: unit u = the BPU blocks from block u*BPU on (BPU = kBpu<T>,
// or 1 for small bf16 messages, see launch_allreduce_flat).
template <typename T, int NR, bool VEC, bool EXACT, int BPU>
__global__ void __launch_bounds__(kThreads, kMinBlocksFp8Flat<NR>)
flat_fp8_kernel(const T *send, T *recv, size_t count, size_t stride, int n) {
    const uint32_t units = static_cast<uint32_t>((count + BPU * kBlock - 1) / (BPU * kBlock));
    const bool wide = rows_16b(recv, stride);
    with_rank_count<NR, EXACT>(n, [&](auto nn) {
        for_each_unit<kPfFlat>(units, [&](uint32_t u) {
            const size_t base = static_cast<size_t>(u) * BPU * kBlock;
            with_full(base + BPU * kBlock <= count, [&](auto full) {
                int valid[BPU];
#pragma unroll
                for (int j = 0; j < BPU; ++j)
                    valid[j] = decltype(full)::value ? 4 : lane_valid(base + j * kBlock, count);
                float acc[BPU][4];
                reduce_blocks_fp8<T, NR, VEC, BPU>(send + base, stride, nn, valid, acc);
                store_blocks<T, VEC, BPU>(recv + base, stride, nn, full, wide, valid, acc);
            });
        });
    });
}

// DDA-tree pass 1, native (one unit body per unit, see rlx_passes.cuh).
template <typename T, int NR, bool VEC, bool EXACT>
__global__ void __launch_bounds__(kThreads, kMinBlocksNative<NR>)
tree_reduce_native_kernel(const T *send, T *recv, size_t count, size_t stride, int n,
                          size_t chunk, FastDiv per_chunk) {
    const uint32_t units = per_chunk.d * static_cast<uint32_t>(n);
    with_rank_count<NR, EXACT>(n, [&](auto nn) {
        for_each_unit<kPn>(units, [&](uint32_t g) {
            tree_reduce_native_unit<T, NR, VEC>(g, send, recv, count, stride, nn, chunk, per_chunk);
        });
    });
}

// DDA-tree pass 1, FP8.
template <typename T, int NR, bool VEC, int P, bool EXACT>
__global__ void __launch_bounds__(kThreads, kMinBlocksFp8<T, NR>)
tree_reduce_fp8_kernel(const T *send, size_t count, size_t stride, int n,
                       uint8_t *ws_codes, float *ws_scales) {
    constexpr int BPU = kBpu<T>;
    const uint32_t units = static_cast<uint32_t>((count + BPU * kBlock - 1) / (BPU * kBlock));
    with_rank_count<NR, EXACT>(n, [&](auto nn) {
        for_each_unit<P>(units, [&](uint32_t u) {
            tree_reduce_fp8_unit<T, NR, VEC>(u, send, count, stride, nn, ws_codes, ws_scales);
        });
    });
}

// ReduceScatter, native: unit = (destination rank r, 32 vectors of chunk r).
template <typename T, int NR, bool VEC, bool EXACT>
__global__ void __launch_bounds__(kThreads, kMinBlocksNative<NR>)
rs_native_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n,
                 FastDiv per_chunk) {
    constexpr int V = VecN<T>::n;
    const uint32_t units = per_chunk.d * static_cast<uint32_t>(n);
    with_rank_count<NR, EXACT>(n, [&](auto nn) {
        for_each_unit<kPn>(units, [&](uint32_t g) {
            const uint32_t r = fast_div(g, per_chunk);
            const size_t u0 = static_cast<size_t>(g - r * per_chunk.d) * 32 * V;
            const size_t j0 = u0 + static_cast<size_t>(lane_id()) * V;
            with_full(u0 + 32 * V <= m, [&](auto full) {
                const int valid = vec_valid_in<V>(j0, m, full);
                if (valid == 0) return;
                float acc[V];
                reduce_vec<T, NR, VEC>(send + r * m + j0, sstride, nn, valid, full, acc);
                storev<T, VEC>(recv + r * rstride + j0, valid, acc);
            });
        });
    });
}

// ReduceScatter, FP8: unit = (destination rank r, kBpu<T> adjacent blocks of
// chunk r); blocks anchored at the chunk start r*m.
template <typename T, int NR, bool VEC, int P, bool EXACT>
__global__ void __launch_bounds__(kThreads, kMinBlocksFp8<T, NR>)
rs_fp8_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n,
              FastDiv per_chunk) {
    constexpr int BPU = kBpu<T>;
    const uint32_t units = per_chunk.d * static_cast<uint32_t>(n);
    const bool wide = rows_16b(recv, rstride);
    with_rank_count<NR, EXACT>(n, [&](auto nn) {
        for_each_unit<P>(units, [&](uint32_t g) {
            const uint32_t r = fast_div(g, per_chunk);
            const size_t j0 = static_cast<size_t>(g - r * per_chunk.d) * BPU * kBlock;
            with_full(j0 + BPU * kBlock <= m, [&](auto full) {
                int valid[BPU];
#pragma unroll
                for (int j = 0; j < BPU; ++j)
                    valid[j] = decltype(full)::value ? 4 : lane_valid(j0 + j * kBlock, m);
                float acc[BPU][4];
                reduce_blocks_fp8<T, NR, VEC, BPU>(send + r * m + j0, sstride, nn, valid, acc);
                store_blocks<T, VEC, BPU>(recv + r * rstride + j0, rstride, 1, full, wide, valid,
                                          acc);
            });
        });
    });
}

// ------------------------------------------------------------- dispatching

// Calls f.template operator()<T, NR, VEC, EX>() for the rank bound NR >= n;
// EX: n == NR (the kernel sums a compile-time number of ranks).
#ifndef RLX_FIXED_RANKS
#define RLX_FIXED_RANKS 1
#endif
template <typename T, int NRV, bool VEC, typename F>
cudaError_t dispatch_exact(int n, F &&f) {
    if (RLX_FIXED_RANKS && n == NRV) return f.template operator()<T, NRV, VEC, true>();
    return f.template operator()<T, NRV, VEC, false>();
}
template <typename F>
cudaError_t dispatch(rlx_dtype dtype, int n, bool vec, F &&f) {
#define RLX_CASE_NR(T, NRV)                                                       \
    if (n <= NRV) return vec ? dispatch_exact<T, NRV, true>(n, f)                 \
                             : dispatch_exact<T, NRV, false>(n, f);
#define RLX_CASE_T(T) \
    RLX_CASE_NR(T, 2) RLX_CASE_NR(T, 4) RLX_CASE_NR(T, 8) RLX_CASE_NR(T, 16)
    if (dtype == RLX_F32) { RLX_CASE_T(float) }
    else { RLX_CASE_T(uint16_t) }
#undef RLX_CASE_T
#undef RLX_CASE_NR
    return cudaErrorInvalidValue;
}

template <typename K, typename... Args>
cudaError_t launch(K kernel, size_t units, size_t units_per_cta, cudaStream_t stream,
                   Args... args) {
    const dim3 grid = grid_for(reinterpret_cast<const void *>(kernel), units, units_per_cta);
    if (grid.x == 0) return cudaErrorInvalidValue;
    return launch_kernel(kernel, grid, stream, args...);
}

constexpr size_t kWarps = kThreads / 32;

// Below one wave of warps (148 SMs x 32), a flat FP8 call on bf16 is bound by
// the latency of each warp's unit, not by bandwidth: units of one block
// instead of two halve that chain and double the warps working on it
// (decode bf16 8 x [32, 8192] from a CUDA graph: 2.7 against 3.2 us).  The
// cluster-form tree keeps two-block units: with one-block units it measured
// slower (5.4 against 5.0 us at the same size).
#ifndef RLX_SMALL_BPU1
#define RLX_SMALL_BPU1 1
#endif
constexpr size_t kSmallUnits = 148 * 32;

}  // namespace

cudaError_t launch_allreduce_flat(const void *send, void *recv, size_t count, size_t stride,
                                  int nranks, rlx_dtype dtype, rlx_wire wire, bool vec,
                                  cudaStream_t stream) {
    return dispatch(dtype, nranks, vec, [&]<typename T, int NR, bool VEC, bool EX>() {
        const T *s = static_cast<const T *>(send);
        T *r = static_cast<T *>(recv);
        if (wire == RLX_WIRE_NATIVE) {
            // the run-time rank count measured faster here than the compile-time
            // one (159.5 against 161.9 us at 8 x 16 Mi fp32)
            const size_t units = ((count + VecN<T>::n - 1) / VecN<T>::n + 31) / 32;
            return launch(flat_native_kernel<T, NR, VEC, false>, units, kWarps * kPn, stream, s, r,
                          count, stride, nranks);
        }
        const size_t units = (count + kBpu<T> * kBlock - 1) / (kBpu<T> * kBlock);
        if (kBpu<T> > 1 && RLX_SMALL_BPU1 && units < kSmallUnits)
            return launch(flat_fp8_kernel<T, NR, VEC, EX, 1>, units * kBpu<T>, kWarps * kPfFlat,
                          stream, s, r, count, stride, nranks);
        return launch(flat_fp8_kernel<T, NR, VEC, EX, kBpu<T>>, units, kWarps * kPfFlat, stream, s,
                      r, count, stride, nranks);
    });
}

cudaError_t launch_tree_reduce(const void *send, void *recv, size_t count, size_t stride,
                               int nranks, size_t chunk, rlx_dtype dtype, rlx_wire wire,
                               uint8_t *ws_codes, float *ws_scales, bool vec,
                               cudaStream_t stream) {
    return dispatch(dtype, nranks, vec, [&]<typename T, int NR, bool VEC, bool EX>() {
        const T *s = static_cast<const T *>(send);
        if (wire == RLX_WIRE_NATIVE) {
            const size_t per = tree_reduce_native_per_chunk<T>(chunk);
            if (per >= (size_t{1} << 32)) return cudaErrorInvalidValue;
            return launch(tree_reduce_native_kernel<T, NR, VEC, EX>,
                          per * static_cast<size_t>(nranks), kWarps * kPn, stream, s,
                          static_cast<T *>(recv), count, stride, nranks, chunk,
                          make_fastdiv(static_cast<uint32_t>(per)));
        }
        const size_t nblk = (count + kBlock - 1) / kBlock;
        const size_t units = (nblk + kBpu<T> - 1) / kBpu<T>;
        if (nblk < RLX_FP8_SMALL_BLOCKS)
            return launch(tree_reduce_fp8_kernel<T, NR, VEC, 1, EX>, units, kWarps, stream, s, count,
                          stride, nranks, ws_codes, ws_scales);
        return launch(tree_reduce_fp8_kernel<T, NR, VEC, kPf, EX>, units, kWarps * kPf, stream, s,
                      count, stride, nranks, ws_codes, ws_scales);
    });
}

cudaError_t launch_reduce_scatter(const void *send, size_t send_stride, void *recv,
                                  size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                                  rlx_wire wire, bool vec, cudaStream_t stream) {
    return dispatch(dtype, nranks, vec, [&]<typename T, int NR, bool VEC, bool EX>() {
        const T *s = static_cast<const T *>(send);
        T *r = static_cast<T *>(recv);
        const size_t nn = static_cast<size_t>(nranks);
        const size_t per = wire == RLX_WIRE_NATIVE
                               ? ((m + VecN<T>::n - 1) / VecN<T>::n + 31) / 32
                               : (m + kBpu<T> * kBlock - 1) / (kBpu<T> * kBlock);
        if (per >= (size_t{1} << 32)) return cudaErrorInvalidValue;
        const FastDiv fd = make_fastdiv(static_cast<uint32_t>(per));
        if (wire == RLX_WIRE_NATIVE)
            return launch(rs_native_kernel<T, NR, VEC, EX>, per * nn, kWarps * kPn, stream, s,
                          send_stride, r, recv_stride, m, nranks, fd);
        if (per * kBpu<T> * nn < RLX_FP8_SMALL_BLOCKS)
            return launch(rs_fp8_kernel<T, NR, VEC, 1, EX>, per * nn, kWarps, stream, s, send_stride,
                          r, recv_stride, m, nranks, fd);
        return launch(rs_fp8_kernel<T, NR, VEC, kPf, EX>, per * nn, kWarps * kPf, stream, s,
                      send_stride, r, recv_stride, m, nranks, fd);
    });
}

}  // namespace rlx
