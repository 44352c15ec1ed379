// rlx_gather.cu -- the distributing passes: DDA-tree pass 2 (all-gather of the
// reduced chunks), the standalone AllGather and AlltoAll, and the one-rank
// copy, on the native and FP8 wires.
//
// DDA-tree pass 2: every rank fetches every reduced chunk ("Meta open-sources
// RCCLX", infolabhq pt, "Direct Data Access (DDA) — De O(N) para O(1) de
// Latência").  AllGather / AlltoAll are two of the LP collectives (RCCLX post,
// es, "Colectivos de mengua precisión"): on the FP8 wire each sender
// quantises what it sends and the receiver dequantises it.
//
// On the native wire these passes move bytes only (16-byte vectors, no
// conversion), so results are bit copies; a warp moves kUnroll x 512
// contiguous bytes per step (lane l takes vectors l, l+32, ...), so each of
// its stores to a destination row continues the previous one.  On the FP8
// wire a warp handles J consecutive 128-element blocks at once (4 elements
// per lane per block; J per element type, see kJa2a and kJag):
// it reads them, applies dequantise(quantise(.)) in registers and writes
// every destination.
// Units of work are numbered in memory order (segment-major) and handed out
// in CTA-sized runs by for_each_unit, so the CTAs in flight stream one
// compact stretch of the data.
#include "rlx_passes.cuh"

namespace rlx {
namespace {

#ifndef RLX_P_COPY
#define RLX_P_COPY 1
#endif
#ifndef RLX_P_GFP8
#define RLX_P_GFP8 1
#endif
constexpr int kPc = RLX_P_COPY;      // units per warp per CTA run, native copies
constexpr int kPg = RLX_P_GFP8;      // units per warp per CTA run, FP8 passes

// ------------------------------------------------------------------ kernels

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
copy_kernel(const T *src, T *dst, size_t n) {
    const uint32_t units = static_cast<uint32_t>(((n + kV<T> - 1) / kV<T> + kWarpVecs - 1) / kWarpVecs);
    for_each_unit<kPc>(units, [&](uint32_t g) {
        with_full(unit_full<T>(g, n), [&](auto full) {
            RawVec<T, VEC> a[kUnroll];
            int valid[kUnroll];
            load_unit<T, VEC>(src, g, n, full, a, valid);
            store_unit<T, VEC>(dst, g, a, valid);
        });
    });
}

// DDA-tree pass 2, native (unit bodies in rlx_passes.cuh).
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
tree_gather_native_kernel(T *recv, size_t count, size_t stride, int n, size_t chunk,
                          FastDiv per_chunk) {
    const uint32_t units = per_chunk.d * static_cast<uint32_t>(n);
    for_each_unit<kPc>(units, [&](uint32_t g) {
        tree_gather_native_unit<T, VEC>(g, recv, count, stride, n, chunk, per_chunk);
    });
}

// DDA-tree pass 2, FP8.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
tree_gather_fp8_kernel(T *recv, size_t count, size_t stride, int n, const uint8_t *ws_codes,
                       const float *ws_scales) {
    const uint32_t units = static_cast<uint32_t>(tree_gather_fp8_units(count));
    for_each_unit<kPg>(units, [&](uint32_t g) {
        tree_gather_fp8_unit<T, VEC>(g, recv, count, stride, n, ws_codes, ws_scales);
    });
}

// AllGather, native: unit = (source rank s, unit of its row).
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
ag_native_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n,
                 FastDiv per_row) {
    const uint32_t units = per_row.d * static_cast<uint32_t>(n);
    for_each_unit<kPc>(units, [&](uint32_t g) {
        const uint32_t s = fast_div(g, per_row);
        const size_t unit = g - s * per_row.d;
        with_full(unit_full<T>(unit, m), [&](auto full) {
            RawVec<T, VEC> a[kUnroll];
            int valid[kUnroll];
            load_unit<T, VEC>(send + s * sstride, unit, m, full, a, valid);
            for (int r = 0; r < n; ++r) store_unit<T, VEC>(recv + r * rstride + s * m, unit, a, valid);
        });
    });
}

// AllGather, FP8: unit = (source rank s, J blocks of its row); blocks
// anchored at the row start.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
ag_fp8_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n,
              FastDiv per_row) {
    const uint32_t units = per_row.d * static_cast<uint32_t>(n);
    const int e0 = lane_id() * 4;
    constexpr int J = kJag<T>;
    for_each_unit<kPg>(units, [&](uint32_t g) {
        const uint32_t s = fast_div(g, per_row);
        const size_t b0 = static_cast<size_t>(g - s * per_row.d) * J;
        with_full((b0 + J) * kBlock <= m, [&](auto full) {
            const T *src = send + s * sstride + b0 * kBlock + e0;
            float v[J][4];
            int valid[J];
#pragma unroll
            for (int j = 0; j < J; ++j) {
                valid[j] = decltype(full)::value ? 4 : lane_valid((b0 + j) * kBlock, m);
                load4<T, VEC>(src + j * kBlock, valid[j], v[j]);
            }
            wire_fp8_blocks<J>(v);
            // row by row: all J blocks of a row before the next row (storing
            // each block to every row in turn measured 5 % slower)
            for (int r = 0; r < n; ++r) {
                T *dst = recv + r * rstride + s * m + b0 * kBlock + e0;
#pragma unroll
                for (int j = 0; j < J; ++j) store4<T, VEC>(dst + j * kBlock, valid[j], v[j]);
            }
        });
    });
}

// AlltoAll, native: unit = (pair p = s*n + r, unit of the chunk): chunk r of
// rank s goes to chunk s of rank r.  Pairs in s-major order read each source
// row front to back.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
a2a_native_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n,
                  FastDiv per_chunk, FastDiv ranks) {
    const uint32_t units = per_chunk.d * static_cast<uint32_t>(n) * static_cast<uint32_t>(n);
    for_each_unit<kPc>(units, [&](uint32_t g) {
        const uint32_t pair = fast_div(g, per_chunk);
        const uint32_t s = fast_div(pair, ranks), r = pair - s * ranks.d;
        const size_t unit = g - pair * per_chunk.d;
        with_full(unit_full<T>(unit, m), [&](auto full) {
            RawVec<T, VEC> a[kUnroll];
            int valid[kUnroll];
            load_unit<T, VEC>(send + static_cast<size_t>(s) * sstride + static_cast<size_t>(r) * m,
                              unit, m, full, a, valid);
            store_unit<T, VEC>(recv + static_cast<size_t>(r) * rstride + static_cast<size_t>(s) * m,
                               unit, a, valid);
        });
    });
}

// AlltoAll, FP8: unit = (pair, J blocks); blocks anchored at the chunk start.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
a2a_fp8_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n,
               FastDiv per_chunk, FastDiv ranks) {
    const uint32_t units = per_chunk.d * static_cast<uint32_t>(n) * static_cast<uint32_t>(n);
    const int e0 = lane_id() * 4;
    constexpr int J = kJa2a<T>;
    for_each_unit<kPg>(units, [&](uint32_t g) {
        const uint32_t pair = fast_div(g, per_chunk);
        const uint32_t s = fast_div(pair, ranks), r = pair - s * ranks.d;
        const size_t b0 = static_cast<size_t>(g - pair * per_chunk.d) * J;
        with_full((b0 + J) * kBlock <= m, [&](auto full) {
            const T *src = send + static_cast<size_t>(s) * sstride + static_cast<size_t>(r) * m +
                           b0 * kBlock + e0;
            T *dst = recv + static_cast<size_t>(r) * rstride + static_cast<size_t>(s) * m +
                     b0 * kBlock + e0;
            int valid[J];
#pragma unroll
            for (int j = 0; j < J; ++j)
                valid[j] = decltype(full)::value ? 4 : lane_valid((b0 + j) * kBlock, m);
            wire_blocks_raw<T, VEC, J>(src, valid, [&](int j, const float (&v)[4]) {
                store4<T, VEC>(dst + j * kBlock, valid[j], v);
            });
        });
    });
}

// ------------------------------------------------------------- dispatching

template <typename F>
cudaError_t dispatch(rlx_dtype dtype, bool vec, F &&f) {
    if (dtype == RLX_F32)
        return vec ? f.template operator()<float, true>() : f.template operator()<float, false>();
    return vec ? f.template operator()<uint16_t, true>() : f.template operator()<uint16_t, false>();
}

template <typename K, typename... Args>
cudaError_t launch(K kernel, size_t units, size_t units_per_cta, cudaStream_t stream,
                   Args... args) {
    const dim3 grid = grid_for(reinterpret_cast<const void *>(kernel), units, units_per_cta);
    if (grid.x == 0) return cudaErrorInvalidValue;
    return launch_kernel(kernel, grid, stream, args...);
}

constexpr size_t kWarps = kThreads / 32;

// units of kWarpVecs vectors, or of kJ / kJd blocks, in n elements
template <typename T> size_t copy_units(size_t n) {
    return ((n + kV<T> - 1) / kV<T> + kWarpVecs - 1) / kWarpVecs;
}
size_t block_units(size_t n, size_t per) { return ((n + kBlock - 1) / kBlock + per - 1) / per; }
bool fits32(size_t v) { return v < (size_t{1} << 32); }

}  // namespace

cudaError_t launch_copy(const void *src, void *dst, size_t n, rlx_dtype dtype, bool vec,
                        cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        return launch(copy_kernel<T, VEC>, copy_units<T>(n), kWarps * kPc, stream,
                      static_cast<const T *>(src), static_cast<T *>(dst), n);
    });
}

cudaError_t launch_tree_gather(void *recv, size_t count, size_t stride, int nranks,
                               size_t chunk, rlx_dtype dtype, rlx_wire wire,
                               const uint8_t *ws_codes, const float *ws_scales, bool vec,
                               cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        T *r = static_cast<T *>(recv);
        if (wire == RLX_WIRE_NATIVE) {
            const size_t per = tree_gather_native_per_chunk<T>(chunk);
            if (!fits32(per)) return cudaErrorInvalidValue;
            return launch(tree_gather_native_kernel<T, VEC>, per * static_cast<size_t>(nranks),
                          kWarps * kPc, stream, r, count, stride, nranks, chunk,
                          make_fastdiv(static_cast<uint32_t>(per)));
        }
        return launch(tree_gather_fp8_kernel<T, VEC>, tree_gather_fp8_units(count), kWarps * kPg,
                      stream, r, count, stride, nranks, ws_codes, ws_scales);
    });
}

cudaError_t launch_all_gather(const void *send, size_t send_stride, void *recv,
                              size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                              rlx_wire wire, bool vec, cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        const T *s = static_cast<const T *>(send);
        T *r = static_cast<T *>(recv);
        const size_t nn = static_cast<size_t>(nranks);
        const size_t per = wire == RLX_WIRE_NATIVE ? copy_units<T>(m) : block_units(m, kJag<T>);
        if (!fits32(per)) return cudaErrorInvalidValue;
        const FastDiv fd = make_fastdiv(static_cast<uint32_t>(per));
        if (wire == RLX_WIRE_NATIVE)
            return launch(ag_native_kernel<T, VEC>, per * nn, kWarps * kPc, stream, s,
                          send_stride, r, recv_stride, m, nranks, fd);
        return launch(ag_fp8_kernel<T, VEC>, per * nn, kWarps * kPg, stream, s, send_stride, r,
                      recv_stride, m, nranks, fd);
    });
}

cudaError_t launch_alltoall(const void *send, size_t send_stride, void *recv,
                            size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                            rlx_wire wire, bool vec, cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        const T *s = static_cast<const T *>(send);
        T *r = static_cast<T *>(recv);
        const size_t pairs = static_cast<size_t>(nranks) * static_cast<size_t>(nranks);
        const size_t per = wire == RLX_WIRE_NATIVE ? copy_units<T>(m) : block_units(m, kJa2a<T>);
        if (!fits32(per)) return cudaErrorInvalidValue;
        const FastDiv fd = make_fastdiv(static_cast<uint32_t>(per));
        const FastDiv fn = make_fastdiv(static_cast<uint32_t>(nranks));
        if (wire == RLX_WIRE_NATIVE)
            return launch(a2a_native_kernel<T, VEC>, per * pairs, kWarps * kPc, stream, s,
                          send_stride, r, recv_stride, m, nranks, fd, fn);
        return launch(a2a_fp8_kernel<T, VEC>, per * pairs, kWarps * kPg, stream, s, send_stride,
                      r, recv_stride, m, nranks, fd, fn);
    });
}

}  // namespace rlx
