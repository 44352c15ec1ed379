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
// conversion), so results are bit copies; each thread keeps kUnroll vectors in
// flight.  On the FP8 wire a warp handles kJ consecutive 128-element blocks
// at once (4 elements per lane per block): it reads them, applies
// dequantise(quantise(.)) in registers and writes every destination.
// Chunked passes walk (chunk, unit) segment-major with a SegCursor, so all
// warps stay within about one chunk (few DRAM streams open at a time).
#include "rlx_device.cuh"
#include "rlx_internal.h"

namespace rlx {
namespace {

constexpr int kUnroll = 4;  // 16-byte vectors in flight per thread (native copies)
constexpr int kJ = 4;       // 128-blocks in flight per warp (FP8 single-source)
constexpr int kJd = 8;      // 128-blocks per warp when reading FP8 payloads

template <typename T> constexpr int kV = 16 / sizeof(T);

// One 16-byte vector (valid elements of it) as raw bits.
template <typename T, bool VEC>
struct RawVec {
    uint4 q;
    T e[kV<T>];
    __device__ __forceinline__ void load(const T *p, int valid) {
        if (VEC && valid == kV<T>) {
            q = __ldcs(reinterpret_cast<const uint4 *>(p));
        } else {
#pragma unroll
            for (int k = 0; k < kV<T>; ++k)
                if (k < valid) e[k] = p[k];
        }
    }
    // default caching, for data written by the previous pass
    __device__ __forceinline__ void load_cached(const T *p, int valid) {
        if (VEC && valid == kV<T>) {
            q = *reinterpret_cast<const uint4 *>(p);
        } else {
#pragma unroll
            for (int k = 0; k < kV<T>; ++k)
                if (k < valid) e[k] = p[k];
        }
    }
    __device__ __forceinline__ void store(T *p, int valid) const {
        if (VEC && valid == kV<T>) {
            __stcs(reinterpret_cast<uint4 *>(p), q);
        } else {
#pragma unroll
            for (int k = 0; k < kV<T>; ++k)
                if (k < valid) p[k] = e[k];
        }
    }
};

template <typename T>
__device__ __forceinline__ int vec_valid(size_t v, size_t nvec, size_t len) {
    if (v >= nvec) return 0;
    const size_t rem = len - v * kV<T>;
    return rem < static_cast<size_t>(kV<T>) ? static_cast<int>(rem) : kV<T>;
}

// ------------------------------------------------------------------ kernels

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
copy_kernel(const T *src, T *dst, size_t n) {
    const size_t nvec = (n + kV<T> - 1) / kV<T>;
    const size_t T_ = threads_in_grid_x();
    for (size_t v0 = thread_in_grid_x(); v0 < nvec; v0 += kUnroll * T_) {
        RawVec<T, VEC> a[kUnroll];
        int valid[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            valid[u] = vec_valid<T>(v0 + u * T_, nvec, n);
            if (valid[u]) a[u].load(src + (v0 + u * T_) * kV<T>, valid[u]);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            if (valid[u]) a[u].store(dst + (v0 + u * T_) * kV<T>, valid[u]);
    }
}

// DDA-tree pass 2, native: chunk c of row c -> chunk c of every other row.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
tree_gather_native_kernel(T *recv, size_t count, size_t stride, int n, size_t chunk) {
    const size_t per = (chunk + kV<T> - 1) / kV<T>;
    const size_t total = per * static_cast<size_t>(n);
    const size_t T_ = threads_in_grid_x();
    SegCursor cur(thread_in_grid_x(), T_, per);
    for (size_t g = thread_in_grid_x(); g < total; g += kUnroll * T_) {
        RawVec<T, VEC> a[kUnroll];
        int valid[kUnroll];
        size_t c[kUnroll], i0[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            c[u] = cur.seg;
            const size_t lo = cur.seg * chunk;
            i0[u] = lo + cur.off * kV<T>;
            valid[u] = 0;
            if (g + u * T_ < total && i0[u] < count) {
                const size_t hi = count - lo < chunk ? count : lo + chunk;
                valid[u] = hi - i0[u] < static_cast<size_t>(kV<T>) ? static_cast<int>(hi - i0[u]) : kV<T>;
                // the owner's chunk was just written by pass 1: default caching
                a[u].load_cached(recv + c[u] * stride + i0[u], valid[u]);
            }
            cur.next();
        }
        for (int r = 0; r < n; ++r) {
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                if (valid[u] && static_cast<size_t>(r) != c[u])
                    a[u].store(recv + r * stride + i0[u], valid[u]);
        }
    }
}

// DDA-tree pass 2, FP8: dequantise the payload blocks into every row.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
tree_gather_fp8_kernel(T *recv, size_t count, size_t stride, int n, const uint8_t *ws_codes,
                       const float *ws_scales) {
    const size_t nblk = (count + kBlock - 1) / kBlock;
    const int e0 = lane_id() * 4;
    for (size_t b0 = warp_in_grid_x() * kJd; b0 < nblk; b0 += warps_in_grid_x() * kJd) {
        float y[kJd][4];
        int valid[kJd];
#pragma unroll
        for (int j = 0; j < kJd; ++j) {
            const size_t b = b0 + j;
            valid[j] = lane_valid(b * kBlock, count);
            if (b < nblk) {
                const uint32_t codes = *reinterpret_cast<const uint32_t *>(ws_codes + b * kBlock + e0);
                dequant4(codes, ws_scales[b], y[j]);
            }
        }
        for (int r = 0; r < n; ++r)
#pragma unroll
            for (int j = 0; j < kJd; ++j)
                store4<T, VEC>(recv + r * stride + (b0 + j) * kBlock + e0, valid[j], y[j]);
    }
}

// AllGather, native: unit = (source rank s, vector of its row).
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
ag_native_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n) {
    const size_t per = (m + kV<T> - 1) / kV<T>;
    const size_t total = per * static_cast<size_t>(n);
    const size_t T_ = threads_in_grid_x();
    SegCursor cur(thread_in_grid_x(), T_, per);
    for (size_t g = thread_in_grid_x(); g < total; g += kUnroll * T_) {
        RawVec<T, VEC> a[kUnroll];
        int valid[kUnroll];
        size_t off[kUnroll];   // element offset within a destination row
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const size_t j0 = cur.off * kV<T>;
            off[u] = cur.seg * m + j0;
            valid[u] = g + u * T_ < total ? vec_valid<T>(cur.off, per, m) : 0;
            if (valid[u]) a[u].load(send + cur.seg * sstride + j0, valid[u]);
            cur.next();
        }
        for (int r = 0; r < n; ++r) {
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                if (valid[u]) a[u].store(recv + r * rstride + off[u], valid[u]);
        }
    }
}

// AllGather, FP8: unit = (source rank s, group of kJ blocks of its row);
// blocks anchored at the row start.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
ag_fp8_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n) {
    const size_t nbm = (m + kBlock - 1) / kBlock;
    const size_t per = (nbm + kJ - 1) / kJ;
    const size_t total = per * static_cast<size_t>(n);
    const int e0 = lane_id() * 4;
    SegCursor cur(warp_in_grid_x(), warps_in_grid_x(), per);
    for (size_t g = warp_in_grid_x(); g < total; g += warps_in_grid_x(), cur.next()) {
        const size_t s = cur.seg, b0 = cur.off * kJ;
        const T *src = send + s * sstride;
        float v[kJ][4];
        int valid[kJ];
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
            valid[j] = lane_valid((b0 + j) * kBlock, m);
            load4<T, VEC>(src + (b0 + j) * kBlock + e0, valid[j], v[j]);
        }
        wire_fp8_blocks<kJ>(v);
        for (int r = 0; r < n; ++r) {
            T *dst = recv + r * rstride + s * m;
#pragma unroll
            for (int j = 0; j < kJ; ++j) store4<T, VEC>(dst + (b0 + j) * kBlock + e0, valid[j], v[j]);
        }
    }
}

// AlltoAll, native: unit = (pair p = s*n + r, vector): chunk r of rank s goes
// to chunk s of rank r.  Pairs in s-major order read each source row front
// to back.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
a2a_native_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n) {
    const size_t per = (m + kV<T> - 1) / kV<T>;
    const size_t nn = static_cast<size_t>(n);
    const size_t total = per * nn * nn;
    const size_t T_ = threads_in_grid_x();
    SegCursor cur(thread_in_grid_x(), T_, per);
    for (size_t g = thread_in_grid_x(); g < total; g += kUnroll * T_) {
        RawVec<T, VEC> a[kUnroll];
        int valid[kUnroll];
        T *dst[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const size_t s = cur.seg / nn, r = cur.seg - s * nn, j0 = cur.off * kV<T>;
            valid[u] = g + u * T_ < total ? vec_valid<T>(cur.off, per, m) : 0;
            dst[u] = recv + r * rstride + s * m + j0;
            if (valid[u]) a[u].load(send + s * sstride + r * m + j0, valid[u]);
            cur.next();
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            if (valid[u]) a[u].store(dst[u], valid[u]);
    }
}

// AlltoAll, FP8: unit = (pair, group of kJ blocks); blocks anchored at the
// chunk start r*m.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
a2a_fp8_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n) {
    const size_t nbm = (m + kBlock - 1) / kBlock;
    const size_t per = (nbm + kJ - 1) / kJ;
    const size_t nn = static_cast<size_t>(n);
    const size_t total = per * nn * nn;
    const int e0 = lane_id() * 4;
    SegCursor cur(warp_in_grid_x(), warps_in_grid_x(), per);
    for (size_t g = warp_in_grid_x(); g < total; g += warps_in_grid_x(), cur.next()) {
        const size_t s = cur.seg / nn, r = cur.seg - s * nn, b0 = cur.off * kJ;
        const T *src = send + s * sstride + r * m;
        T *dst = recv + r * rstride + s * m;
        float v[kJ][4];
        int valid[kJ];
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
            valid[j] = lane_valid((b0 + j) * kBlock, m);
            load4<T, VEC>(src + (b0 + j) * kBlock + e0, valid[j], v[j]);
        }
        wire_fp8_blocks<kJ>(v);
#pragma unroll
        for (int j = 0; j < kJ; ++j) store4<T, VEC>(dst + (b0 + j) * kBlock + e0, valid[j], v[j]);
    }
}

// ------------------------------------------------------------- dispatching

template <typename F>
cudaError_t dispatch(rlx_dtype dtype, bool vec, F &&f) {
    if (dtype == RLX_F32)
        return vec ? f.template operator()<float, true>() : f.template operator()<float, false>();
    return vec ? f.template operator()<uint16_t, true>() : f.template operator()<uint16_t, false>();
}

template <typename K, typename... Args>
cudaError_t launch(K kernel, unsigned segments, size_t jobs_per_segment, size_t jobs_per_cta,
                   cudaStream_t stream, Args... args) {
    const dim3 grid = grid_2d(reinterpret_cast<const void *>(kernel), segments,
                              jobs_per_segment, jobs_per_cta);
    kernel<<<grid, kThreads, 0, stream>>>(args...);
    return cudaGetLastError();
}

constexpr size_t kWarps = kThreads / 32;

template <typename T> size_t nvec_of(size_t n) { return (n + kV<T> - 1) / kV<T>; }
size_t nblk_of(size_t n) { return (n + kBlock - 1) / kBlock; }

}  // namespace

cudaError_t launch_copy(const void *src, void *dst, size_t n, rlx_dtype dtype, bool vec,
                        cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        return launch(copy_kernel<T, VEC>, 1, nvec_of<T>(n), kThreads * kUnroll, stream,
                      static_cast<const T *>(src), static_cast<T *>(dst), n);
    });
}

cudaError_t launch_tree_gather(void *recv, size_t count, size_t stride, int nranks,
                               size_t chunk, rlx_dtype dtype, rlx_wire wire,
                               const uint8_t *ws_codes, const float *ws_scales, bool vec,
                               cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        T *r = static_cast<T *>(recv);
        if (wire == RLX_WIRE_NATIVE)
            return launch(tree_gather_native_kernel<T, VEC>, 1,
                          nvec_of<T>(chunk) * static_cast<size_t>(nranks), kThreads * kUnroll,
                          stream, r, count, stride, nranks, chunk);
        return launch(tree_gather_fp8_kernel<T, VEC>, 1, nblk_of(count), kWarps * kJd, stream, r,
                      count, stride, nranks, ws_codes, ws_scales);
    });
}

cudaError_t launch_all_gather(const void *send, size_t send_stride, void *recv,
                              size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                              rlx_wire wire, bool vec, cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        const T *s = static_cast<const T *>(send);
        T *r = static_cast<T *>(recv);
        const size_t nn = static_cast<size_t>(nranks);
        if (wire == RLX_WIRE_NATIVE)
            return launch(ag_native_kernel<T, VEC>, 1, nvec_of<T>(m) * nn, kThreads * kUnroll,
                          stream, s, send_stride, r, recv_stride, m, nranks);
        return launch(ag_fp8_kernel<T, VEC>, 1, nblk_of(m) * nn, kWarps * kJ, stream, s,
                      send_stride, r, recv_stride, m, nranks);
    });
}

cudaError_t launch_alltoall(const void *send, size_t send_stride, void *recv,
                            size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                            rlx_wire wire, bool vec, cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        const T *s = static_cast<const T *>(send);
        T *r = static_cast<T *>(recv);
        const size_t pairs = static_cast<size_t>(nranks) * static_cast<size_t>(nranks);
        if (wire == RLX_WIRE_NATIVE)
            return launch(a2a_native_kernel<T, VEC>, 1, nvec_of<T>(m) * pairs, kThreads * kUnroll,
                          stream, s, send_stride, r, recv_stride, m, nranks);
        return launch(a2a_fp8_kernel<T, VEC>, 1, nblk_of(m) * pairs, kWarps * kJ, stream, s,
                      send_stride, r, recv_stride, m, nranks);
    });
}

}  // namespace rlx
