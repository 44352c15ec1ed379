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
// conversion), so results are bit copies.  On the FP8 wire one warp handles
// one 128-element block (4 elements per lane): it reads the block once,
// applies dequantise(quantise(.)) in registers and writes every destination.
#include "rlx_device.cuh"
#include "rlx_internal.h"

namespace rlx {
namespace {

// Copy V = 16/sizeof(T) elements (valid of them) as raw bits.
template <typename T, bool VEC>
__device__ __forceinline__ void copyv_load(const T *p, int valid, uint4 &q, T (&e)[16 / sizeof(T)]) {
    constexpr int V = 16 / sizeof(T);
    if (VEC && valid == V) {
        q = __ldcs(reinterpret_cast<const uint4 *>(p));
    } else {
#pragma unroll
        for (int k = 0; k < V; ++k)
            if (k < valid) e[k] = p[k];
    }
}
template <typename T, bool VEC>
__device__ __forceinline__ void copyv_store(T *p, int valid, const uint4 &q, const T (&e)[16 / sizeof(T)]) {
    constexpr int V = 16 / sizeof(T);
    if (VEC && valid == V) {
        __stcs(reinterpret_cast<uint4 *>(p), q);
    } else {
#pragma unroll
        for (int k = 0; k < V; ++k)
            if (k < valid) p[k] = e[k];
    }
}

// ------------------------------------------------------------------ kernels

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
copy_kernel(const T *src, T *dst, size_t n) {
    constexpr int V = 16 / sizeof(T);
    const size_t nvec = (n + V - 1) / V;
    const size_t step = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t v = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec; v += step) {
        const size_t i0 = v * V;
        const int valid = n - i0 < static_cast<size_t>(V) ? static_cast<int>(n - i0) : V;
        uint4 q;
        T e[V];
        copyv_load<T, VEC>(src + i0, valid, q, e);
        copyv_store<T, VEC>(dst + i0, valid, q, e);
    }
}

// DDA-tree pass 2, native: chunk c of row c -> chunk c of every other row.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
tree_gather_native_kernel(T *recv, size_t count, size_t stride, int n, size_t chunk) {
    constexpr int V = 16 / sizeof(T);
    const size_t step = static_cast<size_t>(gridDim.x) * blockDim.x;
    const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (int c = 0; c < n; ++c) {
        const size_t lo = static_cast<size_t>(c) * chunk;
        if (lo >= count) break;
        const size_t hi = count - lo < chunk ? count : lo + chunk;
        const size_t nvec = (hi - lo + V - 1) / V;
        for (size_t v = tid; v < nvec; v += step) {
            const size_t i0 = lo + v * V;
            const int valid = hi - i0 < static_cast<size_t>(V) ? static_cast<int>(hi - i0) : V;
            uint4 q;
            T e[V];
            // the owner's chunk was just written by pass 1: default caching
            if (VEC && valid == V) q = *reinterpret_cast<const uint4 *>(recv + c * stride + i0);
            else copyv_load<T, false>(recv + c * stride + i0, valid, q, e);
            for (int r = 0; r < n; ++r)
                if (r != c) copyv_store<T, VEC>(recv + r * stride + i0, valid, q, e);
        }
    }
}

// DDA-tree pass 2, FP8: dequantise the payload block into every row.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
tree_gather_fp8_kernel(T *recv, size_t count, size_t stride, int n, const uint8_t *ws_codes,
                       const float *ws_scales) {
    const size_t nblk = (count + kBlock - 1) / kBlock;
    const int e0 = lane_id() * 4;
    for (size_t b = global_warp(); b < nblk; b += num_warps()) {
        const size_t base = b * kBlock;
        const int len = count - base < static_cast<size_t>(kBlock) ? static_cast<int>(count - base) : kBlock;
        const int valid = lane_valid(len);
        const uint32_t codes = *reinterpret_cast<const uint32_t *>(ws_codes + base + e0);
        const float s = ws_scales[b];
        float y[4];
        dequant4(codes, s, y);
        for (int r = 0; r < n; ++r) store4<T, VEC>(recv + r * stride + base + e0, valid, y);
    }
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
ag_native_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n) {
    constexpr int V = 16 / sizeof(T);
    const size_t step = static_cast<size_t>(gridDim.x) * blockDim.x;
    const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const size_t nvec = (m + V - 1) / V;
    for (int s = 0; s < n; ++s) {
        for (size_t v = tid; v < nvec; v += step) {
            const size_t j0 = v * V;
            const int valid = m - j0 < static_cast<size_t>(V) ? static_cast<int>(m - j0) : V;
            uint4 q;
            T e[V];
            copyv_load<T, VEC>(send + s * sstride + j0, valid, q, e);
            for (int r = 0; r < n; ++r) copyv_store<T, VEC>(recv + r * rstride + s * m + j0, valid, q, e);
        }
    }
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
ag_fp8_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n) {
    const size_t nbm = (m + kBlock - 1) / kBlock;
    const size_t jobs = nbm * static_cast<size_t>(n);
    const int e0 = lane_id() * 4;
    for (size_t job = global_warp(); job < jobs; job += num_warps()) {
        const size_t s = job / nbm;
        const size_t j0 = (job - s * nbm) * kBlock;
        const int len = m - j0 < static_cast<size_t>(kBlock) ? static_cast<int>(m - j0) : kBlock;
        const int valid = lane_valid(len);
        float v[4];
        load4<T, VEC>(send + s * sstride + j0 + e0, valid, v);
        wire_fp8_block(v);
        for (int r = 0; r < n; ++r) store4<T, VEC>(recv + r * rstride + s * m + j0 + e0, valid, v);
    }
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
a2a_native_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n) {
    constexpr int V = 16 / sizeof(T);
    const size_t step = static_cast<size_t>(gridDim.x) * blockDim.x;
    const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const size_t nvec = (m + V - 1) / V;
    for (int s = 0; s < n; ++s) {
        for (int r = 0; r < n; ++r) {
            const T *src = send + s * sstride + r * m;
            T *dst = recv + r * rstride + s * m;
            for (size_t v = tid; v < nvec; v += step) {
                const size_t j0 = v * V;
                const int valid = m - j0 < static_cast<size_t>(V) ? static_cast<int>(m - j0) : V;
                uint4 q;
                T e[V];
                copyv_load<T, VEC>(src + j0, valid, q, e);
                copyv_store<T, VEC>(dst + j0, valid, q, e);
            }
        }
    }
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
a2a_fp8_kernel(const T *send, size_t sstride, T *recv, size_t rstride, size_t m, int n) {
    const size_t nbm = (m + kBlock - 1) / kBlock;
    const size_t nn = static_cast<size_t>(n);
    const size_t jobs = nbm * nn * nn;
    const int e0 = lane_id() * 4;
    for (size_t job = global_warp(); job < jobs; job += num_warps()) {
        const size_t pair = job / nbm;          // pair = s * n + r
        const size_t j0 = (job - pair * nbm) * kBlock;
        const size_t s = pair / nn, r = pair - s * nn;
        const int len = m - j0 < static_cast<size_t>(kBlock) ? static_cast<int>(m - j0) : kBlock;
        const int valid = lane_valid(len);
        float v[4];
        load4<T, VEC>(send + s * sstride + r * m + j0 + e0, valid, v);
        wire_fp8_block(v);
        store4<T, VEC>(recv + r * rstride + s * m + j0 + e0, valid, v);
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
cudaError_t launch(K kernel, size_t jobs, size_t jobs_per_cta, cudaStream_t stream, Args... args) {
    const int grid = persistent_grid(reinterpret_cast<const void *>(kernel), jobs, jobs_per_cta);
    kernel<<<grid, kThreads, 0, stream>>>(args...);
    return cudaGetLastError();
}

constexpr size_t kWarps = kThreads / 32;

}  // namespace

cudaError_t launch_copy(const void *src, void *dst, size_t n, rlx_dtype dtype, bool vec,
                        cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        const size_t nvec = (n + 16 / sizeof(T) - 1) / (16 / sizeof(T));
        return launch(copy_kernel<T, VEC>, nvec, kThreads, stream, static_cast<const T *>(src),
                      static_cast<T *>(dst), n);
    });
}

cudaError_t launch_tree_gather(void *recv, size_t count, size_t stride, int nranks,
                               size_t chunk, rlx_dtype dtype, rlx_wire wire,
                               const uint8_t *ws_codes, const float *ws_scales, bool vec,
                               cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        T *r = static_cast<T *>(recv);
        if (wire == RLX_WIRE_NATIVE) {
            const size_t nvec = (chunk + 16 / sizeof(T) - 1) / (16 / sizeof(T));
            return launch(tree_gather_native_kernel<T, VEC>, nvec, kThreads, stream, r, count,
                          stride, nranks, chunk);
        }
        const size_t nblk = (count + kBlock - 1) / kBlock;
        return launch(tree_gather_fp8_kernel<T, VEC>, nblk, kWarps, stream, r, count, stride,
                      nranks, ws_codes, ws_scales);
    });
}

cudaError_t launch_all_gather(const void *send, size_t send_stride, void *recv,
                              size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                              rlx_wire wire, bool vec, cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        const T *s = static_cast<const T *>(send);
        T *r = static_cast<T *>(recv);
        if (wire == RLX_WIRE_NATIVE) {
            const size_t nvec = (m + 16 / sizeof(T) - 1) / (16 / sizeof(T));
            return launch(ag_native_kernel<T, VEC>, nvec, kThreads, stream, s, send_stride, r,
                          recv_stride, m, nranks);
        }
        const size_t jobs = (m + kBlock - 1) / kBlock * static_cast<size_t>(nranks);
        return launch(ag_fp8_kernel<T, VEC>, jobs, kWarps, stream, s, send_stride, r,
                      recv_stride, m, nranks);
    });
}

cudaError_t launch_alltoall(const void *send, size_t send_stride, void *recv,
                            size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                            rlx_wire wire, bool vec, cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        const T *s = static_cast<const T *>(send);
        T *r = static_cast<T *>(recv);
        if (wire == RLX_WIRE_NATIVE) {
            const size_t nvec = (m + 16 / sizeof(T) - 1) / (16 / sizeof(T));
            return launch(a2a_native_kernel<T, VEC>, nvec, kThreads, stream, s, send_stride, r,
                          recv_stride, m, nranks);
        }
        const size_t nn = static_cast<size_t>(nranks);
        const size_t jobs = (m + kBlock - 1) / kBlock * nn * nn;
        return launch(a2a_fp8_kernel<T, VEC>, jobs, kWarps, stream, s, send_stride, r,
                      recv_stride, m, nranks);
    });
}

}  // namespace rlx
