// rlx_passes.cuh -- per-unit bodies of the streaming passes, shared by the
// kernels of rlx_reduce.cu and rlx_gather.cu: native 16-byte vector
// reductions and copies, the FP8-wire block reduction, and one unit of each
// DDA-tree pass.
#pragma once

#include "rlx_device.cuh"
#include "rlx_internal.h"

namespace rlx {

// ------------------------------------------------------ native 16-byte vectors

template <typename T> struct VecN { static constexpr int n = 16 / sizeof(T); };

template <typename T, bool VEC>
__device__ __forceinline__ void storev(T *p, int valid, const float (&v)[VecN<T>::n]) {
    constexpr int V = VecN<T>::n;
    if (VEC && valid == V) {
        uint4 q;
        if constexpr (sizeof(T) == 4) {
            q.x = __float_as_uint(v[0]); q.y = __float_as_uint(v[1]);
            q.z = __float_as_uint(v[2]); q.w = __float_as_uint(v[3]);
        } else {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                w[k] = static_cast<uint32_t>(f32_to_bf16_bits(v[2 * k])) |
                       (static_cast<uint32_t>(f32_to_bf16_bits(v[2 * k + 1])) << 16);
            q = make_uint4(w[0], w[1], w[2], w[3]);
        }
        st_stream(reinterpret_cast<uint4 *>(p), q);
    } else {
#pragma unroll
        for (int k = 0; k < V; ++k)
            if (k < valid) Elem<T>::store(p + k, v[k]);
    }
}

// One 16-byte vector kept as raw words (valid elements; the rest +0), so a
// bf16 vector costs 4 registers, not 8, while all ranks are in flight.
template <typename T, bool VEC>
__device__ __forceinline__ uint4 loadv_raw(const T *p, int valid) {
    constexpr int V = VecN<T>::n;
    if (VEC && valid == V) return ld_stream(reinterpret_cast<const uint4 *>(p));
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < V; ++k) {
        if (k < valid) {
            if constexpr (sizeof(T) == 4)
                w[k] = __float_as_uint(Elem<float>::load(reinterpret_cast<const float *>(p) + k));
            else
                w[k / 2] |= static_cast<uint32_t>(ld_stream(reinterpret_cast<const unsigned short *>(p) + k))
                            << (16 * (k % 2));
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Element k (compile-time) of a raw vector, widened to fp32 exactly.
template <typename T, int K>
__device__ __forceinline__ float raw_elem(const uint4 &q) {
    constexpr int word = sizeof(T) == 4 ? K : K / 2;
    const uint32_t w = word == 0 ? q.x : word == 1 ? q.y : word == 2 ? q.z : q.w;
    if constexpr (sizeof(T) == 4) return __uint_as_float(w);
    else return __uint_as_float(K % 2 == 0 ? w << 16 : w & 0xffff0000u);
}

template <typename T, int K = 0>
__device__ __forceinline__ void add_raw(float (&acc)[VecN<T>::n], const uint4 &q, bool first) {
    if constexpr (K < VecN<T>::n) {   // two elements per step (packed add)
        const float2 v = f2(raw_elem<T, K>(q), raw_elem<T, K + 1>(q));
        if (first) {
            acc[K] = v.x;
            acc[K + 1] = v.y;
        } else {
            const float2 s = add2_rn(f2(acc[K], acc[K + 1]), v);
            acc[K] = s.x;
            acc[K + 1] = s.y;
        }
        add_raw<T, K + 2>(acc, q, first);
    }
}

// acc = x_0 + x_1 + ... + x_{n-1} (rank order) of the vector at `src` in each
// of the n rows (row pitch `pitch` elements).  Full vectors issue all n loads
// before the first add; a partial (tail) vector is summed rank by rank, which
// needs few registers and keeps the kernel's register budget for the hot path.
template <typename T, int NR, bool VEC, typename Full>
__device__ __forceinline__ void reduce_vec(const T *src, size_t pitch, int n, int valid, Full,
                                           float (&acc)[VecN<T>::n]) {
    if constexpr (Full::value) {
        uint4 x[NR];
        const T *p = src;   // one running pointer: no per-rank address registers
#pragma unroll
        for (int s = 0; s < NR; ++s) {
            if (s < n) x[s] = loadv_raw<T, VEC>(p, valid);
            p += pitch;
        }
        add_raw<T>(acc, x[0], true);
#pragma unroll
        for (int s = 1; s < NR; ++s)
            if (s < n) add_raw<T>(acc, x[s], false);
    } else {
        add_raw<T>(acc, loadv_raw<T, false>(src, valid), true);
#pragma unroll 1
        for (int s = 1; s < n; ++s) add_raw<T>(acc, loadv_raw<T, false>(src + s * pitch, valid), false);
    }
}

// ---------------------------------------------------- FP8 wire, warp per block

// acc = SUM_s wire(x_s) over the 128-block at `src` in each of n rows, 4
// elements per lane (`valid` of them real; the rest +0).
template <typename T, int NR, bool VEC>
__device__ __forceinline__ void reduce_block_fp8(const T *src, size_t pitch, int n, int valid,
                                                 float (&acc)[4]) {
    float x[NR][4];
    const int e0 = lane_id() * 4;
#pragma unroll
    for (int s = 0; s < NR; ++s) {
        if (s < n) {
            load4<T, VEC>(src + s * pitch + e0, valid, x[s]);
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) x[s][k] = 0.0f;
        }
    }
    wire_fp8_blocks<NR>(x);
    float2 a01 = f2(x[0][0], x[0][1]), a23 = f2(x[0][2], x[0][3]);
#pragma unroll
    for (int s = 1; s < NR; ++s)
        if (s < n) {
            a01 = add2_rn(a01, f2(x[s][0], x[s][1]));
            a23 = add2_rn(a23, f2(x[s][2], x[s][3]));
        }
    acc[0] = a01.x; acc[1] = a01.y; acc[2] = a23.x; acc[3] = a23.y;
}

// Valid elements of a vector starting at element i0 of a segment ending at
// `hi` (V when the unit is full).
template <int V, typename Full>
__device__ __forceinline__ int vec_valid_in(size_t i0, size_t hi, Full) {
    if constexpr (Full::value) {
        return V;
    } else {
        if (i0 >= hi) return 0;
        return hi - i0 < static_cast<size_t>(V) ? static_cast<int>(hi - i0) : V;
    }
}

// ------------------------------------------------------ native copies

#ifndef RLX_UNROLL
#define RLX_UNROLL 4
#endif
#ifndef RLX_J
#define RLX_J 4
#endif
#ifndef RLX_JD
#define RLX_JD 8
#endif
constexpr int kUnroll = RLX_UNROLL;  // 16-byte vectors per lane in flight (native copies)
constexpr int kJ = RLX_J;            // 128-blocks in flight per warp (FP8 single-source)
constexpr int kJd = RLX_JD;          // 128-blocks per warp when reading FP8 payloads

template <typename T> constexpr int kV = 16 / sizeof(T);

// One element read through L2 only.
template <typename T>
__device__ __forceinline__ T load_l2(const T *p) {
    if constexpr (sizeof(T) == 4) {
        return __ldcg(p);
    } else {
        const unsigned short v = __ldcg(reinterpret_cast<const unsigned short *>(p));
        return static_cast<T>(v);
    }
}

// One 16-byte vector (valid elements of it) as raw bits.
template <typename T, bool VEC>
struct RawVec {
    uint4 q;
    T e[kV<T>];
    __device__ __forceinline__ void load(const T *p, int valid) {
        if (VEC && valid == kV<T>) {
            q = ld_stream(reinterpret_cast<const uint4 *>(p));
        } else {
#pragma unroll
            for (int k = 0; k < kV<T>; ++k)
                if (k < valid) e[k] = p[k];
        }
    }
    // for data the previous pass just wrote (possibly from another SM): read
    // through L2 only (ld.global.cg), never from a possibly stale L1 line
    __device__ __forceinline__ void load_through_l2(const T *p, int valid) {
        if (VEC && valid == kV<T>) {
            q = __ldcg(reinterpret_cast<const uint4 *>(p));
        } else {
#pragma unroll
            for (int k = 0; k < kV<T>; ++k)
                if (k < valid) e[k] = load_l2(p + k);
        }
    }
    __device__ __forceinline__ void store(T *p, int valid) const {
        if (VEC && valid == kV<T>) {
            st_stream(reinterpret_cast<uint4 *>(p), q);
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

// Vectors of one unit: unit u of a segment covers vectors
// [u*32*kUnroll, (u+1)*32*kUnroll); lane l takes u*32*kUnroll + k*32 + l, so
// each warp store continues the previous one.
constexpr int kWarpVecs = 32 * kUnroll;

// Loads the unit's vectors of a segment of `len` elements at `src` (Full:
// the unit lies wholly inside the segment, no bounds checks).
template <typename T, bool VEC, bool THROUGH_L2 = false, typename Full>
__device__ __forceinline__ void load_unit(const T *src, size_t unit, size_t len, Full,
                                          RawVec<T, VEC> (&a)[kUnroll], int (&valid)[kUnroll]) {
    const size_t nv = (len + kV<T> - 1) / kV<T>;
    const T *p = src + (unit * kWarpVecs + lane_id()) * kV<T>;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        if constexpr (Full::value) valid[u] = kV<T>;
        else valid[u] = vec_valid<T>(unit * kWarpVecs + u * 32 + lane_id(), nv, len);
        if (valid[u]) {
            if (THROUGH_L2) a[u].load_through_l2(p + u * 32 * kV<T>, valid[u]);
            else a[u].load(p + u * 32 * kV<T>, valid[u]);
        }
    }
}

template <typename T, bool VEC>
__device__ __forceinline__ void store_unit(T *dst, size_t unit, const RawVec<T, VEC> (&a)[kUnroll],
                                           const int (&valid)[kUnroll]) {
    T *p = dst + (unit * kWarpVecs + lane_id()) * kV<T>;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
        if (valid[u]) a[u].store(p + u * 32 * kV<T>, valid[u]);
}

// Is unit `unit` (of kWarpVecs vectors) wholly inside a segment of len elements?
template <typename T>
__device__ __forceinline__ bool unit_full(size_t unit, size_t len) {
    return (unit + 1) * kWarpVecs * kV<T> <= len;
}

// ------------------------------------------------------ DDA-tree pass units

// Pass 1, native: unit g = (chunk c, 32 vectors of it); chunk c -> row c.
template <typename T, int NR, bool VEC>
__device__ __forceinline__ void tree_reduce_native_unit(uint32_t g, const T *send, T *recv,
                                                        size_t count, size_t stride, int n,
                                                        size_t chunk, const FastDiv &per_chunk) {
    constexpr int V = VecN<T>::n;
    const uint32_t c = fast_div(g, per_chunk);
    const size_t lo = static_cast<size_t>(c) * chunk;
    if (lo >= count) return;
    const size_t hi = count - lo < chunk ? count : lo + chunk;
    const size_t u0 = lo + static_cast<size_t>(g - c * per_chunk.d) * 32 * V;
    const size_t i0 = u0 + static_cast<size_t>(lane_id()) * V;
    with_full(u0 + 32 * V <= hi, [&](auto full) {
        const int valid = vec_valid_in<V>(i0, hi, full);
        if (valid == 0) return;
        float acc[V];
        reduce_vec<T, NR, VEC>(send + i0, stride, n, valid, full, acc);
        storev<T, VEC>(recv + c * stride + i0, valid, acc);
    });
}

// Pass 1, FP8: unit b = 128-block b; reduce, then quantise the reduced block
// again into the payload (codes padded to whole blocks, one scale per block).
template <typename T, int NR, bool VEC>
__device__ __forceinline__ void tree_reduce_fp8_unit(uint32_t b, const T *send, size_t count,
                                                     size_t stride, int n, uint8_t *ws_codes,
                                                     float *ws_scales) {
    const int e0 = lane_id() * 4;
    const size_t base = static_cast<size_t>(b) * kBlock;
    with_full(base + kBlock <= count, [&](auto full) {
        const int valid = decltype(full)::value ? 4 : lane_valid(base, count);
        float acc[4];
        reduce_block_fp8<T, NR, VEC>(send + base, stride, n, valid, acc);
        const Scale sc = make_scale(warp_amax4(acc));
        const uint32_t codes = quant4(acc, sc);
        // default caching: pass 2 reads the payload back right away
        *reinterpret_cast<uint32_t *>(ws_codes + base + e0) = codes;
        if (lane_id() == 0) ws_scales[b] = sc.s;
    });
}

// Pass 2, native: unit g = (chunk c, kWarpVecs vectors of it); chunk c of
// row c -> chunk c of every other row.
template <typename T, bool VEC>
__device__ __forceinline__ void tree_gather_native_unit(uint32_t g, T *recv, size_t count,
                                                        size_t stride, int n, size_t chunk,
                                                        const FastDiv &per_chunk) {
    const uint32_t c = fast_div(g, per_chunk);
    const size_t lo = static_cast<size_t>(c) * chunk;
    if (lo >= count) return;
    const size_t len = count - lo < chunk ? count - lo : chunk;
    const size_t unit = g - c * per_chunk.d;
    with_full(unit_full<T>(unit, len), [&](auto full) {
        RawVec<T, VEC> a[kUnroll];
        int valid[kUnroll];
        // the owner's chunk was just written by pass 1: read it through L2
        load_unit<T, VEC, true>(recv + c * stride + lo, unit, len, full, a, valid);
        for (int r = 0; r < n; ++r)
            if (static_cast<uint32_t>(r) != c)
                store_unit<T, VEC>(recv + r * stride + lo, unit, a, valid);
    });
}

// Pass 2, FP8: unit g = kJd payload blocks, dequantised into every row.
template <typename T, bool VEC>
__device__ __forceinline__ void tree_gather_fp8_unit(uint32_t g, T *recv, size_t count,
                                                     size_t stride, int n,
                                                     const uint8_t *ws_codes,
                                                     const float *ws_scales) {
    const size_t nblk = (count + kBlock - 1) / kBlock;
    const int e0 = lane_id() * 4;
    const size_t b0 = static_cast<size_t>(g) * kJd;
    with_full((b0 + kJd) * kBlock <= count, [&](auto full) {
        constexpr bool F = decltype(full)::value;
        const uint8_t *cp = ws_codes + b0 * kBlock + e0;
        float y[kJd][4];
        int valid[kJd];
#pragma unroll
        for (int j = 0; j < kJd; ++j) {
            const size_t b = b0 + j;
            valid[j] = F ? 4 : lane_valid(b * kBlock, count);
            if (F || b < nblk) {   // payload written by pass 1: read through L2
                const uint32_t codes = __ldcg(reinterpret_cast<const unsigned int *>(cp + j * kBlock));
                dequant4(codes, __ldcg(ws_scales + b), y[j]);
            }
        }
        for (int r = 0; r < n; ++r) {
            T *dst = recv + r * stride + b0 * kBlock + e0;
#pragma unroll
            for (int j = 0; j < kJd; ++j) store4<T, VEC>(dst + j * kBlock, valid[j], y[j]);
        }
    });
}

// Unit counts of the two DDA-tree passes.
template <typename T> __host__ __device__ inline size_t tree_reduce_native_per_chunk(size_t chunk) {
    return ((chunk + VecN<T>::n - 1) / VecN<T>::n + 31) / 32;
}
template <typename T> __host__ __device__ inline size_t tree_gather_native_per_chunk(size_t chunk) {
    return ((chunk + kV<T> - 1) / kV<T> + kWarpVecs - 1) / kWarpVecs;
}
__host__ __device__ inline size_t tree_gather_fp8_units(size_t count) {
    return ((count + kBlock - 1) / kBlock + kJd - 1) / kJd;
}

}  // namespace rlx
