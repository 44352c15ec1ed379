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
            q = make_uint4(bf16x2_bits(v[0], v[1]), bf16x2_bits(v[2], v[3]),
                           bf16x2_bits(v[4], v[5]), bf16x2_bits(v[6], v[7]));
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
template <typename T, int NR, bool VEC, typename Full, typename N>
__device__ __forceinline__ void reduce_vec(const T *src, size_t pitch, N n, int valid, Full,
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

// 128-blocks a warp reduces at once on the FP8 wire: a bf16 block is half the
// bytes of an fp32 one, so a bf16 unit takes two adjacent blocks and a warp
// has as many bytes in flight per unit for either type.
#ifndef RLX_BPU_BF16
#define RLX_BPU_BF16 2
#endif
template <typename T> constexpr int kBpu = sizeof(T) == 2 ? RLX_BPU_BF16 : 1;
// 1: one warp vote per unit selects branch-free quantisation when every
// block scale takes the fast quotient; 0: every block branches on its scale.
#ifndef RLX_FAST_VOTE
#define RLX_FAST_VOTE 1
#endif

// acc[j] = SUM_s wire(x_s) over the BPU adjacent 128-blocks at src + 128 j in
// each of n rows, 4 elements per lane (valid[j] of them real; the rest +0).
// Every (rank, block) pair is one FP8 block: its amax is one warp max
// reduction of the lanes' amax keys, and lane l computes the scale of pair
// l % (NR*BPU); the keys and the scales pass through the warp's
// shared-memory slot (publish_scales), and each pair's scale is read from
// there just before the pair is quantised.  The loads stay raw until then,
// so a bf16 pair costs 2 registers.
template <typename T, int NR, bool VEC, int BPU, typename N>
__device__ __forceinline__ void reduce_blocks_fp8(const T *src, size_t pitch, N n,
                                                  const int (&valid)[BPU],
                                                  float (&acc)[BPU][4]) {
    constexpr int K = NR * BPU;
    static_assert(K <= 32 && (K & (K - 1)) == 0, "NR * BPU must be a power of two <= 32");
    const int e0 = lane_id() * 4;
    Raw4<T> x[NR][BPU];
#pragma unroll
    for (int s = 0; s < NR; ++s)
#pragma unroll
        for (int j = 0; j < BPU; ++j)
            x[s][j] = s < n ? load_raw4<T, VEC>(src + s * pitch + j * kBlock + e0, valid[j])
                            : raw4_zero<T>();
    // block (s, j) is pair s*BPU + j; its key goes to the slot as soon as the
    // reduction gives it (four at a time)
    begin_keys();
    if constexpr (K % 4 == 0) {
#pragma unroll
        for (int k = 0; k < K; k += 4) {
            uint32_t q[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                q[i] = __reduce_max_sync(kFull, amax_key(x[(k + i) / BPU][(k + i) % BPU]));
            put_keys(k, q[0], q[1], q[2], q[3]);
        }
    } else {
#pragma unroll
        for (int k = 0; k < K; ++k) put_key(k, __reduce_max_sync(kFull, amax_key(x[k / BPU][k % BPU])));
    }
    // when every scale of the unit takes the fast quotient (the usual case)
    // the quantisation below is straight-line code the compiler can
    // interleave across blocks
    const bool fast = publish_scales<T, K>();
    with_fast(RLX_FAST_VOTE && fast, [&](auto f) {
#pragma unroll
        for (int s = 0; s < NR; ++s) {
            if (s < n) {
#pragma unroll
                for (int j = 0; j < BPU; ++j) {
                    float v[4];
                    widen4(x[s][j], v);
                    wire4<decltype(f)::value>(v, scale_of(s * BPU + j));
                    if (s == 0) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) acc[j][k] = v[k];
                    } else {
                        const float2 lo = add2_rn(f2(acc[j][0], acc[j][1]), f2(v[0], v[1]));
                        const float2 hi = add2_rn(f2(acc[j][2], acc[j][3]), f2(v[2], v[3]));
                        acc[j][0] = lo.x; acc[j][1] = lo.y; acc[j][2] = hi.x; acc[j][3] = hi.y;
                    }
                }
            }
        }
    });
}

// ------------------------------------------------ FP8 wire, one sender's blocks

// What the receiver of one sender holds after J consecutive 128-blocks of it
// crossed the FP8 wire: the warp loads block j at src + 128 j (4 elements
// per lane, valid[j] of them real; the rest +0), finds each block's amax by
// one max reduction of the lanes' amax keys (passed to the warp's
// shared-memory slot four at a time), and then widens, quantises and
// dequantises one block at a time, handing it to emit(j, v) (which stores
// it).  The loads stay raw until their block is converted, so a bf16 block
// holds 2 registers until then instead of 4.
// The scales of the J blocks held raw in x, made known to the warp
// (publish_scales); true when every block takes the fast quotient.
template <typename T, int J>
__device__ __forceinline__ bool scales_of_raw_blocks(const Raw4<T> (&x)[J]) {
    static_assert(J >= 1 && J <= 32 && (J & (J - 1)) == 0, "J must be a power of two <= 32");
    begin_keys();
    if constexpr (J % 4 == 0) {
#pragma unroll
        for (int k = 0; k < J; k += 4) {
            uint32_t q[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) q[i] = __reduce_max_sync(kFull, amax_key(x[k + i]));
            put_keys(k, q[0], q[1], q[2], q[3]);
        }
    } else {
#pragma unroll
        for (int k = 0; k < J; ++k) put_key(k, __reduce_max_sync(kFull, amax_key(x[k])));
    }
    return publish_scales<T, J>();
}

template <typename T, bool VEC, int J, typename Emit>
__device__ __forceinline__ void wire_blocks_raw(const T *src, const int (&valid)[J], Emit &&emit) {
    Raw4<T> x[J];
#pragma unroll
    for (int j = 0; j < J; ++j) x[j] = load_raw4<T, VEC>(src + j * kBlock, valid[j]);
    with_fast(scales_of_raw_blocks<T, J>(x), [&](auto fast) {
#pragma unroll
        for (int j = 0; j < J; ++j) {
            float v[4];
            widen4(x[j], v);
            wire4<decltype(fast)::value>(v, scale_of(j));
            emit(j, v);
        }
    });
}

// The sender side alone: the codes of J consecutive blocks at src (as
// wire_blocks_raw, loads raw until their block is quantised), handed to
// emit(j, codes) as one word of 4 codes per lane; block j's scale is
// scale_of(j).s.x afterwards.
template <typename T, bool VEC, int J, typename Emit>
__device__ __forceinline__ void quant_blocks_raw(const T *src, const int (&valid)[J], Emit &&emit) {
    Raw4<T> x[J];
#pragma unroll
    for (int j = 0; j < J; ++j) x[j] = load_raw4<T, VEC>(src + j * kBlock, valid[j]);
    with_fast(scales_of_raw_blocks<T, J>(x), [&](auto fast) {
#pragma unroll
        for (int j = 0; j < J; ++j) {
            float v[4];
            widen4(x[j], v);
            emit(j, quant4<decltype(fast)::value>(v, scale_of(j)));
        }
    });
}

// ------------------------------------------------------ 16-byte bf16 stores

// Row pieces of 16 bytes for a bf16 block pair held as 4 values per lane per
// block: lane 2i gets elements [8i, 8i+8) of block 0 and lane 2i+1 the same
// elements of block 1 (one exchange with the neighbouring lane), so a warp
// writes the pair with one 16-byte store per lane instead of two of 8 bytes.
// The piece of lane l starts at element bf16_piece(l) of the pair.
__device__ __forceinline__ uint4 bf16_pair_pieces(const float (&v)[2][4]) {
    const uint2 w0 = make_uint2(bf16x2_bits(v[0][0], v[0][1]), bf16x2_bits(v[0][2], v[0][3]));
    const uint2 w1 = make_uint2(bf16x2_bits(v[1][0], v[1][1]), bf16x2_bits(v[1][2], v[1][3]));
    const bool odd = lane_id() & 1;
    const uint2 give = odd ? w0 : w1;
    const uint2 got = make_uint2(__shfl_xor_sync(kFull, give.x, 1), __shfl_xor_sync(kFull, give.y, 1));
    return odd ? make_uint4(got.x, got.y, w1.x, w1.y) : make_uint4(w0.x, w0.y, got.x, got.y);
}
__device__ __forceinline__ int bf16_piece(int lane) { return (lane & 1) * kBlock + (lane >> 1) * 8; }

// May the rows at p (pitch `pitch` elements of T) take 16-byte bf16 stores
// at block-pair offsets?
template <typename T>
__device__ __forceinline__ bool rows_16b(const T *p, size_t pitch) {
    return sizeof(T) == 2 && ((reinterpret_cast<uintptr_t>(p) | pitch * sizeof(T)) & 15) == 0;
}

// Stores the reduced blocks of a unit (acc[j] = block j, 4 values per lane) at
// dst + 128 j in each of `rows` rows `pitch` apart.  A full bf16 block pair
// on 16-byte aligned rows goes out as 16-byte pieces.
template <typename T, bool VEC, int BPU, typename Full, typename R>
__device__ __forceinline__ void store_blocks(T *dst, size_t pitch, R rows, Full, bool wide,
                                             const int (&valid)[BPU], const float (&acc)[BPU][4]) {
    if constexpr (BPU == 2 && sizeof(T) == 2 && Full::value) {
        if (VEC && wide) {
            const uint4 q = bf16_pair_pieces(acc);
            T *p = dst + bf16_piece(lane_id());
            for (int r = 0; r < rows; ++r) st_stream(reinterpret_cast<uint4 *>(p + r * pitch), q);
            return;
        }
    }
    const int e0 = lane_id() * 4;
    for (int r = 0; r < rows; ++r)
#pragma unroll
        for (int j = 0; j < BPU; ++j) store4<T, VEC>(dst + r * pitch + j * kBlock + e0, valid[j], acc[j]);
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
// 128-blocks per warp unit of the single-source FP8 kernels with bf16 data
// (alltoall, all-gather).  The alltoall keeps its loads raw until each block
// is converted (wire_blocks_raw), so 8 bf16 blocks fit the register budget of
// 4 CTAs per SM (62 registers) and halve the per-unit work (indices, the
// scales' division): 221.9 -> 173.6 us at the prefill size.  The all-gather
// stores every block to all N rows and stays at 4.
#ifndef RLX_J_A2A_BF16
#define RLX_J_A2A_BF16 8
#endif
#ifndef RLX_J_AG_BF16
#define RLX_J_AG_BF16 4
#endif
constexpr int kUnroll = RLX_UNROLL;  // 16-byte vectors per lane in flight (native copies)
constexpr int kJ = RLX_J;            // 128-blocks in flight per warp (FP8 single-source, fp32)
template <typename T> constexpr int kJa2a = sizeof(T) == 2 ? RLX_J_A2A_BF16 : RLX_J;
template <typename T> constexpr int kJag = sizeof(T) == 2 ? RLX_J_AG_BF16 : RLX_J;
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
template <typename T, int NR, bool VEC, typename N>
__device__ __forceinline__ void tree_reduce_native_unit(uint32_t g, const T *send, T *recv,
                                                        size_t count, size_t stride, N n,
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

// Pass 1, FP8: unit u = the BPU blocks from block u*BPU on; reduce, then
// quantise each reduced block again into the payload (codes padded to whole
// blocks, one scale per block).
template <typename T, int NR, bool VEC, typename N>
__device__ __forceinline__ void tree_reduce_fp8_unit(uint32_t u, const T *send, size_t count,
                                                     size_t stride, N n, uint8_t *ws_codes,
                                                     float *ws_scales) {
    constexpr int BPU = kBpu<T>;
    const int e0 = lane_id() * 4;
    const size_t base = static_cast<size_t>(u) * BPU * kBlock;
    with_full(base + BPU * kBlock <= count, [&](auto full) {
        int valid[BPU];
#pragma unroll
        for (int j = 0; j < BPU; ++j)
            valid[j] = decltype(full)::value ? 4 : lane_valid(base + j * kBlock, count);
        float acc[BPU][4];
        reduce_blocks_fp8<T, NR, VEC, BPU>(send + base, stride, n, valid, acc);
        Scale2 sc[BPU];
        if constexpr (BPU == 1) {
            sc[0] = pack(make_scale(warp_amax4(acc[0])));
        } else {
            uint32_t key[BPU];
#pragma unroll
            for (int j = 0; j < BPU; ++j) key[j] = __float_as_uint(warp_amax4(acc[j]));
            publish_scales<float, BPU>(key);
#pragma unroll
            for (int j = 0; j < BPU; ++j) sc[j] = scale_of(j);
        }
#pragma unroll
        for (int j = 0; j < BPU; ++j) {
            const size_t bj = base + j * kBlock;
            if (decltype(full)::value || bj < count) {
                const uint32_t codes = quant4(acc[j], sc[j]);
                // default caching: pass 2 reads the payload back right away
                *reinterpret_cast<uint32_t *>(ws_codes + bj + e0) = codes;
                if (lane_id() == 0) ws_scales[bj / kBlock] = sc[j].s.x;
            }
        }
    });
}

// Pass 2, native: unit g = (chunk c, kWarpVecs vectors of it); chunk c of
// row c -> chunk c of every other row.
// (Rows r0, r0 + rstep, ... only: a unit's rows can be split among warps.)
template <typename T, bool VEC>
__device__ __forceinline__ void tree_gather_native_unit(uint32_t g, T *recv, size_t count,
                                                        size_t stride, int n, size_t chunk,
                                                        const FastDiv &per_chunk, int r0 = 0,
                                                        int rstep = 1) {
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
        for (int r = r0; r < n; r += rstep)
            if (static_cast<uint32_t>(r) != c)
                store_unit<T, VEC>(recv + r * stride + lo, unit, a, valid);
    });
}

// Pass 2, FP8: unit g = kJd payload blocks, dequantised into every row
// (rows r0, r0 + rstep, ... only: a unit's rows can be split among warps).
template <typename T, bool VEC>
__device__ __forceinline__ void tree_gather_fp8_unit(uint32_t g, T *recv, size_t count,
                                                     size_t stride, int n,
                                                     const uint8_t *ws_codes,
                                                     const float *ws_scales, int r0 = 0,
                                                     int rstep = 1) {
    const size_t nblk = (count + kBlock - 1) / kBlock;
    const int e0 = lane_id() * 4;
    const size_t b0 = static_cast<size_t>(g) * kJd;
    if constexpr (sizeof(T) == 2 && VEC && kJd % 2 == 0) {
        // bf16 on 16-byte aligned rows, whole unit: lane l takes elements
        // [8l, 8l+8) of every block pair (half-warp l / 16 per block), so each
        // row gets one 16-byte store per lane per pair
        if ((b0 + kJd) * kBlock <= count && rows_16b(recv, stride)) {
            const int l = lane_id();
            uint4 q[kJd / 2];
#pragma unroll
            for (int p = 0; p < kJd / 2; ++p) {
                const size_t b = b0 + 2 * p + (l >> 4);
                const uint2 codes = __ldcg(reinterpret_cast<const uint2 *>(ws_codes + (b0 + 2 * p) * kBlock + 8 * l));
                const float s = __ldcg(ws_scales + b);
                float y[2][4];
                dequant4(codes.x, s, y[0]);
                dequant4(codes.y, s, y[1]);
                q[p] = make_uint4(bf16x2_bits(y[0][0], y[0][1]), bf16x2_bits(y[0][2], y[0][3]),
                                  bf16x2_bits(y[1][0], y[1][1]), bf16x2_bits(y[1][2], y[1][3]));
            }
            for (int r = r0; r < n; r += rstep) {
                T *dst = recv + r * stride + b0 * kBlock + 8 * l;
#pragma unroll
                for (int p = 0; p < kJd / 2; ++p)
                    st_stream(reinterpret_cast<uint4 *>(dst + 2 * p * kBlock), q[p]);
            }
            return;
        }
    }
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
        for (int r = r0; r < n; r += rstep) {
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
