// rlx_device.cuh -- device-side building blocks shared by the rlx kernels.
//
// Element access (vectorised or element-wise), the FP8 E4M3 codec on the
// hardware cvt instructions, the warp-wide block amax, the block scale and the
// "wire" transform dequantise(quantise(x)) of 128-element blocks held as 4
// values per lane of a warp.  Every floating-point step is an explicit
// round-to-nearest intrinsic so that the compiler cannot contract a multiply
// and an add into an FMA that the definition does not have.
#pragma once

#include <cstddef>
#include <cstdint>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace rlx {

constexpr int kBlock = 128;        // elements per FP8 scale block
constexpr float kE4m3Max = 448.0f; // largest finite E4M3 magnitude
constexpr unsigned kFull = 0xffffffffu;
// Below this block scale the quotient x/s falls back to the IEEE division
// (see quotient_rn); at or above it every residual that can change a code is
// exact.  2^-90.
constexpr float kMinFastScale = 0x1p-90f;

// ------------------------------------------------------------ element types

// bf16 <-> fp32: widening is exact; narrowing is round-to-nearest-even.
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Cache policy of the streaming loads and stores (inputs are read once,
// outputs written once): RLX_LD_CS / RLX_ST_CS = 1 use the evict-first
// ".cs" forms, 0 the default write-back forms.
#ifndef RLX_LD_CS
#define RLX_LD_CS 1
#endif
#ifndef RLX_ST_CS
#define RLX_ST_CS 1
#endif

template <typename V>
__device__ __forceinline__ V ld_stream(const V *p) {
#if RLX_LD_CS
    return __ldcs(p);
#else
    return *p;
#endif
}
template <typename V>
__device__ __forceinline__ void st_stream(V *p, V v) {
#if RLX_ST_CS
    __stcs(p, v);
#else
    *p = v;
#endif
}

// Element traits: load/store one element as fp32.
template <typename T> struct Elem;
template <> struct Elem<float> {
    __device__ __forceinline__ static float load(const float *p) { return ld_stream(p); }
    __device__ __forceinline__ static void store(float *p, float v) { st_stream(p, v); }
};
template <> struct Elem<uint16_t> {  // bf16 bit patterns
    __device__ __forceinline__ static float load(const uint16_t *p) {
        return bf16_bits_to_f32(ld_stream(reinterpret_cast<const unsigned short *>(p)));
    }
    __device__ __forceinline__ static void store(uint16_t *p, float v) {
        st_stream(reinterpret_cast<unsigned short *>(p), f32_to_bf16_bits(v));
    }
};

// Four consecutive elements starting at p, `valid` of them real (0..4); the
// rest read as +0.  VEC: p is aligned to 4 elements (16 B fp32, 8 B bf16).
template <typename T, bool VEC>
__device__ __forceinline__ void load4(const T *p, int valid, float (&v)[4]) {
    if (VEC && valid == 4) {
        if constexpr (sizeof(T) == 4) {
            const float4 q = ld_stream(reinterpret_cast<const float4 *>(p));
            v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
        } else {
            const uint2 q = ld_stream(reinterpret_cast<const uint2 *>(p));
            v[0] = __uint_as_float(q.x << 16);
            v[1] = __uint_as_float(q.x & 0xffff0000u);
            v[2] = __uint_as_float(q.y << 16);
            v[3] = __uint_as_float(q.y & 0xffff0000u);
        }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = k < valid ? Elem<T>::load(p + k) : 0.0f;
    }
}

template <typename T, bool VEC>
__device__ __forceinline__ void store4(T *p, int valid, const float (&v)[4]) {
    if (VEC && valid == 4) {
        if constexpr (sizeof(T) == 4) {
            st_stream(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
        } else {
            uint2 q;
            q.x = static_cast<uint32_t>(f32_to_bf16_bits(v[0])) |
                  (static_cast<uint32_t>(f32_to_bf16_bits(v[1])) << 16);
            q.y = static_cast<uint32_t>(f32_to_bf16_bits(v[2])) |
                  (static_cast<uint32_t>(f32_to_bf16_bits(v[3])) << 16);
            st_stream(reinterpret_cast<uint2 *>(p), q);
        }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k < valid) Elem<T>::store(p + k, v[k]);
    }
}

// Four consecutive elements kept as loaded (fp32: 4 words, bf16: 2 words),
// widened to fp32 only where they are used; invalid elements hold +0.
template <typename T> struct Raw4;
template <> struct Raw4<float> { uint4 w; };
template <> struct Raw4<uint16_t> { uint2 w; };

template <typename T, bool VEC>
__device__ __forceinline__ Raw4<T> load_raw4(const T *p, int valid) {
    Raw4<T> r;
    if constexpr (sizeof(T) == 4) {
        if (VEC && valid == 4) {
            r.w = ld_stream(reinterpret_cast<const uint4 *>(p));
        } else {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) w[k] = k < valid ? __float_as_uint(Elem<T>::load(p + k)) : 0u;
            r.w = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else {
        if (VEC && valid == 4) {
            r.w = ld_stream(reinterpret_cast<const uint2 *>(p));
        } else {
            uint32_t w[2] = {0u, 0u};
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < valid)
                    w[k / 2] |= static_cast<uint32_t>(ld_stream(reinterpret_cast<const unsigned short *>(p) + k))
                                << (16 * (k % 2));
            r.w = make_uint2(w[0], w[1]);
        }
    }
    return r;
}

template <typename T> __device__ __forceinline__ Raw4<T> raw4_zero() {
    Raw4<T> r;
    if constexpr (sizeof(T) == 4) r.w = make_uint4(0u, 0u, 0u, 0u);
    else r.w = make_uint2(0u, 0u);
    return r;
}

__device__ __forceinline__ void widen4(const Raw4<float> &r, float (&v)[4]) {
    v[0] = __uint_as_float(r.w.x); v[1] = __uint_as_float(r.w.y);
    v[2] = __uint_as_float(r.w.z); v[3] = __uint_as_float(r.w.w);
}
__device__ __forceinline__ void widen4(const Raw4<uint16_t> &r, float (&v)[4]) {
    v[0] = __uint_as_float(r.w.x << 16); v[1] = __uint_as_float(r.w.x & 0xffff0000u);
    v[2] = __uint_as_float(r.w.y << 16); v[3] = __uint_as_float(r.w.y & 0xffff0000u);
}

// Bits of max |v| over the four elements (a non-negative float's bits; for
// those the integer order is the value order).  bf16 magnitudes are compared
// as 16-bit integers two at a time.
__device__ __forceinline__ uint32_t absmax4_bits(const Raw4<float> &r) {
    const float m = fmaxf(fmaxf(fabsf(__uint_as_float(r.w.x)), fabsf(__uint_as_float(r.w.y))),
                          fmaxf(fabsf(__uint_as_float(r.w.z)), fabsf(__uint_as_float(r.w.w))));
    return __float_as_uint(m);
}
__device__ __forceinline__ uint32_t absmax4_bits(const Raw4<uint16_t> &r) {
    const uint32_t m = __vmaxu2(r.w.x & 0x7fff7fffu, r.w.y & 0x7fff7fffu);
    return max(m & 0xffffu, m >> 16) << 16;
}

// --------------------------------------------------------------- E4M3 codec

// Two fp32 -> two E4M3 codes (round to nearest even, saturating to +-448,
// sign kept); `lo` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Four codes packed in a word (byte k = element k).
__device__ __forceinline__ uint32_t e4m3x4_from_f32(const float (&q)[4]) {
    return e4m3x2_from_f32(q[0], q[1]) | (e4m3x2_from_f32(q[2], q[3]) << 16);
}

// Two E4M3 codes (low byte = first) -> their exact values as fp32.
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t two_codes) {
    uint32_t h2;
    const uint16_t in = static_cast<uint16_t>(two_codes);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    __half2_raw raw;
    raw.x = static_cast<unsigned short>(h2 & 0xffffu);
    raw.y = static_cast<unsigned short>(h2 >> 16);
    return __half22float2(__half2(raw));  // every E4M3 value is exact in f16 and f32
}

// ------------------------------------------------------------ block scales

// max |v| over the 4 values of every lane of the warp (all 32 lanes call).
// For non-negative floats the IEEE bit order is the value order, so the warp
// reduction runs on the integer bits.
__device__ __forceinline__ float warp_amax4(const float (&v)[4]) {
    const float m = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    return __uint_as_float(__reduce_max_sync(kFull, __float_as_uint(m)));
}

// Scale of a block: s = fl32(amax / 448), and y = fl32(1 / s) when the fast
// quotient may be used (s >= 2^-90), else 0.
struct Scale {
    float s, y;
};
__device__ __forceinline__ Scale make_scale(float amax) {
    Scale r;
    r.s = __fdiv_rn(amax, kE4m3Max);
    r.y = r.s >= kMinFastScale ? __frcp_rn(r.s) : 0.0f;
    return r;
}

// Scales of K blocks held by the warp at once (K <= 32, a power of two).
// Lane l computes the division and the reciprocal for block l % K only; the
// results are then broadcast, so a lane pays for one division instead of K.
template <int K>
__device__ __forceinline__ void make_scales(const float (&amax)[K], Scale (&sc)[K]) {
    static_assert(K >= 1 && K <= 32 && (K & (K - 1)) == 0, "K must be a power of two <= 32");
    const int mine = threadIdx.x & (K - 1);
    float a = amax[0];
#pragma unroll
    for (int k = 1; k < K; ++k)
        if (mine == k) a = amax[k];
    const Scale m = make_scale(a);
#pragma unroll
    for (int k = 0; k < K; ++k) {
        sc[k].s = __shfl_sync(kFull, m.s, k);
        sc[k].y = __shfl_sync(kFull, m.y, k);
    }
}

// fl32(x / s), correctly rounded, from y = fl32(1/s) (s >= 2^-90).
// Markstein's division theorem (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): if y approximates 1/s with relative error below 2^-24 and q is a
// faithful approximation of x/s, then the residual s*q - x is exact and
// q - (s*q - x)*y rounded to nearest is the correctly rounded quotient.
// q0 = x*y can be up to 1.5 ulp away, so one correction first makes it
// faithful, the second rounds it correctly.  With s >= 2^-90 every residual
// that can affect an E4M3 code (|x/s| >= 2^-12) is exact; smaller quotients
// keep their sign and a magnitude far below 2^-10, so their code (+-0) is
// right.  The residual is taken as s*q - x (not x - s*q) so that x = -0
// yields -0: the sum of an exact zero product and -0 is then -0.
__device__ __forceinline__ float quotient_rn(float x, float s, float y) {
    float q = __fmul_rn(x, y);
    float r = __fmaf_rn(s, q, -x);
    q = __fmaf_rn(-r, y, q);
    r = __fmaf_rn(s, q, -x);
    return __fmaf_rn(-r, y, q);
}

// Blackwell executes two fp32 lanes per instruction (add/mul/fma .f32x2);
// each lane rounds exactly like the scalar instruction, so the packed forms
// below give the same bits with half the instructions.  A packed product is
// never the addend of a packed add here (such a pair gets fused, see
// dequant4).  RLX_PACKED_F32X2=0 selects the scalar forms.
#ifndef RLX_PACKED_F32X2
#define RLX_PACKED_F32X2 1
#endif

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// quotient_rn on two values sharing (s, y): the same steps, two lanes each.
__device__ __forceinline__ float2 quotient_rn2(float2 x, float s, float y) {
#if RLX_PACKED_F32X2
    const float2 s2 = f2(s, s), y2 = f2(y, y), ny2 = f2(-y, -y), nx = f2(-x.x, -x.y);
    float2 q = __fmul2_rn(x, y2);
    float2 r = __ffma2_rn(s2, q, nx);   // s*q - x
    q = __ffma2_rn(r, ny2, q);          // q - r*y
    r = __ffma2_rn(s2, q, nx);
    return __ffma2_rn(r, ny2, q);
#else
    return f2(quotient_rn(x.x, s, y), quotient_rn(x.y, s, y));
#endif
}

__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
#if RLX_PACKED_F32X2
    return __fadd2_rn(a, b);
#else
    return f2(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y));
#endif
}

// q = fl32(v/s) for 4 values of a block with scale sc; s == 0 gives signed
// zeros, sc.y == 0 selects the IEEE division.  Fast: sc.y != 0 is known.
template <bool Fast>
__device__ __forceinline__ void quotients4(const float (&v)[4], Scale sc, float (&q)[4]) {
    if (Fast || sc.y != 0.0f) {
        const float2 a = quotient_rn2(f2(v[0], v[1]), sc.s, sc.y);
        const float2 b = quotient_rn2(f2(v[2], v[3]), sc.s, sc.y);
        q[0] = a.x; q[1] = a.y; q[2] = b.x; q[3] = b.y;
    } else if (sc.s == 0.0f) {
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = __fmul_rn(v[k], 0.0f);  // +-0 with v's sign
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = __fdiv_rn(v[k], sc.s);
    }
}

// Quantise 4 values of a block with scale sc: code = e4m3_rne_sat(fl32(v/s)).
__device__ __forceinline__ uint32_t quant4(const float (&v)[4], Scale sc) {
    float q[4];
    quotients4<false>(v, sc, q);
    return e4m3x4_from_f32(q);
}

// Dequantise 4 packed codes with scale s: fl32(e4m3(code) * s).  The
// multiply is the scalar __fmul_rn, which is never merged into an FMA: a
// packed multiply whose product fed a packed add was contracted into a packed
// FMA by this toolchain (even as PTX mul.rn.f32x2 / add.rn.f32x2), which skips
// the rounding of the product that the definition requires.
__device__ __forceinline__ void dequant4(uint32_t codes, float s, float (&y)[4]) {
    const float2 a = e4m3x2_to_f32(codes & 0xffffu);
    const float2 b = e4m3x2_to_f32(codes >> 16);
    y[0] = __fmul_rn(a.x, s); y[1] = __fmul_rn(a.y, s);
    y[2] = __fmul_rn(b.x, s); y[3] = __fmul_rn(b.y, s);
}

// dequantise(quantise(v)) of 4 values of a block, in place: the same steps
// as dequant4(quant4(v, sc), sc.s, v), with each pair of codes going straight
// from one conversion to the other instead of through a packed word.
template <bool Fast>
__device__ __forceinline__ void wire4(float (&v)[4], Scale sc) {
    float q[4];
    quotients4<Fast>(v, sc, q);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        const float2 w = e4m3x2_to_f32(e4m3x2_from_f32(q[2 * p], q[2 * p + 1]));
        v[2 * p] = __fmul_rn(w.x, sc.s);
        v[2 * p + 1] = __fmul_rn(w.y, sc.s);
    }
}

// What a receiver holds after K 128-blocks crossed the FP8 wire.  The warp
// holds block k as 4 values per lane in v[k] (lanes past a block's end hold
// +0, which leaves its amax unchanged).  In place.
template <int K>
__device__ __forceinline__ void wire_fp8_blocks(float (&v)[K][4]) {
    float amax[K];
#pragma unroll
    for (int k = 0; k < K; ++k) amax[k] = warp_amax4(v[k]);
    Scale sc[K];
    make_scales<K>(amax, sc);
#pragma unroll
    for (int k = 0; k < K; ++k) wire4<false>(v[k], sc[k]);
}

// ----------------------------------------------------------- work layout

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// n / d for 32-bit n by a multiply and shifts (T. Granlund, P. Montgomery,
// "Division by invariant integers using multiplication", PLDI 1994, sec. 4):
// with l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1,
// q = (t + ((n - t) >> min(l,1))) >> max(l-1,0), t = mulhi(m, n).
struct FastDiv {
    uint32_t d, m, s1, s2;
};
inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t l = 0;
    while (l < 32 && (uint64_t{1} << l) < d) ++l;
    FastDiv f;
    f.d = d;
    f.m = static_cast<uint32_t>((((uint64_t{1} << l) - d) << 32) / d + 1);
    f.s1 = l < 1 ? l : 1;
    f.s2 = l > 0 ? l - 1 : 0;
    return f;
}
__host__ __device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv &f) {
#ifdef __CUDA_ARCH__
    const uint32_t t = __umulhi(f.m, n);
#else
    const uint32_t t = static_cast<uint32_t>((static_cast<uint64_t>(f.m) * n) >> 32);
#endif
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

// Units of work of the calling warp.  The grid covers units 0..total-1 in
// order: CTA b owns units [b*W*P, (b+1)*W*P) (W warps per CTA) and its warps
// take them round-robin, P per warp; a grid smaller than that loops.  CTAs
// are started in index order, so the CTAs resident at any moment work on one
// compact stretch of the data, which keeps few DRAM pages open.  f(g) is
// called with the same g by all 32 lanes.
// Programmatic dependent launch: the kernels are launched so that the next
// kernel on the stream may be scheduled while this one finishes its last
// wave.  Before its first memory access every kernel waits until the grids it
// depends on have completed and their writes are visible (griddepcontrol.wait
// returns at once when there is no such grid), and it lets its own dependents
// be scheduled as soon as all of its CTAs are running.
__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
}

template <int P, typename F>
__device__ __forceinline__ void for_each_unit(uint32_t total, F &&f) {
    constexpr uint32_t W = 256 / 32;   // rlx kernels run 256-thread CTAs
    pdl_begin();                       // every kernel's first memory access comes after this
    const uint32_t w = threadIdx.x >> 5;
    const size_t span = static_cast<size_t>(W) * P;
    for (size_t base = blockIdx.x * span; base < total; base += gridDim.x * span) {
#pragma unroll 1
        for (int p = 0; p < P; ++p) {
            const size_t g = base + static_cast<size_t>(p) * W + w;
            if (g < total) f(static_cast<uint32_t>(g));
        }
    }
}

// Calls f(std::true_type{}) when the unit lies wholly inside its segment
// (every lane owns a full vector of every block), else f(std::false_type{}).
// The two instantiations let the compiler drop all bounds checks, and fold
// the block offsets into the load and store instructions, on full units.
template <typename F>
__device__ __forceinline__ void with_full(bool full, F &&f) {
    if (full) f(std::true_type{});
    else f(std::false_type{});
}

// The number of ranks a reducing kernel sums, as the compile-time NR when the
// call uses every rank slot of the kernel (the usual case: N = 2, 4, 8, 16),
// which removes the per-rank guards, else as a run-time count.
struct RankCount {
    int v;
    __device__ __forceinline__ operator int() const { return v; }
};
template <int NR> struct FixedRanks {
    __device__ __forceinline__ constexpr operator int() const { return NR; }
};
// EXACT (n == NR) is chosen by the host, so each kernel instantiation holds
// one of the two forms and keeps its registers to itself.
template <int NR, bool EXACT, typename F>
__device__ __forceinline__ void with_rank_count(int n, F &&f) {
    if constexpr (EXACT) f(FixedRanks<NR>{});
    else f(RankCount{n});
}

// Calls f(std::true_type{}) when every block scale of the unit takes the fast
// quotient, else f(std::false_type{}).
template <typename F>
__device__ __forceinline__ void with_fast(bool fast, F &&f) {
    if (fast) f(std::true_type{});
    else f(std::false_type{});
}

// Elements of a 128-block that belong to this lane: 0..4.
__device__ __forceinline__ int lane_valid(size_t block_start, size_t len) {
    if (block_start >= len) return 0;
    const size_t rem = len - block_start;
    const int blen = rem < static_cast<size_t>(kBlock) ? static_cast<int>(rem) : kBlock;
    const int v = blen - lane_id() * 4;
    return v < 0 ? 0 : (v > 4 ? 4 : v);
}

}  // namespace rlx
