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
// Two fp32 -> two bf16 (each round-to-nearest-even) in one word, `lo` in the
// low half: one packed conversion instead of two single ones.
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
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
            st_stream(reinterpret_cast<uint2 *>(p), make_uint2(bf16x2_bits(v[0], v[1]),
                                                               bf16x2_bits(v[2], v[3])));
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

// Amax keys: an unsigned word per lane whose integer order is the order of
// max |v| over the lane's four elements, so that one warp max-reduction of the
// keys finds a block's amax, and amax_of<T>(key) turns the winning key into
// the amax.  fp32: the bits of max |v| (for non-negative floats the bit order
// is the value order).  bf16: both 16-bit halves hold the bf16 bits of
// max |v| (magnitudes compared as 16-bit integers two at a time), so the
// 32-bit maximum over lanes is the maximum of the halves and the amax is the
// high half widened exactly.
__device__ __forceinline__ uint32_t amax_key(const Raw4<float> &r) {
    const float m = fmaxf(fmaxf(fabsf(__uint_as_float(r.w.x)), fabsf(__uint_as_float(r.w.y))),
                          fmaxf(fabsf(__uint_as_float(r.w.z)), fabsf(__uint_as_float(r.w.w))));
    return __float_as_uint(m);
}
// 1: a bf16 block's per-lane amax in bf16x2 max arithmetic (measured: one
// ALU instruction less per 4 elements); 0: as 16-bit integers.
#ifndef RLX_AMAX_BF16X2
#define RLX_AMAX_BF16X2 1
#endif
__device__ __forceinline__ uint32_t amax_key(const Raw4<uint16_t> &r) {
#if RLX_AMAX_BF16X2
    // max(|a|, |b|) per half in bf16 arithmetic (sign = xor of the signs,
    // cleared below); max is exact and keeps subnormals
    uint32_t m;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(r.w.x), "r"(r.w.y));
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(m), "r"(__byte_perm(m, 0u, 0x1032)));
    return m & 0x7fff7fffu;
#else
    const uint32_t m = __vmaxu2(r.w.x & 0x7fff7fffu, r.w.y & 0x7fff7fffu);
    return __vmaxu2(m, __byte_perm(m, 0u, 0x1032));   // the larger half in both halves
#endif
}
template <typename T> __device__ __forceinline__ float amax_of(uint32_t key) {
    if constexpr (sizeof(T) == 4) return __uint_as_float(key);
    else return __uint_as_float(key & 0xffff0000u);
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

// How the quotient x / s of the quantiser is formed.  The product is built
// with RLX_QUOTIENT=0: the correctly rounded quotient fl32(x / s), which the
// definition of the codes requires.  The other two exist only for the
// ablation that measures what exactness costs (a profiling build under
// _build/, never the library the package loads):
//   1  x * fl32(448 / amax), one multiply per element (the reciprocal form a
//      faster quantiser would use; it changes some codes);
//   2  __fdiv_rn(x, s) for every element (CUDA's IEEE division);
//   3  the codes of the correctly rounded quotient from two bracketing
//      products (see neg_codes4), with the full quotient only for blocks
//      where the bracket is not decisive.  Gives the same codes as 0.
#ifndef RLX_QUOTIENT
#define RLX_QUOTIENT 0
#endif
constexpr int kQuotient = RLX_QUOTIENT;
static_assert(kQuotient >= 0 && kQuotient <= 3, "RLX_QUOTIENT must be 0, 1, 2 or 3");
constexpr bool kBracket = kQuotient == 3;

// Scale of a block: s = fl32(amax / 448), and ny = -fl32(1 / s) when the fast
// quotient may be used (s >= 2^-90), else 0.  (RLX_QUOTIENT=1: ny =
// -fl32(448 / amax); RLX_QUOTIENT=2: ny = 0, every element takes the IEEE
// division.)  The reciprocal is kept negated because the quantiser works on
// the negated quotient (see neg_quotient2).
// 1: the quotient starts from a two-term reciprocal (see neg_quotient2),
// which saves one of its five packed steps; 0: the plain reciprocal and two
// corrections.  Both give the correctly rounded quotient (the quotient test
// checks both); the two-term form measured slower (bf16 tree pass 1 at a
// quarter of the prefill size: 43.3 against 39.8 us -- the second scale
// load and the extra registers cost more than the step saves), so it is off.
#ifndef RLX_QUOTIENT_2TERM
#define RLX_QUOTIENT_2TERM 0
#endif
constexpr bool k2Term = RLX_QUOTIENT_2TERM && kQuotient == 0;

// With the two-term reciprocal the scale also carries nlo = -y_lo, where
// y_hi = RD(1/s) and y_lo = RN((1 - s*y_hi) * y) >= +0 (so nlo <= -0).
// With RLX_QUOTIENT=3 (nhi, nlo) = (fl32(ny * (1 + 2^-21)),
// fl32(ny * (1 - 2^-21))), the two bracketing multipliers.
struct Scale {
    float s, ny, nhi, nlo;
};
// The reciprocal terms of a scale s for the correctly rounded quotient.
__device__ __forceinline__ Scale reciprocal_terms(float s) {
    Scale r;
    r.s = s;
    r.nhi = r.nlo = 0.0f;
    r.ny = s >= kMinFastScale ? -__frcp_rn(s) : 0.0f;
    if constexpr (k2Term) {
        if (r.ny != 0.0f) {
            const float hi = __frcp_rd(s);
            // 1 - s*hi is exact (hi is a faithful reciprocal) and >= 0
            const float e = __fmaf_rn(-s, hi, 1.0f);
            r.nhi = -hi;
            r.nlo = -__fmul_rn(e, -r.ny);
        }
    }
    return r;
}

__device__ __forceinline__ Scale make_scale(float amax) {
    Scale r;
    r.s = __fdiv_rn(amax, kE4m3Max);
    r.nhi = r.nlo = 0.0f;
    if constexpr (kQuotient == 0) {
        r = reciprocal_terms(r.s);
    } else if constexpr (kBracket) {
        r = reciprocal_terms(r.s);
        r.nhi = __fmul_rn(r.ny, 1.0f + 0x1p-21f);
        r.nlo = __fmul_rn(r.ny, 1.0f - 0x1p-21f);
    } else if constexpr (kQuotient == 1) {
        r.ny = r.s >= kMinFastScale ? -__fdiv_rn(kE4m3Max, amax) : 0.0f;
    } else {
        r.ny = 0.0f;
    }
    return r;
}

// A block scale as the packed two-lane instructions take it: (s, s),
// (ny, ny) (and (nhi, nhi), (nlo, nlo)) in adjacent registers.
struct Scale2 {
    float2 s, ny, nhi, nlo;
};
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ Scale2 pack(Scale sc) {
    return {f2(sc.s, sc.s), f2(sc.ny, sc.ny), f2(sc.nhi, sc.nhi), f2(sc.nlo, sc.nlo)};
}

// Per-warp shared memory through which the lanes of a warp exchange block
// amaxes and scales (a slot per warp of the 256-thread CTA).
constexpr int kWarpsPerCta = 8;
struct alignas(16) WarpScratch {
    float4 scale[32];   // block k: (s, s, ny, ny)
    float4 split[k2Term || kBracket ? 32 : 1];   // block k: (nhi, nhi, nlo, nlo)
    uint32_t key[32];   // block k: its amax key
};
__device__ __forceinline__ WarpScratch &warp_scratch() {
    __shared__ WarpScratch slot[kWarpsPerCta];
    return slot[threadIdx.x >> 5];
}

// Block scales shared by a warp, in three steps for the K blocks of a unit
// (K <= 32, a power of two):
//   begin_keys()          before the first key of the unit is stored (the
//                         previous unit's readers are done with the slot);
//   put_keys(i, ...)      the warp-uniform amax keys (amax_key, after the max
//                         reduction) of blocks i.. go into the slot, as soon
//                         as they are known, so few are held in registers;
//   publish_scales<T,K>() lane l computes the division and the reciprocal
//                         for block l % K only, so a lane pays for one
//                         division instead of K, and writes the scale to the
//                         slot, where scale_of(k) reads it.  Returns true
//                         when every block takes the fast quotient.
__device__ __forceinline__ void begin_keys() { __syncwarp(); }
__device__ __forceinline__ void put_keys(int i, uint32_t k0, uint32_t k1, uint32_t k2,
                                         uint32_t k3) {
    if ((threadIdx.x & 31) == 0)
        *reinterpret_cast<uint4 *>(&warp_scratch().key[i]) = make_uint4(k0, k1, k2, k3);
}
__device__ __forceinline__ void put_key(int i, uint32_t k) {
    if ((threadIdx.x & 31) == 0) warp_scratch().key[i] = k;
}
template <typename T, int K>
__device__ __forceinline__ bool publish_scales() {
    static_assert(K >= 1 && K <= 32 && (K & (K - 1)) == 0, "K must be a power of two <= 32");
    WarpScratch &w = warp_scratch();
    const int lane = threadIdx.x & 31;
    __syncwarp();
    const Scale own = make_scale(amax_of<T>(w.key[lane & (K - 1)]));
    if (lane < K) {
        w.scale[lane] = make_float4(own.s, own.s, own.ny, own.ny);
        if constexpr (k2Term || kBracket)
            w.split[lane] = make_float4(own.nhi, own.nhi, own.nlo, own.nlo);
    }
    const bool fast = __all_sync(kFull, own.ny != 0.0f);
    __syncwarp();
    return fast;
}
// All three steps for keys already held in registers.
template <typename T, int K>
__device__ __forceinline__ bool publish_scales(const uint32_t (&key)[K]) {
    begin_keys();
    if constexpr (K % 4 == 0) {
#pragma unroll
        for (int k = 0; k < K; k += 4) put_keys(k, key[k], key[k + 1], key[k + 2], key[k + 3]);
    } else {
#pragma unroll
        for (int k = 0; k < K; ++k) put_key(k, key[k]);
    }
    return publish_scales<T, K>();
}
__device__ __forceinline__ Scale2 scale_of(int k) {
    const float4 v = warp_scratch().scale[k];
    if constexpr (k2Term || kBracket) {
        const float4 u = warp_scratch().split[k];
        return {f2(v.x, v.y), f2(v.z, v.w), f2(u.x, u.y), f2(u.z, u.w)};
    }
    return {f2(v.x, v.y), f2(v.z, v.w), f2(0.0f, 0.0f), f2(0.0f, 0.0f)};
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

// -fl32(x / s) for two values sharing a scale, exactly: quotient_rn carried
// out on p = -q.  With ny = -y every step is the negation of quotient_rn's
// (round to nearest is symmetric): p0 = x*ny = -q0; the residual
// r' = s*p0 + x is -(s*q0 - x); and p1 = p0 + r'*ny is
// -(q0 - (s*q0 - x)*y) = -q1.  Where quotient_rn's residual cancels exactly
// to +0 this one does too, which leaves p = -q intact since q != 0 there;
// x = +-0 gives p = -+0.  No operand needs a per-element negation.
// (RLX_QUOTIENT=1: p = x * ny.)
// Two-term form (RLX_QUOTIENT_2TERM): y_hi = RD(1/s) and y_lo =
// RN((1 - s*y_hi) * y) approximate 1/s to about 2^-47, so
// q0 = RN(x*y_hi + RN(x*y_lo)) is already faithful and one Markstein step
// rounds it correctly: four packed steps instead of five.  Negated as
// above; since -y_lo is never +0, x*(-y_lo) has the sign of -x when x is a
// zero, and p0 = -+0 for x = +-0 as required.
__device__ __forceinline__ float2 neg_quotient2(float2 x, const Scale2 &sc) {
#if RLX_PACKED_F32X2
    if constexpr (k2Term) {
        const float2 t = __fmul2_rn(x, sc.nlo);
        float2 p = __ffma2_rn(x, sc.nhi, t);    // -RN(x*y_hi + x*y_lo), faithful
        const float2 r = __ffma2_rn(sc.s, p, x);
        return __ffma2_rn(r, sc.ny, p);
    }
    float2 p = __fmul2_rn(x, sc.ny);
    if constexpr (kQuotient == 1) return p;
    float2 r = __ffma2_rn(sc.s, p, x);   // s*p + x = -(s*q - x)
    p = __ffma2_rn(r, sc.ny, p);         // p - r*y
    r = __ffma2_rn(sc.s, p, x);
    return __ffma2_rn(r, sc.ny, p);
#else
    if constexpr (kQuotient == 1) return f2(__fmul_rn(x.x, sc.ny.x), __fmul_rn(x.y, sc.ny.x));
    return f2(-quotient_rn(x.x, sc.s.x, -sc.ny.x), -quotient_rn(x.y, sc.s.x, -sc.ny.x));
#endif
}

__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
#if RLX_PACKED_F32X2
    return __fadd2_rn(a, b);
#else
    return f2(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y));
#endif
}

// p = -fl32(v/s) for 4 values of a block with scale sc, exactly (signed
// zeros included): s == 0 gives -(+-0), ny == 0 the IEEE division by -s.
// Fast: ny != 0 is known.
template <bool Fast>
__device__ __forceinline__ void neg_quotients4(const float (&v)[4], const Scale2 &sc,
                                               float (&p)[4]) {
    if ((Fast && kQuotient != 2) || sc.ny.x != 0.0f) {
        const float2 a = neg_quotient2(f2(v[0], v[1]), sc);
        const float2 b = neg_quotient2(f2(v[2], v[3]), sc);
        p[0] = a.x; p[1] = a.y; p[2] = b.x; p[3] = b.y;
    } else if (sc.s.x == 0.0f) {
#pragma unroll
        for (int k = 0; k < 4; ++k) p[k] = __fmul_rn(v[k], -0.0f);  // zero, sign opposite to v's
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) p[k] = __fdiv_rn(v[k], -sc.s.x);
    }
}

// The codes of -fl32(v/s) for 4 values of a block (byte k = element k).
// RLX_QUOTIENT=3: E, the E4M3 encoding (round to nearest even, saturating),
// is monotone, so if the codes of two values a and b agree, every value
// between them has that code too.  With y = fl32(1/s) (relative error
// <= 2^-24), the products a = fl32(v * fl32(-y * (1 + 2^-21))) and
// b = fl32(v * fl32(-y * (1 - 2^-21))) lie, for every quotient in the fp32
// normal range, at least 2^-21 - 4 * 2^-24 > 2^-24 (relative) beyond -v/s
// on either side, while -fl32(v/s) lies within 2^-24 of it: the correctly
// rounded quotient is bracketed.  (Quotients below the normal range have
// code +-0, as do both products; v = +-0 gives -+0 everywhere.)  So where
// E(a) == E(b) in every lane, E(a) is the code of the correctly rounded
// quotient; a block where some lane's bracket straddles a rounding boundary
// takes the full quotient.  Every lane of the warp calls this.
template <bool Fast>
__device__ __forceinline__ uint32_t neg_codes4(const float (&v)[4], const Scale2 &sc) {
    if constexpr (kBracket) {
        if (Fast || sc.ny.x != 0.0f) {
            const float2 x0 = f2(v[0], v[1]), x1 = f2(v[2], v[3]);
            const float2 a0 = __fmul2_rn(x0, sc.nhi), a1 = __fmul2_rn(x1, sc.nhi);
            const float2 b0 = __fmul2_rn(x0, sc.nlo), b1 = __fmul2_rn(x1, sc.nlo);
            const uint32_t ca = e4m3x2_from_f32(a0.x, a0.y) | (e4m3x2_from_f32(a1.x, a1.y) << 16);
            const uint32_t cb = e4m3x2_from_f32(b0.x, b0.y) | (e4m3x2_from_f32(b1.x, b1.y) << 16);
            if (__all_sync(kFull, ca == cb)) return ca;
        }
    }
    float p[4];
    neg_quotients4<Fast>(v, sc, p);
    return e4m3x4_from_f32(p);
}

// Quantise 4 values of a block with scale sc: code = e4m3_rne_sat(fl32(v/s)).
// The E4M3 encoding is symmetric in the sign (round to nearest even, the
// saturation bound and zero included), so the codes of -q are the codes of q
// with the sign bit of every byte flipped back.
template <bool Fast = false>
__device__ __forceinline__ uint32_t quant4(const float (&v)[4], const Scale2 &sc) {
    return neg_codes4<Fast>(v, sc) ^ 0x80808080u;
}

// Dequantise 4 packed codes with scale s: fl32(e4m3(code) * s).  The
// multiply is the scalar __fmul_rn, which is never merged into an FMA: a
// packed multiply whose product fed a packed add was contracted into a packed
// FMA by this toolchain (even as PTX mul.rn.f32x2 / add.rn.f32x2), which skips
// the rounding of the product that the definition requires.
__device__ __forceinline__ void dequant4(uint32_t codes, float s, float (&y)[4]) {
    const float2 a = e4m3x2_to_f32(codes & 0xffffu);
    const float2 b = e4m3x2_to_f32(codes >> 16);
#if RLX_PACKED_F32X2
    // the products are stored, never added, so the packed multiply is safe here
    const float2 pa = __fmul2_rn(a, f2(s, s)), pb = __fmul2_rn(b, f2(s, s));
    y[0] = pa.x; y[1] = pa.y; y[2] = pb.x; y[3] = pb.y;
#else
    y[0] = __fmul_rn(a.x, s); y[1] = __fmul_rn(a.y, s);
    y[2] = __fmul_rn(b.x, s); y[3] = __fmul_rn(b.y, s);
#endif
}

// dequantise(quantise(v)) of 4 values of a block, in place.  The codes of
// the negated quotient are the codes of -q, whose values are exactly -w, so
// fl32((-w) * (-s)) = fl32(w * s) is the dequantised value (the sign of a
// zero included); each pair of codes goes straight from one conversion to
// the other.
// 1: the dequantising product of the wire is one packed FMA with a -0 addend
// per pair: fl32(w*s + -0) = fl32(w*s) for every w*s (zeros included), and
// the addend, formed at run time as (-s)*0, is not a constant the compiler
// could drop to contract the product into the add that follows.  0: scalar
// multiplies (never contracted).
#ifndef RLX_DEQ_FFMA2
#define RLX_DEQ_FFMA2 0
#endif
template <bool Fast>
__device__ __forceinline__ void wire4(float (&v)[4], const Scale2 &sc) {
    const float ns = -sc.s.x;
    if constexpr (kBracket) {
        const uint32_t c = neg_codes4<Fast>(v, sc);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const float2 w = e4m3x2_to_f32(k == 0 ? c & 0xffffu : c >> 16);
            v[2 * k] = __fmul_rn(w.x, ns);
            v[2 * k + 1] = __fmul_rn(w.y, ns);
        }
        return;
    }
    float p[4];
    neg_quotients4<Fast>(v, sc, p);
#if RLX_DEQ_FFMA2 && RLX_PACKED_F32X2
    const float nz = __fmul_rn(ns, 0.0f);   // -0: s >= 0
    const float2 ns2 = f2(ns, ns), nz2 = f2(nz, nz);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float2 w = e4m3x2_to_f32(e4m3x2_from_f32(p[2 * k], p[2 * k + 1]));
        const float2 y = __ffma2_rn(w, ns2, nz2);
        v[2 * k] = y.x;
        v[2 * k + 1] = y.y;
    }
#else
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float2 w = e4m3x2_to_f32(e4m3x2_from_f32(p[2 * k], p[2 * k + 1]));
        v[2 * k] = __fmul_rn(w.x, ns);
        v[2 * k + 1] = __fmul_rn(w.y, ns);
    }
#endif
}

// Calls f(std::true_type{}) when every block scale of the unit takes the fast
// quotient, else f(std::false_type{}).
template <typename F>
__device__ __forceinline__ void with_fast(bool fast, F &&f) {
    if (fast) f(std::true_type{});
    else f(std::false_type{});
}

// What a receiver holds after K 128-blocks crossed the FP8 wire.  The warp
// holds block k as 4 values per lane in v[k] (lanes past a block's end hold
// +0, which leaves its amax unchanged).  In place.
template <int K>
__device__ __forceinline__ void wire_fp8_blocks(float (&v)[K][4]) {
    uint32_t key[K];
#pragma unroll
    for (int k = 0; k < K; ++k) key[k] = __float_as_uint(warp_amax4(v[k]));
    with_fast(publish_scales<float, K>(key), [&](auto fast) {
#pragma unroll
        for (int k = 0; k < K; ++k) wire4<decltype(fast)::value>(v[k], scale_of(k));
    });
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

// Elements of a 128-block that belong to this lane: 0..4.
__device__ __forceinline__ int lane_valid(size_t block_start, size_t len) {
    if (block_start >= len) return 0;
    const size_t rem = len - block_start;
    const int blen = rem < static_cast<size_t>(kBlock) ? static_cast<int>(rem) : kBlock;
    const int v = blen - lane_id() * 4;
    return v < 0 ? 0 : (v > 4 ? 4 : v);
}

}  // namespace rlx
