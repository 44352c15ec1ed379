// rlx_device.cuh -- device-side building blocks shared by the rlx kernels.
//
// Element access (vectorised 16/8-byte or element-wise), the FP8 E4M3 codec on
// the hardware cvt instructions, the warp-wide block amax, and the "wire"
// transform dequantise(quantise(x)) of one 128-element block held as 4 values
// per lane of a warp.  Every floating-point step is an explicit
// round-to-nearest intrinsic so that the compiler cannot contract a multiply
// and an add into an FMA.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace rlx {

constexpr int kBlock = 128;        // elements per FP8 scale block
constexpr float kE4m3Max = 448.0f; // largest finite E4M3 magnitude
constexpr unsigned kFull = 0xffffffffu;

// ------------------------------------------------------------ element types

// bf16 <-> fp32: widening is exact; narrowing is round-to-nearest-even.
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Element traits: load/store one element as fp32.
template <typename T> struct Elem;
template <> struct Elem<float> {
    using storage = float;
    __device__ __forceinline__ static float load(const float *p) { return __ldcs(p); }
    __device__ __forceinline__ static void store(float *p, float v) { __stcs(p, v); }
};
template <> struct Elem<uint16_t> {  // bf16 bit patterns
    using storage = uint16_t;
    __device__ __forceinline__ static float load(const uint16_t *p) {
        return bf16_bits_to_f32(__ldcs(reinterpret_cast<const unsigned short *>(p)));
    }
    __device__ __forceinline__ static void store(uint16_t *p, float v) {
        __stcs(reinterpret_cast<unsigned short *>(p), f32_to_bf16_bits(v));
    }
};

// Four consecutive elements starting at p, `valid` of them real (0..4); the
// rest read as +0.  VEC: p is aligned to 4 elements (16 B fp32, 8 B bf16).
template <typename T, bool VEC>
__device__ __forceinline__ void load4(const T *p, int valid, float (&v)[4]) {
    if (VEC && valid == 4) {
        if constexpr (sizeof(T) == 4) {
            float4 q = __ldcs(reinterpret_cast<const float4 *>(p));
            v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
        } else {
            uint2 q = __ldcs(reinterpret_cast<const uint2 *>(p));
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
            __stcs(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
        } else {
            uint2 q;
            q.x = static_cast<uint32_t>(f32_to_bf16_bits(v[0])) |
                  (static_cast<uint32_t>(f32_to_bf16_bits(v[1])) << 16);
            q.y = static_cast<uint32_t>(f32_to_bf16_bits(v[2])) |
                  (static_cast<uint32_t>(f32_to_bf16_bits(v[3])) << 16);
            __stcs(reinterpret_cast<uint2 *>(p), q);
        }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k < valid) Elem<T>::store(p + k, v[k]);
    }
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

// ------------------------------------------------------------ block helpers

// max |v| over the 4 values of every lane of the warp (all 32 lanes must call).
// For non-negative floats the IEEE bit order is the value order, so the warp
// reduction runs on the integer bits.
__device__ __forceinline__ float warp_amax4(const float (&v)[4]) {
    uint32_t m = __float_as_uint(v[0]) & 0x7fffffffu;
    m = max(m, __float_as_uint(v[1]) & 0x7fffffffu);
    m = max(m, __float_as_uint(v[2]) & 0x7fffffffu);
    m = max(m, __float_as_uint(v[3]) & 0x7fffffffu);
    return __uint_as_float(__reduce_max_sync(kFull, m));
}

// Block scale s = fl32(amax / 448), correctly rounded.
__device__ __forceinline__ float block_scale(float amax) { return __fdiv_rn(amax, kE4m3Max); }

// Quantise 4 values with scale s: code = e4m3_rne_sat(fl32(v / s)); s == 0
// gives signed zeros.
__device__ __forceinline__ uint32_t quant4(const float (&v)[4], float s) {
    float q[4];
    if (s == 0.0f) {
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = __fmul_rn(v[k], 0.0f);  // +-0 with v's sign
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = __fdiv_rn(v[k], s);
    }
    return e4m3x4_from_f32(q);
}

// Dequantise 4 packed codes with scale s: fl32(e4m3(code) * s).
__device__ __forceinline__ void dequant4(uint32_t codes, float s, float (&y)[4]) {
    const float2 a = e4m3x2_to_f32(codes & 0xffffu);
    const float2 b = e4m3x2_to_f32(codes >> 16);
    y[0] = __fmul_rn(a.x, s);
    y[1] = __fmul_rn(a.y, s);
    y[2] = __fmul_rn(b.x, s);
    y[3] = __fmul_rn(b.y, s);
}

// What a receiver holds after one 128-block crossed the FP8 wire: the warp
// holds the block as 4 values per lane (lanes past the end hold +0, which
// leaves amax unchanged); returns dequantise(quantise(v)) in place.
__device__ __forceinline__ void wire_fp8_block(float (&v)[4]) {
    const float s = block_scale(warp_amax4(v));
    dequant4(quant4(v, s), s, v);
}

// ----------------------------------------------------------- grid helpers

__device__ __forceinline__ size_t global_warp() {
    return (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
}
__device__ __forceinline__ size_t num_warps() {
    return (static_cast<size_t>(gridDim.x) * blockDim.x) >> 5;
}
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// Elements of a 128-block that belong to this lane: 0..4.
__device__ __forceinline__ int lane_valid(int block_len) {
    const int v = block_len - lane_id() * 4;
    return v < 0 ? 0 : (v > 4 ? 4 : v);
}

}  // namespace rlx
