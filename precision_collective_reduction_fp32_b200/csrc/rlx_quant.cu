// rlx_quant.cu -- standalone block quantisation to FP8 E4M3 and its inverse:
// the sender and receiver halves of every low-precision collective (RCCLX
// post, es, "Colectivos de mengua precisión": FP8 on the wire, up to 4:1
// smaller than FP32; "Coletivos de Baixa Precisão — Compressão FP8 com
// Precisão FP32", infolabhq pt).
//
// One warp per 128-element block, 4 elements per lane: the block amax is one
// warp reduction, each lane writes its 4 codes as one 32-bit word.
#include "rlx_device.cuh"
#include "rlx_internal.h"

namespace rlx {
namespace {

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
quantize_kernel(const T *x, size_t rows, size_t n, size_t stride, uint8_t *codes,
                float *scales) {
    const size_t nbr = (n + kBlock - 1) / kBlock;
    const size_t jobs = nbr * rows;
    const int e0 = lane_id() * 4;
    for (size_t job = global_warp(); job < jobs; job += num_warps()) {
        const size_t row = job / nbr;
        const size_t b = job - row * nbr;
        const size_t off = row * stride + b * kBlock;
        const size_t done = b * kBlock;
        const int len = n - done < static_cast<size_t>(kBlock) ? static_cast<int>(n - done) : kBlock;
        const int valid = lane_valid(len);
        float v[4];
        load4<T, VEC>(x + off + e0, valid, v);
        const float s = block_scale(warp_amax4(v));
        const uint32_t q = quant4(v, s);
        uint8_t *dst = codes + off + e0;
        if (VEC && valid == 4) {
            __stcs(reinterpret_cast<unsigned int *>(dst), q);
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < valid) dst[k] = static_cast<uint8_t>(q >> (8 * k));
        }
        if (lane_id() == 0) scales[job] = s;   // job == row * nbr + b
    }
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
dequantize_kernel(const uint8_t *codes, const float *scales, size_t rows, size_t n,
                  size_t stride, T *y) {
    const size_t nbr = (n + kBlock - 1) / kBlock;
    const size_t jobs = nbr * rows;
    const int e0 = lane_id() * 4;
    for (size_t job = global_warp(); job < jobs; job += num_warps()) {
        const size_t row = job / nbr;
        const size_t b = job - row * nbr;
        const size_t off = row * stride + b * kBlock;
        const size_t done = b * kBlock;
        const int len = n - done < static_cast<size_t>(kBlock) ? static_cast<int>(n - done) : kBlock;
        const int valid = lane_valid(len);
        const uint8_t *src = codes + off + e0;
        uint32_t q = 0;
        if (VEC && valid == 4) {
            q = __ldcs(reinterpret_cast<const unsigned int *>(src));
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (k < valid) q |= static_cast<uint32_t>(src[k]) << (8 * k);
        }
        const float s = __ldcs(scales + job);
        float v[4];
        dequant4(q, s, v);
        store4<T, VEC>(y + off + e0, valid, v);
    }
}

template <typename F>
cudaError_t dispatch(rlx_dtype dtype, bool vec, F &&f) {
    if (dtype == RLX_F32)
        return vec ? f.template operator()<float, true>() : f.template operator()<float, false>();
    return vec ? f.template operator()<uint16_t, true>() : f.template operator()<uint16_t, false>();
}

constexpr size_t kWarps = kThreads / 32;

}  // namespace

cudaError_t launch_quantize(const void *x, rlx_dtype dtype, size_t rows, size_t n,
                            size_t stride, uint8_t *codes, float *scales, bool vec,
                            cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        const size_t jobs = (n + kBlock - 1) / kBlock * rows;
        auto k = quantize_kernel<T, VEC>;
        const int grid = persistent_grid(reinterpret_cast<const void *>(k), jobs, kWarps);
        k<<<grid, kThreads, 0, stream>>>(static_cast<const T *>(x), rows, n, stride, codes, scales);
        return cudaGetLastError();
    });
}

cudaError_t launch_dequantize(const uint8_t *codes, const float *scales, size_t rows,
                              size_t n, size_t stride, void *y, rlx_dtype dtype, bool vec,
                              cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        const size_t jobs = (n + kBlock - 1) / kBlock * rows;
        auto k = dequantize_kernel<T, VEC>;
        const int grid = persistent_grid(reinterpret_cast<const void *>(k), jobs, kWarps);
        k<<<grid, kThreads, 0, stream>>>(codes, scales, rows, n, stride, static_cast<T *>(y));
        return cudaGetLastError();
    });
}

}  // namespace rlx
