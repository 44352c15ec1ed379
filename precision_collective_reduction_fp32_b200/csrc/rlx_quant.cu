// rlx_quant.cu -- standalone block quantisation to FP8 E4M3 and its inverse:
// the sender and receiver halves of every low-precision collective (RCCLX
// post, es, "Colectivos de mengua precisión": FP8 on the wire, up to 4:1
// smaller than FP32; "Coletivos de Baixa Precisão — Compressão FP8 com
// Precisão FP32", infolabhq pt).
//
// A warp handles kJ consecutive 128-element blocks of one row at once, 4
// elements per lane per block: each block amax is one warp reduction, each
// lane writes its 4 codes of a block as one 32-bit word.  Rows are the grid's
// y dimension.
#include "rlx_device.cuh"
#include "rlx_internal.h"

namespace rlx {
namespace {

constexpr int kJq = 4;   // blocks per warp, quantise
constexpr int kJd = 8;   // blocks per warp, dequantise

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
quantize_kernel(const T *x, size_t rows, size_t n, size_t stride, uint8_t *codes,
                float *scales) {
    const size_t nbr = (n + kBlock - 1) / kBlock;
    const int e0 = lane_id() * 4;
    for (size_t row = blockIdx.y; row < rows; row += gridDim.y) {
        const T *xr = x + row * stride;
        uint8_t *cr = codes + row * stride;
        float *sr = scales + row * nbr;
        for (size_t b0 = warp_in_grid_x() * kJq; b0 < nbr; b0 += warps_in_grid_x() * kJq) {
            float v[kJq][4];
            int valid[kJq];
            float amax[kJq];
#pragma unroll
            for (int j = 0; j < kJq; ++j) {
                valid[j] = lane_valid((b0 + j) * kBlock, n);
                load4<T, VEC>(xr + (b0 + j) * kBlock + e0, valid[j], v[j]);
            }
#pragma unroll
            for (int j = 0; j < kJq; ++j) amax[j] = warp_amax4(v[j]);
            Scale sc[kJq];
            make_scales<kJq>(amax, sc);
#pragma unroll
            for (int j = 0; j < kJq; ++j) {
                const uint32_t q = quant4(v[j], sc[j]);
                uint8_t *dst = cr + (b0 + j) * kBlock + e0;
                if (VEC && valid[j] == 4) {
                    __stcs(reinterpret_cast<unsigned int *>(dst), q);
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < valid[j]) dst[k] = static_cast<uint8_t>(q >> (8 * k));
                }
            }
            // lane j < kJq stores the scale of block b0 + j
            const int l = lane_id();
            if (l < kJq && b0 + l < nbr) {
                float s = sc[0].s;
#pragma unroll
                for (int j = 1; j < kJq; ++j)
                    if (l == j) s = sc[j].s;
                __stcs(sr + b0 + l, s);
            }
        }
    }
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
dequantize_kernel(const uint8_t *codes, const float *scales, size_t rows, size_t n,
                  size_t stride, T *y) {
    const size_t nbr = (n + kBlock - 1) / kBlock;
    const int e0 = lane_id() * 4;
    for (size_t row = blockIdx.y; row < rows; row += gridDim.y) {
        const uint8_t *cr = codes + row * stride;
        const float *sr = scales + row * nbr;
        T *yr = y + row * stride;
        for (size_t b0 = warp_in_grid_x() * kJd; b0 < nbr; b0 += warps_in_grid_x() * kJd) {
            uint32_t q[kJd];
            float s[kJd];
            int valid[kJd];
#pragma unroll
            for (int j = 0; j < kJd; ++j) {
                const size_t b = b0 + j;
                valid[j] = lane_valid(b * kBlock, n);
                const uint8_t *src = cr + b * kBlock + e0;
                q[j] = 0;
                if (VEC && valid[j] == 4) {
                    q[j] = __ldcs(reinterpret_cast<const unsigned int *>(src));
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < valid[j]) q[j] |= static_cast<uint32_t>(src[k]) << (8 * k);
                }
                s[j] = b < nbr ? __ldcs(sr + b) : 0.0f;
            }
#pragma unroll
            for (int j = 0; j < kJd; ++j) {
                float v[4];
                dequant4(q[j], s[j], v);
                store4<T, VEC>(yr + (b0 + j) * kBlock + e0, valid[j], v);
            }
        }
    }
}

template <typename F>
cudaError_t dispatch(rlx_dtype dtype, bool vec, F &&f) {
    if (dtype == RLX_F32)
        return vec ? f.template operator()<float, true>() : f.template operator()<float, false>();
    return vec ? f.template operator()<uint16_t, true>() : f.template operator()<uint16_t, false>();
}

constexpr size_t kWarps = kThreads / 32;
constexpr unsigned kMaxGridY = 65535;

unsigned row_segments(size_t rows) {
    return rows < kMaxGridY ? static_cast<unsigned>(rows) : kMaxGridY;
}

}  // namespace

cudaError_t launch_quantize(const void *x, rlx_dtype dtype, size_t rows, size_t n,
                            size_t stride, uint8_t *codes, float *scales, bool vec,
                            cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        auto k = quantize_kernel<T, VEC>;
        const dim3 grid = grid_2d(reinterpret_cast<const void *>(k), row_segments(rows),
                                  (n + kBlock - 1) / kBlock, kWarps * kJq);
        k<<<grid, kThreads, 0, stream>>>(static_cast<const T *>(x), rows, n, stride, codes, scales);
        return cudaGetLastError();
    });
}

cudaError_t launch_dequantize(const uint8_t *codes, const float *scales, size_t rows,
                              size_t n, size_t stride, void *y, rlx_dtype dtype, bool vec,
                              cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        auto k = dequantize_kernel<T, VEC>;
        const dim3 grid = grid_2d(reinterpret_cast<const void *>(k), row_segments(rows),
                                  (n + kBlock - 1) / kBlock, kWarps * kJd);
        k<<<grid, kThreads, 0, stream>>>(codes, scales, rows, n, stride, static_cast<T *>(y));
        return cudaGetLastError();
    });
}

}  // namespace rlx
