// rlx_quant.cu -- standalone block quantisation to FP8 E4M3 and its inverse:
// the sender and receiver halves of every low-precision collective (RCCLX
// post, es, "Colectivos de mengua precisión": FP8 on the wire, up to 4:1
// smaller than FP32; "Coletivos de Baixa Precisão — Compressão FP8 com
// Precisão FP32", infolabhq pt).
//
// A warp handles kJq consecutive 128-element blocks of one row at once (4
// for fp32, 8 for bf16), 4 elements per lane per block: each block amax is
// one warp reduction, each lane writes its 4 codes of a block as one 32-bit
// word.  Units (row, group of kJq blocks) are numbered row-major and handed
// out in CTA-sized runs.
#include "rlx_passes.cuh"

namespace rlx {
namespace {

#ifndef RLX_JQ
#define RLX_JQ 4
#endif
// bf16: the loads stay raw until their block is quantised (quant_blocks_raw),
// so 8 blocks per unit fit the register budget; at the prefill size (8 x 32 Mi
// bf16) 170.2 us with widened loads and 4 blocks, 158.8 raw with 4, 135.9 raw
// with 8.
#ifndef RLX_JQ_BF16
#define RLX_JQ_BF16 8
#endif
#ifndef RLX_JDQ
#define RLX_JDQ 8
#endif
#ifndef RLX_P_Q
#define RLX_P_Q 4
#endif
#ifndef RLX_P_DQ
#define RLX_P_DQ 1
#endif
// Resident CTAs per SM requested from the compiler for the quantiser
// (0: no request).
#ifndef RLX_MINB_Q
#define RLX_MINB_Q 0
#endif
template <typename T> constexpr int kJq = sizeof(T) == 2 ? RLX_JQ_BF16 : RLX_JQ;  // blocks per warp unit, quantise
constexpr int kJdq = RLX_JDQ;   // blocks in flight per warp, dequantise
constexpr int kPq = RLX_P_Q;   // units per warp per CTA run, quantise
constexpr int kPdq = RLX_P_DQ; // units per warp per CTA run, dequantise

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads, RLX_MINB_Q)
quantize_kernel(const T *x, size_t rows, size_t n, size_t stride, uint8_t *codes,
                float *scales, FastDiv per_row) {
    const size_t nbr = (n + kBlock - 1) / kBlock;
    const uint32_t units = per_row.d * static_cast<uint32_t>(rows);
    const int e0 = lane_id() * 4;
    for_each_unit<kPq>(units, [&](uint32_t g) {
        const uint32_t row = fast_div(g, per_row);
        const size_t b0 = static_cast<size_t>(g - row * per_row.d) * kJq<T>;
        with_full((b0 + kJq<T>) * kBlock <= n, [&](auto full) {
            constexpr bool F = decltype(full)::value;
            const T *xr = x + row * stride + b0 * kBlock + e0;
            uint8_t *cr = codes + row * stride + b0 * kBlock + e0;
            int valid[kJq<T>];
#pragma unroll
            for (int j = 0; j < kJq<T>; ++j) valid[j] = F ? 4 : lane_valid((b0 + j) * kBlock, n);
            quant_blocks_raw<T, VEC, kJq<T>>(xr, valid, [&](int j, uint32_t q) {
                uint8_t *dst = cr + j * kBlock;
                if (VEC && valid[j] == 4) {
                    st_stream(reinterpret_cast<unsigned int *>(dst), q);
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < valid[j]) dst[k] = static_cast<uint8_t>(q >> (8 * k));
                }
            });
            // lane j < kJq stores the scale of block b0 + j
            const int l = lane_id();
            if (l < kJq<T> && (F || b0 + l < nbr))
                st_stream(scales + row * nbr + b0 + l, scale_of(l).s.x);
        });
    });
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(kThreads)
dequantize_kernel(const uint8_t *codes, const float *scales, size_t rows, size_t n,
                  size_t stride, T *y, FastDiv per_row) {
    const size_t nbr = (n + kBlock - 1) / kBlock;
    const uint32_t units = per_row.d * static_cast<uint32_t>(rows);
    const int e0 = lane_id() * 4;
    for_each_unit<kPdq>(units, [&](uint32_t g) {
        const uint32_t row = fast_div(g, per_row);
        const size_t b0 = static_cast<size_t>(g - row * per_row.d) * kJdq;
        with_full((b0 + kJdq) * kBlock <= n, [&](auto full) {
            constexpr bool F = decltype(full)::value;
            const uint8_t *cr = codes + row * stride + b0 * kBlock + e0;
            const float *sr = scales + row * nbr + b0;
            T *yr = y + row * stride + b0 * kBlock + e0;
            uint32_t q[kJdq];
            float s[kJdq];
            int valid[kJdq];
#pragma unroll
            for (int j = 0; j < kJdq; ++j) {
                valid[j] = F ? 4 : lane_valid((b0 + j) * kBlock, n);
                const uint8_t *src = cr + j * kBlock;
                q[j] = 0;
                if (VEC && valid[j] == 4) {
                    q[j] = ld_stream(reinterpret_cast<const unsigned int *>(src));
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < valid[j]) q[j] |= static_cast<uint32_t>(src[k]) << (8 * k);
                }
                s[j] = (F || b0 + j < nbr) ? ld_stream(sr + j) : 0.0f;
            }
#pragma unroll
            for (int j = 0; j < kJdq; ++j) {
                float v[4];
                dequant4(q[j], s[j], v);
                store4<T, VEC>(yr + j * kBlock, valid[j], v);
            }
        });
    });
}

template <typename F>
cudaError_t dispatch(rlx_dtype dtype, bool vec, F &&f) {
    if (dtype == RLX_F32)
        return vec ? f.template operator()<float, true>() : f.template operator()<float, false>();
    return vec ? f.template operator()<uint16_t, true>() : f.template operator()<uint16_t, false>();
}

constexpr size_t kWarps = kThreads / 32;

template <typename K, typename... Args>
cudaError_t launch_rows(K kernel, size_t rows, size_t n, size_t blocks_per_unit,
                        size_t units_per_warp, cudaStream_t stream, Args... args) {
    const size_t per = ((n + kBlock - 1) / kBlock + blocks_per_unit - 1) / blocks_per_unit;
    if (per >= (size_t{1} << 32) || rows >= (size_t{1} << 32)) return cudaErrorInvalidValue;
    const dim3 grid = grid_for(reinterpret_cast<const void *>(kernel), per * rows,
                               kWarps * units_per_warp);
    if (grid.x == 0) return cudaErrorInvalidValue;
    return launch_kernel(kernel, grid, stream, args..., make_fastdiv(static_cast<uint32_t>(per)));
}

}  // namespace

cudaError_t launch_quantize(const void *x, rlx_dtype dtype, size_t rows, size_t n,
                            size_t stride, uint8_t *codes, float *scales, bool vec,
                            cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        return launch_rows(quantize_kernel<T, VEC>, rows, n, kJq<T>, kPq, stream,
                           static_cast<const T *>(x), rows, n, stride, codes, scales);
    });
}

cudaError_t launch_dequantize(const uint8_t *codes, const float *scales, size_t rows,
                              size_t n, size_t stride, void *y, rlx_dtype dtype, bool vec,
                              cudaStream_t stream) {
    return dispatch(dtype, vec, [&]<typename T, bool VEC>() {
        return launch_rows(dequantize_kernel<T, VEC>, rows, n, kJdq, kPdq, stream, codes, scales, rows,
                           n, stride, static_cast<T *>(y));
    });
}

}  // namespace rlx
