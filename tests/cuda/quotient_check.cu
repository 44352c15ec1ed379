// Test-only kernel: compares the library's fast block quotient (reciprocal +
// two Markstein corrections) with CUDA's IEEE division over every fp32 bit
// pattern in [x_first, x_first + nx) and every scale given: the E4M3 codes of
// the two quotients must always agree, and the quotients themselves bit for
// bit wherever |x/s| >= 2^-12 (below that every code is +-0).  Both forms are
// checked: the scalar quotient_rn, and the packed negated quotient the
// kernels use (neg_quotient2, whose result must be exactly -quotient_rn's,
// and whose sign-flipped codes must be the IEEE quotient's codes) -- in
// whichever form the build selects (RLX_QUOTIENT_2TERM: the two-term
// reciprocal and one correction, else two corrections).
// Built and loaded by tests/test_gpu_quotient.py; not part of the library.
#include <cstdint>
#include <cstdio>
#include <cuda_runtime.h>

#include "../../precision_collective_reduction_fp32_b200/csrc/rlx_device.cuh"

__global__ void quotient_check_kernel(const float *scales, int ns, uint32_t x_first, uint32_t nx,
                                      unsigned long long *mismatches, uint32_t *witness) {
    const size_t step = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nx; i += step) {
        const float x = __uint_as_float(x_first + static_cast<uint32_t>(i));
        for (int k = 0; k < ns; ++k) {
            const float s = scales[k];
            const float y = __frcp_rn(s);
            const float q = rlx::quotient_rn(x, s, y);
            const rlx::Scale2 sc = rlx::pack(rlx::reciprocal_terms(s));
            const float2 p = rlx::neg_quotient2(make_float2(x, -x), sc);   // -q(x), -q(-x)
            const float ref = __fdiv_rn(x, s);
            const bool bits_matter = fabsf(ref) >= 0x1p-12f;
            const uint32_t ref_code = rlx::e4m3x2_from_f32(ref, -ref);
            const bool differ = (bits_matter && __float_as_uint(q) != __float_as_uint(ref)) ||
                                (bits_matter && __float_as_uint(p.x) != (__float_as_uint(ref) ^ 0x80000000u)) ||
                                (bits_matter && __float_as_uint(p.y) != __float_as_uint(ref)) ||
                                rlx::e4m3x2_from_f32(q, -q) != ref_code ||
                                (rlx::e4m3x2_from_f32(p.x, p.y) ^ 0x8080u) != ref_code;
            if (differ) {
                if (atomicAdd(mismatches, 1ull) == 0ull) {
                    witness[0] = __float_as_uint(x);
                    witness[1] = __float_as_uint(s);
                    witness[2] = __float_as_uint(q);
                    witness[3] = __float_as_uint(ref);
                }
            }
        }
    }
}

// Returns 0 on success (mismatch count and a witness in the outputs),
// otherwise the cudaError_t of the failing call.
extern "C" int quotient_check(const float *scales_host, int ns, uint32_t x_first, uint32_t nx,
                              unsigned long long *mismatches_out, uint32_t *witness_out) {
    float *d_s = nullptr;
    unsigned long long *d_m = nullptr;
    uint32_t *d_w = nullptr;
    cudaError_t e = cudaMalloc(&d_s, sizeof(float) * ns);
    if (e == cudaSuccess) e = cudaMalloc(&d_m, sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaMalloc(&d_w, 4 * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMemcpy(d_s, scales_host, sizeof(float) * ns, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(d_m, 0, sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaMemset(d_w, 0, 4 * sizeof(uint32_t));
    if (e == cudaSuccess) {
        quotient_check_kernel<<<148 * 8, 256>>>(d_s, ns, x_first, nx, d_m, d_w);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(mismatches_out, d_m, sizeof(unsigned long long), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(witness_out, d_w, 4 * sizeof(uint32_t), cudaMemcpyDeviceToHost);
    cudaFree(d_s);
    cudaFree(d_m);
    cudaFree(d_w);
    return static_cast<int>(e);
}
