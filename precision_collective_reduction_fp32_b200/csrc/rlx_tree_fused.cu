// rlx_tree_fused.cu -- DDA-tree allreduce in one launch, for small messages.
//
// DDA-tree is a reduce-scatter phase followed by an all-gather phase
// ("Meta open-sources RCCLX", infolabhq pt, "Direct Data Access (DDA) — De
// O(N) para O(1) de Latência"; RCCLX post, es, "Ataque directo a datos
// (DDA)").  For small messages the cost of the separate pass-2 launch is a
// large part of the whole, so this kernel runs pass 1, a grid-wide barrier
// ("every chunk is reduced") and pass 2 in one cooperative launch.  The unit
// bodies are those of the two-launch form (rlx_passes.cuh), so the results
// are bit-identical.  A cooperative launch keeps every CTA of the grid
// resident at once, so the barrier cannot wait on a CTA that is not running;
// the launch itself fails (and nothing runs) if the grid would not fit.
#include <cooperative_groups.h>

#include <map>
#include <mutex>
#include <utility>

#include "rlx_passes.cuh"

namespace cg = cooperative_groups;

namespace rlx {
namespace {

template <typename T, int NR, bool VEC, bool FP8>
__global__ void __launch_bounds__(kThreads)
tree_fused_kernel(const T *send, T *recv, size_t count, size_t stride, int n, size_t chunk,
                  FastDiv per1, FastDiv per2, uint8_t *ws_codes, float *ws_scales) {
    constexpr uint32_t W = kThreads / 32;
    const uint32_t warp = blockIdx.x * W + (threadIdx.x >> 5);
    const uint32_t warps = gridDim.x * W;
    if constexpr (FP8) {
        const uint32_t units = static_cast<uint32_t>((count + kBlock - 1) / kBlock);
        for (uint32_t g = warp; g < units; g += warps)
            tree_reduce_fp8_unit<T, NR, VEC>(g, send, count, stride, n, ws_codes, ws_scales);
    } else {
        const uint32_t units = per1.d * static_cast<uint32_t>(n);
        for (uint32_t g = warp; g < units; g += warps)
            tree_reduce_native_unit<T, NR, VEC>(g, send, recv, count, stride, n, chunk, per1);
    }
    cg::this_grid().sync();   // all chunks reduced (and their writes visible) before pass 2
    if constexpr (FP8) {
        const uint32_t units = static_cast<uint32_t>(tree_gather_fp8_units(count));
        for (uint32_t g = warp; g < units; g += warps)
            tree_gather_fp8_unit<T, VEC>(g, recv, count, stride, n, ws_codes, ws_scales);
    } else {
        const uint32_t units = per2.d * static_cast<uint32_t>(n);
        for (uint32_t g = warp; g < units; g += warps)
            tree_gather_native_unit<T, VEC>(g, recv, count, stride, n, chunk, per2);
    }
}

// Resident CTAs of a kernel on the current device (cached per device).
int coresident_ctas(const void *kernel) {
    static std::mutex mu;
    static std::map<std::pair<int, const void *>, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find({dev, kernel});
    if (it != cache.end()) return it->second;
    int sms = 0, per_sm = 0, coop = 0;
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0);
    const int cap = coop ? sms * per_sm : 0;
    cache[{dev, kernel}] = cap;
    return cap;
}

template <typename F>
cudaError_t dispatch(rlx_dtype dtype, int n, bool vec, bool fp8, F &&f) {
#define RLX_CASE_NR(T, NRV)                                                              \
    if (n <= NRV) {                                                                      \
        if (fp8) return vec ? f.template operator()<T, NRV, true, true>()                \
                            : f.template operator()<T, NRV, false, true>();              \
        return vec ? f.template operator()<T, NRV, true, false>()                        \
                   : f.template operator()<T, NRV, false, false>();                      \
    }
#define RLX_CASE_T(T) \
    RLX_CASE_NR(T, 2) RLX_CASE_NR(T, 4) RLX_CASE_NR(T, 8) RLX_CASE_NR(T, 16)
    if (dtype == RLX_F32) { RLX_CASE_T(float) }
    else { RLX_CASE_T(uint16_t) }
#undef RLX_CASE_T
#undef RLX_CASE_NR
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_tree_fused(const void *send, void *recv, size_t count, size_t stride,
                              int nranks, size_t chunk, rlx_dtype dtype, rlx_wire wire,
                              uint8_t *ws_codes, float *ws_scales, bool vec,
                              cudaStream_t stream) {
    const bool fp8 = wire == RLX_WIRE_FP8_E4M3;
    return dispatch(dtype, nranks, vec, fp8, [&]<typename T, int NR, bool VEC, bool FP8>() {
        auto kernel = tree_fused_kernel<T, NR, VEC, FP8>;
        const size_t p1 = tree_reduce_native_per_chunk<T>(chunk);
        const size_t p2 = tree_gather_native_per_chunk<T>(chunk);
        if (p1 >= (size_t{1} << 32) || p2 >= (size_t{1} << 32)) return cudaErrorInvalidValue;
        const size_t nn = static_cast<size_t>(nranks);
        const size_t units = FP8 ? (count + kBlock - 1) / kBlock : p1 * nn;   // pass 1 is larger
        const int cap = coresident_ctas(reinterpret_cast<const void *>(kernel));
        if (cap <= 0) return cudaErrorCooperativeLaunchTooLarge;
        const size_t want = (units + kThreads / 32 - 1) / (kThreads / 32);
        const unsigned grid = static_cast<unsigned>(want < static_cast<size_t>(cap) ? (want ? want : 1) : cap);
        const T *s = static_cast<const T *>(send);
        T *r = static_cast<T *>(recv);
        int n = nranks;
        FastDiv f1 = make_fastdiv(static_cast<uint32_t>(p1));
        FastDiv f2 = make_fastdiv(static_cast<uint32_t>(p2));
        void *args[] = {&s, &r, &count, &stride, &n, &chunk, &f1, &f2, &ws_codes, &ws_scales};
        return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kernel), dim3(grid),
                                           dim3(kThreads), args, 0, stream);
    });
}

}  // namespace rlx
