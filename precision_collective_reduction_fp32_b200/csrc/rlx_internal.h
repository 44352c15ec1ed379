// rlx_internal.h -- launcher interface between the C ABI layer (rlx_api.cu)
// and the kernel translation units.  Arguments reaching these functions have
// already been validated; `vec` says the vectorised kernels may be used
// (every row and chunk start is aligned as the kernel requires).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/rlx.h"

namespace rlx {

constexpr int kThreads = 256;  // threads per CTA for every kernel

// Grid for `units` units of work, `units_per_cta` per CTA: one CTA per group
// of units (the kernels loop if the grid is smaller).  The unit count must be
// below 2^32 (the kernels index units with 32 bits); larger requests return
// an empty grid.
dim3 grid_for(const void *kernel, size_t units, size_t units_per_cta);

// Launches kernel<<<grid, kThreads, 0, stream>>>(args...) allowing
// programmatic dependent launch (RLX_PDL=1, default): the kernel may be
// scheduled while the previous kernel on the stream finishes; every rlx
// kernel waits for it (griddepcontrol.wait) before touching memory.
#ifndef RLX_PDL
#define RLX_PDL 1
#endif
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, cudaStream_t stream,
                          Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = RLX_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Records a CUDA failure for rlx_last_cuda_error() of the calling thread.
void record_cuda_error(cudaError_t e);

// DDA-flat, all wires.  nranks >= 2.
cudaError_t launch_allreduce_flat(const void *send, void *recv, size_t count, size_t stride,
                                  int nranks, rlx_dtype dtype, rlx_wire wire, bool vec,
                                  cudaStream_t stream);

// DDA-tree pass 1 (reduce-scatter).  Native: writes chunk c into recv row c.
// FP8: writes the requantised chunk codes/scales into the workspace.
cudaError_t launch_tree_reduce(const void *send, void *recv, size_t count, size_t stride,
                               int nranks, size_t chunk, rlx_dtype dtype, rlx_wire wire,
                               uint8_t *ws_codes, float *ws_scales, bool vec,
                               cudaStream_t stream);

// DDA-tree pass 2 (all-gather).
cudaError_t launch_tree_gather(void *recv, size_t count, size_t stride, int nranks,
                               size_t chunk, rlx_dtype dtype, rlx_wire wire,
                               const uint8_t *ws_codes, const float *ws_scales, bool vec,
                               cudaStream_t stream);

// DDA-tree in one launch over thread-block clusters (rlx_tree_cluster.cu):
// the same arguments and results as the two passes above.  tree_cluster_wanted
// says whether a call is small enough for it to be the faster path.
bool tree_cluster_wanted(size_t count, int nranks, size_t chunk, rlx_dtype dtype, rlx_wire wire);
cudaError_t launch_tree_cluster(const void *send, void *recv, size_t count, size_t stride,
                                int nranks, size_t chunk, rlx_dtype dtype, rlx_wire wire,
                                uint8_t *ws_codes, float *ws_scales, bool vec,
                                cudaStream_t stream);

// DDA-tree in one launch with chunk-ready counts (rlx_tree_fused.cu).
// workspace: RLX_TREE_SYNC_BYTES of sync words (zero on entry), then on the
// FP8 wire the payload.  status may be null.
cudaError_t launch_tree_fused(const void *send, void *recv, size_t count, size_t stride,
                              int nranks, size_t chunk, rlx_dtype dtype, rlx_wire wire,
                              void *workspace, int *status, uint64_t limit_ns, bool vec,
                              cudaStream_t stream);

cudaError_t launch_reduce_scatter(const void *send, size_t send_stride, void *recv,
                                  size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                                  rlx_wire wire, bool vec, cudaStream_t stream);

cudaError_t launch_all_gather(const void *send, size_t send_stride, void *recv,
                              size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                              rlx_wire wire, bool vec, cudaStream_t stream);

cudaError_t launch_alltoall(const void *send, size_t send_stride, void *recv,
                            size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                            rlx_wire wire, bool vec, cudaStream_t stream);

// Row copy (every collective with one rank): dst[j] = src[j], j < n.
cudaError_t launch_copy(const void *src, void *dst, size_t n, rlx_dtype dtype, bool vec,
                        cudaStream_t stream);

cudaError_t launch_quantize(const void *x, rlx_dtype dtype, size_t rows, size_t n,
                            size_t stride, uint8_t *codes, float *scales, bool vec,
                            cudaStream_t stream);

cudaError_t launch_dequantize(const uint8_t *codes, const float *scales, size_t rows,
                              size_t n, size_t stride, void *y, rlx_dtype dtype, bool vec,
                              cudaStream_t stream);

}  // namespace rlx
