// rlx_noalloc.cu -- rlx_allreduce_tree_noalloc: the DDA-tree allreduce with
// its FP8 wire payload kept in a fixed device array instead of a
// caller-provided workspace.
//
// Who needs it: callers that cannot call cudaMalloc (or any allocator) at
// the point where they run the collective -- for instance a plug-in that is
// handed only its input and output buffers and owns no allocator, or a
// latency-critical loop that must not allocate because cudaMalloc can
// synchronise the whole device and stall every other stream.
//
// How it works: the payload (codes + scales of the reduced chunks, written
// by pass 1 and read by pass 2) lives in `g_tree_scratch`, a file-scope
// __device__ array of kScratchBytes, enough for RLX_NOALLOC_MAX_COUNT
// elements per rank (16 Mi elements: 16.5 MiB).  Every GPU that loads the
// library holds that array until the process exits.  Host code cannot use the array's name
// as a device address, so on the first call on each device this file asks
// the runtime for the address (cudaGetSymbolAddress, with that device
// current) and caches it; that first call should come before any stream
// capture.  Every call on a device shares the one array and the array keeps
// the last call's contents; nothing in it has to start at zero, because pass
// 1 writes every code and scale of every block before pass 2 reads them.
// Two calls whose kernels overlap on the GPU (different streams, no
// ordering between them) race on the array.
#include <cstdint>
#include <mutex>

#include "rlx_internal.h"

namespace {

constexpr size_t kScratchBytes =
    size_t{RLX_NOALLOC_MAX_COUNT} + size_t{RLX_NOALLOC_MAX_COUNT} / RLX_BLOCK * sizeof(float);

__device__ __align__(256) uint8_t g_tree_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device with that device current.  nullptr (and *err set) on failure.
void *scratch_address(cudaError_t *err) {
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_tree_scratch);
        if (*err != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" rlx_status rlx_allreduce_tree_noalloc(const void *send, void *recv, size_t count,
                                                 size_t stride, int nranks, rlx_dtype dtype,
                                                 rlx_wire wire, rlx_op op, void *stream) {
    const size_t need = rlx_workspace_bytes(RLX_COLL_ALLREDUCE_TREE, count, nranks, dtype, wire);
    // With no workspace, rlx_allreduce_tree checks every other argument and,
    // when they are valid but a payload is needed, returns RLX_ERR_WORKSPACE
    // having launched nothing; native wire, one rank or count 0 need none
    // and run right there.
    const rlx_status st = rlx_allreduce_tree(send, recv, count, stride, nranks, dtype, wire, op,
                                             nullptr, 0, stream);
    if (need == 0 || st != RLX_ERR_WORKSPACE) return st;
    if (need > kScratchBytes) return RLX_ERR_WORKSPACE;   // count > RLX_NOALLOC_MAX_COUNT
    cudaError_t err = cudaSuccess;
    void *ws = scratch_address(&err);
    if (ws == nullptr) {
        rlx::record_cuda_error(err);
        return RLX_ERR_CUDA;
    }
    return rlx_allreduce_tree(send, recv, count, stride, nranks, dtype, wire, op, ws,
                              kScratchBytes, stream);
}
