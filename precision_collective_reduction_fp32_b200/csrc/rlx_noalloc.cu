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
// library holds that array until the process exits.  Host code cannot use
// the array's name as a device address, so this file asks the runtime for
// the address (cudaGetSymbolAddress, with the device current) and caches it
// per device,
// together with the id of the CUDA context it was taken in.  The lookup
// happens on the first call on each device, and again on the first call
// after that device's context was replaced (cudaDeviceReset reloads the
// module, and the array may then sit elsewhere); such a first call should
// come before any stream capture.  Every call on a device shares the one
// array and the array keeps the last call's contents; nothing in it has to
// start at zero, because pass 1 writes every code and scale of every block
// before pass 2 reads them.  Two calls whose kernels overlap on the GPU
// (different streams, no ordering between them) race on the array.
#include <cstdint>
#include <mutex>

#include <cuda.h>

#include "rlx_internal.h"

namespace {

constexpr size_t kScratchBytes =
    size_t{RLX_NOALLOC_MAX_COUNT} + size_t{RLX_NOALLOC_MAX_COUNT} / RLX_BLOCK * sizeof(float);

__device__ __align__(256) uint8_t g_tree_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
struct Slot {
    unsigned long long ctx;   // id of the context the address was taken in (0: none known)
    void *ptr;
};
std::mutex g_mu;
Slot g_slot[kMaxDevices] = {};

// Id of the calling thread's current CUDA context, through the driver's
// cuCtxGetId fetched from the runtime (no link-time dependency on the driver
// library).  false when there is no current context or the query fails.
bool current_context_id(unsigned long long *id) {
    using GetId = CUresult (*)(CUcontext, unsigned long long *);
    static GetId fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<GetId>(p);
    }();
    return fn != nullptr && fn(nullptr, id) == CUDA_SUCCESS && *id != 0;
}

// Device address of the scratch array in the current device's context,
// looked up with that device current on the first call in each context.
// nullptr (and *err set) on failure.
void *scratch_address(cudaError_t *err) {
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    unsigned long long ctx = 0;
    const bool known = current_context_id(&ctx);
    std::lock_guard<std::mutex> lock(g_mu);
    Slot &slot = g_slot[dev];
    if (slot.ptr == nullptr || !known || slot.ctx != ctx) {
        void *p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_tree_scratch);   // makes the context current too
        if (*err != cudaSuccess) return nullptr;
        unsigned long long now = 0;
        slot.ctx = current_context_id(&now) ? now : 0;     // 0: look up again next call
        slot.ptr = p;
    }
    return slot.ptr;
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
