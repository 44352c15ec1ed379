// rlx_api.cu -- the extern "C" boundary of librlx.so: argument checks, choice
// of the vectorised or element-wise kernels, and the order of the passes.
// Nothing here touches the data; every arithmetic step runs in the kernels.
#include <climits>
#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "rlx_internal.h"

namespace rlx {

dim3 grid_for(const void *kernel, size_t units, size_t units_per_cta) {
    if (units >= (size_t{1} << 32)) return dim3(0, 1, 1);
    size_t x = (units + units_per_cta - 1) / units_per_cta;
    if (x == 0) x = 1;
#ifndef RLX_GRID_WAVES
#define RLX_GRID_WAVES 0
#endif
    // RLX_GRID_WAVES > 0 caps the grid at that many waves of resident CTAs.
    if (RLX_GRID_WAVES > 0) {
        static std::mutex mu;
        static std::map<std::pair<int, const void *>, int> cap_cache;
        int dev = 0;
        cudaGetDevice(&dev);
        int cap = 0;
        std::lock_guard<std::mutex> lock(mu);
        auto it = cap_cache.find({dev, kernel});
        if (it != cap_cache.end()) {
            cap = it->second;
        } else {
            int sms = 0, per_sm = 0;
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0);
            cap = sms * (per_sm > 0 ? per_sm : 1);
            cap_cache[{dev, kernel}] = cap;
        }
        const size_t lim = static_cast<size_t>(cap) * RLX_GRID_WAVES;
        if (lim > 0 && x > lim) x = lim;
    }
    if (x > 0x7fffffffu) x = 0x7fffffffu;
    return dim3(static_cast<unsigned>(x), 1, 1);
}

}  // namespace rlx

namespace {

thread_local int g_last_cuda_error = 0;

rlx_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return RLX_OK;
    g_last_cuda_error = static_cast<int>(e);
    return RLX_ERR_CUDA;
}

}  // namespace

void rlx::record_cuda_error(cudaError_t e) { g_last_cuda_error = static_cast<int>(e); }

namespace {

size_t elem_size(rlx_dtype d) { return d == RLX_BF16 ? 2 : 4; }

bool dtype_ok(rlx_dtype d) { return d == RLX_F32 || d == RLX_BF16; }

bool wire_ok(rlx_wire w) { return w == RLX_WIRE_NATIVE || w == RLX_WIRE_FP8_E4M3; }
bool ranks_ok(int n) { return n >= 1 && n <= RLX_MAX_RANKS; }

bool mul(size_t a, size_t b, size_t *out) {
    if (a != 0 && b > SIZE_MAX / a) return false;
    *out = a * b;
    return true;
}

// Every kernel numbers its units of work with 32 bits; up to RLX_MAX_ELEMENTS
// elements per call (all ranks together) the largest unit count stays far
// below 2^32.  No B200 holds more.
bool size_ok(size_t rows, size_t n) {
    size_t total = 0;
    return mul(rows, n, &total) && total <= RLX_MAX_ELEMENTS;
}
// Bytes spanned by `rows` rows of `len` elements at pitch `stride` elements.
bool extent(size_t rows, size_t stride, size_t len, size_t esize, size_t *bytes) {
    size_t a, b;
    if (rows == 0 || len == 0) { *bytes = 0; return true; }
    if (!mul(rows - 1, stride, &a)) return false;
    if (a > SIZE_MAX - len) return false;
    return mul(a + len, esize, &b) && (*bytes = b, true);
}

bool overlap(const void *a, size_t an, const void *b, size_t bn) {
    if (an == 0 || bn == 0) return false;
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + bn && pb < pa + an;
}

bool aligned(const void *p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

// May the vectorised kernels run?  Native-wire kernels move 16-byte vectors,
// FP8-wire kernels move groups of 4 elements; every row start and chunk
// offset (`offsets` in elements) must keep that alignment.
bool vec_ok(rlx_wire wire, size_t esize, std::initializer_list<const void *> ptrs,
            std::initializer_list<size_t> offsets) {
    const size_t bytes = wire == RLX_WIRE_NATIVE ? 16 : 4 * esize;
    const size_t elems = bytes / esize;
    for (const void *p : ptrs)
        if (!aligned(p, bytes)) return false;
    for (size_t o : offsets)
        if (o % elems != 0) return false;
    return true;
}

size_t tree_chunk(size_t count, int nranks) {
    const size_t blocks = (count + RLX_BLOCK - 1) / RLX_BLOCK;
    return (blocks + static_cast<size_t>(nranks) - 1) / static_cast<size_t>(nranks) * RLX_BLOCK;
}

size_t tree_ws_bytes(size_t count) {
    const size_t nblk = (count + RLX_BLOCK - 1) / RLX_BLOCK;
    const size_t raw = nblk * RLX_BLOCK + nblk * sizeof(float);
    return (raw + 255) / 256 * 256;
}

}  // namespace

extern "C" {

const char *rlx_status_string(rlx_status s) {
    switch (s) {
    case RLX_OK: return "success";
    case RLX_ERR_INVALID_ARG: return "invalid argument";
    case RLX_ERR_ALIGNMENT: return "pointer not aligned to its element type";
    case RLX_ERR_UNSUPPORTED: return "unsupported reduction op";
    case RLX_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case RLX_ERR_CUDA: return "CUDA error";
    case RLX_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

int rlx_last_cuda_error(void) { return g_last_cuda_error; }

size_t rlx_workspace_bytes(rlx_coll coll, size_t count, int nranks, rlx_dtype dtype,
                           rlx_wire wire) {
    (void)dtype;
    if (nranks <= 1 || count == 0) return 0;
    if (coll == RLX_COLL_ALLREDUCE_TREE && wire == RLX_WIRE_FP8_E4M3) return tree_ws_bytes(count);
    if (coll == RLX_COLL_ALLREDUCE_TREE_FUSED)
        return RLX_TREE_SYNC_BYTES + (wire == RLX_WIRE_FP8_E4M3 ? tree_ws_bytes(count) : 0);
    return 0;
}

rlx_status rlx_quantize_fp8(const void *x, rlx_dtype dtype, size_t rows, size_t n,
                            size_t stride, uint8_t *codes, float *scales, void *stream) {
    if (!dtype_ok(dtype) || stride < n) return RLX_ERR_INVALID_ARG;
    if (rows == 0 || n == 0) return RLX_OK;
    if (!x || !codes || !scales || !size_ok(rows, n)) return RLX_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    size_t xb, cb, sb, nbr = (n + RLX_BLOCK - 1) / RLX_BLOCK;
    if (!extent(rows, stride, n, es, &xb) || !extent(rows, stride, n, 1, &cb) ||
        !mul(rows, nbr, &sb) || !mul(sb, sizeof(float), &sb))
        return RLX_ERR_INVALID_ARG;
    if (!aligned(x, es) || !aligned(scales, 4)) return RLX_ERR_ALIGNMENT;
    if (overlap(x, xb, codes, cb) || overlap(x, xb, scales, sb) || overlap(codes, cb, scales, sb))
        return RLX_ERR_INVALID_ARG;
    const bool vec = aligned(x, 4 * es) && aligned(codes, 4) && stride % 4 == 0;
    return from_cuda(rlx::launch_quantize(x, dtype, rows, n, stride, codes, scales, vec,
                                          static_cast<cudaStream_t>(stream)));
}

rlx_status rlx_dequantize_fp8(const uint8_t *codes, const float *scales, size_t rows,
                              size_t n, size_t stride, void *y, rlx_dtype dtype,
                              void *stream) {
    if (!dtype_ok(dtype) || stride < n) return RLX_ERR_INVALID_ARG;
    if (rows == 0 || n == 0) return RLX_OK;
    if (!y || !codes || !scales || !size_ok(rows, n)) return RLX_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    size_t yb, cb, sb, nbr = (n + RLX_BLOCK - 1) / RLX_BLOCK;
    if (!extent(rows, stride, n, es, &yb) || !extent(rows, stride, n, 1, &cb) ||
        !mul(rows, nbr, &sb) || !mul(sb, sizeof(float), &sb))
        return RLX_ERR_INVALID_ARG;
    if (!aligned(y, es) || !aligned(scales, 4)) return RLX_ERR_ALIGNMENT;
    if (overlap(y, yb, codes, cb) || overlap(y, yb, scales, sb)) return RLX_ERR_INVALID_ARG;
    const bool vec = aligned(y, 4 * es) && aligned(codes, 4) && stride % 4 == 0;
    return from_cuda(rlx::launch_dequantize(codes, scales, rows, n, stride, y, dtype, vec,
                                            static_cast<cudaStream_t>(stream)));
}

// Checks shared by both allreduce algorithms; fills *bytes with the extent of
// one [nranks][stride] buffer.
static rlx_status check_allreduce(const void *send, void *recv, size_t count, size_t stride,
                                  int nranks, rlx_dtype dtype, rlx_wire wire, rlx_op op,
                                  size_t *bytes) {
    if (!dtype_ok(dtype) || !wire_ok(wire) || !ranks_ok(nranks) || stride < count)
        return RLX_ERR_INVALID_ARG;
    if (op != RLX_SUM) return RLX_ERR_UNSUPPORTED;
    if (count == 0) { *bytes = 0; return RLX_OK; }
    if (!send || !recv || !size_ok(static_cast<size_t>(nranks), count)) return RLX_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    if (!extent(static_cast<size_t>(nranks), stride, count, es, bytes)) return RLX_ERR_INVALID_ARG;
    if (!aligned(send, es) || !aligned(recv, es)) return RLX_ERR_ALIGNMENT;
    if (send != recv && overlap(send, *bytes, recv, *bytes)) return RLX_ERR_INVALID_ARG;
    return RLX_OK;
}

rlx_status rlx_allreduce_flat(const void *send, void *recv, size_t count, size_t stride,
                              int nranks, rlx_dtype dtype, rlx_wire wire, rlx_op op,
                              void *stream) {
    size_t bytes = 0;
    rlx_status st = check_allreduce(send, recv, count, stride, nranks, dtype, wire, op, &bytes);
    if (st != RLX_OK || count == 0) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t es = elem_size(dtype);
    if (nranks == 1) {
        if (send == recv) return RLX_OK;
        return from_cuda(rlx::launch_copy(send, recv, count, dtype,
                                          vec_ok(RLX_WIRE_NATIVE, es, {send, recv}, {}), s));
    }
    const bool vec = vec_ok(wire, es, {send, recv}, {stride});
    return from_cuda(rlx::launch_allreduce_flat(send, recv, count, stride, nranks, dtype, wire,
                                                vec, s));
}

rlx_status rlx_allreduce_tree(const void *send, void *recv, size_t count, size_t stride,
                              int nranks, rlx_dtype dtype, rlx_wire wire, rlx_op op,
                              void *workspace, size_t workspace_bytes, void *stream) {
    size_t bytes = 0;
    rlx_status st = check_allreduce(send, recv, count, stride, nranks, dtype, wire, op, &bytes);
    if (st != RLX_OK || count == 0) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t es = elem_size(dtype);
    if (nranks == 1) {
        if (send == recv) return RLX_OK;
        return from_cuda(rlx::launch_copy(send, recv, count, dtype,
                                          vec_ok(RLX_WIRE_NATIVE, es, {send, recv}, {}), s));
    }
    const size_t chunk = tree_chunk(count, nranks);
    uint8_t *ws_codes = nullptr;
    float *ws_scales = nullptr;
    if (wire == RLX_WIRE_FP8_E4M3) {
        const size_t need = tree_ws_bytes(count);
        if (!workspace || workspace_bytes < need || !aligned(workspace, 16))
            return RLX_ERR_WORKSPACE;
        if (overlap(workspace, need, send, bytes) || overlap(workspace, need, recv, bytes))
            return RLX_ERR_WORKSPACE;
        const size_t nblk = (count + RLX_BLOCK - 1) / RLX_BLOCK;
        ws_codes = static_cast<uint8_t *>(workspace);
        ws_scales = reinterpret_cast<float *>(ws_codes + nblk * RLX_BLOCK);
    }
    const bool vec = vec_ok(wire, es, {send, recv}, {stride});
    // small messages: both passes in one launch over thread-block clusters
    if (rlx::tree_cluster_wanted(count, nranks, chunk, dtype, wire))
        return from_cuda(rlx::launch_tree_cluster(send, recv, count, stride, nranks, chunk, dtype,
                                                  wire, ws_codes, ws_scales, vec, s));
    cudaError_t e = rlx::launch_tree_reduce(send, recv, count, stride, nranks, chunk, dtype, wire,
                                            ws_codes, ws_scales, vec, s);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(rlx::launch_tree_gather(recv, count, stride, nranks, chunk, dtype, wire,
                                             ws_codes, ws_scales, vec, s));
}

rlx_status rlx_allreduce_tree_fused(const void *send, void *recv, size_t count, size_t stride,
                                    int nranks, rlx_dtype dtype, rlx_wire wire, rlx_op op,
                                    void *workspace, size_t workspace_bytes, int *status,
                                    uint64_t wait_limit_ns, void *stream) {
    size_t bytes = 0;
    rlx_status st = check_allreduce(send, recv, count, stride, nranks, dtype, wire, op, &bytes);
    if (st != RLX_OK) return st;
    if (status != nullptr && !aligned(status, alignof(int))) return RLX_ERR_ALIGNMENT;
    if (status != nullptr && (overlap(status, sizeof(int), send, bytes) ||
                              overlap(status, sizeof(int), recv, bytes)))
        return RLX_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t es = elem_size(dtype);
    if (count == 0 || nranks == 1) {
        // nothing waits: the status is RLX_OK as soon as the copy (if any) is queued
        if (count != 0 && send != recv) {
            const cudaError_t e = rlx::launch_copy(send, recv, count, dtype,
                                                   vec_ok(RLX_WIRE_NATIVE, es, {send, recv}, {}), s);
            if (e != cudaSuccess) return from_cuda(e);
        }
        return status != nullptr ? from_cuda(cudaMemsetAsync(status, 0, sizeof(int), s)) : RLX_OK;
    }
    const size_t need = rlx_workspace_bytes(RLX_COLL_ALLREDUCE_TREE_FUSED, count, nranks, dtype, wire);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return RLX_ERR_WORKSPACE;
    if (overlap(workspace, need, send, bytes) || overlap(workspace, need, recv, bytes) ||
        (status != nullptr && overlap(workspace, need, status, sizeof(int))))
        return RLX_ERR_WORKSPACE;
    const bool vec = vec_ok(wire, es, {send, recv}, {stride});
    const uint64_t limit = wait_limit_ns != 0 ? wait_limit_ns : RLX_DEFAULT_WAIT_NS;
    return from_cuda(rlx::launch_tree_fused(send, recv, count, stride, nranks,
                                            tree_chunk(count, nranks), dtype, wire, workspace,
                                            status, limit, vec, s));
}

// Shared checks of the three chunked collectives.
static rlx_status check_chunked(const void *send, size_t sstride, size_t slen, void *recv,
                                size_t rstride, size_t rlen, size_t m, int nranks,
                                rlx_dtype dtype, rlx_wire wire) {
    if (!dtype_ok(dtype) || !wire_ok(wire) || !ranks_ok(nranks)) return RLX_ERR_INVALID_ARG;
    if (m == 0) return RLX_OK;
    size_t sb, rb;
    const size_t es = elem_size(dtype);
    if (slen == 0 || rlen == 0 || sstride < slen || rstride < rlen)
        return RLX_ERR_INVALID_ARG;
    if (!size_ok(static_cast<size_t>(nranks), slen > rlen ? slen : rlen)) return RLX_ERR_INVALID_ARG;
    if (!send || !recv) return RLX_ERR_INVALID_ARG;
    if (!extent(static_cast<size_t>(nranks), sstride, slen, es, &sb) ||
        !extent(static_cast<size_t>(nranks), rstride, rlen, es, &rb))
        return RLX_ERR_INVALID_ARG;
    if (!aligned(send, es) || !aligned(recv, es)) return RLX_ERR_ALIGNMENT;
    if (overlap(send, sb, recv, rb)) return RLX_ERR_INVALID_ARG;
    return RLX_OK;
}

static bool n_times_m(int nranks, size_t m, size_t *out) {
    return mul(static_cast<size_t>(nranks), m, out);
}

rlx_status rlx_reduce_scatter(const void *send, size_t send_stride, void *recv,
                              size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                              rlx_wire wire, rlx_op op, void *stream) {
    size_t nm = 0;
    if (ranks_ok(nranks) && !n_times_m(nranks, m, &nm)) return RLX_ERR_INVALID_ARG;
    rlx_status st = check_chunked(send, send_stride, nm, recv, recv_stride, m, m, nranks, dtype, wire);
    if (st != RLX_OK) return st;
    if (op != RLX_SUM) return RLX_ERR_UNSUPPORTED;
    if (m == 0) return RLX_OK;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t es = elem_size(dtype);
    if (nranks == 1)
        return from_cuda(rlx::launch_copy(send, recv, m, dtype,
                                          vec_ok(RLX_WIRE_NATIVE, es, {send, recv}, {}), s));
    const bool vec = vec_ok(wire, es, {send, recv}, {send_stride, recv_stride, m});
    return from_cuda(rlx::launch_reduce_scatter(send, send_stride, recv, recv_stride, m, nranks,
                                                dtype, wire, vec, s));
}

rlx_status rlx_all_gather(const void *send, size_t send_stride, void *recv,
                          size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                          rlx_wire wire, void *stream) {
    size_t nm = 0;
    if (ranks_ok(nranks) && !n_times_m(nranks, m, &nm)) return RLX_ERR_INVALID_ARG;
    rlx_status st = check_chunked(send, send_stride, m, recv, recv_stride, nm, m, nranks, dtype, wire);
    if (st != RLX_OK || m == 0) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t es = elem_size(dtype);
    if (nranks == 1)
        return from_cuda(rlx::launch_copy(send, recv, m, dtype,
                                          vec_ok(RLX_WIRE_NATIVE, es, {send, recv}, {}), s));
    const bool vec = vec_ok(wire, es, {send, recv}, {send_stride, recv_stride, m});
    return from_cuda(rlx::launch_all_gather(send, send_stride, recv, recv_stride, m, nranks,
                                            dtype, wire, vec, s));
}

rlx_status rlx_alltoall(const void *send, size_t send_stride, void *recv,
                        size_t recv_stride, size_t m, int nranks, rlx_dtype dtype,
                        rlx_wire wire, void *stream) {
    size_t nm = 0;
    if (ranks_ok(nranks) && !n_times_m(nranks, m, &nm)) return RLX_ERR_INVALID_ARG;
    rlx_status st = check_chunked(send, send_stride, nm, recv, recv_stride, nm, m, nranks, dtype, wire);
    if (st != RLX_OK || m == 0) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t es = elem_size(dtype);
    if (nranks == 1)
        return from_cuda(rlx::launch_copy(send, recv, m, dtype,
                                          vec_ok(RLX_WIRE_NATIVE, es, {send, recv}, {}), s));
    const bool vec = vec_ok(wire, es, {send, recv}, {send_stride, recv_stride, m});
    return from_cuda(rlx::launch_alltoall(send, send_stride, recv, recv_stride, m, nranks, dtype,
                                          wire, vec, s));
}

}  // extern "C"
