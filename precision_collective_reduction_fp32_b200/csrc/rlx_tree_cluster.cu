// rlx_tree_cluster.cu -- the DDA-tree in one launch over thread-block
// clusters, for the messages where the kernel boundary between the two
// passes is a large part of the call.
//
// The tree's two passes ("Meta open-sources RCCLX", infolabhq pt, section
// "Direct Data Access (DDA) — De O(N) para O(1) de Latência": a
// reduce-scatter phase, then an all-gather phase) depend on each other only
// element range by element range: the all-gather of a range reads what the
// reduce-scatter of the same range wrote (the owner row's chunk on the native
// wire, the requantised payload on the FP8 wire).  So the work is cut into
// groups of one all-gather unit and the reduce-scatter units that cover the
// same elements, and each cluster of kClusterCtas CTAs takes the groups of
// one contiguous range: its warps run the reduce-scatter units, the cluster
// barrier (arrive with release, wait with acquire semantics at cluster scope)
// makes their writes visible inside the cluster, and then its warps run the
// all-gather units, which read through L2.  No CTA waits on another cluster,
// so there is no flag, ticket or spin-wait: a cluster's CTAs are scheduled
// together, and every thread of every CTA reaches the one barrier exactly
// once.  Results are those of the two-launch tree bit for bit: the same unit
// bodies write the same bytes.
#include <cooperative_groups.h>

#include "rlx_internal.h"
#include "rlx_passes.cuh"

namespace rlx {
namespace {

namespace cg = cooperative_groups;

// CTAs per cluster (measured from a CUDA graph, decode bf16 tree native /
// FP8: 2 CTAs 3.2 / 4.9 us, 4 CTAs 3.4 / 5.3 us, 8 CTAs 3.7 / 5.9 us).
#ifndef RLX_TREE_CLUSTER_CTAS
#define RLX_TREE_CLUSTER_CTAS 2
#endif
constexpr uint32_t kClusterCtas = RLX_TREE_CLUSTER_CTAS;
constexpr uint32_t kClusterWarps = kClusterCtas * kWarpsPerCta;
static_assert(kJd % kBpu<float> == 0 && kJd % kBpu<uint16_t> == 0,
              "an FP8 all-gather unit must cover whole reduce-scatter units");

struct ClusterArgs {
    const void *send;
    void *recv;
    size_t count, stride, chunk;
    uint8_t *ws_codes;
    float *ws_scales;
    uint32_t groups;               // groups = all-gather units
    uint32_t units1;               // FP8: reduce-scatter units (unused on the native wire)
    uint32_t per_group;            // reduce-scatter units (and warps) per group
    uint32_t groups_per_cluster;   // kClusterWarps / per_group
    FastDiv per1, per2;            // native: units per chunk of the two passes
    int n;
};

template <typename T, int NR, bool VEC, bool EXACT, bool FP8>
__global__ void __launch_bounds__(kThreads, NR <= 8 ? 2 : 1)
tree_cluster_kernel(ClusterArgs a) {
    const cg::cluster_group cl = cg::this_cluster();
    pdl_begin();
    const uint32_t cluster = blockIdx.x / kClusterCtas;
    const uint32_t warp = cl.block_rank() * kWarpsPerCta + (threadIdx.x >> 5);
    const uint32_t g0 = cluster * a.groups_per_cluster;
    with_rank_count<NR, EXACT>(a.n, [&](auto nn) {
        // ---- reduce-scatter: warp w takes unit w % per_group of group w / per_group
        const uint32_t gi = warp / a.per_group, sub = warp - gi * a.per_group;
        const uint32_t q = g0 + gi;
        if (gi < a.groups_per_cluster && q < a.groups) {
            if constexpr (FP8) {
                const uint32_t u = q * a.per_group + sub;
                if (u < a.units1)
                    tree_reduce_fp8_unit<T, NR, VEC>(u, static_cast<const T *>(a.send), a.count,
                                                     a.stride, nn, a.ws_codes, a.ws_scales);
            } else {
                const uint32_t c = fast_div(q, a.per2), u2 = q - c * a.per2.d;
                const uint32_t u = u2 * a.per_group + sub;
                if (u < a.per1.d)
                    tree_reduce_native_unit<T, NR, VEC>(c * a.per1.d + u, static_cast<const T *>(a.send),
                                                        static_cast<T *>(a.recv), a.count, a.stride,
                                                        nn, a.chunk, a.per1);
            }
        }
    });
    // every thread of the cluster passes here once: the reduce-scatter writes
    // of the cluster are visible to all of its threads after it
    cl.sync();
    // ---- all-gather: the per_group warps of group w / per_group share its
    // rows (warp w takes rows w % per_group, w % per_group + per_group, ...)
    const uint32_t gj = warp / a.per_group, row0 = warp - gj * a.per_group;
    const uint32_t q2 = g0 + gj;
    if (gj < a.groups_per_cluster && q2 < a.groups) {
        if constexpr (FP8)
            tree_gather_fp8_unit<T, VEC>(q2, static_cast<T *>(a.recv), a.count, a.stride, a.n,
                                         a.ws_codes, a.ws_scales, static_cast<int>(row0),
                                         static_cast<int>(a.per_group));
        else
            tree_gather_native_unit<T, VEC>(q2, static_cast<T *>(a.recv), a.count, a.stride, a.n,
                                            a.chunk, a.per2, static_cast<int>(row0),
                                            static_cast<int>(a.per_group));
    }
}

template <typename F>
cudaError_t dispatch_cluster(rlx_dtype dtype, int n, bool vec, F &&f) {
#define RLX_CLUSTER_NR(T, NRV)                                                                \
    if (n <= NRV) {                                                                           \
        if (n == NRV) return vec ? f.template operator()<T, NRV, true, true>()                \
                                 : f.template operator()<T, NRV, false, true>();              \
        return vec ? f.template operator()<T, NRV, true, false>()                             \
                   : f.template operator()<T, NRV, false, false>();                           \
    }
#define RLX_CLUSTER_T(T) \
    RLX_CLUSTER_NR(T, 2) RLX_CLUSTER_NR(T, 4) RLX_CLUSTER_NR(T, 8) RLX_CLUSTER_NR(T, 16)
    if (dtype == RLX_F32) {
        RLX_CLUSTER_T(float)
    } else {
        RLX_CLUSTER_T(uint16_t)
    }
#undef RLX_CLUSTER_T
#undef RLX_CLUSTER_NR
    return cudaErrorInvalidValue;
}

cudaLaunchConfig_t cluster_config(dim3 grid, cudaStream_t stream, cudaLaunchAttribute (&attr)[2]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClusterCtas;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = RLX_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cfg;
}

}  // namespace

// Whether a call takes the cluster path: while its clusters fill at most a
// few waves of the GPU (2 CTAs per SM).  Measured against the two launches
// (from a CUDA graph, N = 8): decode bf16 [32, 8192] native 3.2 against
// 4.5 us, FP8 4.9 against 7.4 us; quick-start fp32 [10, 20] FP8 3.4 against
// 6.6 us; at 3.5 waves (2 Mi bf16 / 1 Mi fp32 per rank) native and fp32 FP8
// still gain ~1 us, bf16 FP8 loses 1.5 us (its issue-bound reduce-scatter
// runs at 4 CTAs per SM in its own kernel); from 4 Mi fp32 / 8 Mi bf16 per
// rank on, the two launches are faster on both wires.
bool tree_cluster_wanted(size_t count, int nranks, size_t chunk, rlx_dtype dtype, rlx_wire wire) {
    if (nranks < 2 || count == 0) return false;
    const bool bf16 = dtype == RLX_BF16;
    const bool fp8 = wire == RLX_WIRE_FP8_E4M3;
    size_t groups, per_group;
    if (fp8) {
        groups = tree_gather_fp8_units(count);
        per_group = kJd / (bf16 ? kBpu<uint16_t> : kBpu<float>);
    } else {
        const size_t per2 = bf16 ? tree_gather_native_per_chunk<uint16_t>(chunk)
                                 : tree_gather_native_per_chunk<float>(chunk);
        groups = per2 * static_cast<size_t>(nranks);
        per_group = kUnroll;
    }
    const size_t gpc = kClusterWarps / per_group;
    const size_t clusters = (groups + gpc - 1) / gpc;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return false;
    const size_t wave = static_cast<size_t>(sms) * 2 / kClusterCtas;   // clusters per wave
    return clusters <= wave * (fp8 && bf16 ? 1 : 4);
}

cudaError_t launch_tree_cluster(const void *send, void *recv, size_t count, size_t stride,
                                int nranks, size_t chunk, rlx_dtype dtype, rlx_wire wire,
                                uint8_t *ws_codes, float *ws_scales, bool vec,
                                cudaStream_t stream) {
    const bool fp8 = wire == RLX_WIRE_FP8_E4M3;
    return dispatch_cluster(dtype, nranks, vec, [&]<typename T, int NR, bool VEC, bool EX>() {
        ClusterArgs a = {};
        a.send = send;
        a.recv = recv;
        a.count = count;
        a.stride = stride;
        a.chunk = chunk;
        a.ws_codes = ws_codes;
        a.ws_scales = ws_scales;
        a.n = nranks;
        size_t groups, units1 = 0;
        if (fp8) {
            groups = tree_gather_fp8_units(count);
            units1 = ((count + kBlock - 1) / kBlock + kBpu<T> - 1) / kBpu<T>;
            a.per_group = kJd / kBpu<T>;
        } else {
            const size_t per1 = tree_reduce_native_per_chunk<T>(chunk);
            const size_t per2 = tree_gather_native_per_chunk<T>(chunk);
            if (per1 >= (size_t{1} << 31) || per2 >= (size_t{1} << 31)) return cudaErrorInvalidValue;
            a.per1 = make_fastdiv(static_cast<uint32_t>(per1));
            a.per2 = make_fastdiv(static_cast<uint32_t>(per2));
            groups = per2 * static_cast<size_t>(nranks);
            a.per_group = kUnroll;
        }
        if (groups >= (size_t{1} << 31) || units1 >= (size_t{1} << 31)) return cudaErrorInvalidValue;
        a.groups = static_cast<uint32_t>(groups);
        a.units1 = static_cast<uint32_t>(units1);
        a.groups_per_cluster = kClusterWarps / a.per_group;
        const size_t clusters = (groups + a.groups_per_cluster - 1) / a.groups_per_cluster;
        if (clusters * kClusterCtas >= (size_t{1} << 31)) return cudaErrorInvalidValue;
        cudaLaunchAttribute attr[2];
        cudaLaunchConfig_t cfg =
            cluster_config(dim3(static_cast<unsigned>(clusters * kClusterCtas)), stream, attr);
        auto *k = fp8 ? tree_cluster_kernel<T, NR, VEC, EX, true>
                      : tree_cluster_kernel<T, NR, VEC, EX, false>;
        return cudaLaunchKernelEx(&cfg, k, a);
    });
}

}  // namespace rlx
