// rlx_tree_fused.cu -- the DDA-tree allreduce in one kernel launch.
//
// DDA-tree: a reduce-scatter phase (rank c reduces chunk c of every rank's
// buffer) followed by an all-gather phase (every rank fetches every reduced
// chunk), which the pages credit with near-constant latency for somewhat
// larger messages ("Meta open-sources RCCLX", infolabhq pt, "Direct Data
// Access (DDA) — De O(N) para O(1) de Latência"; RCCLX post, es, "Ataque
// directo a datos (DDA)").  rlx_allreduce_tree runs the two phases as two
// launches.  Here both run in one launch, and the all-gather of chunk c
// starts as soon as chunk c is reduced, as a rank of the real collective
// fetches a peer's chunk once the peer's ready flag is up:
//
//   * work queue: the kernel's work is cut into CTA-sized runs of units (the
//     unit bodies of the two-pass kernels, rlx_passes.cuh): tickets 0 .. R1-1
//     are reduce-scatter (pass 1) runs, R1 .. R1+R2-1 all-gather (pass 2)
//     runs, each in memory order (rlx_tree_plan.cuh), and a CTA takes its
//     next ticket from one atomic counter while its current run executes;
//   * chunk-ready counts: after a pass-1 run the CTA adds, with release
//     semantics, how many pass-1 units (native) or 128-blocks (FP8) of each
//     chunk it finished to that chunk's count;
//   * bounded waits: before a pass-2 unit touches chunk c, its warp waits,
//     with acquire loads, until chunk c's count reaches the chunk's total.
//     Every wait gives up after the caller's time limit (%globaltimer) or a
//     fixed number of polls, whichever comes first; the kernel then records
//     the failure, skips the work that depended on the wait, and returns.
//
// Why no CTA can wait forever: tickets are handed out in order, and only to
// CTAs that are running, and every pass-1 run has an earlier ticket than
// every pass-2 run; so a CTA holds a pass-2 ticket only after all pass-1
// work went to running CTAs.  Pass-1 work never waits, so every count a
// pass-2 warp waits for is eventually reached, however many CTAs are
// resident and in whatever order the hardware starts them.
//
// Exit: every CTA counts itself done; the last one clears the ticket, the
// counts and the error word (so the workspace is all zeros again, after a
// timeout too) and writes the call's status (RLX_OK or RLX_ERR_TIMEOUT) to
// the caller's status word.
#include <map>
#include <mutex>

#include "rlx_tree_plan.cuh"

namespace rlx {
namespace {

// The synchronisation words at the start of the workspace (see rlx.h).
struct TreeSync {
    uint32_t ticket;                  // next run to hand out
    uint32_t done;                    // CTAs that have finished
    uint32_t error;                   // nonzero: a wait ran out
    uint32_t reserved;
    uint32_t ready[RLX_MAX_RANKS];    // per chunk: pass-1 work finished
};
static_assert(sizeof(TreeSync) <= RLX_TREE_SYNC_BYTES, "sync words exceed their area");

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_add(uint32_t *p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_acq_rel_add(uint32_t *p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                 : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Polls between two reads of the clock, and the sleep between polls.  The
// poll count bounds a wait even if the clock did not advance.
constexpr uint32_t kPollNs = 64;
constexpr uint64_t kMinPollsPerNs = 32;   // polls allowed: limit_ns / 32 + 64

// A chunk is ready when its count, read as a signed 32-bit number, reaches
// its target (targets are below 2^31): a count that starts negative, e.g.
// INT_MIN, can never get there, which is how a test makes a wait run out.
__device__ __forceinline__ bool chunk_ready(const uint32_t *count, uint32_t target) {
    return static_cast<int32_t>(ld_acquire(count)) >= static_cast<int32_t>(target);
}

// Waits (one lane) until chunk c is ready.  Returns false if the wait ran
// out, or if another wait of this call already ran out (then no time is
// spent waiting here); the failure is recorded in sync->error.
__device__ __noinline__ bool wait_chunk(TreeSync *sync, uint32_t c, uint32_t target,
                                        uint64_t limit_ns) {
    if (chunk_ready(&sync->ready[c], target)) return true;
    const uint64_t t0 = global_ns();
    const uint64_t max_polls = limit_ns / kMinPollsPerNs + 64;
    for (uint64_t poll = 0;; ++poll) {
        if (*reinterpret_cast<volatile uint32_t *>(&sync->error) != 0) return false;
        __nanosleep(kPollNs);
        if (chunk_ready(&sync->ready[c], target)) return true;
        if (poll >= max_polls || global_ns() - t0 > limit_ns) {
            atomicOr(&sync->error, 1u);
            return false;
        }
    }
}

struct FusedArgs {
    const void *send;
    void *recv;
    size_t count, stride, chunk;
    uint8_t *ws_codes;
    float *ws_scales;
    TreeSync *sync;
    int *status;
    uint64_t limit_ns;
    TreePlan plan;
};

// CTAs per SM the kernel is compiled for (MINB, up to 8 ranks).  Both
// passes' unit bodies share its registers: at 2 CTAs per SM they are not
// spilled, at 4 the FP8 instantiations spill a little but twice the warps are
// in flight.  The launcher takes the 2-per-SM form when the runs fit in one
// wave of it (small messages, where the spills add latency: decode bf16 FP8
// from a graph 10.9 against 11.8 us) and the 4-per-SM form beyond (prefill
// bf16: native 205 -> 186 us, FP8 276 -> 244 us; fp32 FP8 at 8 x 16 Mi:
// 229 -> 205 us).
constexpr int kFusedMinbSmall = 2, kFusedMinbLarge = 4;

template <typename T, int NR, bool VEC, bool EXACT, bool FP8, int MINB>
__global__ void __launch_bounds__(kThreads, NR <= 8 ? MINB : 1)
tree_fused_kernel(FusedArgs a) {
    __shared__ uint32_t s_ticket[2];
    __shared__ uint32_t s_done[RLX_MAX_RANKS];
    pdl_begin();
    const int lane = lane_id();
    const uint32_t warp = threadIdx.x >> 5;
    const TreePlan &pl = a.plan;
    const uint32_t total = pl.runs1 + pl.runs2;
    uint32_t ready_mask = 0;   // chunks this warp has seen complete
    bool failed = false;
    if (threadIdx.x == 0) s_ticket[0] = atomicAdd(&a.sync->ticket, 1u);
    with_rank_count<NR, EXACT>(static_cast<int>(pl.n), [&](auto nn) {
        for (uint32_t round = 0;; ++round) {
            if (threadIdx.x < RLX_MAX_RANKS) s_done[threadIdx.x] = 0;
            __syncthreads();
            const uint32_t t = s_ticket[round & 1];
            if (t >= total) break;
            // the next ticket is fetched while this run executes, so the round
            // trip to the counter is off the critical path (a ticket is still
            // only handed to a running CTA, which finishes its current run
            // before it can wait on anything)
            if (threadIdx.x == 0) s_ticket[(round + 1) & 1] = atomicAdd(&a.sync->ticket, 1u);
            bool pass2;
            const uint32_t run = plan_resolve(pl, t, &pass2);   // same in every thread
            const uint32_t g = run * kRunUnits + warp;          // this warp's unit
            if (!pass2) {
                // ---- pass 1: reduce-scatter unit g
                if (g < pl.units1) {
                    if constexpr (!FP8) {
                        tree_reduce_native_unit<T, NR, VEC>(g, static_cast<const T *>(a.send),
                                                            static_cast<T *>(a.recv), a.count,
                                                            a.stride, nn, a.chunk, pl.per1);
                        if (lane == 0) atomicAdd(&s_done[fast_div(g, pl.per1)], 1u);
                    } else {
                        tree_reduce_fp8_unit<T, NR, VEC>(g, static_cast<const T *>(a.send), a.count,
                                                         a.stride, nn, a.ws_codes, a.ws_scales);
                        if (lane == 0) {
                            constexpr uint32_t B = kBpu<T>;
#pragma unroll
                            for (uint32_t j = 0; j < B; ++j) {
                                const uint32_t b = g * B + j;
                                if (b < pl.nblk) atomicAdd(&s_done[fast_div(b, pl.chunk_blocks)], 1u);
                            }
                        }
                    }
                }
                __syncthreads();
                // publish: the CTA's writes (ordered before this thread by the
                // barrier) become visible before the count does
                if (threadIdx.x < pl.n && s_done[threadIdx.x] != 0)
                    red_release_add(&a.sync->ready[threadIdx.x], s_done[threadIdx.x]);
            } else if (g < pl.units2 && !failed) {
                // ---- pass 2: all-gather unit g, once the chunks it reads are ready
                uint32_t c_lo, c_hi;
                plan_pass2_chunks(pl, g, &c_lo, &c_hi);
                // lane 0 waits (acquire); the warp barrier orders the other
                // lanes' reads of the chunk after it
                for (uint32_t c = c_lo; c <= c_hi && !failed; ++c) {
                    if (ready_mask & (1u << c)) continue;
                    int ok = 1;
                    if (lane == 0) ok = wait_chunk(a.sync, c, plan_chunk_target(pl, c), a.limit_ns);
                    if (__shfl_sync(kFull, ok, 0))
                        ready_mask |= 1u << c;
                    else
                        failed = true;
                }
                __syncwarp();
                if (!failed) {
                    if constexpr (!FP8)
                        tree_gather_native_unit<T, VEC>(g, static_cast<T *>(a.recv), a.count, a.stride,
                                                        static_cast<int>(pl.n), a.chunk, pl.per2);
                    else
                        tree_gather_fp8_unit<T, VEC>(g, static_cast<T *>(a.recv), a.count, a.stride,
                                                     static_cast<int>(pl.n), a.ws_codes, a.ws_scales);
                }
            }
            __syncthreads();   // s_done is rewritten next round, s_ticket[round & 1] the one after
        }
    });
    // ---- exit: the last CTA out clears the sync words and reports
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t before = atom_acq_rel_add(&a.sync->done, 1u);
        if (before == gridDim.x - 1) {
            const uint32_t err = *reinterpret_cast<volatile uint32_t *>(&a.sync->error);
            for (int c = 0; c < RLX_MAX_RANKS; ++c) a.sync->ready[c] = 0;
            a.sync->ticket = 0;
            a.sync->error = 0;
            a.sync->done = 0;
            if (a.status != nullptr) *a.status = err != 0 ? RLX_ERR_TIMEOUT : RLX_OK;
        }
    }
}

// Resident CTAs of `kernel` on the current device (cached per device).
int resident_ctas(const void *kernel) {
    static std::mutex mu;
    static std::map<std::pair<int, const void *>, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find({dev, kernel});
    if (it != cache.end()) return it->second;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess)
        return 0;
    const int n = sms * (per_sm > 0 ? per_sm : 1);
    cache[{dev, kernel}] = n;
    return n;
}

template <typename F>
cudaError_t dispatch_fused(rlx_dtype dtype, int n, bool vec, F &&f) {
#define RLX_FUSED_NR(T, NRV)                                                                  \
    if (n <= NRV) {                                                                           \
        if (n == NRV) return vec ? f.template operator()<T, NRV, true, true>()                \
                                 : f.template operator()<T, NRV, false, true>();              \
        return vec ? f.template operator()<T, NRV, true, false>()                             \
                   : f.template operator()<T, NRV, false, false>();                           \
    }
#define RLX_FUSED_T(T) RLX_FUSED_NR(T, 2) RLX_FUSED_NR(T, 4) RLX_FUSED_NR(T, 8) RLX_FUSED_NR(T, 16)
    if (dtype == RLX_F32) { RLX_FUSED_T(float) }
    else { RLX_FUSED_T(uint16_t) }
#undef RLX_FUSED_T
#undef RLX_FUSED_NR
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_tree_fused(const void *send, void *recv, size_t count, size_t stride,
                              int nranks, size_t chunk, rlx_dtype dtype, rlx_wire wire,
                              void *workspace, int *status, uint64_t limit_ns, bool vec,
                              cudaStream_t stream) {
    FusedArgs a = {};
    a.send = send;
    a.recv = recv;
    a.count = count;
    a.stride = stride;
    a.chunk = chunk;
    a.sync = static_cast<TreeSync *>(workspace);
    a.status = status;
    a.limit_ns = limit_ns;
    const bool fp8 = wire == RLX_WIRE_FP8_E4M3;
    if (fp8) {
        const size_t nblk = (count + kBlock - 1) / kBlock;
        a.ws_codes = static_cast<uint8_t *>(workspace) + RLX_TREE_SYNC_BYTES;
        a.ws_scales = reinterpret_cast<float *>(a.ws_codes + nblk * kBlock);
    }
    return dispatch_fused(dtype, nranks, vec, [&]<typename T, int NR, bool VEC, bool EX>() {
        if (!make_tree_plan<T>(count, nranks, chunk, fp8, &a.plan)) return cudaErrorInvalidValue;
        const size_t runs = static_cast<size_t>(a.plan.runs1) + a.plan.runs2;
        // the grid is at most one wave of resident CTAs of the form launched
        auto go = [&]<int MINB>() -> cudaError_t {
            auto *k = fp8 ? tree_fused_kernel<T, NR, VEC, EX, true, MINB>
                          : tree_fused_kernel<T, NR, VEC, EX, false, MINB>;
            const int resident = resident_ctas(reinterpret_cast<const void *>(k));
            if (resident <= 0) return cudaErrorInvalidValue;
            const dim3 grid(static_cast<unsigned>(runs < static_cast<size_t>(resident) ? runs : resident));
            return launch_kernel(k, grid, stream, a);
        };
        const int small = resident_ctas(reinterpret_cast<const void *>(
            fp8 ? tree_fused_kernel<T, NR, VEC, EX, true, kFusedMinbSmall>
                : tree_fused_kernel<T, NR, VEC, EX, false, kFusedMinbSmall>));
        if (small > 0 && runs <= static_cast<size_t>(small))
            return go.template operator()<kFusedMinbSmall>();
        return go.template operator()<kFusedMinbLarge>();
    });
}

}  // namespace rlx
