// rlx_tree_plan.cuh -- the work plan of the one-launch DDA-tree
// (rlx_tree_fused.cu): how its reduce-scatter (pass 1) and all-gather
// (pass 2) units are grouped into runs, what each chunk's ready count must
// reach, and the order in which runs are handed out as tickets.  Host and
// device share these functions: the launcher builds the plan, the kernel
// follows it, and a host-only test checks the ticket order.
#pragma once

#include "rlx_passes.cuh"

namespace rlx {

// Units per run: one per warp of the 256-thread CTA.
constexpr uint32_t kRunUnits = kWarpsPerCta;

struct TreePlan {
    uint32_t n;                   // ranks = chunks
    bool fp8;                     // FP8 wire
    uint32_t runs1, runs2;        // pass-1 / pass-2 runs
    uint32_t units1, units2;      // pass-1 / pass-2 units
    FastDiv per1, per2;           // native: pass-1 / pass-2 units per chunk
    uint32_t bpu;                 // FP8: 128-blocks per pass-1 unit
    uint32_t blocks_per_chunk;    // FP8: 128-blocks per chunk
    FastDiv chunk_blocks;         // FP8: division by blocks_per_chunk
    uint32_t nblk;                // FP8: 128-blocks in count
    uint32_t jd;                  // FP8: 128-blocks per pass-2 unit
};

// Total pass-1 work of chunk c: native units, or 128-blocks on the FP8 wire.
__host__ __device__ inline uint32_t plan_chunk_target(const TreePlan &p, uint32_t c) {
    if (!p.fp8) return p.per1.d;
    const uint32_t lo = c * p.blocks_per_chunk;
    if (lo >= p.nblk) return 0;
    const uint32_t rem = p.nblk - lo;
    return rem < p.blocks_per_chunk ? rem : p.blocks_per_chunk;
}

// The first and last chunk pass-2 unit g reads.
__host__ __device__ inline void plan_pass2_chunks(const TreePlan &p, uint32_t g, uint32_t *c_lo,
                                                  uint32_t *c_hi) {
    if (!p.fp8) {
        *c_lo = *c_hi = fast_div(g, p.per2);
        return;
    }
    const uint32_t b0 = g * p.jd;
    uint32_t b1 = b0 + p.jd;
    if (b1 > p.nblk) b1 = p.nblk;
    *c_lo = fast_div(b0, p.chunk_blocks);
    *c_hi = fast_div(b1 - 1, p.chunk_blocks);
}

// Ticket t -> (pass 2?, run): every reduce-scatter run first, in memory
// order, then every all-gather run.  (Interleaving them -- each all-gather
// run right after the reduce-scatter work of the chunks it reads -- was
// built and measured: no gain on one-wave messages, and the per-run search
// for a ticket's run made many-wave messages slower.)
__host__ __device__ inline uint32_t plan_resolve(const TreePlan &p, uint32_t t, bool *pass2) {
    *pass2 = t >= p.runs1;
    return *pass2 ? t - p.runs1 : t;
}

// The plan for a DDA-tree on `count` elements per rank of T, `nranks` ranks,
// chunks of `chunk` elements (a multiple of 128), built from the unit counts
// of the two-pass kernels' unit bodies.  false if a count does not fit the
// 32-bit indices.
template <typename T>
inline bool make_tree_plan(size_t count, int nranks, size_t chunk, bool fp8, TreePlan *p) {
    *p = TreePlan{};
    p->n = static_cast<uint32_t>(nranks);
    p->fp8 = fp8;
    const size_t nblk = (count + kBlock - 1) / kBlock;
    size_t units1, units2;
    if (!fp8) {
        const size_t per1 = tree_reduce_native_per_chunk<T>(chunk);
        const size_t per2 = tree_gather_native_per_chunk<T>(chunk);
        units1 = per1 * static_cast<size_t>(nranks);
        units2 = per2 * static_cast<size_t>(nranks);
        if (units1 >= (size_t{1} << 31) || units2 >= (size_t{1} << 31)) return false;
        p->per1 = make_fastdiv(static_cast<uint32_t>(per1));
        p->per2 = make_fastdiv(static_cast<uint32_t>(per2));
    } else {
        if (nblk >= (size_t{1} << 31)) return false;
        p->bpu = kBpu<T>;
        p->jd = kJd;
        units1 = (nblk + kBpu<T> - 1) / kBpu<T>;
        units2 = tree_gather_fp8_units(count);
        p->blocks_per_chunk = static_cast<uint32_t>(chunk / kBlock);
        p->chunk_blocks = make_fastdiv(p->blocks_per_chunk);
        p->nblk = static_cast<uint32_t>(nblk);
    }
    p->units1 = static_cast<uint32_t>(units1);
    p->units2 = static_cast<uint32_t>(units2);
    p->runs1 = static_cast<uint32_t>((units1 + kRunUnits - 1) / kRunUnits);
    p->runs2 = static_cast<uint32_t>((units2 + kRunUnits - 1) / kRunUnits);
    return true;
}

}  // namespace rlx
