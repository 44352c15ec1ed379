// Host-only check of the one-launch DDA-tree's work plan (rlx_tree_plan.cuh),
// the same functions the kernel calls: for many shapes,
//   * the ticket order is a bijection onto the reduce-scatter (pass 1) and
//     all-gather (pass 2) runs;
//   * every all-gather run comes after every reduce-scatter run that works on
//     a chunk it reads (the order the kernel's no-deadlock argument needs:
//     the plan hands out all reduce-scatter runs first);
//   * each chunk's ready target equals the reduce-scatter work that reports
//     to it.
// The chunks a unit touches are recomputed here by plain division.
// Exit status 0 = all shapes pass.
#include <cstdint>
#include <cstdio>
#include <vector>

#include "../../precision_collective_reduction_fp32_b200/csrc/rlx_tree_plan.cuh"

template <typename T>
static int check(size_t count, int n, bool fp8) {
    using namespace rlx;
    const size_t nblk = (count + 127) / 128;
    const size_t chunk = 128 * ((nblk + n - 1) / n);          // the DDA-tree's chunk
    TreePlan p;
    if (!make_tree_plan<T>(count, n, chunk, fp8, &p)) return 0;
    const uint32_t total = p.runs1 + p.runs2;
    std::vector<int64_t> pos1(p.runs1, -1), pos2(p.runs2, -1);
    for (uint32_t t = 0; t < total; ++t) {
        bool pass2 = false;
        const uint32_t r = plan_resolve(p, t, &pass2);
        std::vector<int64_t> &pos = pass2 ? pos2 : pos1;
        if (r >= pos.size() || pos[r] != -1) {
            std::printf("not a bijection: count %zu n %d fp8 %d ticket %u\n", count, n, fp8, t);
            return 1;
        }
        pos[r] = t;
    }
    // latest ticket of reduce-scatter work per chunk, and the work per chunk
    std::vector<int64_t> last1(n, -1);
    std::vector<uint64_t> work(n, 0);
    const size_t per1 = fp8 ? 0 : tree_reduce_native_per_chunk<T>(chunk);
    const size_t bpc = chunk / 128;
    for (uint32_t u = 0; u < p.units1; ++u) {
        const int64_t t = pos1[u / kRunUnits];
        if (!fp8) {
            const size_t c = u / per1;
            last1[c] = last1[c] > t ? last1[c] : t;
            work[c] += 1;
        } else {
            for (size_t b = size_t{u} * kBpu<T>; b < size_t{u + 1} * kBpu<T> && b < nblk; ++b) {
                const size_t c = b / bpc;
                last1[c] = last1[c] > t ? last1[c] : t;
                work[c] += 1;
            }
        }
    }
    for (int c = 0; c < n; ++c)
        if (plan_chunk_target(p, c) != work[c]) {
            std::printf("target: count %zu n %d fp8 %d chunk %d: %u vs %llu\n", count, n, fp8, c,
                        plan_chunk_target(p, c), static_cast<unsigned long long>(work[c]));
            return 1;
        }
    const size_t per2 = fp8 ? 0 : tree_gather_native_per_chunk<T>(chunk);
    for (uint32_t g = 0; g < p.units2; ++g) {
        const int64_t t = pos2[g / kRunUnits];
        size_t c_lo, c_hi;
        if (!fp8) {
            c_lo = c_hi = g / per2;
        } else {
            c_lo = (size_t{g} * kJd) / bpc;
            const size_t b1 = size_t{g + 1} * kJd < nblk ? size_t{g + 1} * kJd : nblk;
            c_hi = (b1 - 1) / bpc;
        }
        uint32_t k_lo, k_hi;
        plan_pass2_chunks(p, g, &k_lo, &k_hi);
        if (k_lo != c_lo || k_hi != c_hi) {
            std::printf("pass-2 chunks: count %zu n %d fp8 %d unit %u\n", count, n, fp8, g);
            return 1;
        }
        for (size_t c = c_lo; c <= c_hi; ++c)
            if (last1[c] >= t) {
                std::printf("order: count %zu n %d fp8 %d: all-gather unit %u (ticket %lld) before "
                            "reduce-scatter of chunk %zu (ticket %lld)\n", count, n, fp8, g,
                            static_cast<long long>(t), c, static_cast<long long>(last1[c]));
                return 1;
            }
    }
    return 0;
}

int main() {
    const size_t counts[] = {1, 7, 127, 128, 129, 200, 1000, 1003, 2000, 3077, 4096, 65540, 131075,
                             262144, 600003, size_t{1} << 20, (size_t{3} << 20) + 5};
    const int ranks[] = {2, 3, 4, 5, 7, 8, 16};
    int bad = 0, shapes = 0;
    for (size_t c : counts)
        for (int n : ranks)
            for (int fp8 = 0; fp8 < 2; ++fp8) {
                bad |= check<float>(c, n, fp8);
                bad |= check<uint16_t>(c, n, fp8);
                shapes += 2;
            }
    std::printf(bad ? "FAIL\n" : "ok: %d shapes\n", shapes);
    return bad;
}
