// Host-only check of the multiply-shift divider the kernels use to split a
// unit index into (segment, offset): compares fast_div with the C++ `/`
// for every divisor up to 2^12 against a spread of numerators, and for
// random and edge divisors up to 2^32 - 1.  Exit status 0 = all agree.
#include <cstdint>
#include <cstdio>
#include <random>

#include "../../precision_collective_reduction_fp32_b200/csrc/rlx_device.cuh"

static int check(uint32_t d, uint32_t n) {
    const rlx::FastDiv f = rlx::make_fastdiv(d);
    const uint32_t q = rlx::fast_div(n, f);
    if (q != n / d) {
        std::printf("mismatch: %u / %u = %u, fast_div gave %u\n", n, d, n / d, q);
        return 1;
    }
    return 0;
}

int main() {
    std::mt19937_64 rng(12345);
    const uint32_t edges[] = {0u, 1u, 2u, 3u, 0x7fffffffu, 0x80000000u, 0xfffffffeu, 0xffffffffu};
    int bad = 0;
    for (uint32_t d = 1; d <= 4096 && !bad; ++d) {
        for (uint32_t e : edges) bad |= check(d, e);
        for (uint32_t k = 1; k < 64 && !bad; ++k) {          // around multiples of d
            const uint64_t base = static_cast<uint64_t>(d) * (rng() % (0xffffffffull / d + 1));
            for (int64_t o = -2; o <= 2; ++o) {
                const int64_t nn = static_cast<int64_t>(base) + o;
                if (nn >= 0 && nn <= 0xffffffffll) bad |= check(d, static_cast<uint32_t>(nn));
            }
        }
        for (int k = 0; k < 256 && !bad; ++k) bad |= check(d, static_cast<uint32_t>(rng()));
    }
    for (int t = 0; t < 200000 && !bad; ++t) {
        const int bits = 1 + static_cast<int>(rng() % 32);
        uint32_t d = static_cast<uint32_t>(rng() >> (64 - bits));
        if (d == 0) d = 1;
        bad |= check(d, static_cast<uint32_t>(rng()));
        bad |= check(d, 0xffffffffu);
        bad |= check(d, d - 1);
        bad |= check(d, d);
    }
    for (uint32_t e : edges)
        for (uint32_t e2 : edges)
            if (e) bad |= check(e, e2);
    std::printf(bad ? "FAIL\n" : "ok\n");
    return bad;
}
