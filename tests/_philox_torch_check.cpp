// Host-only cross-check: prints the four output words of torch's own
// Philox4x32-10 engine (ATen/core/PhiloxRNGEngine.h) for each input line
// "c0 c1 c2 c3 k0 k1".  torch keys the engine with (seed lo, seed hi) and
// sets the counter to (offset lo, offset hi, subsequence lo, subsequence hi).
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdint>
#include <cstdio>

int main() {
    unsigned long long c0, c1, c2, c3, k0, k1;
    while (std::scanf("%llu %llu %llu %llu %llu %llu", &c0, &c1, &c2, &c3, &k0, &k1) == 6) {
        uint64_t seed = (uint64_t)k0 | ((uint64_t)k1 << 32);
        uint64_t subseq = (uint64_t)c2 | ((uint64_t)c3 << 32);
        uint64_t offset = (uint64_t)c0 | ((uint64_t)c1 << 32);
        at::philox_engine e(seed, subseq, offset);
        uint32_t w0 = e(), w1 = e(), w2 = e(), w3 = e();
        std::printf("%08x %08x %08x %08x\n", w0, w1, w2, w3);
    }
    return 0;
}
