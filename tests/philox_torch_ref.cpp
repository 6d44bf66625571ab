// Independent Philox4x32-10 for pinning the oracle: PyTorch's header-only
// at::Philox4_32 engine (ATen/core/PhiloxRNGEngine.h), compiled on the host.
// Reads lines "seed subsequence offset" and prints the four 32-bit words of
// one 128-bit output: key = seed, counter = (offset lo, offset hi,
// subsequence lo, subsequence hi).
#include <ATen/core/PhiloxRNGEngine.h>

#include <cstdio>

int main() {
    unsigned long long seed, sub, off;
    while (std::scanf("%llu %llu %llu", &seed, &sub, &off) == 3) {
        at::Philox4_32 engine(seed, sub, off);
        unsigned w0 = engine(), w1 = engine(), w2 = engine(), w3 = engine();
        std::printf("%u %u %u %u\n", w0, w1, w2, w3);
    }
    return 0;
}
