// Host-only driver for the mask helper every attention kernel uses
// (visible_keys in fa_internal.h): prints, for a grid of cases, the first and
// last visible key the helper reports.  Built and run on the CPU by
// test_mask_helper.py, which checks each line against enumeration.
#include <cstdio>

#include "fa_internal.h"

int main() {
    const int windows[][2] = {{-1, -1}, {0, 0}, {1, -1}, {3, 2}, {-1, 0}, {-1, 4}, {5, -1}, {0, 3}};
    for (int s_q = 1; s_q <= 7; ++s_q)
        for (int n = 0; n <= 9; ++n)
            for (int causal = 0; causal <= 1; ++causal)
                for (const auto &w : windows)
                    for (int i = 0; i < s_q; ++i) {
                        int64_t first, last;
                        fa::visible_keys(i, n, s_q, causal, w[0], w[1], first, last);
                        std::printf("%d %d %d %d %d %d %lld %lld\n", i, n, s_q, causal, w[0], w[1],
                                    (long long)first, (long long)last);
                    }
    return 0;
}
