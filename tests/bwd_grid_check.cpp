// Host-only check of fa::bwd_key_tile_fastest (csrc/bwd_grid.h), the backward's choice of
// grid order: compiled and run by tests/test_bwd_grid.py. Prints "ok" and exits 0 when every
// check holds; otherwise prints the failed check and exits 1.
#include <cstdio>

#include "bwd_grid.h"

static int failures = 0;
#define CHECK(cond)                                              \
    do {                                                         \
        if (!(cond)) {                                           \
            std::printf("FAILED line %d: %s\n", __LINE__, #cond); \
            ++failures;                                          \
        }                                                        \
    } while (0)

int main() {
    using fa::bwd_key_tile_fastest;
    const int sms = 148;
    const long long waves12 = 12LL * sms;  // 1776 CTAs
    // one query head per KV head, causal, d = 128: key tile fastest from 12 waves on
    CHECK(bwd_key_tile_fastest(true, 128, 32, 32, 0, 4096, sms));   // B=2 N=8192 H=32
    CHECK(bwd_key_tile_fastest(true, 128, 32, 32, 0, 2048, sms));   // B=1 N=8192, B=2 N=4096
    CHECK(!bwd_key_tile_fastest(true, 128, 32, 32, 0, 1024, sms));  // B=1 N=4096
    CHECK(!bwd_key_tile_fastest(true, 128, 32, 32, 0, 512, sms));   // B=1 N=2048
    CHECK(bwd_key_tile_fastest(true, 128, 8, 8, 0, waves12, sms));  // exactly 12 waves
    CHECK(!bwd_key_tile_fastest(true, 128, 8, 8, 0, waves12 - 1, sms));
    // the threshold follows the SM count
    CHECK(bwd_key_tile_fastest(true, 128, 32, 32, 0, 1200, 100));
    CHECK(!bwd_key_tile_fastest(true, 128, 32, 32, 0, 1199, 100));
    // grouped heads, anchors, d = 64 and no mask keep the other order
    CHECK(!bwd_key_tile_fastest(true, 128, 32, 8, 0, 1 << 20, sms));
    CHECK(!bwd_key_tile_fastest(true, 128, 32, 32, 4, 1 << 20, sms));
    CHECK(!bwd_key_tile_fastest(true, 64, 32, 32, 0, 1 << 20, sms));
    CHECK(!bwd_key_tile_fastest(false, 128, 32, 32, 0, 1 << 20, sms));
    if (failures) return 1;
    std::printf("ok\n");
    return 0;
}
