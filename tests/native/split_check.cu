// Host-side check of the stream-K split-K bookkeeping of the decode-attention
// kernels (nvfp4kv_attention_common.cuh) against brute force: the CTA ranges,
// the owner of a tile, the contributor count of a unit, the partial slot a
// contributor writes and the slot the merge reads, and the unit lookup.
// Compiled by nvcc and run on the CPU; prints "ok" and exits 0 when every
// case agrees.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../../bit_decode_attention_b200/csrc/nvfp4kv_attention_common.cuh"

using namespace nvfp4kv::attn;

static int failures = 0;
#define CHECK(cond, ...)                                   \
    do {                                                   \
        if (!(cond)) {                                     \
            if (failures < 20) std::printf(__VA_ARGS__);   \
            ++failures;                                    \
        }                                                  \
    } while (0)

// every way of cutting T tiles into units of the given lengths, checked for N CTAs
static void check_split(int64_t T, int64_t N, const std::vector<int64_t>& unit_len) {
    // ranges partition [0, T) in order
    CHECK(range_start(0, T, N) == 0, "range_start(0) T=%lld N=%lld\n", (long long)T, (long long)N);
    CHECK(range_start(N, T, N) == T, "range_start(N) T=%lld N=%lld\n", (long long)T, (long long)N);
    std::vector<int64_t> owner(T);
    for (int64_t c = 0; c < N; ++c) {
        const int64_t a = range_start(c, T, N), b = range_start(c + 1, T, N);
        CHECK(a <= b, "ranges out of order c=%lld\n", (long long)c);
        CHECK(a == c * T / N, "range_start closed form c=%lld T=%lld N=%lld\n", (long long)c,
              (long long)T, (long long)N);
        for (int64_t t = a; t < b; ++t) owner[t] = c;
    }
    for (int64_t t = 0; t < T; ++t)
        CHECK(cta_of(t, T, N) == owner[t], "cta_of(%lld) T=%lld N=%lld: %lld, owner %lld\n",
              (long long)t, (long long)T, (long long)N, (long long)cta_of(t, T, N), (long long)owner[t]);
    // units: contributors and slots
    std::vector<std::vector<int64_t>> slots_of_cta(N);
    int64_t U0 = 0;
    for (int64_t len : unit_len) {
        const int64_t U1 = U0 + len;
        // brute force: the distinct owners of the unit's tiles, in order
        std::vector<int64_t> cs;
        for (int64_t t = U0; t < U1; ++t)
            if (cs.empty() || cs.back() != owner[t]) cs.push_back(owner[t]);
        const int ncc = unit_contributors(U0, U1, T, N);
        CHECK(ncc == (int)cs.size(), "contributors U=[%lld,%lld) T=%lld N=%lld: %d vs %zu\n",
              (long long)U0, (long long)U1, (long long)T, (long long)N, ncc, cs.size());
        const int64_t c_first = cta_of(U0, T, N);
        const bool first_odd = range_start(c_first, T, N) < U0;
        for (int j = 0; j < (int)cs.size() && j < ncc; ++j) {
            const int64_t want = partial_slot(cs[j], U0, T, N);     // what contributor j writes
            const int64_t got = contributor_slot(j, U0, c_first, first_odd, T >= N, T, N);   // merge reads
            CHECK(got == want, "slot j=%d U0=%lld T=%lld N=%lld: merge %lld, writer %lld\n", j,
                  (long long)U0, (long long)T, (long long)N, (long long)got, (long long)want);
            CHECK(want == 2 * cs[j] || want == 2 * cs[j] + 1, "slot outside the CTA's pair\n");
            // only split units use a slot
            if (cs.size() > 1) slots_of_cta[cs[j]].push_back(want);
        }
        U0 = U1;
    }
    // a CTA never uses one slot for two units
    for (int64_t c = 0; c < N; ++c) {
        const auto& v = slots_of_cta[c];
        CHECK(v.size() <= 2, "CTA %lld shares %zu units\n", (long long)c, v.size());
        if (v.size() == 2) CHECK(v[0] != v[1], "CTA %lld slot reused\n", (long long)c);
    }
}

// find_unit against an enumeration of (sequence, head, tile)
static void check_find_unit(const std::vector<int32_t>& lens, int Hkv) {
    constexpr int TILE = 128;
    const int B = (int)lens.size();
    std::vector<int32_t> prefix(B + 1, 0);
    for (int b = 0; b < B; ++b) {
        const int ntb = lens[b] > 0 ? (lens[b] + TILE - 1) / TILE : 1;
        prefix[b + 1] = prefix[b] + Hkv * ntb;
    }
    int64_t gt = 0;
    for (int b = 0; b < B; ++b) {
        const int ntb = lens[b] > 0 ? (lens[b] + TILE - 1) / TILE : 1;
        for (int h = 0; h < Hkv; ++h) {
            const int64_t U0 = gt;
            for (int k = 0; k < ntb; ++k, ++gt) {
                const Unit u = find_unit<TILE>(prefix.data(), lens.data(), B, Hkv, gt);
                CHECK(u.b == b && u.h == h && u.U0 == U0 && u.U1 == U0 + ntb && u.L == lens[b] &&
                          u.ntb == ntb,
                      "find_unit gt=%lld: b %d/%d h %d/%d U0 %lld/%lld\n", (long long)gt, u.b, b, u.h, h,
                      (long long)u.U0, (long long)U0);
            }
        }
    }
}

int main() {
    unsigned seed = 12345u;
    auto rnd = [&](unsigned m) {
        seed = seed * 1664525u + 1013904223u;
        return (seed >> 8) % m;
    };
    const int64_t Ns[] = {1, 2, 3, 5, 7, 16, 64, 147, 148, 149, 296, 444};
    for (int64_t N : Ns) {
        for (int64_t T = 1; T <= 700; T += (T < 160 ? 1 : 7)) {
            for (int rep = 0; rep < 3; ++rep) {
                std::vector<int64_t> units;
                int64_t left = T;
                while (left > 0) {
                    int64_t len = rep == 0 ? 1 : 1 + (int64_t)rnd(rep == 1 ? 8 : 200);
                    if (len > left) len = left;
                    units.push_back(len);
                    left -= len;
                }
                check_split(T, N, units);
            }
        }
        // large tile counts: a few long units
        for (int64_t T : {4096LL, 65536LL + 37, (1LL << 22) + 5}) {
            std::vector<int64_t> units;
            int64_t left = T;
            while (left > 0) {
                int64_t len = 1 + (int64_t)rnd((unsigned)(T / 3 + 1));
                if (len > left) len = left;
                units.push_back(len);
                left -= len;
            }
            check_split(T, N, units);
        }
    }
    for (int Hkv : {1, 3, 8}) {
        check_find_unit({0}, Hkv);
        check_find_unit({1, 128, 129, 0, 4097, 300}, Hkv);
        std::vector<int32_t> lens;
        for (int b = 0; b < 64; ++b) lens.push_back((int32_t)rnd(9000));
        check_find_unit(lens, Hkv);
    }
    if (failures) {
        std::printf("%d failures\n", failures);
        return 1;
    }
    std::printf("ok\n");
    return 0;
}
