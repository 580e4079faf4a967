// Host check of the tensor-core kernel's piece scheduler (csrc/tc_sched.cuh).
//
// For many random segment tables, slice sets, tile widths, grid sizes and
// both ways of handing out pieces, it enumerates the pieces of every CTA with
// the same generator the kernel's scheduler warp runs, and checks that
// together they write every (row, column) of every valid segment's slices
// exactly once and nothing else.
//
// Build and run: g++ -O2 -std=c++17 -I <csrc> sched_check.cpp && ./a.out [cases]
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "tc_sched.cuh"

using namespace sgmv::sched;

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;
static uint64_t rnd() {
    rng_state ^= rng_state << 13;
    rng_state ^= rng_state >> 7;
    rng_state ^= rng_state << 17;
    return rng_state;
}
static int64_t uni(int64_t lo, int64_t hi) { return lo + (int64_t)(rnd() % (uint64_t)(hi - lo + 1)); }

struct Case {
    std::vector<int64_t> start, len, idx;
    int64_t T, A;
    int nsl;
    int64_t off[MAX_SLICES], N[MAX_SLICES];
    int bn, grid, mode;
};

static int failures = 0;
#define CHECK(cond, ...)                                   \
    do {                                                   \
        if (!(cond)) {                                     \
            if (failures < 20) {                           \
                std::fprintf(stderr, "FAIL %s:%d: ", __FILE__, __LINE__); \
                std::fprintf(stderr, __VA_ARGS__);         \
                std::fprintf(stderr, "\n");                \
            }                                              \
            ++failures;                                    \
            return -1.0;                                   \
        }                                                  \
    } while (0)

// Returns 0, or -1 on failure.
static double run_case(const Case& k) {
    const int32_t nseg = (int32_t)k.len.size();
    // segment table with the API's guards (rows clipped at T, invalid ids and starts skipped)
    std::vector<SegEntry> segs(nseg);
    for (int32_t b = 0; b < nseg; ++b) {
        const int64_t s = k.start[b], L = k.len[b], a = k.idx[b];
        int64_t end = s + L;
        if (end > k.T) end = k.T;
        const bool ok = a >= 0 && a < k.A && s >= 0 && L > 0 && end > s;
        segs[b] = SegEntry{(int32_t)s, ok ? (int32_t)(end - s) : 0, (int32_t)a, 0};
    }
    SliceTable st;
    st.tile0[0] = 0;
    for (int i = 0; i < MAX_SLICES; ++i) {
        st.off[i] = i < k.nsl ? (int32_t)k.off[i] : 0;
        st.N[i] = i < k.nsl ? (int32_t)k.N[i] : 0;
        st.tile0[i + 1] = st.tile0[i] + (i < k.nsl ? (int32_t)((k.N[i] + k.bn - 1) / k.bn) : 0);
    }
    const int32_t n_tiles = st.tile0[MAX_SLICES];
    const int32_t wmin = 16, wfix = 1;
    int32_t total = 0;
    for (int32_t b = 0; b < nseg; ++b) {
        segs[b].prefix = total;
        total += k.mode == MODE_RR ? all_pieces(segs[b].rows, n_tiles) : contig_weight(segs[b].rows, n_tiles, wmin, wfix);
    }
    int64_t H = 0;
    for (int i = 0; i < k.nsl; ++i) H = H > k.off[i] + k.N[i] ? H : k.off[i] + k.N[i];
    std::vector<uint8_t> cover((size_t)k.T * (size_t)H, 0);
    for (int32_t c = 0; c < k.grid; ++c) {
        Gen g;
        g.segs = segs.data();
        g.st = &st;
        g.nseg = nseg;
        g.n_tiles = n_tiles;
        g.bn = k.bn;
        g.mode = k.mode;
        g.init(c, k.grid, total, wmin, wfix);
        Piece p;
        int guard = 0;
        while (g.next(p)) {
            CHECK(++guard < 10000000, "runaway generator");
            CHECK(p.seg >= 0 && p.seg < nseg && segs[p.seg].rows > 0, "piece of an empty segment %d", p.seg);
            CHECK(p.rows >= 1 && p.rows <= BM, "rows %d", p.rows);
            CHECK(p.blk_row0 == segs[p.seg].row0 + p.rb * BM, "block row");
            CHECK(p.rb * BM < segs[p.seg].rows, "block past the segment");
            CHECK(p.rows == imin(BM, segs[p.seg].rows - p.rb * BM), "block rows");
            CHECK(p.slice >= 0 && p.slice < k.nsl, "slice");
            CHECK(p.ncols >= 1 && p.n0 >= 0 && p.n0 + p.ncols <= k.N[p.slice], "columns %d+%d of %lld", p.n0,
                  p.ncols, (long long)k.N[p.slice]);
            CHECK(p.n0 % k.bn == 0, "n0 %d not on a tile boundary", p.n0);
            CHECK(p.ncols <= k.bn, "piece wider than a tile");
            CHECK(p.col0 == k.off[p.slice] + p.n0, "col0");
            CHECK(p.adapter == segs[p.seg].adapter, "adapter");
            for (int32_t r = p.blk_row0; r < p.blk_row0 + p.rows; ++r)
                for (int32_t n = p.col0; n < p.col0 + p.ncols; ++n) cover[(size_t)r * H + n] += 1;
        }
    }
    // expected coverage: exactly the rows of valid segments, in every slice
    std::vector<uint8_t> want((size_t)k.T * (size_t)H, 0);
    for (int32_t b = 0; b < nseg; ++b)
        for (int32_t r = segs[b].row0; r < segs[b].row0 + segs[b].rows; ++r)
            for (int i = 0; i < k.nsl; ++i)
                for (int64_t n = k.off[i]; n < k.off[i] + k.N[i]; ++n) want[(size_t)r * H + n] += 1;
    for (size_t e = 0; e < cover.size(); ++e)
        CHECK(cover[e] == want[e], "element (%zu, %zu) written %d times, want %d", e / H, e % H, cover[e], want[e]);
    return 0.0;
}

static Case random_case(int shape) {
    Case k;
    const int nseg = shape == 0 ? (int)uni(0, 6) : shape == 1 ? (int)uni(1, 40) : (int)uni(100, 1500);
    k.A = uni(1, 6);
    int64_t row = 0;
    for (int b = 0; b < nseg; ++b) {
        int64_t L;
        const int kind = (int)uni(0, 9);
        if (kind < 3) L = uni(1, 40);
        else if (kind < 6) L = 128 * uni(1, 4);
        else if (kind < 8) L = uni(1, 700);
        else L = uni(-2, 3);                  // empty and negative lengths
        if (shape == 2 && L > 200) L = uni(1, 200);
        row += uni(0, 3) == 0 ? uni(0, 9) : 0;   // gaps
        k.start.push_back(uni(0, 30) == 0 ? -uni(1, 5) : row);
        k.len.push_back(L);
        k.idx.push_back(uni(0, 8) == 0 ? -1 : uni(0, k.A));   // -1 and out-of-range ids
        row += L > 0 ? L : 0;
    }
    k.T = row - (uni(0, 4) == 0 ? uni(0, row > 5 ? 5 : row) : 0);   // sometimes rows past the output
    if (k.T < 1) k.T = 1;
    k.bn = uni(0, 1) ? 128 : 256;
    k.nsl = (int)uni(1, MAX_SLICES);
    int64_t col = 0;
    for (int i = 0; i < k.nsl; ++i) {
        col += 8 * uni(0, 3);
        const int64_t N = shape == 2 ? 8 * uni(1, 40) : 8 * uni(1, 90);
        k.off[i] = col;
        k.N[i] = N;
        col += N;
    }
    k.grid = (int)(uni(0, 2) == 0 ? uni(1, 9) : uni(0, 1) ? 148 : uni(10, 200));
    k.mode = uni(0, 1) ? MODE_RR : MODE_CONTIG;
    return k;
}

int main(int argc, char** argv) {
    const int cases = argc > 1 ? std::atoi(argv[1]) : 3000;
    for (int n = 0; n < cases; ++n) {
        const Case k = random_case(n % 3);
        if (run_case(k) < 0) {
            std::fprintf(stderr, "case %d failed (nseg %zu, grid %d, mode %d, bn %d, slices %d)\n", n, k.len.size(),
                         k.grid, k.mode, k.bn, k.nsl);
            break;
        }
    }
    if (failures) {
        std::printf("FAILED: %d checks\n", failures);
        return 1;
    }
    std::printf("OK: %d cases\n", cases);
    return 0;
}
