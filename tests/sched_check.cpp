// Host check of the tensor-core kernel's piece scheduler (csrc/tc_sched.cuh).
//
// For many random segment tables, slice sets, tile widths, grid sizes and
// every way of handing out pieces, it enumerates the pieces of every CTA with
// the same generator the kernel's scheduler warp runs, and checks that
// together they write every (row, column) of every valid segment's slices
// exactly once and nothing else.  It also reports the largest CTA load over
// the mean (in written elements) for the balanced mode.
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
    int bn, grid, mode, halves, dyn_chunks;
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

// Returns max/mean of the CTAs' loads (elements written), or -1 on failure.
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
        total += k.mode == MODE_BALANCED ? full_pieces(segs[b].rows, n_tiles)
                 : k.mode == MODE_RR || k.mode == MODE_COLS || k.mode == MODE_DYNAMIC ? all_pieces(segs[b].rows, n_tiles)
                                         : contig_weight(segs[b].rows, n_tiles, wmin, wfix);
    }
    Tail tl;
    std::vector<int32_t> inv(nseg + 1);
    if (k.mode == MODE_BALANCED) {
        int32_t cnt[NUM_BUCKETS + 1];
        tail_counts(segs.data(), nseg, cnt);
        tail_layout(tl, cnt, total, k.grid, n_tiles, k.halves);
        tail_inverse(segs.data(), nseg, tl, inv.data());
    }
    int64_t H = 0;
    for (int i = 0; i < k.nsl; ++i) H = H > k.off[i] + k.N[i] ? H : k.off[i] + k.N[i];
    std::vector<uint8_t> cover((size_t)k.T * (size_t)H, 0);
    std::vector<double> load(k.grid, 0.0);
    // dynamic mode: the grid has k.grid + E CTAs; each of the first k.grid takes its own unit, then
    // the remaining units are claimed in an arbitrary order by arbitrary CTAs (here: a shuffled deal)
    const int32_t E = k.mode == MODE_DYNAMIC ? k.dyn_chunks : 0;
    std::vector<int32_t> owner(k.grid + E);
    for (int32_t u = 0; u < k.grid + E; ++u) owner[u] = u < k.grid ? u : (int32_t)uni(0, k.grid - 1);
    for (int32_t u = 0; u < k.grid + E; ++u) {
        const int32_t c = owner[u];
        Gen g;
        g.segs = segs.data();
        g.st = &st;
        g.inv = inv.data();
        g.tl = &tl;
        g.nseg = nseg;
        g.n_tiles = n_tiles;
        g.bn = k.bn;
        g.mode = k.mode;
        if (k.mode == MODE_DYNAMIC) {
            g.E = E;
            g.init(u < k.grid ? u : 0, k.grid, total, wmin, wfix);
            if (u >= k.grid) g.init_unit(u);
        } else {
            if (u >= k.grid) break;
            g.init(c, k.grid, total, wmin, wfix);
        }
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
            CHECK(p.n0 % (k.bn / 2) == 0, "n0 %d not on a half-tile boundary", p.n0);
            CHECK(p.ncols <= k.bn, "piece wider than a tile");
            CHECK(p.col0 == k.off[p.slice] + p.n0, "col0");
            CHECK(p.adapter == segs[p.seg].adapter, "adapter");
            for (int32_t r = p.blk_row0; r < p.blk_row0 + p.rows; ++r)
                for (int32_t n = p.col0; n < p.col0 + p.ncols; ++n) cover[(size_t)r * H + n] += 1;
            load[c] += (double)p.rows * p.ncols;
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
    double mx = 0, sum = 0;
    for (double v : load) {
        mx = v > mx ? v : mx;
        sum += v;
    }
    return sum > 0 ? mx / (sum / k.grid) : 1.0;
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
    k.mode = (int)uni(0, 4);   // MODE_CONTIG, MODE_BALANCED, MODE_RR, MODE_COLS or MODE_DYNAMIC
    k.dyn_chunks = (int)uni(1, 3 * k.grid);
    k.halves = uni(0, 1) ? 2 : 1;
    return k;
}

int main(int argc, char** argv) {
    const int cases = argc > 1 ? std::atoi(argv[1]) : 3000;
    double worst_balanced = 0;
    for (int n = 0; n < cases; ++n) {
        const Case k = random_case(n % 3);
        const double r = run_case(k);
        if (r < 0) {
            std::fprintf(stderr, "case %d failed (nseg %zu, grid %d, mode %d, halves %d, bn %d, slices %d)\n", n,
                         k.len.size(), k.grid, k.mode, k.halves, k.bn, k.nsl);
            break;
        }
        (void)worst_balanced;
    }
    // The round-robin-plus-sorted-tail deal on a QKV-like batch: 16 segments of 64..1024 rows,
    // 2 of them idle, three 4096-column slices, 148 CTAs.
    {
        rng_state = 0x2545F4914F6CDD1Dull;   // a fixed batch, whatever the random cases drew
        Case k;
        int64_t row = 0;
        for (int b = 0; b < 16; ++b) {
            const int64_t L = uni(64, 1024);
            k.start.push_back(row);
            k.len.push_back(L);
            k.idx.push_back(b % 8 == 3 ? -1 : uni(0, 31));
            row += L;
        }
        k.T = row;
        k.A = 32;
        k.nsl = 1;
        k.off[0] = 0;
        k.N[0] = 4096;
        k.bn = 128;
        k.grid = 148;
        k.mode = MODE_BALANCED;
        k.dyn_chunks = 0;
        for (int hv : {1, 2}) {
            k.halves = hv;
            const double r = run_case(k);
            std::printf("qkv-like batch, halves %d: max/mean load %.4f\n", hv, r);
        }
    }
    if (failures) {
        std::printf("FAILED: %d checks\n", failures);
        return 1;
    }
    std::printf("OK: %d cases\n", cases);
    return 0;
}
