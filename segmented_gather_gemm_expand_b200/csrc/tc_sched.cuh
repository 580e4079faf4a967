// Piece scheduler of the tensor-core expand-slice kernel.
//
// A piece is (segment, 128-row block of the segment, column range of one
// n-tile); the kernel's scheduler warp generates the pieces of its CTA in
// order and hands them to the other warps through a queue in shared memory.
// Everything here is plain arithmetic on the segment table, compiled for the
// host too, so that a CPU test can enumerate the pieces of every CTA of a
// grid and check that together they cover every written element exactly once.
//
// Four ways to hand out pieces (the same decision in every CTA):
//
//   balanced   Pieces of full 128-row blocks, in segment order with the n-tile
//              fastest, are dealt round-robin (CTA c takes c, c + G, ...), so
//              that at any moment the CTAs work on neighbouring columns of the
//              same output rows.  Only whole rounds are dealt this way.  The
//              rest -- the last, incomplete round of full pieces and every
//              piece of a partial block (a segment's last block of fewer than
//              128 rows) -- is split into column halves, sorted by the rows
//              of their block (heaviest first: 8-row groups, 16 buckets, a
//              counting sort) and dealt in snake order (CTA 0, 1, ..., G-1,
//              G-1, ..., 0, 0, 1, ...), which evens out the CTAs' loads.
//   round-robin  All pieces, in segment order with the n-tile fastest, dealt
//              round-robin: the balanced deal without its sorted tail.
//   contiguous Each CTA takes the pieces that start in its equal share of the
//              total weight (a piece weighs its 8-row groups, at least a floor,
//              plus its B tile), in the same order; consecutive pieces of a CTA
//              then share their x block, which is converted to the weights'
//              dtype once (used when x's dtype differs from the weights').
//   dynamic    Round-robin without its last rounds: a launch has G0 + E CTAs, of
//              which G0 run at once; unit u < G0 is round-robin share u of the
//              first H pieces (whole rounds, all but the last few), unit
//              G0 + e is chunk e of the rest, cut into E near-equal runs of
//              consecutive pieces.  A CTA processes its own unit, then claims
//              units whose CTAs have not started (cluster launch control, in
//              the kernel) until none is left, so the end of the launch is
//              shared out by how fast each SM actually drains its pieces.
//   columns    Each CTA takes an equal share of the pieces counted in segment
//              order with the row block fastest within each n-tile, so that
//              consecutive pieces of a CTA share their B tile (the adapter's
//              n-tile stays staged while x blocks stream past it).
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define SGMV_HD __host__ __device__ __forceinline__
#else
#define SGMV_HD inline
#endif

namespace sgmv {
namespace sched {

constexpr int BM = 128;                 // rows per block (MMA M, TMEM lanes)
constexpr int GROUP = 8;                // rows per output group
constexpr int GROUPS_PER_BLOCK = BM / GROUP;
constexpr int MAX_SLICES = 4;
constexpr int NUM_BUCKETS = 16;         // a partial block's 8-row groups: 1..16

enum : int32_t { MODE_CONTIG = 0, MODE_BALANCED = 1, MODE_RR = 2, MODE_COLS = 3, MODE_DYNAMIC = 4 };

constexpr int DYN_TAIL_ROUNDS = 3;      // dynamic mode: whole round-robin rounds left to the claimed chunks

struct SegEntry {
    int32_t row0;
    int32_t rows;       // 0: the segment writes nothing (guards applied)
    int32_t adapter;
    int32_t prefix;     // balanced: full-block pieces of earlier segments; round-robin and columns:
                        // all their pieces; contiguous: their weight
};

// The slices of one launch: slice s covers output columns [off[s], off[s] + N[s])
// with its own B; its n-tiles are numbers [tile0[s], tile0[s + 1]).
struct SliceTable {
    int32_t tile0[MAX_SLICES + 1];
    int32_t off[MAX_SLICES];
    int32_t N[MAX_SLICES];
};

struct Piece {
    int32_t seg, rb;      // segment and row block: identify the x block
    int32_t adapter;
    int32_t blk_row0;     // row (of out and x) where the block starts
    int32_t rows;         // rows of the block (1 .. 128)
    int32_t slice;
    int32_t n0;           // first column within the slice
    int32_t col0;         // first output column
    int32_t ncols;        // columns of the piece
};

SGMV_HD int32_t imin(int32_t a, int32_t b) { return a < b ? a : b; }
SGMV_HD int32_t imax(int32_t a, int32_t b) { return a > b ? a : b; }

// Units of one segment in the scan that fills SegEntry::prefix.
SGMV_HD int32_t full_pieces(int32_t rows, int32_t n_tiles) { return rows / BM * n_tiles; }
SGMV_HD int32_t all_pieces(int32_t rows, int32_t n_tiles) { return (rows + BM - 1) / BM * n_tiles; }
SGMV_HD int32_t contig_weight(int32_t rows, int32_t n_tiles, int32_t wmin, int32_t wfix) {
    const int32_t G = (rows + GROUP - 1) / GROUP;
    if (G == 0) return 0;
    const int32_t full = (G - 1) / GROUPS_PER_BLOCK;          // full 128-row blocks
    const int32_t last = G - full * GROUPS_PER_BLOCK;         // groups of the last block
    return (full * imax(GROUPS_PER_BLOCK, wmin) + imax(last, wmin) + (full + 1) * wfix) * n_tiles;
}
// Bucket of a segment's partial last block: its 8-row groups (1..16), 0 if none.
SGMV_HD int32_t partial_bucket(int32_t rows) {
    const int32_t r = rows % BM;
    return r ? (r + GROUP - 1) / GROUP : 0;
}

// Sorted tail of the balanced mode: where each bucket's items start, and the
// segments with a partial block listed by bucket (16 down to 1), then index.
struct Tail {
    int32_t halves;                          // items per tail piece (2: column halves; 1: whole)
    int32_t H, F;                            // full pieces dealt round-robin; all full pieces
    int32_t item0[NUM_BUCKETS + 2];          // item0[r]: first item of bucket r's partial blocks (r = 16..1);
                                             // item0[17] = 0 (the round's leftover full pieces come first)
    int32_t seg0[NUM_BUCKETS + 1];           // seg0[r]: first entry of bucket r in `inv`
    int32_t n_items;
};

// Host (and single-thread) construction of the tail tables and `inv` from a
// segment table whose prefixes count full pieces.  cnt must hold NUM_BUCKETS + 1.
SGMV_HD void tail_counts(const SegEntry* segs, int32_t nseg, int32_t* cnt) {
    for (int r = 0; r <= NUM_BUCKETS; ++r) cnt[r] = 0;
    for (int32_t s = 0; s < nseg; ++s) cnt[partial_bucket(segs[s].rows)] += 1;
}
SGMV_HD void tail_layout(Tail& tl, const int32_t* cnt, int32_t F, int32_t grid, int32_t n_tiles, int32_t halves) {
    tl.halves = halves;
    tl.F = F;
    tl.H = F / grid * grid;
    int32_t item = (F - tl.H) * halves, seg = 0;
    tl.item0[NUM_BUCKETS + 1] = 0;
    for (int r = NUM_BUCKETS; r >= 1; --r) {
        tl.item0[r] = item;
        tl.seg0[r] = seg;
        item += cnt[r] * n_tiles * halves;
        seg += cnt[r];
    }
    tl.seg0[0] = seg;
    tl.item0[0] = item;
    tl.n_items = item;
}
SGMV_HD void tail_inverse(const SegEntry* segs, int32_t nseg, const Tail& tl, int32_t* inv) {
    int32_t fill[NUM_BUCKETS + 1];
    for (int r = 0; r <= NUM_BUCKETS; ++r) fill[r] = r ? tl.seg0[r] : 0;
    for (int32_t s = 0; s < nseg; ++s) {
        const int32_t r = partial_bucket(segs[s].rows);
        if (r) inv[fill[r]++] = s;
    }
}

// The piece generator of one CTA.
struct Gen {
    const SegEntry* segs;
    const SliceTable* st;
    const int32_t* inv;
    const Tail* tl;
    int32_t nseg, n_tiles, bn, mode;
    int32_t c, G;                 // this CTA, grid size
    // balanced: head (round-robin over full pieces) then tail items
    int32_t hs, hloc, f;          // head: segment, piece within its full pieces, global index
    int32_t m, which;             // tail: round and item of the round
    int32_t rr_end;               // round-robin: all pieces
    int32_t cend;                 // columns: end of this CTA's pieces (global; hs, hloc and f walk them)
    int32_t G0, E, Hd;            // dynamic: CTAs that run at once, chunks, pieces dealt round-robin
    // contiguous walk
    int32_t i, rb, j, cur, w_end, nblk, gcw, wmin, wfix;

    // dynamic mode: the pieces of unit u (its own CTA's, or one it claimed)
    SGMV_HD void init_unit(int32_t u) {
        hs = 0;
        hloc = 0;
        if (u < G0) {                 // round-robin share u of the first Hd pieces
            c = u;
            G = G0;
            f = u;
            rr_end = Hd;
            cend = -1;
            head_advance(u);
        } else {                      // chunk u - G0 of the remaining pieces, in order
            const int32_t e = u - G0, T = tl_total - Hd;
            f = Hd + (int32_t)(((int64_t)T * e) / E);
            cend = Hd + (int32_t)(((int64_t)T * (e + 1)) / E);
            head_advance(f);
        }
    }
    int32_t tl_total;             // dynamic: all pieces

    // pieces of segment s that are dealt round-robin
    SGMV_HD int32_t fullp(int32_t s) const {
        return mode == MODE_BALANCED ? full_pieces(segs[s].rows, n_tiles) : all_pieces(segs[s].rows, n_tiles);
    }

    // The piece of block rb of segment s, n-tile j, column half h (h < 0: whole tile).
    // False if the half holds no columns.
    SGMV_HD bool make(int32_t s, int32_t rb_, int32_t j_, int32_t h, Piece& p) const {
        int32_t sl = 0;
        while (j_ >= st->tile0[sl + 1]) ++sl;
        const int32_t n0t = (j_ - st->tile0[sl]) * bn;
        const int32_t tcols = imin(bn, st->N[sl] - n0t);
        if (h < 0) {
            p.n0 = n0t;
            p.ncols = tcols;
        } else {
            const int32_t hc = bn / 2;
            p.n0 = n0t + h * hc;
            p.ncols = imin(hc, tcols - h * hc);
            if (p.ncols <= 0) return false;
        }
        const SegEntry e = segs[s];
        p.seg = s;
        p.rb = rb_;
        p.adapter = e.adapter;
        p.blk_row0 = e.row0 + rb_ * BM;
        p.rows = imin(BM, e.rows - rb_ * BM);
        p.slice = sl;
        p.col0 = st->off[sl] + p.n0;
        return true;
    }

    // ------------------------------------------------------------ balanced
    SGMV_HD void head_advance(int32_t by) {
        hloc += by;
        while (hs < nseg && hloc >= fullp(hs)) {
            hloc -= fullp(hs);
            ++hs;
        }
    }
    // Item i of the sorted tail; false if it is an empty half.
    SGMV_HD bool tail_item(int32_t it, Piece& p) const {
        const int32_t hv = tl->halves;
        if (it < tl->item0[NUM_BUCKETS]) {             // leftover full pieces of the last round
            const int32_t fi = tl->H + it / hv;
            int32_t lo = 0, hi = nseg - 1;             // last segment whose prefix <= fi
            while (lo < hi) {
                const int32_t mid = (lo + hi + 1) / 2;
                if (segs[mid].prefix <= fi) lo = mid;
                else hi = mid - 1;
            }
            while (lo < nseg && fi - segs[lo].prefix >= fullp(lo)) ++lo;   // skip segments without full blocks
            const int32_t local = fi - segs[lo].prefix;
            return make(lo, local / n_tiles, local % n_tiles, hv == 2 ? it % 2 : -1, p);
        }
        int32_t r = NUM_BUCKETS;
        while (r > 1 && it >= tl->item0[r - 1]) --r;
        const int32_t q = it - tl->item0[r];
        const int32_t per = n_tiles * hv;
        const int32_t s = inv[tl->seg0[r] + q / per];
        const int32_t rem = q % per;
        return make(s, segs[s].rows / BM, rem / hv, hv == 2 ? rem % hv : -1, p);
    }

    // ------------------------------------------------------------ contiguous
    SGMV_HD void load_segment_geometry() {
        const int32_t Gg = (segs[i].rows + GROUP - 1) / GROUP;
        nblk = (Gg + GROUPS_PER_BLOCK - 1) / GROUPS_PER_BLOCK;
    }
    SGMV_HD void set_block() {
        const int32_t Gg = (segs[i].rows + GROUP - 1) / GROUP;
        gcw = imax(imin(GROUPS_PER_BLOCK, Gg - rb * GROUPS_PER_BLOCK), wmin) + wfix;
    }
    SGMV_HD void skip_empty() {
        while (i < nseg && segs[i].rows == 0) ++i;
        if (i < nseg) {
            load_segment_geometry();
            cur = segs[i].prefix;
        }
    }
    // The pieces whose start weight lies in [w0, w1).
    SGMV_HD void seek(int32_t w0, int32_t w1) {
        w_end = w1;
        i = nseg;
        rb = j = 0;
        cur = w1;
        if (w0 >= w1 || nseg == 0) return;
        int32_t lo = 0, hi = nseg - 1;   // last segment whose prefix <= w0
        while (lo < hi) {
            const int32_t mid = (lo + hi + 1) / 2;
            if (segs[mid].prefix <= w0) lo = mid;
            else hi = mid - 1;
        }
        i = lo;
        skip_empty();
        if (i >= nseg) return;
        const int32_t local = w0 - segs[i].prefix;
        const int32_t bw = (imax(GROUPS_PER_BLOCK, wmin) + wfix) * n_tiles;   // weight of a full row block
        rb = imin(local / bw, nblk - 1);
        set_block();
        const int32_t rem = local - rb * bw;
        j = (rem + gcw - 1) / gcw;                              // first piece starting at or after w0
        if (j >= n_tiles) {
            j = 0;
            if (++rb == nblk) {
                rb = 0;
                ++i;
                skip_empty();
                if (i >= nseg) return;
                cur = segs[i].prefix;
                set_block();
                return;
            }
            set_block();
        }
        cur = segs[i].prefix + rb * bw + j * gcw;
    }

    // ------------------------------------------------------------ interface
    // total: full pieces (balanced), all pieces (round-robin) or total weight (contiguous).
    SGMV_HD void init(int32_t cta, int32_t grid, int32_t total, int32_t wmin_, int32_t wfix_) {
        c = cta;
        G = grid;
        wmin = wmin_;
        wfix = wfix_;
        rr_end = total;
        if (mode == MODE_DYNAMIC) {
            tl_total = total;
            G0 = grid;                // grid: the CTAs that run at once (the caller passes G0)
            const int32_t rounds = total / G0 - DYN_TAIL_ROUNDS;
            Hd = rounds > 0 ? rounds * G0 : 0;
            init_unit(cta);
        } else if (mode == MODE_COLS) {
            f = (int32_t)(((int64_t)total * c) / G);
            cend = (int32_t)(((int64_t)total * (c + 1)) / G);
            hs = 0;
            hloc = 0;
            head_advance(f);
        } else if (mode != MODE_CONTIG) {
            hs = 0;
            hloc = 0;
            f = c;
            head_advance(c);
            m = 0;
            which = 0;
        } else {
            seek((int32_t)(((int64_t)total * c) / G), (int32_t)(((int64_t)total * (c + 1)) / G));
        }
    }

    SGMV_HD bool next(Piece& p) {
        if (mode == MODE_DYNAMIC) {
            if (cend < 0) {           // a round-robin share
                if (f >= rr_end) return false;
                make(hs, hloc / n_tiles, hloc % n_tiles, -1, p);
                f += G;
                head_advance(G);
                return true;
            }
            if (f >= cend) return false;
            make(hs, hloc / n_tiles, hloc % n_tiles, -1, p);
            ++f;
            head_advance(1);
            return true;
        }
        if (mode == MODE_COLS) {
            if (f >= cend) return false;
            const int32_t nblk_s = (segs[hs].rows + BM - 1) / BM;   // row blocks of the segment: the fastest index
            make(hs, hloc % nblk_s, hloc / nblk_s, -1, p);
            ++f;
            head_advance(1);
            return true;
        }
        if (mode != MODE_CONTIG) {
            while (f < (mode == MODE_RR ? rr_end : tl->H)) {
                const bool ok = make(hs, hloc / n_tiles, hloc % n_tiles, -1, p);
                f += G;
                head_advance(G);
                if (ok) return true;
            }
            if (mode == MODE_RR) return false;
            while (true) {   // tail items c + 2Gm and 2G - 1 - c + 2Gm, in increasing order
                const int32_t it = which == 0 ? c + 2 * G * m : 2 * G - 1 - c + 2 * G * m;
                if (which == 0) which = 1;
                else {
                    which = 0;
                    ++m;
                }
                if (it >= tl->n_items) {
                    if (which == 0) return false;   // the second item of the round is larger still
                    continue;
                }
                if (tail_item(it, p)) return true;
            }
        }
        if (i >= nseg || cur >= w_end) return false;
        make(i, rb, j, -1, p);
        cur += gcw;
        if (++j == n_tiles) {
            j = 0;
            if (++rb == nblk) {
                rb = 0;
                ++i;
                skip_empty();
            }
            if (i < nseg) set_block();
        }
        return true;
    }
};

}  // namespace sched
}  // namespace sgmv
