// Piece scheduler of the tensor-core expand-slice kernel.
//
// A piece is (segment, 128-row block of the segment, one n-tile of columns);
// the kernel's scheduler warp generates the pieces of its CTA in order and
// hands them to the other warps through a queue in shared memory.  Everything
// here is plain arithmetic on the segment table, compiled for the host too, so
// that a CPU test can enumerate the pieces of every CTA of a grid and check
// that together they cover every written element exactly once.
//
// Two ways to hand out pieces (the same decision in every CTA, made by the
// kernel from the segment table):
//
//   round-robin  All pieces, in segment order with the n-tile fastest, dealt
//                round-robin (CTA c takes c, c + G, ...): at any moment the
//                CTAs work on neighbouring columns of the same output rows, and
//                every CTA gets a fair sample of full and partial row blocks.
//   contiguous   Each CTA takes the pieces that start in its equal share of the
//                total weight (a piece weighs its 8-row groups, at least a
//                floor, plus its B tile), in the same order; consecutive pieces
//                of a CTA then share their x block, which is loaded (and, when
//                x's dtype differs from the weights', converted) once.
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

enum : int32_t { MODE_CONTIG = 0, MODE_RR = 1 };

struct SegEntry {
    int32_t row0;
    int32_t rows;       // 0: the segment writes nothing (guards applied)
    int32_t adapter;
    int32_t prefix;     // round-robin: pieces of earlier segments; contiguous: their weight
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
SGMV_HD int32_t all_pieces(int32_t rows, int32_t n_tiles) { return (rows + BM - 1) / BM * n_tiles; }
SGMV_HD int32_t contig_weight(int32_t rows, int32_t n_tiles, int32_t wmin, int32_t wfix) {
    const int32_t G = (rows + GROUP - 1) / GROUP;
    if (G == 0) return 0;
    const int32_t full = (G - 1) / GROUPS_PER_BLOCK;          // full 128-row blocks
    const int32_t last = G - full * GROUPS_PER_BLOCK;         // groups of the last block
    return (full * imax(GROUPS_PER_BLOCK, wmin) + imax(last, wmin) + (full + 1) * wfix) * n_tiles;
}

// The piece generator of one CTA.
struct Gen {
    const SegEntry* segs;
    const SliceTable* st;
    int32_t nseg, n_tiles, bn, mode;
    int32_t c, G;                 // this CTA, grid size
    // round-robin: segment, piece within the segment, global index of the next piece, all pieces
    int32_t hs, hloc, f, rr_end;
    // contiguous walk: segment, row block, n-tile, start weight of the next piece, end of the range,
    // blocks of the segment, weight of a piece of this block, weight floor and fixed part
    int32_t i, rb, j, cur, w_end, nblk, gcw, wmin, wfix;

    // The piece of block rb_ of segment s, n-tile j_.
    SGMV_HD void make(int32_t s, int32_t rb_, int32_t j_, Piece& p) const {
        int32_t sl = 0;
        while (j_ >= st->tile0[sl + 1]) ++sl;
        p.n0 = (j_ - st->tile0[sl]) * bn;
        p.ncols = imin(bn, st->N[sl] - p.n0);
        const SegEntry e = segs[s];
        p.seg = s;
        p.rb = rb_;
        p.adapter = e.adapter;
        p.blk_row0 = e.row0 + rb_ * BM;
        p.rows = imin(BM, e.rows - rb_ * BM);
        p.slice = sl;
        p.col0 = st->off[sl] + p.n0;
    }

    // ------------------------------------------------------------ round-robin
    SGMV_HD void rr_advance(int32_t by) {
        hloc += by;
        while (hs < nseg && hloc >= all_pieces(segs[hs].rows, n_tiles)) {
            hloc -= all_pieces(segs[hs].rows, n_tiles);
            ++hs;
        }
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
    // total: all pieces (round-robin) or the total weight (contiguous).
    SGMV_HD void init(int32_t cta, int32_t grid, int32_t total, int32_t wmin_, int32_t wfix_) {
        c = cta;
        G = grid;
        wmin = wmin_;
        wfix = wfix_;
        hs = hloc = f = rr_end = 0;
        i = rb = j = cur = w_end = nblk = gcw = 0;
        if (mode == MODE_RR) {
            hs = 0;
            hloc = 0;
            f = c;
            rr_end = total;
            rr_advance(c);
        } else {
            seek((int32_t)(((int64_t)total * c) / G), (int32_t)(((int64_t)total * (c + 1)) / G));
        }
    }

    SGMV_HD bool next(Piece& p) {
        if (mode == MODE_RR) {
            if (f >= rr_end) return false;
            make(hs, hloc / n_tiles, hloc % n_tiles, p);
            f += G;
            rr_advance(G);
            return true;
        }
        if (i >= nseg || cur >= w_end) return false;
        make(i, rb, j, p);
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
