// Tensor-core SGMV expand-slice for sm_100a: tcgen05 MMA with the accumulator
// in tensor memory, TMA staging of B, x and the output slice.
//
// One persistent CTA per SM, 384 threads in warp roles.  BN, the n-tile width,
// is 128 or 256 columns (a template parameter); TMEM holds 512 / BN accumulators.
//
//   warp 11   scheduler  builds the segment table (the guards of sgmv.h
//                        applied), generates this CTA's pieces (tc_sched.cuh)
//                        and publishes them, in order, as records in a queue
//                        in shared memory: block, columns, ring position,
//                        x-block reuse, TMEM copy layout.  The other roles only
//                        read records.
//   warp 0    producer   TMA: x for each new 128-row block and B[a]'s BN-row
//                        n-tile (K in 64/32/16/8-column boxes with the matching
//                        swizzle) for each piece.
//   warp 2    loader     in add mode, TMA-loads each piece's old output into
//                        its rows of the shared-memory rings (one ring of
//                        128-byte rows per 128-byte column chunk, in piece
//                        order, freed as the epilogue's stores drain): whole
//                        8-row groups as 2-D boxes of 8..128 rows (128-byte
//                        swizzle), clipped at the slice's last column.
//   warp 1    MMA        rounds x to the weights' dtype into the MMA operand
//                        layout (mixed dtypes), or repeats a short block's rows
//                        over the operand (see below); one elected lane issues
//                        tcgen05.mma (M=128 rows, N=BN columns, K=16 each) into
//                        one of the TMEM accumulators.
//   warps 3-10 epilogue  two groups of four warps take alternate pieces; warp w
//                        owns TMEM lanes 32*(w%4).. (32 rows of the piece) and
//                        all its columns, or, for a piece of at most 64 rows
//                        (computed once per 32- or 64-lane span), its rows in
//                        its span and every 2nd or 4th column chunk: tcgen05.ld
//                        the fp32 sums, add the old output (add mode), round
//                        once to the output dtype, write the tile back in place
//                        in shared memory and TMA-store its whole 8-row groups;
//                        the last < 8 rows of a segment are stored from
//                        registers, so nothing outside the segment's rows is
//                        written.
//
// A piece is (segment, 128-row block of the segment, one n-tile of columns);
// how pieces are handed out to CTAs is described in tc_sched.cuh.  Records
// carry x-block and B-tile reuse flags, so that consecutive pieces of a CTA
// that share either keep it staged.  Every wait on an mbarrier is bounded; a
// wait that gives up sets the device error word and makes the CTA leave its
// loops.
#pragma once

#include <cuda.h>

#include <atomic>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "plan_cache.cuh"
#include "tc_ptx.cuh"
#include "tc_sched.cuh"

namespace sgmv {
namespace tc {

using sched::SegEntry;
using sched::SliceTable;
using sched::Piece;

constexpr int BM = sched::BM;         // rows per MMA tile (TMEM lanes)
constexpr int BM_LOG = 7;
static_assert((1 << BM_LOG) == BM, "BM is a power of two");
constexpr int TMEM_COLS = 512;        // every accumulator of a CTA: all of TMEM
constexpr int GROUP = sched::GROUP;   // rows per work unit
constexpr int THREADS = 384;
constexpr int EPI_WARP0 = 3;          // first epilogue warp
constexpr int EPI_GROUPS = 2;         // epilogue warp groups, taking pieces in turn
constexpr int EPI_WARPS = 4 * EPI_GROUPS;
constexpr int SCHED_WARP = 11;
constexpr int SEG_CAP = 16384;        // most segments a launch takes (the shared-memory table decides below that)
constexpr int WARP_TABLE_MAX = 32;    // segment tables up to this size are built by the scheduler warp alone
constexpr int MAX_KP = 128;           // largest padded rank
constexpr int NUM_YMAPS = 5;          // output boxes of 8, 16, 32, 64, 128 rows
constexpr int MAX_WBLK = 4;           // B tile K blocks (64/32/16/8 columns)
constexpr int MAX_SLICES = sched::MAX_SLICES;   // slices of one output updated by one launch
constexpr int RING_PIECES = 32;       // pieces that may hold ring space at once
constexpr int QS = 64;                // piece records in the queue
// Records a short table's scheduler prepares before the dependency wait.  The
// table's load and scan there are what pays; each held record delays the
// start if the wait ends first.  QKV prefill, us per call by held records
// 0/1/2/4/16: 29.2, 28.8, 28.8, 30.4, 35.6 (30.3 with the table built after
// the wait); the single-tenant batch 48.9, 49.2, 49.6, 50.9, 55.7 (48.5).
constexpr int SPEC_RECORDS = 1;
// an accumulator slot, a ring barrier slot and a queue slot always serve the same epilogue group
static_assert(RING_PIECES % EPI_GROUPS == 0 && QS % EPI_GROUPS == 0, "slot ownership");
constexpr int32_t MODE_AUTO = -1;     // Geometry::mode: decided on the device from the segment table
// record slot readers: producer, loader, MMA warp, and the four warps of the piece's epilogue group
constexpr uint32_t QUEUE_READERS = 3 + 4;

// Geometry fixed per launch (host computes; kernel parameter).
struct Geometry {
    int32_t K;          // rank
    int32_t Kp;         // rank padded to a multiple of 16
    int32_t x_bytes;    // element size of x
    int32_t convert_x;  // x's dtype differs from the weights': round in shared memory
    int32_t n_tiles;    // n-tiles of all slices together
    int32_t ring_rows, stages_w, stages_xo, stages_xr;
    int32_t w_is_bf16;
    int32_t wmin, wfix; // contiguous mode: weight of a piece = max(its 8-row groups, wmin) + wfix
    int32_t mode;       // sched::MODE_CONTIG, or MODE_AUTO: the kernel picks (choose_mode)
    int32_t bn;         // columns per n-tile: 128 or 256 (the kernel's BN)
    // B tile: K split into blocks of 64/32/16/8 columns, each its own TMA box
    // (rows of 2*kb bytes, swizzled by the row width) at w_blk_off in a stage
    int32_t w_nblk;
    int32_t w_blk_k0[MAX_WBLK], w_blk_kb[MAX_WBLK], w_blk_off[MAX_WBLK];
    int32_t w_zero_off; // 16-byte x 128-row zero chunk after an 8-column block (-1: none)
    // MMA descriptors of B for each K=16 step, start address left 0, and the
    // step's byte offset within a stage
    int32_t ksteps;
    uint64_t b_desc_rel[MAX_KP / 16];
    uint32_t b_off[MAX_KP / 16];

    // shared memory offsets (bytes, from the 1024-aligned base)
    int32_t off_y, off_w, off_xo, off_xr, off_seg, off_ends, off_q, off_bar;
    int32_t w_bytes, xo_bytes, xr_bytes;
};

struct YMaps {
    CUtensorMap m[MAX_SLICES][NUM_YMAPS];
};

struct WMaps {
    CUtensorMap m[MAX_SLICES][MAX_WBLK];
};

// The slices of one launch (kernel parameter); copied into shared memory as a
// SliceTable, since reading it from the parameter space through a pointer
// with a data-dependent index costs a slow generic load on every piece.
struct Slices {
    int32_t count;
    int32_t tile0[MAX_SLICES + 1];
    int64_t off[MAX_SLICES];
    int64_t N[MAX_SLICES];
};

// ---------------------------------------------------------------- piece records

enum : int32_t { REC_NEW_X = 1, REC_LAST_X = 2, REC_END = 4, REC_NEW_W = 8, REC_LAST_W = 16 };

// One piece as the roles read it from the queue.
struct PieceRec {
    int32_t adapter;
    int32_t blk_row0;     // row (of out and x) where the 128-row block starts
    int32_t rows;         // rows of the block (1 .. 128)
    int32_t n0;           // first column within the slice
    int32_t col0;         // first output column of the piece
    int32_t ncols;        // columns of the piece
    int32_t slice;
    int32_t rep_log;      // log2 of the copies of the piece's rows in TMEM (1, 2 or 4 copies,
                          // one per 128/copies lanes)
    int32_t shift;        // lane of the piece's first row within each copy (0, 32, 64 or 96)
    int32_t pos;          // first ring row of the piece
    int32_t head_end;     // ring rows handed out up to and including this piece
    int32_t flags;        // REC_NEW_X / REC_LAST_X: first / last piece of its x block in this CTA;
                          // REC_NEW_W / REC_LAST_W: the same for its B tile (adapter, slice, first column)
};

// load_segment read through L2 (ld.global.cg), same guards.  The scheduler of
// a short table reads the metadata once before the preceding grid may have
// finished and once after; the second read must not hit a stale L1 line.
__device__ __forceinline__ int64_t load_meta_l2(const MetaVec& m, int64_t i) {
    if (m.dtype == META_IOTA) return i;
    if (m.dtype == META_ONE) return 1;
    if (m.dtype == SGMV_I64) return __ldcg(reinterpret_cast<const long long*>(m.ptr) + i * m.stride);
    return (int64_t)__ldcg(reinterpret_cast<const int*>(m.ptr) + i * m.stride);
}

__device__ __forceinline__ Segment load_segment_l2(const Problem& p, int64_t b) {
    Segment s;
    s.row0 = load_meta_l2(p.start, b);
    const int64_t L = load_meta_l2(p.len, b);
    s.adapter = load_meta_l2(p.idx, b);
    const int64_t lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    int64_t end = s.row0 + L;
    if (end > lim) end = lim;
    const bool ok = s.adapter >= 0 && s.adapter < p.lora_num && s.row0 >= 0 && L > 0 && end > s.row0;
    s.rows = ok ? end - s.row0 : 0;
    return s;
}

// log2 of the lanes between repeats of a block's rows in the staged x operand:
// the rows rounded up to 32, 64 or 128.
__host__ __device__ __forceinline__ int32_t x_period_log(int32_t rows) { return rows <= 32 ? 5 : rows <= 64 ? 6 : BM_LOG; }

// Place a piece of rows8 rows in a ring of R rows: returns the ring row where it
// starts and advances `head` (rows handed out so far, including skipped ones).
// A piece never wraps: if it does not fit before the ring's end it starts at 0.
__device__ __forceinline__ int32_t ring_place(int32_t& head, int32_t rows8, int32_t R) {
    int32_t pos = head % R;
    if (pos + rows8 > R) {
        head += R - pos;
        pos = 0;
    }
    head += rows8;
    return pos;
}

// Index k of the largest output box (8 << k rows, k <= max_level) that fits in
// `rows` (a positive multiple of 8).
__device__ __forceinline__ int box_level(int rows, int max_level) {
    const int k = 31 - __clz(rows / GROUP);
    return k < max_level ? k : max_level;
}

// Exclusive block-wide scan of units_of(segs[b]) into segs[b].prefix; returns
// the total.  Called by all THREADS threads; ends synchronised.
template <typename UnitsFn>
__device__ int32_t scan_segments(SegEntry* segs, int32_t nseg, int32_t* warp_sums, UnitsFn units_of) {
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    int32_t running = 0;
    for (int32_t base = 0; base < nseg; base += THREADS) {
        const int32_t b = base + tid;
        const int32_t units = b < nseg ? units_of(segs[b]) : 0;
        int32_t v = units;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += t;
        }
        if (lane == 31) warp_sums[warp] = v;
        __syncthreads();
        int32_t warp_off = 0, total = 0;
        for (int w = 0; w < THREADS / 32; ++w) {
            if (w < warp) warp_off += warp_sums[w];
            total += warp_sums[w];
        }
        if (b < nseg) segs[b].prefix = running + warp_off + v - units;
        running += total;
        __syncthreads();
    }
    if (nseg <= 0) __syncthreads();
    return running;
}

// Segment units of the scan: pieces (round-robin) or weight (contiguous).
__device__ __forceinline__ int32_t seg_units(const Geometry& geo, int32_t mode, int32_t rows) {
    if (mode == sched::MODE_RR) return sched::all_pieces(rows, geo.n_tiles);
    return sched::contig_weight(rows, geo.n_tiles, geo.wmin, geo.wfix);
}

// How this launch hands out pieces (the same in every CTA).  A batch whose row
// blocks are mostly partial (short segments: decode-like mixes) takes
// contiguous ranges, which keep each x block and walk one adapter's B tiles in
// order; others are dealt round-robin.  Measured on one B200 (us per call,
// round-robin vs contiguous): QKV prefill 30.7 vs 32.2, single-tenant 51.4 vs
// 54.4, decode-like mix 71.5 vs 52.0.
__device__ __forceinline__ int32_t choose_mode(const Geometry& geo, int32_t partial_blocks, int32_t blocks) {
    if (geo.mode != MODE_AUTO) return geo.mode;
    return 2 * partial_blocks > blocks ? (int32_t)sched::MODE_CONTIG : (int32_t)sched::MODE_RR;
}

// ---------------------------------------------------------------- the kernel

// BN: columns per n-tile (128 or 256); TMEM holds TMEM_COLS / BN accumulators.
template <int OUT_DT, bool ADD, int BN>
__global__ void __launch_bounds__(THREADS, 1)
tc_expand_slice_kernel(const __grid_constant__ WMaps wmaps, const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ YMaps ymaps, Problem p, Geometry geo,
                       const __grid_constant__ Slices sl) {
    constexpr int OUT_BYTES = OUT_DT == SGMV_F32 ? 4 : 2;
    constexpr int NUM_ACC = TMEM_COLS / BN;
    static_assert(NUM_ACC % EPI_GROUPS == 0, "an accumulator slot always serves the same epilogue group");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    __shared__ int s_abort;
    __shared__ uint32_t s_tmem_base;
    __shared__ int32_t s_warp_sums[THREADS / 32];
    __shared__ SliceTable s_sl;
    __shared__ int32_t s_blocks, s_partial;   // row blocks and partial ones (long tables)

    const int tid = threadIdx.x;
    const int warp = tid / 32;
    const int lane = tid % 32;

    SegEntry* segs = reinterpret_cast<SegEntry*>(smem + geo.off_seg);
    PieceRec* recs = reinterpret_cast<PieceRec*>(smem + geo.off_q);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + geo.off_bar);
    const int SW = geo.stages_w, SXO = geo.stages_xo, SXR = geo.stages_xr;
    const int32_t R = geo.ring_rows;
    uint64_t* w_full = bars;
    uint64_t* w_empty = w_full + SW;
    uint64_t* xo_full = w_empty + SW;
    uint64_t* xo_empty = xo_full + SXO;
    uint64_t* xr_full = xo_empty + SXO;
    uint64_t* xr_empty = xr_full + SXR;
    uint64_t* acc_full = xr_empty + SXR;
    uint64_t* acc_empty = acc_full + NUM_ACC;
    uint64_t* y_full = acc_empty + NUM_ACC;     // piece's ring rows ready (loaded, in add mode)
    uint64_t* y_free = y_full + RING_PIECES;     // piece's ring rows no longer read by any store
    uint64_t* q_full = y_free + RING_PIECES;     // queue slot holds a record
    uint64_t* q_empty = q_full + QS;             // queue slot read by every reader

    if (tid == 0) {
        s_abort = 0;
        s_blocks = 0;
        s_partial = 0;
        for (int i = 0; i <= MAX_SLICES; ++i) s_sl.tile0[i] = sl.tile0[i];
        for (int i = 0; i < MAX_SLICES; ++i) {
            s_sl.off[i] = (int32_t)sl.off[i];
            s_sl.N[i] = (int32_t)sl.N[i];
        }
    }
    {
        // The barriers lie back to back from w_full; every thread initialises a
        // few.  acc_empty and y_free count the four warps of an epilogue group,
        // q_empty every reader of a record.
        const int n_bars = (int)(q_empty + QS - bars);
        const int acc_empty0 = (int)(acc_empty - bars), y_free0 = (int)(y_free - bars);
        const int q_empty0 = (int)(q_empty - bars);
        bool did = false;
        for (int b = tid; b < n_bars; b += THREADS) {
            uint32_t count = 1;
            if ((b >= acc_empty0 && b < acc_empty0 + NUM_ACC) || (b >= y_free0 && b < y_free0 + RING_PIECES)) count = 4;
            if (b >= q_empty0) count = QUEUE_READERS;
            mbar_init(smem_u32(&bars[b]), count);
            did = true;
        }
        if (did) fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_x);
        for (int i = 0; i < sl.count; ++i) {
            for (int b = 0; b < geo.w_nblk; ++b) prefetch_tmap(&wmaps.m[i][b]);
            for (int k = 0; k < NUM_YMAPS; ++k) prefetch_tmap(&ymaps.m[i][k]);
        }
    }
    if (warp == 1) tmem_alloc(smem_u32(&s_tmem_base), NUM_ACC * BN);

    // Zero the rank padding of the operand buffers (TMA never writes it): x's
    // chunks past K, and the chunk B's 8-column block points its upper K half at.
    {
        const int kc_real = geo.K / 8, kc_pad = geo.Kp / 8;
        for (int b = 0; b < SW + SXO; ++b) {
            uint8_t* buf;
            int npad;   // 16-byte rows to clear: one per B row (BN) or x row (BM) per missing K chunk
            if (b < SW) {
                if (geo.w_zero_off < 0) continue;
                buf = smem + geo.off_w + b * geo.w_bytes + geo.w_zero_off;
                npad = (kc_pad - kc_real) * BN;
            } else {
                buf = smem + geo.off_xo + (b - SW) * geo.xo_bytes + kc_real * BM * 16;
                npad = (kc_pad - kc_real) * BM;
            }
            for (int q = tid; q < npad; q += THREADS) *reinterpret_cast<uint4*>(buf + q * 16) = make_uint4(0, 0, 0, 0);
        }
    }

    // Warm L2 with the metadata while the preceding kernel may still run.
    for (int32_t b = tid; b < (int32_t)p.batches; b += THREADS) {
        for (const MetaVec* m : {&p.start, &p.len, &p.idx}) {
            if (m->dtype != SGMV_I32 && m->dtype != SGMV_I64) continue;
            const int64_t esz = m->dtype == SGMV_I64 ? 8 : 4;
            prefetch_l2(static_cast<const char*>(m->ptr) + b * m->stride * esz);
        }
    }
    // barriers, the TMEM address, the slice table and the zeroed padding are
    // visible to every role from here
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // Everything below may read memory written by the preceding kernel.  (The
    // scheduler warp of a short segment table waits by itself, after it has
    // prepared its first records from a speculative read of the metadata.)
    // (A one-segment table gains nothing from it: single-tenant batch 48.8 us
    // per call without, 49.2 with.)
    const bool sched_spec = p.batches >= 2 && p.batches <= WARP_TABLE_MAX;
    if (!(warp == SCHED_WARP && sched_spec)) grid_dependency_wait();
    // The next kernel may be scheduled now: its CTAs take SMs as ours leave, and
    // it waits for this grid to finish before it reads anything.
    grid_dependents_launch();

    const int32_t nseg = (int32_t)p.batches;
    int32_t long_table_total = 0, long_table_mode = 0;   // every thread gets the scan's total and the mode
    if (nseg > WARP_TABLE_MAX) {
        // a long segment table: every thread loads and scans (ends synchronised)
        int32_t my_blocks = 0, my_partial = 0;
        for (int32_t b = tid; b < nseg; b += THREADS) {
            const Segment s = load_segment(p, b);
            segs[b] = SegEntry{(int32_t)s.row0, (int32_t)s.rows, (int32_t)s.adapter, 0};
            my_blocks += (int32_t)((s.rows + BM - 1) / BM);
            my_partial += (s.rows % BM) != 0;
        }
        if (my_blocks) atomicAdd(&s_blocks, my_blocks);
        if (my_partial) atomicAdd(&s_partial, my_partial);
        __syncthreads();
        long_table_mode = choose_mode(geo, s_partial, s_blocks);
        long_table_total = scan_segments(segs, nseg, s_warp_sums, [&](const SegEntry& e) {
            return seg_units(geo, long_table_mode, e.rows);
        });
    }

    const uint32_t tmem_base = s_tmem_base;
    volatile int* abort_flag = &s_abort;
    const bool w_bf16 = geo.w_is_bf16 != 0;
    constexpr int CC = 128 / OUT_BYTES;              // columns per 128-byte chunk
    constexpr int NCH = BN / CC;                     // chunks per n-tile
    const int32_t RING_STRIDE = R * 128;             // bytes of one chunk's ring

    if (warp == SCHED_WARP) {
        // ------------------------------------------------------------ scheduler
        // A short table is read and scanned, and its first SPEC_RECORDS record(s)
        // generated into the queue without being published, while the
        // preceding grid may still run.  After the dependency wait the warp
        // reads the metadata again: if it is unchanged the held records are
        // published at once and generation goes on; if not, everything is
        // redone from the new table (pass 1).  Long tables are built by the
        // whole block after the wait and go straight to pass 1.
        bool retry = false;
#pragma unroll 1
        for (int pass = sched_spec ? 0 : 1; pass < 2; ++pass) {
            int spec_bit = pass == 0;
            asm volatile("" : "+r"(spec_bit));   // one copy of the code for both passes
            const bool spec = spec_bit != 0;
            int32_t total, mode;
            SegEntry mine{0, 0, 0, 0};             // this lane's segment (short tables)
            if (nseg <= WARP_TABLE_MAX) {
                if (!spec) grid_dependency_wait();   // (again after a failed speculation: returns at once)
                // a short table: one segment per lane, a warp scan, no block barrier
                SegEntry e{0, 0, 0, 0};
                if (lane < nseg) {
                    const Segment sg = load_segment_l2(p, lane);
                    e = SegEntry{(int32_t)sg.row0, (int32_t)sg.rows, (int32_t)sg.adapter, 0};
                }
                mine = e;
                mode = choose_mode(geo, (int32_t)__reduce_add_sync(0xffffffffu, (e.rows % BM) != 0 ? 1u : 0u),
                                   (int32_t)__reduce_add_sync(0xffffffffu, (uint32_t)((e.rows + BM - 1) / BM)));
                const int32_t units = lane < nseg ? seg_units(geo, mode, e.rows) : 0;
                int32_t v = units;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int32_t t = __shfl_up_sync(0xffffffffu, v, o);
                    if (lane >= o) v += t;
                }
                e.prefix = v - units;
                if (lane < nseg) segs[lane] = e;
                total = __shfl_sync(0xffffffffu, v, 31);
                __syncwarp();
            } else {
                total = long_table_total;
                mode = long_table_mode;
            }
            constexpr int CC_LOG = OUT_BYTES == 4 ? 5 : 6;
            sched::Gen g;
            Piece cur, nxt, prev;
            bool have = false, ok = true;
            int32_t t = 0, head = 0, prev_seg = -1, prev_rb = -1;
            if (lane == 0) {
                g.segs = segs;
                g.st = &s_sl;
                g.nseg = nseg;
                g.n_tiles = geo.n_tiles;
                g.bn = BN;
                g.mode = mode;
                g.init((int32_t)blockIdx.x, (int32_t)gridDim.x, total, geo.wmin, geo.wfix);
                have = g.next(cur);
            }
            // phase 0 (speculative): up to SPEC_RECORDS records, held; phase 1: the rest
#pragma unroll 1
            for (int phase = spec ? 0 : 1; phase < 2; ++phase) {
                const bool hold = phase == 0;
                const int32_t stop = hold ? SPEC_RECORDS : 0x7fffffff;
                if (lane == 0) {
                    while (have && ok && t < stop) {
                        const bool have_n = g.next(nxt);
                        PieceRec r;
                        r.adapter = cur.adapter;
                        r.blk_row0 = cur.blk_row0;
                        r.rows = cur.rows;
                        r.n0 = cur.n0;
                        r.col0 = cur.col0;
                        r.ncols = cur.ncols;
                        r.slice = cur.slice;
                        r.flags = 0;
                        if (cur.seg != prev_seg || cur.rb != prev_rb) r.flags |= REC_NEW_X;
                        if (!have_n || nxt.seg != cur.seg || nxt.rb != cur.rb) r.flags |= REC_LAST_X;
                        if (t == 0 || cur.adapter != prev.adapter || cur.slice != prev.slice || cur.n0 != prev.n0)
                            r.flags |= REC_NEW_W;
                        if (!have_n || nxt.adapter != cur.adapter || nxt.slice != cur.slice || nxt.n0 != cur.n0)
                            r.flags |= REC_LAST_W;
                        // A short piece (rows in 1 or 2 quadrants) is computed in every span
                        // of 32 or 64 lanes: the x block is staged with its rows repeated
                        // (x_period), so each TMEM quadrant holds a copy of the sums, and the
                        // epilogue warps of the copies split the piece's column chunks.  Where
                        // the piece has fewer chunks than copies, its rows instead take turns
                        // in the lanes of a wider span (the pieces of one epilogue group,
                        // every EPI_GROUPS-th, cycle through them).
                        const int32_t span_log = x_period_log(cur.rows);
                        const int32_t nch = (cur.ncols + (1 << CC_LOG) - 1) >> CC_LOG;
                        const int32_t maxrep_log = BM_LOG - span_log;
                        r.rep_log = min(maxrep_log, nch >= 4 ? 2 : nch >= 2 ? 1 : 0);
                        const int32_t turns_mask = (1 << (maxrep_log - r.rep_log)) - 1;
                        r.shift = ((t / EPI_GROUPS) & turns_mask) << span_log;
                        r.pos = ring_place(head, (cur.rows + GROUP - 1) & ~(GROUP - 1), R);
                        r.head_end = head;
                        const int slot = t % QS;
                        // (held records fit the queue: SPEC_RECORDS <= QS, so this wait
                        // passes at once in phase 0)
                        if (!mbar_wait(smem_u32(&q_empty[slot]), ((t / QS) & 1) ^ 1, abort_flag, DEVERR_SCHEDULE)) {
                            ok = false;
                            break;
                        }
                        recs[slot] = r;
                        if (!hold) mbar_arrive(smem_u32(&q_full[slot]));
                        prev_seg = cur.seg;
                        prev_rb = cur.rb;
                        prev = cur;
                        cur = nxt;
                        have = have_n;
                        ++t;
                    }
                }
                __syncwarp();
                if (!hold) break;
                // the speculation is confirmed if every lane's segment reads the same now
                grid_dependency_wait();
                bool same = true;
                if (lane < nseg) {
                    const Segment sg = load_segment_l2(p, lane);
                    same = sg.row0 == mine.row0 && sg.rows == mine.rows && sg.adapter == mine.adapter;
                }
                if (!__all_sync(0xffffffffu, same)) {
                    retry = true;
                    break;
                }
                if (lane == 0)   // publish the held records
                    for (int32_t i = 0; i < t; ++i) mbar_arrive(smem_u32(&q_full[i % QS]));
                __syncwarp();
            }
            if (retry && pass == 0) {
                retry = false;
                continue;   // pass 1: the table again, after the wait, nothing held
            }
            // one end record for each epilogue group (the other roles stop at the first)
            if (lane == 0) {
                for (int e = 0; ok && e < EPI_GROUPS; ++e, ++t) {
                    const int slot = t % QS;
                    if (!mbar_wait(smem_u32(&q_empty[slot]), ((t / QS) & 1) ^ 1, abort_flag, DEVERR_SCHEDULE)) break;
                    recs[slot].flags = REC_END;
                    mbar_arrive(smem_u32(&q_full[slot]));
                }
            }
            break;
        }
        __syncwarp();
    } else if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_keep = policy_evict_last();
            int32_t t = 0, xb = 0, wb = 0;
            const uint32_t w_bytes = (uint32_t)(BN * geo.K * 2);
            const uint32_t x_bytes = (uint32_t)(BM * geo.K * geo.x_bytes);
            while (true) {
                const int slot = t % QS;
                if (!mbar_wait(smem_u32(&q_full[slot]), (t / QS) & 1, abort_flag, DEVERR_TIMEOUT_PRODUCER)) break;
                const PieceRec pc = recs[slot];
                mbar_arrive(smem_u32(&q_empty[slot]));
                if (pc.flags & REC_END) break;
                if (pc.flags & REC_NEW_X) {
                    const int32_t xcur = xb++;
                    if (geo.convert_x) {
                        const int s = xcur % SXR;
                        if (!mbar_wait(smem_u32(&xr_empty[s]), ((xcur / SXR) & 1) ^ 1, abort_flag,
                                       DEVERR_TIMEOUT_PRODUCER))
                            break;
                        mbar_expect_tx(smem_u32(&xr_full[s]), x_bytes);
                        tma_load_2d(smem_u32(smem + geo.off_xr + s * geo.xr_bytes), &tmap_x, 0, pc.blk_row0,
                                    smem_u32(&xr_full[s]), pol_keep);
                    } else {
                        const int s = xcur % SXO;
                        if (!mbar_wait(smem_u32(&xo_empty[s]), ((xcur / SXO) & 1) ^ 1, abort_flag,
                                       DEVERR_TIMEOUT_PRODUCER))
                            break;
                        mbar_expect_tx(smem_u32(&xo_full[s]), x_bytes);
                        tma_load_3d(smem_u32(smem + geo.off_xo + s * geo.xo_bytes), &tmap_x, 0, pc.blk_row0, 0,
                                    smem_u32(&xo_full[s]), pol_keep);
                    }
                }
                if (pc.flags & REC_NEW_W) {
                    const int32_t wcur = wb++;
                    const int s = wcur % SW;
                    if (!mbar_wait(smem_u32(&w_empty[s]), ((wcur / SW) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_PRODUCER))
                        break;
                    mbar_expect_tx(smem_u32(&w_full[s]), w_bytes);
                    for (int b = 0; b < geo.w_nblk; ++b)
                        tma_load_3d(smem_u32(smem + geo.off_w + s * geo.w_bytes + geo.w_blk_off[b]), &wmaps.m[pc.slice][b],
                                    geo.w_blk_k0[b], pc.n0, pc.adapter, smem_u32(&w_full[s]), pol_keep);
                }
                ++t;
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ output-tile loads
        if (lane == 0) {
            const uint64_t pol_stream = policy_evict_first();
            int32_t* ends = reinterpret_cast<int32_t*>(smem + geo.off_ends);   // ring head after each piece
            int32_t t = 0, tail_head = 0, tail_piece = 0;
            bool ok = true;
            while (ok) {
                const int slot = t % QS;
                if (!mbar_wait(smem_u32(&q_full[slot]), (t / QS) & 1, abort_flag, DEVERR_TIMEOUT_PRODUCER)) break;
                const PieceRec pc = recs[slot];
                mbar_arrive(smem_u32(&q_empty[slot]));
                if (pc.flags & REC_END) break;
                // whole 8-row groups: in add mode the rows past the piece in its last
                // group are read but never written back
                const int rows8 = (pc.rows + GROUP - 1) & ~(GROUP - 1);
                // free the oldest pieces until this one fits and its barriers are reusable
                while (tail_piece < t && (pc.head_end - tail_head > R || t - tail_piece >= RING_PIECES)) {
                    const int fi = tail_piece % RING_PIECES;
                    if (!mbar_wait(smem_u32(&y_free[fi]), (tail_piece / RING_PIECES) & 1, abort_flag,
                                   DEVERR_TIMEOUT_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    tail_head = ends[fi];
                    ++tail_piece;
                }
                if (!ok) break;
                ends[t % RING_PIECES] = pc.head_end;
                const uint32_t bar = smem_u32(&y_full[t % RING_PIECES]);
                if (ADD) {
                    const int nch = (pc.ncols + CC - 1) / CC;
                    mbar_expect_tx(bar, (uint32_t)(rows8 * 128 * nch));
                    const uint32_t ring = smem_u32(smem + geo.off_y);
                    for (int c = 0; c < nch; ++c) {
                        for (int r = 0; r < rows8;) {
                            const int k = box_level(rows8 - r, NUM_YMAPS - 1);
                            tma_load_2d(ring + c * RING_STRIDE + (pc.pos + r) * 128, &ymaps.m[pc.slice][k],
                                        pc.col0 + c * CC, pc.blk_row0 + r, bar, pol_stream);
                            r += GROUP << k;
                        }
                    }
                } else {
                    mbar_arrive(bar);
                }
                ++t;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ x rounding (mixed dtypes) + MMA
        int32_t t = 0, xb = 0, xcur = 0, wb = 0, wcur = 0;
        const uint32_t idesc = instr_desc_mn(w_bf16, BM, BN);
        const int kc_real = geo.K / 8, kc_pad = geo.Kp / 8;
        const bool x_bf16 = p.x_dt == SGMV_BF16;
        constexpr int MAX_KSTEPS = MAX_KP / 16;
        const uint64_t a_rel = smem_desc(0, BM * 16, 128);
        while (true) {
            const int slot = t % QS;
            if (!warp_wait(smem_u32(&q_full[slot]), (t / QS) & 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
            const PieceRec pc = recs[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&q_empty[slot]));
            if (pc.flags & REC_END) break;
            if (pc.flags & REC_NEW_X) {
                xcur = xb++;
                const int xs = xcur % SXO;
                const int pmask = (1 << x_period_log(pc.rows)) - 1;   // operand row m holds x row m % period
                if (geo.convert_x) {
                    const int rs = xcur % SXR;
                    if (!warp_wait(smem_u32(&xr_full[rs]), (xcur / SXR) & 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
                    if (!warp_wait(smem_u32(&xo_empty[xs]), ((xcur / SXO) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_MMA))
                        break;
                    // x (its own dtype, row-major) -> weights' dtype, K-major core matrices,
                    // the block's rows repeated every period
                    const uint8_t* xraw = smem + geo.off_xr + rs * geo.xr_bytes;
                    uint8_t* xop = smem + geo.off_xo + xs * geo.xo_bytes;
                    const int row_bytes = geo.K * geo.x_bytes;
                    for (int q = lane; q < BM * kc_pad; q += 32) {
                        const int m = q % BM, kc = q / BM;
                        uint4 outv = make_uint4(0, 0, 0, 0);
                        if (kc < kc_real) {
                            float f[8];
                            const uint8_t* src = xraw + (m & pmask) * row_bytes + kc * 8 * geo.x_bytes;
                            if (geo.x_bytes == 4) {
                                const float4 a = *reinterpret_cast<const float4*>(src);
                                const float4 b = *reinterpret_cast<const float4*>(src + 16);
                                f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w;
                                f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
                            } else {
                                const uint4 a = *reinterpret_cast<const uint4*>(src);
                                const uint32_t u4[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    f[2 * e] = half_bits_to_float(u4[e] & 0xFFFFu, x_bf16);
                                    f[2 * e + 1] = half_bits_to_float(u4[e] >> 16, x_bf16);
                                }
                            }
                            outv.x = pack2(f[0], f[1], w_bf16);
                            outv.y = pack2(f[2], f[3], w_bf16);
                            outv.z = pack2(f[4], f[5], w_bf16);
                            outv.w = pack2(f[6], f[7], w_bf16);
                        }
                        *reinterpret_cast<uint4*>(xop + kc * (BM * 16) + (m / 8) * 128 + (m % 8) * 16) = outv;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&xr_empty[rs]));
                } else {
                    if (!warp_wait(smem_u32(&xo_full[xs]), (xcur / SXO) & 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
                    if (pmask < BM - 1) {
                        // repeat the block's first rows over the whole operand (16-byte
                        // row pieces; K-block kc of row m at kc * BM * 16 + m * 16)
                        uint8_t* xop = smem + geo.off_xo + xs * geo.xo_bytes;
                        const int per = pmask + 1, copies = BM - per;
                        for (int q = lane; q < copies * kc_pad; q += 32) {
                            const int kc = q / copies, m = per + q % copies;
                            *reinterpret_cast<uint4*>(xop + kc * (BM * 16) + m * 16) =
                                *reinterpret_cast<const uint4*>(xop + kc * (BM * 16) + (m & pmask) * 16);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                    }
                }
            }
            const int xs = xcur % SXO;
            if (pc.flags & REC_NEW_W) {
                wcur = wb++;
                if (!warp_wait(smem_u32(&w_full[wcur % SW]), (wcur / SW) & 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
            }
            const int ws = wcur % SW;
            const int as = t % NUM_ACC;
            if (!warp_wait(smem_u32(&acc_empty[as]), ((t / NUM_ACC) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
            tc_fence_after();
            if (lane == 0) {
                // A row m holds x row m % period: every span of `period` TMEM lanes
                // receives the piece's sums (lanes past its rows are never read)
                const uint32_t a_base = smem_u32(smem + geo.off_xo + xs * geo.xo_bytes);
                const uint32_t b_base = smem_u32(smem + geo.off_w + ws * geo.w_bytes);
                const uint32_t d = tmem_base + (uint32_t)(as * BN);
#pragma unroll
                for (int ks = 0; ks < MAX_KSTEPS; ++ks) {
                    if (ks >= geo.ksteps) break;
                    const uint64_t ad = a_rel | (uint64_t)(((a_base + ks * 2 * (BM * 16)) >> 4) & 0x3FFF);
                    const uint64_t bd = geo.b_desc_rel[ks] | (uint64_t)(((b_base + geo.b_off[ks]) >> 4) & 0x3FFF);
                    tc_mma(d, ad, bd, idesc, ks > 0 ? 1u : 0u);
                }
                tc_commit(smem_u32(&acc_full[as]));
                if (pc.flags & REC_LAST_W) tc_commit(smem_u32(&w_empty[ws]));
                if (pc.flags & REC_LAST_X) tc_commit(smem_u32(&xo_empty[xs]));
            }
            __syncwarp();
            ++t;
        }
    } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + EPI_WARPS) {
        // ------------------------------------------------------------ epilogue
        const int q = warp % 4;                  // TMEM lane quadrant of this warp
        const int grp = (warp - EPI_WARP0) / 4;  // this warp's group takes pieces t % EPI_GROUPS == grp
        const int r = q * 32 + lane;             // block row of this thread
        const int ri = r % GROUP;
        constexpr bool out_bf16 = OUT_DT == SGMV_BF16;
        for (int32_t t = grp;; t += EPI_GROUPS) {
            const int slot = t % QS;
            if (!warp_wait(smem_u32(&q_full[slot]), (t / QS) & 1, abort_flag, DEVERR_TIMEOUT_EPILOGUE)) break;
            const PieceRec pc = recs[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&q_empty[slot]));
            if (pc.flags & REC_END) break;
            const int as = t % NUM_ACC;
            if (!warp_wait(smem_u32(&acc_full[as]), (t / NUM_ACC) & 1, abort_flag, DEVERR_TIMEOUT_EPILOGUE)) break;
            tc_fence_after();
            // every warp of the group waits, so that its release of this piece's
            // ring rows below always lands in the right phase
            if (!warp_wait(smem_u32(&y_full[t % RING_PIECES]), (t / RING_PIECES) & 1, abort_flag,
                           DEVERR_TIMEOUT_EPILOGUE))
                break;
            const int full_end = pc.rows & ~(GROUP - 1);
            const int ncols = pc.ncols;
            const int64_t col0 = pc.col0;   // first output column of the piece
            // this warp's copy of the piece (lanes [k * span, (k + 1) * span)) and
            // its column chunks k, k + rep, ...
            const int span_log = BM_LOG - pc.rep_log;
            const int k_copy = (q * 32) >> span_log;
            const int lane0 = ((q * 32) & ((1 << span_log) - 1)) - pc.shift;   // row of this warp's lane 0 within the piece
            const int pr = lane0 + lane;        // this thread's row within the piece
            const bool valid = pr >= 0 && pr < pc.rows;
            // rows past the last whole group go straight to global memory from registers
            const bool tail = pr >= full_end;
            uint8_t* ring = smem + geo.off_y;
            const uint32_t taddr = tmem_base + (uint32_t)(as * BN) + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
            for (int c = k_copy; c < NCH; c += 1 << pc.rep_log) {
                if (c * CC >= ncols) break;     // warp-uniform
                uint32_t v[CC];
#pragma unroll
                for (int sub = 0; sub < CC / 32; ++sub)
                    tmem_ld32(taddr + (uint32_t)(c * CC + sub * 32), *reinterpret_cast<uint32_t(*)[32]>(v + sub * 32));
                tmem_ld_wait();
                if (valid) {
                    uint8_t* rowp = ring + c * RING_STRIDE + (pc.pos + pr) * 128;
                    uint4* grow = reinterpret_cast<uint4*>(reinterpret_cast<char*>(p.out) +
                                                           ((int64_t)(pc.blk_row0 + pr) * p.H + col0 + c * CC) *
                                                               OUT_BYTES);
                    const int kvalid = (min(CC, ncols - c * CC) * OUT_BYTES) / 16;   // 16-byte pieces in the slice
                    uint4 old[8];
                    if (ADD) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) old[k] = *reinterpret_cast<const uint4*>(rowp + ((k ^ ri) * 16));
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        uint4 nv;
                        if (OUT_BYTES == 2) {
                            float a[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) a[e] = __uint_as_float(v[k * 8 + e]);
                            if (ADD) {
                                const uint32_t o[4] = {old[k].x, old[k].y, old[k].z, old[k].w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float2 f = unpack2(o[e], out_bf16);
                                    a[2 * e] += f.x;
                                    a[2 * e + 1] += f.y;
                                }
                            }
                            nv.x = pack2(a[0], a[1], out_bf16);
                            nv.y = pack2(a[2], a[3], out_bf16);
                            nv.z = pack2(a[4], a[5], out_bf16);
                            nv.w = pack2(a[6], a[7], out_bf16);
                        } else {
                            float a[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) a[e] = __uint_as_float(v[k * 4 + e]);
                            if (ADD) {
                                a[0] += __uint_as_float(old[k].x);
                                a[1] += __uint_as_float(old[k].y);
                                a[2] += __uint_as_float(old[k].z);
                                a[3] += __uint_as_float(old[k].w);
                            }
                            nv = make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                                            __float_as_uint(a[3]));
                        }
                        if (!tail) *reinterpret_cast<uint4*>(rowp + ((k ^ ri) * 16)) = nv;
                        else if (k < kvalid) grow[k] = nv;
                    }
                }
            }
            // accumulator no longer needed
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[as]));
            // make the shared-memory writes visible to the bulk-copy engine, then store
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int32_t xcol0 = (int32_t)col0;
                const int row_lo = max(lane0, 0), row_end = min(lane0 + 32, full_end);
                for (int c = k_copy; c < NCH; c += 1 << pc.rep_log) {
                    if (c * CC >= ncols) break;
                    for (int rr = row_lo; rr < row_end;) {
                        const int k = box_level(row_end - rr, 2);
                        tma_store_2d(&ymaps.m[pc.slice][k], xcol0 + c * CC, pc.blk_row0 + rr,
                                     smem_u32(ring + c * RING_STRIDE + (pc.pos + rr) * 128));
                        rr += GROUP << k;
                    }
                }
                bulk_commit();
                // release this piece's ring rows once the stores have read them
                bulk_wait_read<0>();
                mbar_arrive(smem_u32(&y_free[t % RING_PIECES]));
            }
            __syncwarp();
        }
        // the stores must have read shared memory before the CTA exits; the
        // writes themselves complete with the grid
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, NUM_ACC * BN);
}

// ====================================================================== host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

constexpr int SMEM_OPTIN = 232448;      // 227 KB per block on sm_100
constexpr int SMEM_STATIC_RESERVE = 1024;

inline int64_t elem_bytes(int dt) { return dt == SGMV_F32 ? 4 : 2; }
inline bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }
inline int32_t round_up(int32_t v, int32_t m) { return (v + m - 1) / m * m; }

struct Plan {
    Geometry geo;
    int smem_bytes;
    int grid;
    WMaps tw;
    CUtensorMap tx;
    YMaps ty;
    Slices sl;
};

// Scheduling weight of a piece = max(its 8-row groups of output, a floor) + a
// fixed part: its B tile's bytes in units of one group's output bytes, plus
// PIECE_FIXED_GROUPS for the per-piece pipeline work (MMA, barriers, TMA issue).
constexpr int PIECE_WEIGHT_FLOOR = 16;
constexpr int PIECE_FIXED_GROUPS = 0;

// Shared-memory layout: an output ring of at least 4, else 3, 2, 1 whole
// 128-row pieces, with the deepest B pipeline that leaves it room, after the
// segment table and the piece queue.  In add mode the ring also holds the old output loaded ahead of
// the epilogue, and the loads it can keep in flight set the pace: two B
// stages, the rest for the ring (measured on one B200, us per call, 2 B
// stages against the deepest that fits: rank-64 MLP 169.4 vs 178.3; QKV
// prefill and the decode-like mix unchanged; overwrite mode is better with the
// deep B pipeline).  A segment table too long for a ring of one piece leaves
// the call to the generic kernel.
inline bool layout_smem(Geometry& g, int32_t nseg, int32_t out_bytes, bool add, int* total_out) {
    const int sw_deep[] = {8, 6, 4, 3, 2};
    const int sw_two[] = {2};
    const int* sw_opts = add ? sw_two : sw_deep;
    const int n_sw = add ? 1 : 5;
    const int32_t row_bytes = g.bn * out_bytes;            // one ring row across all chunks
    const int num_acc = TMEM_COLS / g.bn;
    const int32_t seg_bytes = round_up(nseg * (int32_t)sizeof(SegEntry), 16);
    const int32_t q_bytes = QS * (int32_t)sizeof(PieceRec);
    const int32_t budget = SMEM_OPTIN - SMEM_STATIC_RESERVE - 1024;   // 1024: base alignment slack
    for (int prefer_rows : {4 * BM, 3 * BM, 2 * BM, BM}) {
        for (int si = 0; si < n_sw; ++si) {
            const int sw = sw_opts[si];
            g.stages_w = sw;
            g.stages_xo = 2;
            g.stages_xr = g.convert_x ? 1 : 0;
            const int n_bars = 2 * sw + 2 * g.stages_xo + 2 * g.stages_xr + 2 * num_acc + 2 * RING_PIECES + 2 * QS;
            const int32_t fixed = sw * g.w_bytes + g.stages_xo * g.xo_bytes + g.stages_xr * g.xr_bytes + seg_bytes +
                                  RING_PIECES * 4 + q_bytes + 8 * n_bars + 64;
            if (fixed >= budget) continue;
            const int32_t rows = ((budget - fixed) / row_bytes) & ~(GROUP - 1);
            if (rows < prefer_rows) continue;
            g.ring_rows = rows;
            int32_t off = 0;
            g.off_y = off;
            off += rows * row_bytes;
            g.off_w = off;
            off += sw * g.w_bytes;
            g.off_xo = off;
            off += g.stages_xo * g.xo_bytes;
            g.off_xr = off;
            off += g.stages_xr * g.xr_bytes;
            g.off_seg = off;
            off += seg_bytes;
            g.off_ends = off;
            off += RING_PIECES * 4;
            g.off_q = round_up(off, 16);
            off = g.off_q + q_bytes;
            g.off_bar = round_up(off, 8);
            off = g.off_bar + 8 * n_bars;
            const int total = off + 1024;
            if (total > SMEM_OPTIN - SMEM_STATIC_RESERVE) continue;
            *total_out = total;
            return true;
        }
    }
    return false;
}

// Conditions one slice must meet for the tensor-core kernel.
inline bool slice_ok(const Problem& p) {
    const int64_t sx = elem_bytes(p.x_dt), so = elem_bytes(p.out_dt);
    if (p.K < 8 || p.K > MAX_KP || p.K % 8 != 0) return false;
    if (p.x_cs != 1 || p.w_ks != 1) return false;
    if (p.x_rs < p.K || p.w_ns < p.K) return false;
    if ((p.x_rs * sx) % 16 || (p.w_ns * 2) % 16) return false;
    if (p.lora_num > 1 && ((p.w_as * 2) % 16 || p.w_as < p.N * p.w_ns)) return false;
    if (!aligned16(p.x) || !aligned16(p.w) || !aligned16(p.out)) return false;
    if ((p.H * so) % 16 || (p.off * so) % 16 || (p.N * so) % 16) return false;
    if (p.batches > SEG_CAP) return false;   // the shared-memory layout sets the real limit
    if (p.out_rows >= (int64_t(1) << 31) || p.x_rows >= (int64_t(1) << 31) || p.off + p.N >= (int64_t(1) << 31))
        return false;
    if (p.lora_num >= (int64_t(1) << 31)) return false;
    return true;
}

// Everything the tensor-core kernel needs for `nsl` slices of one output
// (sharing x, the metadata and the adapter count) with n-tiles of `bn`
// columns, or false if it cannot take the call.
inline bool make_plan_bn(const Problem* ps, int nsl, int sm_count, int bn, Plan* out) {
    if (nsl < 1 || nsl > MAX_SLICES) return false;
    const Problem& p = ps[0];
    for (int i = 0; i < nsl; ++i) {
        if (!slice_ok(ps[i]) || ps[i].w_dt != p.w_dt || ps[i].lora_num != p.lora_num) return false;
        if (ps[i].N == 0) return false;
    }
    const int64_t sx = elem_bytes(p.x_dt), so = elem_bytes(p.out_dt);
    Slices& sl = out->sl;
    sl.count = nsl;
    sl.tile0[0] = 0;
    for (int i = 0; i < nsl; ++i) {
        sl.off[i] = ps[i].off;
        sl.N[i] = ps[i].N;
        sl.tile0[i + 1] = sl.tile0[i] + (int32_t)((ps[i].N + bn - 1) / bn);
    }
    for (int i = nsl; i < MAX_SLICES; ++i) {
        sl.off[i] = 0;
        sl.N[i] = 0;
        sl.tile0[i + 1] = sl.tile0[i];
    }
    const int64_t n_tiles = sl.tile0[nsl];
    const int64_t t_lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    const int64_t max_pieces = (t_lim / BM + p.batches + 1) * n_tiles;
    const int64_t group_bytes = (int64_t)GROUP * bn * so * (p.add ? 2 : 1);
    const int64_t wfix = (bn * p.K * 2 + group_bytes - 1) / group_bytes + PIECE_FIXED_GROUPS;
    const int64_t weight_bound = (t_lim / GROUP + p.batches + 1) * n_tiles + (wfix + PIECE_WEIGHT_FLOOR) * max_pieces;
    if (weight_bound >= (int64_t(1) << 31)) return false;

    Geometry& g = out->geo;
    g.K = (int32_t)p.K;
    g.Kp = round_up((int32_t)p.K, 16);
    g.x_bytes = (int32_t)sx;
    g.convert_x = p.x_dt != p.w_dt;
    g.n_tiles = (int32_t)n_tiles;
    g.w_is_bf16 = p.w_dt == SGMV_BF16;
    g.wmin = PIECE_WEIGHT_FLOOR;
    g.bn = bn;
    // Pieces dealt across the CTAs (the kernel picks, see choose_mode) unless x
    // must be rounded to the weights' dtype: that is done once per x block, so
    // a CTA then takes contiguous pieces and keeps a block across its n-tiles.
    g.mode = g.convert_x ? (int32_t)sched::MODE_CONTIG : MODE_AUTO;
    g.wfix = (int32_t)wfix;
    // B tile: K in blocks of 64 columns, then at most one each of 32, 16, 8
    {
        int k0 = 0, off = 0, nb = 0;
        auto add_block = [&](int kb) {
            g.w_blk_k0[nb] = k0;
            g.w_blk_kb[nb] = kb;
            g.w_blk_off[nb] = off;
            off += round_up(bn * kb * 2, 1024);
            k0 += kb;
            ++nb;
        };
        while (p.K - k0 >= 64 && nb < MAX_WBLK) add_block(64);
        for (int kb : {32, 16, 8})
            if (p.K - k0 >= kb && nb < MAX_WBLK) add_block(kb);
        if (k0 != p.K) return false;
        g.w_nblk = nb;
        g.w_zero_off = -1;
        if (g.w_blk_kb[nb - 1] == 8) {   // the upper K half of the last MMA step reads zeros
            g.w_zero_off = off;
            off += bn * 16;
        }
        g.w_bytes = round_up(off, 1024);
        // B descriptors per K=16 step: swizzle code and 8-row stride follow the
        // block's row width (2*kb bytes); an 8-column block points its upper K
        // half at the zero chunk
        g.ksteps = 0;
        for (int b = 0; b < nb; ++b) {
            const int kb = g.w_blk_kb[b];
            const uint32_t layout = kb == 64 ? 2u : kb == 32 ? 4u : kb == 16 ? 6u : 0u;
            const uint32_t sbo = kb >= 16 ? (uint32_t)(8 * 2 * kb) : 128u;
            const uint32_t lbo = kb >= 16 ? 16u : (uint32_t)(g.w_zero_off - g.w_blk_off[b]);
            const int steps = kb >= 16 ? kb / 16 : 1;
            for (int st = 0; st < steps; ++st) {
                if (g.ksteps == MAX_KP / 16) return false;
                g.b_desc_rel[g.ksteps] = smem_desc(0, lbo, sbo, layout);
                g.b_off[g.ksteps] = (uint32_t)(g.w_blk_off[b] + st * 32);
                ++g.ksteps;
            }
        }
        if (g.ksteps != g.Kp / 16) return false;
    }
    g.xo_bytes = BM * g.Kp * 2;
    g.xr_bytes = round_up(BM * (int32_t)p.K * (int32_t)sx, 1024);
    if (!layout_smem(g, (int32_t)p.batches, (int32_t)so, p.add, &out->smem_bytes)) return false;

    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint32_t ones[5] = {1, 1, 1, 1, 1};
    // B: (K, N rows, adapters); one box per K block, rows of 2*kb bytes swizzled by their width
    for (int si = 0; si < nsl; ++si)
    for (int b = 0; b < g.w_nblk; ++b) {
        const Problem& p = ps[si];
        const cuuint64_t dims[3] = {(cuuint64_t)p.K, (cuuint64_t)p.N, (cuuint64_t)p.lora_num};
        cuuint64_t a_stride = (cuuint64_t)(p.w_as * 2);
        if (p.lora_num == 1) a_stride = (cuuint64_t)round_up((int32_t)(p.N * p.w_ns * 2), 16);
        const cuuint64_t strides[2] = {(cuuint64_t)(p.w_ns * 2), a_stride};
        const int kb = g.w_blk_kb[b];
        const cuuint32_t box[3] = {(cuuint32_t)kb, (cuuint32_t)bn, 1};
        const CUtensorMapSwizzle sw = kb == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                      : kb == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                      : kb == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                 : CU_TENSOR_MAP_SWIZZLE_NONE;
        if (enc(&out->tw.m[si][b], CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(p.w), dims, strides, box, ones,
                CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    if (g.convert_x) {
        // x in its own dtype: (K, rows) row-major, BM rows per box
        const cuuint64_t dims[2] = {(cuuint64_t)p.K, (cuuint64_t)p.x_rows};
        const cuuint64_t strides[1] = {(cuuint64_t)(p.x_rs * sx)};
        const cuuint32_t box[2] = {(cuuint32_t)p.K, (cuuint32_t)BM};
        const CUtensorMapDataType dt = sx == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
        if (enc(&out->tx, dt, 2, const_cast<void*>(p.x), dims, strides, box, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    } else {
        // x already in the weights' dtype: (8 elements, rows, K/8 chunks) -> K-major core matrices
        const cuuint64_t dims[3] = {8, (cuuint64_t)p.x_rows, (cuuint64_t)(p.K / 8)};
        const cuuint64_t strides[2] = {(cuuint64_t)(p.x_rs * 2), 16};
        const cuuint32_t box[3] = {8, (cuuint32_t)BM, (cuuint32_t)(p.K / 8)};
        if (enc(&out->tx, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(p.x), dims, strides, box, ones,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    // out: columns [0, off + N) of each row (clipping at the slice end); boxes of
    // 8 << k rows x 128 bytes with the 128-byte swizzle
    for (int si = 0; si < nsl; ++si)
    for (int k = 0; k < NUM_YMAPS; ++k) {
        const Problem& p = ps[si];
        const cuuint64_t dims[2] = {(cuuint64_t)(p.off + p.N), (cuuint64_t)p.out_rows};
        const cuuint64_t strides[1] = {(cuuint64_t)(p.H * so)};
        const cuuint32_t box[2] = {(cuuint32_t)(128 / so), (cuuint32_t)(GROUP << k)};
        const CUtensorMapDataType dt = so == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
        if (enc(&out->ty.m[si][k], dt, 2, p.out, dims, strides, box, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    int64_t grid = sm_count;
    if (max_pieces < grid) grid = max_pieces;
    out->grid = (int)(grid < 1 ? 1 : grid);
    return true;
}

// n-tile width of a call.  256-column pieces halve the per-piece work (MMA
// issue, barriers, TMA requests) and move 512 contiguous bytes of each output
// row, but a CTA then has half as many pieces, so its pipeline fill and its
// last piece weigh twice as much; B tiles of 256 rows also crowd the output
// ring at rank 64 and up.  Measured on one B200 (us per call, 128 vs 256):
// single-tenant long prefill 66.7 vs 52.0, decode-like mix 80.4 vs 64.7,
// QKV prefill 30.4 vs 33.9, rank-64 MLP 181 vs 277.  So 256 is taken for
// ranks up to 32 with x already in B's dtype when the estimated piece count
// gives every SM at least 16 pieces (overwrite) or 32 (add: loads of the old
// output also wait in the ring).
inline int choose_bn(const Problem* ps, int nsl, int sm_count) {
    const Problem& p = ps[0];
    if (p.K > 32 || p.x_dt != p.w_dt) return 128;
    const int64_t t_lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    int64_t tiles = 0;
    for (int i = 0; i < nsl; ++i) tiles += (ps[i].N + 255) / 256;
    const int64_t est = (t_lim / BM + p.batches) * tiles;
    return est >= (p.add ? 32 : 16) * (int64_t)sm_count ? 256 : 128;
}

// force_bn: 0 lets choose_bn decide; 128 or 256 fixes the width.
inline bool make_plan(const Problem* ps, int nsl, int sm_count, Plan* out, int force_bn = 0) {
    if (nsl < 1 || nsl > MAX_SLICES) return false;
    if (force_bn) return make_plan_bn(ps, nsl, sm_count, force_bn, out);
    if (choose_bn(ps, nsl, sm_count) == 256 && make_plan_bn(ps, nsl, sm_count, 256, out)) return true;
    return make_plan_bn(ps, nsl, sm_count, 128, out);
}

template <int OUT_DT, bool ADD, int BN>
int launch_instance(const Plan& pl, const Problem& p, cudaStream_t stream) {
    auto kern = tc_expand_slice_kernel<OUT_DT, ADD, BN>;
    static std::atomic<uint64_t> configured{0};
    if (!set_smem_limit_once(kern, SMEM_OPTIN - SMEM_STATIC_RESERVE, configured)) return SGMV_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = (size_t)pl.smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, pl.tw, pl.tx, pl.ty, p, pl.geo, pl.sl) != cudaSuccess) return SGMV_ERR_LAUNCH;
    return SGMV_OK;
}

// Plans of recent calls, keyed by every field of the call's slices (pointers,
// dtypes, shapes, strides, metadata, slice offsets and widths, add mode), the
// device, its SM count and the tile width asked for.
struct PlanKey {
    Problem ps[MAX_SLICES];
    int32_t nsl, device, sm_count, force_bn;
};

inline bool cached_plan(const Problem* ps, int nsl, int sm_count, int force_bn, Plan* out) {
    static PlanCache<PlanKey, Plan> cache;
    if (nsl < 1 || nsl > MAX_SLICES) return false;
    PlanKey key;
    std::memset(&key, 0, sizeof(key));
    for (int i = 0; i < nsl; ++i) std::memcpy(&key.ps[i], &ps[i], sizeof(Problem));
    key.nsl = nsl;
    key.sm_count = sm_count;
    key.force_bn = force_bn;
    if (cudaGetDevice(&key.device) != cudaSuccess) return false;
    return cache.get(key, out, [&](Plan* pl) { return make_plan(ps, nsl, sm_count, pl, force_bn); });
}

}  // namespace tc

bool tc_supports(const Problem* ps, int nsl, int sm_count, int force_bn) {
    tc::Plan pl;
    return tc::cached_plan(ps, nsl, sm_count, force_bn, &pl);
}

template <int BN>
int launch_bn(const tc::Plan& pl, const Problem& p, cudaStream_t stream) {
    switch (p.out_dt) {
        case SGMV_F32:
            return p.add ? tc::launch_instance<SGMV_F32, true, BN>(pl, p, stream)
                         : tc::launch_instance<SGMV_F32, false, BN>(pl, p, stream);
        case SGMV_BF16:
            return p.add ? tc::launch_instance<SGMV_BF16, true, BN>(pl, p, stream)
                         : tc::launch_instance<SGMV_BF16, false, BN>(pl, p, stream);
        default:
            return p.add ? tc::launch_instance<SGMV_F16, true, BN>(pl, p, stream)
                         : tc::launch_instance<SGMV_F16, false, BN>(pl, p, stream);
    }
}

int launch_tc(const Problem* ps, int nsl, int sm_count, cudaStream_t stream, int force_bn) {
    tc::Plan pl;
    if (!tc::cached_plan(ps, nsl, sm_count, force_bn, &pl)) return SGMV_ERR_VARIANT;
    const Problem& p = ps[0];
    return pl.geo.bn == 256 ? launch_bn<256>(pl, p, stream) : launch_bn<128>(pl, p, stream);
}

}  // namespace sgmv
