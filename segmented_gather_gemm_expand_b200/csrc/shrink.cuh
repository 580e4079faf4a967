// SGMV shrink on the tensor cores: the LoRA-A projection that produces the
// expand operation's input x.
//
//     out[r, n] = sum_h x[r, h] * A[a][n, h]      (r in segment b, a = lora_idx[b], n < rank)
//
// It is the segmented product of the expand operation with the shapes turned
// round: the reduction runs over the hidden size H (thousands) and the output
// row is `rank` wide.  A work item is (segment, 128-row block, split of H).
// H is cut into 64-column chunks; a pipeline stage holds up to four of them.
// Per chunk the producer warp TMA-loads the block's x rows (the rows the
// segment owns, in 8..128-row boxes, 128-byte swizzle) and A[a]'s rank x 64
// tile, all chunks of a stage at once: with one chunk per stage the x stream
// of the QKV shrink ran at about half the speed (a read-only TMA probe over a
// 4096-wide bf16 matrix: 16.6 us with one 128 x 64 box per stage against 8.3
// us with four neighbouring boxes per stage).  The MMA warp issues M=128,
// N=rank, K=16 tcgen05 MMAs into a TMEM accumulator; the four epilogue warps read the sums back (one row per
// thread) and either round them into out (one split) or store them as fp32
// partial sums in the caller's workspace, which shrink_reduce_kernel adds up
// in split order (deterministic) and rounds into out.
//
// One CTA per SM, 192 threads: warp 0 TMA producer, warp 1 MMA, warps 2-5
// epilogue.  Items are handed out round-robin, the items of full 128-row
// blocks first and those of the segments' partial last blocks after them, so
// that the last, incomplete round of the deal holds the smaller items
// (measured on the QKV shrink: 21.5 against 22.3 us with segment order).
// Every mbarrier wait is bounded and reports a timeout through the device
// error word.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "plan_cache.cuh"
#include "tc_ptx.cuh"

namespace sgmv {
namespace shr {

using namespace sgmv::tc;

constexpr int BM = 128;               // rows per block (TMEM lanes)
constexpr int CH = 64;                // H columns per chunk: 128-byte rows
constexpr int THREADS = 192;
constexpr int NUM_ACC = 2;
constexpr int SEG_CAP = 16384;        // most segments a launch takes (the shared-memory table decides below that)
constexpr int NUM_XMAPS = 5;          // x boxes of 8, 16, 32, 64, 128 rows
constexpr int MAX_RANK = 128;
constexpr int SMEM_LIMIT = 232448 - 1024;   // dynamic shared memory a CTA may opt in to on sm_100

struct SegRow {
    int32_t row0, rows, adapter;
    int32_t prefix;    // full 128-row blocks of earlier segments
    int32_t pprefix;   // earlier segments that end in a partial block
};

struct Geo {
    int32_t R;            // rank (MMA N): multiple of 16, 16..128
    int32_t acc_stride;   // TMEM columns between the accumulators (R rounded up to 32)
    int32_t nchunks;      // ceil(H / CH)
    int32_t splits, cps;  // H splits per block; chunks per split
    int32_t cpst;         // chunks per pipeline stage (1 to 4)
    int32_t stages, stage_bytes;
    int32_t off_seg, off_bar;
    int32_t tmem_cols;
    int64_t t_lim;        // rows of the workspace's row dimension (min of x and out rows)
};

struct XMaps {
    CUtensorMap m[NUM_XMAPS];
};

struct Item {
    int32_t row0, rows, adapter, split, ch0, ch1;
};

// Item `id` of the round-robin sequence: block id / splits, split id % splits.
// Blocks are numbered full ones first (segment order), then every segment's
// partial last block: the last, incomplete round of the deal then holds the
// smaller items, which evens out the CTAs' work.  full_blocks: all full blocks.
__device__ __forceinline__ void decode_item(const SegRow* segs, int32_t nseg, const Geo& g, int32_t full_blocks,
                                            int32_t id, Item& it) {
    const int32_t blk = id / g.splits;
    it.split = id - blk * g.splits;
    const bool partial = blk >= full_blocks;
    const int32_t key = partial ? blk - full_blocks : blk;
    int lo = 0, hi = nseg - 1;   // last segment whose prefix <= key (empty ones share their successor's)
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if ((partial ? segs[mid].pprefix : segs[mid].prefix) <= key) lo = mid;
        else hi = mid - 1;
    }
    const SegRow s = segs[lo];
    const int32_t rb = partial ? s.rows / BM : key - s.prefix;
    it.row0 = s.row0 + rb * BM;
    it.rows = min(BM, s.rows - rb * BM);
    it.adapter = s.adapter;
    it.ch0 = it.split * g.cps;
    it.ch1 = min(g.nchunks, it.ch0 + g.cps);
}

__device__ __forceinline__ int xbox_level(int rows) {   // rows: a positive multiple of 8
    const int k = 31 - __clz(rows / 8);
    return k < NUM_XMAPS - 1 ? k : NUM_XMAPS - 1;
}

template <int OUT_DT>
__global__ void __launch_bounds__(THREADS, 1)
shrink_kernel(const __grid_constant__ XMaps xmaps, const __grid_constant__ CUtensorMap amap, Problem p, Geo g,
              float* ws) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ int s_abort;
    __shared__ uint32_t s_tmem_base;
    __shared__ int32_t s_total_blocks, s_full_blocks;

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    SegRow* segs = reinterpret_cast<SegRow*>(smem + g.off_seg);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + g.off_bar);
    const int S = g.stages;
    uint64_t* full = bars;
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;
    uint64_t* acc_empty = acc_full + NUM_ACC;

    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < S; ++i) {
            mbar_init(smem_u32(&full[i]), 1);
            mbar_init(smem_u32(&empty[i]), 1);
        }
        for (int i = 0; i < NUM_ACC; ++i) {
            mbar_init(smem_u32(&acc_full[i]), 1);
            mbar_init(smem_u32(&acc_empty[i]), 4);     // the four epilogue warps
        }
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        for (int k = 0; k < NUM_XMAPS; ++k) prefetch_tmap(&xmaps.m[k]);
        prefetch_tmap(&amap);
    }
    if (warp == 1) tmem_alloc(smem_u32(&s_tmem_base), (uint32_t)g.tmem_cols);

    // Everything below may read memory written by the preceding kernel.
    grid_dependency_wait();
    // The reduction kernel (split H) may be scheduled now; it waits for this
    // grid to finish before it reads the partial sums.
    grid_dependents_launch();

    // Segment table (guards of sgmv.h applied), the prefix of full row blocks
    // and the count of partial last blocks before each segment.
    const int32_t nseg = (int32_t)p.batches;
    for (int32_t b = tid; b < nseg; b += THREADS) {
        const Segment s = load_segment(p, b);
        segs[b] = SegRow{(int32_t)s.row0, (int32_t)s.rows, (int32_t)s.adapter, 0, 0};
    }
    __syncthreads();
    if (warp == 0) {
        int32_t run_full = 0, run_part = 0;
        for (int32_t base = 0; base < nseg; base += 32) {
            const int32_t b = base + lane;
            const int32_t full = b < nseg ? segs[b].rows / BM : 0;
            const int32_t part = b < nseg ? (segs[b].rows % BM != 0) : 0;
            int32_t v = full, w = part;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t t = __shfl_up_sync(0xffffffffu, v, o);
                const int32_t u = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) {
                    v += t;
                    w += u;
                }
            }
            if (b < nseg) {
                segs[b].prefix = run_full + v - full;
                segs[b].pprefix = run_part + w - part;
            }
            run_full += __shfl_sync(0xffffffffu, v, 31);
            run_part += __shfl_sync(0xffffffffu, w, 31);
        }
        if (lane == 0) {
            s_full_blocks = run_full;
            s_total_blocks = run_full + run_part;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = s_tmem_base;
    const int32_t n_items = s_total_blocks * g.splits;
    const int32_t full_blocks = s_full_blocks;
    volatile int* abort_flag = &s_abort;
    const bool bf16 = p.w_dt == SGMV_BF16;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_x = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            uint32_t q = 0;
            Item it;
            bool ok = true;
            for (int32_t id = blockIdx.x; ok && id < n_items; id += gridDim.x) {
                decode_item(segs, nseg, g, full_blocks, id, it);
                const int rows8 = (it.rows + 7) & ~7;
                for (int32_t ch = it.ch0; ch < it.ch1; ch += g.cpst, ++q) {
                    const int nck = min(g.cpst, it.ch1 - ch);
                    const uint32_t s = q % S;
                    if (!mbar_wait(smem_u32(&empty[s]), ((q / S) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * g.stage_bytes;
                    uint8_t* sa = st + g.cpst * (BM * 128);
                    mbar_expect_tx(smem_u32(&full[s]), (uint32_t)(nck * (rows8 * 128 + g.R * 128)));
                    // the stage's chunks are requested together: neighbouring
                    // 128-byte pieces of each x row are then in flight at once
                    for (int j = 0; j < nck; ++j) {
                        for (int r = 0; r < rows8;) {
                            const int k = xbox_level(rows8 - r);
                            tma_load_2d(smem_u32(st + j * (BM * 128) + r * 128), &xmaps.m[k], (ch + j) * CH,
                                        it.row0 + r, smem_u32(&full[s]), pol_x);
                            r += 8 << k;
                        }
                        tma_load_3d(smem_u32(sa + j * g.R * 128), &amap, (ch + j) * CH, 0, it.adapter,
                                    smem_u32(&full[s]), pol_a);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        const uint32_t idesc = instr_desc_mn(bf16, BM, g.R);
        uint32_t q = 0, n = 0;
        Item it;
        for (int32_t id = blockIdx.x; id < n_items; id += gridDim.x, ++n) {
            decode_item(segs, nseg, g, full_blocks, id, it);
            const uint32_t acc = n % NUM_ACC;
            if (!warp_wait(smem_u32(&acc_empty[acc]), ((n / NUM_ACC) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
            tc_fence_after();
            bool ok = true;
            for (int32_t ch = it.ch0; ch < it.ch1; ch += g.cpst, ++q) {
                const int nck = min(g.cpst, it.ch1 - ch);
                const uint32_t s = q % S;
                if (!warp_wait(smem_u32(&full[s]), (q / S) & 1, abort_flag, DEVERR_TIMEOUT_MMA)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t st = smem_u32(smem + s * g.stage_bytes);
                    for (int j = 0; j < nck; ++j) {
                        const uint32_t xs = st + j * (BM * 128);
                        const uint32_t as = st + g.cpst * (BM * 128) + j * g.R * 128;
#pragma unroll
                        for (int kk = 0; kk < CH / 16; ++kk) {
                            const uint64_t ad = smem_desc(xs + kk * 32, 16, 1024, 2);
                            const uint64_t bd = smem_desc(as + kk * 32, 16, 1024, 2);
                            tc_mma(tmem_base + acc * (uint32_t)g.acc_stride, ad, bd, idesc,
                                   (ch > it.ch0 || j > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    tc_commit(smem_u32(&empty[s]));
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) tc_commit(smem_u32(&acc_full[acc]));
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quad = warp % 4;              // TMEM lane quadrant this warp may read
        const int r = quad * 32 + lane;         // block row of this thread
        uint32_t n = 0;
        Item it;
        for (int32_t id = blockIdx.x; id < n_items; id += gridDim.x, ++n) {
            decode_item(segs, nseg, g, full_blocks, id, it);
            const uint32_t acc = n % NUM_ACC;
            if (!warp_wait(smem_u32(&acc_full[acc]), (n / NUM_ACC) & 1, abort_flag, DEVERR_TIMEOUT_EPILOGUE)) break;
            tc_fence_after();
            const bool valid = r < it.rows;
            const int64_t row = (int64_t)it.row0 + r;
            const uint32_t taddr = tmem_base + acc * (uint32_t)g.acc_stride + ((uint32_t)(quad * 32) << 16);
            for (int c = 0; c < g.R; c += 16) {
                uint32_t v[16];
                tmem_ld16(taddr + (uint32_t)c, v);
                tmem_ld_wait();
                if (!valid) continue;
                if (g.splits > 1) {
                    float4* dst = reinterpret_cast<float4*>(ws + ((int64_t)it.split * g.t_lim + row) * g.R + c);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                             __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                } else if (OUT_DT == SGMV_F32) {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.H + c);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                             __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                } else {
                    constexpr bool ob = OUT_DT == SGMV_BF16;
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.H + c);
#pragma unroll
                    for (int j = 0; j < 2; ++j)
                        dst[j] = make_uint4(pack2(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1]), ob),
                                            pack2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]), ob),
                                            pack2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]), ob),
                                            pack2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]), ob));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[acc]));
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, (uint32_t)g.tmem_cols);
}

// Adds the splits' fp32 partial sums in split order and rounds each sum once
// into out.  A thread takes four neighbouring ranks of one row and issues the
// loads of every split before it adds them (the sums are latency-bound: a few
// MB that the main kernel has just written).  Grid: x = four-rank groups of a
// segment, y = segments (grid-stride).  It lets the next kernel start its
// prologue as soon as it runs.
constexpr int MAX_SPLITS = 16;

template <int OUT_DT>
__global__ void __launch_bounds__(256) shrink_reduce_kernel(Problem p, const float* ws, int splits, int64_t t_lim) {
    grid_dependency_wait();   // the partial sums of the preceding shrink_kernel grid
    grid_dependents_launch();
    const int64_t R = p.N;    // a multiple of 16
    const int64_t q = R / 4;
    const int64_t split_stride = t_lim * R;
    for (int64_t b = blockIdx.y; b < p.batches; b += gridDim.y) {
        const Segment s = load_segment(p, b);
        const int64_t n_vec = s.rows * q;
        for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n_vec; e += (int64_t)gridDim.x * blockDim.x) {
            const int64_t row = s.row0 + e / q, k = (e % q) * 4;
            const float4* src = reinterpret_cast<const float4*>(ws + row * R + k);
            float4 v[MAX_SPLITS];
#pragma unroll
            for (int sp = 0; sp < MAX_SPLITS; ++sp)
                if (sp < splits) v[sp] = src[sp * (split_stride / 4)];
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int sp = 0; sp < MAX_SPLITS; ++sp)
                if (sp < splits) {
                    acc.x += v[sp].x;
                    acc.y += v[sp].y;
                    acc.z += v[sp].z;
                    acc.w += v[sp].w;
                }
            if (OUT_DT == SGMV_F32) {
                *reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.H + k) = acc;
            } else {
                constexpr bool ob = OUT_DT == SGMV_BF16;
                *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.out) + row * p.H + k) =
                    make_uint2(pack2(acc.x, acc.y, ob), pack2(acc.z, acc.w, ob));
            }
        }
    }
}

// ====================================================================== host side

struct Plan {
    Geo geo;
    int smem_bytes;
    int grid;
    XMaps xm;
    CUtensorMap am;
};

// The splits a call would like (a power of two, at most 16 and at most the
// chunk count): the one that minimises the bytes the busiest SM moves, i.e.
// ceil(items / SMs) items of 128 x H/splits x 2 bytes of x, plus its share
// of the partial sums written and read back (2 x splits x rows x rank x 4
// bytes over all SMs), plus ITEM_FIXED_BYTES per item: each item refills the
// chunk pipeline and drains its accumulator, about one DRAM latency of one
// SM's share of the bandwidth.  The block count is estimated from the row
// count and the number of segments (each adds at most one partial block).
// Measured on one B200 for hidden 4096 -> rank 16 over 8772 rows (us per
// call by splits 1/2/4/8/16): 37.4, 24.0, 22.4, 23.8, 25.3; the model picks 4.
constexpr double ITEM_FIXED_BYTES = 64.0 * 1024.0;
inline int preferred_splits(const Problem& p, int sm_count) {
    const int64_t t_lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    const int64_t blocks = (t_lim + BM - 1) / BM + (p.batches < t_lim ? p.batches : t_lim);
    const int64_t nchunks = (p.K + CH - 1) / CH;
    const int64_t G = sm_count > 0 ? sm_count : 1;
    int best = 1;
    double best_cost = 0.0;
    for (int s = 1; s <= 16 && s <= nchunks; s *= 2) {
        const int64_t cps = (nchunks + s - 1) / s;
        const double items_per_sm = (double)((blocks * s + G - 1) / G);
        const double x_bytes = items_per_sm * BM * (double)cps * CH * 2.0;
        const double partial = s > 1 ? 2.0 * s * (double)t_lim * (double)p.N * 4.0 / (double)G : 0.0;
        const double cost = x_bytes + partial + items_per_sm * ITEM_FIXED_BYTES;
        if (s == 1 || cost < best_cost * 0.98) {   // more splits only for a clear gain
            best = s;
            best_cost = cost;
        }
    }
    return best;
}

inline int64_t workspace_bytes_for(const Problem& p, int splits) {
    if (splits <= 1) return 0;
    const int64_t t_lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    return (int64_t)splits * t_lim * p.N * (int64_t)sizeof(float);
}

inline bool supports(const Problem& p) {
    if (p.x_dt != p.w_dt) return false;                       // x is staged as it is: no rounding step
    if (p.N < 16 || p.N > MAX_RANK || p.N % 16) return false;
    if (p.K < 1 || p.K >= (int64_t(1) << 31)) return false;
    if (p.x_cs != 1 || p.w_ks != 1) return false;
    if ((p.x_rs * 2) % 16 || (p.w_ns * 2) % 16 || p.x_rs < p.K || p.w_ns < p.K) return false;
    if (p.lora_num > 1 && ((p.w_as * 2) % 16 || p.w_as < p.N * p.w_ns)) return false;
    if ((reinterpret_cast<uintptr_t>(p.x) & 15) || (reinterpret_cast<uintptr_t>(p.w) & 15) ||
        (reinterpret_cast<uintptr_t>(p.out) & 15))
        return false;
    if (p.out_rows >= (int64_t(1) << 31) || p.x_rows >= (int64_t(1) << 31) || p.lora_num >= (int64_t(1) << 31))
        return false;
    return true;
}

inline bool make_plan(const Problem& p, int sm_count, int splits, tc::EncodeTiledFn enc, Plan* out) {
    if (!supports(p) || !enc || p.batches > SEG_CAP) return false;
    Geo& g = out->geo;
    g.R = (int32_t)p.N;
    g.nchunks = (int32_t)((p.K + CH - 1) / CH);
    g.cps = (g.nchunks + splits - 1) / splits;
    g.splits = (g.nchunks + g.cps - 1) / g.cps;                 // every split gets at least one chunk
    if (g.splits > MAX_SPLITS) return false;
    g.t_lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    // A stage holds up to four chunks (x tiles, then the A tiles; every tile a
    // multiple of 1024 bytes since R % 16 == 0): the widest stage of which at
    // least two fit, then as many stages as fit, at most eight.
    g.stages = 0;
    for (g.cpst = g.cps < 4 ? g.cps : 4; g.cpst >= 1; g.cpst /= 2) {
        g.stage_bytes = g.cpst * (BM * 128 + g.R * 128);
        for (g.stages = 8; g.stages >= 2; --g.stages) {
            g.off_seg = g.stages * g.stage_bytes;
            g.off_bar = (g.off_seg + (int)p.batches * (int)sizeof(SegRow) + 15) & ~15;
            out->smem_bytes = g.off_bar + 8 * (2 * g.stages + 2 * NUM_ACC) + 1024;   // + base alignment slack
            if (out->smem_bytes <= SMEM_LIMIT) break;
        }
        if (g.stages >= 2) break;
    }
    if (g.cpst < 1 || g.stages < 2) return false;
    g.acc_stride = (g.R + 31) / 32 * 32;
    int cols = 32;
    while (cols < NUM_ACC * g.acc_stride) cols *= 2;
    g.tmem_cols = cols;

    const cuuint32_t ones[3] = {1, 1, 1};
    for (int k = 0; k < NUM_XMAPS; ++k) {
        const cuuint64_t dims[2] = {(cuuint64_t)p.K, (cuuint64_t)p.x_rows};
        const cuuint64_t strides[1] = {(cuuint64_t)(p.x_rs * 2)};
        const cuuint32_t box[2] = {(cuuint32_t)CH, (cuuint32_t)(8 << k)};
        if (enc(&out->xm.m[k], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(p.x), dims, strides, box, ones,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    {
        const cuuint64_t dims[3] = {(cuuint64_t)p.K, (cuuint64_t)p.N, (cuuint64_t)p.lora_num};
        cuuint64_t a_stride = (cuuint64_t)(p.w_as * 2);
        if (p.lora_num == 1) a_stride = (cuuint64_t)((p.N * p.w_ns * 2 + 15) / 16 * 16);
        const cuuint64_t strides[2] = {(cuuint64_t)(p.w_ns * 2), a_stride};
        const cuuint32_t box[3] = {(cuuint32_t)CH, (cuuint32_t)p.N, 1};
        if (enc(&out->am, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(p.w), dims, strides, box, ones,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    const int64_t blocks = (g.t_lim + BM - 1) / BM + (p.batches < g.t_lim ? p.batches : g.t_lim);
    int64_t grid = blocks * g.splits;
    if (grid > sm_count) grid = sm_count;
    out->grid = (int)(grid < 1 ? 1 : grid);
    return true;
}

// Plans of recent calls, keyed by every field of the problem, the device, its
// SM count and the split count.
struct PlanKey {
    Problem p;
    int32_t device, sm_count, splits;
};

inline bool cached_plan(const Problem& p, int sm_count, int splits, tc::EncodeTiledFn enc, Plan* out) {
    static PlanCache<PlanKey, Plan> cache;
    PlanKey key;
    std::memset(&key, 0, sizeof(key));
    std::memcpy(&key.p, &p, sizeof(Problem));
    key.sm_count = sm_count;
    key.splits = splits;
    if (cudaGetDevice(&key.device) != cudaSuccess) return false;
    return cache.get(key, out, [&](Plan* pl) { return make_plan(p, sm_count, splits, enc, pl); });
}

template <int OUT_DT>
int launch_dt(const Plan& pl, const Problem& p, float* ws, cudaStream_t stream) {
    auto kern = shrink_kernel<OUT_DT>;
    static std::atomic<uint64_t> configured{0};
    if (!set_smem_limit_once(kern, SMEM_LIMIT, configured)) return SGMV_ERR_CUDA;
    // Both kernels are launched with programmatic stream serialization: each
    // may start its prologue while the kernel before it drains, and waits
    // (griddepcontrol.wait) before it reads global memory.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = (size_t)pl.smem_bytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, pl.xm, pl.am, p, pl.geo, ws) != cudaSuccess) return SGMV_ERR_LAUNCH;
    if (pl.geo.splits > 1) {
        const int64_t rows_guess = (pl.geo.t_lim + p.batches - 1) / (p.batches > 0 ? p.batches : 1);
        int64_t gx = (rows_guess * (p.N / 4) + 255) / 256;
        if (gx < 1) gx = 1;
        if (gx > 1024) gx = 1024;
        cudaLaunchConfig_t rc = {};
        rc.gridDim = dim3((unsigned)gx, (unsigned)(p.batches < 65535 ? p.batches : 65535));
        rc.blockDim = dim3(256);
        rc.stream = stream;
        rc.attrs = attr;
        rc.numAttrs = 1;
        if (cudaLaunchKernelEx(&rc, shrink_reduce_kernel<OUT_DT>, p, (const float*)ws, (int)pl.geo.splits,
                               (int64_t)pl.geo.t_lim) != cudaSuccess)
            return SGMV_ERR_LAUNCH;
    }
    return SGMV_OK;
}

}  // namespace shr
}  // namespace sgmv
