// Row-balanced SGMV shrink: the LoRA-A projection of a prefill batch in one
// launch, with no split of the hidden size and no partial sums.
//
//     out[r, n] = sum_h x[r, h] * A[a][n, h]      (r in segment b, a = lora_idx[b], n < rank)
//
// The rows of all segments are cut into 8-row groups (a segment's last group
// may be partial), numbered in segment order, and CTA c of G takes groups
// [c * total / G, (c + 1) * total / G): every CTA reads the same number of x
// bytes (to one group), so none waits on a heavier neighbour, and every
// output row is summed by one CTA over the whole hidden size (deterministic,
// one rounding).
//
// A CTA owns its rows, so nothing else reads them at the same time: each
// pipeline stage therefore holds CQ consecutive 64-column chunks of the tile's
// rows, loaded back to back, so that every row is read in runs of CQ * 128
// bytes instead of 128-byte pieces a whole x row apart (one DRAM page opened
// per 128 bytes runs at a third of the bandwidth).  CTA c starts at chunk
// (c * CQ) mod nchunks and wraps around, so the CTAs do not all read the same
// columns at once.
//
// A CTA walks its groups in tiles of up to TR rows (64 or 128) made of at most
// PMAX parts, a part being the tile's groups of one segment.  Per 64-column
// chunk of H the producer warp TMA-loads every part's rows into the tile's x
// stage (at the part's row offset, 128-byte swizzle) and every part's A[a]
// rank x 64 tile; the MMA warp issues, for each part, M=128, N=rank, K=16
// tcgen05 MMAs over the WHOLE staged tile into that part's TMEM accumulator,
// so TMEM lane r of accumulator p holds row r of the tile against part p's
// adapter; the four epilogue warps then give each row the sums of its own
// part, round once and store them.  Rows of the tile that belong to no part
// compute garbage that is never read.  With TR = 64 the M=128 operand reads
// 64 rows past the tile, which lie in the next x stage or, for the last one,
// in the A tiles after it: shared memory of this CTA, never written back.
//
// One CTA per SM, 192 threads: warp 0 TMA producer, warp 1 MMA, warps 2-5
// epilogue.  Every mbarrier wait is bounded and reports a timeout through the
// device error word.
#pragma once

#include "shrink.cuh"

namespace sgmv {
namespace shr {

constexpr int RB_THREADS = 192;
constexpr int RB_MAX_STAGES = 16;
constexpr int RB_PMAX = 2;            // parts (segments) per tile
constexpr int RB_SEG_CAP = 16384;
constexpr int RB_CQ = 4;              // most 64-column chunks per pipeline stage

struct RowGeo {
    int32_t R;            // rank (MMA N): multiple of 16, 16..128
    int32_t nchunks;      // ceil(H / CH)
    int32_t tr;           // rows of a tile: 64 or 128
    int32_t stages;
    int32_t cq;           // chunks per stage
    int32_t x_bytes;      // tr * 128: one chunk's x tile
    int32_t a_bytes;      // R * 128: one part's A tile (one chunk)
    int32_t stage_x;      // cq * x_bytes: x tiles of one stage (chunk j at j * x_bytes)
    int32_t stage_a;      // cq * RB_PMAX * a_bytes: A tiles of one stage (chunk j, part p at (j * RB_PMAX + p) * a_bytes)
    int32_t off_a;        // A tiles of every stage, after the x tiles of every stage
    int32_t nstages_tile; // stages of one tile: ceil(nchunks / cq)
    int32_t off_seg, off_bar;
    int32_t acc_cols;     // TMEM columns of one accumulator set (RB_PMAX * R)
    int32_t tmem_cols;
};

struct Part {
    int32_t row0;         // first row (of x and out)
    int32_t rows;         // rows of the part that belong to its segment
    int32_t groups;       // 8-row groups loaded (the last may run past the segment)
    int32_t goff;         // first group of the part within the tile
    int32_t adapter;
};

struct Tile {
    int32_t n;
    Part p[RB_PMAX];
};

// The tiles of one CTA: its groups [g, g_end) in order, cut at RB_PMAX parts
// or tr rows.  Every role runs its own copy.
struct TileWalk {
    const SegRow* segs;   // prefix = 8-row groups of earlier segments
    int32_t nseg, s, g, g_end, tr_groups;

    __device__ __forceinline__ int32_t groups_of(int32_t i) const { return (segs[i].rows + 7) / 8; }

    __device__ __forceinline__ void init(const SegRow* sg, int32_t n, int32_t g0, int32_t g1, int32_t tr) {
        segs = sg;
        nseg = n;
        g = g0;
        g_end = g1;
        tr_groups = tr / 8;
        int32_t lo = 0, hi = n - 1;   // last segment whose prefix <= g0
        while (lo < hi) {
            const int32_t mid = (lo + hi + 1) / 2;
            if (segs[mid].prefix <= g0) lo = mid;
            else hi = mid - 1;
        }
        s = lo;
    }

    __device__ __forceinline__ bool next(Tile& t) {
        t.n = 0;
        int32_t used = 0;
#pragma unroll
        for (int k = 0; k < RB_PMAX; ++k) {   // unrolled: the parts stay in registers
            if (g >= g_end || used >= tr_groups) break;
            while (s < nseg && g >= segs[s].prefix + groups_of(s)) ++s;
            if (s >= nseg) break;
            const int32_t gl = g - segs[s].prefix;
            const int32_t take = min(min(g_end - g, groups_of(s) - gl), tr_groups - used);
            Part& p = t.p[k];
            p.row0 = segs[s].row0 + gl * 8;
            p.rows = min(take * 8, segs[s].rows - gl * 8);
            p.groups = take;
            p.goff = used;
            p.adapter = segs[s].adapter;
            g += take;
            used += take;
            t.n = k + 1;
        }
        return t.n > 0;
    }
};

template <int OUT_DT>
__global__ void __launch_bounds__(RB_THREADS, 1)
shrink_rows_kernel(const __grid_constant__ XMaps xmaps, const __grid_constant__ CUtensorMap amap, Problem p,
                   RowGeo g) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ int s_abort;
    __shared__ uint32_t s_tmem_base;
    __shared__ int32_t s_total_groups;

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
    // Warm L2 with the metadata while the preceding kernel may still run.
    for (int32_t b = tid; b < (int32_t)p.batches; b += RB_THREADS) {
        for (const MetaVec* m : {&p.start, &p.len, &p.idx}) {
            if (m->dtype != SGMV_I32 && m->dtype != SGMV_I64) continue;
            const int64_t esz = m->dtype == SGMV_I64 ? 8 : 4;
            prefetch_l2(static_cast<const char*>(m->ptr) + b * m->stride * esz);
        }
    }

    // Everything below may read memory written by the preceding kernel.
    grid_dependency_wait();
    grid_dependents_launch();

    // Segment table (guards of sgmv.h applied) and the prefix of 8-row groups.
    const int32_t nseg = (int32_t)p.batches;
    for (int32_t b = tid; b < nseg; b += RB_THREADS) {
        const Segment s = load_segment(p, b);
        segs[b] = SegRow{(int32_t)s.row0, (int32_t)s.rows, (int32_t)s.adapter, 0};
    }
    __syncthreads();
    if (warp == 0) {
        int32_t running = 0;
        for (int32_t base = 0; base < nseg; base += 32) {
            const int32_t b = base + lane;
            const int32_t groups = b < nseg ? (segs[b].rows + 7) / 8 : 0;
            int32_t v = groups;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t t = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += t;
            }
            if (b < nseg) segs[b].prefix = running + v - groups;
            running += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) s_total_groups = running;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = s_tmem_base;
    const int32_t total = s_total_groups;
    const int32_t g0 = (int32_t)(((int64_t)total * blockIdx.x) / gridDim.x);
    const int32_t g1 = (int32_t)(((int64_t)total * (blockIdx.x + 1)) / gridDim.x);
    volatile int* abort_flag = &s_abort;
    const bool bf16 = p.w_dt == SGMV_BF16;
    TileWalk walk;
    walk.init(segs, nseg, g0, g1, g.tr);
    Tile t;
    const int32_t ch_first = (int32_t)((blockIdx.x * (unsigned)g.cq) % (unsigned)g.nchunks);   // this CTA's first chunk

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_x = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            uint32_t q = 0;
            bool ok = true;
            while (ok && walk.next(t)) {
                uint32_t chunk_bytes = (uint32_t)(t.n * g.a_bytes);
#pragma unroll
                for (int i = 0; i < RB_PMAX; ++i)
                    if (i < t.n) chunk_bytes += (uint32_t)(t.p[i].groups * 8 * 128);
                for (int32_t k = 0; k < g.nstages_tile; ++k, ++q) {
                    const uint32_t s = q % S;
                    if (!mbar_wait(smem_u32(&empty[s]), ((q / S) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    const int32_t i0 = k * g.cq, i1 = min(g.nchunks, i0 + g.cq);
                    mbar_expect_tx(smem_u32(&full[s]), chunk_bytes * (uint32_t)(i1 - i0));
                    for (int32_t i = i0; i < i1; ++i) {
                        const int32_t ch = (ch_first + i) % g.nchunks;
                        uint8_t* xs = smem + s * g.stage_x + (i - i0) * g.x_bytes;
                        uint8_t* as = smem + g.off_a + s * g.stage_a + (i - i0) * RB_PMAX * g.a_bytes;
#pragma unroll
                        for (int pi = 0; pi < RB_PMAX; ++pi) {
                            if (pi >= t.n) break;
                            const Part& pt = t.p[pi];
                            for (int r = 0; r < pt.groups * 8;) {
                                const int kb = xbox_level(pt.groups * 8 - r);
                                tma_load_2d(smem_u32(xs + (pt.goff * 8 + r) * 128), &xmaps.m[kb], ch * CH, pt.row0 + r,
                                            smem_u32(&full[s]), pol_x);
                                r += 8 << kb;
                            }
                            tma_load_3d(smem_u32(as + pi * g.a_bytes), &amap, ch * CH, 0, pt.adapter,
                                        smem_u32(&full[s]), pol_a);
                        }
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        const uint32_t idesc = instr_desc_mn(bf16, BM, g.R);
        uint32_t q = 0, n = 0;
        bool ok = true;
        while (ok && walk.next(t)) {
            const uint32_t acc = n % NUM_ACC;
            if (!warp_wait(smem_u32(&acc_empty[acc]), ((n / NUM_ACC) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
            tc_fence_after();
            for (int32_t k = 0; k < g.nstages_tile; ++k, ++q) {   // chunks (ch_first + i) % nchunks
                const uint32_t s = q % S;
                if (!warp_wait(smem_u32(&full[s]), (q / S) & 1, abort_flag, DEVERR_TIMEOUT_MMA)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const int32_t i0 = k * g.cq, i1 = min(g.nchunks, i0 + g.cq);
                    for (int32_t i = i0; i < i1; ++i) {
                        const uint32_t xs = smem_u32(smem + s * g.stage_x + (i - i0) * g.x_bytes);
                        const uint32_t as = smem_u32(smem + g.off_a + s * g.stage_a + (i - i0) * RB_PMAX * g.a_bytes);
#pragma unroll
                        for (int pi = 0; pi < RB_PMAX; ++pi) {
                            if (pi >= t.n) break;
#pragma unroll
                            for (int kk = 0; kk < CH / 16; ++kk) {
                                const uint64_t ad = smem_desc(xs + kk * 32, 16, 1024, 2);
                                const uint64_t bd = smem_desc(as + pi * g.a_bytes + kk * 32, 16, 1024, 2);
                                tc_mma(tmem_base + acc * (uint32_t)g.acc_cols + (uint32_t)(pi * g.R), ad, bd, idesc,
                                       (i > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                    }
                    tc_commit(smem_u32(&empty[s]));
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) tc_commit(smem_u32(&acc_full[acc]));
            __syncwarp();
            ++n;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quad = warp % 4;              // TMEM lane quadrant this warp may read
        const int r = quad * 32 + lane;         // tile row of this thread
        uint32_t n = 0;
        while (walk.next(t)) {
            const uint32_t acc = n % NUM_ACC;
            if (!warp_wait(smem_u32(&acc_full[acc]), (n / NUM_ACC) & 1, abort_flag, DEVERR_TIMEOUT_EPILOGUE)) break;
            tc_fence_after();
            int mine = -1;
            int64_t row = 0;
#pragma unroll
            for (int i = 0; i < RB_PMAX; ++i) {
                if (i >= t.n) break;
                const int lo = t.p[i].goff * 8;
                if (r >= lo && r < lo + t.p[i].rows) {
                    mine = i;
                    row = (int64_t)t.p[i].row0 + (r - lo);
                }
            }
#pragma unroll
            for (int i = 0; i < RB_PMAX; ++i) {   // warp-uniform: every lane takes part in each load
                if (i >= t.n) break;
                if (!__any_sync(0xffffffffu, mine == i)) continue;
                const uint32_t taddr =
                    tmem_base + acc * (uint32_t)g.acc_cols + (uint32_t)(i * g.R) + ((uint32_t)(quad * 32) << 16);
                for (int c = 0; c < g.R; c += 16) {
                    uint32_t v[16];
                    tmem_ld16(taddr + (uint32_t)c, v);
                    tmem_ld_wait();
                    if (mine != i) continue;
                    if (OUT_DT == SGMV_F32) {
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
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[acc]));
            ++n;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, (uint32_t)g.tmem_cols);
}

// ====================================================================== host side

struct RowPlan {
    RowGeo geo;
    int smem_bytes;
    int grid;
    XMaps xm;
    CUtensorMap am;
};

// The row-balanced kernel takes a call when every CTA gets at least two
// groups' worth of rows on average and segments are long enough that a tile
// holds few of them (prefill batches); decode-like batches of a few rows per
// segment keep the split-H kernel, which spreads H over the SMs instead.
// rows_layout fills the geometry and shared-memory size, or returns false.
inline bool rows_layout(const Problem& p, int sm_count, RowGeo& g, int* smem_bytes) {
    if (!supports(p) || sm_count < 1) return false;
    const int64_t t_lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    if (p.batches > RB_SEG_CAP || p.batches < 1) return false;
    if (t_lim < 16 * (int64_t)sm_count || t_lim < 32 * p.batches) return false;
    g.R = (int32_t)p.N;
    g.nchunks = (int32_t)((p.K + CH - 1) / CH);
    g.tr = t_lim / sm_count <= 64 ? 64 : 128;
    g.x_bytes = g.tr * 128;
    g.a_bytes = g.R * 128;                          // a multiple of 1024: R % 16 == 0
    const int32_t seg_bytes = ((int32_t)p.batches * (int32_t)sizeof(SegRow) + 15) & ~15;
    // chunks per stage: the most (up to RB_CQ) that still leaves at least 3 stages
    for (g.cq = RB_CQ; g.cq >= 1; g.cq /= 2) {
        g.stage_x = g.cq * g.x_bytes;
        g.stage_a = g.cq * RB_PMAX * g.a_bytes;
        for (g.stages = RB_MAX_STAGES; g.stages >= 2; --g.stages) {
            g.off_a = g.stages * g.stage_x;
            g.off_seg = g.off_a + g.stages * g.stage_a;
            g.off_bar = g.off_seg + seg_bytes;
            *smem_bytes = g.off_bar + 8 * (2 * g.stages + 2 * NUM_ACC) + 1024;   // + base alignment slack
            if (*smem_bytes <= SMEM_LIMIT) break;
        }
        if (g.stages >= 3 || (g.cq == 1 && g.stages >= 2)) break;
    }
    if (g.cq < 1 || g.stages < 2) return false;
    g.nstages_tile = (g.nchunks + g.cq - 1) / g.cq;
    // the M=128 operand of the last chunk of the last stage reads BM - tr rows past its tile: the A tiles cover them
    if (g.stages * g.stage_a < (BM - g.tr) * 128) return false;
    g.acc_cols = RB_PMAX * g.R;
    int cols = 32;
    while (cols < NUM_ACC * g.acc_cols) cols *= 2;
    g.tmem_cols = cols;
    return cols <= 512;
}

inline bool rows_kernel_fits(const Problem& p, int sm_count) {
    RowGeo g;
    int smem = 0;
    return rows_layout(p, sm_count, g, &smem);
}

inline bool make_rows_plan(const Problem& p, int sm_count, tc::EncodeTiledFn enc, RowPlan* out) {
    if (!enc || !rows_layout(p, sm_count, out->geo, &out->smem_bytes)) return false;
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
    out->grid = sm_count;
    return true;
}

template <int OUT_DT>
int launch_rows_dt(const RowPlan& pl, const Problem& p, cudaStream_t stream) {
    auto kern = shrink_rows_kernel<OUT_DT>;
    static std::atomic<uint64_t> configured{0};
    if (!set_smem_limit_once(kern, SMEM_LIMIT, configured)) return SGMV_ERR_CUDA;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.grid);
    cfg.blockDim = dim3(RB_THREADS);
    cfg.dynamicSmemBytes = (size_t)pl.smem_bytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, pl.xm, pl.am, p, pl.geo) == cudaSuccess ? SGMV_OK : SGMV_ERR_LAUNCH;
}

}  // namespace shr
}  // namespace sgmv
