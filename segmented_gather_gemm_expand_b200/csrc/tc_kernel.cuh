// Tensor-core SGMV expand-slice for sm_100a: tcgen05 MMA with the accumulator
// in tensor memory, TMA staging of B, x and the output slice.
//
// Data flow of one CTA (persistent, one per SM, 192 threads):
//
//   warp 0  producer   TMA: B[a] n-tile (once per (segment, n-tile) block),
//                      the x rows of each piece, and (add mode) the output
//                      tile.  Output rows in whole groups of 8 use 2-D
//                      tensor boxes (8 rows x 128 B, 128-byte swizzle); the
//                      last <8 rows of a segment use 1-D bulk copies per row,
//                      so nothing outside the segment's rows is touched.
//   warp 1  MMA        rounds x to the weights' dtype into the MMA operand
//                      layout (rank zero-padded to a multiple of 16), then
//                      one elected lane issues tcgen05.mma (M=128 rows,
//                      N=128 columns, K=16 per instruction) into one of two
//                      TMEM accumulators.
//   warps 2-5 epilogue each owns 32 TMEM lanes (= 32 rows of the tile):
//                      tcgen05.ld the fp32 accumulators, add the old output
//                      (add mode), round once to the output dtype, write the
//                      tile back in place in shared memory, and TMA-store it.
//
// Work is expanded on the device: every CTA builds the table of segments in
// shared memory (guards of sgmv.h applied), counts work units of 8 rows x one
// 128-column n-tile, and takes an equal contiguous range of units; units are
// ordered (segment, n-tile, row group) so the staged B tile is reused over
// all the rows of the range.  Every wait on an mbarrier is bounded; a wait
// that gives up sets the device error word and makes the CTA leave its loops.
#pragma once

#include <cuda.h>

#include <atomic>

#include "common.cuh"

namespace sgmv {

__device__ void raise_device_error(int32_t bits);

namespace tc {

constexpr int BM = 128;               // rows per MMA tile (TMEM lanes)
constexpr int BN = 128;               // columns per n-tile (TMEM columns per accumulator)
constexpr int GROUP = 8;              // rows per work unit
constexpr int MAX_GROUPS = BM / GROUP;
constexpr int THREADS = 192;
constexpr int EPI_WARP0 = 2;
constexpr int SEG_CAP = 1024;         // segments held in shared memory
constexpr int NUM_ACC = 2;            // TMEM accumulators
constexpr int NUM_XOP = 2;            // MMA operand buffers for x
constexpr int NUM_W = 2;              // B tile buffers
constexpr int MAX_KP = 128;           // largest padded rank
constexpr unsigned long long WAIT_LIMIT_CYCLES = 4000000000ull;   // ~2 s

struct SegEntry {
    int32_t row0;
    int32_t rows;
    int32_t adapter;
    int32_t prefix;     // units before this segment
};

// Geometry fixed per launch (host computes; kernel parameter).
struct Geometry {
    int32_t K;          // rank
    int32_t Kp;         // rank padded to a multiple of 16
    int32_t x_bytes;    // element size of x
    int32_t out_bytes;  // element size of out
    int32_t chunk_cols; // output columns per 128-byte chunk
    int32_t n_tiles;    // ceil(N / BN)
    int32_t stages_y;
    int32_t stages_x;
    int32_t w_is_bf16;
    int32_t add;
    // shared memory offsets (bytes, from the 1024-aligned base)
    int32_t off_y, off_xraw, off_xop, off_w, off_seg, off_bar;
    int32_t y_stage_bytes, xraw_stage_bytes, xop_bytes, w_bytes;
};

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait.  Returns false (after raising `err`) if the phase did not
// complete in time or another role of the CTA already gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t err) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > WAIT_LIMIT_CYCLES) {
            *abort_flag = 1;
            raise_device_error(err);
            return false;
        }
    }
}

// The same wait executed by all 32 lanes; the outcome is made warp-uniform so
// that no lane leaves a loop its neighbours stay in.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t err) {
    const bool ok = mbar_wait(bar, parity, abort_flag, err);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int32_t c0, int32_t c1, uint32_t bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void* tmap, int32_t c0, int32_t c1, int32_t c2,
                                            int32_t c3, uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_store_2d(const void* tmap, int32_t c0, int32_t c1, uint32_t src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(c0), "r"(c1), "r"(src)
                 : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(dst)),
                 "r"(src), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// tcgen05 --------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major, no swizzle: 8-row x 16-byte core
// matrices; `lbo` = byte distance between the two 16-byte K halves of one
// K=16 step, `sbo` = byte distance between consecutive 8-row groups.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;   // descriptor version for sm_100
    return d;                 // base offset 0, absolute LBO mode, layout SWIZZLE_NONE (0)
}

// Instruction descriptor of kind::f16: fp32 accumulator, A/B both f16 or
// both bf16, both K-major, M = BM, N = BN.
__host__ __device__ constexpr uint32_t instr_desc(bool bf16) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((uint32_t)(BN >> 3) << 17) |
           ((uint32_t)(BM >> 4) << 24);
}

// ---------------------------------------------------------------- numeric helpers

__device__ __forceinline__ float half_bits_to_float(uint32_t h, bool bf16) {
    if (bf16) return __uint_as_float(h << 16);
    return __half2float(__ushort_as_half((unsigned short)h));
}

__device__ __forceinline__ uint32_t float_to_half_bits(float v, bool bf16) {
    if (bf16) return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
    return (uint32_t)__half_as_ushort(__float2half_rn(v));
}

__device__ __forceinline__ uint32_t pack2(float a, float b, bool bf16) {
    if (bf16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack2(uint32_t u, bool bf16) {
    if (bf16) return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    __half2 h = *reinterpret_cast<__half2*>(&u);
    return __half22float2(h);
}

// ---------------------------------------------------------------- scheduler

// Walks the CTA's contiguous range [u, u_end) of work units.  Every role runs
// an identical copy, so all roles see the same sequence of pieces.
struct Piece {
    int32_t seg;
    int32_t row0;         // first row of out / x
    int32_t nrows;        // 1 .. BM
    int32_t n0;           // first column within the slice
    int32_t adapter;
    bool new_block;       // first piece of a (segment, n-tile) block in this CTA
    bool last_in_block;   // last piece of that block in this CTA
};

struct Walker {
    const SegEntry* segs;
    int32_t n_tiles;
    int32_t i, j, g;      // segment, n-tile, row group
    int32_t u, u_end;
    bool fresh;

    __device__ bool next(Piece& p) {
        if (u >= u_end) return false;
        const SegEntry s = segs[i];
        const int32_t gpb = (s.rows + GROUP - 1) / GROUP;
        int32_t cnt = gpb - g;
        if (cnt > MAX_GROUPS) cnt = MAX_GROUPS;
        if (cnt > u_end - u) cnt = u_end - u;
        p.seg = i;
        p.row0 = s.row0 + g * GROUP;
        p.nrows = min((g + cnt) * GROUP, s.rows) - g * GROUP;
        p.n0 = j * BN;
        p.adapter = s.adapter;
        p.new_block = fresh;
        u += cnt;
        g += cnt;
        const bool block_done = (g == gpb);
        p.last_in_block = block_done || (u >= u_end);
        fresh = block_done;
        if (block_done) {
            g = 0;
            if (++j == n_tiles) {
                j = 0;
                // advance to the next segment with work
                do {
                    ++i;
                } while (u < u_end && segs[i].rows == 0);
            }
        }
        return true;
    }
};

// ---------------------------------------------------------------- the kernel

template <int OUT_BYTES, bool ADD>
__global__ void __launch_bounds__(THREADS, 1)
tc_expand_slice_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_y, Problem p, Geometry geo) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    __shared__ int s_abort;
    __shared__ uint32_t s_tmem_base;
    __shared__ int32_t s_total_units;
    __shared__ int32_t s_warp_sums[THREADS / 32];

    const int tid = threadIdx.x;
    const int warp = tid / 32;
    const int lane = tid % 32;

    SegEntry* segs = reinterpret_cast<SegEntry*>(smem + geo.off_seg);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + geo.off_bar);
    // barrier layout
    const int SY = geo.stages_y, SX = geo.stages_x;
    uint64_t* w_full = bars;
    uint64_t* w_empty = w_full + NUM_W;
    uint64_t* x_full = w_empty + NUM_W;
    uint64_t* x_empty = x_full + SX;
    uint64_t* xop_empty = x_empty + SX;
    uint64_t* acc_full = xop_empty + NUM_XOP;
    uint64_t* acc_empty = acc_full + NUM_ACC;
    uint64_t* y_full = acc_empty + NUM_ACC;
    uint64_t* y_empty = y_full + SY;

    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < NUM_W; ++i) {
            mbar_init(smem_u32(&w_full[i]), 1);
            mbar_init(smem_u32(&w_empty[i]), 1);
        }
        for (int i = 0; i < SX; ++i) {
            mbar_init(smem_u32(&x_full[i]), 1);
            mbar_init(smem_u32(&x_empty[i]), 1);
        }
        for (int i = 0; i < NUM_XOP; ++i) mbar_init(smem_u32(&xop_empty[i]), 1);
        for (int i = 0; i < NUM_ACC; ++i) {
            mbar_init(smem_u32(&acc_full[i]), 1);
            mbar_init(smem_u32(&acc_empty[i]), 4);
        }
        for (int i = 0; i < SY; ++i) {
            mbar_init(smem_u32(&y_full[i]), 1);
            mbar_init(smem_u32(&y_empty[i]), 4);
        }
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_x);
        prefetch_tmap(&tmap_y);
    }
    if (warp == 1) tmem_alloc(smem_u32(&s_tmem_base), NUM_ACC * BN);

    // Zero the rank-padding chunks of the B buffers (TMA never writes them).
    {
        const int kc_real = geo.K / 8, kc_pad = geo.Kp / 8;
        for (int b = 0; b < NUM_W; ++b) {
            uint8_t* wb = smem + geo.off_w + b * geo.w_bytes;
            for (int i = tid; i < (kc_pad - kc_real) * BN; i += THREADS) {
                const int kc = kc_real + i / BN, n = i % BN;
                *reinterpret_cast<uint4*>(wb + kc * BN * 16 + n * 16) = make_uint4(0, 0, 0, 0);
            }
        }
    }

    // Segment table: guards of the API applied, units counted, exclusive scan.
    const int64_t batches = p.batches;
    int32_t running = 0;
    for (int64_t base = 0; base < batches; base += THREADS) {
        const int64_t b = base + tid;
        int32_t units = 0;
        SegEntry e{0, 0, 0, 0};
        if (b < batches) {
            const Segment s = load_segment(p, b);
            e.row0 = (int32_t)s.row0;
            e.rows = (int32_t)s.rows;
            e.adapter = (int32_t)s.adapter;
            units = ((e.rows + GROUP - 1) / GROUP) * geo.n_tiles;
        }
        // block-wide inclusive scan of `units`
        int32_t v = units;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += t;
        }
        if (lane == 31) s_warp_sums[warp] = v;
        __syncthreads();
        int32_t warp_off = 0, total = 0;
        for (int w = 0; w < THREADS / 32; ++w) {
            if (w < warp) warp_off += s_warp_sums[w];
            total += s_warp_sums[w];
        }
        e.prefix = running + warp_off + v - units;
        if (b < batches) segs[b] = e;
        running += total;
        __syncthreads();
    }
    if (tid == 0) s_total_units = running;

    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = s_tmem_base;
    const int32_t U = s_total_units;
    const int32_t u0 = (int32_t)(((int64_t)U * blockIdx.x) / gridDim.x);
    const int32_t u1 = (int32_t)(((int64_t)U * (blockIdx.x + 1)) / gridDim.x);

    Walker walk;
    walk.segs = segs;
    walk.n_tiles = geo.n_tiles;
    walk.u = u0;
    walk.u_end = u1;
    walk.fresh = true;
    walk.i = 0;
    walk.j = 0;
    walk.g = 0;
    if (u0 < u1) {
        // last segment whose prefix <= u0
        int lo = 0, hi = (int)batches - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (segs[mid].prefix <= u0) lo = mid;
            else hi = mid - 1;
        }
        while (segs[lo].rows == 0) ++lo;   // never past a segment with work (u0 < U)
        const int32_t gpb = (segs[lo].rows + GROUP - 1) / GROUP;
        const int32_t local = u0 - segs[lo].prefix;
        walk.i = lo;
        walk.j = local / gpb;
        walk.g = local % gpb;
    }

    volatile int* abort_flag = &s_abort;
    const bool w_bf16 = geo.w_is_bf16 != 0;
    constexpr int CHUNK_COLS = 128 / OUT_BYTES;          // columns per 128-byte row chunk
    constexpr int CHUNKS = BN / CHUNK_COLS;              // chunks per n-tile
    constexpr int CHUNK_STRIDE = BM * 128;               // bytes per chunk column of a stage

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_stream = policy_evict_first();
            const uint64_t pol_keep = policy_evict_last();
            Piece pc;
            int32_t t = 0, wb = 0;
            const uint32_t w_box_bytes = (uint32_t)(BN * geo.K * 2);
            const uint32_t x_box_bytes = (uint32_t)(BM * geo.K * geo.x_bytes);
            while (walk.next(pc)) {
                if (pc.new_block) {
                    const int s = wb % NUM_W;
                    if (!mbar_wait(smem_u32(&w_empty[s]), ((wb / NUM_W) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_PRODUCER))
                        break;
                    mbar_expect_tx(smem_u32(&w_full[s]), w_box_bytes);
                    tma_load_4d(smem_u32(smem + geo.off_w + s * geo.w_bytes), &tmap_w, 0, pc.n0, 0, pc.adapter,
                                smem_u32(&w_full[s]), pol_keep);
                }
                {
                    const int s = t % SX;
                    if (!mbar_wait(smem_u32(&x_empty[s]), ((t / SX) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_PRODUCER))
                        break;
                    mbar_expect_tx(smem_u32(&x_full[s]), x_box_bytes);
                    tma_load_2d(smem_u32(smem + geo.off_xraw + s * geo.xraw_stage_bytes), &tmap_x, 0, pc.row0,
                                smem_u32(&x_full[s]), pol_keep);
                }
                if (ADD) {
                    const int s = t % SY;
                    if (!mbar_wait(smem_u32(&y_empty[s]), ((t / SY) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_PRODUCER))
                        break;
                    const int full_groups = pc.nrows / GROUP;
                    const int tail = pc.nrows - full_groups * GROUP;
                    const int ncols = min(BN, (int)(p.N - pc.n0));
                    const int nch = (ncols + CHUNK_COLS - 1) / CHUNK_COLS;
                    uint32_t bytes = (uint32_t)(full_groups * nch * 1024);
                    for (int c = 0; c < nch; ++c)
                        bytes += (uint32_t)(tail * min(CHUNK_COLS, ncols - c * CHUNK_COLS) * OUT_BYTES);
                    const uint32_t bar = smem_u32(&y_full[s]);
                    mbar_expect_tx(bar, bytes);
                    const uint32_t stage = smem_u32(smem + geo.off_y + s * geo.y_stage_bytes);
                    const int32_t xcol0 = (int32_t)(p.off + pc.n0);
                    for (int c = 0; c < nch; ++c) {
                        for (int g = 0; g < full_groups; ++g)
                            tma_load_2d(stage + c * CHUNK_STRIDE + g * 1024, &tmap_y, xcol0 + c * CHUNK_COLS,
                                        pc.row0 + g * GROUP, bar, pol_stream);
                        const uint32_t tb = (uint32_t)(min(CHUNK_COLS, ncols - c * CHUNK_COLS) * OUT_BYTES);
                        for (int r = full_groups * GROUP; r < pc.nrows; ++r) {
                            const char* src = reinterpret_cast<const char*>(p.out) +
                                              ((int64_t)(pc.row0 + r) * p.H + p.off + pc.n0 + c * CHUNK_COLS) *
                                                  OUT_BYTES;
                            bulk_load(stage + c * CHUNK_STRIDE + (r / GROUP) * 1024 + (r % GROUP) * 128, src, tb,
                                      bar, pol_stream);
                        }
                    }
                }
                if (pc.last_in_block) ++wb;
                ++t;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ x conversion + MMA
        Piece pc;
        int32_t t = 0, wb = 0;
        const uint32_t idesc = instr_desc(w_bf16);
        const int kc_real = geo.K / 8, kc_pad = geo.Kp / 8;
        const int x_row_bytes = geo.K * geo.x_bytes;
        while (walk.next(pc)) {
            const int ws = wb % NUM_W;
            if (pc.new_block) {
                if (!warp_wait(smem_u32(&w_full[ws]), (wb / NUM_W) & 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
            }
            const int xs = t % SX;
            if (!warp_wait(smem_u32(&x_full[xs]), (t / SX) & 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
            const int xo = t % NUM_XOP;
            if (!warp_wait(smem_u32(&xop_empty[xo]), ((t / NUM_XOP) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
            // x (raw dtype, row-major) -> weights' dtype, K-major no-swizzle core matrices
            const uint8_t* xraw = smem + geo.off_xraw + xs * geo.xraw_stage_bytes;
            uint8_t* xop = smem + geo.off_xop + xo * geo.xop_bytes;
            for (int q = lane; q < BM * kc_pad; q += 32) {
                const int m = q % BM, kc = q / BM;
                uint4 outv = make_uint4(0, 0, 0, 0);
                if (kc < kc_real) {
                    float f[8];
                    const uint8_t* src = xraw + m * x_row_bytes + kc * 8 * geo.x_bytes;
                    if (geo.x_bytes == 4) {
                        const float4 a = *reinterpret_cast<const float4*>(src);
                        const float4 b = *reinterpret_cast<const float4*>(src + 16);
                        f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
                    } else {
                        const uint4 a = *reinterpret_cast<const uint4*>(src);
                        const uint32_t u[4] = {a.x, a.y, a.z, a.w};
                        const bool xbf = p.x_dt == SGMV_BF16;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            f[2 * e] = half_bits_to_float(u[e] & 0xFFFFu, xbf);
                            f[2 * e + 1] = half_bits_to_float(u[e] >> 16, xbf);
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
            if (lane == 0) mbar_arrive(smem_u32(&x_empty[xs]));
            const int as = t % NUM_ACC;
            if (!warp_wait(smem_u32(&acc_empty[as]), ((t / NUM_ACC) & 1) ^ 1, abort_flag, DEVERR_TIMEOUT_MMA)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t a_base = smem_u32(xop);
                const uint32_t b_base = smem_u32(smem + geo.off_w + ws * geo.w_bytes);
                const uint32_t d = tmem_base + (uint32_t)(as * BN);
                for (int ks = 0; ks < geo.Kp / 16; ++ks) {
                    const uint64_t ad = smem_desc(a_base + ks * 2 * (BM * 16), BM * 16, 128);
                    const uint64_t bd = smem_desc(b_base + ks * 2 * (BN * 16), BN * 16, 128);
                    tc_mma(d, ad, bd, idesc, ks > 0 ? 1u : 0u);
                }
                tc_commit(smem_u32(&acc_full[as]));
                tc_commit(smem_u32(&xop_empty[xo]));
                if (pc.last_in_block) tc_commit(smem_u32(&w_empty[ws]));
            }
            __syncwarp();
            if (pc.last_in_block) ++wb;
            ++t;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp % 4;                  // TMEM lane quadrant of this warp
        const int r = q * 32 + lane;             // tile row of this thread
        const int grp = r / GROUP, ri = r % GROUP;
        const bool out_bf16 = p.out_dt == SGMV_BF16;
        Piece pc;
        int32_t t = 0;
        while (walk.next(pc)) {
            const int as = t % NUM_ACC;
            const int ys = t % SY;
            if (!warp_wait(smem_u32(&acc_full[as]), (t / NUM_ACC) & 1, abort_flag, DEVERR_TIMEOUT_EPILOGUE)) break;
            tc_fence_after();
            if (ADD) {
                if (!warp_wait(smem_u32(&y_full[ys]), (t / SY) & 1, abort_flag, DEVERR_TIMEOUT_EPILOGUE)) break;
            } else {
                // at most one of this warp's stores (the previous tile's, another
                // stage) may still be reading shared memory
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
            }
            const int nrows = pc.nrows;
            const int nrows8 = nrows & ~(GROUP - 1);
            const int ncols = min(BN, (int)(p.N - pc.n0));
            const int nch = (ncols + CHUNK_COLS - 1) / CHUNK_COLS;
            const bool valid = r < nrows;
            const bool swz = r < nrows8;         // rows in whole groups came through the swizzled boxes
            uint8_t* stage = smem + geo.off_y + ys * geo.y_stage_bytes;
            const uint32_t taddr = tmem_base + (uint32_t)(as * BN) + ((uint32_t)(q * 32) << 16);
            for (int c = 0; c < CHUNKS; ++c) {
                if (c >= nch) break;             // warp-uniform
                uint8_t* rowp = stage + c * CHUNK_STRIDE + grp * 1024 + ri * 128;
                constexpr int SUB = CHUNK_COLS / 32;  // 32-column TMEM loads per chunk
#pragma unroll
                for (int h = 0; h < SUB; ++h) {
                    uint32_t v[32];
                    tmem_ld32(taddr + (uint32_t)(c * CHUNK_COLS + h * 32), v);
                    tmem_ld_wait();
                    if (valid) {
                        if (OUT_BYTES == 2) {
                            // 32 columns = 64 bytes = four 16-byte pieces
#pragma unroll
                            for (int k4 = 0; k4 < 4; ++k4) {
                                const int lc = h * 4 + k4;
                                const int pcn = swz ? (lc ^ ri) : lc;
                                uint4* ptr = reinterpret_cast<uint4*>(rowp + pcn * 16);
                                float a[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) a[e] = __uint_as_float(v[k4 * 8 + e]);
                                if (ADD) {
                                    const uint4 old = *ptr;
                                    const uint32_t o[4] = {old.x, old.y, old.z, old.w};
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        const float2 f = unpack2(o[e], out_bf16);
                                        a[2 * e] += f.x;
                                        a[2 * e + 1] += f.y;
                                    }
                                }
                                uint4 nv;
                                nv.x = pack2(a[0], a[1], out_bf16);
                                nv.y = pack2(a[2], a[3], out_bf16);
                                nv.z = pack2(a[4], a[5], out_bf16);
                                nv.w = pack2(a[6], a[7], out_bf16);
                                *ptr = nv;
                            }
                        } else {
                            // fp32 out: 32 columns = 128 bytes = eight 16-byte pieces
#pragma unroll
                            for (int k8 = 0; k8 < 8; ++k8) {
                                const int pcn = swz ? (k8 ^ ri) : k8;
                                float4* ptr = reinterpret_cast<float4*>(rowp + pcn * 16);
                                float4 a = make_float4(__uint_as_float(v[k8 * 4 + 0]), __uint_as_float(v[k8 * 4 + 1]),
                                                       __uint_as_float(v[k8 * 4 + 2]), __uint_as_float(v[k8 * 4 + 3]));
                                if (ADD) {
                                    const float4 old = *ptr;
                                    a.x += old.x, a.y += old.y, a.z += old.z, a.w += old.w;
                                }
                                *ptr = a;
                            }
                        }
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
                const int32_t xcol0 = (int32_t)(p.off + pc.n0);
                const int r_lo = q * 32, r_hi = min(q * 32 + 32, nrows);
                for (int c = 0; c < nch; ++c) {
                    for (int g = r_lo / GROUP; g * GROUP < min(r_hi, nrows8); ++g)
                        tma_store_2d(&tmap_y, xcol0 + c * CHUNK_COLS, pc.row0 + g * GROUP,
                                     smem_u32(stage + c * CHUNK_STRIDE + g * 1024));
                    const uint32_t tb = (uint32_t)(min(CHUNK_COLS, ncols - c * CHUNK_COLS) * OUT_BYTES);
                    for (int rr = max(r_lo, nrows8); rr < r_hi; ++rr) {
                        char* dst = reinterpret_cast<char*>(p.out) +
                                    ((int64_t)(pc.row0 + rr) * p.H + p.off + pc.n0 + c * CHUNK_COLS) * OUT_BYTES;
                        bulk_store(dst, smem_u32(stage + c * CHUNK_STRIDE + (rr / GROUP) * 1024 + (rr % GROUP) * 128),
                                   tb);
                    }
                }
                bulk_commit();
                if (ADD) {
                    // release the previous tile's stage once its store has read it
                    bulk_wait_read<1>();
                    if (t > 0) mbar_arrive(smem_u32(&y_empty[(t - 1) % SY]));
                }
            }
            __syncwarp();
            ++t;
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, NUM_ACC * BN);
}

}  // namespace tc
}  // namespace sgmv

// ====================================================================== host side

#include <mutex>

namespace sgmv {
namespace tc {

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

constexpr int SMEM_LIMIT = 232448;   // 227 KB opt-in per block on sm_100

inline int64_t elem_bytes(int dt) { return dt == SGMV_F32 ? 4 : 2; }
inline bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }
inline int32_t round_up(int32_t v, int32_t m) { return (v + m - 1) / m * m; }

struct Plan {
    Geometry geo;
    int smem_bytes;
    int grid;
    CUtensorMap tw, tx, ty;
};

// Everything the tensor-core kernel needs, or false if it cannot take the call.
inline bool make_plan(const Problem& p, int sm_count, Plan* out) {
    const int64_t sx = elem_bytes(p.x_dt), so = elem_bytes(p.out_dt);
    if (p.K < 8 || p.K > MAX_KP || p.K % 8 != 0) return false;
    if (p.x_cs != 1 || p.w_ks != 1) return false;
    if (p.x_rs < p.K || p.w_ns < p.K) return false;
    if ((p.x_rs * sx) % 16 || (p.w_ns * 2) % 16) return false;
    if (p.lora_num > 1 && ((p.w_as * 2) % 16 || p.w_as < p.N * p.w_ns)) return false;
    if (!aligned16(p.x) || !aligned16(p.w) || !aligned16(p.out)) return false;
    if ((p.H * so) % 16 || (p.off * so) % 16 || (p.N * so) % 16) return false;
    if (p.batches > SEG_CAP) return false;
    if (p.out_rows >= (int64_t(1) << 31) || p.x_rows >= (int64_t(1) << 31) || p.off + p.N >= (int64_t(1) << 32))
        return false;
    if (p.lora_num >= (int64_t(1) << 31)) return false;
    const int64_t n_tiles = (p.N + BN - 1) / BN;
    const int64_t t_lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    const int64_t unit_bound = (t_lim / GROUP + p.batches + 1) * n_tiles;
    if (unit_bound >= (int64_t(1) << 31)) return false;

    Geometry& g = out->geo;
    g.K = (int32_t)p.K;
    g.Kp = round_up((int32_t)p.K, 16);
    g.x_bytes = (int32_t)sx;
    g.out_bytes = (int32_t)so;
    g.chunk_cols = (int32_t)(128 / so);
    g.n_tiles = (int32_t)n_tiles;
    g.w_is_bf16 = p.w_dt == SGMV_BF16;
    g.add = p.add;
    g.y_stage_bytes = BM * BN * (int32_t)so;
    g.xraw_stage_bytes = round_up(BM * (int32_t)p.K * (int32_t)sx, 1024);
    g.xop_bytes = BM * g.Kp * 2;
    g.w_bytes = BN * g.Kp * 2;
    const int32_t seg_bytes = round_up((int32_t)p.batches * (int32_t)sizeof(SegEntry), 16);
    bool ok = false;
    // Prefer deep output pipelines; shrink until the plan fits.
    const int sy_opts[] = {4, 3, 2};
    const int sx_opts[] = {3, 2};
    for (int sy : sy_opts) {
        for (int sxs : sx_opts) {
            g.stages_y = sy;
            g.stages_x = sxs;
            int32_t off = 0;
            g.off_y = off;
            off += sy * g.y_stage_bytes;
            g.off_xraw = off;
            off += sxs * g.xraw_stage_bytes;
            g.off_xop = off;
            off += NUM_XOP * g.xop_bytes;
            g.off_w = off;
            off += NUM_W * g.w_bytes;
            g.off_seg = off;
            off += seg_bytes;
            g.off_bar = round_up(off, 8);
            off = g.off_bar + 8 * (2 * NUM_W + 2 * sxs + NUM_XOP + 2 * NUM_ACC + 2 * sy);
            const int total = off + 1024;   // alignment slack for the 1024-byte base
            if (total <= SMEM_LIMIT - 1024) {   // static shared variables live in the same budget
                out->smem_bytes = total;
                ok = true;
                break;
            }
        }
        if (ok) break;
    }
    if (!ok) return false;

    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint32_t ones[4] = {1, 1, 1, 1};
    // B: (8 elements, N rows, K/8 chunks, adapters) -> K-major core matrices in shared memory
    {
        const cuuint64_t dims[4] = {8, (cuuint64_t)p.N, (cuuint64_t)(p.K / 8), (cuuint64_t)p.lora_num};
        cuuint64_t a_stride = (cuuint64_t)(p.w_as * 2);
        if (p.lora_num == 1) a_stride = (cuuint64_t)round_up((int32_t)(p.N * p.w_ns * 2), 16);
        const cuuint64_t strides[3] = {(cuuint64_t)(p.w_ns * 2), 16, a_stride};
        const cuuint32_t box[4] = {8, (cuuint32_t)BN, (cuuint32_t)(p.K / 8), 1};
        if (enc(&out->tw, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(p.w), dims, strides, box, ones,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    // x: (K, rows) row-major, BM rows per box
    {
        const cuuint64_t dims[2] = {(cuuint64_t)p.K, (cuuint64_t)p.x_rows};
        const cuuint64_t strides[1] = {(cuuint64_t)(p.x_rs * sx)};
        const cuuint32_t box[2] = {(cuuint32_t)p.K, (cuuint32_t)BM};
        const CUtensorMapDataType dt = sx == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
        if (enc(&out->tx, dt, 2, const_cast<void*>(p.x), dims, strides, box, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    // out: columns [0, off + N) of each row (clipping at the slice end), 8-row boxes of 128 bytes
    {
        const cuuint64_t dims[2] = {(cuuint64_t)(p.off + p.N), (cuuint64_t)p.out_rows};
        const cuuint64_t strides[1] = {(cuuint64_t)(p.H * so)};
        const cuuint32_t box[2] = {(cuuint32_t)(128 / so), (cuuint32_t)GROUP};
        const CUtensorMapDataType dt = so == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
        if (enc(&out->ty, dt, 2, p.out, dims, strides, box, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    int64_t grid = sm_count;
    if (unit_bound < grid) grid = unit_bound;
    out->grid = (int)(grid < 1 ? 1 : grid);
    return true;
}

template <int OUT_BYTES, bool ADD>
int launch_instance(const Plan& pl, const Problem& p, cudaStream_t stream) {
    auto kern = tc_expand_slice_kernel<OUT_BYTES, ADD>;
    static std::atomic<int> configured{0};
    if (configured.load() < pl.smem_bytes) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_LIMIT - 1024) !=
            cudaSuccess)
            return SGMV_ERR_CUDA;
        configured.store(SMEM_LIMIT - 1024);
    }
    kern<<<pl.grid, THREADS, pl.smem_bytes, stream>>>(pl.tw, pl.tx, pl.ty, p, pl.geo);
    return cudaGetLastError() == cudaSuccess ? SGMV_OK : SGMV_ERR_LAUNCH;
}

}  // namespace tc

inline int tc_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return n;
}

bool tc_supports(const Problem& p) {
    tc::Plan pl;
    return tc::make_plan(p, 148, &pl);
}

int launch_tc(const Problem& p, int sm_count, cudaStream_t stream) {
    tc::Plan pl;
    if (!tc::make_plan(p, sm_count, &pl)) return SGMV_ERR_VARIANT;
    if (pl.geo.out_bytes == 4) {
        return p.add ? tc::launch_instance<4, true>(pl, p, stream) : tc::launch_instance<4, false>(pl, p, stream);
    }
    return p.add ? tc::launch_instance<2, true>(pl, p, stream) : tc::launch_instance<2, false>(pl, p, stream);
}

}  // namespace sgmv
