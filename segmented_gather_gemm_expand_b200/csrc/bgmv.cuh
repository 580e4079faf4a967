// BGMV expand-slice: one token per row, each with its own adapter.
//
// The decode counterpart of the expand-slice operation: row b gets
// out[b, off:off+N] (+)= x^[b, :] . B[idx[b]]^T.  With one row per adapter use
// there is no B tile to reuse across rows, so nothing is staged: every thread
// streams the two B rows of its two output columns with 16-byte loads
// (consecutive threads read consecutive rows, so a warp reads one contiguous
// stretch of B).  A row's loads -- its B rows, its x row and, in add mode, the
// old output -- are all issued before the first of them is used, so a row
// costs one memory round trip per 32 ranks, and the register budget leaves
// room for eight CTAs per SM, so enough loads are in flight to cover DRAM
// latency.  When x is already in B's dtype
// each thread reads x's row directly (16-byte loads, served from L1); other x
// dtypes are rounded to B's dtype once per row into shared memory.  Products
// are summed in fp32 in k order and the result (plus the old value in add
// mode) is rounded once.
//
// Grid: x = 256-column tile of the slice, y = rows (grid-stride).  The kernel
// is launched as a programmatic dependent launch and waits for the preceding
// kernel's memory before its first global read.
#pragma once

#include "common.cuh"

namespace sgmv {

constexpr int BGMV_THREADS = 128;
constexpr int BGMV_COLS = 2 * BGMV_THREADS;   // columns per CTA
constexpr int BGMV_MAX_K = 256;
constexpr int BGMV_KC = 32;                   // ranks per round trip
constexpr int BGMV_MIN_CTAS = 8;              // CTAs per SM the register budget must allow

// Element e (0..7) of 8 packed 16-bit values as a float.
__device__ __forceinline__ float half8_elem(const uint4& v, int e, bool bf16) {
    const uint32_t w = e < 2 ? v.x : e < 4 ? v.y : e < 6 ? v.z : v.w;
    const uint32_t h = (e & 1) ? (w >> 16) : (w & 0xFFFFu);
    return bf16 ? __uint_as_float(h << 16) : __half2float(__ushort_as_half((unsigned short)h));
}

// XVEC: x has B's dtype, unit column stride and 16-byte aligned rows.
template <int OUT_DT, bool ADD, bool XVEC>
__global__ void __launch_bounds__(BGMV_THREADS, BGMV_MIN_CTAS)
bgmv_expand_kernel(Problem p) {
    __shared__ float sx[BGMV_MAX_K];
    const int tid = threadIdx.x;
    const bool w_bf16 = p.w_dt == SGMV_BF16;
    const int64_t n = (int64_t)blockIdx.x * BGMV_COLS + 2 * tid;   // first of this thread's two columns
    const int64_t lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    const int K = (int)p.K;
    const bool mine = n < p.N;
    const bool two = n + 1 < p.N;

    asm volatile("griddepcontrol.wait;" ::: "memory");   // launched as a programmatic dependent launch
    for (int64_t b = blockIdx.y; b < p.batches; b += gridDim.y) {
        const int64_t a = load_meta(p.idx, b);
        if (a < 0 || a >= p.lora_num || b >= lim) continue;     // uniform across the CTA
        const int64_t oi = b * p.H + p.off + n;
        float old0 = 0.f, old1 = 0.f;
        if (ADD && mine) {
            old0 = load_elem(p.out, OUT_DT, oi);
            if (two) old1 = load_elem(p.out, OUT_DT, oi + 1);
        }
        if (!XVEC) {
            __syncthreads();   // the previous row's sx is no longer read
            for (int k = tid; k < K; k += BGMV_THREADS)
                sx[k] = round_to(load_elem(p.x, p.x_dt, b * p.x_rs + k * p.x_cs), p.w_dt);
            __syncthreads();
        }
        if (!mine) continue;
        const uint4* w0 = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.w) + a * p.w_as + n * p.w_ns);
        const uint4* w1 = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.w) + a * p.w_as +
                                                         (two ? n + 1 : n) * p.w_ns);
        const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + b * p.x_rs);
        float acc0 = 0.f, acc1 = 0.f;
        for (int k0 = 0; k0 < K; k0 += BGMV_KC) {
            const int kn = min(BGMV_KC, K - k0) / 8;   // 16-byte pieces in this round trip
            uint4 v0[BGMV_KC / 8], v1[BGMV_KC / 8], vx[BGMV_KC / 8];
#pragma unroll
            for (int j = 0; j < BGMV_KC / 8; ++j) {
                if (j < kn) {
                    v0[j] = __ldg(w0 + k0 / 8 + j);
                    v1[j] = __ldg(w1 + k0 / 8 + j);
                    if (XVEC) vx[j] = __ldg(xr + k0 / 8 + j);
                }
            }
#pragma unroll
            for (int j = 0; j < BGMV_KC / 8; ++j) {
                if (j < kn) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float xv = XVEC ? half8_elem(vx[j], e, w_bf16) : sx[k0 + j * 8 + e];
                        acc0 = fmaf(xv, half8_elem(v0[j], e, w_bf16), acc0);
                        acc1 = fmaf(xv, half8_elem(v1[j], e, w_bf16), acc1);
                    }
                }
            }
        }
        store_elem(p.out, OUT_DT, oi, ADD ? old0 + acc0 : acc0);
        if (two) store_elem(p.out, OUT_DT, oi + 1, ADD ? old1 + acc1 : acc1);
    }
}

// ----------------------------------------------------------------------------
// Coalesced variant for ranks that are powers of two (8 .. 256).  A warp load
// of the kernel above touches 32 different 128-byte lines (thread t reads its
// own two B rows), so the L1 tag stage, not DRAM, sets its pace.  Here a warp
// covers 64 B rows of the CTA's 256 and every one of its 16-byte loads reads
// 512 contiguous bytes: K/8 threads share a row, each taking one 16-byte chunk
// (eight ranks), and the row's sum is completed with shuffles.  The 256 sums
// go through shared memory to coalesced output stores; in add mode the old
// values of the thread's two output columns are loaded with the B rows, before
// any of them is used.  (Two token rows per CTA step, with both rows' loads in
// flight, measured slower: the register cost halves the CTAs an SM holds.)
template <int OUT_DT, bool ADD>
__global__ void __launch_bounds__(BGMV_THREADS)
bgmv_coalesced_kernel(Problem p) {
    __shared__ float res[BGMV_COLS];
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const bool w_bf16 = p.w_dt == SGMV_BF16;
    const int K = (int)p.K;
    const int tpr = K / 8;                      // threads per B row (1 .. 32)
    const int rpi = 32 / tpr;                   // rows per warp load
    const int chunk = lane % tpr;               // this thread's 16-byte chunk of a row
    const int64_t n0 = (int64_t)blockIdx.x * BGMV_COLS;
    const int64_t lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    const uint16_t* wbase = static_cast<const uint16_t*>(p.w);
    const int loads = 64 / rpi;                 // warp loads covering the warp's 64 rows

    asm volatile("griddepcontrol.wait;" ::: "memory");   // launched as a programmatic dependent launch
    for (int64_t b = blockIdx.y; b < p.batches; b += gridDim.y) {
        const int64_t a = load_meta(p.idx, b);
        if (a < 0 || a >= p.lora_num || b >= lim) continue;     // uniform across the CTA
        const int64_t oi = b * p.H + p.off + n0;
        float old[2] = {0.f, 0.f};   // add mode: the old values of columns tid and tid + BGMV_THREADS
        if (ADD) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = tid + h * BGMV_THREADS;
                if (n0 + c < p.N) old[h] = load_elem(p.out, OUT_DT, oi + c);
            }
        }
        // this thread's eight ranks of x, rounded to B's dtype
        float xv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) xv[e] = round_to(load_elem(p.x, p.x_dt, b * p.x_rs + (chunk * 8 + e) * p.x_cs), p.w_dt);
        const uint16_t* wa = wbase + a * p.w_as;
        for (int l0 = 0; l0 < loads; l0 += 8) {
            uint4 v[8];
            float part[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t r = n0 + warp * 64 + (int64_t)(l0 + u) * rpi + lane / tpr;
                v[u] = make_uint4(0, 0, 0, 0);
                if (l0 + u < loads && r < p.N)
                    v[u] = __ldg(reinterpret_cast<const uint4*>(wa + r * p.w_ns) + chunk);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float acc = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) acc = fmaf(xv[e], half8_elem(v[u], e, w_bf16), acc);
                part[u] = acc;
            }
            for (int o = tpr / 2; o >= 1; o /= 2) {
#pragma unroll
                for (int u = 0; u < 8; ++u) part[u] += __shfl_xor_sync(0xffffffffu, part[u], o);
            }
            if (chunk == 0) {
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (l0 + u < loads) res[warp * 64 + (l0 + u) * rpi + lane / tpr] = part[u];
            }
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = tid + h * BGMV_THREADS;
            if (n0 + c >= p.N) break;
            const float v = res[c];
            store_elem(p.out, OUT_DT, oi + c, ADD ? old[h] + v : v);
        }
        __syncthreads();   // res is read before the next row overwrites it
    }
}

}  // namespace sgmv
