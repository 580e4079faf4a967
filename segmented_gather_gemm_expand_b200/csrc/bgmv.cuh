// BGMV expand-slice: one token per row, each with its own adapter.
//
// The decode counterpart of the expand-slice operation: row b gets
// out[b, off:off+N] (+)= x^[b, :] . B[idx[b]]^T.  With one row per adapter use
// there is no B tile to reuse across rows, so nothing is staged: every thread
// streams the two B rows of its two output columns with 16-byte loads
// (consecutive threads read consecutive rows, so a warp reads one contiguous
// stretch of B), x's row is rounded to the weights' dtype into shared memory
// once per row, products are summed in fp32 in k order, and the result (plus
// the old value in add mode) is rounded once.
//
// Grid: x = 256-column tile of the slice, y = rows (grid-stride).
#pragma once

#include "common.cuh"

namespace sgmv {

constexpr int BGMV_THREADS = 128;
constexpr int BGMV_COLS = 2 * BGMV_THREADS;   // columns per CTA
constexpr int BGMV_MAX_K = 256;

// Element e (0..7) of 8 packed 16-bit values as a float.
__device__ __forceinline__ float half8_elem(const uint4& v, int e, bool bf16) {
    const uint32_t w = e < 2 ? v.x : e < 4 ? v.y : e < 6 ? v.z : v.w;
    const uint32_t h = (e & 1) ? (w >> 16) : (w & 0xFFFFu);
    return bf16 ? __uint_as_float(h << 16) : __half2float(__ushort_as_half((unsigned short)h));
}

template <int OUT_DT, bool ADD>
__global__ void __launch_bounds__(BGMV_THREADS)
bgmv_expand_kernel(Problem p) {
    __shared__ float sx[BGMV_MAX_K];
    const int tid = threadIdx.x;
    const bool w_bf16 = p.w_dt == SGMV_BF16;
    const int64_t n = (int64_t)blockIdx.x * BGMV_COLS + 2 * tid;   // first of this thread's two columns
    const int64_t lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    const int K = (int)p.K;

    for (int64_t b = blockIdx.y; b < p.batches; b += gridDim.y) {
        const int64_t a = load_meta(p.idx, b);
        if (a < 0 || a >= p.lora_num || b >= lim) continue;     // uniform across the CTA
        __syncthreads();   // the previous row's sx is no longer read
        for (int k = tid; k < K; k += BGMV_THREADS)
            sx[k] = round_to(load_elem(p.x, p.x_dt, b * p.x_rs + k * p.x_cs), p.w_dt);
        __syncthreads();
        if (n >= p.N) continue;
        const bool two = n + 1 < p.N;
        const uint4* w0 = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.w) + a * p.w_as + n * p.w_ns);
        const uint4* w1 = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.w) + a * p.w_as +
                                                         (two ? n + 1 : n) * p.w_ns);
        float acc0 = 0.f, acc1 = 0.f;
        for (int k8 = 0; k8 < K / 8; ++k8) {
            const uint4 v0 = __ldg(w0 + k8);
            const uint4 v1 = __ldg(w1 + k8);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float xv = sx[k8 * 8 + e];
                acc0 = fmaf(xv, half8_elem(v0, e, w_bf16), acc0);
                acc1 = fmaf(xv, half8_elem(v1, e, w_bf16), acc1);
            }
        }
        const int64_t oi = b * p.H + p.off + n;
        if (ADD) {
            acc0 += load_elem(p.out, OUT_DT, oi);
            if (two) acc1 += load_elem(p.out, OUT_DT, oi + 1);
        }
        store_elem(p.out, OUT_DT, oi, acc0);
        if (two) store_elem(p.out, OUT_DT, oi + 1, acc1);
    }
}

}  // namespace sgmv
