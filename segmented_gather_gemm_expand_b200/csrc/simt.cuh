// Generic SGMV expand-slice kernel on the CUDA cores.
//
// Handles every call the API accepts: any rank K (including 0), any strides
// for x and B, any slice offset/width and alignment, all dtype combinations.
// It is the fallback for calls the tensor-core kernel does not take, and the
// independent second implementation the tests compare the fast path with.
//
// Grid: x = n-tile (128 columns) x row-chunk slot, y = segment (grid-stride).
// A CTA of 256 threads owns 128 columns; thread t takes column t % 128 and the
// rows of parity t / 128 within a 32-row chunk.  The rank is consumed in
// chunks of 32: B's chunk is staged in shared memory as fp32 [k][n] and x's
// chunk (already rounded to the weights' dtype) as fp32 [row][k]; products
// are accumulated in fp32 in k order.
#pragma once

#include "common.cuh"

namespace sgmv {

constexpr int SIMT_THREADS = 256;
constexpr int SIMT_NT = 128;     // columns per CTA
constexpr int SIMT_RC = 32;      // rows per chunk
constexpr int SIMT_KC = 32;      // rank chunk
constexpr int SIMT_ROWS_PER_THREAD = SIMT_RC / (SIMT_THREADS / SIMT_NT);

__global__ void __launch_bounds__(SIMT_THREADS)
simt_expand_slice_kernel(Problem p, int n_tiles, int row_slots) {
    __shared__ float sW[SIMT_KC][SIMT_NT];
    __shared__ float sX[SIMT_RC][SIMT_KC + 1];

    const int tid = threadIdx.x;
    const int col = tid % SIMT_NT;
    const int phase = tid / SIMT_NT;
    const int j = blockIdx.x % n_tiles;
    const int z = blockIdx.x / n_tiles;
    const int64_t n0 = (int64_t)j * SIMT_NT;
    const int64_t n = n0 + col;

    for (int64_t b = blockIdx.y; b < p.batches; b += gridDim.y) {
        const Segment seg = load_segment(p, b);
        if (seg.rows == 0) continue;
        const int64_t wbase = seg.adapter * p.w_as;
        for (int64_t c0 = (int64_t)z * SIMT_RC; c0 < seg.rows; c0 += (int64_t)row_slots * SIMT_RC) {
            const int rows_here = (int)min((int64_t)SIMT_RC, seg.rows - c0);
            float acc[SIMT_ROWS_PER_THREAD];
#pragma unroll
            for (int i = 0; i < SIMT_ROWS_PER_THREAD; ++i) acc[i] = 0.f;

            for (int64_t kc = 0; kc < p.K; kc += SIMT_KC) {
                __syncthreads();
                for (int i = tid; i < SIMT_KC * SIMT_NT; i += SIMT_THREADS) {
                    const int kk = i / SIMT_NT, nn = i % SIMT_NT;
                    float v = 0.f;
                    if (kc + kk < p.K && n0 + nn < p.N)
                        v = load_elem(p.w, p.w_dt, wbase + (n0 + nn) * p.w_ns + (kc + kk) * p.w_ks);
                    sW[kk][nn] = v;
                }
                for (int i = tid; i < SIMT_RC * SIMT_KC; i += SIMT_THREADS) {
                    const int rr = i / SIMT_KC, kk = i % SIMT_KC;
                    float v = 0.f;
                    if (rr < rows_here && kc + kk < p.K) {
                        const int64_t r = seg.row0 + c0 + rr;
                        v = round_to(load_elem(p.x, p.x_dt, r * p.x_rs + (kc + kk) * p.x_cs), p.w_dt);
                    }
                    sX[rr][kk] = v;
                }
                __syncthreads();
                const int kmax = (int)min((int64_t)SIMT_KC, p.K - kc);
                for (int kk = 0; kk < kmax; ++kk) {
                    const float wv = sW[kk][col];
#pragma unroll
                    for (int i = 0; i < SIMT_ROWS_PER_THREAD; ++i)
                        acc[i] = fmaf(sX[phase + 2 * i][kk], wv, acc[i]);
                }
            }
            if (n < p.N) {
#pragma unroll
                for (int i = 0; i < SIMT_ROWS_PER_THREAD; ++i) {
                    const int rr = phase + 2 * i;
                    if (rr < rows_here) {
                        const int64_t oi = (seg.row0 + c0 + rr) * p.H + p.off + n;
                        const float v = p.add ? load_elem(p.out, p.out_dt, oi) + acc[i] : acc[i];
                        store_elem(p.out, p.out_dt, oi, v);
                    }
                }
            }
        }
    }
}

}  // namespace sgmv
