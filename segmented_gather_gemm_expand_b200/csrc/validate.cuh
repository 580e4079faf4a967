// Device-side check of the metadata VALUES (sgmv_validate_metadata).
// Writes a bit mask; never traps.  Bits are documented in sgmv.h.
#pragma once

#include "common.cuh"

namespace sgmv {

constexpr int64_t VALIDATE_PAIRWISE_LIMIT = 8192;

__global__ void validate_metadata_kernel(MetaVec start, MetaVec len, MetaVec idx, int64_t batches,
                                         int64_t lora_num, int64_t total_rows, int32_t* status) {
    // One grid; a thread per segment for the per-segment checks and the
    // ordering check, then a grid-stride pairwise overlap check when the
    // starts are not ordered.
    __shared__ int32_t s_bits;
    if (threadIdx.x == 0) s_bits = 0;
    __syncthreads();
    int32_t bits = 0;
    bool unordered = false;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < batches;
         b += (int64_t)gridDim.x * blockDim.x) {
        const int64_t a = load_meta(idx, b), s = load_meta(start, b), L = load_meta(len, b);
        if (a < -1 || a >= lora_num) bits |= 1;
        if (s < 0 || L < 0) bits |= 2;
        const bool valid = a >= 0 && a < lora_num && L > 0 && s >= 0;
        if (valid && s + L > total_rows) bits |= 4;
        if (valid) {
            // next valid segment after b
            for (int64_t c = b + 1; c < batches; ++c) {
                const int64_t a2 = load_meta(idx, c), s2 = load_meta(start, c), L2 = load_meta(len, c);
                if (!(a2 >= 0 && a2 < lora_num && L2 > 0 && s2 >= 0)) continue;
                if (s2 < s) unordered = true;
                else if (s2 < s + L) bits |= 8;
                break;
            }
        }
    }
    if (unordered) bits |= (batches > VALIDATE_PAIRWISE_LIMIT) ? (16 | 32) : 16;
    if (bits) atomicOr(&s_bits, bits);
    __syncthreads();
    if (threadIdx.x == 0 && s_bits) atomicOr(status, s_bits);
}

// Pairwise overlap check, launched only when the ordered check is not enough.
__global__ void validate_overlap_pairwise_kernel(MetaVec start, MetaVec len, MetaVec idx,
                                                 int64_t batches, int64_t lora_num, int32_t* status) {
    if (!(*(volatile int32_t*)status & 16)) return;   // starts were ordered: already checked
    const int64_t pairs = batches * batches;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < pairs;
         q += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = q / batches, c = q % batches;
        if (c <= b) continue;
        const int64_t a1 = load_meta(idx, b), s1 = load_meta(start, b), L1 = load_meta(len, b);
        const int64_t a2 = load_meta(idx, c), s2 = load_meta(start, c), L2 = load_meta(len, c);
        const bool v1 = a1 >= 0 && a1 < lora_num && L1 > 0 && s1 >= 0;
        const bool v2 = a2 >= 0 && a2 < lora_num && L2 > 0 && s2 >= 0;
        if (v1 && v2 && s1 < s2 + L2 && s2 < s1 + L1) atomicOr(status, 8);
    }
}

}  // namespace sgmv
