// Shared device-side definitions of libsgmv: the problem descriptor handed to
// every kernel, metadata/element access, and the rounding helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "sgmv.h"

namespace sgmv {

// One metadata vector (seq_start, seq_len or lora_idx): i32 or i64, any stride,
// or an implicit vector with no memory behind it: element b is b (META_IOTA)
// or 1 (META_ONE), which describes one-token rows (bgmv_expand_slice).
constexpr int32_t META_IOTA = 100;
constexpr int32_t META_ONE = 101;
struct MetaVec {
    const void* ptr;
    int32_t dtype;     // SGMV_I32 | SGMV_I64 | META_IOTA | META_ONE
    int64_t stride;    // elements
};

// Everything a kernel needs about one expand-slice call.  Passed by value
// (kernel parameter space).  Strides are in elements.
struct Problem {
    const void* x;
    int32_t x_dt;
    int64_t x_rows, K, x_rs, x_cs;
    const void* w;
    int32_t w_dt;
    int64_t lora_num, w_as, w_ns, w_ks;     // adapter, row (n) and column (k) strides
    void* out;
    int32_t out_dt;
    int64_t out_rows, H;
    MetaVec start, len, idx;
    int64_t batches, off, N;
    int32_t add;
};

__device__ __forceinline__ int64_t load_meta(const MetaVec& m, int64_t i) {
    if (m.dtype == META_IOTA) return i;
    if (m.dtype == META_ONE) return 1;
    if (m.dtype == SGMV_I64) return __ldg(reinterpret_cast<const long long*>(m.ptr) + i * m.stride);
    return (int64_t)__ldg(reinterpret_cast<const int*>(m.ptr) + i * m.stride);
}

// A segment after the guards of the header: rows [row0, row0 + rows) of out
// get adapter `adapter`; rows == 0 means the segment writes nothing.
struct Segment {
    int64_t row0;
    int64_t rows;
    int64_t adapter;
};

__device__ __forceinline__ Segment load_segment(const Problem& p, int64_t b) {
    Segment s;
    s.row0 = load_meta(p.start, b);
    int64_t L = load_meta(p.len, b);
    s.adapter = load_meta(p.idx, b);
    const int64_t lim = p.out_rows < p.x_rows ? p.out_rows : p.x_rows;
    int64_t end = s.row0 + L;
    if (end > lim) end = lim;
    bool ok = s.adapter >= 0 && s.adapter < p.lora_num && s.row0 >= 0 && L > 0 && end > s.row0;
    s.rows = ok ? end - s.row0 : 0;
    return s;
}

__device__ __forceinline__ float load_elem(const void* p, int dt, int64_t i) {
    if (dt == SGMV_F32) return reinterpret_cast<const float*>(p)[i];
    if (dt == SGMV_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    return __half2float(reinterpret_cast<const __half*>(p)[i]);
}

// Value of v rounded to nearest-even in dtype dt (as a float).
__device__ __forceinline__ float round_to(float v, int dt) {
    if (dt == SGMV_BF16) return __bfloat162float(__float2bfloat16_rn(v));
    if (dt == SGMV_F16) return __half2float(__float2half_rn(v));
    return v;
}

__device__ __forceinline__ void store_elem(void* p, int dt, int64_t i, float v) {
    if (dt == SGMV_F32) reinterpret_cast<float*>(p)[i] = v;
    else if (dt == SGMV_BF16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
    else reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
}

// Device-side error word (per device, lives as long as the module is loaded).
// Kernels OR bits into it instead of trapping.
enum : int32_t {
    DEVERR_TIMEOUT_PRODUCER = 1,
    DEVERR_TIMEOUT_MMA = 2,
    DEVERR_TIMEOUT_EPILOGUE = 4,
    DEVERR_TIMEOUT_CONVERT = 8,
    DEVERR_SCHEDULE = 16
};

// Raises a kernel's dynamic shared-memory limit, once per device: the setting
// belongs to the device's context, so a process that drives several GPUs sets
// it on each (devices past 63 set it on every call).  `done` holds one bit per
// device.  Returns false if the runtime refused.
template <typename Kern>
inline bool set_smem_limit_once(Kern kern, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t(1) << dev) : 0;
    if (bit && (done.load() & bit)) return true;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    if (bit) done.fetch_or(bit);
    return true;
}

}  // namespace sgmv

// Defined in api.cu (relocatable device code is not used; each .cu that needs
// it declares its own accessor).
