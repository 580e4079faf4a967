// libsgmv: the C ABI (include/sgmv.h), host-side validation and dispatch.
//
// This is the library's single translation unit: the kernels live in the
// headers included below, so the device-side error word is one object per
// device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bgmv.cuh"
#include "common.cuh"
#include "simt.cuh"
#include "tc.cuh"
#include "validate.cuh"

namespace sgmv {

__device__ int32_t g_device_error = 0;

__device__ void raise_device_error(int32_t bits) { atomicOr(&g_device_error, bits); }

}  // namespace sgmv

#include "tc_kernel.cuh"
#include "shrink.cuh"

static_assert(SGMV_MAX_SLICES == sgmv::tc::MAX_SLICES, "one fused launch takes every slice of a call");

using namespace sgmv;

namespace {

std::atomic<int> g_forced_variant{SGMV_VARIANT_AUTO};

constexpr int kMaxDevices = 64;
struct DeviceInfo {
    int sm_count = 0;
    int cc_major = 0, cc_minor = 0;
    size_t smem_optin = 0;
    bool ok = false;
};
DeviceInfo g_devinfo[kMaxDevices];
std::mutex g_devinfo_mu;

int device_info(DeviceInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SGMV_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SGMV_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_devinfo_mu);
    DeviceInfo& d = g_devinfo[dev];
    if (!d.ok) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return SGMV_ERR_CUDA;
        d.sm_count = prop.multiProcessorCount;
        d.cc_major = prop.major;
        d.cc_minor = prop.minor;
        d.smem_optin = prop.sharedMemPerBlockOptin;
        d.ok = true;
    }
    *out = d;
    return SGMV_OK;
}

bool is_float_dtype(int dt) { return dt == SGMV_F16 || dt == SGMV_BF16 || dt == SGMV_F32; }
bool is_half_dtype(int dt) { return dt == SGMV_F16 || dt == SGMV_BF16; }
bool is_meta_dtype(int dt) { return dt == SGMV_I32 || dt == SGMV_I64; }

int64_t numel(const sgmv_tensor* t) {
    int64_t n = 1;
    for (int i = 0; i < t->ndim; ++i) n *= t->shape[i];
    return n;
}

// Shape/stride sanity common to every tensor argument.
int check_basic(const sgmv_tensor* t) {
    if (!t) return SGMV_ERR_NULL_ARG;
    if (t->ndim < 1 || t->ndim > 4) return SGMV_ERR_NDIM;
    for (int i = 0; i < t->ndim; ++i) {
        if (t->shape[i] < 0) return SGMV_ERR_SHAPE;
        if (t->stride[i] < 0) return SGMV_ERR_STRIDE;
        if (t->shape[i] > (int64_t(1) << 40) || t->stride[i] > (int64_t(1) << 40)) return SGMV_ERR_TOO_LARGE;
    }
    if (numel(t) > 0 && t->data == nullptr) return SGMV_ERR_NULL_ARG;
    return SGMV_OK;
}

int check_meta(const sgmv_tensor* t, int64_t batches) {
    int rc = check_basic(t);
    if (rc) return rc;
    if (t->ndim != 1) return SGMV_ERR_NDIM;
    if (!is_meta_dtype(t->dtype)) return SGMV_ERR_DTYPE;
    if (t->shape[0] < batches) return SGMV_ERR_BATCHES;
    if (batches > 0 && t->data == nullptr) return SGMV_ERR_NULL_ARG;
    return SGMV_OK;
}

MetaVec meta_of(const sgmv_tensor* t) {
    MetaVec m;
    m.ptr = t->data;
    m.dtype = t->dtype;
    m.stride = t->stride[0];
    return m;
}

struct Call {
    Problem p;
    int64_t max_seq_len;
    bool empty;   // nothing to launch
};

// Full host-side validation; fills the problem descriptor.  Touches no CUDA API.
int validate_call(const sgmv_tensor* x, const sgmv_tensor* w, const sgmv_tensor* out,
                  const sgmv_tensor* s, const sgmv_tensor* l, const sgmv_tensor* idx,
                  int64_t batches, int64_t max_seq_len, int64_t slice_offset, int64_t slice_size,
                  int add_inputs, Call* call) {
    std::memset(call, 0, sizeof(Call));   // zeroed padding too: plans are cached by the bytes of the problem
    int rc;
    if ((rc = check_basic(x))) return rc;
    if ((rc = check_basic(w))) return rc;
    if ((rc = check_basic(out))) return rc;
    if (batches < 0) return SGMV_ERR_BATCHES;
    if (max_seq_len < 0 || slice_size < 0) return SGMV_ERR_SHAPE;
    if ((rc = check_meta(s, batches))) return rc;
    if ((rc = check_meta(l, batches))) return rc;
    if ((rc = check_meta(idx, batches))) return rc;
    if (x->ndim != 2 || out->ndim != 2) return SGMV_ERR_NDIM;
    if (w->ndim != 3 && w->ndim != 4) return SGMV_ERR_NDIM;
    if (!is_float_dtype(x->dtype) || !is_half_dtype(w->dtype) || !is_float_dtype(out->dtype))
        return SGMV_ERR_DTYPE;
    const int wd = w->ndim;
    if (wd == 4 && w->shape[1] != 1) return SGMV_ERR_LAYOUT_4D;
    const int64_t K = x->shape[1];
    if (w->shape[wd - 1] != K) return SGMV_ERR_RANK_MISMATCH;
    if (w->shape[wd - 2] != slice_size) return SGMV_ERR_SLICE_SIZE;
    const int64_t T_out = out->shape[0], H = out->shape[1];
    if (!(out->stride[1] == 1 || H <= 1) || !(out->stride[0] == H || T_out <= 1))
        return SGMV_ERR_OUT_NOT_CONTIGUOUS;
    if (slice_offset < 0 || slice_offset + slice_size > H) return SGMV_ERR_SLICE_RANGE;

    Problem& p = call->p;
    p.x = x->data;
    p.x_dt = x->dtype;
    p.x_rows = x->shape[0];
    p.K = K;
    p.x_rs = x->stride[0];
    p.x_cs = x->stride[1];
    p.w = w->data;
    p.w_dt = w->dtype;
    p.lora_num = w->shape[0];
    p.w_as = w->stride[0];
    p.w_ns = w->stride[wd - 2];
    p.w_ks = w->stride[wd - 1];
    p.out = out->data;
    p.out_dt = out->dtype;
    p.out_rows = T_out;
    p.H = H;
    p.start = meta_of(s);
    p.len = meta_of(l);
    p.idx = meta_of(idx);
    p.batches = batches;
    p.off = slice_offset;
    p.N = slice_size;
    p.add = add_inputs ? 1 : 0;
    call->max_seq_len = max_seq_len;
    call->empty = batches == 0 || slice_size == 0 || T_out == 0 || p.lora_num == 0 || p.x_rows == 0;
    return SGMV_OK;
}

int launch_simt(const Call& c, const DeviceInfo& dev, cudaStream_t stream) {
    const Problem& p = c.p;
    const int64_t n_tiles = (p.N + SIMT_NT - 1) / SIMT_NT;
    if (n_tiles > (1 << 20)) return SGMV_ERR_TOO_LARGE;
    // Row-chunk slots: enough CTAs to fill the GPU for long segments; the
    // kernel grid-strides over chunks, so any value is correct.
    int64_t want_slots = (c.max_seq_len + SIMT_RC - 1) / SIMT_RC;
    const int64_t batches_y = p.batches < 65535 ? p.batches : 65535;
    const int64_t fill = (int64_t)dev.sm_count * 8 / (n_tiles * batches_y) + 1;
    if (want_slots > fill) want_slots = fill;
    if (want_slots < 1) want_slots = 1;
    if (want_slots * n_tiles > 0x7fffffff) want_slots = 0x7fffffff / n_tiles;
    dim3 grid((unsigned)(n_tiles * want_slots), (unsigned)batches_y);
    simt_expand_slice_kernel<<<grid, SIMT_THREADS, 0, stream>>>(p, (int)n_tiles, (int)want_slots);
    return cudaGetLastError() == cudaSuccess ? SGMV_OK : SGMV_ERR_LAUNCH;
}

// n-tile width a forced variant fixes for the tensor-core kernel (0: the library chooses).
int forced_bn(int forced) { return forced == SGMV_VARIANT_TC_WIDE ? 256 : 0; }

// Which variant runs a validated, non-empty call.
int choose_variant(const Call& c, const DeviceInfo& dev, int forced) {
    const bool tc_ok = dev.cc_major == 10 && tc_supports(&c.p, 1, dev.sm_count, forced_bn(forced));
    if (forced == SGMV_VARIANT_SIMT) return SGMV_VARIANT_SIMT;
    if (forced == SGMV_VARIANT_DECODE) return SGMV_ERR_VARIANT;   // bgmv_expand_slice's kernel only
    if (forced == SGMV_VARIANT_TC || forced == SGMV_VARIANT_TC_WIDE)
        return tc_ok ? (int)SGMV_VARIANT_TC : (int)SGMV_ERR_VARIANT;
    return tc_ok ? SGMV_VARIANT_TC : SGMV_VARIANT_SIMT;
}

// Several slices of one output: validate each as a single call, then check
// that the set is well formed (count, disjoint column ranges).  Fills the
// non-empty slices into calls[0..*n_live).
int validate_multi(const sgmv_tensor* x, const sgmv_tensor* const* ws, int num_slices, const sgmv_tensor* out,
                   const sgmv_tensor* s, const sgmv_tensor* l, const sgmv_tensor* idx, int64_t batches,
                   int64_t max_seq_len, const int64_t* offsets, int add_inputs, Call* calls, int* n_live) {
    if (!ws || !offsets) return SGMV_ERR_NULL_ARG;
    if (num_slices < 1 || num_slices > SGMV_MAX_SLICES) return SGMV_ERR_NUM_SLICES;
    *n_live = 0;
    int64_t lo[SGMV_MAX_SLICES], hi[SGMV_MAX_SLICES];
    for (int i = 0; i < num_slices; ++i) {
        if (!ws[i]) return SGMV_ERR_NULL_ARG;
        const int64_t n = ws[i]->ndim >= 2 && ws[i]->ndim <= 4 ? ws[i]->shape[ws[i]->ndim - 2] : -1;
        Call c;
        const int rc = validate_call(x, ws[i], out, s, l, idx, batches, max_seq_len, offsets[i], n < 0 ? 0 : n,
                                     add_inputs, &c);
        if (rc) return rc;
        lo[i] = offsets[i];
        hi[i] = offsets[i] + c.p.N;
        for (int j = 0; j < i; ++j)   // empty ranges overlap nothing
            if (lo[i] < hi[i] && lo[j] < hi[j] && lo[i] < hi[j] && lo[j] < hi[i]) return SGMV_ERR_SLICE_OVERLAP;
        if (!c.empty) calls[(*n_live)++] = c;
    }
    return SGMV_OK;
}

// How the live slices of a multi-slice call are launched: one fused
// tensor-core launch, or (when that cannot take the set) one launch per
// slice, each with its own variant.  Returns the fused variant or a status.
int choose_multi(const Call* calls, int n, const DeviceInfo& dev, int forced, bool* fused) {
    *fused = false;
    if (forced == SGMV_VARIANT_DECODE) return SGMV_ERR_VARIANT;   // bgmv_expand_slice's kernel only
    if (forced != SGMV_VARIANT_SIMT && dev.cc_major == 10) {
        Problem ps[SGMV_MAX_SLICES];
        for (int i = 0; i < n; ++i) ps[i] = calls[i].p;
        if (tc_supports(ps, n, dev.sm_count, forced_bn(forced))) {
            *fused = true;
            return SGMV_VARIANT_TC;
        }
    }
    for (int i = 0; i < n; ++i) {
        const int v = choose_variant(calls[i], dev, forced);
        if (v < 0) return v;
    }
    return forced == SGMV_VARIANT_SIMT ? (int)SGMV_VARIANT_SIMT : 0;
}

// bgmv_expand_slice: the expand-slice validation with row b as a one-token
// segment (start b, length 1); lora_idx stands in for the other two metadata
// tensors in the shape checks, then they become implicit vectors.
int validate_bgmv(const sgmv_tensor* x, const sgmv_tensor* w, const sgmv_tensor* out, const sgmv_tensor* idx,
                  int64_t batches, int64_t slice_offset, int64_t slice_size, int add_inputs, Call* call) {
    const int rc = validate_call(x, w, out, idx, idx, idx, batches, 1, slice_offset, slice_size, add_inputs, call);
    if (rc) return rc;
    call->p.start = MetaVec{nullptr, META_IOTA, 0};
    call->p.len = MetaVec{nullptr, META_ONE, 0};
    call->max_seq_len = 1;
    return SGMV_OK;
}

bool bgmv_fast_ok(const Problem& p) {
    if (p.K < 8 || p.K > BGMV_MAX_K || p.K % 8 != 0 || p.w_ks != 1) return false;
    if ((reinterpret_cast<uintptr_t>(p.w) & 15) || (p.w_ns * 2) % 16) return false;
    if (p.lora_num > 1 && (p.w_as * 2) % 16) return false;
    if ((p.N + BGMV_COLS - 1) / BGMV_COLS > 0x7fffffff) return false;
    return true;
}

int choose_bgmv(const Call& c, int forced) {
    const bool fast = bgmv_fast_ok(c.p);
    if (forced == SGMV_VARIANT_SIMT) return SGMV_VARIANT_SIMT;
    if (forced == SGMV_VARIANT_TC || forced == SGMV_VARIANT_TC_WIDE) return SGMV_ERR_VARIANT;
    if (forced == SGMV_VARIANT_DECODE) return fast ? (int)SGMV_VARIANT_DECODE : (int)SGMV_ERR_VARIANT;
    return fast ? SGMV_VARIANT_DECODE : SGMV_VARIANT_SIMT;
}

// x can be read as 16-byte pieces of B's dtype straight from its rows.
bool bgmv_x_vector(const Problem& p) {
    return p.x_dt == p.w_dt && p.x_cs == 1 && (reinterpret_cast<uintptr_t>(p.x) & 15) == 0 && (p.x_rs * 2) % 16 == 0;
}

// Launched as a programmatic dependent launch: the kernel waits for the
// preceding kernel's memory (griddepcontrol.wait) before its first read.
template <int OUT_DT, bool ADD, bool XVEC>
int launch_bgmv_kernel(const Problem& p, dim3 grid, cudaStream_t stream) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(BGMV_THREADS);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, bgmv_expand_kernel<OUT_DT, ADD, XVEC>, p) == cudaSuccess ? SGMV_OK
                                                                                            : SGMV_ERR_LAUNCH;
}

template <int OUT_DT>
int launch_bgmv_dt(const Problem& p, dim3 grid, cudaStream_t stream) {
    const bool xv = bgmv_x_vector(p);
    if (p.add) return xv ? launch_bgmv_kernel<OUT_DT, true, true>(p, grid, stream)
                         : launch_bgmv_kernel<OUT_DT, true, false>(p, grid, stream);
    return xv ? launch_bgmv_kernel<OUT_DT, false, true>(p, grid, stream)
              : launch_bgmv_kernel<OUT_DT, false, false>(p, grid, stream);
}

// Ranks that are powers of two take the coalesced kernel (every warp load reads
// 512 contiguous bytes of B); the others the two-rows-per-thread kernel.
template <int OUT_DT>
int launch_bgmv_coalesced(const Problem& p, dim3 grid, cudaStream_t stream) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(BGMV_THREADS);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = p.add ? cudaLaunchKernelEx(&cfg, bgmv_coalesced_kernel<OUT_DT, true>, p)
                                : cudaLaunchKernelEx(&cfg, bgmv_coalesced_kernel<OUT_DT, false>, p);
    return e == cudaSuccess ? SGMV_OK : SGMV_ERR_LAUNCH;
}

int launch_bgmv(const Call& c, cudaStream_t stream) {
    const Problem& p = c.p;
    if ((p.K & (p.K - 1)) == 0) {
        dim3 grid((unsigned)((p.N + BGMV_COLS - 1) / BGMV_COLS), (unsigned)(p.batches < 65535 ? p.batches : 65535));
        switch (p.out_dt) {
            case SGMV_F32: return launch_bgmv_coalesced<SGMV_F32>(p, grid, stream);
            case SGMV_BF16: return launch_bgmv_coalesced<SGMV_BF16>(p, grid, stream);
            default: return launch_bgmv_coalesced<SGMV_F16>(p, grid, stream);
        }
    }
    dim3 grid((unsigned)((p.N + BGMV_COLS - 1) / BGMV_COLS), (unsigned)(p.batches < 65535 ? p.batches : 65535));
    switch (p.out_dt) {
        case SGMV_F32: return launch_bgmv_dt<SGMV_F32>(p, grid, stream);
        case SGMV_BF16: return launch_bgmv_dt<SGMV_BF16>(p, grid, stream);
        default: return launch_bgmv_dt<SGMV_F16>(p, grid, stream);
    }
}

// sgmv_shrink: the expand-slice validation with lora_a in the weights' place
// (its N is the rank, its K the hidden size) and the whole output row as the
// slice; add_inputs is off.
int validate_shrink(const sgmv_tensor* x, const sgmv_tensor* a, const sgmv_tensor* out, const sgmv_tensor* s,
                    const sgmv_tensor* l, const sgmv_tensor* idx, int64_t batches, int64_t max_seq_len, Call* call) {
    int rc;
    if ((rc = check_basic(a))) return rc;
    if ((rc = check_basic(out))) return rc;
    if (a->ndim != 3 && a->ndim != 4) return SGMV_ERR_NDIM;
    if (out->ndim != 2) return SGMV_ERR_NDIM;
    const int64_t R = a->shape[a->ndim - 2];
    if ((rc = validate_call(x, a, out, s, l, idx, batches, max_seq_len, 0, R, 0, call))) return rc;
    if (out->shape[1] != R) return SGMV_ERR_OUT_WIDTH;
    return SGMV_OK;
}

// Variant and split count of a validated, non-empty shrink call with the given workspace.
int choose_shrink(const Call& c, const DeviceInfo& dev, int forced, const void* ws, size_t ws_bytes, int* splits) {
    *splits = 1;
    const bool tc_ok = dev.cc_major == 10 && shr::supports(c.p) && c.p.batches <= shr::SEG_CAP;
    int v;
    if (forced == SGMV_VARIANT_SIMT) v = SGMV_VARIANT_SIMT;
    else if (forced == SGMV_VARIANT_DECODE) return SGMV_ERR_VARIANT;
    else if (forced == SGMV_VARIANT_TC || forced == SGMV_VARIANT_TC_WIDE)
        v = tc_ok ? (int)SGMV_VARIANT_TC : (int)SGMV_ERR_VARIANT;
    else v = tc_ok ? SGMV_VARIANT_TC : SGMV_VARIANT_SIMT;
    if (v == SGMV_VARIANT_TC && ws) {
        int sp = shr::preferred_splits(c.p, dev.sm_count);
        while (sp > 1 && (size_t)shr::workspace_bytes_for(c.p, sp) > ws_bytes) sp /= 2;
        *splits = sp;
    }
    return v;
}

int launch_shrink(const Call& c, const DeviceInfo& dev, int splits, float* ws, cudaStream_t stream) {
    shr::Plan pl;
    if (!shr::cached_plan(c.p, dev.sm_count, splits, tc::encode_fn(), &pl)) return SGMV_ERR_VARIANT;
    switch (c.p.out_dt) {
        case SGMV_F32: return shr::launch_dt<SGMV_F32>(pl, c.p, ws, stream);
        case SGMV_BF16: return shr::launch_dt<SGMV_BF16>(pl, c.p, ws, stream);
        default: return shr::launch_dt<SGMV_F16>(pl, c.p, ws, stream);
    }
}

}  // namespace

extern "C" {

int sgmv_shrink(const sgmv_tensor* inputs, const sgmv_tensor* lora_a, const sgmv_tensor* out,
                const sgmv_tensor* seq_start, const sgmv_tensor* seq_len, const sgmv_tensor* lora_idx,
                int64_t batches, int64_t max_seq_len, void* workspace, size_t workspace_bytes, void* stream) {
    Call c;
    int rc = validate_shrink(inputs, lora_a, out, seq_start, seq_len, lora_idx, batches, max_seq_len, &c);
    if (rc) return rc;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 15)) return SGMV_ERR_WORKSPACE;
    if (c.empty) return SGMV_OK;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    int splits = 1;
    const int v = choose_shrink(c, dev, g_forced_variant.load(), workspace, workspace_bytes, &splits);
    if (v < 0) return v;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (v == SGMV_VARIANT_TC) return launch_shrink(c, dev, splits, static_cast<float*>(workspace), st);
    return launch_simt(c, dev, st);
}

}  // extern "C"

// Scratch of sgmv_shrink_static_scratch: the partial sums of split-H shrinks
// for callers that cannot allocate.  In host code this name is only a
// stand-in for the device variable: its device address comes from
// cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) float g_shrink_scratch[SGMV_SHRINK_STATIC_SCRATCH_BYTES / sizeof(float)];

namespace {

float* g_shrink_scratch_ptr[kMaxDevices];
std::mutex g_shrink_scratch_mu;

// Device address of g_shrink_scratch on the current device (looked up on the
// first call there), or nullptr with *rc set.
float* static_scratch(int* rc) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *rc = SGMV_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_shrink_scratch_mu);
    if (!g_shrink_scratch_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_shrink_scratch) != cudaSuccess || !ptr) {
            *rc = SGMV_ERR_CUDA;
            return nullptr;
        }
        g_shrink_scratch_ptr[dev] = static_cast<float*>(ptr);
    }
    *rc = SGMV_OK;
    return g_shrink_scratch_ptr[dev];
}

}  // namespace

extern "C" {

int sgmv_shrink_static_scratch(const sgmv_tensor* inputs, const sgmv_tensor* lora_a, const sgmv_tensor* out,
                               const sgmv_tensor* seq_start, const sgmv_tensor* seq_len,
                               const sgmv_tensor* lora_idx, int64_t batches, int64_t max_seq_len, void* stream) {
    Call c;
    int rc = validate_shrink(inputs, lora_a, out, seq_start, seq_len, lora_idx, batches, max_seq_len, &c);
    if (rc) return rc;
    if (c.empty) return SGMV_OK;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    // exactly what sgmv_shrink does with a workspace of the static array's
    // size: the preferred split count, halved until the partial sums fit
    int splits = 1;
    float* scratch = static_scratch(&rc);
    if (!scratch) return rc;
    const int v = choose_shrink(c, dev, g_forced_variant.load(), scratch, SGMV_SHRINK_STATIC_SCRATCH_BYTES, &splits);
    if (v < 0) return v;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (v == SGMV_VARIANT_TC) return launch_shrink(c, dev, splits, scratch, st);
    return launch_simt(c, dev, st);
}

int sgmv_shrink_plan(const sgmv_tensor* inputs, const sgmv_tensor* lora_a, const sgmv_tensor* out,
                     const sgmv_tensor* seq_start, const sgmv_tensor* seq_len, const sgmv_tensor* lora_idx,
                     int64_t batches, int64_t max_seq_len, size_t workspace_bytes, int* variant, int* splits,
                     size_t* preferred_workspace_bytes) {
    if (!variant || !splits || !preferred_workspace_bytes) return SGMV_ERR_NULL_ARG;
    *variant = 0;
    *splits = 0;
    *preferred_workspace_bytes = 0;
    Call c;
    int rc = validate_shrink(inputs, lora_a, out, seq_start, seq_len, lora_idx, batches, max_seq_len, &c);
    if (rc) return rc;
    if (c.empty) return SGMV_OK;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    int sp = 1;
    static const char dummy = 0;   // a non-null stand-in: only the size matters here
    const int v = choose_shrink(c, dev, g_forced_variant.load(), workspace_bytes ? &dummy : nullptr, workspace_bytes,
                                &sp);
    if (v < 0) return v;
    *variant = v;
    *splits = v == SGMV_VARIANT_TC ? sp : 1;
    if (v == SGMV_VARIANT_TC)
        *preferred_workspace_bytes = (size_t)shr::workspace_bytes_for(c.p, shr::preferred_splits(c.p, dev.sm_count));
    return SGMV_OK;
}

int sgmv_expand(const sgmv_tensor* inputs, const sgmv_tensor* lora_b, const sgmv_tensor* out,
                const sgmv_tensor* seq_start, const sgmv_tensor* seq_len, const sgmv_tensor* lora_idx,
                int64_t batches, int64_t max_seq_len, int add_inputs, void* stream) {
    int rc;
    if ((rc = check_basic(lora_b))) return rc;
    if ((rc = check_basic(out))) return rc;
    if (lora_b->ndim != 3 && lora_b->ndim != 4) return SGMV_ERR_NDIM;
    if (out->ndim != 2) return SGMV_ERR_NDIM;
    const int64_t N = lora_b->shape[lora_b->ndim - 2];
    if (out->shape[1] != N) return SGMV_ERR_OUT_WIDTH;
    return sgmv_expand_slice(inputs, lora_b, out, seq_start, seq_len, lora_idx, batches, max_seq_len, 0, N,
                             add_inputs, stream);
}

int bgmv_expand_slice(const sgmv_tensor* inputs, const sgmv_tensor* lora_b, const sgmv_tensor* out,
                      const sgmv_tensor* lora_idx, int64_t batches, int64_t slice_offset, int64_t slice_size,
                      int add_inputs, void* stream) {
    Call c;
    int rc = validate_bgmv(inputs, lora_b, out, lora_idx, batches, slice_offset, slice_size, add_inputs, &c);
    if (rc) return rc;
    if (c.empty) return SGMV_OK;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    const int v = choose_bgmv(c, g_forced_variant.load());
    if (v < 0) return v;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (v == SGMV_VARIANT_DECODE) return launch_bgmv(c, st);
    return launch_simt(c, dev, st);
}

int bgmv_plan(const sgmv_tensor* inputs, const sgmv_tensor* lora_b, const sgmv_tensor* out,
              const sgmv_tensor* lora_idx, int64_t batches, int64_t slice_offset, int64_t slice_size,
              int add_inputs, int* variant) {
    if (!variant) return SGMV_ERR_NULL_ARG;
    *variant = 0;
    Call c;
    const int rc = validate_bgmv(inputs, lora_b, out, lora_idx, batches, slice_offset, slice_size, add_inputs, &c);
    if (rc) return rc;
    if (c.empty) return SGMV_OK;
    const int v = choose_bgmv(c, g_forced_variant.load());
    if (v < 0) return v;
    *variant = v;
    return SGMV_OK;
}

int sgmv_expand_slice(const sgmv_tensor* inputs, const sgmv_tensor* lora_b, const sgmv_tensor* out,
                      const sgmv_tensor* seq_start, const sgmv_tensor* seq_len,
                      const sgmv_tensor* lora_idx, int64_t batches, int64_t max_seq_len,
                      int64_t slice_offset, int64_t slice_size, int add_inputs, void* stream) {
    Call c;
    int rc = validate_call(inputs, lora_b, out, seq_start, seq_len, lora_idx, batches, max_seq_len,
                           slice_offset, slice_size, add_inputs, &c);
    if (rc) return rc;
    if (c.empty) return SGMV_OK;
    const int forced = g_forced_variant.load();
    if (forced == SGMV_VARIANT_DECODE) return SGMV_ERR_VARIANT;   // bgmv_expand_slice's kernel only
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    const int v = choose_variant(c, dev, forced);
    if (v < 0) return v;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (v == SGMV_VARIANT_TC) return launch_tc(&c.p, 1, dev.sm_count, st, forced_bn(forced));
    return launch_simt(c, dev, st);
}

int sgmv_plan(const sgmv_tensor* inputs, const sgmv_tensor* lora_b, const sgmv_tensor* out,
              const sgmv_tensor* seq_start, const sgmv_tensor* seq_len, const sgmv_tensor* lora_idx,
              int64_t batches, int64_t max_seq_len, int64_t slice_offset, int64_t slice_size,
              int add_inputs, int* variant) {
    if (!variant) return SGMV_ERR_NULL_ARG;
    *variant = 0;
    Call c;
    int rc = validate_call(inputs, lora_b, out, seq_start, seq_len, lora_idx, batches, max_seq_len,
                           slice_offset, slice_size, add_inputs, &c);
    if (rc) return rc;
    if (c.empty) return SGMV_OK;
    const int forced = g_forced_variant.load();
    if (forced == SGMV_VARIANT_DECODE) return SGMV_ERR_VARIANT;   // bgmv_expand_slice's kernel only
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    const int v = choose_variant(c, dev, forced);
    if (v < 0) return v;
    *variant = v;
    return SGMV_OK;
}

int sgmv_expand_multi_slice(const sgmv_tensor* inputs, const sgmv_tensor* const* lora_b, int num_slices,
                            const sgmv_tensor* out, const sgmv_tensor* seq_start, const sgmv_tensor* seq_len,
                            const sgmv_tensor* lora_idx, int64_t batches, int64_t max_seq_len,
                            const int64_t* slice_offsets, int add_inputs, void* stream) {
    Call calls[SGMV_MAX_SLICES];
    int n = 0;
    int rc = validate_multi(inputs, lora_b, num_slices, out, seq_start, seq_len, lora_idx, batches, max_seq_len,
                            slice_offsets, add_inputs, calls, &n);
    if (rc) return rc;
    if (n == 0) return SGMV_OK;
    if (g_forced_variant.load() == SGMV_VARIANT_DECODE) return SGMV_ERR_VARIANT;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    const int forced = g_forced_variant.load();
    bool fused = false;
    const int v = choose_multi(calls, n, dev, forced, &fused);
    if (v < 0) return v;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (fused) {
        Problem ps[SGMV_MAX_SLICES];
        for (int i = 0; i < n; ++i) ps[i] = calls[i].p;
        return launch_tc(ps, n, dev.sm_count, st, forced_bn(forced));
    }
    for (int i = 0; i < n; ++i) {
        const int vi = choose_variant(calls[i], dev, forced);
        rc = vi == SGMV_VARIANT_TC ? launch_tc(&calls[i].p, 1, dev.sm_count, st, forced_bn(forced))
                                   : launch_simt(calls[i], dev, st);
        if (rc) return rc;
    }
    return SGMV_OK;
}

int sgmv_plan_multi_slice(const sgmv_tensor* inputs, const sgmv_tensor* const* lora_b, int num_slices,
                          const sgmv_tensor* out, const sgmv_tensor* seq_start, const sgmv_tensor* seq_len,
                          const sgmv_tensor* lora_idx, int64_t batches, int64_t max_seq_len,
                          const int64_t* slice_offsets, int add_inputs, int* variant, int* launches) {
    if (!variant || !launches) return SGMV_ERR_NULL_ARG;
    *variant = 0;
    *launches = 0;
    Call calls[SGMV_MAX_SLICES];
    int n = 0;
    int rc = validate_multi(inputs, lora_b, num_slices, out, seq_start, seq_len, lora_idx, batches, max_seq_len,
                            slice_offsets, add_inputs, calls, &n);
    if (rc) return rc;
    if (n == 0) return SGMV_OK;
    if (g_forced_variant.load() == SGMV_VARIANT_DECODE) return SGMV_ERR_VARIANT;
    DeviceInfo dev;
    if ((rc = device_info(&dev))) return rc;
    bool fused = false;
    const int v = choose_multi(calls, n, dev, g_forced_variant.load(), &fused);
    if (v < 0) return v;
    *variant = v;
    *launches = fused ? 1 : n;
    return SGMV_OK;
}

int sgmv_validate_metadata(const sgmv_tensor* seq_start, const sgmv_tensor* seq_len,
                           const sgmv_tensor* lora_idx, int64_t batches, int64_t lora_num,
                           int64_t total_rows, int32_t* d_status, void* stream) {
    if (!d_status) return SGMV_ERR_NULL_ARG;
    if (batches < 0) return SGMV_ERR_BATCHES;
    if (lora_num < 0 || total_rows < 0) return SGMV_ERR_SHAPE;
    int rc;
    if ((rc = check_meta(seq_start, batches))) return rc;
    if ((rc = check_meta(seq_len, batches))) return rc;
    if ((rc = check_meta(lora_idx, batches))) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(d_status, 0, sizeof(int32_t), st) != cudaSuccess) return SGMV_ERR_CUDA;
    if (batches == 0) return SGMV_OK;
    const int threads = 256;
    int64_t blocks = (batches + threads - 1) / threads;
    if (blocks > 4096) blocks = 4096;
    validate_metadata_kernel<<<(unsigned)blocks, threads, 0, st>>>(
        meta_of(seq_start), meta_of(seq_len), meta_of(lora_idx), batches, lora_num, total_rows, d_status);
    if (cudaGetLastError() != cudaSuccess) return SGMV_ERR_LAUNCH;
    if (batches <= VALIDATE_PAIRWISE_LIMIT) {
        validate_overlap_pairwise_kernel<<<1024, threads, 0, st>>>(
            meta_of(seq_start), meta_of(seq_len), meta_of(lora_idx), batches, lora_num, d_status);
        if (cudaGetLastError() != cudaSuccess) return SGMV_ERR_LAUNCH;
    }
    return SGMV_OK;
}

const char* sgmv_status_string(int code) {
    switch (code) {
        case SGMV_OK: return "ok";
        case SGMV_ERR_NULL_ARG: return "null descriptor or null data pointer";
        case SGMV_ERR_DTYPE: return "dtype not allowed for this argument";
        case SGMV_ERR_NDIM: return "wrong number of dimensions";
        case SGMV_ERR_RANK_MISMATCH: return "inputs.shape[1] != lora_b.shape[-1] (rank mismatch)";
        case SGMV_ERR_SLICE_SIZE: return "slice_size != lora_b.shape[-2]";
        case SGMV_ERR_LAYOUT_4D: return "4-D lora_b must have shape (lora_num, 1, slice_size, rank)";
        case SGMV_ERR_OUT_NOT_CONTIGUOUS: return "output tensor must be contiguous";
        case SGMV_ERR_SLICE_RANGE: return "slice [offset, offset + size) outside the output width";
        case SGMV_ERR_BATCHES: return "batches negative or larger than a metadata tensor";
        case SGMV_ERR_SHAPE: return "negative extent or max_seq_len";
        case SGMV_ERR_STRIDE: return "negative stride";
        case SGMV_ERR_TOO_LARGE: return "sizes beyond the library's index range";
        case SGMV_ERR_VARIANT: return "the forced kernel variant cannot run this call";
        case SGMV_ERR_NUM_SLICES: return "num_slices outside [1, SGMV_MAX_SLICES]";
        case SGMV_ERR_SLICE_OVERLAP: return "two slices of a multi-slice call overlap";
        case SGMV_ERR_OUT_WIDTH: return "out.shape[1] != lora_b.shape[-2] (plain expand and shrink write whole rows)";
        case SGMV_ERR_WORKSPACE: return "workspace is not 16-byte aligned";
        case SGMV_ERR_SCRATCH: return "reserved status (no entry point returns it)";
        case SGMV_ERR_CUDA: return "a CUDA runtime call failed";
        case SGMV_ERR_LAUNCH: return "kernel launch failed";
        default: return "unknown status";
    }
}

int sgmv_set_variant(int variant) {
    if (variant != SGMV_VARIANT_AUTO && variant != SGMV_VARIANT_SIMT && variant != SGMV_VARIANT_TC &&
        variant != SGMV_VARIANT_DECODE && variant != SGMV_VARIANT_TC_WIDE)
        return SGMV_ERR_VARIANT;
    return g_forced_variant.exchange(variant);
}

int sgmv_device_error(void* stream, int32_t* value) {
    if (!value) return SGMV_ERR_NULL_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t zero = 0;
    if (cudaMemcpyFromSymbolAsync(value, g_device_error, sizeof(int32_t), 0, cudaMemcpyDeviceToHost, st) !=
        cudaSuccess)
        return SGMV_ERR_CUDA;
    if (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int32_t), 0, cudaMemcpyHostToDevice, st) !=
        cudaSuccess)
        return SGMV_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SGMV_ERR_CUDA;
    return SGMV_OK;
}

int sgmv_version(void) { return 100; }

}  // extern "C"
