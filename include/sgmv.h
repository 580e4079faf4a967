/*
 * libsgmv -- SGMV expand-slice for NVIDIA B200 (sm_100a).
 *
 * The operation ("Implementation: Predibase Lorax SGMV Expand Slice Kernel",
 * sections Description, Signature, I/O Contract and Outputs): for every
 * sequence b < batches with start s_b = seq_start[b], length L_b = seq_len[b]
 * and adapter a = lora_idx[b], and every token m < L_b (row r = s_b + m),
 *
 *     out[r, off + n] = (add_inputs ? out[r, off + n] : 0) + sum_k x^[r, k] * B[a][n, k]
 *
 * for n in [0, slice_size), off = slice_offset.  x^ is x rounded to nearest-even
 * in the weights' dtype ("mixed-precision type casting"); products are summed
 * in fp32 and the sum (plus the old value when add_inputs) is rounded to
 * nearest-even in out's dtype once.  Every other element of out keeps its bits:
 * columns outside [off, off + slice_size), rows of segments whose adapter is -1,
 * rows not covered by any segment.
 *
 * Conventions for every entry point:
 *   - Memory: all tensor data pointers are DEVICE pointers on the current CUDA
 *     device.  The caller owns every buffer; the library keeps no pointer after
 *     a call returns and allocates no device memory.
 *   - Streams: work is enqueued on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream).  Nothing synchronises the host, except where a function
 *     says so.
 *   - Errors: a negative status is returned BEFORE anything is enqueued, and
 *     nothing is written, when an argument is invalid.  SGMV_ERR_CUDA /
 *     SGMV_ERR_LAUNCH report a failing CUDA call (the launch may or may not
 *     have been enqueued).  sgmv_status_string() names every code.
 *   - Values inside device tensors (segment starts, lengths, adapter ids)
 *     cannot be checked without a host synchronisation, so the kernels guard
 *     them instead: a segment whose adapter id is outside [0, lora_num), whose
 *     start is negative or whose length is not positive is skipped; rows at or
 *     beyond the row count of `out` or of `inputs` are skipped.  No kernel
 *     reads or writes outside the tensors it is given.  sgmv_validate_metadata()
 *     reports such values without trapping.
 *   - max_seq_len is accepted for signature parity with the page's wrapper,
 *     where it sizes the launch grid; here the grid depends only on the SM
 *     count and the work is expanded from the metadata on the device, so every
 *     token m < L_b is processed even if max_seq_len is smaller.
 */
#ifndef SGMV_H
#define SGMV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SGMV_API __attribute__((visibility("default")))
#else
#define SGMV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Element types. */
typedef enum {
    SGMV_F16 = 0,   /* IEEE binary16 */
    SGMV_BF16 = 1,  /* bfloat16 */
    SGMV_F32 = 2,   /* IEEE binary32 */
    SGMV_I32 = 3,   /* metadata only */
    SGMV_I64 = 4    /* metadata only */
} sgmv_dtype;

/* A strided view of device memory.  shape[i] and stride[i] (in ELEMENTS, not
 * bytes) are meaningful for i < ndim; the rest are ignored. */
typedef struct {
    void* data;
    int32_t dtype;      /* sgmv_dtype */
    int32_t ndim;       /* 1 .. 4 */
    int64_t shape[4];
    int64_t stride[4];
} sgmv_tensor;

/* Status codes. */
enum {
    SGMV_OK = 0,
    SGMV_ERR_NULL_ARG = -1,          /* a descriptor or a non-empty tensor's data is NULL */
    SGMV_ERR_DTYPE = -2,             /* a tensor's dtype is not allowed for its role */
    SGMV_ERR_NDIM = -3,              /* wrong number of dimensions */
    SGMV_ERR_RANK_MISMATCH = -4,     /* inputs.shape[1] != lora_b.shape[-1] */
    SGMV_ERR_SLICE_SIZE = -5,        /* slice_size != lora_b.shape[-2] */
    SGMV_ERR_LAYOUT_4D = -6,         /* 4-D lora_b whose dimension 1 is not 1 */
    SGMV_ERR_OUT_NOT_CONTIGUOUS = -7,/* out is not contiguous row-major */
    SGMV_ERR_SLICE_RANGE = -8,       /* slice_offset < 0 or slice_offset + slice_size > out.shape[1] */
    SGMV_ERR_BATCHES = -9,           /* batches < 0, or a metadata tensor shorter than batches */
    SGMV_ERR_SHAPE = -10,            /* a negative extent, or max_seq_len < 0 */
    SGMV_ERR_STRIDE = -11,           /* a negative stride */
    SGMV_ERR_TOO_LARGE = -12,        /* sizes beyond the library's index range */
    SGMV_ERR_VARIANT = -13,          /* the forced kernel variant cannot run this call */
    SGMV_ERR_NUM_SLICES = -14,       /* num_slices outside [1, SGMV_MAX_SLICES] */
    SGMV_ERR_SLICE_OVERLAP = -15,    /* two non-empty slices of one call share a column */
    SGMV_ERR_OUT_WIDTH = -16,        /* sgmv_expand / sgmv_shrink: out.shape[1] != lora_b/lora_a.shape[-2] */
    SGMV_ERR_WORKSPACE = -17,        /* sgmv_shrink: workspace not 16-byte aligned */
    SGMV_ERR_SCRATCH = -18,          /* reserved (no entry point returns it) */
    SGMV_ERR_CUDA = -20,             /* a CUDA runtime call failed */
    SGMV_ERR_LAUNCH = -21            /* a kernel launch failed */
};

/* Kernel variants (for sgmv_set_variant / sgmv_plan). */
enum {
    SGMV_VARIANT_AUTO = 0,
    SGMV_VARIANT_SIMT = 1,   /* generic CUDA-core kernel: any strides, rank, alignment */
    SGMV_VARIANT_TC = 2,     /* tcgen05 tensor-core kernel with TMA staging */
    SGMV_VARIANT_DECODE = 3, /* bgmv_expand_slice's one-token-per-row kernel (vector loads) */
    SGMV_VARIANT_TC_WIDE = 4 /* the tensor-core kernel with 256-column n-tiles forced (tests); plans report
                                SGMV_VARIANT_TC.  SGMV_VARIANT_TC and AUTO let the library pick 128 or 256 */
};

/*
 * sgmv_expand_slice -- the operation above, in place on `out`.
 *
 *   inputs    (T_x, K)                    f16 | bf16 | f32, any non-negative strides
 *   lora_b    (lora_num, N, K) or (lora_num, 1, N, K)   f16 | bf16, any strides;
 *             N must equal slice_size; the 4-D form's unit dimension is dropped
 *   out       (T_out, H)                  f16 | bf16 | f32, contiguous row-major
 *   seq_start, seq_len, lora_idx  1-D, i32 | i64 (each independently), length
 *             >= batches, any stride; lora_idx == -1 means "no LoRA"
 *   batches, max_seq_len, slice_offset, slice_size, add_inputs: as in the page's
 *             wrapper (sgmv_expand_slice's arguments of the same names).
 *
 * Returns SGMV_OK when the work was enqueued, or a negative status.  Calls with
 * batches == 0, slice_size == 0 or T_out == 0 return SGMV_OK and enqueue nothing.
 * Segments must not overlap (rows written by two segments are undefined).
 */
SGMV_API int sgmv_expand_slice(const sgmv_tensor* inputs, const sgmv_tensor* lora_b, const sgmv_tensor* out,
                      const sgmv_tensor* seq_start, const sgmv_tensor* seq_len,
                      const sgmv_tensor* lora_idx, int64_t batches, int64_t max_seq_len,
                      int64_t slice_offset, int64_t slice_size, int add_inputs, void* stream);

/*
 * sgmv_plan -- validate exactly as sgmv_expand_slice does and report, in
 * *variant, the kernel variant a call with these arguments would launch
 * (SGMV_VARIANT_SIMT or SGMV_VARIANT_TC; 0 when nothing would launch).
 * Launches nothing and touches no tensor data.  May query the current device's
 * properties (once per device).
 */
SGMV_API int sgmv_plan(const sgmv_tensor* inputs, const sgmv_tensor* lora_b, const sgmv_tensor* out,
              const sgmv_tensor* seq_start, const sgmv_tensor* seq_len, const sgmv_tensor* lora_idx,
              int64_t batches, int64_t max_seq_len, int64_t slice_offset, int64_t slice_size,
              int add_inputs, int* variant);

/* Most slices one sgmv_expand_multi_slice call takes. */
#define SGMV_MAX_SLICES 4

/*
 * sgmv_expand_multi_slice -- several slices of one fused output in one call:
 * for each i < num_slices, the operation above with lora_b[i], slice_offset =
 * slice_offsets[i] and slice_size = lora_b[i]'s N (its shape[-2]), all sharing
 * inputs, out, the metadata and add_inputs.  The page explains that the
 * expand-slice kernel is kept apart from plain sgmv_expand so that a later
 * fused operator can update several slices in one launch ("Implementation:
 * Predibase Lorax SGMV Expand Slice Kernel", Description), and that the
 * slices are those of fused projections such as QKV or gate/up (Usage);
 * this is that operator.
 *
 *   lora_b         array of num_slices descriptors, each as lora_b above; they
 *                  may differ in N, strides and adapter count
 *   num_slices     1 .. SGMV_MAX_SLICES
 *   slice_offsets  HOST array of num_slices column offsets
 *
 * The slices' column ranges must be disjoint (else SGMV_ERR_SLICE_OVERLAP),
 * so the result equals the num_slices single-slice calls in any order, bit
 * for bit.  When the tensor-core kernel can take the whole set (same adapter
 * count and weight dtype, the alignment rules it needs) it runs as ONE launch
 * that shares the x tiles, the segment table and the prologue among the
 * slices; otherwise each slice is launched on its own.  Every argument is
 * validated before anything is enqueued.  Slices with N == 0 are skipped.
 */
SGMV_API int sgmv_expand_multi_slice(const sgmv_tensor* inputs, const sgmv_tensor* const* lora_b, int num_slices,
                            const sgmv_tensor* out, const sgmv_tensor* seq_start, const sgmv_tensor* seq_len,
                            const sgmv_tensor* lora_idx, int64_t batches, int64_t max_seq_len,
                            const int64_t* slice_offsets, int add_inputs, void* stream);

/*
 * sgmv_plan_multi_slice -- validate exactly as sgmv_expand_multi_slice does and
 * report the variant (SGMV_VARIANT_TC when the slices run as one fused launch,
 * SGMV_VARIANT_SIMT when the generic kernel is forced, 0 when nothing launches
 * or the slices run as separate launches with their own variants) and, in
 * *launches, how many kernel launches the call makes.  Launches nothing.
 */
SGMV_API int sgmv_plan_multi_slice(const sgmv_tensor* inputs, const sgmv_tensor* const* lora_b, int num_slices,
                          const sgmv_tensor* out, const sgmv_tensor* seq_start, const sgmv_tensor* seq_len,
                          const sgmv_tensor* lora_idx, int64_t batches, int64_t max_seq_len,
                          const int64_t* slice_offsets, int add_inputs, int* variant, int* launches);

/*
 * sgmv_expand -- the standard SGMV expand that the expand-slice operation
 * extends ("Implementation: Predibase Lorax SGMV Expand Slice Kernel",
 * Description): the whole output row is the slice, i.e. the operation above
 * with slice_offset = 0 and slice_size = N, where N = lora_b.shape[-2] must
 * equal out.shape[1] (else SGMV_ERR_OUT_WIDTH).  Every other argument, rule and
 * status is as for sgmv_expand_slice.
 */
SGMV_API int sgmv_expand(const sgmv_tensor* inputs, const sgmv_tensor* lora_b, const sgmv_tensor* out,
                const sgmv_tensor* seq_start, const sgmv_tensor* seq_len, const sgmv_tensor* lora_idx,
                int64_t batches, int64_t max_seq_len, int add_inputs, void* stream);

/*
 * bgmv_expand_slice -- the fixed-length counterpart of the expand-slice
 * operation (the page calls SGMV expand-slice "the variable-length sequence
 * counterpart to the BGMV expand slice kernel", Description): every row b <
 * batches is one token with its own adapter a = lora_idx[b],
 *
 *     out[b, off + n] = (add_inputs ? out[b, off + n] : 0) + sum_k x^[b, k] * B[a][n, k]
 *
 * which is sgmv_expand_slice with seq_start[b] = b and seq_len[b] = 1.  Same
 * tensors, dtypes, rounding, guards and statuses as sgmv_expand_slice, without
 * seq_start, seq_len and max_seq_len; rows at or beyond the row count of
 * inputs or of out are skipped.  Runs a kernel made for one token per row
 * (SGMV_VARIANT_DECODE) when B and x have unit column stride, K is a multiple
 * of 8 no larger than 256 and their rows start on 16-byte boundaries;
 * otherwise the generic CUDA-core kernel.
 */
SGMV_API int bgmv_expand_slice(const sgmv_tensor* inputs, const sgmv_tensor* lora_b, const sgmv_tensor* out,
                      const sgmv_tensor* lora_idx, int64_t batches, int64_t slice_offset, int64_t slice_size,
                      int add_inputs, void* stream);

/*
 * sgmv_shrink -- the LoRA A projection whose output is the expand-slice
 * operation's input (the page describes that input as "the low-rank
 * intermediate activations from the LoRA A projection", I/O Contract):
 *
 *     out[r, n] = sum_h x^[r, h] * A[a][n, h]       for n < R, h < H
 *
 * for every row r of every segment b with adapter a = lora_idx[b], i.e. the
 * expand-slice operation with lora_a in the weights' place (its N is the rank
 * R, its K the hidden size H), the whole output row as the slice, and
 * add_inputs off.  Same dtypes, rounding (x rounded to lora_a's dtype, fp32
 * sums, one rounding), guards, metadata and statuses as sgmv_expand_slice.
 *
 *   inputs    (T_x, H)                        f16 | bf16 | f32, any strides
 *   lora_a    (lora_num, R, H) or (lora_num, 1, R, H)   f16 | bf16, any strides
 *   out       (T_out, R)                      f16 | bf16 | f32, contiguous; out.shape[1]
 *             must equal R (else SGMV_ERR_OUT_WIDTH); rows outside the segments
 *             keep their bits
 *   workspace, workspace_bytes  optional DEVICE scratch (16-byte aligned, else
 *             SGMV_ERR_WORKSPACE), owned by the caller and used only by the
 *             work this call enqueues.  With it the tensor-core kernel splits
 *             H into up to 16 parts (the count a cost model of the busiest
 *             SM's bytes and per-item pipeline work prefers, halved until the
 *             partial sums fit) and adds the fp32 partial sums in a second
 *             kernel, in a fixed order (deterministic); without it (NULL or
 *             too small for two parts) each row block is one work item.
 *             Calls that run at the same time need separate workspaces.
 *
 * The tensor-core path (SGMV_VARIANT_TC) needs x and lora_a in the same half
 * dtype with unit column stride and 16-byte aligned rows, and R a multiple of
 * 16 in 16..128; other calls run the generic kernel.  The segment table is
 * staged in shared memory, which bounds batches (thousands of segments).
 */
SGMV_API int sgmv_shrink(const sgmv_tensor* inputs, const sgmv_tensor* lora_a, const sgmv_tensor* out,
                const sgmv_tensor* seq_start, const sgmv_tensor* seq_len, const sgmv_tensor* lora_idx,
                int64_t batches, int64_t max_seq_len, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device scratch that sgmv_shrink_static_scratch owns on every device. */
#define SGMV_SHRINK_STATIC_SCRATCH_BYTES (8u << 20)

/*
 * sgmv_shrink_static_scratch -- sgmv_shrink for callers that cannot allocate
 * device memory.  The paper has no counterpart: this entry point exists for
 * the caller, not for the method.
 *
 * Some callers are not allowed to allocate: a runtime that reserves all of
 * the GPU's memory when it starts and then forbids further allocations, a
 * plugin host that hands its plugins only their input and output buffers, or
 * a serving loop that must never stall on cudaMalloc, which can synchronise
 * the device.  Such a caller cannot provide sgmv_shrink's workspace, and
 * without one the shrink runs with one work item per row block.  This entry
 * point instead keeps the partial sums in a scratch array that the library
 * itself declares as a file-scope device variable of
 * SGMV_SHRINK_STATIC_SCRATCH_BYTES, which every GPU that loads the library
 * holds until the process exits.  It takes sgmv_shrink's arguments without
 * the workspace and computes exactly (bit for bit) what sgmv_shrink computes
 * with a workspace of SGMV_SHRINK_STATIC_SCRATCH_BYTES: the preferred H split
 * count, halved until the partial sums (splits x min(T_x, T_out) x R x 4
 * bytes) fit, down to one split, which needs no scratch at all.
 *
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and keeps it; make that first call before any
 *     stream capture.  Later calls only read the kept address.
 *   - It allocates nothing and calls no allocating routine.
 *   - Every call on a device shares the one array, and it keeps whatever the
 *     last call left there: each call writes every partial sum before it reads
 *     it, so nothing needs to start at zero, but two calls whose work overlaps
 *     on the GPU (different streams, no ordering between them) race on it.
 */
SGMV_API int sgmv_shrink_static_scratch(const sgmv_tensor* inputs, const sgmv_tensor* lora_a, const sgmv_tensor* out,
                               const sgmv_tensor* seq_start, const sgmv_tensor* seq_len,
                               const sgmv_tensor* lora_idx, int64_t batches, int64_t max_seq_len, void* stream);

/* sgmv_shrink_plan -- validate as sgmv_shrink does and report the variant a
 * call with a workspace of workspace_bytes would launch, its H split count,
 * and the workspace size (bytes) at which it would use its preferred split
 * count (0: the call wants none).  Launches nothing. */
SGMV_API int sgmv_shrink_plan(const sgmv_tensor* inputs, const sgmv_tensor* lora_a, const sgmv_tensor* out,
                     const sgmv_tensor* seq_start, const sgmv_tensor* seq_len, const sgmv_tensor* lora_idx,
                     int64_t batches, int64_t max_seq_len, size_t workspace_bytes, int* variant, int* splits,
                     size_t* preferred_workspace_bytes);

/* bgmv_plan -- validate as bgmv_expand_slice does; *variant receives the
 * kernel variant a call would launch (0 when nothing launches). */
SGMV_API int bgmv_plan(const sgmv_tensor* inputs, const sgmv_tensor* lora_b, const sgmv_tensor* out,
              const sgmv_tensor* lora_idx, int64_t batches, int64_t slice_offset, int64_t slice_size,
              int add_inputs, int* variant);

/*
 * sgmv_validate_metadata -- check the VALUES of the metadata on the device and
 * write a bit mask to *d_status (a device int32; 0 = all well):
 *   1   some lora_idx[b] is < -1 or >= lora_num
 *   2   some seq_start[b] < 0 or seq_len[b] < 0
 *   4   some segment (with a valid adapter) ends past total_rows
 *   8   two segments with valid adapters overlap
 *   16  starts of valid segments are not non-decreasing (overlap was then
 *       checked pairwise, or not at all when batches > 8192 -- bit 32 set)
 *   32  the pairwise overlap check was skipped
 * Never traps.  Enqueued on `stream`; the caller reads *d_status after
 * synchronising.  Same tensor rules as sgmv_expand_slice.
 */
SGMV_API int sgmv_validate_metadata(const sgmv_tensor* seq_start, const sgmv_tensor* seq_len,
                           const sgmv_tensor* lora_idx, int64_t batches, int64_t lora_num,
                           int64_t total_rows, int32_t* d_status, void* stream);

/* Human-readable name of a status code (static storage; never NULL). */
SGMV_API const char* sgmv_status_string(int code);

/*
 * sgmv_set_variant -- force the kernel variant used by later calls from any
 * host thread (SGMV_VARIANT_AUTO restores automatic choice).  A forced variant
 * that cannot run a call makes that call return SGMV_ERR_VARIANT.  Returns the
 * previous setting, or SGMV_ERR_VARIANT for an unknown value.  Meant for tests
 * and benchmarks.
 */
SGMV_API int sgmv_set_variant(int variant);

/*
 * sgmv_device_error -- read and clear the device-side error word of the
 * current device.  Kernels set it (instead of trapping) when a bounded wait on
 * an mbarrier gives up, which only a hardware or driver fault could cause.
 * Synchronises `stream`.  *value receives the word (0 = no error).
 */
SGMV_API int sgmv_device_error(void* stream, int32_t* value);

/* Library version as major*10000 + minor*100 + patch. */
SGMV_API int sgmv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SGMV_H */
