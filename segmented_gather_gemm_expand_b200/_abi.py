"""ctypes declarations of libsgmv's C ABI (include/sgmv.h).

Argument marshalling only; no computation happens here.  Loading fails loudly
when the library has not been built: there is no fallback implementation.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsgmv.so")

# sgmv_dtype
F16, BF16, F32, I32, I64 = 0, 1, 2, 3, 4

SGMV_OK = 0
VARIANT_AUTO, VARIANT_SIMT, VARIANT_TC, VARIANT_DECODE, VARIANT_TC_WIDE = 0, 1, 2, 3, 4

STATUS_NAMES = {
    0: "SGMV_OK", -1: "SGMV_ERR_NULL_ARG", -2: "SGMV_ERR_DTYPE", -3: "SGMV_ERR_NDIM",
    -4: "SGMV_ERR_RANK_MISMATCH", -5: "SGMV_ERR_SLICE_SIZE", -6: "SGMV_ERR_LAYOUT_4D",
    -7: "SGMV_ERR_OUT_NOT_CONTIGUOUS", -8: "SGMV_ERR_SLICE_RANGE", -9: "SGMV_ERR_BATCHES",
    -10: "SGMV_ERR_SHAPE", -11: "SGMV_ERR_STRIDE", -12: "SGMV_ERR_TOO_LARGE",
    -13: "SGMV_ERR_VARIANT", -14: "SGMV_ERR_NUM_SLICES", -15: "SGMV_ERR_SLICE_OVERLAP",
    -16: "SGMV_ERR_OUT_WIDTH", -17: "SGMV_ERR_WORKSPACE",
    -18: "SGMV_ERR_SCRATCH",
    -20: "SGMV_ERR_CUDA", -21: "SGMV_ERR_LAUNCH",
}
MAX_SLICES = 4
STATUS = {v: k for k, v in STATUS_NAMES.items()}


class SgmvTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


def make_tensor(data_ptr, dtype, shape, strides):
    t = SgmvTensor()
    t.data = ctypes.c_void_p(int(data_ptr)) if data_ptr else None
    t.dtype = int(dtype)
    t.ndim = len(shape)
    for i, (s, st) in enumerate(zip(shape, strides)):
        t.shape[i] = int(s)
        t.stride[i] = int(st)
    return t


_lib = None


def load():
    """Load libsgmv.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsgmv.so not found at {LIB_PATH}; build it with "
                          "`python segmented_gather_gemm_expand_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(SgmvTensor)
    i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    lib.sgmv_expand_slice.restype = i32
    lib.sgmv_expand_slice.argtypes = [P, P, P, P, P, P, i64, i64, i64, i64, i32, vp]
    lib.sgmv_plan.restype = i32
    lib.sgmv_plan.argtypes = [P, P, P, P, P, P, i64, i64, i64, i64, i32, ctypes.POINTER(i32)]
    PP = ctypes.POINTER(P)
    I64P = ctypes.POINTER(i64)
    lib.sgmv_expand_multi_slice.restype = i32
    lib.sgmv_expand_multi_slice.argtypes = [P, PP, i32, P, P, P, P, i64, i64, I64P, i32, vp]
    lib.sgmv_plan_multi_slice.restype = i32
    lib.sgmv_plan_multi_slice.argtypes = [P, PP, i32, P, P, P, P, i64, i64, I64P, i32,
                                          ctypes.POINTER(i32), ctypes.POINTER(i32)]
    lib.sgmv_expand.restype = i32
    lib.sgmv_expand.argtypes = [P, P, P, P, P, P, i64, i64, i32, vp]
    lib.bgmv_expand_slice.restype = i32
    lib.bgmv_expand_slice.argtypes = [P, P, P, P, i64, i64, i64, i32, vp]
    lib.bgmv_plan.restype = i32
    lib.bgmv_plan.argtypes = [P, P, P, P, i64, i64, i64, i32, ctypes.POINTER(i32)]
    sz = ctypes.c_size_t
    lib.sgmv_shrink.restype = i32
    lib.sgmv_shrink.argtypes = [P, P, P, P, P, P, i64, i64, vp, sz, vp]
    lib.sgmv_shrink_static_scratch.restype = i32
    lib.sgmv_shrink_static_scratch.argtypes = [P, P, P, P, P, P, i64, i64, vp]
    lib.sgmv_shrink_plan.restype = i32
    lib.sgmv_shrink_plan.argtypes = [P, P, P, P, P, P, i64, i64, sz, ctypes.POINTER(i32), ctypes.POINTER(i32),
                                     ctypes.POINTER(sz)]
    lib.sgmv_validate_metadata.restype = i32
    lib.sgmv_validate_metadata.argtypes = [P, P, P, i64, i64, i64, vp, vp]
    lib.sgmv_status_string.restype = ctypes.c_char_p
    lib.sgmv_status_string.argtypes = [i32]
    lib.sgmv_set_variant.restype = i32
    lib.sgmv_set_variant.argtypes = [i32]
    lib.sgmv_device_error.restype = i32
    lib.sgmv_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
    lib.sgmv_version.restype = i32
    lib.sgmv_version.argtypes = []
    _lib = lib
    return lib
