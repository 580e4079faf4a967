"""Host-only checks of the C ABI (no GPU needed, no kernel launched).

- libsgmv.so loads and exports every function include/sgmv.h declares;
- every status code has a name;
- invalid arguments return their specific error code before any CUDA call
  (these calls use fake, never-dereferenced data pointers).
"""
import ctypes
import os
import re

import pytest

from segmented_gather_gemm_expand_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"SGMV_API\s+[\w\s\*]+?\b((?:sgmv|bgmv)_\w+)\s*\(", text)
    return names


def test_library_exports_every_declared_symbol():
    lib = _abi.load()
    names = declared_functions()
    assert "sgmv_expand_slice" in names and len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version():
    lib = _abi.load()
    for code, name in _abi.STATUS_NAMES.items():
        s = lib.sgmv_status_string(code).decode()
        assert s and s != "unknown status", name
    assert lib.sgmv_status_string(-999).decode() == "unknown status"
    assert lib.sgmv_version() >= 100


def test_set_variant_round_trip():
    lib = _abi.load()
    prev = lib.sgmv_set_variant(_abi.VARIANT_SIMT)
    assert prev == _abi.VARIANT_AUTO
    assert lib.sgmv_set_variant(_abi.VARIANT_AUTO) == _abi.VARIANT_SIMT
    assert lib.sgmv_set_variant(7) == _abi.STATUS["SGMV_ERR_VARIANT"]


FAKE = 0x10000   # never dereferenced: every case below fails validation first


def good_args(**over):
    T, K, A, N, H, B = 20, 16, 3, 128, 384, 4
    a = dict(
        x=_abi.make_tensor(FAKE, _abi.BF16, (T, K), (K, 1)),
        w=_abi.make_tensor(FAKE, _abi.BF16, (A, N, K), (N * K, K, 1)),
        out=_abi.make_tensor(FAKE, _abi.BF16, (T, H), (H, 1)),
        s=_abi.make_tensor(FAKE, _abi.I64, (B,), (1,)),
        l=_abi.make_tensor(FAKE, _abi.I64, (B,), (1,)),
        i=_abi.make_tensor(FAKE, _abi.I32, (B,), (1,)),
        batches=B, max_seq_len=7, off=128, size=N, add=0,
    )
    a.update(over)
    return a


def call(a):
    lib = _abi.load()
    r = ctypes.byref
    return lib.sgmv_expand_slice(r(a["x"]), r(a["w"]), r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]),
                                 a["batches"], a["max_seq_len"], a["off"], a["size"], a["add"], None)


def plan(a):
    lib = _abi.load()
    r = ctypes.byref
    v = ctypes.c_int(-1)
    rc = lib.sgmv_plan(r(a["x"]), r(a["w"]), r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]),
                       a["batches"], a["max_seq_len"], a["off"], a["size"], a["add"], r(v))
    return rc, v.value


T, K, A, N, H, B = 20, 16, 3, 128, 384, 4
BAD_CASES = {
    "x_dtype_int": (dict(x=_abi.make_tensor(FAKE, _abi.I32, (T, K), (K, 1))), "SGMV_ERR_DTYPE"),
    "w_dtype_f32": (dict(w=_abi.make_tensor(FAKE, _abi.F32, (A, N, K), (N * K, K, 1))), "SGMV_ERR_DTYPE"),
    "out_dtype_i64": (dict(out=_abi.make_tensor(FAKE, _abi.I64, (T, H), (H, 1))), "SGMV_ERR_DTYPE"),
    "meta_dtype_f16": (dict(s=_abi.make_tensor(FAKE, _abi.F16, (B,), (1,))), "SGMV_ERR_DTYPE"),
    "x_3d": (dict(x=_abi.make_tensor(FAKE, _abi.BF16, (T, K, 1), (K, 1, 1))), "SGMV_ERR_NDIM"),
    "w_2d": (dict(w=_abi.make_tensor(FAKE, _abi.BF16, (N, K), (K, 1))), "SGMV_ERR_NDIM"),
    "meta_2d": (dict(l=_abi.make_tensor(FAKE, _abi.I64, (B, 1), (1, 1))), "SGMV_ERR_NDIM"),
    "rank_mismatch": (dict(x=_abi.make_tensor(FAKE, _abi.BF16, (T, 8), (8, 1))), "SGMV_ERR_RANK_MISMATCH"),
    "slice_size_mismatch": (dict(size=64), "SGMV_ERR_SLICE_SIZE"),
    "w_4d_bad_unit_dim": (dict(w=_abi.make_tensor(FAKE, _abi.BF16, (A, 2, N, K), (2 * N * K, N * K, K, 1))),
                          "SGMV_ERR_LAYOUT_4D"),
    "out_transposed": (dict(out=_abi.make_tensor(FAKE, _abi.BF16, (T, H), (1, T))), "SGMV_ERR_OUT_NOT_CONTIGUOUS"),
    "out_row_pitch": (dict(out=_abi.make_tensor(FAKE, _abi.BF16, (T, H), (H + 8, 1))), "SGMV_ERR_OUT_NOT_CONTIGUOUS"),
    "slice_past_width": (dict(off=300), "SGMV_ERR_SLICE_RANGE"),
    "negative_offset": (dict(off=-1), "SGMV_ERR_SLICE_RANGE"),
    "negative_batches": (dict(batches=-1), "SGMV_ERR_BATCHES"),
    "meta_shorter_than_batches": (dict(batches=5), "SGMV_ERR_BATCHES"),
    "negative_max_seq_len": (dict(max_seq_len=-3), "SGMV_ERR_SHAPE"),
    "negative_extent": (dict(x=_abi.make_tensor(FAKE, _abi.BF16, (-1, K), (K, 1))), "SGMV_ERR_SHAPE"),
    "negative_stride": (dict(x=_abi.make_tensor(FAKE, _abi.BF16, (T, K), (-K, 1))), "SGMV_ERR_STRIDE"),
    "null_x_data": (dict(x=_abi.make_tensor(0, _abi.BF16, (T, K), (K, 1))), "SGMV_ERR_NULL_ARG"),
    "null_meta_data": (dict(i=_abi.make_tensor(0, _abi.I32, (B,), (1,))), "SGMV_ERR_NULL_ARG"),
    "huge_extent": (dict(out=_abi.make_tensor(FAKE, _abi.BF16, (1 << 41, H), (H, 1))), "SGMV_ERR_TOO_LARGE"),
}


@pytest.mark.parametrize("case", sorted(BAD_CASES))
def test_invalid_arguments_fail_before_launch(case):
    over, code = BAD_CASES[case]
    a = good_args(**over)
    assert call(a) == _abi.STATUS[code]
    rc, v = plan(a)
    assert rc == _abi.STATUS[code] and v == 0


def test_null_descriptor():
    lib = _abi.load()
    a = good_args()
    r = ctypes.byref
    rc = lib.sgmv_expand_slice(None, r(a["w"]), r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]),
                               4, 7, 128, 128, 0, None)
    assert rc == _abi.STATUS["SGMV_ERR_NULL_ARG"]


def test_validate_metadata_rejects_bad_arguments():
    lib = _abi.load()
    a = good_args()
    r = ctypes.byref
    assert lib.sgmv_validate_metadata(r(a["s"]), r(a["l"]), r(a["i"]), 4, 3, 20, None, None) == \
        _abi.STATUS["SGMV_ERR_NULL_ARG"]
    assert lib.sgmv_validate_metadata(r(a["s"]), r(a["l"]), r(a["i"]), 9, 3, 20, FAKE, None) == \
        _abi.STATUS["SGMV_ERR_BATCHES"]
    assert lib.sgmv_validate_metadata(r(a["s"]), r(a["l"]), r(a["i"]), 4, -1, 20, FAKE, None) == \
        _abi.STATUS["SGMV_ERR_SHAPE"]


def test_empty_calls_need_no_device_and_launch_nothing():
    # batches == 0 and slice_size == 0 return OK before any CUDA call.
    assert call(good_args(batches=0)) == 0
    empty_w = _abi.make_tensor(FAKE, _abi.BF16, (A, 0, K), (0, K, 1))
    assert call(good_args(w=empty_w, size=0)) == 0


# --- several slices of one output (sgmv_expand_multi_slice) -----------------

def call_multi(a, ws, offs, n=None):
    lib = _abi.load()
    r = ctypes.byref
    n = len(ws) if n is None else n
    arr = (ctypes.POINTER(_abi.SgmvTensor) * max(len(ws), 1))(*[ctypes.pointer(w) for w in ws])
    off_arr = (ctypes.c_int64 * max(len(offs), 1))(*offs)
    rc = lib.sgmv_expand_multi_slice(r(a["x"]), arr, n, r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]),
                                     a["batches"], a["max_seq_len"], off_arr, a["add"], None)
    v, k = ctypes.c_int(-1), ctypes.c_int(-1)
    rc2 = lib.sgmv_plan_multi_slice(r(a["x"]), arr, n, r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]),
                                    a["batches"], a["max_seq_len"], off_arr, a["add"], r(v), r(k))
    assert rc2 == rc
    if rc:
        assert v.value == 0 and k.value == 0
    return rc


def wslice(n):
    return _abi.make_tensor(FAKE, _abi.BF16, (A, n, K), (n * K, K, 1))


def test_multi_slice_overlapping_ranges_rejected():
    a = good_args()
    assert call_multi(a, [wslice(128), wslice(128)], [0, 64]) == _abi.STATUS["SGMV_ERR_SLICE_OVERLAP"]
    assert call_multi(a, [wslice(128), wslice(64), wslice(64)], [0, 256, 300]) == \
        _abi.STATUS["SGMV_ERR_SLICE_OVERLAP"]
    # the same slice twice
    assert call_multi(a, [wslice(128), wslice(128)], [128, 128]) == _abi.STATUS["SGMV_ERR_SLICE_OVERLAP"]


def test_multi_slice_count_and_null_checks():
    lib = _abi.load()
    a = good_args()
    assert call_multi(a, [wslice(64)] * 5, [0, 64, 128, 192, 256]) == _abi.STATUS["SGMV_ERR_NUM_SLICES"]
    assert call_multi(a, [wslice(64)], [0], n=0) == _abi.STATUS["SGMV_ERR_NUM_SLICES"]
    r = ctypes.byref
    off_arr = (ctypes.c_int64 * 1)(0)
    assert lib.sgmv_expand_multi_slice(r(a["x"]), None, 1, r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]),
                                       4, 7, off_arr, 0, None) == _abi.STATUS["SGMV_ERR_NULL_ARG"]
    arr = (ctypes.POINTER(_abi.SgmvTensor) * 1)(ctypes.pointer(wslice(64)))
    assert lib.sgmv_expand_multi_slice(r(a["x"]), arr, 1, r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]),
                                       4, 7, None, 0, None) == _abi.STATUS["SGMV_ERR_NULL_ARG"]
    arr2 = (ctypes.POINTER(_abi.SgmvTensor) * 2)(ctypes.pointer(wslice(64)), None)
    off2 = (ctypes.c_int64 * 2)(0, 64)
    assert lib.sgmv_expand_multi_slice(r(a["x"]), arr2, 2, r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]),
                                       4, 7, off2, 0, None) == _abi.STATUS["SGMV_ERR_NULL_ARG"]


def test_multi_slice_validates_every_slice():
    a = good_args()
    # slice 2 reaches past the output width
    assert call_multi(a, [wslice(128), wslice(128)], [0, 300]) == _abi.STATUS["SGMV_ERR_SLICE_RANGE"]
    # slice 2 has the wrong rank
    bad_rank = _abi.make_tensor(FAKE, _abi.BF16, (A, 64, 8), (64 * 8, 8, 1))
    assert call_multi(a, [wslice(64), bad_rank], [0, 64]) == _abi.STATUS["SGMV_ERR_RANK_MISMATCH"]
    bad_dt = _abi.make_tensor(FAKE, _abi.F32, (A, 64, K), (64 * K, K, 1))
    assert call_multi(a, [bad_dt], [0]) == _abi.STATUS["SGMV_ERR_DTYPE"]
    assert call_multi(a, [wslice(64), _abi.make_tensor(FAKE, _abi.BF16, (64, K), (K, 1))], [0, 64]) == \
        _abi.STATUS["SGMV_ERR_NDIM"]


def test_multi_slice_empty_needs_no_device():
    # every slice empty, or no batches: OK before any CUDA call
    a = good_args()
    assert call_multi(a, [wslice(0), wslice(0)], [0, 0]) == 0
    assert call_multi(good_args(batches=0), [wslice(128), wslice(128)], [0, 128]) == 0
    # an empty slice inside a non-empty one overlaps nothing
    assert call_multi(good_args(batches=0), [wslice(128), wslice(0)], [0, 64]) == 0


# ------------------------------------------------------------ plain expand and BGMV

def test_plain_expand_rejects_a_partial_width_output():
    lib = _abi.load()
    a = good_args()          # out is wider than lora_b's N: a slice call, not a plain expand
    r = ctypes.byref
    rc = lib.sgmv_expand(r(a["x"]), r(a["w"]), r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]),
                         a["batches"], a["max_seq_len"], a["add"], None)
    assert rc == _abi.STATUS["SGMV_ERR_OUT_WIDTH"]
    w2 = _abi.make_tensor(FAKE, _abi.BF16, (A, N), (N, 1))
    assert lib.sgmv_expand(r(a["x"]), r(w2), r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]), 4, 7, 0, None) == \
        _abi.STATUS["SGMV_ERR_NDIM"]
    assert lib.sgmv_expand(r(a["x"]), None, r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]), 4, 7, 0, None) == \
        _abi.STATUS["SGMV_ERR_NULL_ARG"]


BGMV_BAD = {
    "idx_shorter_than_batches": (dict(batches=5), "SGMV_ERR_BATCHES"),
    "slice_past_width": (dict(off=300), "SGMV_ERR_SLICE_RANGE"),
    "slice_size_mismatch": (dict(size=64), "SGMV_ERR_SLICE_SIZE"),
    "w_dtype_f32": (dict(w=_abi.make_tensor(FAKE, _abi.F32, (A, N, K), (N * K, K, 1))), "SGMV_ERR_DTYPE"),
    "idx_dtype_f16": (dict(i=_abi.make_tensor(FAKE, _abi.F16, (B,), (1,))), "SGMV_ERR_DTYPE"),
    "rank_mismatch": (dict(x=_abi.make_tensor(FAKE, _abi.BF16, (T, 8), (8, 1))), "SGMV_ERR_RANK_MISMATCH"),
    "negative_batches": (dict(batches=-2), "SGMV_ERR_BATCHES"),
}


@pytest.mark.parametrize("case", sorted(BGMV_BAD))
def test_bgmv_invalid_arguments_fail_before_launch(case):
    lib = _abi.load()
    over, code = BGMV_BAD[case]
    a = good_args(**over)
    r = ctypes.byref
    rc = lib.bgmv_expand_slice(r(a["x"]), r(a["w"]), r(a["out"]), r(a["i"]), a["batches"], a["off"], a["size"],
                               a["add"], None)
    assert rc == _abi.STATUS[code]
    v = ctypes.c_int(-1)
    rc = lib.bgmv_plan(r(a["x"]), r(a["w"]), r(a["out"]), r(a["i"]), a["batches"], a["off"], a["size"],
                       a["add"], r(v))
    assert rc == _abi.STATUS[code] and v.value == 0


def test_decode_variant_is_only_for_bgmv():
    """Forcing the one-token kernel makes expand-slice calls report SGMV_ERR_VARIANT (before any launch)."""
    lib = _abi.load()
    prev = lib.sgmv_set_variant(3)
    try:
        a = good_args()
        assert call(a) == _abi.STATUS["SGMV_ERR_VARIANT"]
    finally:
        lib.sgmv_set_variant(prev)


# ------------------------------------------------------------ shrink

def shrink_args(**over):
    T, H, A, R, B = 20, 256, 3, 16, 4
    a = dict(
        x=_abi.make_tensor(FAKE, _abi.BF16, (T, H), (H, 1)),
        w=_abi.make_tensor(FAKE, _abi.BF16, (A, R, H), (R * H, H, 1)),
        out=_abi.make_tensor(FAKE, _abi.F32, (T, R), (R, 1)),
        s=_abi.make_tensor(FAKE, _abi.I64, (B,), (1,)),
        l=_abi.make_tensor(FAKE, _abi.I64, (B,), (1,)),
        i=_abi.make_tensor(FAKE, _abi.I32, (B,), (1,)),
        batches=B, max_seq_len=7, ws=None, ws_bytes=0,
    )
    a.update(over)
    return a


def shrink_call(a):
    lib = _abi.load()
    r = ctypes.byref
    return lib.sgmv_shrink(r(a["x"]), r(a["w"]), r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]), a["batches"],
                           a["max_seq_len"], a["ws"], a["ws_bytes"], None)


SHRINK_BAD = {
    "out_width_not_rank": (dict(out=_abi.make_tensor(FAKE, _abi.F32, (20, 32), (32, 1))), "SGMV_ERR_OUT_WIDTH"),
    "hidden_size_mismatch": (dict(x=_abi.make_tensor(FAKE, _abi.BF16, (20, 128), (128, 1))), "SGMV_ERR_RANK_MISMATCH"),
    "a_2d": (dict(w=_abi.make_tensor(FAKE, _abi.BF16, (16, 256), (256, 1))), "SGMV_ERR_NDIM"),
    "a_f32": (dict(w=_abi.make_tensor(FAKE, _abi.F32, (3, 16, 256), (16 * 256, 256, 1))), "SGMV_ERR_DTYPE"),
    "a_4d_bad_unit_dim": (dict(w=_abi.make_tensor(FAKE, _abi.BF16, (3, 2, 16, 256), (2 * 16 * 256, 16 * 256, 256, 1))),
                          "SGMV_ERR_LAYOUT_4D"),
    "out_not_contiguous": (dict(out=_abi.make_tensor(FAKE, _abi.F32, (20, 16), (17, 1))), "SGMV_ERR_OUT_NOT_CONTIGUOUS"),
    "meta_short": (dict(batches=6), "SGMV_ERR_BATCHES"),
    "misaligned_workspace": (dict(ws=FAKE + 4, ws_bytes=1 << 20), "SGMV_ERR_WORKSPACE"),
}


@pytest.mark.parametrize("case", sorted(SHRINK_BAD))
def test_shrink_invalid_arguments_fail_before_launch(case):
    over, code = SHRINK_BAD[case]
    assert shrink_call(shrink_args(**over)) == _abi.STATUS[code]


def test_shrink_plan_null_outputs():
    lib = _abi.load()
    a = shrink_args()
    r = ctypes.byref
    v = ctypes.c_int(0)
    assert lib.sgmv_shrink_plan(r(a["x"]), r(a["w"]), r(a["out"]), r(a["s"]), r(a["l"]), r(a["i"]), 4, 7, 0,
                                r(v), None, None) == _abi.STATUS["SGMV_ERR_NULL_ARG"]
