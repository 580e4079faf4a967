"""CPU oracle for SGMV expand-slice -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py`
may import this package.  The CUDA library (`segmented_gather_gemm_expand_b200`)
never imports it and shares no code with it.

The arithmetic lives in `sgmv_oracle.c` (plain C, fp64 triple loop, one
rounding at the end); this module only marshals numpy arrays.  The operation
follows "Implementation: Predibase Lorax SGMV Expand Slice Kernel" (sections
Description, I/O Contract and Outputs): for each sequence b, each token m of
its segment and each n in the slice,
``out[s_b+m, off+n] = (add ? out[s_b+m, off+n] : 0) + x[s_b+m, :] . B[idx_b][n, :]``.

Dtypes are named 'f16', 'bf16', 'f32'.  Half-width tensors are passed as uint16
bit patterns, f32 tensors as float32 arrays.
"""
import ctypes
import os

import numpy as np

from . import build as _build

DTYPES = {"f16": 0, "bf16": 1, "f32": 2}

_lib = None


def _load():
    global _lib
    if _lib is None:
        # SGMV_ORACLE_LIB: used only by the mutation test, which loads a copy of
        # this oracle compiled with a deliberate bug to show the pins catch it.
        path = os.environ.get("SGMV_ORACLE_LIB") or _build.build()
        lib = ctypes.CDLL(path)
        i64, i32, vp, dp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.POINTER(ctypes.c_double)
        lib.orc_expand_slice.restype = i64
        lib.orc_expand_slice.argtypes = [vp, i32, i64, i64, i64, i64,
                                         vp, i32, i64, i64, i64, i64,
                                         vp, i32, i64, i64,
                                         vp, vp, vp, i64, i64, i64, i32, vp, i32]
        lib.orc_decode16.restype = ctypes.c_double
        lib.orc_decode16.argtypes = [ctypes.c_uint16, i32]
        lib.orc_encode16.restype = ctypes.c_uint16
        lib.orc_encode16.argtypes = [ctypes.c_double, i32]
        lib.orc_decode16_array.restype = None
        lib.orc_decode16_array.argtypes = [vp, vp, i64, i32]
        lib.orc_encode16_array.restype = None
        lib.orc_encode16_array.argtypes = [vp, vp, i64, i32]
        lib.orc_max_threads.restype = i32
        lib.orc_max_threads.argtypes = []
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().orc_max_threads())


def _storage_dtype(dt: str):
    return np.float32 if dt == "f32" else np.uint16


def decode(bits, dt: str) -> np.ndarray:
    """Bit patterns (uint16) of dtype `dt` -> exact float64 values.  f32 arrays pass through."""
    if dt == "f32":
        return np.asarray(bits, dtype=np.float32).astype(np.float64)
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    _load().orc_decode16_array(b.ctypes.data, out.ctypes.data, b.size, DTYPES[dt])
    return out


def encode(values, dt: str) -> np.ndarray:
    """float64 values -> dtype `dt` storage (uint16 bits, or float32), nearest-even."""
    v = np.ascontiguousarray(values, dtype=np.float64)
    if dt == "f32":
        return v.astype(np.float32)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().orc_encode16_array(v.ctypes.data, out.ctypes.data, v.size, DTYPES[dt])
    return out


def _elem_strides(a: np.ndarray):
    return [s // a.itemsize for s in a.strides]


def expand_slice(x, x_dt, w, w_dt, out, out_dt, seq_start, seq_len, lora_idx,
                 slice_offset, slice_size, add_inputs, batches=None, nthreads=1,
                 return_pre=False):
    """Run the oracle.  Returns a NEW array holding the updated `out`
    (and, if `return_pre`, a float64 (rows, slice_size) array of the values
    before the final rounding, NaN where nothing was written).

    x: (T, K) storage array (may be strided); w: (A, N, K) or (A, 1, N, K)
    storage array (may be strided); out: (T_out, H) storage array.
    """
    lib = _load()
    assert x.dtype == _storage_dtype(x_dt) and w.dtype == _storage_dtype(w_dt)
    assert out.dtype == _storage_dtype(out_dt)
    assert w_dt in ("f16", "bf16"), "weights are f16 or bf16"
    if w.ndim == 4:
        assert w.shape[1] == 1, "4-D weights must be (lora_num, 1, N, K)"
        w3 = w[:, 0]
    else:
        w3 = w
    A, N, K = w3.shape
    assert N == slice_size and x.shape[1] == K
    y = np.array(out, copy=True, order="C")
    T_out, H = y.shape
    assert 0 <= slice_offset and slice_offset + slice_size <= H
    ss = np.ascontiguousarray(seq_start, dtype=np.int64)
    sl = np.ascontiguousarray(seq_len, dtype=np.int64)
    li = np.ascontiguousarray(lora_idx, dtype=np.int64)
    B = len(ss) if batches is None else int(batches)
    assert len(ss) >= B and len(sl) >= B and len(li) >= B
    xs = _elem_strides(x)
    ws = _elem_strides(w3)
    pre = None
    pre_ptr = None
    if return_pre:
        pre = np.full((T_out, N), np.nan, dtype=np.float64)
        pre_ptr = pre.ctypes.data
    lib.orc_expand_slice(x.ctypes.data, DTYPES[x_dt], x.shape[0], K, xs[0], xs[1],
                         w3.ctypes.data, DTYPES[w_dt], A, ws[0], ws[1], ws[2],
                         y.ctypes.data, DTYPES[out_dt], T_out, H,
                         ss.ctypes.data, sl.ctypes.data, li.ctypes.data, B,
                         int(slice_offset), int(slice_size), int(bool(add_inputs)), pre_ptr,
                         int(nthreads))
    if return_pre:
        return y, pre
    return y


def expand(x, x_dt, w, w_dt, out, out_dt, seq_start, seq_len, lora_idx, add_inputs, batches=None,
           nthreads=1, return_pre=False):
    """The standard SGMV expand that the slice operation extends ("Implementation:
    Predibase Lorax SGMV Expand Slice Kernel", Description): the whole output
    row is the slice, so this is expand_slice with slice_offset 0 and
    slice_size = lora_b's N, which must equal out's width."""
    N = w.shape[-2]
    assert out.shape[1] == N, "plain expand writes whole rows: out's width must equal lora_b's N"
    return expand_slice(x, x_dt, w, w_dt, out, out_dt, seq_start, seq_len, lora_idx, 0, N, add_inputs,
                        batches=batches, nthreads=nthreads, return_pre=return_pre)


def bgmv_expand_slice(x, x_dt, w, w_dt, out, out_dt, lora_idx, slice_offset, slice_size, add_inputs,
                      batches=None, nthreads=1, return_pre=False):
    """BGMV expand-slice, the fixed-length counterpart the same page names
    (Description): row b (b < batches) is one token with adapter lora_idx[b],
    i.e. expand_slice with seq_start[b] = b and seq_len[b] = 1."""
    li = np.asarray(lora_idx, dtype=np.int64)
    B = len(li) if batches is None else int(batches)
    starts = np.arange(B, dtype=np.int64)
    lens = np.ones(B, dtype=np.int64)
    return expand_slice(x, x_dt, w, w_dt, out, out_dt, starts, lens, li[:B], slice_offset, slice_size,
                        add_inputs, batches=B, nthreads=nthreads, return_pre=return_pre)


def shrink(x, x_dt, a, a_dt, out, out_dt, seq_start, seq_len, lora_idx, batches=None, nthreads=1,
           return_pre=False):
    """The LoRA A projection that produces the expand input ("Implementation:
    Predibase Lorax SGMV Expand Slice Kernel", I/O Contract, inputs):
    out[r, n] = sum_h x[r, h] * A[a][n, h] over the rows of every segment.  It
    is the same segmented product as expand_slice with A (lora_num, R, H) in
    the weights' place, R output columns written from column 0, and no add."""
    R = a.shape[-2]
    assert out.shape[1] == R, "shrink writes whole rows: out's width must equal the rank"
    return expand_slice(x, x_dt, a, a_dt, out, out_dt, seq_start, seq_len, lora_idx, 0, R, False,
                        batches=batches, nthreads=nthreads, return_pre=return_pre)


def run_problem(p, nthreads=1, return_pre=False, out=None, call=0):
    """Run the oracle on a `sgmv_inputs.Problem` (one of its slice calls)."""
    c = p.calls[call]
    return expand_slice(p.x, p.x_dt, c.w, p.w_dt, p.y0 if out is None else out, p.out_dt,
                        p.seq_start, p.seq_len, p.lora_idx, c.slice_offset, c.slice_size,
                        p.add_inputs, nthreads=nthreads, return_pre=return_pre)


def run_problem_all_calls(p, nthreads=1):
    """Apply every slice call of the problem in order; returns the final output."""
    y = p.y0
    for i in range(len(p.calls)):
        y = run_problem(p, nthreads=nthreads, out=y, call=i)
    return y
