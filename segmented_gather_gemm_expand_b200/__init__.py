"""SGMV expand-slice for NVIDIA B200 (sm_100a): Python binding of libsgmv.

The binding only turns torch tensors into the C ABI's descriptors and passes
torch's current CUDA stream; every step of the operation runs in libsgmv's
CUDA kernels.  The operation and its arguments follow the wrapper described on
"Implementation: Predibase Lorax SGMV Expand Slice Kernel" (sections Signature
and I/O Contract):

    sgmv_expand_slice(inputs, lora_b_weights, output_tensor, b_seq_start_loc,
                      seq_len_tensor, lora_indices_tensor, batches,
                      max_seq_length, slice_offset, slice_size, add_inputs=False)

updates ``output_tensor[start_b + m, slice_offset:slice_offset + slice_size]``
for every sequence b with ``lora_indices_tensor[b] != -1`` and token m, with
``inputs[start_b + m] @ lora_b_weights[idx_b].T`` (added to the old values when
``add_inputs``).

``sgmv_expand_multi_slice`` updates several disjoint slices of one fused
output (the QKV or gate/up projections the page's Usage section names) in a
single call, which the page's Description anticipates as a fused operator.
``sgmv_expand`` is the standard expand the slice operation extends (the whole
output row is the slice), and ``bgmv_expand_slice`` its fixed-length
counterpart with one token per row (both named in the page's Description).
``sgmv_shrink`` is the LoRA-A projection that produces the expand's input
(I/O Contract, inputs).
"""
import ctypes

import torch

from . import _abi

__all__ = ["sgmv_expand_slice", "sgmv_expand_multi_slice", "sgmv_expand", "bgmv_expand_slice", "sgmv_shrink",
           "shrink_plan", "plan",
           "plan_multi_slice", "bgmv_plan", "validate_metadata", "set_variant", "device_error", "SgmvError",
           "VARIANT_AUTO", "VARIANT_SIMT", "VARIANT_TC", "VARIANT_DECODE", "VARIANT_TC_WIDE", "library_path"]

VARIANT_AUTO, VARIANT_SIMT, VARIANT_TC = _abi.VARIANT_AUTO, _abi.VARIANT_SIMT, _abi.VARIANT_TC
VARIANT_DECODE = _abi.VARIANT_DECODE
VARIANT_TC_WIDE = _abi.VARIANT_TC_WIDE
library_path = _abi.LIB_PATH

_DTYPES = {torch.float16: _abi.F16, torch.bfloat16: _abi.BF16, torch.float32: _abi.F32,
           torch.int32: _abi.I32, torch.int64: _abi.I64}

_lib = _abi.load()


class SgmvError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = _lib.sgmv_status_string(code).decode()
        super().__init__(f"{where}: {_abi.STATUS_NAMES.get(code, code)} ({msg})")


def _desc(t: torch.Tensor) -> _abi.SgmvTensor:
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return _abi.make_tensor(t.data_ptr(), _DTYPES[t.dtype], t.shape, t.stride())


def _stream_handle(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _args(inputs, lora_b_weights, output_tensor, b_seq_start_loc, seq_len_tensor,
          lora_indices_tensor):
    ts = [inputs, lora_b_weights, output_tensor, b_seq_start_loc, seq_len_tensor, lora_indices_tensor]
    for t in ts:
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors on the same device")
        if t.device != output_tensor.device:
            raise ValueError("all tensors must be on the same device")
    return [_desc(t) for t in ts]


def sgmv_expand_slice(inputs, lora_b_weights, output_tensor, b_seq_start_loc, seq_len_tensor,
                      lora_indices_tensor, batches, max_seq_length, slice_offset, slice_size,
                      add_inputs=False):
    """In-place SGMV expand-slice on ``output_tensor`` (enqueued on torch's current stream)."""
    d = _args(inputs, lora_b_weights, output_tensor, b_seq_start_loc, seq_len_tensor,
              lora_indices_tensor)
    with torch.cuda.device(output_tensor.device):
        rc = _lib.sgmv_expand_slice(*[ctypes.byref(x) for x in d], int(batches), int(max_seq_length),
                                    int(slice_offset), int(slice_size), int(bool(add_inputs)),
                                    _stream_handle(output_tensor.device))
    if rc != 0:
        raise SgmvError(rc, "sgmv_expand_slice")
    return output_tensor


def sgmv_expand(inputs, lora_b_weights, output_tensor, b_seq_start_loc, seq_len_tensor,
                lora_indices_tensor, batches, max_seq_length, add_inputs=False):
    """In-place standard SGMV expand: ``output_tensor`` is as wide as the slice
    (``lora_b_weights.shape[-2]``), which starts at column 0."""
    d = _args(inputs, lora_b_weights, output_tensor, b_seq_start_loc, seq_len_tensor,
              lora_indices_tensor)
    with torch.cuda.device(output_tensor.device):
        rc = _lib.sgmv_expand(*[ctypes.byref(x) for x in d], int(batches), int(max_seq_length),
                              int(bool(add_inputs)), _stream_handle(output_tensor.device))
    if rc != 0:
        raise SgmvError(rc, "sgmv_expand")
    return output_tensor


def _bgmv_args(inputs, lora_b_weights, output_tensor, lora_indices_tensor):
    ts = [inputs, lora_b_weights, output_tensor, lora_indices_tensor]
    for t in ts:
        if not t.is_cuda or t.device != output_tensor.device:
            raise ValueError("all tensors must be CUDA tensors on the same device")
    return [_desc(t) for t in ts]


def bgmv_expand_slice(inputs, lora_b_weights, output_tensor, lora_indices_tensor, slice_offset, slice_size,
                      add_inputs=False, batches=None):
    """In-place BGMV expand-slice: row b of ``inputs`` is one token with adapter
    ``lora_indices_tensor[b]``; ``batches`` defaults to ``inputs.shape[0]``."""
    batches = inputs.shape[0] if batches is None else batches
    d = _bgmv_args(inputs, lora_b_weights, output_tensor, lora_indices_tensor)
    with torch.cuda.device(output_tensor.device):
        rc = _lib.bgmv_expand_slice(*[ctypes.byref(x) for x in d], int(batches), int(slice_offset),
                                    int(slice_size), int(bool(add_inputs)), _stream_handle(output_tensor.device))
    if rc != 0:
        raise SgmvError(rc, "bgmv_expand_slice")
    return output_tensor


def bgmv_plan(inputs, lora_b_weights, output_tensor, lora_indices_tensor, slice_offset, slice_size,
              add_inputs=False, batches=None) -> int:
    """Kernel variant a bgmv_expand_slice call with these arguments would launch (0 = none)."""
    batches = inputs.shape[0] if batches is None else batches
    d = _bgmv_args(inputs, lora_b_weights, output_tensor, lora_indices_tensor)
    v = ctypes.c_int(0)
    with torch.cuda.device(output_tensor.device):
        rc = _lib.bgmv_plan(*[ctypes.byref(x) for x in d], int(batches), int(slice_offset), int(slice_size),
                            int(bool(add_inputs)), ctypes.byref(v))
    if rc != 0:
        raise SgmvError(rc, "bgmv_plan")
    return v.value


def _ws(workspace):
    if workspace is None:
        return None, 0
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size()


def sgmv_shrink(inputs, lora_a_weights, output_tensor, b_seq_start_loc, seq_len_tensor, lora_indices_tensor,
                batches, max_seq_length, workspace=None):
    """In-place SGMV shrink: ``output_tensor[r] = inputs[r] @ lora_a_weights[idx_b].T`` for the rows of
    every segment.  ``workspace``: optional contiguous CUDA tensor of scratch (see ``shrink_plan``)."""
    d = _args(inputs, lora_a_weights, output_tensor, b_seq_start_loc, seq_len_tensor, lora_indices_tensor)
    wp, wb = _ws(workspace)
    with torch.cuda.device(output_tensor.device):
        rc = _lib.sgmv_shrink(*[ctypes.byref(x) for x in d], int(batches), int(max_seq_length), wp, wb,
                              _stream_handle(output_tensor.device))
    if rc != 0:
        raise SgmvError(rc, "sgmv_shrink")
    return output_tensor


def shrink_plan(inputs, lora_a_weights, output_tensor, b_seq_start_loc, seq_len_tensor, lora_indices_tensor,
                batches, max_seq_length, workspace_bytes=0):
    """(variant, splits, preferred workspace bytes) of a shrink call with a workspace of that size."""
    d = _args(inputs, lora_a_weights, output_tensor, b_seq_start_loc, seq_len_tensor, lora_indices_tensor)
    v, sp, pref = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_size_t(0)
    with torch.cuda.device(output_tensor.device):
        rc = _lib.sgmv_shrink_plan(*[ctypes.byref(x) for x in d], int(batches), int(max_seq_length),
                                   int(workspace_bytes), ctypes.byref(v), ctypes.byref(sp), ctypes.byref(pref))
    if rc != 0:
        raise SgmvError(rc, "sgmv_shrink_plan")
    return v.value, sp.value, pref.value


def _multi_args(inputs, lora_b_list, output_tensor, b_seq_start_loc, seq_len_tensor,
                lora_indices_tensor, slice_offsets):
    lora_b_list = list(lora_b_list)
    offs = [int(o) for o in slice_offsets]
    if len(offs) != len(lora_b_list):
        raise ValueError("slice_offsets must have one entry per lora_b tensor")
    d = _args(inputs, output_tensor, output_tensor, b_seq_start_loc, seq_len_tensor,
              lora_indices_tensor)
    for w in lora_b_list:
        if not w.is_cuda or w.device != output_tensor.device:
            raise ValueError("all tensors must be CUDA tensors on the same device")
    ws = [_desc(w) for w in lora_b_list]
    n = len(ws)
    arr = (ctypes.POINTER(_abi.SgmvTensor) * max(n, 1))(*[ctypes.pointer(w) for w in ws])
    off_arr = (ctypes.c_int64 * max(n, 1))(*offs)
    keep = (ws, arr, off_arr)   # the descriptors must outlive the call
    return d[0], arr, n, d[2], d[3], d[4], d[5], off_arr, keep


def sgmv_expand_multi_slice(inputs, lora_b_list, output_tensor, b_seq_start_loc, seq_len_tensor,
                            lora_indices_tensor, batches, max_seq_length, slice_offsets,
                            add_inputs=False):
    """In-place expand-slice of every (lora_b_list[i], slice_offsets[i]) pair on
    ``output_tensor`` in one call; slice i's size is ``lora_b_list[i].shape[-2]``.
    The slices' column ranges must be disjoint."""
    x, arr, n, out, s, l, idx, offs, _keep = _multi_args(
        inputs, lora_b_list, output_tensor, b_seq_start_loc, seq_len_tensor, lora_indices_tensor,
        slice_offsets)
    with torch.cuda.device(output_tensor.device):
        rc = _lib.sgmv_expand_multi_slice(ctypes.byref(x), arr, n, ctypes.byref(out), ctypes.byref(s),
                                          ctypes.byref(l), ctypes.byref(idx), int(batches),
                                          int(max_seq_length), offs, int(bool(add_inputs)),
                                          _stream_handle(output_tensor.device))
    if rc != 0:
        raise SgmvError(rc, "sgmv_expand_multi_slice")
    return output_tensor


def plan_multi_slice(inputs, lora_b_list, output_tensor, b_seq_start_loc, seq_len_tensor,
                     lora_indices_tensor, batches, max_seq_length, slice_offsets, add_inputs=False):
    """(variant, launches) a multi-slice call with these arguments would make."""
    x, arr, n, out, s, l, idx, offs, _keep = _multi_args(
        inputs, lora_b_list, output_tensor, b_seq_start_loc, seq_len_tensor, lora_indices_tensor,
        slice_offsets)
    v, k = ctypes.c_int(0), ctypes.c_int(0)
    with torch.cuda.device(output_tensor.device):
        rc = _lib.sgmv_plan_multi_slice(ctypes.byref(x), arr, n, ctypes.byref(out), ctypes.byref(s),
                                        ctypes.byref(l), ctypes.byref(idx), int(batches),
                                        int(max_seq_length), offs, int(bool(add_inputs)),
                                        ctypes.byref(v), ctypes.byref(k))
    if rc != 0:
        raise SgmvError(rc, "sgmv_plan_multi_slice")
    return v.value, k.value


def plan(inputs, lora_b_weights, output_tensor, b_seq_start_loc, seq_len_tensor, lora_indices_tensor,
         batches, max_seq_length, slice_offset, slice_size, add_inputs=False) -> int:
    """Kernel variant a call with these arguments would launch (0 = none)."""
    d = _args(inputs, lora_b_weights, output_tensor, b_seq_start_loc, seq_len_tensor,
              lora_indices_tensor)
    v = ctypes.c_int(0)
    with torch.cuda.device(output_tensor.device):
        rc = _lib.sgmv_plan(*[ctypes.byref(x) for x in d], int(batches), int(max_seq_length),
                            int(slice_offset), int(slice_size), int(bool(add_inputs)), ctypes.byref(v))
    if rc != 0:
        raise SgmvError(rc, "sgmv_plan")
    return v.value


def validate_metadata(b_seq_start_loc, seq_len_tensor, lora_indices_tensor, batches, lora_num,
                      total_rows) -> int:
    """Device check of the metadata values; returns the status bit mask (synchronises)."""
    dev = b_seq_start_loc.device
    status = torch.empty(1, dtype=torch.int32, device=dev)
    d = [_desc(t) for t in (b_seq_start_loc, seq_len_tensor, lora_indices_tensor)]
    with torch.cuda.device(dev):
        rc = _lib.sgmv_validate_metadata(*[ctypes.byref(x) for x in d], int(batches), int(lora_num),
                                         int(total_rows), ctypes.c_void_p(status.data_ptr()),
                                         _stream_handle(dev))
    if rc != 0:
        raise SgmvError(rc, "sgmv_validate_metadata")
    return int(status.item())


def set_variant(variant: int) -> int:
    """Force a kernel variant for later calls (VARIANT_AUTO restores the default)."""
    rc = _lib.sgmv_set_variant(int(variant))
    if rc < 0:
        raise SgmvError(rc, "sgmv_set_variant")
    return rc


def device_error(device=None) -> int:
    """Read and clear the device error word (non-zero only after a kernel gave up a wait)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    v = ctypes.c_int32(0)
    with torch.cuda.device(dev):
        rc = _lib.sgmv_device_error(_stream_handle(dev), ctypes.byref(v))
    if rc != 0:
        raise SgmvError(rc, "sgmv_device_error")
    return v.value
