"""sgmv_shrink_static_scratch: the shrink for callers that cannot allocate.

Some callers may not allocate device memory at all (a runtime that reserves
the whole GPU up front, a plugin host that only passes buffers in and out, a
serving loop that must not stall on cudaMalloc).  This entry point keeps the
shrink's partial sums in scratch the library declares itself, so such a
caller gets the same result as sgmv_shrink with a workspace of its own.  The
test calls it through the C ABI twice in a row, on different inputs, and
checks each result against sgmv_shrink's within the tolerance the other tests
use; it also checks that a call needing more scratch than the library holds is
refused before anything is written.  It lives in a file of its own, collected
last, and passes alone in a fresh process or after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import sgmv_inputs as gen
import segmented_gather_gemm_expand_b200 as sg
from segmented_gather_gemm_expand_b200 import _abi
from sgmv_testlib import compare, from_torch, to_torch

pytestmark = pytest.mark.gpu


def shrink_problem(seed, lengths, H, R, A, out_dt):
    return gen.custom(seed=seed, lengths=lengths, K=H, N=R, H=R, offset=0, num_adapters=A, add_inputs=False,
                      out_dt=out_dt)


def device_args(p):
    c = p.calls[0]
    x, a, y = to_torch(p.x, p.x_dt), to_torch(c.w, p.w_dt), to_torch(p.y0, p.out_dt)
    meta = [torch.as_tensor(np.asarray(m)).cuda() for m in (p.seq_start, p.seq_len, p.lora_idx)]
    return x, a, y, meta


def static_scratch_call(x, a, y, meta, p):
    """The new entry point, called through the C ABI with ctypes."""
    d = [sg._desc(t) for t in (x, a, y, *meta)]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sg._lib.sgmv_shrink_static_scratch(*[ctypes.byref(t) for t in d], p.batches, p.max_seq_len, stream)


def written_rows(p):
    rows = np.zeros(p.y0.shape[0], dtype=bool)
    for s, L, ai in zip(p.seq_start, p.seq_len, p.lora_idx):
        if 0 <= ai < p.calls[0].w.shape[0] and L > 0:
            rows[s:s + L] = True
    return rows


@pytest.mark.parametrize("case", [0, 1])
def test_two_calls_in_a_row_match_the_workspace_entry_point(case):
    sg.set_variant(sg.VARIANT_AUTO)
    problems = [shrink_problem(31, [300, 64, 9, 700], H=2048, R=16, A=4, out_dt="bf16"),
                shrink_problem(32, [128, 5, 400], H=1000, R=32, A=3, out_dt="f32")]
    if case:
        problems.reverse()
    for p in problems:                      # two calls in a row on one device
        x, a, y, meta = device_args(p)
        v, splits, pref = sg.shrink_plan(x, a, y, *meta, p.batches, p.max_seq_len, 1 << 30)
        assert v == sg.VARIANT_TC and splits > 1
        assert pref <= _abi_static_bytes()
        ws = torch.empty(pref, dtype=torch.uint8, device="cuda")
        y_ref = y.clone()
        sg.sgmv_shrink(x, a, y_ref, *meta, p.batches, p.max_seq_len, workspace=ws)
        rc = static_scratch_call(x, a, y, meta, p)
        assert rc == 0, _abi.STATUS_NAMES.get(rc, rc)
        torch.cuda.synchronize()
        assert sg.device_error() == 0
        compare(from_torch(y, p.out_dt), from_torch(y_ref, p.out_dt), p.y0, p, written_rows(p), 0,
                p.calls[0].w.shape[-2])


def test_a_call_needing_more_scratch_is_refused():
    sg.set_variant(sg.VARIANT_AUTO)
    p = shrink_problem(33, [2100], H=4096, R=128, A=1, out_dt="f32")   # splits x 2100 rows x 128 x 4 B > 8 MiB
    x, a, y, meta = device_args(p)
    _, splits, pref = sg.shrink_plan(x, a, y, *meta, p.batches, p.max_seq_len, 1 << 40)
    assert pref > _abi_static_bytes(), (splits, pref)
    rc = static_scratch_call(x, a, y, meta, p)
    assert rc == _abi.STATUS["SGMV_ERR_SCRATCH"]
    torch.cuda.synchronize()
    assert np.array_equal(from_torch(y, p.out_dt), p.y0)


def _abi_static_bytes():
    return 8 << 20          # SGMV_SHRINK_STATIC_SCRATCH_BYTES in include/sgmv.h
