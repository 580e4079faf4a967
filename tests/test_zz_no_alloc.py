"""sgmv_shrink_static_scratch: the shrink for callers that cannot allocate.

Some callers may not allocate device memory at all (a runtime that reserves
the whole GPU up front, a plugin host that only passes buffers in and out, a
serving loop that must not stall on cudaMalloc).  This entry point keeps the
shrink's split-H partial sums in scratch the library declares itself, so such
a caller gets exactly what sgmv_shrink computes with a workspace of the same
size (SGMV_SHRINK_STATIC_SCRATCH_BYTES, 8 MiB).

The test calls it through the C ABI twice in a row, on different inputs, and
checks each result bit for bit against sgmv_shrink given an 8 MiB workspace of
its own (same split count, same fixed-order reduction), and every element
against the CPU oracle's shrink within the tolerance the other tests use.  The
inputs include a segment with adapter -1 and one of length zero, whose rows
must keep their bits.  A call whose preferred split count needs more than
8 MiB of partial sums runs with fewer splits, as sgmv_shrink does.  The file
is collected last and passes alone in a fresh process or after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sgmv_inputs as gen
import segmented_gather_gemm_expand_b200 as sg
from segmented_gather_gemm_expand_b200 import _abi
from sgmv_testlib import compare_every_element, from_torch, report, to_torch

pytestmark = pytest.mark.gpu

STATIC_BYTES = 8 << 20          # SGMV_SHRINK_STATIC_SCRATCH_BYTES in include/sgmv.h


def shrink_problem(seed, lengths, H, R, A, out_dt, idx=None):
    return gen.custom(seed=seed, lengths=lengths, K=H, N=R, H=R, offset=0, num_adapters=A, add_inputs=False,
                      out_dt=out_dt, idx=idx)


def device_args(p):
    c = p.calls[0]
    x, a, y = to_torch(p.x, p.x_dt), to_torch(c.w, p.w_dt), to_torch(p.y0, p.out_dt)
    meta = [torch.as_tensor(np.asarray(m)).cuda() for m in (p.seq_start, p.seq_len, p.lora_idx)]
    return x, a, y, meta


def static_scratch_call(x, a, y, meta, p):
    """The entry point under test, called through the C ABI with ctypes."""
    d = [sg._desc(t) for t in (x, a, y, *meta)]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sg._lib.sgmv_shrink_static_scratch(*[ctypes.byref(t) for t in d], p.batches, p.max_seq_len, stream)


def written_rows(p):
    rows = np.zeros(p.y0.shape[0], dtype=bool)
    for s, L, ai in zip(p.seq_start, p.seq_len, p.lora_idx):
        if 0 <= ai < p.calls[0].w.shape[0] and L > 0:
            rows[s:s + L] = True
    return rows


def oracle_shrink(p):
    return oracle.shrink(p.x, p.x_dt, p.calls[0].w, p.w_dt, p.y0, p.out_dt, p.seq_start, p.seq_len, p.lora_idx,
                         nthreads=oracle.max_threads())


def check_one(p, name):
    x, a, y, meta = device_args(p)
    v, splits, _ = sg.shrink_plan(x, a, y, *meta, p.batches, p.max_seq_len, STATIC_BYTES)
    ws = torch.empty(STATIC_BYTES, dtype=torch.uint8, device="cuda")
    y_ref = y.clone()
    sg.sgmv_shrink(x, a, y_ref, *meta, p.batches, p.max_seq_len, workspace=ws)
    rc = static_scratch_call(x, a, y, meta, p)
    assert rc == 0, _abi.STATUS_NAMES.get(rc, rc)
    torch.cuda.synchronize()
    assert sg.device_error() == 0
    got, want = from_torch(y, p.out_dt), from_torch(y_ref, p.out_dt)
    assert np.array_equal(got, want), "differs from sgmv_shrink with an 8 MiB workspace"
    rows = written_rows(p)
    err, count = compare_every_element(got, oracle_shrink(p), p, [(rows, 0, p.calls[0].w.shape[-2])])
    assert count == int(rows.sum()) * p.calls[0].w.shape[-2]
    report(f"static_scratch/{name}", variant=v, splits=splits, compared=count, max_abs_err=err)
    return v, splits


PROBLEMS = {
    # a -1 segment and a zero-length segment among them: their rows keep their bits
    "bf16_out": dict(seed=31, lengths=[300, 64, 0, 9, 700, 40], H=2048, R=16, A=4, out_dt="bf16",
                     idx=[0, -1, 2, 1, 3, 2]),
    "f32_out": dict(seed=32, lengths=[128, 5, 400, 0], H=1000, R=32, A=3, out_dt="f32", idx=[2, 0, 1, 0]),
}


@pytest.mark.parametrize("order", [0, 1])
def test_two_calls_in_a_row_match_the_workspace_entry_point(order):
    sg.set_variant(sg.VARIANT_AUTO)
    names = sorted(PROBLEMS)
    if order:
        names.reverse()
    for name in names:                      # two calls in a row on one device
        v, splits = check_one(shrink_problem(**PROBLEMS[name]), name)
        assert v == sg.VARIANT_TC and splits > 1


def test_a_call_whose_preferred_splits_do_not_fit_runs_with_fewer():
    sg.set_variant(sg.VARIANT_AUTO)
    p = shrink_problem(33, [2100], H=4096, R=128, A=1, out_dt="f32")   # splits x 2100 rows x 128 x 4 B > 8 MiB
    x, a, y, meta = device_args(p)
    _, pref_splits, pref = sg.shrink_plan(x, a, y, *meta, p.batches, p.max_seq_len, 1 << 40)
    assert pref > STATIC_BYTES, (pref_splits, pref)
    v, splits = check_one(p, "preferred_splits_too_large")
    assert v == sg.VARIANT_TC and splits < pref_splits
