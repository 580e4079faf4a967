"""Launch plans are kept between calls (keyed by every field of the call); these
tests check that a kept plan is only reused for a call it fits.

Each call's result is compared, element by element, with the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
import sgmv_inputs as gen
import segmented_gather_gemm_expand_b200 as sg
from sgmv_testlib import DeviceProblem, compare_every_element, meta_tensors, to_torch, written_rows

pytestmark = pytest.mark.gpu

SHAPE = dict(K=16, N=1024, H=2048, offset=512, num_adapters=4)


def check(dp: DeviceProblem, p: gen.Problem, call=0):
    """Compare dp's output with the oracle run on p (the problem whose data dp now holds)."""
    torch.cuda.synchronize()
    assert sg.device_error() == 0
    gpu = dp.result()
    ref = oracle.run_problem(p, nthreads=oracle.max_threads(), call=call)
    c = p.calls[call]
    _, count = compare_every_element(gpu, ref, p, [(written_rows(p, call), c.slice_offset, c.slice_size)])
    assert count > 0


def fresh_output(dp: DeviceProblem):
    dp.y = to_torch(dp.p.y0, dp.p.out_dt)


def test_problems_of_one_shape_in_other_buffers():
    """Same shapes, other buffers: calls alternate between them and each writes its own output."""
    lengths = [300, 50, 700, 130]
    p1 = gen.custom(1, lengths=lengths, **SHAPE)
    p2 = gen.custom(2, lengths=lengths, **SHAPE)
    d1, d2 = DeviceProblem(p1), DeviceProblem(p2)
    for _ in range(2):
        for dp, p in ((d1, p1), (d2, p2)):
            fresh_output(dp)
            dp.run()
            check(dp, p)


def test_new_contents_in_the_same_buffers():
    """Same buffers refilled with another problem (other segment lengths, ids, values): the kept plan
    holds pointers only, so the call computes on the new contents."""
    p1 = gen.custom(3, lengths=[300, 50, 700, 130], **SHAPE)
    p2 = gen.custom(4, lengths=[700, 130, 50, 300], idx=[2, -1, 0, 3], **SHAPE)
    dp = DeviceProblem(p1)
    dp.run()
    check(dp, p1)
    dp.x.copy_(to_torch(p2.x, p2.x_dt))
    dp.ws[0].copy_(to_torch(p2.calls[0].w, p2.w_dt))
    dp.y.copy_(to_torch(p2.y0, p2.out_dt))
    for mine, new in zip((dp.start, dp.len, dp.idx), meta_tensors(p2)):
        mine.copy_(new)
    dp.p = p2
    dp.run()
    check(dp, p2)


def test_same_buffers_other_slice():
    """Same buffers, another slice offset: another plan."""
    p = gen.custom(5, lengths=[400, 9, 260], **dict(SHAPE, offset=0))
    dp = DeviceProblem(p)
    dp.run()
    check(dp, p)
    q = gen.custom(5, lengths=[400, 9, 260], **dict(SHAPE, offset=1024))
    q.y0 = p.y0
    dq = DeviceProblem(q)
    dq.x, dq.ws, dq.y, dq.start, dq.len, dq.idx = dp.x, dp.ws, to_torch(q.y0, q.out_dt), dp.start, dp.len, dp.idx
    dq.run()
    check(dq, q)


def test_shrink_same_buffers_other_workspace():
    """Same shrink buffers with and without a workspace (other split counts), twice each."""
    p = gen.custom(6, lengths=[513, 64, 9], K=2048, N=16, H=16, offset=0, num_adapters=2, add_inputs=False,
                   out_dt="f32")
    c = p.calls[0]
    x, a = to_torch(p.x, p.x_dt), to_torch(c.w, p.w_dt)
    meta = meta_tensors(p)
    _, _, pref = sg.shrink_plan(x, a, to_torch(p.y0, p.out_dt), *meta, p.batches, p.max_seq_len, 1 << 30)
    ws = torch.empty(max(pref, 16), dtype=torch.uint8, device="cuda")
    ref = oracle.shrink(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.seq_start, p.seq_len, p.lora_idx)
    rows = written_rows(p)
    for workspace in (ws, None, ws, None):
        y = to_torch(p.y0, p.out_dt)
        sg.sgmv_shrink(x, a, y, *meta, p.batches, p.max_seq_len, workspace=workspace)
        torch.cuda.synchronize()
        assert sg.device_error() == 0
        _, count = compare_every_element(y.cpu().numpy(), ref, p, [(rows, 0, 16)])
        assert count == int(rows.sum()) * 16


def test_metadata_written_on_the_device_just_before_the_call():
    """The scheduler of a short segment table reads the metadata before the preceding kernel may have
    finished and checks it again afterwards; here a device copy rewrites the metadata right before each
    call (same stream, no synchronisation), alternating between two batches of different lengths."""
    lengths_a = [300, 50, 700, 130]
    lengths_b = [700, 130, 50, 300]
    pa = gen.custom(7, lengths=lengths_a, **SHAPE)
    pb = gen.custom(7, lengths=lengths_b, idx=[1, 3, -1, 0], **SHAPE)
    pb.x = pa.x
    pb.calls[0] = pa.calls[0]
    dp = DeviceProblem(pa)
    meta = {"a": meta_tensors(pa), "b": meta_tensors(pb)}
    for name, p in (("b", pb), ("a", pa), ("b", pb)):
        dp.y = to_torch(p.y0, p.out_dt)
        for mine, new in zip((dp.start, dp.len, dp.idx), meta[name]):
            mine.copy_(new, non_blocking=True)
        dp.p = p
        dp.run()
        check(dp, p)
