"""GPU parity of SGMV shrink (the LoRA A projection) against the CPU oracle.

out[r, n] = sum_h x^[r, h] * A[a][n, h] for the rows of every segment: the
expand operation's segmented product with the reduction over the hidden size.
Tolerance as in the expand tests, with the hidden size as the reduction length.
"""
import numpy as np
import pytest
import torch

import oracle
import sgmv_inputs as gen
import segmented_gather_gemm_expand_b200 as sg
from sgmv_testlib import compare, compare_every_element, from_torch, report, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset_variant():
    yield
    sg.set_variant(sg.VARIANT_AUTO)


def shrink_problem(seed, lengths, H, R, A, **kw):
    kw.setdefault("out_dt", "f32")
    return gen.custom(seed=seed, lengths=lengths, K=H, N=R, H=R, offset=0, num_adapters=A, add_inputs=False, **kw)


def run_shrink(p, variant=sg.VARIANT_AUTO, workspace=True, nthreads=1):
    c = p.calls[0]
    x, a, y = to_torch(p.x, p.x_dt), to_torch(c.w, p.w_dt), to_torch(p.y0, p.out_dt)
    meta = [torch.as_tensor(np.asarray(m)).cuda() for m in (p.seq_start, p.seq_len, p.lora_idx)]
    sg.set_variant(variant)
    _, _, pref = sg.shrink_plan(x, a, y, *meta, p.batches, p.max_seq_len, 1 << 30)
    ws = torch.empty(max(pref, 16), dtype=torch.uint8, device="cuda") if workspace else None
    v, splits, _ = sg.shrink_plan(x, a, y, *meta, p.batches, p.max_seq_len, 0 if ws is None else ws.numel())
    sg.sgmv_shrink(x, a, y, *meta, p.batches, p.max_seq_len, workspace=ws)
    torch.cuda.synchronize()
    assert sg.device_error() == 0
    gpu = from_torch(y, p.out_dt)
    ref = oracle.shrink(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.seq_start, p.seq_len, p.lora_idx,
                        nthreads=nthreads)
    rows = np.zeros(p.y0.shape[0], dtype=bool)
    lim = min(p.y0.shape[0], p.x.shape[0])
    for s, L, ai in zip(p.seq_start, p.seq_len, p.lora_idx):
        if 0 <= ai < c.w.shape[0] and s >= 0 and L > 0:
            rows[s:min(s + L, lim)] = True
    compare(gpu, ref, p.y0, p, rows, 0, c.w.shape[-2])
    return v, splits, gpu


MIXED = [300, 0, 5, 128, 77, 1]


@pytest.mark.parametrize("R", [16, 32, 64, 128])
@pytest.mark.parametrize("workspace", [True, False])
def test_shrink_tensor_cores_ranks(R, workspace):
    p = shrink_problem(R, MIXED, H=1000, R=R, A=4, idx=[3, 1, -1, 0, 2, 1])
    v, splits, _ = run_shrink(p, workspace=workspace)
    assert v == sg.VARIANT_TC
    assert (splits > 1) == workspace


@pytest.mark.parametrize("x_dt,out_dt", [("bf16", "bf16"), ("f16", "f16"), ("bf16", "f32"), ("f16", "bf16")])
def test_shrink_dtypes(x_dt, out_dt):
    p = shrink_problem(2, MIXED, H=512, R=16, A=3, x_dt=x_dt, w_dt=x_dt, out_dt=out_dt)
    v, _, _ = run_shrink(p)
    assert v == sg.VARIANT_TC


@pytest.mark.parametrize("case", [dict(R=8), dict(R=16, x_dt="f32", w_dt="bf16"), dict(R=24), dict(R=16, x_col_pad=3)])
def test_shrink_generic_kernel_cases(case):
    """Ranks that are not multiples of 16, x in another dtype than A, unaligned x rows: the generic kernel."""
    R = case.pop("R")
    p = shrink_problem(3, [40, 3, 17], H=200, R=R, A=2, **case)
    v, _, _ = run_shrink(p)
    assert v == sg.VARIANT_SIMT


def test_shrink_forced_generic_kernel_agrees():
    p = shrink_problem(4, MIXED, H=700, R=32, A=4)
    v, _, _ = run_shrink(p, variant=sg.VARIANT_SIMT)
    assert v == sg.VARIANT_SIMT


def test_shrink_split_and_unsplit_results_agree():
    p = shrink_problem(5, [513, 64, 9], H=2048, R=16, A=2, out_dt="f32")
    _, s1, a = run_shrink(p, workspace=False)
    _, s2, b = run_shrink(p, workspace=True)
    assert s1 == 1 and s2 > 1
    np.testing.assert_allclose(a, b, rtol=1e-5, atol=1e-4)


def test_shrink_invalid_ids_and_rows_past_the_output():
    p = shrink_problem(6, [30, 20, 10, 5], H=256, R=16, A=3, idx=[0, -1, 7, 2])
    run_shrink(p)


@pytest.mark.parametrize("H", [64, 65, 4096])
def test_shrink_hidden_sizes(H):
    p = shrink_problem(7, [130, 7], H=H, R=16, A=2)
    run_shrink(p)


def test_shrink_qkv_prefill_sized():
    """The shrink that feeds the fused-QKV prefill batch: 16 sequences U[64,1024], hidden 4096, rank 16."""
    rng = np.random.default_rng(0)
    lengths = rng.integers(64, 1025, 16)
    idx = rng.integers(0, 32, 16)
    idx[rng.permutation(16)[:2]] = -1
    p = shrink_problem(8, lengths.tolist(), H=4096, R=16, A=32, idx=idx.tolist(), out_dt="bf16")
    import oracle as o
    v, splits, _ = run_shrink(p, nthreads=o.max_threads())
    assert v == sg.VARIANT_TC and splits > 1


# ---------------------------------------------------------------- prefill-sized batches

def prefill_check(p, name):
    """Run sgmv_shrink on a prefill-sized batch with the workspace it prefers, and compare every element
    with the oracle's shrink; the same call twice gives the same bits (fixed-order partial sums)."""
    c = p.calls[0]
    x, a, y = to_torch(p.x, p.x_dt), to_torch(c.w, p.w_dt), to_torch(p.y0, p.out_dt)
    meta = [torch.as_tensor(np.asarray(m)).cuda() for m in (p.seq_start, p.seq_len, p.lora_idx)]
    v, splits, pref = sg.shrink_plan(x, a, y, *meta, p.batches, p.max_seq_len, 1 << 30)
    assert v == sg.VARIANT_TC, (v, splits, pref)
    ws = torch.empty(max(pref, 16), dtype=torch.uint8, device="cuda")
    sg.sgmv_shrink(x, a, y, *meta, p.batches, p.max_seq_len, workspace=ws)
    torch.cuda.synchronize()
    assert sg.device_error() == 0
    gpu = from_torch(y, p.out_dt)
    ref = oracle.shrink(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.seq_start, p.seq_len, p.lora_idx,
                        nthreads=oracle.max_threads())
    rows = np.zeros(p.y0.shape[0], dtype=bool)
    lim = min(p.y0.shape[0], p.x.shape[0])
    for s_, L, ai in zip(p.seq_start, p.seq_len, p.lora_idx):
        if 0 <= ai < c.w.shape[0] and s_ >= 0 and L > 0:
            rows[s_:min(s_ + L, lim)] = True
    err, count = compare_every_element(gpu, ref, p, [(rows, 0, c.w.shape[-2])])
    assert count == int(rows.sum()) * c.w.shape[-2]
    report(f"shrink_prefill/{name}", compared=count, max_abs_err=err, splits=splits)
    y2 = to_torch(p.y0, p.out_dt)
    sg.sgmv_shrink(x, a, y2, *meta, p.batches, p.max_seq_len, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(from_torch(y2, p.out_dt), gpu)


ROW_CASES = {
    # lengths, hidden, rank, adapters, extra keywords
    "rank16_bf16": dict(lengths=[700, 0, 1300, 64, 5, 900, 33], H=4096, R=16, A=4, idx=[0, 1, 2, -1, 3, 1, 2],
                        out_dt="bf16"),
    "rank32_f32_out": dict(lengths=[1000, 1500, 77], H=1000, R=32, A=3, out_dt="f32"),
    "rank64_f16": dict(lengths=[2000, 600], H=520, R=64, A=2, x_dt="f16", w_dt="f16", out_dt="f16"),
    "rank128": dict(lengths=[1200, 1300], H=256, R=128, A=2, out_dt="f32"),
    "short_segments_two_per_tile": dict(lengths=[40, 36, 45, 9] * 20, H=512, R=16, A=5, out_dt="bf16"),
    "tiles_of_128_rows": dict(lengths=[5000, 4000, 3000, 1], H=384, R=16, A=3, out_dt="bf16"),
    "gaps_invalid_ids_rows_past_out": dict(lengths=[900, 800, 700, 600], starts=[3, 1000, 1900, 2650], H=640,
                                           R=16, A=2, idx=[0, 5, 1, -1], extra_rows=7, out_dt="f32"),
}


@pytest.mark.parametrize("case", sorted(ROW_CASES))
def test_shrink_prefill_sized(case):
    kw = dict(ROW_CASES[case])
    p = shrink_problem(len(case), **kw)
    prefill_check(p, case)


def test_shrink_prefill_out_shorter_than_x():
    """Rows at or past the output's row count are skipped (the output has fewer rows than x)."""
    p = shrink_problem(9, [1500, 1500], H=512, R=16, A=2, out_dt="bf16")
    p.y0 = np.ascontiguousarray(p.y0[:2800])
    prefill_check(p, "out_shorter_than_x")


def test_shrink_workload_every_element():
    """The qkv_shrink workload (the bench's shrink line) at full size, every element."""
    prefill_check(gen.WORKLOADS["qkv_shrink"](), "qkv_shrink")
