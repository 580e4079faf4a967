"""GPU parity of sgmv_expand_multi_slice: several disjoint slices of one fused
output (the QKV or gate/up projections the page's Usage section names) in one
call.

The fused launch computes every piece exactly as a single-slice launch of the
same kernel does (same operand order, same fp32 accumulation, one rounding),
so its output must equal the single-slice calls bit for bit; against the
oracle it must be within the stated tolerance inside every slice and
bit-exact everywhere else.
"""
import numpy as np
import pytest
import torch

import oracle
import sgmv_inputs as gen
import segmented_gather_gemm_expand_b200 as sg
from sgmv_testlib import DeviceProblem, compare, from_torch, run_multi, written_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset_variant():
    yield
    sg.set_variant(sg.VARIANT_AUTO)


def multi_problem(seed, *, lengths, K, Ns, offs, H, num_adapters, x_dt="bf16", w_dt="bf16",
                  out_dt="bf16", add_inputs=True, layout4d=False, idx=None):
    """A problem whose calls are the slices (Ns[i] columns at offs[i]) of one output."""
    p = gen.custom(seed=seed, lengths=lengths, K=K, N=Ns[0], H=H, offset=offs[0],
                   num_adapters=num_adapters, x_dt=x_dt, w_dt=w_dt, out_dt=out_dt,
                   add_inputs=add_inputs, layout4d=layout4d, idx=idx)
    rng = np.random.default_rng(seed + 1000)
    calls = []
    for n, o in zip(Ns, offs):
        w = gen.normal(rng, (num_adapters, n, K), 0.02, w_dt)
        if layout4d:
            w = w[:, None]
        calls.append(gen.SliceCall(w, o, n))
    p.calls = calls
    return p


def oracle_all(p):
    ref = p.y0
    for c in range(len(p.calls)):
        ref = oracle.run_problem(p, out=ref, call=c)
    return ref


def check_against_oracle(gpu, ref, p):
    outside = np.ones(gpu.shape, dtype=bool)
    for c, call in enumerate(p.calls):
        outside[np.ix_(written_rows(p, c), np.arange(call.slice_offset, call.slice_offset + call.slice_size))] = False
    bad = np.nonzero((gpu != p.y0) & outside)
    assert bad[0].size == 0, f"{bad[0].size} untouched elements changed"
    for c, call in enumerate(p.calls):
        compare(gpu, ref, np.where(outside, p.y0, gpu), p, written_rows(p, c), call.slice_offset,
                call.slice_size)


def fused_vs_single(p, expect_launches=None):
    """Run the multi-slice call and the single-slice calls; both checked."""
    dm = DeviceProblem(p)
    variant, launches = run_multi(dm, plan_only=True)
    if expect_launches is not None:
        assert launches == expect_launches, (variant, launches)
    run_multi(dm)
    ds = DeviceProblem(p)
    for c in range(len(p.calls)):
        ds.run(c)
    torch.cuda.synchronize()
    assert sg.device_error() == 0
    gm, gs = dm.result(), ds.result()
    check_against_oracle(gm, oracle_all(p), p)
    return gm, gs, variant, launches


CASES = {
    "three_equal": dict(lengths=[300, 129, 7, 128, 257], K=16, Ns=[256, 256, 256], offs=[0, 256, 512],
                        H=768, num_adapters=4),
    "unequal_sizes_gaps": dict(lengths=[40, 200, 1, 131], K=32, Ns=[136, 64, 200], offs=[8, 200, 400],
                               H=640, num_adapters=3),
    "reversed_order": dict(lengths=[90, 17, 260], K=16, Ns=[128, 128, 128], offs=[256, 128, 0], H=512,
                           num_adapters=2, idx=[1, -1, 0]),
    "four_slices_f32_out_overwrite": dict(lengths=[33, 140, 5], K=64, Ns=[64, 72, 128, 16],
                                          offs=[0, 64, 136, 264], H=296, num_adapters=3, out_dt="f32",
                                          add_inputs=False),
    "mixed_precision_4d": dict(lengths=[70, 3, 190], K=64, Ns=[192, 192], offs=[0, 192], H=384,
                               num_adapters=3, x_dt="f32", layout4d=True),
    "rank8_f16": dict(lengths=[500, 12], K=8, Ns=[128, 256], offs=[256, 0], H=384, num_adapters=2,
                      x_dt="f16", w_dt="f16", out_dt="f16", add_inputs=False),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_fused_multi_slice_matches_oracle_and_single_calls(case):
    p = multi_problem(sum(map(ord, case)) % 997, **CASES[case])
    gm, gs, variant, launches = fused_vs_single(p, expect_launches=1)
    assert variant == sg.VARIANT_TC
    assert np.array_equal(gm, gs), "fused launch differs from the single-slice launches"


def test_unfusable_slices_run_as_separate_launches():
    # slice 2 has an odd width: the tensor-core kernel cannot take it, so the
    # call splits into one launch per slice
    p = multi_problem(5, lengths=[60, 9, 130], K=16, Ns=[128, 61, 128], offs=[0, 128, 192], H=320,
                      num_adapters=2)
    gm, gs, variant, launches = fused_vs_single(p, expect_launches=3)
    assert variant == 0
    assert np.array_equal(gm, gs)


def test_forced_generic_kernel_runs_each_slice():
    p = multi_problem(6, lengths=[60, 9, 130], K=16, Ns=[128, 128], offs=[0, 128], H=256, num_adapters=2)
    sg.set_variant(sg.VARIANT_SIMT)
    gm, gs, variant, launches = fused_vs_single(p, expect_launches=2)
    assert variant == sg.VARIANT_SIMT
    assert np.array_equal(gm, gs)


def test_single_slice_through_multi_entry_point():
    p = multi_problem(7, lengths=[100, 28], K=16, Ns=[256], offs=[128], H=512, num_adapters=2)
    gm, gs, variant, launches = fused_vs_single(p, expect_launches=1)
    assert np.array_equal(gm, gs)


def test_empty_slice_is_skipped():
    p = multi_problem(8, lengths=[50, 20], K=16, Ns=[128, 0, 128], offs=[0, 128, 128], H=256,
                      num_adapters=2)
    gm, gs, variant, launches = fused_vs_single(p, expect_launches=1)
    assert np.array_equal(gm, gs)


# The full-size workloads of several slices (QKV prefill, gate/up MLP) run through the fused
# launch in test_parity_gpu.test_workload_full_size_every_element, against the oracle at every
# element and against the separate calls bit for bit.
