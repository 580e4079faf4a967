"""GPU parity: the CUDA library against the CPU oracle on the same seeded inputs.

Every test runs each kernel variant that can take the case.  Inside the written
slice the results must be within the stated tolerance (see sgmv_testlib);
everything else in the output must keep its bits.
"""
import numpy as np
import pytest
import torch

import oracle
import sgmv_inputs as gen
import segmented_gather_gemm_expand_b200 as sg
from sgmv_testlib import (DeviceProblem, compare, compare_every_element, from_torch, report, run_multi,
                          to_torch, written_rows)

pytestmark = pytest.mark.gpu

VARIANTS = {"simt": sg.VARIANT_SIMT, "tc": sg.VARIANT_TC, "tc_wide": sg.VARIANT_TC_WIDE}


@pytest.fixture(autouse=True)
def _reset_variant():
    yield
    sg.set_variant(sg.VARIANT_AUTO)


def use_variant(name, dp: DeviceProblem, call=0):
    """Force a variant; returns False (and restores auto) if it cannot take the case."""
    sg.set_variant(VARIANTS[name])
    try:
        dp.plan(call)
    except sg.SgmvError as e:
        sg.set_variant(sg.VARIANT_AUTO)
        if e.code == -13:
            return False
        raise
    return True


def regions(p, calls=None):
    calls = range(len(p.calls)) if calls is None else calls
    return [(written_rows(p, c), p.calls[c].slice_offset, p.calls[c].slice_size) for c in calls]


def check_full(p: gen.Problem, variant: str, calls=None):
    """Run every call on the GPU and the oracle; compare the whole output."""
    dp = DeviceProblem(p)
    calls = list(range(len(p.calls))) if calls is None else calls
    if not use_variant(variant, dp):
        pytest.skip(f"{variant} does not take this case")
    ref = p.y0
    for c in calls:
        dp.run(c)
        ref = oracle.run_problem(p, out=ref, call=c)
    torch.cuda.synchronize()
    gpu = dp.result()
    assert sg.device_error() == 0
    check_regions(gpu, ref, p, regions(p, calls))
    return gpu, ref


def check_regions(gpu, ref, p, regs, check_rows=None):
    outside = np.ones(gpu.shape, dtype=bool)
    for rows, c0, n in regs:
        outside[np.ix_(rows, np.arange(c0, c0 + n))] = False
    bad = np.nonzero((gpu != p.y0) & outside)
    assert bad[0].size == 0, f"{bad[0].size} untouched elements changed (first {bad[0][0]},{bad[1][0]})"
    for rows, c0, n in regs:
        compare(gpu, ref, np.where(outside, p.y0, gpu), p, rows, c0, n, check_rows=check_rows)


# ------------------------------------------------------------------ small cases

@pytest.mark.parametrize("variant", VARIANTS)
def test_tiny_workload(variant):
    check_full(gen.tiny(), variant)


EDGE = {
    "one_token_segments": dict(lengths=[1, 1, 1, 1, 1], K=16, N=64, H=64, offset=0, num_adapters=3),
    "zero_length_mixed": dict(lengths=[0, 5, 0, 3, 0], K=16, N=64, H=128, offset=64, num_adapters=2),
    "all_minus_one": dict(lengths=[4, 5], K=16, N=64, H=64, offset=0, num_adapters=2, idx=[-1, -1]),
    "multi_tile_ragged": dict(lengths=[300, 129, 7, 128, 257], K=16, N=320, H=640, offset=256,
                              num_adapters=4),
    "n_not_multiple_of_8": dict(lengths=[9, 17], K=16, N=61, H=100, offset=3, num_adapters=2),
    "odd_offset_f32_out": dict(lengths=[33, 5], K=32, N=72, H=200, offset=7, num_adapters=2,
                               out_dt="f32"),
    "gaps_and_extra_rows": dict(lengths=[3, 40, 9], starts=[2, 10, 60], K=16, N=128, H=256,
                                offset=128, num_adapters=3, extra_rows=11),
    "strided_x_and_w": dict(lengths=[50, 14], K=16, N=96, H=192, offset=32, num_adapters=2,
                            x_col_pad=5, w_row_pad=3),
    "layout_4d": dict(lengths=[70, 3, 19], K=32, N=128, H=256, offset=128, num_adapters=3,
                      layout4d=True),
    "int32_metadata": dict(lengths=[64, 65, 1], K=16, N=128, H=128, offset=0, num_adapters=2,
                           meta_dt="int32"),
    "overwrite_mode": dict(lengths=[40, 90], K=16, N=256, H=512, offset=256, num_adapters=2,
                           add_inputs=False),
    "wide_slice": dict(lengths=[20, 150], K=16, N=1000, H=1100, offset=40, num_adapters=2),
}


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("case", sorted(EDGE))
def test_edge_cases(case, variant):
    check_full(gen.custom(seed=sum(map(ord, case)) % 1000, **EDGE[case]), variant)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("K", [1, 7, 8, 16, 17, 32, 48, 64, 128])
def test_ranks(K, variant):
    p = gen.custom(seed=K, lengths=[37, 130, 2], K=K, N=136, H=272, offset=136, num_adapters=3)
    check_full(p, variant)


# The tensor-core kernel hands pieces out round-robin when full 128-row blocks
# and partial ones are mixed (at most half of the pieces partial), and in
# contiguous ranges otherwise; these cases put each mode through ranks, dtypes
# and a segment table longer than one pass of its block-wide scan.
MIXED_BLOCKS = [256, 3, 384, 130, 1, 128]          # 7 full blocks, 3 partial: round-robin


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("K,out_dt", [(8, "bf16"), (16, "f16"), (24, "bf16"), (64, "f32"), (128, "bf16")])
def test_mixed_block_lengths(K, out_dt, variant):
    p = gen.custom(seed=40 + K, lengths=MIXED_BLOCKS, K=K, N=200, H=456, offset=128, num_adapters=4,
                   x_dt="f16" if out_dt == "f16" else "bf16", w_dt="f16" if out_dt == "f16" else "bf16",
                   out_dt=out_dt)
    check_full(p, variant)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("share_short", [0.1, 0.9])
def test_many_segments(share_short, variant):
    """800 segments (more than one 352-wide scan pass): 10% short segments picks
    round-robin, 90% short picks contiguous ranges."""
    rng = np.random.default_rng(int(share_short * 100))
    short = rng.random(800) < share_short
    lengths = np.where(short, rng.integers(1, 20, 800), 128 * rng.integers(1, 3, 800))
    idx = rng.integers(-1, 6, 800)
    p = gen.custom(seed=11, lengths=lengths.tolist(), K=16, N=64, H=192, offset=64, num_adapters=6,
                   idx=idx.tolist())
    check_full(p, variant)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("x_dt", gen.ALL_DTYPES)
@pytest.mark.parametrize("w_dt", gen.HALF_DTYPES)
@pytest.mark.parametrize("out_dt", gen.ALL_DTYPES)
def test_dtype_combinations(x_dt, w_dt, out_dt, variant):
    p = gen.custom(seed=3, lengths=[45, 140, 6], K=16, N=128, H=384, offset=128, num_adapters=3,
                   x_dt=x_dt, w_dt=w_dt, out_dt=out_dt, idx=[2, 0, 1])
    check_full(p, variant)


@pytest.mark.parametrize("variant", VARIANTS)
def test_integer_inputs_bit_exact(variant):
    p = gen.custom(seed=8, lengths=[33, 129, 5], K=64, N=128, H=256, offset=0, num_adapters=3,
                   integer=True, idx=[1, 2, 0])
    gpu, ref = check_full(p, variant)
    assert np.array_equal(oracle.decode(gpu, "bf16"), oracle.decode(ref, "bf16"))


@pytest.mark.parametrize("variant", VARIANTS)
def test_out_of_range_metadata_is_skipped_and_guards_hold(variant):
    """idx >= lora_num, idx < -1, negative start, segment past the last row."""
    T, H, N, K = 64, 256, 128, 16
    p = gen.custom(seed=4, lengths=[10, 8, 6, 9, 30], starts=[0, 12, 22, 30, 50], K=K, N=N, H=H,
                   offset=128, num_adapters=2, idx=[0, 5, -7, 1, 1])
    p.seq_start = p.seq_start.copy()
    p.seq_start[2] = -4                        # negative start (its idx is also invalid)
    # y0 has 80 rows; segment 4 runs to row 80 -> give out only 64 rows: rows >= 64 skipped
    p.y0 = np.ascontiguousarray(p.y0[:T])
    dp = DeviceProblem(p)
    if not use_variant(variant, dp):
        pytest.skip("variant does not take this case")
    # embed out in a guarded buffer
    G = 4096
    buf = torch.empty(G + T * H + G, dtype=torch.bfloat16, device="cuda")
    canary = torch.full((G,), 7.0, dtype=torch.bfloat16, device="cuda")
    buf[:G] = canary
    buf[G + T * H:] = canary
    y = buf[G:G + T * H].view(T, H)
    y.copy_(dp.y)
    dp.run(out=y)
    torch.cuda.synchronize()
    assert torch.equal(buf[:G], canary) and torch.equal(buf[G + T * H:], canary)
    gpu = from_torch(y, "bf16")
    ref = oracle.run_problem(p)
    check_regions(gpu, ref, p, regions(p))


@pytest.mark.parametrize("variant", VARIANTS)
def test_max_seq_len_smaller_than_segments(variant):
    """Every token m < L_b is processed even if max_seq_len understates the longest segment."""
    p = gen.custom(seed=12, lengths=[200, 17], K=16, N=128, H=128, offset=0, num_adapters=2)
    dp = DeviceProblem(p)
    if not use_variant(variant, dp):
        pytest.skip("variant does not take this case")
    dp.run(max_seq_len=4)
    torch.cuda.synchronize()
    check_regions(dp.result(), oracle.run_problem(p), p, regions(p))


@pytest.mark.parametrize("variant", VARIANTS)
def test_overwrite_ignores_nan(variant):
    p = gen.custom(seed=13, lengths=[70, 9], K=16, N=128, H=256, offset=128, num_adapters=2,
                   add_inputs=False)
    p.y0 = gen.to_storage(np.full(p.y0.shape, np.nan, np.float32), "bf16")
    check_full(p, variant)


# ------------------------------------------------------------------ invariants, bit-exact

@pytest.mark.parametrize("variant", VARIANTS)
def test_invariants_bit_exact(variant):
    base = dict(lengths=[130, 7, 64, 250, 1], K=32, N=256, H=768, offset=256, num_adapters=4,
                idx=[3, -1, 0, 2, 1])
    p = gen.custom(seed=21, **base)
    dp = DeviceProblem(p)
    if not use_variant(variant, dp):
        pytest.skip("variant does not take this case")
    dp.run()
    ref = from_torch(dp.y, "bf16")
    # deterministic
    dp2 = DeviceProblem(p)
    dp2.run()
    assert np.array_equal(from_torch(dp2.y, "bf16"), ref)
    # 3-D vs 4-D
    q = gen.custom(seed=21, layout4d=True, **base)
    dq = DeviceProblem(q)
    dq.run()
    assert np.array_equal(from_torch(dq.y, "bf16"), ref)
    # segment order
    perm = np.array([3, 0, 4, 2, 1])
    p2 = gen.custom(seed=21, **base)
    p2.seq_start, p2.seq_len, p2.lora_idx = p.seq_start[perm], p.seq_len[perm], p.lora_idx[perm]
    d3 = DeviceProblem(p2)
    d3.run()
    assert np.array_equal(from_torch(d3.y, "bf16"), ref)
    # split into two calls over disjoint segments
    p3 = gen.custom(seed=21, **base)
    d4 = DeviceProblem(p3)
    for part in ([0, 2], [1, 3, 4]):
        sub = gen.custom(seed=21, **base)
        sub.seq_start, sub.seq_len, sub.lora_idx = p.seq_start[part], p.seq_len[part], p.lora_idx[part]
        ds = DeviceProblem(sub)
        ds.run(out=d4.y)
    assert np.array_equal(from_torch(d4.y, "bf16"), ref)


@pytest.mark.parametrize("variant", VARIANTS)
def test_add_equals_old_plus_overwrite_result(variant):
    base = dict(lengths=[90, 40], K=16, N=128, H=128, offset=0, num_adapters=2, out_dt="f32")
    p = gen.custom(seed=22, **base)
    dp = DeviceProblem(p)
    if not use_variant(variant, dp):
        pytest.skip("variant does not take this case")
    dp.run(add=True)
    d2 = DeviceProblem(p)
    d2.run(add=False)
    torch.cuda.synchronize()
    a = from_torch(dp.y, "f32").astype(np.float64)
    o = from_torch(d2.y, "f32").astype(np.float64)
    y0 = p.y0.astype(np.float64)
    rows = written_rows(p)
    np.testing.assert_allclose(a[rows, :128], y0[rows, :128] + o[rows, :128], rtol=0, atol=1e-5)
    assert np.array_equal(a[~rows], y0[~rows]) and np.array_equal(o[~rows], y0[~rows])


# ------------------------------------------------------------------ the five workloads, full size

def oracle_all_calls(p):
    ref = p.y0
    for c in range(len(p.calls)):
        ref = oracle.run_problem(p, out=ref, call=c, nthreads=oracle.max_threads())
    return ref


@pytest.mark.parametrize("name", ["tiny", "qkv_prefill", "mlp_mixed", "long_single", "decode_mix"])
def test_workload_full_size_every_element(name):
    """Every written element of every slice of the workload against the oracle (the multi-threaded C
    oracle computes the whole output once); every other element bit-exact.  Each variant that takes
    the case runs it, and for workloads of several slices so does the fused multi-slice launch, which
    must also equal the separate calls bit for bit."""
    p = gen.WORKLOADS[name]()
    ref = oracle_all_calls(p)
    regs = regions(p)
    expected = int(sum(int(rows.sum()) * n for rows, _, n in regs))
    single = {}
    for variant in VARIANTS:
        dp = DeviceProblem(p)
        if not use_variant(variant, dp):
            report(f"{name}/{variant}", skipped="variant does not take this case")
            continue
        for c in range(len(p.calls)):
            dp.run(c)
        torch.cuda.synchronize()
        assert sg.device_error() == 0
        gpu = dp.result()
        del dp
        torch.cuda.empty_cache()
        sg.set_variant(sg.VARIANT_AUTO)
        err, count = compare_every_element(gpu, ref, p, regs)
        assert count == expected, (count, expected)
        report(f"{name}/{variant}", compared=count, max_abs_err=err, out_dtype=p.out_dt, rank=p.rank)
        single[variant] = gpu
    if len(p.calls) > 1:
        dm = DeviceProblem(p)
        assert run_multi(dm, plan_only=True) == (sg.VARIANT_TC, 1)
        run_multi(dm)
        torch.cuda.synchronize()
        assert sg.device_error() == 0
        gm = dm.result()
        del dm
        torch.cuda.empty_cache()
        err, count = compare_every_element(gm, ref, p, regs)
        assert count == expected, (count, expected)
        report(f"{name}/fused_multi_slice", compared=count, max_abs_err=err, out_dtype=p.out_dt, rank=p.rank)
        # the library's automatic choice for the separate calls is the tensor-core kernel (checked below)
        assert np.array_equal(gm, single["tc"]), "fused launch differs from the separate tensor-core calls"


def test_auto_picks_tensor_cores_for_the_workloads():
    """On compute capability 10.x every workload's calls take the tensor-core kernel."""
    major, _ = torch.cuda.get_device_capability()
    assert major == 10, "the tensor-core kernel is built for sm_100a"
    sg.set_variant(sg.VARIANT_AUTO)
    for name in ["tiny", "qkv_prefill", "mlp_mixed", "long_single", "decode_mix"]:
        p = gen.WORKLOADS[name]()
        dp = DeviceProblem(p)
        for c in range(len(p.calls)):
            assert dp.plan(c) == sg.VARIANT_TC, (name, c)
        if len(p.calls) > 1:
            assert run_multi(dp, plan_only=True) == (sg.VARIANT_TC, 1), name


# Each CTA of the tensor-core kernel handles more pieces than its output ring has
# barrier slots (32), so ring space and barrier phases are reused many times over,
# in both ways of handing out pieces.  The oracle checks every element.
MANY_PIECES = {
    # almost all blocks partial: contiguous ranges
    "contiguous": dict(short_share=1.0),
    # 40 % partial blocks: round-robin
    "round_robin": dict(short_share=0.4),
}


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("case", sorted(MANY_PIECES))
def test_more_pieces_per_cta_than_ring_slots(case, variant):
    rng = np.random.default_rng(77 if case == "contiguous" else 78)
    B = 1000
    short = rng.random(B) < MANY_PIECES[case]["short_share"]
    lengths = np.where(short, rng.integers(1, 128, B), 128)
    idx = rng.integers(-1, 8, B)
    N = 1536                           # 12 n-tiles of 128 columns, 6 of 256
    p = gen.custom(seed=79, lengths=lengths.tolist(), K=16, N=N, H=N + 256, offset=128, num_adapters=8,
                   idx=idx.tolist())
    dp = DeviceProblem(p)
    if not use_variant(variant, dp):
        pytest.skip(f"{variant} does not take this case")
    dp.run()
    torch.cuda.synchronize()
    assert sg.device_error() == 0
    gpu = dp.result()
    ref = oracle.run_problem(p, nthreads=oracle.max_threads())
    err, count = compare_every_element(gpu, ref, p, regions(p))
    active = (p.lora_idx >= 0) & (p.lora_idx < 8)
    pieces = int((np.ceil(lengths[active] / 128) * (N // (256 if variant == "tc_wide" else 128))).sum())
    report(f"many_pieces_{case}/{variant}", compared=count, max_abs_err=err,
           pieces_per_cta=pieces / torch.cuda.get_device_properties(0).multi_processor_count)
    assert pieces > 32 * torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("variant", ["auto", "tc_wide"])
def test_thousands_of_segments_take_the_tensor_cores(variant):
    """4096 segments (short, full-block and longer ones mixed, ids -1 and out of range among them): the
    segment table stays in shared memory, the tensor-core kernel takes the call and every element
    matches the oracle."""
    rng = np.random.default_rng(4096)
    B = 4096
    kind = rng.random(B)
    lengths = np.where(kind < 0.6, rng.integers(1, 41, B), np.where(kind < 0.8, 128, rng.integers(129, 301, B)))
    idx = rng.integers(-1, 17, B)                 # 16 is out of range: skipped like -1
    p = gen.custom(seed=96, lengths=lengths.tolist(), K=16, N=256, H=512, offset=128, num_adapters=16,
                   idx=idx.tolist())
    dp = DeviceProblem(p)
    if variant == "auto":
        sg.set_variant(sg.VARIANT_AUTO)
        assert dp.plan() == sg.VARIANT_TC
    else:
        assert use_variant(variant, dp)
    dp.run()
    torch.cuda.synchronize()
    assert sg.device_error() == 0
    gpu = dp.result()
    ref = oracle.run_problem(p, nthreads=oracle.max_threads())
    err, count = compare_every_element(gpu, ref, p, regions(p))
    report(f"segments_4096/{variant}", compared=count, max_abs_err=err)


# ------------------------------------------------------------------ metadata validation

def test_validate_metadata_bits():
    dev = "cuda"

    def run(starts, lens, idx, A=4, rows=100):
        t = lambda a: torch.tensor(a, dtype=torch.int64, device=dev)
        return sg.validate_metadata(t(starts), t(lens), t(idx), len(starts), A, rows)

    assert run([0, 4, 10], [4, 6, 3], [0, 1, -1]) == 0
    assert run([0, 4], [4, 6], [0, 9]) & 1
    assert run([0, -4], [4, 6], [0, 1]) & 2
    assert run([0, 95], [4, 6], [0, 1]) & 4
    assert run([0, 2], [4, 6], [0, 1]) & 8
    st = run([10, 0], [4, 6], [0, 1])
    assert st & 16 and not st & 8
    assert run([4, 0], [6, 6], [0, 1]) & 8


@pytest.mark.parametrize("case", ["multi_tile_ragged", "wide_slice", "odd_offset_f32_out", "overwrite_mode"])
def test_tile_widths_give_identical_bits(case):
    """128- and 256-column n-tiles run the same MMA steps for every output element, so the results
    must agree bit for bit (this is what lets the library pick the width per call)."""
    p = gen.custom(seed=sum(map(ord, case)) % 1000, **EDGE[case])
    outs = []
    for v in (sg.VARIANT_TC, sg.VARIANT_TC_WIDE):
        dp = DeviceProblem(p)
        sg.set_variant(v)
        try:
            dp.plan(0)
        except sg.SgmvError as e:
            pytest.skip(f"variant {v} does not take this case ({e.code})")
        dp.run(0)
        torch.cuda.synchronize()
        outs.append(dp.result())
    assert sg.device_error() == 0
    assert np.array_equal(outs[0], outs[1])
