"""Pins for the CPU oracle: each check compares it with something other than itself.

- the fp16 / bfloat16 codecs against numpy's IEEE binary16 and torch's
  bfloat16 on all 65536 bit patterns, and the encoder against a brute-force
  nearest-value search with exact rational arithmetic;
- the page's worked example (lengths [4, 6] give starts [0, 4]);
- a dense per-adapter formulation with numpy's fp64 matmul;
- exact rational arithmetic (Fraction) element by element on tiny inputs;
- small-integer inputs whose results are exact;
- invariants: untouched rows/columns, add = old + product, scaling, segment
  order, adapter relabelling, 3-D vs 4-D layout, split calls, K = 1.
"""
import bisect
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import sgmv_inputs as gen

HERE = os.path.dirname(os.path.abspath(__file__))


# --------------------------------------------------------------- independent codecs

def indep_decode(storage, dt):
    a = np.asarray(storage)
    if dt == "f32":
        return a.astype(np.float64)
    if dt == "f16":
        return np.ascontiguousarray(a, dtype=np.uint16).view(np.float16).astype(np.float64)
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).to(torch.float64).numpy()


def indep_cast(values_f64, dt):
    """Round values (each exactly representable in float32) to dtype dt, as float64."""
    v = np.asarray(values_f64, dtype=np.float64)
    if dt == "f32":
        return v.astype(np.float32).astype(np.float64)
    if dt == "f16":
        return v.astype(np.float16).astype(np.float64)
    f32 = v.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), v, equal_nan=True)
    return torch.from_numpy(f32).to(torch.bfloat16).to(torch.float64).numpy()


def positive_table(dt):
    """Ascending finite non-negative values of a 16-bit format with their bit patterns."""
    last = 0x7BFF if dt == "f16" else 0x7F7F
    bits = np.arange(0, last + 1, dtype=np.uint32).astype(np.uint16)
    vals = indep_decode(bits, dt)
    assert np.all(np.diff(vals) > 0)
    return [Fraction(float(v)) for v in vals], bits


_TABLES = {}


def brute_round(v: float, dt: str) -> int:
    """Nearest representable value (ties to the even pattern), by exhaustive search."""
    if dt not in _TABLES:
        _TABLES[dt] = positive_table(dt)
    vals, bits = _TABLES[dt]
    sign = 0x8000 if np.signbit(v) else 0
    x = Fraction(abs(float(v)))
    emax_next = vals[-1] + (vals[-1] - vals[-2])        # 2^(emax+1): the first value past max
    inf_bits = 0x7C00 if dt == "f16" else 0x7F80
    cand = []
    i = bisect.bisect_left(vals, x)
    for j in (i - 1, i):
        if 0 <= j < len(vals):
            cand.append((abs(vals[j] - x), int(bits[j])))
    if x > vals[-1]:
        cand.append((abs(emax_next - x), inf_bits))
    cand.sort(key=lambda c: (c[0], c[1] & 1))
    return sign | cand[0][1]


# --------------------------------------------------------------- codec pins

@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_decode_all_bit_patterns(dt):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = indep_decode(bits, dt)
    got = oracle.decode(bits, dt)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    m = ~np.isnan(ref)
    assert np.array_equal(ref[m], got[m])
    assert np.array_equal(np.signbit(ref[m]), np.signbit(got[m]))


def _encode_probe_values(dt, rng):
    vals, _ = positive_table(dt)
    fv = np.array([float(v) for v in vals])
    picks = rng.integers(1, len(fv) - 1, size=400)
    mids = (fv[picks] + fv[picks + 1]) / 2.0                 # exact ties
    near = np.concatenate([np.nextafter(mids, 0), np.nextafter(mids, np.inf)])
    top = fv[-1]
    step = fv[-1] - fv[-2]
    edges = np.array([top, top + step / 2, np.nextafter(top + step / 2, 0),
                      np.nextafter(top + step / 2, np.inf), top * 4, fv[1] / 2, fv[1] / 4,
                      np.nextafter(fv[1] / 2, np.inf), fv[1] * 1.5, fv[1] * 2.5, 0.0])
    logs = np.exp(rng.uniform(np.log(fv[1] / 8), np.log(top * 2), size=2000))
    v = np.concatenate([mids, near, edges, logs, rng.standard_normal(500)])
    return np.concatenate([v, -v])


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_encode_is_correct_rounding(dt):
    rng = np.random.default_rng(1)
    v = _encode_probe_values(dt, rng)
    got = oracle.encode(v, dt)
    want = np.array([brute_round(x, dt) for x in v], dtype=np.uint16)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(v[i], hex(got[i]), hex(want[i])) for i in bad[:5]]


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_encode_matches_library_on_float32_inputs(dt):
    rng = np.random.default_rng(2)
    f = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        (rng.standard_normal(2000) * 1e-6).astype(np.float32),
                        (rng.standard_normal(2000) * 7e4).astype(np.float32)])
    got = oracle.encode(f.astype(np.float64), dt)
    want = gen.to_storage(f, dt)
    assert np.array_equal(got, want)


def test_encode_special_values():
    assert oracle.encode(np.array([np.inf]), "f16")[0] == 0x7C00
    assert oracle.encode(np.array([-np.inf]), "bf16")[0] == 0xFF80
    assert oracle.encode(np.array([-0.0]), "f16")[0] == 0x8000
    assert np.isnan(oracle.decode(oracle.encode(np.array([np.nan]), "bf16"), "bf16")[0])
    assert oracle.encode(np.array([65520.0]), "f16")[0] == 0x7C00     # max + half ulp: tie to inf
    assert oracle.encode(np.array([65519.99]), "f16")[0] == 0x7BFF


# --------------------------------------------------------------- helpers for the operation

def dense_reference(p: gen.Problem, call: int = 0):
    """Per-row adapter ids, then one fp64 matmul per adapter (numpy)."""
    c = p.calls[call]
    w = c.w[:, 0] if c.w.ndim == 4 else c.w
    A, N, K = w.shape
    T_out = p.y0.shape[0]
    aid = np.full(T_out, -1, dtype=np.int64)
    for s, L, a in zip(p.seq_start, p.seq_len, p.lora_idx):
        if 0 <= a < A and s >= 0 and L > 0:
            hi = min(s + L, T_out, p.x.shape[0])
            aid[s:hi] = a
    xh = indep_cast(indep_decode(p.x, p.x_dt), p.w_dt)
    wd = indep_decode(w, p.w_dt)
    y = indep_decode(p.y0, p.out_dt)[:, c.slice_offset:c.slice_offset + N]
    pre = np.full((T_out, N), np.nan)
    for a in np.unique(aid[aid >= 0]):
        rows = np.nonzero(aid == a)[0]
        acc = xh[rows] @ wd[a].T
        pre[rows] = (y[rows] + acc) if p.add_inputs else acc
    return aid, pre


def ulp_of(values, dt):
    """Spacing of the format at each value's magnitude (bf16/f16), floored at the subnormal step."""
    f = 10 if dt == "f16" else 7
    emin = -14 if dt == "f16" else -126
    mag = np.abs(values)
    e = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    e = np.maximum(e, emin)
    return np.ldexp(1.0, (e - f).astype(int))


def check_against_dense(p, call=0):
    c = p.calls[call]
    out, pre = oracle.run_problem(p, return_pre=True, call=call)
    aid, want = dense_reference(p, call)
    written = aid >= 0
    assert np.array_equal(np.isnan(pre[written]).any(axis=1), np.zeros(written.sum(), bool))
    assert np.all(np.isnan(pre[~written]))
    np.testing.assert_allclose(pre[written], want[written], rtol=1e-12, atol=1e-12)
    # final values: the nearest representable value to the fp64 result
    got = indep_decode(out, p.out_dt)[:, c.slice_offset:c.slice_offset + c.slice_size]
    if p.out_dt == "f32":
        assert np.array_equal(got[written], want[written].astype(np.float32).astype(np.float64))
    else:
        err = np.abs(got[written] - want[written])
        assert np.all(err <= 0.5 * ulp_of(got[written], p.out_dt) * (1 + 1e-9))
    # untouched bits
    mask = np.ones(p.y0.shape, dtype=bool)
    mask[np.ix_(written, np.arange(c.slice_offset, c.slice_offset + c.slice_size))] = False
    assert np.array_equal(out[mask], p.y0[mask])
    return out, pre


# --------------------------------------------------------------- the page's worked example

def test_worked_example_starts():
    g = json.load(open(os.path.join(HERE, "golden", "worked_example.json")))
    assert gen.exclusive_cumsum(g["lengths"]).tolist() == g["starts"]
    assert gen.tiny().seq_start.tolist() == gen.exclusive_cumsum([4, 6, 3, 7]).tolist() == [0, 4, 10, 13]


def test_worked_example_rows_follow_their_segment():
    """Lengths [4, 6] with starts [0, 4]: rows 0-3 take adapter idx[0], rows 4-9 idx[1]."""
    g = json.load(open(os.path.join(HERE, "golden", "worked_example.json")))
    A, N, K, H = 3, 8, 1, 8
    x = gen.to_storage(np.ones((10, K), np.float32), "f16")
    w = gen.to_storage(np.repeat(np.arange(1, A + 1, dtype=np.float32), N).reshape(A, N, K), "f16")
    y0 = gen.to_storage(np.full((10, H), 100.0, np.float32), "f16")
    idx = [2, 0]
    out = oracle.expand_slice(x, "f16", w, "f16", y0, "f16", g["starts"], g["lengths"], idx, 0, N, False)
    vals = oracle.decode(out, "f16")
    assert np.all(vals[0:4] == idx[0] + 1) and np.all(vals[4:10] == idx[1] + 1)


# --------------------------------------------------------------- dense formulation

DENSE_CASES = [
    dict(lengths=[5, 1, 9, 3], K=16, N=24, H=64, offset=8, num_adapters=3, x_dt="bf16", w_dt="bf16", out_dt="bf16"),
    dict(lengths=[7, 2, 4], K=8, N=16, H=40, offset=16, num_adapters=2, x_dt="f16", w_dt="f16", out_dt="f16", add_inputs=False),
    dict(lengths=[3, 6, 2, 5], K=32, N=12, H=12, offset=0, num_adapters=4, x_dt="f32", w_dt="bf16", out_dt="bf16", layout4d=True),
    dict(lengths=[4, 4], K=16, N=8, H=32, offset=24, num_adapters=2, x_dt="f32", w_dt="f16", out_dt="f32"),
    dict(lengths=[6, 3, 1], K=7, N=10, H=30, offset=5, num_adapters=3, x_dt="bf16", w_dt="f16", out_dt="f16", x_col_pad=3, w_row_pad=2),
    dict(lengths=[2, 9], K=64, N=16, H=48, offset=32, num_adapters=2, x_dt="f16", w_dt="bf16", out_dt="f32", add_inputs=False),
]


@pytest.mark.parametrize("case", range(len(DENSE_CASES)))
def test_oracle_matches_dense_matmul(case):
    kw = dict(DENSE_CASES[case])
    kw.setdefault("idx", None)
    p = gen.custom(seed=10 + case, **kw)
    if kw["idx"] is None:
        p.lora_idx[0] = -1
    check_against_dense(p)


def test_oracle_with_gaps_and_tail_rows():
    p = gen.custom(seed=3, lengths=[3, 4, 2], starts=[1, 7, 13], K=16, N=16, H=32, offset=16,
                   num_adapters=2, extra_rows=5)
    check_against_dense(p)


@pytest.mark.parametrize("name", ["tiny"])
def test_tiny_workload_against_dense(name):
    check_against_dense(gen.WORKLOADS[name]())


# --------------------------------------------------------------- exact rational brute force

def brute_force_exact(p: gen.Problem):
    """Every element from exact rational arithmetic and exhaustive rounding."""
    c = p.calls[0]
    w = c.w[:, 0] if c.w.ndim == 4 else c.w
    A, N, K = w.shape
    xv = indep_decode(p.x, p.x_dt)
    wv = indep_decode(w, p.w_dt)
    yv = indep_decode(p.y0, p.out_dt)
    out = p.y0.copy()
    for s, L, a in zip(p.seq_start, p.seq_len, p.lora_idx):
        if not (0 <= a < A):
            continue
        for r in range(s, s + L):
            for n in range(N):
                tot = Fraction(0)
                for k in range(K):
                    xr = Fraction(float(indep_cast(np.array([xv[r, k]]), p.w_dt)[0]))
                    tot += xr * Fraction(float(wv[a, n, k]))
                if p.add_inputs:
                    tot += Fraction(float(yv[r, c.slice_offset + n]))
                if p.out_dt == "f32":
                    out[r, c.slice_offset + n] = np.float32(float(tot))
                else:
                    out[r, c.slice_offset + n] = brute_round(float(tot), p.out_dt)
    return out


@pytest.mark.parametrize("x_dt,w_dt,out_dt,add", [("bf16", "bf16", "bf16", True), ("f16", "f16", "f16", False),
                                                 ("f32", "bf16", "f16", True), ("bf16", "f16", "bf16", True)])
def test_oracle_matches_exact_brute_force(x_dt, w_dt, out_dt, add):
    p = gen.custom(seed=5, lengths=[3, 2, 4], K=6, N=5, H=9, offset=2, num_adapters=3, idx=[1, -1, 2],
                   x_dt=x_dt, w_dt=w_dt, out_dt=out_dt, add_inputs=add, w_scale=0.3)
    assert np.array_equal(oracle.run_problem(p), brute_force_exact(p))


def test_rank_one_is_an_outer_product():
    p = gen.custom(seed=6, lengths=[4, 3], K=1, N=7, H=7, offset=0, num_adapters=2, idx=[1, 0])
    out = oracle.run_problem(p)
    assert np.array_equal(out, brute_force_exact(p))


# --------------------------------------------------------------- exact integers

@pytest.mark.parametrize("out_dt", ["bf16", "f16", "f32"])
def test_integer_inputs_are_exact(out_dt):
    p = gen.custom(seed=7, lengths=[5, 8, 3], K=64, N=16, H=40, offset=8, num_adapters=3, idx=[2, 0, 1],
                   x_dt="bf16", w_dt="bf16", out_dt=out_dt, integer=True)
    out = oracle.run_problem(p)
    xi = indep_decode(p.x, "bf16").astype(np.int64)
    wi = indep_decode(p.calls[0].w, "bf16").astype(np.int64)
    yi = indep_decode(p.y0, out_dt).astype(np.int64)
    want = yi.copy()
    for s, L, a in zip(p.seq_start, p.seq_len, p.lora_idx):
        want[s:s + L, 8:24] += xi[s:s + L] @ wi[a].T
    assert np.abs(want).max() <= 256           # exactly representable in every output dtype
    assert np.array_equal(indep_decode(out, out_dt), want.astype(np.float64))


# --------------------------------------------------------------- invariants

def _base_problem(seed=11, **over):
    kw = dict(lengths=[6, 3, 7, 2, 5], K=16, N=24, H=72, offset=24, num_adapters=4,
              idx=[3, -1, 0, 2, 1], x_dt="bf16", w_dt="bf16", out_dt="bf16")
    kw.update(over)
    return gen.custom(seed=seed, **kw)


def test_minus_one_rows_and_outside_columns_unchanged():
    p = _base_problem()
    p.y0[:] = gen.to_storage(np.full(p.y0.shape, np.nan, np.float32), "bf16")  # NaN must survive too
    out = oracle.run_problem(p)
    s, L = p.seq_start[1], p.seq_len[1]
    assert np.array_equal(out[s:s + L], p.y0[s:s + L])
    assert np.array_equal(out[:, :24], p.y0[:, :24]) and np.array_equal(out[:, 48:], p.y0[:, 48:])


def test_out_of_range_adapter_is_skipped():
    p = _base_problem(idx=[3, 7, 0, -5, 1])
    out = oracle.run_problem(p)
    for b in (1, 3):
        s, L = p.seq_start[b], p.seq_len[b]
        assert np.array_equal(out[s:s + L], p.y0[s:s + L])


def test_add_equals_old_plus_product():
    p = _base_problem(add_inputs=True)
    _, pre_add = oracle.run_problem(p, return_pre=True)
    p.add_inputs = False
    _, pre_over = oracle.run_problem(p, return_pre=True)
    y = indep_decode(p.y0, "bf16")[:, 24:48]
    m = ~np.isnan(pre_add)
    assert np.array_equal(pre_add[m], (y + pre_over)[m])


def test_overwrite_ignores_old_values():
    p = _base_problem(add_inputs=False)
    a = oracle.run_problem(p)
    p.y0 = gen.to_storage(np.full(p.y0.shape, np.nan, np.float32), "bf16")
    b = oracle.run_problem(p)
    written = np.zeros(p.y0.shape[0], bool)
    for s, L, i in zip(p.seq_start, p.seq_len, p.lora_idx):
        if i >= 0:
            written[s:s + L] = True
    assert np.array_equal(a[written, 24:48], b[written, 24:48])


def test_scaling_x_or_w_by_two_scales_the_product():
    p = _base_problem(add_inputs=False)
    _, pre = oracle.run_problem(p, return_pre=True)
    p2 = _base_problem(add_inputs=False)
    p2.x = gen.to_storage(indep_decode(p.x, "bf16").astype(np.float32) * 2, "bf16")
    _, pre_x2 = oracle.run_problem(p2, return_pre=True)
    p3 = _base_problem(add_inputs=False)
    p3.calls[0].w = gen.to_storage(indep_decode(p.calls[0].w, "bf16").astype(np.float32) * 2, "bf16")
    _, pre_w2 = oracle.run_problem(p3, return_pre=True)
    m = ~np.isnan(pre)
    assert np.array_equal(pre_x2[m], 2 * pre[m]) and np.array_equal(pre_w2[m], 2 * pre[m])


def test_linearity_in_x():
    p = _base_problem(add_inputs=False, x_dt="f32", w_dt="bf16")
    _, pa = oracle.run_problem(p, return_pre=True)
    x1 = p.x.copy()
    p.x = gen.normal(np.random.default_rng(99), x1.shape, 1.0, "f32")
    _, pb = oracle.run_problem(p, return_pre=True)
    x2 = p.x.copy()
    # choose x1, x2 whose casts to bf16 add exactly: use the casts themselves
    c1 = indep_cast(x1.astype(np.float64), "bf16")
    c2 = indep_cast(x2.astype(np.float64), "bf16")
    p.x = (c1 + c2).astype(np.float32)
    _, pab = oracle.run_problem(p, return_pre=True)
    exact = np.array_equal(indep_cast(p.x.astype(np.float64), "bf16"), c1 + c2)
    m = ~np.isnan(pa)
    if exact:
        np.testing.assert_allclose(pab[m], pa[m] + pb[m], rtol=1e-12, atol=1e-12)
    else:  # the sum itself had to round; linearity holds to bf16 precision of x
        np.testing.assert_allclose(pab[m], pa[m] + pb[m], rtol=0, atol=0.05)


def test_segment_order_and_adapter_relabelling_do_not_matter():
    p = _base_problem()
    ref = oracle.run_problem(p)
    perm = np.array([4, 2, 0, 3, 1])
    q = _base_problem()
    q.seq_start, q.seq_len, q.lora_idx = p.seq_start[perm], p.seq_len[perm], p.lora_idx[perm]
    assert np.array_equal(oracle.run_problem(q), ref)
    relabel = np.array([2, 0, 3, 1])               # new position of old adapter a
    r = _base_problem()
    w_new = np.empty_like(p.calls[0].w)
    w_new[relabel] = p.calls[0].w
    r.calls[0].w = w_new
    r.lora_idx = np.where(p.lora_idx >= 0, relabel[np.maximum(p.lora_idx, 0)], -1)
    assert np.array_equal(oracle.run_problem(r), ref)


def test_three_d_and_four_d_layouts_agree():
    p = _base_problem()
    q = _base_problem()
    q.calls[0].w = p.calls[0].w[:, None]
    assert np.array_equal(oracle.run_problem(p), oracle.run_problem(q))


def test_split_into_two_calls_matches_one_call():
    p = _base_problem()
    ref = oracle.run_problem(p)
    first, second = [0, 2, 4], [1, 3]
    q = _base_problem()
    q.seq_start, q.seq_len, q.lora_idx = p.seq_start[first], p.seq_len[first], p.lora_idx[first]
    mid = oracle.run_problem(q)
    q.seq_start, q.seq_len, q.lora_idx = p.seq_start[second], p.seq_len[second], p.lora_idx[second]
    assert np.array_equal(oracle.run_problem(q, out=mid), ref)


def test_mixed_precision_casts_x_to_the_weight_dtype():
    """fp32 x must be rounded to bf16 first: compare with and without the cast."""
    p = _base_problem(x_dt="f32", add_inputs=False)
    _, pre = oracle.run_problem(p, return_pre=True)
    aid, want = dense_reference(p)
    m = aid >= 0
    np.testing.assert_allclose(pre[m], want[m], rtol=1e-12, atol=1e-12)
    w = indep_decode(p.calls[0].w, "bf16")
    uncast = np.full_like(want, np.nan)
    for a in np.unique(aid[m]):
        rows = aid == a
        uncast[rows] = p.x[rows].astype(np.float64) @ w[a].T
    assert np.abs(uncast[m] - pre[m]).max() > 1e-4


def test_nthreads_do_not_change_results():
    p = _base_problem()
    assert np.array_equal(oracle.run_problem(p, nthreads=1), oracle.run_problem(p, nthreads=4))
