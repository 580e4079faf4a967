"""Pins for the oracle's plain SGMV expand and BGMV expand-slice (CPU only).

Both are defined on "Implementation: Predibase Lorax SGMV Expand Slice Kernel"
(Description) relative to the expand-slice operation: plain expand writes the
whole output row, and BGMV is the fixed-length counterpart with one token per
row.  The oracle reaches them through its expand-slice routine, so here they
are pinned against other formulations: one numpy fp64 matmul per adapter over
the rows that use it, exact small-integer inputs, and the rows and columns
that must keep their bits.
"""
import numpy as np
import pytest

import oracle
import sgmv_inputs as gen
from test_oracle_pins import indep_cast, indep_decode, ulp_of


def dense_rows(x, x_dt, w, w_dt, y0, out_dt, row_adapter, col0, add):
    """pre-rounding values per row from one fp64 matmul per adapter (numpy)."""
    w3 = w[:, 0] if w.ndim == 4 else w
    A, N, K = w3.shape
    xh = indep_cast(indep_decode(x, x_dt), w_dt)
    wd = indep_decode(w3, w_dt)
    y = indep_decode(y0, out_dt)[:, col0:col0 + N]
    pre = np.full((y0.shape[0], N), np.nan)
    for a in np.unique(row_adapter[row_adapter >= 0]):
        rows = np.nonzero(row_adapter == a)[0]
        acc = xh[rows] @ wd[a].T
        pre[rows] = y[rows] + acc if add else acc
    return pre


def check_rounded(out, pre_want, written, col0, N, out_dt, y0):
    got = indep_decode(out, out_dt)[:, col0:col0 + N]
    if out_dt == "f32":
        assert np.array_equal(got[written], pre_want[written].astype(np.float32).astype(np.float64))
    else:
        err = np.abs(got[written] - pre_want[written])
        assert np.all(err <= 0.5 * ulp_of(got[written], out_dt) * (1 + 1e-9))
    mask = np.ones(y0.shape, dtype=bool)
    mask[np.ix_(written, np.arange(col0, col0 + N))] = False
    assert np.array_equal(out[mask], y0[mask])


@pytest.mark.parametrize("out_dt,add", [("bf16", True), ("f16", False), ("f32", True)])
def test_bgmv_matches_dense_per_adapter(out_dt, add):
    B, K, N, H, off, A = 37, 24, 40, 100, 17, 5
    p = gen.custom(seed=5, lengths=[1] * B, K=K, N=N, H=H, offset=off, num_adapters=A, out_dt=out_dt,
                   x_dt="f32", w_dt="bf16", add_inputs=add,
                   idx=[(3 * b) % (A + 2) - 1 for b in range(B)])   # includes -1 and A (out of range)
    c = p.calls[0]
    out, pre = oracle.bgmv_expand_slice(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.lora_idx, off, N, add,
                                        return_pre=True)
    ra = np.where((p.lora_idx >= 0) & (p.lora_idx < A), p.lora_idx, -1)
    want = dense_rows(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, ra, off, add)
    written = ra >= 0
    assert written.any() and (~written).any()
    np.testing.assert_allclose(pre[written], want[written], rtol=1e-12, atol=1e-12)
    assert np.all(np.isnan(pre[~written]))
    check_rounded(out, want, written, off, N, out_dt, p.y0)


def test_bgmv_rows_beyond_batches_are_untouched():
    B, K, N, A = 12, 16, 32, 3
    p = gen.custom(seed=6, lengths=[1] * B, K=K, N=N, H=N, offset=0, num_adapters=A, idx=[b % A for b in range(B)])
    c = p.calls[0]
    out = oracle.bgmv_expand_slice(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.lora_idx, 0, N, True, batches=7)
    assert np.array_equal(out[7:], p.y0[7:])
    assert not np.array_equal(out[:7], p.y0[:7])


def test_bgmv_integer_inputs_are_exact():
    B, K, N, A = 20, 16, 48, 4     # |sum| <= 3 + 16 * 9 < 256: every value exact in bf16
    p = gen.custom(seed=7, lengths=[1] * B, K=K, N=N, H=N + 8, offset=8, num_adapters=A, integer=True,
                   idx=[b % A for b in range(B)])
    c = p.calls[0]
    out = oracle.bgmv_expand_slice(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.lora_idx, 8, N, True)
    xi = indep_decode(p.x, p.x_dt).astype(np.int64)
    wi = indep_decode(c.w, p.w_dt).astype(np.int64)
    yi = indep_decode(p.y0, p.out_dt).astype(np.int64)
    for b in range(B):
        exact = yi[b, 8:8 + N] + wi[p.lora_idx[b]] @ xi[b]
        assert np.array_equal(indep_decode(out[b, 8:8 + N], p.out_dt), exact.astype(np.float64))


def test_bgmv_equals_sgmv_with_one_token_segments_in_any_order():
    """A batch of one-token rows is an SGMV batch whose segments may come in any order."""
    B, K, N, A = 25, 16, 64, 6
    p = gen.custom(seed=8, lengths=[1] * B, K=K, N=N, H=2 * N, offset=N, num_adapters=A)
    c = p.calls[0]
    out_b = oracle.bgmv_expand_slice(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.lora_idx, N, N, True)
    perm = np.random.default_rng(1).permutation(B)
    out_s = oracle.expand_slice(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, perm, np.ones(B, np.int64),
                                p.lora_idx[perm], N, N, True)
    assert np.array_equal(out_b, out_s)


@pytest.mark.parametrize("add", [True, False])
def test_plain_expand_matches_dense_over_whole_rows(add):
    lengths = [5, 0, 9, 3]
    K, N, A = 16, 72, 3
    p = gen.custom(seed=9, lengths=lengths, K=K, N=N, H=N, offset=0, num_adapters=A, add_inputs=add,
                   idx=[2, 0, -1, 1])
    c = p.calls[0]
    out, pre = oracle.expand(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.seq_start, p.seq_len, p.lora_idx,
                             add, return_pre=True)
    ra = np.full(p.y0.shape[0], -1)
    for s, L, a in zip(p.seq_start, p.seq_len, p.lora_idx):
        if a >= 0:
            ra[s:s + L] = a
    want = dense_rows(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, ra, 0, add)
    written = ra >= 0
    np.testing.assert_allclose(pre[written], want[written], rtol=1e-12, atol=1e-12)
    check_rounded(out, want, written, 0, N, p.out_dt, p.y0)


def test_plain_expand_requires_whole_rows():
    p = gen.custom(seed=10, lengths=[4], K=16, N=32, H=40, offset=0, num_adapters=1)
    c = p.calls[0]
    with pytest.raises(AssertionError):
        oracle.expand(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.seq_start, p.seq_len, p.lora_idx, True)


# ------------------------------------------------------------------ shrink

def shrink_problem(seed, lengths, H, R, A, **kw):
    """x (T, H), lora_a (A, R, H) in calls[0].w, out (T, R)."""
    return gen.custom(seed=seed, lengths=lengths, K=H, N=R, H=R, offset=0, num_adapters=A, add_inputs=False, **kw)


@pytest.mark.parametrize("x_dt,a_dt,out_dt", [("bf16", "bf16", "f32"), ("f16", "f16", "bf16"), ("f32", "bf16", "f16")])
def test_shrink_matches_dense_per_adapter(x_dt, a_dt, out_dt):
    p = shrink_problem(11, [7, 0, 20, 3], H=300, R=16, A=3, idx=[2, 1, 0, -1], x_dt=x_dt, w_dt=a_dt, out_dt=out_dt)
    c = p.calls[0]
    out, pre = oracle.shrink(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.seq_start, p.seq_len, p.lora_idx,
                             return_pre=True)
    ra = np.full(p.y0.shape[0], -1)
    for s, L, a in zip(p.seq_start, p.seq_len, p.lora_idx):
        if a >= 0:
            ra[s:s + L] = a
    want = dense_rows(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, ra, 0, False)
    written = ra >= 0
    np.testing.assert_allclose(pre[written], want[written], rtol=1e-12, atol=1e-12)
    check_rounded(out, want, written, 0, 16, out_dt, p.y0)


def test_shrink_integer_inputs_are_exact():
    p = shrink_problem(12, [5, 9], H=64, R=32, A=2, idx=[1, 0], integer=True, out_dt="f32")
    c = p.calls[0]
    out = oracle.shrink(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.seq_start, p.seq_len, p.lora_idx)
    xi = indep_decode(p.x, p.x_dt).astype(np.int64)
    ai = indep_decode(c.w, p.w_dt).astype(np.int64)
    for s, L, a in zip(p.seq_start, p.seq_len, p.lora_idx):
        exact = xi[s:s + L] @ ai[a].T
        assert np.array_equal(out[s:s + L].astype(np.float64), exact.astype(np.float64))


def test_shrink_then_expand_is_the_lora_delta():
    """Shrink into an fp32 intermediate, then expand: the slice gets x . A^T . B^T (the LoRA update)."""
    H, R, N, A = 96, 16, 40, 2
    p = shrink_problem(13, [6, 4], H=H, R=R, A=A, idx=[1, 0], out_dt="f32", y_scale=0.0)
    a = p.calls[0].w
    mid = oracle.shrink(p.x, p.x_dt, a, p.w_dt, p.y0, "f32", p.seq_start, p.seq_len, p.lora_idx)
    rng = np.random.default_rng(3)
    b = gen.normal(rng, (A, N, R), 0.02, "bf16")
    y0 = np.zeros((10, N), np.float32)
    y = oracle.expand(mid, "f32", b, "bf16", y0, "f32", p.seq_start, p.seq_len, p.lora_idx, False)
    xd = indep_decode(p.x, p.x_dt)
    for s, L, ai in zip(p.seq_start, p.seq_len, p.lora_idx):
        delta = xd[s:s + L] @ indep_decode(a[ai], "bf16").T
        delta = indep_cast(delta.astype(np.float32).astype(np.float64), "bf16") @ indep_decode(b[ai], "bf16").T
        np.testing.assert_allclose(y[s:s + L], delta, rtol=1e-5, atol=1e-6)
