"""GPU parity of plain SGMV expand and BGMV expand-slice against the CPU oracle.

Plain expand is the slice operation over the whole output row; BGMV is its
one-token-per-row counterpart ("Implementation: Predibase Lorax SGMV Expand
Slice Kernel", Description).  Same tolerance and bit-exactness rules as the
expand-slice parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
import sgmv_inputs as gen
import segmented_gather_gemm_expand_b200 as sg
from sgmv_testlib import compare, from_torch, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset_variant():
    yield
    sg.set_variant(sg.VARIANT_AUTO)


def bgmv_problem(seed, B, K, N, H, off, A, **kw):
    return gen.custom(seed=seed, lengths=[1] * B, K=K, N=N, H=H, offset=off, num_adapters=A, **kw)


def run_bgmv(p, variant, batches=None, idx_dt=torch.int64):
    c = p.calls[0]
    x = to_torch(p.x, p.x_dt)
    w = to_torch(c.w, p.w_dt)
    y = to_torch(p.y0, p.out_dt)
    idx = torch.as_tensor(np.asarray(p.lora_idx), dtype=idx_dt).cuda()
    B = p.batches if batches is None else batches
    sg.set_variant(variant)
    v = sg.bgmv_plan(x, w, y, idx, c.slice_offset, c.slice_size, p.add_inputs, batches=B)
    sg.bgmv_expand_slice(x, w, y, idx, c.slice_offset, c.slice_size, p.add_inputs, batches=B)
    torch.cuda.synchronize()
    assert sg.device_error() == 0
    gpu = from_torch(y, p.out_dt)
    ref = oracle.bgmv_expand_slice(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.lora_idx, c.slice_offset,
                                   c.slice_size, p.add_inputs, batches=B)
    A = c.w.shape[0]
    lim = min(p.y0.shape[0], p.x.shape[0], B)
    rows = np.zeros(p.y0.shape[0], dtype=bool)
    li = np.asarray(p.lora_idx)
    rows[:lim] = (li[:lim] >= 0) & (li[:lim] < A)
    compare(gpu, ref, p.y0, p, rows, c.slice_offset, c.slice_size)
    return v


BGMV_VARIANTS = {"auto": sg.VARIANT_AUTO, "simt": sg.VARIANT_SIMT}


@pytest.mark.parametrize("variant", BGMV_VARIANTS)
@pytest.mark.parametrize("K", [8, 16, 32, 64, 128, 256])
def test_bgmv_ranks(K, variant):
    p = bgmv_problem(K, B=70, K=K, N=300, H=700, off=256, A=5)
    v = run_bgmv(p, BGMV_VARIANTS[variant])
    assert v == (sg.VARIANT_DECODE if variant == "auto" else sg.VARIANT_SIMT)


@pytest.mark.parametrize("variant", BGMV_VARIANTS)
@pytest.mark.parametrize("x_dt,w_dt,out_dt", [("f32", "bf16", "bf16"), ("f16", "f16", "f16"), ("bf16", "bf16", "f32"),
                                              ("f16", "bf16", "f16"), ("f32", "f16", "f32")])
def test_bgmv_dtypes(x_dt, w_dt, out_dt, variant):
    p = bgmv_problem(2, B=33, K=32, N=256, H=512, off=256, A=4, x_dt=x_dt, w_dt=w_dt, out_dt=out_dt)
    run_bgmv(p, BGMV_VARIANTS[variant])


@pytest.mark.parametrize("variant", BGMV_VARIANTS)
def test_bgmv_odd_width_offset_and_invalid_ids(variant):
    """Odd slice width and offset; ids -1, lora_num and -5 leave their rows alone; overwrite mode."""
    B, A = 29, 4
    idx = [(b % (A + 3)) - 2 for b in range(B)]          # -2 .. A: several invalid ids
    p = bgmv_problem(3, B=B, K=16, N=61, H=100, off=3, A=A, idx=idx, add_inputs=False)
    run_bgmv(p, BGMV_VARIANTS[variant], idx_dt=torch.int32)


@pytest.mark.parametrize("variant", BGMV_VARIANTS)
def test_bgmv_batches_smaller_than_rows(variant):
    p = bgmv_problem(4, B=40, K=16, N=128, H=128, off=0, A=3)
    run_bgmv(p, BGMV_VARIANTS[variant], batches=23)


@pytest.mark.parametrize("K,pad", [(32, 8), (64, 16), (16, 0), (8, 0)])
def test_bgmv_dense_and_padded_b_rows(K, pad):
    """Dense and padded B rows (row stride K or K + pad) both take the decode kernel; slices of 1, 255, 256
    and 257 columns cover a CTA's 256-column tile whole, partly and with one column over."""
    for N in (1, 255, 256, 257):
        p = bgmv_problem(K + N + pad, B=37, K=K, N=N, H=N + 40, off=24, A=4, w_row_pad=pad,
                         idx=[(i * 3) % 6 - 1 for i in range(37)])
        assert run_bgmv(p, sg.VARIANT_AUTO) == sg.VARIANT_DECODE


def test_bgmv_strided_x_takes_the_decode_kernel():
    p = bgmv_problem(5, B=20, K=24, N=96, H=192, off=96, A=3, x_col_pad=3)
    assert run_bgmv(p, sg.VARIANT_AUTO) == sg.VARIANT_DECODE


@pytest.mark.parametrize("case", [dict(K=12), dict(K=16, w_row_pad=1)])
def test_bgmv_layouts_the_decode_kernel_does_not_take(case):
    """K not a multiple of 8, or B rows not on 16-byte boundaries: the generic kernel runs,
    and forcing the decode kernel is refused before any launch."""
    p = bgmv_problem(6, B=18, N=80, H=160, off=80, A=3, **case)
    assert run_bgmv(p, sg.VARIANT_AUTO) == sg.VARIANT_SIMT
    c = p.calls[0]
    sg.set_variant(sg.VARIANT_DECODE)
    x, w, y = to_torch(p.x, p.x_dt), to_torch(c.w, p.w_dt), to_torch(p.y0, p.out_dt)
    idx = torch.as_tensor(np.asarray(p.lora_idx)).cuda()
    with pytest.raises(sg.SgmvError) as e:
        sg.bgmv_expand_slice(x, w, y, idx, c.slice_offset, c.slice_size, True)
    assert e.value.code == -13
    torch.cuda.synchronize()
    assert np.array_equal(from_torch(y, p.out_dt), p.y0)


@pytest.mark.parametrize("variant", BGMV_VARIANTS)
def test_bgmv_decode_batch_full_size(variant):
    """256 one-token rows with distinct adapters (26 at -1), rank 32, a 5120-wide slice of a 15360-wide output."""
    rng = np.random.default_rng(0)
    idx = rng.permutation(256)
    idx[rng.permutation(256)[:26]] = -1
    p = bgmv_problem(7, B=256, K=32, N=5120, H=15360, off=5120, A=256, idx=idx.tolist())
    run_bgmv(p, BGMV_VARIANTS[variant])


def test_bgmv_empty_batch_writes_nothing():
    p = bgmv_problem(8, B=4, K=16, N=64, H=64, off=0, A=2)
    c = p.calls[0]
    x, w, y = to_torch(p.x, p.x_dt), to_torch(c.w, p.w_dt), to_torch(p.y0, p.out_dt)
    idx = torch.as_tensor(np.asarray(p.lora_idx)).cuda()
    assert sg.bgmv_plan(x, w, y, idx, 0, 64, True, batches=0) == 0
    sg.bgmv_expand_slice(x, w, y, idx, 0, 64, True, batches=0)
    torch.cuda.synchronize()
    assert np.array_equal(from_torch(y, p.out_dt), p.y0)


# ------------------------------------------------------------------ plain expand

@pytest.mark.parametrize("variant", {"simt": sg.VARIANT_SIMT, "tc": sg.VARIANT_TC})
@pytest.mark.parametrize("add", [True, False])
def test_plain_expand(variant, add):
    p = gen.custom(seed=21, lengths=[130, 0, 7, 300, 64], K=16, N=384, H=384, offset=0, num_adapters=4,
                   idx=[3, 1, -1, 0, 2], add_inputs=add)
    c = p.calls[0]
    x, w, y = to_torch(p.x, p.x_dt), to_torch(c.w, p.w_dt), to_torch(p.y0, p.out_dt)
    meta = [torch.as_tensor(np.asarray(a)).cuda() for a in (p.seq_start, p.seq_len, p.lora_idx)]
    sg.set_variant({"simt": sg.VARIANT_SIMT, "tc": sg.VARIANT_TC}[variant])
    sg.sgmv_expand(x, w, y, *meta, p.batches, p.max_seq_len, add)
    torch.cuda.synchronize()
    assert sg.device_error() == 0
    gpu = from_torch(y, p.out_dt)
    ref = oracle.expand(p.x, p.x_dt, c.w, p.w_dt, p.y0, p.out_dt, p.seq_start, p.seq_len, p.lora_idx, add)
    rows = np.zeros(p.y0.shape[0], dtype=bool)
    for s, L, a in zip(p.seq_start, p.seq_len, p.lora_idx):
        if a >= 0:
            rows[s:s + L] = True
    compare(gpu, ref, p.y0, p, rows, 0, 384)


def test_plain_expand_rejects_partial_width():
    p = gen.custom(seed=22, lengths=[8], K=16, N=64, H=128, offset=0, num_adapters=1)
    c = p.calls[0]
    x, w, y = to_torch(p.x, p.x_dt), to_torch(c.w, p.w_dt), to_torch(p.y0, p.out_dt)
    meta = [torch.as_tensor(np.asarray(a)).cuda() for a in (p.seq_start, p.seq_len, p.lora_idx)]
    with pytest.raises(sg.SgmvError) as e:
        sg.sgmv_expand(x, w, y, *meta, 1, 8, True)
    assert e.value.code == -16
