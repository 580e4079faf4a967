"""Helpers shared by the tests: moving seeded problems to the GPU, running the
CUDA library on them, and comparing with the oracle under the stated tolerance.

Tolerance inside the written slice (per element, against the oracle's rounded
output value v):
  fp32 out:      |gpu - v| <= 1e-4 * sqrt(K)
  fp16/bf16 out: |gpu - v| <= 2 * ulp_out(v) + 1e-3
where ulp_out(v) is the spacing of the output format at |v| (floored at the
subnormal spacing).  Everything outside the written slice must be bit-exact.
"""
import numpy as np
import torch

import sgmv_inputs as gen

TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def to_torch(storage: np.ndarray, dt: str, device="cuda") -> torch.Tensor:
    """Storage array (possibly a strided view) -> torch tensor with the same strides."""
    a = storage
    strides = [st // a.itemsize for st in a.strides]
    assert all(st >= 0 for st in strides)
    span = 1 + sum((n - 1) * st for n, st in zip(a.shape, strides)) if a.size else 0
    flat = np.array(np.lib.stride_tricks.as_strided(a, shape=(span,), strides=(a.itemsize,)))
    t = torch.from_numpy(flat.view(np.int16) if dt != "f32" else flat)
    if dt != "f32":
        t = t.view(TORCH_DT[dt])
    t = t.to(device)
    return t.as_strided(tuple(a.shape), tuple(strides), 0)


def from_torch(t: torch.Tensor, dt: str) -> np.ndarray:
    t = t.detach().contiguous().cpu()
    if dt == "f32":
        return t.numpy().copy()
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def meta_tensors(p: gen.Problem, device="cuda"):
    tdt = torch.int64 if p.meta_dt == "int64" else torch.int32
    return [torch.as_tensor(np.asarray(a), dtype=tdt).to(device) for a in (p.seq_start, p.seq_len, p.lora_idx)]


class DeviceProblem:
    def __init__(self, p: gen.Problem, device="cuda"):
        self.p = p
        self.x = to_torch(p.x, p.x_dt, device)
        self.ws = [to_torch(c.w, p.w_dt, device) for c in p.calls]
        self.y = to_torch(p.y0, p.out_dt, device)
        self.start, self.len, self.idx = meta_tensors(p, device)

    def run(self, call=0, out=None, max_seq_len=None, add=None, batches=None):
        import segmented_gather_gemm_expand_b200 as sg
        c = self.p.calls[call]
        y = self.y if out is None else out
        sg.sgmv_expand_slice(self.x, self.ws[call], y, self.start, self.len, self.idx,
                             self.p.batches if batches is None else batches,
                             self.p.max_seq_len if max_seq_len is None else max_seq_len,
                             c.slice_offset, c.slice_size,
                             self.p.add_inputs if add is None else add)
        return y

    def plan(self, call=0):
        import segmented_gather_gemm_expand_b200 as sg
        c = self.p.calls[call]
        return sg.plan(self.x, self.ws[call], self.y, self.start, self.len, self.idx, self.p.batches,
                       self.p.max_seq_len, c.slice_offset, c.slice_size, self.p.add_inputs)

    def result(self) -> np.ndarray:
        return from_torch(self.y, self.p.out_dt)


def written_rows(p: gen.Problem, call=0) -> np.ndarray:
    """Boolean mask over out's rows that the call writes (guards of the header applied)."""
    c = p.calls[call]
    A = c.w.shape[0]
    T_out = p.y0.shape[0]
    lim = min(T_out, p.x.shape[0])
    m = np.zeros(T_out, dtype=bool)
    for s, L, a in zip(p.seq_start[:p.batches], p.seq_len[:p.batches], p.lora_idx[:p.batches]):
        if 0 <= a < A and s >= 0 and L > 0:
            m[s:min(s + L, lim)] = True
    return m


def decode(storage, dt):
    import oracle
    return oracle.decode(storage, dt)


def ulp_out(v: np.ndarray, dt: str) -> np.ndarray:
    f = 10 if dt == "f16" else 7
    emin = -14 if dt == "f16" else -126
    mag = np.abs(v)
    e = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    e = np.maximum(e, emin)
    return np.ldexp(1.0, (e - f).astype(int))


def tolerance(v: np.ndarray, dt: str, K: int) -> np.ndarray:
    if dt == "f32":
        return np.full(v.shape, 1e-4 * np.sqrt(max(K, 1)))
    return 2.0 * ulp_out(v, dt) + 1e-3


def compare(gpu: np.ndarray, ref: np.ndarray, y0: np.ndarray, p: gen.Problem, rows_mask: np.ndarray,
            col0: int, ncols: int, check_rows=None):
    """Assert: slice elements of `rows_mask` rows within tolerance, all else bit-exact.

    check_rows: optional boolean mask of rows whose slice values are compared
    (others in rows_mask are only required to differ from nothing: skipped).
    Returns the max error over compared elements.
    """
    dt = p.out_dt
    outside = np.ones(gpu.shape, dtype=bool)
    outside[np.ix_(rows_mask, np.arange(col0, col0 + ncols))] = False
    bad = np.nonzero((gpu != y0) & outside)
    assert bad[0].size == 0, f"{bad[0].size} untouched elements changed, first at {bad[0][0]},{bad[1][0]}"
    sel = rows_mask if check_rows is None else (rows_mask & check_rows)
    if not sel.any():
        return 0.0
    g = decode(gpu[sel, col0:col0 + ncols], dt)
    r = decode(ref[sel, col0:col0 + ncols], dt)
    both_nan = np.isnan(g) & np.isnan(r)
    same_inf = np.isinf(g) & np.isinf(r) & (np.sign(g) == np.sign(r))
    ok_special = both_nan | same_inf
    finite = ~ok_special
    assert np.all(np.isfinite(g[finite]) == np.isfinite(r[finite])), "non-finite mismatch"
    err = np.abs(g[finite] - r[finite])
    tol = tolerance(r[finite], dt, p.rank)
    worst = np.argmax(err - tol) if err.size else 0
    assert np.all(err <= tol), (f"max err {err.max():.3g} over tol; worst gpu={g[finite][worst]!r} "
                                f"ref={r[finite][worst]!r} tol={tol[worst]:.3g}")
    return float(err.max()) if err.size else 0.0


def run_multi(dp: DeviceProblem, calls=None, out=None, plan_only=False):
    """All (or the listed) slice calls of dp's problem as ONE multi-slice call.

    plan_only: return (variant, launches) instead of running."""
    import segmented_gather_gemm_expand_b200 as sg
    p = dp.p
    calls = list(range(len(p.calls))) if calls is None else list(calls)
    ws = [dp.ws[c] for c in calls]
    offs = [p.calls[c].slice_offset for c in calls]
    y = dp.y if out is None else out
    fn = sg.plan_multi_slice if plan_only else sg.sgmv_expand_multi_slice
    return fn(dp.x, ws, y, dp.start, dp.len, dp.idx, p.batches, p.max_seq_len, offs, p.add_inputs)


def _bits(a: np.ndarray) -> np.ndarray:
    """The storage's bit patterns (so that NaNs compare by their bits)."""
    return a.view(np.uint32) if a.dtype == np.float32 else a


def compare_every_element(gpu: np.ndarray, ref: np.ndarray, p: gen.Problem, regs, chunk_rows: int = 1024):
    """Compare a whole output with the oracle's, element by element, in row chunks.

    regs: [(rows_mask, col0, ncols), ...], the written regions.  Inside them every
    element must be within the stated tolerance of the oracle's value; every
    other element must keep the bits of p.y0.  Returns (max |err|, elements
    compared inside the regions).
    """
    dt = p.out_dt
    T, H = gpu.shape
    worst, count = 0.0, 0
    for r0 in range(0, T, chunk_rows):
        r1 = min(T, r0 + chunk_rows)
        g, rf, y0 = gpu[r0:r1], ref[r0:r1], p.y0[r0:r1]
        outside = np.ones(g.shape, dtype=bool)
        for rows, c0, n in regs:
            outside[np.ix_(rows[r0:r1], np.arange(c0, c0 + n))] = False
        bad = np.nonzero((_bits(g) != _bits(y0)) & outside)
        assert bad[0].size == 0, (f"{bad[0].size} untouched elements changed, first at row "
                                  f"{r0 + bad[0][0]}, column {bad[1][0]}")
        for rows, c0, n in regs:
            sel = rows[r0:r1]
            if not sel.any():
                continue
            gv = decode(g[sel, c0:c0 + n], dt)
            rv = decode(rf[sel, c0:c0 + n], dt)
            special = (np.isnan(gv) & np.isnan(rv)) | (np.isinf(gv) & np.isinf(rv) & (np.sign(gv) == np.sign(rv)))
            fin = ~special
            assert np.array_equal(np.isfinite(gv[fin]), np.isfinite(rv[fin])), f"non-finite mismatch in rows {r0}..{r1}"
            err = np.abs(gv[fin] - rv[fin])
            tol = tolerance(rv[fin], dt, p.rank)
            if err.size:
                i = np.argmax(err - tol)
                assert err[i] <= tol[i], (f"rows {r0}..{r1}: err {err[i]:.3g} > tol {tol[i]:.3g} "
                                          f"(gpu {gv[fin][i]!r}, oracle {rv[fin][i]!r})")
                worst = max(worst, float(err.max()))
            count += int(gv.size)
    return worst, count


def report(name: str, **fields):
    """Print a parity record, and append it as a JSON line to $SGMV_PARITY_REPORT if set."""
    import json
    import os
    rec = dict(test=name, **fields)
    print(json.dumps(rec))
    path = os.environ.get("SGMV_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")
