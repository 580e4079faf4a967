"""Seeded synthetic inputs for SGMV expand-slice.

This module only draws random numbers and lays them out; it holds none of the
operation's arithmetic.  Both the CPU oracle's tests and the CUDA path's tests
and benchmark take their inputs from here.

Storage convention (host, numpy): 'f16' and 'bf16' tensors are uint16 bit
patterns, 'f32' tensors are float32.  Normals are drawn as float32 from
`numpy.random.default_rng(seed)`, scaled, and rounded to nearest-even into
the storage dtype.

Workloads (shapes and distributions of the multi-tenant LoRA prefill/decode
cases the operation serves; lengths, adapters and -1 entries as stated):
  tiny          4 sequences [4,6,3,7], fp16, slice 128 at offset 128, overwrite
  qkv_prefill   Llama-7B fused QKV: 16 seqs U{64..1024}, r=16, 3 slices of 4096
  mlp_mixed     gate/up: 64 seqs Geom(mean 256) <= 2048, r=64, fp32 x, 4-D bf16 B
  long_single   1 x 32768 tokens, r=8, fp16, write-only
  decode_mix    256 seqs Zipf(1.2) clipped [1,64], r=32, distinct adapters
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import numpy as np

HALF_DTYPES = ("f16", "bf16")
ALL_DTYPES = ("f16", "bf16", "f32")


def storage_dtype(dt: str):
    return np.float32 if dt == "f32" else np.uint16


def to_storage(values: np.ndarray, dt: str) -> np.ndarray:
    """float32/float64 values -> storage of dtype `dt` (nearest-even)."""
    v = np.asarray(values)
    if dt == "f32":
        return v.astype(np.float32)
    if dt == "f16":
        return v.astype(np.float32).astype(np.float16).view(np.uint16)
    if dt == "bf16":
        import torch  # conversion only
        t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
        return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(dt)


def normal(rng: np.random.Generator, shape, scale: float, dt: str) -> np.ndarray:
    v = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        v *= np.float32(scale)
    return to_storage(v, dt)


def small_ints(rng: np.random.Generator, shape, lo: int, hi: int, dt: str) -> np.ndarray:
    return to_storage(rng.integers(lo, hi + 1, size=shape).astype(np.float32), dt)


@dataclasses.dataclass
class SliceCall:
    w: np.ndarray            # (A, N, K) or (A, 1, N, K) storage array
    slice_offset: int
    slice_size: int


@dataclasses.dataclass
class Problem:
    name: str
    x: np.ndarray            # (T, K) storage array, possibly a strided view
    x_dt: str
    w_dt: str
    y0: np.ndarray           # (T_out, H) storage array, contiguous
    out_dt: str
    seq_start: np.ndarray    # int64 (B,)
    seq_len: np.ndarray      # int64 (B,)
    lora_idx: np.ndarray     # int64 (B,)
    add_inputs: bool
    calls: List[SliceCall]
    meta_dt: str = "int64"   # dtype the metadata is handed to the library in
    seed: int = 0
    op: str = "slice"        # "slice": sgmv_expand_slice; "bgmv": one token per row (starts b, lengths 1);
                             # "shrink": sgmv_shrink (x is (T, H), calls[0].w is lora_a (A, R, H), out (T, R))

    @property
    def batches(self) -> int:
        return int(len(self.seq_len))

    @property
    def rank(self) -> int:
        return int(self.x.shape[1])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_len.max()) if len(self.seq_len) else 0

    @property
    def total_tokens(self) -> int:
        return int(self.y0.shape[0])

    def active_tokens(self) -> int:
        """Tokens whose adapter index is valid (rows that get written)."""
        A = self.calls[0].w.shape[0]
        ok = (self.lora_idx >= 0) & (self.lora_idx < A)
        return int(self.seq_len[ok].clip(min=0).sum())


def exclusive_cumsum(lengths: Sequence[int]) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    out = np.zeros(len(lengths), dtype=np.int64)
    if len(lengths) > 1:
        out[1:] = np.cumsum(lengths[:-1])
    return out


def _minus_one_mask(rng, B: int, frac: float) -> np.ndarray:
    """Exactly round(frac*B) entries, chosen by a seeded permutation."""
    k = int(round(frac * B))
    mask = np.zeros(B, dtype=bool)
    if k:
        mask[rng.permutation(B)[:k]] = True
    return mask


# ---------------------------------------------------------------- workloads

def tiny(seed: int = 0) -> Problem:
    rng = np.random.default_rng(seed)
    lengths = np.array([4, 6, 3, 7], dtype=np.int64)
    starts = np.array([0, 4, 10, 13], dtype=np.int64)
    idx = np.array([0, 2, -1, 1], dtype=np.int64)
    x = normal(rng, (20, 16), 1.0, "f16")
    w = normal(rng, (3, 128, 16), 0.05, "f16")
    y0 = normal(rng, (20, 384), 1.0, "f16")
    return Problem("tiny", x, "f16", "f16", y0, "f16", starts, lengths, idx, False,
                   [SliceCall(w, 128, 128)], seed=seed)


def qkv_prefill(seed: int = 0) -> Problem:
    rng = np.random.default_rng(seed)
    B, K, A, N = 16, 16, 32, 4096
    lengths = rng.integers(64, 1024 + 1, size=B).astype(np.int64)
    idx = rng.integers(0, A, size=B).astype(np.int64)
    idx[_minus_one_mask(rng, B, 0.10)] = -1
    T = int(lengths.sum())
    x = normal(rng, (T, K), 1.0, "bf16")
    calls = [SliceCall(normal(rng, (A, N, K), 0.02, "bf16"), off, N) for off in (0, 4096, 8192)]
    y0 = normal(rng, (T, 3 * N), 1.0, "bf16")
    return Problem("qkv_prefill", x, "bf16", "bf16", y0, "bf16", exclusive_cumsum(lengths),
                   lengths, idx, True, calls, seed=seed)


def mlp_mixed(seed: int = 0) -> Problem:
    rng = np.random.default_rng(seed)
    B, K, A, N = 64, 64, 128, 11008
    lengths = np.minimum(rng.geometric(1.0 / 256.0, size=B), 2048).astype(np.int64)
    idx = rng.integers(0, A, size=B).astype(np.int64)
    T = int(lengths.sum())
    x = normal(rng, (T, K), 1.0, "f32")
    calls = [SliceCall(normal(rng, (A, 1, N, K), 0.02, "bf16"), off, N) for off in (0, N)]
    y0 = normal(rng, (T, 2 * N), 1.0, "bf16")
    return Problem("mlp_mixed", x, "f32", "bf16", y0, "bf16", exclusive_cumsum(lengths),
                   lengths, idx, True, calls, seed=seed)


def long_single(seed: int = 0) -> Problem:
    rng = np.random.default_rng(seed)
    T, K, N = 32768, 8, 4096
    lengths = np.array([T], dtype=np.int64)
    idx = np.array([0], dtype=np.int64)
    x = normal(rng, (T, K), 1.0, "f16")
    w = normal(rng, (1, N, K), 0.02, "f16")
    y0 = normal(rng, (T, N), 1.0, "f16")
    return Problem("long_single", x, "f16", "f16", y0, "f16", np.zeros(1, np.int64), lengths, idx,
                   False, [SliceCall(w, 0, N)], seed=seed)


def decode_mix(seed: int = 0) -> Problem:
    rng = np.random.default_rng(seed)
    B, K, A, N = 256, 32, 256, 5120
    lengths = np.clip(rng.zipf(1.2, size=B), 1, 64).astype(np.int64)
    idx = rng.permutation(A)[:B].astype(np.int64)
    idx[_minus_one_mask(rng, B, 0.10)] = -1
    T = int(lengths.sum())
    x = normal(rng, (T, K), 1.0, "bf16")
    w = normal(rng, (A, N, K), 0.02, "bf16")
    y0 = normal(rng, (T, 3 * N), 1.0, "bf16")
    return Problem("decode_mix", x, "bf16", "bf16", y0, "bf16", exclusive_cumsum(lengths),
                   lengths, idx, True, [SliceCall(w, 5120, N)], seed=seed)


def decode_bgmv(seed: int = 0) -> Problem:
    """The decode step of the decode-like mix: one token per sequence (the BGMV
    case), 256 sequences with distinct adapters out of 256, 10% at -1."""
    rng = np.random.default_rng(seed)
    B, K, A, N = 256, 32, 256, 5120
    lengths = np.ones(B, dtype=np.int64)
    idx = rng.permutation(A)[:B].astype(np.int64)
    idx[_minus_one_mask(rng, B, 0.10)] = -1
    x = normal(rng, (B, K), 1.0, "bf16")
    w = normal(rng, (A, N, K), 0.02, "bf16")
    y0 = normal(rng, (B, 3 * N), 1.0, "bf16")
    return Problem("decode_bgmv", x, "bf16", "bf16", y0, "bf16", exclusive_cumsum(lengths),
                   lengths, idx, True, [SliceCall(w, 5120, N)], seed=seed, op="bgmv")


def qkv_shrink(seed: int = 0) -> Problem:
    """The LoRA-A step that feeds the fused-QKV prefill batch: the same 16
    sequences (lengths U[64,1024], 10% at -1, 32 adapters), hidden size 4096
    projected to rank 16, bf16 in and out."""
    rng = np.random.default_rng(seed)
    B, R, A, H = 16, 16, 32, 4096
    lengths = rng.integers(64, 1024 + 1, size=B).astype(np.int64)
    idx = rng.integers(0, A, size=B).astype(np.int64)
    idx[_minus_one_mask(rng, B, 0.10)] = -1
    T = int(lengths.sum())
    x = normal(rng, (T, H), 1.0, "bf16")
    a = normal(rng, (A, R, H), 0.02, "bf16")
    y0 = normal(rng, (T, R), 1.0, "bf16")
    return Problem("qkv_shrink", x, "bf16", "bf16", y0, "bf16", exclusive_cumsum(lengths), lengths, idx, False,
                   [SliceCall(a, 0, R)], seed=seed, op="shrink")


WORKLOADS = {
    "tiny": tiny,
    "qkv_prefill": qkv_prefill,
    "mlp_mixed": mlp_mixed,
    "long_single": long_single,
    "decode_mix": decode_mix,
    "decode_bgmv": decode_bgmv,
    "qkv_shrink": qkv_shrink,
}


# ------------------------------------------------------------ custom cases

def custom(seed: int = 0, *, lengths: Sequence[int], K: int, N: int, H: int, offset: int,
           num_adapters: int, x_dt: str = "bf16", w_dt: str = "bf16", out_dt: str = "bf16",
           idx: Optional[Sequence[int]] = None, starts: Optional[Sequence[int]] = None,
           extra_rows: int = 0, add_inputs: bool = True, layout4d: bool = False,
           x_col_pad: int = 0, w_row_pad: int = 0, x_scale: float = 1.0, w_scale: float = 0.02,
           y_scale: float = 1.0, integer: bool = False, meta_dt: str = "int64",
           n_calls: int = 1) -> Problem:
    """A problem with explicit segment structure.

    starts=None packs the segments back to back (exclusive cumulative sum);
    extra_rows adds untouched rows after the last segment; x_col_pad makes x a
    strided column view of a wider buffer; w_row_pad makes B's row stride K +
    w_row_pad; integer=True draws small integers in [-3, 3] (exact sums).
    """
    rng = np.random.default_rng(seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    B = len(lengths)
    if idx is None:
        idx = rng.integers(0, num_adapters, size=B)
    idx = np.asarray(idx, dtype=np.int64)
    if starts is None:
        starts = exclusive_cumsum(lengths)
        T = int(lengths.sum()) + extra_rows
    else:
        starts = np.asarray(starts, dtype=np.int64)
        T = int(max([0] + [s + l for s, l in zip(starts, lengths)])) + extra_rows

    def draw(shape, scale, dt):
        if integer:
            return small_ints(rng, shape, -3, 3, dt)
        return normal(rng, shape, scale, dt)

    xbuf = draw((T, K + x_col_pad), x_scale, x_dt)
    x = xbuf[:, :K]
    calls = []
    for c in range(n_calls):
        wbuf = draw((num_adapters, N, K + w_row_pad), w_scale, w_dt)
        w = wbuf[:, :, :K]
        if layout4d:
            w = w[:, None]
        calls.append(SliceCall(w, offset + c * N if n_calls > 1 else offset, N))
    y0 = draw((T, H), y_scale, out_dt)
    return Problem("custom", x, x_dt, w_dt, np.ascontiguousarray(y0), out_dt, starts, lengths, idx,
                   add_inputs, calls, meta_dt=meta_dt, seed=seed)
