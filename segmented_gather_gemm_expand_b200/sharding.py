"""Host-side helpers for running SGMV expand-slice on several GPUs.

Every output row depends only on its own input row and its segment's adapter
("Implementation: Predibase Lorax SGMV Expand Slice Kernel", Description:
each token's slice is its input times its sequence's B matrix), so a batch
shards across GPUs with no exchange: each rank takes a contiguous set of
whole sequences (plus a copy of the adapters they use) and runs the same
call on its rows.  Nothing here touches a GPU.
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np


def partition_segments(seq_len: Sequence[int], lora_idx: Sequence[int], world: int,
                       lora_num: int | None = None) -> list:
    """Split sequence indices [0, B) into `world` contiguous ranges with about
    equal numbers of rows that get written (sequences whose adapter is valid).

    Returns a list of (begin, end) index pairs, one per rank; ranges may be
    empty.  Deterministic: every rank computes the same split.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    L = np.asarray(seq_len, dtype=np.int64).clip(min=0)
    idx = np.asarray(lora_idx, dtype=np.int64)
    ok = idx >= 0
    if lora_num is not None:
        ok &= idx < lora_num
    work = np.where(ok, L, 0)
    csum = np.concatenate([[0], np.cumsum(work)])
    total = int(csum[-1])
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        # first sequence whose cumulative work reaches the target
        b = int(np.searchsorted(csum, target, side="left"))
        bounds.append(max(bounds[-1], min(b, len(L))))
    bounds.append(len(L))
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def local_metadata(seq_start, seq_len, lora_idx, part: Tuple[int, int]):
    """The metadata of one rank's sequences, with starts renumbered so that the
    rank's rows are packed from row 0, and the global rows they came from.

    Returns (starts, lens, idx, rows) where `rows` indexes the global rows the
    rank owns, in the order of its local rows.
    """
    b0, b1 = part
    s = np.asarray(seq_start, dtype=np.int64)[b0:b1]
    L = np.asarray(seq_len, dtype=np.int64)[b0:b1].clip(min=0)
    a = np.asarray(lora_idx, dtype=np.int64)[b0:b1]
    rows = np.concatenate([np.arange(x, x + n) for x, n in zip(s, L)]) if len(L) else np.zeros(0, np.int64)
    starts = np.zeros(len(L), dtype=np.int64)
    if len(L) > 1:
        starts[1:] = np.cumsum(L[:-1])
    return starts, L, a, rows
