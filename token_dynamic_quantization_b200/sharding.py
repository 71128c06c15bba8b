"""Row sharding across ranks (one process per GPU).

Rows are independent units of per-token quantization (aclnnDynamicQuantV2,
"Formula": one scale per row), so a batch shards into contiguous row ranges
with no exchange between ranks. The only cross-row input is the MoE group
index (aclnnDynamicQuantV2, "Description"), whose cumulative end rows are
rebased to each shard's first row.
"""

from __future__ import annotations

import numpy as np


def row_range(rows: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [start, end) of ``rows`` owned by ``rank`` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    return rows * rank // world, rows * (rank + 1) // world


def rebase_group_index(group_index, start: int, end: int) -> np.ndarray:
    """Cumulative end rows of every expert, seen from a shard [start, end).

    Entry e becomes clip(group_index[e] - start, 0, end - start): the shard's
    local row i belongs to the smallest e with start + i < group_index[e],
    and rows past the last group stay past it.
    """
    gi = np.asarray(group_index, dtype=np.int64)
    return np.clip(gi - start, 0, end - start).astype(np.int32)
