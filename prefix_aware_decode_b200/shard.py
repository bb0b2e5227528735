"""Data-parallel sharding of one decode batch across ranks (host logic).

Requests are grouped by the page id of their first block: requests in
different groups share no prefix, so whole groups (root subtrees of the tree
block table) are assigned to ranks and no shared node is split across GPUs.
Groups go to the least-loaded rank in decreasing order of KV tokens (longest
processing time first), so ranks receive about the same number of KV bytes.
No data-path collective is needed: each rank runs the full pack-forward-merge
on its own requests.
"""
from __future__ import annotations

import heapq
from typing import List

import numpy as np


def shard_by_root(block_table: np.ndarray, kv_lens: np.ndarray, world: int) -> List[np.ndarray]:
    """Returns, per rank, the sorted request indices it owns."""
    B = len(kv_lens)
    first = block_table[np.arange(B), 0]
    groups = {}
    for b in range(B):
        groups.setdefault(int(first[b]), []).append(b)
    # weight of a root subtree: its distinct tokens are at most the sum of its requests' tokens;
    # use the sum (what query-centric reads would cost) as the balancing key
    items = sorted(((int(kv_lens[g].sum()), tuple(g)) for g in groups.values()), reverse=True)
    heap = [(0, r) for r in range(world)]
    owned = [[] for _ in range(world)]
    for w, g in items:
        load, r = heapq.heappop(heap)
        owned[r].extend(g)
        heapq.heappush(heap, (load + w, r))
    return [np.array(sorted(o), dtype=np.int64) for o in owned]


def local_batch(block_table: np.ndarray, kv_lens: np.ndarray, q: np.ndarray, owned: np.ndarray):
    """The rank's slice of the batch (block table rows, kv lens, q rows)."""
    return (np.ascontiguousarray(block_table[owned]), np.ascontiguousarray(kv_lens[owned]),
            np.ascontiguousarray(q[owned]))
