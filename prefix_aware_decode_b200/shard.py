"""Data-parallel sharding of one decode batch across ranks (host logic).

Data parallelism: requests are grouped by the page id of their first block: requests in
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


# ------------------------------------------------------------- context parallel

def context_slices(block_table: np.ndarray, kv_lens: np.ndarray, world: int):
    """Context-parallel split of one batch: the pages of every request are cut
    into `world` contiguous, page-aligned slices, slice r going to rank r, so a
    long session's KV is spread over the GPUs.  Returns, per rank,
    (requests, block_table, kv_lens): the requests holding at least one token
    in the rank's slice, their slice's page ids (from column 0) and token
    counts.  Requests that share a prefix share it inside each slice too (the
    slices are cut at the same page positions), so each rank's plan still packs
    the shared pages.  Slice boundaries sit at page multiples, so only a
    request's last slice may end inside a page."""
    P = 16
    B = len(kv_lens)
    npg = (kv_lens.astype(np.int64) + P - 1) // P
    out = []
    for r in range(world):
        lo = npg * r // world
        hi = npg * (r + 1) // world
        reqs = np.nonzero(hi > lo)[0]
        width = int((hi - lo)[reqs].max()) if len(reqs) else 1
        bt = np.full((len(reqs), max(1, width)), -1, dtype=np.int32)
        kl = np.zeros(len(reqs), dtype=np.int32)
        for i, b in enumerate(reqs):
            bt[i, :hi[b] - lo[b]] = block_table[b, lo[b]:hi[b]]
            kl[i] = min(int(kv_lens[b]), int(hi[b]) * P) - int(lo[b]) * P
        out.append((reqs.astype(np.int64), bt, kl))
    return out


def exchange_context_parts(reqs, out_f32, lse_f32, batch: int, out, lse=None, group=None):
    """The exchange step of context parallelism on GPUs: every rank's
    (request ids, fp32 out [n][Hq][D], lse [n][Hq]) of its slice, padded to the
    largest slice, is all-gathered over NCCL (torch.distributed, the process
    group's backend), and the rows are merged on the device by pa_merge_rows
    into out (bf16 [batch][Hq][D]) and lse.  Every rank ends with the whole
    batch's result.  All tensors are CUDA tensors."""
    import torch
    import torch.distributed as dist

    from ._binding import merge_rows

    world = dist.get_world_size(group)
    n = torch.tensor([len(reqs)], device=out_f32.device, dtype=torch.int64)
    dist.all_reduce(n, op=dist.ReduceOp.MAX, group=group)
    R = max(1, int(n.item()))
    Hq, D = out_f32.shape[1], out_f32.shape[2]
    req = torch.full((R,), -1, dtype=torch.int32, device=out_f32.device)
    o = torch.zeros((R, Hq, D), dtype=torch.float32, device=out_f32.device)
    ls = torch.full((R, Hq), float("-inf"), dtype=torch.float32, device=out_f32.device)
    k = len(reqs)
    req[:k] = torch.as_tensor(np.asarray(reqs), dtype=torch.int32, device=out_f32.device)
    o[:k] = out_f32[:k]
    ls[:k] = lse_f32[:k]
    all_req = torch.empty((world, R), dtype=torch.int32, device=out_f32.device)
    all_o = torch.empty((world, R, Hq, D), dtype=torch.float32, device=out_f32.device)
    all_l = torch.empty((world, R, Hq), dtype=torch.float32, device=out_f32.device)
    dist.all_gather_into_tensor(all_req, req, group=group)
    dist.all_gather_into_tensor(all_o, o, group=group)
    dist.all_gather_into_tensor(all_l, ls, group=group)
    merge_rows(all_req, all_o, all_l, batch, out, lse)
