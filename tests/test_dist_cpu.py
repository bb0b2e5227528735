"""World-size-2 data-parallel path on CPU (gloo): each rank plans its root
subtrees with the C planner, executes the plan image in fp64, and the gathered
result equals the oracle over the whole batch."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    import torch

    import prefix_aware_decode_b200 as pad
    from plan_exec import Image, check_structure, execute
    from prefix_aware_decode_b200 import workload as wl
    from prefix_aware_decode_b200.shard import local_batch, shard_by_root

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        roots = wl.random_tree(seed=31, n_queries=12, depth=2, shared_pages=(1, 3), leaf_tokens=(1, 40))
        w = wl.build_workload("dp", roots, Hq=8, Hkv=2, D=64, seed=9)
        owned = shard_by_root(w.block_table, w.kv_lens, world)
        assert sum(len(o) for o in owned) == w.B
        mine = owned[rank]
        bt, kl, qq = local_batch(w.block_table, w.kv_lens, w.q, mine)
        out = np.zeros((w.B, w.Hq, w.D))
        lse = np.zeros((w.B, w.Hq))
        if len(mine):
            plan = pad.Plan(kl, bt, w.num_pages, w.Hq, w.Hkv, w.D)
            img = Image(plan.host_image())
            check_structure(img, kl, bt)
            o, l = execute(img, qq, w.k_pool, w.v_pool)
            out[mine], lse[mine] = o, l
        t_out, t_lse = torch.from_numpy(out), torch.from_numpy(lse)
        dist.all_reduce(t_out)
        dist.all_reduce(t_lse)
        if rank == 0:
            import oracle
            ro, rl = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
            q.put((float(np.abs(t_out.numpy() - ro).max()), float(np.abs(t_lse.numpy() - rl).max()),
                   [len(o) for o in owned]))
    finally:
        dist.destroy_process_group()


def _cp_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

    import prefix_aware_decode_b200 as pad
    from plan_exec import Image, check_structure, execute
    from prefix_aware_decode_b200 import workload as wl
    from prefix_aware_decode_b200.shard import context_slices

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # long sessions (config-5 shaped, scaled down): every rank holds a
        # page-aligned slice of every session's KV and plans it on its own
        w = wl.make_config(5, scale=1 / 64)
        reqs, bt, kl = context_slices(w.block_table, w.kv_lens, world)[rank]
        plan = pad.Plan(kl, bt, w.num_pages, w.Hq, w.Hkv, w.D)
        img = Image(plan.host_image())
        check_structure(img, kl, bt)
        o, l = execute(img, w.q[reqs], w.k_pool, w.v_pool)
        parts = [None] * world
        dist.all_gather_object(parts, (reqs, o, l))
        if rank == 0:
            import oracle
            # the exchange step's combine, done here with the oracle's merge
            # (on GPUs: pa_merge_rows after an NCCL all-gather)
            out = np.zeros((w.B, w.Hq, w.D))
            lse = np.zeros((w.B, w.Hq))
            for b in range(w.B):
                for h in range(w.Hq):
                    rows = [(o_[list(r_).index(b), h], l_[list(r_).index(b), h]) for r_, o_, l_ in parts if b in r_]
                    out[b, h], lse[b, h] = oracle.merge(np.stack([x[0] for x in rows]), np.array([x[1] for x in rows]))
            ro, rl = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
            q.put((float(np.abs(out - ro).max()), float(np.abs(lse - rl).max()),
                   [int(p_[2].shape[0]) for p_ in parts], plan.stats()["num_kept_shared"]))
    finally:
        dist.destroy_process_group()


def test_two_rank_context_parallel_sessions_match_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    err_o, err_l, rows, kept = q.get(timeout=5)
    assert err_o < 1e-12 and err_l < 1e-12
    assert all(r > 0 for r in rows)  # both ranks hold part of every session
    assert kept > 0                  # the slice of a shared context is still packed as shared


def test_context_slices_cover_each_token_once():
    from prefix_aware_decode_b200 import workload as wl
    from prefix_aware_decode_b200.shard import context_slices
    w = wl.make_config(3, with_values=False, scale=0.25)
    for world in (2, 3, 5):
        seen = {b: [] for b in range(w.B)}
        for reqs, bt, kl in context_slices(w.block_table, w.kv_lens, world):
            assert (kl > 0).all()
            for i, b in enumerate(reqs):
                n = (int(kl[i]) + 15) // 16
                seen[int(b)].extend(bt[i, :n].tolist())
                assert int(kl[i]) % 16 == 0 or seen[int(b)][-1] == w.block_table[b, (w.kv_lens[b] - 1) // 16]
        for b in range(w.B):
            n = (int(w.kv_lens[b]) + 15) // 16
            assert seen[b] == w.block_table[b, :n].tolist()


def test_two_rank_sharded_batch_matches_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    err_o, err_l, sizes = q.get(timeout=5)
    assert err_o < 1e-12 and err_l < 1e-12
    assert all(s > 0 for s in sizes)


def test_shard_by_root_keeps_subtrees_whole():
    from prefix_aware_decode_b200 import workload as wl
    from prefix_aware_decode_b200.shard import shard_by_root
    w = wl.make_config(3, with_values=False, scale=0.25)
    owned = shard_by_root(w.block_table, w.kv_lens, 4)
    roots = [set(w.block_table[o, 0].tolist()) for o in owned if len(o)]
    for i in range(len(roots)):
        for j in range(i + 1, len(roots)):
            assert not (roots[i] & roots[j])
    assert sorted(np.concatenate(owned).tolist()) == list(range(w.B))
    w5 = wl.make_config(5, with_values=False, scale=0.25)
    owned5 = shard_by_root(w5.block_table, w5.kv_lens, 4)
    loads = [int(w5.kv_lens[o].sum()) for o in owned5]
    assert max(loads) <= 2 * min(loads)
