"""Stateful sessions on the GPU, through the C ABI against the fp64 oracle.

- Chunk append (prefix-aware grouped prefill): each session appends a chunk of
  new tokens; every new token attends over the context and the chunk up to
  itself (pa_plan_create_append).  Chunks of 1, 5, 16 and 19 tokens, G in
  {1, 4, 8}, D in {64, 128}.
- Registered queries against live sessions: sessions grow and fork over
  several steps (session.SessionPool), their registered queries are batched at
  every step and planned by pa_plan_advance while the batch keeps its
  requests (pa_plan_create after a fork or a new registration).
Tolerances as in test_gpu_parity (gpu_util).
"""
import numpy as np
import pytest
import torch

import oracle
import prefix_aware_decode_b200 as pad
from prefix_aware_decode_b200 import workload as wl
from prefix_aware_decode_b200.session import SessionPool

from gpu_util import assert_close, bf16_dev, compare

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_chunk_append_matches_the_oracle_rows(G, D):
    ctx = np.array([0, 37, 48, 1000, 2333, 4096], dtype=np.int32)
    chunk = np.array([5, 19, 1, 16, 19, 16], dtype=np.int32)
    Hkv = 8 if D == 128 else 2
    w, q = wl.session_chunks(ctx, chunk, Hq=G * Hkv, Hkv=Hkv, D=D, seed=100 * G + D)
    row_req = np.repeat(np.arange(len(ctx)), chunk)
    row_pos = np.concatenate([c + np.arange(n) for c, n in zip(ctx, chunk)])
    ref_o, ref_l = oracle.attend_rows(q, row_req, row_pos, w.k_pool, w.v_pool, w.block_table)
    qd, kd, vd = bf16_dev(q), bf16_dev(w.k_pool), bf16_dev(w.v_pool)
    for fused in (False, True):
        plan = pad.Plan.append(ctx, chunk, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
        st = plan.stats()
        assert st["batch"] == len(row_req) and st["num_kept_shared"] >= 1
        ws = plan.alloc_workspace()
        out = torch.empty((len(row_req), w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((len(row_req), w.Hq), dtype=torch.float32, device="cuda")
        plan.upload(ws)
        if fused:
            plan.attend(qd, kd, vd, ws, out, lse)
        else:
            plan.forward(qd, kd, vd, ws)
            plan.merge(ws, out, lse)
        assert plan.device_status(ws) == pad.PA_OK
        assert_close(compare(out, lse, ref_o, ref_l), f"append G={G} D={D} fused={fused}")
        plan.close()


class DevPools:
    """K/V pools of a SessionPool: host copies written as the allocator says,
    mirrored to the device before each step."""

    def __init__(self, n_pages, Hkv, D, seed):
        self.rng = np.random.default_rng(seed)
        self.Hkv, self.D = Hkv, D
        self.k = np.full((n_pages, Hkv, 16, D), wl.BF16_NAN, dtype=np.uint16)
        self.v = self.k.copy()

    def bf(self, *shape):
        return (self.rng.normal(size=shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)

    def write(self, runs):
        for page, slot, n in runs:
            self.k[page, :, slot:slot + n] = self.bf(self.Hkv, n, self.D)
            self.v[page, :, slot:slot + n] = self.bf(self.Hkv, n, self.D)

    def copy(self, copies):
        for src, dst, n in copies:
            self.k[dst, :, :n] = self.k[src, :, :n]
            self.v[dst, :, :n] = self.v[src, :, :n]


def test_registered_queries_against_growing_sessions():
    Hkv, D, G = 8, 128, 4
    n_pages = 4096
    pool = SessionPool(n_pages, 16)
    kvp = DevPools(n_pages, Hkv, D, seed=7)
    rng = np.random.default_rng(8)
    q_of = {}

    def register(sid, n):
        for _ in range(n):
            qid = len(q_of)
            q_of[qid] = kvp.bf(G * Hkv, D)
            pool.register(sid, qid)

    for sid, n in ((0, 3000), (1, 1500), (2, 777)):
        pool.open(sid)
        kvp.write(pool.append(sid, n))
        register(sid, 16 if sid == 0 else 4)
    plan, prev_reqs = None, None
    for step in range(8):
        if step == 3:  # a fork of session 0 with queries of its own: the batch changes
            kvp.copy(pool.fork(3, parent=0))
            register(3, 8)
        for sid in sorted(pool._sessions):
            kvp.write(pool.append(sid, int(rng.integers(1, 300))))
        pool.check()
        qids, sids, bt, kv = pool.batch()
        reqs = list(zip(qids, sids))
        if plan is not None and reqs == prev_reqs:
            nxt = plan.advance(kv, bt, n_pages)
            plan.close()
            plan = nxt
        else:
            if plan is not None:
                plan.close()
            plan = pad.Plan(kv, bt, n_pages, G * Hkv, Hkv, D, flags=pad.PA_PLAN_KEEP_PACK)
        prev_reqs = reqs
        q = np.stack([q_of[i] for i in qids])
        qd, kd, vd = bf16_dev(q), bf16_dev(kvp.k), bf16_dev(kvp.v)
        ws = plan.alloc_workspace()
        out = torch.empty((len(qids), G * Hkv, D), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((len(qids), G * Hkv), dtype=torch.float32, device="cuda")
        plan.upload(ws)
        plan.attend(qd, kd, vd, ws, out, lse)
        assert plan.device_status(ws) == pad.PA_OK
        ref_o, ref_l = oracle.attend_paged(q, kvp.k, kvp.v, bt, kv)
        assert_close(compare(out, lse, ref_o, ref_l), f"live sessions step {step}")
    assert plan.stats()["num_kept_shared"] >= 1
    plan.close()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_slices_merged_on_the_device(world):
    # long sessions (config-5 shaped, 4 sessions x 16 queries): the batch's
    # pages cut into `world` page-aligned slices (one per rank), each slice
    # planned and run on its own with an fp32 result (pa_merge_f32), the rows
    # stacked as an all-gather would deliver them, and merged by pa_merge_rows
    from prefix_aware_decode_b200.shard import context_slices

    w = wl.make_config(5, scale=0.125)
    qd, kd, vd = bf16_dev(w.q), bf16_dev(w.k_pool), bf16_dev(w.v_pool)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    parts = context_slices(w.block_table, w.kv_lens, world)
    R = max(len(reqs) for reqs, _, _ in parts)
    all_req = torch.full((world, R), -1, dtype=torch.int32, device="cuda")
    all_o = torch.zeros((world, R, w.Hq, w.D), dtype=torch.float32, device="cuda")
    all_l = torch.full((world, R, w.Hq), float("-inf"), dtype=torch.float32, device="cuda")
    for r, (reqs, bt, kl) in enumerate(parts):
        plan = pad.Plan(kl, bt, w.num_pages, w.Hq, w.Hkv, w.D)
        assert plan.stats()["num_kept_shared"] >= 1  # each slice of a session is still packed as shared
        ws = plan.alloc_workspace()
        qr = qd[torch.as_tensor(reqs, device="cuda")].contiguous()
        plan.upload(ws)
        plan.forward(qr, kd, vd, ws)
        o32 = torch.empty((len(reqs), w.Hq, w.D), dtype=torch.float32, device="cuda")
        l32 = torch.empty((len(reqs), w.Hq), dtype=torch.float32, device="cuda")
        plan.merge_f32(ws, o32, l32)
        # the fp32 result rounds to exactly what the bf16 merge writes
        o16 = torch.empty((len(reqs), w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
        l16 = torch.empty_like(l32)
        plan.merge(ws, o16, l16)
        assert plan.device_status(ws) == pad.PA_OK
        assert torch.equal(o32.to(torch.bfloat16).view(torch.int16), o16.view(torch.int16))
        assert torch.equal(l32, l16)
        all_req[r, :len(reqs)] = torch.as_tensor(reqs, dtype=torch.int32, device="cuda")
        all_o[r, :len(reqs)] = o32
        all_l[r, :len(reqs)] = l32
        plan.close()
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    pad.merge_rows(all_req, all_o, all_l, w.B, out, lse)
    torch.cuda.synchronize()
    assert_close(compare(out, lse, ref_o, ref_l), f"context parallel, {world} slices")
