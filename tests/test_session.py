"""Session page allocator (stateful sessions): page bookkeeping, forks, and the
decode batch of registered queries planned and executed against the oracle."""
import numpy as np
import pytest

import oracle
import prefix_aware_decode_b200 as pad
from prefix_aware_decode_b200.session import SessionPool

from plan_exec import Image, check_structure, execute

P, HKV, D, G = 16, 2, 64, 4


class Pools:
    """Numpy K/V pools written as the allocator says (the caller's side)."""

    def __init__(self, n_pages, seed):
        self.rng = np.random.default_rng(seed)
        self.k = np.full((n_pages, HKV, P, D), 0x7FC0, dtype=np.uint16)  # NaN until written
        self.v = self.k.copy()

    def bf(self, *shape):
        return (self.rng.normal(size=shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)

    def write(self, runs):
        for page, slot, n in runs:
            self.k[page, :, slot:slot + n] = self.bf(HKV, n, D)
            self.v[page, :, slot:slot + n] = self.bf(HKV, n, D)

    def copy(self, copies):
        for src, dst, n in copies:
            self.k[dst, :, :n] = self.k[src, :, :n]
            self.v[dst, :, :n] = self.v[src, :, :n]


def run_batch(pool, kv_pool, q_of, plan=None):
    qids, _, bt, kv = pool.batch()
    q = np.stack([q_of[i] for i in qids])
    if plan is None:
        # these sessions are small (tens of tokens): the profit model would
        # inline them, so sharing is forced to exercise the shared path
        plan = pad.Plan(kv, bt, pool.num_pages, G * HKV, HKV, D,
                        flags=pad.PA_PLAN_KEEP_PACK | pad.PA_PLAN_ALWAYS_SHARE)
    else:
        plan = plan.advance(kv, bt, pool.num_pages)
    img = Image(plan.host_image())
    check_structure(img, kv, bt, P)
    out, lse = execute(img, q, kv_pool.k, kv_pool.v)
    ref_o, ref_l = oracle.attend_paged(q, kv_pool.k, kv_pool.v, bt, kv)
    np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)
    return plan


def test_sessions_grow_fork_and_serve_their_registered_queries():
    pool = SessionPool(64, P)
    kvp = Pools(64, seed=1)
    rng = np.random.default_rng(2)
    q_of = {}
    # two sessions with contexts that end inside a page, a fork of the first
    for sid, n in ((0, 70), (1, 45)):
        pool.open(sid)
        kvp.write(pool.append(sid, n))
    kvp.copy(pool.fork(2, parent=0))
    kvp.write(pool.append(2, 9))  # the fork diverges after the parent's 70 tokens
    pool.check()
    assert pool.pages(2)[:4] == pool.pages(0)[:4] and pool.pages(2)[4] != pool.pages(0)[4]
    for sid, nq in ((0, 3), (1, 2), (2, 4)):
        for j in range(nq):
            qid = 10 * sid + j
            q_of[qid] = kvp.bf(G * HKV, D)
            pool.register(sid, qid)
    plan = run_batch(pool, kvp, q_of)
    st = plan.stats()
    assert st["num_kept_shared"] >= 1  # a session's full pages are one shared node
    # decode steps: data arrives for every session, the same queries are asked again
    for _ in range(6):
        for sid in (0, 1, 2):
            kvp.write(pool.append(sid, int(rng.integers(0, 20))))
        pool.check()
        plan = run_batch(pool, kvp, q_of, plan)
    # closing the parent frees the pages only it held; the fork keeps the shared ones
    before = pool.free_pages
    pages0, pages2 = set(pool.pages(0)), set(pool.pages(2))
    shared = pages0 & pages2
    assert shared
    pool.close(0)
    pool.check()
    assert pool.free_pages == before + len(pages0 - pages2)
    for p in shared:
        assert p in pool.pages(2)
    pool.close(1)
    pool.close(2)
    pool.check()
    assert pool.free_pages == 64


def test_allocator_accounting():
    pool = SessionPool(8, P)
    pool.open(0)
    assert pool.append(0, 40) == [(0, 0, 16), (1, 0, 16), (2, 0, 8)]
    assert pool.append(0, 10) == [(2, 8, 8), (3, 0, 2)]
    assert pool.tokens(0) == 50 and pool.free_pages == 4
    copies = pool.fork(1, parent=0)
    assert copies == [(3, 4, 2)]  # the partial last page is copied, full pages shared
    assert pool.pages(1) == [0, 1, 2, 4] and pool.free_pages == 3
    pool.check()
    pool.close(0)
    assert pool.free_pages == 4  # only page 3 was the parent's alone
    pool.close(1)
    assert pool.free_pages == 8
    pool.check()
    pool.open(5)
    with pytest.raises(MemoryError):
        pool.append(5, 9 * 16)
    with pytest.raises(KeyError):
        pool.open(5)
