"""Persistent paged KV for stateful sessions (host bookkeeping).

"Attention Once Is All You Need" keeps a session's KV cache alive across
queries and advances it as data arrives, so a query only pays for itself; its
registered questions ("Flash Queries") are evaluated against the live session.
This module is the page allocator behind that workload: it owns the page ids
of one pool, grows sessions token by token, forks a session off another's
prefix (full pages are shared by reference, a partial last page is copied), and
builds the decode batch of every registered query for the planner
(pa_plan_create, or pa_plan_advance between steps, since a session only grows).

It moves no data: appends and forks return the page slots the caller writes
new K/V into, and the page copies a fork needs; the device pools stay the
caller's.  Shared pages are reference-counted and go back to the free list
when no session holds them.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import numpy as np


@dataclass
class _Session:
    pages: List[int] = field(default_factory=list)
    n_tokens: int = 0
    queries: List[int] = field(default_factory=list)  # registered query ids


class SessionPool:
    """Page allocator of one paged KV pool shared by many sessions."""

    def __init__(self, num_pages: int, page_size: int = 16):
        if num_pages < 1 or page_size < 1:
            raise ValueError("num_pages and page_size must be positive")
        self.num_pages = int(num_pages)
        self.P = int(page_size)
        self._free = list(range(self.num_pages - 1, -1, -1))  # pop() gives the lowest id
        self._ref = np.zeros(self.num_pages, dtype=np.int64)
        self._sessions: Dict[int, _Session] = {}

    # ------------------------------------------------------------ pages
    @property
    def free_pages(self) -> int:
        return len(self._free)

    def _take(self) -> int:
        if not self._free:
            raise MemoryError("KV pool has no free page")
        p = self._free.pop()
        self._ref[p] = 1
        return p

    def _drop(self, p: int):
        self._ref[p] -= 1
        if self._ref[p] == 0:
            self._free.append(p)
        elif self._ref[p] < 0:
            raise RuntimeError(f"page {p} released more often than held")

    # ------------------------------------------------------------ sessions
    def open(self, sid: int):
        if sid in self._sessions:
            raise KeyError(f"session {sid} exists")
        self._sessions[sid] = _Session()

    def fork(self, sid: int, parent: int) -> List[Tuple[int, int, int]]:
        """New session `sid` holding parent's whole KV.  Full pages are shared;
        a partial last page is copied into a page of the new session's own.
        Returns the copies to make: (src_page, dst_page, tokens)."""
        if sid in self._sessions:
            raise KeyError(f"session {sid} exists")
        par = self._sessions[parent]
        s = _Session(n_tokens=par.n_tokens)
        full = par.n_tokens // self.P
        copies = []
        for p in par.pages[:full]:
            self._ref[p] += 1
            s.pages.append(p)
        rest = par.n_tokens - full * self.P
        if rest:
            dst = self._take()
            s.pages.append(dst)
            copies.append((par.pages[full], dst, rest))
        self._sessions[sid] = s
        return copies

    def append(self, sid: int, n_tokens: int) -> List[Tuple[int, int, int]]:
        """Grows session `sid` by n_tokens.  Returns where their K/V go, as
        (page, first slot, slot count) runs in token order.  A shared last
        page is never written: a session that shares its partial last page is
        impossible (forks copy it), and full pages take no new tokens."""
        if n_tokens < 0:
            raise ValueError("n_tokens must be >= 0")
        s = self._sessions[sid]
        runs = []
        left = n_tokens
        while left > 0:
            slot = s.n_tokens % self.P
            if slot == 0:
                s.pages.append(self._take())
            page = s.pages[-1]
            if self._ref[page] != 1:
                raise RuntimeError("a partial page is shared")
            take = min(left, self.P - slot)
            runs.append((page, slot, take))
            s.n_tokens += take
            left -= take
        return runs

    def close(self, sid: int):
        s = self._sessions.pop(sid)
        for p in s.pages:
            self._drop(p)

    def register(self, sid: int, qid: int):
        """A query (one decode token) of session `sid` to be evaluated at every step."""
        self._sessions[sid].queries.append(int(qid))

    def unregister(self, sid: int, qid: int):
        self._sessions[sid].queries.remove(int(qid))

    def tokens(self, sid: int) -> int:
        return self._sessions[sid].n_tokens

    def pages(self, sid: int) -> List[int]:
        return list(self._sessions[sid].pages)

    # ------------------------------------------------------------ batches
    def batch(self, sessions=None):
        """The decode batch of every registered query: one request per query
        over its session's whole KV.  Returns (query ids, session of each
        request, block_table int32 [B][max_pages] with -1 past the pages,
        kv_lens int32 [B]).  Queries of one session share all of its pages, so
        the planner packs the session as one shared node."""
        sids = sorted(self._sessions) if sessions is None else list(sessions)
        rows = [(sid, q) for sid in sids for q in self._sessions[sid].queries if self._sessions[sid].n_tokens > 0]
        B = len(rows)
        width = max([len(self._sessions[sid].pages) for sid, _ in rows] + [1])
        bt = np.full((B, width), -1, dtype=np.int32)
        kv = np.zeros(B, dtype=np.int32)
        for i, (sid, _) in enumerate(rows):
            s = self._sessions[sid]
            bt[i, :len(s.pages)] = s.pages
            kv[i] = s.n_tokens
        return [q for _, q in rows], [sid for sid, _ in rows], bt, kv

    def check(self):
        """Invariants: every held page is referenced once per session holding
        it, free pages are unreferenced and each listed once."""
        count = np.zeros(self.num_pages, dtype=np.int64)
        for s in self._sessions.values():
            if len(s.pages) != -(-s.n_tokens // self.P):
                raise AssertionError("page count does not match the token count")
            for p in s.pages:
                count[p] += 1
        if not np.array_equal(count, self._ref):
            raise AssertionError("reference counts differ from the sessions' pages")
        free = np.array(self._free, dtype=np.int64)
        if len(set(self._free)) != len(self._free) or (self._ref[free] != 0).any():
            raise AssertionError("free list broken")
        if len(self._free) + int((self._ref > 0).sum()) != self.num_pages:
            raise AssertionError("pages lost")
