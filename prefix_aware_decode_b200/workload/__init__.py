"""Seeded synthetic decode-attention workloads.

This module only builds inputs: the prefix tree of each batch, the paged K/V
pools, the block tables and the queries.  It holds no attention arithmetic; the
fp64 oracle and the CUDA path both read what it produces.

Workload shapes follow the PAT review ("PAT: Accelerating LLM Decoding via
Prefix-Aware Attention", section 三, Figure 4 and Figure 5: hierarchical shared
prefixes such as system prompt -> tool/template -> per-request suffix) and the
stateful-streaming summary ("Attention Once Is All You Need", 方法拆解: a
persistent session context probed by registered queries).  The paged layout
follows PagedAttention as described on the short-term-memory page
(长上下文的关键技术栈, PagedAttention 与 vLLM) and its KV-append rule
(技术原理: K_t, V_t are appended before attending), so every request's own
token is the last entry of its KV.

Layouts (all little-endian, C-contiguous):
  q        uint16 (bf16 bits) [B][Hq][D]
  k_pool   uint16 (bf16 bits) [num_pages][Hkv][P][D]   (same for v_pool)
  block_table int32 [B][max_pages], unused entries -1
  kv_lens  int32 [B]

Random values: SplitMix64-seeded xoshiro256** streams with Box-Muller normals
(gen.c).  Each physical page is its own stream keyed by its page id.  Unused
pages and the slots past kv_len in a request's last page hold bf16 NaN
(0x7FC0) so that any read outside the valid KV shows up in the output.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

PAGE_SIZE = 16
BF16_NAN = 0x7FC0

TAG_K, TAG_V, TAG_Q, TAG_LEN, TAG_PERM, TAG_TAIL_K, TAG_TAIL_V = 1, 2, 3, 4, 5, 6, 7

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libpagen.so")
_lib = None


def build_generator(force: bool = False) -> str:
    """Compile gen.c into libpagen.so next to it (gcc, -O2)."""
    import subprocess

    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        tmp = _LIB_PATH + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", src,
                               "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _gen():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            build_generator()
        lib = ctypes.CDLL(_LIB_PATH)
        u64, i64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        lib.pagen_u64.argtypes = [u64, u64, u64, i64, vp]
        lib.pagen_unit.argtypes = [u64, u64, u64, i64, vp]
        lib.pagen_normal_f64.argtypes = [u64, u64, u64, i64, vp]
        lib.pagen_normal_bf16.argtypes = [u64, u64, u64, i64, vp]
        lib.pagen_permutation.argtypes = [u64, u64, i64, vp]
        lib.pagen_fill_pages.argtypes = [u64, u64, vp, i64, i64, vp, ctypes.c_int]
        lib.pagen_fill_u16.argtypes = [vp, i64, ctypes.c_uint16]
        for f in (lib.pagen_u64, lib.pagen_unit, lib.pagen_normal_f64, lib.pagen_normal_bf16,
                  lib.pagen_permutation, lib.pagen_fill_pages, lib.pagen_fill_u16):
            f.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def unit_stream(seed: int, tag: int, index: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _gen().pagen_unit(seed, tag, index, n, _ptr(out))
    return out


def normal_stream(seed: int, tag: int, index: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _gen().pagen_normal_f64(seed, tag, index, n, _ptr(out))
    return out


def normal_bf16(seed: int, tag: int, index: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    _gen().pagen_normal_bf16(seed, tag, index, n, _ptr(out))
    return out


def permutation(seed: int, tag: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _gen().pagen_permutation(seed, tag, n, _ptr(out))
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


class Uniform:
    """Sequential uniform draws from one stream, consumed in a fixed order."""

    def __init__(self, seed: int, tag: int, index: int = 0, block: int = 4096):
        self.seed, self.tag, self.index, self.block = seed, tag, index, block
        self.buf = np.empty(0)
        self.pos = 0
        self.drawn = 0

    def unit(self) -> float:
        if self.pos >= len(self.buf):
            # one long stream: regenerate it with a larger prefix and skip what was used
            self.buf = unit_stream(self.seed, self.tag, self.index, self.drawn + self.block)[self.drawn:]
            self.pos = 0
        self.pos += 1
        self.drawn += 1
        return float(self.buf[self.pos - 1])

    def randint(self, lo: int, hi: int) -> int:
        """Integer uniform on the inclusive range [lo, hi]."""
        v = lo + int(self.unit() * (hi - lo + 1))
        return min(v, hi)


@dataclass
class Node:
    """One node of a request prefix tree: a run of tokens, stored in its own pages.

    `length` counts tokens.  A node with children is shared by all requests below
    it and must hold whole pages.  A leaf belongs to exactly one request, and its
    last token is that request's own (appended) token.  `cow_tail`, when set on a
    leaf, is (session id, r): the leaf's first r tokens are copies of that
    session's tail tokens (copy-on-write of a partial last page).
    """

    length: int
    children: List["Node"] = field(default_factory=list)
    cow_tail: Optional[tuple] = None
    query: int = -1  # filled in for leaves
    pages: Optional[np.ndarray] = None


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    P: int
    seed: int
    kv_lens: np.ndarray
    block_table: np.ndarray
    num_pages: int
    q: np.ndarray
    k_pool: np.ndarray
    v_pool: np.ndarray
    unique_tokens: int
    roots: list = field(repr=False, default_factory=list)

    @property
    def naive_tokens(self) -> int:
        return int(self.kv_lens.sum())

    @property
    def kv_bytes_per_token(self) -> int:
        return 2 * self.Hkv * self.D * 2

    @property
    def unique_kv_bytes(self) -> int:
        return self.unique_tokens * self.kv_bytes_per_token

    @property
    def prefix_ratio(self) -> float:
        """Share of request KV tokens that lie in nodes shared by more than one request."""
        shared = 0

        def walk(n: Node, nreq: int):
            nonlocal shared
            cnt = _count_leaves(n)
            if cnt > 1:
                shared += n.length * cnt
            for c in n.children:
                walk(c, cnt)

        for r in self.roots:
            walk(r, 0)
        return shared / max(1, self.naive_tokens)

    def describe(self) -> dict:
        return dict(name=self.name, B=self.B, Hq=self.Hq, Hkv=self.Hkv, D=self.D, P=self.P,
                    seed=self.seed, num_pages=self.num_pages, unique_tokens=self.unique_tokens,
                    naive_tokens=self.naive_tokens, unique_kv_bytes=self.unique_kv_bytes,
                    prefix_ratio=round(self.prefix_ratio, 4))


def _count_leaves(n: Node) -> int:
    if not n.children:
        return 1
    return sum(_count_leaves(c) for c in n.children)


def _leaves(n: Node) -> List[Node]:
    if not n.children:
        return [n]
    out = []
    for c in n.children:
        out.extend(_leaves(c))
    return out


def build_workload(name: str, roots: List[Node], Hq: int, Hkv: int, D: int, seed: int,
                   P: int = PAGE_SIZE, spare_frac: float = 0.05, nthreads: Optional[int] = None,
                   with_values: bool = True) -> Workload:
    """Lay a prefix forest out in a paged pool and draw its values.

    Pages are drawn from a seeded random permutation of the pool, so a request's
    pages are scattered like a real paged cache.  The pool holds ceil(5%) spare,
    NaN-filled pages beyond the used ones.
    """
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    # assign queries in leaf order
    leaves: List[Node] = []
    for r in roots:
        leaves.extend(_leaves(r))
    B = len(leaves)
    for i, lf in enumerate(leaves):
        lf.query = i

    def node_pages(n: Node) -> int:
        return -(-n.length // P)

    def check(n: Node, depth_tokens: int):
        if n.children:
            if n.length % P != 0:
                raise ValueError("a shared node must hold whole pages")
            for c in n.children:
                check(c, depth_tokens + n.length)
        elif n.length < 1 and depth_tokens < 1:
            raise ValueError("every request needs at least one token")

    for r in roots:
        check(r, 0)

    # DFS order of nodes for page assignment
    order: List[Node] = []

    def dfs(n: Node):
        order.append(n)
        for c in n.children:
            dfs(c)

    for r in roots:
        dfs(r)
    used = sum(node_pages(n) for n in order)
    num_pages = used + max(1, math.ceil(spare_frac * used))
    perm = permutation(seed, TAG_PERM, num_pages)
    cursor = 0
    for n in order:
        k = node_pages(n)
        n.pages = perm[cursor:cursor + k].copy()
        cursor += k
    spare = perm[cursor:]

    # block tables
    paths = []

    def collect(n: Node, prefix: list):
        cur = prefix + [n]
        if not n.children:
            paths.append(cur)
        for c in n.children:
            collect(c, cur)

    for r in roots:
        collect(r, [])
    kv_lens = np.zeros(B, dtype=np.int32)
    tables = []
    for path in paths:
        b = path[-1].query
        kv_lens[b] = sum(n.length for n in path)
        tables.append((b, np.concatenate([n.pages for n in path if len(n.pages)])))
    max_pages = max(len(t) for _, t in tables)
    block_table = np.full((B, max_pages), -1, dtype=np.int32)
    for b, t in tables:
        block_table[b, :len(t)] = t
    unique_tokens = int(sum(n.length for n in order))

    elems = Hkv * P * D
    if with_values:
        k_pool = np.empty((num_pages, Hkv, P, D), dtype=np.uint16)
        v_pool = np.empty((num_pages, Hkv, P, D), dtype=np.uint16)
        used_ids = perm[:cursor].copy()
        g = _gen()
        g.pagen_fill_pages(seed, TAG_K, _ptr(used_ids), len(used_ids), elems, _ptr(k_pool), nthreads)
        g.pagen_fill_pages(seed, TAG_V, _ptr(used_ids), len(used_ids), elems, _ptr(v_pool), nthreads)
        for p in spare:
            k_pool[p] = BF16_NAN
            v_pool[p] = BF16_NAN
        for lf in leaves:
            if lf.cow_tail is not None:
                sess, r = lf.cow_tail
                if r > 0:
                    tk = normal_bf16(seed, TAG_TAIL_K, sess, Hkv * r * D).reshape(Hkv, r, D)
                    tv = normal_bf16(seed, TAG_TAIL_V, sess, Hkv * r * D).reshape(Hkv, r, D)
                    k_pool[lf.pages[0], :, :r, :] = tk
                    v_pool[lf.pages[0], :, :r, :] = tv
            tail = lf.length % P
            if tail and len(lf.pages):
                k_pool[lf.pages[-1], :, tail:, :] = BF16_NAN
                v_pool[lf.pages[-1], :, tail:, :] = BF16_NAN
        q = np.empty((B, Hq, D), dtype=np.uint16)
        for b in range(B):
            q[b] = normal_bf16(seed, TAG_Q, b, Hq * D).reshape(Hq, D)
    else:
        k_pool = v_pool = q = None
    return Workload(name=name, B=B, Hq=Hq, Hkv=Hkv, D=D, P=P, seed=seed, kv_lens=kv_lens,
                    block_table=block_table, num_pages=num_pages, q=q, k_pool=k_pool, v_pool=v_pool,
                    unique_tokens=unique_tokens, roots=roots)


# ----------------------------------------------------------------- the five configs

CONFIG_NAMES = {
    1: "tiny GQA decode: B=4, 8/2 heads, D=64, shared 256 + suffix U[16,64]",
    2: "Llama-3-8B-shaped decode layer: B=64, 32/8 heads, D=128, shared 2048 + suffix U[128,1024]",
    3: "3-level prefix tree: root 4096 -> 8 x 1024 -> 32 leaves U[64,2048] each, B=256, 32/8, D=128",
    4: "no sharing, skewed: B=128, lognormal(median 2048, sigma 1) clipped [32,32768], 32/8, D=128",
    5: "stateful sessions: 32 x context U[32768,131072] x 16 single-token queries, B=512, 32/8, D=128",
}


def config1_stream(n: int, seed: int = 1001, with_values: bool = True) -> "Workload":
    """n independent problems shaped like config 1 (each: one shared 256-token
    prefix and 4 suffixes uniform 16-64 tokens, 8/2 heads, D 64) in one batch of
    4n requests: the amortised form of config 1, whose single instance is too
    small to leave the launch latency."""
    u = Uniform(seed, TAG_LEN)
    roots = [Node(256, [Node(u.randint(16, 64)) for _ in range(4)]) for _ in range(n)]
    return build_workload(f"config 1 x {n}", roots, 8, 2, 64, seed, with_values=with_values)


def session_chunks(ctx_lens, chunk_lens, Hq: int, Hkv: int, D: int, seed: int):
    """Sessions that each append a chunk of new tokens (the prefix-aware
    grouped prefill of stateful sessions): session s holds ctx_lens[s] context
    tokens followed by its chunk_lens[s] new tokens, all already in the paged
    pool (append, then attend).  Returns (workload, q_rows): the workload's
    request s is session s over all its tokens; q_rows uint16 [sum chunk][Hq][D]
    are the new tokens' queries, sessions in order, each chunk in token order."""
    roots = [Node(int(c) + int(n)) for c, n in zip(ctx_lens, chunk_lens)]
    w = build_workload("chunks", roots, Hq, Hkv, D, seed)
    rows = int(np.sum(chunk_lens))
    q = np.empty((rows, Hq, D), dtype=np.uint16)
    for r in range(rows):
        q[r] = normal_bf16(seed, TAG_Q, 1 << 20 | r, Hq * D).reshape(Hq, D)
    return w, q


def config_tree(config: int, seed: int, scale: float = 1.0):
    """Return (roots, Hq, Hkv, D) for one of the five configs.

    `scale` < 1 shrinks batch sizes / lengths proportionally (used only for quick
    CPU tests; the named configs use scale 1).
    """
    u = Uniform(seed, TAG_LEN)
    if config == 1:
        leaves = [Node(u.randint(16, 64)) for _ in range(4)]
        return [Node(256, leaves)], 8, 2, 64
    if config == 2:
        B = max(1, int(round(64 * scale)))
        leaves = [Node(u.randint(128, 1024)) for _ in range(B)]
        return [Node(2048, leaves)], 32, 8, 128
    if config == 3:
        nb = 8
        per = max(1, int(round(32 * scale)))
        branches = [Node(1024, [Node(u.randint(64, 2048)) for _ in range(per)]) for _ in range(nb)]
        return [Node(4096, branches)], 32, 8, 128
    if config == 4:
        B = max(1, int(round(128 * scale)))
        z = normal_stream(seed, TAG_LEN, 1, B)
        lens = np.floor(np.clip(2048.0 * np.exp(1.0 * z), 32, 32768) + 0.5).astype(int)
        return [Node(int(n)) for n in lens], 32, 8, 128
    if config == 5:
        S = max(1, int(round(32 * scale)))
        roots = []
        for s in range(S):
            L = u.randint(32768, 131072)
            if scale < 1.0:
                L = max(P_ALIGN, int(L * scale))
            full = (L // PAGE_SIZE) * PAGE_SIZE
            r = L - full
            leaves = [Node(r + 1, cow_tail=(s, r)) for _ in range(16)]
            roots.append(Node(full, leaves))
        return roots, 32, 8, 128
    raise ValueError(f"unknown config {config}")


P_ALIGN = 64


def make_config(config: int, seed: Optional[int] = None, scale: float = 1.0,
                nthreads: Optional[int] = None, with_values: bool = True) -> Workload:
    """Build config 1..5 with its default seed 1000 + config."""
    if seed is None:
        seed = 1000 + config
    roots, Hq, Hkv, D = config_tree(config, seed, scale)
    name = f"config{config}" + ("" if scale == 1.0 else f"@{scale:g}")
    return build_workload(name, roots, Hq, Hkv, D, seed, nthreads=nthreads, with_values=with_values)


def random_tree(seed: int, n_queries: int, depth: int = 2, shared_pages=(1, 8), leaf_tokens=(1, 80),
                fanout=(1, 4)) -> List[Node]:
    """A small random prefix forest for tests: shared nodes of whole pages, ragged leaves."""
    u = Uniform(seed, TAG_LEN, 7)
    remaining = [n_queries]

    def make(level: int) -> Node:
        if level >= depth or remaining[0] <= 1:
            remaining[0] -= 1
            return Node(u.randint(*leaf_tokens))
        k = min(remaining[0], u.randint(*fanout))
        kids = []
        for _ in range(k):
            if remaining[0] <= 0:
                break
            kids.append(make(level + 1))
        if not kids:
            remaining[0] -= 1
            return Node(u.randint(*leaf_tokens))
        return Node(PAGE_SIZE * u.randint(*shared_pages), kids)

    roots = []
    while remaining[0] > 0:
        roots.append(make(0))
    return roots
