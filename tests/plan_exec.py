"""CPU executor of a plan image (test utility; neither the oracle nor the product).

It reads the bytes pa_plan_upload would send (layout in include/pa.h), runs
every forward segment in fp64 with the oracle's dense attention, and merges each
(request, head)'s partial rows with the oracle's log-sum-exp merge.  It also
checks the plan's structure: every (request, kv head) reads each of its tokens
exactly once, every partial row is written once, and the SIMT tile list matches
the segments.
"""
import ctypes

import numpy as np

import oracle
from prefix_aware_decode_b200 import PaImageHeader
from prefix_aware_decode_b200 import workload as wl


class Image:
    def __init__(self, buf: np.ndarray):
        h = PaImageHeader.from_buffer_copy(buf[: ctypes.sizeof(PaImageHeader)].tobytes())
        assert h.magic == 0x50414231
        self.h = h

        def arr(off, n, dt=np.int32, cols=None):
            a = np.frombuffer(buf, dtype=dt, count=n * (cols or 1), offset=off)
            return a.reshape(n, cols) if cols else a

        self.items = arr(h.off_nodes, h.num_items, cols=4)  # page_off, n_tokens, n_queries, query_off
        segs8 = arr(h.off_segs, h.num_segments, cols=8)
        self.segs = segs8[:, :6]  # item, kv_head, page_begin, n_tokens, prow, query
        self.seg_sole = segs8[:, 6]
        self.seg_page_start = segs8[:, 7]
        n_pages = (h.off_queries - h.off_pages) // 4
        self.pages = arr(h.off_pages, n_pages)
        self.queries = arr(h.off_queries, (h.off_seg_prows - h.off_queries) // 4)
        self.seg_prows = arr(h.off_seg_prows, (h.off_mma_segs - h.off_seg_prows) // 4)
        self.mma_segs = arr(h.off_mma_segs, 2 if h.num_segments_mma else 1)
        self.counters = arr(h.off_counters, h.batch * h.num_kv_heads)
        self.warp_segs = arr(h.off_warp_segs, h.simt_warps + 1)
        self.prow_off = arr(h.off_prow_off, h.batch * h.num_kv_heads + 1)
        self.tail_pairs = arr(h.off_tail_pairs, h.num_tail_pairs)
        self.mix_pairs = arr(h.off_mix_pairs, h.num_mix_pairs, cols=2)


def check_structure(img: Image, kv_lens, block_table, P=16):
    h = img.h
    B, Hkv, G = h.batch, h.num_kv_heads, h.num_q_heads // h.num_kv_heads
    nseg_simt = h.num_segments_simt
    # the tensor-core work units form one list, longest first, taken by the
    # CTAs from the header's counter (zero after upload); arrival counters
    # start at zero
    if h.num_segments_mma:
        assert list(img.mma_segs) == [0, h.num_segments_mma]
        assert 1 <= h.mma_ctas <= h.num_segments_mma
        toks = img.segs[nseg_simt:, 3]
        assert np.all(np.diff(toks) <= 0)
    else:
        assert h.mma_ctas == 0
    assert h.mma_next == 0
    assert np.all(img.counters == 0)
    # small-row launch: 8 warps per CTA, or 6 when its warps stream long runs
    assert h.simt_warps_per_cta in (6, 8)
    # pairs with tensor-core rows; the tail list holds those without SIMT rows, ascending
    mma_pairs, simt_rows = set(), {}
    for si in range(nseg_simt, h.num_segments):
        item, g, pb, nt, prow, q = img.segs[si]
        po, itok, nq, qo = img.items[item]
        mma_pairs.update(int(b) * Hkv + int(g) for b in img.queries[qo: qo + nq])
    for si in range(nseg_simt):
        item, g, pb, nt, prow, q = img.segs[si]
        bg = int(q) * Hkv + int(g)
        simt_rows[bg] = simt_rows.get(bg, 0) + 1
    modes = {int(m) & 3 for m in img.seg_sole[:nseg_simt]}
    mixed_to_tail = 3 in modes
    assert not (mixed_to_tail and 2 in modes)
    mixed = sorted(bg for bg in mma_pairs if bg in simt_rows)
    assert list(img.tail_pairs) == sorted(bg for bg in mma_pairs if mixed_to_tail or bg not in simt_rows)
    # the mixed pairs (both classes' rows) not sent to the tail launch: each in
    # exactly one mix_pairs entry with its SIMT row count, at most 3 per warp
    # (entry k belongs to warp k mod W), other entries empty
    if mixed_to_tail:
        assert h.num_mix_pairs == 0 and len(mixed) > 3 * h.simt_warps
    else:
        got = [(int(bg), int(n)) for bg, n in img.mix_pairs if bg >= 0]
        assert sorted(got) == [(bg, simt_rows[bg]) for bg in mixed]
        assert all(int(bg) == -1 and int(n) == -1 for bg, n in img.mix_pairs if bg < 0)
        per_warp = np.bincount([k % max(1, h.simt_warps) for k in range(h.num_mix_pairs) if img.mix_pairs[k, 0] >= 0],
                               minlength=max(1, h.simt_warps))
        assert per_warp.max(initial=0) <= 3
    # warp lists partition the SIMT segments, in order; page_start and the
    # combine mode (tail merge, sole row or arrival counted) are consistent
    assert img.warp_segs[0] == 0 and img.warp_segs[-1] == nseg_simt
    assert np.all(np.diff(img.warp_segs) > 0) or nseg_simt == 0
    for si in range(h.num_segments):
        item, g, pb, nt, prow, q = img.segs[si]
        assert img.seg_page_start[si] == img.items[item][0] + pb
        if si < nseg_simt:
            n_rows = img.prow_off[q * Hkv + g + 1] - img.prow_off[q * Hkv + g]
            bg = int(q) * Hkv + int(g)
            want = (3 if mixed_to_tail else 2) if bg in mma_pairs else (1 if n_rows == 1 else 0)
            assert img.seg_sole[si] & 3 == want
            assert img.seg_sole[si] >> 2 == simt_rows[bg]
        else:
            # a tensor-core unit names its item's request list itself
            assert q == img.items[item][3] and img.seg_sole[si] == img.items[item][2]
    # coverage: each (request, kv head) reads each token (page, slot) exactly once
    seen = {}
    prows_written = np.zeros(h.num_partial_rows, dtype=np.int64)
    for si in range(h.num_segments):
        item, g, pb, nt, prow, q0 = img.segs[si]
        po, itok, nq, qo = img.items[item]
        assert 1 <= nt and pb * P + nt <= itok
        qs = img.queries[qo: qo + nq]
        if si < nseg_simt:
            prs = [prow]
        else:
            prs = img.seg_prows[prow: prow + nq]
        for b, pr in zip(qs, prs):
            assert img.prow_off[b * Hkv + g] <= pr < img.prow_off[b * Hkv + g + 1]
            prows_written[pr] += 1
            for tok in range(pb * P, pb * P + nt):
                key = (int(b), int(g), int(img.pages[po + tok // P]), tok % P)
                seen[key] = seen.get(key, 0) + 1
    assert np.all(prows_written == 1)
    assert all(v == 1 for v in seen.values())
    for b in range(B):
        n = int(kv_lens[b])
        for g in range(Hkv):
            for tok in range(n):
                assert seen.get((b, g, int(block_table[b, tok // P]), tok % P)) == 1, (b, g, tok)
    assert len(seen) == int(np.sum(kv_lens)) * Hkv


def execute(img: Image, q, k_pool, v_pool, scale=None, P=16):
    """Run the plan in fp64: returns (out[B][Hq][D], lse[B][Hq])."""
    h = img.h
    B, Hq, Hkv, D = h.batch, h.num_q_heads, h.num_kv_heads, h.head_dim
    G = Hq // Hkv
    po_ = np.zeros((h.num_partial_rows, G, D))
    pl_ = np.full((h.num_partial_rows, G), -np.inf)
    kf = wl.bf16_bits_to_f32(k_pool).astype(np.float64)
    vf = wl.bf16_bits_to_f32(v_pool).astype(np.float64)
    qf = wl.bf16_bits_to_f32(q).astype(np.float64)
    for si in range(h.num_segments):
        item, g, pb, nt, prow, q0 = img.segs[si]
        po, itok, nq, qo = img.items[item]
        toks = np.arange(pb * P, pb * P + nt)
        pg = img.pages[po + toks // P]
        K = kf[pg, g, toks % P]
        V = vf[pg, g, toks % P]
        qs = img.queries[qo: qo + nq]
        prs = [prow] if si < h.num_segments_simt else img.seg_prows[prow: prow + nq]
        for b, pr in zip(qs, prs):
            for r in range(G):
                o, l = oracle.attend_dense(qf[b, g * G + r], K, V, scale)
                po_[pr, r] = o
                pl_[pr, r] = l
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for hh in range(Hq):
            g, r = hh // G, hh % G
            a, e = img.prow_off[b * Hkv + g], img.prow_off[b * Hkv + g + 1]
            out[b, hh], lse[b, hh] = oracle.merge(po_[a:e, r], pl_[a:e, r])
    return out, lse
