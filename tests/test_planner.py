"""Pack stage on the host: tree structure, coverage, validation, and the plan
executed on the CPU (fp64) against the oracle."""
import numpy as np
import pytest

import oracle
import prefix_aware_decode_b200 as pad
from prefix_aware_decode_b200 import workload as wl

from plan_exec import Image, check_structure, execute


def make_plan(w, **kw):
    return pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D, **kw)


def test_exports_match_header(repo_root):
    import ctypes
    import os
    import re
    hdr = open(os.path.join(repo_root, "include", "pa.h")).read()
    declared = re.findall(r"^\s*(?:pa_status|void|const char \*)\s*(pa_\w+)\s*\(", hdr, re.M)
    assert declared, "no declarations found"
    L = pad.lib()
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) <= set(pad._binding.EXPORTS) | {"pa_plan_stats"}
    assert ctypes.sizeof(pad._binding.PaConfig) == 36


@pytest.mark.parametrize("config", [1, 2, 3, 4, 5])
def test_config_plans_cover_every_token(config):
    w = wl.make_config(config, with_values=False, scale=1.0 if config in (1, 2) else 0.125)
    p = make_plan(w)
    st = p.stats()
    check_structure(Image(p.host_image()), w.kv_lens, w.block_table)
    assert st["unique_tokens"] == w.unique_tokens
    assert st["naive_tokens"] == w.naive_tokens
    assert st["read_tokens"] >= st["unique_tokens"]


def test_config2_tree_and_classes():
    w = wl.make_config(2, with_values=False)
    st = make_plan(w).stats()
    assert st["num_nodes"] == 65 and st["num_shared_nodes"] == 1 and st["num_kept_shared"] == 1
    # 256 rows of the shared root -> 2 query tiles of 128 rows on the tensor-core class
    assert st["num_items"] == 64 + 2
    assert 0 < st["mma_ctas"] < 148 and st["simt_warps"] <= (148 - st["mma_ctas"]) * 8  # at most 8 per CTA
    assert st["num_segments_mma"] > 0 and st["num_segments_simt"] > 0


def test_config4_has_no_tensor_core_work():
    w = wl.make_config(4, with_values=False)
    st = make_plan(w).stats()
    assert st["num_segments_mma"] == 0 and st["num_shared_nodes"] == 0
    assert st["read_tokens"] == st["unique_tokens"] == st["naive_tokens"]


def test_no_sharing_mode_reads_naive_tokens():
    w = wl.make_config(2, with_values=False)
    st = make_plan(w, flags=pad.PA_PLAN_NO_SHARING).stats()
    assert st["num_kept_shared"] == 0 and st["num_segments_mma"] == 0
    assert st["read_tokens"] == st["naive_tokens"]


@pytest.mark.parametrize("seed", range(6))
def test_random_forests_execute_to_oracle(seed):
    G = [1, 2, 4, 8][seed % 4]
    D = [64, 128][seed % 2]
    roots = wl.random_tree(seed=100 + seed, n_queries=7, depth=3, shared_pages=(1, 4), leaf_tokens=(1, 40))
    w = wl.build_workload("rand", roots, Hq=2 * G, Hkv=2, D=D, seed=500 + seed)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    for flags, chunk in [(0, 0), (pad.PA_PLAN_ALWAYS_SHARE, 16), (pad.PA_PLAN_NO_SHARING, 32),
                         (pad.PA_PLAN_ALWAYS_SHARE, 0)]:
        p = make_plan(w, flags=flags, max_chunk_tokens=chunk)
        img = Image(p.host_image())
        check_structure(img, w.kv_lens, w.block_table)
        out, lse = execute(img, w.q, w.k_pool, w.v_pool)
        np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)


def test_config1_executes_to_oracle():
    w = wl.make_config(1)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    for chunk in (0, 16, 48):
        img = Image(make_plan(w, max_chunk_tokens=chunk).host_image())
        out, lse = execute(img, w.q, w.k_pool, w.v_pool)
        np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)


def test_requests_ending_inside_the_tree():
    # request 0's KV is exactly the shared prefix of requests 1 and 2 (full pages)
    P = 16
    bt = np.array([[5, 6, -1, -1], [5, 6, 7, -1], [5, 6, 8, 9]], dtype=np.int32)
    kv = np.array([32, 40, 50], dtype=np.int32)
    for flags in (0, pad.PA_PLAN_ALWAYS_SHARE, pad.PA_PLAN_NO_SHARING):
        p = pad.Plan(kv, bt, 10, 4, 1, 64, flags=flags)
        check_structure(Image(p.host_image()), kv, bt, P)
    # two identical full requests
    bt2 = np.array([[3, 4], [3, 4]], dtype=np.int32)
    p = pad.Plan(np.array([32, 32], dtype=np.int32), bt2, 5, 4, 1, 64, flags=pad.PA_PLAN_ALWAYS_SHARE)
    check_structure(Image(p.host_image()), np.array([32, 32]), bt2, P)


def test_validation_errors():
    bt = np.array([[1, 2], [1, 3]], dtype=np.int32)
    ok = np.array([20, 30], dtype=np.int32)
    pad.Plan(ok, bt, 4, 8, 2, 64)
    cases = [
        (dict(kv_lens=np.array([0, 30], dtype=np.int32)), pad.PA_ERR_INVALID),      # empty request
        (dict(kv_lens=np.array([20, 33], dtype=np.int32)), pad.PA_ERR_INVALID),     # beyond max_pages * P
        (dict(num_pages=3), pad.PA_ERR_INVALID),                                     # page id 3 out of range
        (dict(num_q_heads=12, num_kv_heads=4), pad.PA_ERR_UNSUPPORTED),              # G = 3
        (dict(num_q_heads=8, num_kv_heads=3), pad.PA_ERR_INVALID),                   # not a multiple
        (dict(head_dim=96), pad.PA_ERR_UNSUPPORTED),
        (dict(page_size=32), pad.PA_ERR_UNSUPPORTED),
    ]
    for kw, code in cases:
        args = dict(kv_lens=ok, block_table=bt, num_pages=4, num_q_heads=8, num_kv_heads=2, head_dim=64)
        args.update(kw)
        with pytest.raises(pad.PaError) as e:
            pad.Plan(**args)
        assert e.value.status == code, kw


@pytest.mark.parametrize("flags", [0, pad.PA_PLAN_ALWAYS_SHARE, pad.PA_PLAN_NO_SHARING])
def test_partially_filled_shared_pages(flags):
    # a page several requests hold is packed as shared only where it is full
    # for all of them; a page that is the last, partial page of some of them is
    # read by each of those in its own item (sessions whose queries share the
    # session's partial last page; a request that continues in a page another
    # one ends in)
    P, Hkv, D, Hq = 16, 2, 64, 8
    rng = np.random.default_rng(3)
    bf = lambda *sh: (rng.normal(size=sh).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    n_pages = 12
    k, v = bf(n_pages, Hkv, P, D), bf(n_pages, Hkv, P, D)
    cases = [
        # three queries of one session: pages 4, 5 full, page 6 holds 7 tokens
        (np.array([[4, 5, 6]] * 3, dtype=np.int32), np.array([39, 39, 39], dtype=np.int32)),
        # request 0 ends 10 tokens into page 1, request 1 fills it and goes on
        (np.array([[1, 2], [1, 3]], dtype=np.int32), np.array([10, 30], dtype=np.int32)),
        # the same page partial for two requests of different lengths, full for a third
        (np.array([[7, 8, 9], [7, 8, 10], [7, 8, 11]], dtype=np.int32), np.array([20, 28, 40], dtype=np.int32)),
        # a shared run of full pages, then one page partial for all four at different lengths
        (np.array([[0, 1, 2]] * 4, dtype=np.int32), np.array([33, 35, 40, 47], dtype=np.int32)),
    ]
    for bt, kv in cases:
        q = bf(len(kv), Hq, D)
        p = pad.Plan(kv, bt, n_pages, Hq, Hkv, D, flags=flags)
        img = Image(p.host_image())
        check_structure(img, kv, bt, P)
        out, lse = execute(img, q, k, v)
        ref_o, ref_l = oracle.attend_paged(q, k, v, bt, kv)
        np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)
    # the session's full pages stay one shared node
    p = pad.Plan(cases[0][1], cases[0][0], n_pages, Hq, Hkv, D, flags=pad.PA_PLAN_ALWAYS_SHARE)
    assert p.stats()["num_kept_shared"] == 1 and p.stats()["num_segments_mma"] > 0


@pytest.mark.parametrize("flags", [0, pad.PA_PLAN_ALWAYS_SHARE, pad.PA_PLAN_NO_SHARING])
def test_out_of_range_page_ids_anywhere_are_rejected(flags):
    # pages 0-1 are shared by all three requests, page 2 by the first two,
    # page 3 is each request's own (4 full pages each, pool of 10 pages)
    bt = np.array([[5, 6, 7, 2], [5, 6, 7, 3], [5, 6, 8, 9]], dtype=np.int32)
    kv = np.array([64, 64, 64], dtype=np.int32)
    pad.Plan(kv, bt, 10, 4, 1, 64, flags=flags)
    bad_cases = []
    b = bt.copy(); b[:, 1] = 10; bad_cases.append(b)      # in a run shared by three
    b = bt.copy(); b[:2, 2] = 11; bad_cases.append(b)     # in a run shared by two
    b = bt.copy(); b[2, 3] = 12; bad_cases.append(b)      # in one request's own page
    b = bt.copy(); b[1, 2] = -1; bad_cases.append(b)      # negative
    for i, b in enumerate(bad_cases):
        with pytest.raises(pad.PaError) as e:
            pad.Plan(kv, b, 10, 4, 1, 64, flags=flags)
        assert e.value.status == pad.PA_ERR_INVALID, i
    # an entry past a request's last page is never read
    ignored = bt.copy()
    ignored[0, 3] = 99
    pad.Plan(np.array([48, 64, 64], dtype=np.int32), ignored, 10, 4, 1, 64, flags=flags)


def test_plan_is_deterministic():
    w = wl.make_config(3, with_values=False, scale=0.25)
    a = make_plan(w).host_image()
    # a plan of other inputs in between leaves other bytes in the pooled host
    # buffers; the alignment gaps of the image are zeroed, so the bytes match
    other = make_plan(wl.make_config(2, with_values=False, scale=0.5))
    other.close()
    b = make_plan(w).host_image()
    assert np.array_equal(a, b)


def tensor_core_units(w, flags=0):
    p = make_plan(w, flags=flags)
    img = Image(p.host_image())
    h = img.h
    ns = h.num_segments_simt
    pages = [(int(img.segs[i][3]) + 15) // 16 for i in range(ns, h.num_segments)]
    runs = {}
    for i in range(ns, h.num_segments):
        item, g = int(img.segs[i][0]), int(img.segs[i][1])
        runs.setdefault((item, g), []).append(i)
    return h, img, pages, runs


@pytest.mark.parametrize("config", [1, 2, 3, 5])
def test_tensor_core_work_units_cover_each_run_in_pieces_of_at_least_32_pages(config):
    # at most one tensor-core CTA per 16 pages of tensor-core work (a small
    # shared prefix, config 1: 16 pages x 2 kv heads, is not spread over many
    # CTAs that each pay the segment's fixed cost); every (item, kv head) run
    # is covered by consecutive pieces of at least 32 pages (or the whole run),
    # and there are at least as many pieces as CTAs
    w = wl.make_config(config, with_values=False)
    # config 1's small prefix is inlined by the profit model; shared on purpose here
    h, img, pages, runs = tensor_core_units(w, flags=pad.PA_PLAN_ALWAYS_SHARE if config == 1 else 0)
    mma_pages = sum(pages)
    assert 1 <= h.mma_ctas <= -(-mma_pages // 16) and h.mma_ctas <= len(pages)
    if config == 1:
        assert h.mma_ctas <= 2
    ns = h.num_segments_simt
    for (item, g), ids in runs.items():
        segs = sorted((int(img.segs[i][2]), pages[i - ns]) for i in ids)  # (page_begin, pages)
        assert segs[0][0] == 0
        for (b0, n0), (b1, _) in zip(segs, segs[1:]):
            assert b1 == b0 + n0
        total = sum(n for _, n in segs)
        assert total == -(-int(img.items[item][1]) // 16)
        assert len(segs) == 1 or min(n for _, n in segs) >= 32


@pytest.mark.parametrize("config", [3, 5])
def test_tensor_core_work_units_longest_first_and_short_at_the_end(config):
    # guided self-scheduling: the CTAs take the units longest first from a
    # shared counter, so a CTA that runs faster takes more of them; the units
    # shrink as the queue drains, each cut about a 2 x CTAs-th of the work not
    # yet cut, so the last units, which decide when the launch ends on a slow
    # SM, are short, while most of the work still runs in long units (config 5:
    # 256 runs of 2k-8k pages over 147 CTAs; config 3: 128-row root runs of 256
    # pages and 64-page branch runs)
    w = wl.make_config(config, with_values=False)
    h, img, pages, runs = tensor_core_units(w)
    W, n = sum(pages), h.mma_ctas
    assert pages == sorted(pages, reverse=True)
    assert pages[0] <= -(-W // (2 * n)) + 64
    assert max(pages[-n:]) <= 64 and sum(pages[-n:]) <= W // 8
    # about 2 ln(W / (2 n 64)) + 2 units per CTA, not many more
    assert len(pages) <= n * (2 * np.log(max(2.0, W / (2 * n * 64))) + 4) + len(runs)


# ------------------------------------------------------------- decode steps

def decode_steps(w, steps, seed):
    """Yields (kv_lens, block_table, k_pool, v_pool, num_pages) after each of
    `steps` decode steps: every request appends 0-2 tokens (random bf16 K/V),
    taking a fresh page of its own whenever its last page is full."""
    rng = np.random.default_rng(seed)
    P = w.P
    kv = w.kv_lens.astype(np.int32).copy()
    spare = w.B * (2 * steps // P + 2)
    k = np.concatenate([w.k_pool, np.full((spare,) + w.k_pool.shape[1:], wl.BF16_NAN, np.uint16)])
    v = np.concatenate([w.v_pool, np.full((spare,) + w.v_pool.shape[1:], wl.BF16_NAN, np.uint16)])
    cols = w.block_table.shape[1] + 2 * steps // P + 2
    bt = np.full((w.B, cols), -1, np.int32)
    bt[:, :w.block_table.shape[1]] = w.block_table
    free = w.num_pages
    for _ in range(steps):
        for b in range(w.B):
            for _ in range(int(rng.integers(0, 3))):
                pos = int(kv[b])
                pg, slot = pos // P, pos % P
                if slot == 0:
                    bt[b, pg] = free
                    free += 1
                page = bt[b, pg]
                k[page, :, slot, :] = rng.normal(size=(w.Hkv, w.D)).astype(np.float32).view(np.uint32) >> 16
                v[page, :, slot, :] = rng.normal(size=(w.Hkv, w.D)).astype(np.float32).view(np.uint32) >> 16
                kv[b] += 1
        yield kv.copy(), bt.copy(), k, v, free


@pytest.mark.parametrize("seed", range(4))
def test_advanced_plans_execute_to_oracle(seed):
    # pa_plan_advance: the tree of the first step is carried over; each
    # request's own tail takes the new tokens.  Every step's plan must cover
    # each token once and execute to the oracle, and count the same tokens as
    # a plan made from scratch
    G = [1, 2, 4, 8][seed % 4]
    D = [64, 128][seed % 2]
    roots = wl.random_tree(seed=300 + seed, n_queries=9, depth=3, shared_pages=(1, 4), leaf_tokens=(1, 40))
    w = wl.build_workload("rand", roots, Hq=2 * G, Hkv=2, D=D, seed=700 + seed)
    p = make_plan(w, flags=pad.PA_PLAN_KEEP_PACK, max_chunk_tokens=32 * (seed % 2))
    for kv, bt, k, v, n_pages in decode_steps(w, steps=20, seed=seed):
        p = p.advance(kv, bt, n_pages)
        img = Image(p.host_image())
        check_structure(img, kv, bt)
        out, lse = execute(img, w.q, k, v)
        ref_o, ref_l = oracle.attend_paged(w.q, k, v, bt, kv)
        np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)
        st = p.stats()
        full = pad.Plan(kv, bt, n_pages, w.Hq, w.Hkv, w.D, max_chunk_tokens=32 * (seed % 2)).stats()
        for key in ("unique_tokens", "naive_tokens", "read_tokens", "num_shared_nodes", "num_kept_shared"):
            assert st[key] == full[key], key


def test_advance_falls_back_and_checks_its_inputs():
    roots = wl.random_tree(seed=41, n_queries=6, depth=2, shared_pages=(1, 3), leaf_tokens=(1, 40))
    w = wl.build_workload("rand", roots, Hq=8, Hkv=2, D=64, seed=42)
    kept = make_plan(w, flags=pad.PA_PLAN_KEEP_PACK)
    # a plan made without PA_PLAN_KEEP_PACK cannot be advanced
    with pytest.raises(pad.PaError) as e:
        make_plan(w).advance(w.kv_lens, w.block_table, w.num_pages)
    assert e.value.status == pad.PA_ERR_INVALID
    # a request that shrank: planned from scratch, same structure as pa_plan_create
    kv = w.kv_lens.copy()
    b = int(np.argmax(kv))
    kv[b] -= 1
    p = kept.advance(kv, w.block_table, w.num_pages)
    check_structure(Image(p.host_image()), kv, w.block_table)
    assert p.stats()["unique_tokens"] == make_plan(w).stats()["unique_tokens"] - 1
    # a new page id outside the pool is rejected
    steps = decode_steps(w, steps=16, seed=3)
    kv2, bt2, _, _, n_pages = next(steps)
    grown = np.nonzero(kv2 > w.kv_lens)[0]
    assert len(grown)
    bad = bt2.copy()
    for r in grown:
        bad[r, (kv2[r] - 1) // 16] = n_pages + 5 if (kv2[r] - 1) // 16 >= (w.kv_lens[r] + 15) // 16 else bad[r, (kv2[r] - 1) // 16]
    if np.array_equal(bad, bt2):
        pytest.skip("no request took a new page in the first step")
    with pytest.raises(pad.PaError) as e:
        kept.advance(kv2, bad, n_pages)
    assert e.value.status == pad.PA_ERR_INVALID


def test_advance_gives_a_request_that_ended_at_a_shared_node_its_own_tail():
    # request 0's KV is exactly the shared node [5, 6] of requests 0-2 (kept
    # shared), so it has no item of its own; its next token goes to a new page
    P, Hkv, D, Hq = 16, 1, 64, 4
    rng = np.random.default_rng(5)
    n_pages = 12
    bf = lambda *s: (rng.normal(size=s).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    k, v = bf(n_pages, Hkv, P, D), bf(n_pages, Hkv, P, D)
    q = bf(3, Hq, D)
    bt = np.array([[5, 6, -1, -1], [5, 6, 7, -1], [5, 6, 8, 9]], dtype=np.int32)
    kv = np.array([32, 40, 50], dtype=np.int32)
    p = pad.Plan(kv, bt, n_pages, Hq, Hkv, D, flags=pad.PA_PLAN_ALWAYS_SHARE | pad.PA_PLAN_KEEP_PACK)
    before = Image(p.host_image())
    assert sum(1 for it in before.items if it[2] == 1 and int(before.queries[it[3]]) == 0) == 0
    bt2 = bt.copy()
    bt2[0, 2] = 10
    for kv2 in (np.array([33, 41, 50], dtype=np.int32), np.array([40, 47, 51], dtype=np.int32)):
        p2 = p.advance(kv2, bt2, n_pages)
        img = Image(p2.host_image())
        check_structure(img, kv2, bt2, P)
        out, lse = execute(img, q, k, v)
        ref_o, ref_l = oracle.attend_paged(q, k, v, bt2, kv2)
        np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)
        assert p2.stats()["num_kept_shared"] == 1


@pytest.mark.parametrize("config,scale", [(5, 1 / 64), (3, 1 / 16)])
def test_advanced_plans_of_session_and_tree_batches(config, scale):
    # shapes with tensor-core items of many rows (config 5: sessions of 16
    # requests over one context; config 3: a three-level tree), a few decode
    # steps through pa_plan_advance, executed against the oracle
    w = wl.make_config(config, scale=scale)
    p = make_plan(w, flags=pad.PA_PLAN_KEEP_PACK)
    assert p.stats()["num_segments_mma"] > 0
    for kv, bt, k, v, n_pages in decode_steps(w, steps=3, seed=config):
        p = p.advance(kv, bt, n_pages)
        img = Image(p.host_image())
        check_structure(img, kv, bt)
        out, lse = execute(img, w.q, k, v)
        ref_o, ref_l = oracle.attend_paged(w.q, k, v, bt, kv)
        np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)
        assert p.stats()["num_segments_mma"] > 0


@pytest.mark.parametrize("num_sms", [1, 2, 3])
def test_plans_for_very_few_sms(num_sms):
    # both tile classes with one to three SMs: each class still gets at least
    # one CTA (with one SM the two launches run one after the other)
    w = wl.make_config(2, scale=0.125)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    p = make_plan(w, num_sms=num_sms)
    st = p.stats()
    assert st["mma_ctas"] >= 1 and st["simt_warps"] >= 1
    img = Image(p.host_image())
    wpc = img.h.simt_warps_per_cta
    assert st["mma_ctas"] + -(-st["simt_warps"] // wpc) <= max(2, num_sms)
    check_structure(img, w.kv_lens, w.block_table)
    out, lse = execute(img, w.q, w.k_pool, w.v_pool)
    np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)


def test_random_plans_and_advances_against_the_oracle():
    # a fixed-seed sweep over tree shapes, GQA groups, head dims, SM counts,
    # planner flags and chunk caps: a plan, then decode steps through
    # pa_plan_advance (some requests shrink, which plans from scratch), every
    # plan checked for coverage and the last one executed against the oracle
    rng = np.random.default_rng(2024)
    done = 0
    while done < 60:
        seed = int(rng.integers(1 << 30))
        G, D, Hkv = int(rng.choice([1, 2, 4, 8])), int(rng.choice([64, 128])), int(rng.choice([1, 2]))
        roots = wl.random_tree(seed=seed, n_queries=int(rng.integers(2, 20)), depth=int(rng.integers(1, 4)),
                               shared_pages=(1, int(rng.integers(1, 6))), leaf_tokens=(1, int(rng.integers(2, 80))))
        w = wl.build_workload("sweep", roots, Hq=G * Hkv, Hkv=Hkv, D=D, seed=seed % 1000)
        flags = int(rng.choice([0, pad.PA_PLAN_ALWAYS_SHARE, pad.PA_PLAN_NO_SHARING]))
        p = make_plan(w, flags=flags | pad.PA_PLAN_KEEP_PACK, num_sms=int(rng.choice([1, 2, 7, 148])),
                      max_chunk_tokens=int(rng.choice([0, 16, 64])))
        for kv, bt, k, v, n_pages in decode_steps(w, steps=int(rng.integers(1, 8)), seed=seed % 97):
            kv = kv.copy()
            b = int(rng.integers(0, w.B))
            if rng.random() < 0.2 and kv[b] > w.kv_lens[b]:
                kv[b] -= 1
            p = p.advance(kv, bt, n_pages)
            img = Image(p.host_image())
            check_structure(img, kv, bt)
        out, lse = execute(img, w.q, k, v)
        ref_o, ref_l = oracle.attend_paged(w.q, k, v, bt, kv)
        np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)
        done += 1


def test_random_partially_shared_pages_against_the_oracle():
    # block tables whose rows share random prefixes of a few page chains and
    # end anywhere (so shared pages are often partial for some holders), then
    # grown in place; plan, advance and execute against the oracle
    rng = np.random.default_rng(77)
    P = 16
    for _ in range(40):
        B, maxp = int(rng.integers(1, 10)), int(rng.integers(1, 7))
        Hkv, G, D = int(rng.choice([1, 2])), int(rng.choice([1, 2, 4, 8])), int(rng.choice([64, 128]))
        chains = [rng.permutation(100)[:maxp] for _ in range(int(rng.integers(1, 4)))]
        bt = np.full((B, maxp), -1, np.int32)
        nxt = 100
        for b in range(B):
            share = int(rng.integers(0, maxp + 1))
            bt[b, :share] = chains[int(rng.integers(0, len(chains)))][:share]
            bt[b, share:] = np.arange(nxt, nxt + maxp - share)
            nxt += maxp - share
        kv = rng.integers(1, maxp * P + 1, size=B).astype(np.int32)
        bf = lambda *sh: (rng.normal(size=sh).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        k, v, q = bf(nxt, Hkv, P, D), bf(nxt, Hkv, P, D), bf(B, G * Hkv, D)
        flags = int(rng.choice([0, pad.PA_PLAN_ALWAYS_SHARE, pad.PA_PLAN_NO_SHARING]))
        p = pad.Plan(kv, bt, nxt, G * Hkv, Hkv, D, flags=flags | pad.PA_PLAN_KEEP_PACK)
        kv2 = np.minimum(kv + rng.integers(0, 20, size=B), maxp * P).astype(np.int32)
        for plan, lens in ((p, kv), (p.advance(kv2, bt, nxt), kv2)):
            img = Image(plan.host_image())
            check_structure(img, lens, bt)
            out, lse = execute(img, q, k, v)
            ref_o, ref_l = oracle.attend_paged(q, k, v, bt, lens)
            np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)


@pytest.mark.parametrize("G,D", [(1, 64), (4, 128), (8, 64)])
def test_append_plan_executes_to_the_oracle_rows(G, D):
    # chunks of 1, 5, 16 and 19 new tokens over contexts that end on and off
    # page boundaries (0 tokens included): each row must see the context and
    # the chunk up to itself, nothing after it
    ctx = np.array([0, 37, 48, 200, 333], dtype=np.int32)
    chunk = np.array([5, 19, 1, 16, 19], dtype=np.int32)
    w, q = wl.session_chunks(ctx, chunk, Hq=2 * G, Hkv=2, D=D, seed=11 * G + D)
    plan = pad.Plan.append(ctx, chunk, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
    st = plan.stats()
    assert st["batch"] == chunk.sum()
    img = Image(plan.host_image())
    row_req = np.repeat(np.arange(len(ctx)), chunk)
    row_pos = np.concatenate([c + np.arange(n) for c, n in zip(ctx, chunk)])
    check_structure(img, (row_pos + 1).astype(np.int32), w.block_table[row_req])
    o, l = execute(img, q, w.k_pool, w.v_pool)
    ro, rl = oracle.attend_rows(q, row_req, row_pos, w.k_pool, w.v_pool, w.block_table)
    assert np.abs(o - ro).max() < 1e-12 and np.abs(l - rl).max() < 1e-12
    # the rows of a session with a long context share its full pages
    assert st["num_kept_shared"] >= 1
    plan.close()


def test_append_plan_rejects_bad_chunks():
    bt = np.zeros((1, 4), np.int32)
    with pytest.raises(pad.PaError):
        pad.Plan.append([10], [0], bt, 4, 8, 2, 64)
    with pytest.raises(pad.PaError):
        pad.Plan.append([60], [5], bt, 4, 8, 2, 64)  # 65 tokens > 4 pages


def test_small_row_warps_per_cta():
    # 6 warps per CTA when the small-row class streams long runs of D = 128
    # tiles on most SMs (configs 3 and 4), else 8: short runs (config 2), a
    # class of one CTA beside the tensor-core launch (config 5), D = 64
    want = {2: 8, 3: 6, 4: 6, 5: 8}
    for c, wpc in want.items():
        w = wl.make_config(c, with_values=False)
        img = Image(make_plan(w).host_image())
        assert img.h.simt_warps_per_cta == wpc, c
        # the warp lists cover whole CTAs of that many warps at most
        assert img.h.simt_warps <= (148 - img.h.mma_ctas) * wpc
    # long independent requests: 6 warps at D = 128, 8 at D = 64
    roots = wl.random_tree(seed=5, n_queries=128, depth=0, leaf_tokens=(4000, 6000))
    for D, wpc in ((128, 6), (64, 8)):
        wd = wl.build_workload("long", roots, Hq=32, Hkv=8, D=D, seed=5, with_values=False)
        assert Image(make_plan(wd).host_image()).h.simt_warps_per_cta == wpc, D


def test_binding_host_arrays():
    # host arrays reach the library by address: the buffer-protocol address is
    # the array's data, other dtypes and layouts are converted, read-only
    # arrays still work, and a wrong rank is refused
    from prefix_aware_decode_b200 import _binding as B

    a = np.arange(64, dtype=np.int32)
    assert B._host_ptr(a) == a.ctypes.data
    assert B._host_i32(a, 1) is a
    b = B._host_i32(np.arange(12, dtype=np.int64).reshape(3, 4)[:, ::2], 2)
    assert b.dtype == np.int32 and b.flags.c_contiguous and b.tolist() == [[0, 2], [4, 6], [8, 10]]
    ro = np.arange(8, dtype=np.int32)
    ro.flags.writeable = False
    assert B._host_ptr(ro) == ro.ctypes.data
    with pytest.raises(ValueError):
        B._host_i32(a, 2)
