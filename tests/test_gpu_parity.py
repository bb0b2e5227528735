"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Inputs are the seeded synthetic workloads (NaN-poisoned spare pages and
tails).  Tolerances (gpu_util): max abs 2e-3 wherever |o| < 1, and half a bf16
ulp plus 2^-15 |o| above (where rounding the output to bf16 alone exceeds
2e-3); max relative 1e-2 floored by the row rms; 1e-4 on fp32 lse.  Configs
1-4 are compared on every request, config 5 on three queries of each of its
32 sessions (the first and the last among them).
"""
import numpy as np
import pytest
import torch

import oracle
import prefix_aware_decode_b200 as pad
from prefix_aware_decode_b200 import workload as wl

from gpu_util import DevWorkload, assert_close, compare, run

pytestmark = pytest.mark.gpu

_cache = {}


def dev_config(c, scale=1.0):
    key = (c, scale)
    if key not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        _cache[key] = DevWorkload(wl.make_config(c, scale=scale))
    return _cache[key]


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("config", [1, 2])
def test_small_configs_full_parity(config, fused):
    dw = dev_config(config)
    w = dw.w
    out, lse, st, _ = run(dw, fused=fused)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    m = compare(out, lse, ref_o, ref_l)
    assert_close(m, f"config {config}")


@pytest.mark.parametrize("config", [2, 3, 4])
def test_large_configs_full_parity(config):
    # every request of the workload, both the two-launch path (pa_forward +
    # pa_merge) and the fused one (pa_attend)
    dw = dev_config(config)
    w = dw.w
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    res = {}
    for fused in (False, True):
        out, lse, st, _ = run(dw, fused=fused)
        assert_close(compare(out, lse, ref_o, ref_l), f"config {config} fused={fused}")
        res[fused] = (out, lse)
    # the fused merge combines a pair's partial rows in the same fixed order
    # whichever arrival merges it (config 2: 512 mixed pairs, each counted by
    # a designated small-row warp once the tensor-core launch has finished;
    # config 3: 2048 mixed pairs, more than 3 per small-row warp, merged by the
    # tail merge launch)
    assert torch.equal(res[True][0].view(torch.int16), res[False][0].view(torch.int16))
    assert torch.equal(res[True][1], res[False][1])
    if config == 2:
        assert st["num_segments_mma"] > 0 and st["num_tail_pairs"] == 0
    if config == 3:
        assert st["num_segments_mma"] > 0 and st["num_tail_pairs"] > 0


def test_config5_every_session_parity():
    # 32 sessions x 16 registered queries (request 16 s + j is query j of
    # session s): the first and the last query of every session, plus one
    # from the middle of each, against the oracle
    dw = dev_config(5)
    w = dw.w
    S = w.B // 16
    qs = np.array(sorted({16 * s + j for s in range(S) for j in (0, 15, (5 * s) % 14 + 1)}), dtype=np.int32)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens, queries=qs)
    for fused in (False, True):
        out, lse, st, _ = run(dw, fused=fused)
        assert st["num_segments_mma"] > 0
        assert_close(compare(out, lse, ref_o, ref_l, queries=qs), f"config 5 fused={fused} ({len(qs)} queries)")
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("flags,chunk", [(pad.PA_PLAN_NO_SHARING, 0), (pad.PA_PLAN_ALWAYS_SHARE, 64),
                                         (0, 16), (pad.PA_PLAN_ALWAYS_SHARE, 16)])
def test_plan_modes_match_oracle(flags, chunk):
    dw = dev_config(2, scale=0.25)
    w = dw.w
    out, lse, st, _ = run(dw, flags=flags, max_chunk_tokens=chunk)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    assert_close(compare(out, lse, ref_o, ref_l), f"flags {flags} chunk {chunk}")


@pytest.mark.parametrize("G,D", [(1, 64), (2, 128), (4, 64), (4, 128), (8, 64), (8, 128), (1, 128), (2, 64)])
def test_random_forests_gqa_and_head_dim(G, D):
    roots = wl.random_tree(seed=G * 10 + D, n_queries=24, depth=3, shared_pages=(1, 12), leaf_tokens=(1, 300),
                           fanout=(1, 6))
    w = wl.build_workload("rand", roots, Hq=4 * G, Hkv=4, D=D, seed=G * 1000 + D)
    dw = DevWorkload(w)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    for flags, chunk in [(0, 0), (pad.PA_PLAN_ALWAYS_SHARE, 32), (pad.PA_PLAN_NO_SHARING, 0)]:
        out, lse, st, _ = run(dw, flags=flags, max_chunk_tokens=chunk)
        assert_close(compare(out, lse, ref_o, ref_l), f"G={G} D={D} flags={flags}")


@pytest.mark.parametrize("fused", [False, True])
def test_edge_lengths_and_ragged_tails(fused):
    lens = [1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 255, 256, 257, 1000, 4099]
    roots = [wl.Node(n) for n in lens]
    # plus a shared prefix whose children end 0..17 tokens after it
    roots.append(wl.Node(48, [wl.Node(n) for n in (1, 5, 16, 17)]))
    w = wl.build_workload("edges", roots, Hq=32, Hkv=8, D=128, seed=4242)
    dw = DevWorkload(w)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    for flags, chunk in [(0, 0), (pad.PA_PLAN_ALWAYS_SHARE, 16), (0, 32)]:
        out, lse, st, _ = run(dw, flags=flags, max_chunk_tokens=chunk, fused=fused)
        assert_close(compare(out, lse, ref_o, ref_l), f"edges flags={flags} chunk={chunk}")


@pytest.mark.parametrize("fused", [False, True])
def test_pairs_with_tensor_core_rows_only(fused):
    # requests 0 and 1 hold the same four full pages and nothing else, so their
    # (request, kv head) pairs have tensor-core partial rows only (merged by the
    # tail merge launch in the fused path); requests 2 and 3 share those pages
    # too and go on, so theirs mix tensor-core and SIMT rows
    base = wl.make_config(1)
    bt = base.block_table.copy()
    kv = base.kv_lens.copy()
    bt[1, :4] = bt[0, :4]
    kv[0] = kv[1] = 64
    w = wl.Workload(**{**base.__dict__, "block_table": bt, "kv_lens": kv})
    dw = DevWorkload(w)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    out, lse, st, _ = run(dw, flags=pad.PA_PLAN_ALWAYS_SHARE, fused=fused)
    assert st["num_tail_pairs"] == 2 * w.Hkv and st["mma_ctas"] >= 1
    assert_close(compare(out, lse, ref_o, ref_l), "tensor-core-only pairs")


def test_single_key_returns_v_row_bit_exact():
    roots = [wl.Node(1) for _ in range(16)]
    w = wl.build_workload("one", roots, Hq=32, Hkv=8, D=128, seed=77)
    dw = DevWorkload(w)
    out, lse, st, _ = run(dw)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    G = w.Hq // w.Hkv
    for b in range(w.B):
        page = w.block_table[b, 0]
        for h in range(w.Hq):
            assert np.array_equal(got[b, h], w.v_pool[page, h // G, 0]), (b, h)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    assert np.abs(lse.cpu().numpy() - ref_l).max() <= 1e-4


def test_results_are_bit_reproducible():
    dw = dev_config(2, scale=0.25)
    a, la, _, _ = run(dw)
    b, lb, _, _ = run(dw)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)) and torch.equal(la, lb)


@pytest.mark.parametrize("flags", [0, pad.PA_PLAN_ALWAYS_SHARE])
def test_bounded_wait_reports_timeout_and_context_survives(flags):
    """A forward that never receives one of its loads must give up after the
    configured limit, record PA_ERR_TIMEOUT in the workspace, and leave the
    context usable (a normal run right after it still matches the oracle)."""
    w = wl.make_config(1)
    dw = DevWorkload(w)
    out, lse, st, status = run(dw, flags=flags | pad.PA_PLAN_FAULT_DROP_LOAD, wait_timeout_us=20000,
                               check_status=False)
    assert status == pad.PA_ERR_TIMEOUT
    out, lse, st, status = run(dw, flags=flags)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    assert_close(compare(out, lse, ref_o, ref_l), "after timeout")


def test_attend_convenience_and_validation():
    dw = dev_config(1)
    w = dw.w
    out, lse = pad.attend(dw.q, dw.k, dw.v, w.block_table, w.kv_lens)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    assert_close(compare(out, lse, ref_o, ref_l), "attend()")
    plan = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
    ws = plan.alloc_workspace()
    # a workspace that is too small, or misaligned pointers, are refused before anything is enqueued
    assert plan._lib.pa_plan_upload(plan.handle, ws.data_ptr(), 16, None) == pad.PA_ERR_NOMEM
    assert plan._lib.pa_forward(plan.handle, dw.q.data_ptr() + 2, dw.k.data_ptr(), dw.v.data_ptr(),
                                ws.data_ptr(), None) == pad.PA_ERR_INVALID
    plan.close()


def test_decode_step_matches_plan_path():
    dw = dev_config(2, scale=0.25)
    w = dw.w
    a, la, _, _ = run(dw)
    plan = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
    ws = plan.alloc_workspace()
    plan.close()
    out = torch.empty_like(a)
    lse = torch.empty_like(la)
    step = pad.DecodeStep(w.num_pages, w.Hq, w.Hkv, w.D, dw.q, dw.k, dw.v, ws, out, lse)
    for _ in range(2):  # the arrival counters are left at zero: a second step gives the same bits
        step(w.kv_lens, w.block_table)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), a.view(torch.int16)) and torch.equal(lse, la)


def test_arrival_counters_return_to_zero_with_mixed_pairs():
    # mixed pairs (tensor-core and small-row rows) are merged by the last
    # small-row arriver after the tensor-core launch; the merging warp puts the
    # pair's arrival counter back to zero, and the launch's last take of a
    # tensor-core work unit puts the unit counter back to zero, so the uploaded
    # plan gives the same bits launch after launch
    import ctypes

    dw = dev_config(2, scale=0.25)
    w = dw.w
    plan = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
    st = plan.stats()
    assert st["mma_ctas"] > 0 and st["simt_warps"] > 0 and st["num_tail_pairs"] == 0
    h = pad.PaImageHeader.from_buffer_copy(plan.host_image()[: ctypes.sizeof(pad.PaImageHeader)].tobytes())
    n_words = w.B * w.Hkv
    ws = plan.alloc_workspace()
    plan.upload(ws)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    first = None
    for _ in range(4):
        out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        plan.attend(dw.q, dw.k, dw.v, ws, out, lse)
        torch.cuda.synchronize()
        words = ws[h.off_counters: h.off_counters + 4 * n_words].cpu().numpy().view(np.int32)
        assert not words.any(), np.nonzero(words)
        # the counter of tensor-core work units taken is back at zero too
        off_next = pad.PaImageHeader.mma_next.offset
        assert int(ws[off_next:off_next + 4].cpu().numpy().view(np.int32)[0]) == 0
        if first is None:
            first = (out.clone(), lse.clone())
            assert_close(compare(out, lse, ref_o, ref_l), "attend() with mixed pairs")
        else:
            assert torch.equal(out.view(torch.int16), first[0].view(torch.int16)) and torch.equal(lse, first[1])
    assert plan.device_status(ws) == pad.PA_OK
    plan.close()


def test_advanced_plan_on_the_device_matches_the_oracle():
    # pa_plan_advance over a few decode steps of a config-2-shaped batch: the
    # carried-over plan runs through the same kernels and matches the oracle
    w = wl.make_config(2, scale=0.25)
    P = w.P
    rng = np.random.default_rng(11)
    kv = w.kv_lens.astype(np.int32).copy()
    bt = np.full((w.B, w.block_table.shape[1] + 2), -1, np.int32)
    bt[:, :w.block_table.shape[1]] = w.block_table
    spare = 2 * w.B
    k = np.concatenate([w.k_pool, np.full((spare,) + w.k_pool.shape[1:], wl.BF16_NAN, np.uint16)])
    v = np.concatenate([w.v_pool, np.full((spare,) + w.v_pool.shape[1:], wl.BF16_NAN, np.uint16)])
    n_pages, free = w.num_pages + spare, w.num_pages
    plan = pad.Plan(kv, bt, n_pages, w.Hq, w.Hkv, w.D, flags=pad.PA_PLAN_KEEP_PACK)
    q = torch.from_numpy(w.q.view(np.int16)).cuda().view(torch.bfloat16)
    for step in range(3):
        for b in range(w.B):
            for _ in range(int(rng.integers(1, 4))):
                pos = int(kv[b])
                if pos % P == 0:
                    bt[b, pos // P] = free
                    free += 1
                page = bt[b, pos // P]
                k[page, :, pos % P, :] = rng.normal(size=(w.Hkv, w.D)).astype(np.float32).view(np.uint32) >> 16
                v[page, :, pos % P, :] = rng.normal(size=(w.Hkv, w.D)).astype(np.float32).view(np.uint32) >> 16
                kv[b] += 1
        nxt = plan.advance(kv, bt, n_pages)
        plan.close()
        plan = nxt
        kd = torch.from_numpy(k.view(np.int16)).cuda().view(torch.bfloat16)
        vd = torch.from_numpy(v.view(np.int16)).cuda().view(torch.bfloat16)
        ws = plan.alloc_workspace()
        plan.upload(ws)
        out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        plan.attend(q, kd, vd, ws, out, lse)
        torch.cuda.synchronize()
        assert plan.device_status(ws) == pad.PA_OK
        ref_o, ref_l = oracle.attend_paged(w.q, k, v, bt, kv)
        assert_close(compare(out, lse, ref_o, ref_l), f"advanced plan, step {step}")
    plan.close()


def test_decode_steps_alternating_batches_and_one_plan_over_several_pools():
    # pa_decode_step uploads each step's plan into one of two device slots on a
    # copy stream of its own (config 1's 3.8 KB image on the compute stream
    # itself, config 2's on the copy stream, so the slots switch between the
    # two ways); alternating two different batches must give each batch its
    # own result every time
    wa = wl.make_config(1)
    wb = wl.make_config(2, scale=0.25)
    da, db = DevWorkload(wa), DevWorkload(wb)
    refs = {}
    for name, w in (("a", wa), ("b", wb)):
        refs[name] = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    outs = {}
    for name, w, d in (("a", wa, da), ("b", wb, db)):
        p = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
        ws = p.alloc_workspace()
        p.close()
        o = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
        l = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        outs[name] = (pad.DecodeStep(w.num_pages, w.Hq, w.Hkv, w.D, d.q, d.k, d.v, ws, o, l), o, l, w)
    for step in range(6):
        name = "ab"[step % 2]
        stepper, o, l, w = outs[name]
        stepper(w.kv_lens, w.block_table)
        if step >= 4:
            torch.cuda.synchronize()
            assert_close(compare(o, l, *refs[name]), f"alternating step {step} ({name})")
    # one uploaded plan read with three different pool pairs (as the layers of
    # a model would): each result matches the oracle over that pool pair
    w, d = wb, db
    p = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
    ws = p.alloc_workspace()
    p.upload(ws)
    # other contents with the NaN poison in the same places: K and V swapped,
    # K with its signs flipped
    flip = lambda a: (a.view(np.uint16) ^ np.uint16(0x8000)).view(a.dtype)
    for layer, (k_np, v_np) in enumerate([(w.k_pool, w.v_pool), (w.v_pool, w.k_pool), (flip(w.k_pool), w.v_pool)]):
        k_d = torch.from_numpy(np.ascontiguousarray(k_np).view(np.int16)).cuda().view(torch.bfloat16)
        v_d = torch.from_numpy(np.ascontiguousarray(v_np).view(np.int16)).cuda().view(torch.bfloat16)
        o = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
        l = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        p.attend(d.q, k_d, v_d, ws, o, l)
        torch.cuda.synchronize()
        ref = oracle.attend_paged(w.q, k_np, v_np, w.block_table, w.kv_lens)
        assert_close(compare(o, l, *ref), f"pool pair {layer}")
    assert p.device_status(ws) == pad.PA_OK
    p.close()


@pytest.mark.parametrize("flags", [pad.PA_PLAN_NO_SHARING, pad.PA_PLAN_ALWAYS_SHARE])
def test_debug_checks_catch_a_corrupted_page_id(flags):
    """PA_PLAN_DEBUG_CHECKS range-checks every page id the kernels read from
    the device image before any load is issued.  The pools here hold 8 NaN
    pages more than the plan declares, and the uploaded image's first page id
    is overwritten with one of them: still inside the allocation (an unchecked
    read would stay in bounds) but past the declared pool, so the check must
    record PA_ERR_DEVICE.  The first page id belongs to request 0's own item
    (small-row class) without sharing, and to the shared prefix (tensor-core
    class) with it.  A clean run on the same plan is correct again."""
    import ctypes

    w = wl.make_config(1)
    extra = np.full((8,) + w.k_pool.shape[1:], wl.BF16_NAN, np.uint16)
    k = torch.from_numpy(np.concatenate([w.k_pool, extra]).view(np.int16)).cuda().view(torch.bfloat16)
    v = torch.from_numpy(np.concatenate([w.v_pool, extra]).view(np.int16)).cuda().view(torch.bfloat16)
    q = torch.from_numpy(w.q.view(np.int16)).cuda().view(torch.bfloat16)
    plan = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D,
                    flags=flags | pad.PA_PLAN_DEBUG_CHECKS)
    h = pad.PaImageHeader.from_buffer_copy(plan.host_image()[: ctypes.sizeof(pad.PaImageHeader)].tobytes())
    ws = plan.alloc_workspace()
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    plan.upload(ws)
    torch.cuda.synchronize()
    ws[h.off_pages:h.off_pages + 4].view(torch.int32).fill_(w.num_pages + 3)
    plan.attend(q, k, v, ws, out, lse)
    assert plan.device_status(ws) == pad.PA_ERR_DEVICE
    plan.upload(ws)
    plan.attend(q, k, v, ws, out, lse)
    assert plan.device_status(ws) == pad.PA_OK
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    assert_close(compare(out, lse, ref_o, ref_l), "debug checks, clean run")
    plan.close()


@pytest.mark.parametrize("config,scale", [(2, 0.25), (5, 0.125)])
def test_canaries_around_outputs_and_workspace_survive(config, scale):
    # every device buffer the library writes (workspace, out, lse) sits inside
    # a larger allocation with a canary pattern of 4 KiB on both sides; the
    # two-launch path, the fused path and the fp32 merge leave the canaries as
    # they were
    w = wl.make_config(config, scale=scale)
    dw = DevWorkload(w)
    pad_b = 4096
    canary = 0x5A

    def guarded(nbytes):
        buf = torch.full((nbytes + 2 * pad_b,), canary, dtype=torch.uint8, device="cuda")
        return buf, buf[pad_b:pad_b + nbytes]

    def intact(buf, nbytes):
        return bool((buf[:pad_b] == canary).all() and (buf[pad_b + nbytes:] == canary).all())

    plan = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
    nws = (plan.workspace_bytes + 255) // 256 * 256
    wsb, ws = guarded(nws)
    nout, nlse, nf32 = w.B * w.Hq * w.D * 2, w.B * w.Hq * 4, w.B * w.Hq * w.D * 4
    outb, out_raw = guarded(nout)
    lseb, lse_raw = guarded(nlse)
    f32b, f32_raw = guarded(nf32)
    out = out_raw.view(torch.bfloat16).view(w.B, w.Hq, w.D)
    lse = lse_raw.view(torch.float32).view(w.B, w.Hq)
    o32 = f32_raw.view(torch.float32).view(w.B, w.Hq, w.D)
    plan.upload(ws)
    plan.forward(dw.q, dw.k, dw.v, ws)
    plan.merge(ws, out, lse)
    plan.merge_f32(ws, o32, lse)
    plan.attend(dw.q, dw.k, dw.v, ws, out, lse)
    assert plan.device_status(ws) == pad.PA_OK
    torch.cuda.synchronize()
    assert intact(wsb, nws) and intact(outb, nout) and intact(lseb, nlse) and intact(f32b, nf32)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    assert_close(compare(out, lse, ref_o, ref_l), f"canaries config {config}")
    plan.close()
