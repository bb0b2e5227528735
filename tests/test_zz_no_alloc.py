"""pa_attend_noalloc: the fused forward on the library's static device
workspace, for callers that cannot allocate device memory at the point where
they run attention (a memory pool that refuses further allocation, an
allocator-free runtime, a hook that must not touch the caching allocator).

The entry point runs the same kernels on the same plan image as pa_attend, so
its results must equal pa_attend's bit for bit; they are also checked against
the fp64 oracle.  Each case makes two calls in a row: the array keeps the
previous call's contents, so the second call also checks that each call resets
what must start at zero (status word, arrival counters).

This file is collected last, so a run that stops at its first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
import prefix_aware_decode_b200 as pad
from prefix_aware_decode_b200 import workload as wl

from gpu_util import DevWorkload, assert_close, compare

pytestmark = pytest.mark.gpu


def _workspace_result(plan, dw):
    w = dw.w
    ws = plan.alloc_workspace()
    ref = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    plan.upload(ws)
    plan.attend(dw.q, dw.k, dw.v, ws, ref, ref_lse)
    torch.cuda.synchronize()
    assert plan.device_status(ws) == pad.PA_OK
    return ref, ref_lse


def _check_noalloc(plan, dw, ref, ref_lse, ref_o, ref_l, what):
    w = dw.w
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        plan.attend_noalloc(dw.q, dw.k, dw.v, out, lse)
        torch.cuda.synchronize()
        assert plan.device_status(None) == pad.PA_OK
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"{what}: out differs (call {call})"
        assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32)), f"{what}: lse differs (call {call})"
        assert_close(compare(out, lse, ref_o, ref_l), f"{what} call {call}")


@pytest.mark.parametrize("config,scale", [(1, 1.0), (2, 0.25)])
def test_noalloc_equals_workspace_entry_point(config, scale):
    dw = DevWorkload(wl.make_config(config, scale=scale))
    w = dw.w
    plan = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
    ref, ref_lse = _workspace_result(plan, dw)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    _check_noalloc(plan, dw, ref, ref_lse, ref_o, ref_l, f"noalloc config {config}")
    plan.close()


def test_noalloc_on_an_advanced_plan():
    # a plan carried over by pa_plan_advance (every request one token longer)
    base = wl.make_config(2, scale=0.25)
    rng = np.random.default_rng(5)
    k, v = base.k_pool.copy(), base.v_pool.copy()
    kv = base.kv_lens.astype(np.int32).copy()
    bt = base.block_table.copy()
    first = pad.Plan(kv, bt, base.num_pages, base.Hq, base.Hkv, base.D, flags=pad.PA_PLAN_KEEP_PACK)
    grow = kv % base.P != 0  # room left in the last page: the new token goes there
    for b in np.nonzero(grow)[0]:
        page, slot = bt[b, kv[b] // base.P], kv[b] % base.P
        k[page, :, slot, :] = (rng.normal(size=(base.Hkv, base.D)).astype(np.float32).view(np.uint32) >> 16)
        v[page, :, slot, :] = (rng.normal(size=(base.Hkv, base.D)).astype(np.float32).view(np.uint32) >> 16)
    kv = kv + grow.astype(np.int32)
    plan = first.advance(kv, bt, base.num_pages)
    first.close()
    w = wl.Workload(**{**base.__dict__, "k_pool": k, "v_pool": v, "kv_lens": kv})
    dw = DevWorkload(w)
    ref, ref_lse = _workspace_result(plan, dw)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    _check_noalloc(plan, dw, ref, ref_lse, ref_o, ref_l, "noalloc advanced plan")
    plan.close()


def test_noalloc_status_reports_a_timeout_then_recovers():
    # one load is left out on purpose, so the kernel's bounded wait gives up
    # after 20 ms and records PA_ERR_TIMEOUT in the static array; the status is
    # read through pa_get_device_status with no workspace, and the next call on
    # the same array is correct again
    dw = DevWorkload(wl.make_config(1))
    w = dw.w
    bad = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D,
                   flags=pad.PA_PLAN_FAULT_DROP_LOAD, wait_timeout_us=20000)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    bad.attend_noalloc(dw.q, dw.k, dw.v, out)
    torch.cuda.synchronize()
    assert bad.device_status(None) == pad.PA_ERR_TIMEOUT
    bad.close()
    plan = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
    ref, ref_lse = _workspace_result(plan, dw)
    ref_o, ref_l = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    _check_noalloc(plan, dw, ref, ref_lse, ref_o, ref_l, "noalloc after a timeout")
    plan.close()


def test_noalloc_refuses_plans_beyond_its_array():
    # 64 requests x 2048 tokens with every page its own work unit: the fp32
    # partial rows alone need far more than the array's 24 MiB
    roots = [wl.Node(2048) for _ in range(64)]
    w = wl.build_workload("big", roots, Hq=32, Hkv=8, D=128, seed=3, with_values=False)
    plan = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D, max_chunk_tokens=16)
    assert plan.workspace_bytes > 24 << 20
    q = torch.zeros((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((1, w.Hkv, 16, w.D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(pad.PaError) as e:
        plan.attend_noalloc(q, pool, pool, out)
    assert e.value.status == pad.PA_ERR_NOMEM
    plan.close()
