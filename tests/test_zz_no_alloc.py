"""pa_attend_noalloc: the fused forward on the library's static device
workspace, for callers that cannot allocate device memory where they run
attention.  Checked against the caller-workspace entry point pa_attend on two
calls in a row (the array keeps the previous call's contents, so the second
call also checks that the plan upload resets what must start at zero).

This file is collected last, so a run that stops at its first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import prefix_aware_decode_b200 as pad
from prefix_aware_decode_b200 import workload as wl

from gpu_util import DevWorkload, assert_close, compare

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("config,scale", [(1, 1.0), (2, 0.25)])
def test_noalloc_matches_workspace_entry_point(config, scale):
    dw = DevWorkload(wl.make_config(config, scale=scale))
    w = dw.w
    plan = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
    ws = plan.alloc_workspace()
    ref = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    plan.upload(ws)
    plan.attend(dw.q, dw.k, dw.v, ws, ref, ref_lse)
    torch.cuda.synchronize()
    ref_np = ref.float().cpu().numpy().astype(np.float64)
    ref_lse_np = ref_lse.cpu().numpy().astype(np.float64)
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        plan.attend_noalloc(dw.q, dw.k, dw.v, out, lse)
        torch.cuda.synchronize()
        assert_close(compare(out, lse, ref_np, ref_lse_np), f"noalloc config {config}")
    plan.close()


def test_noalloc_refuses_plans_beyond_its_array():
    # 64 requests x 2048 tokens with every page its own work unit: the fp32
    # partial rows alone need far more than 24 MiB
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
