"""Helpers for the GPU parity tests: device copies of a workload, the CUDA path
through the C ABI, and the comparison against the fp64 oracle."""
import numpy as np
import torch

import prefix_aware_decode_b200 as pad

# Tolerances on bf16 outputs and fp32 lse against the fp64 oracle.
MAX_ABS = 2e-3   # absolute, where |o| <= 0.256; above that the bound is one bf16 ulp,
                 # 2^-7 |o|: the output rounding (half an ulp) plus the bf16 rounding of
                 # p in the tensor-core p.V product (2^-9 relative per weight)
MAX_REL = 1e-2   # |g - o| / max(|o|, rms of the (request, head) row of o)
MAX_LSE = 1e-4


def bf16_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


class DevWorkload:
    def __init__(self, w):
        self.w = w
        self.q = bf16_dev(w.q)
        self.k = bf16_dev(w.k_pool)
        self.v = bf16_dev(w.v_pool)


def run(dw: DevWorkload, flags=0, max_chunk_tokens=0, wait_timeout_us=0, check_status=True, fused=False):
    """Plan + upload + forward + merge through the C ABI; returns (out, lse, plan stats, status).

    fused: pa_attend (merge inside the forward launches, plus the tail merge
    launch) instead of pa_forward followed by pa_merge."""
    w = dw.w
    plan = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D, flags=flags,
                    max_chunk_tokens=max_chunk_tokens, wait_timeout_us=wait_timeout_us)
    ws = plan.alloc_workspace()
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    plan.upload(ws)
    if fused:
        plan.attend(dw.q, dw.k, dw.v, ws, out, lse)
    else:
        plan.forward(dw.q, dw.k, dw.v, ws)
        plan.merge(ws, out, lse)
    status = plan.device_status(ws)
    torch.cuda.synchronize()
    if check_status:
        assert status == pad.PA_OK, pad._binding.STATUS_NAMES.get(status)
    st = plan.stats()
    plan.close()
    return out, lse, st, status


def compare(out: torch.Tensor, lse: torch.Tensor, ref_o: np.ndarray, ref_l: np.ndarray, queries=None) -> dict:
    g = out.float().cpu().numpy().astype(np.float64)
    gl = lse.cpu().numpy().astype(np.float64)
    if queries is not None:
        g, gl = g[queries], gl[queries]
    err = np.abs(g - ref_o)
    rms = np.sqrt(np.mean(ref_o ** 2, axis=-1, keepdims=True))
    rel = err / np.maximum(np.abs(ref_o), rms)
    abs_bound = np.maximum(MAX_ABS, np.abs(ref_o) * 2.0 ** -7)
    return dict(max_abs=float(err.max()), max_rel=float(rel.max()), max_lse=float(np.abs(gl - ref_l).max()),
                abs_over_bound=float((err / abs_bound).max()),
                finite=bool(np.isfinite(g).all() and np.isfinite(gl).all()),
                rel_unfloored=float((err / np.maximum(np.abs(ref_o), 1e-30)).max()),
                rel_rownorm=float((np.linalg.norm(g - ref_o, axis=-1) / np.linalg.norm(ref_o, axis=-1)).max()))


def assert_close(m: dict, what: str = ""):
    assert m["finite"], f"{what}: non-finite output {m}"
    assert m["abs_over_bound"] <= 1.0, f"{what}: max abs {m}"
    assert m["max_rel"] <= MAX_REL, f"{what}: max rel {m}"
    assert m["max_lse"] <= MAX_LSE, f"{what}: lse {m}"
