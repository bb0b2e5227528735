"""Helpers for the GPU parity tests: device copies of a workload, the CUDA path
through the C ABI, and the comparison against the fp64 oracle."""
import numpy as np
import torch

import prefix_aware_decode_b200 as pad

# Tolerances on bf16 outputs and fp32 lse against the fp64 oracle.
#
# Absolute: |g - o| <= max(MAX_ABS, half_ulp_bf16(|o|) + FP32_SLACK * max(1, |o|)).
# The kernels produce an fp32 value y and round it to bf16 (round to nearest
# even), so |g - o| <= half_ulp(y) + |y - o|.  Below |o| = 1 half an ulp is at
# most 2^-9 = 1.953e-3 and the bound is exactly MAX_ABS, as long as the fp32
# error |y - o| stays under 2^-15 (3.05e-5); at |o| >= 1 the bf16 rounding of
# the output alone exceeds 2e-3, so there the bound is that rounding plus the
# same fp32 slack, relative.  FP32_SLACK covers the tensor-core class's split
# of p into two bf16 terms (each weight kept to 2^-16 relative, unbiased) and
# fp32 accumulation; the CUDA-core class is far inside it.
MAX_ABS = 2e-3
FP32_SLACK = 2.0 ** -15
MAX_REL = 1e-2   # |g - o| / max(|o|, rms of the (request, head) row of o)
MAX_LSE = 1e-4


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers (8 significant bits) at |x|: 2^(e - 8)
    for |x| in [2^e, 2^(e+1))."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def abs_bound(ref_o: np.ndarray) -> np.ndarray:
    a = np.abs(ref_o)
    return np.maximum(MAX_ABS, half_ulp_bf16(a) + FP32_SLACK * np.maximum(1.0, a))


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
    small = np.abs(ref_o) < 1.0
    return dict(max_abs=float(err.max()), max_rel=float(rel.max()), max_lse=float(np.abs(gl - ref_l).max()),
                abs_over_bound=float((err / abs_bound(ref_o)).max()),
                max_abs_below_1=float(err[small].max()) if small.any() else 0.0,
                finite=bool(np.isfinite(g).all() and np.isfinite(gl).all()),
                rel_unfloored=float((err / np.maximum(np.abs(ref_o), 1e-30)).max()),
                rel_rownorm=float((np.linalg.norm(g - ref_o, axis=-1) / np.linalg.norm(ref_o, axis=-1)).max()),
                n_rows=int(ref_o.shape[0] * ref_o.shape[1]))


def report(m: dict, what: str):
    print(f"[parity] {what}: abs_over_bound={m['abs_over_bound']:.3f} max_abs={m['max_abs']:.2e} "
          f"max_abs(|o|<1)={m['max_abs_below_1']:.2e} max_rel={m['max_rel']:.2e} max_lse={m['max_lse']:.2e} "
          f"rows={m['n_rows']}")


def assert_close(m: dict, what: str = ""):
    report(m, what)
    assert m["finite"], f"{what}: non-finite output {m}"
    assert m["abs_over_bound"] <= 1.0, f"{what}: max abs {m}"
    assert m["max_abs_below_1"] <= MAX_ABS, f"{what}: max abs where |o| < 1 {m}"
    assert m["max_rel"] <= MAX_REL, f"{what}: max rel {m}"
    assert m["max_lse"] <= MAX_LSE, f"{what}: lse {m}"
