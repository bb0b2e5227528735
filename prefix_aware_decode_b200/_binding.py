"""ctypes binding of libpa.so (include/pa.h).  Argument marshalling only.

Every step of the decode-attention path (pack, forward, merge) runs inside the
library: the planner in C++ on the host, forward and merge as sm_100a kernels.
Loading fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_NOMEM, PA_ERR_CUDA, PA_ERR_TIMEOUT, PA_ERR_DEVICE = range(7)
PA_PLAN_NO_SHARING = 1 << 0
PA_PLAN_ALWAYS_SHARE = 1 << 1
PA_PLAN_DEBUG_CHECKS = 1 << 2
PA_PLAN_KEEP_PACK = 1 << 3
PA_PLAN_FAULT_DROP_LOAD = 1 << 8

STATUS_NAMES = {0: "PA_OK", 1: "PA_ERR_INVALID", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_NOMEM", 4: "PA_ERR_CUDA",
                5: "PA_ERR_TIMEOUT", 6: "PA_ERR_DEVICE"}


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class PaConfig(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("softmax_scale", ctypes.c_float), ("num_sms", ctypes.c_int32),
                ("max_chunk_tokens", ctypes.c_int32), ("flags", ctypes.c_uint32), ("wait_timeout_us", ctypes.c_int32)]


class PaPlanStats(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_nodes", ctypes.c_int32), ("num_shared_nodes", ctypes.c_int32),
                ("num_kept_shared", ctypes.c_int32), ("num_items", ctypes.c_int32), ("num_segments", ctypes.c_int32),
                ("num_segments_simt", ctypes.c_int32), ("num_segments_mma", ctypes.c_int32),
                ("num_partial_rows", ctypes.c_int32), ("simt_warps", ctypes.c_int32), ("mma_ctas", ctypes.c_int32),
                ("num_tail_pairs", ctypes.c_int32), ("unique_tokens", ctypes.c_int64), ("naive_tokens", ctypes.c_int64), ("read_tokens", ctypes.c_int64),
                ("unique_kv_bytes", ctypes.c_int64), ("read_kv_bytes", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_uint64), ("image_bytes", ctypes.c_uint64), ("plan_us", ctypes.c_double)]


class PaImageHeader(ctypes.Structure):
    _fields_ = ([("magic", ctypes.c_uint32), ("status", ctypes.c_int32), ("fault_a", ctypes.c_int32),
                 ("fault_b", ctypes.c_int32)]
                + [(n, ctypes.c_int32) for n in ("batch", "num_q_heads", "num_kv_heads", "head_dim", "page_size",
                                                 "num_items", "num_segments", "num_segments_simt", "num_segments_mma",
                                                 "simt_warps", "num_partial_rows", "mma_ctas", "num_tail_pairs",
                                                 "mma_next", "num_mix_pairs", "simt_warps_per_cta")]
                + [(n, ctypes.c_uint64) for n in ("off_nodes", "off_segs", "off_pages", "off_queries",
                                                  "off_seg_prows", "off_mma_segs", "off_counters", "off_warp_segs",
                                                  "off_prow_off", "off_tail_pairs", "off_mix_pairs", "off_partial_lse",
                                                  "off_partial_o",
                                                  "image_bytes",
                                                  "workspace_bytes")])


# exported names, in the order pa.h declares them
EXPORTS = ["pa_plan_create", "pa_plan_advance", "pa_plan_create_append", "pa_plan_workspace_size", "pa_plan_upload", "pa_forward", "pa_merge", "pa_merge_f32", "pa_merge_rows", "pa_attend",
           "pa_get_device_status", "pa_plan_get_stats", "pa_plan_host_image", "pa_plan_set_profile_events",
           "pa_decode_step", "pa_attend_noalloc", "pa_plan_destroy", "pa_status_string"]

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it first (python -c 'import __graft_entry__ as g; "
                           "g.build()'); there is no fallback path")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    st = ctypes.c_int
    L.pa_plan_create.argtypes = [ctypes.POINTER(PaConfig), i32, vp, vp, i32, i32, ctypes.POINTER(vp)]
    L.pa_plan_create.restype = st
    L.pa_plan_advance.argtypes = [vp, vp, vp, i32, i32, ctypes.POINTER(vp)]
    L.pa_plan_advance.restype = st
    L.pa_plan_create_append.argtypes = [ctypes.POINTER(PaConfig), i32, vp, vp, vp, i32, i32, ctypes.POINTER(vp)]
    L.pa_plan_create_append.restype = st
    L.pa_plan_workspace_size.argtypes = [vp, ctypes.POINTER(sz)]
    L.pa_plan_workspace_size.restype = st
    L.pa_plan_upload.argtypes = [vp, vp, sz, vp]
    L.pa_plan_upload.restype = st
    L.pa_forward.argtypes = [vp, vp, vp, vp, vp, vp]
    L.pa_forward.restype = st
    L.pa_merge.argtypes = [vp, vp, vp, vp, vp]
    L.pa_merge.restype = st
    L.pa_merge_f32.argtypes = [vp, vp, vp, vp, vp]
    L.pa_merge_f32.restype = st
    L.pa_merge_rows.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    L.pa_merge_rows.restype = st
    L.pa_attend.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
    L.pa_attend.restype = st
    L.pa_get_device_status.argtypes = [vp, vp, vp, ctypes.POINTER(ctypes.c_int)]
    L.pa_get_device_status.restype = st
    L.pa_plan_get_stats.argtypes = [vp, ctypes.POINTER(PaPlanStats)]
    L.pa_plan_get_stats.restype = st
    L.pa_plan_host_image.argtypes = [vp, vp, sz]
    L.pa_plan_host_image.restype = st
    L.pa_plan_set_profile_events.argtypes = [vp, ctypes.POINTER(vp), i32]
    L.pa_plan_set_profile_events.restype = st
    L.pa_decode_step.argtypes = [ctypes.POINTER(PaConfig), i32, vp, vp, i32, i32, vp, vp, vp, vp, sz, vp, sz, vp,
                                 vp, ctypes.POINTER(vp), vp, ctypes.POINTER(vp)]
    L.pa_decode_step.restype = st
    L.pa_attend_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp]
    L.pa_attend_noalloc.restype = st
    L.pa_plan_destroy.argtypes = [vp]
    L.pa_plan_destroy.restype = None
    L.pa_status_string.argtypes = [st]
    L.pa_status_string.restype = ctypes.c_char_p
    _lib = L
    return L


def _check(status: int, where: str):
    if status != PA_OK:
        raise PaError(status, where)


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _host_ptr(a: np.ndarray) -> int:
    """Address of a host array's data (the buffer protocol: a fraction of the
    cost of ndarray.ctypes per call)."""
    try:
        return ctypes.addressof(ctypes.c_char.from_buffer(a))
    except (TypeError, ValueError, BufferError):  # read-only or empty arrays
        return a.ctypes.data


def _host_i32(a, ndim: int) -> np.ndarray:
    """a as a C-contiguous int32 array of `ndim` dimensions (no copy when it is one)."""
    if not (isinstance(a, np.ndarray) and a.dtype == np.int32 and a.flags.c_contiguous):
        a = np.ascontiguousarray(a, dtype=np.int32)
    if a.ndim != ndim:
        raise ValueError(f"expected a {ndim}-d host array, got {a.ndim}-d")
    return a


def _dptr(t, name: str, align: int = 16) -> int:
    p = t.data_ptr()
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if p % align:
        raise ValueError(f"{name} must be {align}-byte aligned")
    return p


class Plan:
    """A pack-stage plan for one decode batch (wraps pa_plan)."""

    def __init__(self, kv_lens, block_table, num_pages: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 page_size: int = 16, softmax_scale: float = 0.0, num_sms: int = 0, max_chunk_tokens: int = 0,
                 flags: int = 0, wait_timeout_us: int = 0):
        self._lib = lib()
        self._h = None
        kv = np.ascontiguousarray(kv_lens, dtype=np.int32)
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        if bt.ndim != 2 or kv.ndim != 1 or bt.shape[0] != kv.shape[0]:
            raise ValueError("block_table must be [B][max_pages] and kv_lens [B]")
        cfg = PaConfig(num_q_heads, num_kv_heads, head_dim, page_size, softmax_scale, num_sms, max_chunk_tokens,
                       flags, wait_timeout_us)
        h = ctypes.c_void_p()
        _check(self._lib.pa_plan_create(ctypes.byref(cfg), kv.shape[0], _host_ptr(kv), _host_ptr(bt),
                                        bt.shape[1], int(num_pages), ctypes.byref(h)), "pa_plan_create")
        self._h = h
        self.B, self.Hq, self.Hkv, self.D = int(kv.shape[0]), num_q_heads, num_kv_heads, head_dim

    @classmethod
    def append(cls, ctx_lens, chunk_lens, block_table, num_pages: int, num_q_heads: int, num_kv_heads: int,
               head_dim: int, page_size: int = 16, softmax_scale: float = 0.0, num_sms: int = 0,
               max_chunk_tokens: int = 0, flags: int = 0, wait_timeout_us: int = 0) -> "Plan":
        """Plan for chunks of new tokens appended to sessions
        (pa_plan_create_append): one row per new token, sessions in order;
        row i of session s attends over tokens 0 .. ctx_lens[s] + i."""
        ctx = np.ascontiguousarray(ctx_lens, dtype=np.int32)
        ch = np.ascontiguousarray(chunk_lens, dtype=np.int32)
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        if bt.ndim != 2 or ctx.ndim != 1 or ch.shape != ctx.shape or bt.shape[0] != ctx.shape[0]:
            raise ValueError("block_table must be [S][max_pages], ctx_lens and chunk_lens [S]")
        self = cls.__new__(cls)
        self._lib = lib()
        cfg = PaConfig(num_q_heads, num_kv_heads, head_dim, page_size, softmax_scale, num_sms, max_chunk_tokens,
                       flags, wait_timeout_us)
        h = ctypes.c_void_p()
        _check(self._lib.pa_plan_create_append(ctypes.byref(cfg), ctx.shape[0], ctx.ctypes.data, ch.ctypes.data,
                                               bt.ctypes.data, bt.shape[1], int(num_pages), ctypes.byref(h)),
               "pa_plan_create_append")
        self._h = h
        self.B, self.Hq, self.Hkv, self.D = int(ch.sum()), num_q_heads, num_kv_heads, head_dim
        return self

    def advance(self, kv_lens, block_table, num_pages: int) -> "Plan":
        """The next decode step's plan of the same batch (pa_plan_advance): this
        plan must have been made with PA_PLAN_KEEP_PACK; the first
        ceil(old kv_len / page_size) entries of every row must be unchanged."""
        kv = np.ascontiguousarray(kv_lens, dtype=np.int32)
        bt = np.ascontiguousarray(block_table, dtype=np.int32)
        if bt.ndim != 2 or kv.ndim != 1 or bt.shape[0] != kv.shape[0] or kv.shape[0] != self.B:
            raise ValueError("block_table must be [B][max_pages] and kv_lens [B], B as before")
        h = ctypes.c_void_p()
        _check(self._lib.pa_plan_advance(self._h, _host_ptr(kv), _host_ptr(bt), bt.shape[1], int(num_pages),
                                         ctypes.byref(h)), "pa_plan_advance")
        nxt = Plan.__new__(Plan)
        nxt._lib, nxt._h = self._lib, h
        nxt.B, nxt.Hq, nxt.Hkv, nxt.D = self.B, self.Hq, self.Hkv, self.D
        return nxt

    def close(self):
        if self._h is not None and self._h.value:
            self._lib.pa_plan_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    def stats(self) -> dict:
        s = PaPlanStats()
        _check(self._lib.pa_plan_get_stats(self._h, ctypes.byref(s)), "pa_plan_get_stats")
        return {n: getattr(s, n) for n, _ in PaPlanStats._fields_}

    @property
    def workspace_bytes(self) -> int:
        n = ctypes.c_size_t()
        _check(self._lib.pa_plan_workspace_size(self._h, ctypes.byref(n)), "pa_plan_workspace_size")
        return n.value

    def host_image(self) -> np.ndarray:
        n = self.stats()["image_bytes"]
        buf = np.zeros(n, dtype=np.uint8)
        _check(self._lib.pa_plan_host_image(self._h, buf.ctypes.data, n), "pa_plan_host_image")
        return buf

    def alloc_workspace(self, device=None):
        import torch
        n = (self.workspace_bytes + 255) // 256 * 256
        return torch.empty(n, dtype=torch.uint8, device=device or "cuda")

    def upload(self, ws, stream=None):
        _check(self._lib.pa_plan_upload(self._h, _dptr(ws, "workspace", 256), ws.numel() * ws.element_size(),
                                        _stream_ptr(stream)), "pa_plan_upload")

    def forward(self, q, k_pool, v_pool, ws, stream=None):
        _check(self._lib.pa_forward(self._h, _dptr(q, "q"), _dptr(k_pool, "k_pool"), _dptr(v_pool, "v_pool"),
                                    _dptr(ws, "workspace", 256), _stream_ptr(stream)), "pa_forward")

    def merge(self, ws, out, lse=None, stream=None):
        _check(self._lib.pa_merge(self._h, _dptr(ws, "workspace", 256), _dptr(out, "out"),
                                  _dptr(lse, "lse", 4) if lse is not None else None, _stream_ptr(stream)),
               "pa_merge")

    def merge_f32(self, ws, out, lse=None, stream=None):
        """pa_merge_f32: out fp32 [B][Hq][D], not rounded (a rank's part of a
        context-parallel batch)."""
        _check(self._lib.pa_merge_f32(self._h, _dptr(ws, "workspace", 256), _dptr(out, "out"),
                                      _dptr(lse, "lse", 4) if lse is not None else None, _stream_ptr(stream)),
               "pa_merge_f32")

    def attend(self, q, k_pool, v_pool, ws, out, lse=None, stream=None):
        _check(self._lib.pa_attend(self._h, _dptr(q, "q"), _dptr(k_pool, "k_pool"), _dptr(v_pool, "v_pool"),
                                   _dptr(ws, "workspace", 256), _dptr(out, "out"),
                                   _dptr(lse, "lse", 4) if lse is not None else None, _stream_ptr(stream)),
               "pa_attend")

    def set_profile_events(self, events):
        """events: up to four torch.cuda.Event (or None), see pa_plan_set_profile_events."""
        self._prof_events = list(events)  # keep them alive
        arr = (ctypes.c_void_p * 4)()
        for i, e in enumerate(self._prof_events):
            arr[i] = None if e is None else e.cuda_event
        _check(self._lib.pa_plan_set_profile_events(self._h, arr, len(self._prof_events)),
               "pa_plan_set_profile_events")

    def attend_noalloc(self, q, k_pool, v_pool, out, lse=None, stream=None):
        """pa_attend with the library's static device workspace (no allocation)."""
        _check(self._lib.pa_attend_noalloc(self._h, _dptr(q, "q"), _dptr(k_pool, "k_pool"), _dptr(v_pool, "v_pool"),
                                           _dptr(out, "out"), _dptr(lse, "lse", 4) if lse is not None else None,
                                           _stream_ptr(stream)), "pa_attend_noalloc")

    def device_status(self, ws, stream=None) -> int:
        """The device status word of the workspace `ws`; ws=None reads the
        static workspace of attend_noalloc."""
        out = ctypes.c_int()
        _check(self._lib.pa_get_device_status(self._h, _dptr(ws, "workspace", 256) if ws is not None else None,
                                              _stream_ptr(stream), ctypes.byref(out)), "pa_get_device_status")
        return out.value


def merge_rows(part_req, part_o, part_lse, batch: int, out, lse=None, stream=None):
    """pa_merge_rows: combine rows gathered from several parts of the KV.
    part_req int32 [P][R] (ascending, -1 padding last), part_o fp32 [P][R][Hq][D],
    part_lse fp32 [P][R][Hq] (CUDA tensors); out bf16 [batch][Hq][D]."""
    P, R = part_req.shape
    Hq, D = part_o.shape[2], part_o.shape[3]
    _check(lib().pa_merge_rows(P, R, batch, Hq, D, _dptr(part_req, "part_req", 4), _dptr(part_o, "part_o"),
                               _dptr(part_lse, "part_lse", 4), _dptr(out, "out"),
                               _dptr(lse, "lse", 4) if lse is not None else None, _stream_ptr(stream)),
           "pa_merge_rows")


def attend(q, k_pool, v_pool, block_table, kv_lens, softmax_scale: float = 0.0, flags: int = 0,
           max_chunk_tokens: int = 0, return_lse: bool = True, stream=None):
    """One decode step: plan on the host, then forward + merge on the GPU.

    q bf16 [B][Hq][D], k_pool/v_pool bf16 [num_pages][Hkv][P][D] (CUDA tensors);
    block_table int32 [B][max_pages] and kv_lens int32 [B] (host arrays or CPU tensors).
    Returns (out bf16 [B][Hq][D], lse fp32 [B][Hq]).
    """
    import torch
    B, Hq, D = q.shape
    num_pages, Hkv, P, _ = k_pool.shape
    bt = block_table.cpu().numpy() if hasattr(block_table, "cpu") else block_table
    kl = kv_lens.cpu().numpy() if hasattr(kv_lens, "cpu") else kv_lens
    plan = Plan(kl, bt, num_pages, Hq, Hkv, D, P, softmax_scale=softmax_scale, flags=flags,
                max_chunk_tokens=max_chunk_tokens)
    ws = plan.alloc_workspace(q.device)
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if return_lse else None
    plan.upload(ws, stream)
    plan.attend(q, k_pool, v_pool, ws, out, lse, stream)
    torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
    plan.close()
    return out, lse


class DecodeStep:
    """Repeated decode steps through pa_decode_step (one C call per step).

    The fixed arguments (shapes, pools, workspace, image buffer, outputs) are
    marshalled once; each call passes the step's kv_lens / block_table (host
    arrays).  `images` is the device buffer whose two halves hold the plan
    images of consecutive steps (allocated here, image_bytes per half, when
    not given).
    """

    def __init__(self, num_pages, num_q_heads, num_kv_heads, head_dim, q, k_pool, v_pool, workspace, out, lse=None,
                 page_size=16, softmax_scale=0.0, flags=0, max_chunk_tokens=0, stream=None, images=None,
                 image_bytes=8 << 20):
        import torch
        self._lib = lib()
        self.cfg = PaConfig(num_q_heads, num_kv_heads, head_dim, page_size, softmax_scale, 0, max_chunk_tokens,
                            flags, 0)
        self.num_pages = int(num_pages)
        if images is None:
            images = torch.empty(2 * ((image_bytes + 255) // 256 * 256), dtype=torch.uint8, device=q.device)
        self.images = images
        self.args = (_dptr(q, "q"), _dptr(k_pool, "k_pool"), _dptr(v_pool, "v_pool"),
                     _dptr(workspace, "workspace", 256), workspace.numel() * workspace.element_size(),
                     _dptr(images, "images", 256), images.numel() * images.element_size(),
                     _dptr(out, "out"), _dptr(lse, "lse", 4) if lse is not None else None)
        self.stream = _stream_ptr(stream)
        self._events = None

    def set_pools(self, k_pool, v_pool):
        a = list(self.args)
        a[1], a[2] = _dptr(k_pool, "k_pool"), _dptr(v_pool, "v_pool")
        self.args = tuple(a)

    def __call__(self, kv_lens: np.ndarray, block_table: np.ndarray, events=None):
        ev = None
        if events is not None:
            self._events = (ctypes.c_void_p * 4)(*[e.cuda_event if e is not None else None for e in events])
            ev = self._events
        q, k, v, ws, wsb, im, imb, out, lse = self.args
        kv_lens, block_table = _host_i32(kv_lens, 1), _host_i32(block_table, 2)
        if block_table.shape[0] != kv_lens.shape[0]:
            raise ValueError("block_table must be [B][max_pages] and kv_lens [B]")
        _check(self._lib.pa_decode_step(ctypes.byref(self.cfg), kv_lens.shape[0], _host_ptr(kv_lens),
                                        _host_ptr(block_table), block_table.shape[1], self.num_pages, q, k, v,
                                        ws, wsb, im, imb, out, lse, ev, self.stream, None), "pa_decode_step")
