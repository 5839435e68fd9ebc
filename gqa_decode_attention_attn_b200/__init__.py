"""B200 (sm_100a) decode-time grouped-query attention.

Thin Python binding over the C ABI in ``include/gqa_decode.h``
(``lib/libgqa_decode_b200.so``).  This module only marshals torch tensors into
pointers and sizes; every step of the computation runs in the library's CUDA
kernels.  There is no fallback: if the library is missing or a CUDA device is
absent, calls raise.

    out = gqa_decode(q, k_cache, v_cache, block_table, seq_lens)

q [B, Hq, D] bf16; caches [num_blocks, Hkv, block_size, D] bf16 (paged, with
block_table [B, max_blocks] int32) or [B, Hkv, capacity, D] (block_table=None);
seq_lens [B] int32 -- all on the same CUDA device.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libgqa_decode_b200.so")

GQA_OK = 0
GQA_ERR_WORKSPACE_TOO_SMALL = 3
DEV_BAD_BLOCK = 1
DEV_BAD_LENGTH = 2
DEV_TIMEOUT = 4

EXPORTED = ("gqa_decode_workspace_size", "gqa_decode", "gqa_decode_states", "gqa_merge_states",
            "gqa_status", "gqa_decode_host_buffer_bytes", "gqa_decode_host", "gqa_error_string",
            "gqa_decode_noalloc", "gqa_decode_fixed_split_workspace_size",
            "gqa_decode_fixed_split", "gqa_select_schedule", "gqa_decode_auto",
            "gqa_decode_multi", "gqa_decode_fp8", "gqa_decode_fp8_auto", "gqa_decode_timeline",
            "gqa_decode_plan", "gqa_set_wait_limit", "gqa_stream_floor")
GQA_ERR_SCRATCH_LIMIT = 6
TIMELINE_COLS = 8  # values per CTA row of gqa_decode_timeline
KERNEL_TENSOR_CORE = 1
KERNEL_CUDA_CORE = 2


class _Plan(ctypes.Structure):
    """gqa_plan of include/gqa_decode.h."""
    _fields_ = [("kernel", ctypes.c_int), ("heads_per_pass", ctypes.c_int),
                ("head_chunks", ctypes.c_int), ("num_splits", ctypes.c_int),
                ("grid", ctypes.c_int), ("threads_per_cta", ctypes.c_int),
                ("cooperative", ctypes.c_int), ("merge_launch", ctypes.c_int),
                ("tile_tokens", ctypes.c_int), ("ring_stages", ctypes.c_int),
                ("box_rows", ctypes.c_int), ("tiles", ctypes.c_longlong),
                ("smem_bytes", ctypes.c_size_t), ("workspace_bytes", ctypes.c_size_t),
                ("kernel_name", ctypes.c_char * 64)]

_lib = None


class GqaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn}: {error_string(code)} (code {code})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m gqa_decode_attention_attn_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.gqa_decode_workspace_size.argtypes = [I, I, I, I, I, ctypes.POINTER(SZ)]
    lib.gqa_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, SZ, P]
    lib.gqa_decode_states.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, SZ, P]
    lib.gqa_merge_states.argtypes = [P, P, P, I, I, I, P, P, P]
    lib.gqa_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint)]
    lib.gqa_decode_host_buffer_bytes.argtypes = [I, I, I, I, I, I, I, I]
    lib.gqa_decode_host_buffer_bytes.restype = SZ
    lib.gqa_decode_host.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, SZ, P, SZ, P]
    lib.gqa_decode_fixed_split_workspace_size.argtypes = [I, I, I, I, I, I, ctypes.POINTER(SZ)]
    lib.gqa_decode_fixed_split.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, I, P, SZ, P]
    lib.gqa_select_schedule.argtypes = [I, I, I, I, P, I, I, ctypes.POINTER(I), P]
    lib.gqa_decode_auto.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, I, I, P, SZ, P]
    lib.gqa_decode_multi.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, P, SZ, P]
    lib.gqa_decode_fp8.argtypes = [P, P, P, F, F, P, P, P, I, I, I, I, I, F, I, I, P, SZ, P]
    lib.gqa_decode_fp8_auto.argtypes = [P, P, P, F, F, P, P, P, P, I, I, I, I, I, F, I, I, P, SZ,
                                        P]
    lib.gqa_decode_timeline.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, I, P, I,
                                        ctypes.POINTER(I), P, SZ, P]
    lib.gqa_decode_plan.argtypes = [I, I, I, I, I, I, I, I, I, I, P, I, ctypes.POINTER(_Plan)]
    lib.gqa_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, P]
    lib.gqa_set_wait_limit.argtypes = [ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_ulonglong)]
    lib.gqa_stream_floor.argtypes = [P, P, ctypes.c_longlong, I, P, SZ, P]
    lib.gqa_error_string.argtypes = [I]
    lib.gqa_error_string.restype = ctypes.c_char_p
    for name in ("gqa_decode_workspace_size", "gqa_decode", "gqa_decode_states",
                 "gqa_merge_states", "gqa_status", "gqa_decode_host",
                 "gqa_decode_fixed_split_workspace_size", "gqa_decode_fixed_split",
                 "gqa_select_schedule", "gqa_decode_auto", "gqa_decode_multi",
                 "gqa_decode_fp8", "gqa_decode_fp8_auto", "gqa_decode_plan", "gqa_decode_noalloc",
                 "gqa_decode_timeline", "gqa_set_wait_limit", "gqa_stream_floor"):
        getattr(lib, name).restype = I
    _lib = lib
    return lib


def set_wait_limit(ns: int) -> int:
    """Limit of each in-kernel wait for progress, for launches from now on (0: the
    default 1.5 s); returns the previous limit in ns (gqa_set_wait_limit)."""
    prev = ctypes.c_ulonglong(0)
    _check("gqa_set_wait_limit", load_library().gqa_set_wait_limit(int(ns), ctypes.byref(prev)))
    return prev.value


FLOOR_TILE_BYTES = 128 * 256  # one 128-row tile of 256-byte rows (gqa_stream_floor)


def stream_floor(k: torch.Tensor, v: torch.Tensor, nbytes: int, ctas: int,
                 workspace: Optional[Workspace] = None, stream=None) -> None:
    """Stream the first `nbytes` bytes of k and of v (a multiple of FLOOR_TILE_BYTES)
    through the decode kernels' TMA rings with no arithmetic, over `ctas` CTAs: the
    measurement reference of gqa_stream_floor.  Asynchronous; a wait that ran out
    shows in workspace.status()."""
    lib = load_library()
    dev = k.device
    for t, n in ((k, "k"), (v, "v")):
        if t.device != dev or dev.type != "cuda":
            raise ValueError(f"{n} must be a CUDA tensor on {dev}")
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
        if nbytes > t.numel() * t.element_size():
            raise ValueError(f"{n} holds fewer than {nbytes} bytes")
    if nbytes <= 0 or nbytes % FLOOR_TILE_BYTES:
        raise ValueError(f"nbytes must be a positive multiple of {FLOOR_TILE_BYTES}")
    ws = workspace or default_workspace(dev)
    buf = ws.get(256)
    _check("gqa_stream_floor", lib.gqa_stream_floor(_ptr(k), _ptr(v), nbytes // 256, int(ctas),
                                                    _ptr(buf), buf.numel(), _stream_ptr(stream)))


def error_string(code: int) -> str:
    return load_library().gqa_error_string(int(code)).decode()


def _check(fn: str, rc: int) -> None:
    if rc != GQA_OK:
        raise GqaError(fn, rc)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _shape(q, k_cache, block_table):
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [B, Hq, D] and caches [blocks, Hkv, block_size, D]")
    B, Hq, D = q.shape
    nb, Hkv, bs, D2 = k_cache.shape
    if D2 != D:
        raise ValueError("head_dim of q and the cache differ")
    mb = 0 if block_table is None else block_table.shape[1]
    return B, Hq, Hkv, D, bs, mb, nb


def _require(t: torch.Tensor, name: str, dtype, device) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_size(B: int, Hq: int, Hkv: int, D: int, device: int | None = None) -> int:
    lib = load_library()
    dev = torch.cuda.current_device() if device is None else int(device)
    out = ctypes.c_size_t(0)
    _check("gqa_decode_workspace_size", lib.gqa_decode_workspace_size(B, Hq, Hkv, D, dev,
                                                                      ctypes.byref(out)))
    return out.value


class Workspace:
    """A zero-initialised device workspace that grows on demand (one per device and
    stream; calls sharing it must not overlap on the GPU)."""

    def __init__(self, device=None):
        self.device = torch.device("cuda", torch.cuda.current_device() if device is None
                                   else torch.device(device).index)
        self.buf = torch.zeros(0, dtype=torch.uint8, device=self.device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        return self.buf

    def status(self, stream=None) -> int:
        """Device status bits since the last call (synchronises the stream)."""
        lib = load_library()
        v = ctypes.c_uint(0)
        _check("gqa_status", lib.gqa_status(_ptr(self.buf), _stream_ptr(stream), ctypes.byref(v)))
        return v.value


_workspaces: dict = {}


def default_workspace(device) -> Workspace:
    key = (torch.device(device).index, torch.cuda.current_stream(device).cuda_stream)
    if key not in _workspaces:
        _workspaces[key] = Workspace(device)
    return _workspaces[key]


def gqa_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
               block_table: Optional[torch.Tensor], seq_lens: torch.Tensor,
               out: Optional[torch.Tensor] = None, scale: Optional[float] = None,
               workspace: Optional[Workspace] = None, stream=None) -> torch.Tensor:
    """Decode attention; returns out [B, Hq, D] bf16 (see include/gqa_decode.h)."""
    lib = load_library()
    B, Hq, Hkv, D, bs, mb, nb = _shape(q, k_cache, block_table)
    dev = q.device
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _require(t, n, torch.bfloat16, dev)
    _require(seq_lens, "seq_lens", torch.int32, dev)
    if block_table is not None:
        _require(block_table, "block_table", torch.int32, dev)
    if out is None:
        out = torch.empty_like(q)
    _require(out, "out", torch.bfloat16, dev)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws = default_workspace(dev) if workspace is None else workspace
    buf = ws.get(workspace_size(B, Hq, Hkv, D, dev.index))
    with torch.cuda.device(dev):
        rc = lib.gqa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                            _ptr(seq_lens), _ptr(out), B, Hq, Hkv, D, bs, scale, mb, nb,
                            _ptr(buf), buf.numel(), _stream_ptr(stream))
    _check("gqa_decode", rc)
    return out


def fixed_split_workspace_size(B: int, Hq: int, Hkv: int, D: int, num_splits: int,
                               device: int | None = None) -> int:
    lib = load_library()
    dev = torch.cuda.current_device() if device is None else device
    n = ctypes.c_size_t()
    _check("gqa_decode_fixed_split_workspace_size",
           lib.gqa_decode_fixed_split_workspace_size(B, Hq, Hkv, D, num_splits, dev,
                                                     ctypes.byref(n)))
    return n.value


def gqa_decode_fixed_split(q, k_cache, v_cache, block_table, seq_lens, num_splits: int,
                           out=None, scale=None, workspace: Optional[Workspace] = None,
                           stream=None) -> torch.Tensor:
    """The fixed-split comparator (see include/gqa_decode.h): same result as gqa_decode."""
    lib = load_library()
    B, Hq, Hkv, D, bs, mb, nb = _shape(q, k_cache, block_table)
    dev = q.device
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _require(t, n, torch.bfloat16, dev)
    _require(seq_lens, "seq_lens", torch.int32, dev)
    if block_table is not None:
        _require(block_table, "block_table", torch.int32, dev)
    if out is None:
        out = torch.empty_like(q)
    _require(out, "out", torch.bfloat16, dev)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws = default_workspace(dev) if workspace is None else workspace
    buf = ws.get(fixed_split_workspace_size(B, Hq, Hkv, D, num_splits, dev.index))
    with torch.cuda.device(dev):
        rc = lib.gqa_decode_fixed_split(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                        _ptr(seq_lens), _ptr(out), B, Hq, Hkv, D, bs, scale, mb,
                                        nb, int(num_splits), _ptr(buf), buf.numel(),
                                        _stream_ptr(stream))
    _check("gqa_decode_fixed_split", rc)
    return out


def gqa_decode_timeline(q, k_cache, v_cache, block_table, seq_lens, num_splits: int = 0,
                        out=None, scale=None, workspace: Optional[Workspace] = None,
                        stream=None):
    """gqa_decode (num_splits = 0, stream-K) or the fixed split (num_splits >= 1) that
    also records the decode kernel's per-CTA timeline (see include/gqa_decode.h).
    Returns (out, timeline): timeline is int64 [grid, 8] on the device, rows
    (start ns, end ns, SM id, tiles, first TMA ns, first scores ns, streamed ns,
    merged ns); the last four are 0 where not recorded."""
    lib = load_library()
    B, Hq, Hkv, D, bs, mb, nb = _shape(q, k_cache, block_table)
    dev = q.device
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _require(t, n, torch.bfloat16, dev)
    _require(seq_lens, "seq_lens", torch.int32, dev)
    if block_table is not None:
        _require(block_table, "block_table", torch.int32, dev)
    if out is None:
        out = torch.empty_like(q)
    _require(out, "out", torch.bfloat16, dev)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws = default_workspace(dev) if workspace is None else workspace
    need = (fixed_split_workspace_size(B, Hq, Hkv, D, num_splits, dev.index) if num_splits > 0
            else workspace_size(B, Hq, Hkv, D, dev.index))
    buf = ws.get(need)
    grid = ctypes.c_int(0)
    # A buffer too small for the grid is refused before launch, with the grid reported.
    tl = torch.zeros((1, TIMELINE_COLS), dtype=torch.int64, device=dev)
    with torch.cuda.device(dev):
        for _ in range(2):
            rc = lib.gqa_decode_timeline(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                         _ptr(seq_lens), _ptr(out), B, Hq, Hkv, D, bs, scale, mb,
                                         nb, int(num_splits), _ptr(tl), tl.shape[0],
                                         ctypes.byref(grid), _ptr(buf), buf.numel(),
                                         _stream_ptr(stream))
            if rc == GQA_ERR_WORKSPACE_TOO_SMALL and grid.value > tl.shape[0]:
                tl = torch.zeros((grid.value, TIMELINE_COLS), dtype=torch.int64, device=dev)
                continue
            break
    _check("gqa_decode_timeline", rc)
    return out, tl[:grid.value]


def timeline_summary(timeline) -> dict:
    """Tail-wave figures of one step's timeline (rows as gqa_decode_timeline returns):
    span = last CTA end - first CTA start; busy = sum of CTA durations over
    (CTAs x span); tail idle = 1 - busy; start and end times of the CTAs relative to
    the first start (ends over the CTAs that had tiles); and, where the phases were
    recorded, their median and maximum times after each CTA's own start."""
    import numpy as np
    t = np.asarray(timeline.cpu() if hasattr(timeline, "cpu") else timeline, dtype=np.int64)
    if t.ndim != 2 or t.shape[1] != TIMELINE_COLS or t.shape[0] == 0:
        raise ValueError(f"timeline must be a non-empty [rows, {TIMELINE_COLS}] array")
    start, end, sm, tiles = t[:, 0], t[:, 1], t[:, 2], t[:, 3]
    if np.any(end < start):
        raise ValueError("a CTA ends before it starts")
    t0 = start.min()
    span = float(end.max() - t0)
    busy = float((end - start).sum()) / (len(t) * span) if span > 0 else 1.0
    work = tiles > 0
    ends = (end[work] if work.any() else end) - t0
    return {
        "ctas": int(len(t)), "ctas_with_work": int(work.sum()), "sms": int(len(np.unique(sm))),
        "tiles": int(tiles.sum()), "span_us": span / 1e3, "busy_frac": busy,
        "tail_idle": 1.0 - busy, "start_us_max": float(start.max() - t0) / 1e3,
        "end_us_min": float(ends.min()) / 1e3, "end_us_median": float(np.median(ends)) / 1e3,
        "end_us_max": float(ends.max()) / 1e3,
        "phases_us": _phases(t),
    }


def _phases(t) -> dict:
    import numpy as np
    out = {}
    for col, name in ((4, "first_tma"), (5, "first_scores"), (6, "streamed"), (7, "merged")):
        rec = t[:, col] > 0
        if rec.any():
            d = (t[rec, col] - t[rec, 0]) / 1e3
            out[name] = {"median": float(np.median(d)), "max": float(d.max())}
    return out


def gqa_decode_auto(q, k_cache, v_cache, block_table, seq_lens, seq_lens_host=None, out=None,
                    scale=None, workspace: Optional[Workspace] = None, stream=None) -> torch.Tensor:
    """gqa_decode with the runtime schedule selection; seq_lens_host: int32 CPU tensor
    (a copy of seq_lens; taken from the device, with a sync, when omitted)."""
    lib = load_library()
    B, Hq, Hkv, D, bs, mb, nb = _shape(q, k_cache, block_table)
    dev = q.device
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _require(t, n, torch.bfloat16, dev)
    _require(seq_lens, "seq_lens", torch.int32, dev)
    if block_table is not None:
        _require(block_table, "block_table", torch.int32, dev)
    host = seq_lens.cpu() if seq_lens_host is None else seq_lens_host
    if host.device.type != "cpu" or host.dtype != torch.int32 or not host.is_contiguous() \
            or host.numel() != B:
        raise ValueError("seq_lens_host must be a contiguous int32 CPU tensor of length B")
    if out is None:
        out = torch.empty_like(q)
    _require(out, "out", torch.bfloat16, dev)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws = default_workspace(dev) if workspace is None else workspace
    buf = ws.get(workspace_size(B, Hq, Hkv, D, dev.index))
    with torch.cuda.device(dev):
        rc = lib.gqa_decode_auto(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                 _ptr(seq_lens), ctypes.c_void_p(host.data_ptr()), _ptr(out), B, Hq,
                                 Hkv, D, bs, scale, mb, nb, _ptr(buf), buf.numel(),
                                 _stream_ptr(stream))
    _check("gqa_decode_auto", rc)
    return out


def gqa_decode_fp8(q, k8, v8, k_scale: float, v_scale: float, block_table, seq_lens, out=None,
                   scale=None, workspace: Optional[Workspace] = None, stream=None) -> torch.Tensor:
    """Decode over an FP8 E4M3 cache: k8, v8 uint8 (or float8_e4m3fn) in the bf16 caches'
    layouts, values e4m3 * k_scale / e4m3 * v_scale.  Returns out [B, Hq, D] bf16."""
    import torch as _t
    lib = load_library()
    k8 = k8.view(_t.uint8) if k8.dtype != _t.uint8 else k8
    v8 = v8.view(_t.uint8) if v8.dtype != _t.uint8 else v8
    B, Hq, Hkv, D, bs, mb, nb = _shape(q, k8, block_table)
    dev = q.device
    _require(q, "q", _t.bfloat16, dev)
    _require(k8, "k_cache", _t.uint8, dev)
    _require(v8, "v_cache", _t.uint8, dev)
    _require(seq_lens, "seq_lens", _t.int32, dev)
    if block_table is not None:
        _require(block_table, "block_table", _t.int32, dev)
    if out is None:
        out = _t.empty_like(q)
    _require(out, "out", _t.bfloat16, dev)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws = default_workspace(dev) if workspace is None else workspace
    buf = ws.get(workspace_size(B, Hq, Hkv, D, dev.index))
    with _t.cuda.device(dev):
        rc = lib.gqa_decode_fp8(_ptr(q), _ptr(k8), _ptr(v8), float(k_scale), float(v_scale),
                                _ptr(block_table), _ptr(seq_lens), _ptr(out), B, Hq, Hkv, D, bs,
                                scale, mb, nb, _ptr(buf), buf.numel(), _stream_ptr(stream))
    _check("gqa_decode_fp8", rc)
    return out


def gqa_decode_fp8_auto(q, k8, v8, k_scale: float, v_scale: float, block_table, seq_lens,
                        seq_lens_host=None, out=None, scale=None,
                        workspace: Optional[Workspace] = None, stream=None) -> torch.Tensor:
    """gqa_decode_fp8 with the runtime schedule selection of gqa_decode_auto;
    seq_lens_host: int32 CPU tensor (a copy of seq_lens; taken from the device, with a
    sync, when omitted)."""
    lib = load_library()
    k8 = k8.view(torch.uint8) if k8.dtype != torch.uint8 else k8
    v8 = v8.view(torch.uint8) if v8.dtype != torch.uint8 else v8
    B, Hq, Hkv, D, bs, mb, nb = _shape(q, k8, block_table)
    dev = q.device
    _require(q, "q", torch.bfloat16, dev)
    _require(k8, "k_cache", torch.uint8, dev)
    _require(v8, "v_cache", torch.uint8, dev)
    _require(seq_lens, "seq_lens", torch.int32, dev)
    if block_table is not None:
        _require(block_table, "block_table", torch.int32, dev)
    host = seq_lens.cpu() if seq_lens_host is None else seq_lens_host
    if host.device.type != "cpu" or host.dtype != torch.int32 or not host.is_contiguous() \
            or host.numel() != B:
        raise ValueError("seq_lens_host must be a contiguous int32 CPU tensor of length B")
    if out is None:
        out = torch.empty_like(q)
    _require(out, "out", torch.bfloat16, dev)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws = default_workspace(dev) if workspace is None else workspace
    buf = ws.get(workspace_size(B, Hq, Hkv, D, dev.index))
    with torch.cuda.device(dev):
        rc = lib.gqa_decode_fp8_auto(_ptr(q), _ptr(k8), _ptr(v8), float(k_scale),
                                     float(v_scale), _ptr(block_table), _ptr(seq_lens),
                                     ctypes.c_void_p(host.data_ptr()), _ptr(out), B, Hq, Hkv, D,
                                     bs, scale, mb, nb, _ptr(buf), buf.numel(),
                                     _stream_ptr(stream))
    _check("gqa_decode_fp8_auto", rc)
    return out


def gqa_decode_multi(q, k_cache, v_cache, block_table, seq_lens, out=None, scale=None,
                     workspace: Optional[Workspace] = None, stream=None) -> torch.Tensor:
    """Several query tokens per request (speculative verification): q [B, Q, Hq, D] bf16;
    token i of request b sees keys t <= L_b - Q + i.  Returns out [B, Q, Hq, D]."""
    lib = load_library()
    if q.dim() != 4:
        raise ValueError("q must be [B, Q, Hq, D]")
    B, Q, Hq, D = q.shape
    _, _, Hkv, _, bs, mb, nb = _shape(q.view(B, Q * Hq, D), k_cache, block_table)
    dev = q.device
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _require(t, n, torch.bfloat16, dev)
    _require(seq_lens, "seq_lens", torch.int32, dev)
    if block_table is not None:
        _require(block_table, "block_table", torch.int32, dev)
    if out is None:
        out = torch.empty_like(q)
    _require(out, "out", torch.bfloat16, dev)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws = default_workspace(dev) if workspace is None else workspace
    buf = ws.get(workspace_size(B, Hq, Hkv, D, dev.index))
    with torch.cuda.device(dev):
        rc = lib.gqa_decode_multi(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                  _ptr(seq_lens), _ptr(out), B, Q, Hq, Hkv, D, bs, scale, mb, nb,
                                  _ptr(buf), buf.numel(), _stream_ptr(stream))
    _check("gqa_decode_multi", rc)
    return out


def decode_plan(B: int, Hq: int, Hkv: int, D: int, block_size: int, paged: bool,
                num_blocks: int = 0, qlen: int = 1, kv_fp8: bool = False, num_splits: int = 0,
                seq_lens_host=None, device: int | None = None) -> dict:
    """What a call would launch (the C ABI's gqa_decode_plan): kernel, template
    parameters, schedule, grid, LeanTiles.  num_splits: -1 = gqa_decode_auto's choice
    (needs seq_lens_host and a device), 0 = stream-K, n = fixed split.  device < 0
    skips the device query (grid -1 for stream-K)."""
    lib = load_library()
    if device is None:
        device = torch.cuda.current_device()
    lens = None
    if seq_lens_host is not None:
        lens = (seq_lens_host.detach().to("cpu", torch.int32).contiguous()
                if torch.is_tensor(seq_lens_host)
                else torch.tensor(list(seq_lens_host), dtype=torch.int32))
        if lens.numel() != B:
            raise ValueError("seq_lens_host must hold B lengths")
    pl = _Plan()
    _check("gqa_decode_plan",
           lib.gqa_decode_plan(B, Hq, Hkv, D, block_size, int(bool(paged)), num_blocks, qlen,
                               int(bool(kv_fp8)), num_splits,
                               None if lens is None else ctypes.c_void_p(lens.data_ptr()),
                               int(device), ctypes.byref(pl)))
    out = {name: getattr(pl, name) for name, _ in _Plan._fields_}
    out["kernel_name"] = pl.kernel_name.decode()
    return out


def select_schedule(seq_lens, Hq: int, Hkv: int, D: int, num_sms: int, max_splits: int = 64):
    """Host-side schedule choice: (num_splits, est_us) with num_splits = 0 for the
    stream-K gqa_decode, n > 0 for gqa_decode_fixed_split with n chunks; est_us =
    (stream-K estimate, best fixed-split estimate or -1).  max_splits = 1 gives the
    choice gqa_decode_auto makes."""
    lib = load_library()
    lens = (seq_lens.detach().to("cpu", torch.int32).contiguous() if torch.is_tensor(seq_lens)
            else torch.tensor(list(seq_lens), dtype=torch.int32))
    ns = ctypes.c_int()
    est = (ctypes.c_float * 2)()
    _check("gqa_select_schedule",
           lib.gqa_select_schedule(lens.numel(), Hq, Hkv, D, ctypes.c_void_p(lens.data_ptr()),
                                   int(num_sms), int(max_splits), ctypes.byref(ns), est))
    return ns.value, (est[0], est[1])


def gqa_decode_states(q, k_cache, v_cache, block_table, kv_begin, kv_end, scale=None,
                      workspace: Optional[Workspace] = None, stream=None):
    """Partial states over [kv_begin[b], kv_end[b]): (acc [B,Hq,D], m [B,Hq], l [B,Hq]) fp32,
    natural-log units, acc not normalised."""
    lib = load_library()
    B, Hq, Hkv, D, bs, mb, nb = _shape(q, k_cache, block_table)
    dev = q.device
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _require(t, n, torch.bfloat16, dev)
    _require(kv_begin, "kv_begin", torch.int32, dev)
    _require(kv_end, "kv_end", torch.int32, dev)
    if block_table is not None:
        _require(block_table, "block_table", torch.int32, dev)
    acc = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    m = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    l = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    ws = default_workspace(dev) if workspace is None else workspace
    buf = ws.get(workspace_size(B, Hq, Hkv, D, dev.index))
    with torch.cuda.device(dev):
        rc = lib.gqa_decode_states(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                   _ptr(kv_begin), _ptr(kv_end), _ptr(acc), _ptr(m), _ptr(l),
                                   B, Hq, Hkv, D, bs, scale, mb, nb, _ptr(buf), buf.numel(),
                                   _stream_ptr(stream))
    _check("gqa_decode_states", rc)
    return acc, m, l


def gqa_merge_states(acc: torch.Tensor, m: torch.Tensor, l: torch.Tensor, stream=None):
    """Merge S partial states: acc [S, N, D], m/l [S, N] fp32 -> (out [N, D] bf16, lse [N])."""
    lib = load_library()
    S, N, D = acc.shape
    dev = acc.device
    _require(acc, "acc", torch.float32, dev)
    _require(m, "m", torch.float32, dev)
    _require(l, "l", torch.float32, dev)
    if m.shape != (S, N) or l.shape != (S, N):
        raise ValueError("m and l must be [S, N]")
    out = torch.empty((N, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((N,), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        rc = lib.gqa_merge_states(_ptr(acc), _ptr(m), _ptr(l), S, N, D, _ptr(out), _ptr(lse),
                                  _stream_ptr(stream))
    _check("gqa_merge_states", rc)
    return out, lse


class HostDecoder:
    """gqa_decode over HOST tensors: each call copies the inputs host->device, runs the
    kernel and copies the output back (the C ABI's gqa_decode_host)."""

    def __init__(self, B, Hq, Hkv, D, block_size, max_blocks, num_blocks, paged, device=None):
        lib = load_library()
        self.dims = (B, Hq, Hkv, D, block_size, max_blocks, num_blocks)
        self.paged = bool(paged)
        self.device = torch.device("cuda", torch.cuda.current_device() if device is None
                                   else torch.device(device).index)
        nbytes = lib.gqa_decode_host_buffer_bytes(B, Hq, Hkv, D, block_size, max_blocks,
                                                  num_blocks, int(paged))
        self.dbuf = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.ws = Workspace(self.device)
        self.wsbuf = self.ws.get(workspace_size(B, Hq, Hkv, D, self.device.index))

    def h2d_bytes(self, q, k_cache, v_cache, block_table, seq_lens) -> int:
        n = q.numel() * 2 + k_cache.numel() * 2 + v_cache.numel() * 2 + seq_lens.numel() * 4
        return n + (0 if block_table is None else block_table.numel() * 4)

    def __call__(self, q, k_cache, v_cache, block_table, seq_lens, out, scale=None, stream=None):
        lib = load_library()
        B, Hq, Hkv, D, bs, mb, nb = self.dims
        scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
        with torch.cuda.device(self.device):
            rc = lib.gqa_decode_host(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                     _ptr(seq_lens), _ptr(out), B, Hq, Hkv, D, bs, scale, mb, nb,
                                     _ptr(self.dbuf), self.dbuf.numel(), _ptr(self.wsbuf),
                                     self.wsbuf.numel(), _stream_ptr(stream))
        _check("gqa_decode_host", rc)
        return out


def gqa_decode_noalloc(q, k_cache, v_cache, block_table, seq_lens, out=None, scale=None,
                       stream=None):
    """gqa_decode for callers that cannot allocate device memory: the library uses
    its own fixed 16 MiB device scratch instead of a workspace.  Calls on one device
    share that scratch, so they must not overlap on the GPU.  (`out` is allocated
    here only when the caller passes none.)  Tensors are checked as gqa_decode
    checks them, before anything is launched."""
    lib = load_library()
    B, Hq, Hkv, D, bs, mb, nb = _shape(q, k_cache, block_table)
    dev = q.device
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _require(t, n, torch.bfloat16, dev)
    _require(seq_lens, "seq_lens", torch.int32, dev)
    if block_table is not None:
        _require(block_table, "block_table", torch.int32, dev)
    if out is None:
        out = torch.empty_like(q)
    _require(out, "out", torch.bfloat16, dev)
    if tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must have q's shape")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    with torch.cuda.device(dev):
        rc = lib.gqa_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                    _ptr(seq_lens), _ptr(out), B, Hq, Hkv, D, bs, scale, mb, nb,
                                    _stream_ptr(stream))
    _check("gqa_decode_noalloc", rc)
    return out
