"""fp64 CPU oracle for decode-time grouped-query attention (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``gqa_decode_attention_attn_b200``) never imports, links or calls it, and the two
share no code: the C source here is compiled with the host C compiler into its
own shared object.

The arithmetic lives in ``gqa_oracle.c`` (plain double-precision loops, two-pass
softmax).  This module only compiles that file on first use, marshals arrays
and splits query rows across host threads; it adds no arithmetic of its own.

Inputs are the raw bf16 bit patterns (``uint16``) of q, K and V, exactly as the
CUDA path receives them, plus int32 block table / lengths.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.c")
_LIB = os.path.join(_HERE, "libgqa_oracle.so")
_lock = threading.Lock()
_lib = None

ORACLE_ERRORS = {1: "bad argument", 2: "block id outside the pool", 3: "out of memory"}


def build(force: bool = False, src: str = _SRC, lib: str = _LIB) -> str:
    """Compile the oracle C source into a shared object (IEEE semantics, no contraction)."""
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
               "-std=c11", src, "-o", lib + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(lib + ".tmp", lib)
    return lib


def host_threads() -> int:
    """Host cores this process may run on (affinity mask)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _bits(x) -> np.ndarray:
    """Contiguous uint16 view of bf16 data given as a torch tensor or a uint16 array."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        x = x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
    arr = np.ascontiguousarray(np.asarray(x))
    if arr.dtype != np.uint16:
        raise TypeError(f"expected bf16 bit patterns (uint16), got {arr.dtype}")
    return arr


def _bytes8(x) -> np.ndarray:
    """Contiguous uint8 view of FP8 E4M3 data (torch float8_e4m3fn or uint8, numpy uint8)."""
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu").contiguous()
        if x.dtype != torch.uint8:
            x = x.view(torch.uint8)
        x = x.numpy()
    arr = np.ascontiguousarray(np.asarray(x))
    if arr.dtype != np.uint8:
        raise TypeError(f"expected FP8 E4M3 bytes (uint8), got {arr.dtype}")
    return arr


def _i32(x) -> np.ndarray | None:
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x), dtype=np.int32)


def _ptr(a) -> ctypes.c_void_p | None:
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _shape(q, k_cache, block_table):
    B, Hq, D = q.shape
    num_blocks, Hkv, block_size, D2 = k_cache.shape
    if D2 != D:
        raise ValueError("head_dim of q and the cache differ")
    max_blocks = 0 if block_table is None else block_table.shape[1]
    return B, Hq, Hkv, D, block_size, max_blocks, num_blocks


def _split(n_rows: int, threads: int):
    threads = max(1, min(threads, n_rows))
    edges = np.linspace(0, n_rows, threads + 1).astype(np.int64)
    return [(int(edges[i]), int(edges[i + 1])) for i in range(threads) if edges[i + 1] > edges[i]]


def _run_spans(fn, spans):
    if len(spans) == 1:
        fn(spans[0])
    else:
        with ThreadPoolExecutor(len(spans)) as ex:
            list(ex.map(fn, spans))


class Oracle:
    """The oracle functions bound to one compiled copy of the C source."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        P, I, I64, Dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_gqa_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, Dbl, I64, I64, P]
        lib.oracle_gqa_decode.restype = I
        lib.oracle_gqa_decode_multi.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, I, Dbl, I64,
                                                I64, P]
        lib.oracle_gqa_decode_multi.restype = I
        lib.oracle_gqa_decode_states.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, Dbl,
                                                 I64, I64, P, P, P]
        lib.oracle_gqa_decode_states.restype = I
        lib.oracle_merge_states.argtypes = [P, P, P, I, I, I, P, P]
        lib.oracle_merge_states.restype = I
        lib.oracle_gqa_decode_fp8.argtypes = [P, P, P, Dbl, Dbl, P, P, I, I, I, I, I, I, I, Dbl,
                                              I64, I64, P]
        lib.oracle_gqa_decode_fp8.restype = I
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = Dbl
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = Dbl
        self.lib = lib

    def gqa_decode(self, q, k_cache, v_cache, block_table, seq_lens, scale: float,
                   rows=None, threads: int | None = None) -> np.ndarray:
        """Attention output in float64.

        q: [B, Hq, D] bf16; k_cache, v_cache: [num_blocks, Hkv, block_size, D] bf16
        (contiguous caches: [B, Hkv, capacity, D] with block_table=None);
        block_table: [B, max_blocks] int32 or None; seq_lens: [B] int32.
        rows: optional (row_begin, row_end) over the flattened [B*Hq] query rows.
        Returns [B, Hq, D] (or [row_end-row_begin, D] when rows is given).
        """
        lib = self.lib
        qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
        bt, sl = _i32(block_table), _i32(seq_lens)
        B, Hq, Hkv, D, bs, max_blocks, num_blocks = _shape(qb, kb, bt)
        r0, r1 = (0, B * Hq) if rows is None else rows
        out = np.zeros((r1 - r0, D), dtype=np.float64)
        threads = host_threads() if threads is None else threads

        def run(span):
            a, b = span
            rc = lib.oracle_gqa_decode(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), _ptr(sl), B, Hq,
                                       Hkv, D, bs, max_blocks, num_blocks, float(scale),
                                       r0 + a, r0 + b,
                                       ctypes.c_void_p(out.ctypes.data + a * D * 8))
            if rc:
                raise RuntimeError(f"oracle_gqa_decode: {ORACLE_ERRORS.get(rc, rc)}")

        _run_spans(run, _split(r1 - r0, threads))
        return out.reshape(B, Hq, D) if rows is None else out

    def gqa_decode_fp8(self, q, k8, v8, k_scale: float, v_scale: float, block_table, seq_lens,
                       scale: float, rows=None, threads: int | None = None) -> np.ndarray:
        """Decode over an FP8 E4M3 cache (values e4m3 * k_scale, e4m3 * v_scale); k8, v8
        have the bf16 caches' shapes with one byte per element.  Returns [B, Hq, D]."""
        lib = self.lib
        qb, kb, vb = _bits(q), _bytes8(k8), _bytes8(v8)
        bt, sl = _i32(block_table), _i32(seq_lens)
        B, Hq, Hkv, D, bs, max_blocks, num_blocks = _shape(qb, kb, bt)
        r0, r1 = (0, B * Hq) if rows is None else rows
        out = np.zeros((r1 - r0, D), dtype=np.float64)
        threads = host_threads() if threads is None else threads

        def run(span):
            a, b = span
            rc = lib.oracle_gqa_decode_fp8(_ptr(qb), _ptr(kb), _ptr(vb), float(k_scale),
                                           float(v_scale), _ptr(bt), _ptr(sl), B, Hq, Hkv, D, bs,
                                           max_blocks, num_blocks, float(scale), r0 + a, r0 + b,
                                           ctypes.c_void_p(out.ctypes.data + a * D * 8))
            if rc:
                raise RuntimeError(f"oracle_gqa_decode_fp8: {ORACLE_ERRORS.get(rc, rc)}")

        _run_spans(run, _split(r1 - r0, threads))
        return out.reshape(B, Hq, D) if rows is None else out

    def e4m3_to_double(self, bits: int) -> float:
        """Exact widening of one FP8 E4M3 byte."""
        return self.lib.oracle_e4m3_to_double(int(bits))

    def gqa_decode_multi(self, q, k_cache, v_cache, block_table, seq_lens, scale: float,
                         rows=None, threads: int | None = None) -> np.ndarray:
        """Several query tokens per request (speculative verification): q [B, Q, Hq, D];
        query token i of request b attends keys t <= L_b - Q + i.  Returns [B, Q, Hq, D]
        float64 (or [row_end-row_begin, D] over the flattened [B*Q*Hq] rows)."""
        lib = self.lib
        qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
        bt, sl = _i32(block_table), _i32(seq_lens)
        B, Q, Hq, D = qb.shape
        _, _, Hkv, D2, bs, max_blocks, num_blocks = _shape(qb.reshape(B, Q * Hq, D), kb, bt)
        r0, r1 = (0, B * Q * Hq) if rows is None else rows
        out = np.zeros((r1 - r0, D), dtype=np.float64)
        threads = host_threads() if threads is None else threads

        def run(span):
            a, b = span
            rc = lib.oracle_gqa_decode_multi(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), _ptr(sl), B,
                                             Q, Hq, Hkv, D, bs, max_blocks, num_blocks,
                                             float(scale), r0 + a, r0 + b,
                                             ctypes.c_void_p(out.ctypes.data + a * D * 8))
            if rc:
                raise RuntimeError(f"oracle_gqa_decode_multi: {ORACLE_ERRORS.get(rc, rc)}")

        _run_spans(run, _split(r1 - r0, threads))
        return out.reshape(B, Q, Hq, D) if rows is None else out

    def gqa_decode_states(self, q, k_cache, v_cache, block_table, kv_begin, kv_end,
                          scale: float, threads: int | None = None):
        """Partial softmax states over per-request key ranges [kv_begin[b], kv_end[b]).

        Returns (acc [B, Hq, D], m [B, Hq], l [B, Hq]) in float64, natural-log
        units, acc not normalised.
        """
        lib = self.lib
        qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
        bt, k0, k1 = _i32(block_table), _i32(kv_begin), _i32(kv_end)
        B, Hq, Hkv, D, bs, max_blocks, num_blocks = _shape(qb, kb, bt)
        n = B * Hq
        acc = np.zeros((n, D), dtype=np.float64)
        m = np.zeros(n, dtype=np.float64)
        l = np.zeros(n, dtype=np.float64)
        threads = host_threads() if threads is None else threads

        def run(span):
            a, b = span
            rc = lib.oracle_gqa_decode_states(
                _ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), _ptr(k0), _ptr(k1), B, Hq, Hkv, D, bs,
                max_blocks, num_blocks, float(scale), a, b,
                ctypes.c_void_p(acc.ctypes.data + a * D * 8),
                ctypes.c_void_p(m.ctypes.data + a * 8), ctypes.c_void_p(l.ctypes.data + a * 8))
            if rc:
                raise RuntimeError(f"oracle_gqa_decode_states: {ORACLE_ERRORS.get(rc, rc)}")

        _run_spans(run, _split(n, threads))
        return acc.reshape(B, Hq, D), m.reshape(B, Hq), l.reshape(B, Hq)

    def merge_states(self, acc, m, l):
        """Exact merge of S partial states: acc [S, N, D], m [S, N], l [S, N] (float64).

        Returns (out [N, D], lse [N]).
        """
        acc = np.ascontiguousarray(acc, dtype=np.float64)
        m = np.ascontiguousarray(m, dtype=np.float64)
        l = np.ascontiguousarray(l, dtype=np.float64)
        S, N, D = acc.shape
        if m.shape != (S, N) or l.shape != (S, N):
            raise ValueError("m and l must be [S, N]")
        out = np.zeros((N, D), dtype=np.float64)
        lse = np.zeros(N, dtype=np.float64)
        rc = self.lib.oracle_merge_states(_ptr(acc), _ptr(m), _ptr(l), S, N, D, _ptr(out),
                                          _ptr(lse))
        if rc:
            raise RuntimeError(f"oracle_merge_states: {ORACLE_ERRORS.get(rc, rc)}")
        return out, lse

    def bf16_to_double(self, bits: int) -> float:
        """Exact widening of one bf16 bit pattern."""
        return self.lib.oracle_bf16_to_double(int(bits))


def default() -> Oracle:
    """The oracle compiled from this directory's C source (built on first use)."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = Oracle(build())
    return _lib


def gqa_decode(*args, **kw):
    return default().gqa_decode(*args, **kw)


def gqa_decode_fp8(*args, **kw):
    return default().gqa_decode_fp8(*args, **kw)


def e4m3_to_double(bits: int) -> float:
    return default().e4m3_to_double(bits)


def gqa_decode_multi(*args, **kw):
    return default().gqa_decode_multi(*args, **kw)


def gqa_decode_states(*args, **kw):
    return default().gqa_decode_states(*args, **kw)


def merge_states(*args, **kw):
    return default().merge_states(*args, **kw)


def bf16_to_double(bits: int) -> float:
    return default().bf16_to_double(bits)
