"""CPU: the C-ABI library loads, exports every symbol its header declares, and
rejects bad arguments on the host before touching the GPU."""
import ctypes
import os
import re

import pytest

import gqa_decode_attention_attn_b200 as gq
from gqa_decode_attention_attn_b200 import build as gbuild

HEADER_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


def declared_symbols():
    names = []
    for f in sorted(os.listdir(HEADER_DIR)):
        if f.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, f)).read()
            names += re.findall(r"GQA_API\s+[\w\s\*]+?\b(gqa_\w+)\s*\(", text)
    return names


@pytest.fixture(scope="module")
def lib():
    gbuild.build()
    return gq.load_library()


def test_header_declares_entry_points():
    names = declared_symbols()
    for n in ("gqa_decode", "gqa_merge_states", "gqa_decode_states", "gqa_status",
              "gqa_decode_workspace_size", "gqa_decode_host", "gqa_error_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_symbols():
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
        assert n in gq.EXPORTED


def test_error_strings(lib):
    assert gq.error_string(0) == "ok"
    assert "workspace" in gq.error_string(3)
    assert gq.error_string(99) == "unknown error"


def _decode_rc(lib, B=1, Hq=4, Hkv=1, D=128, bs=16, scale=0.1, q=16, k=16, v=16, out=16,
               lens=16, ws=16):
    P = ctypes.c_void_p
    return lib.gqa_decode(P(q), P(k), P(v), None, P(lens), P(out), B, Hq, Hkv, D, bs, scale,
                          0, 0, P(ws), 1 << 20, None)


def test_host_argument_checks(lib):
    assert _decode_rc(lib, B=-1) == 1              # negative batch
    assert _decode_rc(lib, Hq=6, Hkv=4) == 1        # Hq not a multiple of Hkv
    assert _decode_rc(lib, D=96) == 2               # unsupported head dim
    assert _decode_rc(lib, B=4097) == 2             # above GQA_MAX_BATCH
    assert _decode_rc(lib, scale=float("nan")) == 1
    assert _decode_rc(lib, q=0) == 1                # null pointer
    assert _decode_rc(lib, k=24) == 4               # not 16-byte aligned
    sz = ctypes.c_size_t()
    assert lib.gqa_decode_workspace_size(1, 4, 1, 80, 0, ctypes.byref(sz)) == 2
    assert lib.gqa_merge_states(None, None, None, 1, 0, 8, None, None, None) == 0   # N = 0
    assert lib.gqa_merge_states(None, None, None, 1, 4, 8, None, None, None) == 1
    assert lib.gqa_decode_host_buffer_bytes(2, 4, 1, 128, 64, 0, 0, 0) > 2 * 4 * 128 * 2


def test_timeline_argument_checks(lib):
    P, I = ctypes.c_void_p, ctypes.c_int
    grid = I(-5)

    def rc(timeline=16, rows=8, splits=0, B=1):
        return lib.gqa_decode_timeline(P(16), P(16), P(16), None, P(16), P(16), B, 4, 1, 128, 16,
                                       0.1, 0, 0, splits, None if timeline is None else P(timeline),
                                       rows, ctypes.byref(grid), P(16), 1 << 20, None)

    assert rc(timeline=None) == 1       # no timeline buffer
    assert rc(timeline=20) == 1         # not 8-byte aligned
    assert rc(splits=-1) == 1
    assert rc(rows=-1) == 1
    assert rc(B=-1) == 1                # the shape checks of gqa_decode
    assert rc(B=0) == 0 and grid.value == 0   # empty batch: nothing launched, no rows


def test_wait_limit_arguments(lib):
    """gqa_set_wait_limit: 0 restores the 1.5 s default, 1 us .. 10 s accepted."""
    with pytest.raises(gq.GqaError):
        gq.set_wait_limit(10)            # below 1 us
    with pytest.raises(gq.GqaError):
        gq.set_wait_limit(10 ** 11)      # above 10 s
    assert gq.set_wait_limit(5_000_000) == 1_500_000_000
    assert gq.set_wait_limit(0) == 5_000_000
    assert gq.set_wait_limit(0) == 1_500_000_000


def test_stream_floor_argument_checks(lib):
    """gqa_stream_floor rejects bad arguments on the host, before any CUDA call."""
    P = ctypes.c_void_p

    def rc(k=16, v=16, rows=256, ctas=4, ws=16, ws_bytes=256):
        return lib.gqa_stream_floor(None if k is None else P(k), None if v is None else P(v),
                                    rows, ctas, None if ws is None else P(ws), ws_bytes, None)

    assert rc(k=None) == 1
    assert rc(ws=None) == 1
    assert rc(rows=0) == 1
    assert rc(rows=200) == 1            # not a whole number of 128-row tiles
    assert rc(rows=1 << 31) == 1        # row coordinates are 32-bit
    assert rc(ctas=0) == 1
    assert rc(ws_bytes=8) == 3          # no room for the status word
    assert rc(v=24) == 4                # not 16-byte aligned
