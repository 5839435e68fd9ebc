"""GPU: gqa_decode_noalloc, the entry point for callers that cannot allocate
device memory (it keeps its scratch in a fixed array inside the library instead
of taking a workspace).  It must give the same results as gqa_decode, call after
call, even though every call reuses the same scratch.

This file is named to be collected last, so a failure here cannot hide the
results of the other GPU tests.
"""
import ctypes

import pytest
import torch

import oracle
from gpu_util import MAX_ABS, REL_RMS, as_f64, parity
from workloads import make_problem

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    import gqa_decode_attention_attn_b200 as gq
    lib = gq.load_library()
    fn = lib.gqa_decode_noalloc
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, P]
    fn.restype = I
    return gq, fn


def _call(fn, d, out):
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ptr(d.q), ptr(d.k_cache), ptr(d.v_cache), ptr(d.block_table), ptr(d.seq_lens),
              ptr(out), d.B, d.Hq, d.Hkv, d.D, d.block_size, d.scale, d.max_blocks,
              d.num_blocks, stream)


def test_noalloc_matches_gqa_decode_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required")
    gq, fn = _noalloc_fn()
    # Long paged requests (split over many CTAs, so tickets and partial slots in
    # the scratch are exercised) and a contiguous case with a different shape.
    cases = [make_problem("paged", 4, 32, 8, 128, [20000, 3, 9000, 4097], seed=77,
                          block_size=16, spare_blocks=4),
             make_problem("contig", 2, 16, 4, 64, [30000, 1000], seed=78),
             # the 64-head kernel's larger partial-state slots, and D = 256
             make_problem("mqa", 2, 64, 1, 128, [30000, 777], seed=81, block_size=64),
             make_problem("d256", 2, 16, 4, 256, [20000, 300], seed=82, block_size=16)]
    for p in cases:
        d = p.to("cuda")
        expect = gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                               scale=p.scale)
        torch.cuda.synchronize()
        for call in range(2):
            out = torch.full_like(d.q, float("nan"))
            assert _call(fn, d, out) == 0
            torch.cuda.synchronize()
            parity(out, as_f64(expect), f"{p.name} call {call}")
        # and against the oracle, once
        ref = oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale)
        parity(out, ref, f"{p.name} vs oracle")


def test_noalloc_rejects_shapes_beyond_its_limits():
    gq, fn = _noalloc_fn()
    p = make_problem("big", 1, 4, 1, 128, [16], seed=79).to("cuda")
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    out = torch.empty_like(p.q)
    # B above GQA_MAX_BATCH: rejected on the host, nothing launched.
    rc = fn(ptr(p.q), ptr(p.k_cache), ptr(p.v_cache), None, ptr(p.seq_lens), ptr(out),
            4097, 4, 1, 128, p.block_size, p.scale, 0, 0, None)
    assert rc == 2 and "unsupported" in gq.error_string(rc)
    assert "16 MiB" in gq.error_string(gq.GQA_ERR_SCRATCH_LIMIT)


def test_noalloc_scratch_covers_every_shape_within_the_maxima():
    """The header's claim: every shape within GQA_MAX_BATCH and GQA_MAX_QHEADS needs
    no more scratch than the fixed 16 MiB (gqa_decode_workspace_size is what the
    entry point compares against), at the extreme batch and head counts."""
    gq, _ = _noalloc_fn()
    limit = 16 << 20
    for D in (64, 128, 256):
        for Hq, Hkv in ((256, 1), (256, 256), (256, 64), (4, 1)):
            need = gq.workspace_size(4096, Hq, Hkv, D)
            assert need <= limit, (D, Hq, Hkv, need)


def test_noalloc_python_wrapper_checks_and_matches():
    """The Python wrapper checks its tensors before anything is launched (a CPU
    length array or a float32 output would otherwise reach the kernel as a bad
    pointer) and otherwise returns gqa_decode's result."""
    gq, _ = _noalloc_fn()
    p = make_problem("wrap", 2, 32, 8, 128, [5000, 77], seed=80, block_size=16, spare_blocks=2)
    d = p.to("cuda")
    with pytest.raises(ValueError):
        gq.gqa_decode_noalloc(d.q, d.k_cache, d.v_cache, d.block_table, p.seq_lens)
    with pytest.raises(ValueError):
        gq.gqa_decode_noalloc(d.q, d.k_cache, d.v_cache, p.block_table, d.seq_lens)
    with pytest.raises(TypeError):
        gq.gqa_decode_noalloc(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                              out=torch.empty(d.q.shape, dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError):
        gq.gqa_decode_noalloc(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                              out=torch.empty(2, 128, 32, dtype=torch.bfloat16,
                                              device="cuda").transpose(1, 2))
    expect = gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, scale=p.scale)
    for _ in range(2):
        got = gq.gqa_decode_noalloc(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                                    scale=p.scale)
        torch.cuda.synchronize()
        parity(got, as_f64(expect), "python wrapper")
