"""GPU: the per-CTA timeline entry point (gqa_decode_timeline) computes what
gqa_decode and gqa_decode_fixed_split compute, bit for bit, and records one sane
row (start ns, end ns, SM id, tiles, then the phase times of a tensor-core CTA)
per CTA of the decode kernel's grid."""
import ctypes
import math

import pytest
import torch

import gqa_decode_attention_attn_b200 as gq
import oracle
from gpu_util import parity
from workloads import make_problem

pytestmark = pytest.mark.gpu


def _rows_ok(tl, tiles=None, phases=True):
    t = tl.cpu()
    assert t.dim() == 2 and t.shape[1] == gq.TIMELINE_COLS and t.shape[0] >= 1
    assert torch.all(t[:, 0] > 0) and torch.all(t[:, 1] >= t[:, 0])
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert torch.all((t[:, 2] >= 0) & (t[:, 2] < sms))
    if tiles is not None:
        assert int(t[:, 3].sum()) == tiles
    work = t[:, 3] > 0
    if phases:
        # start <= first TMA <= first scores <= streamed <= merged <= end, CTAs with work
        w = t[work]
        seq = [w[:, 0], w[:, 4], w[:, 5], w[:, 6], w[:, 7], w[:, 1]]
        for a, b in zip(seq, seq[1:]):
            assert torch.all(a <= b)
        assert torch.all(t[~work][:, 4:] == 0)
    else:
        assert torch.all(t[:, 4:] == 0)
    return t


def test_stream_k_timeline_on_the_tensor_cores():
    lens = [100000, 3001]
    p = make_problem("tl", 2, 32, 2, 128, lens, seed=4401, block_size=64)
    d = p.to("cuda")
    ws = gq.Workspace(d.q.device)
    ref = gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, scale=p.scale,
                        workspace=ws)
    out, tl = gq.gqa_decode_timeline(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                                     scale=p.scale, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert torch.equal(out, ref)
    parity(out, oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale),
           "timeline")
    # Every tile of every (request, KV head) once: G = 16 is one head chunk.
    t = _rows_ok(tl, 2 * sum(math.ceil(L / 128) for L in lens))
    # The cooperative grid holds one CTA per SM, each on its own SM, all with work.
    assert len(set(t[:, 2].tolist())) == t.shape[0]
    # Stream-K partition of the W tiles over the P CTAs: CTA c runs [cW/P, (c+1)W/P).
    W, P = 2 * sum(math.ceil(L / 128) for L in lens), t.shape[0]
    assert t[:, 3].tolist() == [(c + 1) * W // P - c * W // P for c in range(P)]
    s = gq.timeline_summary(tl)
    assert s["ctas_with_work"] == t.shape[0] and 0.0 <= s["tail_idle"] < 1.0


def test_fixed_split_timeline():
    lens = [3000, 1, 700, 129]
    p = make_problem("tlfs", 4, 32, 8, 128, lens, seed=4402, block_size=None)
    d = p.to("cuda")
    ws = gq.Workspace(d.q.device)
    ref = gq.gqa_decode_fixed_split(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, 3,
                                    scale=p.scale, workspace=ws)
    out, tl = gq.gqa_decode_timeline(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                                     num_splits=3, scale=p.scale, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert torch.equal(out, ref)
    t = _rows_ok(tl, 8 * sum(math.ceil(L / 128) for L in lens))
    assert t.shape[0] == 4 * 8 * 3  # one CTA per (request, KV head, chunk)
    # Chunk i of a segment of nb tiles holds tiles [i nb / 3, (i + 1) nb / 3).
    nb = [math.ceil(L / 128) for L in lens]
    assert t[:, 3].tolist() == [(i + 1) * nb[b] // 3 - i * nb[b] // 3
                                for b in range(4) for _ in range(8) for i in range(3)]


def test_cuda_core_timeline():
    p = make_problem("tlsimt", 2, 8, 8, 128, [5000, 77], seed=4403, block_size=16)  # G = 1
    d = p.to("cuda")
    ws = gq.Workspace(d.q.device)
    ref = gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, scale=p.scale,
                        workspace=ws)
    out, tl = gq.gqa_decode_timeline(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                                     scale=p.scale, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert torch.equal(out, ref)
    t = _rows_ok(tl, phases=False)
    assert int(t[:, 3].sum()) > 0


def test_timeline_buffer_too_small_launches_nothing():
    p = make_problem("tlsmall", 1, 32, 2, 128, [20000], seed=4404, block_size=None)
    d = p.to("cuda")
    ws = gq.Workspace(d.q.device)
    lib = gq.load_library()
    out = torch.full_like(d.q, 7.0)
    tl = torch.zeros((1, gq.TIMELINE_COLS), dtype=torch.int64, device="cuda")
    grid = ctypes.c_int(0)
    B, Hq, Hkv, D, bs, mb, nb = gq._shape(d.q, d.k_cache, d.block_table)
    buf = ws.get(gq.workspace_size(B, Hq, Hkv, D, 0))
    rc = lib.gqa_decode_timeline(gq._ptr(d.q), gq._ptr(d.k_cache), gq._ptr(d.v_cache),
                                 gq._ptr(d.block_table), gq._ptr(d.seq_lens), gq._ptr(out), B, Hq,
                                 Hkv, D, bs, p.scale, mb, nb, 0, gq._ptr(tl), 1,
                                 ctypes.byref(grid), gq._ptr(buf), buf.numel(),
                                 gq._stream_ptr(None))
    torch.cuda.synchronize()
    assert rc == gq.GQA_ERR_WORKSPACE_TOO_SMALL and grid.value > 1
    assert torch.all(out == 7.0) and torch.all(tl == 0)
