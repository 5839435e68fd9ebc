"""GPU: a bounded in-kernel wait that cannot end runs out, and the kernel returns.

The owners of a split (request, KV head) publish their partial states by raising
the segment's counter in the workspace and wait until all of them have (the
co-resident merge).  Here the counter of one segment is preset so that its low
16 bits wrap to 0 on the first publish and never reach the owner count, and the
wait limit is cut to 2 ms (gqa_set_wait_limit).  Every owner's wait then runs
out: the kernel must set GQA_DEV_TIMEOUT, write NaN to that segment's rows,
finish the other segment normally, and leave a workspace that gqa_status cleans
for the next call.  Nothing traps or waits without a limit.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import parity
from workloads import make_problem

pytestmark = pytest.mark.gpu

STATUS_BYTES = 256  # the workspace's status word area; ticket counters follow


def test_merge_wait_runs_out_and_reports():
    import gqa_decode_attention_attn_b200 as gq
    gq.load_library()
    # Two requests, one KV head, G = 16 (one head chunk): two segments of 469
    # tiles, each split over about half of the persistent CTAs.
    p = make_problem("timeout", 2, 16, 1, 128, [60000, 60000], seed=90, block_size=64)
    d = p.to("cuda")
    plan = gq.decode_plan(p.B, p.Hq, p.Hkv, p.D, p.block_size, True, p.num_blocks,
                          seq_lens_host=p.seq_lens)
    assert plan["kernel"] == gq.KERNEL_TENSOR_CORE and plan["cooperative"] == 1
    assert plan["grid"] > 2  # so each segment is split over several owners
    ref = oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale)
    ws = gq.Workspace("cuda")
    buf = ws.get(gq.workspace_size(p.B, p.Hq, p.Hkv, p.D))
    counters = buf[STATUS_BYTES:STATUS_BYTES + 4 * 16].view(torch.int32)
    seg = 1  # (request 1, KV head 0, head chunk 0), the last segment of the order
    counters[seg] = 0xFFFF
    prev = gq.set_wait_limit(2_000_000)
    try:
        out = gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                            scale=p.scale, workspace=ws)
        torch.cuda.synchronize()
    finally:
        gq.set_wait_limit(0)
    assert prev == 1_500_000_000
    status = ws.status()
    assert status & gq.DEV_TIMEOUT, status
    o = out.float().cpu()
    assert torch.isnan(o[1]).all(), "the segment whose wait ran out has NaN rows"
    parity(out[0], ref.reshape(2, 16, 128)[0], "the other segment")
    # gqa_status cleared the counters: the next call on the same workspace is clean.
    out2 = gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, scale=p.scale,
                         workspace=ws)
    assert ws.status() == 0
    parity(out2, ref, "next call")

