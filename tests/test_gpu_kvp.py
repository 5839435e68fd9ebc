"""Sequence-sharded decode on the GPU kernels.

Each emulated rank keeps only its own pages in the block table (the others are
-1, which the kernel reports as GQA_DEV_BAD_BLOCK if it reads them), computes its
partial states with ``gqa_decode_states`` and the merge of all ranks' states runs
in ``gqa_merge_states``; the result must match the unsplit oracle.  A second test
drives ``kvp.kvp_decode`` through a real one-rank NCCL group.
"""
import multiprocessing as mp
import socket

import pytest
import torch

import gqa_decode_attention_attn_b200 as gq
import oracle
import workloads
from gpu_util import parity
from gqa_decode_attention_attn_b200 import kvp

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,bs,lens,shape", [
    (2, 16, [1000, 37, 5, 0], (32, 8, 128)),
    (4, 64, [20000, 4096, 63, 640], (32, 2, 128)),
    (8, 16, [3000, 129, 1], (16, 4, 256)),
])
def test_sharded_states_merge_match_oracle(world, bs, lens, shape):
    Hq, Hkv, D = shape
    p = workloads.make_problem("kvp", len(lens), Hq, Hkv, D, lens, seed=9000 + world,
                               block_size=bs)
    dev = torch.device("cuda", 0)
    d = p.to(dev)
    ws = gq.Workspace(dev)
    accs, ms, ls = [], [], []
    for r in range(world):
        k0, k1 = kvp.shard_bounds(p.seq_lens, world, r, align=bs)
        table = p.block_table.clone()
        for b in range(p.B):
            lo, hi = int(k0[b]) // bs, -(-int(k1[b]) // bs)
            table[b, :lo] = -1
            table[b, hi:] = -1
        acc, m, l = gq.gqa_decode_states(d.q, d.k_cache, d.v_cache, table.to(dev), k0.to(dev),
                                         k1.to(dev), scale=p.scale, workspace=ws)
        assert ws.status() == 0
        accs.append(acc)
        ms.append(m)
        ls.append(l)
    N = p.B * Hq
    out, _ = gq.gqa_merge_states(torch.stack(accs).view(world, N, D),
                                 torch.stack(ms).view(world, N), torch.stack(ls).view(world, N))
    ref = oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale)
    parity(out.view(p.B, Hq, D).cpu(), ref)


def test_kvp_decode_one_rank_nccl():
    import kvp_gpu_worker

    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    proc = ctx.Process(target=kvp_gpu_worker.run, args=(port, results))
    proc.start()
    try:
        item = results.get(timeout=300)
    finally:
        proc.join(timeout=60)
        if proc.is_alive():
            proc.kill()
    assert item[0] == "ok", item
    _, q, k, v, table, lens, scale, out = item
    ref = oracle.gqa_decode(q, k, v, table, lens, scale)
    parity(out, ref)
    assert proc.exitcode == 0
