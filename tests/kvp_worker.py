"""Rank body for the sequence-sharded decode test (spawned; gloo on CPU).

Each rank keeps only the block-table entries of its own pages (the rest are
-1, which the oracle rejects if it ever reads them), computes the fp64 partial
states of its token range with the oracle, exchanges them with
``kvp.exchange_states`` and merges them with the oracle's exact merge.
"""
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def run(rank: int, world: int, port: int, case: dict, results) -> None:
    import oracle
    import workloads
    from gqa_decode_attention_attn_b200 import kvp

    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world)
        p = workloads.make_problem("kvp", case["B"], case["Hq"], case["Hkv"], case["D"],
                                   case["lens"], seed=case["seed"],
                                   block_size=case["block_size"])
        bs = p.block_size
        k0, k1 = kvp.shard_bounds(p.seq_lens, world, rank, align=bs)
        table = p.block_table.clone()
        for b in range(p.B):
            owned = set(range(int(k0[b]) // bs, -(-int(k1[b]) // bs)))
            for j in range(table.shape[1]):
                if j not in owned:
                    table[b, j] = -1
        acc, m, l = oracle.gqa_decode_states(p.q, p.k_cache, p.v_cache, table, k0, k1,
                                             p.scale, threads=2)
        A, M, L = kvp.exchange_states(torch.from_numpy(acc), torch.from_numpy(m),
                                      torch.from_numpy(l))
        out, lse = oracle.merge_states(A.numpy(), M.numpy(), L.numpy())
        full = oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens,
                                 p.scale, threads=2)
        results.put((rank, out.reshape(full.shape), full, lse, A.shape[0],
                     k0.tolist(), k1.tolist()))
        dist.destroy_process_group()
    except Exception as e:  # report to the parent instead of hanging it
        results.put((rank, repr(e)))
        raise
