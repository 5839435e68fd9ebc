"""Rank body for the one-GPU run of ``kvp.kvp_decode`` over a real NCCL group
(world size 1: the states, the collective and the merge all run on cuda:0)."""
import os
import sys

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def run(port: int, results) -> None:
    import workloads
    from gqa_decode_attention_attn_b200 import kvp

    try:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, device_id=dev)
        p = workloads.make_problem("kvp1", 3, 32, 8, 128, [700, 64, 1], seed=777, block_size=16)
        d = p.to(dev)
        k0, k1 = kvp.shard_bounds(p.seq_lens, 1, 0, align=16)
        out, lse = kvp.kvp_decode(d.q, d.k_cache, d.v_cache, d.block_table, k0.to(dev),
                                  k1.to(dev), scale=p.scale)
        torch.cuda.synchronize()
        results.put(("ok", p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale,
                     out.cpu()))
        dist.destroy_process_group()
    except Exception as e:
        results.put(("error", repr(e)))
        raise
