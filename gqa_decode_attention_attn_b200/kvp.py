"""Sequence-sharded (KV-parallel) decode across ranks.

Each rank holds the pages of a contiguous token range of every request.  It
computes the partial softmax states (acc, m, l) of every query row over that
range with ``gqa_decode_states``.  The ranks all-gather the states and merge
them exactly with ``gqa_merge_states``.

Only B*Hq*(D+2) fp32 values per rank cross the interconnect per step, against
4*D*Hkv bytes per cached token read from HBM, so the exchange stays small
whatever the context length.

The merge is exact because partial states over disjoint key ranges combine by
rescaling to a common maximum (LeanAttention decode tiles digest, section "Exact
softmax that merges piece by piece"; FlashDecoding's split-KV reduction in
"Attention co-design for long-context inference", section "FlashAttention and
GEMM shapes").

Ranks take the same collective steps in the same order; the process group is
the caller's (NCCL for CUDA tensors, gloo for CPU tensors).
"""
from __future__ import annotations

from typing import Sequence

import torch


def shard_bounds(seq_lens: Sequence[int], world: int, rank: int, align: int = 1):
    """Token range [begin, end) of every request that ``rank`` owns.

    Request b's L_b tokens are cut into ceil(L_b / align) chunks of ``align`` tokens
    (a page, so that no page straddles two ranks).  Rank r takes a contiguous run
    of chunks; runs differ in length by at most one chunk, and the longer runs go
    to the lower ranks.  The ranges of ranks 0..world-1 are disjoint and cover
    [0, L_b).  A rank whose run is empty gets begin = end.

    Returns two int32 CPU tensors of length B.
    """
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of size {world}")
    if align < 1:
        raise ValueError("align must be positive")
    lens = [int(x) for x in (seq_lens.tolist() if torch.is_tensor(seq_lens) else seq_lens)]
    begin, end = [], []
    for L in lens:
        if L < 0:
            raise ValueError("negative sequence length")
        chunks = -(-L // align)
        per, rem = divmod(chunks, world)
        c0 = rank * per + min(rank, rem)
        c1 = c0 + per + (1 if rank < rem else 0)
        begin.append(min(L, c0 * align))
        end.append(min(L, c1 * align))
    return torch.tensor(begin, dtype=torch.int32), torch.tensor(end, dtype=torch.int32)


def exchange_states(acc: torch.Tensor, m: torch.Tensor, l: torch.Tensor, group=None):
    """All-gather every rank's partial states.

    acc [..., D], m [...], l [...] (same leading shape, N rows in all) become
    acc [S, N, D], m [S, N], l [S, N] with S = world size, ordered by rank.  The
    three tensors travel packed as one [N, D + 2] buffer in one collective.
    """
    import torch.distributed as dist

    D = acc.shape[-1]
    N = m.numel()
    if l.numel() != N or acc.numel() != N * D:
        raise ValueError("acc, m and l disagree in their row count")
    world = dist.get_world_size(group)
    pack = torch.cat([acc.reshape(N, D), m.reshape(N, 1).to(acc.dtype),
                      l.reshape(N, 1).to(acc.dtype)], dim=1).contiguous()
    gathered = torch.empty((world * N, D + 2), dtype=pack.dtype, device=pack.device)
    dist.all_gather_into_tensor(gathered, pack, group=group)
    g = gathered.view(world, N, D + 2)
    return g[:, :, :D].contiguous(), g[:, :, D].contiguous(), g[:, :, D + 1].contiguous()


def kvp_decode(q, k_cache, v_cache, block_table, kv_begin, kv_end, group=None, scale=None,
               workspace=None, stream=None):
    """Decode attention for one step when the KV cache is sharded by tokens.

    The arguments are this rank's: its cache pool, and its block table, whose
    entries for tokens outside [kv_begin[b], kv_end[b]) are never read.
    kv_begin/kv_end are int32 [B] on the device, as ``shard_bounds`` gives them.
    Every rank returns the full output, bf16 [B, Hq, D], and lse [B, Hq] (natural
    log).  ``stream`` (a torch.cuda.Stream, or None for the current one) carries the
    kernels and the collective alike.
    """
    from . import gqa_decode_states, gqa_merge_states

    B, Hq, D = q.shape
    acc, m, l = gqa_decode_states(q, k_cache, v_cache, block_table, kv_begin, kv_end,
                                  scale=scale, workspace=workspace, stream=stream)
    if stream is None:
        A, M, Ls = exchange_states(acc, m, l, group)
    else:
        with torch.cuda.stream(stream):
            A, M, Ls = exchange_states(acc, m, l, group)
    out, lse = gqa_merge_states(A, M, Ls, stream=stream)
    return out.view(B, Hq, D), lse.view(B, Hq)
