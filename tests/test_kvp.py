"""Sequence-sharded (KV-parallel) decode: shard bounds and the state exchange.

The exchange runs as world_size 2 and 3 gloo process groups on CPU; the partial
states and the merge come from the fp64 oracle, so the test checks the host
logic (ranges, packing, rank order) against the unsplit oracle result.  The
exactness of merging disjoint ranges is the property stated in the LeanAttention
decode tiles digest, section "Exact softmax that merges piece by piece".
"""
import multiprocessing as mp
import random
import socket

import numpy as np
import pytest

from gqa_decode_attention_attn_b200 import kvp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_bounds_cover_disjoint_aligned(world):
    rng = random.Random(world)
    lens = [0, 1, 5, 16, 17, 1000] + [rng.randrange(0, 5000) for _ in range(20)]
    for align in (1, 16, 64):
        spans = [kvp.shard_bounds(lens, world, r, align) for r in range(world)]
        for b, L in enumerate(lens):
            prev = 0
            sizes = []
            for r in range(world):
                k0, k1 = int(spans[r][0][b]), int(spans[r][1][b])
                assert k0 == prev and k0 <= k1 <= L
                if k0 < L:
                    assert k0 % align == 0
                sizes.append(-(-(k1 - k0) // align))
                prev = k1
            assert prev == L
            assert max(sizes) - min(sizes) <= 1
            assert sizes == sorted(sizes, reverse=True)


def test_shard_bounds_rejects_bad_arguments():
    with pytest.raises(ValueError):
        kvp.shard_bounds([4], 2, 2)
    with pytest.raises(ValueError):
        kvp.shard_bounds([4], 2, 0, align=0)
    with pytest.raises(ValueError):
        kvp.shard_bounds([-1], 1, 0)


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_and_merge_equals_unsplit(world):
    import kvp_worker

    case = dict(B=4, Hq=8, Hkv=2, D=64, lens=[100, 37, 5, 0], seed=4242, block_size=16)
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=kvp_worker.run, args=(r, world, port, case, results))
             for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            item = results.get(timeout=180)
            assert len(item) > 2, f"rank {item[0]} failed: {item[1]}"
            got[item[0]] = item[1:]
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for p in procs:
        assert p.exitcode == 0
    ref_out = got[0][0]
    for r in range(world):
        out, full, lse, S, k0, k1 = got[r]
        assert S == world
        # every rank holds the same merged result, bit for bit
        assert np.array_equal(out, ref_out)
        np.testing.assert_allclose(out, full, rtol=0, atol=1e-12)
        # a request with no keys gives out = 0 and lse = -inf
        assert np.all(out[3] == 0.0) and np.all(np.isneginf(lse.reshape(4, 8)[3]))
    # the short request lives on rank 0 only
    assert got[0][4][2] == 0 and got[0][5][2] == 5
