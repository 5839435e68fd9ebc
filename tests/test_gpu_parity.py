"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bar: max-abs error <= 1e-2 and relative RMS error <= 2e-3 per case over all
outputs; index handling (block tables, lengths) bit-exact, checked through
poisoned slots that must never be read and through permutation invariance.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import as_f64, parity
from workloads import make_problem

pytestmark = pytest.mark.gpu

gq = None


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    global gq
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import gqa_decode_attention_attn_b200 as mod
    mod.load_library()
    gq = mod
    yield


def run(p, out=None, workspace=None):
    d = p.to("cuda")
    return gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, out=out,
                         scale=p.scale, workspace=workspace)


def ref(p, rows=None):
    return oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale,
                             rows=rows)


# --------------------------------------------------------------------- small, many shapes

SMALL = [
    # B, Hq, Hkv, D, lens, block_size
    (1, 4, 1, 128, [512], None),
    (3, 8, 2, 128, [1, 63, 200], None),
    (2, 8, 8, 128, [64, 65], None),                     # G = 1 (MHA)
    (2, 8, 1, 128, [129, 7], None),                     # G = 8 (MQA)
    (2, 6, 2, 128, [100, 33], None),                    # G = 3 (padded head chunk)
    (2, 12, 2, 128, [300, 5], 16),                      # G = 6
    (2, 24, 2, 64, [333, 129], 16),                     # G = 12: two head chunks
    (1, 32, 2, 128, [1000], 64),                        # G = 16
    (1, 64, 1, 128, [777], 64),                         # G = 64
    (4, 8, 2, 64, [128, 127, 129, 1], 16),
    (3, 4, 2, 256, [31, 32, 95], 8),
    (2, 16, 4, 256, [500, 1], 32),
    (5, 8, 4, 128, [0, 17, 0, 250, 64], 16),            # empty requests
    (2, 4, 1, 128, [70, 70], 1),                        # one-token pages
    (2, 4, 2, 128, [101, 55], 3),                       # pages not a power of two
    (2, 4, 2, 128, [1000, 999], 100),
    # tensor-core path (D = 128, G >= 8): pages of 8..256 tokens, ragged tiles
    (3, 16, 2, 128, [129, 1, 300], 8),
    (2, 24, 2, 128, [511, 130], 32),                    # G = 12: padded head chunk
    (2, 32, 1, 128, [1000, 127], 128),                  # G = 32: two head chunks
    (1, 16, 1, 128, [700], 256),
    (2, 8, 1, 128, [5000, 3000], None),                 # contiguous, capacity 5005
    (4, 64, 4, 128, [2048, 2047, 1, 130], 16),
    # one long segment spread over every CTA: group merges plus a segment merge
    (1, 4, 1, 128, [100000], None),
    (1, 16, 1, 128, [200000], 64),
    (1, 2, 1, 64, [150000], 16),
    # the 64-heads-per-pass tensor-core kernel (G > 16 at D = 128)
    (3, 48, 1, 128, [129, 1, 4000], 16),                # G = 48: padded 64-head pass
    (2, 128, 1, 128, [3000, 257], 32),                  # G = 128: two 64-head passes
    (4, 64, 2, 128, [5000, 1, 0, 777], None),           # contiguous, an empty request
    (1, 64, 1, 128, [150000], 64),                      # one long segment over every CTA
    (2, 32, 1, 128, [130, 9000], 8),                    # G = 32, 8-token pages
    # tensor-core path at D = 256 (two ring slots per tile)
    (2, 16, 4, 256, [3000, 129], 16),                   # G = 4, 16-token pages
    (2, 32, 2, 256, [700, 1], None),                    # G = 16, contiguous
    (3, 24, 2, 256, [128, 127, 4097], 64),              # G = 12: padded head chunk
    (1, 8, 1, 256, [100000], 64),                       # one long segment over every CTA
    # tensor-core path at D = 64
    (2, 32, 4, 64, [3001, 77], 32),                     # G = 8
    (2, 16, 2, 64, [1000, 999], None),                  # contiguous
    (1, 8, 1, 64, [120000], 64),                        # one long segment over every CTA
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_D{c[3]}_bs{c[5]}")
def test_small_shapes(case):
    B, Hq, Hkv, D, lens, bs = case
    p = make_problem("small", B, Hq, Hkv, D, lens, seed=100 + sum(lens) + D, block_size=bs,
                     spare_blocks=3 if bs else 0, capacity=None if bs else max(lens) + 5)
    out = run(p)
    torch.cuda.synchronize()
    parity(out, ref(p), str(case))


# Key outliers move the softmax reference maximum in the middle of a run, also in
# the last tile of a piece: every rescaling path of both kernels, with many
# segments and pieces per CTA.
OUTLIER = [
    # B, Hq, Hkv, D, lens, block_size, outlier scale
    (16, 32, 8, 128, [3000] * 16, None, 8.0),
    (8, 64, 4, 128, [4000, 100, 3000, 7, 5000, 1200, 999, 2500], 16, 8.0),
    (8, 64, 4, 128, [4000, 100, 3000, 7, 5000, 1200, 999, 2500], 16, 24.0),
    (2, 32, 2, 128, [60000, 30000], 64, 16.0),
    (6, 8, 1, 128, [2000, 1, 4097, 640, 130, 9000], 32, 16.0),
    (1, 16, 1, 128, [100000], None, 24.0),
    (4, 16, 4, 64, [5000, 3000, 1, 700], 16, 16.0),
    (4, 64, 1, 128, [6000, 3000, 1, 900], 16, 16.0),    # 64-head passes
    (1, 64, 1, 128, [100000], 64, 24.0),                # 64-head passes, split segment
    (4, 16, 4, 256, [5000, 3000, 1, 700], 16, 16.0),    # D = 256
    (1, 16, 2, 256, [60000], 64, 24.0),                 # D = 256, split segment
]


@pytest.mark.parametrize("case", OUTLIER,
                         ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_D{c[3]}_bs{c[5]}_x{c[6]:g}")
def test_key_outliers_rescale(case):
    B, Hq, Hkv, D, lens, bs, xs = case
    p = make_problem("outliers", B, Hq, Hkv, D, lens, seed=300 + sum(lens) + int(xs), block_size=bs,
                     key_outlier_frac=0.02, key_outlier_scale=xs)
    out = run(p)
    torch.cuda.synchronize()
    parity(out, ref(p), str(case), bf16_scaled=True)


def test_empty_batch_and_all_empty_requests():
    p = make_problem("empty", 3, 4, 1, 128, [0, 0, 0], seed=5, block_size=16)
    out = run(p)
    assert torch.all(out.float() == 0)
    p = make_problem("empty0", 0, 4, 1, 128, [], seed=5)
    assert run(p).numel() == 0


def test_single_key_returns_value_row():
    p = make_problem("one", 2, 8, 2, 128, [1, 1], seed=6)
    out = run(p).cpu()
    for b in range(2):
        for h in range(8):
            assert torch.equal(out[b, h], p.v_cache[b, h // 4, 0])


# --------------------------------------------------------------------- the five workloads

FULL = ["tiny", "llama3_8b", "long_256k"] + [f"sweep_{a}_{b}_{c}" for a, b, c in workloads.SWEEP]


def run_auto(p, out=None, workspace=None):
    """The bench's path: gqa_decode_auto with the host copy of the lengths."""
    d = p.to("cuda")
    return gq.gqa_decode_auto(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                              p.seq_lens.to(torch.int32).contiguous(), out=out, scale=p.scale,
                              workspace=workspace)


@pytest.mark.parametrize("name", FULL)
def test_workload_full_parity(name):
    """Every output of the full-size workload, through gqa_decode (stream-K) and
    gqa_decode_auto (the schedule the bench times), under the plain bar."""
    p = workloads.workload(name)
    r = ref(p)
    out = run(p)
    torch.cuda.synchronize()
    parity(out, r, name)
    out = run_auto(p)
    torch.cuda.synchronize()
    parity(out, r, name + " (auto)")


def test_varlen_paged_full():
    """Full-size variable-length paged batch: all 64 requests element by element
    (poisoned tail slots and unused table entries are never read), through both
    schedules."""
    p = workloads.workload("varlen_paged")
    r = ref(p)
    for fn, what in ((run, "stream-K"), (run_auto, "auto")):
        out = fn(p)
        torch.cuda.synchronize()
        parity(out, r, f"varlen_paged ({what})")


def test_auto_on_pages_the_tensor_cores_do_not_take():
    """gqa_decode_auto on page sizes the tensor-core kernel cannot tile (3, 100 tokens)
    with G = 4: the same result as gqa_decode, against the oracle."""
    for bs, lens in ((3, [50, 2000]), (100, [4000, 17])):
        p = make_problem("autopage", 2, 32, 8, 128, lens, seed=11 + bs, block_size=bs,
                         spare_blocks=2)
        r = ref(p)
        parity(run_auto(p), r, f"auto, {bs}-token pages")
        parity(run(p), r, f"decode, {bs}-token pages")
        dec = gq.HostDecoder(p.B, p.Hq, p.Hkv, p.D, p.block_size, p.max_blocks, p.num_blocks,
                             True)
        out = torch.empty_like(p.q)
        dec(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, out, scale=p.scale)
        parity(out, r, f"host buffers, {bs}-token pages")


# --------------------------------------------------------------------- invariants

def test_paging_permutation_bit_identical():
    """Renaming physical blocks leaves the GPU result bit-identical (the schedule
    depends only on the lengths)."""
    lens = [3000, 17, 1025]
    p = make_problem("perm", 3, 16, 4, 128, lens, seed=7, block_size=16, spare_blocks=5)
    a = run(p).cpu()
    perm = torch.randperm(p.num_blocks, generator=torch.Generator().manual_seed(8))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(p.num_blocks)
    p.k_cache = p.k_cache[inv].contiguous()
    p.v_cache = p.v_cache[inv].contiguous()
    valid = p.block_table >= 0
    p.block_table[valid] = perm[p.block_table[valid].long()].to(torch.int32)
    b = run(p).cpu()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_deterministic_repeat():
    p = workloads.workload("tiny")
    d = p.to("cuda")
    outs = [gq.gqa_decode(d.q, d.k_cache, d.v_cache, None, d.seq_lens).clone() for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


@pytest.mark.parametrize("name", ["long_256k", "one_segment_200k", "varlen_small", "mqa_200k", "d256_100k"])
def test_split_segments_bitwise_repeat(name):
    """Segments split over many CTAs are merged in a fixed order, so repeated calls
    give bit-identical outputs whatever the CTAs' timing (other work and an L2
    flush run between the calls to perturb it)."""
    if name == "long_256k":
        p = workloads.workload(name)
    elif name == "one_segment_200k":
        p = make_problem(name, 1, 16, 1, 128, [200000], seed=21, block_size=64)
    elif name == "d256_100k":  # D = 256 on the tensor cores
        p = make_problem(name, 1, 16, 2, 256, [100000], seed=24, block_size=64)
    elif name == "mqa_200k":   # the 64-heads-per-pass kernel
        p = make_problem(name, 2, 64, 1, 128, [200000, 31000], seed=23, block_size=64)
    else:
        p = make_problem(name, 6, 32, 8, 128, [40000, 1, 9000, 700, 25000, 3], seed=22,
                         block_size=16)
    d = p.to("cuda")
    junk = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    outs = []
    for i in range(4):
        junk.fill_(i)
        if i % 2:
            torch.cuda._sleep(1000 * (i + 1))
        outs.append(gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                                  scale=p.scale).clone())
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


def test_plan_matches_what_runs():
    """gqa_decode_plan's grid is the grid the timeline entry point records, for the
    stream-K and the one-CTA-per-segment schedule."""
    for name in ("long_256k", "tiny", "sweep_64_1_128"):
        p = workloads.workload(name)
        d = p.to("cuda")
        lens = p.seq_lens.to(torch.int32)
        auto = gq.decode_plan(p.B, p.Hq, p.Hkv, p.D, p.block_size, p.paged, p.num_blocks,
                              num_splits=-1, seq_lens_host=lens)
        for ns in (0, 1):
            plan = gq.decode_plan(p.B, p.Hq, p.Hkv, p.D, p.block_size, p.paged, p.num_blocks,
                                  num_splits=ns, seq_lens_host=lens)
            _, tl = gq.gqa_decode_timeline(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                                           num_splits=ns, scale=p.scale)
            torch.cuda.synchronize()
            assert tl.shape[0] == plan["grid"] > 0
            assert int(tl[:, 3].sum()) == plan["tiles"]
            assert plan["workspace_bytes"] > 0 and plan["smem_bytes"] > 0
        assert auto["num_splits"] == (1 if name == "tiny" else 0)


def test_contiguous_equals_paged():
    lens = [700, 300]
    p = make_problem("paged", 2, 8, 2, 128, lens, seed=9, block_size=64)
    cap = max(lens)
    kc = torch.full((2, 2, cap, 128), float("nan"), dtype=torch.bfloat16)
    vc = kc.clone()
    for b, L in enumerate(lens):
        t = torch.arange(L)
        blk = p.block_table[b, t // 64].long()
        kc[b, :, :L] = p.k_cache[blk, :, t % 64].transpose(0, 1)
        vc[b, :, :L] = p.v_cache[blk, :, t % 64].transpose(0, 1)
    a = run(p).cpu()
    c = workloads.Problem("contig", p.q, kc, vc, None, p.seq_lens, p.scale)
    b = run(c).cpu()
    parity(b, as_f64(a), "contiguous vs paged")


# --------------------------------------------------------------------- states and merge

def test_states_split_merge_matches_decode_and_oracle():
    lens = [2000, 513, 64]
    p = make_problem("split", 3, 16, 4, 128, lens, seed=10, block_size=16)
    d = p.to("cuda")
    full = gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, scale=p.scale)
    cuts = [[0, 1, 700, 2000], [0, 300, 301, 513], [0, 0, 64, 64]]
    pieces = []
    for s in range(3):
        b0 = torch.tensor([c[s] for c in cuts], dtype=torch.int32, device="cuda")
        b1 = torch.tensor([c[s + 1] for c in cuts], dtype=torch.int32, device="cuda")
        pieces.append(gq.gqa_decode_states(d.q, d.k_cache, d.v_cache, d.block_table, b0, b1,
                                           scale=p.scale))
        # states against the oracle's states
        acc, m, l = oracle.gqa_decode_states(p.q, p.k_cache, p.v_cache, p.block_table,
                                             b0.cpu(), b1.cpu(), p.scale)
        gm = as_f64(pieces[-1][1])
        fin = np.isfinite(m)
        assert np.array_equal(fin, np.isfinite(gm))
        assert np.allclose(gm[fin], m[fin], rtol=1e-5, atol=1e-5)
        ga, gl = as_f64(pieces[-1][0]), as_f64(pieces[-1][2])
        # compare normalised pieces (acc / l) where non-empty
        nz = l > 0
        assert np.allclose(gl[nz], l[nz], rtol=1e-4)
        parity(torch.from_numpy((ga[nz] / gl[nz][:, None])), acc[nz] / l[nz][:, None],
               f"piece {s}")
    acc = torch.stack([x[0] for x in pieces]).reshape(3, -1, 128)
    m = torch.stack([x[1] for x in pieces]).reshape(3, -1)
    l = torch.stack([x[2] for x in pieces]).reshape(3, -1)
    merged, lse = gq.gqa_merge_states(acc, m, l)
    torch.cuda.synchronize()
    r = ref(p)
    parity(merged.view(3, 16, 128), r, "merged vs oracle")
    parity(merged.view(3, 16, 128), as_f64(full), "merged vs gqa_decode")


def test_merge_states_against_oracle():
    # States shaped like real attention pieces: normalised outputs of O(0.1),
    # normalisers in [1, 100], maxima spread over a few units.
    g = torch.Generator().manual_seed(11)
    S, N, D = 5, 37, 128
    l = torch.rand((S, N), generator=g) * 99 + 1
    acc = torch.randn((S, N, D), generator=g) * 0.1 * l[..., None]
    m = torch.randn((S, N), generator=g) * 4
    m[1, :10] = -math.inf
    l[1, :10] = 0
    acc[1, :10] = 0
    m[:, 36] = -math.inf
    l[:, 36] = 0
    acc[:, 36] = 0
    out, lse = gq.gqa_merge_states(acc.cuda(), m.cuda(), l.cuda())
    torch.cuda.synchronize()
    r_out, r_lse = oracle.merge_states(acc.double().numpy(), m.double().numpy(),
                                       l.double().numpy())
    parity(out, r_out, "merge_states")
    gl = lse.cpu().double().numpy()
    assert gl[36] == -np.inf
    assert np.allclose(gl[:36], r_lse[:36], rtol=1e-6, atol=1e-5)


# --------------------------------------------------------------------- errors, no faults

@pytest.mark.parametrize("Hq", [4, 64])
def test_bad_block_id_sets_status_and_nan_rows(Hq):
    lens = [100, 90]
    p = make_problem("badblk", 2, Hq, 1, 128, lens, seed=12, block_size=16)
    p.block_table[1, 2] = p.num_blocks + 1000          # out of the pool: must not be read
    ws = gq.Workspace("cuda")
    out = run(p, workspace=ws)
    st = ws.status()
    assert st & gq.DEV_BAD_BLOCK
    o = out.cpu().float()
    assert torch.isnan(o[1]).all()
    r = ref(make_problem("badblk", 2, Hq, 1, 128, lens, seed=12, block_size=16))
    parity(out[0], r[0], "unaffected request")
    assert ws.status() == 0                             # cleared by the read


def test_length_above_capacity_sets_status():
    p = make_problem("badlen", 2, 4, 1, 128, [10, 20], seed=13, block_size=16)
    p.seq_lens[0] = 10 ** 6
    ws = gq.Workspace("cuda")
    out = run(p, workspace=ws)
    assert ws.status() & gq.DEV_BAD_LENGTH
    assert torch.isnan(out[0].float()).all()
    assert torch.isfinite(out[1].float()).all()


def test_workspace_too_small_is_an_error():
    p = make_problem("ws", 1, 4, 1, 128, [10], seed=14).to("cuda")
    ws = gq.Workspace("cuda")
    ws.buf = torch.zeros(64, dtype=torch.uint8, device="cuda")
    ws.get = lambda n: ws.buf
    with pytest.raises(gq.GqaError) as e:
        gq.gqa_decode(p.q, p.k_cache, p.v_cache, None, p.seq_lens, workspace=ws)
    assert e.value.code == gq.GQA_ERR_WORKSPACE_TOO_SMALL


def test_workspace_reused_across_shapes():
    """One workspace serves calls of different shapes in turn (counters stay at zero
    between calls)."""
    ws = gq.Workspace("cuda")
    shapes = [("a", 1, 4, 1, 128, [512], None), ("b", 16, 32, 8, 128, [3000] * 16, None),
              ("c", 2, 8, 2, 64, [900, 17], 16), ("d", 64, 8, 8, 128, [300] * 64, 16),
              ("a", 1, 4, 1, 128, [512], None)]
    for name, B, Hq, Hkv, D, lens, bs in shapes:
        p = make_problem(name, B, Hq, Hkv, D, lens, seed=B + D, block_size=bs)
        out = run(p, workspace=ws)
        torch.cuda.synchronize()
        parity(out, ref(p), f"shape {name}")
    assert ws.status() == 0


def test_max_batch():
    B = 4096
    lens = [(i * 37) % 300 for i in range(B)]
    p = make_problem("maxb", B, 8, 2, 64, lens, seed=15, block_size=16)
    out = run(p)
    torch.cuda.synchronize()
    rows = (1000 * 8, 1100 * 8)
    parity(out.view(-1, 64)[rows[0]:rows[1]], ref(p, rows=rows), "B=4096 sample")


def test_host_buffer_entry_point():
    p = make_problem("host", 2, 8, 2, 128, [300, 77], seed=16, block_size=16)
    dec = gq.HostDecoder(p.B, p.Hq, p.Hkv, p.D, p.block_size, p.max_blocks, p.num_blocks, True)
    pin = lambda t: t.pin_memory()
    out = torch.empty_like(p.q).pin_memory()
    dec(pin(p.q), pin(p.k_cache), pin(p.v_cache), pin(p.block_table), pin(p.seq_lens), out,
        scale=p.scale)
    parity(out, ref(p), "host-buffer call")
