// schedule.cuh -- kernel parameters and the stream-K LeanTile schedule shared by
// the decode kernels.
//
// Work decomposition (LeanAttention decode tiles digest, sections "Exact softmax
// that merges piece by piece" and "Hardware-sized work units"):
//   * the key range of every (request b, KV head kvh, head chunk hc) -- a
//     "segment" -- is cut into tiles of T tokens: n_b = ceil(len_b / T);
//   * tiles are numbered in one global order (b, kvh, hc, tile), W tiles in all;
//   * persistent CTA c of P takes the contiguous run [c*W/P, (c+1)*W/P), so every
//     CTA gets the same number of tiles (+-1) whatever the length mix;
//   * a segment split over several CTAs is merged exactly by the CTA that
//     finishes its piece last (ticket counter per segment; no waiting).
// Query heads of one KV head are processed in chunks of GC heads (hc), so the
// register-resident accumulators stay bounded for large groups.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace gqa {

constexpr unsigned DEV_BAD_BLOCK = 1u;
constexpr unsigned DEV_BAD_LENGTH = 2u;
constexpr unsigned DEV_TIMEOUT = 4u;

// Default upper bound on any single in-kernel wait for progress (a pipeline stage,
// another CTA's partial state); a healthy wait lasts microseconds.  A launch may
// carry a shorter one (Params::wait_ns).  The waits at exit for the CTA's own
// copies and tensor-core work in flight always use this default.
constexpr uint64_t WAIT_LIMIT_NS = 1500000000ull;

// Per-CTA timeline row (Params::timeline): start ns, end ns, SM id, tiles, then the
// phases of a tensor-core CTA with work (0 elsewhere): first TMA issue, first
// scores ready, end of streaming (last piece closed), end of merging.
constexpr int TL_COLS = 8;

struct Params {
    const uint16_t *q;            // [B, Hq, D] bf16
    const uint16_t *k;            // [num_blocks, Hkv, block_size, D] bf16
    const uint16_t *v;
    const int32_t *block_table;   // [B, max_blocks] or null (contiguous)
    const int32_t *seq_lens;      // [B]          (decode mode)
    const int32_t *kv_begin;      // [B]          (states mode)
    const int32_t *kv_end;        // [B]          (states mode)
    uint16_t *out;                // [B, Hq, D] bf16        (decode mode)
    float *st_acc;                // [B, Hq, D]             (states mode)
    float *st_m;                  // [B, Hq]
    float *st_l;                  // [B, Hq]
    unsigned *status;             // device status word
    int *counters;                // one ticket per segment
    int *gcounters;               // one ticket per CTA-group merge (index: leader slot)
    float *slots;                 // 2 partial states per CTA
    int B, Hq, Hkv, G, block_size, max_blocks, num_blocks;
    int hch;                      // head chunks per KV head
    int nsplit;                   // 0: stream-K runs; n > 0: fixed split, CTA = (segment, chunk)
    int qlen;                     // query tokens per request (1: decode; > 1: speculative verify)
    int R;                        // query rows per KV head: qlen * G
    int64_t capacity;             // tokens a request can hold
    uint32_t bs_magic;            // token -> page division by block_size (see page_of)
    int bs_shift;
    float qscale;                 // scale * log2(e) (* k_scale for FP8): scores in log2 units
    float vscale;                 // FP8 cache: v_scale, applied to the output (1 for bf16)
    unsigned long long *timeline; // optional [grid][TL_COLS], see TL_COLS
    uint64_t wait_ns;             // limit of each wait for progress (see WAIT_LIMIT_NS)
};

// floor(t / block_size) for 0 <= t < 2^31 without a divide: with l = ceil(log2 bs)
// and m = floor(2^32 (2^l - bs) / bs) + 1 (computed on the host),
// floor(t / bs) = (umulhi(m, t) + t) >> l (division by an invariant integer,
// Granlund & Montgomery 1994).
__device__ __forceinline__ int page_of(const Params &p, int t)
{
    const uint32_t u = (uint32_t)t;
    return (int)((__umulhi(p.bs_magic, u) + u) >> p.bs_shift);
}

// Quotient of non-negative x by positive y, in 32 bits when both fit (the
// 64-bit division is several times longer, and the prologue and the merge tail
// call these on their critical paths).
__device__ __forceinline__ int64_t div_nonneg(int64_t x, int64_t y)
{
    if ((((uint64_t)x | (uint64_t)y) >> 32) == 0)
        return (int64_t)((uint32_t)x / (uint32_t)y);
    return x / y;
}

// Walks the global tile order one tile at a time.  prefix[b] = sum of n_b'
// (b' < b) lives in shared memory; units = Hkv * hch segments per request.  Only
// init() divides; next() is increments and compares.
// Global tile order: head chunk outermost, then request, KV head, tile, i.e.
// (hc, b, kvh, j).  With one head chunk this is (b, kvh, j).  With several, the
// CTAs of the chunks run over the same (b, kvh, j) ranges side by side (exactly
// when the grid divides by the chunk count), so a K/V tile is read from HBM once
// and from L2 by the other chunks.  A segment is the nb tiles of one
// (b, kvh, hc); W = hch * Hkv * prefix[B].
struct TileIter {
    int b, kvh, hc;
    int j;         // tile index inside the segment
    int nb;        // tiles in the segment
    int64_t seg0;  // global index of the segment's first tile

    __device__ __forceinline__ void init(int64_t i, const int *prefix, int B, int64_t units,
                                         int hch)
    {
        const int64_t hkv = div_nonneg(units, hch);
        const int64_t w1 = hkv * prefix[B];  // tiles per head chunk
        hc = (int)div_nonneg(i, w1);
        const int64_t i1 = i - (int64_t)hc * w1;
        int lo = 0, hi = B;  // hkv*prefix[lo] <= i1 < hkv*prefix[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (hkv * prefix[mid] <= i1)
                lo = mid;
            else
                hi = mid;
        }
        b = lo;
        nb = prefix[lo + 1] - prefix[lo];
        const int64_t local = i1 - hkv * prefix[lo];
        kvh = (int)div_nonneg(local, nb);
        j = (int)(local - (int64_t)kvh * nb);
        seg0 = (int64_t)hc * w1 + hkv * prefix[lo] + (int64_t)kvh * nb;
    }

    // Advance to the next tile; the caller guarantees one exists.
    __device__ __forceinline__ void next(const int *prefix, int B, int Hkv, int hch)
    {
        (void)hch;
        if (++j < nb)
            return;
        j = 0;
        seg0 += nb;
        if (++kvh < Hkv)
            return;
        kvh = 0;
        // Next request with tiles; past the last one, the next head chunk's first.
        do {
            ++b;
        } while (b < B && prefix[b + 1] == prefix[b]);
        if (b == B) {
            ++hc;
            b = 0;
            while (prefix[b + 1] == prefix[b])
                ++b;
        }
        nb = prefix[b + 1] - prefix[b];
    }
};

// run_start(c) = floor(c * W / P) for consecutive c without dividing:
// (q, r) tracks the quotient and remainder of c * W by P.
struct RunWalker {
    int64_t q, r, qw, rw, P;
    __device__ __forceinline__ RunWalker(int64_t c, int64_t W, int64_t P_)
    {
        P = P_;
        qw = W / P;
        rw = W - qw * P;
        const int64_t cw = c * W;
        q = cw / P;
        r = cw - q * P;
    }
    __device__ __forceinline__ int64_t start() const { return q; }
    __device__ __forceinline__ void next()
    {
        q += qw;
        r += rw;
        if (r >= P) {
            r -= P;
            ++q;
        }
    }
};

// First tile of CTA c, and the CTA whose run holds tile i.
__device__ __forceinline__ int64_t run_start(int64_t c, int64_t W, int64_t P)
{
    return div_nonneg(c * W, P);
}
__device__ __forceinline__ int64_t tile_owner(int64_t i, int64_t W, int64_t P)
{
    return div_nonneg((i + 1) * P - 1, W);
}

// Requested key range of request b; returns false for an invalid range.
template <bool STATES>
__device__ __forceinline__ bool request_range(const Params &p, int b, int64_t &begin, int64_t &len)
{
    int64_t b0 = 0, b1;
    if (STATES) {
        b0 = p.kv_begin[b];
        b1 = p.kv_end[b];
    } else {
        b1 = p.seq_lens[b];
    }
    // With qlen > 1 query tokens the request must hold at least qlen tokens.
    bool ok = b0 >= 0 && b1 >= b0 && b1 <= p.capacity && (STATES || p.qlen <= 1 || b1 >= p.qlen);
    begin = ok ? b0 : 0;
    len = ok ? b1 - b0 : 0;
    return ok;
}

// Output row of query row r (0 <= r < R) of (request b, KV head kvh): query token
// r / G, head kvh * G + r % G, in the [B, qlen, Hq] row order of q and out.
__device__ __forceinline__ int64_t out_row(const Params &p, int b, int kvh, int r)
{
    const int i = r / p.G, h = r - i * p.G;
    return ((int64_t)b * p.qlen + i) * p.Hq + (int64_t)kvh * p.G + h;
}

// out_row for one query token per request (qlen = 1): no division.
__device__ __forceinline__ int64_t out_row_q1(const Params &p, int b, int kvh, int r)
{
    return (int64_t)b * p.Hq + (int64_t)kvh * p.G + r;
}

// Bounded wait on an mbarrier phase (at most p.wait_ns).  On timeout: status bit,
// CTA abort flag.
__device__ __forceinline__ bool bounded_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             const Params &p)
{
    if (mbar_try_wait(bar, parity))
        return true;
    if (*abort_flag)
        return false;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag)
            return false;
        if (global_timer_ns() - t0 > p.wait_ns) {
            atomicOr(p.status, DEV_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// Writes one finished output element (and, in states mode, m and l).
template <bool STATES>
__device__ __forceinline__ void write_result(const Params &p, int64_t row, int d, int D, float a,
                                             float ms, float ls, bool poisoned)
{
    if (STATES) {
        p.st_acc[row * D + d] = poisoned ? __int_as_float(0x7fc00000) : a;
        if (d == 0) {
            p.st_m[row] = ms == -INFINITY ? -INFINITY : ms * 0.69314718055994531f;
            p.st_l[row] = poisoned ? __int_as_float(0x7fc00000) : ls;
        }
    } else {
        // (fast reciprocal division: well inside the bf16 output's precision)
        float o = poisoned ? __int_as_float(0x7fc00000) : (ls > 0.f ? __fdividef(p.vscale * a, ls) : 0.f);
        __nv_bfloat16 h = __float2bfloat16_rn(o);
        p.out[row * D + d] = *reinterpret_cast<uint16_t *>(&h);
    }
}


// Slot of one partial state: acc [NH][D], then m [NH] and l [NH] (log2 units),
// padded to a 16-byte multiple so float4 loads stay aligned.
__host__ __device__ constexpr int slot_floats(int NH, int D) { return NH * D + ((2 * NH + 3) / 4) * 4; }

// ---------------------------------------------------------------------------
// Exact merge of partial pieces (LeanAttention decode tiles digest, section
// "Exact softmax that merges piece by piece"): every piece keeps its own maximum,
// normaliser and weighted values; rescaling all of them to the common maximum and
// adding is exact in any order.  Pieces are combined in CTA order, so the result
// does not depend on which CTA arrived last.
//
// Two levels, so that no single CTA reads every piece of a long segment: the
// owners of a segment are grouped by MERGE_GROUP consecutive CTAs; the last
// arriver of each group merges the group's pieces into the slot of the group's
// first owner, then takes the segment ticket; the last group merger combines the
// group results (one group: it writes the output directly).
constexpr int MERGE_GROUP = 8;

__host__ __device__ constexpr int merge_scratch_floats(int NP, int NT, int P)
{
    return P + 8;  // the slot list (ints)
}

// Merges the n slots listed in `list` (shared memory), in list order.  Every
// thread owns R float4 outputs and merges them online, four pieces per round
// trip to L2: load (m, l, acc) of the pieces, raise the running maximum, rescale
// and add.  No barriers: threads never exchange data.  dst_slot == nullptr: the
// result goes to output rows row0 .. row0 + rows - 1; otherwise it is written to
// dst_slot as a partial state again (log2 units); dst_slot may be one of the
// sources, so every thread finishes reading (barrier bar_id) before any writes.
template <int NP, int D, int NT, bool STATES>
__device__ __forceinline__ void merge_slots(const Params &p, const int *list, int n,
                                            float *dst_slot, int rows, int64_t row0, int t,
                                            int bar_id)
{
    constexpr int SF = slot_floats(NP, D);
    constexpr int NF4 = NP * D / 4;                  // float4 outputs
    constexpr int R = (NF4 + NT - 1) / NT;
    constexpr int U = R >= 4 ? 4 : 8 / R;            // pieces per round trip
    float4 acc[R];
    float mrun[R], lrun[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        mrun[r] = -INFINITY;
        lrun[r] = 0.f;
    }
    for (int o0 = 0; o0 < n; o0 += U) {
        float4 v[U][R];
        float mv[U][R], lv[U][R];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const bool have = o0 + u < n;
            const float *sl = p.slots + (int64_t)(have ? list[o0 + u] : list[0]) * SF;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int f = t + r * NT;
                const bool ok = have && f < NF4;
                const int g = ok ? (4 * f) / D : 0;
                v[u][r] = ok ? __ldcg(reinterpret_cast<const float4 *>(sl) + f) : make_float4(0.f, 0.f, 0.f, 0.f);
                mv[u][r] = ok ? __ldcg(sl + NP * D + g) : -INFINITY;
                lv[u][r] = ok ? __ldcg(sl + NP * D + NP + g) : 0.f;
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float mnew = mrun[r];
#pragma unroll
            for (int u = 0; u < U; ++u)
                mnew = fmaxf(mnew, mv[u][r]);
            if (mnew == -INFINITY)
                continue;  // nothing non-empty yet
            const float sc = fast_exp2(mrun[r] - mnew);  // exp2(-inf) = 0
            float4 a = make_float4(acc[r].x * sc, acc[r].y * sc, acc[r].z * sc, acc[r].w * sc);
            float l = lrun[r] * sc;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const float w = mv[u][r] == -INFINITY ? 0.f : fast_exp2(mv[u][r] - mnew);
                a.x = fmaf(w, v[u][r].x, a.x);
                a.y = fmaf(w, v[u][r].y, a.y);
                a.z = fmaf(w, v[u][r].z, a.z);
                a.w = fmaf(w, v[u][r].w, a.w);
                l = fmaf(w, lv[u][r], l);
            }
            acc[r] = a;
            lrun[r] = l;
            mrun[r] = mnew;
        }
    }
    if (dst_slot)
        named_barrier_sync(bar_id, NT);
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int f = t + r * NT;
        if (f >= NF4)
            continue;
        const int g = (4 * f) / D, d = (4 * f) % D;
        if (dst_slot) {
            reinterpret_cast<float4 *>(dst_slot)[f] = acc[r];
            if (d == 0) {
                dst_slot[NP * D + g] = mrun[r];
                dst_slot[NP * D + NP + g] = lrun[r];
            }
            continue;
        }
        if (g >= rows)
            continue;
        const float ls = lrun[r], ms = mrun[r];
        const bool bad = ls != ls;
        write_result<STATES>(p, row0 + g, d, D, acc[r].x, ms, ls, bad);
        write_result<STATES>(p, row0 + g, d + 1, D, acc[r].y, ms, ls, bad);
        write_result<STATES>(p, row0 + g, d + 2, D, acc[r].z, ms, ls, bad);
        write_result<STATES>(p, row0 + g, d + 3, D, acc[r].w, ms, ls, bad);
    }
}

// Ticket: atomic add with acquire-release semantics at GPU scope.  Called by one
// thread after a CTA barrier, it publishes every write the CTA made before the
// barrier (release) and, for the last arriver, makes every other CTA's published
// writes visible to this CTA after the next barrier (acquire).
__device__ __forceinline__ int ticket_add(int *counter, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(counter), "r"(v) : "memory");
    return old;
}

// A partial piece whose slot is written and whose ticket is still to be taken.
// Tickets (and the merges they may trigger) wait until the CTA has streamed all
// its tiles: the segment cannot complete before its other owners reach the end
// of their runs anyway, and a merge in mid-run would stall this CTA's pipeline.
struct PendingPiece {
    int64_t seg0, first, end, vseg, row0;  // row0: first output row (qlen = 1 kernels)
    int nb, rows;
    int b, kvh, r0;                        // request, KV head, first query row (any qlen)
};

// Slot of CTA cc's piece of the segment starting at tile seg0, or -1 if cc owns
// no tile (its run is empty).
__device__ __forceinline__ int piece_slot(int64_t cc, int64_t seg0, int64_t W, int64_t P)
{
    const int64_t s0 = run_start(cc, W, P), s1 = run_start(cc + 1, W, P);
    return s0 == s1 ? -1 : (int)(2 * cc + (s0 < seg0 ? 1 : 0));
}

// Called by all NT threads after this CTA wrote its partial piece of a segment
// (tiles [piece_first, piece_end) of [seg0, seg0 + nb)) to its slot.  Takes the
// group ticket and, for the last arriver of the group, merges the group and
// takes the segment ticket; the last group merger writes the output.
// counters: per-segment ticket (index vseg); gcounters: per-group tickets (index =
// slot of the group's first owner).  Both are left at zero by whoever finishes.
// merge(list, n, dst_slot) combines the n listed slots (merge_slots bound to
// this segment's rows).
template <int NP, int D, int NT, bool STATES, class MergeFn>
__device__ __forceinline__ void finish_partial(const Params &p, int64_t c, int64_t seg0, int nb,
                                               int64_t piece_first, int64_t piece_end,
                                               int64_t vseg, int64_t W, int64_t P, float *scr,
                                               int *flag, int t, int bar_id, MergeFn &&merge)
{
    int *list = reinterpret_cast<int *>(scr);  // slot list: <= P ints
    const int64_t seg1 = seg0 + nb;
    named_barrier_sync(bar_id, NT);  // this CTA's slot writes precede the ticket
    const int64_t c0 = tile_owner(seg0, W, P), c1 = tile_owner(seg1 - 1, W, P);
    const int64_t g = c / MERGE_GROUP;
    const int64_t ga = max(c0, g * MERGE_GROUP), gb = min(c1, g * MERGE_GROUP + MERGE_GROUP - 1);
    const bool one_group = c0 / MERGE_GROUP == c1 / MERGE_GROUP;
    if (t == 0) {
        // Group ticket (tiles of this segment owned by the group's CTAs).
        const int64_t gt0 = max(seg0, run_start(ga, W, P)), gt1 = min(seg1, run_start(gb + 1, W, P));
        int lead = -1;
        for (int64_t cc = ga; cc <= gb && lead < 0; ++cc)
            lead = piece_slot(cc, seg0, W, P);
        const int mine = (int)(piece_end - piece_first);
        const int old = ticket_add(&p.gcounters[lead], mine);
        flag[0] = (old + mine == (int)(gt1 - gt0)) ? 1 : 0;
        flag[1] = lead;
        flag[2] = (int)(gt1 - gt0);
    }
    named_barrier_sync(bar_id, NT);
    if (!*reinterpret_cast<volatile int *>(flag))
        return;
    const int lead = flag[1], gtiles = flag[2];
    // Group merge: the group's owners in CTA order.
    {
        const int no = (int)(gb - ga + 1);
        for (int o = t; o < no; o += NT)
            list[o] = piece_slot(ga + o, seg0, W, P);
        named_barrier_sync(bar_id, NT);
        if (t == 0) {
            int m = 0;
            for (int o = 0; o < no; ++o)
                if (list[o] >= 0)
                    list[m++] = list[o];
            flag[3] = m;
        }
        named_barrier_sync(bar_id, NT);
        const int m = flag[3];
        float *dst = one_group ? nullptr : p.slots + (int64_t)lead * slot_floats(NP, D);
        merge(list, m, dst);
        if (t == 0)
            p.gcounters[lead] = 0;
    }
    if (one_group)
        return;
    // Segment ticket, counted in tiles; the last group merger combines the groups.
    named_barrier_sync(bar_id, NT);  // the group result precedes the ticket
    if (t == 0) {
        const int old = ticket_add(&p.counters[vseg], gtiles);
        flag[0] = (old + gtiles == nb) ? 1 : 0;
    }
    named_barrier_sync(bar_id, NT);
    if (!*reinterpret_cast<volatile int *>(flag))
        return;
    {
        const int64_t g0 = c0 / MERGE_GROUP, g1 = c1 / MERGE_GROUP;
        const int ng = (int)(g1 - g0 + 1);
        for (int o = t; o < ng; o += NT) {
            const int64_t gg = g0 + o;
            const int64_t a = max(c0, gg * MERGE_GROUP), z = min(c1, gg * MERGE_GROUP + MERGE_GROUP - 1);
            int s = -1;
            for (int64_t cc = a; cc <= z && s < 0; ++cc)
                s = piece_slot(cc, seg0, W, P);
            list[o] = s;
        }
        named_barrier_sync(bar_id, NT);
        if (t == 0) {
            int m = 0;
            for (int o = 0; o < ng; ++o)
                if (list[o] >= 0)
                    list[m++] = list[o];
            flag[3] = m;
            p.counters[vseg] = 0;
        }
        named_barrier_sync(bar_id, NT);
        merge(list, flag[3], static_cast<float *>(nullptr));
    }
}

}  // namespace gqa
