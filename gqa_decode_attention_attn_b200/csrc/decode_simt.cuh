// decode_simt.cuh -- persistent stream-K decode-attention kernel, CUDA-core
// arithmetic (used when few query heads share a KV head, so that q.K^T is too
// thin to be a dense contraction).
//
// Per CTA: one producer warp and NC consumer warps.
//   producer  walks the CTA's run of tiles and, for each tile, issues bulk
//             asynchronous copies (one per page piece) of the K and V rows into a
//             STAGES-deep shared-memory ring; completion is counted in bytes on a
//             "full" mbarrier, and consumers hand slots back on an "empty" one.
//   consumers split every tile's T tokens evenly.  A warp reads a token row with
//             16-byte loads, D/8 lanes per token; every KV row is loaded once from
//             HBM and reused by all GC query heads of the chunk.  q.k partial dots
//             are reduced across the token's lanes with butterfly shuffles, then
//             the online softmax (running max m, running sum l, in log2 units)
//             rescales the fp32 accumulators and adds p * V.
//   epilogue  at the end of a segment piece the NC warp states are merged in
//             shared memory; a whole segment writes bf16 output directly, a
//             partial one stores (acc, m, l) in its workspace slot and takes a
//             ticket; the CTA completing the segment merges all pieces in CTA
//             order (deterministic) and writes the output.
// FlashAttention-style fusion of BMM1 -> online softmax -> BMM2 (Attention
// co-design for long-context inference, section "FlashAttention and GEMM
// shapes"); exact piecewise merge (LeanAttention decode tiles digest, section
// "Exact softmax that merges piece by piece").
#pragma once

#include <cuda_bf16.h>

#include "schedule.cuh"

namespace gqa {

template <int D, int GC>
struct SimtCfg {
    static constexpr int NC = 8;                       // consumer warps
    static constexpr int THREADS = (NC + 1) * 32;
    static constexpr int T = 32768 / (4 * D);          // tokens per tile: 32 KB of K+V
    static constexpr int STAGES = 4;
    static constexpr int LPT = D / 8;                  // lanes per token (16 B each)
    static constexpr int TPW = 32 / LPT;               // tokens per warp step
    static constexpr int TOKW = T / NC;                // tokens per warp per tile
    static constexpr int STEPS = TOKW / TPW;           // warp steps per tile
    static constexpr int TILE_ELEMS = T * D;
    static constexpr int SCRATCH_PER_WARP = GC * D + ((2 * GC + 3) / 4) * 4;  // 16-byte multiple
    static constexpr size_t RING_BYTES = 2ull * STAGES * TILE_ELEMS * sizeof(uint16_t);
    static constexpr size_t BAR_OFF = RING_BYTES;
    static constexpr size_t FLAG_OFF = BAR_OFF + 2 * STAGES * sizeof(uint64_t);
    static constexpr size_t SCRATCH_OFF = FLAG_OFF + 32 * sizeof(int);
    static constexpr size_t PREFIX_OFF = SCRATCH_OFF + (size_t)NC * SCRATCH_PER_WARP * sizeof(float);
    static constexpr int SLOT_FLOATS = GC * (D + 2);   // one partial state
    static size_t smem_bytes(int B) { return PREFIX_OFF + (size_t)(B + 1) * sizeof(int); }
    static_assert(STEPS >= 1 && TOKW % TPW == 0, "tile must split evenly over warps");
    static_assert(2 * STAGES <= 24, "flag area");
};

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
        float o = poisoned ? __int_as_float(0x7fc00000) : (ls > 0.f ? a / ls : 0.f);
        __nv_bfloat16 h = __float2bfloat16_rn(o);
        p.out[row * D + d] = *reinterpret_cast<uint16_t *>(&h);
    }
}

template <int D, int GC, bool STATES>
__global__ void __launch_bounds__(SimtCfg<D, GC>::THREADS, 1)
    gqa_decode_simt_kernel(const Params p)
{
    using C = SimtCfg<D, GC>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint16_t *kring = reinterpret_cast<uint16_t *>(smem);
    uint16_t *vring = kring + C::STAGES * C::TILE_ELEMS;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + C::STAGES;
    int *stage_bad = reinterpret_cast<int *>(smem + C::FLAG_OFF);  // [STAGES]
    int *stage_n = stage_bad + C::STAGES;                           // [STAGES] valid tokens
    volatile int *abort_flag = stage_bad + 24;
    int *last_flag = stage_bad + 25;
    int *poison_flag = stage_bad + 26;
    float *scratch = reinterpret_cast<float *>(smem + C::SCRATCH_OFF);
    int *prefix = reinterpret_cast<int *>(smem + C::PREFIX_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.B;

    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::NC);
            stage_bad[s] = 0;
        }
        *abort_flag = 0;
        *last_flag = 0;
        *poison_flag = 0;
        fence_mbar_init();
    }
    // Tiles per request, then an exclusive prefix sum (warp 0).
    for (int b = tid; b < B; b += C::THREADS) {
        int64_t begin, len;
        bool ok = request_range<STATES>(p, b, begin, len);
        if (!ok && blockIdx.x == 0)
            atomicOr(p.status, DEV_BAD_LENGTH);
        prefix[b + 1] = (int)((len + C::T - 1) / C::T);
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < B; base += 32) {
            int b = base + lane;
            int x = b < B ? prefix[b + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o)
                    x += y;
            }
            if (b < B)
                prefix[b + 1] = carry + x;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0)
            prefix[0] = 0;
    }
    __syncthreads();

    const int64_t units = (int64_t)p.Hkv * p.hch;
    const int64_t W = units * prefix[B];
    const int64_t P = gridDim.x, c = blockIdx.x;
    const int64_t start = run_start(c, W, P), end = run_start(c + 1, W, P);

    // Requests without tiles (empty, or an invalid range) get their rows here.
    for (int b = (int)c; b < B; b += (int)P) {
        if (prefix[b + 1] != prefix[b])
            continue;
        int64_t begin, len;
        bool bad = !request_range<STATES>(p, b, begin, len);
        for (int e = tid; e < p.Hq * D; e += C::THREADS)
            write_result<STATES>(p, (int64_t)b * p.Hq + e / D, e % D, D, 0.f, -INFINITY, 0.f, bad);
    }
    if (start >= end)
        return;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol = l2_evict_first_policy();
        int64_t k = 0;
        for (int64_t i = start; i < end; ++i, ++k) {
            const int s = (int)(k % C::STAGES);
            const uint32_t ph = (uint32_t)((k / C::STAGES) & 1);
            if (k >= C::STAGES && !bounded_wait(&empty[s], ph ^ 1u, abort_flag, p.status))
                break;
            const Tile t = locate_tile(i, prefix, B, units, p.hch);
            int64_t begin, len;
            request_range<STATES>(p, t.b, begin, len);
            const int64_t tok0 = begin + (int64_t)t.j * C::T;
            const int64_t n = min((int64_t)C::T, len - (int64_t)t.j * C::T);
            const int64_t bs = p.block_size;
            const int64_t pg0 = tok0 / bs, pg1 = (tok0 + n - 1) / bs;
            const int npieces = (int)(pg1 - pg0 + 1);
            uint32_t bytes = 0;
            bool bad = false;
            for (int pc = lane; pc < npieces; pc += 32) {
                const int64_t pg = pg0 + pc;
                const int64_t blk = p.block_table ? p.block_table[(int64_t)t.b * p.max_blocks + pg] : t.b;
                if (p.block_table && (blk < 0 || blk >= p.num_blocks)) {
                    bad = true;
                } else {
                    const int64_t a = max(tok0, pg * bs), z = min(tok0 + n, (pg + 1) * bs);
                    bytes += (uint32_t)((z - a) * D * 2 * 2);
                }
            }
            bad = __any_sync(0xffffffffu, bad);
#pragma unroll
            for (int o = 16; o; o >>= 1)
                bytes += __shfl_xor_sync(0xffffffffu, bytes, o);
            if (lane == 0) {
                stage_bad[s] = bad ? 1 : 0;
                stage_n[s] = (int)n;
                if (bad)
                    atomicOr(p.status, DEV_BAD_BLOCK);
                mbar_arrive_expect_tx(&full[s], bytes);
            }
            __syncwarp();
            for (int pc = lane; pc < npieces; pc += 32) {
                const int64_t pg = pg0 + pc;
                const int64_t blk = p.block_table ? p.block_table[(int64_t)t.b * p.max_blocks + pg] : t.b;
                if (p.block_table && (blk < 0 || blk >= p.num_blocks))
                    continue;
                const int64_t a = max(tok0, pg * bs), z = min(tok0 + n, (pg + 1) * bs);
                const int64_t src = ((blk * p.Hkv + t.kvh) * bs + (a - pg * bs)) * D;
                const int64_t dst = (int64_t)s * C::TILE_ELEMS + (a - tok0) * D;
                const uint32_t nb = (uint32_t)((z - a) * D * 2);
                bulk_copy_g2s(kring + dst, p.k + src, nb, &full[s], pol);
                bulk_copy_g2s(vring + dst, p.v + src, nb, &full[s], pol);
            }
        }
        // Never leave copies in flight: wait for the last issued phase of each slot.
        if (lane == 0) {
            for (int64_t kk = max((int64_t)0, k - C::STAGES); kk < k; ++kk) {
                const int s = (int)(kk % C::STAGES);
                const uint32_t ph = (uint32_t)((kk / C::STAGES) & 1);
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(&full[s], ph) && global_timer_ns() - t0 < WAIT_LIMIT_NS) {
                }
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int cw = warp - 1;               // consumer warp index
    const int ctid = tid - 32;             // consumer thread index
    const int grp = lane / C::LPT;         // token slot inside a warp step
    const int d0 = (lane % C::LPT) * 8;    // this lane's 8 dimensions
    const int G = p.G;

    float qf[GC][8], acc[GC][8], m[GC], l[GC];
    bool poisoned = false;
    Tile cur{};
    int64_t piece_first = start;
    int64_t k = 0;

    for (int64_t i = start; i < end; ++i, ++k) {
        const Tile t = locate_tile(i, prefix, B, units, p.hch);
        if (i == start || t.seg0 != cur.seg0) {
            cur = t;
            piece_first = i;
            poisoned = false;
#pragma unroll
            for (int g = 0; g < GC; ++g) {
                const int hg = t.hc * GC + g;  // head inside the group
                uint4 w = make_uint4(0, 0, 0, 0);
                if (hg < G)
                    w = __ldg(reinterpret_cast<const uint4 *>(
                        p.q + (((int64_t)t.b * p.Hq + (int64_t)t.kvh * G + hg) * D + d0)));
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float lo, hi;
                    bf16x2_to_float2(ww[j], lo, hi);
                    qf[g][2 * j] = lo * p.qscale;
                    qf[g][2 * j + 1] = hi * p.qscale;
                }
                m[g] = -INFINITY;
                l[g] = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    acc[g][j] = 0.f;
            }
        }

        const int s = (int)(k % C::STAGES);
        const uint32_t ph = (uint32_t)((k / C::STAGES) & 1);
        const bool ready = bounded_wait(&full[s], ph, abort_flag, p.status);
        if (!ready) {
            poisoned = true;
        } else {
            poisoned |= stage_bad[s] != 0;
            const int n = stage_n[s];
            const uint16_t *Ks = kring + s * C::TILE_ELEMS;
            const uint16_t *Vs = vring + s * C::TILE_ELEMS;

            float sc[C::STEPS][GC];
            bool valid[C::STEPS];
#pragma unroll
            for (int st = 0; st < C::STEPS; ++st) {
                const int tt = cw * C::TOKW + st * C::TPW + grp;
                valid[st] = tt < n;
                uint4 w = make_uint4(0, 0, 0, 0);
                if (valid[st])
                    w = *reinterpret_cast<const uint4 *>(Ks + tt * D + d0);
                float kf[8];
                bf16x2_to_float2(w.x, kf[0], kf[1]);
                bf16x2_to_float2(w.y, kf[2], kf[3]);
                bf16x2_to_float2(w.z, kf[4], kf[5]);
                bf16x2_to_float2(w.w, kf[6], kf[7]);
#pragma unroll
                for (int g = 0; g < GC; ++g) {
                    float a = 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        a = fmaf(qf[g][j], kf[j], a);
                    sc[st][g] = a;
                }
            }
            // Full dot products: butterfly over the LPT lanes of each token.
#pragma unroll
            for (int o = C::LPT / 2; o >= 1; o >>= 1)
#pragma unroll
                for (int st = 0; st < C::STEPS; ++st)
#pragma unroll
                    for (int g = 0; g < GC; ++g)
                        sc[st][g] += __shfl_xor_sync(0xffffffffu, sc[st][g], o);
            // Online softmax over this warp's tokens of the tile (scores become
            // probabilities in place).
#pragma unroll
            for (int g = 0; g < GC; ++g) {
                float mx = -INFINITY;
#pragma unroll
                for (int st = 0; st < C::STEPS; ++st)
                    if (valid[st])
                        mx = fmaxf(mx, sc[st][g]);
#pragma unroll
                for (int o = C::LPT; o < 32; o <<= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const float mnew = fmaxf(m[g], mx);
                const float muse = mnew == -INFINITY ? 0.f : mnew;
                const float alpha = exp2f(m[g] - muse);
                float ps = 0.f;
#pragma unroll
                for (int st = 0; st < C::STEPS; ++st) {
                    sc[st][g] = valid[st] ? exp2f(sc[st][g] - muse) : 0.f;
                    ps += sc[st][g];
                }
                l[g] = l[g] * alpha + ps;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    acc[g][j] *= alpha;
                m[g] = mnew;
            }
#pragma unroll
            for (int st = 0; st < C::STEPS; ++st) {
                if (!valid[st])
                    continue;
                const int tt = cw * C::TOKW + st * C::TPW + grp;
                const uint4 w = *reinterpret_cast<const uint4 *>(Vs + tt * D + d0);
                float vf[8];
                bf16x2_to_float2(w.x, vf[0], vf[1]);
                bf16x2_to_float2(w.y, vf[2], vf[3]);
                bf16x2_to_float2(w.z, vf[4], vf[5]);
                bf16x2_to_float2(w.w, vf[6], vf[7]);
#pragma unroll
                for (int g = 0; g < GC; ++g)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        acc[g][j] = fmaf(sc[st][g], vf[j], acc[g][j]);
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]);

        const bool piece_end = (i + 1 == end) || (i + 1 == t.seg0 + t.nb);
        if (!piece_end)
            continue;

        // ------------------------------------------------------------ epilogue
        // Token slots of a warp share m; add their l and acc.
#pragma unroll
        for (int g = 0; g < GC; ++g) {
#pragma unroll
            for (int o = C::LPT; o < 32; o <<= 1) {
                l[g] += __shfl_xor_sync(0xffffffffu, l[g], o);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    acc[g][j] += __shfl_xor_sync(0xffffffffu, acc[g][j], o);
            }
        }
        float *mine = scratch + cw * C::SCRATCH_PER_WARP;
        if (grp == 0) {
#pragma unroll
            for (int g = 0; g < GC; ++g) {
                float4 *dst = reinterpret_cast<float4 *>(mine + g * D + d0);
                dst[0] = make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
                dst[1] = make_float4(acc[g][4], acc[g][5], acc[g][6], acc[g][7]);
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int g = 0; g < GC; ++g) {
                mine[GC * D + g] = m[g];
                mine[GC * D + GC + g] = l[g];
            }
            if (poisoned)
                atomicOr(poison_flag, 1);
        }
        named_barrier_sync(1, C::NC * 32);

        const bool pois = *reinterpret_cast<volatile int *>(poison_flag) != 0;
        const bool complete = piece_first == cur.seg0 && i + 1 == cur.seg0 + cur.nb;
        const int rows = min(GC, G - cur.hc * GC);
        const int64_t row0 = (int64_t)cur.b * p.Hq + (int64_t)cur.kvh * G + (int64_t)cur.hc * GC;
        const int64_t vseg = ((int64_t)cur.b * p.Hkv + cur.kvh) * p.hch + cur.hc;
        float *slot = p.slots + (2 * c + (piece_first == start ? 0 : 1)) * (int64_t)C::SLOT_FLOATS;

        for (int e = ctid; e < GC * D; e += C::NC * 32) {
            const int g = e / D, d = e - (e / D) * D;
            if (g >= rows)
                continue;
            float ms = -INFINITY;
#pragma unroll
            for (int w = 0; w < C::NC; ++w)
                ms = fmaxf(ms, scratch[w * C::SCRATCH_PER_WARP + GC * D + g]);
            float a = 0.f, ls = 0.f;
#pragma unroll
            for (int w = 0; w < C::NC; ++w) {
                const float *sw = scratch + w * C::SCRATCH_PER_WARP;
                const float mw = sw[GC * D + g];
                const float wt = mw == -INFINITY ? 0.f : exp2f(mw - ms);
                a = fmaf(wt, sw[g * D + d], a);
                ls = fmaf(wt, sw[GC * D + GC + g], ls);
            }
            if (complete) {
                write_result<STATES>(p, row0 + g, d, D, a, ms, ls, pois);
            } else {
                slot[g * D + d] = a;
                if (d == 0) {
                    slot[GC * D + g] = ms;
                    slot[GC * D + GC + g] = pois ? __int_as_float(0x7fc00000) : ls;
                }
            }
        }
        named_barrier_sync(1, C::NC * 32);

        if (!complete) {
            if (ctid == 0) {
                *poison_flag = 0;
                __threadfence();
                const int ntiles = (int)(i + 1 - piece_first);
                const int old = atomicAdd(&p.counters[vseg], ntiles);
                *last_flag = (old + ntiles == cur.nb) ? 1 : 0;
            }
            named_barrier_sync(1, C::NC * 32);
            if (*reinterpret_cast<volatile int *>(last_flag)) {
                __threadfence();
                const int64_t seg1 = cur.seg0 + cur.nb;
                const int64_t c0 = tile_owner(cur.seg0, W, P), c1 = tile_owner(seg1 - 1, W, P);
                for (int e = ctid; e < GC * D; e += C::NC * 32) {
                    const int g = e / D, d = e - (e / D) * D;
                    if (g >= rows)
                        continue;
                    float ms = -INFINITY;
                    for (int64_t cc = c0; cc <= c1; ++cc) {
                        const int64_t s0 = run_start(cc, W, P);
                        if (s0 == run_start(cc + 1, W, P))
                            continue;
                        const float *sl = p.slots + (2 * cc + (s0 < cur.seg0 ? 1 : 0)) * (int64_t)C::SLOT_FLOATS;
                        ms = fmaxf(ms, __ldcg(sl + GC * D + g));
                    }
                    float a = 0.f, ls = 0.f;
                    for (int64_t cc = c0; cc <= c1; ++cc) {
                        const int64_t s0 = run_start(cc, W, P);
                        if (s0 == run_start(cc + 1, W, P))
                            continue;
                        const float *sl = p.slots + (2 * cc + (s0 < cur.seg0 ? 1 : 0)) * (int64_t)C::SLOT_FLOATS;
                        const float mw = __ldcg(sl + GC * D + g);
                        const float wt = mw == -INFINITY ? 0.f : exp2f(mw - ms);
                        a = fmaf(wt, __ldcg(sl + g * D + d), a);
                        ls = fmaf(wt, __ldcg(sl + GC * D + GC + g), ls);
                    }
                    write_result<STATES>(p, row0 + g, d, D, a, ms, ls, ls != ls);
                }
                if (ctid == 0)
                    p.counters[vseg] = 0;
            }
        } else if (ctid == 0) {
            *poison_flag = 0;
        }
        named_barrier_sync(1, C::NC * 32);
    }
}

}  // namespace gqa
