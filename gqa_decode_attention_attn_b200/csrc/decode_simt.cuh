// decode_simt.cuh -- persistent stream-K decode-attention kernel, CUDA-core
// arithmetic (used when few query heads share a KV head, so that q.K^T is too
// thin to be a dense contraction: G query heads give M = G rows).
//
// Per CTA: one producer warp and NC consumer warps.
//   producer  walks the CTA's run of tiles and, for each tile, issues bulk
//             asynchronous copies (one per page piece) of the K and V rows into a
//             STAGES-deep shared-memory ring; completion is counted in bytes on a
//             "full" mbarrier, and consumers hand slots back on an "empty" one.
//   consumers split every tile's T tokens evenly.  A warp reads token rows with
//             16-byte shared loads, D/8 lanes per token; every KV row is loaded
//             once from HBM and reused by all GC query heads of the chunk.
//             BMM1: packed fp32 FMAs (two lanes of math per instruction) give
//             per-lane partial dots, which a transposed butterfly reduces across
//             the token's lanes so that each lane ends with whole scores.
//             Online softmax: running max m and sum l per head, in log2 units
//             (scale * log2 e is folded into q), one SFU exponential per score;
//             the fp32 accumulators are rescaled only when a maximum moved.
//             BMM2: packed FMAs of p * V into fp32 accumulators.
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
#include <cuda_fp8.h>

#include <type_traits>

#include "schedule.cuh"

namespace gqa {

// F8: the cache holds FP8 E4M3 bytes (one scale per tensor, folded into q for K
// and applied at the output for V) instead of bf16.
template <int D, int GC, bool F8 = false>
struct SimtCfg {
    static constexpr int KB = F8 ? 1 : 2;              // bytes per cache element
    // 7 consumer warps + 1 producer = 256 threads: the register allocator grants
    // up to 255 registers per thread only to CTAs of at most 256 threads, and each
    // warp needs ~200 to keep 8 steps (16 tokens at D = 128) in flight per tile.
    static constexpr int NC = 7;                       // consumer warps
    static constexpr int THREADS = (NC + 1) * 32;
    static constexpr int STEPS = 8;                    // warp steps per tile
    static constexpr int LPT = D / 8;                  // lanes per token (16 B each)
    static constexpr int TPW = 32 / LPT;               // tokens per warp step
    static constexpr int TOKW = STEPS * TPW;           // tokens per warp per tile
    static constexpr int T = NC * TOKW;                // tokens per tile: 56 KB of K+V
    // Shared-memory budget: the FP8 ring holds twice the tiles in the same bytes.
    static constexpr int STAGES = ((D == 256 && GC == 8) ? 2 : 3) * (F8 ? 2 : 1);
    static constexpr int NV = STEPS * GC;              // partial dots per lane
    static constexpr int NF = NV >= LPT ? NV / LPT : 1;  // whole scores per lane
    static constexpr int REP = NV >= LPT ? 1 : LPT / NV; // lanes sharing one score
    static constexpr int NS = TOKW * GC;               // scores per warp per tile
    static constexpr int NSL = (NS + 31) / 32;         // scores per lane (softmax)
    static constexpr int TILE_ELEMS = T * D;
    static constexpr int SCRATCH_PER_WARP = GC * D + ((2 * GC + 3) / 4) * 4;  // 16-byte multiple
    static constexpr int PSCR_PER_WARP = ((NS + GC + 3) / 4) * 4;              // scores + alphas
    static constexpr size_t RING_BYTES = 2ull * STAGES * TILE_ELEMS * KB;
    static constexpr size_t BAR_OFF = RING_BYTES;
    static constexpr size_t FLAG_OFF = BAR_OFF + 2 * STAGES * sizeof(uint64_t);
    static constexpr size_t SCRATCH_OFF = FLAG_OFF + 32 * sizeof(int);
    static constexpr size_t PSCR_OFF = SCRATCH_OFF + (size_t)NC * SCRATCH_PER_WARP * sizeof(float);
    static constexpr size_t MSCR_OFF = PSCR_OFF + (size_t)NC * PSCR_PER_WARP * sizeof(float);
    static constexpr size_t PREFIX_OFF =
        MSCR_OFF + (size_t)merge_scratch_floats(GC, NC * 32, 512) * sizeof(float);
    static constexpr int SLOT_FLOATS = slot_floats(GC, D);  // one partial state
    static size_t smem_bytes(int B) { return PREFIX_OFF + (size_t)(B + 1) * sizeof(int); }
    static_assert(STEPS >= 1 && TOKW % TPW == 0, "tile must split evenly over warps");
    static_assert(32 % GC == 0 && GC <= 8, "head chunk must divide the warp");
    static_assert(2 * STAGES <= 24, "flag area");
    static_assert(PREFIX_OFF + (4096 + 1) * sizeof(int) <= 232448, "shared memory at the largest batch");
};

// Transposed butterfly: NV partial sums per lane, reduced across the LPT lanes of
// a token.  While a lane still holds two or more values, each level hands half of
// them to the partner and keeps the other half (one shuffle per kept value);
// afterwards plain butterflies finish.  Lane s (= lane % LPT) ends with the NF
// whole sums of flat indices NF * (s / REP) + j.
template <int LPT, int NV>
__device__ __forceinline__ void transpose_reduce(float (&v)[NV], int lane)
{
#pragma unroll
    for (int lvl = 0; (LPT >> (lvl + 1)) >= 1; ++lvl) {
        const int m = LPT >> (lvl + 1);
        const int n = NV >> lvl;
        if (n >= 2) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int j = 0; j < n / 2; ++j) {
                const float send = upper ? v[j] : v[j + n / 2];
                const float keep = upper ? v[j + n / 2] : v[j];
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
        }
    }
}

// Eight consecutive cache elements: one uint4 of bf16 or one uint2 of FP8 E4M3.
// Typed (not char) so that the compiler may keep shared-memory loads and stores
// of other types apart.
template <bool F8>
using Vec8 = typename std::conditional<F8, uint2, uint4>::type;

// Eight cache elements as four float2, exactly.
template <bool F8>
__device__ __forceinline__ void load8(const Vec8<F8> &w, float2 &a, float2 &b, float2 &c, float2 &d)
{
    if constexpr (F8) {
        const uint32_t ww[2] = {w.x, w.y};
        float2 f[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
                (__nv_fp8x2_storage_t)((ww[j >> 1] >> (16 * (j & 1))) & 0xffffu), __NV_E4M3);
            f[j] = __half22float2(*reinterpret_cast<const __half2 *>(&h));
        }
        a = f[0];
        b = f[1];
        c = f[2];
        d = f[3];
    } else {
        a = bf16x2_to_float2(w.x);
        b = bf16x2_to_float2(w.y);
        c = bf16x2_to_float2(w.z);
        d = bf16x2_to_float2(w.w);
    }
}

template <int D, int GC, bool STATES, bool F8 = false>
__global__ void __launch_bounds__(SimtCfg<D, GC, F8>::THREADS, 1)
    gqa_decode_simt_kernel(const Params p)
{
    using C = SimtCfg<D, GC, F8>;
    constexpr int KB = C::KB;
    extern __shared__ __align__(128) unsigned char smem[];
    // The rings, typed by element (bf16 bits or FP8 bytes; the other pair unused).
    uint16_t *kring = reinterpret_cast<uint16_t *>(smem);
    uint16_t *vring = kring + C::STAGES * C::TILE_ELEMS;
    uint8_t *kring8 = smem;
    uint8_t *vring8 = kring8 + C::STAGES * C::TILE_ELEMS;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *empty = full + C::STAGES;
    int *stage_bad = reinterpret_cast<int *>(smem + C::FLAG_OFF);  // [STAGES]
    int *stage_n = stage_bad + C::STAGES;                           // [STAGES] valid tokens
    volatile int *abort_flag = stage_bad + 24;
    int *last_flag = stage_bad + 25;
    int *poison_flag = stage_bad + 26;
    int *merge_flags = stage_bad + 28;                              // [4]
    float *scratch = reinterpret_cast<float *>(smem + C::SCRATCH_OFF);
    float *pscr = reinterpret_cast<float *>(smem + C::PSCR_OFF);
    float *mscr = reinterpret_cast<float *>(smem + C::MSCR_OFF);
    int *prefix = reinterpret_cast<int *>(smem + C::PREFIX_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.B;
    const uint64_t t_start = global_timer_ns();

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
    if (start >= end) {
        if (p.timeline && tid == 0) {
            unsigned sm;
            asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
            unsigned long long *rec = p.timeline + TL_COLS * c;
            rec[0] = t_start;
            rec[1] = global_timer_ns();
            rec[2] = sm;
            rec[3] = 0;
            for (int x = 4; x < TL_COLS; ++x)
                rec[x] = 0;
        }
        return;
    }

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol = l2_evict_first_policy();
        TileIter it;
        it.init(start, prefix, B, units, p.hch);
        int cur_b = -1;
        int begin = 0, len = 0;
        int k = 0;
        for (int64_t i = start; i < end; ++i, ++k) {
            if (i > start)
                it.next(prefix, B, p.Hkv, p.hch);
            const int s = k % C::STAGES;
            const uint32_t ph = (uint32_t)((k / C::STAGES) & 1);
            if (k >= C::STAGES && !bounded_wait(&empty[s], ph ^ 1u, abort_flag, p))
                break;
            if (it.b != cur_b) {
                cur_b = it.b;
                int64_t b0, l0;
                request_range<STATES>(p, cur_b, b0, l0);
                begin = (int)b0;
                len = (int)l0;
            }
            // Tokens [tok0, tok0 + n) of the request; one copy per page piece.
            const int tok0 = begin + it.j * C::T;
            const int n = min(C::T, len - it.j * C::T);
            const int bs = p.block_size;
            const int pg0 = page_of(p, tok0);
            const int npieces = page_of(p, tok0 + n - 1) - pg0 + 1;
            const int32_t *row = p.block_table ? p.block_table + (int64_t)it.b * p.max_blocks : nullptr;
            // Pass 1: block ids and their bounds; bytes only need a sum when some
            // piece is skipped.
            int64_t blk0 = it.b;
            bool bad = false;
            for (int pc = lane; pc < npieces; pc += 32) {
                const int64_t blk = row ? row[pg0 + pc] : it.b;
                if (pc == lane)
                    blk0 = blk;
                if (row && (blk < 0 || blk >= p.num_blocks))
                    bad = true;
            }
            uint32_t bytes = (uint32_t)n * D * 2 * KB;
            if (__any_sync(0xffffffffu, bad)) {
                uint32_t skip = 0;
                for (int pc = lane; pc < npieces; pc += 32) {
                    const int64_t blk = row ? row[pg0 + pc] : it.b;
                    if (blk < 0 || blk >= p.num_blocks) {
                        const int pg = pg0 + pc;
                        skip += (uint32_t)(min((int64_t)tok0 + n, (int64_t)(pg + 1) * bs) -
                                           max((int64_t)tok0, (int64_t)pg * bs)) * D * 2 * KB;
                    }
                }
#pragma unroll
                for (int o = 16; o; o >>= 1)
                    skip += __shfl_xor_sync(0xffffffffu, skip, o);
                bytes -= skip;
                if (lane == 0)
                    atomicOr(p.status, DEV_BAD_BLOCK);
            }
            if (lane == 0) {
                stage_bad[s] = bytes != (uint32_t)n * D * 2 * KB;
                stage_n[s] = n;
                mbar_arrive_expect_tx(&full[s], bytes);
            }
            __syncwarp();
            // Pass 2: issue the copies (K and V rows of each piece).
            for (int pc = lane; pc < npieces; pc += 32) {
                const int64_t blk = pc == lane ? blk0 : (row ? row[pg0 + pc] : it.b);
                if (row && (blk < 0 || blk >= p.num_blocks))
                    continue;
                const int pg = pg0 + pc;
                const int a = max(tok0, pg * bs);
                const int z = (int)min((int64_t)tok0 + n, (int64_t)(pg + 1) * bs);
                const int64_t src = ((blk * p.Hkv + it.kvh) * (int64_t)bs + (a - pg * bs)) * D;
                const int dst = s * C::TILE_ELEMS + (a - tok0) * D;
                const uint32_t nb = (uint32_t)(z - a) * D * KB;
                if constexpr (F8) {
                    bulk_copy_g2s(kring8 + dst, reinterpret_cast<const uint8_t *>(p.k) + src, nb, &full[s], pol);
                    bulk_copy_g2s(vring8 + dst, reinterpret_cast<const uint8_t *>(p.v) + src, nb, &full[s], pol);
                } else {
                    bulk_copy_g2s(kring + dst, p.k + src, nb, &full[s], pol);
                    bulk_copy_g2s(vring + dst, p.v + src, nb, &full[s], pol);
                }
            }
        }
        // Never leave copies in flight: wait for the last issued phase of each slot.
        if (lane == 0) {
            for (int kk = max(0, k - C::STAGES); kk < k; ++kk) {
                const int s = kk % C::STAGES;
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
    const int sub = lane % C::LPT;
    const int d0 = sub * 8;                // this lane's 8 dimensions
    const int G = p.G;
    float *ps = pscr + cw * C::PSCR_PER_WARP;  // this warp's scores / probabilities
    float *alpha_s = ps + C::NS;

    float2 q2[GC][4], acc[GC][4];
    float m_h = -INFINITY, l_h = 0.f;      // running max / sum of head (lane % GC)
    bool poisoned = false;
    TileIter it, cur;
    it.init(start, prefix, B, units, p.hch);
    cur = it;
    int64_t piece_first = start;
    int k = 0;
    PendingPiece pending[2];  // a run has at most a first and a last partial piece
    int npending = 0;

    for (int64_t i = start; i < end; ++i, ++k) {
        if (i > start)
            it.next(prefix, B, p.Hkv, p.hch);
        if (i == start || it.seg0 != cur.seg0) {
            cur = it;
            piece_first = i;
            poisoned = false;
            m_h = -INFINITY;
            l_h = 0.f;
#pragma unroll
            for (int g = 0; g < GC; ++g) {
                const int hg = it.hc * GC + g;  // head inside the group
                uint4 w = make_uint4(0, 0, 0, 0);
                if (hg < G)
                    w = __ldg(reinterpret_cast<const uint4 *>(
                        p.q + (((int64_t)it.b * p.Hq + (int64_t)it.kvh * G + hg) * D + d0)));
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = bf16x2_to_float2(ww[j]);
                    q2[g][j] = make_float2(f.x * p.qscale, f.y * p.qscale);
                    acc[g][j] = make_float2(0.f, 0.f);
                }
            }
        }

        const int s = k % C::STAGES;
        const uint32_t ph = (uint32_t)((k / C::STAGES) & 1);
        const bool ready = bounded_wait(&full[s], ph, abort_flag, p);
        if (!ready) {
            poisoned = true;
        } else {
            poisoned |= stage_bad[s] != 0;
            const int n = stage_n[s];
            const uint16_t *Ks = kring + s * C::TILE_ELEMS;
            const uint16_t *Vs = vring + s * C::TILE_ELEMS;
            const uint8_t *Ks8 = kring8 + s * C::TILE_ELEMS;
            const uint8_t *Vs8 = vring8 + s * C::TILE_ELEMS;
            const int tok_base = cw * C::TOKW;  // this warp's first token in the tile

            // BMM1: partial dots over this lane's 8 dimensions.
            float part[C::NV];
#pragma unroll
            for (int st = 0; st < C::STEPS; ++st) {
                const int tt = tok_base + st * C::TPW + grp;
                float2 k0, k1, k2, k3;
                if constexpr (F8) {
                    uint2 w = make_uint2(0, 0);
                    if (tt < n)
                        w = *reinterpret_cast<const uint2 *>(Ks8 + tt * D + d0);
                    load8<true>(w, k0, k1, k2, k3);
                } else {
                    uint4 w = make_uint4(0, 0, 0, 0);
                    if (tt < n)
                        w = *reinterpret_cast<const uint4 *>(Ks + tt * D + d0);
                    k0 = bf16x2_to_float2(w.x);
                    k1 = bf16x2_to_float2(w.y);
                    k2 = bf16x2_to_float2(w.z);
                    k3 = bf16x2_to_float2(w.w);
                }
#pragma unroll
                for (int g = 0; g < GC; ++g) {
                    float2 a = __fmul2_rn(q2[g][0], k0);
                    a = __ffma2_rn(q2[g][1], k1, a);
                    a = __ffma2_rn(q2[g][2], k2, a);
                    a = __ffma2_rn(q2[g][3], k3, a);
                    part[st * GC + g] = a.x + a.y;
                }
            }
            transpose_reduce<C::LPT, C::NV>(part, lane);
            // Scores to shared memory in (token, head) order.
            if (sub % C::REP == 0) {
#pragma unroll
                for (int j = 0; j < C::NF; ++j) {
                    const int f = C::NF * (sub / C::REP) + j;
                    ps[((f / GC) * C::TPW + grp) * GC + (f % GC)] = part[j];
                }
            }
            __syncwarp();

            // Online softmax.  Lane handles scores sigma = lane + 32 r; all of them
            // belong to head lane % GC.
            float sc[C::NSL];
            float mx = -INFINITY;
#pragma unroll
            for (int r = 0; r < C::NSL; ++r) {
                const int sg = lane + 32 * r;
                const bool ok = sg < C::NS && tok_base + sg / GC < n;
                sc[r] = ok ? ps[sg] : -INFINITY;
                mx = fmaxf(mx, sc[r]);
            }
#pragma unroll
            for (int o = GC; o < 32; o <<= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_new = fmaxf(m_h, mx);
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            const float alpha = fast_exp2(m_h - m_use);
            float lsum = 0.f;
#pragma unroll
            for (int r = 0; r < C::NSL; ++r) {
                const int sg = lane + 32 * r;
                const float pr = fast_exp2(sc[r] - m_use);  // exp2(-inf) = 0
                lsum += pr;
                if (sg < C::NS)
                    ps[sg] = pr;
            }
            l_h = l_h * alpha + lsum;
            m_h = m_new;
            const bool rescale = __any_sync(0xffffffffu, alpha != 1.f);
            if (rescale && lane < GC)
                alpha_s[lane] = alpha;
            __syncwarp();
            if (rescale) {
#pragma unroll
                for (int g = 0; g < GC; ++g) {
                    const float a = alpha_s[g];
                    const float2 a2 = make_float2(a, a);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        acc[g][j] = __fmul2_rn(acc[g][j], a2);
                }
            }
            // BMM2: acc += p * V over this lane's tokens and dimensions.
#pragma unroll
            for (int st = 0; st < C::STEPS; ++st) {
                const int tl = st * C::TPW + grp;  // token inside this warp's share
                if (tok_base + tl >= n)
                    continue;
                float2 v0, v1, v2, v3;
                if constexpr (F8) {
                    load8<true>(*reinterpret_cast<const uint2 *>(Vs8 + (tok_base + tl) * D + d0), v0, v1,
                                v2, v3);
                } else {
                    const uint4 w = *reinterpret_cast<const uint4 *>(Vs + (tok_base + tl) * D + d0);
                    v0 = bf16x2_to_float2(w.x);
                    v1 = bf16x2_to_float2(w.y);
                    v2 = bf16x2_to_float2(w.z);
                    v3 = bf16x2_to_float2(w.w);
                }
                float pv[GC];
                if constexpr (GC % 4 == 0) {
#pragma unroll
                    for (int g = 0; g < GC; g += 4) {
                        const float4 f = *reinterpret_cast<const float4 *>(ps + tl * GC + g);
                        pv[g] = f.x;
                        pv[g + 1] = f.y;
                        pv[g + 2] = f.z;
                        pv[g + 3] = f.w;
                    }
                } else {
#pragma unroll
                    for (int g = 0; g < GC; ++g)
                        pv[g] = ps[tl * GC + g];
                }
#pragma unroll
                for (int g = 0; g < GC; ++g) {
                    const float2 pp = make_float2(pv[g], pv[g]);
                    acc[g][0] = __ffma2_rn(pp, v0, acc[g][0]);
                    acc[g][1] = __ffma2_rn(pp, v1, acc[g][1]);
                    acc[g][2] = __ffma2_rn(pp, v2, acc[g][2]);
                    acc[g][3] = __ffma2_rn(pp, v3, acc[g][3]);
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]);

        const bool piece_end = (i + 1 == end) || (i + 1 == it.seg0 + it.nb);
        if (!piece_end)
            continue;

        // ------------------------------------------------------------ epilogue
        // Lanes of one head share m; add their l.  Token slots of a warp share m;
        // add their accumulators.
        float l_tot = l_h;
#pragma unroll
        for (int o = GC; o < 32; o <<= 1)
            l_tot += __shfl_xor_sync(0xffffffffu, l_tot, o);
#pragma unroll
        for (int g = 0; g < GC; ++g)
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int o = C::LPT; o < 32; o <<= 1) {
                    acc[g][j].x += __shfl_xor_sync(0xffffffffu, acc[g][j].x, o);
                    acc[g][j].y += __shfl_xor_sync(0xffffffffu, acc[g][j].y, o);
                }
        float *mine = scratch + cw * C::SCRATCH_PER_WARP;
        if (grp == 0) {
#pragma unroll
            for (int g = 0; g < GC; ++g) {
                float4 *dst = reinterpret_cast<float4 *>(mine + g * D + d0);
                dst[0] = make_float4(acc[g][0].x, acc[g][0].y, acc[g][1].x, acc[g][1].y);
                dst[1] = make_float4(acc[g][2].x, acc[g][2].y, acc[g][3].x, acc[g][3].y);
            }
        }
        if (lane < GC) {
            mine[GC * D + lane] = m_h;
            mine[GC * D + GC + lane] = l_tot;
        }
        if (lane == 0 && poisoned)
            atomicOr(poison_flag, 1);
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
                const float wt = mw == -INFINITY ? 0.f : fast_exp2(mw - ms);
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
            if (ctid == 0)
                *poison_flag = 0;
            pending[npending++] = PendingPiece{cur.seg0, piece_first, i + 1, vseg, row0, cur.nb, rows};
        } else if (ctid == 0) {
            *poison_flag = 0;
        }
        named_barrier_sync(1, C::NC * 32);
    }

    for (int x = 0; x < npending; ++x) {
        const PendingPiece &pp = pending[x];
        finish_partial<GC, D, C::NC * 32, STATES>(
            p, c, pp.seg0, pp.nb, pp.first, pp.end, pp.vseg, W, P, mscr, merge_flags, ctid, 1,
            [&](const int *list, int n, float *dst) {
                merge_slots<GC, D, C::NC * 32, STATES>(p, list, n, dst, pp.rows, pp.row0, ctid, 1);
            });
        named_barrier_sync(1, C::NC * 32);
    }

    if (p.timeline && ctid == 0) {
        unsigned sm;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
        unsigned long long *rec = p.timeline + TL_COLS * c;
        rec[0] = t_start;
        rec[1] = global_timer_ns();
        rec[2] = sm;
        rec[3] = (unsigned long long)(end - start);
        for (int x = 4; x < TL_COLS; ++x)
            rec[x] = 0;
    }
}

}  // namespace gqa
