// decode_tc.cuh -- persistent stream-K decode attention on the 5th-generation
// tensor cores (tcgen05), for groups of G >= 8 query heads per KV head where
// q.K^T is a real dense contraction (M = 128 tokens, N = 16 heads, K = D = 128).
//
// Same LeanTile schedule as the CUDA-core kernel (schedule.cuh): each CTA walks a
// contiguous run of 128-token tiles of (request, KV head, 16-head chunk) segments.
// Roles (one CTA per SM, 7 warps):
//   warps 0, 6 TMA: each tile's K rows (warp 0) and V rows (warp 6) arrive as
//              128-byte-swizzled boxes (one per page, two 64-column halves) into
//              separate 3-slot rings: a K slot frees as soon as BMM1 has read it,
//              a V slot only after BMM2, so K loads run further ahead.
//   warp 1     MMA (one thread): BMM1  S^T[128 x 16] = K[128 x 128] . Q^T, with K
//              and Q K-major; BMM2  O^T[128 x 16] = V^T . P^T, with V read
//              MN-major straight from the swizzled TMA boxes and P from shared
//              memory.  P is passed as two bf16 terms, hi and lo, so that P itself
//              carries ~16 significant bits: they are the two halves of one
//              N = 32 operand, since an MMA of N <= 128 costs the tensor pipe the
//              same ~90 cycles whatever N is.  Accumulators live in tensor
//              memory, two buffers each.
//   warps 2-5  softmax + correction (thread = TMEM lane): read S rows, take the
//              tile maximum per head across the 128 tokens, update the running
//              maximum lazily (only when it grows by more than 2^8), write
//              P = exp2(s - m) as bf16, and fold each tile's O into fp32 registers
//              rescaled by the running-maximum changes.
// Piece epilogue, partial-state slots and last-arriver merge as in the CUDA-core
// kernel.  (Attention co-design for long-context inference, sections "FlashAttention
// and GEMM shapes" and "Effect of group size G": decode GEMM-M equals G; LeanAttention
// decode tiles digest, sections "Exact softmax that merges piece by piece" and
// "Hardware-sized work units".)
#pragma once

#include "schedule.cuh"
#include "tc.cuh"

namespace gqa {

struct TcCfg {
    // (merge scratch lives in the P buffers: checked below)
    static constexpr int D = 128, T = 128, NP = 16;  // head dim, tile tokens, heads per MMA
    static constexpr int STAGES = 3;                   // slots per ring (K ring, V ring)
    static constexpr int THREADS = 224;
    static constexpr int BOX_BYTES = T * 128;          // one 64-column half of a tile: 16 KB
    static constexpr int TILE_BYTES = 2 * BOX_BYTES;   // K or V tile
    static constexpr int V_RING_OFF = STAGES * TILE_BYTES;
    static constexpr int QBUF_BYTES = 2 * NP * 128;    // two halves, NP rows of 128 B
    static constexpr int NO = 2 * NP;                  // BMM2 columns: P_hi heads, P_lo heads
    static constexpr int P_LBO = (NO / 8) * 128;       // P: stride between 8-token groups
    static constexpr int PBUF_BYTES = (T / 8) * P_LBO;
    static constexpr int S_COL = 0, O_COL = 2 * NP;    // TMEM columns: S x2, O x2 (NO wide)
    static constexpr int TMEM_COLS = 128;              // >= 2 * NP + 2 * NO, power of two
    static constexpr float LAZY = 8.f;                 // rescale only when max grows > 2^8
    static constexpr size_t Q_OFF = (size_t)2 * STAGES * TILE_BYTES;
    static constexpr size_t P_OFF = Q_OFF + 2 * QBUF_BYTES;
    static constexpr size_t BAR_OFF = P_OFF + 2 * PBUF_BYTES;
    static constexpr int NBAR = 4 * STAGES + 13;
    static constexpr size_t MISC_OFF = BAR_OFF + NBAR * 8;
    // floats: tile maxima [2][4][NP], piece sums [4][NP], merge maxima [NP]
    static constexpr size_t RED_OFF = MISC_OFF + 64 * 4;
    static constexpr size_t PREFIX_OFF = RED_OFF + 13 * NP * 4 + 64;
    static constexpr int SLOT_FLOATS = slot_floats(NP, D);
    static constexpr int MAX_BATCH = 1024;
    // +1024: the dynamic shared-memory base is re-aligned to 1024 bytes in-kernel.
    static size_t smem_bytes(int B) { return PREFIX_OFF + (size_t)(B + 1) * sizeof(int) + 1024; }
};
static_assert(merge_scratch_floats(TcCfg::NP, 128, 512) * 4 <= 2 * TcCfg::PBUF_BYTES,
              "merge scratch must fit in the P buffers");
static_assert(TcCfg::O_COL + 2 * TcCfg::NO <= TcCfg::TMEM_COLS, "tensor memory columns");

// Max or sum of NV per-lane values across the 32 lanes of a warp, transposed so
// that lane l ends with the result for index l / (32 / NV) (NV <= 32).
template <int NV, bool MAX>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[NV], int lane)
{
#pragma unroll
    for (int lvl = 0; (32 >> (lvl + 1)) >= 1; ++lvl) {
        const int m = 32 >> (lvl + 1);
        const int n = NV >> lvl;
        if (n >= 2) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int j = 0; j < n / 2; ++j) {
                const float send = upper ? v[j] : v[j + n / 2];
                const float keep = upper ? v[j + n / 2] : v[j];
                const float got = __shfl_xor_sync(0xffffffffu, send, m);
                v[j] = MAX ? fmaxf(keep, got) : keep + got;
            }
        } else {
            const float got = __shfl_xor_sync(0xffffffffu, v[0], m);
            v[0] = MAX ? fmaxf(v[0], got) : v[0] + got;
        }
    }
    return v[0];
}

__global__ void __launch_bounds__(TcCfg::THREADS, 1)
    gqa_decode_tc_kernel(const Params p, const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv, int box_rows)
{
    using C = TcCfg;
    constexpr int S = C::STAGES, NP = C::NP, D = C::D, T = C::T;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    unsigned char *ring = smem;
    unsigned char *qbuf = smem + C::Q_OFF;
    unsigned char *pbuf = smem + C::P_OFF;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *k_full = bars, *k_empty = bars + S, *v_full = bars + 2 * S, *v_empty = bars + 3 * S;
    uint64_t *s_full = bars + 4 * S, *s_free = s_full + 2, *p_full = s_free + 2;
    uint64_t *o_full = p_full + 2, *o_free = o_full + 2, *q_full = o_free + 2, *drain = q_full + 2;
    int *misc = reinterpret_cast<int *>(smem + C::MISC_OFF);
    int *stage_n = misc, *stage_bad = misc + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 16);
    volatile int *abort_flag = misc + 17;
    int *last_flag = misc + 18, *poison_flag = misc + 19;
    float *red = reinterpret_cast<float *>(smem + C::RED_OFF);
    int *prefix = reinterpret_cast<int *>(smem + C::PREFIX_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.B;
    const uint64_t t_start = global_timer_ns();

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
            stage_bad[s] = 0;
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 128);
            mbar_init(&p_full[b], 128);
            mbar_init(&o_full[b], 1);
            mbar_init(&o_free[b], 128);
            mbar_init(&q_full[b], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        *last_flag = 0;
        *poison_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    for (int b = tid; b < B; b += C::THREADS) {
        int64_t begin, len;
        const bool ok = request_range<false>(p, b, begin, len);
        if (!ok && blockIdx.x == 0)
            atomicOr(p.status, DEV_BAD_LENGTH);
        prefix[b + 1] = (int)((len + T - 1) / T);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < B; base += 32) {
            const int b = base + lane;
            int x = b < B ? prefix[b + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
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
    const int G = p.G;

    for (int b = (int)c; b < B; b += (int)P) {
        if (prefix[b + 1] != prefix[b])
            continue;
        int64_t begin, len;
        const bool bad = !request_range<false>(p, b, begin, len);
        for (int e = tid; e < p.Hq * D; e += C::THREADS)
            write_result<false>(p, (int64_t)b * p.Hq + e / D, e % D, D, 0.f, -INFINITY, 0.f, bad);
    }

    if (start < end && (warp == 0 || warp == 6)) {
        // ---------------------------------------------------------------- TMA
        const bool is_k = warp == 0;
        const CUtensorMap *map = is_k ? &tmk : &tmv;
        unsigned char *base = ring + (is_k ? 0 : C::V_RING_OFF);
        uint64_t *full = is_k ? k_full : v_full, *emptyb = is_k ? k_empty : v_empty;
        const uint64_t pol = l2_evict_first_policy();
        TileIter it;
        it.init(start, prefix, B, units, p.hch);
        int cur_b = -1, len = 0, k = 0;
        for (int64_t i = start; i < end; ++i, ++k) {
            if (i > start)
                it.next(prefix, B, p.Hkv, p.hch);
            const int s = k % S;
            const uint32_t ph = (uint32_t)((k / S) & 1);
            if (k >= S && !bounded_wait(&emptyb[s], ph ^ 1u, abort_flag, p.status))
                break;
            if (it.b != cur_b) {
                cur_b = it.b;
                int64_t b0, l0;
                request_range<false>(p, cur_b, b0, l0);
                len = (int)l0;
            }
            const int tok0 = it.j * T;
            const int n = min(T, len - tok0);
            const int nbox = (n + box_rows - 1) / box_rows;
            bool bad = false;
            int row = 0;
            if (lane < nbox) {
                const int t = tok0 + lane * box_rows;
                if (p.block_table) {
                    const int pg = page_of(p, t);
                    const int64_t blk = p.block_table[(int64_t)it.b * p.max_blocks + pg];
                    bad = blk < 0 || blk >= p.num_blocks;
                    row = bad ? 0 : (int)((blk * p.Hkv + it.kvh) * p.block_size + (t - pg * p.block_size));
                } else {
                    row = (int)(((int64_t)it.b * p.Hkv + it.kvh) * p.block_size + t);
                }
            }
            const unsigned badmask = __ballot_sync(0xffffffffu, bad);
            if (lane == 0) {
                // Tile metadata travels with the V slot: a V slot is recycled only
                // after every softmax thread has posted this tile's P, while a K
                // slot may be refilled before a slow softmax thread looks at it.
                if (!is_k) {
                    stage_n[s] = n;
                    stage_bad[s] = badmask != 0;
                    if (badmask)
                        atomicOr(p.status, DEV_BAD_BLOCK);
                }
                const uint32_t boxes = (uint32_t)(nbox - __popc(badmask));
                mbar_arrive_expect_tx(&full[s], boxes * 2u * (uint32_t)box_rows * 128u);
            }
            __syncwarp();
            if (lane < nbox && !bad) {
                unsigned char *d = base + (size_t)s * C::TILE_BYTES + (size_t)lane * box_rows * 128;
                tma_load_2d(d, map, 0, row, &full[s], pol);
                tma_load_2d(d + C::BOX_BYTES, map, 64, row, &full[s], pol);
            }
        }
        if (lane == 0) {
            for (int kk = max(0, k - S); kk < k; ++kk) {
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(&full[kk % S], (uint32_t)((kk / S) & 1)) &&
                       global_timer_ns() - t0 < WAIT_LIMIT_NS) {
                }
            }
        }
    } else if (start < end && warp == 1) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t idesc1 = umma_idesc_bf16(128, NP, 0, 0);
            const uint32_t idesc2 = umma_idesc_bf16(128, C::NO, 1, 1);
            const uint32_t ring_a = smem_addr(ring), q_a = smem_addr(qbuf), p_a = smem_addr(pbuf);
            const int ntiles = (int)(end - start);
            TileIter it1;
            it1.init(start, prefix, B, units, p.hch);
            int64_t seg1 = -1;
            int piece1 = 0;
            bool ok = true;
            auto mma1 = [&](int k) {
                if (k > 0)
                    it1.next(prefix, B, p.Hkv, p.hch);
                if (it1.seg0 != seg1) {
                    seg1 = it1.seg0;
                    ++piece1;
                }
                const int s = k % S, b = k & 1, qb = (piece1 - 1) & 1;
                ok = ok && bounded_wait(&k_full[s], (uint32_t)((k / S) & 1), abort_flag, p.status);
                if (k >= 2)
                    ok = ok && bounded_wait(&s_free[b], (uint32_t)(((k - 2) >> 1) & 1), abort_flag, p.status);
                ok = ok && bounded_wait(&q_full[qb], (uint32_t)(((piece1 - 1) >> 1) & 1), abort_flag, p.status);
                if (!ok)
                    return;
                tc_fence_after_sync();
                const uint32_t ka = ring_a + (uint32_t)(s * C::TILE_BYTES);
                const uint32_t qa = q_a + (uint32_t)(qb * C::QBUF_BYTES);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (uint32_t)((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32);
                    const uint32_t qoff = (uint32_t)((kk >> 2) * NP * 128 + (kk & 3) * 32);
                    umma_bf16(tbase + (uint32_t)(C::S_COL + b * NP), umma_smem_desc(ka + off, 16, 1024, SMEM_LAYOUT_SW128),
                              umma_smem_desc(qa + qoff, 16, 1024, SMEM_LAYOUT_SW128), idesc1, kk > 0);
                }
                umma_commit(&s_full[b]);
                umma_commit(&k_empty[s]);
            };
            auto mma2 = [&](int k) {
                const int s = k % S, b = k & 1;
                ok = ok && bounded_wait(&p_full[b], (uint32_t)((k >> 1) & 1), abort_flag, p.status);
                ok = ok && bounded_wait(&v_full[s], (uint32_t)((k / S) & 1), abort_flag, p.status);
                if (k >= 2)
                    ok = ok && bounded_wait(&o_free[b], (uint32_t)(((k - 2) >> 1) & 1), abort_flag, p.status);
                if (!ok)
                    return;
                tc_fence_after_sync();
                const uint32_t va = ring_a + (uint32_t)(C::V_RING_OFF + s * C::TILE_BYTES);
                const uint32_t pa = p_a + (uint32_t)(b * C::PBUF_BYTES);
#pragma unroll
                for (int kk = 0; kk < T / 16; ++kk) {
                    umma_bf16(tbase + (uint32_t)(C::O_COL + b * C::NO),
                              umma_smem_desc(va + (uint32_t)(kk * 2048), C::BOX_BYTES, 1024, SMEM_LAYOUT_SW128),
                              umma_smem_desc(pa + (uint32_t)(2 * kk * C::P_LBO), C::P_LBO, 128, SMEM_LAYOUT_NONE),
                              idesc2, kk > 0);
                }
                umma_commit(&o_full[b]);
                umma_commit(&v_empty[s]);
            };
            mma1(0);
            for (int k = 0; k < ntiles && ok; ++k) {
                if (k + 1 < ntiles)
                    mma1(k + 1);
                mma2(k);
            }
            // Nothing of ours may still be running on the tensor cores at exit.
            umma_commit(drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < WAIT_LIMIT_NS) {
            }
        }
    } else if (start < end) {
        // ------------------------------------------------------ softmax + correction
        const int q4 = warp & 3;                 // TMEM lane quadrant of this warp
        const int ti = q4 * 32 + lane;           // token row (S) and d row (O)
        const int stid = tid - 64;               // 0..127 among the softmax threads
        const uint32_t tlane = tbase + ((uint32_t)(q4 * 32) << 16);
        const float qscale = p.qscale;
        float m_ref[NP], l_t[NP], acc[NP], alpha_prev[NP];
        PendingPiece pending[2];  // a run has at most a first and a last partial piece
        int npending = 0;
        bool poisoned = false, pend = false;
        TileIter it, cur;
        it.init(start, prefix, B, units, p.hch);
        cur = it;
        int64_t piece_first = start;
        int piece = 0;
        bool ok = true;

        auto correction = [&](int kc) {
            const int bc = kc & 1;
            float o[NP];
            if (ok && bounded_wait(&o_full[bc], (uint32_t)((kc >> 1) & 1), abort_flag, p.status)) {
                float olo[NP];
                tc_fence_after_sync();
                tmem_load16(tlane + (uint32_t)(C::O_COL + bc * C::NO), o);
                tmem_load16(tlane + (uint32_t)(C::O_COL + bc * C::NO + NP), olo);
                tc_fence_before_sync();
#pragma unroll
                for (int g = 0; g < NP; ++g)
                    o[g] += olo[g];
            } else {
                ok = false;
                poisoned = true;
#pragma unroll
                for (int g = 0; g < NP; ++g)
                    o[g] = 0.f;
            }
            mbar_arrive(&o_free[bc]);
#pragma unroll
            for (int g = 0; g < NP; ++g)
                acc[g] = fmaf(acc[g], alpha_prev[g], o[g]);
        };

        auto epilogue = [&](int64_t last_excl) {
            // Normaliser per head: sum of every token thread's partial.
            float lv[NP];
#pragma unroll
            for (int g = 0; g < NP; ++g)
                lv[g] = l_t[g];
            const float mine = warp_transpose_reduce<NP, false>(lv, lane);
            float *lred = red + 8 * NP;
            if ((lane & 1) == 0)
                lred[q4 * NP + (lane >> 1)] = mine;
            if (poisoned)
                atomicOr(poison_flag, 1);
            named_barrier_sync(1, 128);
            float lsum[NP];
#pragma unroll
            for (int g = 0; g < NP; ++g)
                lsum[g] = lred[g] + lred[NP + g] + lred[2 * NP + g] + lred[3 * NP + g];
            const bool pois = *reinterpret_cast<volatile int *>(poison_flag) != 0;
            const bool complete = piece_first == cur.seg0 && last_excl == cur.seg0 + cur.nb;
            const int rows = min(NP, G - cur.hc * NP);
            const int64_t row0 = (int64_t)cur.b * p.Hq + (int64_t)cur.kvh * G + (int64_t)cur.hc * NP;
            const int64_t vseg = ((int64_t)cur.b * p.Hkv + cur.kvh) * p.hch + cur.hc;
            float *slot = p.slots + (2 * c + (piece_first == start ? 0 : 1)) * (int64_t)C::SLOT_FLOATS;
            if (complete) {
#pragma unroll
                for (int g = 0; g < NP; ++g)
                    if (g < rows)
                        write_result<false>(p, row0 + g, ti, D, acc[g], m_ref[g], lsum[g], pois);
            } else {
#pragma unroll
                for (int g = 0; g < NP; ++g)
                    slot[g * D + ti] = acc[g];
                if (ti < NP) {
                    float mv = m_ref[0], lvv = lsum[0];
#pragma unroll
                    for (int g = 1; g < NP; ++g)
                        if (g == ti) {
                            mv = m_ref[g];
                            lvv = lsum[g];
                        }
                    slot[NP * D + ti] = mv;
                    slot[NP * D + NP + ti] = pois ? __int_as_float(0x7fc00000) : lvv;
                }
            }
            named_barrier_sync(1, 128);
            if (!complete) {
                if (stid == 0)
                    *poison_flag = 0;
                pending[npending++] = PendingPiece{cur.seg0, piece_first, last_excl, vseg, row0, cur.nb, rows};
            } else if (stid == 0) {
                *poison_flag = 0;
            }
            named_barrier_sync(1, 128);
        };

        int k = 0;
        for (int64_t i = start; i < end; ++i, ++k) {
            if (i > start)
                it.next(prefix, B, p.Hkv, p.hch);
            if (i == start || it.seg0 != cur.seg0) {
                // Q of the new (request, KV head, head chunk) goes out first: the MMA
                // warp issues this tile's BMM1 before the previous tile's BMM2, and
                // closing the previous piece below waits on that BMM2.  Layout: the
                // 128-byte-swizzled K-major form the tensor cores read (row g,
                // 16-byte chunk cc of a 64-column half at chunk position cc ^ (g & 7)).
                ++piece;
                unsigned char *qd = qbuf + ((piece - 1) & 1) * C::QBUF_BYTES;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int x = stid + 128 * r;
                    const int half = x >> 7, g = (x & 127) >> 3, cc = x & 7;
                    uint4 w = make_uint4(0, 0, 0, 0);
                    if (it.hc * NP + g < G)
                        w = __ldg(reinterpret_cast<const uint4 *>(
                            p.q + (((int64_t)it.b * p.Hq + (int64_t)it.kvh * G + it.hc * NP + g) * D +
                                   half * 64 + cc * 8)));
                    *reinterpret_cast<uint4 *>(qd + half * NP * 128 + g * 128 + ((cc ^ (g & 7)) << 4)) = w;
                }
                fence_proxy_async_smem();
                mbar_arrive(&q_full[(piece - 1) & 1]);
                if (i > start) {
                    if (pend)
                        correction(k - 1);
                    pend = false;
                    epilogue(i);
                }
                cur = it;
                piece_first = i;
                poisoned = false;
#pragma unroll
                for (int g = 0; g < NP; ++g) {
                    m_ref[g] = -INFINITY;
                    l_t[g] = 0.f;
                    acc[g] = 0.f;
                    alpha_prev[g] = 1.f;
                }
            }

            const int s = k % S, b = k & 1;
            float sc[NP];
            int n = 0;
            if (ok && bounded_wait(&v_full[s], (uint32_t)((k / S) & 1), abort_flag, p.status) &&
                bounded_wait(&s_full[b], (uint32_t)((k >> 1) & 1), abort_flag, p.status)) {
                n = stage_n[s];
                poisoned |= stage_bad[s] != 0;
                tc_fence_after_sync();
                tmem_load16(tlane + (uint32_t)(C::S_COL + b * NP), sc);
                tc_fence_before_sync();
            } else {
                ok = false;
                poisoned = true;
            }
            mbar_arrive(&s_free[b]);
            const bool valid = ti < n;
            float mx[NP];
#pragma unroll
            for (int g = 0; g < NP; ++g) {
                sc[g] = valid ? sc[g] * qscale : -INFINITY;
                mx[g] = sc[g];
            }
            // Tile maximum per head over the 128 tokens: warp, then the 4 warps.
            const float wmax = warp_transpose_reduce<NP, true>(mx, lane);
            float *tred = red + (k & 1) * 4 * NP;
            if ((lane & 1) == 0)
                tred[q4 * NP + (lane >> 1)] = wmax;
            named_barrier_sync(1, 128);
            float alpha[NP], pr[NP];
#pragma unroll
            for (int g = 0; g < NP; ++g) {
                const float tm = fmaxf(fmaxf(tred[g], tred[NP + g]), fmaxf(tred[2 * NP + g], tred[3 * NP + g]));
                const float m_new = tm > m_ref[g] + C::LAZY ? tm : m_ref[g];
                alpha[g] = m_new == m_ref[g] ? 1.f : fast_exp2(m_ref[g] - m_new);
                m_ref[g] = m_new;
                pr[g] = (valid && m_new != -INFINITY) ? fast_exp2(sc[g] - m_new) : 0.f;
                l_t[g] = fmaf(l_t[g], alpha[g], pr[g]);
            }
            // P = hi + lo, both bf16, as one N = 32 operand (hi heads, then lo
            // heads) in the no-swizzle MN-major layout: token ti's 8-head groups
            // are 16-byte rows of 8x8 core matrices.
            unsigned char *pd = pbuf + b * C::PBUF_BYTES + (ti >> 3) * C::P_LBO + (ti & 7) * 16;
#pragma unroll
            for (int ng = 0; ng < NP / 8; ++ng) {
                uint32_t whi[4], wlo[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float a = pr[ng * 8 + 2 * j], bb = pr[ng * 8 + 2 * j + 1];
                    __nv_bfloat162 hi = __floats2bfloat162_rn(a, bb);
                    const float2 hf = __bfloat1622float2(hi);
                    __nv_bfloat162 lo = __floats2bfloat162_rn(a - hf.x, bb - hf.y);
                    whi[j] = *reinterpret_cast<uint32_t *>(&hi);
                    wlo[j] = *reinterpret_cast<uint32_t *>(&lo);
                }
                *reinterpret_cast<uint4 *>(pd + ng * 128) = make_uint4(whi[0], whi[1], whi[2], whi[3]);
                *reinterpret_cast<uint4 *>(pd + (NP / 8 + ng) * 128) =
                    make_uint4(wlo[0], wlo[1], wlo[2], wlo[3]);
            }
            // Rows past the valid tokens may hold anything (stale tiles, poison):
            // zero this token's V row so that 0-weight rows add exact zeros.
            if (!valid) {
                unsigned char *vr = ring + C::V_RING_OFF + (size_t)s * C::TILE_BYTES + ti * 128;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc)
                        *reinterpret_cast<uint4 *>(vr + h * C::BOX_BYTES + cc * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            mbar_arrive(&p_full[b]);
            if (pend)
                correction(k - 1);
#pragma unroll
            for (int g = 0; g < NP; ++g)
                alpha_prev[g] = alpha[g];
            pend = true;
        }
        if (pend)
            correction(k - 1);
        epilogue(end);
        // Tickets and merges after streaming; the P buffers are idle: merge scratch.
        for (int x = 0; x < npending; ++x) {
            const PendingPiece &pp = pending[x];
            finish_partial<NP, D, 128, false>(p, c, pp.seg0, pp.nb, pp.first, pp.end, pp.vseg, W, P,
                                              pp.rows, pp.row0, reinterpret_cast<float *>(pbuf),
                                              misc + 20, stid, 1);
            named_barrier_sync(1, 128);
        }
    }

    // Timeline record and tensor-memory release.
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tbase, C::TMEM_COLS);
    }
    if (p.timeline && tid == 0) {
        unsigned sm;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
        unsigned long long *rec = p.timeline + 4 * c;
        rec[0] = t_start;
        rec[1] = global_timer_ns();
        rec[2] = sm;
        rec[3] = (unsigned long long)(end - start);
    }
}

}  // namespace gqa
