// decode_tc_wide.cuh -- the tensor-core decode kernel for large groups: 17 to 64
// query heads per KV head in one pass (multi-query attention with 64 heads on one
// KV head, or G = 32, 48; larger groups take several passes of 64).  Each K/V tile
// is streamed once per pass and meets all of the pass's heads in one BMM1 of
// N = 64 and one BMM2 of N = 128 (P_hi | P_lo), where the 16-head kernel
// (decode_tc.cuh) would stream it once per 16 heads and issue four times the MMAs.
// (Attention co-design for long-context inference, section "Effect of group size
// G": decode GEMM-M equals G, so a larger group turns the same KV bytes into more
// useful work per tile.)
//
// Same schedule, TMA and MMA roles and pipeline as the 16-head kernel; what differs:
//   - shared memory: two K slots and three V slots of 32 KB (a V slot is held until
//     the softmax has posted P, a K slot only until BMM1 has read it), one 16 KB Q
//     buffer and one 32 KB P buffer (P of tile k+1 is computed while BMM2 reads P
//     of tile k, and stored once it has);
//   - tensor memory: S 2 x 64 columns, O 2 x 128 columns, and the folded O rows
//     (64 columns) that the 16-head kernel keeps in registers (512 allocated);
//   - softmax: four warpgroups of 128 threads (thread = token row), each carrying 16
//     of the 64 heads, so that every SM sub-partition runs four softmax warps; the
//     reference maxima and the fold weights, equal for every thread, live in shared
//     memory; the pipeline barriers take one arrival per softmax warp.
// Head dimension 128, bf16 cache, one query token per request.
#pragma once

#include "decode_tc.cuh"

namespace gqa {

struct TcWide {
    static constexpr int T = 128, NP = 64, D = 128;
    static constexpr int NGRP = 4;                        // softmax warpgroups
    static constexpr int HPT = NP / NGRP;                 // heads per softmax thread
    static constexpr int THREADS = 128 * (1 + NGRP);      // warps 0, 1, 6, 7: roles
    static constexpr int SMT = 128 * NGRP;                // softmax threads
    static constexpr int BOX_BYTES = T * 128;              // one 64-column half: 16 KB
    static constexpr int SLOT_BYTES = 2 * BOX_BYTES;       // one K or V tile: 32 KB
    static constexpr int SK = 2, SV = 3;                   // K and V ring slots
    static constexpr int QBUF_BYTES = 2 * NP * 128;        // two halves of NP rows of 128 B
    static constexpr int NO = 2 * NP;                      // BMM2 columns: P_hi heads, P_lo heads
    static constexpr int P_LBO = (NO / 8) * 128;           // P: stride between 8-token groups
    static constexpr int PBUF_BYTES = (T / 8) * P_LBO;     // 32 KB
    static constexpr int S_COL = 0, O_COL = 2 * NP;        // TMEM: S x2 (NP), O x2 (NO),
    static constexpr int ACC_COL = O_COL + 2 * NO;         // the folded O rows (NP)
    static constexpr int TMEM_COLS = 512;
    static constexpr float LAZY = TcCfg::LAZY;
    static constexpr size_t V_RING_OFF = (size_t)SK * SLOT_BYTES;
    static constexpr size_t Q_OFF = V_RING_OFF + (size_t)SV * SLOT_BYTES;
    static constexpr size_t P_OFF = Q_OFF + QBUF_BYTES;
    static constexpr size_t BAR_OFF = P_OFF + PBUF_BYTES;
    static constexpr int NBAR = 2 * SK + 2 * SV + 16;
    static constexpr size_t MISC_OFF = BAR_OFF + NBAR * 8;
    // floats: reference maxima [NP], rescale factors [NP], pending fold weights
    // [NP], tile maxima [4][NP], normaliser sums [4][NP]
    static constexpr size_t RED_OFF = MISC_OFF + 64 * 4;
    static constexpr size_t PREFIX_OFF = RED_OFF + 11 * NP * 4;
    static constexpr int SLOT_FLOATS = slot_floats(NP, D);
    static size_t smem_bytes(int B) { return PREFIX_OFF + (size_t)(B + 1) * sizeof(int) + 1024; }
    static_assert(ACC_COL + NP <= TMEM_COLS, "tensor memory columns");
    static_assert(Q_OFF % 1024 == 0 && V_RING_OFF % 1024 == 0, "swizzled buffers are 1024-byte aligned");
    static_assert(SV <= 8, "stage_n and stage_bad hold 8 slots");
    static_assert(HPT % 16 == 0 && 1024 % SMT == 0, "softmax split");
    static_assert(PREFIX_OFF + (TcCfg::MAX_BATCH + 1) * sizeof(int) + 1024 <= 227 * 1024,
                  "shared memory per CTA");
    // Segment merge: the owner list (<= 512 ints) in the P buffer; the gathered
    // slices (E = NP x D outputs, slices rounded to 4 elements; per owner at most
    // E / D + 2 heads) in the rings.
    static_assert(512 * 4 <= PBUF_BYTES, "owner list must fit in the P buffer");
    static_assert((NP * D + 4 * 512 + 3 * (NP + 4 * 512 / D + 2 * 512) + 2 * (NP + 2)) * 4 <= Q_OFF,
                  "gathered slices must fit in the rings");
};

__global__ void __launch_bounds__(TcWide::THREADS, 1)
    gqa_decode_tc_wide_kernel(const Params p, const __grid_constant__ CUtensorMap tmk,
                              const __grid_constant__ CUtensorMap tmv, int box_rows)
{
    using C = TcWide;
    constexpr int SK = C::SK, SV = C::SV, NP = C::NP, D = C::D, T = C::T;
    constexpr int SMT = C::SMT;
    constexpr int HPT = C::HPT, NCH = HPT / 16;  // heads per softmax thread; chunks of 16 columns
    constexpr int SLOT = C::SLOT_FLOATS;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    unsigned char *ring = smem;
    unsigned char *qbuf = smem + C::Q_OFF;
    unsigned char *pbuf = smem + C::P_OFF;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *k_full = bars, *k_empty = bars + SK, *v_full = bars + 2 * SK, *v_empty = v_full + SV;
    uint64_t *s_full = v_empty + SV, *s_free = s_full + 2, *p_full = s_free + 2;
    uint64_t *p_free = p_full + 1, *o_full = p_free + 1, *o_free = o_full + 2, *q_full = o_free + 2;
    uint64_t *drain = q_full + 1;  // two: one per MMA-issuing thread
    int *misc = reinterpret_cast<int *>(smem + C::MISC_OFF);
    int *stage_n = misc, *stage_bad = misc + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 16);
    volatile int *abort_flag = misc + 17;
    int *poison_flag = misc + 19;
    volatile int *ctl = misc + 28;  // the softmax moved its reference max at this tile
    float *mref_s = reinterpret_cast<float *>(smem + C::RED_OFF);
    float *alpha_s = mref_s + NP, *apend_s = alpha_s + NP, *tred = apend_s + NP, *lred = tred + 4 * NP;
    int *prefix = reinterpret_cast<int *>(smem + C::PREFIX_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.B;
    const uint64_t t_start = global_timer_ns();

    if (tid == 32 * 2)
        tma_prefetch_map(&tmk);
    else if (tid == 32 * 3)
        tma_prefetch_map(&tmv);
    if (tid == 0) {
        for (int s = 0; s < SK; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < SV; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
            stage_bad[s] = 0;
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], SMT / 32);  // one arrival per softmax warp
            mbar_init(&o_full[b], 1);
            mbar_init(&o_free[b], SMT / 32);
        }
        mbar_init(p_full, SMT / 32);
        mbar_init(p_free, 1);
        mbar_init(q_full, SMT / 32);
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        *abort_flag = 0;
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
    // Stream-K runs, or (nsplit = 1) one CTA per (request, KV head, head pass).
    int64_t start, end;
    if (p.nsplit == 0) {
        start = run_start(c, W, P);
        end = run_start(c + 1, W, P);
    } else {
        const int64_t j = div_nonneg(c, p.nsplit), i = c - j * p.nsplit;
        const int b = (int)div_nonneg(j, units);
        const int64_t u = j - (int64_t)b * units, kv = div_nonneg(u, p.hch), hc = u - kv * p.hch;
        const int64_t nbj = prefix[b + 1] - prefix[b];
        const int64_t seg0 = hc * p.Hkv * prefix[B] + (int64_t)p.Hkv * prefix[b] + kv * nbj;
        start = seg0 + div_nonneg(i * nbj, p.nsplit);
        end = seg0 + div_nonneg((i + 1) * nbj, p.nsplit);
    }

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
        const int S = is_k ? SK : SV;
        const CUtensorMap *map = is_k ? &tmk : &tmv;
        unsigned char *base = ring + (is_k ? 0 : C::V_RING_OFF);
        uint64_t *full = is_k ? k_full : v_full, *emptyb = is_k ? k_empty : v_empty;
        const uint64_t pol = p.hch > 1 ? l2_evict_normal_policy() : l2_evict_first_policy();
        TileIter it;
        it.init(start, prefix, B, units, p.hch);
        auto box_row = [&](const TileIter &ti, int tok0) -> int {
            const int t = tok0 + lane * box_rows;
            if (!p.block_table)
                return (int)(((int64_t)ti.b * p.Hkv + ti.kvh) * p.block_size + t);
            const int pg = page_of(p, t);
            const int64_t blk = p.block_table[(int64_t)ti.b * p.max_blocks + pg];
            if (blk < 0 || blk >= p.num_blocks)
                return -1;
            return (int)((blk * p.Hkv + ti.kvh) * p.block_size + (t - pg * p.block_size));
        };
        int cur_b = -1, len = 0, k = 0;
        for (int64_t i = start; i < end; ++i, ++k) {
            if (i > start)
                it.next(prefix, B, p.Hkv, p.hch);
            const int s = k % S;
            const uint32_t ph = (uint32_t)((k / S) & 1);
            if (k >= S && !bounded_wait(&emptyb[s], ph ^ 1u, abort_flag, p))
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
                row = box_row(it, tok0);
                bad = row < 0;
                row = bad ? 0 : row;
            }
            const unsigned badmask = __ballot_sync(0xffffffffu, bad);
            if (lane == 0) {
                if (!is_k) {  // tile metadata travels with the V slot
                    stage_n[s] = n;
                    stage_bad[s] = badmask != 0;
                    if (badmask)
                        atomicOr(p.status, DEV_BAD_BLOCK);
                }
                const uint32_t boxes = (uint32_t)(nbox - __popc(badmask));
                mbar_arrive_expect_tx(&full[s], boxes * 2u * (uint32_t)box_rows * 128u);
                if (p.timeline && is_k && k == 0)
                    p.timeline[TL_COLS * c + 4] = global_timer_ns();
            }
            __syncwarp();
            if (lane < nbox && !bad) {
                unsigned char *d = base + (size_t)s * C::SLOT_BYTES + (size_t)lane * box_rows * 128;
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
    } else if (start < end && (warp == 1 || warp == 7)) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t ring_a = smem_addr(ring), q_a = smem_addr(qbuf), p_a = smem_addr(pbuf);
            const int ntiles = (int)(end - start);
            bool ok = true;
            if (warp == 1) {
                // BMM1: S^T[128 x 64] = K[128 x 128] . Q^T, both K-major.
                const uint32_t idesc1 = umma_idesc_bf16(128, NP, 0, 0);
                TileIter it1;
                it1.init(start, prefix, B, units, p.hch);
                int64_t seg1 = -1;
                int piece1 = 0;
                for (int k = 0; k < ntiles && ok; ++k) {
                    if (k > 0)
                        it1.next(prefix, B, p.Hkv, p.hch);
                    if (it1.seg0 != seg1) {
                        seg1 = it1.seg0;
                        ++piece1;
                    }
                    const int s = k % SK, b = k & 1;
                    ok = bounded_wait(&k_full[s], (uint32_t)((k / SK) & 1), abort_flag, p) &&
                         (k < 2 || bounded_wait(&s_free[b], (uint32_t)(((k - 2) >> 1) & 1), abort_flag, p)) &&
                         bounded_wait(q_full, (uint32_t)((piece1 - 1) & 1), abort_flag, p);
                    if (!ok)
                        break;
                    tc_fence_after_sync();
                    const uint32_t ka = ring_a + (uint32_t)(s * C::SLOT_BYTES);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (uint32_t)((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32);
                        const uint32_t qoff = (uint32_t)((kk >> 2) * NP * 128 + (kk & 3) * 32);
                        umma_bf16(tbase + (uint32_t)(C::S_COL + b * NP),
                                  umma_smem_desc(ka + off, 16, 1024, SMEM_LAYOUT_SW128),
                                  umma_smem_desc(q_a + qoff, 16, 1024, SMEM_LAYOUT_SW128), idesc1, kk > 0);
                    }
                    umma_commit(&s_full[b]);
                    umma_commit(&k_empty[s]);
                }
            } else {
                // BMM2: O^T[128 x 128] += V^T . [P_hi | P_lo]^T into the open O buffer
                // (closed by a moved reference or at a piece end; use u in buffer u & 1).
                const uint32_t idesc2 = umma_idesc_bf16(128, C::NO, 1, 1);
                TileIter itp;
                itp.init(start, prefix, B, units, p.hch);
                int64_t segp = itp.seg0;
                int u = 0;
                bool fresh = true;
                for (int k = 0; k < ntiles && ok; ++k) {
                    const int s = k % SV;
                    if (!bounded_wait(p_full, (uint32_t)(k & 1), abort_flag, p)) {
                        ok = false;
                        break;
                    }
                    if (*ctl && !fresh) {
                        umma_commit(&o_full[u & 1]);
                        ++u;
                        fresh = true;
                    }
                    ok = (!fresh || u < 2 ||
                          bounded_wait(&o_free[u & 1], (uint32_t)(((u - 2) >> 1) & 1), abort_flag, p)) &&
                         bounded_wait(&v_full[s], (uint32_t)((k / SV) & 1), abort_flag, p);
                    if (!ok)
                        break;
                    bool piece_ends = true;
                    if (k + 1 < ntiles) {
                        itp.next(prefix, B, p.Hkv, p.hch);
                        piece_ends = itp.seg0 != segp;
                        segp = itp.seg0;
                    }
                    tc_fence_after_sync();
                    const uint32_t va = ring_a + (uint32_t)(C::V_RING_OFF + s * C::SLOT_BYTES);
#pragma unroll
                    for (int kk = 0; kk < T / 16; ++kk)
                        umma_bf16(tbase + (uint32_t)(C::O_COL + (u & 1) * C::NO),
                                  umma_smem_desc(va + (uint32_t)(kk * 2048), C::BOX_BYTES, 1024, SMEM_LAYOUT_SW128),
                                  umma_smem_desc(p_a + (uint32_t)(2 * kk * C::P_LBO), C::P_LBO, 128, SMEM_LAYOUT_NONE),
                                  idesc2, kk > 0 || !fresh);
                    fresh = false;
                    umma_commit(&v_empty[s]);
                    umma_commit(p_free);
                    if (piece_ends) {
                        umma_commit(&o_full[u & 1]);
                        ++u;
                        fresh = true;
                    }
                }
            }
            (void)ok;
            uint64_t *dr = &drain[warp == 1 ? 0 : 1];
            umma_commit(dr);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(dr, 0) && global_timer_ns() - t0 < WAIT_LIMIT_NS) {
            }
        }
    } else if (start < end && (warp >= 2 && warp != 6 && warp != 7)) {
        // ------------------------------------------------------ softmax + correction
        // NGRP warpgroups (warps 2-5, then 8-11, 12-15, ...) each cover all 128 TMEM
        // lanes; group hg carries heads hg * HPT .. hg * HPT + HPT - 1 of the pass.
        const int q4 = warp & 3;                 // TMEM lane quadrant of this warp
        const int ti = q4 * 32 + lane;           // token row (S) and d row (O)
        const int hg = warp < 8 ? 0 : (warp - 4) >> 2;
        const int stid = warp < 8 ? tid - 64 : tid - 128 * (hg + 1);  // 0..127 within the group
        const int sid = hg * 128 + stid;         // 0..SMT-1 among the softmax threads
        const int h0 = hg * HPT;                 // first head of this thread
        const uint32_t tlane = tbase + ((uint32_t)(q4 * 32) << 16);
        const uint32_t acol = tlane + (uint32_t)(C::ACC_COL + h0);  // this thread's acc columns
        const float4 *mref4 = reinterpret_cast<const float4 *>(mref_s + h0);
        const float qscale = p.qscale;
        // The softmax warps arrive on the pipeline barriers once per warp: the warp's
        // writes (and its tensor-memory reads, fenced by the caller) are ordered
        // before lane 0's release by __syncwarp.
        auto warp_arrive = [&](uint64_t *bar) {
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar);
        };
        // l_t: this token's share of each of its heads' normalisers.  The closed O
        // buffers are folded into acc, this d row's HPT columns of TMEM (ACC_COL),
        // relative to the current reference maxima (mref_s).
        float l_t[HPT];
        PendingPiece pending[2];
        int npending = 0;
        bool poisoned = false;
        TileIter it, cur;
        it.init(start, prefix, B, units, p.hch);
        cur = it;
        int64_t piece_first = start;
        int u = 0;
        bool ok = true;

        // acc[ch] = acc[ch] * w + add, 16 columns at a time.  (tcgen05.ld / st are
        // warp-collective: every lane of a warp takes part or none does.)
        auto acc_update = [&](int ch, const float (&add)[16], const float *w) {
            float a[16];
            tmem_load<16>(acol + 16 * ch, a);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                a[j] = fmaf(a[j], w ? w[j] : 1.f, add[j]);
            tmem_store16(acol + 16 * ch, a);
        };

        // Fold closed O buffer use u into acc (scaled by apend_s when `weighted`) and
        // hand the buffer back.
        auto fold = [&](bool weighted) {
            const int bc = u & 1;
            const bool got = __all_sync(0xffffffffu, ok && bounded_wait(&o_full[bc], (uint32_t)((u >> 1) & 1),
                                                                         abort_flag, p));
            if (got) {
                tc_fence_after_sync();
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch) {
                    float o[16], olo[16], w[16];
                    tmem_load<16>(tlane + (uint32_t)(C::O_COL + bc * C::NO + h0 + 16 * ch), o);
                    tmem_load<16>(tlane + (uint32_t)(C::O_COL + bc * C::NO + NP + h0 + 16 * ch), olo);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        w[j] = weighted ? apend_s[h0 + 16 * ch + j] : 1.f;
                        o[j] = (o[j] + olo[j]) * w[j];
                    }
                    acc_update(ch, o, nullptr);
                }
            } else {
                ok = false;
                poisoned = true;
            }
            tc_fence_before_sync();
            warp_arrive(&o_free[bc]);
            ++u;
        };

        auto epilogue = [&](int64_t last_excl) {
            fold(false);
            // Normaliser per head: the 128 token threads' partials, 16 heads at a time
            // through a transposed warp reduction, then the four warps.
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                float lv[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    lv[j] = l_t[16 * ch + j];
                const float mine = warp_transpose_reduce<16, false>(lv, lane);
                if ((lane & 1) == 0)
                    lred[q4 * NP + h0 + 16 * ch + (lane >> 1)] = mine;
            }
            if (poisoned)
                atomicOr(poison_flag, 1);
            named_barrier_sync(1, SMT);
            const bool pois = *reinterpret_cast<volatile int *>(poison_flag) != 0;
            const bool complete = piece_first == cur.seg0 && last_excl == cur.seg0 + cur.nb;
            const int rows = min(NP, p.R - cur.hc * NP);
            const int r0 = cur.hc * NP;
            const int64_t vseg = ((int64_t)cur.b * p.Hkv + cur.kvh) * p.hch + cur.hc;
            float *slot = p.slots + (p.nsplit ? c : 2 * c + (piece_first == start ? 0 : 1)) * (int64_t)SLOT;
            auto lsum = [&](int g) {
                return lred[g] + lred[NP + g] + lred[2 * NP + g] + lred[3 * NP + g];
            };
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                float a[16];
                tmem_load<16>(acol + 16 * ch, a);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int g = h0 + 16 * ch + j;
                    if (!complete)
                        slot[g * D + ti] = a[j];
                    else if (g < rows)
                        write_result<false>(p, out_row_q1(p, cur.b, cur.kvh, r0 + g), ti, D, a[j], mref_s[g],
                                            lsum(g), pois);
                }
            }
            if (!complete && sid < NP) {
                slot[NP * D + sid] = mref_s[sid];
                slot[NP * D + NP + sid] = pois ? __int_as_float(0x7fc00000) : lsum(sid);
            }
            named_barrier_sync(1, SMT);
            if (!complete)
                pending[npending++] =
                    PendingPiece{cur.seg0, piece_first, last_excl, vseg, 0, cur.nb, rows, cur.b, cur.kvh, r0};
            if (sid == 0)
                *poison_flag = 0;
            named_barrier_sync(1, SMT);
        };

        bool fold_pend = false;
        uint64_t t_scores = 0;
        int k = 0;
        for (int64_t i = start;; ++i, ++k) {
            const bool past = i == end;
            if (i > start && !past)
                it.next(prefix, B, p.Hkv, p.hch);
            const bool first_tile = !past && (i == start || it.seg0 != cur.seg0);
            if (first_tile) {
                // Q of the new (request, KV head, head pass) in the 128-byte-swizzled
                // K-major layout BMM1 reads.  Every BMM1 of the previous piece has
                // completed: its last S has been consumed.
#pragma unroll
                for (int r = 0; r < 1024 / SMT; ++r) {
                    const int x = sid + SMT * r;
                    const int half = x >> 9, g = (x >> 3) & (NP - 1), cc = x & 7;
                    uint4 w = make_uint4(0, 0, 0, 0);
                    if (it.hc * NP + g < p.R)
                        w = __ldg(reinterpret_cast<const uint4 *>(
                            p.q + (out_row_q1(p, it.b, it.kvh, it.hc * NP + g) * D + half * 64 + cc * 8)));
                    *reinterpret_cast<uint4 *>(qbuf + half * NP * 128 + g * 128 + ((cc ^ (g & 7)) << 4)) = w;
                }
                fence_proxy_async_smem();
                warp_arrive(q_full);
            }
            if (first_tile || past) {
                if (i > start) {
                    if (fold_pend)
                        fold(true);
                    fold_pend = false;
                    epilogue(i);
                }
                if (past)
                    break;
                cur = it;
                piece_first = i;
                poisoned = false;
                float zero[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    zero[j] = 0.f;
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch)
                    tmem_store16(acol + 16 * ch, zero);
#pragma unroll
                for (int j = 0; j < HPT; ++j)
                    l_t[j] = 0.f;
                if (sid < NP)
                    mref_s[sid] = -INFINITY;
                named_barrier_sync(1, SMT);
            }

            const int s = k % SV, b = k & 1;
            int n = 0;
            const bool have = __all_sync(0xffffffffu, ok && bounded_wait(&v_full[s], (uint32_t)((k / SV) & 1),
                                                                          abort_flag, p) &&
                                                          bounded_wait(&s_full[b], (uint32_t)((k >> 1) & 1),
                                                                       abort_flag, p));
            // This thread's HPT scores of the tile (the S buffer is released only after
            // P has been computed from them).
            float sc[HPT];
            if (have) {
                n = stage_n[s];
                poisoned |= stage_bad[s] != 0;
                tc_fence_after_sync();
                tmem_load<HPT>(tlane + (uint32_t)(C::S_COL + b * NP + h0), sc);
                if (k == 0 && sid == 0 && p.timeline)
                    t_scores = global_timer_ns();
            } else {
                ok = false;
                poisoned = true;
            }
            // A buffer closed at the previous tile is folded before this tile may
            // rescale acc (and before its weights in apend_s can change).
            if (fold_pend)
                fold(true);
            fold_pend = false;
            const bool valid = have && ti < n;
            // Lazy rescale test: does any score exceed its head's reference by more
            // than 2^LAZY?  (x = scaled score relative to the reference.)
            float xmax = -INFINITY;
            if (valid) {
#pragma unroll
                for (int q = 0; q < HPT / 4; ++q) {
                    const float4 m4 = mref4[q];
                    xmax = fmaxf(xmax, fmaxf(fmaxf(fmaf(sc[4 * q], qscale, -m4.x), fmaf(sc[4 * q + 1], qscale, -m4.y)),
                                             fmaxf(fmaf(sc[4 * q + 2], qscale, -m4.z), fmaf(sc[4 * q + 3], qscale, -m4.w))));
                }
            }
            const bool moved = named_barrier_or(1, SMT, !(xmax <= C::LAZY));
            if (moved) {
                // Tile maximum per head over the 128 tokens: warp, then the 4 warps.
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch) {
                    float mx[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        mx[j] = valid ? sc[16 * ch + j] * qscale : -INFINITY;
                    const float wmax = warp_transpose_reduce<16, true>(mx, lane);
                    if ((lane & 1) == 0)
                        tred[q4 * NP + h0 + 16 * ch + (lane >> 1)] = wmax;
                }
                named_barrier_sync(1, SMT);
                if (sid < NP) {
                    const int g = sid;
                    const float tm = fmaxf(fmaxf(tred[g], tred[NP + g]), fmaxf(tred[2 * NP + g], tred[3 * NP + g]));
                    const float m_old = mref_s[g];
                    const float m_new = tm > m_old + C::LAZY ? tm : m_old;
                    const float a = m_new == m_old ? 1.f : fast_exp2(m_old - m_new);
                    mref_s[g] = m_new;
                    alpha_s[g] = a;
                    apend_s[g] = a;  // the weights of the O buffer this tile closes
                }
                named_barrier_sync(1, SMT);
                float zero[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    zero[j] = 0.f;
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch) {
                    float a[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        a[j] = alpha_s[h0 + 16 * ch + j];
                        l_t[16 * ch + j] *= a[j];
                    }
                    acc_update(ch, zero, a);
                }
            }
            // P = 2^x as hi + lo, both bf16, computed before the P buffer is free: hi
            // keeps the top 16 bits of p (truncation), lo = p - hi (exact in fp32)
            // rounded to bf16, so hi + lo carries about 16 significant bits.
            uint32_t whi[HPT / 2], wlo[HPT / 2];
#pragma unroll
            for (int q = 0; q < HPT / 4; ++q) {
                const float4 m4 = mref4[q];
                const float mq[4] = {m4.x, m4.y, m4.z, m4.w};
                float pr[4], lo[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float x = valid ? fmaf(sc[4 * q + j], qscale, -mq[j]) : -INFINITY;
                    pr[j] = fast_exp2(x);  // 0 for an invalid token
                    l_t[4 * q + j] += pr[j];
                    lo[j] = pr[j] - __uint_as_float(__float_as_uint(pr[j]) & 0xffff0000u);
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    whi[2 * q + j] = __byte_perm(__float_as_uint(pr[2 * j]), __float_as_uint(pr[2 * j + 1]), 0x7632);
                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(lo[2 * j], lo[2 * j + 1]);
                    wlo[2 * q + j] = *reinterpret_cast<const uint32_t *>(&l2);
                }
            }
            tc_fence_before_sync();
            warp_arrive(&s_free[b]);
            // The P buffer was last read by BMM2 of the previous tile.
            if (k >= 1 && ok && !bounded_wait(p_free, (uint32_t)((k - 1) & 1), abort_flag, p)) {
                ok = false;
                poisoned = true;
            }
            // No-swizzle MN-major layout: token ti's 8-head groups are 16-byte rows of
            // 8x8 core matrices; P_hi heads in core groups 0..NP/8-1, P_lo heads in
            // NP/8..2NP/8-1.
            unsigned char *pd = pbuf + (ti >> 3) * C::P_LBO + (ti & 7) * 16;
#pragma unroll
            for (int q = 0; q < HPT / 8; ++q) {
                const int ng = h0 / 8 + q;
                *reinterpret_cast<uint4 *>(pd + ng * 128) =
                    make_uint4(whi[4 * q], whi[4 * q + 1], whi[4 * q + 2], whi[4 * q + 3]);
                *reinterpret_cast<uint4 *>(pd + (NP / 8 + ng) * 128) =
                    make_uint4(wlo[4 * q], wlo[4 * q + 1], wlo[4 * q + 2], wlo[4 * q + 3]);
            }
            // Rows past the valid tokens may hold anything (stale tiles, poison):
            // zero this token's V row so that 0-weight rows add exact zeros.
            if (hg == 0 && !(ti < n)) {
                unsigned char *vr = ring + C::V_RING_OFF + (size_t)s * C::SLOT_BYTES + ti * 128;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc)
                        *reinterpret_cast<uint4 *>(vr + h * C::BOX_BYTES + cc * 16) = make_uint4(0, 0, 0, 0);
            }
            // A moved reference closes the open O buffer (unless this tile opens a
            // piece, whose buffer is fresh anyway).
            const bool close = moved && !first_tile;
            if (sid == 0)
                *ctl = close ? 1 : 0;
            fence_proxy_async_smem();
            warp_arrive(p_full);
            fold_pend = close;
        }
        const uint64_t t_streamed = p.timeline ? global_timer_ns() : 0;
        if (p.nsplit)
            npending = 0;  // one CTA per segment: every piece is whole
        for (int x = 0; x < npending; ++x)
            publish_piece(p, pending[x].vseg, sid, 1, SMT);
        for (int x = 0; x < npending; ++x) {
            const PendingPiece &pp = pending[x];
            merge_segment_gather<NP, D, SMT, false>(p, c, pp.seg0, pp.nb, pp.first, pp.vseg, W, P, pp.rows,
                                                    pp.b, pp.kvh, pp.r0, reinterpret_cast<int *>(pbuf),
                                                    reinterpret_cast<float *>(ring), misc + 20, sid, 1,
                                                    abort_flag);
        }
        if (p.timeline && sid == 0) {
            unsigned long long *rec = p.timeline + TL_COLS * c;
            rec[5] = t_scores;
            rec[6] = t_streamed;
            rec[7] = global_timer_ns();
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tbase, C::TMEM_COLS);
    }
    if (p.timeline && tid == 0) {
        unsigned sm;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
        unsigned long long *rec = p.timeline + TL_COLS * c;
        rec[0] = t_start;
        rec[1] = global_timer_ns();
        rec[2] = sm;
        rec[3] = (unsigned long long)(end - start);
        if (start >= end)
            for (int x = 4; x < TL_COLS; ++x)
                rec[x] = 0;
    }
}

}  // namespace gqa
