// decode_tc.cuh -- persistent stream-K decode attention on the 5th-generation
// tensor cores (tcgen05), for groups of G >= 4 query heads per KV head (D = 64, 128 or
// 256; decode_tc_wide.cuh takes more than 16 heads per KV head at D = 128).
// The MMAs run M = 128 tokens by N = 16 heads; the softmax threads carry only
// the NV <= 16 heads that exist.
//
// Same LeanTile schedule as the CUDA-core kernel (schedule.cuh): each CTA walks a
// contiguous run of 128-token tiles of (request, KV head, 16-head chunk) segments.
// Roles (one CTA per SM, 8 warps):
//   warps 0, 6 TMA: each tile's K rows (warp 0) and V rows (warp 6) arrive as
//              128-byte-swizzled boxes (one per page, two 64-column halves) into
//              separate 3-slot rings: a K slot frees as soon as BMM1 has read it,
//              a V slot only after BMM2.
//   warp 1     BMM1 (one thread): S^T[128 x 16] = K[128 x 128] . Q^T, K and Q
//              K-major, into one of two TMEM S buffers.
//   warp 7     BMM2 (one thread): O^T[128 x 32] += V^T . [P_hi | P_lo]^T, V read
//              MN-major straight from the swizzled TMA boxes, P from shared
//              memory as two bf16 terms (hi and lo) so that P carries ~16
//              significant bits; the two terms are the halves of one N = 32
//              operand, since an MMA of N <= 128 costs the same ~90 cycles.  O
//              accumulates in TMEM across tiles while the softmax reference
//              maximum stays put (two O buffers: one open, one being read back).
//              Two issuing threads let a late K tile never hold back the BMM2 that
//              frees a V slot.
//   warps 2-5  softmax (thread = TMEM lane = token row): read S, and while no
//              score exceeds the reference maximum by more than 2^8 (one
//              barrier-OR per tile decides) write P = 2^(s - m) directly; otherwise
//              take the tile maximum, move the reference, rescale, and have BMM2
//              close the open O buffer, which is folded into fp32 registers.
// Pieces: whole segments are written at once; split segments are merged by all
// of their owners together after streaming (gather_merge.cuh; the launch is
// cooperative, so every CTA is resident).  (Attention co-design for long-context
// inference, sections "FlashAttention and GEMM shapes" and "Effect of group size
// G": decode GEMM-M equals G; LeanAttention decode tiles digest, sections "Exact
// softmax that merges piece by piece" and "Hardware-sized work units".)
#pragma once

#include <cuda_fp8.h>

#include "gather_merge.cuh"
#include "schedule.cuh"
#include "tc.cuh"

namespace gqa {

struct TcCfg {
    // (merge scratch lives in the P buffers: checked below)
    static constexpr int T = 128, NP = 16;             // tile tokens, heads per MMA
    static constexpr int THREADS = 256;
    static constexpr int BOX_BYTES = T * 128;          // one 64-column half of a tile: 16 KB
    static constexpr int QBUF_BYTES = 2 * NP * 128;    // two halves, NP rows of 128 B
    static constexpr int NO = 2 * NP;                  // BMM2 columns: P_hi heads, P_lo heads
    static constexpr int P_LBO = (NO / 8) * 128;       // P: stride between 8-token groups
    static constexpr int PBUF_BYTES = (T / 8) * P_LBO;
    static constexpr int S_COL = 0, O_COL = 2 * NP;    // TMEM columns: S x2, O x2 (NO wide)
    static constexpr int TMEM_COLS = 128;              // >= 2 * NP + 2 * NO, power of two
    static constexpr float LAZY = 8.f;                 // rescale only when max grows > 2^8
    static constexpr int SLOT_FLOATS = slot_floats(NP, 128);  // the larger head dimension
    static constexpr int MAX_BATCH = 1024;
};
static_assert(TcCfg::O_COL + 2 * TcCfg::NO <= TcCfg::TMEM_COLS, "tensor memory columns");

// Shared-memory layout for head dimension D (F8: an FP8 E4M3 cache, D = 128).  A
// ring slot holds one K or V tile of 128-byte boxes (one box row per token):
// two boxes at bf16 D = 128 (32 KB, three slots per ring), one at bf16 D = 64
// (16 KB, five slots per ring, so that as many bytes stay in flight).  FP8 tiles
// are 256 tokens (TH = 2 halves of 128): one box row per token, 32 KB, three
// slots per ring, so that a pipeline step moves 64 KB as at bf16 D = 128; BMM1
// writes each half's scores to its own TMEM columns, BMM2 runs K = 256 tokens,
// each softmax thread carries two token rows, and Q has one buffer (the rings and
// the 12 KB P buffers then fit).  At bf16 D = 64 BMM2 still runs M = 128 over
// V^T; its rows 64..127 come from one 16 KB block of zeros shared by every V slot
// (the operand's leading-byte offset points there).  At 8 bits one box row spans all 128 rows
// of V^T.  At bf16 D = 256 a tile's two 128-column halves are two consecutive
// slots of the 32 KB rings (SUB = 2): BMM1 accumulates S over both, BMM2 writes
// each half's O rows to its own TMEM columns; Q (8 KB) has one buffer, so that the
// rings keep three slots.
template <int D, bool F8 = false>
struct TcGeom {
    static_assert(!F8 || D == 128, "FP8 tiles are built for D = 128");
    static constexpr int SUB = D == 256 ? 2 : 1;           // ring slots per tile
    // 128-token halves per tile: FP8 tiles are 256 tokens (64 KB of K and V, as a
    // bf16 tile at D = 128), so that each pipeline step moves as many bytes.
    static constexpr int TH = F8 ? 2 : 1;
    static constexpr int TILE = TcCfg::T * TH;             // tokens per tile
    static constexpr int BOXES = (F8 ? D : 2 * D / SUB) / 128;  // 128-byte boxes per token row of a slot
    static constexpr bool NEED_ZERO = !F8 && D == 64;
    static constexpr int STAGES = (BOXES == 1 && !F8) ? 5 : 3;  // slots per ring (K ring, V ring)
    static constexpr int SLOT_BYTES = BOXES * TcCfg::BOX_BYTES * TH;
    static constexpr int QBUFS = (D == 256 || F8) ? 1 : 2;  // Q buffers
    // P buffer: bf16 hi | lo for 16 heads per 128 tokens, or FP8's three E4M3 terms
    // (three 128-byte core matrices per 8 tokens) for a 256-token tile.
    static constexpr int PBUF = F8 ? (TILE / 8) * 3 * 128 : TcCfg::PBUF_BYTES;
    static constexpr int QBUF = (D == 256 ? 2 : 1) * TcCfg::QBUF_BYTES;
    static constexpr size_t V_RING_OFF = (size_t)STAGES * SLOT_BYTES;
    static constexpr size_t ZERO_OFF = 2 * V_RING_OFF;                 // NEED_ZERO only
    static constexpr size_t Q_OFF = ZERO_OFF + (NEED_ZERO ? TcCfg::BOX_BYTES : 0);
    static constexpr size_t P_OFF = Q_OFF + QBUFS * QBUF;
    static constexpr size_t BAR_OFF = P_OFF + 2 * PBUF;
    static constexpr int NBAR = 4 * STAGES + 16;
    static constexpr size_t MISC_OFF = BAR_OFF + NBAR * 8;
    // floats: tile maxima [2][4][NP], piece sums [4][NP], merge maxima [NP], then
    // (FP8) the per-row scales of the piece's Q terms [NP]
    static constexpr size_t RED_OFF = MISC_OFF + 64 * 4;
    static constexpr size_t PREFIX_OFF = RED_OFF + 13 * TcCfg::NP * 4 + 64;
    // +1024: the dynamic shared-memory base is re-aligned to 1024 bytes in-kernel.
    static size_t smem_bytes(int B) { return PREFIX_OFF + (size_t)(B + 1) * sizeof(int) + 1024; }
    // Segment merge: the owner list (<= 512 ints) in the P buffers; the gathered
    // slices, at most E + 4 no + 3 no (E / D + 2) + 2 NP floats (E <= NP x D
    // outputs, no <= 512 owners, slices rounded to 4 elements), in the rings.
    static_assert(512 * 4 <= 2 * PBUF, "owner list must fit in the P buffers");
    static_assert((16 * D + 4 * 512 + 3 * 512 * (16 + 2) + 32) * 4 <= 2 * V_RING_OFF,
                  "gathered slices must fit in the rings");
    static_assert(STAGES <= 8, "stage_n and stage_bad hold 8 slots");
    static_assert(Q_OFF % 1024 == 0 && ZERO_OFF % 1024 == 0, "swizzled buffers are 1024-byte aligned");
    static_assert(PREFIX_OFF + (TcCfg::MAX_BATCH + 1) * sizeof(int) + 1024 <= 227 * 1024,
                  "shared memory per CTA");
};

// One float to E4M3 (round to nearest even, saturating) and back, exactly.
__device__ __forceinline__ uint32_t to_e4m3(float x)
{
    return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float e4m3_value(uint32_t b)
{
    const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3);
    return __half2float(__half(h));
}
// x as two E4M3 terms, x ~ hi + lo / 16 (lo carries the remainder scaled by 16).
__device__ __forceinline__ void split_e4m3(float x, uint32_t &hi, uint32_t &lo)
{
    hi = to_e4m3(x);
    lo = to_e4m3((x - e4m3_value(hi)) * 16.f);
}

// x as three E4M3 terms, x ~ t1 + t2 / 16 + t3 / 256 (about 12 significant bits;
// each term carries the remainder of the ones before it, scaled by 16).
__device__ __forceinline__ void split3_e4m3(float x, uint32_t &t1, uint32_t &t2, uint32_t &t3)
{
    t1 = to_e4m3(x);
    const float r1 = (x - e4m3_value(t1)) * 16.f;
    t2 = to_e4m3(r1);
    t3 = to_e4m3((r1 - e4m3_value(t2)) * 16.f);
}

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

// NV: query heads the softmax threads carry (4, 8 or 16 = the MMA width NP);
// the MMAs always run NP = 16 columns, and columns NV..NP-1 of S and O are
// never read (zero Q rows in, P left as is: an O column depends on its P column only).
// MQ: several query tokens per request (causal mask inside them); the one-token
// decode instantiation carries no mask code.
// DH: head dimension, 64, 128 or 256.  At 64, BMM1 takes 4 K-steps over the one
// 64-column half that is loaded, and BMM2 still runs M = 128 over V^T with rows
// 64..127 read from a block of zeros (written once, never loaded), so the O rows
// 64..127 are zero and are not read back.  At 256 (one query token, bf16) each
// tile's two 128-column halves come through two ring slots (TcGeom::SUB).
// F8: the cache holds FP8 E4M3 (D = 128), in 256-token tiles (TcGeom::TH): the
// MMAs run kind::f8f6f4 (K = 32) on the cache bytes as loaded.  Q enters as two E4M3 terms, t1 + t2 / 16 (exact for
// bf16 q after the row's power-of-two scaling), side by side in N = 32 (one term
// per 16 columns); P as three, t1 + t2 / 16 + t3 / 256, in N = 48: two terms
// leave the weights of the keys that dominate a row 8 significant bits, whose
// error alone can move a bf16 output by one unit.  The softmax and the fold add
// the column blocks back.  Scores are scaled by p.qscale (which holds the
// K scale) and by the power of two that brought each Q row into E4M3's range.
template <int NV, bool MQ, int DH = 128, bool F8 = false>
__global__ void __launch_bounds__(TcCfg::THREADS, 1)
    gqa_decode_tc_kernel(const Params p, const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv, int box_rows)
{
    using C = TcCfg;
    using L = TcGeom<DH, F8>;
    constexpr int TH = L::TH;                       // 128-token halves per tile
    constexpr int S = L::STAGES, NP = C::NP, D = DH, T = L::TILE;
    constexpr int HALVES = L::BOXES;  // 128-byte boxes loaded per token row of a slot
    constexpr int SUB = L::SUB;       // ring slots per tile (2 at D = 256)
    constexpr int QH = D / 64;        // 64-column halves of a bf16 Q row
    constexpr int QBUFS = L::QBUFS;
    constexpr int SW = F8 ? 2 * NP : NP;            // S columns per buffer
    constexpr int SWB = SW * TH;                     // S columns per buffer, all halves
    constexpr int OC = F8 ? 2 * SWB : C::O_COL;     // first O column
    constexpr int KSTEP = F8 ? 32 : 16;             // MMA K per instruction
    // FP8 P: per 8-token group, two 128-byte core matrices along N (16 E4M3 heads
    // per 16-byte row: term 1, then term 2).
    constexpr int NO = F8 ? 3 * NP : C::NO;         // BMM2 columns: the P terms side by side
    constexpr int P8_LBO = 3 * 128;                 // FP8 P: three core matrices per 8 tokens
    constexpr int TMEM_COLS = (F8 || SUB == 2) ? 256 : C::TMEM_COLS;
    static_assert(OC + 2 * NO * SUB <= TMEM_COLS, "tensor memory columns");
    static_assert(!F8 || (T / 8) * P8_LBO <= L::PBUF, "FP8 P buffer");
    static_assert(D == 64 || D == 128 || (D == 256 && !MQ && !F8), "head dimension");
    constexpr int SLOT = slot_floats(NV, D);
    constexpr int LPH = 32 / NV;  // lanes per head after a transposed warp reduction
    static_assert(NV == 4 || NV == 8 || NV == 16, "softmax head count");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    unsigned char *ring = smem;
    unsigned char *qbuf = smem + L::Q_OFF;
    unsigned char *pbuf = smem + L::P_OFF;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *k_full = bars, *k_empty = bars + S, *v_full = bars + 2 * S, *v_empty = bars + 3 * S;
    uint64_t *s_full = bars + 4 * S, *s_free = s_full + 2, *p_full = s_free + 2;
    uint64_t *o_full = p_full + 2, *o_free = o_full + 2, *q_full = o_free + 2, *p_free = q_full + 2;
    uint64_t *drain = p_free + 2;  // two: one per MMA-issuing thread
    int *misc = reinterpret_cast<int *>(smem + L::MISC_OFF);
    int *stage_n = misc, *stage_bad = misc + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 16);
    volatile int *abort_flag = misc + 17;
    int *last_flag = misc + 18, *poison_flag = misc + 19;
    volatile int *ctl = misc + 28;  // per P buffer: the softmax moved its reference max
    float *red = reinterpret_cast<float *>(smem + L::RED_OFF);
    int *prefix = reinterpret_cast<int *>(smem + L::PREFIX_OFF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.B;
    const uint64_t t_start = global_timer_ns();

    // The tensor maps are fetched while the barriers, TMEM and the tile prefix sums
    // are set up.
    if (tid == 32 * 2)
        tma_prefetch_map(&tmk);
    else if (tid == 32 * 3)
        tma_prefetch_map(&tmv);
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
            mbar_init(&p_free[b], 1);
        }
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        *abort_flag = 0;
        *last_flag = 0;
        *poison_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    if constexpr (L::NEED_ZERO) {
        // The block BMM2 reads as V^T rows 64..127 stays zero for the whole launch.
        // Likewise Q's upper half.
        for (int x = tid; x < C::BOX_BYTES / 16; x += C::THREADS)
            reinterpret_cast<uint4 *>(ring + L::ZERO_OFF)[x] = make_uint4(0, 0, 0, 0);
        for (int x = tid; x < QBUFS * L::QBUF / 16; x += C::THREADS)
            reinterpret_cast<uint4 *>(qbuf)[x] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
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
    // Stream-K: CTA c takes tiles [cW/P, (c+1)W/P) of the global order.  Fixed
    // split (the FlashDecoding comparator): CTA c takes chunk c % nsplit of
    // segment c / nsplit, the chunks cutting the segment's tiles evenly.
    int64_t start, end;
    if (p.nsplit == 0) {
        start = run_start(c, W, P);
        end = run_start(c + 1, W, P);
    } else {
        // Segment j = (b, kvh, hc) in that order; its first tile in the global order
        // (hc, b, kvh, tile).
        const int64_t j = div_nonneg(c, p.nsplit), i = c - j * p.nsplit;
        const int b = (int)div_nonneg(j, units);
        const int64_t u = j - (int64_t)b * units, kv = div_nonneg(u, p.hch), hc = u - kv * p.hch;
        const int64_t nbj = prefix[b + 1] - prefix[b];
        const int64_t seg0 = hc * p.Hkv * prefix[B] + (int64_t)p.Hkv * prefix[b] + kv * nbj;
        start = seg0 + div_nonneg(i * nbj, p.nsplit);
        end = seg0 + div_nonneg((i + 1) * nbj, p.nsplit);
    }
    const int G = p.G;

    for (int b = (int)c; b < B; b += (int)P) {
        if (prefix[b + 1] != prefix[b])
            continue;
        int64_t begin, len;
        const bool bad = !request_range<false>(p, b, begin, len);
        for (int e = tid; e < p.qlen * p.Hq * D; e += C::THREADS)
            write_result<false>(p, (int64_t)b * p.qlen * p.Hq + e / D, e % D, D, 0.f, -INFINITY, 0.f, bad);
    }

    if (start < end && (warp == 0 || warp == 6)) {
        // ---------------------------------------------------------------- TMA
        const bool is_k = warp == 0;
        const CUtensorMap *map = is_k ? &tmk : &tmv;
        unsigned char *base = ring + (is_k ? 0 : L::V_RING_OFF);
        uint64_t *full = is_k ? k_full : v_full, *emptyb = is_k ? k_empty : v_empty;
        // K/V are read once, except when several 16-head chunks of a KV head (G > 16)
        // stream the same tiles at about the same time: then L2 keeps them for the
        // other chunks.
        const uint64_t pol = p.hch > 1 ? l2_evict_normal_policy() : l2_evict_first_policy();
        TileIter it;
        it.init(start, prefix, B, units, p.hch);
        // Global row of this lane's box of tile `ti` (lane < boxes), or -1 for a
        // block id outside the pool.
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
        int cur_b = -1, len = 0, ks = 0;  // ks: ring slots filled (SUB per tile)
        if constexpr (SUB == 1) {
            for (int64_t i = start; i < end; ++i, ++ks) {
                if (i > start)
                    it.next(prefix, B, p.Hkv, p.hch);
                const int s = ks % S;
                const uint32_t ph = (uint32_t)((ks / S) & 1);
                if (ks >= S && !bounded_wait(&emptyb[s], ph ^ 1u, abort_flag, p))
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
                    mbar_arrive_expect_tx(&full[s], boxes * (uint32_t)HALVES * (uint32_t)box_rows * 128u);
                    if (p.timeline && is_k && ks == 0)
                        p.timeline[TL_COLS * c + 4] = global_timer_ns();
                }
                __syncwarp();
                if (lane < nbox && !bad) {
                    unsigned char *d = base + (size_t)s * L::SLOT_BYTES + (size_t)lane * box_rows * 128;
                    tma_load_2d(d, map, 0, row, &full[s], pol);
                    if constexpr (HALVES == 2)
                        tma_load_2d(d + C::BOX_BYTES, map, 64, row, &full[s], pol);
                }
            }
        } else {
            // D = 256: the tile's two column halves go to two consecutive slots.
            bool stop = false;
            for (int64_t i = start; i < end && !stop; ++i) {
                if (i > start)
                    it.next(prefix, B, p.Hkv, p.hch);
                int n = 0, nbox = 0, row = 0;
                bool bad = false;
                unsigned badmask = 0;
#pragma unroll
                for (int sub = 0; sub < SUB; ++sub, ++ks) {
                    const int s = ks % S;
                    const uint32_t ph = (uint32_t)((ks / S) & 1);
                    if (ks >= S && !bounded_wait(&emptyb[s], ph ^ 1u, abort_flag, p)) {
                        stop = true;
                        break;
                    }
                    if (sub == 0) {
                        if (it.b != cur_b) {
                            cur_b = it.b;
                            int64_t b0, l0;
                            request_range<false>(p, cur_b, b0, l0);
                            len = (int)l0;
                        }
                        const int tok0 = it.j * T;
                        n = min(T, len - tok0);
                        nbox = (n + box_rows - 1) / box_rows;
                        if (lane < nbox) {
                            row = box_row(it, tok0);
                            bad = row < 0;
                            row = bad ? 0 : row;
                        }
                        badmask = __ballot_sync(0xffffffffu, bad);
                    }
                    if (lane == 0) {
                        if (!is_k) {
                            stage_n[s] = n;
                            stage_bad[s] = badmask != 0;
                            if (badmask)
                                atomicOr(p.status, DEV_BAD_BLOCK);
                        }
                        const uint32_t boxes = (uint32_t)(nbox - __popc(badmask));
                        mbar_arrive_expect_tx(&full[s], boxes * (uint32_t)HALVES * (uint32_t)box_rows * 128u);
                        if (p.timeline && is_k && ks == 0)
                            p.timeline[TL_COLS * c + 4] = global_timer_ns();
                    }
                    __syncwarp();
                    if (lane < nbox && !bad) {
                        unsigned char *d = base + (size_t)s * L::SLOT_BYTES + (size_t)lane * box_rows * 128;
                        tma_load_2d(d, map, sub * 128, row, &full[s], pol);
                        tma_load_2d(d + C::BOX_BYTES, map, sub * 128 + 64, row, &full[s], pol);
                    }
                }
            }
        }
        if (lane == 0) {
            for (int kk = max(0, ks - S); kk < ks; ++kk) {
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(&full[kk % S], (uint32_t)((kk / S) & 1)) &&
                       global_timer_ns() - t0 < WAIT_LIMIT_NS) {
                }
            }
        }
    } else if (start < end && (warp == 1 || warp == 7)) {
        // ---------------------------------------------------------------- MMA
        // Two issuing threads: warp 1 issues every BMM1, warp 7 every BMM2, each in
        // tile order and each waiting (asleep) only for its own operands, so a late
        // K tile never holds back the BMM2 that frees a V slot.  tcgen05.commit
        // tracks the MMAs of the committing thread alone.
        if (lane == 0) {
            const uint32_t ring_a = smem_addr(ring), q_a = smem_addr(qbuf), p_a = smem_addr(pbuf);
            const int ntiles = (int)(end - start);
            bool ok = true;
            if (warp == 1) {
                const uint32_t idesc1 = F8 ? umma_idesc_e4m3(128, SW, 0, 0) : umma_idesc_bf16(128, NP, 0, 0);
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
                    const int b = k & 1, qb = QBUFS == 2 ? (piece1 - 1) & 1 : 0;
                    const uint32_t qpar = (uint32_t)((QBUFS == 2 ? (piece1 - 1) >> 1 : piece1 - 1) & 1);
                    const uint32_t qa = q_a + (uint32_t)(qb * L::QBUF);
#pragma unroll
                    for (int sub = 0; sub < SUB && ok; ++sub) {
                        const int ks = k * SUB + sub, s = ks % S;
                        ok = bounded_wait(&k_full[s], (uint32_t)((ks / S) & 1), abort_flag, p) &&
                             (sub > 0 || k < 2 ||
                              bounded_wait(&s_free[b], (uint32_t)(((k - 2) >> 1) & 1), abort_flag, p)) &&
                             (sub > 0 || bounded_wait(&q_full[qb], qpar, abort_flag, p));
                        if (!ok)
                            break;
                        tc_fence_after_sync();
                        const uint32_t ka = ring_a + (uint32_t)(s * L::SLOT_BYTES);
#pragma unroll
                        for (int th = 0; th < TH; ++th) {
                            // token half th (FP8): slot rows 128 th .., into its own S columns
#pragma unroll
                            for (int kk = 0; kk < D / SUB / KSTEP; ++kk) {
                                // 32 bytes of every row per instruction: 16 bf16 or 32 E4M3 elements.
                                const uint32_t off = (uint32_t)((th + (kk >> 2)) * C::BOX_BYTES + (kk & 3) * 32);
                                const uint32_t qoff = (uint32_t)((2 * sub + (kk >> 2)) * NP * 128 + (kk & 3) * 32);
                                const uint64_t ad = umma_smem_desc(ka + off, 16, 1024, SMEM_LAYOUT_SW128);
                                const uint64_t bd = umma_smem_desc(qa + qoff, 16, 1024, SMEM_LAYOUT_SW128);
                                if constexpr (F8)
                                    umma_e4m3(tbase + (uint32_t)(C::S_COL + b * SWB + th * SW), ad, bd, idesc1, kk > 0);
                                else
                                    umma_bf16(tbase + (uint32_t)(C::S_COL + b * SWB), ad, bd, idesc1, sub > 0 || kk > 0);
                            }
                        }
                        if (sub == SUB - 1)
                            umma_commit(&s_full[b]);
                        umma_commit(&k_empty[s]);
                    }
                }
            } else {
                // O accumulates in one TMEM buffer across tiles while the softmax
                // reference maximum stays put.  A buffer is closed (committed to
                // o_full) when the softmax moves the reference (ctl flag of the tile)
                // or when a piece ends; the next tile opens the other buffer afresh.
                // Closes are counted by `u`: use u lives in buffer u & 1.
                const uint32_t idesc2 = F8 ? umma_idesc_e4m3(128, NO, 1, 1) : umma_idesc_bf16(128, NO, 1, 1);
                TileIter itp;
                itp.init(start, prefix, B, units, p.hch);
                int64_t segp = itp.seg0;
                int u = 0;
                bool fresh = true;
                for (int k = 0; k < ntiles && ok; ++k) {
                    const int b = k & 1;
                    if (!bounded_wait(&p_full[b], (uint32_t)((k >> 1) & 1), abort_flag, p)) {
                        ok = false;
                        break;
                    }
                    if (ctl[b] && !fresh) {
                        umma_commit(&o_full[u & 1]);
                        ++u;
                        fresh = true;
                    }
                    ok = !fresh || u < 2 ||
                         bounded_wait(&o_free[u & 1], (uint32_t)(((u - 2) >> 1) & 1), abort_flag, p);
                    if (!ok)
                        break;
                    // Does the piece end with tile k?  (itp runs one tile ahead.)
                    bool piece_ends = true;
                    if (k + 1 < ntiles) {
                        itp.next(prefix, B, p.Hkv, p.hch);
                        piece_ends = itp.seg0 != segp;
                        segp = itp.seg0;
                    }
                    const uint32_t pa = p_a + (uint32_t)(b * L::PBUF);
#pragma unroll
                    for (int sub = 0; sub < SUB && ok; ++sub) {
                        // O^T rows of head-dimension half `sub` (D = 256) in their own columns.
                        const int ks = k * SUB + sub, s = ks % S;
                        ok = bounded_wait(&v_full[s], (uint32_t)((ks / S) & 1), abort_flag, p);
                        if (!ok)
                            break;
                        tc_fence_after_sync();
                        const uint32_t va_off = (uint32_t)(L::V_RING_OFF + s * L::SLOT_BYTES);
                        const uint32_t va = ring_a + va_off;
                        // V^T rows 64..127: the slot's upper half, or the zero block at D = 64.
                        const uint32_t vlbo = HALVES == 2 ? (uint32_t)C::BOX_BYTES : (uint32_t)L::ZERO_OFF - va_off;
                        const uint32_t ocol = tbase + (uint32_t)(OC + (u & 1) * NO * SUB + sub * NO);
#pragma unroll
                        for (int kk = 0; kk < T / KSTEP; ++kk) {
                            if constexpr (F8) {
                                // 32 tokens per instruction: 4 KB of V rows, four 8-token groups of P.
                                umma_e4m3(ocol,
                                          umma_smem_desc(va + (uint32_t)(kk * 4096), C::BOX_BYTES, 1024,
                                                         SMEM_LAYOUT_SW128),
                                          umma_smem_desc(pa + (uint32_t)(4 * kk * P8_LBO), P8_LBO, 128,
                                                         SMEM_LAYOUT_NONE),
                                          idesc2, kk > 0 || !fresh);
                            } else {
                                umma_bf16(ocol,
                                          umma_smem_desc(va + (uint32_t)(kk * 2048), vlbo, 1024, SMEM_LAYOUT_SW128),
                                          umma_smem_desc(pa + (uint32_t)(2 * kk * C::P_LBO), C::P_LBO, 128, SMEM_LAYOUT_NONE),
                                          idesc2, kk > 0 || !fresh);
                            }
                        }
                        umma_commit(&v_empty[s]);
                    }
                    if (!ok)
                        break;
                    fresh = false;
                    umma_commit(&p_free[b]);
                    if (piece_ends) {
                        umma_commit(&o_full[u & 1]);
                        ++u;
                        fresh = true;
                    }
                }
            }
            (void)ok;
            // Nothing of ours may still be running on the tensor cores at exit.
            uint64_t *dr = &drain[warp == 1 ? 0 : 1];
            umma_commit(dr);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(dr, 0) && global_timer_ns() - t0 < WAIT_LIMIT_NS) {
            }
        }
    } else if (start < end) {
        // ------------------------------------------------------ softmax + correction
        const int q4 = warp & 3;                 // TMEM lane quadrant of this warp
        const int ti = q4 * 32 + lane;           // token row (S) and d row (O)
        const int stid = tid - 64;               // 0..127 among the softmax threads
        const uint32_t tlane = tbase + ((uint32_t)(q4 * 32) << 16);
        const float qscale = p.qscale;
        // FP8: score scale per head of the current piece (qscale over its Q row's
        // power-of-two range factor).
        float qs[F8 ? NV : 1];
#pragma unroll
        for (int g = 0; g < (F8 ? NV : 1); ++g)
            qs[g] = qscale;
        auto qsc = [&](int g) -> float {
            if constexpr (F8)
                return qs[g];
            else
                return qscale;
        };
        // FP8: the piece's Q rows as two E4M3 terms in the 128-byte-swizzled K-major
        // layout BMM1 reads, term 1 in rows 0..NP-1 and term 2 in rows NP..2NP-1.
        // Each row is first scaled by the power of two that brings its largest
        // magnitude into [2^7, 2^8); red[13 NP + g] receives the inverse.  Thread
        // stid converts 8 elements of rows stid / 16 and stid / 16 + 8: the 16
        // threads of a row are 16 consecutive lanes.
        auto load_q_e4m3 = [&](unsigned char *qd, const TileIter &ti) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int x = stid + 128 * r;
                const int g = x >> 4, c8 = x & 15;  // row, 8-element chunk of it
                uint4 w = make_uint4(0, 0, 0, 0);
                if (ti.hc * NP + g < p.R)
                    w = __ldg(reinterpret_cast<const uint4 *>(
                        p.q + (out_row(p, ti.b, ti.kvh, ti.hc * NP + g) * D + c8 * 8)));
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                float v[8];
                float mx = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v[2 * j] = __uint_as_float(ww[j] << 16);  // bf16 widening, exact
                    v[2 * j + 1] = __uint_as_float(ww[j] & 0xffff0000u);
                    mx = fmaxf(mx, fmaxf(fabsf(v[2 * j]), fabsf(v[2 * j + 1])));
                }
#pragma unroll
                for (int o = 8; o > 0; o >>= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                int sh = 0;
                if (mx > 0.f)
                    sh = min(max(7 - (((__float_as_int(mx) >> 23) & 0xff) - 127), -100), 100);
                const float up = __int_as_float((127 + sh) << 23), down = __int_as_float((127 - sh) << 23);
                uint32_t t1[2] = {0u, 0u}, t2[2] = {0u, 0u};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t hi, lo;
                    split_e4m3(v[j] * up, hi, lo);
                    t1[j >> 2] |= hi << (8 * (j & 3));
                    t2[j >> 2] |= lo << (8 * (j & 3));
                }
                const int c16 = c8 >> 1, sub = (c8 & 1) * 8, g2 = g + NP;
                *reinterpret_cast<uint2 *>(qd + g * 128 + (((c16 ^ (g & 7)) << 4) + sub)) =
                    make_uint2(t1[0], t1[1]);
                *reinterpret_cast<uint2 *>(qd + g2 * 128 + (((c16 ^ (g2 & 7)) << 4) + sub)) =
                    make_uint2(t2[0], t2[1]);
                if (c8 == 0)
                    red[13 * NP + g] = down;
            }
        };
        // acc holds the closed O buffers, relative to the current reference m_ref
        // (the open TMEM buffer shares that reference).
        float m_ref[NV], l_t[NV], acc[SUB][NV];
        PendingPiece pending[2];  // a run has at most a first and a last partial piece
        int npending = 0;
        bool poisoned = false;
        TileIter it, cur;
        it.init(start, prefix, B, units, p.hch);
        cur = it;
        int64_t piece_first = start;
        int piece = 0, u = 0;
        bool ok = true;

        // Fold closed O buffer use u (scaled by w[g]) into acc and hand it back.
        auto fold = [&](const float (&w)[NV]) {
            const int bc = u & 1;
            float o[SUB][NV];
            if (ok && bounded_wait(&o_full[bc], (uint32_t)((u >> 1) & 1), abort_flag, p)) {
                tc_fence_after_sync();
#pragma unroll
                for (int sub = 0; sub < SUB; ++sub) {
                    float olo[NV];
                    const uint32_t oc = tlane + (uint32_t)(OC + bc * NO * SUB + sub * NO);
                    tmem_load<NV>(oc, o[sub]);
                    tmem_load<NV>(oc + NP, olo);
                    if constexpr (F8) {
                        // P terms 2 and 3 carry x16 and x256.
                        float o3[NV];
                        tmem_load<NV>(oc + 2 * NP, o3);
#pragma unroll
                        for (int g = 0; g < NV; ++g)
                            o[sub][g] = fmaf(fmaf(o3[g], 1.f / 16.f, olo[g]), 1.f / 16.f, o[sub][g]);
                    } else {
#pragma unroll
                        for (int g = 0; g < NV; ++g)
                            o[sub][g] += olo[g];
                    }
                }
                tc_fence_before_sync();
            } else {
                ok = false;
                poisoned = true;
#pragma unroll
                for (int sub = 0; sub < SUB; ++sub)
#pragma unroll
                    for (int g = 0; g < NV; ++g)
                        o[sub][g] = 0.f;
            }
            mbar_arrive(&o_free[bc]);
            ++u;
#pragma unroll
            for (int sub = 0; sub < SUB; ++sub)
#pragma unroll
                for (int g = 0; g < NV; ++g)
                    acc[sub][g] = fmaf(o[sub][g], w[g], acc[sub][g]);
        };

        auto epilogue = [&](int64_t last_excl) {
            float one[NV];
#pragma unroll
            for (int g = 0; g < NV; ++g)
                one[g] = 1.f;
            fold(one);
            // Normaliser per head: sum of every token thread's partial.
            float lv[NV];
#pragma unroll
            for (int g = 0; g < NV; ++g)
                lv[g] = l_t[g];
            const float mine = warp_transpose_reduce<NV, false>(lv, lane);
            float *lred = red + 8 * NP;
            if (lane % LPH == 0)
                lred[q4 * NV + lane / LPH] = mine;
            if (poisoned)
                atomicOr(poison_flag, 1);
            named_barrier_sync(1, 128);
            float lsum[NV];
#pragma unroll
            for (int g = 0; g < NV; ++g)
                lsum[g] = lred[g] + lred[NV + g] + lred[2 * NV + g] + lred[3 * NV + g];
            const bool pois = *reinterpret_cast<volatile int *>(poison_flag) != 0;
            const bool complete = piece_first == cur.seg0 && last_excl == cur.seg0 + cur.nb;
            const int rows = min(NV, p.R - cur.hc * NP);
            const int r0 = cur.hc * NP;
            const int64_t vseg = ((int64_t)cur.b * p.Hkv + cur.kvh) * p.hch + cur.hc;
            float *slot = p.slots + (p.nsplit ? c : 2 * c + (piece_first == start ? 0 : 1)) * (int64_t)SLOT;
            if (complete) {
#pragma unroll
                for (int sub = 0; sub < SUB; ++sub)
#pragma unroll
                    for (int g = 0; g < NV; ++g)
                        if (g < rows && ti + 128 * sub < D)
                            write_result<false>(p, MQ ? out_row(p, cur.b, cur.kvh, r0 + g) : out_row_q1(p, cur.b, cur.kvh, r0 + g),
                                                ti + 128 * sub, D, acc[sub][g], m_ref[g], lsum[g], pois);
            } else {
#pragma unroll
                for (int sub = 0; sub < SUB; ++sub)
#pragma unroll
                    for (int g = 0; g < NV; ++g)
                        if (ti + 128 * sub < D)
                            slot[g * D + ti + 128 * sub] = acc[sub][g];
                if (ti < NV) {
                    float mv = m_ref[0], lvv = lsum[0];
#pragma unroll
                    for (int g = 1; g < NV; ++g)
                        if (g == ti) {
                            mv = m_ref[g];
                            lvv = lsum[g];
                        }
                    slot[NV * D + ti] = mv;
                    slot[NV * D + NV + ti] = pois ? __int_as_float(0x7fc00000) : lvv;
                }
            }
            named_barrier_sync(1, 128);
            if (!complete) {
                if (stid == 0)
                    *poison_flag = 0;
                pending[npending++] =
                    PendingPiece{cur.seg0, piece_first, last_excl, vseg, 0, cur.nb, rows, cur.b, cur.kvh, r0};
            } else if (stid == 0) {
                *poison_flag = 0;
            }
            named_barrier_sync(1, 128);
        };

        // A buffer closed by a moved reference is folded one tile later: its close
        // is committed with the tile's BMM2, which the MMA warp issues only after
        // the next tile's BMM1, and that may wait for the next piece's Q.
        float alpha_pend[NV];
        bool fold_pend = false;
        auto flush_fold = [&]() {
            if (fold_pend)
                fold(alpha_pend);
            fold_pend = false;
        };

        int len_b = -1;
        int64_t req_len = 0;
        uint64_t t_scores = 0;
        int k = 0;
        // One pass past the last tile (i == end) closes the last piece, so that the
        // piece epilogue is written out once.
        for (int64_t i = start;; ++i, ++k) {
            const bool past = i == end;
            if (i > start && !past)
                it.next(prefix, B, p.Hkv, p.hch);
            const bool first_tile = !past && (i == start || it.seg0 != cur.seg0);
            if (first_tile) {
                // Q of the new (request, KV head, head chunk) goes out first: the MMA
                // warp issues this tile's BMM1 before the previous tile's BMM2, and
                // closing the previous piece below waits on that BMM2.  Layout: the
                // 128-byte-swizzled K-major form the tensor cores read (row g,
                // 16-byte chunk cc of a 64-column half at chunk position cc ^ (g & 7)).
                ++piece;
                const int qb = QBUFS == 2 ? (piece - 1) & 1 : 0;
                unsigned char *qd = qbuf + qb * L::QBUF;
                if constexpr (F8) {
                    load_q_e4m3(qd, it);
                } else {
#pragma unroll
                for (int r = 0; r < QH; ++r) {
                    const int x = stid + 128 * r;
                    const int half = x >> 7, g = (x & 127) >> 3, cc = x & 7;
                    uint4 w = make_uint4(0, 0, 0, 0);
                    if (it.hc * NP + g < p.R)
                        w = __ldg(reinterpret_cast<const uint4 *>(
                            p.q + (out_row(p, it.b, it.kvh, it.hc * NP + g) * D + half * 64 + cc * 8)));
                    *reinterpret_cast<uint4 *>(qd + half * NP * 128 + g * 128 + ((cc ^ (g & 7)) << 4)) = w;
                }
                }
                fence_proxy_async_smem();
                mbar_arrive(&q_full[qb]);
                if constexpr (F8) {
                    named_barrier_sync(1, 128);  // the rows' range factors are in red
#pragma unroll
                    for (int g = 0; g < NV; ++g)
                        qs[g] = qscale * red[13 * NP + g];
                }
            }
            if (first_tile || past) {
                if (i > start) {
                    flush_fold();
                    epilogue(i);
                }
                if (past)
                    break;
                cur = it;
                piece_first = i;
                poisoned = false;
#pragma unroll
                for (int g = 0; g < NV; ++g) {
                    m_ref[g] = -INFINITY;
                    l_t[g] = 0.f;
#pragma unroll
                    for (int sub = 0; sub < SUB; ++sub)
                        acc[sub][g] = 0.f;
                }
            }

            const int s = (k * SUB) % S, b = k & 1;  // the tile's (first) V slot
            float sc[TH][NV];
            int n = 0;
            bool have_v = ok;
#pragma unroll
            for (int sub = 0; sub < SUB; ++sub)
                have_v = have_v && bounded_wait(&v_full[(k * SUB + sub) % S],
                                                (uint32_t)(((k * SUB + sub) / S) & 1), abort_flag, p);
            if (have_v && bounded_wait(&s_full[b], (uint32_t)((k >> 1) & 1), abort_flag, p)) {
                n = stage_n[s];
                poisoned |= stage_bad[s] != 0;
                tc_fence_after_sync();
                if constexpr (F8) {
#pragma unroll
                    for (int th = 0; th < TH; ++th) {
                        float s2[NV];
                        tmem_load<NV>(tlane + (uint32_t)(C::S_COL + b * SWB + th * SW), sc[th]);
                        tmem_load<NV>(tlane + (uint32_t)(C::S_COL + b * SWB + th * SW + NP), s2);
#pragma unroll
                        for (int g = 0; g < NV; ++g)
                            sc[th][g] = fmaf(s2[g], 1.f / 16.f, sc[th][g]);  // the second Q term carries x16
                    }
                } else {
                    tmem_load<NV>(tlane + (uint32_t)(C::S_COL + b * SWB), sc[0]);
                }
                tc_fence_before_sync();
                if (k == 0 && stid == 0 && p.timeline)
                    t_scores = global_timer_ns();
            } else {
                ok = false;
                poisoned = true;
            }
            mbar_arrive(&s_free[b]);
            flush_fold();  // before this tile may rescale acc again
            bool valid[TH];
#pragma unroll
            for (int th = 0; th < TH; ++th)
                valid[th] = ti + 128 * th < n;
            // Several query tokens (qlen > 1): query row r is token r / G at position
            // L - qlen + r / G and sees keys up to its own position, so a key `past`
            // places beyond L - qlen is hidden from the rows of tokens before it.
            bool see[TH][NV];
#pragma unroll
            for (int th = 0; th < TH; ++th)
#pragma unroll
                for (int g = 0; g < NV; ++g)
                    see[th][g] = valid[th];
            if (MQ) {
                if (it.b != len_b) {
                    len_b = it.b;
                    int64_t b0, l0;
                    request_range<false>(p, len_b, b0, l0);
                    req_len = l0;
                }
                const int64_t past = (int64_t)it.j * T + ti - (req_len - p.qlen);
                if (past > 0) {  // only the last qlen - 1 keys of a request
#pragma unroll
                    for (int g = 0; g < NV; ++g)
                        see[0][g] = see[0][g] && past <= (it.hc * NP + g) / G;
                }
            }
            // x = scaled score relative to the reference.  While no score of the tile
            // exceeds its reference by more than 2^LAZY, P = 2^x <= 2^LAZY is used as
            // is and nothing is rescaled: one barrier-OR decides that for the CTA.
            float x[TH][NV];
            float xmax = -INFINITY;
#pragma unroll
            for (int th = 0; th < TH; ++th)
#pragma unroll
                for (int g = 0; g < NV; ++g) {
                    x[th][g] = see[th][g] ? fmaf(sc[th][g], qsc(g), -m_ref[g]) : -INFINITY;
                    xmax = fmaxf(xmax, x[th][g]);
                }
            const bool moved = named_barrier_or(1, 128, !(xmax <= C::LAZY));
            float alpha[NV];
            if (moved) {
                // Tile maximum per head over the 128 tokens: warp, then the 4 warps.
                float mx[NV];
#pragma unroll
                for (int g = 0; g < NV; ++g) {
                    mx[g] = see[0][g] ? sc[0][g] * qsc(g) : -INFINITY;
#pragma unroll
                    for (int th = 1; th < TH; ++th)
                        mx[g] = fmaxf(mx[g], see[th][g] ? sc[th][g] * qsc(g) : -INFINITY);
                }
                const float wmax = warp_transpose_reduce<NV, true>(mx, lane);
                float *tred = red + (k & 1) * 4 * NP;
                if (lane % LPH == 0)
                    tred[q4 * NV + lane / LPH] = wmax;
                named_barrier_sync(1, 128);
#pragma unroll
                for (int g = 0; g < NV; ++g) {
                    const float tm = fmaxf(fmaxf(tred[g], tred[NV + g]), fmaxf(tred[2 * NV + g], tred[3 * NV + g]));
                    const float m_new = tm > m_ref[g] + C::LAZY ? tm : m_ref[g];
                    alpha[g] = m_new == m_ref[g] ? 1.f : fast_exp2(m_ref[g] - m_new);
                    m_ref[g] = m_new;
#pragma unroll
                    for (int th = 0; th < TH; ++th)
                        x[th][g] = (see[th][g] && m_new != -INFINITY) ? fmaf(sc[th][g], qsc(g), -m_new) : -INFINITY;
                    l_t[g] *= alpha[g];
#pragma unroll
                    for (int sub = 0; sub < SUB; ++sub)
                        acc[sub][g] *= alpha[g];
                }
            }
            // This P buffer was last read by BMM2 two tiles ago.
            if (k >= 2 && ok && !bounded_wait(&p_free[b], (uint32_t)(((k - 2) >> 1) & 1), abort_flag, p)) {
                ok = false;
                poisoned = true;
            }
            float prh[TH][NV];
#pragma unroll
            for (int th = 0; th < TH; ++th)
#pragma unroll
                for (int g = 0; g < NV; ++g) {
                    prh[th][g] = fast_exp2(x[th][g]);
                    l_t[g] += prh[th][g];
                }
            // P = hi + lo, both bf16, as one N = 32 operand (hi heads in columns
            // 0..NP-1, lo heads in NP..2NP-1) in the no-swizzle MN-major layout:
            // token ti's 8-head groups are 16-byte rows of 8x8 core matrices.
            if constexpr (F8) {
                // P = t1 + t2 / 16 + t3 / 256, all E4M3, as one N = 48 operand (term
                // i of the heads in bytes 0..NP-1 of the token's 16-byte row of core
                // matrix i), no-swizzle MN-major.
#pragma unroll
                for (int th = 0; th < TH; ++th) {
                    const float (&pr)[NV] = prh[th];
                    const int tt = ti + 128 * th;  // the token of this half
                    unsigned char *pd8 = pbuf + b * L::PBUF + (tt >> 3) * P8_LBO + (tt & 7) * 16;
                    uint32_t w1[(NV + 3) / 4], w2[(NV + 3) / 4], w3[(NV + 3) / 4];
#pragma unroll
                    for (int j = 0; j < (NV + 3) / 4; ++j)
                        w1[j] = w2[j] = w3[j] = 0u;
#pragma unroll
                    for (int g = 0; g < NV; ++g) {
                        uint32_t t1, t2, t3;
                        split3_e4m3(pr[g], t1, t2, t3);
                        w1[g >> 2] |= t1 << (8 * (g & 3));
                        w2[g >> 2] |= t2 << (8 * (g & 3));
                        w3[g >> 2] |= t3 << (8 * (g & 3));
                    }
                    if constexpr (NV == 4) {
                        *reinterpret_cast<uint32_t *>(pd8) = w1[0];
                        *reinterpret_cast<uint32_t *>(pd8 + 128) = w2[0];
                        *reinterpret_cast<uint32_t *>(pd8 + 256) = w3[0];
                    } else if constexpr (NV == 8) {
                        *reinterpret_cast<uint2 *>(pd8) = make_uint2(w1[0], w1[1]);
                        *reinterpret_cast<uint2 *>(pd8 + 128) = make_uint2(w2[0], w2[1]);
                        *reinterpret_cast<uint2 *>(pd8 + 256) = make_uint2(w3[0], w3[1]);
                    } else {
                        *reinterpret_cast<uint4 *>(pd8) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
                        *reinterpret_cast<uint4 *>(pd8 + 128) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
                        *reinterpret_cast<uint4 *>(pd8 + 256) = make_uint4(w3[0], w3[1], w3[2], w3[3]);
                    }
                }
            } else {
                const float (&pr)[NV] = prh[0];
                unsigned char *pd = pbuf + b * L::PBUF + (ti >> 3) * C::P_LBO + (ti & 7) * 16;
                constexpr int NW = NV / 2;  // bf16 pairs per term
                uint32_t whi[NW], wlo[NW];
#pragma unroll
                for (int j = 0; j < NW; ++j) {
                    const float a = pr[2 * j], bb = pr[2 * j + 1];
                    __nv_bfloat162 hi = __floats2bfloat162_rn(a, bb);
                    const float2 hf = __bfloat1622float2(hi);
                    __nv_bfloat162 lo = __floats2bfloat162_rn(a - hf.x, bb - hf.y);
                    whi[j] = *reinterpret_cast<uint32_t *>(&hi);
                    wlo[j] = *reinterpret_cast<uint32_t *>(&lo);
                }
                if constexpr (NV == 4) {
                    *reinterpret_cast<uint2 *>(pd) = make_uint2(whi[0], whi[1]);
                    *reinterpret_cast<uint2 *>(pd + (NP / 8) * 128) = make_uint2(wlo[0], wlo[1]);
                } else {
#pragma unroll
                    for (int ng = 0; ng < NV / 8; ++ng) {
                        *reinterpret_cast<uint4 *>(pd + ng * 128) =
                            make_uint4(whi[4 * ng], whi[4 * ng + 1], whi[4 * ng + 2], whi[4 * ng + 3]);
                        *reinterpret_cast<uint4 *>(pd + (NP / 8 + ng) * 128) =
                            make_uint4(wlo[4 * ng], wlo[4 * ng + 1], wlo[4 * ng + 2], wlo[4 * ng + 3]);
                    }
                }
            }
            // Rows past the valid tokens may hold anything (stale tiles, poison):
            // zero this token's V row so that 0-weight rows add exact zeros.
#pragma unroll
            for (int th = 0; th < TH; ++th) {
                if (valid[th])
                    continue;
#pragma unroll
                for (int sub = 0; sub < SUB; ++sub) {
                    unsigned char *vr = ring + L::V_RING_OFF + (size_t)((k * SUB + sub) % S) * L::SLOT_BYTES +
                                        (ti + 128 * th) * 128;
#pragma unroll
                    for (int h = 0; h < HALVES; ++h)
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc)
                            *reinterpret_cast<uint4 *>(vr + h * C::BOX_BYTES + cc * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            // A moved reference closes the open O buffer (unless this tile opens a
            // piece, whose buffer is fresh anyway).
            const bool close = moved && !first_tile;
            if (stid == 0)
                ctl[b] = close ? 1 : 0;
            fence_proxy_async_smem();
            mbar_arrive(&p_full[b]);
            if (close) {
#pragma unroll
                for (int g = 0; g < NV; ++g)
                    alpha_pend[g] = alpha[g];
                fold_pend = true;
            }
        }
        const uint64_t t_streamed = p.timeline ? global_timer_ns() : 0;
        // Split segments: publish every partial piece of this run, then merge this
        // CTA's share of each (all owners are resident: cooperative launch).  Every
        // tile has been consumed, so the P buffers and the rings are scratch.
        if (p.nsplit)
            npending = 0;  // fixed split: merge_split_kernel combines the chunks
        for (int x = 0; x < npending; ++x)
            publish_piece(p, pending[x].vseg, stid, 1, 128);
        for (int x = 0; x < npending; ++x) {
            const PendingPiece &pp = pending[x];
            merge_segment_gather<NV, D, 128, MQ>(p, c, pp.seg0, pp.nb, pp.first, pp.vseg, W, P, pp.rows,
                                             pp.b, pp.kvh, pp.r0, reinterpret_cast<int *>(pbuf),
                                             reinterpret_cast<float *>(ring), misc + 20, stid, 1,
                                             abort_flag);
        }
        if (p.timeline && stid == 0) {
            unsigned long long *rec = p.timeline + TL_COLS * c;
            rec[5] = t_scores;
            rec[6] = t_streamed;
            rec[7] = global_timer_ns();
        }
    }

    // Timeline record and tensor-memory release.
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tbase, TMEM_COLS);
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

// Second kernel of the fixed-split comparator: one thread per output element
// (segment j, head g, column d) merges the segment's chunks (slot c of chunk CTA
// c) in chunk order; a segment with fewer than two non-empty chunks was written by
// the decode kernel itself.  (Attention co-design for long-context inference,
// section "FlashAttention and GEMM shapes": FlashDecoding's split-KV reduction.)
template <int NV, int DH = 128>
__global__ void __launch_bounds__(128)
    merge_split_kernel(const Params p)
{
    constexpr int D = DH, NP = TcCfg::NP, T = TcCfg::T;
    constexpr int SLOT = slot_floats(NV, D);
    constexpr int U = 8;  // chunks per batch of independent loads
    const int64_t units = (int64_t)p.Hkv * p.hch;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t j = gid / (NV * D);
    if (j >= (int64_t)p.B * units)
        return;
    const int e = (int)(gid - j * (NV * D)), g = e / D, d = e - g * D;
    const int b = (int)(j / units);
    const int u = (int)(j - (int64_t)b * units), kvh = u / p.hch, hc = u - kvh * p.hch;
    if (g >= min(NV, p.R - hc * NP))
        return;
    int64_t begin, len;
    request_range<false>(p, b, begin, len);
    const int64_t nb = (len + T - 1) / T;
    const int ns = p.nsplit;
    if ((nb < ns ? nb : (int64_t)ns) < 2)
        return;  // at most one non-empty chunk: written by the decode kernel
    const float *base = p.slots + j * ns * SLOT;
    auto nonempty = [&](int i) { return (int64_t)(i + 1) * nb / ns > (int64_t)i * nb / ns; };
    float mx = -INFINITY;
    for (int i0 = 0; i0 < ns; i0 += U) {
        float mv[U];
#pragma unroll
        for (int q = 0; q < U; ++q)
            mv[q] = (i0 + q < ns && nonempty(i0 + q)) ? __ldcg(base + (i0 + q) * SLOT + NV * D + g)
                                                       : -INFINITY;
#pragma unroll
        for (int q = 0; q < U; ++q)
            mx = fmaxf(mx, mv[q]);
    }
    float a = 0.f, ls = 0.f;
    for (int i0 = 0; i0 < ns; i0 += U) {
        float mv[U], lv[U], av[U];
#pragma unroll
        for (int q = 0; q < U; ++q) {
            const bool have = i0 + q < ns && nonempty(i0 + q);
            const float *sl = base + (i0 + q) * SLOT;
            mv[q] = have ? __ldcg(sl + NV * D + g) : -INFINITY;
            lv[q] = have ? __ldcg(sl + NV * D + NV + g) : 0.f;
            av[q] = have ? __ldcg(sl + g * D + d) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < U; ++q) {
            const float w = mv[q] == -INFINITY ? 0.f : fast_exp2(mv[q] - mx);
            a = fmaf(w, av[q], a);
            ls = fmaf(w, lv[q], ls);
        }
    }
    write_result<false>(p, out_row(p, b, kvh, hc * NP + g), d, D, a, mx, ls, ls != ls);
}

}  // namespace gqa
