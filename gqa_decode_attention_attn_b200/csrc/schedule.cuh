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

// Upper bound on any single in-kernel wait; a healthy wait lasts microseconds.
constexpr uint64_t WAIT_LIMIT_NS = 1500000000ull;

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
    float *slots;                 // 2 partial states per CTA
    int B, Hq, Hkv, G, block_size, max_blocks, num_blocks;
    int hch;                      // head chunks per KV head
    int64_t capacity;             // tokens a request can hold
    uint32_t bs_magic;            // token -> page division by block_size (see page_of)
    int bs_shift;
    float qscale;                 // scale * log2(e): scores are kept in log2 units
    unsigned long long *timeline; // optional [grid][4]: start ns, end ns, SM id, tiles
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

// Walks the global tile order one tile at a time.  prefix[b] = sum of n_b'
// (b' < b) lives in shared memory; units = Hkv * hch segments per request.  Only
// init() divides; next() is increments and compares.
struct TileIter {
    int b, kvh, hc;
    int j;         // tile index inside the segment
    int nb;        // tiles in the segment
    int64_t seg0;  // global index of the segment's first tile

    __device__ __forceinline__ void init(int64_t i, const int *prefix, int B, int64_t units,
                                         int hch)
    {
        int lo = 0, hi = B;  // units*prefix[lo] <= i < units*prefix[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (units * prefix[mid] <= i)
                lo = mid;
            else
                hi = mid;
        }
        b = lo;
        nb = prefix[lo + 1] - prefix[lo];
        const int64_t local = i - units * prefix[lo];
        const int64_t vs = local / nb;
        j = (int)(local - vs * nb);
        kvh = (int)(vs / hch);
        hc = (int)(vs - (int64_t)kvh * hch);
        seg0 = units * prefix[lo] + vs * nb;
    }

    // Advance to the next tile; the caller guarantees one exists.
    __device__ __forceinline__ void next(const int *prefix, int B, int Hkv, int hch)
    {
        if (++j < nb)
            return;
        j = 0;
        seg0 += nb;
        if (++hc < hch)
            return;
        hc = 0;
        if (++kvh < Hkv)
            return;
        kvh = 0;
        do {
            ++b;
        } while (b < B - 1 && prefix[b + 1] == prefix[b]);
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
    return c * W / P;
}
__device__ __forceinline__ int64_t tile_owner(int64_t i, int64_t W, int64_t P)
{
    return ((i + 1) * P - 1) / W;
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
    bool ok = b0 >= 0 && b1 >= b0 && b1 <= p.capacity;
    begin = ok ? b0 : 0;
    len = ok ? b1 - b0 : 0;
    return ok;
}

// Bounded wait on an mbarrier phase.  On timeout: status bit, CTA abort flag.
__device__ __forceinline__ bool bounded_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             unsigned *status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    if (*abort_flag)
        return false;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag)
            return false;
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) {
            atomicOr(status, DEV_TIMEOUT);
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
        float o = poisoned ? __int_as_float(0x7fc00000) : (ls > 0.f ? a / ls : 0.f);
        __nv_bfloat16 h = __float2bfloat16_rn(o);
        p.out[row * D + d] = *reinterpret_cast<uint16_t *>(&h);
    }
}

}  // namespace gqa
