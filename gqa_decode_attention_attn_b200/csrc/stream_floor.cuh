// stream_floor.cuh -- the measurement reference for the decode kernels: K and V
// bytes pulled through the same 2-D TMA boxes (two 64-column halves of 128-byte
// swizzled rows, 128-row tiles, L2 evict-first) into the same three-slot rings of
// 32 KB, with no attention arithmetic: a slot is handed back as soon as its tile
// has landed.  CTA c of P takes tiles [cW/P, (c+1)W/P) of the W tiles, as the
// stream-K decode schedule does.
//
// A decode step reads its K and V once from HBM and is bound by that read
// (Attention co-design for long-context inference, section "Difference between
// prefill and decode", Equation 1 and Figure 2: decode sits below the roofline
// ridge).  Timed like a decode step over the same number of bytes, this kernel
// gives the floor that streaming alone reaches under that timing (launch, first-byte
// latency, loaded-memory throughput); what a decode kernel takes beyond it is what
// its attention pipeline adds.  Every wait is bounded: on expiry the status word
// gets DEV_TIMEOUT and the CTA stops issuing.
#pragma once

#include "schedule.cuh"
#include "tc.cuh"

namespace gqa {

struct FloorCfg {
    static constexpr int T = 128;                  // rows per tile
    static constexpr int STAGES = 3;               // slots per ring
    static constexpr int BOX_BYTES = T * 128;      // one 64-column half of a tile
    static constexpr int SLOT_BYTES = 2 * BOX_BYTES;
    static constexpr int THREADS = 96;             // K loads, V loads, release
    static constexpr size_t BAR_OFF = (size_t)2 * STAGES * SLOT_BYTES;
    static constexpr size_t SMEM = BAR_OFF + 4 * STAGES * 8 + 1024;  // +1024: re-alignment
};

__device__ __forceinline__ bool floor_wait(uint64_t *bar, uint32_t parity, unsigned *status,
                                           uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > limit_ns) {
            atomicOr(status, DEV_TIMEOUT);
            return false;
        }
    return true;
}

__global__ void __launch_bounds__(FloorCfg::THREADS, 1)
    stream_floor_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                        int64_t W, unsigned *status, uint64_t limit_ns)
{
    using C = FloorCfg;
    constexpr int S = C::STAGES;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *k_full = bars, *k_empty = bars + S, *v_full = bars + 2 * S, *v_empty = bars + 3 * S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();
    const int64_t P = gridDim.x, c = blockIdx.x;
    const int64_t t0 = run_start(c, W, P);
    const int n = (int)(run_start(c + 1, W, P) - t0);
    if (warp < 2 && lane == 0) {
        const bool is_k = warp == 0;
        const CUtensorMap *map = is_k ? &tmk : &tmv;
        uint64_t *full = is_k ? k_full : v_full, *emptyb = is_k ? k_empty : v_empty;
        unsigned char *base = smem + (is_k ? 0 : (size_t)S * C::SLOT_BYTES);
        const uint64_t pol = l2_evict_first_policy();
        int k = 0;
        for (; k < n; ++k) {
            const int s = k % S;
            if (k >= S && !floor_wait(&emptyb[s], (uint32_t)(((k / S) & 1) ^ 1), status, limit_ns))
                break;
            mbar_arrive_expect_tx(&full[s], (uint32_t)C::SLOT_BYTES);
            const int row = (int)((t0 + k) * C::T);
            tma_load_2d(base + (size_t)s * C::SLOT_BYTES, map, 0, row, &full[s], pol);
            tma_load_2d(base + (size_t)s * C::SLOT_BYTES + C::BOX_BYTES, map, 64, row, &full[s], pol);
        }
        // No copy of ours may still be landing at exit.
        for (int kk = k > S ? k - S : 0; kk < k; ++kk)
            floor_wait(&full[kk % S], (uint32_t)((kk / S) & 1), status, limit_ns);
    } else if (warp == 2 && lane == 0) {
        for (int k = 0; k < n; ++k) {
            const int s = k % S;
            const uint32_t ph = (uint32_t)((k / S) & 1);
            if (!floor_wait(&k_full[s], ph, status, limit_ns) || !floor_wait(&v_full[s], ph, status, limit_ns))
                break;
            mbar_arrive(&k_empty[s]);
            mbar_arrive(&v_empty[s]);
        }
    }
    __syncthreads();
}

}  // namespace gqa
