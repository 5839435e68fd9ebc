// gather_merge.cuh -- exact merge of a split segment by all of its owner CTAs at
// once, for kernels launched cooperatively (every CTA of the grid resident).
//
// The owners of a segment (the CTAs whose runs cut it) each publish their partial
// piece (acc, m, l in a workspace slot) with one release increment of the
// segment's counter.  Then every owner waits until all pieces are published and
// merges its own share of the segment's outputs: owner k of no takes elements
// [k E / no, (k+1) E / no) of the E = rows x D outputs, gathers that slice of
// every piece (and the pieces' m and l for the heads the slice touches) into
// shared memory in one round of loads, rescales to the common maximum and adds
// (LeanAttention decode tiles digest, section "Exact softmax that merges piece by
// piece").  Pieces are added in CTA order, so the result does not depend on
// timing.  Compared with a last-arriver merge chain this puts one wait and one
// gather after the slowest owner instead of two ticket round trips and two
// serial merges.
//
// counters[vseg]: bits 0..15 count published pieces, bits 16..31 count finished
// slices; the owner that finishes the last slice resets the word to zero.  Waits
// are bounded (Params::wait_ns): on expiry the kernel's status gets DEV_TIMEOUT and
// the slice is written as NaN.
#pragma once

#include "schedule.cuh"

namespace gqa {

__device__ __forceinline__ void red_release_add(int *addr, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire(const int *addr)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
    return v;
}

// All NT threads, after this CTA wrote its piece of segment vseg to its slot.
__device__ __forceinline__ void publish_piece(const Params &p, int64_t vseg, int t, int bar_id,
                                              int nt)
{
    named_barrier_sync(bar_id, nt);  // every thread's slot writes precede the release
    if (t == 0)
        red_release_add(&p.counters[vseg], 1);
}

// All NT threads.  Segment [seg0, seg0 + nb) of KV unit vseg; this CTA (c) owns
// the piece starting at tile piece_first.  NV rows per slot, `rows` of them real:
// query rows r0 .. r0 + rows - 1 of (request b, KV head kvh), written to
// out_row(p, b, kvh, r).  list: >= no ints of shared memory; buf: shared floats
// for the gathered slices (see the bound in the kernel).
template <int NV, int D, int NT, bool MQ>
__device__ __forceinline__ void merge_segment_gather(const Params &p, int64_t c, int64_t seg0,
                                                     int nb, int64_t piece_first, int64_t vseg,
                                                     int64_t W, int64_t P, int rows, int b, int kvh,
                                                     int r0,
                                                     int *list, float *buf, int *flag, int t,
                                                     int bar_id, volatile int *abort_flag)
{
    constexpr int SF = slot_floats(NV, D);
    // Owners: with W >= P every run holds a tile, so they are the consecutive CTAs
    // c0 .. c1; with W < P every tile has an owner of its own.
    const bool dense = W >= P;
    const int64_t c0 = tile_owner(seg0, W, P);
    const int no = dense ? (int)(tile_owner(seg0 + nb - 1, W, P) - c0 + 1) : nb;
    const int k = dense ? (int)(c - c0) : (int)(piece_first - seg0);
    for (int i = t; i < no; i += NT) {
        const int64_t cc = dense ? c0 + i : tile_owner(seg0 + i, W, P);
        list[i] = (int)(2 * cc + (run_start(cc, W, P) < seg0 ? 1 : 0));
    }
    if (t == 0) {
        bool ok = true;
        const uint64_t t0 = global_timer_ns();
        while ((ld_acquire(&p.counters[vseg]) & 0xFFFF) < no) {
            if (*abort_flag || global_timer_ns() - t0 > p.wait_ns) {
                ok = false;
                break;
            }
        }
        if (!ok && !*abort_flag) {
            atomicOr(p.status, DEV_TIMEOUT);
            *abort_flag = 1;
        }
        flag[0] = ok ? 1 : 0;
    }
    named_barrier_sync(bar_id, NT);
    const bool ok = *reinterpret_cast<volatile int *>(flag) != 0;

    // Slices start on 4-element boundaries, so every piece's slice is whole float4s.
    const int E4 = rows * D / 4;
    const int e0 = 4 * (int)((int64_t)k * E4 / no), e1 = 4 * (int)((int64_t)(k + 1) * E4 / no);
    const int Ec = e1 - e0;
    if (Ec > 0) {
        const int g0 = e0 / D, NH = (e1 - 1) / D - g0 + 1;
        float *acc_s = buf;            // [no][Ec]
        float *m_s = acc_s + no * Ec;  // [no][NH]
        float *l_s = m_s + no * NH;    // [no][NH]
        float *w_s = l_s + no * NH;    // [no][NH]
        float *hm_s = w_s + no * NH;   // [NH] common maximum
        float *hl_s = hm_s + NH;       // [NH] merged normaliser
        if (ok) {
            // Per round, up to UA float4 of slices and UH (m, l) pairs per thread are
            // in flight together before any is stored: one round trip to L2 for
            // slices of up to UA x NT float4 in all (every shape here).
            constexpr int UA = 8, UH = 2;
            const int Ec4 = Ec / 4, na4 = no * Ec4, nh = no * NH;
            for (int r0 = 0; r0 * NT * UA < na4 || r0 * NT * UH < nh; ++r0) {
                float4 av[UA];
                float mv[UH], lv[UH];
#pragma unroll
                for (int q = 0; q < UH; ++q) {
                    const int x = (r0 * UH + q) * NT + t;
                    const int i = x < nh ? x / NH : 0, g = g0 + (x - i * NH);
                    const float *sl = p.slots + (int64_t)list[i] * SF;
                    mv[q] = x < nh ? __ldcg(sl + NV * D + g) : 0.f;
                    lv[q] = x < nh ? __ldcg(sl + NV * D + NV + g) : 0.f;
                }
#pragma unroll
                for (int q = 0; q < UA; ++q) {
                    const int x = (r0 * UA + q) * NT + t;
                    const int i = x < na4 ? x / Ec4 : 0;
                    av[q] = x < na4 ? __ldcg(reinterpret_cast<const float4 *>(
                                          p.slots + (int64_t)list[i] * SF + e0) + (x - i * Ec4))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int q = 0; q < UH; ++q) {
                    const int x = (r0 * UH + q) * NT + t;
                    if (x < nh) {
                        m_s[x] = mv[q];
                        l_s[x] = lv[q];
                    }
                }
#pragma unroll
                for (int q = 0; q < UA; ++q) {
                    const int x = (r0 * UA + q) * NT + t;
                    if (x < na4)
                        reinterpret_cast<float4 *>(acc_s)[x] = av[q];
                }
            }
        }
        named_barrier_sync(bar_id, NT);
        if (ok) {
            // Per head: common maximum, piece weights, merged normaliser (one warp each).
            const int lane = t & 31;
            for (int h = t >> 5; h < NH; h += NT / 32) {
                float mx = -INFINITY;
                for (int i = lane; i < no; i += 32)
                    mx = fmaxf(mx, m_s[i * NH + h]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                float ls = 0.f;
                for (int i = lane; i < no; i += 32) {
                    const float mi = m_s[i * NH + h];
                    const float w = mi == -INFINITY ? 0.f : fast_exp2(mi - mx);
                    w_s[i * NH + h] = w;
                    ls = fmaf(w, l_s[i * NH + h], ls);
                }
                // Sum in a fixed lane order, so the result does not depend on timing.
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    ls += __shfl_xor_sync(0xffffffffu, ls, o);
                if (lane == 0) {
                    hm_s[h] = mx;
                    hl_s[h] = ls;
                }
            }
        }
        named_barrier_sync(bar_id, NT);
        // TPE adjacent threads share an element (few elements, many pieces), each
        // summing every TPE-th piece; a fixed shuffle tree combines them.
        const int TPE = Ec <= NT / 4 ? 4 : (Ec <= NT / 2 ? 2 : 1);
        const int per = NT / TPE, sub = t % TPE;
        for (int x0 = 0; x0 < Ec; x0 += per) {
            const int x = x0 + t / TPE;
            const int e = e0 + x, g = e / D, h = g - g0;
            float a = 0.f;
            if (ok && x < Ec)
                for (int i = sub; i < no; i += TPE)
                    a = fmaf(w_s[i * NH + h], acc_s[i * Ec + x], a);
            for (int o = 1; o < TPE; o <<= 1)
                a += __shfl_xor_sync(0xffffffffu, a, o);
            if (sub != 0 || x >= Ec)
                continue;
            if (!ok) {
                write_result<false>(p, MQ ? out_row(p, b, kvh, r0 + g) : out_row_q1(p, b, kvh, r0 + g), e - g * D, D, 0.f, 0.f, 0.f, true);
                continue;
            }
            const float ls = hl_s[h];
            write_result<false>(p, MQ ? out_row(p, b, kvh, r0 + g) : out_row_q1(p, b, kvh, r0 + g), e - g * D, D, a, hm_s[h], ls, ls != ls);
        }
    }
    named_barrier_sync(bar_id, NT);  // list and buf are reused by the next segment
    if (t == 0 && ok) {
        const int old = atomicAdd(&p.counters[vseg], 1 << 16);
        if ((old >> 16) == no - 1)
            atomicExch(&p.counters[vseg], 0);
    }
}

}  // namespace gqa
