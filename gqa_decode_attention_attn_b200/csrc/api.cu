// api.cu -- the C ABI declared in include/gqa_decode.h: argument checks,
// per-device launch geometry, workspace carving and kernel dispatch.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <queue>
#include <vector>
#include <algorithm>
#include <atomic>

#include "decode_simt.cuh"
#include "decode_tc.cuh"
#include "decode_tc_wide.cuh"
#include "gqa_decode.h"
#include "merge_states.cuh"
#include "stream_floor.cuh"

namespace gqa {
namespace {

constexpr int MAX_DEVICES = 64;
constexpr size_t STATUS_BYTES = 256;
constexpr float LOG2E = 1.4426950408889634f;

// Smallest group (query heads per KV head) that runs on the tensor-core kernel.
constexpr int TC_MIN_G = 4;

// Schedule selector cost model (gqa_select_schedule, gqa_decode_auto), fitted to
// this library's tensor-core kernel on B200: a CTA streams K+V at
// min(SCHED_SM_GBS, SCHED_HBM_GBS / active CTAs) -- one SM alone is limited by
// its own copies in flight, many share the HBM -- after a start-up of
// SCHED_CTA_US (prologue and the first tile's trip from HBM); a split segment
// adds the merge tail SCHED_MERGE_US to stream-K and a second launch plus merge
// SCHED_SPLIT_MERGE_US to fixed split.
constexpr double SCHED_SM_GBS = 79.0;
constexpr double SCHED_HBM_GBS = 6300.0;
constexpr double SCHED_CTA_US = 3.0;
constexpr double SCHED_MERGE_US = 3.0;
constexpr double SCHED_SPLIT_MERGE_US = 5.0;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Limit of each in-kernel wait for progress, for launches from now on
// (gqa_set_wait_limit).
std::atomic<unsigned long long> g_wait_ns{WAIT_LIMIT_NS};

// Query heads per chunk for the CUDA-core kernel: the next power of two >= G,
// capped at 8 (larger groups run as several chunks).
int head_chunk(int G)
{
    int gc = 1;
    while (gc < G && gc < 8)
        gc <<= 1;
    return gc;
}

using KernelFn = void (*)(Params);

template <int D, int GC, bool ST, bool F8>
KernelFn simt_fn()
{
    return gqa_decode_simt_kernel<D, GC, ST, F8>;
}

struct Variant {
    KernelFn fn;
    int threads;
    size_t smem_max;                  // shared memory at the largest batch
    size_t (*smem)(int B);
    int slot_floats;
    int tile_tokens;                  // tokens per LeanTile
    int stages;                       // ring stages
};

template <int D, int GC, bool ST, bool F8>
Variant make_variant()
{
    using C = SimtCfg<D, GC, F8>;
    return Variant{simt_fn<D, GC, ST, F8>(), C::THREADS, C::smem_bytes(GQA_MAX_BATCH), &C::smem_bytes,
                   C::SLOT_FLOATS, C::T, C::STAGES};
}

template <bool ST, bool F8>
bool pick_gc(int D, int GC, Variant &v)
{
#define GQA_CASE(DD, GG)                       \
    if (D == DD && GC == GG) {                 \
        v = make_variant<DD, GG, ST, F8>();    \
        return true;                           \
    }
    GQA_CASE(64, 1) GQA_CASE(64, 2) GQA_CASE(64, 4) GQA_CASE(64, 8)
    GQA_CASE(128, 1) GQA_CASE(128, 2) GQA_CASE(128, 4) GQA_CASE(128, 8)
    GQA_CASE(256, 1) GQA_CASE(256, 2) GQA_CASE(256, 4) GQA_CASE(256, 8)
#undef GQA_CASE
    return false;
}

bool pick_variant(int D, int G, bool states, Variant &v, bool fp8 = false)
{
    const int gc = head_chunk(G);
    if (fp8)
        return !states && pick_gc<false, true>(D, gc, v);
    return states ? pick_gc<true, false>(D, gc, v) : pick_gc<false, false>(D, gc, v);
}

// Per-device cache: SM count and, per kernel, resident CTAs per SM.
struct DeviceGeom {
    int sms = 0;
    bool ready = false;
};
std::mutex g_mu;
DeviceGeom g_dev[MAX_DEVICES];
struct FnGeom {
    const void *fn;
    int device;
    int ctas_per_sm;
};
FnGeom g_fn[256];
int g_nfn = 0;

int current_device(int &dev)
{
    return cudaGetDevice(&dev) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

// Persistent grid for a kernel on a device: SMs x resident CTAs per SM.
int persistent_ctas_fn(const void *fn, int threads, size_t smem_max, int dev, int &ctas)
{
    std::lock_guard<std::mutex> lock(g_mu);
    if (dev < 0 || dev >= MAX_DEVICES)
        return GQA_ERR_UNSUPPORTED;
    if (!g_dev[dev].ready) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return GQA_ERR_CUDA;
        g_dev[dev].sms = sms;
        g_dev[dev].ready = true;
    }
    for (int i = 0; i < g_nfn; ++i) {
        if (g_fn[i].fn == fn && g_fn[i].device == dev) {
            ctas = g_dev[dev].sms * g_fn[i].ctas_per_sm;
            if (ctas > 512)
                ctas = 512;
            return GQA_OK;
        }
    }
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess)
        return GQA_ERR_CUDA;
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess)
        return GQA_ERR_CUDA;
    int per_sm = 0;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_max);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem_max);
    if (prev != dev)
        cudaSetDevice(prev);
    if (e != cudaSuccess || per_sm < 1)
        return GQA_ERR_CUDA;
    if (g_nfn < 256)
        g_fn[g_nfn++] = FnGeom{fn, dev, per_sm};
    ctas = g_dev[dev].sms * per_sm;
    if (ctas > 512)  // merge scratch is sized for at most 512 persistent CTAs
        ctas = 512;
    return GQA_OK;
}

int persistent_ctas(const Variant &v, int dev, int &ctas)
{
    return persistent_ctas_fn(reinterpret_cast<const void *>(v.fn), v.threads, v.smem_max, dev,
                              ctas);
}

// Tensor-core kernel for G query heads per KV head: the softmax carries 4, 8 or
// 16 heads (the smallest that holds G, capped at the MMA width 16).
using TcKernelFn = void (*)(Params, CUtensorMap, CUtensorMap, int);
template <bool MQ, int DH>
TcKernelFn tc_kernel_nv(int G)
{
    if (G <= 4)
        return gqa_decode_tc_kernel<4, MQ, DH>;
    if (G <= 8)
        return gqa_decode_tc_kernel<8, MQ, DH>;
    return gqa_decode_tc_kernel<16, MQ, DH>;
}

TcKernelFn tc_kernel_for(int G, bool mq = false, int D = 128, bool fp8 = false)
{
    if (fp8) {  // FP8 E4M3 cache: D = 128, one query token
        if (G <= 4)
            return gqa_decode_tc_kernel<4, false, 128, true>;
        if (G <= 8)
            return gqa_decode_tc_kernel<8, false, 128, true>;
        return gqa_decode_tc_kernel<16, false, 128, true>;
    }
    if (D == 64)
        return mq ? tc_kernel_nv<true, 64>(G) : tc_kernel_nv<false, 64>(G);
    if (D == 256)  // one query token (the plan keeps several on the CUDA-core kernel's check)
        return tc_kernel_nv<false, 256>(G);
    return mq ? tc_kernel_nv<true, 128>(G) : tc_kernel_nv<false, 128>(G);
}

using MergeFn = void (*)(Params);
template <int DH>
MergeFn tc_merge_nv(int G)
{
    if (G <= 4)
        return merge_split_kernel<4, DH>;
    if (G <= 8)
        return merge_split_kernel<8, DH>;
    return merge_split_kernel<16, DH>;
}

MergeFn tc_merge_for(int G, int D = 128)
{
    return D == 64 ? tc_merge_nv<64>(G) : D == 256 ? tc_merge_nv<256>(G) : tc_merge_nv<128>(G);
}

size_t tc_smem_bytes(int D, int B, bool fp8 = false)
{
    if (fp8)
        return TcGeom<128, true>::smem_bytes(B);
    return D == 64 ? TcGeom<64>::smem_bytes(B) : D == 256 ? TcGeom<256>::smem_bytes(B) : TcGeom<128>::smem_bytes(B);
}

// Floats of one partial-state slot of the 16-head tensor-core kernel at head dimension D.
int tc_slot_floats(int D)
{
    return D == 256 ? slot_floats(TcCfg::NP, 256) : TcCfg::SLOT_FLOATS;
}

int tc_ctas(int G, int dev, int &ctas, bool mq = false, int D = 128, bool fp8 = false)
{
    return persistent_ctas_fn(reinterpret_cast<const void *>(tc_kernel_for(G, mq, D, fp8)),
                              TcCfg::THREADS, tc_smem_bytes(D, TcCfg::MAX_BATCH, fp8), dev, ctas);
}

// The wide tensor-core kernel (64 heads per pass) takes bf16 caches at D = 128
// with one query token and more than 16 query heads per KV head; the fixed split
// into several chunks (merge_split_kernel) stays on the 16-head kernel.
bool tc_wide(int R, int D, bool mq, bool fp8, int nsplit)
{
    return !mq && !fp8 && D == 128 && R > TcCfg::NP && nsplit <= 1;
}

int tc_wide_ctas(int dev, int &ctas)
{
    return persistent_ctas_fn(reinterpret_cast<const void *>(gqa_decode_tc_wide_kernel), TcWide::THREADS,
                              TcWide::smem_bytes(TcCfg::MAX_BATCH), dev, ctas);
}

// Head dimensions the tensor-core kernel is built for (256: one query token, bf16).
bool tc_head_dim(int D)
{
    return D == 64 || D == 128 || D == 256;
}

// ---- tensor-core path: applicability and tensor maps -------------------------

// Tokens per TMA box along the cache rows: one box per page, 128 for big pages.
int tc_box_rows(bool paged, int block_size)
{
    if (!paged)
        return 128;
    if (block_size >= 128)
        return block_size % 128 == 0 ? 128 : 0;
    return (block_size >= 8 && 128 % block_size == 0) ? block_size : 0;
}

// R = query rows per KV head (query tokens x G).
bool tc_applicable(bool states, int B, int Hkv, int D, int block_size, bool paged,
                   int num_blocks, int R)
{
    if (states || !tc_head_dim(D) || R < TC_MIN_G || B > TcCfg::MAX_BATCH)
        return false;
    if (tc_box_rows(paged, block_size) == 0)
        return false;
    const int64_t blocks = paged ? num_blocks : B;
    const int64_t rows = blocks * Hkv * (int64_t)block_size;
    return rows > 0 && rows < (int64_t(1) << 31);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2-D view of a cache as [rows, D] bf16 (or FP8 bytes); boxes of 128 bytes (64
// bf16 or 128 FP8 columns) x box_rows rows, 128-byte swizzle (the layout the
// tensor cores read), zero fill out of range.
bool encode_kv_map(CUtensorMap *map, const void *base, int64_t rows, int box_rows, int D,
                   bool fp8 = false)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const int eb = fp8 ? 1 : 2;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * eb};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / eb), (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct WorkspaceLayout {
    size_t counters_off, gcounters_off, slots_off, total;
};

// Fixed layout: [status | ticket counters for the largest shape | partial-state
// slots].  The counters never move, so whatever shape a call has, each counter it
// touches is either still zero from allocation or was reset by the call that last
// used it; slots of one call can never alias counters of another.
constexpr size_t COUNTERS_BYTES = sizeof(int) * (size_t)GQA_MAX_BATCH * GQA_MAX_QHEADS;
constexpr size_t GCOUNTERS_BYTES = sizeof(int) * 2 * 512;  // one per slot of <= 512 CTAs

WorkspaceLayout layout_for(int ctas, int slot_floats)
{
    WorkspaceLayout w;
    w.counters_off = STATUS_BYTES;
    w.gcounters_off = w.counters_off + COUNTERS_BYTES;
    w.slots_off = w.gcounters_off + GCOUNTERS_BYTES;
    w.total = align_up(w.slots_off + sizeof(float) * 2 * (size_t)ctas * slot_floats, 256);
    return w;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_shape(int B, int Hq, int Hkv, int D, int block_size, const int32_t *block_table,
                int max_blocks, int num_blocks, float scale)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || block_size <= 0 || Hq % Hkv != 0)
        return GQA_ERR_INVALID_ARG;
    if (!std::isfinite(scale))
        return GQA_ERR_INVALID_ARG;
    if (block_table && (max_blocks <= 0 || num_blocks < 0))
        return GQA_ERR_INVALID_ARG;
    if (D != 64 && D != 128 && D != 256)
        return GQA_ERR_UNSUPPORTED;
    if (B > GQA_MAX_BATCH || Hq > GQA_MAX_QHEADS)
        return GQA_ERR_UNSUPPORTED;
    return GQA_OK;
}

// Everything a call's launch depends on, decided on the host from the shape
// alone: which kernel, how many query heads one pass carries, the grid, shared
// memory and the workspace layout.  run_decode launches from it and
// gqa_decode_plan reports it, so the two cannot disagree.
struct Plan {
    bool use_tc = false;   // tensor-core kernel (else the CUDA-core kernel)
    bool mq = false;       // several query tokens per request
    bool fp8 = false;
    bool wide = false;     // the 64-heads-per-pass tensor-core kernel
    Variant v{};           // CUDA-core kernel variant
    int G = 0, R = 0;      // query heads per KV head; query rows per KV head
    int nv = 0;            // heads one pass carries (tensor cores: 4, 8, 16, 64; CUDA cores: GC)
    int hch = 0;           // passes (head chunks) per KV head
    int nsplit = 0;        // 0: stream-K; n > 0: fixed split into n chunks
    int ctas = 0;          // persistent grid; -1 when no device was given
    int64_t items = 0;     // fixed split: CTAs of the decode kernel
    int64_t grid = 0;      // CTAs of the decode kernel
    int threads = 0;
    int tile_tokens = 0;
    int stages = 0;
    size_t smem = 0;       // dynamic shared memory per CTA
    int box_rows = 0;      // tensor cores: tokens per TMA box
    WorkspaceLayout w{};
};

// dev < 0: no device query (the grid and the workspace are left at -1 / 0).
int make_plan(bool states, int B, int Hq, int Hkv, int D, int block_size, bool paged,
              int num_blocks, int qlen, bool fp8, int nsplit, int dev, Plan &pl)
{
    pl = Plan{};
    if (qlen < 1 || qlen > GQA_MAX_QLEN)
        return GQA_ERR_INVALID_ARG;
    pl.G = Hq / Hkv;
    pl.R = qlen * pl.G;
    pl.mq = qlen > 1;
    pl.fp8 = fp8;
    // FP8 caches run on the tensor cores at D = 128 (one query token), else on the
    // CUDA-core kernel.
    pl.use_tc = (!fp8 || (D == 128 && qlen == 1)) && (D != 256 || qlen == 1) &&
                tc_applicable(states, B, Hkv, D, block_size, paged, num_blocks, pl.R);
    if (!pl.use_tc && !pick_variant(D, pl.G, states, pl.v, fp8))
        return GQA_ERR_UNSUPPORTED;
    if (!pl.use_tc && qlen > 1)  // several query tokens run on the tensor-core kernel only
        return GQA_ERR_UNSUPPORTED;
    if (nsplit > 0 && !pl.use_tc)
        return GQA_ERR_UNSUPPORTED;
    pl.wide = pl.use_tc && tc_wide(pl.R, D, pl.mq, fp8, nsplit);
    if (pl.wide) {
        pl.hch = (pl.R + TcWide::NP - 1) / TcWide::NP;
        pl.nv = TcWide::NP;
        pl.threads = TcWide::THREADS;
        pl.tile_tokens = TcWide::T;
        pl.stages = TcWide::SV;
        pl.smem = TcWide::smem_bytes(B);
        pl.box_rows = tc_box_rows(paged, block_size);
    } else if (pl.use_tc) {
        pl.hch = (pl.R + TcCfg::NP - 1) / TcCfg::NP;
        pl.nv = pl.R <= 4 ? 4 : (pl.R <= 8 ? 8 : 16);
        pl.threads = TcCfg::THREADS;
        pl.tile_tokens = fp8 ? TcGeom<128, true>::TILE : TcCfg::T;
        pl.stages = fp8 ? TcGeom<128, true>::STAGES
                        : (D == 64 ? TcGeom<64>::STAGES : D == 256 ? TcGeom<256>::STAGES : TcGeom<128>::STAGES);
        pl.smem = tc_smem_bytes(D, B, fp8);
        pl.box_rows = tc_box_rows(paged, block_size);
    } else {
        const int gc = head_chunk(pl.G);
        pl.hch = (pl.G + gc - 1) / gc;
        pl.nv = gc;
        pl.threads = pl.v.threads;
        pl.tile_tokens = pl.v.tile_tokens;
        pl.stages = pl.v.stages;
        pl.smem = pl.v.smem(B);
    }
    pl.nsplit = nsplit > 0 ? nsplit : 0;
    pl.items = nsplit > 0 ? (int64_t)B * Hkv * pl.hch * nsplit : 0;
    if (pl.items > (int64_t)1 << 30)
        return GQA_ERR_INVALID_ARG;
    if (dev < 0) {
        pl.ctas = -1;
        pl.grid = nsplit > 0 ? pl.items : -1;
        return GQA_OK;
    }
    int rc = pl.wide     ? tc_wide_ctas(dev, pl.ctas)
             : pl.use_tc ? tc_ctas(pl.R, dev, pl.ctas, pl.mq, D, fp8)
                         : persistent_ctas(pl.v, dev, pl.ctas);
    if (rc)
        return rc;
    // One chunk per segment (nsplit = 1) always finishes its segment: no slots.
    const int tc_slot = pl.wide ? TcWide::SLOT_FLOATS : tc_slot_floats(D);
    pl.w = nsplit > 1    ? layout_for((int)((pl.items + 1) / 2), tc_slot)
           : nsplit == 1 ? layout_for(0, tc_slot)
                         : layout_for(pl.ctas, pl.use_tc ? tc_slot : pl.v.slot_floats);
    pl.grid = nsplit > 0 ? pl.items : pl.ctas;
    return GQA_OK;
}

// nsplit = 0: the stream-K schedule; nsplit > 0: the fixed-split comparator
// (tensor-core shapes only), a grid of one CTA per (segment, chunk) followed by
// merge_split_kernel.
int run_decode(bool states, const void *q, const void *k_cache, const void *v_cache,
               const int32_t *block_table, const int32_t *seq_lens, const int32_t *kv_begin,
               const int32_t *kv_end, void *out, float *acc, float *m, float *l, int B, int Hq,
               int Hkv, int D, int block_size, float scale, int max_blocks, int num_blocks,
               void *workspace, size_t workspace_bytes, void *stream, int nsplit = 0,
               int qlen = 1, bool fp8 = false, float k_scale = 1.0f, float v_scale = 1.0f,
               unsigned long long *timeline = nullptr, int timeline_rows = 0,
               int *grid_out = nullptr)
{
    int rc = check_shape(B, Hq, Hkv, D, block_size, block_table, max_blocks, num_blocks, scale);
    if (rc)
        return rc;
    if (grid_out)
        *grid_out = 0;
    if (B == 0)
        return GQA_OK;
    // An empty pool (num_blocks == 0) is never read: its caches may be null.
    const bool empty_pool = block_table && num_blocks == 0;
    if (!q || !workspace || (!empty_pool && (!k_cache || !v_cache)))
        return GQA_ERR_INVALID_ARG;
    if (states ? (!kv_begin || !kv_end || !acc || !m || !l) : (!seq_lens || !out))
        return GQA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || (out && !aligned16(out)))
        return GQA_ERR_MISALIGNED;
    // Shape errors first (no device query), then the plan for the current device.
    Plan pl;
    if ((rc = make_plan(states, B, Hq, Hkv, D, block_size, block_table != nullptr, num_blocks, qlen,
                        fp8, nsplit, -1, pl)))
        return rc;
    int dev = 0;
    if ((rc = current_device(dev)))
        return rc;
    if ((rc = make_plan(states, B, Hq, Hkv, D, block_size, block_table != nullptr, num_blocks, qlen,
                        fp8, nsplit, dev, pl)))
        return rc;
    const bool use_tc = pl.use_tc;
    const int G = pl.G, R = pl.R, ctas = pl.ctas;
    const int64_t items = pl.items;
    const WorkspaceLayout w = pl.w;
    if (workspace_bytes < w.total)
        return GQA_ERR_WORKSPACE_TOO_SMALL;
    // The decode kernel's grid: one timeline row (TL_COLS values) per CTA.
    const int64_t grid = pl.grid;
    if (grid_out)
        *grid_out = (int)grid;
    if (timeline && timeline_rows < grid)
        return GQA_ERR_WORKSPACE_TOO_SMALL;

    unsigned char *ws = static_cast<unsigned char *>(workspace);
    Params p{};
    p.q = static_cast<const uint16_t *>(q);
    p.k = static_cast<const uint16_t *>(k_cache);
    p.v = static_cast<const uint16_t *>(v_cache);
    p.block_table = block_table;
    p.seq_lens = seq_lens;
    p.kv_begin = kv_begin;
    p.kv_end = kv_end;
    p.out = static_cast<uint16_t *>(out);
    p.st_acc = acc;
    p.st_m = m;
    p.st_l = l;
    p.status = reinterpret_cast<unsigned *>(ws);
    p.counters = reinterpret_cast<int *>(ws + w.counters_off);
    p.gcounters = reinterpret_cast<int *>(ws + w.gcounters_off);
    p.slots = reinterpret_cast<float *>(ws + w.slots_off);
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = G;
    p.qlen = qlen;
    p.R = R;
    p.block_size = block_size;
    p.max_blocks = block_table ? max_blocks : 1;
    p.num_blocks = block_table ? num_blocks : B;
    p.hch = pl.hch;
    p.nsplit = nsplit > 0 ? nsplit : 0;
    p.capacity = block_table ? (int64_t)max_blocks * block_size : (int64_t)block_size;
    p.qscale = scale * LOG2E * (fp8 ? k_scale : 1.0f);
    p.vscale = fp8 ? v_scale : 1.0f;
    p.timeline = timeline;
    p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    // Magic number for t / block_size (t < 2^31): see page_of().
    {
        int l = 0;
        while ((1ll << l) < block_size)
            ++l;
        const uint64_t m = ((((uint64_t)1 << l) - (uint64_t)block_size) << 32) / (uint64_t)block_size + 1;
        p.bs_magic = (uint32_t)m;
        p.bs_shift = l;
    }

    if (use_tc) {
        const int box_rows = pl.box_rows;
        const int64_t rows = (block_table ? (int64_t)num_blocks : (int64_t)B) * Hkv * block_size;
        CUtensorMap tmk, tmv;
        if (!encode_kv_map(&tmk, k_cache, rows, box_rows, D, fp8) ||
            !encode_kv_map(&tmv, v_cache, rows, box_rows, D, fp8))
            return GQA_ERR_CUDA;
        if (nsplit > 0) {
            // Fixed split: as many CTAs as chunks, in waves; no CTA waits for another.
            const cudaStream_t st = static_cast<cudaStream_t>(stream);
            const TcKernelFn fn = pl.wide ? gqa_decode_tc_wide_kernel : tc_kernel_for(R, qlen > 1, D, fp8);
            fn<<<(unsigned)items, pl.threads, pl.smem, st>>>(p, tmk, tmv, box_rows);
            if (B > 0 && nsplit > 1) {
                const int64_t threads = (int64_t)B * Hkv * pl.hch * pl.nv * D;
                tc_merge_for(R, D)<<<(unsigned)((threads + 127) / 128), 128, 0, st>>>(p);
            }
            return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
        }
        // Cooperative launch: the owners of a split segment wait for one another's
        // pieces, so every CTA of the grid must be resident (the launch fails
        // rather than run otherwise).
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)ctas);
        cfg.blockDim = dim3(pl.threads);
        cfg.dynamicSmemBytes = pl.smem;
        cfg.stream = static_cast<cudaStream_t>(stream);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const TcKernelFn fn = pl.wide ? gqa_decode_tc_wide_kernel : tc_kernel_for(R, qlen > 1, D, fp8);
        if (cudaLaunchKernelEx(&cfg, fn, p, tmk, tmv, box_rows) != cudaSuccess)
            return GQA_ERR_CUDA;
    } else {
        pl.v.fn<<<ctas, pl.threads, pl.smem, static_cast<cudaStream_t>(stream)>>>(p);
    }
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace
}  // namespace gqa

using namespace gqa;

// The schedule selector (gqa_select_schedule, gqa_decode_auto): fixed split
// with 1, 2, 4, ..., max_splits chunks against stream-K.  kv_fp8: an FP8 cache,
// whose tensor-core tiles are 256 tokens of one byte per element and which runs
// 16-head passes only.
int select_schedule(int B, int Hq, int Hkv, int D, const int32_t *seq_lens, int num_sms,
                    int max_splits, int *num_splits, float *est_us, bool kv_fp8 = false)
{
    if (!num_splits || num_sms <= 0 || (B > 0 && !seq_lens))
        return GQA_ERR_INVALID_ARG;
    int rc = check_shape(B, Hq, Hkv, D, 1, nullptr, 0, 0, 1.0f);
    if (rc)
        return rc;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] < 0)
            return GQA_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    const bool tc = tc_head_dim(D) && G >= TC_MIN_G && B <= TcCfg::MAX_BATCH;
    // Segments per request: head passes per KV head.  Stream-K and one chunk per
    // segment take the wide kernel's 64-head passes where it applies; a split into
    // several chunks runs 16-head passes.
    const int64_t units16 = (int64_t)Hkv * (tc ? (G + TcCfg::NP - 1) / TcCfg::NP
                                               : (G + head_chunk(G) - 1) / head_chunk(G));
    const int64_t units = tc && tc_wide(G, D, false, kv_fp8, 0)
                              ? (int64_t)Hkv * ((G + TcWide::NP - 1) / TcWide::NP) : units16;
    // Microseconds per 128-token K+V tile for a CTA while `active` CTAs stream.
    const int Tt = kv_fp8 ? TcGeom<128, true>::TILE : TcCfg::T;  // tokens per LeanTile
    const double tile_bytes = (kv_fp8 ? 2.0 : 4.0) * Tt * D;
    auto tile_us = [&](int64_t active) {
        const double gbs = std::min(SCHED_SM_GBS, SCHED_HBM_GBS / (double)std::max<int64_t>(active, 1));
        return tile_bytes / (gbs * 1e3);
    };
    std::vector<int64_t> nb(B);
    int64_t W = 0;
    for (int b = 0; b < B; ++b) {
        nb[b] = ((int64_t)seq_lens[b] + Tt - 1) / Tt;
        W += units * nb[b];
    }
    const int64_t P = num_sms;
    if (W == 0) {  // nothing to stream: any schedule is a no-op
        *num_splits = 0;
        if (est_us) {
            est_us[0] = 0.0f;
            est_us[1] = tc ? 0.0f : -1.0f;
        }
        return GQA_OK;
    }
    // Does any segment straddle two stream-K runs?  (tile_owner of its first and
    // last tile differ.)
    bool sk_split = false;
    int64_t seg0 = 0;
    for (int b = 0; b < B && !sk_split; ++b)
        for (int64_t u = 0; u < units && !sk_split; ++u, seg0 += nb[b])
            if (nb[b] > 0 && ((seg0 + 1) * P - 1) / W != ((seg0 + nb[b]) * P - 1) / W)
                sk_split = true;
    const int64_t sk_active = std::min(P, W);
    const double sk = (W + sk_active - 1) / sk_active * tile_us(sk_active) + SCHED_CTA_US +
                      (sk_split ? SCHED_MERGE_US : 0.0);
    // Fixed split: chunks are handed to SMs in index order as SMs free up.
    double best = -1.0;
    int best_s = 1;
    if (tc) {
        for (int sp = 1; sp <= max_splits; sp *= 2) {
            const int64_t un = sp == 1 ? units : units16;
            if ((int64_t)B * un * sp > ((int64_t)1 << 21))
                break;  // keep the host-side estimate cheap
            int64_t items = 0;
            for (int b = 0; b < B; ++b)
                items += un * std::min<int64_t>(nb[b], sp);
            const double tu = tile_us(std::min(P, items));
            std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
            for (int64_t i = 0; i < P; ++i)
                free_at.push(0.0);
            double makespan = 0.0;
            bool any_split = false;
            for (int b = 0; b < B; ++b)
                for (int64_t u = 0; u < un; ++u) {
                    int nonempty = 0;
                    for (int i = 0; i < sp; ++i) {
                        const int64_t len = (int64_t)(i + 1) * nb[b] / sp - (int64_t)i * nb[b] / sp;
                        const double t0 = free_at.top();
                        free_at.pop();
                        const double t1 = t0 + (len > 0 ? SCHED_CTA_US + len * tu : 0.0);
                        free_at.push(t1);
                        makespan = std::max(makespan, t1);
                        nonempty += len > 0;
                    }
                    any_split |= nonempty > 1;
                }
            const double t = makespan + (any_split ? SCHED_SPLIT_MERGE_US : 0.0);
            if (best < 0.0 || t < best) {
                best = t;
                best_s = sp;
            }
        }
    }
    // On a tie the fixed split wins: it needs neither a cooperative launch nor merges.
    *num_splits = (tc && best <= sk) ? best_s : 0;
    if (est_us) {
        est_us[0] = (float)sk;
        est_us[1] = tc ? (float)best : -1.0f;
    }
    return GQA_OK;
}

// gqa_decode_auto's choice between stream-K (0) and one CTA per (request, KV
// head) (1).  The second runs on the tensor-core kernel only, so a shape that
// kernel does not take (a page size its TMA boxes cannot tile, too many rows
// for a tensor map, a small group) stays on stream-K.
static int auto_splits(int B, int Hq, int Hkv, int D, int block_size, bool paged, int num_blocks,
                       const int32_t *seq_lens_host, int sms, int &ns, bool kv_fp8 = false)
{
    ns = 0;
    int rc = select_schedule(B, Hq, Hkv, D, seq_lens_host, sms, 1, &ns, nullptr, kv_fp8);
    if (rc)
        return rc;
    if (ns && !tc_applicable(false, B, Hkv, D, block_size, paged, num_blocks, Hq / Hkv))
        ns = 0;
    if (kv_fp8 && D != 128)  // FP8 runs on the tensor cores at D = 128 only; elsewhere stream-K
        ns = 0;
    return GQA_OK;
}

extern "C" {

int gqa_decode_workspace_size(int B, int Hq, int Hkv, int D, int device, size_t *bytes)
{
    if (!bytes)
        return GQA_ERR_INVALID_ARG;
    int rc = check_shape(B, Hq, Hkv, D, 1, nullptr, 0, 0, 1.0f);
    if (rc)
        return rc;
    size_t best = 0;
    for (int states = 0; states < 2; ++states) {
        Variant v;
        if (!pick_variant(D, Hq / Hkv, states != 0, v))
            return GQA_ERR_UNSUPPORTED;
        int ctas = 0;
        if ((rc = persistent_ctas(v, device, ctas)))
            return rc;
        const size_t t = layout_for(ctas, v.slot_floats).total;
        best = t > best ? t : best;
    }
    if (tc_head_dim(D)) {  // the tensor-core kernel (also for several query tokens)
        int ctas = 0;
        if ((rc = tc_ctas(TC_MIN_G, device, ctas)))
            return rc;
        const size_t t = layout_for(ctas, tc_slot_floats(D)).total;
        best = t > best ? t : best;
    }
    if (tc_wide(Hq / Hkv, D, false, false, 0)) {  // 64 heads per pass: larger slots
        int ctas = 0;
        if ((rc = tc_wide_ctas(device, ctas)))
            return rc;
        const size_t t = layout_for(ctas, TcWide::SLOT_FLOATS).total;
        best = t > best ? t : best;
    }
    *bytes = best;
    return GQA_OK;
}

int gqa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
               const int32_t *seq_lens, void *out, int B, int Hq, int Hkv, int D, int block_size,
               float scale, int max_blocks_per_seq, int num_blocks, void *workspace,
               size_t workspace_bytes, void *stream)
{
    return run_decode(false, q, k_cache, v_cache, block_table, seq_lens, nullptr, nullptr, out,
                      nullptr, nullptr, nullptr, B, Hq, Hkv, D, block_size, scale,
                      max_blocks_per_seq, num_blocks, workspace, workspace_bytes, stream);
}

int gqa_decode_fixed_split_workspace_size(int B, int Hq, int Hkv, int D, int num_splits, int device,
                                          size_t *bytes)
{
    if (!bytes || num_splits <= 0)
        return GQA_ERR_INVALID_ARG;
    int rc = check_shape(B, Hq, Hkv, D, 1, nullptr, 0, 0, 1.0f);
    if (rc)
        return rc;
    (void)device;
    const int G = Hq / Hkv;
    const int64_t items = (int64_t)B * Hkv * ((G + TcCfg::NP - 1) / TcCfg::NP) * num_splits;
    if (items > (int64_t)1 << 30)
        return GQA_ERR_INVALID_ARG;
    *bytes = layout_for(num_splits > 1 ? (int)((items + 1) / 2) : 0, tc_slot_floats(D)).total;
    return GQA_OK;
}

int gqa_decode_timeline(const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_table, const int32_t *seq_lens, void *out, int B,
                        int Hq, int Hkv, int D, int block_size, float scale,
                        int max_blocks_per_seq, int num_blocks, int num_splits,
                        unsigned long long *timeline, int timeline_rows, int *grid,
                        void *workspace, size_t workspace_bytes, void *stream)
{
    if (!timeline || timeline_rows < 0 || num_splits < 0 ||
        reinterpret_cast<uintptr_t>(timeline) % alignof(unsigned long long) != 0)
        return GQA_ERR_INVALID_ARG;
    return run_decode(false, q, k_cache, v_cache, block_table, seq_lens, nullptr, nullptr, out,
                      nullptr, nullptr, nullptr, B, Hq, Hkv, D, block_size, scale,
                      max_blocks_per_seq, num_blocks, workspace, workspace_bytes, stream,
                      num_splits, 1, false, 1.0f, 1.0f, timeline, timeline_rows, grid);
}

int gqa_decode_fixed_split(const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *block_table, const int32_t *seq_lens, void *out, int B,
                           int Hq, int Hkv, int D, int block_size, float scale,
                           int max_blocks_per_seq, int num_blocks, int num_splits,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    if (num_splits <= 0)
        return GQA_ERR_INVALID_ARG;
    return run_decode(false, q, k_cache, v_cache, block_table, seq_lens, nullptr, nullptr, out,
                      nullptr, nullptr, nullptr, B, Hq, Hkv, D, block_size, scale,
                      max_blocks_per_seq, num_blocks, workspace, workspace_bytes, stream,
                      num_splits);
}

int gqa_select_schedule(int B, int Hq, int Hkv, int D, const int32_t *seq_lens, int num_sms,
                        int max_splits, int *num_splits, float *est_us)
{
    if (max_splits < 1 || max_splits > 64)
        return GQA_ERR_INVALID_ARG;
    return select_schedule(B, Hq, Hkv, D, seq_lens, num_sms, max_splits, num_splits, est_us);
}

int gqa_decode_auto(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_table, const int32_t *seq_lens,
                    const int32_t *seq_lens_host, void *out, int B, int Hq, int Hkv, int D,
                    int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                    void *workspace, size_t workspace_bytes, void *stream)
{
    int dev = 0, sms = 0, rc;
    if ((rc = current_device(dev)))
        return rc;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GQA_ERR_CUDA;
    int ns = 0;
    if ((rc = auto_splits(B, Hq, Hkv, D, block_size, block_table != nullptr, num_blocks,
                          seq_lens_host, sms, ns)))
        return rc;
    return run_decode(false, q, k_cache, v_cache, block_table, seq_lens, nullptr, nullptr, out,
                      nullptr, nullptr, nullptr, B, Hq, Hkv, D, block_size, scale,
                      max_blocks_per_seq, num_blocks, workspace, workspace_bytes, stream, ns);
}

int gqa_decode_plan(int B, int Hq, int Hkv, int D, int block_size, int paged, int num_blocks,
                    int qlen, int kv_fp8, int num_splits, const int32_t *seq_lens_host, int device,
                    gqa_plan *plan)
{
    if (!plan || num_splits < -1)
        return GQA_ERR_INVALID_ARG;
    std::memset(plan, 0, sizeof *plan);
    int rc = check_shape(B, Hq, Hkv, D, block_size, paged ? &B : nullptr, 1,
                         paged ? num_blocks : 0, 1.0f);
    if (rc)
        return rc;
    if (paged && num_blocks < 0)
        return GQA_ERR_INVALID_ARG;
    if (B > 0 && num_splits == -1 && (!seq_lens_host || device < 0))
        return GQA_ERR_INVALID_ARG;
    if (seq_lens_host)
        for (int b = 0; b < B; ++b)
            if (seq_lens_host[b] < 0)
                return GQA_ERR_INVALID_ARG;
    if (kv_fp8 && (qlen != 1))
        return GQA_ERR_UNSUPPORTED;
    int ns = num_splits;
    if (ns == -1 && B > 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
            return GQA_ERR_CUDA;
        if ((rc = auto_splits(B, Hq, Hkv, D, block_size, paged != 0, num_blocks, seq_lens_host, sms,
                              ns, kv_fp8 != 0)))
            return rc;
    }
    ns = ns < 0 ? 0 : ns;
    plan->num_splits = ns;
    plan->tiles = -1;
    plan->grid = -1;
    if (B == 0) {  // nothing is launched
        plan->grid = 0;
        plan->tiles = 0;
        return GQA_OK;
    }
    Plan pl;
    if ((rc = make_plan(false, B, Hq, Hkv, D, block_size, paged != 0, num_blocks, qlen,
                        kv_fp8 != 0, ns, device, pl)))
        return rc;
    plan->kernel = pl.use_tc ? GQA_KERNEL_TENSOR_CORE : GQA_KERNEL_CUDA_CORE;
    plan->heads_per_pass = pl.nv;
    plan->head_chunks = pl.hch;
    plan->grid = (int)pl.grid;
    plan->threads_per_cta = pl.threads;
    plan->cooperative = pl.use_tc && ns == 0;
    plan->merge_launch = ns > 1;
    plan->tile_tokens = pl.tile_tokens;
    plan->ring_stages = pl.stages;
    plan->box_rows = pl.box_rows;
    plan->smem_bytes = pl.smem;
    plan->workspace_bytes = device >= 0 ? pl.w.total : 0;
    if (seq_lens_host) {
        long long tiles = 0;
        for (int b = 0; b < B; ++b)
            tiles += ((long long)seq_lens_host[b] + pl.tile_tokens - 1) / pl.tile_tokens;
        plan->tiles = tiles * Hkv * pl.hch;
    }
    if (pl.wide)
        std::snprintf(plan->kernel_name, sizeof plan->kernel_name, "gqa_decode_tc_wide_kernel<NV=%d,D=%d>",
                      pl.nv, D);
    else if (pl.use_tc)
        std::snprintf(plan->kernel_name, sizeof plan->kernel_name,
                      "gqa_decode_tc_kernel<NV=%d,MQ=%d,D=%d,F8=%d>", pl.nv, pl.mq ? 1 : 0, D,
                      kv_fp8 ? 1 : 0);
    else
        std::snprintf(plan->kernel_name, sizeof plan->kernel_name,
                      "gqa_decode_simt_kernel<D=%d,GC=%d,ST=0,F8=%d>", D, pl.nv, kv_fp8 ? 1 : 0);
    return GQA_OK;
}

int gqa_decode_multi(const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *block_table, const int32_t *seq_lens, void *out, int B,
                     int qlen, int Hq, int Hkv, int D, int block_size, float scale,
                     int max_blocks_per_seq, int num_blocks, void *workspace,
                     size_t workspace_bytes, void *stream)
{
    return run_decode(false, q, k_cache, v_cache, block_table, seq_lens, nullptr, nullptr, out,
                      nullptr, nullptr, nullptr, B, Hq, Hkv, D, block_size, scale,
                      max_blocks_per_seq, num_blocks, workspace, workspace_bytes, stream, 0, qlen);
}

int gqa_decode_fp8(const void *q, const void *k_cache, const void *v_cache, float k_scale,
                   float v_scale, const int32_t *block_table, const int32_t *seq_lens, void *out,
                   int B, int Hq, int Hkv, int D, int block_size, float scale,
                   int max_blocks_per_seq, int num_blocks, void *workspace,
                   size_t workspace_bytes, void *stream)
{
    if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || k_scale <= 0.f || v_scale <= 0.f)
        return GQA_ERR_INVALID_ARG;
    return run_decode(false, q, k_cache, v_cache, block_table, seq_lens, nullptr, nullptr, out,
                      nullptr, nullptr, nullptr, B, Hq, Hkv, D, block_size, scale,
                      max_blocks_per_seq, num_blocks, workspace, workspace_bytes, stream, 0, 1,
                      true, k_scale, v_scale);
}

int gqa_decode_fp8_auto(const void *q, const void *k_cache, const void *v_cache, float k_scale,
                        float v_scale, const int32_t *block_table, const int32_t *seq_lens,
                        const int32_t *seq_lens_host, void *out, int B, int Hq, int Hkv, int D,
                        int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                        void *workspace, size_t workspace_bytes, void *stream)
{
    if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || k_scale <= 0.f || v_scale <= 0.f)
        return GQA_ERR_INVALID_ARG;
    int dev = 0, sms = 0, rc;
    if ((rc = current_device(dev)))
        return rc;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GQA_ERR_CUDA;
    int ns = 0;
    if ((rc = auto_splits(B, Hq, Hkv, D, block_size, block_table != nullptr, num_blocks,
                          seq_lens_host, sms, ns, true)))
        return rc;
    return run_decode(false, q, k_cache, v_cache, block_table, seq_lens, nullptr, nullptr, out,
                      nullptr, nullptr, nullptr, B, Hq, Hkv, D, block_size, scale,
                      max_blocks_per_seq, num_blocks, workspace, workspace_bytes, stream, ns, 1,
                      true, k_scale, v_scale);
}

int gqa_decode_states(const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_table, const int32_t *kv_begin, const int32_t *kv_end,
                      float *acc, float *m, float *l, int B, int Hq, int Hkv, int D,
                      int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                      void *workspace, size_t workspace_bytes, void *stream)
{
    return run_decode(true, q, k_cache, v_cache, block_table, nullptr, kv_begin, kv_end, nullptr,
                      acc, m, l, B, Hq, Hkv, D, block_size, scale, max_blocks_per_seq, num_blocks,
                      workspace, workspace_bytes, stream);
}

int gqa_merge_states(const float *acc, const float *m, const float *l, int S, int N, int D,
                     void *out, float *lse, void *stream)
{
    if (S < 0 || N < 0 || D <= 0)
        return GQA_ERR_INVALID_ARG;
    if (N == 0)
        return GQA_OK;
    if (!out || (S > 0 && (!acc || !m || !l)))
        return GQA_ERR_INVALID_ARG;
    const int blocks = (N + MERGE_WARPS - 1) / MERGE_WARPS;
    merge_states_kernel<<<blocks, MERGE_WARPS * 32, 0, static_cast<cudaStream_t>(stream)>>>(
        acc, m, l, S, N, D, static_cast<uint16_t *>(out), lse);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

int gqa_status(void *workspace, void *stream, unsigned *device_error)
{
    if (!workspace || !device_error)
        return GQA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return GQA_ERR_CUDA;
    if (cudaMemcpy(&v, workspace, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
        return GQA_ERR_CUDA;
    // After a device error some tickets may be left mid-count: clear them too.
    if (v && cudaMemset(workspace, 0, STATUS_BYTES + COUNTERS_BYTES + GCOUNTERS_BYTES) != cudaSuccess)
        return GQA_ERR_CUDA;
    *device_error = v;
    return GQA_OK;
}

struct HostLayout {
    size_t q, k, v, bt, lens, out, total;
};

static HostLayout host_layout(int B, int Hq, int Hkv, int D, int block_size, int max_blocks,
                              int num_blocks, int paged)
{
    HostLayout h;
    const size_t nb = paged ? (size_t)num_blocks : (size_t)B;
    const size_t qbytes = (size_t)B * Hq * D * 2;
    const size_t kv = nb * Hkv * (size_t)block_size * D * 2;
    h.q = 0;
    h.k = align_up(h.q + qbytes, 256);
    h.v = align_up(h.k + kv, 256);
    h.bt = align_up(h.v + kv, 256);
    h.lens = align_up(h.bt + (paged ? (size_t)B * max_blocks * 4 : 0), 256);
    h.out = align_up(h.lens + (size_t)B * 4, 256);
    h.total = align_up(h.out + qbytes, 256);
    return h;
}

size_t gqa_decode_host_buffer_bytes(int B, int Hq, int Hkv, int D, int block_size,
                                    int max_blocks_per_seq, int num_blocks, int paged)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || block_size <= 0)
        return 0;
    return host_layout(B, Hq, Hkv, D, block_size, max_blocks_per_seq, num_blocks, paged).total;
}

int gqa_decode_host(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_table, const int32_t *seq_lens, void *out, int B, int Hq,
                    int Hkv, int D, int block_size, float scale, int max_blocks_per_seq,
                    int num_blocks, void *device_buffer, size_t device_buffer_bytes,
                    void *workspace, size_t workspace_bytes, void *stream)
{
    int rc = check_shape(B, Hq, Hkv, D, block_size, block_table, max_blocks_per_seq, num_blocks,
                         scale);
    if (rc)
        return rc;
    if (!q || !k_cache || !v_cache || !seq_lens || !out || !device_buffer)
        return GQA_ERR_INVALID_ARG;
    const int paged = block_table != nullptr;
    const HostLayout h =
        host_layout(B, Hq, Hkv, D, block_size, max_blocks_per_seq, num_blocks, paged);
    if (device_buffer_bytes < h.total)
        return GQA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char *dbuf = static_cast<unsigned char *>(device_buffer);
    const size_t nb = paged ? (size_t)num_blocks : (size_t)B;
    const size_t qbytes = (size_t)B * Hq * D * 2;
    const size_t kv = nb * Hkv * (size_t)block_size * D * 2;
    bool ok = cudaMemcpyAsync(dbuf + h.q, q, qbytes, cudaMemcpyHostToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(dbuf + h.k, k_cache, kv, cudaMemcpyHostToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(dbuf + h.v, v_cache, kv, cudaMemcpyHostToDevice, s) == cudaSuccess;
    if (paged)
        ok = ok && cudaMemcpyAsync(dbuf + h.bt, block_table, (size_t)B * max_blocks_per_seq * 4,
                                   cudaMemcpyHostToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(dbuf + h.lens, seq_lens, (size_t)B * 4, cudaMemcpyHostToDevice,
                               s) == cudaSuccess;
    if (!ok)
        return GQA_ERR_CUDA;
    rc = gqa_decode_auto(dbuf + h.q, dbuf + h.k, dbuf + h.v,
                         paged ? reinterpret_cast<const int32_t *>(dbuf + h.bt) : nullptr,
                         reinterpret_cast<const int32_t *>(dbuf + h.lens), seq_lens, dbuf + h.out,
                         B, Hq, Hkv, D, block_size, scale, max_blocks_per_seq, num_blocks,
                         workspace, workspace_bytes, stream);
    if (rc)
        return rc;
    if (cudaMemcpyAsync(out, dbuf + h.out, qbytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GQA_ERR_CUDA;
    return cudaStreamSynchronize(s) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

int gqa_stream_floor(const void *k, const void *v, long long rows, int ctas, void *workspace,
                     size_t workspace_bytes, void *stream)
{
    using C = FloorCfg;
    if (!k || !v || !workspace || rows < C::T || rows % C::T != 0 || rows > (1ll << 31) - C::T ||
        ctas < 1)
        return GQA_ERR_INVALID_ARG;
    if (workspace_bytes < STATUS_BYTES)
        return GQA_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(k) || !aligned16(v) || !aligned16(workspace))
        return GQA_ERR_MISALIGNED;
    int dev = 0, max_ctas = 0;
    if (current_device(dev) != GQA_OK)
        return GQA_ERR_CUDA;
    const int rc = persistent_ctas_fn(reinterpret_cast<const void *>(stream_floor_kernel), C::THREADS,
                                      C::SMEM, dev, max_ctas);
    if (rc != GQA_OK)
        return rc;
    if (ctas > max_ctas)
        return GQA_ERR_INVALID_ARG;
    CUtensorMap tmk, tmv;
    if (!encode_kv_map(&tmk, k, rows, C::T, 128) || !encode_kv_map(&tmv, v, rows, C::T, 128))
        return GQA_ERR_CUDA;
    stream_floor_kernel<<<ctas, C::THREADS, C::SMEM, static_cast<cudaStream_t>(stream)>>>(
        tmk, tmv, rows / C::T, static_cast<unsigned *>(workspace), g_wait_ns.load());
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

int gqa_set_wait_limit(unsigned long long ns, unsigned long long *previous)
{
    if (ns != 0 && (ns < 1000ull || ns > 10000000000ull))
        return GQA_ERR_INVALID_ARG;
    const unsigned long long old = g_wait_ns.exchange(ns ? ns : WAIT_LIMIT_NS);
    if (previous)
        *previous = old;
    return GQA_OK;
}

const char *gqa_error_string(int code)
{
    switch (code) {
    case GQA_OK: return "ok";
    case GQA_ERR_INVALID_ARG: return "invalid argument";
    case GQA_ERR_UNSUPPORTED: return "unsupported shape (D must be 64, 128 or 256; B <= 4096)";
    case GQA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case GQA_ERR_MISALIGNED: return "bf16 tensor not 16-byte aligned";
    case GQA_ERR_CUDA: return "CUDA runtime error";
    case GQA_ERR_SCRATCH_LIMIT: return "shape needs more scratch than gqa_decode_noalloc's fixed 16 MiB";
    default: return "unknown error";
    }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// gqa_decode_noalloc: gqa_decode for callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc at all: code running under another
// runtime's memory pool, plug-ins whose host owns every allocation, or
// latency-critical paths that forbid allocator calls.  They still
// own q, the caches and out, but cannot hand us a workspace.  For them the
// scratch gqa_decode needs (status word, ticket counters, partial-state slots)
// lives in one fixed array in this library's device image.  Every GPU that loads
// the library keeps that array until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = 16u << 20;  // 16 MiB per device

// Device-side scratch shared by every gqa_decode_noalloc call on a device.  In
// host code this name is only a handle; its device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void *g_noalloc_addr[gqa::MAX_DEVICES] = {};

// Device address of the scratch array on the current device, looked up once per
// device (the first call on a device does it).
int noalloc_scratch(int dev, void **addr)
{
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return GQA_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *addr = g_noalloc_addr[dev];
    return GQA_OK;
}

}  // namespace

extern "C" int gqa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *block_table, const int32_t *seq_lens, void *out,
                                  int B, int Hq, int Hkv, int D, int block_size, float scale,
                                  int max_blocks_per_seq, int num_blocks, void *stream)
{
    int rc = check_shape(B, Hq, Hkv, D, block_size, block_table, max_blocks_per_seq, num_blocks,
                         scale);
    if (rc)
        return rc;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return GQA_ERR_CUDA;
    if (dev < 0 || dev >= MAX_DEVICES)
        return GQA_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(dev, &scratch)))
        return rc;
    size_t need = 0;
    if ((rc = gqa_decode_workspace_size(B, Hq, Hkv, D, dev, &need)))
        return rc;
    if (need > NOALLOC_SCRATCH_BYTES)
        return GQA_ERR_SCRATCH_LIMIT;
    // The status word and the ticket counters this call can touch (per segment and
    // per CTA group) must start at zero; a previous call that hit a device error
    // may have left them set.
    const size_t clear = STATUS_BYTES + sizeof(int) * (size_t)B * Hq;
    if (cudaMemsetAsync(scratch, 0, clear, static_cast<cudaStream_t>(stream)) != cudaSuccess ||
        cudaMemsetAsync(static_cast<unsigned char *>(scratch) + STATUS_BYTES + COUNTERS_BYTES, 0,
                        GCOUNTERS_BYTES, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return GQA_ERR_CUDA;
    return gqa_decode(q, k_cache, v_cache, block_table, seq_lens, out, B, Hq, Hkv, D, block_size,
                      scale, max_blocks_per_seq, num_blocks, scratch, NOALLOC_SCRATCH_BYTES, stream);
}
