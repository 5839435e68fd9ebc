/*
 * gqa_decode.h -- C ABI of the B200 (sm_100a) decode-attention library
 * (libgqa_decode_b200.so).
 *
 * Operation (Attention co-design for long-context inference, sections
 * "Difference between prefill and decode" and "FlashAttention and GEMM shapes";
 * LeanAttention decode tiles digest, sections "Prefill and decode have different
 * shapes" and "Exact softmax that merges piece by piece"):
 *
 *   for every request b < B and query head h < Hq, with G = Hq / Hkv and
 *   KV head kvh = h / G,
 *       out[b, h, :] = softmax_t( scale * q[b, h, :] . K[b, kvh, t, :] ) V[b, kvh, t, :]
 *   over the cached tokens 0 <= t < seq_lens[b].  One query token per head;
 *   every cached key is visible (no mask inside a single decode query).
 *
 * Data types and layouts (all row-major, innermost index last):
 *   q, out         bf16 [B, Hq, D]
 *   k_cache,
 *   v_cache        bf16 [num_blocks, Hkv, block_size, D]   (paged pool)
 *                  bf16 [B, Hkv, block_size, D]            (block_table == NULL:
 *                       contiguous cache, block_size = per-request capacity)
 *   block_table    int32 [B, max_blocks_per_seq]; logical block j of request b
 *                  is physical block block_table[b * max_blocks_per_seq + j]
 *                  (Essential LLM optimization techniques (2), section
 *                  "PagedAttention", Figure 6-13); entries past a request's
 *                  last block are never read.
 *   seq_lens       int32 [B]
 *   bf16 values are passed as their 16-bit patterns; accumulation is fp32.
 *
 * Pointers: unless a function says otherwise, every pointer is a DEVICE pointer
 * on the current CUDA device, borrowed for the duration of the call (and of the
 * asynchronous work it enqueues); the library never frees or retains it.
 * q, k_cache, v_cache and out must be 16-byte aligned.  `stream` is a
 * cudaStream_t passed as void* (NULL = legacy default stream).
 *
 * Errors: every entry point returns GQA_OK (0) or a positive GQA_ERR_* code
 * after checking its arguments on the host; nothing is enqueued on error.
 * Problems only the device can see (a block id outside [0, num_blocks), a
 * length above the capacity, a bounded wait that ran out) never fault or trap:
 * the kernel skips the offending reads, writes NaN to the affected output rows
 * and ORs a GQA_DEV_* bit into a status word inside the workspace, which
 * gqa_status() reads back.
 */
#ifndef GQA_DECODE_H
#define GQA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GQA_API __attribute__((visibility("default")))
#else
#define GQA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Host-side return codes. */
#define GQA_OK 0
#define GQA_ERR_INVALID_ARG 1         /* null pointer, negative size, Hq % Hkv != 0, ... */
#define GQA_ERR_UNSUPPORTED 2         /* D not in {64, 128, 256}, B or Hq above the maxima */
#define GQA_ERR_WORKSPACE_TOO_SMALL 3 /* workspace_bytes below gqa_decode_workspace_size() */
#define GQA_ERR_MISALIGNED 4          /* a bf16 tensor not 16-byte aligned */
#define GQA_ERR_CUDA 5                /* a CUDA runtime call failed (launch, copy, ...) */
#define GQA_ERR_SCRATCH_LIMIT 6       /* gqa_decode_noalloc: shape needs more than its fixed scratch */

/* Device-side status bits (gqa_status). */
#define GQA_DEV_BAD_BLOCK 1u   /* a block-table entry outside [0, num_blocks) */
#define GQA_DEV_BAD_LENGTH 2u  /* a length < 0 or above the cache capacity */
#define GQA_DEV_TIMEOUT 4u     /* a bounded wait inside the kernel gave up */

#define GQA_MAX_BATCH 4096   /* requests per call */
#define GQA_MAX_QHEADS 256   /* query heads per request */
#define GQA_MAX_QLEN 16      /* query tokens per request (gqa_decode_multi) */

/*
 * Bytes of device workspace gqa_decode / gqa_decode_states need for this shape
 * on `device` (independent of the lengths; a few MiB).  The workspace holds a
 * status word, ticket counters at a fixed offset (room for GQA_MAX_BATCH x
 * GQA_MAX_QHEADS) and two partial softmax states per persistent CTA.  It must be
 * zero-filled once when allocated; every completed call leaves the counters at
 * zero again, so one workspace serves calls of any shape in turn.  After
 * gqa_status reports a device error it re-zeroes the counters itself.  Calls
 * that share one workspace must not overlap on the GPU (use one stream, or one
 * workspace per stream).
 */
GQA_API int gqa_decode_workspace_size(int B, int Hq, int Hkv, int D, int device, size_t *bytes);

/*
 * Decode attention for one layer and one decode step (the operation above).
 * Stream-K schedule: the context of every (request, KV head) is cut into
 * fixed-size tiles; tiles are ordered (request, KV head, tile) and every
 * persistent CTA takes one contiguous run of that global order, so long
 * requests spread over many SMs (LeanAttention decode tiles digest, sections
 * "Exact softmax that merges piece by piece" and "Hardware-sized work units").
 * A (request, KV head) split across CTAs is merged exactly from the partial
 * states.  On the tensor-core kernels (D = 64, 128 or 256, at least 4 query heads
 * per KV head -- more than 16 at D = 128 run 64 heads per pass -- pages of 8..128
 * tokens dividing 128 or multiples of 128, B <= 1024) the launch
 * is cooperative: every CTA is resident, and the owners of a split segment wait
 * (bounded, GQA_DEV_TIMEOUT on expiry) for one another and merge one slice of its
 * outputs each; the launch fails with GQA_ERR_CUDA rather than run when the grid
 * cannot be resident.  On the CUDA-core kernel the CTA that arrives last merges,
 * and no CTA waits.
 *
 *   block_table        NULL for a contiguous cache
 *   max_blocks_per_seq row stride of block_table (ignored when it is NULL)
 *   num_blocks         pool size, for bounds checks (ignored when block_table is NULL)
 *   scale              softmax scale, usually 1/sqrt(D)
 */
GQA_API int gqa_decode(const void *q, const void *k_cache, const void *v_cache,
               const int32_t *block_table, const int32_t *seq_lens, void *out,
               int B, int Hq, int Hkv, int D, int block_size, float scale,
               int max_blocks_per_seq, int num_blocks,
               void *workspace, size_t workspace_bytes, void *stream);

/*
 * Fixed-split comparator (FlashDecoding-style, the prior art the LeanAttention
 * decode tiles digest measures against in "Evaluation figures and their scope"):
 * the tiles of every (request, KV head) are cut into num_splits even chunks, one
 * CTA per chunk (a grid of B * Hkv * ceil(G / 16) * num_splits CTAs run in
 * waves), and a second kernel merges each segment's chunks exactly.  Same
 * arguments and result as gqa_decode; tensor-core shapes only (else
 * GQA_ERR_UNSUPPORTED); workspace from gqa_decode_fixed_split_workspace_size,
 * zero-filled once.  It exists to measure the stream-K schedule against.
 */
GQA_API int gqa_decode_fixed_split_workspace_size(int B, int Hq, int Hkv, int D, int num_splits,
                                                  int device, size_t *bytes);
GQA_API int gqa_decode_fixed_split(const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *block_table, const int32_t *seq_lens, void *out,
                                   int B, int Hq, int Hkv, int D, int block_size, float scale,
                                   int max_blocks_per_seq, int num_blocks, int num_splits,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Per-CTA timeline of one decode step, for measuring how evenly the work units
 * spread over the SMs and how long the last CTA trails (the tail wave the
 * LeanAttention decode tiles digest sets out to remove, sections "Hardware-sized
 * work units" and "Evaluation figures and their scope").  Computes exactly what
 * gqa_decode (num_splits = 0, the stream-K schedule) or gqa_decode_fixed_split
 * (num_splits >= 1) computes, with the same arguments, workspace and errors, and
 * in addition writes one row per CTA of the decode kernel's grid:
 *   timeline  DEVICE buffer, unsigned 64-bit [timeline_rows][8], 8-byte aligned,
 *             borrowed.  Row c = { start ns, end ns, SM id, tiles, first TMA ns,
 *             first scores ns, streamed ns, merged ns }: the GPU's global
 *             nanosecond timer when CTA c began and when it finished (after any
 *             merge it took part in), the SM it ran on, and the number of tiles
 *             (work units) in its run: 128 tokens each on the tensor-core
 *             kernel, the kernel's own tile size on the CUDA cores.  For a
 *             tensor-core CTA with work, the last four are the timer when it
 *             issued its first K tile, when the first tile's scores were ready,
 *             when its last piece was closed, and when its merges were done;
 *             they are 0 for other CTAs and on the CUDA cores.
 *   grid      HOST int or NULL; receives the number of rows written (0 for B = 0).
 * timeline_rows below the grid returns GQA_ERR_WORKSPACE_TOO_SMALL without
 * launching (grid is still set), so a caller may size the buffer from a first
 * call.  A NULL or misaligned timeline, or num_splits < 0, is GQA_ERR_INVALID_ARG.
 * The second kernel of the fixed split records no rows.
 */
GQA_API int gqa_decode_timeline(const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_table, const int32_t *seq_lens, void *out,
                                int B, int Hq, int Hkv, int D, int block_size, float scale,
                                int max_blocks_per_seq, int num_blocks, int num_splits,
                                unsigned long long *timeline, int timeline_rows, int *grid,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * Runtime schedule selection on the host (LeanAttention decode tiles digest,
 * section "Runtime selection policy": the choice depends on the batch's context
 * length distribution, the heads per device, the head dimension and the SM
 * count).  seq_lens is a HOST array [B].  A cost model of this library on B200
 * (per-CTA streaming rate, shared HBM bandwidth, start-up and merge costs)
 * estimates the stream-K schedule and the fixed split with 1, 2, 4, ...,
 * max_splits (<= 64) chunks, chunks assigned to SMs in order as they free up.
 * *num_splits = 0 selects gqa_decode (stream-K), n > 0 selects
 * gqa_decode_fixed_split with n chunks.  est_us (NULL or float[2]) receives the
 * two estimates: stream-K, best fixed split (-1 when fixed split does not apply).
 * Contention from other kernels, which the digest also lists, is not modelled.
 */
GQA_API int gqa_select_schedule(int B, int Hq, int Hkv, int D, const int32_t *seq_lens, int num_sms,
                                int max_splits, int *num_splits, float *est_us);

/*
 * gqa_decode with the runtime selection of the LeanAttention decode tiles digest
 * ("Runtime selection policy": short contexts or large batches fill the GPU with
 * one CTA per (request, KV head) and need no reduction; long contexts, few heads
 * per device and uneven batches want stream-K).  seq_lens_host is a HOST copy of
 * seq_lens [B]; gqa_select_schedule's cost model, restricted to the two choices
 * stream-K and one chunk per segment, picks the schedule.  Same arguments,
 * workspace (gqa_decode_workspace_size) and result as gqa_decode.
 */
GQA_API int gqa_decode_auto(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_table, const int32_t *seq_lens,
                            const int32_t *seq_lens_host, void *out, int B, int Hq, int Hkv, int D,
                            int block_size, float scale, int max_blocks_per_seq, int num_blocks,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * What a call would launch, reported without launching anything: the kernel
 * and its template parameters, the schedule, the grid and the LeanTile count
 * (the work units of LeanAttention decode tiles digest, section
 * "Hardware-sized work units").  The library's own launch path decides from the
 * same host-side plan, so the report is what runs.
 *   paged          1: a paged pool of num_blocks blocks (block_table non-NULL);
 *                  0: a contiguous cache (block_size = per-request capacity)
 *   qlen           query tokens per request (1: gqa_decode; > 1: gqa_decode_multi)
 *   kv_fp8         1: an FP8 E4M3 cache (gqa_decode_fp8; qlen must be 1)
 *   num_splits     -1: the choice gqa_decode_auto (gqa_decode_fp8_auto) makes (needs
 *                  seq_lens_host and a device); 0: stream-K; n > 0:
 *                  gqa_decode_fixed_split
 *   seq_lens_host  HOST int32 [B] or NULL; with it, plan->tiles is filled in
 *   device         CUDA device for the grid and workspace size; < 0: no device
 *                  query (grid = -1 for stream-K, workspace_bytes = 0)
 *   plan           HOST, written on GQA_OK
 * Errors: those gqa_decode would return for the shape (GQA_ERR_UNSUPPORTED for a
 * schedule or format the shape cannot run), GQA_ERR_INVALID_ARG for a NULL plan,
 * num_splits < -1, a negative length, or num_splits = -1 without lengths or a
 * device.  B = 0 gives kernel = 0 (nothing is launched).
 */
#define GQA_KERNEL_TENSOR_CORE 1  /* gqa_decode_tc_kernel: tcgen05 MMAs, TMA tiles */
#define GQA_KERNEL_CUDA_CORE 2    /* gqa_decode_simt_kernel: packed FMAs on CUDA cores */
typedef struct gqa_plan {
    int kernel;              /* GQA_KERNEL_*, 0 when nothing is launched */
    int heads_per_pass;      /* query rows one pass carries (tensor cores: 4, 8, 16, 64) */
    int head_chunks;         /* passes per KV head */
    int num_splits;          /* 0: stream-K; n > 0: fixed split into n chunks */
    int grid;                /* CTAs of the decode kernel (-1: no device given) */
    int threads_per_cta;
    int cooperative;         /* 1: cooperative launch (every CTA resident) */
    int merge_launch;        /* 1: a second kernel merges the fixed-split chunks */
    int tile_tokens;         /* tokens per LeanTile (256 on the FP8 tensor-core kernel) */
    int ring_stages;         /* shared-memory ring slots per K (and per V) stream */
    int box_rows;            /* tensor cores: tokens per TMA box (0 on CUDA cores) */
    long long tiles;         /* LeanTiles of the step (-1 without seq_lens_host) */
    size_t smem_bytes;       /* dynamic shared memory per CTA */
    size_t workspace_bytes;  /* workspace the call needs on `device` */
    char kernel_name[64];    /* e.g. "gqa_decode_tc_kernel<NV=4,MQ=0,D=128,F8=0>" */
} gqa_plan;
GQA_API int gqa_decode_plan(int B, int Hq, int Hkv, int D, int block_size, int paged,
                            int num_blocks, int qlen, int kv_fp8, int num_splits,
                            const int32_t *seq_lens_host, int device, gqa_plan *plan);

/*
 * Several query tokens per request: the verification pass of speculative
 * decoding, where the large model scores the qlen drafted positions in one pass
 * (Inference optimization: KV cache, MQA/GQA, batching..., section 5
 * "Speculative decoding").  The drafted tokens' keys and values are already in
 * the cache: request b holds L_b >= qlen tokens and query token i sits at
 * position L_b - qlen + i, seeing the keys t <= L_b - qlen + i (causal inside the
 * qlen new tokens).
 *   q, out  [B, qlen, Hq, D] bf16; everything else as gqa_decode.
 * 1 <= qlen <= GQA_MAX_QLEN; qlen = 1 is gqa_decode.  Runs on the tensor-core
 * kernel (D = 64 or 128, qlen * Hq / Hkv >= 4, its page sizes, B <= 1024), the query
 * rows of one KV head (qlen x G) sharing every K/V tile; other shapes return
 * GQA_ERR_UNSUPPORTED for qlen > 1.  A request with L_b < qlen gets NaN rows and
 * GQA_DEV_BAD_LENGTH.  Workspace: gqa_decode_workspace_size(B, Hq, Hkv, D, ...).
 */
GQA_API int gqa_decode_multi(const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *block_table, const int32_t *seq_lens, void *out,
                             int B, int qlen, int Hq, int Hkv, int D, int block_size, float scale,
                             int max_blocks_per_seq, int num_blocks, void *workspace,
                             size_t workspace_bytes, void *stream);

/*
 * gqa_decode over an FP8 E4M3 cache (the FP8 KV cache of Attention co-design for
 * long-context inference, list of techniques): k_cache and v_cache hold one byte
 * per element in the bf16 caches' layouts; element values are e4m3(byte) * k_scale
 * and e4m3(byte) * v_scale (one scale per tensor, > 0).  q and out stay bf16.  A
 * decode step reads half the bytes.  At D = 128 with at least 4 query heads per
 * KV head (and the tensor-core kernel's page sizes, B <= 1024) it runs on the
 * tensor cores over 256-token LeanTiles (64 KB of K and V per step, as a bf16
 * tile of 128 tokens): kind::f8f6f4 MMAs read the cache bytes as loaded; q
 * enters as two E4M3 terms (t1 + t2 / 16, each q row first scaled by a power of
 * two) and the softmax weights as three (t1 + t2 / 16 + t3 / 256); accumulation
 * in fp32.  Other shapes run on the CUDA-core kernel, the E4M3 bytes widened
 * exactly in registers.  k_scale is
 * folded into the scores, v_scale applied to the output.  Workspace:
 * gqa_decode_workspace_size.  Errors as gqa_decode.
 */
GQA_API int gqa_decode_fp8(const void *q, const void *k_cache, const void *v_cache, float k_scale,
                           float v_scale, const int32_t *block_table, const int32_t *seq_lens,
                           void *out, int B, int Hq, int Hkv, int D, int block_size, float scale,
                           int max_blocks_per_seq, int num_blocks, void *workspace,
                           size_t workspace_bytes, void *stream);

/*
 * gqa_decode_fp8 with gqa_decode_auto's runtime selection (stream-K, or one CTA
 * per (request, KV head) when that already fills the GPU), given a HOST copy of
 * the lengths, seq_lens_host int32 [B] (read during the call only).  The cost
 * model takes the FP8 kernel's tiles (256 tokens, one byte per element) and its
 * 16-head passes.  FP8 caches off the tensor cores (D != 128) always take
 * stream-K.  Arguments, workspace, results and errors otherwise as gqa_decode_fp8.
 */
GQA_API int gqa_decode_fp8_auto(const void *q, const void *k_cache, const void *v_cache,
                                float k_scale, float v_scale, const int32_t *block_table,
                                const int32_t *seq_lens, const int32_t *seq_lens_host, void *out,
                                int B, int Hq, int Hkv, int D, int block_size, float scale,
                                int max_blocks_per_seq, int num_blocks, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * Partial softmax states of every query row over the key range
 * [kv_begin[b], kv_end[b]) of request b (both int32 [B], device):
 *   m[b, h]      = max_t s_t                      (natural-log units)
 *   l[b, h]      = sum_t exp(s_t - m)
 *   acc[b, h, :] = sum_t exp(s_t - m) V_t         (not normalised)
 * acc is fp32 [B, Hq, D]; m and l are fp32 [B, Hq].  An empty range gives
 * m = -inf, l = 0, acc = 0.  Feeding the states of disjoint ranges that cover
 * [0, L_b) to gqa_merge_states reproduces gqa_decode (LeanAttention decode tiles
 * digest, section "Exact softmax that merges piece by piece").
 */
GQA_API int gqa_decode_states(const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *block_table, const int32_t *kv_begin,
                      const int32_t *kv_end, float *acc, float *m, float *l,
                      int B, int Hq, int Hkv, int D, int block_size, float scale,
                      int max_blocks_per_seq, int num_blocks,
                      void *workspace, size_t workspace_bytes, void *stream);

/*
 * Exact merge of S partial states per row (LeanAttention decode tiles digest,
 * section "Exact softmax that merges piece by piece"):
 *   m* = max_i m_i,  w_i = exp(m_i - m*) (0 when m_i = -inf),
 *   out = bf16( sum_i w_i acc_i / sum_i w_i l_i ),  lse = m* + log(sum_i w_i l_i).
 * acc fp32 [S, N, D]; m, l fp32 [S, N]; out bf16 [N, D]; lse fp32 [N] or NULL.
 * Pieces are combined in index order, so the result does not depend on timing.
 * A row whose pieces are all empty gives out = 0 and lse = -inf.
 */
GQA_API int gqa_merge_states(const float *acc, const float *m, const float *l, int S, int N, int D,
                     void *out, float *lse, void *stream);

/*
 * Synchronises `stream`, returns the device status bits accumulated in
 * `workspace` since the last call in *device_error (0 = clean), and clears them.
 */
GQA_API int gqa_status(void *workspace, void *stream, unsigned *device_error);

/*
 * gqa_decode with HOST buffers: copies q, k_cache, v_cache, block_table and
 * seq_lens from host memory into `device_buffer` (at least
 * gqa_decode_host_buffer_bytes() bytes, device), runs gqa_decode_auto (the
 * lengths are on the host already), copies out back to host memory and
 * synchronises the stream.  Pinned host memory gives asynchronous,
 * full-bandwidth copies.  Same shapes and errors as gqa_decode.
 */
GQA_API size_t gqa_decode_host_buffer_bytes(int B, int Hq, int Hkv, int D, int block_size,
                                    int max_blocks_per_seq, int num_blocks, int paged);
GQA_API int gqa_decode_host(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_table, const int32_t *seq_lens, void *out,
                    int B, int Hq, int Hkv, int D, int block_size, float scale,
                    int max_blocks_per_seq, int num_blocks,
                    void *device_buffer, size_t device_buffer_bytes,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * gqa_decode without a workspace argument, for callers that cannot allocate
 * device memory (nothing here calls cudaMalloc, cudaFree or an allocating
 * library routine).  The pages describe no such call; it exists for callers
 * that run under an allocator they do not control -- inside another runtime's
 * memory pool, in a plug-in whose host owns every allocation, or on a path where
 * allocator calls are forbidden -- and so cannot pass the workspace gqa_decode
 * wants.  Arguments, layouts and results are those of gqa_decode.
 *
 * Scratch: one fixed 16 MiB array inside the library's device image, held by
 * every GPU that loads the library until the process exits.  A shape whose
 * scratch need (gqa_decode_workspace_size) exceeds 16 MiB is rejected with
 * GQA_ERR_SCRATCH_LIMIT; B above GQA_MAX_BATCH or Hq above GQA_MAX_QHEADS with
 * GQA_ERR_UNSUPPORTED.  On B200 every shape within those maxima fits.
 *
 * The first call on each device looks up the array's device address (with that
 * device current); make that first call before any stream capture.  Each call
 * first clears, on `stream`, the status word and the ticket counters it can use.
 * All calls on a device share the one array and it keeps the last call's
 * contents, so calls that overlap on the GPU (different streams, no ordering
 * between them) race and give wrong results: order them, e.g. on one stream.
 * Device-side errors (bad block ids, lengths) still yield NaN rows as in
 * gqa_decode; the status word is not exposed.
 */
GQA_API int gqa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *block_table, const int32_t *seq_lens, void *out,
                               int B, int Hq, int Hkv, int D, int block_size, float scale,
                               int max_blocks_per_seq, int num_blocks, void *stream);

/*
 * The longest any wait inside the decode kernels for progress may last -- a
 * pipeline stage, or the partial states of the other CTAs sharing a split
 * (request, KV head) -- before the kernel gives up on it: it then sets
 * GQA_DEV_TIMEOUT, stops streaming, writes NaN to the rows it could not finish
 * and returns (the LeanAttention decode tiles digest's split pieces are merged by
 * CTAs that wait for one another; a wait that cannot end must not hang the GPU).
 * Healthy waits last microseconds; the default limit is 1.5 s.  The setting is
 * process-wide and applies to calls launched after this returns.  ns = 0
 * restores the default; otherwise 1e3 <= ns <= 1e10, else GQA_ERR_INVALID_ARG.
 * *previous (HOST, may be NULL) receives the limit in force before.  The waits at
 * exit for the kernel's own copies and tensor-core work in flight keep the
 * default limit whatever is set here, so no CTA leaves with work outstanding.
 */
GQA_API int gqa_set_wait_limit(unsigned long long ns, unsigned long long *previous);

/*
 * Measurement reference, not part of the attention path: streams k and v, each
 * a contiguous bf16 array of `rows` rows of 128 columns (256 bytes per row;
 * rows a positive multiple of 128, below 2^31), through the decode kernels'
 * TMA boxes and three-slot rings of 32 KB with no arithmetic, over `ctas`
 * CTAs (1 .. resident CTAs of the device), CTA c taking 128-row tiles
 * [c W / ctas, (c+1) W / ctas) of the W = rows / 128 as the stream-K decode
 * schedule does.  A decode step is bound by reading its K and V from HBM
 * (Attention co-design for long-context inference, section "Difference between
 * prefill and decode", Equation 1 and Figure 2), so this kernel, timed like a
 * step over the step's K and V bytes, gives the floor that streaming alone
 * reaches under that timing.  The bytes are read, never interpreted.
 * k, v, workspace: DEVICE, 16-byte aligned; workspace as for gqa_decode (at
 * least its status word): a bounded wait that runs out sets GQA_DEV_TIMEOUT
 * there.  Returns GQA_OK, GQA_ERR_INVALID_ARG, GQA_ERR_WORKSPACE_TOO_SMALL,
 * GQA_ERR_MISALIGNED or GQA_ERR_CUDA; asynchronous.
 */
GQA_API int gqa_stream_floor(const void *k, const void *v, long long rows, int ctas,
                             void *workspace, size_t workspace_bytes, void *stream);

/* Human-readable text for a GQA_ERR_* code. */
GQA_API const char *gqa_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* GQA_DECODE_H */
