/*
 * lora_sgmv.h -- C ABI of the heterogeneous-batch LoRA delta for B200 (sm_100a).
 *
 * The operation.  A batch of T tokens, each naming its own adapter i = id[t] and that
 * adapter's rank r_i, receives the low-rank update of one projection of one layer:
 *
 *     v[t, 0:r_i]        = x[t, 0:h] . A_i^T                (shrink, scale 1, fp32 result)
 *     y[t, off + n]     += s_i * sum_k v[t, k] * B_i[n, k]   (expand, n < o)
 *
 * Sources (multi-LoRA serving pages):
 *   - "TGI Multi-LoRA: Deploy Once, Serve 30 Models", section "Technical Foundation: LoRA"
 *     (frozen base weight plus two small trained matrices A and B) and section "How
 *     Multi-LoRA Serving Works" (one adapter id per request; requests for different adapters
 *     share one forward pass as a heterogeneous batch).
 *   - "Compress then Serve" review thread, authors' rebuttal on Punica: SGMV groups the
 *     requests that use the same LoRA model; the add_lora_slice_with_sigma pseudocode
 *     applies A with scale 1 into an fp32 buffer of shape (tokens, R), then B with the
 *     scale into the column slice [y_offset, y_offset + y_slice_size) of y, the adapter of
 *     each token coming from a per-token index vector (its "indices").
 *   - "how does this differ from S-LoRA?" (LoRAX issue): adapters of different ranks in one
 *     batch, served by one kernel.
 *
 * Layouts (all row-major, element type E = bf16 or fp32 as the table says):
 *   x  [T, ldx]   first h columns used           y  [T, ldy]   columns [y_offset, y_offset+o)
 *   A_i [r_i, h]  (PEFT lora_A orientation)      B_i [o, r_i]  (PEFT lora_B orientation)
 *   v  [T, ldv]   fp32, indexed by token (not by sorted position)
 *
 * Alignment: every pointer to x, y, A_i, B_i, v is 16-byte aligned; h, o, ldx, ldy and
 * y_offset are multiples of 16 / sizeof(E); ldv is a multiple of 4.  Violations return
 * LORA_ERR_UNSUPPORTED before anything is launched.
 *
 * Streams.  Every call enqueues on the given CUDA stream (a cudaStream_t passed as void*;
 * NULL is the legacy default stream).  The hot calls (lora_build_segments, lora_shrink,
 * lora_expand, lora_sgmv, lora_bgmv) never allocate, never synchronise the host, and never
 * read device memory from the host.
 *
 * Errors.  Each call returns LORA_OK (0) or a negative LORA_ERR_* code.  Problems the host
 * can see (null pointers, sizes, alignment, workspace size) are rejected before launch.
 * Problems only the device can see -- an id outside [-1, n), a segment entry out of range,
 * a bounded wait that ran out -- never trap: the offending token or segment is skipped and
 * a bit is latched into the table's device status word, which lora_get_status reads.
 * There is no CPU fallback: an unsupported configuration is an error.
 *
 * Ownership.  The caller owns x, y, v, ids, segment arrays, workspace and every A_i / B_i
 * buffer, and keeps the weights alive while a table refers to them.  A table owns only its
 * device descriptor array (adapter pointers, ranks, scales) and its status word.
 */
#ifndef LORA_SGMV_H
#define LORA_SGMV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types of a table (x, y, A_i and B_i share it). */
#define LORA_F32 0
#define LORA_BF16 1

/* Return codes. */
#define LORA_OK 0
#define LORA_ERR_INVALID_ARG (-1)   /* null pointer, negative size, bad id in host data   */
#define LORA_ERR_UNSUPPORTED (-2)   /* rank > LORA_MAX_RANK, alignment, dtype, size limits */
#define LORA_ERR_WORKSPACE (-3)     /* workspace pointer null or smaller than required      */
#define LORA_ERR_CUDA (-4)          /* a CUDA runtime call failed                           */
#define LORA_ERR_TIMEOUT (-5)       /* a device-side bounded wait ran out (status word)     */
#define LORA_ERR_DEVICE_STATUS (-6) /* lora_get_status found a latched device error         */

/* Bits of the device status word. */
#define LORA_STATUS_BAD_ID 1u       /* an id outside [-1, n) was skipped                    */
#define LORA_STATUS_TIMEOUT 2u      /* a bounded wait gave up; that block stopped early     */
#define LORA_STATUS_BAD_SEGMENT 4u  /* a segment entry (adapter, bounds, perm) was skipped */

/* Limits. */
#define LORA_MAX_RANK 128            /* largest r_i a table accepts                        */
#define LORA_MAX_SEGMENT_TOKENS 8192 /* largest T lora_build_segments sorts in one call    */

typedef struct lora_table lora_table; /* opaque */

/* Segments: tokens grouped by adapter, so that all requests of one LoRA model are served
 * together ("Compress then Serve" review thread, authors' rebuttal on Punica, SGMV).
 * Segment s covers sorted positions [seg_ptr[s], seg_ptr[s+1]); the token at sorted position
 * p is perm[p], or p itself when perm is NULL (tokens already contiguous per adapter, as in
 * prefill).  All arrays are device memory and may be produced by lora_build_segments. */
typedef struct lora_segments {
    const int32_t *perm;        /* [>= seg_ptr[num_segs]] token index per sorted position, or NULL */
    const int32_t *seg_ptr;     /* [max_segs + 1] */
    const int32_t *seg_adapter; /* [max_segs]    adapter of each segment */
    const int32_t *num_segs;    /* [1]           number of segments S (<= max_segs) */
    int32_t T;                  /* rows of x and y */
    int32_t max_segs;           /* capacity of the segment arrays (host value) */
    int32_t max_seg_len;        /* host hint: no segment is longer (0 = unknown) */
    int32_t reserved;
} lora_segments;

/* Register the adapters of one (layer, projection).  A and B are HOST arrays of n DEVICE
 * pointers; A[i] is [ranks[i], h_in], B[i] is [h_out, ranks[i]], both of element type dtype.
 * ranks[i] in [1, LORA_MAX_RANK]; scales[i] is s_i.  The descriptor array is copied to the
 * device on `stream`.  Stands in for the stacked per-layer weights and layer index of the
 * pseudocode: one table per (layer, projection), adapters neither contiguous nor padded. */
int lora_table_create(lora_table **out, int32_t n_adapters, int32_t h_in, int32_t h_out,
                      int32_t dtype, const void *const *A, const void *const *B,
                      const int32_t *ranks, const float *scales, void *stream);

/* Three-stage (compressed) form, "Compress then Serve" review thread, authors' rebuttal on
 * Punica, pseudocode of add_lora_slice_with_sigma: between the A step (scale 1) and the B
 * step (scale s_i) each token's intermediate passes through its adapter's small matrix:
 *   LORA_SIGMA_FULL: sigma[i] is [ranks[i], ranks[i]] row-major, v'[k] = sum_m sigma[i][k, m] v[m]
 *   LORA_SIGMA_DIAG: sigma[i] holds ranks[i] values,              v'[k] = sigma[i][k] * v[k]
 * (the pages' JD-Full and JD-Diag).  sigma is a HOST array of n DEVICE pointers to fp32 values
 * (4-byte aligned), kept alive by the caller while the table uses them; LORA_SIGMA_NONE
 * (sigma may be NULL) returns to the plain form.  Adapters of one compression cluster share
 * A_c and B_c simply by passing the same A / B pointers to lora_table_create.  Every compute
 * call then applies Sigma in fp32 on chip; lora_shrink writes v' (steps 1 and 2) and
 * lora_expand takes v' as given.  Tables with Sigma use the decode kernels (no tcgen05 path).
 * The descriptor update is copied on `stream` and synchronised; do not call it while calls
 * that use the table are in flight. */
#define LORA_SIGMA_NONE 0
#define LORA_SIGMA_FULL 1
#define LORA_SIGMA_DIAG 2
int lora_table_set_sigma(lora_table *table, int32_t kind, const float *const *sigma, void *stream);

/* Free the table's device memory (synchronises the device first).  NULL is accepted. */
int lora_table_destroy(lora_table *table);

/* Table metadata (any output pointer may be NULL). */
int lora_table_info(const lora_table *table, int32_t *n_adapters, int32_t *h_in,
                    int32_t *h_out, int32_t *max_rank, int32_t *dtype);

/* Bytes of device workspace that lora_sgmv and lora_bgmv need for T tokens (a multiple of
 * 256; 0 is never returned). */
size_t lora_workspace_bytes(const lora_table *table, int32_t T);

/* Segment bookkeeping (SGMV grouping): a stable sort of the tokens by adapter id.
 * Outputs, all device arrays: perm[T] (token of each sorted position; only the first
 * seg_ptr[num_segs] entries are written), seg_ptr[n + 1], seg_adapter[n], num_segs[1].
 * Segments come in ascending adapter id, one per adapter with at least one token, tokens in
 * batch order inside a segment.  id -1 means "no adapter" and is left out; other ids outside
 * [0, n) are left out and latch LORA_STATUS_BAD_ID.  T <= LORA_MAX_SEGMENT_TOKENS.
 * Bit-exact: the result is unique. */
int lora_build_segments(const lora_table *table, const int32_t *d_ids, int32_t T,
                        int32_t *d_perm, int32_t *d_seg_ptr, int32_t *d_seg_adapter,
                        int32_t *d_num_segs, void *stream);

/* Shrink step alone: v[t, 0:r_i] = x[t] . A_i^T for every token of every segment (fp32
 * accumulation, scale 1).  Columns >= r_i of v and rows of tokens outside all segments are
 * not written.  ldv >= the table's max rank. */
int lora_shrink(const lora_table *table, const lora_segments *seg, const void *x,
                int64_t ldx, float *v, int32_t ldv, void *stream);

/* Expand step alone: y[t, y_offset + n] = round(y[t, y_offset + n] + s_i * v[t, 0:r_i] . B_i[n])
 * for every token of every segment, n < o, rounding once to nearest-even in E. */
int lora_expand(const lora_table *table, const lora_segments *seg, const float *v,
                int32_t ldv, void *y, int64_t ldy, int32_t y_offset, void *stream);

/* SGMV: shrink and expand for sorted segments, in place on the y slice.  Picks the path:
 *  - the tcgen05 tensor-core path (prefill) for every segment when the hint max_seg_len
 *    reaches the "prefill_min_seg_len" option (256), perm is NULL, and the table is
 *    tensor-core capable (bf16, every rank a multiple of 8 and at most 64, no Sigma);
 *  - otherwise, in a batch of at least "tc_min_tokens" (1024) tokens on a tensor-core capable
 *    table with the workspace given, a split decided on the device from the segment lengths:
 *    segments of at least "tc_min_seg_len" (64) tokens run on the tcgen05 kernels, which
 *    gather their token rows through perm (TMA four-row gathers), and the shorter ones on the
 *    fused cluster kernel; both launches read the same segment table;
 *  - otherwise every segment runs on the fused cluster kernel (decode).
 * The tcgen05 kernels keep their intermediate (bf16 hi + lo) in the workspace; the fused
 * kernel needs none, so ws may be NULL when ws_bytes is 0 (every segment then runs on the
 * fused kernel); a path that needs the workspace requires ws_bytes >=
 * lora_workspace_bytes(table, seg->T). */
int lora_sgmv(const lora_table *table, const lora_segments *seg, const void *x, int64_t ldx,
              void *y, int64_t ldy, int32_t y_offset, void *ws, size_t ws_bytes, void *stream);

/* Grouped SGMV: P <= LORA_MAX_GROUP projections of one batch in one launch, e.g. the q, k and
 * v (and o) projections of a layer, each with its own adapter table but one shared segment
 * table (the same adapter id selects adapter i of every table).  Projection p computes
 * y[p][t, y_offset[p] + n] += s_i * (x[p][t] . A_i^T) . B_i^T exactly as lora_sgmv with
 * tables[p] would, and per output the arithmetic is the same as that call's, so results
 * match it bit for bit (at the same "decode_cluster" width).  The per-call y_offset /
 * y_slice_size of the pages' pseudocode ("Compress then Serve" review thread, add_lora_slice)
 * is what lets q, k and v write their slices of one fused output.
 * Arguments: host arrays of P entries (tables, x, ldx, y, ldy, y_offset); the tables must
 * have the same n, dtype and device; x[p] may repeat (q, k and v share x); the output
 * slices must not overlap (LORA_ERR_INVALID_ARG), because the projections update y
 * concurrently.  Device errors latch into tables[0]'s status word.  When a table qualifies
 * for the tcgen05 path (long contiguous segments) or the "split" option is set, the call
 * runs lora_sgmv once per table instead (ws as for lora_sgmv). */
#define LORA_MAX_GROUP 4
int lora_sgmv_grouped(const lora_table *const *tables, int32_t P, const lora_segments *seg,
                      const void *const *x, const int64_t *ldx, void *const *y, const int64_t *ldy,
                      const int32_t *y_offset, void *ws, size_t ws_bytes, void *stream);

/* Layer output with the frozen base weight, fused with the adapter term ("TGI Multi-LoRA"
 * page, "Technical Foundation: LoRA": the pretrained W stays frozen and the adapter adds
 * B A x; "predibase/lorax" repository page: one forward pass of the layer):
 *   y[t, y_offset + n] = (accumulate ? y[t, y_offset + n] : 0) + sum_j x[t, j] W[n, j]
 *                        + s_i * sum_k B_i[n, k] (x[t] . A_i[k])       (n < o)
 * for every token t < seg->T; tokens outside all segments get the first two terms only.
 * W is [o, ldw] row-major bf16 (a linear layer's weight; the first h columns are used),
 * 16-byte aligned, ldw a multiple of 8.  Runs on the tcgen05 tensor cores: the shrink stores
 * s_i * (x . A_i^T) as bf16 hi + lo in the workspace, then one persistent kernel accumulates
 * x W^T and that intermediate times B_i in the same tensor-memory tile and writes y once.
 * Requires a bf16 table whose ranks are multiples of 8 and at most 64 without Sigma, and
 * seg->perm == NULL (tokens contiguous per segment, segments in position order); otherwise
 * LORA_ERR_UNSUPPORTED.  accumulate is 0 or 1.  ws_bytes >= lora_workspace_bytes(table, T).
 * The products are rounded once, to bf16, per output (fp32 accumulation). */
int lora_sgmv_base(const lora_table *table, const lora_segments *seg, const void *x, int64_t ldx,
                   const void *W, int64_t ldw, void *y, int64_t ldy, int32_t y_offset,
                   int32_t accumulate, void *ws, size_t ws_bytes, void *stream);

/* BGMV: the same update driven by per-token ids (d_ids[T], device) without a caller-built
 * segment table, as the per-token "indices" of the pseudocode.  Tokens sharing an adapter
 * are grouped on the device so each adapter's weights are read once per group.  For
 * T <= 1024 and n <= 4096 this is one launch that needs no workspace; larger batches sort
 * into the workspace first. */
int lora_bgmv(const lora_table *table, const int32_t *d_ids, int32_t T, const void *x,
              int64_t ldx, void *y, int64_t ldy, int32_t y_offset, void *ws, size_t ws_bytes,
              void *stream);

/* Several adapters merged per token (the Lorax pages' per-request weighted ensembles):
 *   y[t, y_offset + n] += sum_{j < K, ids[t, j] >= 0} w[t, j] * s_i * (B_i (A_i x[t]))[n]
 * d_ids and d_w are [T, K] row-major DEVICE arrays (int32 ids, -1 = empty slot; fp32
 * weights), 1 <= K <= LORA_MAX_MERGE.  Runs one BGMV pass per slot, in slot order, with the
 * weight folded into the scale.  With a workspace of at least
 *   W + T * h_out * 4 bytes,   W = lora_workspace_bytes(table, T) rounded up to 256,
 * (16-byte aligned) the passes add into an fp32 sum held after the first W bytes (zeroed
 * first) and a last launch rounds y + sum once, as one weighted update; with less (or no)
 * workspace y is rounded to its type after each slot (K roundings).  Batches above 1024 tokens
 * or 4096 adapters sort each slot into the workspace (ws_bytes >= lora_workspace_bytes(table,
 * T)); otherwise ws may be NULL.  The "split" option does not apply. */
#define LORA_MAX_MERGE 8
int lora_bgmv_merged(const lora_table *table, const int32_t *d_ids, const float *d_w, int32_t T,
                     int32_t K, const void *x, int64_t ldx, void *y, int64_t ldy, int32_t y_offset,
                     void *ws, size_t ws_bytes, void *stream);

/* Read (and with reset != 0, clear) the table's device status word into *h_status.
 * Synchronises `stream`.  Returns LORA_OK when the word is 0, LORA_ERR_TIMEOUT when the
 * timeout bit is set, otherwise LORA_ERR_DEVICE_STATUS. */
int lora_get_status(const lora_table *table, uint32_t *h_status, int32_t reset, void *stream);

/* SGMV without any workspace from the caller.  There is no counterpart on the multi-LoRA
 * pages; it exists for callers that cannot allocate device memory themselves (a framework
 * that owns all GPU memory through its own allocator, a runtime with a fixed memory budget,
 * or a path where a cudaMalloc/cudaFree and the synchronisation it may bring is not allowed).
 * Same arguments and result as lora_sgmv minus the workspace: it runs lora_shrink into a
 * library-owned device array of LORA_NOALLOC_SCRATCH_FLOATS floats (1 MiB, held on every GPU
 * that loads the library until the process exits), then lora_expand from it.  Limit:
 * seg->T * ldv <= LORA_NOALLOC_SCRATCH_FLOATS with ldv = max rank rounded up to 4, else
 * LORA_ERR_WORKSPACE is returned and nothing is launched.  It calls no allocating routine.
 * The first call on a device looks up the array's address on that device (make that first
 * call outside any stream capture).  All calls share the one array: calls that can overlap on
 * the GPU (different streams, or different host threads) race on it and must be serialised by
 * the caller.  The array keeps the last call's contents; nothing relies on it starting at 0.
 * The current device must be the table's device (else LORA_ERR_INVALID_ARG).  The looked-up
 * address is kept for the life of the process, so the library must not be used on a device
 * after cudaDeviceReset (or any other teardown of that device's primary context). */
#define LORA_NOALLOC_SCRATCH_FLOATS 262144
int lora_sgmv_noalloc(const lora_table *table, const lora_segments *seg, const void *x, int64_t ldx,
                      void *y, int64_t ldy, int32_t y_offset, void *stream);

/* Static text for a return code. */
const char *lora_status_string(int code);

/* Runtime knobs (process-wide, for tuning and tests).  key: "pdl" (0/1, programmatic
 * dependent launch between consecutive calls), "decode_stages", "decode_ctas_per_sm",
 * "decode_cluster" (0: automatic, else 1, 2, 4 or 8 CTAs sharing one decode work unit; the
 * width changes the fp32 summation order, so results can differ in the last bits between
 * widths), "decode_max_clusters" (0: every co-resident cluster; else an upper bound on
 * the persistent decode grid, for tuning), "prefill_ksplit" (4, the default, or 8 CTAs splitting
 * h in the tcgen05 shrink), "prefill_min_seg_len" (segment-length hint at or above which lora_sgmv takes the tcgen05
 * path; 0 disables that path), "split" (1: lora_sgmv runs lora_shrink then lora_expand
 * through the workspace instead of the fused kernel), "wait_limit_ns" (bound of every
 * device-side wait of the following launches; 0: the default of about 2 s), "inject_stall"
 * (tests only: a bit mask, 1 decode kernels, 2 tcgen05 shrink, 4 tcgen05 expand, that arms one
 * pipeline stage per unit or tile without ever loading it, so the bounded wait on it runs
 * out, LORA_STATUS_TIMEOUT is latched and the kernel drains its copies, releases tensor
 * memory and returns; results are then invalid), "tc_min_seg_len" (segments at least this
 * long take the tcgen05 kernels in mixed batches; 0 disables that split), "tc_min_tokens"
 * (smallest batch that considers the split), "decode_balance" (segment tables on the cluster
 * kernel: -1, the default, cuts the units into runs of about equal estimated work per cluster
 * when the table's ranks differ by 2x or more, else deals them with a fixed stride; 0 always the
 * stride, 1 always the runs; results are bit-identical either way), "decode_shared_exchange"
 * (lora_sgmv_grouped on the cluster kernel: 1, the default, runs each unit's shrink tiles of
 * every projection first and exchanges their partials across the cluster once, then the
 * expand tiles; 0 exchanges once per projection; tables with Sigma_i always take the latter;
 * results are bit-identical either way).  Returns LORA_ERR_INVALID_ARG for an unknown key. */
int lora_set_option(const char *key, int64_t value);
int lora_get_option(const char *key, int64_t *value);

/* Launch counters (diagnostics, process-wide): the number of launches of each of the library's
 * kernels that the CUDA runtime has accepted since the library was loaded.  kind runs from 0 to
 * LORA_KERNEL_KINDS - 1 (0 the decode kernel, 1 and 2 the two segment-building kernels, 3 and
 * 4 the tcgen05 shrink and expand, 5 the fused base GEMM, 6 the merged ensembles' final
 * rounding).  lora_kernel_name returns the
 * kernel's name (static text; NULL outside that range) and lora_kernel_launches its count (-1
 * outside that range).  A count says that a launch was enqueued, not that it has finished;
 * lora_get_status reports what the device found.  Tests read them to see which path a call
 * took. */
#define LORA_KERNEL_KINDS 7
const char *lora_kernel_name(int32_t kind);
int64_t lora_kernel_launches(int32_t kind);

#ifdef __cplusplus
}
#endif

#endif /* LORA_SGMV_H */
