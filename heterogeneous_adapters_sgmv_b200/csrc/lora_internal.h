// Host-side internals shared by the translation units of liblora_sgmv.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "lora_sgmv.h"

struct CUtensorMap_st;
struct lora_table;

namespace lora {
struct AdapterDesc;

// Decode kernel modes: shrink+expand fused, shrink only (v to global), expand only (v from global).
enum DecodeMode : int { kModeFused = 0, kModeShrink = 1, kModeExpand = 2 };
// Where the work units come from: a segment table, or per-token ids grouped on the device.
enum UnitSource : int { kSrcSegments = 0, kSrcIds = 1 };

// One projection (one adapter table with its activations) of a decode launch.  A grouped
// launch carries up to kMaxProj of them over one segment table.
struct ProjParams {
    const AdapterDesc *desc;
    const void *tmA;       // device array of 128-byte tensor maps, one per adapter (A_i slices)
    const void *x;
    void *y;
    int64_t ldx, ldy;
    int32_t h, o;          // in/out features
    int32_t y_off;
    int32_t sigma_kind;    // LORA_SIGMA_* of the table
};
constexpr int kMaxProj = 4;

struct DecodeParams {
    ProjParams pj[kMaxProj];
    int32_t P;             // projections in this launch (1 unless grouped)
    int32_t n, R;          // adapters per table, max rank over the launch's tables
    int32_t ldv;
    float *v;
    const int32_t *perm, *seg_ptr, *seg_adapter, *num_segs;
    int32_t max_segs;
    const int32_t *ids;
    int32_t ids_stride;    // element stride of ids (slot k of a [T, K] ensemble: ids + k, stride K)
    const float *tok_w;    // per-token weights (merged ensembles), or null for weight 1
    int32_t w_stride;
    int32_t T;
    uint32_t *status;
    uint64_t wait_ns;      // bound of every device-side wait (option "wait_limit_ns")
    int32_t inject;        // test-only stall injection (option "inject_stall"), 0 in normal use
    int32_t long_len;      // segments of at least this many tokens are served elsewhere (0: none)
    int32_t balance;       // segment tables: cost-balanced runs of units per cluster (1) or a fixed stride (0)
    int32_t mx;            // grouped launch: one exchange per unit for all projections' shrinks (no Sigma)
    float *yacc;           // fused / expand: add the scaled delta to this fp32 [T, ldacc] array instead of
    int64_t ldacc;         // rounding it into y (merged ensembles summed before their one rounding), or null
    int32_t stages;        // pipeline depth
    int32_t stage_bytes;   // bytes of one stage (header + data)
    int32_t ids_smem;      // kSrcIds: bytes of the id / leader scratch in shared memory
};

struct Options {
    int64_t pdl = 1;
    int64_t decode_stages = 0;       // 0: automatic
    int64_t decode_ctas_per_sm = 0;  // 0: automatic
    int64_t decode_cluster = 0;      // 0: automatic; else 1, 2, 4 or 8 CTAs per cluster
    int64_t decode_max_clusters = 0; // 0: as many as are co-resident
    int64_t prefill_min_seg_len = 256;
    int64_t prefill_ksplit = 4;      // CTAs splitting h in the tcgen05 shrink (4 or 8)
    int64_t split = 0;
    int64_t wait_limit_ns = 0;       // 0: the default bound (about 2 s)
    int64_t inject_stall = 0;        // test-only: bit 0 decode, bit 1 prefill shrink, bit 2 prefill expand
    int64_t tc_min_seg_len = 64;     // mixed batches: segments this long take the tcgen05 kernels (0: never)
    int64_t tc_min_tokens = 1024;    // ... in batches of at least this many tokens
    int64_t decode_balance = -1;     // segment units: -1 by the tables' rank spread, 0 fixed stride, 1 balanced runs
    int64_t decode_shared_exchange = 1;  // grouped launches: one cluster exchange per unit for all projections
};
// Bound of the device-side waits for the next launch.
uint64_t wait_limit_ns();
Options &options();

// Host-side count of accepted launches per kernel (lora_kernel_launches).
enum KernelKind {
    kKernDecode = 0, kKernCountSegments, kKernBuildSegments, kKernPrefillShrink, kKernPrefillExpand,
    kKernBaseGemm, kKernMergeFinish, kKernKinds
};
void note_launch(KernelKind k);

// Launchers (return a LORA_* code).
int launch_decode(int mode, int src, const DecodeParams &p, int dtype, cudaStream_t s);
int launch_build_segments(const int32_t *ids, int32_t T, int32_t n, int32_t *perm, int32_t *seg_ptr,
                          int32_t *seg_adapter, int32_t *num_segs, uint32_t *status, cudaStream_t s);
// Tensor maps of every adapter for the tcgen05 prefill path (no-op when the table does not qualify).
int prefill_build_maps(lora_table *t);
// tcgen05 shrink alone (contiguous segments, prefill-capable table): v receives the bf16 hi and
// lo parts ([T, 64] each) of x . A_i^T, multiplied by s_i when fold_scale.
int launch_prefill_shrink(const lora_table *t, const lora_segments *seg, const void *x, int64_t ldx, void *v,
                          bool fold_scale, cudaStream_t s);
// Fused layer output (base_gemm.cu): y = (y if accumulate) + x W^T + the adapter term, from the
// scale-folded intermediate v that launch_prefill_shrink wrote.
// after_shrink: launch_prefill_shrink was the launch just before on `s` (lets the kernel start
// its base-product tiles before the shrink has finished).
int launch_base_gemm(const lora_table *t, const lora_segments *seg, const void *x, int64_t ldx, const void *W,
                     int64_t ldw, void *y, int64_t ldy, int32_t y_off, int accumulate, const void *v, bool after_shrink,
                     cudaStream_t s);
// y[t, y_off + n] = round(y[t, y_off + n] + yacc[t, n]) for t < T, n < o (merge.cu).
int launch_merge_finish(void *y, int64_t ldy, int32_t y_off, const float *yacc, int64_t ldacc, int32_t T, int32_t o,
                        int dtype, cudaStream_t s);
// Encode the TMA tensor map of A_i [rank, h] used by the decode shrink (host side).
int encode_tmap_A(void *out128, const void *A, int dtype, int h, int rank);

}  // namespace lora

struct lora_table {
    int32_t n, h, o, dtype, max_rank, min_rank;
    int device;
    lora::AdapterDesc *d_desc;
    uint32_t *d_status;
    std::vector<const void *> A, B;
    std::vector<int32_t> ranks;
    std::vector<float> scales;
    // per-adapter TMA tensor maps of A_i (device array of 128-byte CUtensorMap)
    void *d_tmaps;
    // prefill path (bf16, ranks multiple of 8 and <= 64): 128-byte-swizzled maps of A_i, B_i
    void *d_tmaps_pfA, *d_tmaps_pfB;
    // three-stage form: LORA_SIGMA_* and the per-adapter Sigma_i pointers (device, fp32)
    int32_t sigma_kind;
    std::vector<const float *> sigma;
};
