// Prefill path of the LoRA delta for long, contiguous segments on the 5th-generation tensor
// cores (tcgen05): per segment the shrink v = x . A_i^T (scale 1, fp32) and the expand
// y += s_i * v . B_i^T are dense contractions ("Compress then Serve" review thread,
// add_lora_slice pseudocode; "TGI Multi-LoRA" page, "Technical Foundation: LoRA").
//
// Shrink kernel: one cluster of KS CTAs (4, or 8 with the "prefill_ksplit" option) per
// (segment, 128-token tile); CTA j takes the j-th KS-th of h.  A producer thread streams x
// and A_i tiles (64 columns of h, 128-byte swizzle) with 2-D tensor-map TMA loads into a
// 4-deep ring; one thread issues tcgen05.mma (M = 128 tokens, N = rank rounded up to 16,
// K = 16) accumulating in tensor memory; the partials are summed in fixed CTA order through
// distributed shared memory, and the fp32 sum is stored as bf16 hi + lo (v = hi + lo to about
// 16 bits, zero past the rank).
//
// Expand kernel: persistent CTAs over the (128-token tile, 128-column tile of o) pairs.  Both
// parts of the intermediate come in by TMA, already in the 128-byte-swizzled K-major layout
// the tensor core reads, and are multiplied with the B_i tile (TMA) in 8 MMAs of K = 16.  The
// y tile arrives by TMA; the epilogue reads the accumulator from tensor memory row by row,
// adds s_i * acc to y in shared memory, rounds once to bf16, and writes a full tile back with
// TMA stores, a partial one with coalesced 16-byte stores masked to the segment, so
// neighbouring segments are never touched.
//
// No TMA multicast.  Every wait is bounded; on timeout a status bit is latched, in-flight
// copies are drained and tensor memory is released before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "lora_common.cuh"
#include "lora_internal.h"
#include "tcgen05.cuh"

namespace lora {
#ifdef LORA_TRACE
// instrumented builds only: per-CTA clock64 phase marks of the tcgen05 shrink
__device__ unsigned long long lora_trace_shrink[4096 * 16];
#define SHRINK_MARK(slot)                                                              \
    do {                                                                               \
        if (blockIdx.x < 4096u) ::lora::lora_trace_shrink[blockIdx.x * 16 + (slot)] = clock64(); \
    } while (0)
// and per-tile marks of the persistent expand: [CTA][tile 0..63, 64 = start][event 0..3]
__device__ unsigned long long lora_trace_expand[160 * 65 * 4];
#define EXPAND_MARK(i, e)                                                                          \
    do {                                                                                           \
        if (blockIdx.x < 160u && (i) <= 64) ::lora::lora_trace_expand[(blockIdx.x * 65 + (i)) * 4 + (e)] = clock64(); \
    } while (0)
#define EXPAND_GMARK(e)                                                                            \
    do {                                                                                           \
        if (blockIdx.x < 160u) ::lora::lora_trace_expand[(blockIdx.x * 65 + 64) * 4 + (e)] = globaltimer_ns(); \
    } while (0)
#else
#define EXPAND_GMARK(e) \
    do {                \
    } while (0)
#define SHRINK_MARK(slot) \
    do {                  \
    } while (0)
#define EXPAND_MARK(i, e) \
    do {                  \
    } while (0)
#endif
namespace {

constexpr int kTileM = 128;          // tokens per tile
constexpr int kTileN = 128;          // columns of o per expand tile
constexpr int kBK = 64;              // columns of h per shrink k-block (128 bytes of bf16)
constexpr int kStagesMax = 4;        // shrink pipeline depth
// (eight stages with the split of 4 measured slower: 17.4 against 16.3 us)
__host__ __device__ constexpr int shrink_stages(int) { return 4; }
constexpr int kThreadsPF = 128;      // 4 warps: one TMEM lane quarter each
constexpr int kMaxRankPF = 64;

struct PrefillParams {
    CUtensorMap tmap_io;          // shrink: x [T, h]; expand: y slice [T, o]   (box 64 x 128)
    CUtensorMap tmap_vhi, tmap_vlo;   // expand: intermediate hi / lo parts [T, 64] bf16 (box 64 x 128)
    const AdapterDesc *desc;
    const uint8_t *tm_A;          // per adapter: tensor map of A_i, box 64 x roundup(r, 16)
    const uint8_t *tm_B;          // per adapter: tensor map of B_i, box 64 x 128
    const int32_t *seg_ptr, *seg_adapter, *num_segs;
    int32_t max_segs, T, h, o, n;
    uint16_t *v_hi, *v_lo;        // the fp32 intermediate as bf16 hi + lo, [T, 64] each, zero past the rank
    void *y;
    int64_t ldy;
    int32_t y_off;
    uint32_t *status;
    uint64_t wait_ns;             // bound of every device-side wait
    int32_t inject;               // test-only stall injection: bit 1 shrink, bit 2 expand
    int32_t fold_scale;           // shrink: store s_i * v instead of v (fused base product)
    const int32_t *perm;          // token of each sorted position, or null (tokens contiguous)
    int32_t min_len;              // only segments of at least this many tokens (0: all)
    CUtensorMap tmap_g;           // perm: x [T, h] (shrink) or the y slice (expand), box 64 x 1
    int32_t *tile_ctr;            // expand: next tile of the shared pool (zeroed by the shrink), or null
};

// 4-row gather (TMA tile::gather4, one-row box, 128-byte swizzle) of columns [c0, c0 + 64) of
// rows r0..r3 into 512 bytes of shared memory, counted on `bar`.  The rows land exactly as
// rows 4k .. 4k + 3 of a tiled box would at the same shared-memory offset.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const void *tmap, int32_t c0, int32_t r0, int32_t r1,
                                            int32_t r2, int32_t r3, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
        : "memory");
}

// Tokens of rows 4 lane .. 4 lane + 3 of a tile at sorted positions [row0, row0 + rows): rows
// past the tile repeat its last row (their results are never stored); an entry outside [0, T)
// latches LORA_STATUS_BAD_SEGMENT and reads row 0 instead.
__device__ __forceinline__ void tile_tokens(const PrefillParams &p, int row0, int rows, int tk[4])
{
    const int lane = threadIdx.x & 31;
    bool bad = false;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int r = min(4 * lane + q, rows - 1);
        int t = p.perm[row0 + r];
        if (t < 0 || t >= p.T) {
            bad = true;
            t = 0;
        }
        tk[q] = t;
    }
    if (bad) atomicOr(p.status, LORA_STATUS_BAD_SEGMENT);
}

// Map a global 128-token tile index to (segment, first row, rows).  One warp scans the
// segment table 32 entries at a time; each lane loads its entry's bounds and adapter together
// with the segment count (one round trip per window rather than one per dependent value).
// Returns false when the index is past the last tile.
__device__ bool find_tile(const PrefillParams &p, int g, int *seg, int *row0, int *rows, int *adapter)
{
    const int lane = threadIdx.x & 31;
    const int ns_raw = *p.num_segs;
    int base_tiles = 0;
    for (int s0 = 0; s0 < p.max_segs; s0 += 32) {
        const int s = s0 + lane;
        int p0 = 0, p1 = 0, a = -1;
        if (s < p.max_segs) {
            p0 = p.seg_ptr[s];
            p1 = p.seg_ptr[s + 1];
            a = p.seg_adapter[s];
        }
        const int nseg = min(ns_raw, p.max_segs);
        if (s0 >= nseg) break;
        int len = (s < nseg) ? max(0, min(p1, p.T) - max(p0, 0)) : 0;   // bad bounds: empty
        if (len < p.min_len) len = 0;   // a short segment is served by the decode kernel
        const int tiles = (len + kTileM - 1) / kTileM;
        int incl = tiles;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += o;
        }
        const int excl = base_tiles + incl - tiles;
        const bool hit = (g >= excl) && (g < excl + tiles);
        const uint32_t m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            const int start = max(__shfl_sync(0xffffffffu, p0, src), 0);
            const int end = min(__shfl_sync(0xffffffffu, p1, src), p.T);
            *seg = s0 + src;
            *row0 = start + (g - __shfl_sync(0xffffffffu, excl, src)) * kTileM;
            *rows = min(kTileM, end - *row0);
            *adapter = __shfl_sync(0xffffffffu, a, src);
            return true;
        }
        base_tiles += __shfl_sync(0xffffffffu, incl, 31);
    }
    return false;
}

struct __align__(8) ShrinkCtl {
    uint64_t full[kStagesMax];
    uint64_t empty[kStagesMax];
    uint64_t done;
    uint32_t tmem_base;
    int32_t info[5];   // valid, row0, rows, adapter, rank
    float scale;       // multiplier of the stored intermediate (1, or s_i when folding)
};

template <int KS>
__global__ void __launch_bounds__(kThreadsPF, 1) prefill_shrink_kernel(const __grid_constant__ PrefillParams p)
{
    constexpr int kRowsPerCta = kTileM / KS;   // rows of the tile each CTA reduces
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int kXBytes = kTileM * 128;              // 16 KiB
    constexpr int kABytes = kMaxRankPF * 128;          //  8 KiB (room for rank <= 64)
    constexpr int kStageBytes = kXBytes + kABytes;
    constexpr int kStages = shrink_stages(KS);
    ShrinkCtl &ctl = *reinterpret_cast<ShrinkCtl *>(smem + kStages * kStageBytes);
    float *part = reinterpret_cast<float *>(smem);     // [128][PRS] fp32, reuses the ring after the MMAs
    constexpr int PRS = kMaxRankPF + 4;                // padded row stride of the partial

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t crank = cluster_ctarank();
    const int g = (int)cluster_id_x();

    if (tid == 0) SHRINK_MARK(0);
    // set-up that touches no global memory runs before the wait on the previous kernel
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(smem_u32(&ctl.full[i]), 1);
            mbar_init(smem_u32(&ctl.empty[i]), 1);
        }
        mbar_init(smem_u32(&ctl.done), 1);
        fence_mbar_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctl.tmem_base), 64);
        tmem_relinquish();
    }
    pdl_wait();
    pdl_launch_dependents();
    if (tid == 0) SHRINK_MARK(1);
    // the expand that follows deals the last tiles from a shared counter; the wait above means
    // the previous expand on this workspace has finished with it
    if (blockIdx.x == 0 && tid == 0 && p.tile_ctr) *p.tile_ctr = 0;

    if (warp == 0) {
        int s, row0 = 0, rows = 0, a = 0;
        const bool ok = find_tile(p, g, &s, &row0, &rows, &a);
        if (lane == 0) {
            const bool good = ok && a >= 0 && a < p.n && rows > 0;
            if (ok && !good && crank == 0) atomicOr(p.status, LORA_STATUS_BAD_SEGMENT);
            ctl.info[0] = good ? 1 : 0;
            ctl.info[1] = row0;
            ctl.info[2] = rows;
            ctl.info[3] = a;
            ctl.info[4] = good ? p.desc[a].rank : 0;
            ctl.scale = (good && p.fold_scale) ? p.desc[a].scale : 1.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool valid = ctl.info[0] != 0;
    const int row0 = ctl.info[1], rows = ctl.info[2], a = ctl.info[3], r = ctl.info[4];
    const float vscale = ctl.scale;
    if (tid == 0) SHRINK_MARK(2);
    const int npad = (r + 15) & ~15;
    const uint32_t tmem = ctl.tmem_base;
    const int nkb_all = (p.h + kBK - 1) / kBK;
    const int kb0 = (int)((int64_t)crank * nkb_all / KS);
    const int kb1 = (int)((int64_t)(crank + 1) * nkb_all / KS);
    const int nkb = valid ? kb1 - kb0 : 0;
    bool ok = true;

    if (valid && nkb > 0) {
        if (warp == 0) {
            // producer: x tile (128 tokens x 64 columns) and A_i tile (npad rows x 64 columns);
            // with a permutation each lane gathers four of the tile's token rows
            const void *tA = p.tm_A + (size_t)a * 128;
            const uint32_t bytes = (uint32_t)(kXBytes + npad * 128);
            int tk[4] = {0, 0, 0, 0};
            if (p.perm) tile_tokens(p, row0, rows, tk);
            int issued = 0;
            bool stalled = false;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kStages, m = kb / kStages;
                if (m >= 1 &&
                    !__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.empty[s]), (m - 1) & 1, p.status, p.wait_ns))) {
                    stalled = true;
                    break;
                }
                uint8_t *st = smem + s * kStageBytes;
                const uint32_t fb = smem_u32(&ctl.full[s]);
                ++issued;
                const int k0 = (kb0 + kb) * kBK;
                // test-only stall: the first k-block is armed but never loaded
                const bool load = !((p.inject & 2) && kb == 0);
                if (lane == 0) {
                    mbar_arrive_expect_tx(fb, bytes);
                    if (load) {
                        if (!p.perm) tma_load_2d(smem_u32(st), &p.tmap_io, k0, row0, fb);
                        tma_load_2d(smem_u32(st + kXBytes), tA, k0, 0, fb);
                    }
                }
                __syncwarp();
                if (p.perm && load) tma_gather4(smem_u32(st + lane * 512), &p.tmap_g, k0, tk[0], tk[1], tk[2], tk[3], fb);
                if (lane == 0 && kb == 0) SHRINK_MARK(3);
            }
            // After a timeout the ring is given up early: wait (bounded) for the copies of the
            // last stages issued, so none is still writing when the ring is reused below.
            if (lane == 0 && (stalled || (p.inject & 2)))
                for (int kb = max(0, issued - kStages); kb < issued; ++kb)
                    mbar_wait(smem_u32(&ctl.full[kb % kStages]), (kb / kStages) & 1, p.status, p.wait_ns);
        } else if (warp == 1 && lane == 0) {
            // MMA issuer
            const uint32_t idesc = idesc_bf16(kTileM, npad);
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kStages, m = kb / kStages;
                if (!mbar_wait(smem_u32(&ctl.full[s]), m & 1, p.status, p.wait_ns)) break;
                tc_fence_after();
                if (kb == 0) SHRINK_MARK(4);
                if (kb == nkb - 1) SHRINK_MARK(5);
                uint8_t *st = smem + s * kStageBytes;
                const uint64_t ad = sw128_desc(smem_u32(st));
                const uint64_t bd = sw128_desc(smem_u32(st + kXBytes));
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k)
                    umma_bf16(tmem, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                umma_commit(smem_u32(&ctl.empty[s]));
            }
            umma_commit(smem_u32(&ctl.done));
        }
        __syncwarp();
        ok = mbar_wait(smem_u32(&ctl.done), 0, p.status, p.wait_ns);
        tc_fence_after();
        if (tid == 0) SHRINK_MARK(6);
    }
    // ---- epilogue: partial [128][npad] from tensor memory (zeros when this CTA had no k-blocks)
    // The ring is free: all MMAs and loads that fed them are complete.  A wait that ran out in
    // any thread makes every thread skip the (warp-collective) tensor-memory loads.
    ok = __syncthreads_and(ok) != 0;
    const int m = warp * 32 + lane;   // row of the tile = TMEM lane
    if (valid) {
        for (int c0 = 0; c0 < npad; c0 += 32) {
            float acc[32];
            if (nkb > 0 && ok) {
                tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, acc);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (c0 + i < npad) part[m * PRS + c0 + i] = acc[i];
        }
    }
    if (tid == 0) SHRINK_MARK(7);
    cluster_sync_all();   // every CTA's partial is visible to its peers
    if (tid == 0) SHRINK_MARK(8);
    if (valid) {
        // CTA j reduces rows [16 j, 16 j + 16) over the 8 partials, in CTA order
        const uint32_t part_addr = smem_u32(part);
        // Four columns per load (r is a multiple of 8 on this path; same order of additions).
        // The sum is stored as bf16 hi + lo (v = hi + lo to about 16 bits), the layout the
        // expand's tensor-core operand takes by TMA; columns past r are zero.
        constexpr int q4all = kMaxRankPF / 4;
        const int q4 = r >> 2;
        for (int e = tid; e < kRowsPerCta * q4all; e += kThreadsPF) {
            const int rr = crank * kRowsPerCta + e / q4all, kq = e % q4all, k = kq * 4;
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            if (kq < q4) {
                float4 pv[KS];
#pragma unroll
                for (int j = 0; j < KS; ++j) pv[j] = ld_dsmem_f32x4(part_addr + 4u * (rr * PRS + k), j);
#pragma unroll
                for (int j = 0; j < KS; ++j) {
                    sum.x += pv[j].x;
                    sum.y += pv[j].y;
                    sum.z += pv[j].z;
                    sum.w += pv[j].w;
                }
            }
            if (rr < rows) {
                sum.x *= vscale;   // exact when the scale is 1
                sum.y *= vscale;
                sum.z *= vscale;
                sum.w *= vscale;
                const __nv_bfloat162 h01 = __floats2bfloat162_rn(sum.x, sum.y);
                const __nv_bfloat162 h23 = __floats2bfloat162_rn(sum.z, sum.w);
                const float2 g01 = __bfloat1622float2(h01), g23 = __bfloat1622float2(h23);
                const __nv_bfloat162 l01 = __floats2bfloat162_rn(sum.x - g01.x, sum.y - g01.y);
                const __nv_bfloat162 l23 = __floats2bfloat162_rn(sum.z - g23.x, sum.w - g23.y);
                const int64_t off = (int64_t)(row0 + rr) * kMaxRankPF + k;
                *reinterpret_cast<uint2 *>(p.v_hi + off) =
                    make_uint2(*reinterpret_cast<const uint32_t *>(&h01), *reinterpret_cast<const uint32_t *>(&h23));
                *reinterpret_cast<uint2 *>(p.v_lo + off) =
                    make_uint2(*reinterpret_cast<const uint32_t *>(&l01), *reinterpret_cast<const uint32_t *>(&l23));
            }
        }
    }
    if (tid == 0) SHRINK_MARK(9);
    cluster_sync_all();   // no peer reads this CTA's partial any more
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 64);
    if (tid == 0) SHRINK_MARK(10);
}

// ----------------------------------------------------------------------------------------
// Persistent expand: CTA b walks tiles [b * total / G, (b + 1) * total / G) of the
// (128-token tile, 128-column tile) grid, columns fastest, so consecutive tiles share the
// intermediate tile.  Warp roles:
//   warp 0      producer: loads the bf16 hi + lo intermediate tile (double-buffered) when the
//               token tile changes, and streams y tiles (4-stage ring) and B_i tiles (2-stage
//               ring: the MMA releases a B tile as soon as it has read it, while a y tile is
//               held through the epilogue and its store) by TMA;
//   warp 1      MMA issuer (one thread) into two TMEM accumulators used alternately;
//   warps 2..9  epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 and columns
//               64 ((w - 2) / 4) .. +63, adds s * acc to y in place in shared memory; a full
//               tile goes back by two TMA stores, whose shared-memory reads are awaited only at
//               the next tile (the y stage is released one tile late, the epilogue moves on at
//               once); a partial tile by coalesced 16-byte stores masked to the segment.
constexpr int kEpiWarps = 8;
constexpr int kThreadsEX = (2 + kEpiWarps) * 32;
constexpr int kExYStages = 4;
constexpr int kExBStages = 2;
constexpr int kExYBytes = 32768;                       // y tile: two 64-column boxes of 128 rows
constexpr int kExBBytes = 16384;                       // B_i tile: 128 rows of o x 64 ranks
constexpr int kExVBytes = 32768;                       // hi + lo intermediate tile
constexpr int kExPoolPerCta = 3;                       // tiles per CTA dealt from the shared pool
constexpr int kExPreTiles = 1;                         // tiles loaded before the wait on the shrink
                                                       // (<= kExBStages; 2 measured 0.3 us slower)

struct ExTileInfo {
    int32_t row0, rows, col0, ncols, vb;
    float scale;
};

struct __align__(8) ExpandCtl {
    uint64_t yfull[kExYStages], yempty[kExYStages];
    uint64_t bfull[kExBStages], bempty[kExBStages];
    uint64_t vfull[2], vempty[2];
    uint64_t accfull[2], accempty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int32_t total_m;
    ExTileInfo info[kExYStages];   // per y stage; written before the tile's B and y loads are armed
};

__device__ int count_m_tiles(const PrefillParams &p)
{
    const int lane = threadIdx.x & 31;
    const int ns_raw = *p.num_segs;
    int tot = 0;
    for (int s0 = 0; s0 < p.max_segs; s0 += 32) {
        const int s = s0 + lane;
        int p0 = 0, p1 = 0;
        if (s < p.max_segs) {
            p0 = p.seg_ptr[s];
            p1 = p.seg_ptr[s + 1];
        }
        const int nseg = min(ns_raw, p.max_segs);
        if (s0 >= nseg) break;
        int len = (s < nseg) ? max(0, min(p1, p.T) - max(p0, 0)) : 0;
        if (len < p.min_len) len = 0;
        int tiles = (len + kTileM - 1) / kTileM;
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) tiles += __shfl_xor_sync(0xffffffffu, tiles, d);
        tot += tiles;
    }
    return tot;
}

__global__ void __launch_bounds__(kThreadsEX, 1) prefill_expand_kernel(const __grid_constant__ PrefillParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *vbuf = smem;                                    // [2][hi 16 KiB | lo 16 KiB]
    uint8_t *yring = smem + 2 * kExVBytes;                   // [kExYStages][y 32 KiB]
    uint8_t *bring = yring + kExYStages * kExYBytes;         // [kExBStages][B 16 KiB]
    ExpandCtl &ctl = *reinterpret_cast<ExpandCtl *>(bring + kExBStages * kExBBytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NT = (p.o + kTileN - 1) / kTileN;
    if (tid == 0) EXPAND_MARK(64, 0);
    if (tid == 0) EXPAND_GMARK(2);

    if (tid == 0) {
        for (int i = 0; i < kExYStages; ++i) {
            mbar_init(smem_u32(&ctl.yfull[i]), 1);
            mbar_init(smem_u32(&ctl.yempty[i]), kEpiWarps);
        }
        for (int i = 0; i < kExBStages; ++i) {
            mbar_init(smem_u32(&ctl.bfull[i]), 1);
            mbar_init(smem_u32(&ctl.bempty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&ctl.vfull[i]), 1);
            mbar_init(smem_u32(&ctl.vempty[i]), 1);
            mbar_init(smem_u32(&ctl.accfull[i]), 1);
            mbar_init(smem_u32(&ctl.accempty[i]), kEpiWarps);
        }
        mbar_init(smem_u32(&ctl.mma_done), 1);
        fence_mbar_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctl.tmem_base), 256);
        tmem_relinquish();
    }
    // The shrink that precedes this kernel writes only the intermediate and the tile counter,
    // and it lets this grid launch only after its own wait on everything before it: the
    // segment table, y and the weights are final already.  Only the producer's intermediate
    // loads and counter grabs wait for the shrink (below).
    pdl_launch_dependents();
    if (warp == 0) {
        const int tm = count_m_tiles(p);
        if (lane == 0) ctl.total_m = tm;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) EXPAND_MARK(64, 1);
    const uint32_t tmem = ctl.tmem_base;
    const int total = ctl.total_m * NT;
    // Each CTA first takes a contiguous share of the tiles (consecutive tiles share the
    // intermediate tile); the last ~kExPoolPerCta per CTA form a pool dealt one at a time
    // from a counter, so CTAs that started late or ran slow take fewer of them.  Without a
    // counter every tile is in the contiguous shares.
    const int G = (int)gridDim.x, b = (int)blockIdx.x;
    const int S = p.tile_ctr ? max(0, total / G - kExPoolPerCta) : 0;
    const int t0 = p.tile_ctr ? b * S : (int)((int64_t)b * total / G);
    const int t1 = p.tile_ctr ? t0 + S : (int)((int64_t)(b + 1) * total / G);
    const int pool0 = G * S;   // first pool tile (with a counter)
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int cur_g = -1, vcount = 0, row0 = 0, rows = 0, a = 0, vb = 0, nissued = 0;
        int tk[4] = {0, 0, 0, 0};   // with a permutation: tokens of rows 4 lane .. 4 lane + 3
        float sc = 0.f;
        int grab = 0;   // lane 0: pool index taken ahead of its use
        // The first tiles of the share (kExPreTiles, within one token tile): their y and B_i
        // tiles are loaded before the wait on the shrink (tile info included); the loop then
        // adds the intermediate load.
        int npre = 0;
        if ((p.tile_ctr ? S >= 1 : t0 < t1) && !(p.inject & 4)) {
            const int g = t0 / NT;
            int sg;
            if (!find_tile(p, g, &sg, &row0, &rows, &a) || a < 0 || a >= p.n) {
                if (lane == 0 && t0 - g * NT == 0) atomicOr(p.status, LORA_STATUS_BAD_SEGMENT);
                row0 = 0;
                rows = 0;
                a = 0;
            }
            sc = p.desc[a].scale;
            cur_g = g;
            if (p.perm && rows > 0) tile_tokens(p, row0, rows, tk);
            const int avail = p.tile_ctr ? S : t1 - t0;
            for (int i = 0; i < kExPreTiles && i < avail && (t0 + i) / NT == g; ++i) {
                const int nt = t0 + i - g * NT;
                if (lane == 0) {
                    EXPAND_MARK(i, 0);
                    ExTileInfo &inf = ctl.info[i];
                    inf.row0 = row0;
                    inf.rows = rows;
                    inf.col0 = nt * kTileN;
                    inf.ncols = min(kTileN, p.o - nt * kTileN);
                    inf.vb = 0;
                    inf.scale = sc;
                    uint8_t *yst = yring + i * kExYBytes;
                    const uint32_t yb = smem_u32(&ctl.yfull[i]), bb = smem_u32(&ctl.bfull[i]);
                    mbar_arrive_expect_tx(yb, kExYBytes);
                    mbar_arrive_expect_tx(bb, kExBBytes);
                    tma_load_2d(smem_u32(bring + i * kExBBytes), p.tm_B + (size_t)a * 128, 0, nt * kTileN, bb);
                    if (!p.perm) {
                        tma_load_2d(smem_u32(yst), &p.tmap_io, nt * kTileN, row0, yb);
                        tma_load_2d(smem_u32(yst + 16384), &p.tmap_io, nt * kTileN + 64, row0, yb);
                    }
                }
                __syncwarp();
                if (p.perm) {
                    const uint32_t yst = smem_u32(yring + i * kExYBytes), yb = smem_u32(&ctl.yfull[i]);
                    tma_gather4(yst + lane * 512, &p.tmap_g, nt * kTileN, tk[0], tk[1], tk[2], tk[3], yb);
                    tma_gather4(yst + 16384 + lane * 512, &p.tmap_g, nt * kTileN + 64, tk[0], tk[1], tk[2], tk[3],
                                yb);
                }
                __syncwarp();
                ++npre;
            }
        }
        pdl_wait();
        for (int i = 0; ok; ++i) {
            // the tile of stage i: the share, then pool tiles (the next index is taken one tile
            // ahead, so the counter's round trip overlaps the tile before)
            int t;
            if (!p.tile_ctr) {
                t = t0 + i;
                if (t >= t1) break;
            } else {
                if (lane == 0 && i == max(S - 1, 0)) grab = atomicAdd(p.tile_ctr, 1);
                if (i < S) {
                    t = t0 + i;
                } else {
                    t = pool0 + __shfl_sync(0xffffffffu, grab, 0);
                    if (t >= total) break;
                    if (lane == 0) grab = atomicAdd(p.tile_ctr, 1);
                }
            }
            const int sy = i % kExYStages, sb = i % kExBStages;
            const int g = t / NT, nt = t - g * NT;
            const bool pre_i = i < npre;   // this tile's y and B_i are loaded already
            const bool pre_v = i == 0 && npre > 0;   // its token tile was found above
            if (g != cur_g || pre_v) {
                int sg;
                if (pre_v) {
                    // (tile found above)
                } else if (!find_tile(p, g, &sg, &row0, &rows, &a) || a < 0 || a >= p.n) {
                    // a bad segment entry: keep the pipeline fed, store nothing for this tile
                    if (lane == 0 && nt == 0) atomicOr(p.status, LORA_STATUS_BAD_SEGMENT);
                    row0 = 0;
                    rows = 0;
                    a = 0;
                }
                if (!pre_v) {
                    sc = p.desc[a].scale;
                    cur_g = g;
                    if (p.perm && rows > 0) tile_tokens(p, row0, rows, tk);
                }
                vb = vcount & 1;
                if (vcount >= 2 && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.vempty[vb]),
                                                                     ((vcount >> 1) - 1) & 1, p.status, p.wait_ns))) {
                    ok = false;
                    break;
                }
                // intermediate tile: hi and lo parts (128 rows x 64 columns each) by TMA; rows
                // past the segment belong to no output of this tile and are masked at the store
                if (lane == 0) {
                    uint8_t *vhi = vbuf + vb * kExVBytes;
                    const uint32_t vf = smem_u32(&ctl.vfull[vb]);
                    mbar_arrive_expect_tx(vf, (uint32_t)kExVBytes);
                    tma_load_2d(smem_u32(vhi), &p.tmap_vhi, 0, row0, vf);
                    tma_load_2d(smem_u32(vhi + 16384), &p.tmap_vlo, 0, row0, vf);
                }
                __syncwarp();
                ++vcount;
            }
            if (i >= kExYStages && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.yempty[sy]),
                                                                      ((i / kExYStages) - 1) & 1, p.status, p.wait_ns))) {
                ok = false;
                break;
            }
            if (i >= kExBStages && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.bempty[sb]),
                                                                      ((i / kExBStages) - 1) & 1, p.status, p.wait_ns))) {
                ok = false;
                break;
            }
            // test-only stall: the first tile's stages are armed but never loaded
            const bool load = !((p.inject & 4) && i == 0);
            if (lane == 0 && !pre_i) {
                EXPAND_MARK(i, 0);
                ExTileInfo &inf = ctl.info[sy];
                inf.row0 = row0;
                inf.rows = rows;
                inf.col0 = nt * kTileN;
                inf.ncols = min(kTileN, p.o - nt * kTileN);
                inf.vb = vb;
                inf.scale = sc;
                uint8_t *yst = yring + sy * kExYBytes;
                const uint32_t yb = smem_u32(&ctl.yfull[sy]), bb = smem_u32(&ctl.bfull[sb]);
                mbar_arrive_expect_tx(yb, kExYBytes);
                mbar_arrive_expect_tx(bb, kExBBytes);
                if (load) {
                    tma_load_2d(smem_u32(bring + sb * kExBBytes), p.tm_B + (size_t)a * 128, 0, nt * kTileN, bb);
                    if (!p.perm) {
                        tma_load_2d(smem_u32(yst), &p.tmap_io, nt * kTileN, row0, yb);
                        tma_load_2d(smem_u32(yst + 16384), &p.tmap_io, nt * kTileN + 64, row0, yb);
                    }
                }
            }
            __syncwarp();
            if (p.perm && load && !pre_i) {   // the y tile's rows, four per lane
                const uint32_t yst = smem_u32(yring + sy * kExYBytes);
                const uint32_t yb = smem_u32(&ctl.yfull[sy]);
                tma_gather4(yst + lane * 512, &p.tmap_g, nt * kTileN, tk[0], tk[1], tk[2], tk[3], yb);
                tma_gather4(yst + 16384 + lane * 512, &p.tmap_g, nt * kTileN + 64, tk[0], tk[1], tk[2], tk[3], yb);
            }
            ++nissued;
            __syncwarp();
        }
        // end of the tiles: a stage whose info has rows = -1, with its barriers completed by
        // plain arrivals, tells the MMA issuer and the epilogue to stop
        int sentinel = 0;
        if (ok) {
            const int i = nissued, sy = i % kExYStages, sb = i % kExBStages;
            const bool oky = i < kExYStages || __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.yempty[sy]),
                                                                                   ((i / kExYStages) - 1) & 1,
                                                                                   p.status, p.wait_ns));
            const bool okb = i < kExBStages || __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.bempty[sb]),
                                                                                   ((i / kExBStages) - 1) & 1,
                                                                                   p.status, p.wait_ns));
            if (oky && okb && lane == 0) {
                ctl.info[sy].rows = -1;
                mbar_arrive(smem_u32(&ctl.yfull[sy]));
                mbar_arrive(smem_u32(&ctl.bfull[sb]));
            }
            sentinel = (oky && okb) ? 1 : 0;
            __syncwarp();
        }
        // drain: every TMA issued by this CTA has landed before shared memory is released.  The
        // stages of the last tiles armed hold the loads still in flight; earlier tiles' stages
        // were consumed before reuse (the end-of-tiles stage reused one more of each ring, and
        // waiting on that stage's older phase would never succeed).
        const int n = nissued;
        if (lane == 0) {
            for (int i = max(0, n + sentinel - kExYStages); i < n; ++i)
                mbar_wait(smem_u32(&ctl.yfull[i % kExYStages]), (i / kExYStages) & 1, p.status, p.wait_ns);
            for (int i = max(0, n + sentinel - kExBStages); i < n; ++i)
                mbar_wait(smem_u32(&ctl.bfull[i % kExBStages]), (i / kExBStages) & 1, p.status, p.wait_ns);
            for (int c = max(0, vcount - 2); c < vcount; ++c)
                mbar_wait(smem_u32(&ctl.vfull[c & 1]), (c >> 1) & 1, p.status, p.wait_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(kTileM, kTileN);
            int vuse = 0, prev_vb = -1;
            for (int i = 0;; ++i) {
                const int sy = i % kExYStages, sb = i % kExBStages, ab = i & 1;
                if (!mbar_wait(smem_u32(&ctl.bfull[sb]), (i / kExBStages) & 1, p.status, p.wait_ns)) break;
                EXPAND_MARK(i, 1);
                if (ctl.info[sy].rows < 0) {
                    // end of the tiles: complete the accumulator barrier the epilogue waits on
                    // next (once it is done with this accumulator's previous tile)
                    if (i < 2 || mbar_wait(smem_u32(&ctl.accempty[ab]), ((i >> 1) - 1) & 1, p.status, p.wait_ns))
                        umma_commit(smem_u32(&ctl.accfull[ab]));
                    break;
                }
                const int vb = ctl.info[sy].vb;
                if (vb != prev_vb) {
                    if (prev_vb >= 0) umma_commit(smem_u32(&ctl.vempty[prev_vb]));   // old tile may be rebuilt
                    if (!mbar_wait(smem_u32(&ctl.vfull[vb]), (vuse >> 1) & 1, p.status, p.wait_ns)) break;
                    ++vuse;
                    prev_vb = vb;
                }
                if (i >= 2 && !mbar_wait(smem_u32(&ctl.accempty[ab]), ((i >> 1) - 1) & 1, p.status, p.wait_ns)) break;
                tc_fence_after();
                const uint64_t dh = sw128_desc(smem_u32(vbuf + vb * kExVBytes));
                const uint64_t dl = sw128_desc(smem_u32(vbuf + vb * kExVBytes + 16384));
                const uint64_t db = sw128_desc(smem_u32(bring + sb * kExBBytes));
                const uint32_t acc = tmem + (uint32_t)(ab * kTileN);
#pragma unroll
                for (int k = 0; k < 4; ++k) umma_bf16(acc, dh + 2 * k, db + 2 * k, idesc, k != 0 ? 1u : 0u);
#pragma unroll
                for (int k = 0; k < 4; ++k) umma_bf16(acc, dl + 2 * k, db + 2 * k, idesc, 1u);
                umma_commit(smem_u32(&ctl.accfull[ab]));
                umma_commit(smem_u32(&ctl.bempty[sb]));
            }
            // every MMA of this CTA has completed before tensor memory is released
            umma_commit(smem_u32(&ctl.mma_done));
            mbar_wait(smem_u32(&ctl.mma_done), 0, p.status, p.wait_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quarter
        const int half = (warp - 2) >> 2;       // column half of the tile
        const int m = q * 32 + lane;            // row of the tile
        const int ew = warp - 2;                // epilogue warp 0..7
        int pending = -1;                       // ew 0: y stage whose TMA store is still reading it
        for (int i = 0;; ++i) {
            const int sy = i % kExYStages, ab = i & 1;
            // every epilogue warp leaves together if any lane ran out of time (the tensor-memory
            // loads below are warp-collective and the warps meet at a named barrier)
            const bool oka = mbar_wait(smem_u32(&ctl.accfull[ab]), (i >> 1) & 1, p.status, p.wait_ns);
            const bool okf = mbar_wait(smem_u32(&ctl.yfull[sy]), (i / kExYStages) & 1, p.status, p.wait_ns);
            if (!named_bar_and(3, kEpiWarps * 32, oka && okf)) break;
            tc_fence_after();
            if (ew == 0 && lane == 0) EXPAND_MARK(i, 2);
            const ExTileInfo inf = ctl.info[sy];
            if (inf.rows < 0) break;   // end of the tiles (the same for every thread)
            uint8_t *yt = yring + sy * kExYBytes + half * 16384;   // this half's 64-column box
            float acc[64];
            tmem_ld64(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * kTileN + half * 64), acc);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl.accempty[ab]));   // the accumulator is in registers
            uint4 w[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) w[c] = *reinterpret_cast<const uint4 *>(yt + sw128_off(m, c));
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t *wv = reinterpret_cast<uint32_t *>(&w[c]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float y0 = fmaf(inf.scale, acc[c * 8 + 2 * e], bf16_lo(wv[e]));
                    const float y1 = fmaf(inf.scale, acc[c * 8 + 2 * e + 1], bf16_hi(wv[e]));
                    wv[e] = pack_bf16x2(y0, y1);
                }
                *reinterpret_cast<uint4 *>(yt + sw128_off(m, c)) = w[c];
            }
            fence_proxy_async_smem();            // the updated tile is read by the TMA unit below
            named_bar_sync(2, kEpiWarps * 32);   // the whole tile is updated in shared memory
            const bool full_tile = !p.perm && inf.rows == kTileM && inf.ncols == kTileN;
            if (full_tile) {
                if (ew == 0 && lane == 0) {
                    const uint32_t yt0 = smem_u32(yring + sy * kExYBytes);
                    tma_store_2d(&p.tmap_io, yt0, inf.col0, inf.row0);
                    tma_store_2d(&p.tmap_io, yt0 + 16384, inf.col0 + 64, inf.row0);
                    bulk_commit_group();
                    // the previous tile's store has read its stage: release that stage now
                    if (pending >= 0) {
                        bulk_wait_group_read1();
                        mbar_arrive(smem_u32(&ctl.yempty[pending]));
                    }
                    EXPAND_MARK(i, 3);
                }
                if (ew == 0) pending = sy;
            } else {
                // coalesced stores masked to the segment's rows and to o: epilogue warp ew stores
                // rows 16 ew .. 16 ew + 15, two per step
                // (with a permutation, row rr of the tile is token perm[row0 + rr])
                uint8_t *yg = static_cast<uint8_t *>(p.y);
                const int chunk = lane & 15;
#pragma unroll 1
                for (int rr = ew * 16 + (lane >> 4); rr < ew * 16 + 16; rr += 2) {
                    if (rr < inf.rows && chunk * 8 < inf.ncols) {
                        const int tok = p.perm ? p.perm[inf.row0 + rr] : inf.row0 + rr;
                        if (tok < 0 || tok >= p.T) continue;   // latched when the rows were gathered
                        const uint8_t *box = yring + sy * kExYBytes + (chunk >= 8 ? 16384 : 0);
                        const uint4 wv = *reinterpret_cast<const uint4 *>(box + sw128_off(rr, chunk & 7));
                        *reinterpret_cast<uint4 *>(
                            yg + ((int64_t)tok * p.ldy + p.y_off + inf.col0 + chunk * 8) * 2) = wv;
                    }
                }
                if (ew == 0 && lane == 0 && pending >= 0) {   // no store group of this tile to keep
                    bulk_wait_group_read0();
                    mbar_arrive(smem_u32(&ctl.yempty[pending]));
                }
                if (ew == 0) pending = -1;
            }
            __syncwarp();
            // warps 1..7, and warp 0 for a tile without a TMA store, release the stage now
            if (lane == 0 && !(ew == 0 && pending == sy)) mbar_arrive(smem_u32(&ctl.yempty[sy]));
        }
        if (ew == 0 && lane == 0) {
            if (pending >= 0) {
                bulk_wait_group_read0();
                mbar_arrive(smem_u32(&ctl.yempty[pending]));
            }
            bulk_wait_group0();   // this CTA's tile stores are complete
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 256);
    if (tid == 0) EXPAND_GMARK(3);
}

// ------------------------------------------------------------------- host side

constexpr int shrink_smem(int ks) { return shrink_stages(ks) * (kTileM * 128 + kMaxRankPF * 128) + 256 + 1024; }
constexpr int kExpandSmem = 2 * kExVBytes + kExYStages * kExYBytes + kExBStages * kExBBytes + (int)sizeof(ExpandCtl) + 1024;
static_assert(kExpandSmem <= 227 * 1024, "expand shared memory");
static_assert(shrink_stages(8) * (kTileM * 128 + kMaxRankPF * 128) >= kTileM * (kMaxRankPF + 4) * 4, "partial fits ring");
static_assert(shrink_smem(4) <= 227 * 1024, "shrink shared memory");

}  // namespace

bool prefill_supported(const lora_table *t)
{
    return t && t->d_tmaps_pfA && t->d_tmaps_pfB && t->sigma_kind == LORA_SIGMA_NONE;
}

// Tensor maps of every adapter for the prefill path (bf16 tables, ranks multiple of 8, <= 64).
int prefill_build_maps(lora_table *t)
{
    if (t->dtype != LORA_BF16) return LORA_OK;
    for (int i = 0; i < t->n; ++i)
        if (t->ranks[i] > kMaxRankPF || t->ranks[i] % 8) return LORA_OK;
    std::vector<uint8_t> ha((size_t)t->n * 128), hb((size_t)t->n * 128);
    for (int i = 0; i < t->n; ++i) {
        const int r = t->ranks[i];
        if (encode_sw128(reinterpret_cast<CUtensorMap *>(ha.data() + (size_t)i * 128), t->A[i], t->h, r, t->h,
                         (r + 15) & ~15) != LORA_OK ||
            encode_sw128(reinterpret_cast<CUtensorMap *>(hb.data() + (size_t)i * 128), t->B[i], r, t->o, r, kTileN) !=
                LORA_OK)
            return LORA_OK;   // leave the path off for this table
    }
    if (cudaMalloc(&t->d_tmaps_pfA, ha.size()) != cudaSuccess) return LORA_ERR_CUDA;
    if (cudaMalloc(&t->d_tmaps_pfB, hb.size()) != cudaSuccess) return LORA_ERR_CUDA;
    if (cudaMemcpy(t->d_tmaps_pfA, ha.data(), ha.size(), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(t->d_tmaps_pfB, hb.data(), hb.size(), cudaMemcpyHostToDevice) != cudaSuccess)
        return LORA_ERR_CUDA;
    return LORA_OK;
}

namespace {

// Upper bound of the 128-token tiles of the segments with at least min_len tokens: one partial
// tile per segment at most, and no more such segments than T / min_len.
int tile_bound(const lora_segments *seg, int min_len)
{
    const int segs = min_len > 0 ? std::min(seg->max_segs, seg->T / min_len) : seg->max_segs;
    return segs + (seg->T + kTileM - 1) / kTileM;
}

PrefillParams prefill_params(const lora_table *t, const lora_segments *seg, void *v)
{
    PrefillParams p;
    std::memset(&p, 0, sizeof p);
    p.desc = t->d_desc;
    p.tm_A = static_cast<const uint8_t *>(t->d_tmaps_pfA);
    p.tm_B = static_cast<const uint8_t *>(t->d_tmaps_pfB);
    p.seg_ptr = seg->seg_ptr;
    p.seg_adapter = seg->seg_adapter;
    p.num_segs = seg->num_segs;
    p.max_segs = seg->max_segs;
    p.T = seg->T;
    p.h = t->h;
    p.o = t->o;
    p.n = t->n;
    p.v_hi = static_cast<uint16_t *>(v);
    p.v_lo = p.v_hi + (int64_t)seg->T * kMaxRankPF;
    p.status = t->d_status;
    p.wait_ns = wait_limit_ns();
    p.inject = (int32_t)(options().inject_stall & 6);
    p.perm = seg->perm;
    return p;
}

int set_prefill_attributes()
{
    static bool attr_done[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return LORA_ERR_CUDA;
    if (!attr_done[dev]) {
        if (cudaFuncSetAttribute(prefill_shrink_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 shrink_smem(8)) != cudaSuccess ||
            cudaFuncSetAttribute(prefill_shrink_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 shrink_smem(4)) != cudaSuccess ||
            cudaFuncSetAttribute(prefill_expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kExpandSmem) !=
                cudaSuccess)
            return LORA_ERR_CUDA;
        attr_done[dev] = true;
    }
    return LORA_OK;
}

// The tcgen05 shrink: clusters of KS CTAs (split of h), one cluster per 128-token tile of a
// segment; the intermediate (times s_i when fold_scale) goes to v as bf16 hi + lo [T, 64] each.
int launch_shrink_kernel(PrefillParams &p, const lora_table *t, const lora_segments *seg, const void *x, int64_t ldx,
                         cudaStream_t s)
{
    const Options &opt = options();
    const int mt_bound = tile_bound(seg, p.min_len);
    int rc = encode_sw128(&p.tmap_io, x, (uint64_t)t->h, (uint64_t)seg->T, (uint64_t)ldx, kTileM);
    if (rc != LORA_OK) return rc;
    // with a permutation the x rows are gathered four at a time (one-row boxes)
    if (p.perm && (rc = encode_sw128(&p.tmap_g, x, (uint64_t)t->h, (uint64_t)seg->T, (uint64_t)ldx, 1)) != LORA_OK)
        return rc;
    cudaLaunchConfig_t cfg = {};
    const int KS = opt.prefill_ksplit == 8 ? 8 : 4;
    cfg.gridDim = dim3(KS * mt_bound);
    cfg.blockDim = dim3(kThreadsPF);
    cfg.dynamicSmemBytes = shrink_smem(KS);
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = KS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    int na = 1;
    if (opt.pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    const cudaError_t e = KS == 4 ? cudaLaunchKernelEx(&cfg, prefill_shrink_kernel<4>, p)
                                  : cudaLaunchKernelEx(&cfg, prefill_shrink_kernel<8>, p);
    if (e != cudaSuccess) return LORA_ERR_CUDA;
    note_launch(kKernPrefillShrink);
    return LORA_OK;
}

}  // namespace

int launch_prefill_shrink(const lora_table *t, const lora_segments *seg, const void *x, int64_t ldx, void *v,
                          bool fold_scale, cudaStream_t s)
{
    if (!prefill_supported(t)) return LORA_ERR_UNSUPPORTED;
    int rc = set_prefill_attributes();
    if (rc != LORA_OK) return rc;
    PrefillParams p = prefill_params(t, seg, v);
    p.fold_scale = fold_scale ? 1 : 0;
    return launch_shrink_kernel(p, t, seg, x, ldx, s);
}

int launch_prefill(const lora_table *t, const lora_segments *seg, const void *x, int64_t ldx, void *y, int64_t ldy,
                   int32_t y_off, void *v, int32_t *tile_ctr, int32_t min_len, cudaStream_t s)
{
    if (!prefill_supported(t)) return LORA_ERR_UNSUPPORTED;
    int rc = set_prefill_attributes();
    if (rc != LORA_OK) return rc;
    PrefillParams p = prefill_params(t, seg, v);
    p.y = y;
    p.ldy = ldy;
    p.y_off = y_off;
    p.min_len = min_len;
    p.tile_ctr = tile_ctr;
    const int mt_bound = tile_bound(seg, min_len);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return LORA_ERR_CUDA;
    const Options &opt = options();
    if ((rc = launch_shrink_kernel(p, t, seg, x, ldx, s)) != LORA_OK) return rc;
    // expand: persistent, one CTA per SM over all (128-token tile, 128-column tile) pairs
    if ((rc = encode_sw128(&p.tmap_vhi, p.v_hi, kMaxRankPF, (uint64_t)seg->T, kMaxRankPF, kTileM)) != LORA_OK ||
        (rc = encode_sw128(&p.tmap_vlo, p.v_lo, kMaxRankPF, (uint64_t)seg->T, kMaxRankPF, kTileM)) != LORA_OK)
        return rc;
    rc = encode_sw128(&p.tmap_io, static_cast<uint8_t *>(y) + (int64_t)y_off * 2, (uint64_t)t->o, (uint64_t)seg->T,
                      (uint64_t)ldy, kTileM);
    if (rc != LORA_OK) return rc;
    if (p.perm && (rc = encode_sw128(&p.tmap_g, static_cast<uint8_t *>(y) + (int64_t)y_off * 2, (uint64_t)t->o,
                                     (uint64_t)seg->T, (uint64_t)ldy, 1)) != LORA_OK)
        return rc;
    {
        cudaLaunchConfig_t cfg = {};
        static int n_sms[64];
        if (!n_sms[dev]) cudaDeviceGetAttribute(&n_sms[dev], cudaDevAttrMultiProcessorCount, dev);
        const int tiles_bound = mt_bound * ((t->o + kTileN - 1) / kTileN);
        cfg.gridDim = dim3(max(1, min(n_sms[dev], tiles_bound)));
        cfg.blockDim = dim3(kThreadsEX);
        cfg.dynamicSmemBytes = kExpandSmem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        int na = 0;
        if (opt.pdl) {
            attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[na].val.programmaticStreamSerializationAllowed = 1;
            ++na;
        }
        cfg.attrs = attr;
        cfg.numAttrs = na;
        if (cudaLaunchKernelEx(&cfg, prefill_expand_kernel, p) != cudaSuccess) return LORA_ERR_CUDA;
        note_launch(kKernPrefillExpand);
    }
    return LORA_OK;
}

}  // namespace lora

#ifdef LORA_TRACE
// Instrumented builds only: copy the shrink's per-CTA phase marks to the host.
extern "C" int lora_trace_read_shrink(unsigned long long *host, int n)
{
    if (n > 4096 * 16) n = 4096 * 16;
    return cudaMemcpyFromSymbol(host, lora::lora_trace_shrink, sizeof(unsigned long long) * n) == cudaSuccess ? 0 : -4;
}

extern "C" int lora_trace_read_expand(unsigned long long *host, int n)
{
    if (n > 160 * 65 * 4) n = 160 * 65 * 4;
    return cudaMemcpyFromSymbol(host, lora::lora_trace_expand, sizeof(unsigned long long) * n) == cudaSuccess ? 0 : -4;
}
#endif
