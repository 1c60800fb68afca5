// Layer output with the frozen base weight, fused with the adapter term, on the 5th-generation
// tensor cores:
//
//     y[t, off + n] = (y[t, off + n] if accumulating) + sum_j x[t, j] W[n, j]
//                     + s_i * sum_k B_i[n, k] (sum_j x[t, j] A_i[k, j])
//
// ("TGI Multi-LoRA" page, "Technical Foundation: LoRA": the pretrained weight stays frozen and
// the adapter adds its low-rank term to the layer's output; "predibase/lorax" repository
// page: the adapter is applied within the layer's single forward pass.)
//
// Two launches.  The tcgen05 shrink (prefill.cu) stores s_i * (x . A_i^T) per token as bf16
// hi + lo.  Then this persistent kernel computes every (128-token tile, 256-column tile) of the
// output in ONE tensor-memory accumulator: 64-column k-blocks of x against W, then, for tiles
// of a segment with an adapter, two more k-blocks -- the intermediate's hi and lo parts
// against B_i (rank padded to 64 by the TMA zero fill) -- so the adapter term is summed by the
// tensor core and y is written once (read only when accumulating).
//
// Warp roles: warp 0 streams k-blocks by TMA into a 4-deep ring (x or intermediate tile
// 16 KiB + W or B_i tile 32 KiB per stage); warp 1 allocates tensor memory and one lane
// issues tcgen05.mma (M = 128, N = 256, K = 16) into two accumulators used alternately; warps
// 2..5 drain an accumulator (tcgen05.ld, one output row per thread), round once to bf16 and
// store while the next tile accumulates.  Tiles never straddle a segment: the rows [0, T) are
// cut into pieces (before the first segment, each segment, after the last) and each piece into
// 128-row tiles, so a tile has one adapter (or none); rows past a partial tile's piece are
// computed but not stored.  No TMA multicast.  Every wait is bounded; after a timeout the
// kernel drains its copies and MMAs and releases tensor memory before returning.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "lora_common.cuh"
#include "lora_internal.h"
#include "tcgen05.cuh"

namespace lora {
namespace {

constexpr int kBM = 128;                       // tokens per tile (MMA M, TMEM lanes)
constexpr int kBN = 256;                       // output columns per tile (MMA N)
constexpr int kBK = 64;                        // k-block: 64 bf16 = one 128-byte swizzled row
constexpr int kBStages = 4;
constexpr int kBABytes = kBM * 128;            // x (or intermediate) k-block tile
constexpr int kBBBytes = kBN * 128;            // W (or B_i) k-block tile
constexpr int kBStageBytes = kBABytes + kBBBytes;
constexpr int kBEpiWarps = 4;
constexpr int kBThreads = (2 + kBEpiWarps) * 32;
constexpr int kBRankPad = 64;                  // the intermediate's columns (ranks <= 64)

struct BaseParams {
    CUtensorMap tm_x;             // x [T, h], box 64 x 128
    CUtensorMap tm_w;             // W [o, h], box 64 x 256
    CUtensorMap tm_vhi, tm_vlo;   // s_i * intermediate, bf16 hi / lo parts [T, 64], box 64 x 128
    const uint8_t *tm_B;          // per adapter: B_i [o, r], box 64 x 128 (rank zero-filled to 64)
    const int32_t *seg_ptr, *seg_adapter, *num_segs;
    int32_t max_segs, T, h, o, n;
    void *y;
    int64_t ldy;
    int32_t y_off;
    int32_t accumulate;
    uint32_t *status;
    uint64_t wait_ns;
    int32_t early;                // 1: the shrink was launched just before (see the kernel)
};

struct __align__(8) BaseCtl {
    uint64_t full[kBStages], empty[kBStages];
    uint64_t accfull[2], accempty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int32_t total_m;
};

// Row tiles of [0, T).  The pieces are [0, seg_ptr[0]) (no adapter), segment s =
// [seg_ptr[s], seg_ptr[s + 1]) with adapter seg_adapter[s], and [seg_ptr[S], T) (no adapter).
// Boundaries are clamped to [0, T] and made non-decreasing (running maximum), so the pieces
// partition [0, T) even when the table is malformed (*bad is then set).  Every piece is cut into
// 128-row tiles.  Warp-collective; returns the number of tiles, and for 0 <= g < that number
// the first row, the row count and the adapter (-1: none) of tile g.
__device__ int base_row_tiles(const BaseParams &p, int g, int *row0, int *rows, int *adapter, bool *bad)
{
    const int lane = threadIdx.x & 31;
    const int S = max(0, min(*p.num_segs, p.max_segs));
    const int npieces = S + 2;
    int prev_end = 0, tile_base = 0;
    bool badl = false;
    for (int q0 = 0; q0 < npieces; q0 += 32) {
        const int q = q0 + lane;
        const int raw_end = (q <= S) ? p.seg_ptr[q] : p.T;   // piece q ends where segment q starts
        const int end = min(p.T, max(0, raw_end));
        badl |= (q <= S) && (raw_end < 0 || raw_end > p.T);
        int m = max(end, prev_end);
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, m, d);
            if (lane >= d) m = max(m, o);
        }
        int start = __shfl_up_sync(0xffffffffu, m, 1);
        if (lane == 0) start = prev_end;
        badl |= (q < npieces) && (end < start);
        const int len = q < npieces ? m - start : 0;
        const int tiles = (len + kBM - 1) / kBM;
        int incl = tiles;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += o;
        }
        const int excl = tile_base + incl - tiles;
        const uint32_t hit = __ballot_sync(0xffffffffu, g >= excl && g < excl + tiles);
        if (hit) {
            const int src = __ffs(hit) - 1;
            const int qs = __shfl_sync(0xffffffffu, q, src);
            const int r0 = __shfl_sync(0xffffffffu, start, src) + (g - __shfl_sync(0xffffffffu, excl, src)) * kBM;
            *row0 = r0;
            *rows = min(kBM, __shfl_sync(0xffffffffu, m, src) - r0);
            int a = (qs >= 1 && qs <= S) ? p.seg_adapter[qs - 1] : -1;
            if (qs >= 1 && qs <= S && (a < 0 || a >= p.n)) {
                badl = true;
                a = -1;
            }
            *adapter = a;
        }
        tile_base += __shfl_sync(0xffffffffu, incl, 31);
        prev_end = __shfl_sync(0xffffffffu, m, 31);
    }
    *bad = __any_sync(0xffffffffu, badl);
    return tile_base;
}

__global__ void __launch_bounds__(kBThreads, 1) base_gemm_kernel(const __grid_constant__ BaseParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    BaseCtl &ctl = *reinterpret_cast<BaseCtl *>(ring + kBStages * kBStageBytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NT = (p.o + kBN - 1) / kBN;
    const int nkb = (p.h + kBK - 1) / kBK;

    if (tid == 0) {
        for (int i = 0; i < kBStages; ++i) {
            mbar_init(smem_u32(&ctl.full[i]), 1);
            mbar_init(smem_u32(&ctl.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&ctl.accfull[i]), 1);
            mbar_init(smem_u32(&ctl.accempty[i]), kBEpiWarps);
        }
        mbar_init(smem_u32(&ctl.mma_done), 1);
        fence_mbar_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctl.tmem_base), 512);   // two 256-column accumulators
        tmem_relinquish();
    }
    // Programmatic launch: the shrink that precedes this kernel signals its dependents only
    // after its own wait on the grid before it, so x, W, y and the segment table are final when
    // this kernel starts; only the intermediate the shrink writes needs the wait, which the
    // producer performs before its first adapter k-block.  Without that shrink every thread
    // waits here.
    if (!p.early) pdl_wait();
    pdl_launch_dependents();
    if (warp == 0) {
        int r0, rw, ad;
        bool bad = false;
        const int tm = base_row_tiles(p, -1, &r0, &rw, &ad, &bad);
        if (lane == 0) {
            ctl.total_m = tm;
            if (bad && blockIdx.x == 0) atomicOr(p.status, LORA_STATUS_BAD_SEGMENT);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem_base;
    const int MT = ctl.total_m;
    const int total = MT * NT;

    // Tiles t = blockIdx.x, + gridDim.x, ...: row tile g = t % MT fastest, so the CTAs working at
    // one time share a few W column tiles (read from DRAM once, then from L2) and all of x.
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int cur_g = -1, row0 = 0, rows = 0, a = -1, kbi = 0;
        bool ok = true, bad = false, waited = !p.early;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const int g = t % MT, nt = t / MT;
            if (g != cur_g) {
                base_row_tiles(p, g, &row0, &rows, &a, &bad);
                cur_g = g;
            }
            const int nk = nkb + (a >= 0 ? 2 : 0);
            if (a >= 0 && !waited) {   // the intermediate is the shrink's output
                pdl_wait();
                waited = true;
            }
            for (int kb = 0; kb < nk; ++kb, ++kbi) {
                const int s = kbi % kBStages, m = kbi / kBStages;
                if (m >= 1 &&
                    !__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.empty[s]), (m - 1) & 1, p.status, p.wait_ns))) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    uint8_t *st = ring + s * kBStageBytes;
                    const uint32_t fb = smem_u32(&ctl.full[s]);
                    mbar_arrive_expect_tx(fb, kBStageBytes);
                    if (kb < nkb) {
                        tma_load_2d(smem_u32(st), &p.tm_x, kb * kBK, row0, fb);
                        tma_load_2d(smem_u32(st + kBABytes), &p.tm_w, kb * kBK, nt * kBN, fb);
                    } else {
                        // the adapter's k-blocks: intermediate part (hi, then lo) against B_i,
                        // whose 256 rows come as two 128-row boxes
                        tma_load_2d(smem_u32(st), kb == nkb ? &p.tm_vhi : &p.tm_vlo, 0, row0, fb);
                        const void *tb = p.tm_B + (size_t)a * 128;
                        tma_load_2d(smem_u32(st + kBABytes), tb, 0, nt * kBN, fb);
                        tma_load_2d(smem_u32(st + kBABytes + kBBBytes / 2), tb, 0, nt * kBN + kBN / 2, fb);
                    }
                }
                __syncwarp();
            }
        }
        // drain: the copies of the last stages armed have landed before shared memory is
        // released (earlier stages were consumed by the MMAs before being re-armed)
        if (lane == 0)
            for (int i = max(0, kbi - kBStages); i < kbi; ++i)
                mbar_wait(smem_u32(&ctl.full[i % kBStages]), (i / kBStages) & 1, p.status, p.wait_ns);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc = idesc_bf16(kBM, kBN);
        int cur_g = -1, row0 = 0, rows = 0, a = -1, kbi = 0, li = 0;
        bool ok = true, bad = false;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++li) {
            const int g = t % MT;
            if (g != cur_g) {
                base_row_tiles(p, g, &row0, &rows, &a, &bad);
                cur_g = g;
            }
            const int nk = nkb + (a >= 0 ? 2 : 0);
            const int ab = li & 1;
            if (li >= 2 &&
                !__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.accempty[ab]), ((li >> 1) - 1) & 1, p.status, p.wait_ns))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t acc = tmem + (uint32_t)(ab * kBN);
            for (int kb = 0; kb < nk; ++kb, ++kbi) {
                const int s = kbi % kBStages, m = kbi / kBStages;
                if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.full[s]), m & 1, p.status, p.wait_ns))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint8_t *st = ring + s * kBStageBytes;
                    const uint64_t ad = sw128_desc(smem_u32(st));
                    const uint64_t bd = sw128_desc(smem_u32(st + kBABytes));
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k) umma_bf16(acc, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                    umma_commit(smem_u32(&ctl.empty[s]));   // the stage is free once these MMAs finish
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) umma_commit(smem_u32(&ctl.accfull[ab]));
            __syncwarp();
        }
        // every MMA of this CTA has completed before tensor memory is released
        if (lane == 0) {
            umma_commit(smem_u32(&ctl.mma_done));
            mbar_wait(smem_u32(&ctl.mma_done), 0, p.status, p.wait_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;          // TMEM lane quarter of this warp
        const int mrow = q * 32 + lane;  // tile row of this thread
        int cur_g = -1, row0 = 0, rows = 0, a = -1, li = 0;
        bool bad = false;
        uint16_t *y = static_cast<uint16_t *>(p.y);
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++li) {
            const int g = t % MT, nt = t / MT;
            if (g != cur_g) {
                base_row_tiles(p, g, &row0, &rows, &a, &bad);
                cur_g = g;
            }
            const int ab = li & 1;
            // every epilogue warp leaves together if any lane ran out of time
            const bool okw = mbar_wait(smem_u32(&ctl.accfull[ab]), (li >> 1) & 1, p.status, p.wait_ns);
            if (!named_bar_and(2, kBEpiWarps * 32, okw)) break;
            tc_fence_after();
            const int col0 = nt * kBN;
            const bool row_ok = mrow < rows;
            uint16_t *yrow = y + (int64_t)(row0 + (row_ok ? mrow : 0)) * p.ldy + p.y_off + col0;
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * kBN + c0), v);
                const int ncol = min(32, p.o - col0 - c0);
                if (row_ok && ncol > 0) {
#pragma unroll
                    for (int pc = 0; pc < 4; ++pc) {
                        if (pc * 8 < ncol) {
                            uint4 *dst = reinterpret_cast<uint4 *>(yrow + c0 + pc * 8);
                            uint32_t w[4];
                            if (p.accumulate) {
                                const uint4 old = *dst;
                                const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    w[e] = pack_bf16x2(v[pc * 8 + 2 * e] + bf16_lo(ow[e]),
                                                       v[pc * 8 + 2 * e + 1] + bf16_hi(ow[e]));
                            } else {
#pragma unroll
                                for (int e = 0; e < 4; ++e) w[e] = pack_bf16x2(v[pc * 8 + 2 * e], v[pc * 8 + 2 * e + 1]);
                            }
                            *dst = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl.accempty[ab]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

constexpr int kBaseSmem = kBStages * kBStageBytes + (int)sizeof(BaseCtl) + 1024;
static_assert(kBaseSmem <= 227 * 1024, "base GEMM shared memory");

}  // namespace

int launch_base_gemm(const lora_table *t, const lora_segments *seg, const void *x, int64_t ldx, const void *W,
                     int64_t ldw, void *y, int64_t ldy, int32_t y_off, int accumulate, const void *v, bool after_shrink,
                     cudaStream_t s)
{
    BaseParams p;
    std::memset(&p, 0, sizeof p);
    const uint16_t *v_hi = static_cast<const uint16_t *>(v);
    const uint16_t *v_lo = v_hi + (int64_t)seg->T * kBRankPad;
    int rc;
    if ((rc = encode_sw128(&p.tm_x, x, (uint64_t)t->h, (uint64_t)seg->T, (uint64_t)ldx, kBM)) != LORA_OK ||
        (rc = encode_sw128(&p.tm_w, W, (uint64_t)t->h, (uint64_t)t->o, (uint64_t)ldw, kBN)) != LORA_OK ||
        (rc = encode_sw128(&p.tm_vhi, v_hi, kBRankPad, (uint64_t)seg->T, kBRankPad, kBM)) != LORA_OK ||
        (rc = encode_sw128(&p.tm_vlo, v_lo, kBRankPad, (uint64_t)seg->T, kBRankPad, kBM)) != LORA_OK)
        return rc;
    p.tm_B = static_cast<const uint8_t *>(t->d_tmaps_pfB);
    p.seg_ptr = seg->seg_ptr;
    p.seg_adapter = seg->seg_adapter;
    p.num_segs = seg->num_segs;
    p.max_segs = seg->max_segs;
    p.T = seg->T;
    p.h = t->h;
    p.o = t->o;
    p.n = t->n;
    p.y = y;
    p.ldy = ldy;
    p.y_off = y_off;
    p.accumulate = accumulate;
    p.status = t->d_status;
    p.wait_ns = wait_limit_ns();
    p.early = (after_shrink && options().pdl) ? 1 : 0;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return LORA_ERR_CUDA;
    static bool attr_done[64];
    static int n_sms[64];
    if (!attr_done[dev]) {
        if (cudaFuncSetAttribute(base_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBaseSmem) !=
            cudaSuccess)
            return LORA_ERR_CUDA;
        cudaDeviceGetAttribute(&n_sms[dev], cudaDevAttrMultiProcessorCount, dev);
        attr_done[dev] = true;
    }
    const int64_t mt_bound = (int64_t)seg->max_segs + 2 + (seg->T + kBM - 1) / kBM;
    const int64_t tiles_bound = mt_bound * ((t->o + kBN - 1) / kBN);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(n_sms[dev], tiles_bound)));
    cfg.blockDim = dim3(kBThreads);
    cfg.dynamicSmemBytes = kBaseSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    int na = 0;
    if (options().pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, base_gemm_kernel, p) != cudaSuccess) return LORA_ERR_CUDA;
    note_launch(kKernBaseGemm);
    return LORA_OK;
}

}  // namespace lora
