// Decode-time LoRA delta on CUDA cores: shrink (x . A_i^T -> fp32 rank-space intermediate,
// scale 1) and expand (y += s_i * v . B_i^T into a column slice of y), fused in one kernel or
// run as separate steps ("Compress then Serve" review thread, add_lora_slice pseudocode;
// "TGI Multi-LoRA" page, "Technical Foundation: LoRA").
//
// Design for sm_100a:
//  * A cluster of 8 CTAs owns one work unit at a time: up to 16 tokens of one adapter (one
//    SGMV segment chunk, or one group of equal ids in the per-token BGMV form).  CTA j of the
//    cluster streams the j-th eighth of h for the shrink and the j-th eighth of o for the
//    expand, so each adapter's A_i and B_i are read exactly once per unit and every token of
//    the unit reuses that read.
//  * One producer warp per CTA moves all operands with untiled bulk async copies (TMA engine,
//    no multicast) into a ring of shared-memory stages guarded by mbarriers; it runs ahead
//    across units, so B_i and y of a unit are in flight while its shrink is computed.
//  * Shrink: warp-level split-K.  A lane owns 16 bytes at two places of each 1 KiB row; 8
//    partial dot products per lane are folded across the warp with a transposed butterfly
//    (9 shuffles) instead of 8 separate reductions.
//  * The 8 partial intermediates of a cluster are summed in a fixed CTA order through
//    distributed shared memory, synchronised by remote mbarrier arrivals (no grid barrier, no
//    atomics, bit-identical run to run).
//  * Expand: each thread owns two output columns (bf16) and all tokens of the unit, reads its
//    B rows once from shared memory and updates y from the staged copy; results are rounded
//    once (round-to-nearest-even) and stored with coalesced 32-bit stores.
//  * Persistent grid: as many clusters as fit, each walking the unit list with a stride.
#include <climits>
#include <cstdio>
#include <mutex>

#include "lora_common.cuh"
#include "lora_internal.h"

namespace lora {
namespace {

constexpr int kCluster = 8;
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;   // + one producer warp
constexpr int kTokChunk = 16;               // tokens per work unit
constexpr int kRowBytes = 1024;             // one staged row of a tile
constexpr int kMaxStages = 4;
constexpr int kHeaderBytes = 128;

enum : int32_t { kTileShrink = 1, kTileExpand = 2, kTileEnd = 3 };
enum : int32_t { kFlagFirst = 1, kFlagLast = 2 };

struct __align__(16) StageHeader {
    int32_t kind, flags, adapter, rank;
    float scale;
    int32_t L, off, len;        // tokens; first column (shrink: of h, expand: row of o) and extent
    int32_t tok[kTokChunk];
};
static_assert(sizeof(StageHeader) <= kHeaderBytes, "header");

struct __align__(8) SmemCtl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t vready[2];
    uint64_t vfree[2];
    int32_t n_groups;
    int32_t pending[kTokChunk];  // producer's token list while grouping ids
};
constexpr int kCtlBytes = 256;
static_assert(sizeof(SmemCtl) <= kCtlBytes, "ctl");

template <typename E> struct Tr;
template <> struct Tr<__nv_bfloat16> {
    static constexpr int ESZ = 2, EPC = 8, CPT = 2;
};
template <> struct Tr<float> {
    static constexpr int ESZ = 4, EPC = 4, CPT = 1;
};

__host__ __device__ constexpr int round_up(int a, int b) { return (a + b - 1) / b * b; }

struct Layout {
    int ids_off, v_off, stage_off, RP, total;
};

__host__ __device__ inline Layout make_layout(int src, int R, int n, int T, int stages, int stage_bytes)
{
    Layout l;
    l.RP = round_up(R, 8);
    l.ids_off = kCtlBytes;
    const int ids_bytes = (src == kSrcIds) ? round_up(4 * (2 * T + n), 128) : 0;
    l.v_off = l.ids_off + ids_bytes;
    const int v_bytes = round_up(3 * kTokChunk * l.RP * 4, 128);   // vpart[2] + vfull
    l.stage_off = l.v_off + v_bytes;
    l.total = l.stage_off + stages * stage_bytes;
    return l;
}

// 16 staged bytes -> EPC floats
__device__ __forceinline__ void load16(const uint8_t *p, float *o, __nv_bfloat16 *)
{
    const uint4 w = *reinterpret_cast<const uint4 *>(p);
    o[0] = bf16_lo(w.x); o[1] = bf16_hi(w.x); o[2] = bf16_lo(w.y); o[3] = bf16_hi(w.y);
    o[4] = bf16_lo(w.z); o[5] = bf16_hi(w.z); o[6] = bf16_lo(w.w); o[7] = bf16_hi(w.w);
}
__device__ __forceinline__ void load16(const uint8_t *p, float *o, float *)
{
    const float4 w = *reinterpret_cast<const float4 *>(p);
    o[0] = w.x; o[1] = w.y; o[2] = w.z; o[3] = w.w;
}

// Sum 8 per-lane values over the 32 lanes of a warp.  On return lane L holds the total of
// value index (L >> 2) & 7.  Fixed order, so the result is deterministic.
__device__ __forceinline__ float warp_reduce8(float (&a)[8], int lane)
{
    {
        const bool up = lane & 16;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float send = up ? a[q] : a[q + 4];
            const float keep = up ? a[q + 4] : a[q];
            a[q] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
    }
    {
        const bool up = lane & 8;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const float send = up ? a[q] : a[q + 2];
            const float keep = up ? a[q + 2] : a[q];
            a[q] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
    }
    {
        const bool up = lane & 4;
        const float send = up ? a[0] : a[1];
        const float keep = up ? a[1] : a[0];
        a[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    float r = a[0];
    r += __shfl_xor_sync(0xffffffffu, r, 2);
    r += __shfl_xor_sync(0xffffffffu, r, 1);
    return r;
}

template <typename E, int MODE, int SRC>
__global__ void __launch_bounds__(kThreads, 1)
lora_decode_kernel(const __grid_constant__ DecodeParams p)
{
    using T_ = Tr<E>;
    constexpr int ESZ = T_::ESZ, EPC = T_::EPC, CPT = T_::CPT;
    constexpr int W = kRowBytes / ESZ;          // elements of one staged row
    constexpr int CHUNKS = kRowBytes / 16;      // 16-byte chunks per staged row

    extern __shared__ __align__(128) uint8_t smem[];
    SmemCtl &ctl = *reinterpret_cast<SmemCtl *>(smem);
    const Layout lay = make_layout(SRC, p.R, p.n, p.T, p.stages, p.stage_bytes);
    float *vpart = reinterpret_cast<float *>(smem + lay.v_off);            // [2][kTokChunk][RP]
    float *vfull = vpart + 2 * kTokChunk * lay.RP;                          // [kTokChunk][RP]
    uint8_t *stage_base = smem + lay.stage_off;
    const int RP = lay.RP;
    const int S = p.stages;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t crank = cluster_ctarank();
    const int cid = (int)cluster_id_x(), G = (int)nclusters_x();

    pdl_wait();
    pdl_launch_dependents();

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&ctl.full[s]), 1);
            mbar_init(smem_u32(&ctl.empty[s]), kConsumerWarps);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(smem_u32(&ctl.vready[q]), kCluster);
            mbar_init(smem_u32(&ctl.vfree[q]), kCluster);
        }
        fence_mbar_init_cluster();
    }

    // Per-token ids: group equal ids on the device.  A group is led by the first token that
    // carries its id; groups are listed in the order of their leaders.
    int32_t *ids_s = reinterpret_cast<int32_t *>(smem + lay.ids_off);
    int32_t *first = ids_s + p.T;
    int32_t *leaders = first + p.n;
    if (SRC == kSrcIds) {
        bool bad = false;
        for (int t = tid; t < p.T; t += kThreads) {
            const int32_t a = p.ids[t];
            ids_s[t] = a;
            bad |= (a < -1 || a >= p.n);
        }
        for (int i = tid; i < p.n; i += kThreads) first[i] = INT_MAX;
        if (__syncthreads_or(bad) && tid == 0 && crank == 0) atomicOr(p.status, LORA_STATUS_BAD_ID);
        for (int t = tid; t < p.T; t += kThreads) {
            const int32_t a = ids_s[t];
            if (a >= 0 && a < p.n) atomicMin(&first[a], t);
        }
        __syncthreads();
        if (warp == 0) {
            int cnt = 0;
            for (int base = 0; base < p.T; base += 32) {
                const int t = base + lane;
                const int32_t a = t < p.T ? ids_s[t] : -1;
                const bool lead = a >= 0 && a < p.n && first[a] == t;
                const uint32_t m = __ballot_sync(0xffffffffu, lead);
                if (lead) leaders[cnt + __popc(m & ((1u << lane) - 1u))] = t;
                cnt += __popc(m);
            }
            if (lane == 0) ctl.n_groups = cnt;
        }
    }
    cluster_sync_all();   // barrier inits visible cluster-wide; group list ready

    // h and o ranges of this CTA, in 16-byte chunks of h and EPC-row groups of o
    const int hchunks = p.h / EPC, ogroups = p.o / EPC;
    const int hc0 = (int)((int64_t)crank * hchunks / kCluster);
    const int hc1 = (int)((int64_t)(crank + 1) * hchunks / kCluster);
    const int og0 = (int)((int64_t)crank * ogroups / kCluster);
    const int og1 = (int)((int64_t)(crank + 1) * ogroups / kCluster);
    const int n_shrink = (MODE == kModeExpand) ? 0 : max(1, (hc1 - hc0 + CHUNKS - 1) / CHUNKS);
    const int orows = (og1 - og0) * EPC;
    const int n_expand = (MODE == kModeShrink) ? 0 : (orows + W - 1) / W;

    if (warp == kConsumerWarps) {
        // ================================ producer warp ================================
        int issued = 0;
        bool alive = true;
        auto next_stage = [&](StageHeader *&hdr, uint8_t *&data, uint32_t &full_bar) -> bool {
            const int s = issued % S;
            const int m = issued / S;
            if (m >= 1 && !mbar_wait(smem_u32(&ctl.empty[s]), (m - 1) & 1, p.status)) return false;
            hdr = reinterpret_cast<StageHeader *>(stage_base + (size_t)s * p.stage_bytes);
            data = stage_base + (size_t)s * p.stage_bytes + kHeaderBytes;
            full_bar = smem_u32(&ctl.full[s]);
            return true;
        };
        // Issue every tile of one unit: adapter a, tokens tok[0, L) (valid in lane l < L).
        auto emit_unit = [&](int a, int my_tok, int L) {
            const AdapterDesc d = p.desc[a];
            const int r = d.rank;
            const uint8_t *Ab = static_cast<const uint8_t *>(d.A);
            const uint8_t *Bb = static_cast<const uint8_t *>(d.B);
            const int ntiles = n_shrink + n_expand;
            for (int j = 0; j < ntiles && alive; ++j) {
                StageHeader *hdr;
                uint8_t *data;
                uint32_t fb;
                if (!next_stage(hdr, data, fb)) {
                    alive = false;
                    break;
                }
                const bool shrink = j < n_shrink;
                int off, len;
                uint32_t bytes;
                if (shrink) {
                    const int c0 = hc0 + j * CHUNKS;
                    const int c1 = min(hc1, c0 + CHUNKS);
                    off = c0 * EPC;
                    len = max(0, c1 - c0) * EPC;
                    bytes = (uint32_t)((r + L) * len * ESZ);
                } else {
                    const int jj = j - n_shrink;
                    off = og0 * EPC + jj * W;
                    len = min(W, orows - jj * W);
                    bytes = (uint32_t)(len * r * ESZ + L * len * ESZ);
                }
                if (lane < L) hdr->tok[lane] = my_tok;
                if (lane == 0) {
                    hdr->kind = shrink ? kTileShrink : kTileExpand;
                    const int first_j = shrink ? 0 : n_shrink;
                    const int last_j = shrink ? n_shrink - 1 : ntiles - 1;
                    hdr->flags = (j == first_j ? kFlagFirst : 0) | (j == last_j ? kFlagLast : 0);
                    hdr->adapter = a;
                    hdr->rank = r;
                    hdr->scale = d.scale;
                    hdr->L = L;
                    hdr->off = off;
                    hdr->len = len;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive_expect_tx(fb, bytes);
                __syncwarp();
                if (len > 0) {
                    const uint32_t dst = smem_u32(data);
                    if (shrink) {
                        // r rows of A_i, then L rows of x, each len elements from column `off`
                        for (int c = lane; c < r; c += 32)
                            bulk_g2s(dst + c * kRowBytes, Ab + ((int64_t)c * p.h + off) * ESZ, len * ESZ, fb);
                        // x rows (token of row l lives in lane l)
                        for (int l = 0; l < L; ++l) {
                            const int t = __shfl_sync(0xffffffffu, my_tok, l);
                            if (lane == (l & 31))
                                bulk_g2s(dst + (r + l) * kRowBytes,
                                         static_cast<const uint8_t *>(p.x) + ((int64_t)t * p.ldx + off) * ESZ,
                                         len * ESZ, fb);
                        }
                    } else {
                        const int yoff = round_up(len * r * ESZ, 128);
                        if (lane == 0) bulk_g2s(dst, Bb + (int64_t)off * r * ESZ, len * r * ESZ, fb);
                        for (int l = 0; l < L; ++l) {
                            const int t = __shfl_sync(0xffffffffu, my_tok, l);
                            if (lane == ((l + 1) & 31))
                                bulk_g2s(dst + yoff + l * kRowBytes,
                                         static_cast<uint8_t *>(p.y) +
                                             ((int64_t)t * p.ldy + p.y_off + off) * ESZ,
                                         len * ESZ, fb);
                        }
                    }
                }
                ++issued;
            }
        };

        if (SRC == kSrcSegments) {
            const int nseg = min(*p.num_segs, p.max_segs);
            for (int s = cid; s < nseg && alive; s += G) {
                const int a = p.seg_adapter[s];
                const int p0 = p.seg_ptr[s], p1 = p.seg_ptr[s + 1];
                if (a < 0 || a >= p.n || p0 < 0 || p1 < p0 || p1 > p.T) {
                    if (lane == 0 && crank == 0) atomicOr(p.status, LORA_STATUS_BAD_SEGMENT);
                    continue;
                }
                for (int q = p0; q < p1 && alive; q += kTokChunk) {
                    const int L0 = min(kTokChunk, p1 - q);
                    int t = -1;
                    if (lane < L0) t = p.perm ? p.perm[q + lane] : q + lane;
                    const bool ok = lane < L0 && t >= 0 && t < p.T;
                    const uint32_t m = __ballot_sync(0xffffffffu, ok);
                    if (m != __ballot_sync(0xffffffffu, lane < L0) && lane == 0 && crank == 0)
                        atomicOr(p.status, LORA_STATUS_BAD_SEGMENT);
                    // compact valid tokens to lanes 0..popc(m)-1
                    const int dst_lane = __popc(m & ((1u << lane) - 1u));
                    int my_tok = 0;
                    for (int l = 0; l < L0; ++l) {
                        const int tl = __shfl_sync(0xffffffffu, t, l);
                        const int dl = __shfl_sync(0xffffffffu, dst_lane, l);
                        if (((m >> l) & 1u) && lane == dl) my_tok = tl;
                    }
                    const int L = __popc(m);
                    if (L > 0) emit_unit(a, my_tok, L);
                }
            }
        } else {
            const int ng = ctl.n_groups;
            for (int g = cid; g < ng && alive; g += G) {
                const int t0 = leaders[g];
                const int a = ids_s[t0];
                int cnt = 0;
                for (int base = t0; base < p.T && alive; base += 32) {
                    const int t = base + lane;
                    const bool match = t < p.T && ids_s[t] == a;
                    uint32_t m = __ballot_sync(0xffffffffu, match);
                    while (m && alive) {
                        const int take = min(__popc(m), kTokChunk - cnt);
                        const int rk = __popc(m & ((1u << lane) - 1u));
                        if (((m >> lane) & 1u) && rk < take) ctl.pending[cnt + rk] = t;
                        for (int i = 0; i < take; ++i) m &= m - 1u;
                        cnt += take;
                        __syncwarp();
                        if (cnt == kTokChunk) {
                            const int my_tok = ctl.pending[lane & (kTokChunk - 1)];
                            __syncwarp();
                            emit_unit(a, my_tok, cnt);
                            cnt = 0;
                        }
                    }
                }
                if (cnt > 0 && alive) {
                    const int my_tok = ctl.pending[lane & (kTokChunk - 1)];
                    __syncwarp();
                    emit_unit(a, my_tok, cnt);
                }
            }
        }
        // end marker
        if (alive) {
            StageHeader *hdr;
            uint8_t *data;
            uint32_t fb;
            if (next_stage(hdr, data, fb)) {
                if (lane == 0) {
                    hdr->kind = kTileEnd;
                    mbar_arrive(fb);
                }
                ++issued;
            }
        }
        // drain: no bulk copy may still be writing into this CTA's shared memory at exit
        for (int i = max(0, issued - S); i < issued; ++i)
            mbar_wait(smem_u32(&ctl.full[i % S]), (i / S) & 1, p.status);
        return;
    }

    // =================================== consumers ===================================
    int u = 0;   // units whose intermediate has been reduced (fused / shrink modes)
    for (int it = 0;; ++it) {
        const int s = it % S;
        if (!mbar_wait(smem_u32(&ctl.full[s]), (it / S) & 1, p.status)) break;
        const StageHeader &hdr = *reinterpret_cast<const StageHeader *>(stage_base + (size_t)s * p.stage_bytes);
        const uint8_t *data = stage_base + (size_t)s * p.stage_bytes + kHeaderBytes;
        const int kind = hdr.kind;
        if (kind == kTileEnd) break;
        const int r = hdr.rank, L = hdr.L, flags = hdr.flags, len = hdr.len, off = hdr.off;
        bool ok = true;

        if (kind == kTileShrink) {
            const int q = u & 1;
            float *vp = vpart + q * kTokChunk * RP;
            if ((flags & kFlagFirst) && u >= 2)
                ok = mbar_wait_cluster(smem_u32(&ctl.vfree[q]), ((u >> 1) - 1) & 1, p.status);
            if (!ok) break;
            // ---- partial shrink over this CTA's slice of h: P[l][k] = sum_j X[l][j] A[k][j]
            const int nchunks = len / EPC;
            const int cA = lane, cB = lane + 32;
            const int nkg = (r + 7) >> 3;
            for (int slot = warp; slot < L * nkg; slot += kConsumerWarps) {
                const int l = slot / nkg, kg = slot - l * nkg;
                float xv[2 * EPC];
                const uint8_t *xr = data + (r + l) * kRowBytes;
                if (cA < nchunks) load16(xr + cA * 16, xv, (E *)nullptr);
                else for (int e = 0; e < EPC; ++e) xv[e] = 0.f;
                if (cB < nchunks) load16(xr + cB * 16, xv + EPC, (E *)nullptr);
                else for (int e = 0; e < EPC; ++e) xv[EPC + e] = 0.f;
                float acc[8];
#pragma unroll
                for (int qq = 0; qq < 8; ++qq) {
                    acc[qq] = 0.f;
                    const int k = kg * 8 + qq;
                    if (k < r) {
                        const uint8_t *ar = data + k * kRowBytes;
                        float av[EPC];
                        if (cA < nchunks) {
                            load16(ar + cA * 16, av, (E *)nullptr);
#pragma unroll
                            for (int e = 0; e < EPC; ++e) acc[qq] = fmaf(xv[e], av[e], acc[qq]);
                        }
                        if (cB < nchunks) {
                            load16(ar + cB * 16, av, (E *)nullptr);
#pragma unroll
                            for (int e = 0; e < EPC; ++e) acc[qq] = fmaf(xv[EPC + e], av[e], acc[qq]);
                        }
                    }
                }
                const float tot = warp_reduce8(acc, lane);
                const int k = kg * 8 + ((lane >> 2) & 7);
                if ((lane & 3) == 0 && k < r) {
                    float *dst = vp + l * RP + k;
                    *dst = (flags & kFlagFirst) ? tot : *dst + tot;
                }
            }
            if (flags & kFlagLast) {
                // ---- sum the cluster's partials in CTA order 0..7 through distributed smem
                named_bar_sync(1, kConsumers);
                if (tid == 0)
                    for (int j = 0; j < kCluster; ++j) mbar_arrive_remote(smem_u32(&ctl.vready[q]), j);
                ok = mbar_wait_cluster(smem_u32(&ctl.vready[q]), (u >> 1) & 1, p.status);
                if (!ok) break;
                const uint32_t vp_addr = smem_u32(vp);
                for (int e = tid; e < L * RP; e += kConsumers) {
                    const int l = e / RP, k = e - l * RP;
                    float acc = 0.f;
                    if (k < r)
                        for (int j = 0; j < kCluster; ++j) acc += ld_dsmem_f32(vp_addr + 4u * (l * RP + k), j);
                    vfull[e] = acc;
                }
                named_bar_sync(1, kConsumers);
                if (tid == 0)
                    for (int j = 0; j < kCluster; ++j) mbar_arrive_remote(smem_u32(&ctl.vfree[q]), j);
                if (MODE == kModeShrink && crank == 0) {
                    for (int e = tid; e < L * r; e += kConsumers) {
                        const int l = e / r, k = e - l * r;
                        p.v[(int64_t)hdr.tok[l] * p.ldv + k] = vfull[l * RP + k];
                    }
                }
                ++u;
            }
        } else {  // kTileExpand
            if (MODE == kModeExpand && (flags & kFlagFirst)) {
                named_bar_sync(1, kConsumers);
                for (int e = tid; e < L * RP; e += kConsumers) {
                    const int l = e / RP, k = e - l * RP;
                    vfull[e] = (k < r) ? p.v[(int64_t)hdr.tok[l] * p.ldv + k] : 0.f;
                }
                named_bar_sync(1, kConsumers);
            }
            const int c = tid * CPT;   // first column of this thread within the tile
            if (c < len) {
                const int yoff = round_up(len * r * ESZ, 128);
                float acc[kTokChunk][CPT];
#pragma unroll
                for (int l = 0; l < kTokChunk; ++l)
#pragma unroll
                    for (int j = 0; j < CPT; ++j) acc[l][j] = 0.f;
                if ((r % EPC) == 0) {
                    for (int k = 0; k < r; k += EPC) {
                        float b[CPT][EPC];
#pragma unroll
                        for (int j = 0; j < CPT; ++j) load16(data + ((c + j) * r + k) * ESZ, b[j], (E *)nullptr);
#pragma unroll
                        for (int l = 0; l < kTokChunk; ++l) {
                            if (l < L) {
                                const float *vr = vfull + l * RP + k;
                                float vv[EPC];
#pragma unroll
                                for (int e = 0; e < EPC; e += 4) {
                                    const float4 t4 = *reinterpret_cast<const float4 *>(vr + e);
                                    vv[e] = t4.x; vv[e + 1] = t4.y; vv[e + 2] = t4.z; vv[e + 3] = t4.w;
                                }
#pragma unroll
                                for (int j = 0; j < CPT; ++j)
#pragma unroll
                                    for (int e = 0; e < EPC; ++e) acc[l][j] = fmaf(vv[e], b[j][e], acc[l][j]);
                            }
                        }
                    }
                } else {
                    for (int k = 0; k < r; ++k) {
                        float b[CPT];
#pragma unroll
                        for (int j = 0; j < CPT; ++j) {
                            const E *bp = reinterpret_cast<const E *>(data) + (c + j) * r + k;
                            b[j] = (float)(*bp);
                        }
#pragma unroll
                        for (int l = 0; l < kTokChunk; ++l)
                            if (l < L)
#pragma unroll
                                for (int j = 0; j < CPT; ++j) acc[l][j] = fmaf(vfull[l * RP + k], b[j], acc[l][j]);
                    }
                }
                const float sc = hdr.scale;
#pragma unroll
                for (int l = 0; l < kTokChunk; ++l) {
                    if (l < L) {
                        const uint8_t *yr = data + yoff + l * kRowBytes + c * ESZ;
                        const int64_t gofs = (int64_t)hdr.tok[l] * p.ldy + p.y_off + off + c;
                        if constexpr (CPT == 2) {
                            const uint32_t w = *reinterpret_cast<const uint32_t *>(yr);
                            const float y0 = fmaf(sc, acc[l][0], bf16_lo(w));
                            const float y1 = fmaf(sc, acc[l][1], bf16_hi(w));
                            *reinterpret_cast<uint32_t *>(static_cast<E *>(p.y) + gofs) = pack_bf16x2(y0, y1);
                        } else {
                            const float w = *reinterpret_cast<const float *>(yr);
                            static_cast<float *>(p.y)[gofs] = fmaf(sc, acc[l][0], w);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctl.empty[s]));
    }
    // No CTA of the cluster may leave while a peer can still read its partials or arrive on
    // its barriers: wait for the last release of each intermediate slot.
    if (MODE != kModeExpand) {
        if (u >= 1) mbar_wait_cluster(smem_u32(&ctl.vfree[(u - 1) & 1]), ((u - 1) >> 1) & 1, p.status);
        if (u >= 2) mbar_wait_cluster(smem_u32(&ctl.vfree[(u - 2) & 1]), ((u - 2) >> 1) & 1, p.status);
    }
}

template <typename E, int MODE, int SRC>
int launch_one(const DecodeParams &p0, cudaStream_t s)
{
    auto kern = lora_decode_kernel<E, MODE, SRC>;
    DecodeParams p = p0;
    const Options &opt = options();
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LORA_ERR_CUDA;
    static std::once_flag once[64];
    static int max_optin[64];
    static int n_sms[64];
    if (dev >= 64) return LORA_ERR_UNSUPPORTED;
    std::call_once(once[dev], [&] {
        cudaDeviceGetAttribute(&max_optin[dev], cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaDeviceGetAttribute(&n_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    });
    // Pipeline depth: aim for two CTAs per SM unless told otherwise.
    const int stage_bytes = kHeaderBytes + (p.R + kTokChunk) * kRowBytes;
    const int fixed = make_layout(SRC, p.R, p.n, p.T, 0, stage_bytes).total;
    int ctas_per_sm = opt.decode_ctas_per_sm > 0 ? (int)opt.decode_ctas_per_sm : 2;
    int stages = (int)opt.decode_stages;
    if (stages <= 0) {
        const int budget = (228 * 1024) / ctas_per_sm - 1024 - fixed;
        stages = min(kMaxStages, budget / stage_bytes);
        if (stages < 2) stages = 2;
    }
    stages = max(2, min(kMaxStages, stages));
    const Layout lay = make_layout(SRC, p.R, p.n, p.T, stages, stage_bytes);
    if (lay.total > max_optin[dev]) return LORA_ERR_UNSUPPORTED;
    p.stages = stages;
    p.stage_bytes = stage_bytes;
    static int smem_set[64];
    if (smem_set[dev] < lay.total) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total) != cudaSuccess)
            return LORA_ERR_CUDA;
        smem_set[dev] = lay.total;
    }

    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)lay.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = kCluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cfg.gridDim = dim3(kCluster);
    // co-resident clusters for this shared-memory size (cached: a host query, not a stream op)
    static int occ_smem[64], occ_clusters[64];
    if (occ_smem[dev] != lay.total) {
        int mc = 0;
        if (cudaOccupancyMaxActiveClusters(&mc, (void *)kern, &cfg) != cudaSuccess || mc < 1)
            mc = max(1, n_sms[dev] / kCluster);
        occ_clusters[dev] = mc;
        occ_smem[dev] = lay.total;
    }
    const int max_clusters = occ_clusters[dev];
    const int units_bound = max(1, min(p.T, (SRC == kSrcSegments) ? p.max_segs : p.n));
    const int G = max(1, min(max_clusters, units_bound));
    cfg.gridDim = dim3(G * kCluster);
    if (opt.pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return LORA_ERR_CUDA;
    return LORA_OK;
}

template <typename E>
int launch_typed(int mode, int src, const DecodeParams &p, cudaStream_t s)
{
    if (src == kSrcSegments) {
        if (mode == kModeFused) return launch_one<E, kModeFused, kSrcSegments>(p, s);
        if (mode == kModeShrink) return launch_one<E, kModeShrink, kSrcSegments>(p, s);
        return launch_one<E, kModeExpand, kSrcSegments>(p, s);
    }
    if (mode == kModeFused) return launch_one<E, kModeFused, kSrcIds>(p, s);
    return LORA_ERR_UNSUPPORTED;
}

}  // namespace

int launch_decode(int mode, int src, const DecodeParams &p, int dtype, cudaStream_t s)
{
    if (dtype == LORA_BF16) return launch_typed<__nv_bfloat16>(mode, src, p, s);
    if (dtype == LORA_F32) return launch_typed<float>(mode, src, p, s);
    return LORA_ERR_UNSUPPORTED;
}

size_t decode_ids_limit_bytes(int n, int T) { return (size_t)round_up(4 * (2 * T + n), 128); }

}  // namespace lora
