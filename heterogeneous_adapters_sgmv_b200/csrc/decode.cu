// Decode-time LoRA delta on CUDA cores: shrink (x . A_i^T -> fp32 rank-space intermediate,
// scale 1) and expand (y += s_i * v . B_i^T into a column slice of y), fused in one kernel or
// run as separate steps ("Compress then Serve" review thread, add_lora_slice pseudocode;
// "TGI Multi-LoRA" page, "Technical Foundation: LoRA").
//
// Design for sm_100a:
//  * A cluster of CL CTAs (8 by default; 4, 2 or 1 through the "decode_cluster" option or when
//    the exchange buffers of wider clusters do not fit) owns one work unit at a time: up to 16
//    tokens of one adapter (a 16-token chunk of an SGMV segment, or of a group of equal ids in
//    the per-token BGMV form).  CTA j of the cluster streams the j-th CL-th of h for the shrink
//    and the j-th CL-th of o for the expand, so each adapter's A_i and B_i are read once per
//    unit and every token of the unit reuses that read.  Segment chunks are dealt to clusters
//    round-robin (or, when the table's ranks differ, in runs of about equal estimated work),
//    so a long segment spreads over many clusters.
//  * One producer warp per CTA runs ahead across units: it stages this CTA's slice of A_i with
//    2-D tensor-map TMA loads (one or two instructions per unit) and its slice of B_i with one
//    bulk copy, into a ring of shared-memory stages guarded by mbarriers, and hints the unit's
//    x and y rows into L2.  No multicast anywhere.
//  * Consumer warps load the next tile's x (or y) rows with coalesced 128-bit loads while the
//    current tile computes.  Shrink: warp-level split-K; a warp owns rank rows k = warp + 8 i, a
//    lane 16 bytes at two places of each 1 KiB row; two tokens x two rows are formed at once
//    (bf16 x bf16 -> fp32 fused multiply-adds straight from the packed words, even and odd
//    elements in two chains) and folded across the warp by one transposed butterfly.
//  * Each CTA pushes its partial intermediate into every peer's shared memory with st.async
//    (completion counted in bytes on the peer's mbarrier); every CTA then sums the CL partials
//    in fixed CTA order.  No atomics, no grid barrier: bit-identical run to run.  A cluster of
//    one keeps its own sum and exchanges nothing.  The three-stage form applies the adapter's
//    Sigma_i (full or diagonal) to the summed intermediate here.
//  * Expand: a thread owns two output columns (bf16) and takes the unit's tokens two or four
//    at a time, sharing each B_i load; it walks its B rows from a rotated 16-byte chunk so a
//    quarter warp hits distinct shared-memory banks; one rounding (nearest-even) per output,
//    coalesced 32-bit stores.  A per-token weight (merged ensembles) multiplies the scale; with
//    an fp32 sum (merged ensembles rounded once) the term is added there instead of into y.
//  * A grouped launch carries up to four projections (tables, x, y slices); each unit runs
//    the shrink tiles of every projection, one cluster exchange of all their partials, then
//    the expand tiles, back to back on the same cluster.
//  * Short kernels like this one are dominated by instruction fetch and dependent latency, so
//    the per-unit code is kept to a few compact loops (no run-time integer division), and
//    work that reads no input (barrier set-up; in the direct BGMV mode the adapter descriptor
//    and the copies of the first stages of the cluster's adapter) happens before the wait on
//    the previous grid.
//  * Persistent grid: as many clusters as fit, each walking the unit list with a stride.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <climits>
#include <mutex>
#include <type_traits>

#include "lora_common.cuh"
#include "lora_internal.h"

namespace lora {
#ifdef LORA_TRACE
__device__ unsigned long long lora_trace_buf[kTraceCtas * kTraceSlots];
#endif
namespace {

constexpr int kMaxCluster = 8;
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;   // + one producer warp
constexpr int kTokChunk = 16;               // tokens per work unit
// Cost-balanced split of segment-table units over the clusters: a unit's estimated work is a
// fixed part plus tokens x rank, in the proportion measured on this kernel (about 2.5 us per
// unit plus 21 ns per token-rank at 4096 -> 4096).
constexpr int kUnitFixedCost = 120;
constexpr int kRowBytes = 1024;             // h-subtile row (shrink) / o-subtile span (expand);
                                            // 512 for ranks above 64 (smaller stages)
constexpr int kBoxBytes = 512;              // one TMA box row of A
constexpr int kMaxStages = 4;
constexpr int kHeaderBytes = 256;

enum : int32_t { kTileShrink = 1, kTileExpand = 2, kTileEnd = 3 };
enum : int32_t { kFlagFirst = 1, kFlagLast = 2 };

struct __align__(16) StageHeader {
    int32_t kind, flags, adapter, rank;
    float scale;
    int32_t L, off, len;   // tokens; first column of h (shrink) or row of o (expand); extent
    int32_t proj;          // projection of a grouped launch
    int32_t skind;         // LORA_SIGMA_*: the unit's Sigma_i (three-stage form)
    const float *sigma;
    int32_t tok[kTokChunk];
    float tw[kTokChunk];   // per-token weight of a merged ensemble slot (1 otherwise)
};
static_assert(sizeof(StageHeader) <= kHeaderBytes, "header");

struct __align__(8) SmemCtl {
    uint64_t full[kMaxStages];    // TMA data landed (tx bytes) + producer arrival
    uint64_t meta[kMaxStages];    // header written (producer arrival)
    uint64_t empty[kMaxStages];   // consumer warps released the stage
    uint64_t recv;                // peers' partials landed (tx bytes) + own arrival
    uint64_t freed;               // every peer finished reading its partials of the last unit
    int32_t n_groups;
    int32_t pending[kTokChunk];   // producer's token list while grouping ids
};
constexpr int kCtlBytes = 256;
#ifndef LORA_TRACE_TILE0
#define LORA_TRACE_TILE0 0
#endif
constexpr int kTraceTile0 = LORA_TRACE_TILE0;   // instrumented builds: first of the two traced tiles
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
    int ids_off, xs_off, ys_off, vpart_off, recv_off, vsum_off, stage_off, RP, total;
};

__host__ __device__ inline int row_bytes_for(int R) { return R > 64 ? kRowBytes / 2 : kRowBytes; }

// VP: projections whose intermediates share one exchange (a grouped launch with one exchange
// per unit), else 1.  A token's row of the partial / intermediate holds VP slices of RP floats.
__host__ __device__ inline Layout make_layout(int src, int R, int n, int T, int stages, int stage_bytes, int CL,
                                              int VP)
{
    Layout l;
    const int rowb = row_bytes_for(R);
    l.RP = round_up(R, 8);
    const int VS = VP * l.RP;
    l.ids_off = kCtlBytes;
    // ids, first member and count per adapter, leaders, weights, chunk offsets per group
    const int ids_bytes = (src == kSrcIds) ? round_up(4 * (4 * T + n + 1), 128) : 0;
    // x rows (shrink tiles) and y rows (expand tiles) share one buffer: a tile stages only one
    // of them, after every consumer is done with the previous tile's
    l.xs_off = l.ids_off + ids_bytes;
    l.ys_off = l.xs_off;
    l.vpart_off = l.ys_off + kTokChunk * rowb;
    l.recv_off = l.vpart_off + round_up(kTokChunk * VS * 4, 128);
    if (CL > 1) {
        l.vsum_off = l.recv_off + CL * kTokChunk * VS * 4;
        l.stage_off = l.vsum_off + round_up(kTokChunk * VS * 4, 128);
    } else {   // no exchange: the CTA's own partial is the unit's intermediate
        l.recv_off = l.vsum_off = l.vpart_off;
        l.stage_off = l.vpart_off + round_up(kTokChunk * VS * 4, 128);
    }
    l.total = l.stage_off + stages * stage_bytes;
    return l;
}

__device__ __forceinline__ void cvt16(const uint4 w, float *o, __nv_bfloat16 *)
{
    o[0] = bf16_lo(w.x); o[1] = bf16_hi(w.x); o[2] = bf16_lo(w.y); o[3] = bf16_hi(w.y);
    o[4] = bf16_lo(w.z); o[5] = bf16_hi(w.z); o[6] = bf16_lo(w.w); o[7] = bf16_hi(w.w);
}
__device__ __forceinline__ void cvt16(const uint4 w, float *o, float *)
{
    o[0] = __uint_as_float(w.x); o[1] = __uint_as_float(w.y);
    o[2] = __uint_as_float(w.z); o[3] = __uint_as_float(w.w);
}

__device__ __forceinline__ int ceil_log2(int v) { return v <= 1 ? 0 : 32 - __clz(v - 1); }

// lo += a.lo * b.lo and hi += a.hi * b.hi for packed bf16 pairs, each product taken exactly and
// added with one rounding (a bf16 x bf16 fused multiply-add into fp32, no unpacking).
__device__ __forceinline__ void fma_bf16x2(uint32_t a, uint32_t b, float &lo, float &hi)
{
    asm("{\n .reg .b16 al, ah, bl, bh;\n"
        " mov.b32 {al, ah}, %2;\n"
        " mov.b32 {bl, bh}, %3;\n"
        " fma.rn.f32.bf16 %0, al, bl, %0;\n"
        " fma.rn.f32.bf16 %1, ah, bh, %1;\n}"
        : "+f"(lo), "+f"(hi)
        : "r"(a), "r"(b));
}


template <typename E, int MODE, int SRC, int CL>
__global__ void __launch_bounds__(kThreads, 2) lora_decode_kernel(const __grid_constant__ DecodeParams p)
{
    using T_ = Tr<E>;
    constexpr int ESZ = T_::ESZ, EPC = T_::EPC, CPT = T_::CPT;
    constexpr int BOXW = kBoxBytes / ESZ;       // elements of one TMA box row
    const int rowb = row_bytes_for(p.R);        // bytes of one staged row
    const int W = rowb / ESZ;                   // elements of one h-subtile / rows of one o-subtile
    const int CHUNKS = rowb / 16;               // 16-byte chunks per staged row (64 or 32)
    const int lgC = CHUNKS == 64 ? 6 : 5;

    extern __shared__ __align__(128) uint8_t smem[];
    SmemCtl &ctl = *reinterpret_cast<SmemCtl *>(smem);
    const int VP = p.mx ? p.P : 1;   // projections sharing one exchange per unit
    const Layout lay = make_layout(SRC, p.R, p.n, p.T, p.stages, p.stage_bytes, CL, VP);
    uint8_t *xs = smem + lay.xs_off;
    uint8_t *ys = smem + lay.ys_off;
    float *vpart = reinterpret_cast<float *>(smem + lay.vpart_off);   // [kTokChunk][RP] this CTA's partial
    float *recv = reinterpret_cast<float *>(smem + lay.recv_off);     // [CL][kTokChunk][RP] from peers
    float *vsum = reinterpret_cast<float *>(smem + lay.vsum_off);     // [kTokChunk][RP] the unit's intermediate
    uint8_t *stage_base = smem + lay.stage_off;
    const int RP = lay.RP;
    const int lgRP = ceil_log2(RP);
    const int VS = VP * RP;                // floats per token row of vpart / recv / vsum
    const int lgVS = ceil_log2(VS);
    const int S = p.stages;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t crank = cluster_ctarank();
    const int cid = (int)cluster_id_x(), G = (int)nclusters_x();

    if (tid == 0) LORA_TRACE_MARK(0);
    // Set-up that reads no input may overlap the previous grid (programmatic launch).
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&ctl.full[s]), 1);
            mbar_init(smem_u32(&ctl.meta[s]), 1);
            mbar_init(smem_u32(&ctl.empty[s]), kConsumerWarps);
        }
        mbar_init(smem_u32(&ctl.recv), 1);
        mbar_init(smem_u32(&ctl.freed), CL);
        fence_mbar_init_cluster();
    }
    __syncthreads();            // barriers initialised for this CTA
    if (CL > 1) cluster_arrive_relaxed();   // peers wait for this before their first remote access

    // This CTA's share of projection pi: a range of h in 16-byte chunks (shrink) and a range
    // of o in EPC-row groups (expand), and the tiles they make.
    const int lgW = lgC + 4 - (ESZ == 2 ? 1 : 2);   // W = 2^lgW
    struct Geo {
        int hc0, hc1, og0, orows, n_shrink, n_expand;
    };
    auto geo_of = [&](int pi) -> Geo {
        Geo g;
        const int hchunks = p.pj[pi].h / EPC, ogroups = p.pj[pi].o / EPC;
        g.hc0 = (int)((int64_t)crank * hchunks / CL);
        g.hc1 = (int)((int64_t)(crank + 1) * hchunks / CL);
        g.og0 = (int)((int64_t)crank * ogroups / CL);
        const int og1 = (int)((int64_t)(crank + 1) * ogroups / CL);
        g.n_shrink = (MODE == kModeExpand) ? 0 : max(1, (g.hc1 - g.hc0 + CHUNKS - 1) >> lgC);
        g.orows = (og1 - g.og0) * EPC;
        g.n_expand = (MODE == kModeShrink) ? 0 : (g.orows + W - 1) >> lgW;
        return g;
    };
    // Geometry of tile j of a unit: shrink tiles first (a slice of h, A by TMA boxes), then
    // expand tiles (W rows of o, one bulk copy of B).  Returns the bytes the tile brings in.
    auto tile_geom = [&](const Geo &g, int j, int r, int &off, int &len, int &nbox) -> uint32_t {
        if (j < g.n_shrink) {
            const int c0 = g.hc0 + j * CHUNKS;
            const int c1 = min(g.hc1, c0 + CHUNKS);
            off = c0 * EPC;
            len = max(0, c1 - c0) * EPC;
            nbox = (len + BOXW - 1) / BOXW;
            return (uint32_t)(nbox * r * kBoxBytes);
        }
        const int jj = j - g.n_shrink;
        off = g.og0 * EPC + jj * W;
        len = min(W, g.orows - jj * W);
        nbox = 0;
        return (uint32_t)(len * r * ESZ);
    };
    // One thread: expect the bytes of tile j of adapter a (projection pi) on stage s and start
    // its copies.
    auto issue_tile = [&](const Geo &g, int pi, int j, int a, const AdapterDesc &d, int s) {
        int off, len, nbox;
        const uint32_t bytes = tile_geom(g, j, d.rank, off, len, nbox);
        const uint32_t data = smem_u32(stage_base + (size_t)s * p.stage_bytes + kHeaderBytes);
        const uint32_t fb = smem_u32(&ctl.full[s]);
        mbar_arrive_expect_tx(fb, bytes);
        // Test-only stall (option "inject_stall"): the first tile of every unit is armed but its
        // copies are never started, so its phase never completes and the consumers' bounded
        // wait runs out.  No copy is in flight for it.
        if (p.inject && j == 0) return;
        if (j < g.n_shrink) {
            const char *tmapA = reinterpret_cast<const char *>(p.pj[pi].tmA) + (size_t)a * 128;
            for (int b = 0; b < nbox; ++b) tma_load_2d(data + b * d.rank * kBoxBytes, tmapA, off + b * BOXW, 0, fb);
        } else if (len > 0) {
            bulk_g2s(data, static_cast<const uint8_t *>(d.B) + (int64_t)off * d.rank * ESZ, len * d.rank * ESZ, fb);
        }
    };

    // Per-token ids: tokens with equal ids form one group.  With no more adapters than
    // clusters and at most two tokens per adapter on average, cluster c owns adapter c and its
    // producer scans the ids itself.  Otherwise a group is led by the first token carrying its
    // id, groups are listed in leader order, and their 16-token chunks are numbered group by
    // group and dealt to the clusters round-robin (so a heavy group spreads over many).
    int32_t *ids_s = reinterpret_cast<int32_t *>(smem + lay.ids_off);
    int32_t *first = ids_s + p.T;       // per adapter: first member (low 16 bits), count (high)
    int32_t *leaders = first + p.n;
    float *w_s = reinterpret_cast<float *>(leaders + p.T);   // per-token merge weights (ids form)
    int32_t *chunk0 = reinterpret_cast<int32_t *>(w_s + p.T);   // [groups + 1] first chunk of each group
    const bool direct_ids = (SRC == kSrcIds) && p.n <= G && p.T <= 2 * p.n;
    // The adapter table is immutable after creation: in direct mode this cluster's descriptor
    // and tensor map are fetched before waiting for the previous grid.
    // The weights are immutable too, so the copies of the first stages of this cluster's
    // adapter start here as well; the tiles are handed to the consumers (with no tokens if the
    // adapter turns out to be unused) once the ids are known.
    // A consumer thread starts them, so the producer warp goes straight on to the ids.
    AdapterDesc pre_desc = {};
    const Geo geo0 = geo_of(0);
    const int npre_all = (direct_ids && cid < p.n) ? min(geo0.n_shrink + geo0.n_expand, S) : 0;
    int npre = 0;
    if (npre_all > 0 && warp == kConsumerWarps) {
        pre_desc = p.pj[0].desc[cid];
        npre = npre_all;
    }
    if (npre_all > 0 && tid == 0) {
        const AdapterDesc d0 = p.pj[0].desc[cid];
        for (int j = 0; j < npre_all; ++j) issue_tile(geo0, 0, j, cid, d0, j);
        if (p.pj[0].sigma_kind != LORA_SIGMA_NONE) {
            const int sbytes = (p.pj[0].sigma_kind == LORA_SIGMA_FULL ? d0.rank * d0.rank : d0.rank) * 4;
            for (int c = 0; c < sbytes; c += 128) prefetch_l2(reinterpret_cast<const uint8_t *>(d0.sigma) + c);
        }
    }
    pdl_wait();
    pdl_launch_dependents();
    if (SRC == kSrcIds && !direct_ids) {
        bool bad = false;
        for (int t0 = tid; t0 < p.T; t0 += 4 * kThreads) {
            int32_t v[4];
            float wv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int t = t0 + kThreads * q;
                v[q] = t < p.T ? p.ids[(int64_t)t * p.ids_stride] : -1;
                wv[q] = (t < p.T && p.tok_w) ? p.tok_w[(int64_t)t * p.w_stride] : 1.f;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int t = t0 + kThreads * q;
                if (t < p.T) {
                    ids_s[t] = v[q];
                    w_s[t] = wv[q];
                    bad |= (v[q] < -1 || v[q] >= p.n);
                }
            }
        }
        for (int i = tid; i < p.n; i += kThreads) first[i] = 0xffff;
        if (__syncthreads_or(bad) && tid == 0 && crank == 0 && cid == 0) atomicOr(p.status, LORA_STATUS_BAD_ID);
        for (int t = tid; t < p.T; t += kThreads) {
            const int32_t a = ids_s[t];
            if (a >= 0 && a < p.n) atomicMin(&first[a], t);
        }
        __syncthreads();
        for (int t = tid; t < p.T; t += kThreads) {   // member counts in the high half (T <= 1024)
            const int32_t a = ids_s[t];
            if (a >= 0 && a < p.n) atomicAdd(&first[a], 1 << 16);
        }
        __syncthreads();
        if (warp == 0) {
            int cnt = 0, chunks = 0;
            for (int base = 0; base < p.T; base += 32) {
                const int t = base + lane;
                const int32_t a = t < p.T ? ids_s[t] : -1;
                const int32_t f = (a >= 0 && a < p.n) ? first[a] : 0;
                const bool lead = a >= 0 && a < p.n && (f & 0xffff) == t;
                const uint32_t m = __ballot_sync(0xffffffffu, lead);
                const int nch = lead ? ((f >> 16) + kTokChunk - 1) / kTokChunk : 0;
                int incl = nch;
#pragma unroll
                for (int dl = 1; dl < 32; dl <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, dl);
                    if (lane >= dl) incl += v;
                }
                if (lead) {
                    const int gi = cnt + __popc(m & ((1u << lane) - 1u));
                    leaders[gi] = t;
                    chunk0[gi] = chunks + incl - nch;
                }
                cnt += __popc(m);
                chunks += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) {
                ctl.n_groups = cnt;
                chunk0[cnt] = chunks;
            }
        }
        __syncthreads();
    }
    // Segment tables: every thread helps stage each segment's length and rank for the
    // producer's cost-balanced split of the units (below).  The stage ring is free until the
    // producer's first tile, so it holds them (8 bytes per segment; larger tables keep the
    // fixed stride).
    int2 *segw = reinterpret_cast<int2 *>(stage_base);
    const int nseg_sc = (SRC == kSrcSegments) ? min(*p.num_segs, p.max_segs) : 0;
    const bool use_part = SRC == kSrcSegments && p.balance &&
                          (int64_t)nseg_sc * (int64_t)sizeof(int2) <= (int64_t)p.stages * p.stage_bytes;
    if (use_part) {
        bool bad = false;
        for (int s0 = tid; s0 < nseg_sc; s0 += 2 * kThreads) {
            int av[2], q0[2], q1[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int sg = s0 + u * kThreads;
                av[u] = -1;
                q0[u] = q1[u] = 0;
                if (sg < nseg_sc) {
                    av[u] = p.seg_adapter[sg];
                    q0[u] = p.seg_ptr[sg];
                    q1[u] = p.seg_ptr[sg + 1];
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int sg = s0 + u * kThreads;
                if (sg < nseg_sc) {
                    const bool okseg = av[u] >= 0 && av[u] < p.n && q0[u] >= 0 && q1[u] >= q0[u] && q1[u] <= p.T;
                    bad |= !okseg;
                    int len = okseg ? q1[u] - q0[u] : 0;
                    if (p.long_len != 0 && len >= p.long_len) len = 0;   // served by the tensor-core kernels
                    segw[sg] = make_int2(len, len > 0 ? p.pj[0].desc[av[u]].rank : 0);
                }
            }
        }
        if (__syncthreads_or(bad) && tid == 0 && crank == 0 && cid == 0) atomicOr(p.status, LORA_STATUS_BAD_SEGMENT);
    }
    if (tid == 0) LORA_TRACE_MARK(1);

    if (warp == kConsumerWarps) {
        // ================================ producer warp ================================
        int issued = 0, ps = 0, pround = 0;   // tiles issued; stage and round of the next one
        bool alive = true;
        if (direct_ids) {
            // stage the ids for this warp's scan; cluster 0 CTA 0 reports bad ids
            // (loads issued four at a time per lane: the ids are on every unit's critical path)
            bool bad = false;
            for (int t0 = lane; t0 < p.T; t0 += 4 * 32) {
                int32_t v[4];
                float wv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int t = t0 + 32 * q;
                    v[q] = t < p.T ? p.ids[(int64_t)t * p.ids_stride] : -1;
                    wv[q] = (t < p.T && p.tok_w) ? p.tok_w[(int64_t)t * p.w_stride] : 1.f;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int t = t0 + 32 * q;
                    if (t < p.T) {
                        ids_s[t] = v[q];
                        w_s[t] = wv[q];
                        bad |= (v[q] < -1 || v[q] >= p.n);
                    }
                }
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0 && crank == 0 && cid == 0)
                atomicOr(p.status, LORA_STATUS_BAD_ID);
            __syncwarp();
        }
        // Walk this cluster's units; each yields (adapter, descriptor, tokens in lanes 0..L-1).
        // Segment tables: units are the 16-token chunks of the segments, numbered segment by
        // segment.  The units are cut into G contiguous runs of about equal estimated work and
        // cluster c takes run c (with the segments staged), else units c, c + G, ...; a long
        // segment spreads over many clusters either way.  A fixed stride can stack several heavy
        // units (many tokens of a high-rank adapter) on one cluster; the runs keep each
        // cluster's work within one unit of the average.  The warp holds a window of 32 segments
        // (lane l: segment sb + l) with the inclusive prefix count of their units and slides it
        // forward as units are taken.
        const int nseg = (SRC == kSrcSegments) ? min(*p.num_segs, p.max_segs) : 0;
        int sb = -32, ubase = 0, w_p0 = 0, w_p1 = 0, w_sa = -1, w_nu = 0, w_incl = 0, w_total = 0;
        int un = cid, un_end = INT_MAX, un_step = G;
        if (use_part) {
            // lane l sums the segments [l B, l B + B): estimated work and units, then scans
            const int B = (nseg + 31) / 32;
            const int s_lo = min(nseg, lane * B), s_hi = min(nseg, s_lo + B);
            long long C = 0;
            int U = 0;
            for (int sg = s_lo; sg < s_hi; ++sg) {
                const int2 e = segw[sg];
                const int nu = (e.x + kTokChunk - 1) / kTokChunk;
                C += (long long)kUnitFixedCost * nu + (long long)e.x * e.y;
                U += nu;
            }
            long long Ci = C;
            int Ui = U;
#pragma unroll
            for (int dl = 1; dl < 32; dl <<= 1) {
                const long long vc = __shfl_up_sync(0xffffffffu, Ci, dl);
                const int vu = __shfl_up_sync(0xffffffffu, Ui, dl);
                if (lane >= dl) {
                    Ci += vc;
                    Ui += vu;
                }
            }
            const long long tot = __shfl_sync(0xffffffffu, Ci, 31);
            const long long Gl = G;
            // units whose doubled midpoint m (twice the work before them plus their own) has
            // m G < X: per segment in closed form (its units cost cf but the last, cl)
            int cnt_lo = 0, cnt_hi = 0;
            {
                long long P = Ci - C;
                const long long Xlo = 2 * tot * cid, Xhi = 2 * tot * (cid + 1);
                for (int sg = s_lo; sg < s_hi; ++sg) {
                    const int2 e = segw[sg];
                    const int nu = (e.x + kTokChunk - 1) / kTokChunk;
                    if (nu == 0) continue;
                    const long long cf = kUnitFixedCost + (long long)kTokChunk * e.y;
                    const long long cl = kUnitFixedCost + (long long)(e.x - kTokChunk * (nu - 1)) * e.y;
                    const long long mlast = 2 * P + 2 * (long long)(nu - 1) * cf + cl;
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        const long long X = w == 0 ? Xlo : Xhi;
                        int c = 0;
                        const long long Y = X - 2 * P * Gl;
                        if (nu > 1 && Y > 0) {
                            const long long q = (Y + cf * Gl - 1) / (cf * Gl);
                            c = (int)min((long long)(nu - 1), q / 2);
                        }
                        if (mlast * Gl < X) c = nu;
                        if (w == 0) cnt_lo += c;
                        else cnt_hi += c;
                    }
                    P += (long long)kUnitFixedCost * nu + (long long)e.x * e.y;
                }
            }
#pragma unroll
            for (int dl = 16; dl >= 1; dl >>= 1) {
                cnt_lo += __shfl_xor_sync(0xffffffffu, cnt_lo, dl);
                cnt_hi += __shfl_xor_sync(0xffffffffu, cnt_hi, dl);
            }
            un = cnt_lo;
            un_end = cnt_hi;
            un_step = 1;
            if (un < un_end) {
                // start the window at the window of 32 segments that holds unit `un`
                const int ub = Ui - U;   // units before this lane's segments
                int hs = -1;
                if (un >= ub && un < Ui) {
                    int acc = ub;
                    for (int sg = s_lo; sg < s_hi; ++sg) {
                        acc += (segw[sg].x + kTokChunk - 1) / kTokChunk;
                        if (un < acc) {
                            hs = sg;
                            break;
                        }
                    }
                }
                const int hsw = __reduce_max_sync(0xffffffffu, hs);
                const int s0w = hsw / 32 * 32;
                int before = 0;
                for (int sg = s_lo; sg < min(s_hi, s0w); ++sg) before += (segw[sg].x + kTokChunk - 1) / kTokChunk;
                before = __reduce_add_sync(0xffffffffu, before);
                sb = s0w - 32;
                ubase = before;
            }
        }
        int g = cid, base = -1, cnt = 0, gi = 0;
        for (;;) {
            int a = -1, my_tok = 0, L = 0;
            AdapterDesc d = {};
            if (SRC == kSrcSegments) {
                while (L == 0) {
                    if (un >= un_end) break;   // this cluster's run is done
                    while (un >= ubase + w_total && sb + 32 < nseg) {
                        ubase += w_total;
                        sb += 32;
                        const int sg = sb + lane;
                        w_nu = 0;
                        w_sa = -1;
                        w_p0 = w_p1 = 0;
                        if (sg < nseg) {
                            w_sa = p.seg_adapter[sg];
                            w_p0 = p.seg_ptr[sg];
                            w_p1 = p.seg_ptr[sg + 1];
                            if (w_sa >= 0 && w_sa < p.n && w_p0 >= 0 && w_p1 >= w_p0 && w_p1 <= p.T) {
                                // a long segment served by the tensor-core kernels has no units here
                                if (p.long_len == 0 || w_p1 - w_p0 < p.long_len)
                                    w_nu = (w_p1 - w_p0 + kTokChunk - 1) / kTokChunk;
                            }
                            else if (cid == 0 && crank == 0)   // every cluster scans every segment
                                atomicOr(p.status, LORA_STATUS_BAD_SEGMENT);
                        }
                        w_incl = w_nu;
#pragma unroll
                        for (int dl = 1; dl < 32; dl <<= 1) {
                            const int v = __shfl_up_sync(0xffffffffu, w_incl, dl);
                            if (lane >= dl) w_incl += v;
                        }
                        w_total = __shfl_sync(0xffffffffu, w_incl, 31);
                    }
                    if (un >= ubase + w_total) break;   // this cluster has no units left
                    const int hl = __ffs(__ballot_sync(0xffffffffu, ubase + w_incl > un)) - 1;
                    const int sa = __shfl_sync(0xffffffffu, w_sa, hl);
                    const int p1 = __shfl_sync(0xffffffffu, w_p1, hl);
                    const int first_unit = ubase + __shfl_sync(0xffffffffu, w_incl - w_nu, hl);
                    const int start = __shfl_sync(0xffffffffu, w_p0, hl) + (un - first_unit) * kTokChunk;
                    un += un_step;
                    d = p.pj[0].desc[sa];
                    const int L0 = min(kTokChunk, p1 - start);
                    int t = -1;
                    if (lane < L0) t = p.perm ? p.perm[start + lane] : start + lane;
                    const bool ok = lane < L0 && t >= 0 && t < p.T;
                    const uint32_t m = __ballot_sync(0xffffffffu, ok);
                    if (m != __ballot_sync(0xffffffffu, lane < L0) && lane == 0 && crank == 0)
                        atomicOr(p.status, LORA_STATUS_BAD_SEGMENT);
                    // compact the valid tokens to lanes 0 .. popc(m) - 1, order kept
                    const int dst = __popc(m & ((1u << lane) - 1u));
                    if (ok) ctl.pending[dst] = t;
                    __syncwarp();
                    my_tok = ctl.pending[lane & (kTokChunk - 1)];
                    __syncwarp();
                    L = __popc(m);
                    a = sa;
                }
            } else if (!direct_ids) {
                // chunk `un` of the numbering: members 16 k .. 16 k + 15 of group gi, in batch
                // order, found by scanning the ids from the group's first member
                const int ng = ctl.n_groups;
                if (un < chunk0[ng]) {
                    while (chunk0[gi + 1] <= un) ++gi;
                    const int t0 = leaders[gi];
                    const int ga = ids_s[t0];
                    int skip = (un - chunk0[gi]) * kTokChunk;
                    int c = 0;
                    for (int bs = t0; bs < p.T && c < kTokChunk; bs += 32) {
                        const int t = bs + lane;
                        const uint32_t m = __ballot_sync(0xffffffffu, t < p.T && ids_s[t] == ga);
                        const int pc = __popc(m);
                        if (skip >= pc) {
                            skip -= pc;
                            continue;
                        }
                        const int take = min(pc - skip, kTokChunk - c);
                        const int rk = __popc(m & ((1u << lane) - 1u)) - skip;
                        if (((m >> lane) & 1u) && rk >= 0 && rk < take) ctl.pending[c + rk] = t;
                        c += take;
                        skip = 0;
                    }
                    __syncwarp();
                    my_tok = ctl.pending[lane & (kTokChunk - 1)];
                    __syncwarp();
                    L = c;
                    a = ga;
                    d = p.pj[0].desc[ga];
                    un += G;
                }
            } else {
                const int ng = min(p.n, cid + 1);
                while (g < ng && L == 0) {
                    const int t0 = 0;
                    const int ga = g;
                    if (base < 0) base = t0;
                    // gather up to kTokChunk members of group g, resuming at `base`
                    while (base < p.T && cnt < kTokChunk) {
                        const int t = base + lane;
                        const uint32_t m = __ballot_sync(0xffffffffu, t < p.T && ids_s[t] == ga);
                        const int take = min(__popc(m), kTokChunk - cnt);
                        const int rk = __popc(m & ((1u << lane) - 1u));
                        if (((m >> lane) & 1u) && rk < take) ctl.pending[cnt + rk] = t;
                        cnt += take;
                        if (take < __popc(m)) {
                            // resume just after the last member taken
                            uint32_t mm = m;
                            for (int i = 0; i < take; ++i) mm &= mm - 1u;
                            base += __ffs(mm) - 1;
                        } else {
                            base += 32;
                        }
                    }
                    __syncwarp();
                    if (cnt > 0) {
                        my_tok = ctl.pending[lane & (kTokChunk - 1)];
                        L = cnt;
                        a = ga;
                        d = pre_desc;
                    }
                    __syncwarp();
                    cnt = 0;
                    if (base >= p.T) {
                        g += G;
                        base = -1;
                    }
                }
            }
            if (L == 0 && npre > 0) {   // copies already started: hand them over with no tokens
                a = cid;
                d = pre_desc;
            } else if (L == 0 || !alive) {
                break;
            }

            // ---- issue every tile of this unit, once per projection (the first npre tiles of
            // projection 0 were started before the grid dependency wait)
            if (lane == 0) LORA_TRACE_MARK(2);
            const int skip = npre;
            npre = 0;
            // With a shared exchange (grouped launch, option decode_shared_exchange) the unit's
            // shrink tiles of every projection come first, then all its expand tiles: the
            // consumers exchange the projections' partials once, after the last shrink tile.
            const int npass = p.mx ? 2 : 1;
            for (int step = 0; step < npass * p.P && alive; ++step) {
                const int pass = step / p.P, pi = step - pass * p.P;
                const ProjParams &pj = p.pj[pi];
                const AdapterDesc dd = pi == 0 ? d : pj.desc[a];
                const Geo g = pi == 0 ? geo0 : geo_of(pi);
                const int r = dd.rank;
                const int ntiles = g.n_shrink + g.n_expand;
                const int j0 = (p.mx && pass == 1) ? g.n_shrink : 0;
                const int j1 = (p.mx && pass == 0) ? g.n_shrink : ntiles;
                if (pj.sigma_kind != LORA_SIGMA_NONE) {   // the consumers read Sigma_i after the shrink
                    const int sbytes = (pj.sigma_kind == LORA_SIGMA_FULL ? r * r : r) * 4;
                    for (int c = lane * 128; c < sbytes; c += 32 * 128)
                        prefetch_l2(reinterpret_cast<const uint8_t *>(dd.sigma) + c);
                }
                for (int j = j0; j < j1; ++j) {
                    const int s = ps, m = pround;
                    if (m >= 1 && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.empty[s]), (m - 1) & 1, p.status,
                                                                      p.wait_ns))) {
                        alive = false;
                        break;
                    }
                    StageHeader *hdr = reinterpret_cast<StageHeader *>(stage_base + (size_t)s * p.stage_bytes);
                    const bool shrink = j < g.n_shrink;
                    int off, len, nbox;
                    tile_geom(g, j, r, off, len, nbox);
                    if (lane < L) {
                        hdr->tok[lane] = my_tok;
                        hdr->tw[lane] = SRC == kSrcIds ? w_s[my_tok]
                                        : !p.tok_w ? 1.f
                                                   : p.tok_w[(int64_t)my_tok * p.w_stride];
                    }
                    if (lane == 0) {
                        hdr->kind = shrink ? kTileShrink : kTileExpand;
                        const int first_j = shrink ? 0 : g.n_shrink;
                        const int last_j = shrink ? g.n_shrink - 1 : ntiles - 1;
                        // the exchange follows the last shrink tile (of the last projection when shared)
                        const bool last = j == last_j && !(shrink && p.mx && pi != p.P - 1);
                        hdr->flags = (j == first_j ? kFlagFirst : 0) | (last ? kFlagLast : 0);
                        hdr->adapter = a;
                        hdr->rank = r;
                        hdr->scale = dd.scale;
                        hdr->L = L;
                        hdr->off = off;
                        hdr->len = len;
                        hdr->proj = pi;
                        hdr->skind = pj.sigma_kind;
                        hdr->sigma = dd.sigma;
                    }
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(smem_u32(&ctl.meta[s]));
                        if (pi > 0 || j >= skip) issue_tile(g, pi, j, a, dd, s);
                    }
                    // L2 hints for the rows the consumers load for this tile (lane l: row l)
                    if (lane < L && (shrink || !p.yacc)) {
                        const uint8_t *row =
                            shrink ? static_cast<const uint8_t *>(pj.x) + ((int64_t)my_tok * pj.ldx + off) * ESZ
                                   : static_cast<const uint8_t *>(pj.y) + ((int64_t)my_tok * pj.ldy + pj.y_off + off) * ESZ;
                        for (int c = 0; c < len * ESZ; c += 128) prefetch_l2(row + c);
                    }
                    ++issued;
                    if (++ps == S) {
                        ps = 0;
                        ++pround;
                    }
                    if (lane == 0) LORA_TRACE_MARK(shrink ? 3 : 4);
                }
            }
        }
        // end marker
        if (alive) {
            const int s = ps, m = pround;
            if (m < 1 || __all_sync(0xffffffffu, mbar_wait(smem_u32(&ctl.empty[s]), (m - 1) & 1, p.status, p.wait_ns))) {
                if (lane == 0) {
                    reinterpret_cast<StageHeader *>(stage_base + (size_t)s * p.stage_bytes)->kind = kTileEnd;
                    mbar_arrive(smem_u32(&ctl.meta[s]));
                    mbar_arrive(smem_u32(&ctl.full[s]));
                }
                ++issued;
            }
        }
        // drain: no copy may still be writing into this CTA's shared memory at exit
        for (int i = max(0, issued - S); i < issued; ++i)
            mbar_wait(smem_u32(&ctl.full[i % S]), (i / S) & 1, p.status, p.wait_ns);
        return;
    }

    // =================================== consumers ===================================
    // The global rows a tile reads (x for a shrink tile, y for an expand tile) are loaded into
    // registers while the previous tile computes, and written to shared memory once every
    // consumer is done with that tile.  Element e = (row l, chunk c) with c < CHUNKS; four per
    // thread at most (16 rows x CHUNKS chunks).
    int u = 0;   // units whose intermediate has been exchanged (fused / shrink modes)
    bool cluster_waited = false;
    uint4 ld[4];
    auto stage_header = [&](int st) -> const StageHeader & {
        return *reinterpret_cast<const StageHeader *>(stage_base + (size_t)st * p.stage_bytes);
    };
    auto load_rows = [&](const StageHeader &h) {
        const bool xr = h.kind == kTileShrink;
        const int L = h.L, nch = h.len / EPC;
        const ProjParams &pj = p.pj[h.proj];
        const uint8_t *src = xr ? static_cast<const uint8_t *>(pj.x) + (int64_t)h.off * ESZ
                                : static_cast<const uint8_t *>(pj.y) + ((int64_t)pj.y_off + h.off) * ESZ;
        const int64_t ld_row = (xr ? pj.ldx : pj.ldy) * ESZ;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + kConsumers * i;
            const int l = e >> lgC, c = e & (CHUNKS - 1);
            ld[i] = make_uint4(0, 0, 0, 0);
            // with an fp32 sum (merged ensembles) the expand never reads y
            if (l < L && c < nch && (xr || !p.yacc))
                ld[i] = *reinterpret_cast<const uint4 *>(src + h.tok[l] * ld_row + c * 16);
        }
    };
    bool live = named_bar_and(1, kConsumers, mbar_wait(smem_u32(&ctl.meta[0]), 0, p.status, p.wait_ns));
    if (live && stage_header(0).kind != kTileEnd) load_rows(stage_header(0));
    int s = 0;          // stage of tile `it`
    uint32_t ph = 0;    // its phase parity
    for (int it = 0; live; ++it) {
        const int s1 = s + 1 == S ? 0 : s + 1;        // stage of the next tile
        const uint32_t ph1 = s1 == 0 ? ph ^ 1u : ph;
        if (tid == 0 && (unsigned)(it - kTraceTile0) < 2u) LORA_TRACE_MARK(5 + 5 * (it - kTraceTile0));
        const StageHeader &hdr = stage_header(s);
        const int kind = hdr.kind;
        if (kind == kTileEnd) break;
        const int r = hdr.rank, L = hdr.L, flags = hdr.flags, len = hdr.len, off = hdr.off;
        const int po = p.mx ? hdr.proj * RP : 0;   // this projection's slice of a token row
        const uint8_t *data = stage_base + (size_t)s * p.stage_bytes + kHeaderBytes;
        const int nch = len / EPC;   // 16-byte chunks per staged row
        if (tid == 0 && u < 6 && kind == kTileShrink && (flags & kFlagFirst)) LORA_TRACE_MARK(40 + 4 * u);

        named_bar_sync(1, kConsumers);   // every consumer is done with the previous tile's buffers
        if (tid == 0 && (unsigned)(it - kTraceTile0) < 2u) LORA_TRACE_MARK(6 + 5 * (it - kTraceTile0));
        uint8_t *rows = kind == kTileShrink ? xs : ys;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + kConsumers * i;
            const int l = e >> lgC, c = e & (CHUNKS - 1);
            if (l < L && c < nch) *reinterpret_cast<uint4 *>(rows + l * rowb + c * 16) = ld[i];
        }
        // next tile's rows (its stage was released S - 1 tiles ago, so its header comes
        // without waiting on this tile)
        const bool okm = mbar_wait(smem_u32(&ctl.meta[s1]), ph1, p.status, p.wait_ns);
        if (okm && stage_header(s1).kind != kTileEnd) load_rows(stage_header(s1));
        const bool okf = mbar_wait(smem_u32(&ctl.full[s]), ph, p.status, p.wait_ns);
        if (tid == 0 && (unsigned)(it - kTraceTile0) < 2u) LORA_TRACE_MARK(7 + 5 * (it - kTraceTile0));
        // every consumer stops together if any of them ran out of time
        if (!named_bar_and(1, kConsumers, okm && okf)) break;
        if (tid == 0 && (unsigned)(it - kTraceTile0) < 2u) LORA_TRACE_MARK(8 + 5 * (it - kTraceTile0));

        if (kind == kTileShrink) {
            const bool first = flags & kFlagFirst;
            if (first && hdr.skind != LORA_SIGMA_NONE) {   // Sigma_i is read after the exchange
                const int sbytes = (hdr.skind == LORA_SIGMA_FULL ? r * r : r) * 4;
                for (int c = tid * 128; c < sbytes; c += kConsumers * 128)
                    prefetch_l1(reinterpret_cast<const uint8_t *>(hdr.sigma) + c);
            }
            // ---- partial shrink over this CTA's slice of h: warp w owns rows w, w + 8, ...;
            // A is staged as [box][row][512 B] (box 1 after r rows of box 0), x as [token][row].
            // Two tokens x two rows at a time: a lane forms the four partial dot products over
            // its 16 elements, and one transposed butterfly folds all four across the warp.
            const bool okA = lane < nch, okB = lane + 32 < nch;
            const uint4 z = make_uint4(0, 0, 0, 0);
            if (ESZ == 2 && warp < r) {
                for (int l = 0; l < L; l += 2) {
                    const bool l2 = l + 1 < L;
                    const uint8_t *xr0 = xs + l * rowb, *xr1 = xr0 + rowb;
                    const uint4 x00 = okA ? *reinterpret_cast<const uint4 *>(xr0 + lane * 16) : z;
                    const uint4 x01 = okB ? *reinterpret_cast<const uint4 *>(xr0 + 512 + lane * 16) : z;
                    const uint4 x10 = l2 && okA ? *reinterpret_cast<const uint4 *>(xr1 + lane * 16) : z;
                    const uint4 x11 = l2 && okB ? *reinterpret_cast<const uint4 *>(xr1 + 512 + lane * 16) : z;
                    const uint32_t xw0[8] = {x00.x, x00.y, x00.z, x00.w, x01.x, x01.y, x01.z, x01.w};
                    const uint32_t xw1[8] = {x10.x, x10.y, x10.z, x10.w, x11.x, x11.y, x11.z, x11.w};
                    for (int k = warp; k < r; k += 2 * kConsumerWarps) {
                        const bool k2 = k + kConsumerWarps < r;
                        float p[4];
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const uint8_t *row = data + (k + q * kConsumerWarps) * kBoxBytes;
                            const bool ok = q == 0 || k2;
                            const uint4 a0 = ok && okA ? *reinterpret_cast<const uint4 *>(row + lane * 16) : z;
                            const uint4 a1 = ok && okB ? *reinterpret_cast<const uint4 *>(row + r * kBoxBytes + lane * 16) : z;
                            const uint32_t aw[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                            float s0 = 0.f, s1 = 0.f, t0 = 0.f, t1 = 0.f;
#pragma unroll
                            for (int w = 0; w < 8; ++w) {
                                fma_bf16x2(xw0[w], aw[w], s0, s1);
                                fma_bf16x2(xw1[w], aw[w], t0, t1);
                            }
                            p[q] = s0 + s1;
                            p[2 + q] = t0 + t1;
                        }
                        const bool hi16 = lane & 16, hi8 = lane & 8;
                        float k0 = hi16 ? p[2] : p[0], k1 = hi16 ? p[3] : p[1];
                        k0 += __shfl_xor_sync(0xffffffffu, hi16 ? p[0] : p[2], 16);
                        k1 += __shfl_xor_sync(0xffffffffu, hi16 ? p[1] : p[3], 16);
                        float tot = hi8 ? k1 : k0;
                        tot += __shfl_xor_sync(0xffffffffu, hi8 ? k0 : k1, 8);
                        tot += __shfl_xor_sync(0xffffffffu, tot, 4);
                        tot += __shfl_xor_sync(0xffffffffu, tot, 2);
                        tot += __shfl_xor_sync(0xffffffffu, tot, 1);
                        if ((lane & 7) == 0 && (!hi16 || l2) && (!hi8 || k2)) {
                            float *dst = vpart + (l + (hi16 ? 1 : 0)) * VS + po + k + (hi8 ? kConsumerWarps : 0);
                            *dst = first ? tot : *dst + tot;
                        }
                    }
                }
            } else if (warp < r) {
                for (int l = 0; l < L; l += 2) {
                    const bool l2 = l + 1 < L;
                    const uint8_t *xr0 = xs + l * rowb, *xr1 = xr0 + rowb;
                    float xv0[2 * EPC], xv1[2 * EPC];
                    cvt16(okA ? *reinterpret_cast<const uint4 *>(xr0 + lane * 16) : z, xv0, (E *)nullptr);
                    cvt16(okB ? *reinterpret_cast<const uint4 *>(xr0 + 512 + lane * 16) : z, xv0 + EPC, (E *)nullptr);
                    cvt16(l2 && okA ? *reinterpret_cast<const uint4 *>(xr1 + lane * 16) : z, xv1, (E *)nullptr);
                    cvt16(l2 && okB ? *reinterpret_cast<const uint4 *>(xr1 + 512 + lane * 16) : z, xv1 + EPC,
                          (E *)nullptr);
                    if (tid == 0 && l == 0 && (unsigned)(it - kTraceTile0) < 2u) LORA_TRACE_MARK(26 + 3 * (it - kTraceTile0));
                    for (int k = warp; k < r; k += 2 * kConsumerWarps) {
                        const bool k2 = k + kConsumerWarps < r;
                        float p[4];   // (token l, row k), (l, k + 8), (l + 1, k), (l + 1, k + 8)
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const uint8_t *row = data + (k + q * kConsumerWarps) * kBoxBytes;
                            const bool ok = q == 0 || k2;
                            float av[2 * EPC];
                            cvt16(ok && okA ? *reinterpret_cast<const uint4 *>(row + lane * 16) : z, av, (E *)nullptr);
                            cvt16(ok && okB ? *reinterpret_cast<const uint4 *>(row + r * kBoxBytes + lane * 16) : z,
                                  av + EPC, (E *)nullptr);
                            float s0 = 0.f, s1 = 0.f, t0 = 0.f, t1 = 0.f;
#pragma unroll
                            for (int e = 0; e < EPC; ++e) {
                                s0 = fmaf(xv0[e], av[e], s0);
                                s1 = fmaf(xv0[EPC + e], av[EPC + e], s1);
                                t0 = fmaf(xv1[e], av[e], t0);
                                t1 = fmaf(xv1[EPC + e], av[EPC + e], t1);
                            }
                            p[q] = s0 + s1;
                            p[2 + q] = t0 + t1;
                        }
                        // lane ends with value j = (lane >> 3) & 3, summed over all 32 lanes
                        if (tid == 0 && l == 0 && k == warp && (unsigned)(it - kTraceTile0) < 2u)
                            LORA_TRACE_MARK(27 + 3 * (it - kTraceTile0));
                        const bool hi16 = lane & 16, hi8 = lane & 8;
                        float k0 = hi16 ? p[2] : p[0], k1 = hi16 ? p[3] : p[1];
                        k0 += __shfl_xor_sync(0xffffffffu, hi16 ? p[0] : p[2], 16);
                        k1 += __shfl_xor_sync(0xffffffffu, hi16 ? p[1] : p[3], 16);
                        float tot = hi8 ? k1 : k0;
                        tot += __shfl_xor_sync(0xffffffffu, hi8 ? k0 : k1, 8);
                        tot += __shfl_xor_sync(0xffffffffu, tot, 4);
                        tot += __shfl_xor_sync(0xffffffffu, tot, 2);
                        tot += __shfl_xor_sync(0xffffffffu, tot, 1);
                        if ((lane & 7) == 0 && (!hi16 || l2) && (!hi8 || k2)) {
                            float *dst = vpart + (l + (hi16 ? 1 : 0)) * VS + po + k + (hi8 ? kConsumerWarps : 0);
                            *dst = first ? tot : *dst + tot;
                        }
                        if (tid == 0 && l == 0 && k == warp && (unsigned)(it - kTraceTile0) < 2u)
                            LORA_TRACE_MARK(28 + 3 * (it - kTraceTile0));
                    }
                }
            }
            if (flags & kFlagLast) {
                if (tid == 0) LORA_TRACE_MARK(15);
                if (tid == 0 && u < 6) LORA_TRACE_MARK(41 + 4 * u);
                named_bar_sync(1, kConsumers);
                if (tid == 0) LORA_TRACE_MARK(16);
                if constexpr (CL > 1) {
                    // ---- push the partial into every CTA of the cluster (this one included)
                    if (!cluster_waited) {
                        cluster_wait_acquire();   // every peer has initialised its barriers
                        cluster_waited = true;
                    }
                    // (a wait that ran out here is acted on, by all consumers together, at the
                    // barrier after the sum)
                    const bool okF =
                        u < 1 || mbar_wait_cluster(smem_u32(&ctl.freed), (u - 1) & 1, p.status, p.wait_ns);
                    if (tid == 0) LORA_TRACE_MARK(17);
                    const int nq = L * VS / 4;            // float4 quads of the partial
                    const int lgq = ceil_log2(nq);
                    const uint32_t my_slot = smem_u32(recv + crank * kTokChunk * VS);
                    const uint32_t rbar = smem_u32(&ctl.recv);
                    for (int e = tid; e < (CL << lgq); e += kConsumers) {
                        const int peer = e >> lgq, qd = e & ((1 << lgq) - 1);
                        if (qd < nq) {
                            const float4 v = *reinterpret_cast<const float4 *>(vpart + qd * 4);
                            st_async_v4(my_slot + qd * 16, rbar, peer, v);
                        }
                    }
                    if (tid == 0) mbar_arrive_expect_tx(rbar, (uint32_t)(CL * nq * 16));
                    if (tid == 0) LORA_TRACE_MARK(18);
                    const bool okR = mbar_wait_cluster(rbar, u & 1, p.status, p.wait_ns);
                    if (tid == 0) LORA_TRACE_MARK(19);
                    // ---- sum the CL partials in CTA order (entries k >= r are never read; with a
                    // shared exchange each projection's slice is summed whole)
                    const int kmax = p.mx ? VS : r;
                    for (int e = tid; e < (L << lgVS); e += kConsumers) {
                        const int l = e >> lgVS, k = e & ((1 << lgVS) - 1);
                        if (k < kmax) {
                            float acc = 0.f;
#pragma unroll
                            for (int j = 0; j < CL; ++j) acc += recv[(j * kTokChunk + l) * VS + k];
                            vsum[l * VS + k] = acc;
                        }
                    }
                    if (tid == 0) LORA_TRACE_MARK(20);
                    if (!named_bar_and(1, kConsumers, okF && okR)) break;
                    if (tid == 0) LORA_TRACE_MARK(21);
                    if (tid < CL) mbar_arrive_remote_relaxed(smem_u32(&ctl.freed), tid);
                    if (tid == 0) LORA_TRACE_MARK(22);
                }
                // (with CL == 1 vpart is vsum and already complete)
                if (hdr.skind == LORA_SIGMA_FULL) {
                    // ---- three-stage form, full Sigma_i: v[l] <- Sigma_i v[l] in fp32.  Thread
                    // (k, g) forms output row k for tokens g, g + G, ...: each load of Sigma_i's
                    // row k serves all of them; products are added in ascending m.
                    const float *S = hdr.sigma;
                    const int lgR = ceil_log2(r);
                    const int G = kConsumers >> lgR;    // token groups (>= 2: r <= 128)
                    const int k = tid & ((1 << lgR) - 1), g = tid >> lgR;
                    float w[8];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) w[jj] = 0.f;
                    if (k < r) {
                        const float *Sk = S + (size_t)k * r;
                        if ((r & 3) == 0 && (reinterpret_cast<uintptr_t>(S) & 15) == 0) {
                            for (int m = 0; m < r; m += 4) {
                                const float4 s4 = __ldg(reinterpret_cast<const float4 *>(Sk + m));
#pragma unroll
                                for (int jj = 0; jj < 8; ++jj) {
                                    const int l = g + G * jj;
                                    if (l < L) {
                                        const float4 v4 = *reinterpret_cast<const float4 *>(vsum + l * RP + m);
                                        w[jj] = fmaf(s4.x, v4.x, w[jj]);
                                        w[jj] = fmaf(s4.y, v4.y, w[jj]);
                                        w[jj] = fmaf(s4.z, v4.z, w[jj]);
                                        w[jj] = fmaf(s4.w, v4.w, w[jj]);
                                    }
                                }
                            }
                        } else {
                            for (int m = 0; m < r; ++m) {
                                const float sv = __ldg(Sk + m);
#pragma unroll
                                for (int jj = 0; jj < 8; ++jj) {
                                    const int l = g + G * jj;
                                    if (l < L) w[jj] = fmaf(sv, vsum[l * RP + m], w[jj]);
                                }
                            }
                        }
                    }
                    named_bar_sync(1, kConsumers);
                    if (k < r) {
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj) {
                            const int l = g + G * jj;
                            if (l < L) vsum[l * RP + k] = w[jj];
                        }
                    }
                    if (MODE == kModeShrink) named_bar_sync(1, kConsumers);
                } else if (hdr.skind == LORA_SIGMA_DIAG) {
                    // ---- diagonal Sigma_i: v[l][k] <- Sigma_i[k] v[l][k], in place
                    const float *S = hdr.sigma;
                    for (int e = tid; e < (L << lgRP); e += kConsumers) {
                        const int l = e >> lgRP, k = e & ((1 << lgRP) - 1);
                        if (k < r) vsum[l * RP + k] = __ldg(S + k) * vsum[l * RP + k];
                    }
                    if (MODE == kModeShrink) named_bar_sync(1, kConsumers);
                }
                if (MODE == kModeShrink && (CL == 1 || crank == 0)) {
                    for (int e = tid; e < (L << lgRP); e += kConsumers) {
                        const int l = e >> lgRP, k = e & ((1 << lgRP) - 1);
                        if (k < r) p.v[(int64_t)hdr.tok[l] * p.ldv + k] = vsum[l * RP + k];
                    }
                }
                if (tid == 0 && u < 6) LORA_TRACE_MARK(42 + 4 * u);
                ++u;
            }
        } else {  // kTileExpand
            if (MODE == kModeExpand && (flags & kFlagFirst)) {
                for (int e = tid; e < (L << lgRP); e += kConsumers) {
                    const int l = e >> lgRP, k = e & ((1 << lgRP) - 1);
                    if (k < r) vsum[l * RP + k] = p.v[(int64_t)hdr.tok[l] * p.ldv + k];
                }
                named_bar_sync(1, kConsumers);
            }
            const float sc = hdr.scale;
            const ProjParams &pj = p.pj[hdr.proj];
            const int c = tid * CPT;   // first column of this thread within the tile
            // starting chunk of this thread's B rows (bf16: rows of 2 r bytes, two per thread)
            int krot = 0;
            if (CPT == 2 && (r % EPC) == 0) {
                const int nchk = r / EPC;
                if ((nchk & (nchk - 1)) == 0) {
                    const int sh = r >= 32 ? 0 : (r == 16 ? 1 : 2);
                    krot = ((tid >> sh) & (nchk - 1)) * EPC;
                }
            }
            // TG tokens per pass share each load (and unpacking) of this thread's B rows: two
            // for the 1-2 token units of wide batches, four for larger units.  Per
            // output the products are added in one fixed order (the thread's rotated chunk
            // order) whatever TG is.  Rows of vsum past L hold stale values; their sums are
            // formed but never stored.
            auto expand_pass = [&](auto tg, int l0) {
                constexpr int TG = decltype(tg)::value;
                const uint8_t *brow = data + (size_t)c * r * ESZ;   // CPT consecutive rows of B
                float acc[TG][CPT];
#pragma unroll
                for (int q = 0; q < TG; ++q)
#pragma unroll
                    for (int j = 0; j < CPT; ++j) acc[q][j] = 0.f;
                if ((r % EPC) == 0) {
                    // Each thread starts its walk over the 16-byte chunks of its B rows at a
                    // rotated chunk, so the lanes of a quarter warp read different bank groups
                    // (rows of 2 r bytes would otherwise put them on one group).
                    for (int kk = 0; kk < r; kk += EPC) {
                        int k = kk + krot;
                        if (k >= r) k -= r;
                        float b[CPT][EPC];
#pragma unroll
                        for (int j = 0; j < CPT; ++j)
                            cvt16(*reinterpret_cast<const uint4 *>(brow + ((size_t)j * r + k) * ESZ), b[j],
                                  (E *)nullptr);
#pragma unroll
                        for (int q = 0; q < TG; ++q) {
                            const float *vr = vsum + (l0 + q) * VS + po + k;
                            float v[EPC];
#pragma unroll
                            for (int e = 0; e < EPC; e += 4) {
                                const float4 a4 = *reinterpret_cast<const float4 *>(vr + e);
                                v[e] = a4.x; v[e + 1] = a4.y; v[e + 2] = a4.z; v[e + 3] = a4.w;
                            }
#pragma unroll
                            for (int j = 0; j < CPT; ++j)
#pragma unroll
                                for (int e = 0; e < EPC; ++e) acc[q][j] = fmaf(v[e], b[j][e], acc[q][j]);
                        }
                    }
                } else {
                    for (int k = 0; k < r; ++k) {
#pragma unroll
                        for (int j = 0; j < CPT; ++j) {
                            const float b = (float)reinterpret_cast<const E *>(brow)[j * r + k];
#pragma unroll
                            for (int q = 0; q < TG; ++q) acc[q][j] = fmaf(vsum[(l0 + q) * VS + po + k], b, acc[q][j]);
                        }
                    }
                }
                if (tid == 0 && l0 == 0 && (unsigned)(it - kTraceTile0) < 2u) LORA_TRACE_MARK(32 + 2 * (it - kTraceTile0));
#pragma unroll
                for (int q = 0; q < TG; ++q) {
                    const int l = l0 + q;
                    if (l >= L) break;
                    const float sl = sc * hdr.tw[l];   // exact when the weight is 1
                    const uint8_t *yr = ys + l * rowb + c * ESZ;
                    const int64_t gofs = (int64_t)hdr.tok[l] * pj.ldy + pj.y_off + off + c;
                    if (p.yacc) {
                        // merged ensembles: the slot's term goes into the fp32 sum, rounded
                        // into y once after the last slot
                        float *ya = p.yacc + (int64_t)hdr.tok[l] * p.ldacc + off + c;
#pragma unroll
                        for (int j = 0; j < CPT; ++j) ya[j] = fmaf(sl, acc[q][j], ya[j]);
                    } else if constexpr (CPT == 2) {
                        const uint32_t w = *reinterpret_cast<const uint32_t *>(yr);
                        const float y0 = fmaf(sl, acc[q][0], bf16_lo(w));
                        const float y1 = fmaf(sl, acc[q][1], bf16_hi(w));
                        *reinterpret_cast<uint32_t *>(static_cast<E *>(pj.y) + gofs) = pack_bf16x2(y0, y1);
                    } else {
                        const float w = *reinterpret_cast<const float *>(yr);
                        static_cast<float *>(pj.y)[gofs] = fmaf(sl, acc[q][0], w);
                    }
                }
                if (tid == 0 && l0 == 0 && (unsigned)(it - kTraceTile0) < 2u) LORA_TRACE_MARK(33 + 2 * (it - kTraceTile0));
            };
            if (c < len) {
                if (L <= 2)
                    expand_pass(std::integral_constant<int, 2>(), 0);
                else
                    for (int l0 = 0; l0 < L; l0 += 4) expand_pass(std::integral_constant<int, 4>(), l0);
            }
        }
        if (tid == 0 && (unsigned)(it - kTraceTile0) < 2u) LORA_TRACE_MARK(9 + 5 * (it - kTraceTile0));
        if (tid == 0 && kind == kTileExpand && (flags & kFlagLast) && u >= 1 && u <= 6) LORA_TRACE_MARK(43 + 4 * (u - 1));
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctl.empty[s]));
        s = s1;
        ph = ph1;
    }
    if (tid == 0) LORA_TRACE_MARK(24);
    // No CTA may leave while a peer can still arrive on its barriers: wait until every peer
    // has released the partials of the last unit.
    if (CL > 1 && MODE != kModeExpand && u >= 1) mbar_wait_cluster(smem_u32(&ctl.freed), (u - 1) & 1, p.status, p.wait_ns);
    if (tid == 0) LORA_TRACE_MARK(25);
}

// Shared-memory size, pipeline depth and co-resident cluster count of one instantiation.
struct LaunchShape {
    int stages, stage_bytes, smem, clusters;
};

template <typename E, int MODE, int SRC, int CL>
int launch_shape(const DecodeParams &p, LaunchShape &ls)
{
    auto kern = lora_decode_kernel<E, MODE, SRC, CL>;
    const Options &opt = options();
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LORA_ERR_CUDA;
    if (dev >= 64) return LORA_ERR_UNSUPPORTED;
    static std::once_flag once[64];
    static int max_optin[64];
    static int n_sms[64];
    std::call_once(once[dev], [&] {
        cudaDeviceGetAttribute(&max_optin[dev], cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaDeviceGetAttribute(&n_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    });
    // Pipeline depth: aim for two CTAs per SM unless told otherwise.
    const int stage_bytes = kHeaderBytes + p.R * row_bytes_for(p.R);
    const int VP = p.mx ? p.P : 1;
    const int fixed = make_layout(SRC, p.R, p.n, p.T, 0, stage_bytes, CL, VP).total;
    const int ctas_per_sm = opt.decode_ctas_per_sm > 0 ? (int)opt.decode_ctas_per_sm : 2;
    int stages = (int)opt.decode_stages;
    if (stages <= 0) {
        const int budget = (228 * 1024) / ctas_per_sm - 1024 - fixed;
        stages = max(2, min(kMaxStages, budget / stage_bytes));
    }
    // at least two stages: consumers read the next tile's header before releasing this one
    stages = max(2, min(kMaxStages, stages));
    while (stages > 2 && make_layout(SRC, p.R, p.n, p.T, stages, stage_bytes, CL, VP).total > max_optin[dev])
        --stages;
    const Layout lay = make_layout(SRC, p.R, p.n, p.T, stages, stage_bytes, CL, VP);
    if (lay.total > max_optin[dev]) return LORA_ERR_UNSUPPORTED;
    static int smem_set[64];
    if (smem_set[dev] < lay.total) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total) != cudaSuccess)
            return LORA_ERR_CUDA;
        smem_set[dev] = lay.total;
    }
    // co-resident clusters for this shared-memory size (cached: a host query, not a stream op)
    static int occ_smem[64], occ_clusters[64];
    if (occ_smem[dev] != lay.total) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CL;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.blockDim = dim3(kThreads);
        cfg.gridDim = dim3(CL);
        cfg.dynamicSmemBytes = (size_t)lay.total;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int mc = 0;
        if (cudaOccupancyMaxActiveClusters(&mc, (void *)kern, &cfg) != cudaSuccess || mc < 1)
            mc = max(1, n_sms[dev] / CL);
        occ_clusters[dev] = mc;
        occ_smem[dev] = lay.total;
    }
    ls.stages = stages;
    ls.stage_bytes = stage_bytes;
    ls.smem = lay.total;
    ls.clusters = occ_clusters[dev];
    return LORA_OK;
}

template <typename E, int MODE, int SRC, int CL>
int launch_one(const DecodeParams &p0, int units, cudaStream_t s)
{
    auto kern = lora_decode_kernel<E, MODE, SRC, CL>;
    LaunchShape ls;
    const int rc = launch_shape<E, MODE, SRC, CL>(p0, ls);
    if (rc != LORA_OK) return rc;
    DecodeParams p = p0;
    p.stages = ls.stages;
    p.stage_bytes = ls.stage_bytes;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)ls.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = CL;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    if (options().pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    int G = max(1, min(ls.clusters, units));
    if (options().decode_max_clusters > 0) G = min(G, (int)options().decode_max_clusters);
    cfg.gridDim = dim3(G * CL);
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return LORA_ERR_CUDA;
    note_launch(kKernDecode);
    return LORA_OK;
}

// Cluster width for a launch: 8 CTAs share each unit unless the "decode_cluster" option asks
// for fewer (1, 2 or 4).  Narrow clusters run more units side by side but stream each unit's
// weights through fewer SMs; measured on the decode workloads here, 8 was never slower.
template <typename E, int MODE, int SRC>
int launch_mode(const DecodeParams &p, cudaStream_t s)
{
    // units: an upper bound on the work units (16-token chunks of one adapter's tokens)
    const int units = max(1, min(p.T, ((SRC == kSrcSegments) ? p.max_segs : p.n) + (p.T + kTokChunk - 1) / kTokChunk));
    const int64_t forced = options().decode_cluster;
    int CL = (forced == 1 || forced == 2 || forced == 4) ? (int)forced : kMaxCluster;
    // The widest width whose pipeline fits in shared memory (the partial-exchange buffers grow
    // with the width).  A shared exchange (grouped launch) multiplies those buffers by the
    // projection count; it is dropped where it would not fit at a width, or would leave fewer
    // than three pipeline stages, so that it never costs cluster width or depth.
    DecodeParams q = p;
    auto shape = [&](int cl, LaunchShape &ls) {
        if (cl == 8) return launch_shape<E, MODE, SRC, 8>(q, ls);
        if (cl == 4) return launch_shape<E, MODE, SRC, 4>(q, ls);
        if (cl == 2) return launch_shape<E, MODE, SRC, 2>(q, ls);
        return launch_shape<E, MODE, SRC, 1>(q, ls);
    };
    for (;; CL >>= 1) {
        LaunchShape ls;
        int rc = shape(CL, ls);
        if (q.mx && (rc == LORA_ERR_UNSUPPORTED || (rc == LORA_OK && ls.stages < 3))) {
            q.mx = 0;
            rc = shape(CL, ls);
        }
        if (rc == LORA_OK || CL == 1 || rc != LORA_ERR_UNSUPPORTED) break;
    }
    switch (CL) {
    case 8: return launch_one<E, MODE, SRC, 8>(q, units, s);
    case 4: return launch_one<E, MODE, SRC, 4>(q, units, s);
    case 2: return launch_one<E, MODE, SRC, 2>(q, units, s);
    default: return launch_one<E, MODE, SRC, 1>(q, units, s);
    }
}

template <typename E>
int launch_typed(int mode, int src, const DecodeParams &p, cudaStream_t s)
{
    if (src == kSrcSegments) {
        if (mode == kModeFused) return launch_mode<E, kModeFused, kSrcSegments>(p, s);
        if (mode == kModeShrink) return launch_mode<E, kModeShrink, kSrcSegments>(p, s);
        return launch_mode<E, kModeExpand, kSrcSegments>(p, s);
    }
    if (mode == kModeFused) return launch_mode<E, kModeFused, kSrcIds>(p, s);
    return LORA_ERR_UNSUPPORTED;
}

}  // namespace

int launch_decode(int mode, int src, const DecodeParams &p, int dtype, cudaStream_t s)
{
    if (!p.pj[0].tmA || p.P < 1 || p.P > kMaxProj) return LORA_ERR_INVALID_ARG;
    if (dtype == LORA_BF16) return launch_typed<__nv_bfloat16>(mode, src, p, s);
    if (dtype == LORA_F32) return launch_typed<float>(mode, src, p, s);
    return LORA_ERR_UNSUPPORTED;
}

// Tensor map of one adapter's A_i [rank, h] for the shrink: boxes of 512 bytes by `rank` rows,
// no swizzle, zero fill past the end of h.
int encode_tmap_A(void *out128, const void *A, int dtype, int h, int rank)
{
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *fn = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!encode) return LORA_ERR_CUDA;
    const int esz = dtype == LORA_BF16 ? 2 : 4;
    const cuuint64_t dims[2] = {(cuuint64_t)h, (cuuint64_t)rank};
    const cuuint64_t strides[1] = {(cuuint64_t)h * esz};
    const cuuint32_t box[2] = {(cuuint32_t)(kBoxBytes / esz), (cuuint32_t)rank};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult rc = encode(reinterpret_cast<CUtensorMap *>(out128),
                               dtype == LORA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                               2, const_cast<void *>(A), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return rc == CUDA_SUCCESS ? LORA_OK : LORA_ERR_UNSUPPORTED;
}

}  // namespace lora

#ifdef LORA_TRACE
// Instrumented builds only: copy the per-CTA phase marks to the host (n <= 4096 * 32 values).
extern "C" int lora_trace_read(unsigned long long *host, int n)
{
    if (n > lora::kTraceCtas * lora::kTraceSlots) n = lora::kTraceCtas * lora::kTraceSlots;
    return cudaMemcpyFromSymbol(host, lora::lora_trace_buf, sizeof(unsigned long long) * n) == cudaSuccess ? 0 : -4;
}
extern "C" int lora_trace_clear(void)
{
    static unsigned long long zero[lora::kTraceCtas * lora::kTraceSlots];
    return cudaMemcpyToSymbol(lora::lora_trace_buf, zero, sizeof zero) == cudaSuccess ? 0 : -4;
}
#endif
