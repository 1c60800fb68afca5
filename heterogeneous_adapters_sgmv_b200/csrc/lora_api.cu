// C ABI of liblora_sgmv.so: adapter tables, host-side validation, workspace carving and the
// choice of device path.  Nothing here computes the delta; every step runs in the kernels of
// decode.cu, segments.cu and prefill.cu.
#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "lora_common.cuh"
#include "lora_internal.h"

namespace lora {

static int64_t env_or(const char *name, int64_t dflt)
{
    const char *v = std::getenv(name);
    if (!v || !*v) return dflt;
    return std::strtoll(v, nullptr, 10);
}

static std::atomic<int64_t> g_launches[kKernKinds];
static const char *const kKernelNames[kKernKinds] = {
    "lora_decode_kernel", "count_segments_kernel", "build_segments_kernel", "prefill_shrink_kernel",
    "prefill_expand_kernel", "base_gemm_kernel", "merge_finish_kernel",
};

void note_launch(KernelKind k) { g_launches[k].fetch_add(1, std::memory_order_relaxed); }

Options &options()
{
    static Options o;
    static std::once_flag once;
    std::call_once(once, [] {
        o.pdl = env_or("LORA_PDL", o.pdl);
        o.decode_stages = env_or("LORA_DECODE_STAGES", o.decode_stages);
        o.decode_ctas_per_sm = env_or("LORA_DECODE_CTAS_PER_SM", o.decode_ctas_per_sm);
        o.decode_cluster = env_or("LORA_DECODE_CLUSTER", o.decode_cluster);
        o.decode_max_clusters = env_or("LORA_DECODE_MAX_CLUSTERS", o.decode_max_clusters);
        o.prefill_min_seg_len = env_or("LORA_PREFILL_MIN_SEG_LEN", o.prefill_min_seg_len);
        o.prefill_ksplit = env_or("LORA_PREFILL_KSPLIT", o.prefill_ksplit);
        o.split = env_or("LORA_SPLIT", o.split);
        o.tc_min_seg_len = env_or("LORA_TC_MIN_SEG_LEN", o.tc_min_seg_len);
        o.tc_min_tokens = env_or("LORA_TC_MIN_TOKENS", o.tc_min_tokens);
        o.decode_balance = env_or("LORA_DECODE_BALANCE", o.decode_balance);
        o.decode_shared_exchange = env_or("LORA_DECODE_SHARED_EXCHANGE", o.decode_shared_exchange);
    });
    return o;
}

uint64_t wait_limit_ns()
{
    const int64_t v = options().wait_limit_ns;
    return v > 0 ? (uint64_t)v : kWaitLimitNs;
}

// prefill.cu
bool prefill_supported(const lora_table *t);
int launch_prefill(const lora_table *t, const lora_segments *seg, const void *x, int64_t ldx, void *y,
                   int64_t ldy, int32_t y_off, void *v, int32_t *tile_ctr, int32_t min_len, cudaStream_t s);

}  // namespace lora

using namespace lora;

namespace {

static_assert(kMaxProj == LORA_MAX_GROUP, "grouped-call limit");
static_assert(kKernKinds == LORA_KERNEL_KINDS, "kernel kinds");
constexpr int kBgmvMaxT = 1024;
constexpr int kBgmvMaxN = 4096;

inline bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int esz(int dtype) { return dtype == LORA_BF16 ? 2 : 4; }
inline int epc(int dtype) { return 16 / esz(dtype); }
inline size_t up256(size_t b) { return (b + 255) & ~size_t(255); }
inline int ldv_of(const lora_table *t) { return (t->max_rank + 3) & ~3; }

struct WsLayout {
    size_t v, perm, seg_ptr, seg_adapter, num_segs, tile_ctr, total;
};

WsLayout ws_layout(const lora_table *t, int32_t T)
{
    WsLayout w;
    size_t off = 0;
    w.v = off;
    // the fp32 intermediate, or (tcgen05 path) its bf16 hi and lo parts of 64 columns each
    size_t vbytes = (size_t)T * ldv_of(t) * sizeof(float);
    if (t->d_tmaps_pfA) vbytes = std::max(vbytes, (size_t)T * 64 * 2 * sizeof(uint16_t));
    off += up256(vbytes);
    w.perm = off;
    off += up256((size_t)T * sizeof(int32_t));
    w.seg_ptr = off;
    off += up256((size_t)(t->n + 1) * sizeof(int32_t));
    w.seg_adapter = off;
    off += up256((size_t)t->n * sizeof(int32_t));
    w.num_segs = off;
    w.tile_ctr = off + 128;   // the tcgen05 expand's tile counter, in the same 256-byte block
    off += 256;
    w.total = off;
    return w;
}

int check_table(const lora_table *t)
{
    if (!t || !t->d_desc) return LORA_ERR_INVALID_ARG;
    return LORA_OK;
}

int check_io(const lora_table *t, const void *x, int64_t ldx, const void *y, int64_t ldy, int32_t y_off,
             bool need_x, bool need_y)
{
    const int e = epc(t->dtype);
    if (need_x) {
        if (!x) return LORA_ERR_INVALID_ARG;
        if (ldx < t->h) return LORA_ERR_INVALID_ARG;
        if (!al16(x) || ldx % e) return LORA_ERR_UNSUPPORTED;
    }
    if (need_y) {
        if (!y) return LORA_ERR_INVALID_ARG;
        if (y_off < 0 || ldy < (int64_t)y_off + t->o) return LORA_ERR_INVALID_ARG;
        if (!al16(y) || ldy % e || y_off % e) return LORA_ERR_UNSUPPORTED;
    }
    return LORA_OK;
}

int check_segments(const lora_segments *seg)
{
    if (!seg || !seg->seg_ptr || !seg->seg_adapter || !seg->num_segs) return LORA_ERR_INVALID_ARG;
    if (seg->T < 0 || seg->max_segs < 0) return LORA_ERR_INVALID_ARG;
    return LORA_OK;
}

// Whether the decode kernel cuts segment-table units into cost-balanced runs per cluster: it
// pays when unit costs differ widely, i.e. when the ranks do (measured: multi-rank 57.7 -> 45.3
// us per step; with one rank the staging of the table costs more than the balance gains).
int32_t balance_for(int min_rank, int max_rank)
{
    const int64_t o = options().decode_balance;
    if (o >= 0) return o ? 1 : 0;
    return max_rank >= 2 * min_rank ? 1 : 0;
}

DecodeParams base_params(const lora_table *t)
{
    DecodeParams p;
    std::memset(&p, 0, sizeof p);
    p.pj[0].desc = t->d_desc;
    p.pj[0].tmA = t->d_tmaps;
    p.pj[0].h = t->h;
    p.pj[0].o = t->o;
    p.pj[0].sigma_kind = t->sigma_kind;
    p.P = 1;
    p.ids_stride = 1;
    p.w_stride = 1;
    p.n = t->n;
    p.R = t->max_rank;
    p.balance = balance_for(t->min_rank, t->max_rank);
    p.status = t->d_status;
    p.wait_ns = wait_limit_ns();
    p.inject = (int32_t)(options().inject_stall & 1);
    return p;
}

void set_segments(DecodeParams &p, const lora_segments *seg)
{
    p.perm = seg->perm;
    p.seg_ptr = seg->seg_ptr;
    p.seg_adapter = seg->seg_adapter;
    p.num_segs = seg->num_segs;
    p.max_segs = seg->max_segs;
    p.T = seg->T;
}

}  // namespace

extern "C" {

int lora_table_create(lora_table **out, int32_t n, int32_t h, int32_t o, int32_t dtype,
                      const void *const *A, const void *const *B, const int32_t *ranks,
                      const float *scales, void *stream)
{
    if (!out || !A || !B || !ranks || !scales) return LORA_ERR_INVALID_ARG;
    *out = nullptr;
    if (n < 1 || h < 1 || o < 1) return LORA_ERR_INVALID_ARG;
    if (dtype != LORA_BF16 && dtype != LORA_F32) return LORA_ERR_UNSUPPORTED;
    if (h % epc(dtype) || o % epc(dtype)) return LORA_ERR_UNSUPPORTED;
    int max_rank = 0, min_rank = LORA_MAX_RANK;
    for (int i = 0; i < n; ++i) {
        if (!A[i] || !B[i]) return LORA_ERR_INVALID_ARG;
        if (ranks[i] < 1) return LORA_ERR_INVALID_ARG;
        if (ranks[i] > LORA_MAX_RANK) return LORA_ERR_UNSUPPORTED;
        if (!al16(A[i]) || !al16(B[i])) return LORA_ERR_UNSUPPORTED;
        if (ranks[i] > max_rank) max_rank = ranks[i];
        if (ranks[i] < min_rank) min_rank = ranks[i];
    }
    lora_table *t = new (std::nothrow) lora_table();
    if (!t) return LORA_ERR_INVALID_ARG;
    t->n = n;
    t->h = h;
    t->o = o;
    t->dtype = dtype;
    t->max_rank = max_rank;
    t->min_rank = min_rank;
    t->d_desc = nullptr;
    t->d_status = nullptr;
    t->d_tmaps = nullptr;
    t->d_tmaps_pfA = nullptr;
    t->d_tmaps_pfB = nullptr;
    t->sigma_kind = LORA_SIGMA_NONE;
    if (cudaGetDevice(&t->device) != cudaSuccess) {
        delete t;
        return LORA_ERR_CUDA;
    }
    t->A.assign(A, A + n);
    t->B.assign(B, B + n);
    t->ranks.assign(ranks, ranks + n);
    t->scales.assign(scales, scales + n);
    AdapterDesc *h_desc = new (std::nothrow) AdapterDesc[n];
    if (!h_desc) {
        delete t;
        return LORA_ERR_INVALID_ARG;
    }
    for (int i = 0; i < n; ++i) {
        h_desc[i].A = A[i];
        h_desc[i].B = B[i];
        h_desc[i].rank = ranks[i];
        h_desc[i].scale = scales[i];
        h_desc[i].sigma = nullptr;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int rc = LORA_OK;
    std::vector<uint8_t> h_tmaps((size_t)n * 128, 0);
    for (int i = 0; i < n && rc == LORA_OK; ++i)
        rc = encode_tmap_A(h_tmaps.data() + (size_t)i * 128, A[i], dtype, h, ranks[i]);
    if (rc == LORA_OK &&
        (cudaMalloc(&t->d_desc, sizeof(AdapterDesc) * n) != cudaSuccess ||
         cudaMalloc(&t->d_tmaps, (size_t)n * 128) != cudaSuccess || cudaMalloc(&t->d_status, 256) != cudaSuccess ||
         cudaMemcpyAsync(t->d_desc, h_desc, sizeof(AdapterDesc) * n, cudaMemcpyHostToDevice, s) != cudaSuccess ||
         cudaMemcpyAsync(t->d_tmaps, h_tmaps.data(), (size_t)n * 128, cudaMemcpyHostToDevice, s) != cudaSuccess ||
         cudaMemsetAsync(t->d_status, 0, 256, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess))
        rc = LORA_ERR_CUDA;
    delete[] h_desc;
    if (rc == LORA_OK) rc = prefill_build_maps(t);
    if (rc != LORA_OK) {
        lora_table_destroy(t);
        return rc;
    }
    *out = t;
    return LORA_OK;
}

int lora_table_set_sigma(lora_table *t, int32_t kind, const float *const *sigma, void *stream)
{
    if (!t || !t->d_desc) return LORA_ERR_INVALID_ARG;
    if (kind != LORA_SIGMA_NONE && kind != LORA_SIGMA_FULL && kind != LORA_SIGMA_DIAG) return LORA_ERR_INVALID_ARG;
    if (kind != LORA_SIGMA_NONE) {
        if (!sigma) return LORA_ERR_INVALID_ARG;
        for (int i = 0; i < t->n; ++i) {
            if (!sigma[i]) return LORA_ERR_INVALID_ARG;
            if (reinterpret_cast<uintptr_t>(sigma[i]) & 3u) return LORA_ERR_UNSUPPORTED;
        }
    }
    std::vector<AdapterDesc> h_desc(t->n);
    for (int i = 0; i < t->n; ++i) {
        h_desc[i].A = t->A[i];
        h_desc[i].B = t->B[i];
        h_desc[i].rank = t->ranks[i];
        h_desc[i].scale = t->scales[i];
        h_desc[i].sigma = kind == LORA_SIGMA_NONE ? nullptr : sigma[i];
    }
    int prev = 0;
    if (cudaGetDevice(&prev) != cudaSuccess || cudaSetDevice(t->device) != cudaSuccess) return LORA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool ok = cudaMemcpyAsync(t->d_desc, h_desc.data(), sizeof(AdapterDesc) * t->n, cudaMemcpyHostToDevice,
                                    s) == cudaSuccess &&
                    cudaStreamSynchronize(s) == cudaSuccess;
    cudaSetDevice(prev);
    if (!ok) return LORA_ERR_CUDA;
    t->sigma_kind = kind;
    t->sigma.assign(kind == LORA_SIGMA_NONE ? nullptr : sigma, kind == LORA_SIGMA_NONE ? nullptr : sigma + t->n);
    return LORA_OK;
}

int lora_table_destroy(lora_table *t)
{
    if (!t) return LORA_OK;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(t->device);
    cudaDeviceSynchronize();
    if (t->d_desc) cudaFree(t->d_desc);
    if (t->d_status) cudaFree(t->d_status);
    if (t->d_tmaps) cudaFree(t->d_tmaps);
    if (t->d_tmaps_pfA) cudaFree(t->d_tmaps_pfA);
    if (t->d_tmaps_pfB) cudaFree(t->d_tmaps_pfB);
    cudaSetDevice(prev);
    delete t;
    return LORA_OK;
}

int lora_table_info(const lora_table *t, int32_t *n, int32_t *h, int32_t *o, int32_t *max_rank, int32_t *dtype)
{
    if (!t) return LORA_ERR_INVALID_ARG;
    if (n) *n = t->n;
    if (h) *h = t->h;
    if (o) *o = t->o;
    if (max_rank) *max_rank = t->max_rank;
    if (dtype) *dtype = t->dtype;
    return LORA_OK;
}

size_t lora_workspace_bytes(const lora_table *t, int32_t T)
{
    if (!t || T < 0) return 256;
    return ws_layout(t, T).total;
}

int lora_build_segments(const lora_table *t, const int32_t *d_ids, int32_t T, int32_t *d_perm,
                        int32_t *d_seg_ptr, int32_t *d_seg_adapter, int32_t *d_num_segs, void *stream)
{
    int rc = check_table(t);
    if (rc) return rc;
    if (T < 0 || !d_seg_ptr || !d_seg_adapter || !d_num_segs) return LORA_ERR_INVALID_ARG;
    if (T > 0 && (!d_ids || !d_perm)) return LORA_ERR_INVALID_ARG;
    if (T > LORA_MAX_SEGMENT_TOKENS) return LORA_ERR_UNSUPPORTED;
    return launch_build_segments(d_ids, T, t->n, d_perm, d_seg_ptr, d_seg_adapter, d_num_segs, t->d_status,
                                 static_cast<cudaStream_t>(stream));
}

int lora_shrink(const lora_table *t, const lora_segments *seg, const void *x, int64_t ldx, float *v,
                int32_t ldv, void *stream)
{
    int rc = check_table(t);
    if (rc) return rc;
    if ((rc = check_segments(seg))) return rc;
    if ((rc = check_io(t, x, ldx, nullptr, 0, 0, true, false))) return rc;
    if (!v || ldv < t->max_rank) return LORA_ERR_INVALID_ARG;
    if (ldv % 4 || !al16(v)) return LORA_ERR_UNSUPPORTED;
    if (seg->T == 0 || seg->max_segs == 0) return LORA_OK;
    DecodeParams p = base_params(t);
    set_segments(p, seg);
    p.pj[0].x = x;
    p.pj[0].ldx = ldx;
    p.v = v;
    p.ldv = ldv;
    return launch_decode(kModeShrink, kSrcSegments, p, t->dtype, static_cast<cudaStream_t>(stream));
}

int lora_expand(const lora_table *t, const lora_segments *seg, const float *v, int32_t ldv, void *y,
                int64_t ldy, int32_t y_off, void *stream)
{
    int rc = check_table(t);
    if (rc) return rc;
    if ((rc = check_segments(seg))) return rc;
    if ((rc = check_io(t, nullptr, 0, y, ldy, y_off, false, true))) return rc;
    if (!v || ldv < t->max_rank) return LORA_ERR_INVALID_ARG;
    if (ldv % 4 || !al16(v)) return LORA_ERR_UNSUPPORTED;
    if (seg->T == 0 || seg->max_segs == 0) return LORA_OK;
    DecodeParams p = base_params(t);
    set_segments(p, seg);
    p.pj[0].y = y;
    p.pj[0].ldy = ldy;
    p.pj[0].y_off = y_off;
    p.v = const_cast<float *>(v);
    p.ldv = ldv;
    return launch_decode(kModeExpand, kSrcSegments, p, t->dtype, static_cast<cudaStream_t>(stream));
}

int lora_sgmv(const lora_table *t, const lora_segments *seg, const void *x, int64_t ldx, void *y,
              int64_t ldy, int32_t y_off, void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_table(t);
    if (rc) return rc;
    if ((rc = check_segments(seg))) return rc;
    if ((rc = check_io(t, x, ldx, y, ldy, y_off, true, true))) return rc;
    if (seg->T == 0 || seg->max_segs == 0) return LORA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Options &opt = options();
    const bool prefill = opt.prefill_min_seg_len > 0 && seg->max_seg_len >= opt.prefill_min_seg_len &&
                         seg->perm == nullptr && prefill_supported(t);
    if (prefill || opt.split) {
        const WsLayout w = ws_layout(t, seg->T);
        if (!ws || ws_bytes < w.total) return LORA_ERR_WORKSPACE;
        if (!al16(ws)) return LORA_ERR_UNSUPPORTED;
        float *v = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + w.v);
        int32_t *ctr = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + w.tile_ctr);
        if (prefill) return launch_prefill(t, seg, x, ldx, y, ldy, y_off, v, ctr, 0, s);
        if ((rc = lora_shrink(t, seg, x, ldx, v, ldv_of(t), stream))) return rc;
        return lora_expand(t, seg, v, ldv_of(t), y, ldy, y_off, stream);
    }
    DecodeParams p = base_params(t);
    set_segments(p, seg);
    p.pj[0].x = x;
    p.pj[0].ldx = ldx;
    p.pj[0].y = y;
    p.pj[0].ldy = ldy;
    p.pj[0].y_off = y_off;
    // Mixed batches (segments of any length, in any token order, e.g. from lora_build_segments):
    // in a batch of at least "tc_min_tokens" tokens the segments of at least "tc_min_seg_len"
    // tokens go to the tcgen05 kernels (rows gathered through perm), the shorter ones to the
    // decode kernel.  Both read the same segment table and split it by length on the device.
    const bool mixed = opt.tc_min_seg_len > 0 && seg->T >= opt.tc_min_tokens && prefill_supported(t) && ws &&
                       ws_bytes >= ws_layout(t, seg->T).total && al16(ws);
    if (mixed) p.long_len = (int32_t)opt.tc_min_seg_len;
    if ((rc = launch_decode(kModeFused, kSrcSegments, p, t->dtype, s)) != LORA_OK || !mixed) return rc;
    const WsLayout w = ws_layout(t, seg->T);
    float *v = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + w.v);
    int32_t *ctr = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + w.tile_ctr);
    return launch_prefill(t, seg, x, ldx, y, ldy, y_off, v, ctr, (int32_t)opt.tc_min_seg_len, s);
}

int lora_sgmv_base(const lora_table *t, const lora_segments *seg, const void *x, int64_t ldx, const void *W,
                   int64_t ldw, void *y, int64_t ldy, int32_t y_off, int32_t accumulate, void *ws, size_t ws_bytes,
                   void *stream)
{
    int rc = check_table(t);
    if (rc) return rc;
    if ((rc = check_segments(seg))) return rc;
    if ((rc = check_io(t, x, ldx, y, ldy, y_off, true, true))) return rc;
    if (!W || ldw < t->h || (accumulate != 0 && accumulate != 1)) return LORA_ERR_INVALID_ARG;
    if (!al16(W) || ldw % 8) return LORA_ERR_UNSUPPORTED;
    // tensor-core tiles only: bf16 tables with ranks that are multiples of 8 up to 64, no
    // Sigma, tokens contiguous per segment
    if (!prefill_supported(t) || seg->perm != nullptr) return LORA_ERR_UNSUPPORTED;
    if (seg->T == 0) return LORA_OK;
    const WsLayout w = ws_layout(t, seg->T);
    if (!ws || ws_bytes < w.total) return LORA_ERR_WORKSPACE;
    if (!al16(ws)) return LORA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void *v = static_cast<uint8_t *>(ws) + w.v;
    const bool shrink = seg->max_segs > 0;
    if (shrink && (rc = launch_prefill_shrink(t, seg, x, ldx, v, true, s)) != LORA_OK) return rc;
    return launch_base_gemm(t, seg, x, ldx, W, ldw, y, ldy, y_off, accumulate, v, shrink, s);
}

int lora_sgmv_grouped(const lora_table *const *tables, int32_t P, const lora_segments *seg,
                      const void *const *x, const int64_t *ldx, void *const *y, const int64_t *ldy,
                      const int32_t *y_off, void *ws, size_t ws_bytes, void *stream)
{
    if (!tables || !x || !ldx || !y || !ldy || !y_off) return LORA_ERR_INVALID_ARG;
    if (P < 1 || P > kMaxProj) return LORA_ERR_INVALID_ARG;
    int rc;
    if ((rc = check_segments(seg))) return rc;
    for (int i = 0; i < P; ++i) {
        if ((rc = check_table(tables[i]))) return rc;
        if (tables[i]->n != tables[0]->n || tables[i]->dtype != tables[0]->dtype ||
            tables[i]->device != tables[0]->device)
            return LORA_ERR_INVALID_ARG;
        if ((rc = check_io(tables[i], x[i], ldx[i], y[i], ldy[i], y_off[i], true, true))) return rc;
    }
    // The output slices must not overlap: the projections update y concurrently.
    const int e = esz(tables[0]->dtype);
    for (int i = 0; i < P; ++i)
        for (int j = i + 1; j < P; ++j) {
            const int64_t a0 = y_off[i], a1 = a0 + tables[i]->o, b0 = y_off[j], b1 = b0 + tables[j]->o;
            if (y[i] == y[j] && ldy[i] == ldy[j]) {
                if (a0 < b1 && b0 < a1) return LORA_ERR_INVALID_ARG;
                continue;
            }
            const int64_t rows = seg->T > 0 ? seg->T - 1 : 0;
            const uintptr_t pi0 = reinterpret_cast<uintptr_t>(y[i]) + (uintptr_t)(a0 * e);
            const uintptr_t pi1 = reinterpret_cast<uintptr_t>(y[i]) + (uintptr_t)((rows * ldy[i] + a1) * e);
            const uintptr_t pj0 = reinterpret_cast<uintptr_t>(y[j]) + (uintptr_t)(b0 * e);
            const uintptr_t pj1 = reinterpret_cast<uintptr_t>(y[j]) + (uintptr_t)((rows * ldy[j] + b1) * e);
            if (pi0 < pj1 && pj0 < pi1) return LORA_ERR_INVALID_ARG;
        }
    if (seg->T == 0 || seg->max_segs == 0) return LORA_OK;
    const Options &opt = options();
    bool separate = opt.split != 0;
    for (int i = 0; i < P; ++i)
        separate |= opt.prefill_min_seg_len > 0 && seg->max_seg_len >= opt.prefill_min_seg_len &&
                    seg->perm == nullptr && prefill_supported(tables[i]);
    if (separate) {   // long segments (tcgen05 path) or the split option: one call per table
        for (int i = 0; i < P; ++i)
            if ((rc = lora_sgmv(tables[i], seg, x[i], ldx[i], y[i], ldy[i], y_off[i], ws, ws_bytes, stream)))
                return rc;
        return LORA_OK;
    }
    DecodeParams p = base_params(tables[0]);
    set_segments(p, seg);
    p.P = P;
    for (int i = 0; i < P; ++i) {
        const lora_table *t = tables[i];
        ProjParams &pj = p.pj[i];
        pj.desc = t->d_desc;
        pj.tmA = t->d_tmaps;
        pj.h = t->h;
        pj.o = t->o;
        pj.x = x[i];
        pj.ldx = ldx[i];
        pj.y = y[i];
        pj.ldy = ldy[i];
        pj.y_off = y_off[i];
        pj.sigma_kind = t->sigma_kind;
        if (t->max_rank > p.R) p.R = t->max_rank;
        p.balance |= balance_for(t->min_rank, t->max_rank);
    }
    // one exchange per unit for all projections, unless a projection applies Sigma_i after its
    // own exchange
    p.mx = (P > 1 && opt.decode_shared_exchange) ? 1 : 0;
    for (int i = 0; i < P; ++i)
        if (tables[i]->sigma_kind != LORA_SIGMA_NONE) p.mx = 0;
    return launch_decode(kModeFused, kSrcSegments, p, tables[0]->dtype, static_cast<cudaStream_t>(stream));
}

int lora_bgmv(const lora_table *t, const int32_t *d_ids, int32_t T, const void *x, int64_t ldx, void *y,
              int64_t ldy, int32_t y_off, void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_table(t);
    if (rc) return rc;
    if (T < 0) return LORA_ERR_INVALID_ARG;
    if ((rc = check_io(t, x, ldx, y, ldy, y_off, true, true))) return rc;
    if (T == 0) return LORA_OK;
    if (!d_ids) return LORA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T <= kBgmvMaxT && t->n <= kBgmvMaxN && !options().split) {
        DecodeParams p = base_params(t);
        p.ids = d_ids;
        p.T = T;
        p.pj[0].x = x;
        p.pj[0].ldx = ldx;
        p.pj[0].y = y;
        p.pj[0].ldy = ldy;
        p.pj[0].y_off = y_off;
        return launch_decode(kModeFused, kSrcIds, p, t->dtype, s);
    }
    // Larger batches: sort into the workspace, then run the segmented form.
    if (T > LORA_MAX_SEGMENT_TOKENS) return LORA_ERR_UNSUPPORTED;
    const WsLayout w = ws_layout(t, T);
    if (!ws || ws_bytes < w.total) return LORA_ERR_WORKSPACE;
    if (!al16(ws)) return LORA_ERR_UNSUPPORTED;
    uint8_t *b = static_cast<uint8_t *>(ws);
    lora_segments seg;
    std::memset(&seg, 0, sizeof seg);
    seg.perm = reinterpret_cast<int32_t *>(b + w.perm);
    seg.seg_ptr = reinterpret_cast<int32_t *>(b + w.seg_ptr);
    seg.seg_adapter = reinterpret_cast<int32_t *>(b + w.seg_adapter);
    seg.num_segs = reinterpret_cast<int32_t *>(b + w.num_segs);
    seg.T = T;
    seg.max_segs = t->n;
    if ((rc = lora_build_segments(t, d_ids, T, const_cast<int32_t *>(seg.perm), const_cast<int32_t *>(seg.seg_ptr),
                                  const_cast<int32_t *>(seg.seg_adapter), const_cast<int32_t *>(seg.num_segs),
                                  stream)))
        return rc;
    return lora_sgmv(t, &seg, x, ldx, y, ldy, y_off, ws, ws_bytes, stream);
}

int lora_bgmv_merged(const lora_table *t, const int32_t *d_ids, const float *d_w, int32_t T, int32_t K,
                     const void *x, int64_t ldx, void *y, int64_t ldy, int32_t y_off, void *ws, size_t ws_bytes,
                     void *stream)
{
    int rc = check_table(t);
    if (rc) return rc;
    if (T < 0 || K < 1 || K > LORA_MAX_MERGE) return LORA_ERR_INVALID_ARG;
    if ((rc = check_io(t, x, ldx, y, ldy, y_off, true, true))) return rc;
    if (T == 0) return LORA_OK;
    if (!d_ids || !d_w) return LORA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool direct = T <= kBgmvMaxT && t->n <= kBgmvMaxN;
    if (!direct && T > LORA_MAX_SEGMENT_TOKENS) return LORA_ERR_UNSUPPORTED;
    const WsLayout w = ws_layout(t, T);
    if (!direct && (!ws || ws_bytes < w.total)) return LORA_ERR_WORKSPACE;
    if (!direct && !al16(ws)) return LORA_ERR_UNSUPPORTED;
    // One pass per slot, in slot order: each pass is the BGMV update of that slot's adapters
    // with the per-token weight folded into the scale.  With room for an fp32 [T, o] sum after
    // the workspace's own areas the passes add into that sum (zeroed first) and one last launch
    // rounds y + sum once; otherwise y is rounded after each pass.
    const size_t acc_off = (w.total + 255) / 256 * 256;
    const size_t acc_bytes = (size_t)T * t->o * sizeof(float);
    float *yacc = (ws && al16(ws) && ws_bytes >= acc_off + acc_bytes)
                      ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + acc_off)
                      : nullptr;
    if (yacc && cudaMemsetAsync(yacc, 0, acc_bytes, s) != cudaSuccess) return LORA_ERR_CUDA;
    for (int k = 0; k < K; ++k) {
        DecodeParams p = base_params(t);
        p.pj[0].x = x;
        p.pj[0].ldx = ldx;
        p.pj[0].y = y;
        p.pj[0].ldy = ldy;
        p.pj[0].y_off = y_off;
        p.tok_w = d_w + k;
        p.w_stride = K;
        p.yacc = yacc;
        p.ldacc = t->o;
        if (direct) {
            p.ids = d_ids + k;
            p.ids_stride = K;
            p.T = T;
            rc = launch_decode(kModeFused, kSrcIds, p, t->dtype, s);
        } else {
            // slot k's ids into the workspace (the intermediate area, unused by the fused
            // kernel), then the segment bookkeeping and the segmented kernel
            uint8_t *b = static_cast<uint8_t *>(ws);
            int32_t *col = reinterpret_cast<int32_t *>(b + w.v);
            if (cudaMemcpy2DAsync(col, sizeof(int32_t), d_ids + k, sizeof(int32_t) * K, sizeof(int32_t), T,
                                  cudaMemcpyDeviceToDevice, s) != cudaSuccess)
                return LORA_ERR_CUDA;
            lora_segments seg;
            std::memset(&seg, 0, sizeof seg);
            seg.perm = reinterpret_cast<int32_t *>(b + w.perm);
            seg.seg_ptr = reinterpret_cast<int32_t *>(b + w.seg_ptr);
            seg.seg_adapter = reinterpret_cast<int32_t *>(b + w.seg_adapter);
            seg.num_segs = reinterpret_cast<int32_t *>(b + w.num_segs);
            seg.T = T;
            seg.max_segs = t->n;
            if ((rc = lora_build_segments(t, col, T, const_cast<int32_t *>(seg.perm),
                                          const_cast<int32_t *>(seg.seg_ptr), const_cast<int32_t *>(seg.seg_adapter),
                                          const_cast<int32_t *>(seg.num_segs), stream)))
                return rc;
            set_segments(p, &seg);
            rc = launch_decode(kModeFused, kSrcSegments, p, t->dtype, s);
        }
        if (rc) return rc;
    }
    if (yacc) return launch_merge_finish(y, ldy, y_off, yacc, t->o, T, t->o, t->dtype, s);
    return LORA_OK;
}

int lora_get_status(const lora_table *t, uint32_t *h_status, int32_t reset, void *stream)
{
    if (!t || !h_status) return LORA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t w = 0;
    if (cudaMemcpyAsync(&w, t->d_status, sizeof w, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return LORA_ERR_CUDA;
    if (reset && (cudaMemsetAsync(t->d_status, 0, sizeof w, s) != cudaSuccess ||
                  cudaStreamSynchronize(s) != cudaSuccess))
        return LORA_ERR_CUDA;
    *h_status = w;
    if (w == 0) return LORA_OK;
    return (w & LORA_STATUS_TIMEOUT) ? LORA_ERR_TIMEOUT : LORA_ERR_DEVICE_STATUS;
}

const char *lora_status_string(int code)
{
    switch (code) {
    case LORA_OK: return "ok";
    case LORA_ERR_INVALID_ARG: return "invalid argument";
    case LORA_ERR_UNSUPPORTED: return "unsupported configuration (rank, alignment, dtype or size limit)";
    case LORA_ERR_WORKSPACE: return "workspace missing or too small";
    case LORA_ERR_CUDA: return "CUDA runtime error";
    case LORA_ERR_TIMEOUT: return "a device-side bounded wait ran out";
    case LORA_ERR_DEVICE_STATUS: return "the device latched an error (bad id or segment entry)";
    default: return "unknown status";
    }
}

int lora_set_option(const char *key, int64_t value)
{
    if (!key) return LORA_ERR_INVALID_ARG;
    Options &o = options();
    if (!std::strcmp(key, "pdl")) o.pdl = value;
    else if (!std::strcmp(key, "decode_stages")) o.decode_stages = value;
    else if (!std::strcmp(key, "decode_ctas_per_sm")) o.decode_ctas_per_sm = value;
    else if (!std::strcmp(key, "decode_cluster")) o.decode_cluster = value;
    else if (!std::strcmp(key, "decode_max_clusters")) o.decode_max_clusters = value;
    else if (!std::strcmp(key, "prefill_min_seg_len")) o.prefill_min_seg_len = value;
    else if (!std::strcmp(key, "prefill_ksplit")) o.prefill_ksplit = value;
    else if (!std::strcmp(key, "split")) o.split = value;
    else if (!std::strcmp(key, "wait_limit_ns")) o.wait_limit_ns = value;
    else if (!std::strcmp(key, "inject_stall")) o.inject_stall = value;
    else if (!std::strcmp(key, "tc_min_seg_len")) o.tc_min_seg_len = value;
    else if (!std::strcmp(key, "tc_min_tokens")) o.tc_min_tokens = value;
    else if (!std::strcmp(key, "decode_balance")) o.decode_balance = value;
    else if (!std::strcmp(key, "decode_shared_exchange")) o.decode_shared_exchange = value;
    else return LORA_ERR_INVALID_ARG;
    return LORA_OK;
}

int lora_get_option(const char *key, int64_t *value)
{
    if (!key || !value) return LORA_ERR_INVALID_ARG;
    const Options &o = options();
    if (!std::strcmp(key, "pdl")) *value = o.pdl;
    else if (!std::strcmp(key, "decode_stages")) *value = o.decode_stages;
    else if (!std::strcmp(key, "decode_ctas_per_sm")) *value = o.decode_ctas_per_sm;
    else if (!std::strcmp(key, "decode_cluster")) *value = o.decode_cluster;
    else if (!std::strcmp(key, "decode_max_clusters")) *value = o.decode_max_clusters;
    else if (!std::strcmp(key, "prefill_min_seg_len")) *value = o.prefill_min_seg_len;
    else if (!std::strcmp(key, "prefill_ksplit")) *value = o.prefill_ksplit;
    else if (!std::strcmp(key, "split")) *value = o.split;
    else if (!std::strcmp(key, "wait_limit_ns")) *value = o.wait_limit_ns;
    else if (!std::strcmp(key, "inject_stall")) *value = o.inject_stall;
    else if (!std::strcmp(key, "tc_min_seg_len")) *value = o.tc_min_seg_len;
    else if (!std::strcmp(key, "tc_min_tokens")) *value = o.tc_min_tokens;
    else if (!std::strcmp(key, "decode_balance")) *value = o.decode_balance;
    else if (!std::strcmp(key, "decode_shared_exchange")) *value = o.decode_shared_exchange;
    else return LORA_ERR_INVALID_ARG;
    return LORA_OK;
}

const char *lora_kernel_name(int32_t kind)
{
    return kind >= 0 && kind < kKernKinds ? kKernelNames[kind] : nullptr;
}

int64_t lora_kernel_launches(int32_t kind)
{
    return kind >= 0 && kind < kKernKinds ? g_launches[kind].load(std::memory_order_relaxed) : -1;
}

}  // extern "C"
