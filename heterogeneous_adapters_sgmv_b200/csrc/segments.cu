// Segment bookkeeping for SGMV: a stable sort of the batch's tokens by adapter id, giving
// the grouping of same-adapter requests that SGMV multiplies segment by segment ("Compress
// then Serve" review thread, authors' rebuttal on Punica).
//
// Two single-CTA (1024-thread) kernels, both giving the unique stable order, bit-identical
// run to run:
//  * counting sort, for decode-sized batches (T <= 512, n < 8192): one histogram of the
//    adapter ids in shared memory (warp-aggregated atomics: counts only, not positions), one
//    exclusive scan of packed (count, non-empty) pairs giving each adapter's first position
//    and its segment index at once, then every token is placed at its adapter's first position plus the number of earlier
//    tokens with the same adapter, so positions never depend on timing (that count costs
//    O(T^2) compares over the block, which is why larger batches take the radix sort);
//  * least-significant-digit radix sort for the rest (8-bit digits, as many passes as the
//    adapter count needs).  Every pass is stable: each warp owns a contiguous run of the
//    input, counts its digits into a private histogram row, the rows are scanned digit-major
//    / warp-minor, and each warp scatters its run in order.
#include <climits>

#include "lora_common.cuh"
#include "lora_internal.h"

namespace lora {
namespace {

constexpr int kSegThreads = 1024;
constexpr int kSegWarps = kSegThreads / 32;
constexpr int kHistEntries = 256 * kSegWarps;

// In-place exclusive scan of a[0, count) (count <= 8192) over all 1024 threads; *total gets
// the sum.  Ends with a __syncthreads().
__device__ void block_exclusive_scan(int32_t *a, int count, int32_t *warp_sums, int32_t *total)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (count + kSegThreads - 1) / kSegThreads;
    const int beg = min(tid * per, count), end = min(beg + per, count);
    int32_t local = 0;
    for (int i = beg; i < end; ++i) local += a[i];
    int32_t incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int32_t o = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += o;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int32_t w = warp_sums[lane];
        int32_t wi = w;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t o = __shfl_up_sync(0xffffffffu, wi, d);
            if (lane >= d) wi += o;
        }
        warp_sums[lane] = wi - w;
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    int32_t run = warp_sums[warp] + incl - local;
    for (int i = beg; i < end; ++i) {
        const int32_t v = a[i];
        a[i] = run;
        run += v;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kSegThreads, 1)
build_segments_kernel(const int32_t *__restrict__ ids, int32_t T, int32_t n, int32_t *__restrict__ perm,
                      int32_t *__restrict__ seg_ptr, int32_t *__restrict__ seg_adapter,
                      int32_t *__restrict__ num_segs, uint32_t *__restrict__ status)
{
    pdl_wait();
    pdl_launch_dependents();

    extern __shared__ __align__(16) int32_t sm[];
    int32_t *keyA = sm, *valA = sm + T, *keyB = sm + 2 * T, *valB = sm + 3 * T;
    int32_t *hist = sm + 4 * T;   // kHistEntries, later reused for the boundary scan (T <= 8192)
    __shared__ int32_t warp_sums[kSegWarps];
    __shared__ int32_t total, valid_s;
    __shared__ uint32_t bad;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        bad = 0;
        valid_s = 0;
    }
    __syncthreads();
    // Keys: the adapter id; "no adapter" (-1) and out-of-range ids get the sentinel n, which
    // sorts after every real adapter and is dropped below.
    for (int t = tid; t < T; t += kSegThreads) {
        const int32_t id = ids[t];
        int32_t key = n;
        if (id >= 0 && id < n)
            key = id;
        else if (id != -1)
            bad = 1;
        keyA[t] = key;
        valA[t] = t;
    }
    __syncthreads();
    if (tid == 0 && bad) atomicOr(status, LORA_STATUS_BAD_ID);

    const int bits = 32 - __clz(n);                       // enough bits for keys 0..n
    const int chunk = (((T + kSegWarps - 1) / kSegWarps) + 31) & ~31;
    const int wbeg = warp * chunk, wend = min(wbeg + chunk, T);
    for (int shift = 0; shift < bits; shift += 8) {
        const int D = min(8, bits - shift);
        const uint32_t dmask = (1u << D) - 1u;
        const int nb = 1 << D;
        for (int i = tid; i < nb * kSegWarps; i += kSegThreads) hist[i] = 0;
        __syncthreads();
        // per-warp digit counts (row `warp` of a digit-major table)
        for (int base = wbeg; base < wend; base += 32) {
            const int t = base + lane;
            const bool ok = t < wend;
            const uint32_t d = ok ? ((uint32_t)keyA[t] >> shift) & dmask : 0xffffffffu;
            const uint32_t peers = __match_any_sync(0xffffffffu, d);
            if (ok && lane == __ffs(peers) - 1) hist[d * kSegWarps + warp] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();
        block_exclusive_scan(hist, nb * kSegWarps, warp_sums, &total);
        // stable scatter of each warp's run
        for (int base = wbeg; base < wend; base += 32) {
            const int t = base + lane;
            const bool ok = t < wend;
            const uint32_t d = ok ? ((uint32_t)keyA[t] >> shift) & dmask : 0xffffffffu;
            const uint32_t peers = __match_any_sync(0xffffffffu, d);
            if (ok) {
                const int pos = hist[d * kSegWarps + warp] + __popc(peers & ((1u << lane) - 1u));
                keyB[pos] = keyA[t];
                valB[pos] = valA[t];
            }
            __syncwarp();
            if (ok && lane == __ffs(peers) - 1) hist[d * kSegWarps + warp] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();
        int32_t *tk = keyA; keyA = keyB; keyB = tk;
        int32_t *tv = valA; valA = valB; valB = tv;
    }

    // Segment starts: first position of every distinct real key.
    for (int p = tid; p < T; p += kSegThreads) {
        const int32_t k = keyA[p];
        hist[p] = (k < n && (p == 0 || keyA[p - 1] != k)) ? 1 : 0;
        if (k < n && (p + 1 == T || keyA[p + 1] >= n)) valid_s = p + 1;
    }
    __syncthreads();
    block_exclusive_scan(hist, T, warp_sums, &total);
    const int32_t S = total;
    for (int p = tid; p < T; p += kSegThreads) {
        const int32_t k = keyA[p];
        if (k < n && (p == 0 || keyA[p - 1] != k)) {
            seg_ptr[hist[p]] = p;
            seg_adapter[hist[p]] = k;
        }
    }
    const int32_t valid = valid_s;
    for (int p = tid; p < valid; p += kSegThreads) perm[p] = valA[p];
    if (tid == 0) {
        seg_ptr[S] = valid;
        *num_segs = S;
    }
}

// Counting sort (see above).  Shared memory: cnt[n + 1], key[T].  One scan gives both the first
// position of each adapter and its segment index: entry i holds (count_i << 16) | (count_i > 0)
// before the scan, so after it the high half is the position and the low half the number of
// non-empty adapters before i (T <= 512 and n <= 8191 keep both halves below 2^16).
__global__ void __launch_bounds__(kSegThreads, 1)
count_segments_kernel(const int32_t *__restrict__ ids, int32_t T, int32_t n, int32_t *__restrict__ perm,
                      int32_t *__restrict__ seg_ptr, int32_t *__restrict__ seg_adapter,
                      int32_t *__restrict__ num_segs, uint32_t *__restrict__ status)
{
    pdl_wait();
    pdl_launch_dependents();

    extern __shared__ __align__(16) int32_t sm[];
    int32_t *cnt = sm, *key_s = sm + (n + 1);
    __shared__ int32_t warp_sums[kSegWarps];
    __shared__ int32_t total;
    __shared__ uint32_t bad;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) bad = 0;
    for (int i = tid; i <= n; i += kSegThreads) cnt[i] = 0;
    __syncthreads();
    // keys (out-of-range ids and -1 get the sentinel n) and their histogram
    for (int t0 = 0; t0 < T; t0 += kSegThreads) {
        const int t = t0 + tid;
        const bool ok = t < T;
        int32_t key = n;
        if (ok) {
            const int32_t id = ids[t];
            if (id >= 0 && id < n)
                key = id;
            else if (id != -1)
                bad = 1;
            key_s[t] = key;
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, ok ? key : -1);
        if (ok && lane == __ffs(peers) - 1) atomicAdd(&cnt[key], __popc(peers));
    }
    __syncthreads();
    if (tid == 0 && bad) atomicOr(status, LORA_STATUS_BAD_ID);
    for (int i = tid; i <= n; i += kSegThreads) {
        const int32_t c = cnt[i];
        cnt[i] = (c << 16) | (i < n && c > 0 ? 1 : 0);
    }
    __syncthreads();
    block_exclusive_scan(cnt, n + 1, warp_sums, &total);   // cnt[i]: (first position << 16) | segment
    const int32_t valid = cnt[n] >> 16;
    const int32_t segs = cnt[n] & 0xFFFF;
    for (int i = tid; i < n; i += kSegThreads) {
        const int32_t e = cnt[i];
        if ((cnt[i + 1] >> 16) > (e >> 16)) {
            seg_ptr[e & 0xFFFF] = e >> 16;
            seg_adapter[e & 0xFFFF] = i;
        }
    }
    if (tid == 0) {
        seg_ptr[segs] = valid;
        *num_segs = segs;
    }
    // Place every token at its adapter's first position plus the number of earlier tokens with
    // the same adapter (the stable order), all tokens at once: a thread counts the matches
    // among the keys before its token, read from shared memory in step by its warp's lanes
    // (one broadcast per key), 32 keys per step.
    for (int t0 = warp * 32; t0 < T; t0 += kSegThreads) {
        const int t = t0 + lane;
        const bool ok = t < T;
        const int32_t key = ok ? key_s[t] : -1;
        int rank = 0;
        for (int u0 = 0; u0 < t0; u0 += 32) {
            const int32_t ku = key_s[u0 + lane];
#pragma unroll
            for (int j = 0; j < 32; ++j) rank += __shfl_sync(0xffffffffu, ku, j) == key;
        }
        // the warp's own earlier lanes
        const uint32_t peers = __match_any_sync(0xffffffffu, key);
        rank += __popc(peers & ((1u << lane) - 1u));
        if (ok && key < n) perm[(cnt[key] >> 16) + rank] = t;
    }
}

constexpr int kCountMaxT = 512;   // above this the radix sort is faster (measured)
constexpr int kCountMaxN = 8191;
static_assert(kCountMaxT < 32768 && kCountMaxN < 65536, "packed (position, segment) scan");

}  // namespace

int launch_build_segments(const int32_t *ids, int32_t T, int32_t n, int32_t *perm, int32_t *seg_ptr,
                          int32_t *seg_adapter, int32_t *num_segs, uint32_t *status, cudaStream_t s)
{
    const bool counting = T <= kCountMaxT && n <= kCountMaxN;
    const size_t smem = counting ? (size_t)(n + 1 + T) * sizeof(int32_t)
                                 : (size_t)(4 * T + kHistEntries) * sizeof(int32_t);
    static bool attr_set = false;
    if (!attr_set) {
        const int max_smem = (4 * LORA_MAX_SEGMENT_TOKENS + kHistEntries) * (int)sizeof(int32_t);
        const int max_count = (kCountMaxN + 1 + kCountMaxT) * (int)sizeof(int32_t);
        if (cudaFuncSetAttribute(build_segments_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 max_smem) != cudaSuccess ||
            cudaFuncSetAttribute(count_segments_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 max_count) != cudaSuccess)
            return LORA_ERR_CUDA;
        attr_set = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kSegThreads);
    cfg.dynamicSmemBytes = smem;
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
    if (cudaLaunchKernelEx(&cfg, counting ? count_segments_kernel : build_segments_kernel, ids, T, n, perm,
                           seg_ptr, seg_adapter, num_segs, status) != cudaSuccess)
        return LORA_ERR_CUDA;
    note_launch(counting ? kKernCountSegments : kKernBuildSegments);
    return LORA_OK;
}

}  // namespace lora
