// lora_sgmv_noalloc: the two-step SGMV (shrink into an fp32 intermediate, then expand) with the
// intermediate held in a fixed array that the library owns, so the caller never has to
// provide or allocate workspace.
//
// Who needs this: code that must not allocate device memory on its own -- for instance a
// serving loop whose framework owns every byte of the GPU through its own allocator, a
// runtime with a fixed memory budget decided at start-up, or a latency-critical path where a
// cudaMalloc/cudaFree (which can synchronise the device) is not acceptable.  Such callers
// pass only inputs and outputs.
//
// The array lives in device global memory for as long as the library is loaded, on every
// GPU that loads it.  Its device address is looked up once per device, with that device
// current, on the first call made on that device, and kept for the life of the process: the
// library must not be used on a device after cudaDeviceReset (or anything else that tears
// down that device's primary context), because the kept address would then be stale.
#include <mutex>

#include "lora_common.cuh"
#include "lora_internal.h"

namespace {

static __device__ __align__(256) float g_noalloc_scratch[LORA_NOALLOC_SCRATCH_FLOATS];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float *g_scratch[kMaxDevices];

// Device address of the array on the current device (looked up once per device).
int scratch_for_current_device(float **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LORA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return LORA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LORA_ERR_CUDA;
        g_scratch[dev] = static_cast<float *>(p);
    }
    *out = g_scratch[dev];
    return LORA_OK;
}

}  // namespace

extern "C" int lora_sgmv_noalloc(const lora_table *table, const lora_segments *seg, const void *x, int64_t ldx,
                                 void *y, int64_t ldy, int32_t y_offset, void *stream)
{
    if (!table || !seg) return LORA_ERR_INVALID_ARG;
    if (seg->T < 0) return LORA_ERR_INVALID_ARG;
    // The array used is the current device's; the table's descriptors live on table->device.
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return LORA_ERR_CUDA;
    if (dev != table->device) return LORA_ERR_INVALID_ARG;
    const int32_t ldv = (table->max_rank + 3) & ~3;
    if ((int64_t)seg->T * ldv > LORA_NOALLOC_SCRATCH_FLOATS) return LORA_ERR_WORKSPACE;
    float *v = nullptr;
    int rc = scratch_for_current_device(&v);
    if (rc != LORA_OK) return rc;
    // The intermediate needs no clearing: the shrink writes v[t, 0:r_i] for every token it
    // covers before the expand reads exactly those entries.
    rc = lora_shrink(table, seg, x, ldx, v, ldv, stream);
    if (rc != LORA_OK) return rc;
    return lora_expand(table, seg, v, ldv, y, ldy, y_offset, stream);
}
