// Last step of a merged ensemble summed in fp32 (lora_bgmv_merged with the larger workspace):
// the K slots' weighted adapter terms were added into an fp32 array by the decode kernel, one
// pass per slot; this kernel adds that sum to y and rounds once to y's type ("Lorax" pages: a
// request's adapters combined into one weighted update of the layer output).
#include <cuda_bf16.h>

#include <algorithm>

#include "lora_common.cuh"
#include "lora_internal.h"

namespace lora {
namespace {

constexpr int kMergeThreads = 256;

// Two consecutive outputs per thread (o is a multiple of 8 for bf16, 4 for fp32), grid-stride.
template <typename E>
__global__ void __launch_bounds__(kMergeThreads) merge_finish_kernel(E *__restrict__ y, int64_t ldy, int32_t y_off,
                                                                     const float *__restrict__ yacc, int64_t ldacc,
                                                                     int32_t T, int32_t o)
{
    pdl_wait();
    pdl_launch_dependents();
    const int half = o / 2;
    const int64_t pairs = (int64_t)T * half;
    for (int64_t e = (int64_t)blockIdx.x * kMergeThreads + threadIdx.x; e < pairs;
         e += (int64_t)gridDim.x * kMergeThreads) {
        const int64_t t = e / half;
        const int n = (int)(e - t * half) * 2;
        const float2 a = *reinterpret_cast<const float2 *>(yacc + t * ldacc + n);
        E *py = y + t * ldy + y_off + n;
        if constexpr (sizeof(E) == 2) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(py);
            *reinterpret_cast<uint32_t *>(py) = pack_bf16x2(bf16_lo(w) + a.x, bf16_hi(w) + a.y);
        } else {
            py[0] = py[0] + a.x;
            py[1] = py[1] + a.y;
        }
    }
}

}  // namespace

int launch_merge_finish(void *y, int64_t ldy, int32_t y_off, const float *yacc, int64_t ldacc, int32_t T, int32_t o,
                        int dtype, cudaStream_t s)
{
    if (T <= 0 || o <= 0) return LORA_OK;
    int dev = 0, n_sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return LORA_ERR_CUDA;
    const int64_t pairs = (int64_t)T * (o / 2);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>(4 * n_sms, (pairs + kMergeThreads - 1) / kMergeThreads)));
    cfg.blockDim = dim3(kMergeThreads);
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
    const cudaError_t e =
        dtype == LORA_BF16
            ? cudaLaunchKernelEx(&cfg, merge_finish_kernel<__nv_bfloat16>, static_cast<__nv_bfloat16 *>(y), ldy, y_off,
                                 yacc, ldacc, T, o)
            : cudaLaunchKernelEx(&cfg, merge_finish_kernel<float>, static_cast<float *>(y), ldy, y_off, yacc, ldacc, T, o);
    if (e != cudaSuccess) return LORA_ERR_CUDA;
    note_launch(kKernMergeFinish);
    return LORA_OK;
}

}  // namespace lora
