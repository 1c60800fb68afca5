// Prefill path for long contiguous segments (tcgen05 tensor cores); not yet available in
// this build: lora_sgmv keeps long segments on the decode kernels.
#include "lora_common.cuh"
#include "lora_internal.h"

namespace lora {

bool prefill_supported(const lora_table *) { return false; }

int launch_prefill(const lora_table *, const lora_segments *, const void *, int64_t, void *, int64_t, int32_t,
                   float *, int32_t, cudaStream_t)
{
    return LORA_ERR_UNSUPPORTED;
}

}  // namespace lora
