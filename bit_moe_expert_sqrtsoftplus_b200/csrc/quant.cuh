// quant.cuh -- offline block encoders (fp32 -> Q8_0 / Q2_K), host interface.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kQuantQ80 = MOE_QUANT_Q8_0;
constexpr int kQuantQ2K = MOE_QUANT_Q2_K;
constexpr int kQuantQ4K = MOE_QUANT_Q4_K;

// Encodes nblocks blocks (32 values per Q8_0 block, 256 per Q2_K or Q4_K
// block) from x into out (34-, 84- or 144-byte blocks) on `stream`; blocks
// holding a non-finite value are written as zeros and added to *nonfinite
// when it is not null.
cudaError_t quantize_blocks(int format, const float *x, int64_t nblocks, void *out, int32_t *nonfinite,
                            cudaStream_t stream, int num_sms);

}  // namespace moe
