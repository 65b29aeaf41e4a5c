// Internal interface of the partial-result merge (attn_merge.cu).  Not installed.
#pragma once

#include <cuda_runtime.h>

namespace ea {

// (o_acc, lse_acc) <- merge of itself with (o_part, lse_part): rows x d, o_acc float32,
// o_part bf16 (part_f32 == 0) or float32, all contiguous.
cudaError_t launch_merge_partials(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                                  long long rows, int d, int part_f32, cudaStream_t stream);

}  // namespace ea
