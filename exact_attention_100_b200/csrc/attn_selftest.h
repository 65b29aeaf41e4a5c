// Internal interface of the bounded-wait self-test (attn_selftest.cu).  Not installed.
#pragma once

#include <cuda_runtime.h>

namespace ea {

// One CTA whose thread 0 waits on an mbarrier that nothing arrives at: the library's bounded
// wait gives up after its limit and ORs the timeout bit into *status.
cudaError_t launch_wait_selftest(int* status, cudaStream_t stream);

}  // namespace ea
