// E4M3 instantiation of the attention forward (kernel template in attn_fwd_kernel.cuh).
#include "attn_fwd_kernel.cuh"

namespace ea {

cudaError_t setup_fwd_fp8_kernels() { return set_fwd_smem_attr<128, 2, ElemE4m3>(); }

cudaError_t launch_attn_fwd_fp8(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                const CUtensorMap& o, const FwdParams& p, int num_sms, cudaStream_t stream) {
  if (d != 128) return cudaErrorInvalidValue;
  return launch_fwd<128, 2, ElemE4m3>(q, k, v, o, p, num_sms, stream);
}

}  // namespace ea
