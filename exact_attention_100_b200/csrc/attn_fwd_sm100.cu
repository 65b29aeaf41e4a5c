// bf16 instantiations of the attention forward (kernel template in attn_fwd_kernel.cuh).
#include "attn_fwd_kernel.cuh"

namespace ea {

int fwd_units_per_tile_pair(int d) { return d == 256 ? 1 : 2; }

cudaError_t setup_fwd_bf16_kernels() {
  cudaError_t e = set_fwd_smem_attr<64, 2, ElemBf16>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<128, 2, ElemBf16>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<256, 1, ElemBf16>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<64, 2, ElemBf16, true>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<128, 2, ElemBf16, true>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<256, 1, ElemBf16, true>();
  return e;
}

cudaError_t launch_attn_fwd_bf16(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                 const CUtensorMap& o, const FwdParams& p, int num_sms, cudaStream_t stream) {
  const bool vl = p.cu_q != nullptr;
  switch (d) {
    case 64:
      return vl ? launch_fwd<64, 2, ElemBf16, true>(q, k, v, o, p, num_sms, stream)
                : launch_fwd<64, 2, ElemBf16>(q, k, v, o, p, num_sms, stream);
    case 128:
      return vl ? launch_fwd<128, 2, ElemBf16, true>(q, k, v, o, p, num_sms, stream)
                : launch_fwd<128, 2, ElemBf16>(q, k, v, o, p, num_sms, stream);
    case 256:
      return vl ? launch_fwd<256, 1, ElemBf16, true>(q, k, v, o, p, num_sms, stream)
                : launch_fwd<256, 1, ElemBf16>(q, k, v, o, p, num_sms, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace ea
