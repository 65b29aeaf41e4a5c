// E4M3 instantiations of the attention forward (kernel template in attn_fwd_kernel.cuh): fixed-length
// and packed variable-length batches.
#include "attn_fwd_kernel.cuh"

namespace ea {

cudaError_t setup_fwd_fp8_kernels() {
  cudaError_t e = set_fwd_smem_attr<64, 2, ElemE4m3>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<128, 2, ElemE4m3>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<256, 1, ElemE4m3>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<64, 2, ElemE4m3, true>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<128, 2, ElemE4m3, true>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<256, 1, ElemE4m3, true>();
  return e;
}

cudaError_t launch_attn_fwd_fp8(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                const CUtensorMap& o, const FwdParams& p, int num_sms, cudaStream_t stream) {
  const bool vl = p.cu_q != nullptr;
  switch (d) {
    case 64:  // rows of 64 bytes: 64-byte TMA boxes and swizzle
      return vl ? launch_fwd<64, 2, ElemE4m3, true>(q, k, v, o, p, num_sms, stream)
                : launch_fwd<64, 2, ElemE4m3>(q, k, v, o, p, num_sms, stream);
    case 128:
      return vl ? launch_fwd<128, 2, ElemE4m3, true>(q, k, v, o, p, num_sms, stream)
                : launch_fwd<128, 2, ElemE4m3>(q, k, v, o, p, num_sms, stream);
    case 256:  // one Q tile per unit, S double-buffered in TMEM (two O tiles of 256 columns do not fit)
      return vl ? launch_fwd<256, 1, ElemE4m3, true>(q, k, v, o, p, num_sms, stream)
                : launch_fwd<256, 1, ElemE4m3>(q, k, v, o, p, num_sms, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace ea
