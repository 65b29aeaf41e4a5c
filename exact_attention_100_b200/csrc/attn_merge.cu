// Merge of two partial attention results of the same queries over disjoint key sets: the
// step a sequence-sharded (ring) attention takes after each hop.  With l = exp(LSE) the softmax
// denominator of a part, the union gives O = (l_a O_a + l_b O_b) / (l_a + l_b) and
// LSE = log(l_a + l_b) -- the running rescale of the tiled recurrence ("FlashAttention-2/3",
// section "技术原理") applied to two finished parts.  A part with LSE = -inf (no visible key)
// contributes nothing.
//
// Bandwidth-bound: one warp per row, each lane four columns per step (16-byte loads of the
// float32 accumulator, 8-byte loads of a bf16 part); the weights are computed once per row in
// float32, shifted by the larger LSE so that neither exponential overflows.

#include <cuda_bf16.h>

#include <cstdint>

#include "attn_merge.h"

namespace ea {

namespace {

template <bool PartF32>
__global__ void __launch_bounds__(256) merge_partials_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                             const void* __restrict__ o_part,
                                                             const float* __restrict__ lse_part, long long rows,
                                                             int d) {
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    const float la = lse_acc[row], lb = lse_part[row];
    const float m = fmaxf(la, lb);
    if (m == -INFINITY) continue;  // neither part sees a key: the accumulator stays (0, -inf)
    const float wa = la == -INFINITY ? 0.f : expf(la - m);
    const float wb = lb == -INFINITY ? 0.f : expf(lb - m);
    const float tot = wa + wb;
    const float ca = wa / tot, cb = wb / tot;
    float* acc = o_acc + row * d;
    for (int c = lane * 4; c < d; c += 128) {
      float4 a = *reinterpret_cast<const float4*>(acc + c);
      float4 b;
      if constexpr (PartF32) {
        b = *reinterpret_cast<const float4*>(static_cast<const float*>(o_part) + row * d + c);
      } else {
        const uint2 w = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(o_part) + row * d + c);
        b = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u), __uint_as_float(w.y << 16),
                        __uint_as_float(w.y & 0xFFFF0000u));
      }
      a.x = ca * a.x + cb * b.x;
      a.y = ca * a.y + cb * b.y;
      a.z = ca * a.z + cb * b.z;
      a.w = ca * a.w + cb * b.w;
      *reinterpret_cast<float4*>(acc + c) = a;
    }
    if (lane == 0) lse_acc[row] = m + logf(tot);
  }
}

}  // namespace

cudaError_t launch_merge_partials(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                                  long long rows, int d, int part_f32, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long want = (rows + 7) / 8;                 // 8 rows (warps) per block of 256 threads
  const long long cap = static_cast<long long>(sms) * 8;  // a few waves; the kernel strides over rows
  const int grid = static_cast<int>(want < cap ? want : cap);
  if (part_f32)
    merge_partials_kernel<true><<<grid, 256, 0, stream>>>(o_acc, lse_acc, o_part, lse_part, rows, d);
  else
    merge_partials_kernel<false><<<grid, 256, 0, stream>>>(o_acc, lse_acc, o_part, lse_part, rows, d);
  return cudaGetLastError();
}

}  // namespace ea
