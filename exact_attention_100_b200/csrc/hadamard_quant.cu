// Random-sign Hadamard transform + per-block E4M3 quantisation (bandwidth-bound pre-kernel).
//
// "FlashAttention-3", section "FP8 路径与低精度误差": outliers in Q and K are spread by
// x~ = H D x (D random signs, H Hadamard) before FP8 quantisation; the transform costs
// O(d log d) and is memory-bound.  "FlashAttention-2/3", section "FA-3：拥抱 Hopper",
// feature 3: the FP8 scales are per block, not global.
//
// One CTA per (batch*head, 128-row block).  A row of d bf16 is spread over d/8 lanes, 8
// consecutive elements (16 bytes) per lane, so one warp-wide load covers 32*16 contiguous
// bytes.  The unnormalised transform y = H_d (D x) is computed in float32 with butterfly
// stages of stride 1, 2, 4 inside each lane's 8 values and 8, 16, ... across lanes by warp
// shuffles -- the textbook stage order, so every element sees the same float32 additions in
// the same order as a plain sequential transform.  The block's largest |y| sets
// s_u = max(amax / 448, 2^-126); codes are E4M3(y * (1/s_u)) (round to nearest even,
// saturating); the stored dequantisation scale is s_u * post_scale (post_scale = 1/sqrt(d)
// with the transform, 1 without).

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "attn_kernels.h"

namespace ea {

template <int D, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
    hadamard_quant_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ x8, float* __restrict__ scales,
                          const signed char* __restrict__ signs, int N, int n_blocks, float post_scale) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerStep = 32 / kLanesPerRow;
  constexpr int kRowsPerWarp = 128 / WARPS;
  constexpr int kSteps = kRowsPerWarp / kRowsPerStep;
  static_assert(kSteps * kRowsPerStep * WARPS == 128, "row split");

  __shared__ float warp_max[WARPS];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int blk = blockIdx.x % n_blocks;
  const int bh = blockIdx.x / n_blocks;
  const int sub_row = lane / kLanesPerRow;
  const int col0 = (lane % kLanesPerRow) * 8;
  const size_t head_base = static_cast<size_t>(bh) * N * D;
  const int row_base = blk * 128 + warp * kRowsPerWarp + sub_row;

  float v[kSteps][8];
  // load (rows past the sequence end are zero and do not raise the block max)
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const int row = row_base + s * kRowsPerStep;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (row < N) w = __ldg(reinterpret_cast<const uint4*>(x + head_base + static_cast<size_t>(row) * D + col0));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[s][2 * e] = __uint_as_float(ws[e] << 16);
      v[s][2 * e + 1] = __uint_as_float(ws[e] & 0xFFFF0000u);
    }
  }

  if (signs != nullptr) {
    float sg[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sg[e] = (__ldg(signs + col0 + e) == -1) ? -1.f : 1.f;
#pragma unroll
    for (int s = 0; s < kSteps; ++s) {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[s][e] *= sg[e];
      // strides 1, 2, 4: inside the lane
#pragma unroll
      for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if ((e & h) == 0) {
            const float a = v[s][e], b = v[s][e + h];
            v[s][e] = __fadd_rn(a, b);
            v[s][e + h] = __fsub_rn(a, b);
          }
        }
      }
      // strides 8 .. D/2: partner lane differs in bit (h/8) of the lane index within the row
#pragma unroll
      for (int hl = 1; hl < kLanesPerRow; hl <<= 1) {
        const bool upper = (lane & hl) != 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float other = __shfl_xor_sync(0xffffffffu, v[s][e], hl);
          v[s][e] = upper ? __fsub_rn(other, v[s][e]) : __fadd_rn(v[s][e], other);
        }
      }
    }
  }

  float amax = 0.f;
#pragma unroll
  for (int s = 0; s < kSteps; ++s)
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[s][e]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) warp_max[warp] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < WARPS; ++w) amax = fmaxf(amax, warp_max[w]);

  const float s_u = fmaxf(__fdiv_rn(amax, 448.f), 1.17549435e-38f);
  const float rcp = __frcp_rn(s_u);
  if (threadIdx.x == 0) scales[static_cast<size_t>(bh) * n_blocks + blk] = __fmul_rn(s_u, post_scale);

#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const int row = row_base + s * kRowsPerStep;
    if (row >= N) continue;
    uint32_t packed[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
          make_float2(__fmul_rn(v[s][4 * h], rcp), __fmul_rn(v[s][4 * h + 1], rcp)), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
          make_float2(__fmul_rn(v[s][4 * h + 2], rcp), __fmul_rn(v[s][4 * h + 3], rcp)), __NV_SATFINITE, __NV_E4M3);
      packed[h] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    *reinterpret_cast<uint2*>(x8 + head_base + static_cast<size_t>(row) * D + col0) = make_uint2(packed[0], packed[1]);
  }
}

cudaError_t launch_hadamard_quant(const void* x, void* x8, float* scales, const signed char* signs, int BH, int N,
                                  int d, float post_scale, cudaStream_t stream) {
  const int n_blocks = (N + 127) / 128;
  const long long grid = static_cast<long long>(BH) * n_blocks;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* out = static_cast<uint8_t*>(x8);
  switch (d) {
    case 64:
      hadamard_quant_kernel<64, 8><<<(unsigned)grid, 256, 0, stream>>>(xb, out, scales, signs, N, n_blocks, post_scale);
      break;
    case 128:
      hadamard_quant_kernel<128, 8><<<(unsigned)grid, 256, 0, stream>>>(xb, out, scales, signs, N, n_blocks, post_scale);
      break;
    case 256:
      hadamard_quant_kernel<256, 16><<<(unsigned)grid, 512, 0, stream>>>(xb, out, scales, signs, N, n_blocks, post_scale);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace ea
