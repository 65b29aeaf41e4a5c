// Random-sign Hadamard transform + per-block E4M3 quantisation (bandwidth-bound pre-kernel).
//
// "FlashAttention-3", section "FP8 路径与低精度误差": outliers in Q and K are spread by
// x~ = H D x (D random signs, H Hadamard) before FP8 quantisation; the transform costs
// O(d log d) and is memory-bound.  "FlashAttention-2/3", section "FA-3：拥抱 Hopper",
// feature 3: the FP8 scales are per block, not global.
//
// Persistent grid: each CTA walks over (tensor, batch*head, 128-row block) units.  A block is
// brought into shared memory by TMA (128-byte swizzle, rows past the sequence end read as
// zero); two blocks are in flight per CTA, the next load being issued as soon as every thread
// has copied the current block into registers.  One thread holds a whole row (d = 64, 128) or
// 64 elements of it (d = 256, four adjacent lanes per row, with or without the rotary
// embedding; at d = 64 and 128 the rotary embedding has hq_rope_kernel below): the
// unnormalised transform y = H_d (D x) runs in float32 registers with butterfly stages of
// stride 1, 2, ..., inside a thread and the remaining strides between the lanes of a row -- the
// textbook stage order, so every element sees the same float32 additions in the same order
// as a plain sequential transform.  The block's largest |y| sets s_u = max(amax / 448, 2^-126);
// codes are E4M3(y * (1/s_u)) (round to nearest even, saturating); the stored dequantisation
// scale is s_u * post_scale (post_scale = 1/sqrt(d) with the transform, 1 without).  At
// d = 256 the codes of a warp's 8 rows are gathered in shared memory and written 512 contiguous
// bytes per store instruction (per-thread stores of 16-byte pieces of 8 rows took 9% longer),
// and each of the two butterfly stages between lanes moves every value across lanes once: the
// two lanes of a pair each keep half of the positions and receive the partner's values for
// them (one shuffle per position instead of one per element; the launch was bound by the
// shared-memory/shuffle crossbar, 86 -> 70 us for Q/K/V [2, 8, 8192, 256]).
//
// With ROPE (d = 256; d = 64 and 128 have hq_rope_kernel below), the tensors marked for it are
// first given the rotary position embedding the same page names as a bandwidth-bound step to
// fuse with the transform: coordinates i and i + d/2 of row n are rotated by the angle whose
// cosine and sine the caller's tables hold at [i, n], in float32 with each product and the sum
// rounded (no fused multiply-add); then D (an exact sign flip) and the butterflies run on the
// rotated float32 row.  The tables are frequency-major so that the 32 rows of a warp read one
// contiguous 128-byte line per frequency (row-major tables cost each warp load 32 lines and made
// the kernel L1-bound).  Four lanes hold a row; the partner coordinate sits two lanes away.
//
// Packed batches (VL): tensor t holds B sequences of different lengths, rows cu_t[b] ..
// cu_t[b+1]-1 of a [total_t, H, d] tensor, and is quantised in 128-row blocks of each sequence,
// so that a block never mixes two sequences: a block's rows past its sequence's end (the next
// sequence's rows, which the TMA box reads) count as zero and are not written.  Block j of
// sequence b, head h has scale [b, h, j] of a [B, H, ceil(max_len_t / 128)] array; blocks past a
// sequence's end are skipped (their barrier phase completes without a load).

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "attn_kernels.h"
#include "sm100_ptx.cuh"

namespace ea {

// (a0, a1) += (b0, b1) and (a0, a1) -= (b0, b1) as packed f32x2 operations
__device__ __forceinline__ void add2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb;\n\tmov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
      "add.rn.f32x2 ra, ra, rb;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
}
__device__ __forceinline__ void sub2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb;\n\tmov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
      "sub.rn.f32x2 ra, ra, rb;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
}
// (v0, v1) <- (s * v0 + o0, s * v1 + o1), one packed f32x2 fma; with s = +-1 the product is
// exact and the result is the correctly rounded o +- v
__device__ __forceinline__ void fma2_rn(float& v0, float& v1, float s, float o0, float o1) {
  asm("{\n\t.reg .b64 rv, rs, ro;\n\tmov.b64 rv, {%0, %1};\n\tmov.b64 rs, {%2, %2};\n\t"
      "mov.b64 ro, {%3, %4};\n\tfma.rn.f32x2 rv, rs, rv, ro;\n\tmov.b64 {%0, %1}, rv;\n\t}"
      : "+f"(v0), "+f"(v1) : "f"(s), "f"(o0), "f"(o1));
}

// (a0, a1) *= (b, b) as one packed f32x2 multiply (each lane rounds like a scalar multiply)
__device__ __forceinline__ void mul2(float& a0, float& a1, float b) {
  asm("{\n\t.reg .b64 ra, rb;\n\tmov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %2};\n\t"
      "mul.rn.f32x2 ra, ra, rb;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(b));
}

// Bounded wait of this thread on `bar`; on running out it flags `abort_s` and the status word.
// Callers reach a __syncthreads() before they act on `abort_s`, so the CTA leaves together.
__device__ __forceinline__ void thread_wait(uint64_t* bar, uint32_t parity, volatile int* abort_s, int* status) {
  const uint32_t a = smem_addr(bar);
  if (bar_try_wait(a, parity)) return;
  const unsigned long long t0 = global_timer_ns();
  while (!bar_try_wait(a, parity)) {
    if (*abort_s || global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_s = 1;
      atomicOr(status, kDevStatusTimeout);
      return;
    }
  }
}

template <int D, bool ROPE = false>
struct HqCfg {
  static_assert(!ROPE || D == 256, "the rotary embedding at d = 64 and 128 is hq_rope_kernel");
  // elements of a row held by one thread: the whole row at d = 64 and 128, a quarter at d = 256
  // (ROPE implies d = 256)
  static constexpr int kElems = (D == 256 || ROPE) ? 64 : D;
  static constexpr int kThreadsPerRow = D / kElems;
  static constexpr int kThreads = 128 * kThreadsPerRow;
  static constexpr int kBoxes = D / 64;             // 128-byte TMA boxes per row
  static constexpr int kBufBytes = 128 * D * 2;
  static constexpr int kCtasPerSm = D == 256 ? 1 : (D == 128 ? 3 : 5);
  // d = 256: the codes of a warp's 8 rows go through shared memory (2 KB per warp), so that
  // every store instruction writes 512 contiguous bytes
  static constexpr bool kStaged = kThreadsPerRow == 4;
  static constexpr int kSmem = 2 * kBufBytes + (kStaged ? kThreads / 32 * 8 * D : 0) + 1024;
};

// Up to three tensors of one shape in one launch (Q and K with the transform, V without).
struct HqJob {
  uint8_t* x8[3];
  float* scales[3];
  float post[3];
  int transform[3];
  int rope[3];        // ROPE kernels: rotate this tensor's rows first
  const float* cos;   // [d/2, n_pos] float32 rotary tables, frequency-major (ROPE kernels)
  const float* sin;
  int n_pos;
  int blocks_per_tensor;
  int H;              // heads: batch*head bh = b * H + h reaches the maps as (h, b)
  // packed batches (VL kernels): per tensor the B + 1 row offsets, the rows of the tensor, the
  // scale blocks per (sequence, head) = ceil(longest sequence / 128), and the first unit
  const int* cu[3];
  int total[3];
  int nbmax[3];
  int unit0[4];
};

// One 128-row block of a packed tensor: sequence row range and where its scale goes.
struct VlBlock {
  int t, bh, j;   // tensor, b * H + h, block of the sequence
  int row0;       // first row of the block in the [total, H, d] tensor
  int rows;       // rows of the block inside the sequence (0: past its end, or bad offsets)
  bool bad;       // offsets out of order, outside the tensor or longer than nbmax blocks
};

__device__ __forceinline__ VlBlock vl_block(int u, const HqJob& job) {
  VlBlock r;
  r.t = u < job.unit0[1] ? 0 : (u < job.unit0[2] ? 1 : 2);
  const int rem = u - (r.t == 0 ? 0 : (r.t == 1 ? job.unit0[1] : job.unit0[2]));
  const int nbm = r.t == 0 ? job.nbmax[0] : (r.t == 1 ? job.nbmax[1] : job.nbmax[2]);
  const int* cu = r.t == 0 ? job.cu[0] : (r.t == 1 ? job.cu[1] : job.cu[2]);
  const int total = r.t == 0 ? job.total[0] : (r.t == 1 ? job.total[1] : job.total[2]);
  r.j = rem % nbm;
  r.bh = rem / nbm;
  const int b = r.bh / job.H;
  const int s0 = __ldg(cu + b), s1 = __ldg(cu + b + 1);
  r.bad = !(0 <= s0 && s0 <= s1 && s1 <= total && (s1 - s0 + 127) / 128 <= nbm);
  r.row0 = s0 + r.j * 128;
  r.rows = r.bad ? 0 : min(128, max(0, s1 - r.row0));
  return r;
}

template <int D, bool ROPE, bool VL>
__global__ void __launch_bounds__(HqCfg<D, ROPE>::kThreads, HqCfg<D, ROPE>::kCtasPerSm)
    hadamard_quant_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                          const __grid_constant__ CUtensorMap tm2, const HqJob job,
                          const signed char* __restrict__ signs, int N, int n_blocks, int total_blocks, int* status) {
  using C = HqCfg<D, ROPE>;
  constexpr int kE = C::kElems;
  constexpr int kWarps = C::kThreads / 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ float warp_max[2][kWarps];
  __shared__ int abort_s;
  __shared__ __align__(16) uint32_t smask[D / 2];  // bf16x2 sign-bit masks of D (bits 15 and 31)

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int row = tid / C::kThreadsPerRow;   // row of the block
  const int part = tid % C::kThreadsPerRow;  // which kE-element part of the row

  if (tid == 0) {
    bar_init(&bar[0], 1);
    bar_init(&bar[1], 1);
    abort_s = 0;
    fence_barrier_init();
    prefetch_tensor_map(&tm0);
    prefetch_tensor_map(&tm1);
    prefetch_tensor_map(&tm2);
  }
  for (int i = tid; i < D / 2; i += C::kThreads) {
    uint32_t m = 0u;
    if (signs != nullptr) {
      if (__ldg(signs + 2 * i) == -1) m |= 0x00008000u;
      if (__ldg(signs + 2 * i + 1) == -1) m |= 0x80000000u;
    }
    smask[i] = m;
  }
  __syncthreads();

  auto issue = [&](int u, int buf) {
    if constexpr (VL) {
      // packed tensors are [total, H, d]: the maps are (d, rows, heads, 1)
      const VlBlock vb = vl_block(u, job);
      if (vb.rows == 0) {  // past the sequence's end: complete the phase without a load
        bar_arrive(&bar[buf]);
        return;
      }
      const CUtensorMap* tm = vb.t == 0 ? &tm0 : (vb.t == 1 ? &tm1 : &tm2);
      bar_arrive_expect_tx(&bar[buf], C::kBufBytes);
#pragma unroll
      for (int bx = 0; bx < C::kBoxes; ++bx)
        tma_load_4d(smem + buf * C::kBufBytes + bx * 16384, tm, &bar[buf], bx * 64, vb.row0, vb.bh % job.H, 0);
    } else {
      const int t = u / job.blocks_per_tensor;
      const int b = u - t * job.blocks_per_tensor;
      const int blk = b % n_blocks;
      const int bh = b / n_blocks;
      const CUtensorMap* tm = t == 0 ? &tm0 : (t == 1 ? &tm1 : &tm2);
      bar_arrive_expect_tx(&bar[buf], C::kBufBytes);
#pragma unroll
      for (int bx = 0; bx < C::kBoxes; ++bx)
        tma_load_4d(smem + buf * C::kBufBytes + bx * 16384, tm, &bar[buf], bx * 64, blk * 128, bh % job.H,
                    bh / job.H);
    }
  };

  // two blocks in flight: block i of this CTA goes to buffer i % 2, and the load of block i + 2
  // is issued as soon as every thread has read block i into registers
  if (tid == 0) {
    if (static_cast<int>(blockIdx.x) < total_blocks) issue(blockIdx.x, 0);
    if (static_cast<int>(blockIdx.x + gridDim.x) < total_blocks) issue(blockIdx.x + gridDim.x, 1);
  }
  int it = 0;
  for (int u = blockIdx.x; u < total_blocks; u += gridDim.x, ++it) {
    const int buf = it & 1;
    thread_wait(&bar[buf], (it >> 1) & 1, &abort_s, status);

    int t, blk, bh, rows_valid = 128;
    long long vl_row0 = 0;
    if constexpr (VL) {
      const VlBlock vb = vl_block(u, job);
      if (vb.bad && tid == 0 && vb.j == 0) atomicOr(status, kDevStatusBadSeqlens);
      if (vb.rows == 0) {
        // nothing loaded, nothing written; the CTA still meets at the barrier every block has
        __syncthreads();
        if (abort_s) break;
        if (tid == 0 && u + 2 * static_cast<int>(gridDim.x) < total_blocks) issue(u + 2 * gridDim.x, buf);
        continue;
      }
      t = vb.t;
      blk = vb.j;
      bh = vb.bh;
      rows_valid = vb.rows;
      vl_row0 = vb.row0;
    } else {
      t = u / job.blocks_per_tensor;
      const int b = u - t * job.blocks_per_tensor;
      blk = b % n_blocks;
      bh = b / n_blocks;
    }
    // explicit selects keep the parameter block out of local memory
    const bool transform = (t == 0 ? job.transform[0] : (t == 1 ? job.transform[1] : job.transform[2])) != 0;
    const uint8_t* sb = smem + buf * C::kBufBytes;
    // four lanes per row, transformed rows: the odd lanes hold the two halves of their part
    // swapped (v[j] = element part * kE + (j + 32) % 64), so that the exchanges between lanes
    // send the same registers on every lane (see the lane stages below)
    const int sh = (C::kThreadsPerRow == 4 && transform) ? 32 * (part & 1) : 0;

    // this thread's kE elements of its row: element e0 = part*kE + 8c.. lives in box e0/64 at
    // 16-byte chunk ((e0 % 64) / 8) ^ (row % 8) of the row (128-byte swizzle).  With the
    // transform, D x is a flip of bf16 sign bits, and the stride-1 butterflies of H run here.
    float v[kE];
    // x = the raw bf16 row part, as float32
    auto unpack_raw = [&]() {
#pragma unroll
      for (int c = 0; c < kE / 8; ++c) {
        const int e0 = part * kE + ((c * 8 + sh) & (kE - 1));
        const uint4 w = *reinterpret_cast<const uint4*>(sb + (e0 >> 6) * 16384 + row * 128 +
                                                        ((((e0 & 63) >> 3) ^ (row & 7)) << 4));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          v[c * 8 + 2 * k] = __uint_as_float(ws[k] << 16);
          v[c * 8 + 2 * k + 1] = __uint_as_float(ws[k] & 0xFFFF0000u);
        }
      }
    };
    // D x as a flip of bf16 sign bits, fused with the stride-1 butterflies of H
    auto unpack_signed_stage1 = [&]() {
#pragma unroll
      for (int c = 0; c < kE / 8; ++c) {
        const int e0 = part * kE + ((c * 8 + sh) & (kE - 1));
        uint4 w = *reinterpret_cast<const uint4*>(sb + (e0 >> 6) * 16384 + row * 128 +
                                                  ((((e0 & 63) >> 3) ^ (row & 7)) << 4));
        const uint4 mk = *reinterpret_cast<const uint4*>(&smask[e0 / 2]);
        const uint32_t ws[4] = {w.x ^ mk.x, w.y ^ mk.y, w.z ^ mk.z, w.w ^ mk.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float lo = __uint_as_float(ws[k] << 16);
          const float hi = __uint_as_float(ws[k] & 0xFFFF0000u);
          v[c * 8 + 2 * k] = lo + hi;
          v[c * 8 + 2 * k + 1] = lo - hi;
        }
      }
    };
    // the butterflies of stride 2 .. D/2
    auto later_stages = [&]() {
      // strides 2 .. kE/2 inside the thread, on register pairs (e, e+1): one packed add and one
      // packed sub make two butterflies, each lane rounding like a scalar operation
      constexpr int kLastLocal = C::kThreadsPerRow == 4 ? kE / 2 : kE;  // handled apart below
#pragma unroll
      for (int h = 2; h < kLastLocal; h <<= 1) {
#pragma unroll
        for (int e = 0; e < kE; e += 2) {
          if ((e & h) == 0) {
            float s0 = v[e], s1 = v[e + 1], d0 = v[e], d1 = v[e + 1];
            add2(s0, s1, v[e + h], v[e + h + 1]);
            sub2(d0, d1, v[e + h], v[e + h + 1]);
            v[e] = s0;
            v[e + 1] = s1;
            v[e + h] = d0;
            v[e + h + 1] = d1;
          }
        }
      }
      if constexpr (C::kThreadsPerRow == 4) {
        // Every butterfly below is fl(x + y) or fl(x - y) of its lower element x and upper
        // element y, as an fma with multipliers +-1 (exact) and one rounding -- the value and
        // the sign of a zero of the textbook stage.
        // Stride 32, inside the thread; with swapped halves (odd lanes) element j sits at
        // v[32 + j] and j + 32 at v[j]: v[j] <- s1 v[j] + v[32+j], v[32+j] <- -s1 v[32+j] + v[j].
        const float s1 = (part & 1) ? -1.f : 1.f;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float a0 = v[j], a1 = v[j + 1], b0 = v[32 + j], b1 = v[33 + j];
          fma2_rn(a0, a1, s1, v[32 + j], v[33 + j]);
          fma2_rn(b0, b1, -s1, v[j], v[j + 1]);
          v[j] = a0;
          v[j + 1] = a1;
          v[32 + j] = b0;
          v[33 + j] = b1;
        }
        // Strides 64 and 128 between lanes.  At each, a lane pair holds the two elements of 32
        // butterflies' worth of positions each; every lane keeps v[t], sends v[32 + t] and
        // computes the butterflies of its kept positions with the received value r:
        // v[t] <- b1 r + a1 v[t], v[32+t] <- b2 r + a2 v[t] (a, b = +-1 by lane).
        // Stride 64 (lanes p, p^1; part p holds elements 64p ..): lane 0 keeps elements 0..31
        // and sends 32..63, lane 1 keeps 96..127 and sends 64..95; sums and differences land
        // so that the stride-128 exchange sends v[32 + t] again:
        //   lane 0: v[t] = e(t),      v[32+t] = e(64+t)      lane 1: e(32+t),  e(96+t)
        //   lane 2: v[t] = e(192+t),  v[32+t] = e(128+t)     lane 3: e(224+t), e(160+t)
        {
          const float a1 = part == 3 ? -1.f : 1.f, b1 = part == 2 ? -1.f : 1.f;
          const float a2 = part == 1 ? -1.f : 1.f, b2 = part == 0 ? -1.f : 1.f;
#pragma unroll
          for (int t = 0; t < 32; t += 2) {
            float r0 = __shfl_xor_sync(0xffffffffu, v[32 + t], 1);
            float r1 = __shfl_xor_sync(0xffffffffu, v[33 + t], 1);
            float w0 = v[t], w1 = v[t + 1], x0 = v[t], x1 = v[t + 1];
            mul2(w0, w1, a1);
            mul2(x0, x1, a2);
            float q0 = r0, q1 = r1;
            fma2_rn(r0, r1, b1, w0, w1);
            fma2_rn(q0, q1, b2, x0, x1);
            v[t] = r0;
            v[t + 1] = r1;
            v[32 + t] = q0;
            v[33 + t] = q1;
          }
        }
        // Stride 128 (lanes p, p^2): lane p ends with v[t] = e(32p + t), v[32+t] = e(128 + 32p + t)
        {
          const float a = part >= 2 ? -1.f : 1.f;
#pragma unroll
          for (int t = 0; t < 32; t += 2) {
            const float r0 = __shfl_xor_sync(0xffffffffu, v[32 + t], 2);
            const float r1 = __shfl_xor_sync(0xffffffffu, v[33 + t], 2);
            float s0 = v[t], s1_ = v[t + 1], w0 = v[t], w1 = v[t + 1];
            add2(s0, s1_, r0, r1);
            mul2(w0, w1, a);
            float d0 = r0, d1 = r1;
            fma2_rn(d0, d1, -a, w0, w1);
            v[t] = s0;
            v[t + 1] = s1_;
            v[32 + t] = d0;
            v[33 + t] = d1;
          }
        }
      }
    };
    // rotary embedding of the float32 row (pairs i, i + D/2), then, with the transform, the sign
    // flips of D and the stride-1 butterflies
    auto rotate_row = [&]() {
      // rows past the sequence end hold zeros (TMA fill): any table row leaves them zero
      const int pos = min(blk * 128 + row, N - 1);
      const size_t np = static_cast<size_t>(job.n_pos);
      if constexpr (ROPE) {  // (d = 256: four lanes per row)
        // the lower half of the parts holds coordinates 0 .. D/2-1, the upper half their
        // partners D/2 .. D-1, kThreadsPerRow/2 lanes away
        constexpr int kHalf = C::kThreadsPerRow / 2;
        const bool upper = part >= kHalf;
        const int i0 = (part % kHalf) * kE;
        // v[e] is coordinate part * kE + (e + sh) % kE: frequency i0 + (e + sh) % kE
        const float* cr = job.cos + i0 * np + pos;
        const float* sr = job.sin + i0 * np + pos;
        const long long lo_off = static_cast<long long>(sh) * static_cast<long long>(np);
#pragma unroll
        for (int e = 0; e < kE; ++e) {
          const long long off = (e < kE / 2 ? lo_off : -lo_off) + static_cast<long long>(e) * static_cast<long long>(np);
          const float c = __ldg(cr + off), s = __ldg(sr + off);
          const float own = v[e];
          const float other = __shfl_xor_sync(0xffffffffu, own, kHalf);
          v[e] = upper ? __fadd_rn(__fmul_rn(own, c), __fmul_rn(other, s))
                       : __fsub_rn(__fmul_rn(own, c), __fmul_rn(other, s));
        }
      }
    };
    auto signed_stage1 = [&]() {
#pragma unroll
      for (int e = 0; e < kE; e += 2) {
        const uint32_t mk = smask[(part * kE + ((e + sh) & (kE - 1))) / 2];
        const float a = __uint_as_float(__float_as_uint(v[e]) ^ (mk << 16));
        const float b = __uint_as_float(__float_as_uint(v[e + 1]) ^ (mk & 0x80000000u));
        v[e] = a + b;
        v[e + 1] = a - b;
      }
    };

    if constexpr (ROPE) {
      const bool rotate = (t == 0 ? job.rope[0] : (t == 1 ? job.rope[1] : job.rope[2])) != 0;
      if (rotate) {
        unpack_raw();
        rotate_row();
        if (transform) {
          signed_stage1();
          later_stages();
        }
      } else if (transform) {
        unpack_signed_stage1();
        later_stages();
      } else {
        unpack_raw();
      }
    } else {
      if (transform) {
        unpack_signed_stage1();
        later_stages();
      } else {
        unpack_raw();
      }
    }

    if constexpr (VL) {
      // rows of the next sequence inside the box: zero (the transform of a zero row is zero)
      if (row >= rows_valid) {
#pragma unroll
        for (int e = 0; e < kE; ++e) v[e] = 0.f;
      }
    }
    // block amax: four chains in the thread, then the lanes, then the warps
    float am[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < kE; ++e) am[e & 3] = fmaxf(am[e & 3], fabsf(v[e]));
    float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
    // non-negative, never NaN: the unsigned order of the bits is the order of the values
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    if (lane == 0) warp_max[buf][warp] = amax;
    // every thread has read buffer `buf` and posted its warp maximum
    __syncthreads();
    if (abort_s) break;
    if (tid == 0 && u + 2 * static_cast<int>(gridDim.x) < total_blocks) issue(u + 2 * gridDim.x, buf);
    amax = warp_max[buf][0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) amax = fmaxf(amax, warp_max[buf][w]);

    uint8_t* const x8 = t == 0 ? job.x8[0] : (t == 1 ? job.x8[1] : job.x8[2]);
    float* const scales = t == 0 ? job.scales[0] : (t == 1 ? job.scales[1] : job.scales[2]);
    const float post = t == 0 ? job.post[0] : (t == 1 ? job.post[1] : job.post[2]);
    const float s_u = fmaxf(__fdiv_rn(amax, 448.f), 1.17549435e-38f);
    const float rcp = __frcp_rn(s_u);
    const int nbs = VL ? (t == 0 ? job.nbmax[0] : (t == 1 ? job.nbmax[1] : job.nbmax[2])) : n_blocks;
    if (tid == 0) scales[static_cast<size_t>(bh) * nbs + blk] = __fmul_rn(s_u, post);

    const int grow = blk * 128 + row;
    if constexpr (C::kStaged && !VL) {
      // logical 16-byte chunk ch of warp row rw at physical chunk ch ^ g, g = 2 * (ch / 8) + rw % 2:
      // the 8 lanes of each quarter-warp access hit 8 different bank groups, for the writes
      // (two rows, four parts) and for the reads (one row, eight chunks)
      uint8_t* const ws = smem + 2 * C::kBufBytes + warp * (8 * D);
      const int rw = lane >> 2;
#pragma unroll
      for (int c = 0; c < kE / 16; ++c) {
        // the row's 16-byte chunk of v[16c ..]: transformed rows end the lane stages with
        // elements 32 part .. and 128 + 32 part .., the others hold part * kE ..
        const int ch = transform ? (c < 2 ? 2 * part + c : 8 + 2 * part + (c - 2)) : 4 * part + c;
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = c * 16 + 4 * k;
          float a0 = v[e], a1 = v[e + 1], a2 = v[e + 2], a3 = v[e + 3];
          mul2(a0, a1, rcp);
          mul2(a2, a3, rcp);
          const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a0, a1), __NV_SATFINITE, __NV_E4M3);
          const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(a2, a3), __NV_SATFINITE, __NV_E4M3);
          w[k] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
        }
        *reinterpret_cast<uint4*>(ws + rw * D + ((ch ^ (2 * (ch >> 3) + (rw & 1))) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      __syncwarp();
      const int row0 = blk * 128 + warp * 8;  // sequence row of the warp's first row
      uint8_t* const gout = x8 + (static_cast<size_t>(bh) * N + row0) * D;
#pragma unroll
      for (int i = 0; i < 8 * D / 512; ++i) {
        const int rr = 2 * i + (lane >> 4);
        const int ch = lane & 15;
        const uint4 val = *reinterpret_cast<const uint4*>(ws + rr * D + ((ch ^ (2 * (ch >> 3) + (rr & 1))) << 4));
        if (row0 + rr < N) *reinterpret_cast<uint4*>(gout + 512 * i + 16 * lane) = val;
      }
      __syncwarp();
    } else if (VL ? row < rows_valid : grow < N) {
      // contiguous outputs: [BH, N, d], or [total, H, d] for packed tensors
      uint8_t* out = VL ? x8 + ((vl_row0 + row) * job.H + bh % job.H) * D
                        : x8 + (static_cast<size_t>(bh) * N + grow) * D;
#pragma unroll
      for (int c = 0; c < kE / 16; ++c) {
        // the row's 16-byte chunk of v[16c ..] (four lanes per row: as in the staged stores)
        const int ch = (C::kThreadsPerRow == 4 && transform) ? (c < 2 ? 2 * part + c : 8 + 2 * part + (c - 2))
                                                             : part * (kE / 16) + c;
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = c * 16 + 4 * k;
          float a0 = v[e], a1 = v[e + 1], a2 = v[e + 2], a3 = v[e + 3];
          mul2(a0, a1, rcp);
          mul2(a2, a3, rcp);
          const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a0, a1), __NV_SATFINITE, __NV_E4M3);
          const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(a2, a3), __NV_SATFINITE, __NV_E4M3);
          w[k] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
        }
        *reinterpret_cast<uint4*>(out + ch * 16) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  // no TMA copy may still be in flight when the CTA exits: after an abort at block `it`, blocks
  // it and it + 1 may have been issued and not waited for
  if (tid == 0) {
    const int issued = total_blocks > static_cast<int>(blockIdx.x)
                           ? (total_blocks - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                                 static_cast<int>(gridDim.x)
                           : 0;
    for (int i = it; i < issued && i < it + 2; ++i) {
      const uint32_t a = smem_addr(&bar[i & 1]);
      const unsigned long long t0 = global_timer_ns();
      while (!bar_try_wait(a, (i >> 1) & 1)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          atomicOr(status, kDevStatusTimeout);
          break;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Rotary embedding + transform + quantisation for d = 64 and 128 (d = 256 keeps the kernel above).
//
// One thread holds a whole row, so that the rotation (coordinates i and i + d/2) and every
// butterfly stage stay inside the thread, in the textbook stage order.  The 128 x d/2 slice of
// each table that a 128-row block needs is staged once per position block in shared memory,
// position-major with its 16-byte chunks permuted so that the 8 rows of a quarter warp read
// distinct banks; the units are ordered position block first, so that one staged slice serves
// every head and tensor at those positions (the tables are read from DRAM once).  A CTA works on
// kSlots blocks at a time, one 128-thread slot each, with its own TMA buffers, barrier phases and
// named barrier; with one buffer per slot (d = 128, where a row takes the registers of two) the
// next block's load is issued as soon as the slot has unpacked the current one.  A warp's codes go
// through shared memory (rows permuted in 16-byte chunks), so that each store instruction writes
// 512 contiguous bytes of the output instead of one 16-byte piece of 32 rows.
//
// Rounding is that of the oracle's composition: products and the sum of the rotation each
// rounded, the sign flips of D exact and applied to the rotated values, each butterfly rounded
// once.  A packed f32x2 multiply is fused by the assembler into a following packed add or sub
// even with .rn, so the rotation's products are packed fmas with a run-time -0.0 addend.
template <int D>
struct HqRopeCfg {
  static constexpr int kSlots = D == 128 ? 3 : 4;
  static constexpr int kBufs = D == 128 ? 1 : 2;     // TMA buffers per slot
  static constexpr int kThreads = 128 * kSlots;
  static constexpr int kBufBytes = 128 * D * 2;      // one bf16 block
  static constexpr int kTabBytes = 128 * (D / 2) * 4;  // one table slice, float32
  static constexpr int kOutBytes = 128 * D;          // one block of codes, staged per warp for the store
  static constexpr int kSmem = 2 * kTabBytes + kSlots * (kBufs * kBufBytes + kOutBytes) + 1024;
};

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// (a0, a1) *= (b0, b1), each lane rounded once, as a packed fma whose addend z is -0.0 known
// only at run time (x + (-0) = x for every x, zeros included); an fma's result is never fused
// into another operation
__device__ __forceinline__ void mul2r(float& a0, float& a1, float b0, float b1, float z) {
  asm("{\n\t.reg .b64 ra, rb, rz;\n\tmov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
      "mov.b64 rz, {%4, %4};\n\tfma.rn.f32x2 ra, ra, rb, rz;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1), "f"(z));
}

// bounded wait that reports whether the phase completed
__device__ __forceinline__ bool slot_wait(uint64_t* bar, uint32_t parity, volatile int* abort_s, int* status) {
  const uint32_t a = smem_addr(bar);
  if (bar_try_wait(a, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (!bar_try_wait(a, parity)) {
    if (*abort_s || global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_s = 1;
      atomicOr(status, kDevStatusTimeout);
      return false;
    }
  }
  return true;
}

// The units of slot `slot` in the CTA's range [lo, hi): the range is cut at multiples of P (the
// units of one position block) into segments, and slot s takes units a + s, a + s + S, ... of
// segment [a, b).  slot_first: the slot's first unit at or after segment start `a`, or hi.
__device__ __forceinline__ int slot_first(int a, int hi, int P, int slot) {
  while (a < hi) {
    const int b = min(hi, (a / P + 1) * P);
    if (a + slot < b) return a + slot;
    a = b;
  }
  return hi;
}
template <int S>
__device__ __forceinline__ int slot_next(int u, int hi, int P, int slot) {
  const int b = min(hi, (u / P + 1) * P);
  return u + S < b ? u + S : slot_first(b, hi, P, slot);
}

template <int D>
__global__ void __launch_bounds__(HqRopeCfg<D>::kThreads, 1)
    hq_rope_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                   const __grid_constant__ CUtensorMap tm2, const HqJob job, const signed char* __restrict__ signs,
                   int N, int n_blocks, int BH, int ntensors, int* status) {
  using C = HqRopeCfg<D>;
  constexpr int S = C::kSlots;
  constexpr int NB = C::kBufs;
  constexpr int kBoxes = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  float* const tab_c = reinterpret_cast<float*>(smem);
  float* const tab_s = reinterpret_cast<float*>(smem + C::kTabBytes);
  uint8_t* const bufs = smem + 2 * C::kTabBytes;
  uint8_t* const outs = bufs + S * NB * C::kBufBytes;
  __shared__ __align__(8) uint64_t bar[S][NB];
  __shared__ float warp_max[S][2][4];
  __shared__ int abort_s[S];
  __shared__ __align__(16) float fsig[D];  // the signs of D as +-1.0f
  __shared__ float zero_s;                 // -0.0f, read back as an opaque value

  const int tid = threadIdx.x;
  const int slot = tid >> 7;
  const int row = tid & 127;  // row of the block
  const int lane = tid & 31;
  const int swarp = row >> 5;  // warp within the slot

  if (tid == 0) {
    // one thread initialises every slot's barriers, so that its fence publishes them all to
    // the TMA unit
    for (int i = 0; i < S; ++i) {
      for (int j = 0; j < NB; ++j) bar_init(&bar[i][j], 1);
      abort_s[i] = 0;
    }
    zero_s = -0.0f;
    fence_barrier_init();
    prefetch_tensor_map(&tm0);
    prefetch_tensor_map(&tm1);
    prefetch_tensor_map(&tm2);
  }
  for (int i = tid; i < D; i += C::kThreads) fsig[i] = (signs != nullptr && __ldg(signs + i) == -1) ? -1.f : 1.f;
  __syncthreads();
  const float zneg = *static_cast<volatile float*>(&zero_s);

  const int P = ntensors * BH;  // units of one position block: (tensor, batch*head)
  const long long U = static_cast<long long>(n_blocks) * P;
  const int lo = static_cast<int>(U * blockIdx.x / gridDim.x);
  const int hi = static_cast<int>(U * (blockIdx.x + 1) / gridDim.x);
  const bool producer = row == 0;
  uint64_t* const sbar = bar[slot];
  uint8_t* const sbuf = bufs + slot * NB * C::kBufBytes;
  volatile int* const sabort = &abort_s[slot];

  auto issue = [&](int u, int buf) {
    const int blk = u / P;
    const int rem = u - blk * P;
    const int t = rem / BH;
    const int bh = rem - t * BH;
    const CUtensorMap* tm = t == 0 ? &tm0 : (t == 1 ? &tm1 : &tm2);
    bar_arrive_expect_tx(&sbar[buf], C::kBufBytes);
#pragma unroll
    for (int bx = 0; bx < kBoxes; ++bx)
      tma_load_4d(sbuf + buf * C::kBufBytes + bx * 16384, tm, &sbar[buf], bx * 64, blk * 128, bh % job.H, bh / job.H);
  };

  int pre = hi;    // producer: the next unit to load
  int issued = 0;  // producer: loads issued, and waits of its own that completed
  int waited = 0;
  if (producer) {
    pre = slot_first(lo, hi, P, slot);
    for (int j = 0; j < NB && pre < hi; ++j) {
      issue(pre, j);
      ++issued;
      pre = slot_next<S>(pre, hi, P, slot);
    }
  }

  int k = 0;  // units of this slot so far
  for (int a = lo; a < hi;) {
    const int blk = a / P;
    const int b = min(hi, (blk + 1) * P);
    const int t_first = (a - blk * P) / BH, t_last = (b - 1 - blk * P) / BH;
    bool need = false;
    for (int t = t_first; t <= t_last; ++t) need |= (t == 0 ? job.rope[0] : (t == 1 ? job.rope[1] : job.rope[2])) != 0;
    __syncthreads();  // every slot is done with the previous slice
    if (need) {
      // the slice of this position block (rows past the sequence end take the last position's
      // entries; their values are zero), every load of the thread in flight before its stores
      constexpr int kRowsPer = C::kThreads / 128;
      constexpr int kPer = (D / 2 + kRowsPer - 1) / kRowsPer;
      const size_t np = static_cast<size_t>(job.n_pos);
      const int pos = min(blk * 128 + row, N - 1);
      float cv[kPer], sv[kPer];
#pragma unroll
      for (int m = 0; m < kPer; ++m) {
        const int i = slot + m * kRowsPer;
        if (i < D / 2) {
          cv[m] = __ldg(job.cos + i * np + pos);
          sv[m] = __ldg(job.sin + i * np + pos);
        }
      }
#pragma unroll
      for (int m = 0; m < kPer; ++m) {
        const int i = slot + m * kRowsPer;
        if (i < D / 2) {
          const int ch = i >> 2;
          const int idx = row * (D / 2) + ((ch ^ ((row + (ch >> 3)) & 7)) << 2) + (i & 3);
          tab_c[idx] = cv[m];
          tab_s[idx] = sv[m];
        }
      }
    }
    __syncthreads();
    if (b < hi) {
      // bring the next position block's slice into L2 while this one is worked on
      const int pos0 = (blk + 1) * 128;
      const size_t np = static_cast<size_t>(job.n_pos);
      for (int l = tid; l < 2 * (D / 2) * 4; l += C::kThreads) {
        const int i = (l >> 2) % (D / 2), j = l & 3;
        const float* tb = l < (D / 2) * 4 ? job.cos : job.sin;
        if (pos0 + 32 * j < job.n_pos)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(tb + i * np + pos0 + 32 * j));
      }
    }

    for (int u = a + slot; u < b; u += S, ++k) {
      const int buf = NB == 1 ? 0 : (k & 1);
      const uint32_t parity = NB == 1 ? (k & 1) : ((k >> 1) & 1);
      const int rem = u - blk * P;
      const int t = rem / BH;
      const int bh = rem - t * BH;
      if (!*sabort) {
        const bool ok = slot_wait(&sbar[buf], parity, sabort, status);
        if (producer && ok) ++waited;
      }
      const bool rotate = (t == 0 ? job.rope[0] : (t == 1 ? job.rope[1] : job.rope[2])) != 0;
      const bool transform = (t == 0 ? job.transform[0] : (t == 1 ? job.transform[1] : job.transform[2])) != 0;
      const uint8_t* sb = sbuf + buf * C::kBufBytes;

      // v[c] = coordinate c of the row
      float v[D];
#pragma unroll
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const int e0 = 8 * c8;
        const uint4 w = *reinterpret_cast<const uint4*>(sb + (e0 >> 6) * 16384 + row * 128 +
                                                        ((((e0 & 63) >> 3) ^ (row & 7)) << 4));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          v[e0 + 2 * m] = __uint_as_float(ws[m] << 16);
          v[e0 + 2 * m + 1] = __uint_as_float(ws[m] & 0xFFFF0000u);
        }
      }
      if constexpr (NB == 1) {
        // the slot has read its buffer: load the next block into it
        named_bar_sync(1 + slot, 128);
        if (!*sabort && producer && pre < hi) {
          issue(pre, 0);
          ++issued;
          pre = slot_next<S>(pre, hi, P, slot);
        }
      }
      if (rotate) {
        // (x_i, x_{i+d/2}) -> (x_i c - x_{i+d/2} s, x_{i+d/2} c + x_i s), frequency i
#pragma unroll
        for (int q = 0; q < D / 8; ++q) {
          const int idx = row * (D / 2) + ((q ^ ((row + (q >> 3)) & 7)) << 2);
          const float4 c4 = *reinterpret_cast<const float4*>(tab_c + idx);
          const float4 s4 = *reinterpret_cast<const float4*>(tab_s + idx);
          const float cs[4] = {c4.x, c4.y, c4.z, c4.w};
          const float sn[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
          for (int m = 0; m < 4; m += 2) {
            const int j = 4 * q + m;
            float al0 = v[j], al1 = v[j + 1], bl0 = v[D / 2 + j], bl1 = v[D / 2 + j + 1];
            float ah0 = bl0, ah1 = bl1, bh0 = al0, bh1 = al1;
            mul2r(al0, al1, cs[m], cs[m + 1], zneg);  // x_lo c
            mul2r(bl0, bl1, sn[m], sn[m + 1], zneg);  // x_hi s
            mul2r(ah0, ah1, cs[m], cs[m + 1], zneg);  // x_hi c
            mul2r(bh0, bh1, sn[m], sn[m + 1], zneg);  // x_lo s
            sub2(al0, al1, bl0, bl1);
            add2(ah0, ah1, bh0, bh1);
            v[j] = al0;
            v[j + 1] = al1;
            v[D / 2 + j] = ah0;
            v[D / 2 + j + 1] = ah1;
          }
        }
      }
      if (transform) {
        // D (exact sign flips) fused with the stride-1 butterflies: (s_e x_e) +- s_{e+1} x_{e+1}
#pragma unroll
        for (int q = 0; q < D / 4; ++q) {
          const float4 sg = *reinterpret_cast<const float4*>(fsig + 4 * q);
          const float sgs[4] = {sg.x, sg.y, sg.z, sg.w};
#pragma unroll
          for (int m = 0; m < 4; m += 2) {
            const int e = 4 * q + m;
            const float x = v[e] * sgs[m];
            const float y = v[e + 1];
            v[e] = fmaf(sgs[m + 1], y, x);
            v[e + 1] = fmaf(-sgs[m + 1], y, x);
          }
        }
        // strides 2 .. d/2 on register pairs (e, e+1): a packed add and a packed sub make two
        // butterflies
#pragma unroll
        for (int h = 2; h < D; h <<= 1) {
#pragma unroll
          for (int e = 0; e < D; e += 2) {
            if ((e & h) == 0) {
              float s0 = v[e], s1 = v[e + 1], d0 = v[e], d1 = v[e + 1];
              add2(s0, s1, v[e + h], v[e + h + 1]);
              sub2(d0, d1, v[e + h], v[e + h + 1]);
              v[e] = s0;
              v[e + 1] = s1;
              v[e + h] = d0;
              v[e + h + 1] = d1;
            }
          }
        }
      }

      float am[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < D; ++e) am[e & 3] = fmaxf(am[e & 3], fabsf(v[e]));
      float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
      // non-negative, never NaN: the unsigned order of the bits is the order of the values
      amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
      if (lane == 0) warp_max[slot][k & 1][swarp] = amax;
      // every warp of the slot has posted its maximum (and, with two buffers, read buffer `buf`)
      named_bar_sync(1 + slot, 128);
      if (*sabort) continue;
      if constexpr (NB == 2) {
        if (producer && pre < hi) {
          issue(pre, buf);
          ++issued;
          pre = slot_next<S>(pre, hi, P, slot);
        }
      }
      amax = fmaxf(fmaxf(warp_max[slot][k & 1][0], warp_max[slot][k & 1][1]),
                   fmaxf(warp_max[slot][k & 1][2], warp_max[slot][k & 1][3]));

      uint8_t* const x8 = t == 0 ? job.x8[0] : (t == 1 ? job.x8[1] : job.x8[2]);
      float* const scales = t == 0 ? job.scales[0] : (t == 1 ? job.scales[1] : job.scales[2]);
      const float post = t == 0 ? job.post[0] : (t == 1 ? job.post[1] : job.post[2]);
      const float s_u = fmaxf(__fdiv_rn(amax, 448.f), 1.17549435e-38f);
      const float rcp = __frcp_rn(s_u);
      if (producer) scales[static_cast<size_t>(bh) * n_blocks + blk] = __fmul_rn(s_u, post);
      {
        // the warp's 32 rows of codes: row r at r * D, 16-byte chunk c at chunk c ^ ((r / G) % CPR),
        // G rows per 128-byte line, CPR chunks per row (conflict-free writes and reads)
        constexpr int CPR = D / 16;
        constexpr int G = 128 / D;
        uint8_t* const ws = outs + (slot * 4 + swarp) * (32 * D);
#pragma unroll
        for (int c = 0; c < CPR; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int e = 16 * c + 4 * m;
            float a0 = v[e], a1 = v[e + 1], a2 = v[e + 2], a3 = v[e + 3];
            mul2(a0, a1, rcp);
            mul2(a2, a3, rcp);
            const __nv_fp8x2_storage_t l = __nv_cvt_float2_to_fp8x2(make_float2(a0, a1), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t h = __nv_cvt_float2_to_fp8x2(make_float2(a2, a3), __NV_SATFINITE, __NV_E4M3);
            w[m] = static_cast<uint32_t>(l) | (static_cast<uint32_t>(h) << 16);
          }
          *reinterpret_cast<uint4*>(ws + lane * D + ((c ^ ((lane / G) % CPR)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        __syncwarp();
        const int row0 = blk * 128 + swarp * 32;  // sequence row of the warp's first row
        uint8_t* const gout = x8 + (static_cast<size_t>(bh) * N + row0) * D;
#pragma unroll
        for (int i = 0; i < 32 * D / 512; ++i) {
          const int rr = i * (512 / D) + lane / CPR;
          const int c = lane % CPR;
          const uint4 val = *reinterpret_cast<const uint4*>(ws + rr * D + ((c ^ ((rr / G) % CPR)) << 4));
          if (row0 + rr < N) *reinterpret_cast<uint4*>(gout + 512 * i + 16 * lane) = val;
        }
        __syncwarp();
      }
    }
    a = b;
  }
  // no TMA copy may still be in flight when the CTA exits: after an abort, the slot's loads from
  // its first unwaited one on may not have landed
  if (producer) {
    for (int i = waited; i < issued; ++i) {
      const uint32_t ad = smem_addr(&sbar[NB == 1 ? 0 : (i & 1)]);
      const uint32_t par = NB == 1 ? (i & 1) : ((i >> 1) & 1);
      const unsigned long long t0 = global_timer_ns();
      while (!bar_try_wait(ad, par)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          atomicOr(status, kDevStatusTimeout);
          break;
        }
      }
    }
  }
}

template <int D>
static cudaError_t launch_hq_rope(const CUtensorMap* tm, int ntensors, const HqJob& job0, const signed char* signs,
                                  int BH, int N, int num_sms, int* status, cudaStream_t stream) {
  using C = HqRopeCfg<D>;
  const int n_blocks = (N + 127) / 128;
  const long long total = static_cast<long long>(BH) * n_blocks * ntensors;
  if (total > 0x7FFFFFFFLL - 65536) return cudaErrorInvalidValue;
  const long long want = (total + C::kSlots - 1) / C::kSlots;
  const int grid = static_cast<int>(want < num_sms ? want : num_sms);
  hq_rope_kernel<D><<<grid, C::kThreads, C::kSmem, stream>>>(tm[0], tm[ntensors > 1 ? 1 : 0],
                                                             tm[ntensors > 2 ? 2 : 0], job0, signs, N, n_blocks, BH,
                                                             ntensors, status);
  return cudaGetLastError();
}

template <int D, bool ROPE, bool VL = false>
static cudaError_t launch_hq(const CUtensorMap* tm, int ntensors, const HqJob& job0, const signed char* signs, int BH,
                             int N, int num_sms, int* status, cudaStream_t stream) {
  using C = HqCfg<D, ROPE>;
  const int n_blocks = (N + 127) / 128;
  HqJob job = job0;
  long long total = 0;
  if constexpr (VL) {
    // units: every (sequence, head, block up to the longest sequence's) of each tensor
    for (int t = 0; t < 3; ++t) {
      job.unit0[t] = static_cast<int>(t < ntensors ? total : 0x7FFFFFFF);
      if (t < ntensors) total += static_cast<long long>(BH) * job.nbmax[t];
      if (total > 0x7FFFFFFFLL - 65536) return cudaErrorInvalidValue;
    }
    job.unit0[3] = static_cast<int>(total);
  } else {
    const long long per = static_cast<long long>(BH) * n_blocks;
    total = per * ntensors;
    if (total > 0x7FFFFFFFLL - 65536) return cudaErrorInvalidValue;  // u + 2 * grid stays an int
    job.blocks_per_tensor = static_cast<int>(per);
  }
  const long long cap = static_cast<long long>(num_sms) * C::kCtasPerSm;
  const int grid = static_cast<int>(total < cap ? total : cap);
  hadamard_quant_kernel<D, ROPE, VL><<<grid, C::kThreads, C::kSmem, stream>>>(
      tm[0], tm[ntensors > 1 ? 1 : 0], tm[ntensors > 2 ? 2 : 0], job, signs, N, n_blocks, static_cast<int>(total),
      status);
  return cudaGetLastError();
}

template <int D>
static cudaError_t set_hq_attr() {
  cudaError_t e = cudaFuncSetAttribute(hadamard_quant_kernel<D, false, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, HqCfg<D>::kSmem);
  if (e == cudaSuccess) {
    if constexpr (D == 256)
      e = cudaFuncSetAttribute(hadamard_quant_kernel<D, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               HqCfg<D, true>::kSmem);
    else
      e = cudaFuncSetAttribute(hq_rope_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, HqRopeCfg<D>::kSmem);
  }
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(hadamard_quant_kernel<D, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             HqCfg<D>::kSmem);
  return e;
}

cudaError_t launch_hadamard_quant_varlen(const CUtensorMap* tm, int ntensors, uint8_t* const* x8, float* const* scales,
                                         const float* post, const int* transform, const signed char* signs, int B,
                                         int H, const int* const* cu, const int* total, const int* max_len, int d,
                                         int num_sms, int* status, cudaStream_t stream) {
  if (ntensors < 1 || ntensors > 3) return cudaErrorInvalidValue;
  HqJob job{};
  for (int t = 0; t < 3; ++t) {
    const int s = t < ntensors ? t : 0;
    job.x8[t] = x8[s];
    job.scales[t] = scales[s];
    job.post[t] = post[s];
    job.transform[t] = transform[s];
    job.cu[t] = cu[s];
    job.total[t] = total[s];
    job.nbmax[t] = (max_len[s] + 127) / 128;
    if (job.nbmax[t] < 1) return cudaErrorInvalidValue;
  }
  job.H = H;
  const int BH = B * H;
  switch (d) {
    case 64:
      return launch_hq<64, false, true>(tm, ntensors, job, signs, BH, 0, num_sms, status, stream);
    case 128:
      return launch_hq<128, false, true>(tm, ntensors, job, signs, BH, 0, num_sms, status, stream);
    case 256:
      return launch_hq<256, false, true>(tm, ntensors, job, signs, BH, 0, num_sms, status, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t setup_hadamard_quant_kernels() {
  cudaError_t e = set_hq_attr<64>();
  if (e == cudaSuccess) e = set_hq_attr<128>();
  if (e == cudaSuccess) e = set_hq_attr<256>();
  return e;
}

cudaError_t launch_hadamard_quant(const CUtensorMap* tm, int ntensors, uint8_t* const* x8, float* const* scales,
                                  const float* post, const int* transform, const signed char* signs, int BH, int H,
                                  int N, int d, const int* rope, const float* cos, const float* sin, int n_pos,
                                  int num_sms, int* status, cudaStream_t stream) {
  if (ntensors < 1 || ntensors > 3) return cudaErrorInvalidValue;
  const bool with_rope = rope != nullptr;
  if (with_rope && (cos == nullptr || sin == nullptr)) return cudaErrorInvalidValue;
  HqJob job{};
  for (int t = 0; t < 3; ++t) {
    const int s = t < ntensors ? t : 0;
    job.x8[t] = x8[s];
    job.scales[t] = scales[s];
    job.post[t] = post[s];
    job.transform[t] = transform[s];
    job.rope[t] = with_rope ? rope[s] : 0;
  }
  job.cos = cos;
  job.sin = sin;
  job.H = H;
  job.n_pos = n_pos;
  switch (d) {
    case 64:
      return with_rope ? launch_hq_rope<64>(tm, ntensors, job, signs, BH, N, num_sms, status, stream)
                       : launch_hq<64, false>(tm, ntensors, job, signs, BH, N, num_sms, status, stream);
    case 128:
      return with_rope ? launch_hq_rope<128>(tm, ntensors, job, signs, BH, N, num_sms, status, stream)
                       : launch_hq<128, false>(tm, ntensors, job, signs, BH, N, num_sms, status, stream);
    case 256:
      return with_rope ? launch_hq<256, true>(tm, ntensors, job, signs, BH, N, num_sms, status, stream)
                       : launch_hq<256, false>(tm, ntensors, job, signs, BH, N, num_sms, status, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace ea
