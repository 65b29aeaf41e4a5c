// Backward pass of the exact attention forward, sm_100a (B200): tcgen05 + TMEM + TMA.
//
// The pages state that the backward exists and recomputes the softmax from what the forward
// kept ("FlashAttention-3", section "适用范围和工程限制"; "Flash Attention V3 解析", section
// 2.1, "反向重计算").  With P = softmax(scale Q K^T) rebuilt from the forward's LSE:
//     dV = P^T dO,   dP = dO V^T,   dS = P * (dP - D),   D_i = sum_c dO_ic O_ic,
//     dQ = scale dS K,   dK = scale dS^T Q.
//
// Three launches:
//   bwd_prep_kernel   D and LSE * log2 e per row into a padded workspace (bandwidth-bound).
//   bwd_dkdv_kernel   one CTA per (batch*head, 128-key block): S^T = K Q^T and dP^T = V dO^T per
//                     128-query block, P^T and dS^T back into TMEM, dV += P^T dO, dK += dS^T Q.
//   bwd_dq_kernel     one CTA per (batch*head, 128-query block): S = Q K^T and dP = dO V^T per
//                     128-key block, dS into TMEM, dQ += dS K.
// dQ gets its own pass (recomputing S and dP) instead of atomic additions from the dK/dV
// kernel ("Flash Attention V3 解析", section 4.2): no float atomics, deterministic results.
//
// Roles (both main kernels, 320 threads): warps 0-7 form the softmax backward and the epilogue,
// one TMEM lane (a row of S or S^T) per thread of warps w and w + 4, which take the first and
// the second 64 columns of each block (no exchange between them: LSE and D are given); warp 8
// lane 0 issues every tcgen05.mma, warp 9 lane 0 is the TMA producer.  Every mbarrier wait is
// bounded (wait_bar).

#include <cuda_bf16.h>

#include "attn_kernels.h"
#include "sm100_ptx.cuh"

namespace ea {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// (y0, y1) = (a0 b0 + c0, a1 b1 + c1): one packed f32x2 FMA (each lane rounds like fmaf)
__device__ __forceinline__ void f2_fma(float& y0, float& y1, float a0, float a1, float b0, float b1, float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 ra, ra, rb, rc;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "=f"(y0), "=f"(y1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
// (y0, y1) = ((a0 - b0) m0, (a1 - b1) m1): packed f32x2 subtract, then multiply
__device__ __forceinline__ void f2_sub_mul(float& y0, float& y1, float a0, float a1, float b0, float b1, float m0,
                                           float m1) {
  asm("{\n\t.reg .b64 ra, rb, rm;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rm, {%6, %7};\n\t"
      "sub.rn.f32x2 ra, ra, rb;\n\tmul.rn.f32x2 ra, ra, rm;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "=f"(y0), "=f"(y1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(m0), "f"(m1));
}

// p = 2^x for a pair on the special-function unit.  (Moving a quarter of the pairs to the FMA
// pipe, as the forward does, measured 14% slower here: the pass keeps 128 P values live and the
// extra instructions cost more than the MUFU time they save.)
__device__ __forceinline__ void exp2_pair(float& p0, float& p1, float x0, float x1) {
  p0 = ex2_approx(x0);
  p1 = ex2_approx(x1);
}

// The sequence of one (batch entry, head) pair: fixed-length batches take every field from the
// parameters, packed batches (VL) read the row ranges from the offset arrays.
struct BSeq {
  int h, bc;        // head; batch coordinate of the tensors (0 for packed batches)
  int N, Nk;        // query and key lengths
  int nb, nbk;      // 128-row query and key blocks
  int off;          // Nk - N: key j is visible to query i iff j <= i + off (causal)
  int q0, k0;       // first query and key row (0 unless packed)
  long long lse0;   // LSE index of the sequence's row 0 for this head
  bool bad;         // packed offsets out of order, outside the tensors or too long
};

template <bool VL>
__device__ __forceinline__ BSeq bseq_of(int bh, const BwdParams& p) {
  BSeq s;
  const int b = bh / p.H;
  s.h = bh - b * p.H;
  s.bad = false;
  if constexpr (!VL) {
    s.bc = b;
    s.N = p.N;
    s.Nk = p.Nk;
    s.nb = p.n_blocks;
    s.nbk = p.nbk;
    s.off = p.off;
    s.q0 = s.k0 = 0;
    s.lse0 = static_cast<long long>(bh) * p.N;
  } else {
    int q0 = __ldg(p.cu_q + b), q1 = __ldg(p.cu_q + b + 1);
    int k0 = __ldg(p.cu_k + b), k1 = __ldg(p.cu_k + b + 1);
    if (!(0 <= q0 && q0 <= q1 && q1 <= p.total_q && q1 - q0 <= p.N && 0 <= k0 && k0 <= k1 && k1 <= p.total_k &&
          k1 - k0 <= p.Nk)) {
      s.bad = true;
      q0 = q1 = k0 = k1 = 0;
    }
    s.bc = 0;
    s.N = q1 - q0;
    s.Nk = k1 - k0;
    s.nb = (s.N + 127) / 128;
    s.nbk = (s.Nk + 127) / 128;
    s.off = s.Nk - s.N;
    s.q0 = q0;
    s.k0 = k0;
    s.lse0 = static_cast<long long>(s.h) * p.total_q + q0;
  }
  return s;
}

// ------------------------------------------------------------------------------ preparation
// One row per group of d/16 lanes: D = sum_c dO * O (f32), lse2 = LSE * log2 e; rows past N get
// D = 0 and lse2 = +inf, so that their P (= 2^(s - lse2)) is exactly zero in the main kernels.
template <int D, bool VL>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdParams p) {
  constexpr int kLanes = D / 16;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = t / kLanes;  // over BH * n_pad
  const int part = static_cast<int>(t % kLanes);
  const long long total = static_cast<long long>(p.BH) * p.n_pad;
  const bool in_range = row < total;
  const int bh = in_range ? static_cast<int>(row / p.n_pad) : 0;
  const int r = in_range ? static_cast<int>(row % p.n_pad) : 0;
  const BSeq S = bseq_of<VL>(bh, p);
  if constexpr (VL) {
    if (S.bad && in_range && r == 0 && part == 0) atomicOr(p.status, kDevStatusBadSeqlens);
  }
  const bool valid = in_range && r < S.N;
  float acc = 0.f;
  if (valid) {
    const long long row_q = S.q0 + r;
    const long long oo = S.bc * p.o_sb + S.h * p.o_sh + row_q * p.o_sn + part * 16;
    const long long od = S.bc * p.do_sb + S.h * p.do_sh + row_q * p.do_sn + part * 16;
    const uint4* po = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.o) + oo);
    const uint4* pd = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.dout) + od);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint4 a = __ldg(po + c), b = __ldg(pd + c);
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc = fmaf(__uint_as_float(wa[k] << 16), __uint_as_float(wb[k] << 16), acc);
        acc = fmaf(__uint_as_float(wa[k] & 0xFFFF0000u), __uint_as_float(wb[k] & 0xFFFF0000u), acc);
      }
    }
  }
#pragma unroll
  for (int o = kLanes / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (in_range && part == 0) {
    p.delta[row] = valid ? acc : 0.f;
    p.lse2[row] = valid ? p.lse[S.lse0 + r] * kLog2e : INFINITY;
  }
}

// --------------------------------------------------------------------------- shared pieces
template <int D>
struct BwdCfg {
  static constexpr int kBoxBytes = 128 * 128;            // a 128-row x 128-byte column box
  static constexpr int kBoxes = D * 2 / 128;             // column boxes of a bf16 row
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // 128 rows x D bf16
  static constexpr int kThreads = 320;
  static constexpr int kComputeWarps = 8;   // two per TMEM lane quarter, one per column half
  static constexpr int kMmaWarp = 8;
  static constexpr int kLoadWarp = 9;
  static constexpr uint32_t kIdS = make_idesc(128, 128, 1, false);  // S-type products, both K-major
  static constexpr uint32_t kIdD = make_idesc(128, D, 1, true);     // accumulations, B MN-major
};

// Loads a 128-row tile at rows [row0, row0 + 128) of head h, batch coordinate bc: one 128-row x
// 128-byte TMA box per column box (4-D maps (d, rows, heads, batch), as the forward's).
template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row0, int h,
                                          int bc) {
  using C = BwdCfg<D>;
#pragma unroll
  for (int b = 0; b < C::kBoxes; ++b) tma_load_4d(dst + b * C::kBoxBytes, map, bar, b * 64, row0, h, bc);
}

// X[tmem, 128 x 128] = A B^T with A and B 128 x D tiles in shared memory, both K-major.
template <int D>
__device__ __forceinline__ void mma_abt(uint32_t d_tmem, uint32_t a_base, uint32_t b_base) {
  using C = BwdCfg<D>;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
    mma_f16_ss(d_tmem, make_sdesc_sw128(a_base + off, 16, 1024), make_sdesc_sw128(b_base + off, 16, 1024),
               C::kIdS, kk > 0 ? 1u : 0u);
  }
}

// Acc[tmem, 128 x D] (+)= X B with X 128 x 128 bf16 in TMEM (packed pairs) and B a 128 x D tile
// in shared memory read MN-major (its rows are the contraction index).  X's contraction index
// 16 kk .. 16 kk + 15 sits at TMEM column x_tmem + (kk / 4) * half_stride + (kk % 4) * 8: the two
// 64-wide halves of X are 32 columns each, half_stride apart.
template <int D>
__device__ __forceinline__ void mma_xb(uint32_t d_tmem, uint32_t x_tmem, uint32_t half_stride, uint32_t b_base,
                                       bool acc) {
  using C = BwdCfg<D>;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    mma_f16_ts(d_tmem, x_tmem + (kk >> 2) * half_stride + (kk & 3) * 8,
               make_sdesc_sw128(b_base + kk * 16 * 128, C::kBoxBytes, 1024), C::kIdD, (acc || kk > 0) ? 1u : 0u);
}

// Stores kCols columns of one row of an f32 TMEM accumulator (this thread's lane), times `mul`,
// as bf16 or f32 at out + row_off.
template <int kCols>
__device__ __forceinline__ void store_row(uint32_t t_acc, void* out, size_t row_off, float mul, bool fp32,
                                          bool valid) {
#pragma unroll 1
  for (int cc = 0; cc < kCols / 32; ++cc) {
    uint32_t r[32];
    tmem_ld_32cols(t_acc + 32 * cc, r);
    tmem_ld_wait(r);
    if (!valid) continue;
    if (fp32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + row_off + 32 * cc);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_float4(__uint_as_float(r[4 * i]) * mul, __uint_as_float(r[4 * i + 1]) * mul,
                             __uint_as_float(r[4 * i + 2]) * mul, __uint_as_float(r[4 * i + 3]) * mul);
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + row_off + 32 * cc);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * mul, __uint_as_float(r[8 * i + 1]) * mul);
        w.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * mul, __uint_as_float(r[8 * i + 3]) * mul);
        w.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * mul, __uint_as_float(r[8 * i + 5]) * mul);
        w.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * mul, __uint_as_float(r[8 * i + 7]) * mul);
        dst[i] = w;
      }
    }
  }
}

__device__ __forceinline__ int unit_of(int k) {
  const int g = gridDim.x;
  return k * g + ((k & 1) ? (g - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x));
}

// k-th unit of this CTA from a host-built work list (tab: [gridDim.x + 1] offsets, then unit
// ids), or the round-robin order without one; past the end of the list a value >= every unit.
__device__ __forceinline__ int unit_of(int k, const int* tab) {
  if (tab != nullptr) {
    const int i = __ldg(tab + blockIdx.x) + k;
    return i < __ldg(tab + blockIdx.x + 1) ? __ldg(tab + gridDim.x + 1 + i) : 0x7FFFFFFF;
  }
  return unit_of(k);
}

// dS mode: index of tile (query block i, key block kb) of batch*head bh in the workspace
__device__ __forceinline__ long long ds_tile_index(const BwdParams& p, int bh, int i, int kb) {
  const long long base = static_cast<long long>(bh) * p.ds_tiles;
  if (p.ds_rect) return base + static_cast<long long>(i) * p.ds_nbk + kb;
  return base + (p.causal ? static_cast<long long>(i) * (i + 1) / 2 + kb : static_cast<long long>(i) * p.n_blocks + kb);
}

// dK/dV unit u: key block kb of head bh and the first query block i0 that sees any of its keys
// (causal, bottom-right: query r sees key c iff c <= r + off); i0 >= n_blocks: no query does.
// `present`: the block lies inside its sequence (always, unless packed).
struct KvUnit {
  int bh, kb, i0;
  bool present;
  BSeq S;
};
template <bool VL>
__device__ __forceinline__ KvUnit kv_unit(int u, const BwdParams& p) {
  KvUnit U;
  U.bh = u % p.BH;
  U.kb = u / p.BH;
  U.S = bseq_of<VL>(U.bh, p);
  U.present = U.kb < U.S.nbk;
  const int first_q = U.kb * 128 - U.S.off;  // the smallest query that sees the block's first key
  U.i0 = (!p.causal || first_q <= 0) ? 0 : first_q / 128;
  return U;
}

// dQ unit u: query block qb of head bh (causal: longest first) and its number n of visible key
// blocks (0: its rows see no key).
struct QUnit {
  int bh, qb, n;
  bool present;
  BSeq S;
};
template <bool VL>
__device__ __forceinline__ QUnit q_unit(int u, const BwdParams& p) {
  QUnit U;
  U.bh = u % p.BH;
  U.qb = p.causal ? p.n_blocks - 1 - u / p.BH : u / p.BH;
  U.S = bseq_of<VL>(U.bh, p);
  U.present = U.qb < U.S.nb;
  if (!p.causal) {
    U.n = U.S.nbk;
  } else {
    const int last = min(U.qb * 128 + 127, U.S.N - 1) + U.S.off;
    U.n = last < 0 ? 0 : min(last / 128 + 1, U.S.nbk);
  }
  return U;
}

// Zero rows [row_off, +cols) of a bf16 or f32 gradient (rows that no query or no key reaches).
template <int kCols>
__device__ __forceinline__ void zero_row(void* out, size_t row_off, bool fp32) {
  for (int c = 0; c < kCols; c += 4) {
    if (fp32)
      *reinterpret_cast<float4*>(static_cast<float*>(out) + row_off + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    else
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + row_off + c) = make_uint2(0u, 0u);
  }
}

__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity, int* status) {
  const uint32_t a = smem_addr(bar);
  const unsigned long long t0 = global_timer_ns();
  while (!bar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, kDevStatusTimeout);
      return;
    }
  }
}

// --------------------------------------------------------------------------- dK / dV kernel
// Unit u: bh = u % BH, key block kb = u / BH (causal: longest first, kb = 0 visits every query
// block).  Query blocks i = (causal ? kb : 0) .. n_blocks - 1 stream through two stages of
// shared memory (Q_i, dO_i, and the workspace rows of lse2 and D).
// TMEM columns: S^T [0,128) (then P^T as bf16 pairs in [0,64)), dP^T [128,256) (then dS^T in
// [128,192)), dV [256, 256+D), dK [256+D, 256+2D).
template <int D>
struct DkdvCfg : BwdCfg<D> {
  static constexpr int kStages = 2;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = BwdCfg<D>::kTileBytes;
  static constexpr int kStageOff = 2 * BwdCfg<D>::kTileBytes;
  static constexpr int kStageBytes = 2 * BwdCfg<D>::kTileBytes + 1024;  // Q, dO, lse2[128], D[128]
  static constexpr int kBarOff = kStageOff + kStages * kStageBytes;
  // kv_full, kv_empty, st_full[2], st_empty[2], st_s (S^T in TMEM), st_dp (dP^T in TMEM),
  // pt_full (P^T written), dst_full (dS^T written), dkv_done, dkv_free, drain
  static constexpr int kNumBars = 2 + 2 * kStages + 7;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(256 + 2 * D <= 512, "TMEM budget");
};

template <int D, bool VL, bool DS = false>
__global__ void __launch_bounds__(BwdCfg<D>::kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const BwdParams p) {
  using C = DkdvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 1;
  uint64_t* st_full = bars + 2;
  uint64_t* st_empty = st_full + C::kStages;
  uint64_t* st_s = st_empty + C::kStages;
  uint64_t* st_dp = st_s + 1;
  uint64_t* pt_full = st_dp + 1;
  uint64_t* dst_full = pt_full + 1;
  uint64_t* dkv_done = dst_full + 1;
  uint64_t* dkv_free = dkv_done + 1;
  uint64_t* drain_bar = dkv_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  if (threadIdx.x == 0) {
    bar_init(kv_full, 1);
    bar_init(kv_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      bar_init(&st_full[s], 1);
      bar_init(&st_empty[s], 1);
    }
    bar_init(st_s, 1);
    bar_init(st_dp, 1);
    bar_init(pt_full, C::kComputeWarps);
    bar_init(dst_full, C::kComputeWarps);
    bar_init(dkv_done, 1);
    bar_init(dkv_free, C::kComputeWarps);
    bar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kLoadWarp && lane == 0) {
    prefetch_tensor_map(&tmQ);
    prefetch_tensor_map(&tmK);
    prefetch_tensor_map(&tmV);
    prefetch_tensor_map(&tmdO);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const AbortState ab{abort_flag, p.status};
  const int num_units = p.BH * p.nbk;

  if (warp < C::kComputeWarps) {
    // ===================================== softmax backward: one key row, one half of the queries
    const int row = (warp & 3) * 32 + lane;
    const int h = warp >> 2;  // queries [64h, 64h + 64) of each block
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    uint32_t qc = 0, uit = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = unit_of(k, p.kv_tab);
      if (u >= num_units) break;
      const KvUnit U = kv_unit<VL>(u, p);
      if constexpr (VL) {
        if (!U.present) continue;  // past its sequence's keys: every role skips it
      }
      const BSeq& S = U.S;
      const int kb = U.kb, i0 = U.i0, nb = S.nb;
      const int key_g = kb * 128 + row;
      const long long key_row = S.k0 + key_g;
      const size_t off_v = static_cast<size_t>(S.bc * p.dv_sb + S.h * p.dv_sh + key_row * p.dv_sn) + h * (D / 2);
      const size_t off_k = static_cast<size_t>(S.bc * p.dk_sb + S.h * p.dk_sh + key_row * p.dk_sn) + h * (D / 2);
      if (i0 >= nb) {
        // no query sees these keys (causal, more keys than queries): dK = dV = 0
        if (key_g < S.Nk) {
          zero_row<D / 2>(p.dv, off_v, p.g_fp32 != 0);
          zero_row<D / 2>(p.dk, off_k, p.g_fp32 != 0);
        }
        continue;
      }
      for (int i = i0; i < nb && ok; ++i, ++qc) {
        const uint32_t st = qc % C::kStages;
        // the stage's lse2 / D rows arrived with its TMA transaction count
        ok = warp_all(wait_bar(&st_full[st], (qc / C::kStages) & 1u, ab));
        if (!ok) break;
        const float* lse2 = reinterpret_cast<const float*>(smem + C::kStageOff + st * C::kStageBytes +
                                                           2 * C::kTileBytes);
        const float* dlt = lse2 + 128;
        // some query of block i misses some key of block kb (bottom-right causal mask)
        const bool diag = p.causal && kb * 128 + 127 > i * 128 + S.off;
        // pass 1, from S^T alone: P^T, kept in registers and stored as bf16 over this half's first
        // 32 S^T columns [64h, 64h + 32) (already read by this thread)
        ok = warp_all(wait_bar(st_s, qc & 1u, ab));
        if (!ok) break;
        tc_fence_after();
        float pr[64];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sv[32];
          tmem_ld_32cols(lane_base + 64 * h + 32 * c, sv);
          tmem_ld_wait(sv);
          uint32_t pk[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int ql = 32 * c + 2 * t;  // query pair within this half
            const int qq = 64 * h + ql;     // ... within the block
            float p0, p1;
            float x0, x1;
            f2_fma(x0, x1, __uint_as_float(sv[2 * t]), __uint_as_float(sv[2 * t + 1]), p.scale_log2, p.scale_log2,
                   -lse2[qq], -lse2[qq + 1]);
            exp2_pair(p0, p1, x0, x1);
            if (diag && i * 128 + qq + S.off < key_g) p0 = 0.f;  // key after the query's diagonal
            if (diag && i * 128 + qq + 1 + S.off < key_g) p1 = 0.f;
            pr[ql] = p0;
            pr[ql + 1] = p1;
          }
#pragma unroll
          for (int t = 0; t < 16; ++t) pk[t] = pack_bf16x2(pr[32 * c + 2 * t], pr[32 * c + 2 * t + 1]);
          tmem_st_16cols(lane_base + 64 * h + 16 * c, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(pt_full);
        // pass 2, from dP^T: dS^T = P^T (dP^T - D) as bf16 over dP^T columns [128 + 64h, +32)
        ok = warp_all(wait_bar(st_dp, qc & 1u, ab));
        if (!ok) break;
        tc_fence_after();
        // dS mode: tile (i, kb) of the workspace, stored chunk-major (16-byte chunk j of query
        // columns [8j, 8j + 8) for all 128 key rows, then chunk j + 1), so that a warp's store of
        // one chunk writes 512 contiguous bytes; the layout is the tensor core's non-swizzled
        // MN-major operand layout, which the dQ pass copies into shared memory as it is
        // A key row past the sequence end stores zeros: the dQ pass multiplies the tile by a K tile
        // whose rows there are the next sequence's keys (packed) or TMA's zero fill, and a finite
        // zero keeps both out of dQ (an unmasked score of such a row need not even be finite).
        uint8_t* ds_tile = nullptr;
        [[maybe_unused]] const bool ds_keep = key_g < S.Nk;
        if constexpr (DS) ds_tile = static_cast<uint8_t*>(p.ds) + ds_tile_index(p, U.bh, i, kb) * (128 * 128 * 2) + row * 16;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t dp[32];
          tmem_ld_32cols(lane_base + 128 + 64 * h + 32 * c, dp);
          tmem_ld_wait(dp);
          uint32_t dk[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int ql = 32 * c + 2 * t;
            const int q0 = 64 * h + ql;
            float y0, y1;
            f2_sub_mul(y0, y1, __uint_as_float(dp[2 * t]), __uint_as_float(dp[2 * t + 1]), dlt[q0], dlt[q0 + 1], pr[ql],
                       pr[ql + 1]);
            dk[t] = pack_bf16x2(y0, y1);
          }
          tmem_st_16cols(lane_base + 128 + 64 * h + 16 * c, dk);
          if constexpr (DS) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)  // chunk 8h + 4c + v4: queries 64h + 32c + 8 v4 .. + 8
              *reinterpret_cast<uint4*>(ds_tile + (8 * h + 4 * c + v4) * 2048) =
                  ds_keep ? make_uint4(dk[4 * v4], dk[4 * v4 + 1], dk[4 * v4 + 2], dk[4 * v4 + 3])
                          : make_uint4(0u, 0u, 0u, 0u);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(dst_full);

      }
      if (!ok) break;
      // epilogue: dV and scale * dK of this key block
      ok = warp_all(wait_bar(dkv_done, uit & 1u, ab));
      if (!ok) break;
      tc_fence_after();
      const bool valid = key_g < S.Nk;
      store_row<D / 2>(lane_base + 256 + h * (D / 2), p.dv, off_v, 1.f, p.g_fp32 != 0, valid);
      store_row<D / 2>(lane_base + 256 + D + h * (D / 2), p.dk, off_k, p.scale, p.g_fp32 != 0, valid);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(dkv_free);
      ++uit;
    }
  } else if (warp == C::kMmaWarp) {
    if (lane == 0) {
      // ================================================================== MMA issuer
      const uint32_t k_base = smem_addr(smem + C::kKOff);
      const uint32_t v_base = smem_addr(smem + C::kVOff);
      uint32_t qc = 0, uc = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_of(k, p.kv_tab);
        if (u >= num_units) break;
        const KvUnit U = kv_unit<VL>(u, p);
        if constexpr (VL) {
          if (!U.present) continue;
        }
        const int i0 = U.i0, nb = U.S.nb;
        if (i0 >= nb) continue;  // no query sees the block: nothing loaded, nothing to compute
        if (!(ok = wait_bar(kv_full, uc & 1u, ab))) break;
        auto q_at = [&](uint32_t c) { return smem_addr(smem + C::kStageOff + (c % C::kStages) * C::kStageBytes); };
        // S^T and dP^T of the unit's first query block
        if (!(ok = wait_bar(&st_full[qc % C::kStages], (qc / C::kStages) & 1u, ab))) break;
        mma_abt<D>(tmem, k_base, q_at(qc));                              // S^T = K Q^T
        tc_commit(st_s);
        mma_abt<D>(tmem + 128, v_base, q_at(qc) + C::kTileBytes);       // dP^T = V dO^T
        tc_commit(st_dp);
        // K and V are read only by S^T and dP^T: once the unit's last pair has been issued, their
        // completion frees the buffer, so the next unit's K and V load during this unit's last
        // block and epilogue
        if (i0 + 1 >= nb) tc_commit(kv_empty);
        for (int i = i0; i < nb && ok; ++i, ++qc) {
          const uint32_t q_base = q_at(qc);
          const uint32_t do_base = q_base + C::kTileBytes;
          const bool next = i + 1 < nb;
          if (!(ok = wait_bar(pt_full, qc & 1u, ab))) break;
          tc_fence_after();
          if (i == i0) {
            // the previous unit's epilogue must be done reading dV / dK
            if (!(ok = wait_bar(dkv_free, (uc & 1u) ^ 1u, ab))) break;
            tc_fence_after();
          }
          mma_xb<D>(tmem + 256, tmem, 64, do_base, i > i0);  // dV += P^T dO
          if (next) {
            // S^T of the next block replaces P^T, which dV (issued first) has read
            if (!(ok = wait_bar(&st_full[(qc + 1) % C::kStages], ((qc + 1) / C::kStages) & 1u, ab))) break;
            mma_abt<D>(tmem, k_base, q_at(qc + 1));
            tc_commit(st_s);
          }
          if (!(ok = wait_bar(dst_full, qc & 1u, ab))) break;
          tc_fence_after();
          mma_xb<D>(tmem + 256 + D, tmem + 128, 64, q_base, i > i0);  // dK += dS^T Q
          tc_commit(&st_empty[qc % C::kStages]);
          if (next) {
            mma_abt<D>(tmem + 128, v_base, q_at(qc + 1) + C::kTileBytes);
            tc_commit(st_dp);
            if (i + 2 >= nb) tc_commit(kv_empty);  // that was the unit's last dP^T
          }
        }
        if (!ok) break;
        tc_commit(dkv_done);
        ++uc;
      }
      tc_commit(drain_bar);
      drain(drain_bar, 0, p.status);
    }
  } else {
    if (lane == 0) {
      // =============================================================== TMA producer
      uint32_t qc = 0, uc = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_of(k, p.kv_tab);
        if (u >= num_units) break;
        const KvUnit U = kv_unit<VL>(u, p);
        if constexpr (VL) {
          if (!U.present) continue;
        }
        const BSeq& S = U.S;
        const int bh = U.bh, kb = U.kb, i0 = U.i0, nb = S.nb;
        if (i0 >= nb) continue;
        if (uc > 0 && !(ok = wait_bar(kv_empty, (uc - 1u) & 1u, ab))) break;
        bar_arrive_expect_tx(kv_full, 2 * C::kTileBytes);
        load_tile<D>(smem + C::kKOff, &tmK, kv_full, S.k0 + kb * 128, S.h, S.bc);
        load_tile<D>(smem + C::kVOff, &tmV, kv_full, S.k0 + kb * 128, S.h, S.bc);
        ++uc;
        for (int i = i0; i < nb && ok; ++i, ++qc) {
          const uint32_t st = qc % C::kStages;
          if (!(ok = wait_bar(&st_empty[st], ((qc / C::kStages) & 1u) ^ 1u, ab))) break;
          uint8_t* base = smem + C::kStageOff + st * C::kStageBytes;
          bar_arrive_expect_tx(&st_full[st], 2 * C::kTileBytes + 1024);
          load_tile<D>(base, &tmQ, &st_full[st], S.q0 + i * 128, S.h, S.bc);
          load_tile<D>(base + C::kTileBytes, &tmdO, &st_full[st], S.q0 + i * 128, S.h, S.bc);
          const size_t w = static_cast<size_t>(bh) * p.n_pad + static_cast<size_t>(i) * 128;
          bulk_load_g2s(base + 2 * C::kTileBytes, p.lse2 + w, 512, &st_full[st]);
          bulk_load_g2s(base + 2 * C::kTileBytes + 512, p.delta + w, 512, &st_full[st]);
        }
      }
      // every issued copy lands before the CTA can exit
      if (uc > 0) drain(kv_full, (uc - 1u) & 1u, p.status);
      const uint32_t first = qc > static_cast<uint32_t>(C::kStages) ? qc - C::kStages : 0u;
      for (uint32_t i = first; i < qc; ++i) drain(&st_full[i % C::kStages], (i / C::kStages) & 1u, p.status);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------ dQ kernel
// Unit u: bh = u % BH, query block qb (causal: longest first).  K_j and V_j stream through two
// rings (K: 3 slots, since dQ(j) is issued a block late and holds K_j; V: 2).  TMEM columns:
// S [0,128), dP [128,256), dQ [256, 256+D), dS double buffer [384, 448) and [448, 512) (bf16
// pairs).  The single MMA thread is the tensor pipe's timeline (an issue returns about when the
// pipe has taken it), so it issues in order of urgency: S(j+1) as soon as the softmax has read
// S(j), then dQ(j-1), then dP(j+1) once dS(j) is written.
template <int D>
struct DqCfg : BwdCfg<D> {
  static constexpr int kQOff = 0;
  static constexpr int kDoOff = BwdCfg<D>::kTileBytes;
  static constexpr int kKSlots = 3;
  static constexpr int kVSlots = 2;
  static constexpr int kKOff = 2 * BwdCfg<D>::kTileBytes;
  static constexpr int kVOff = kKOff + kKSlots * BwdCfg<D>::kTileBytes;
  static constexpr int kBarOff = kVOff + kVSlots * BwdCfg<D>::kTileBytes;
  // kfull[3], kempty[3], vfull[2], vempty[2], qdo_full, qdo_empty, s_full, dp_full, s_free,
  // ds_full[2], dq_done, dq_free, drain
  static constexpr int kNumBars = 2 * (kKSlots + kVSlots) + 10;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(256 + D <= 384, "TMEM budget");
};

template <int D, bool VL>
__global__ void __launch_bounds__(BwdCfg<D>::kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const BwdParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* kfull = bars;
  uint64_t* kempty = kfull + C::kKSlots;
  uint64_t* vfull = kempty + C::kKSlots;
  uint64_t* vempty = vfull + C::kVSlots;
  uint64_t* qdo_full = vempty + C::kVSlots;
  uint64_t* qdo_empty = qdo_full + 1;
  uint64_t* s_full = qdo_empty + 1;  // S in TMEM
  uint64_t* dp_full = s_full + 1;    // dP in TMEM
  uint64_t* s_free = dp_full + 1;    // the softmax has read S (pass 1 done)
  uint64_t* ds_full = s_free + 1;    // [2] dS written
  uint64_t* dq_done = ds_full + 2;
  uint64_t* dq_free = dq_done + 1;
  uint64_t* drain_bar = dq_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kKSlots; ++i) {
      bar_init(&kfull[i], 1);
      bar_init(&kempty[i], 1);
    }
    for (int i = 0; i < C::kVSlots; ++i) {
      bar_init(&vfull[i], 1);
      bar_init(&vempty[i], 1);
    }
    bar_init(qdo_full, 1);
    bar_init(qdo_empty, 1);
    bar_init(s_full, 1);
    bar_init(dp_full, 1);
    bar_init(s_free, C::kComputeWarps);
    bar_init(&ds_full[0], C::kComputeWarps);
    bar_init(&ds_full[1], C::kComputeWarps);
    bar_init(dq_done, 1);
    bar_init(dq_free, C::kComputeWarps);
    bar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kLoadWarp && lane == 0) {
    prefetch_tensor_map(&tmQ);
    prefetch_tensor_map(&tmK);
    prefetch_tensor_map(&tmV);
    prefetch_tensor_map(&tmdO);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const AbortState ab{abort_flag, p.status};
  const int num_units = p.BH * p.n_blocks;

  if (warp < C::kComputeWarps) {
    // ===================================== softmax backward: one query row, one half of the keys
    const int row = (warp & 3) * 32 + lane;
    const int h = warp >> 2;  // keys [64h, 64h + 64) of each block
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    uint32_t sc = 0, uit = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = unit_of(k);
      if (u >= num_units) break;
      const QUnit U = q_unit<VL>(u, p);
      if constexpr (VL) {
        if (!U.present) continue;  // past its sequence's queries: every role skips it
      }
      const BSeq& S = U.S;
      const int bh = U.bh, qb = U.qb, n = U.n;
      const int q_g = qb * 128 + row;
      const size_t off_q = static_cast<size_t>(S.bc * p.dq_sb + S.h * p.dq_sh + (S.q0 + static_cast<long long>(q_g)) *
                                               p.dq_sn) + h * (D / 2);
      if (n == 0) {
        // these queries see no key (causal, more queries than keys, or no keys): dQ = 0
        if (q_g < S.N) zero_row<D / 2>(p.dq, off_q, p.g_fp32 != 0);
        continue;
      }
      const size_t w = static_cast<size_t>(bh) * p.n_pad + q_g;
      const float lse2 = p.lse2[w];  // +inf on padded rows: P = 0 there
      const float dlt = p.delta[w];
      for (int j = 0; j < n && ok; ++j, ++sc) {
        const uint32_t t_ds = lane_base + 384 + (sc & 1u) * 64;
        const bool mask = (j * 128 + 128 > S.Nk) || (p.causal && j * 128 + 127 > qb * 128 + S.off);
        const int lim = min(S.Nk, p.causal ? q_g + S.off + 1 : S.Nk) - j * 128;  // visible keys of this block
        // pass 1, from S alone: P in registers; then S's columns may take the next block
        ok = warp_all(wait_bar(s_full, sc & 1u, ab));
        if (!ok) break;
        tc_fence_after();
        float pr[64];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sv[32];
          tmem_ld_32cols(lane_base + 64 * h + 32 * c, sv);
          tmem_ld_wait(sv);
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int kl = 32 * c + 2 * t;  // key pair within this half
            const int kk = 64 * h + kl;     // ... within the block
            float p0, p1;
            float x0, x1;
            f2_fma(x0, x1, __uint_as_float(sv[2 * t]), __uint_as_float(sv[2 * t + 1]), p.scale_log2, p.scale_log2,
                   -lse2, -lse2);
            exp2_pair(p0, p1, x0, x1);
            if (mask && kk >= lim) p0 = 0.f;
            if (mask && kk + 1 >= lim) p1 = 0.f;
            pr[kl] = p0;
            pr[kl + 1] = p1;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(s_free);
        // pass 2, from dP: dS = P (dP - D) as bf16 into the dS buffer of this block
        ok = warp_all(wait_bar(dp_full, sc & 1u, ab));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t dp[32];
          tmem_ld_32cols(lane_base + 128 + 64 * h + 32 * c, dp);
          tmem_ld_wait(dp);
          uint32_t dk[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int k0 = 32 * c + 2 * t;
            float y0, y1;
            f2_sub_mul(y0, y1, __uint_as_float(dp[2 * t]), __uint_as_float(dp[2 * t + 1]), dlt, dlt, pr[k0], pr[k0 + 1]);
            dk[t] = pack_bf16x2(y0, y1);
          }
          tmem_st_16cols(t_ds + 32 * h + 16 * c, dk);  // the buffer holds the 128 keys in order
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(&ds_full[sc & 1u]);
      }
      if (!ok) break;
      ok = warp_all(wait_bar(dq_done, uit & 1u, ab));
      if (!ok) break;
      tc_fence_after();
      store_row<D / 2>(lane_base + 256 + h * (D / 2), p.dq, off_q, p.scale, p.g_fp32 != 0, q_g < S.N);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(dq_free);
      ++uit;
    }
  } else if (warp == C::kMmaWarp) {
    if (lane == 0) {
      // ================================================================== MMA issuer
      const uint32_t q_base = smem_addr(smem + C::kQOff);
      const uint32_t do_base = smem_addr(smem + C::kDoOff);
      const uint32_t k_ring = smem_addr(smem + C::kKOff);
      const uint32_t v_ring = smem_addr(smem + C::kVOff);
      uint32_t kit = 0, vit = 0, qit = 0, sc = 0, uc = 0;
      bool ok = true;
      auto k_addr = [&](uint32_t idx) { return k_ring + (idx % C::kKSlots) * C::kTileBytes; };
      auto v_addr = [&](uint32_t idx) { return v_ring + (idx % C::kVSlots) * C::kTileBytes; };
      auto k_wait = [&](uint32_t idx) { return wait_bar(&kfull[idx % C::kKSlots], (idx / C::kKSlots) & 1u, ab); };
      auto v_wait = [&](uint32_t idx) { return wait_bar(&vfull[idx % C::kVSlots], (idx / C::kVSlots) & 1u, ab); };
      for (int k = 0; ok; ++k) {
        const int u = unit_of(k);
        if (u >= num_units) break;
        const QUnit U = q_unit<VL>(u, p);
        if constexpr (VL) {
          if (!U.present) continue;
        }
        const int n = U.n;
        const uint32_t kb0 = kit, vb0 = vit;  // K_j = kb0 + j, V_j = vb0 + j
        kit += n;
        vit += n;
        if (!(ok = wait_bar(qdo_full, qit & 1u, ab))) break;
        ++qit;
        if (n == 0) {  // the unit's queries see no key: release Q, dO; no dQ
          tc_commit(qdo_empty);
          continue;
        }
        bool dq_started = false;
        // dQ(j) += dS(j) K_j, from the dS buffer of global block number `blk`
        auto issue_dq = [&](int j, uint32_t blk) {
          if (!dq_started) {
            // the previous unit's epilogue must be done reading dQ
            if (!wait_bar(dq_free, (uc & 1u) ^ 1u, ab)) return false;
            tc_fence_after();
            dq_started = true;
          }
          mma_xb<D>(tmem + 256, tmem + 384 + (blk & 1u) * 64, 32, k_addr(kb0 + j), j > 0);
          tc_commit(&kempty[(kb0 + j) % C::kKSlots]);
          return true;
        };
        // S(0), dP(0)
        if (!(ok = k_wait(kb0)) || !(ok = v_wait(vb0))) break;
        mma_abt<D>(tmem, q_base, k_addr(kb0));
        tc_commit(s_full);
        mma_abt<D>(tmem + 128, do_base, v_addr(vb0));
        tc_commit(dp_full);
        tc_commit(&vempty[vb0 % C::kVSlots]);
        // Q and dO are read only by S and dP: once the unit's last pair has been issued, their
        // completion frees the buffer for the next unit's Q and dO (dQ reads dS and K)
        if (n == 1) tc_commit(qdo_empty);
        for (int j = 0; j < n && ok; ++j, ++sc) {
          const bool next = j + 1 < n;
          if (next) {
            // S(j+1) as soon as the softmax has read S(j) (its pass 1)
            if (!(ok = k_wait(kb0 + j + 1))) break;
            if (!(ok = wait_bar(s_free, sc & 1u, ab))) break;
            tc_fence_after();
            mma_abt<D>(tmem, q_base, k_addr(kb0 + j + 1));
            tc_commit(s_full);
          }
          if (j > 0 && !(ok = issue_dq(j - 1, sc - 1))) break;
          // dP(j+1) once dS(j) is written (pass 2 has read dP(j))
          if (!(ok = wait_bar(&ds_full[sc & 1u], (sc >> 1) & 1u, ab))) break;
          tc_fence_after();
          if (next) {
            if (!(ok = v_wait(vb0 + j + 1))) break;
            mma_abt<D>(tmem + 128, do_base, v_addr(vb0 + j + 1));
            tc_commit(dp_full);
            tc_commit(&vempty[(vb0 + j + 1) % C::kVSlots]);
            if (j + 2 == n) tc_commit(qdo_empty);  // that was the unit's last dP
          }
        }
        if (!ok) break;
        if (!(ok = issue_dq(n - 1, sc - 1))) break;
        if (!ok) break;
        tc_commit(dq_done);
        ++uc;
      }
      tc_commit(drain_bar);
      drain(drain_bar, 0, p.status);
    }
  } else {
    if (lane == 0) {
      // =============================================================== TMA producer
      uint32_t kit = 0, vit = 0, qit = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_of(k);
        if (u >= num_units) break;
        const QUnit U = q_unit<VL>(u, p);
        if constexpr (VL) {
          if (!U.present) continue;
        }
        const BSeq& S = U.S;
        const int qb = U.qb, n = U.n;
        if (qit > 0 && !(ok = wait_bar(qdo_empty, (qit - 1u) & 1u, ab))) break;
        bar_arrive_expect_tx(qdo_full, 2 * C::kTileBytes);
        load_tile<D>(smem + C::kQOff, &tmQ, qdo_full, S.q0 + qb * 128, S.h, S.bc);
        load_tile<D>(smem + C::kDoOff, &tmdO, qdo_full, S.q0 + qb * 128, S.h, S.bc);
        ++qit;
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t ks = kit % C::kKSlots;
          if (!(ok = wait_bar(&kempty[ks], ((kit / C::kKSlots) & 1u) ^ 1u, ab))) break;
          bar_arrive_expect_tx(&kfull[ks], C::kTileBytes);
          load_tile<D>(smem + C::kKOff + ks * C::kTileBytes, &tmK, &kfull[ks], S.k0 + j * 128, S.h, S.bc);
          ++kit;
          const uint32_t vs = vit % C::kVSlots;
          if (!(ok = wait_bar(&vempty[vs], ((vit / C::kVSlots) & 1u) ^ 1u, ab))) break;
          bar_arrive_expect_tx(&vfull[vs], C::kTileBytes);
          load_tile<D>(smem + C::kVOff + vs * C::kTileBytes, &tmV, &vfull[vs], S.k0 + j * 128, S.h, S.bc);
          ++vit;
        }
      }
      // every issued copy lands before the CTA can exit
      const uint32_t kf = kit > static_cast<uint32_t>(C::kKSlots) ? kit - C::kKSlots : 0u;
      for (uint32_t i = kf; i < kit; ++i) drain(&kfull[i % C::kKSlots], (i / C::kKSlots) & 1u, p.status);
      const uint32_t vf = vit > static_cast<uint32_t>(C::kVSlots) ? vit - C::kVSlots : 0u;
      for (uint32_t i = vf; i < vit; ++i) drain(&vfull[i % C::kVSlots], (i / C::kVSlots) & 1u, p.status);
      if (qit > 0) drain(qdo_full, (qit - 1u) & 1u, p.status);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ dQ from stored dS (dS mode)
// Unit u: query block i of head bh (causal: longest first) and its key blocks kb = 0 .. n-1,
// streamed through a ring of slots that each hold the bf16 dS^T tile (i, kb) written by the dK/dV
// kernel (one 32 KB bulk copy: it is stored in the non-swizzled MN-major operand layout) and the
// K tile kb (TMA): dQ_i += dS(i, kb) K_kb on the tensor cores, A = dS read MN-major (queries
// contiguous in 16-byte chunks), B = K read MN-major (d contiguous, 128-byte swizzle).  No S, P or dP is
// recomputed: five products in all instead of seven.  dQ is double-buffered in TMEM (2 x D
// columns) so that one unit's epilogue overlaps the next unit's products.  Roles: warps 0-3 the
// epilogue (one TMEM lane quarter each), warp 4 lane 0 the MMA issuer, warp 5 lane 0 the TMA
// producer.  Fixed-length batches, equal query and key lengths.
template <int D>
struct DqDsCfg {
  static constexpr int kDsBytes = 128 * 128 * 2;             // one dS^T tile (chunk-major)
  static constexpr int kKBytes = BwdCfg<D>::kTileBytes;      // one K tile
  static constexpr int kSlotBytes = kDsBytes + kKBytes;
  static constexpr int kSlots = 3;
  static constexpr int kThreads = 192;
  static constexpr int kMmaWarp = 4;
  static constexpr int kLoadWarp = 5;
  static constexpr int kBarOff = kSlots * kSlotBytes;
  // full[kSlots], empty[kSlots], dq_done[2], dq_free[2], drain
  static constexpr int kNumBars = 2 * kSlots + 5;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static constexpr uint32_t kTmemCols = 2 * D;
  // M = 128 queries, N = D, K = 16 keys per instruction; A and B both MN-major
  static constexpr uint32_t kIdQ = make_idesc(128, D, 1, true) | (1u << 15);
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

template <int D, bool VL>
__global__ void __launch_bounds__(DqDsCfg<D>::kThreads, 1)
    bwd_dq_ds_kernel(const __grid_constant__ CUtensorMap tmK, const BwdParams p) {
  using C = DqDsCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = full + C::kSlots;
  uint64_t* dq_done = empty + C::kSlots;
  uint64_t* dq_free = dq_done + 2;
  uint64_t* drain_bar = dq_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kSlots; ++s) {
      bar_init(&full[s], 1);
      bar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      bar_init(&dq_done[b], 1);
      bar_init(&dq_free[b], 4);
    }
    bar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kLoadWarp && lane == 0) {
    prefetch_tensor_map(&tmK);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const AbortState ab{abort_flag, p.status};
  const int num_units = p.BH * p.n_blocks;

  if (warp < 4) {
    // ================================================================ epilogue: scale * dQ
    const int row = warp * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t uc = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = unit_of(k, p.q_tab);
      if (u >= num_units) break;
      const QUnit U = q_unit<VL>(u, p);
      if constexpr (VL) {
        if (!U.present) continue;  // past its sequence's queries: every role skips it
      }
      const BSeq& S = U.S;
      const int q_g = U.qb * 128 + row;
      const size_t off_q = static_cast<size_t>(S.bc * p.dq_sb + S.h * p.dq_sh +
                                               (S.q0 + static_cast<long long>(q_g)) * p.dq_sn);
      if (U.n == 0) {  // these queries see no key: dQ = 0 (no products, no TMEM buffer)
        if (q_g < S.N) zero_row<D>(p.dq, off_q, p.g_fp32 != 0);
        continue;
      }
      const uint32_t buf = uc & 1u;
      ok = warp_all(wait_bar(&dq_done[buf], (uc >> 1) & 1u, ab));
      if (!ok) break;
      tc_fence_after();
      store_row<D>(lane_base + buf * D, p.dq, off_q, p.scale, p.g_fp32 != 0, q_g < S.N);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(&dq_free[buf]);
      ++uc;
    }
  } else if (warp == C::kMmaWarp) {
    if (lane == 0) {
      // ================================================================== MMA issuer
      const uint32_t ring = smem_addr(smem);
      uint32_t it = 0, uc = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_of(k, p.q_tab);
        if (u >= num_units) break;
        const QUnit U = q_unit<VL>(u, p);
        if constexpr (VL) {
          if (!U.present) continue;
        }
        if (U.n == 0) continue;
        const uint32_t buf = uc & 1u;
        // the epilogue of the unit before last must be done reading this dQ buffer
        if (!(ok = wait_bar(&dq_free[buf], ((uc >> 1) & 1u) ^ 1u, ab))) break;
        tc_fence_after();
        for (int j = 0; j < U.n && ok; ++j, ++it) {
          const uint32_t s = it % C::kSlots;
          // TMA-filled shared memory read by the tensor core: the wait alone orders it
          if (!(ok = wait_bar(&full[s], (it / C::kSlots) & 1u, ab))) break;
          const uint32_t a_base = ring + s * C::kSlotBytes;
          const uint32_t b_base = a_base + C::kDsBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ss(tmem + buf * D, make_sdesc_mn_noswz(a_base + kk * 256, 2048, 128),
                       make_sdesc_sw128(b_base + kk * 16 * 128, BwdCfg<D>::kBoxBytes, 1024), C::kIdQ,
                       (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&dq_done[buf]);
        ++uc;
      }
      tc_commit(drain_bar);
      drain(drain_bar, 0, p.status);
    }
  } else {
    if (lane == 0) {
      // =============================================================== TMA producer
      uint32_t it = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_of(k, p.q_tab);
        if (u >= num_units) break;
        const QUnit U = q_unit<VL>(u, p);
        if constexpr (VL) {
          if (!U.present) continue;
        }
        const BSeq& S = U.S;
        for (int j = 0; j < U.n && ok; ++j, ++it) {
          const uint32_t s = it % C::kSlots;
          if (!(ok = wait_bar(&empty[s], ((it / C::kSlots) & 1u) ^ 1u, ab))) break;
          uint8_t* dst = smem + s * C::kSlotBytes;
          bar_arrive_expect_tx(&full[s], C::kSlotBytes);
          bulk_load_g2s(dst, static_cast<const uint8_t*>(p.ds) + ds_tile_index(p, U.bh, U.qb, j) * C::kDsBytes,
                        C::kDsBytes, &full[s]);
          load_tile<D>(dst + C::kDsBytes, &tmK, &full[s], S.k0 + j * 128, S.h, S.bc);
        }
      }
      // every issued copy lands before the CTA can exit
      const uint32_t first = it > static_cast<uint32_t>(C::kSlots) ? it - C::kSlots : 0u;
      for (uint32_t i = first; i < it; ++i) drain(&full[i % C::kSlots], (i / C::kSlots) & 1u, p.status);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, bool VL>
cudaError_t setup_d() {
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<D, VL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       DkdvCfg<D>::kSmemAlloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(bwd_dq_kernel<D, VL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DqCfg<D>::kSmemAlloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(bwd_dkdv_kernel<D, VL, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DkdvCfg<D>::kSmemAlloc);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(bwd_dq_ds_kernel<D, VL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DqDsCfg<D>::kSmemAlloc);
  return e;
}

template <int D, bool VL>
cudaError_t launch_d_ds(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dout,
                        const BwdParams& p, int num_sms, cudaStream_t stream) {
  const long long rows = static_cast<long long>(p.BH) * p.n_pad;
  const long long threads = rows * (D / 16);
  const long long blocks = (threads + 255) / 256;
  if (blocks > 0x7FFFFFFFLL || p.ds == nullptr || (p.cu_q != nullptr) != VL) return cudaErrorInvalidValue;
  bwd_prep_kernel<D, VL><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int kv_units = p.BH * p.nbk;
  const int kv_grid = kv_units < num_sms ? kv_units : num_sms;
  bwd_dkdv_kernel<D, VL, true><<<kv_grid, BwdCfg<D>::kThreads, DkdvCfg<D>::kSmemAlloc, stream>>>(q, k, v, dout, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int q_units = p.BH * p.n_blocks;
  const int q_grid = q_units < num_sms ? q_units : num_sms;
  bwd_dq_ds_kernel<D, VL><<<q_grid, DqDsCfg<D>::kThreads, DqDsCfg<D>::kSmemAlloc, stream>>>(k, p);
  return cudaGetLastError();
}

template <int D, bool VL>
cudaError_t launch_d(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dout,
                     const BwdParams& p, int num_sms, cudaStream_t stream) {
  const long long rows = static_cast<long long>(p.BH) * p.n_pad;
  const long long threads = rows * (D / 16);
  const long long blocks = (threads + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  bwd_prep_kernel<D, VL><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int kv_units = p.BH * p.nbk;
  const int kv_grid = kv_units < num_sms ? kv_units : num_sms;
  bwd_dkdv_kernel<D, VL><<<kv_grid, BwdCfg<D>::kThreads, DkdvCfg<D>::kSmemAlloc, stream>>>(q, k, v, dout, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int q_units = p.BH * p.n_blocks;
  const int q_grid = q_units < num_sms ? q_units : num_sms;
  bwd_dq_kernel<D, VL><<<q_grid, BwdCfg<D>::kThreads, DqCfg<D>::kSmemAlloc, stream>>>(q, k, v, dout, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t setup_bwd_kernels() {
  cudaError_t e = setup_d<64, false>();
  if (e == cudaSuccess) e = setup_d<128, false>();
  if (e == cudaSuccess) e = setup_d<64, true>();
  if (e == cudaSuccess) e = setup_d<128, true>();
  return e;
}

cudaError_t launch_attn_bwd(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                            const CUtensorMap& dout, const BwdParams& p, int num_sms, cudaStream_t stream) {
  const bool vl = p.cu_q != nullptr;
  switch (d) {
    case 64:
      return vl ? launch_d<64, true>(q, k, v, dout, p, num_sms, stream)
                : launch_d<64, false>(q, k, v, dout, p, num_sms, stream);
    case 128:
      return vl ? launch_d<128, true>(q, k, v, dout, p, num_sms, stream)
                : launch_d<128, false>(q, k, v, dout, p, num_sms, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_bwd_ds(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                               const CUtensorMap& dout, const BwdParams& p, int num_sms,
                               cudaStream_t stream) {
  const bool vl = p.cu_q != nullptr;
  switch (d) {
    case 64:
      return vl ? launch_d_ds<64, true>(q, k, v, dout, p, num_sms, stream)
                : launch_d_ds<64, false>(q, k, v, dout, p, num_sms, stream);
    case 128:
      return vl ? launch_d_ds<128, true>(q, k, v, dout, p, num_sms, stream)
                : launch_d_ds<128, false>(q, k, v, dout, p, num_sms, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace ea
