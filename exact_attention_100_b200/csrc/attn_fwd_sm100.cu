// Exact attention forward for sm_100a (B200): persistent, warp-specialised, tcgen05 + TMEM.
//
// What one CTA computes: for a unit (one batch*head, NQ consecutive 128-row Q tiles) the
// tiled recurrence of "FlashAttention-2/3", section "技术原理" (outer loop over Q blocks,
// inner loop over K/V blocks, running row max m and row sum l), in the FA-2 form with the
// normalisation deferred to the end ("FlashAttention-2/3", FA-2 improvement 1), writing O and
// the per-row logsumexp ("Flash Attention V3 解析", section 2.2).  Causal units skip the K/V
// blocks that are entirely masked (same section).
//
// Roles (warp specialisation, "FlashAttention-3", section "异步搬运与异步计算"):
//   warps 0..4*NQ-1      softmax warpgroup q = warp/4: one thread per S row (TMEM lane)
//   next 4 warps         correction warpgroup: lazy O rescale in TMEM, then the epilogue
//   next warp            MMA issuer (one thread issues every tcgen05.mma)
//   next warp            TMA producer (one thread; fills the K/V ring and the Q tiles)
//   last 2 warps         idle (keep the CTA a whole number of warpgroups)
//
// Overlap ("FlashAttention-3", sections "Ping-pong 调度" and "同一个 warpgroup 内部也能再叠一层"):
// with NQ = 2 the MMA issue order per K/V block j is PV0(j), S0(j+1), PV1(j), S1(j+1), so the
// tensor core computes one tile's GEMMs while the other tile's softmax runs.
//
// TMEM (512 columns x 128 lanes, f32): S_q at columns [128q, 128q+128); P_q (bf16 pairs)
// overwrites the first 64 of them; O_q at [128*NQ + D*q, +D).
//
// Lazy rescale: a row's reference max m moves only when a block max exceeds it by more than
// kTau (base-2 units); then the correction warpgroup multiplies that row of O by
// alpha = 2^(m_old - m_new) before the next P.V accumulates (l is rescaled by the softmax
// thread).  O and l always refer to the same m, so O / l is exact; p <= 2^kTau.

#include <cuda_bf16.h>

#include "attn_kernels.h"
#include "sm100_ptx.cuh"

namespace ea {

constexpr float kTau = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D, int NQ>
struct FwdCfg {
  static constexpr int kBoxBytes = 128 * 128;             // one TMA box: 128 rows x 128 bytes
  static constexpr int kBoxes = D / 64;                   // 64 bf16 per 128-byte row
  static constexpr int kTileBytes = kBoxes * kBoxBytes;   // 128 rows x D bf16
  static constexpr int kSlots = D == 64 ? 8 : (D == 128 ? 4 : 2);
  static constexpr int kSCol = 0;
  static constexpr int kOCol = NQ * 128;
  static constexpr int kTmemCols = 512;
  static constexpr int kCorrWarp0 = 4 * NQ;
  static constexpr int kMmaWarp = 4 * NQ + 4;
  static constexpr int kLoadWarp = 4 * NQ + 5;
  static constexpr int kThreads = (4 * NQ + 8) * 32;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = NQ * kTileBytes;
  static constexpr int kBarOff = kRingOff + kSlots * kTileBytes;
  static constexpr int kNumBars = 2 * kSlots + 2 + 4 * NQ + 1;
  static constexpr int kAlphaOff = kBarOff + ((kNumBars * 8 + 15) / 16) * 16;
  static constexpr int kRowMOff = kAlphaOff + NQ * 2 * 128 * 4;
  static constexpr int kRowLOff = kRowMOff + NQ * 128 * 4;
  static constexpr int kMiscOff = kRowLOff + NQ * 128 * 4;
  static constexpr int kSmemBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;  // room to align the base to 1024 bytes
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(NQ * 128 + NQ * D <= kTmemCols, "TMEM budget");
};

struct Unit {
  int bh;
  int tile0;     // index of the first 128-row Q tile of the unit
  int n[2];      // K/V blocks each Q tile visits (0: tile lies past the sequence end)
  int n_max;
};

template <int NQ>
__device__ __forceinline__ Unit decode_unit(int u, const FwdParams& p) {
  Unit U;
  const int r = u / p.BH;
  U.bh = u - r * p.BH;
  const int pair = p.causal ? (p.n_pairs - 1 - r) : r;  // causal: longest units first
  U.tile0 = pair * NQ;
  U.n_max = 0;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int t = U.tile0 + q;
    int n = 0;
    if (q < NQ && t * 128 < p.N) n = p.causal ? min(t + 1, p.n_blocks) : p.n_blocks;
    U.n[q] = n;
    U.n_max = max(U.n_max, n);
  }
  return U;
}

// k-th unit of this CTA: round-robin over CTAs, alternating direction every round.
__device__ __forceinline__ int unit_index(int k) {
  const int g = gridDim.x;
  return k * g + ((k & 1) ? (g - 1 - (int)blockIdx.x) : (int)blockIdx.x);
}

// Bounded wait that ignores the abort flag: used at exit to let this thread's own async
// copies and MMAs finish before shared memory and TMEM are released.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* status) {
  const uint32_t a = smem_addr(bar);
  const unsigned long long t0 = global_timer_ns();
  while (!bar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, kDevStatusTimeout);
      return;
    }
  }
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, int NQ>
__global__ void __launch_bounds__(FwdCfg<D, NQ>::kThreads, 1)
    attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D, NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kSlots;
  uint64_t* q_full = bars + 2 * C::kSlots;
  uint64_t* q_empty = q_full + 1;
  uint64_t* s_full = q_full + 2;
  uint64_t* p_full = s_full + NQ;
  uint64_t* o_corr = p_full + NQ;
  uint64_t* o_done = o_corr + NQ;
  uint64_t* drain = o_done + NQ;
  float* alpha_s = reinterpret_cast<float*>(smem + C::kAlphaOff);
  float* row_m = reinterpret_cast<float*>(smem + C::kRowMOff);
  float* row_l = reinterpret_cast<float*>(smem + C::kRowLOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kSlots; ++i) {
      bar_init(&full[i], 1);
      bar_init(&empty[i], 1);
    }
    bar_init(q_full, 1);
    bar_init(q_empty, 1);
    for (int q = 0; q < NQ; ++q) {
      bar_init(&s_full[q], 1);
      bar_init(&p_full[q], 128);
      bar_init(&o_corr[q], 128);
      bar_init(&o_done[q], 1);
    }
    bar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kLoadWarp && lane == 0) {
    prefetch_tensor_map(&tmQ);
    prefetch_tensor_map(&tmK);
    prefetch_tensor_map(&tmV);
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

  if (warp < 4 * NQ) {
    // ------------------------------------------------------------------ softmax warpgroups
    const int q = warp >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tS = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + C::kSCol + q * 128;
    const float sl2 = p.scale_log2;
    uint32_t sit = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = unit_index(k);
      if (u >= p.num_units) break;
      const Unit U = decode_unit<NQ>(u, p);
      const int n = U.n[q];
      const int tile_row0 = (U.tile0 + q) * 128;
      const int row_g = tile_row0 + row;
      int lim_row = p.N;  // keys [0, lim_row) are visible to this row
      if (p.causal) lim_row = min(lim_row, row_g + 1);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        ok = warp_all(wait_bar(&s_full[q], sit & 1, ab));
        if (!ok) break;
        tc_fence_after();
        const int key0 = j * 128;
        const bool need_mask = (key0 + 128 > p.N) || (p.causal && key0 + 127 > tile_row0);
        const int lim = lim_row - key0;
        uint32_t r[32];
        // pass 1: row max of the block
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld_32cols(tS + 32 * c, r);
          tmem_ld_wait(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float s = __uint_as_float(r[i]);
            mx = (need_mask && 32 * c + i >= lim) ? mx : fmaxf(mx, s);
          }
        }
        const float mb = mx * sl2;
        float alpha = 1.f;
        if (mb - m > kTau) {
          alpha = ex2_approx(m - mb);
          m = mb;
          l *= alpha;
        }
        // pass 2: p = 2^(s*scale*log2e - m), row sum in f32, P to TMEM as bf16
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld_32cols(tS + 32 * c, r);
          tmem_ld_wait(r);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float p0 = ex2_approx(fmaf(__uint_as_float(r[i]), sl2, -m));
            float p1 = ex2_approx(fmaf(__uint_as_float(r[i + 1]), sl2, -m));
            if (need_mask) {
              if (32 * c + i >= lim) p0 = 0.f;
              if (32 * c + i + 1 >= lim) p1 = 0.f;
            }
            l += p0 + p1;
            pk[i >> 1] = pack_bf16x2(p0, p1);
          }
          tmem_st_16cols(tS + 16 * c, pk);
        }
        tmem_st_wait();
        alpha_s[(q * 2 + (sit & 1)) * 128 + row] = alpha;
        if (j == n - 1) {
          row_m[q * 128 + row] = m;
          row_l[q * 128 + row] = l;
        }
        tc_fence_before();
        bar_arrive(&p_full[q]);
        ++sit;
      }
    }
  } else if (warp < C::kCorrWarp0 + 4) {
    // ------------------------------------------------------- correction warpgroup + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t pit[NQ], oit[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) pit[q] = oit[q] = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = unit_index(k);
      if (u >= p.num_units) break;
      const Unit U = decode_unit<NQ>(u, p);
      for (int j = 0; j < U.n_max && ok; ++j) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          if (j >= U.n[q] || !ok) continue;
          ok = warp_all(wait_bar(&p_full[q], pit[q] & 1, ab));
          if (!ok) continue;
          const float alpha = alpha_s[(q * 2 + (pit[q] & 1)) * 128 + row];
          ++pit[q];
          if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            // PV_q(j-1) must have landed before O_q is rescaled
            ok = warp_all(wait_bar(&o_done[q], (oit[q] - 1) & 1, ab));
            if (!ok) continue;
            tc_fence_after();
            const uint32_t tO = tmem + lane_off + C::kOCol + q * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t r[32];
              tmem_ld_32cols(tO + 32 * c, r);
              tmem_ld_wait(r);
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
              tmem_st_32cols(tO + 32 * c, r);
            }
            tmem_st_wait();
          }
          tc_fence_before();
          bar_arrive(&o_corr[q]);
          ++oit[q];
        }
      }
      if (!ok) break;
      // epilogue: O / l to global memory, LSE = (m + log2 l) ln 2
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        if (U.n[q] == 0 || !ok) continue;
        ok = warp_all(wait_bar(&o_done[q], (oit[q] - 1) & 1, ab));
        if (!ok) continue;
        tc_fence_after();
        const float m = row_m[q * 128 + row];
        const float l = row_l[q * 128 + row];
        const float inv = 1.f / l;
        const int row_g = (U.tile0 + q) * 128 + row;
        const bool valid = row_g < p.N;
        const size_t orow = (static_cast<size_t>(U.bh) * p.N + row_g) * D;
        const uint32_t tO = tmem + lane_off + C::kOCol + q * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32cols(tO + 32 * c, r);
          tmem_ld_wait(r);
          if (!valid) continue;
          if (p.o_fp32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                                   __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + orow + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv, __uint_as_float(r[8 * i + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv, __uint_as_float(r[8 * i + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv, __uint_as_float(r[8 * i + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv, __uint_as_float(r[8 * i + 7]) * inv);
              dst[i] = w;
            }
          }
        }
        if (valid && p.lse != nullptr)
          p.lse[static_cast<size_t>(U.bh) * p.N + row_g] = (m + lg2_approx(l)) * kLn2;
      }
    }
  } else if (warp == C::kMmaWarp) {
    // ------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = make_idesc(128, 128, 1u, false);  // S = Q K^T, both K-major
      constexpr uint32_t kIdPV = make_idesc(128, D, 1u, true);    // O += P V, V is MN-major
      const uint32_t q_base = smem_addr(smem + C::kQOff);
      const uint32_t ring_base = smem_addr(smem + C::kRingOff);
      uint32_t it = 0, qit = 0;
      uint32_t cit[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) cit[q] = 0;

      auto issue_s = [&](int q, uint32_t slot) {
        const uint32_t d = tmem + C::kSCol + q * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
          const uint64_t a = make_sdesc_sw128(q_base + q * C::kTileBytes + off, 16, 1024);
          const uint64_t b = make_sdesc_sw128(ring_base + slot * C::kTileBytes + off, 16, 1024);
          mma_f16_ss(d, a, b, kIdS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int q, uint32_t slot, bool acc) {
        const uint32_t d = tmem + C::kOCol + q * D;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = tmem + C::kSCol + q * 128 + kk * 8;  // 16 bf16 of P = 8 columns
          const uint64_t b = make_sdesc_sw128(ring_base + slot * C::kTileBytes + kk * 16 * 128, C::kBoxBytes, 1024);
          mma_f16_ts(d, a, b, kIdPV, (acc || kk > 0) ? 1u : 0u);
        }
      };

      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_index(k);
        if (u >= p.num_units) break;
        const Unit U = decode_unit<NQ>(u, p);
        ok = wait_bar(q_full, qit & 1, ab);
        ++qit;
        if (!ok) break;
        // K_0
        const uint32_t ks0 = it % C::kSlots;
        ok = wait_bar(&full[ks0], (it / C::kSlots) & 1, ab);
        ++it;
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          if (U.n[q] > 0) {
            issue_s(q, ks0);
            tc_commit(&s_full[q]);
          }
        tc_commit(&empty[ks0]);
        if (U.n_max == 1) tc_commit(q_empty);
        for (int j = 0; j < U.n_max; ++j) {
          const uint32_t vs = it % C::kSlots;
          ok = wait_bar(&full[vs], (it / C::kSlots) & 1, ab);
          ++it;
          if (!ok) break;
          tc_fence_after();
          if (j < U.n[0]) {
            ok = wait_bar(&o_corr[0], cit[0] & 1, ab);
            if (!ok) break;
            tc_fence_after();
            issue_pv(0, vs, j > 0);
            tc_commit(&o_done[0]);
            ++cit[0];
          }
          const bool more = j + 1 < U.n_max;
          uint32_t ks = 0;
          if (more) {
            ks = it % C::kSlots;
            ok = wait_bar(&full[ks], (it / C::kSlots) & 1, ab);
            ++it;
            if (!ok) break;
            tc_fence_after();
            if (j + 1 < U.n[0]) {
              issue_s(0, ks);
              tc_commit(&s_full[0]);
            }
          }
          if (NQ == 2 && j < U.n[NQ - 1]) {
            ok = wait_bar(&o_corr[NQ - 1], cit[NQ - 1] & 1, ab);
            if (!ok) break;
            tc_fence_after();
            issue_pv(NQ - 1, vs, j > 0);
            tc_commit(&o_done[NQ - 1]);
            ++cit[NQ - 1];
          }
          tc_commit(&empty[vs]);
          if (more) {
            if (NQ == 2 && j + 1 < U.n[NQ - 1]) {
              issue_s(NQ - 1, ks);
              tc_commit(&s_full[NQ - 1]);
            }
            tc_commit(&empty[ks]);
            if (j + 2 == U.n_max) tc_commit(q_empty);
          }
        }
      }
      // every MMA issued so far must complete before TMEM is released
      tc_commit(drain);
      drain_wait(drain, 0, p.status);
    }
  } else if (warp == C::kLoadWarp) {
    // ------------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0, qit = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_index(k);
        if (u >= p.num_units) break;
        const Unit U = decode_unit<NQ>(u, p);
        if (qit > 0) {
          ok = wait_bar(q_empty, (qit - 1) & 1, ab);
          if (!ok) break;
        }
        bar_arrive_expect_tx(q_full, NQ * C::kTileBytes);
#pragma unroll
        for (int q = 0; q < NQ; ++q)
#pragma unroll
          for (int b = 0; b < C::kBoxes; ++b)
            tma_load_3d(smem + C::kQOff + q * C::kTileBytes + b * C::kBoxBytes, &tmQ, q_full, b * 64,
                        (U.tile0 + q) * 128, U.bh);
        ++qit;
        for (int j = 0; j < U.n_max && ok; ++j) {
#pragma unroll
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t s = it % C::kSlots;
            ok = wait_bar(&empty[s], ((it / C::kSlots) & 1) ^ 1, ab);
            if (!ok) break;
            bar_arrive_expect_tx(&full[s], C::kTileBytes);
            uint8_t* dst = smem + C::kRingOff + s * C::kTileBytes;
#pragma unroll
            for (int b = 0; b < C::kBoxes; ++b)
              tma_load_3d(dst + b * C::kBoxBytes, kv ? &tmV : &tmK, &full[s], b * 64, j * 128, U.bh);
            ++it;
          }
        }
      }
      // let every issued copy land before the CTA can exit
      const uint32_t first = it > (uint32_t)C::kSlots ? it - C::kSlots : 0u;
      for (uint32_t i = first; i < it; ++i) drain_wait(&full[i % C::kSlots], (i / C::kSlots) & 1, p.status);
      if (qit > 0) drain_wait(q_full, (qit - 1) & 1, p.status);
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

template <int D, int NQ>
static cudaError_t set_fwd_smem_attr() {
  return cudaFuncSetAttribute(attn_fwd_bf16_kernel<D, NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              FwdCfg<D, NQ>::kSmemAlloc);
}

cudaError_t setup_fwd_bf16_kernels() {
  cudaError_t e = set_fwd_smem_attr<64, 2>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<128, 2>();
  if (e == cudaSuccess) e = set_fwd_smem_attr<256, 1>();
  return e;
}

template <int D, int NQ>
static cudaError_t launch_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const FwdParams& p,
                              int num_sms, cudaStream_t stream) {
  using C = FwdCfg<D, NQ>;
  const int grid = p.num_units < num_sms ? p.num_units : num_sms;
  attn_fwd_bf16_kernel<D, NQ><<<grid, C::kThreads, C::kSmemAlloc, stream>>>(q, k, v, p);
  return cudaGetLastError();
}

int fwd_units_per_tile_pair(int d) { return d == 256 ? 1 : 2; }

cudaError_t launch_attn_fwd_bf16(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                 const FwdParams& p, int num_sms, cudaStream_t stream) {
  switch (d) {
    case 64:
      return launch_fwd<64, 2>(q, k, v, p, num_sms, stream);
    case 128:
      return launch_fwd<128, 2>(q, k, v, p, num_sms, stream);
    case 256:
      return launch_fwd<256, 1>(q, k, v, p, num_sms, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace ea
