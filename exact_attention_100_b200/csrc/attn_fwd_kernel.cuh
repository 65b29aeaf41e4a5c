// Exact attention forward for sm_100a (B200): persistent, warp-specialised, tcgen05 + TMEM.
// One template serves the bf16 forward and the E4M3 forward (Elem = ElemBf16 / ElemE4m3).
//
// What one CTA computes: for a unit (one batch*head and NQ consecutive 128-row Q tiles) the
// tiled recurrence of "FlashAttention-2/3", section "技术原理" (outer loop over Q blocks,
// inner loop over K/V blocks, running row max m and row sum l), in the FA-2 form with the
// normalisation deferred to the end ("FlashAttention-2/3", FA-2 improvement 1), writing O and
// the per-row logsumexp ("Flash Attention V3 解析", section 2.2).  Causal units skip the K/V
// blocks that are entirely masked (same section) and run longest first.
//
// Roles (warp specialisation, "FlashAttention-3", section "异步搬运与异步计算"):
//   warps 0..4*NQ-1   softmax warpgroup q = warp/4: one thread per S row (= TMEM lane)
//   next 4 warps      correction warpgroup: the epilogue of a finished Q tile (O / l into
//                     shared-memory stage buffers, LSE), on events from the MMA thread
//   next warp         MMA issuer (one thread issues every tcgen05.mma)
//   next warp         TMA producer (one thread; Q tiles and a ring of K/V slots)
//   next warp         store warp (one thread): TMA stores of the staged O slices and bulk
//                     copies of the LSE rows ("Flash Attention V3 解析", section 3.2.1: the
//                     asynchronous copy engine moves tiles both ways)
//   remaining warp    idle (the CTA is a whole number of warpgroups)
//
// Overlap ("FlashAttention-3", sections "Ping-pong 调度" and "同一个 warpgroup 内部也能再叠一层";
// "Flash Attention V3 解析", section 3.2.3):
//   NQ = 2: per K/V block j the MMA order is PV0(j), S0(j+1), PV1(j), S1(j+1): the tensor core
//           runs one tile's GEMMs while the other tile's softmax runs.  On a unit's last block
//           S0(0) of the next unit goes in before PV1, so units overlap too.
//   NQ = 1: S is double-buffered in TMEM and S(j+1) is issued before PV(j), so the softmax of
//           block j+1 overlaps P.V of block j.
//
// TMEM (512 columns x 128 lanes of 32 bit): S buffers of 128 columns at [0, 256); P (packed
// bf16 or E4M3) overwrites the first columns of its S buffer; O_q at [256 + D*q, +D).
//
// Lazy rescale: a row's reference max m moves only when a block max exceeds it by more than
// Elem::kTau (base-2 units).  The softmax thread then multiplies l, and its row of O in TMEM,
// by alpha = 2^(m_old - m_new) itself, before it hands P over: the P.V of the previous block,
// the last MMA that wrote O, has completed by then (with two Q tiles it was issued before S of
// this block, and one thread issues every MMA in order; with one tile the thread waits on
// pv_done), and the next P.V waits for this P.  O and l always refer to the same m, so O / l
// is exact, and p <= 2^kTau.
//
// Softmax arithmetic per block: one TMEM load of the whole row, eight independent max chains,
// x = s * c - m with packed f32x2 FMAs, p = 2^x on the special-function unit for most pairs
// and, for a quarter of them, on the FMA pipe (2^x = 2^n * q(x - n) with n = round(x) and q a
// cubic fitted on [-1/2, 1/2], relative error < 1e-4), packed f32x2 row sums.

#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "attn_kernels.h"
#include "sm100_ptx.cuh"

namespace ea {

constexpr float kLn2 = 0.6931471805599453f;

struct ElemBf16 {
  static constexpr int kBytes = 2;
  static constexpr bool kFp8 = false;
  static constexpr uint32_t kFmt = 1;   // bf16 in kind::f16
  static constexpr int kKeysPerMma = 16;  // K of one P.V MMA
  static constexpr float kTau = 8.0f;
  static constexpr int kPCols = 64;     // TMEM columns of a 128-key P row
};

struct ElemE4m3 {
  static constexpr int kBytes = 1;
  static constexpr bool kFp8 = true;
  static constexpr uint32_t kFmt = 0;   // e4m3 in kind::f8f6f4
  static constexpr int kKeysPerMma = 32;
  // p <= 2^6, and P is stored as p * 4 * (s_v(j) / max_j s_v(j)) <= 256 < 448.  A larger P
  // scale keeps smaller p above the E4M3 subnormal floor but forces a lower threshold: 16 with
  // threshold 4 rescaled O on most steps of the outlier workload and was 3.5% slower
  static constexpr float kTau = 6.0f;
  static constexpr float kPScale = 4.0f;
  static constexpr int kPCols = 32;
};

// Schedule of a packed batch in shared memory: at most this many sequences and tile pairs.
constexpr int kVlSchedSeqs = 1024, kVlSchedRounds = 1023;

template <int D, int NQ, class E>
struct FwdCfg {
  // one TMA box: 128 rows x 128 bytes (128-byte swizzle), or x 64 bytes (64-byte swizzle) where
  // a row has only 64 bytes (E4M3, d = 64)
  static constexpr int kBoxRow = D * E::kBytes < 128 ? D * E::kBytes : 128;
  static constexpr int kBoxBytes = 128 * kBoxRow;
  static constexpr int kBoxes = D * E::kBytes / kBoxRow;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;       // 128 rows x D elements
  // K/V ring: as many slots as 192 KB hold besides Q, at most 8 (2 for bf16 d = 256)
  static constexpr int kSlots = (196608 - NQ * kTileBytes) / kTileBytes > 8 ? 8
                                                                            : (196608 - NQ * kTileBytes) / kTileBytes;
  static constexpr int kSBufs = NQ == 1 ? 2 : NQ;             // S buffers in TMEM
  static constexpr int kOCol = 256;
  static constexpr int kTmemCols = 512;
  static constexpr int kCorrWarp0 = 4 * NQ;
  static constexpr int kMmaWarp = 4 * NQ + 4;
  static constexpr int kLoadWarp = 4 * NQ + 5;
  static constexpr int kEpiWarp = 4 * NQ + 6;                 // issues the TMA stores of O and LSE
  static constexpr int kThreads = (4 * NQ + 8) * 32;
  static constexpr int kEvents = 4;                           // correction event ring
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = NQ * kTileBytes;
  // O leaves through two stage buffers of 128 rows x 64 bytes (32 bf16 or 16 f32 columns, the
  // O map's box, 64-byte swizzle) and the LSE of a tile through [2][128] f32
  static constexpr int kStageBytes = 128 * 64;
  static constexpr int kStageOff = kRingOff + kSlots * kTileBytes;
  static constexpr int kLseStageOff = kStageOff + 2 * kStageBytes;
  static constexpr int kBarOff = kLseStageOff + 2 * 128 * 4;
  // full[kSlots], empty[kSlots], q_full, q_empty, s_full[kSBufs], p_full[kSBufs], pv_done[NQ],
  // o_done[NQ], o_free[NQ], ev_full[kEvents], ev_empty[kEvents], drain, st_full[2], st_empty[2]
  static constexpr int kNumBars = 2 * kSlots + 2 + 2 * kSBufs + 3 * NQ + 2 * kEvents + 1 + 4;
  static constexpr int kRowMOff = kBarOff + ((kNumBars * 8 + 15) / 16) * 16;
  static constexpr int kRowLOff = kRowMOff + NQ * 2 * 128 * 4;
  static constexpr int kEventOff = kRowLOff + NQ * 2 * 128 * 4;  // [kEvents][4] int
  static constexpr int kStageInfoOff = kEventOff + kEvents * 16;  // [2][8] int: what a stage holds
  static constexpr int kMiscOff = kStageInfoOff + 2 * 8 * 4;
  // packed batches: sorted sequence keys [kSchedSeqs] and the unit prefix [kSchedRounds + 1]
  static constexpr int kSchedSeqs = kVlSchedSeqs, kSchedRounds = kVlSchedRounds;
  static constexpr int kSchedOff = kMiscOff + 16;
  static constexpr int kSmemBytes = kSchedOff + (kSchedSeqs + kSchedRounds + 1) * 4;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;        // room to align the base to 1024 bytes
  static_assert(kSlots >= 2, "K/V ring");
  static_assert(kStageOff % 1024 == 0, "stage buffers: 64-byte swizzle atoms");
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(kSBufs * 128 <= kOCol && kOCol + NQ * D <= kTmemCols, "TMEM budget");
  // register split (setmaxnreg) for NQ = 2: 2 softmax warpgroups, 1 correction, 1 MMA/TMA
  static constexpr uint32_t kRegSoftmax = 168, kRegCorr = 80, kRegOther = 96;
  static_assert(NQ != 2 || (2 * kRegSoftmax + kRegCorr + kRegOther) * 128 == 65536, "register split");
};

enum : int { kEvEpilogue = 1, kEvEnd = 2 };

// The sequence of one (batch entry, head) pair.  Fixed-length batches take every field from
// the parameters; packed variable-length batches (VL) read the sequence's row range from the
// offset arrays.
struct Seq {
  int h, bc;        // head; batch coordinate of Q, K, V and O (0 for packed sequences)
  int N, Nk;        // query and key lengths
  int nbk;          // ceil(Nk / 128)
  int off;          // Nk - N: key j is visible to query i iff j <= i + off (causal)
  int q0, k0;       // first row of the sequence in Q/O and in K/V (0 unless packed)
  long long lse0;   // LSE index of the sequence's row 0 for this head
  bool bad;         // packed offsets out of order, outside the tensors or too long
};

template <bool VL>
__device__ __forceinline__ Seq seq_of(int bh, const FwdParams& p) {
  Seq s;
  const int b = bh / p.H;
  s.h = bh - b * p.H;
  s.bad = false;
  if constexpr (!VL) {
    s.bc = b;
    s.N = p.N;
    s.Nk = p.Nk;
    s.nbk = p.nbk;
    s.off = p.off;
    s.q0 = s.k0 = 0;
    s.lse0 = static_cast<long long>(bh) * p.N;
  } else {
    int q0 = __ldg(p.cu_q + b), q1 = __ldg(p.cu_q + b + 1);
    int k0 = __ldg(p.cu_k + b), k1 = __ldg(p.cu_k + b + 1);
    // p.N is the longest query length the launch was sized for; a sequence that breaks a
    // bound is treated as empty (nothing read or written for it) and reported
    if (!(0 <= q0 && q0 <= q1 && q1 <= p.total_q && q1 - q0 <= p.N && 0 <= k0 && k0 <= k1 && k1 <= p.total_k &&
          k1 - k0 <= p.max_nk)) {
      s.bad = true;
      q0 = q1 = k0 = k1 = 0;
    }
    s.bc = 0;
    s.N = q1 - q0;
    s.Nk = k1 - k0;
    s.nbk = (s.Nk + 127) / 128;
    s.off = s.Nk - s.N;
    s.q0 = q0;
    s.k0 = k0;
    s.lse0 = static_cast<long long>(s.h) * p.total_q + q0;
  }
  return s;
}

struct Unit {
  int bh;
  int tile0;     // index of the first 128-row Q tile of the unit
  int n[2];      // K/V blocks each Q tile visits (0: no visible key, or past the sequence end)
  int n_max;
  bool present;  // the unit's first tile starts inside its sequence (always, unless packed)
  Seq s;
};

// Unit u of the launch.  Fixed-length batches (and packed ones without the schedule): round
// r = u / BH, (batch, head) = u % BH, tile pair n_pairs - 1 - r when causal (longest units
// first) or r.  Packed batches with the schedule (`sched` = the sorted sequence keys, then the
// unit prefix C[0..n_pairs]): round r holds, for tile pair n_pairs - 1 - r, every sequence that
// has that pair (a prefix of the sorted keys) times every head, so no unit is empty.
template <int NQ, bool VL>
__device__ __forceinline__ Unit decode_unit(int u, const FwdParams& p, const int* sched) {
  Unit U;
  int pair;
  if (VL && sched != nullptr) {
    const int* pre = sched + kVlSchedSeqs;
    int lo = 0, hi = p.n_pairs;  // pre[lo] <= u < pre[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= u) lo = mid;
      else hi = mid;
    }
    const int idx = u - pre[lo];
    const int i = idx / p.H;
    U.bh = (sched[i] & 0xFFFF) * p.H + (idx - i * p.H);
    pair = p.n_pairs - 1 - lo;
  } else {
    const int r = u / p.BH;
    U.bh = u - r * p.BH;
    pair = p.causal ? (p.n_pairs - 1 - r) : r;  // causal: longest units first
  }
  U.s = seq_of<VL>(U.bh, p);
  U.tile0 = pair * NQ;
  U.present = U.tile0 * 128 < U.s.N;
  U.n_max = 0;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int t = U.tile0 + q;
    int n = 0;
    if (q < NQ && t * 128 < U.s.N) {
      if (!p.causal) {
        n = U.s.nbk;
      } else {
        // keys up to the tile's last row + off (bottom-right alignment); 0 if even it sees none
        const int last = min(t * 128 + 127, U.s.N - 1) + U.s.off;
        n = last < 0 ? 0 : min(last / 128 + 1, U.s.nbk);
      }
    }
    U.n[q] = n;
    U.n_max = max(U.n_max, n);
  }
  return U;
}

// k-th unit of this CTA: from the host's work lists (tab: [gridDim.x + 1] offsets, then unit
// ids), or else round-robin over CTAs, alternating direction every round.  Past the end of its
// list a CTA gets a value >= num_units.
__device__ __forceinline__ int unit_index(int k, const int* tab) {
  if (tab != nullptr) {
    const int i = __ldg(tab + blockIdx.x) + k;
    return i < __ldg(tab + blockIdx.x + 1) ? __ldg(tab + gridDim.x + 1 + i) : 0x7FFFFFFF;
  }
  const int g = gridDim.x;
  return k * g + ((k & 1) ? (g - 1 - (int)blockIdx.x) : (int)blockIdx.x);
}

// Bounded wait that ignores the abort flag: used at exit so that this thread's own async
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

// (x0, x1) <- (s0 * c + nm, s1 * c + nm), one packed f32x2 FMA
__device__ __forceinline__ void fma2_bcast(float& x0, float& x1, float s0, float s1, float c, float nm) {
  asm("{\n\t.reg .b64 ra, rc, rm, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rc, {%4, %4};\n\t"
      "mov.b64 rm, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rc, rm;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(x0), "=f"(x1)
      : "f"(s0), "f"(s1), "f"(c), "f"(nm));
}

// (a0, a1) += (b0, b1), one packed f32x2 add
__device__ __forceinline__ void add2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%0, %1};\n\t"
      "mov.b64 rb, {%2, %3};\n\t"
      "add.rn.f32x2 ra, ra, rb;\n\t"
      "mov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// Loads a 128-column row slice of S (this thread's lane) with four loads and one wait.
__device__ __forceinline__ void tmem_ld_row128(uint32_t taddr, uint32_t (&r)[128]) {
  uint32_t(&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
  uint32_t(&b)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
  uint32_t(&c)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[64]);
  uint32_t(&d)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[96]);
  tmem_ld_32cols(taddr, a);
  tmem_ld_32cols(taddr + 32, b);
  tmem_ld_32cols(taddr + 64, c);
  tmem_ld_32cols(taddr + 96, d);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 128; i += 8)
    asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), "+r"(r[i + 5]),
                 "+r"(r[i + 6]), "+r"(r[i + 7]));
}

// Softmax of one 128-key block for this thread's row.  r holds the raw scores; on return the
// packed P of the block is in pk (kPCols words), and the function returns sum_j p_j (not yet
// scaled back for E4M3).  c = softmax scale * log2 e (times the Q/K block scales for E4M3);
// nm = -(reference max) (+ log2 of the P scale for E4M3).
template <class E, bool kMasked>
__device__ __forceinline__ float softmax_block(uint32_t (&r)[128], uint32_t* pk, float c, float nm) {
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  float pv[4];
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    float x0, x1, p0, p1;
    fma2_bcast(x0, x1, __uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), c, nm);
    if (!kMasked && (i & 3) == 3) {
      exp2_fma_pair(p0, p1, x0, x1);
    } else {
      p0 = ex2_approx(x0);
      p1 = ex2_approx(x1);
    }
    add2(acc[2 * (i & 3)], acc[2 * (i & 3) + 1], p0, p1);
    if constexpr (E::kFp8) {
      pv[2 * (i & 1)] = p0;
      pv[2 * (i & 1) + 1] = p1;
      if (i & 1) pk[i >> 1] = pack_e4m3x4(pv[0], pv[1], pv[2], pv[3]);
    } else {
      pk[i] = pack_bf16x2(p0, p1);
    }
  }
  add2(acc[0], acc[1], acc[2], acc[3]);
  add2(acc[4], acc[5], acc[6], acc[7]);
  add2(acc[0], acc[1], acc[4], acc[5]);
  return acc[0] + acc[1];
}

template <int D, int NQ, class E, bool VL>
__global__ void __launch_bounds__(FwdCfg<D, NQ, E>::kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdParams p) {
  using C = FwdCfg<D, NQ, E>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* full = bars;                   // [kSlots] K/V slot loaded
  uint64_t* empty = full + C::kSlots;      // [kSlots] K/V slot released by the MMAs
  uint64_t* q_full = empty + C::kSlots;
  uint64_t* q_empty = q_full + 1;
  uint64_t* s_full = q_empty + 1;          // [kSBufs] S ready in TMEM
  uint64_t* p_full = s_full + C::kSBufs;   // [kSBufs] P ready in TMEM (softmax warps)
  uint64_t* pv_done = p_full + C::kSBufs;  // [NQ] one completion per P.V of the tile (commit, NQ = 1)
  uint64_t* o_done = pv_done + NQ;         // [NQ] the last P.V of a tile finished (commit)
  uint64_t* o_free = o_done + NQ;          // [NQ] epilogue finished reading O (correction warps)
  uint64_t* ev_full = o_free + NQ;         // [kEvents] event posted (MMA thread)
  uint64_t* ev_empty = ev_full + C::kEvents;  // [kEvents] event taken (correction warps)
  uint64_t* drain = ev_empty + C::kEvents;
  uint64_t* st_full = drain + 1;           // [2] stage buffer written (128 correction threads)
  uint64_t* st_empty = st_full + 2;        // [2] stage buffer read by its store (store warp)
  uint8_t* stage = smem + C::kStageOff;                                   // [2][128 rows][64 B]
  float* lse_stage = reinterpret_cast<float*>(smem + C::kLseStageOff);    // [2][128]
  volatile int* stage_info = reinterpret_cast<volatile int*>(smem + C::kStageInfoOff);  // [2][8]
  // [NQ][2][128], slot = parity of the tile's unit count: a tile with a single K/V block writes
  // the next unit's values before the previous epilogue has necessarily read its own
  float* row_m = reinterpret_cast<float*>(smem + C::kRowMOff);     // base-2 LSE
  float* row_l = reinterpret_cast<float*>(smem + C::kRowLOff);     // divisor of O
  volatile int* events = reinterpret_cast<volatile int*>(smem + C::kEventOff);  // [kEvents][4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kSlots; ++i) {
      bar_init(&full[i], 1);
      bar_init(&empty[i], 1);
    }
    bar_init(q_full, 1);
    bar_init(q_empty, 1);
    for (int b = 0; b < C::kSBufs; ++b) {
      bar_init(&s_full[b], 1);
      bar_init(&p_full[b], 4);  // one arrive per softmax warp
    }
    for (int q = 0; q < NQ; ++q) {
      bar_init(&pv_done[q], 1);
      bar_init(&o_done[q], 1);
      bar_init(&o_free[q], 4);
    }
    for (int e = 0; e < C::kEvents; ++e) {
      bar_init(&ev_full[e], 1);
      bar_init(&ev_empty[e], 4);
    }
    bar_init(drain, 1);
    for (int b = 0; b < 2; ++b) {
      bar_init(&st_full[b], 128);
      bar_init(&st_empty[b], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kLoadWarp && lane == 0) {
    prefetch_tensor_map(&tmQ);
    prefetch_tensor_map(&tmK);
    prefetch_tensor_map(&tmV);
  }
  if (warp == C::kEpiWarp && lane == 0) prefetch_tensor_map(&tmO);
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  const int* sched = nullptr;
  int num_units = p.num_units;
  if constexpr (VL) {
    if (p.vl_sched) {
      // every CTA builds the same schedule: sequence keys (n_pairs - pairs) << 16 | b sorted
      // ascending (bitonic sort; unique keys, so the order is the same in every CTA), then the
      // units per round, prefix-summed
      int* key = reinterpret_cast<int*>(smem + C::kSchedOff);
      int* pre = key + C::kSchedSeqs;
      const int B = p.BH / p.H;
      int Bp = 1;
      while (Bp < B) Bp <<= 1;
      for (int i = threadIdx.x; i < Bp; i += C::kThreads) {
        int k = 0x7FFFFFFF;  // padding sorts last
        if (i < B) {
          const Seq s = seq_of<true>(i * p.H, p);
          if (s.bad && blockIdx.x == 0) atomicOr(p.status, kDevStatusBadSeqlens);
          const int pairs = (s.N + 128 * NQ - 1) / (128 * NQ);
          k = ((p.n_pairs - pairs) << 16) | i;
        }
        key[i] = k;
      }
      __syncthreads();
      for (int kk = 2; kk <= Bp; kk <<= 1) {
        for (int j = kk >> 1; j > 0; j >>= 1) {
          for (int i = threadIdx.x; i < Bp; i += C::kThreads) {
            const int ixj = i ^ j;
            if (ixj > i) {
              const int a = key[i], b = key[ixj];
              if ((a > b) == ((i & kk) == 0)) {
                key[i] = b;
                key[ixj] = a;
              }
            }
          }
          __syncthreads();
        }
      }
      // round r has every sequence whose key >> 16 is <= r, i.e. with at least n_pairs - r pairs
      for (int r = threadIdx.x; r < p.n_pairs; r += C::kThreads) {
        int lo = 0, hi = B;  // first index whose key >> 16 exceeds r
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if ((key[mid] >> 16) <= r) lo = mid + 1;
          else hi = mid;
        }
        pre[r + 1] = lo * p.H;
      }
      __syncthreads();
      if (warp == 0) {
        // inclusive scan of pre[1..n_pairs] by one warp: each lane a contiguous chunk
        const int per = (p.n_pairs + 31) / 32;
        const int r0 = 1 + lane * per;
        int sum = 0;
        for (int r = r0; r < r0 + per && r <= p.n_pairs; ++r) sum += pre[r];
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        int run = incl - sum;
        for (int r = r0; r < r0 + per && r <= p.n_pairs; ++r) {
          run += pre[r];
          pre[r] = run;
        }
        if (lane == 0) pre[0] = 0;
      }
      sched = key;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if constexpr (VL) {
    if (sched != nullptr) num_units = sched[C::kSchedSeqs + p.n_pairs];
  }
  const AbortState ab{abort_flag, p.status};
  const int nb = p.n_blocks;

  if (warp < 4 * NQ) {
    // ==================================================================== softmax warpgroups
    if constexpr (NQ == 2) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kRegSoftmax));
    const int q = warp >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t sit = 0;  // S blocks consumed by this warpgroup so far
    uint32_t uit = 0;  // units this warpgroup's tile took part in
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = unit_index(k, p.unit_tab);
      if (u >= num_units) break;
      const Unit U = decode_unit<NQ, VL>(u, p, sched);
      const Seq& S = U.s;
      const int n = U.n[q];
      const int tile_row0 = (U.tile0 + q) * 128;
      const int row_g = tile_row0 + row;
      if (n == 0) {
        // a tile inside the sequence whose rows see no key (causal, more queries than keys, or
        // an empty key sequence): O = 0 and LSE = -inf, written here; no MMA or epilogue event
        // concerns it.  A tile past the sequence end is skipped by every role.
        if (tile_row0 < S.N) {
          if (row_g < S.N) {
            const long long orow = S.bc * p.o_sb + S.h * p.o_sh + static_cast<long long>(S.q0 + row_g) * p.o_sn;
            for (int c = 0; c < D; c += 4) {
              if (p.o_fp32)
                *reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
              else
                *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.o) + orow + c) = make_uint2(0u, 0u);
            }
            if (p.lse != nullptr) p.lse[S.lse0 + row_g] = -INFINITY;
          }
        }
        continue;
      }
      int lim_row = S.Nk;  // keys [0, lim_row) are visible to this row (<= 0: none)
      if (p.causal) lim_row = min(lim_row, row_g + S.off + 1);
      float c_base = p.scale_log2;
      float ps_log2_base = 0.f, l_div = 1.f;
      const float* ks = nullptr;
      const float* vs = nullptr;
      float kj = 1.f, vj = 1.f;
      if constexpr (E::kFp8) {
        // the Q block scale folds into c; P is stored as p * kPScale * s_v(j) / max_j s_v(j)
        c_base *= __ldg(p.q_scale + static_cast<size_t>(U.bh) * nb + U.tile0 + q);
        ks = p.k_scale + static_cast<size_t>(U.bh) * p.kv_sstride;
        vs = p.v_scale + static_cast<size_t>(U.bh) * p.kv_sstride;
        float vmax = 0.f;
        for (int b = lane; b < S.nbk; b += 32) vmax = fmaxf(vmax, __ldg(vs + b));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
        ps_log2_base = lg2_approx(E::kPScale / vmax);
        l_div = E::kPScale / vmax;
        kj = __ldg(ks);
        vj = __ldg(vs);
      }
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        float c = c_base, ps_log2 = 0.f;
        if constexpr (E::kFp8) {
          c *= kj;
          ps_log2 = ps_log2_base + lg2_approx(vj);
          if (j + 1 < n) {  // next block's scales, ahead of their use
            kj = __ldg(ks + j + 1);
            vj = __ldg(vs + j + 1);
          }
        }
        const uint32_t sbuf = (C::kSBufs == NQ) ? static_cast<uint32_t>(q) : (sit & 1u);
        const uint32_t sphase = (C::kSBufs == NQ) ? (sit & 1u) : ((sit >> 1) & 1u);
        ok = warp_all(wait_bar(&s_full[sbuf], sphase, ab));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = lane_base + sbuf * 128;
        uint32_t r[128];
        tmem_ld_row128(tS, r);
        const int key0 = j * 128;
        const bool need_mask = (key0 + 128 > S.Nk) || (p.causal && key0 + 127 > tile_row0 + S.off);
        if (need_mask) {
          const int lim = lim_row - key0;
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= lim) r[i] = __float_as_uint(-INFINITY);
        }
        // row max: eight independent two-input max chains.  (The three-input max.f32 gave
        // wrong partial maxima on masked rows in this kernel on B200 and is not used.)
        float mx[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) mx[t] = __uint_as_float(r[t]);
#pragma unroll
        for (int i = 8; i < 128; i += 8)
#pragma unroll
          for (int t = 0; t < 8; ++t) mx[t] = fmaxf(mx[t], __uint_as_float(r[i + t]));
        const float mb =
            fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * c;
        float alpha = 1.f;
        if (mb > m + E::kTau) {
          alpha = ex2_approx(m - mb);
          m = mb;
          l *= alpha;
        }
        uint32_t pk[E::kPCols];
        float lb;
        if (need_mask) {
          // only a masked block can leave a row without any visible key so far (m = -inf,
          // possible when there are more queries than keys): its p must come out 0, not NaN
          lb = softmax_block<E, true>(r, pk, c, ps_log2 - (m == -INFINITY ? 0.f : m));
        } else {
          lb = softmax_block<E, false>(r, pk, c, ps_log2 - m);
        }
        if constexpr (E::kFp8) lb *= ex2_approx(-ps_log2);
        l += lb;
        tmem_st_32cols(tS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        if constexpr (!E::kFp8) tmem_st_32cols(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        tmem_st_wait();
        if (__any_sync(0xffffffffu, alpha != 1.f) && j > 0) {
          // the reference max moved: O *= alpha for this warp's rows, once the previous block's
          // P.V has landed.  With two Q tiles it has (it was issued before S of this block); with
          // one, S of this block goes in first, so wait for completion number sit of pv_done.
          if constexpr (NQ == 1) {
            ok = warp_all(wait_bar(&pv_done[q], (sit - 1u) & 1u, ab));
            if (!ok) break;
          }
          tc_fence_after();
          const uint32_t tO = lane_base + C::kOCol + q * D;
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld_32cols(tO + 32 * cc, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st_32cols(tO + 32 * cc, o);
          }
          tmem_st_wait();
        }
        if (j == n - 1) {
          row_m[(q * 2 + (uit & 1u)) * 128 + row] = m + lg2_approx(l);
          row_l[(q * 2 + (uit & 1u)) * 128 + row] = l * l_div;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(&p_full[sbuf]);
        ++sit;
      }
      ++uit;
    }
  } else if (warp < C::kCorrWarp0 + 4) {
    // ========================================= correction warpgroup: rescale and epilogue events
    if constexpr (NQ == 2) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegCorr));
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t eit = 0;
    uint32_t stc = 0;  // stage buffers filled so far (buffer stc & 1)
    bool ok = true;
    // waits until stage buffer stc & 1 is free again (its previous store has read it)
    auto stage_acquire = [&]() {
      return warp_all(wait_bar(&st_empty[stc & 1u], ((stc >> 1) & 1u) ^ 1u, ab));
    };
    // hands the stage buffer to the store warp: info = {kind, x, row, head, batch, lse, lse lo, hi}
    auto stage_release = [&](int x, int y, int h, int bc, bool lse, long long lse_idx) {
      volatile int* info = stage_info + (stc & 1u) * 8;
      if (row == 0) {
        info[0] = 1;
        info[1] = x;
        info[2] = y;
        info[3] = h;
        info[4] = bc;
        info[5] = lse ? 1 : 0;
        info[6] = static_cast<int>(lse_idx & 0xFFFFFFFFll);
        info[7] = static_cast<int>(lse_idx >> 32);
      }
      fence_proxy_async_smem();
      bar_arrive(&st_full[stc & 1u]);
      ++stc;
    };
    while (ok) {
      const uint32_t es = eit % C::kEvents;
      ok = warp_all(wait_bar(&ev_full[es], (eit / C::kEvents) & 1u, ab));
      if (!ok) break;
      const int kq = events[es * 4 + 0];
      const uint32_t c = static_cast<uint32_t>(events[es * 4 + 1]);
      const int bh = events[es * 4 + 2];
      const int tile = events[es * 4 + 3];
      __syncwarp();
      if (lane == 0) bar_arrive(&ev_empty[es]);
      ++eit;
      const int kind = kq & 0xff;
      const int q = (kq >> 8) & 0xff;
      const int uslot = kq >> 16;
      if (kind == kEvEnd) {
        // tells the store warp to finish
        if ((ok = stage_acquire())) {
          if (row == 0) stage_info[(stc & 1u) * 8] = 0;
          bar_arrive(&st_full[stc & 1u]);
        }
        break;
      }
      const uint32_t tO = tmem + lane_off + C::kOCol + q * D;
      {
        // epilogue: the MMA thread committed o_done (phase c) after the tile's last P.V
        ok = warp_all(wait_bar(&o_done[q], c & 1u, ab));
        if (!ok) break;
        tc_fence_after();
        const float lse2 = row_m[(q * 2 + uslot) * 128 + row];
        const float ls = row_l[(q * 2 + uslot) * 128 + row];
        const float inv = ls > 0.f ? 1.f / ls : 0.f;  // a row with no visible key: O = 0
        const int row_g = tile * 128 + row;
        const Seq S = seq_of<VL>(bh, p);
        const bool valid = row_g < S.N;
        // A tile leaves through the stage buffers and the TMA store (rows past the tensor's end
        // are clipped by the copy); only the last tile of a packed sequence, whose rows past the
        // sequence's end belong to the next sequence, is written row by row instead.
        const bool staged = !VL || tile * 128 + 128 <= S.N;
        if (staged) {
          const long long lse_first = S.lse0 + tile * 128;
          const bool lse_bulk = p.lse != nullptr && tile * 128 + 128 <= S.N && (lse_first & 3) == 0;
          if (p.lse != nullptr && !lse_bulk && valid) p.lse[S.lse0 + row_g] = lse2 * kLn2;
          const int sw = (row >> 1) & 3;  // 64-byte swizzle: 16-byte chunk c of row r sits at c ^ ((r >> 1) & 3)
#pragma unroll 1
          for (int cc = 0; cc < D / 32 && ok; ++cc) {
            uint32_t r[32];
            tmem_ld_32cols(tO + 32 * cc, r);
            tmem_ld_wait(r);
            if (cc == D / 32 - 1) {
              // O is in registers: the next unit's first P.V may overwrite it in TMEM
              tc_fence_before();
              __syncwarp();
              if (lane == 0) bar_arrive(&o_free[q]);
            }
            if (p.o_fp32) {
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                if (!(ok = stage_acquire())) break;
                uint8_t* dst = stage + (stc & 1u) * C::kStageBytes + row * 64;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  *reinterpret_cast<float4*>(dst + ((i ^ sw) << 4)) =
                      make_float4(__uint_as_float(r[16 * h2 + 4 * i]) * inv, __uint_as_float(r[16 * h2 + 4 * i + 1]) * inv,
                                  __uint_as_float(r[16 * h2 + 4 * i + 2]) * inv,
                                  __uint_as_float(r[16 * h2 + 4 * i + 3]) * inv);
                const bool with_lse = lse_bulk && cc == 0 && h2 == 0;
                if (with_lse) lse_stage[(stc & 1u) * 128 + row] = lse2 * kLn2;
                stage_release(32 * cc + 16 * h2, S.q0 + tile * 128, S.h, S.bc, with_lse, lse_first);
              }
            } else {
              if (!(ok = stage_acquire())) break;
              uint8_t* dst = stage + (stc & 1u) * C::kStageBytes + row * 64;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv, __uint_as_float(r[8 * i + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv, __uint_as_float(r[8 * i + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv, __uint_as_float(r[8 * i + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv, __uint_as_float(r[8 * i + 7]) * inv);
                *reinterpret_cast<uint4*>(dst + ((i ^ sw) << 4)) = w;
              }
              const bool with_lse = lse_bulk && cc == 0;
              if (with_lse) lse_stage[(stc & 1u) * 128 + row] = lse2 * kLn2;
              stage_release(32 * cc, S.q0 + tile * 128, S.h, S.bc, with_lse, lse_first);
            }
          }
          if (!ok) break;
        } else {
          const long long orow = S.bc * p.o_sb + S.h * p.o_sh + static_cast<long long>(S.q0 + row_g) * p.o_sn;
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t r[32];
            tmem_ld_32cols(tO + 32 * cc, r);
            tmem_ld_wait(r);
            if (cc == D / 32 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) bar_arrive(&o_free[q]);
            }
            if (!valid) continue;
            if (p.o_fp32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow + 32 * cc);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                                     __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + orow + 32 * cc);
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
          if (valid && p.lse != nullptr) p.lse[S.lse0 + row_g] = lse2 * kLn2;
        }
      }
    }
  } else {
    if constexpr (NQ == 2) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegOther));
    if (warp == C::kMmaWarp && lane == 0) {
      // ======================================================================= MMA issuer
      constexpr uint32_t kIdS = make_idesc(128, 128, E::kFmt, false);  // S = Q K^T, both K-major
      constexpr uint32_t kIdPV = make_idesc(128, D, E::kFmt, true);    // O += P V, V MN-major
      const uint32_t q_base = smem_addr(smem + C::kQOff);
      const uint32_t ring_base = smem_addr(smem + C::kRingOff);
      uint32_t it = 0, qit = 0, sc = 0, ev = 0;
      // per tile: P.V issued, units (o_free phases), o_done commits
      uint32_t pc[NQ], uc[NQ], od[NQ];
#pragma unroll
      for (int q = 0; q < NQ; ++q) pc[q] = uc[q] = od[q] = 0;

      auto slot_of = [&](uint32_t idx) { return idx % C::kSlots; };
      // TMA-filled shared memory read by the tensor core stays in the async proxy: the wait alone
      // orders it (no tcgen05 fence)
      auto wait_loaded = [&](uint32_t idx) {
        return wait_bar(&full[idx % C::kSlots], (idx / C::kSlots) & 1u, ab);
      };
      // operand descriptors for the tiles' swizzle: 8-row atoms of 8 * kBoxRow bytes
      auto sdesc = [](uint32_t addr, uint32_t lbo) {
        return C::kBoxRow == 128 ? make_sdesc_sw128(addr, lbo, 1024) : make_sdesc_sw64(addr, lbo, 512);
      };
      auto issue_s = [&](int q, uint32_t slot, uint32_t buf) {
        const uint32_t d = tmem + buf * 128;
        constexpr int kStepsPerBox = C::kBoxRow / 32;  // 32-byte K steps inside a row of a box
#pragma unroll
        for (int kk = 0; kk < D * E::kBytes / 32; ++kk) {
          const uint32_t off = (kk / kStepsPerBox) * C::kBoxBytes + (kk % kStepsPerBox) * 32;
          const uint64_t a = sdesc(q_base + q * C::kTileBytes + off, 16);
          const uint64_t b = sdesc(ring_base + slot * C::kTileBytes + off, 16);
          if constexpr (E::kFp8)
            mma_f8_ss(d, a, b, kIdS, kk > 0 ? 1u : 0u);
          else
            mma_f16_ss(d, a, b, kIdS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int q, uint32_t slot, uint32_t buf, bool acc) {
        const uint32_t d = tmem + C::kOCol + q * D;
#pragma unroll
        for (int kk = 0; kk < 128 / E::kKeysPerMma; ++kk) {
          const uint32_t a = tmem + buf * 128 + kk * 8;  // kKeysPerMma keys of P = 8 columns
          const uint64_t b =
              sdesc(ring_base + slot * C::kTileBytes + kk * E::kKeysPerMma * C::kBoxRow, C::kBoxBytes);
          if constexpr (E::kFp8)
            mma_f8_ts(d, a, b, kIdPV, (acc || kk > 0) ? 1u : 0u);
          else
            mma_f16_ts(d, a, b, kIdPV, (acc || kk > 0) ? 1u : 0u);
        }
      };
      auto push_event = [&](int kind, int q, uint32_t c, int bh, int tile, uint32_t uslot) {
        const uint32_t es = ev % C::kEvents;
        if (!wait_bar(&ev_empty[es], ((ev / C::kEvents) & 1u) ^ 1u, ab)) return false;
        events[es * 4 + 0] = kind | (q << 8) | static_cast<int>(uslot << 16);
        events[es * 4 + 1] = static_cast<int>(c);
        events[es * 4 + 2] = bh;
        events[es * 4 + 3] = tile;
        bar_arrive(&ev_full[es]);
        ++ev;
        return true;
      };
      // P.V of tile q for block j: wait for P, keep O safe (epilogue / lazy rescale), issue.
      // n_q: K/V blocks of tile q in this unit; bh and tile0 identify the unit for its epilogue
      auto pv_step = [&](int q, int j, int n_q, int bh, int tile0, uint32_t vslot, uint32_t buf) {
        // P of this block sits in S buffer `buf`; that buffer's p_full completes once per use
        const uint32_t pphase = (C::kSBufs == NQ) ? (pc[q] & 1u) : ((pc[q] >> 1) & 1u);
        if (!wait_bar(&p_full[buf], pphase, ab)) return false;
        if (j == 0) {
          // P.V 0 overwrites O: the previous unit's epilogue of this tile must be done with it
          if (!wait_bar(&o_free[q], (uc[q] & 1u) ^ 1u, ab)) return false;
          ++uc[q];
        }
        tc_fence_after();
        issue_pv(q, vslot, buf, j > 0);
        if constexpr (NQ == 1) tc_commit(&pv_done[q]);  // a lazy rescale of the next block waits for it
        if (j == n_q - 1) {
          // uc[q] was counted at j == 0 of this unit: the softmax wrote slot (uc[q] - 1) & 1
          tc_commit(&o_done[q]);
          if (!push_event(kEvEpilogue, q, od[q]++, bh, tile0 + q, (uc[q] - 1u) & 1u)) return false;
        }
        ++pc[q];
        return true;
      };

      bool ok = true;
      // Two Q tiles: on a unit's last step, once tile 0 has had its last P.V, S0(0) of the next
      // unit goes in before tile 1's last P.V as soon as that unit's Q and K_0 have landed, so
      // that tile 0's softmax of the next unit overlaps the end of this one.  (Its Q was
      // requested when this unit's last S went in; K_0 needs one ring slot.)  The MMA thread
      // polls both events: whichever comes first goes first, so a late load never holds back
      // tile 1's last P.V.  Returns whether S0 was issued.
      bool s0_early = false;
      auto issue_next_s0 = [&](int k) {
        int k2 = k + 1;
        Unit U2;
        for (;; ++k2) {
          const int u2 = unit_index(k2, p.unit_tab);
          if (u2 >= num_units) return false;
          U2 = decode_unit<NQ, VL>(u2, p, sched);
          if constexpr (VL) {
            if (!U2.present) continue;
          }
          break;
        }
        if (U2.n_max == 0 || U2.n[0] == 0) return false;
        // `it` is the next unit's K_0; P1 of this step completes p_full[1] phase pc[1] & 1
        const uint32_t a_q = smem_addr(q_full), a_k = smem_addr(&full[slot_of(it)]), a_p = smem_addr(&p_full[1]);
        const uint32_t ph_q = qit & 1u, ph_k = (it / C::kSlots) & 1u, ph_p = pc[1] & 1u;
        const unsigned long long t0 = global_timer_ns();
        for (uint32_t n = 0;; ++n) {
          if (bar_test_wait(a_q, ph_q) && bar_test_wait(a_k, ph_k)) break;
          if (bar_test_wait(a_p, ph_p)) return false;
          if ((n & 15u) == 15u && (*ab.flag || global_timer_ns() - t0 > kWaitLimitNs)) return false;
        }
        ++qit;
        issue_s(0, slot_of(it), 0);
        tc_commit(&s_full[0]);
        return true;
      };
      for (int k = 0; ok; ++k) {
        const int u = unit_index(k, p.unit_tab);
        if (u >= num_units) break;
        const Unit U = decode_unit<NQ, VL>(u, p, sched);
        if constexpr (VL) {
          if (!U.present) continue;  // past its sequence's end: the producer skips it too
        }
        const uint32_t base = it;  // ring index of K_0; K_j = base + 2j, V_j = base + 2j + 1
        it += 2u * U.n_max;
        if (!s0_early) {  // (an early S0 already waited for this unit's Q and K_0)
          ok = wait_bar(q_full, qit & 1u, ab);
          ++qit;
          if (!ok) break;
        }
        if (U.n_max == 0) {  // no tile of the unit sees a key: nothing to compute, Q is free again
          tc_commit(q_empty);
          continue;
        }
        if (!s0_early && !(ok = wait_loaded(base))) break;
        if constexpr (NQ == 2) {
#pragma unroll
          for (int q = 0; q < NQ; ++q)
            if (U.n[q] > 0 && !(q == 0 && s0_early)) {
              issue_s(q, slot_of(base), q);
              tc_commit(&s_full[q]);
            }
          s0_early = false;
          tc_commit(&empty[slot_of(base)]);
          if (U.n_max == 1) tc_commit(q_empty);
          for (int j = 0; j < U.n_max && ok; ++j) {
            const uint32_t vi = base + 2 * j + 1, ki = base + 2 * j + 2;
            const bool more = j + 1 < U.n_max;
            // both waits come before the wait for P: a completed barrier still costs a round
            // trip, which here overlaps the softmax instead of sitting between P.V and S
            if (!(ok = wait_loaded(vi))) break;
            if (more && !(ok = wait_loaded(ki))) break;
            if (j < U.n[0] && !(ok = pv_step(0, j, U.n[0], U.bh, U.tile0, slot_of(vi), 0))) break;
            if (more) {
              if (j + 1 < U.n[0]) {
                issue_s(0, slot_of(ki), 0);
                tc_commit(&s_full[0]);
              }
            } else if (j < U.n[1]) {
              s0_early = issue_next_s0(k);
            }
            if (j < U.n[1] && !(ok = pv_step(1, j, U.n[1], U.bh, U.tile0, slot_of(vi), 1))) break;
            tc_commit(&empty[slot_of(vi)]);
            if (more) {
              if (j + 1 < U.n[1]) {
                issue_s(1, slot_of(ki), 1);
                tc_commit(&s_full[1]);
              }
              tc_commit(&empty[slot_of(ki)]);
              if (j + 2 == U.n_max) tc_commit(q_empty);
            }
          }
        } else {
          // one Q tile, S double-buffered: S(j+1) goes in before P.V(j)
          issue_s(0, slot_of(base), sc & 1u);
          tc_commit(&s_full[sc & 1u]);
          ++sc;
          tc_commit(&empty[slot_of(base)]);
          if (U.n_max == 1) tc_commit(q_empty);
          for (int j = 0; j < U.n_max && ok; ++j) {
            const uint32_t vi = base + 2 * j + 1, ki = base + 2 * j + 2;
            const uint32_t pbuf = (sc - 1u) & 1u;  // buffer holding P(j)
            if (j + 1 < U.n_max) {
              if (!(ok = wait_loaded(ki))) break;
              issue_s(0, slot_of(ki), sc & 1u);
              tc_commit(&s_full[sc & 1u]);
              ++sc;
              tc_commit(&empty[slot_of(ki)]);
              if (j + 2 == U.n_max) tc_commit(q_empty);
            }
            if (!(ok = wait_loaded(vi))) break;
            if (!(ok = pv_step(0, j, U.n[0], U.bh, U.tile0, slot_of(vi), pbuf))) break;
            tc_commit(&empty[slot_of(vi)]);
          }
        }
      }
      if (ok) push_event(kEvEnd, 0, 0, 0, 0, 0);
      // every MMA issued so far must complete before TMEM is released
      tc_commit(drain);
      drain_wait(drain, 0, p.status);
    } else if (warp == C::kLoadWarp && lane == 0) {
      // ====================================================================== TMA producer
      uint32_t it = 0, qit = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_index(k, p.unit_tab);
        if (u >= num_units) break;
        const Unit U = decode_unit<NQ, VL>(u, p, sched);
        const Seq& S = U.s;
        if constexpr (VL) {
          if (S.bad && U.tile0 == 0) atomicOr(p.status, kDevStatusBadSeqlens);
          if (!U.present) continue;
        }
        if (qit > 0 && !(ok = wait_bar(q_empty, (qit - 1u) & 1u, ab))) break;
        bar_arrive_expect_tx(q_full, NQ * C::kTileBytes);
#pragma unroll
        for (int q = 0; q < NQ; ++q)
#pragma unroll
          for (int b = 0; b < C::kBoxes; ++b)
            tma_load_4d(smem + C::kQOff + q * C::kTileBytes + b * C::kBoxBytes, &tmQ, q_full,
                        b * (C::kBoxRow / E::kBytes), S.q0 + (U.tile0 + q) * 128, S.h, S.bc);
        ++qit;
        for (int j = 0; j < U.n_max && ok; ++j) {
#pragma unroll
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t s = it % C::kSlots;
            if (!(ok = wait_bar(&empty[s], ((it / C::kSlots) & 1u) ^ 1u, ab))) break;
            bar_arrive_expect_tx(&full[s], C::kTileBytes);
            uint8_t* dst = smem + C::kRingOff + s * C::kTileBytes;
#pragma unroll
            for (int b = 0; b < C::kBoxes; ++b)
              tma_load_4d(dst + b * C::kBoxBytes, kv ? &tmV : &tmK, &full[s], b * (C::kBoxRow / E::kBytes),
                          S.k0 + j * 128, S.h, S.bc);
            ++it;
          }
        }
      }
      // let every issued copy land before the CTA can exit
      const uint32_t first = it > static_cast<uint32_t>(C::kSlots) ? it - C::kSlots : 0u;
      for (uint32_t i = first; i < it; ++i) drain_wait(&full[i % C::kSlots], (i / C::kSlots) & 1u, p.status);
      if (qit > 0) drain_wait(q_full, (qit - 1u) & 1u, p.status);
    } else if (warp == C::kEpiWarp && lane == 0) {
      // ======================================================================== store warp
      uint32_t stc = 0;
      while (wait_bar(&st_full[stc & 1u], (stc >> 1) & 1u, ab)) {
        const uint32_t b = stc & 1u;
        const volatile int* info = stage_info + b * 8;
        if (info[0] == 0) break;  // the correction warpgroup has finished
        tma_store_4d(&tmO, stage + b * C::kStageBytes, info[1], info[2], info[3], info[4]);
        if (info[5]) {
          const long long idx = (static_cast<long long>(info[7]) << 32) | static_cast<unsigned int>(info[6]);
          bulk_store_s2g(p.lse + idx, lse_stage + b * 128, 128 * 4);
        }
        bulk_commit_group();
        bulk_wait_read_all();  // the buffer may be refilled once its store has read it
        bar_arrive(&st_empty[b]);
        ++stc;
      }
      bulk_wait_all();  // every store performed before the CTA exits
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

template <int D, int NQ, class E, bool VL = false>
cudaError_t set_fwd_smem_attr() {
  return cudaFuncSetAttribute(attn_fwd_kernel<D, NQ, E, VL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              FwdCfg<D, NQ, E>::kSmemAlloc);
}

template <int D, int NQ, class E, bool VL = false>
cudaError_t launch_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& o,
                       const FwdParams& p, int num_sms, cudaStream_t stream) {
  using C = FwdCfg<D, NQ, E>;
  const int grid = fwd_grid(p, num_sms);
  attn_fwd_kernel<D, NQ, E, VL><<<grid, C::kThreads, C::kSmemAlloc, stream>>>(q, k, v, o, p);
  return cudaGetLastError();
}

}  // namespace ea
