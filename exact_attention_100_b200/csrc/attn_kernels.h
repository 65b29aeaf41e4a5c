// Internal interface between the C ABI (attn_api.cu) and the kernels.  Not installed.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <vector>

namespace ea {

// Device status word bits (OR-ed into the library's per-device status word).
constexpr int kDevStatusTimeout = 1;
constexpr int kDevStatusBadSeqlens = 2;  // packed-sequence offsets that break their bounds

// Parameters of the attention forward kernels (bf16 and E4M3).
struct FwdParams {
  void* o;          // [BH, N, d] bf16 or f32
  float* lse;       // [BH, N] or nullptr
  int* status;      // device status word
  const float* q_scale;  // E4M3 only: [BH, n_blocks] block scales
  const float* k_scale;
  const float* v_scale;
  int N;            // query length (rows of Q, O, LSE)
  int BH;           // batch * heads
  int n_blocks;     // ceil(N / 128): Q tiles
  int Nk;           // key length (rows of K, V)
  int nbk;          // ceil(Nk / 128): K/V blocks
  int off;          // Nk - N: causal key j is visible to query i iff j <= i + off (bottom-right)
  int H;            // heads (bh = b * H + h)
  long long o_sb;   // element strides of O for batch, head and row (d is contiguous)
  long long o_sh;
  long long o_sn;
  int n_pairs;      // ceil(n_blocks / Q tiles per unit)
  int num_units;    // BH * n_pairs
  float scale_log2; // softmax scale * log2(e)
  int causal;
  int o_fp32;
  // Packed variable-length batches (bf16 only): sequence b holds rows [cu_q[b], cu_q[b+1]) of
  // Q and O and rows [cu_k[b], cu_k[b+1]) of K and V (device arrays of B + 1 entries); N is
  // then the longest query length the launch covers, BH = B * H, and LSE is [H, total_q].
  // cu_q == nullptr for fixed-length batches.
  const int* cu_q;
  const int* cu_k;
  int total_q;
  int total_k;
  // packed batches with B <= 1024 and n_pairs <= 1023: every CTA sorts the sequences by their
  // number of tile pairs and deals out only the units that exist, longest first
  int vl_sched;
  // fixed-length batches: per-CTA work lists from fwd_unit_schedule in device memory, or
  // nullptr for the kernel's round-robin order
  const int* unit_tab;
  // E4M3: blocks per (batch, head) row of k_scale and v_scale (nbk; for packed batches
  // ceil(max_nk / 128)); packed batches: the longest key sequence allowed (longer ones are
  // reported as bad offsets)
  int kv_sstride;
  int max_nk;
};

// CTAs of a persistent forward launch: one per SM, or one per unit if there are fewer.
int fwd_grid(const FwdParams& p, int num_sms);

// Work lists of the forward kernels for the fixed-length launch p on `grid` CTAs, nq Q tiles per
// unit, head dim d, elem_bytes per K/V element: out = [grid + 1 list offsets][num_units unit
// ids]; CTA b computes the units out[grid + 1 + i], i in [out[b], out[b + 1]), in that order.
// Returns false (out untouched) for launches left to the round-robin order (packed batches,
// more than 2^20 units).
bool fwd_unit_schedule(const FwdParams& p, int nq, int d, int elem_bytes, int grid, std::vector<int>* out);

// The table of fwd_unit_schedule in device memory on the current device, built on the first
// launch of a shape and cached until free_unit_tables (nullptr: round-robin order).
const int* fwd_unit_table(const FwdParams& p, int nq, int d, int elem_bytes, int grid, cudaStream_t stream);
void free_unit_tables();

// Q tiles of 128 rows handled together by one unit of the bf16 kernel for head dim d.
int fwd_units_per_tile_pair(int d);

// Sets the kernels' shared-memory attributes on the current device (once per device).
cudaError_t setup_kernels_for_current_device();

// The forward kernels read Q, K and V through 4-D maps (d, rows, heads, batch) with a box of
// 128 bytes x 128 rows x 1 x 1, 128-byte swizzle: any layout with d contiguous and 16-byte-aligned
// strides.  They store O through a 4-D map of the same form over O (bf16 or f32) with a box of
// 64 bytes x 128 rows x 1 x 1 and 64-byte swizzle.
cudaError_t launch_attn_fwd_bf16(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                 const CUtensorMap& o, const FwdParams& p, int num_sms, cudaStream_t stream);

cudaError_t launch_attn_fwd_fp8(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                const CUtensorMap& o, const FwdParams& p, int num_sms, cudaStream_t stream);

// Parameters of the backward kernels (bf16 inputs, d = 64 or 128).
struct BwdParams {
  const float* lse;       // forward LSE [BH, N] (natural log), read by the preparation kernel
  const void* o;          // forward O [BH, N, d] bf16 (preparation kernel)
  const void* dout;       // dO [BH, N, d] bf16 (preparation kernel)
  float* delta;           // workspace [BH, n_pad]: rowsum(dO * O), 0 on padded rows
  float* lse2;            // workspace [BH, n_pad]: LSE * log2 e, +inf on padded rows
  void* dq;               // [BH, N, d] bf16 or f32
  void* dk;
  void* dv;
  int* status;
  int N;                  // query length (rows of Q, O, dO, LSE, dQ)
  int BH;
  int n_blocks;           // ceil(N / 128): query blocks
  int n_pad;              // n_blocks * 128
  int Nk;                 // key length (rows of K, V, dK, dV)
  int nbk;                // ceil(Nk / 128)
  int off;                // Nk - N: causal key j is visible to query i iff j <= i + off
  float scale;
  float scale_log2;       // scale * log2 e
  int causal;
  int g_fp32;             // gradients stored as f32 (else bf16)
  int H;                  // heads (bh = b * H + h)
  // element strides (batch, head, row) of O and dO (read by the preparation kernel) and of the
  // gradients (d contiguous); Q, K, V and dO reach the main kernels through 4-D tensor maps
  long long o_sb, o_sh, o_sn, do_sb, do_sh, do_sn;
  long long dq_sb, dq_sh, dq_sn, dk_sb, dk_sh, dk_sn, dv_sb, dv_sh, dv_sn;
  // packed batches (cu_q == nullptr: fixed lengths): sequence b owns query rows
  // [cu_q[b], cu_q[b+1]) and key rows [cu_k[b], cu_k[b+1]); N and Nk are then the longest
  // lengths the launch covers, LSE is [H, total_q], and the workspace keeps n_pad rows per
  // (sequence, head)
  const int* cu_q;
  const int* cu_k;
  int total_q;
  int total_k;
  // dS mode (ds == nullptr: dQ recomputes S and dP): the dK/dV kernel also writes its bf16 dS^T
  // tiles to ds, [BH][ds_tiles] tiles of 32 KB, tile (i, kb) of query block i and key block kb
  // at i (i + 1) / 2 + kb (causal) or i * n_blocks + kb, each [16 chunks of 8 queries][128 key
  // rows][8 queries], and dQ is formed from them; fixed-length batches, equal lengths
  void* ds;
  long long ds_tiles;
  // packed batches: tiles indexed i * ds_nbk + kb per (sequence, head), ds_tiles = n_blocks *
  // ds_nbk (ds_rect = 1), for any per-sequence lengths
  int ds_rect;
  int ds_nbk;
  // dS mode: per-CTA work lists of the dK/dV kernel and of the dQ pass (bwd_unit_table), or
  // nullptr for the round-robin order
  const int* kv_tab;
  const int* q_tab;
};

// Work lists of the backward's dK/dV kernel (kind 1: units u = kb * BH + bh) or of the dQ pass
// from stored dS (kind 2: units u = r * BH + bh, query block n_blocks - 1 - r causal, else r),
// in the form of fwd_unit_schedule: longest first within groups of heads whose streamed tensors
// (Q and dO, or K) fit 32 MB, dealt by greedy list scheduling; fixed-length batches only.
bool bwd_unit_schedule(const BwdParams& p, int kind, int d, int grid, std::vector<int>* out);
const int* bwd_unit_table(const BwdParams& p, int kind, int d, int grid, cudaStream_t stream);

cudaError_t setup_bwd_kernels();
// D and LSE*log2e into the workspace, then dK/dV and dQ; q/k/v/dout are 4-D maps as for the
// forward (p.cu_q selects the packed-batch kernels).
cudaError_t launch_attn_bwd(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                            const CUtensorMap& dout, const BwdParams& p, int num_sms, cudaStream_t stream);

// The dS mode: D and LSE * log2 e, then dK/dV writing the dS^T tiles, then dQ = scale dS K
// streamed from them (each 32 KB tile stored chunk-major: 16-byte chunks of 8 queries for the
// 128 key rows, chunk after chunk, the tensor core's non-swizzled MN-major operand layout).
cudaError_t launch_attn_bwd_ds(int d, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                               const CUtensorMap& dout, const BwdParams& p, int num_sms, cudaStream_t stream);

// Hadamard + per-block E4M3 quantisation of 1..3 tensors of one shape [B, H, N, d] in one launch:
// tm[t] is a 4-D tiled map (d, rows, heads, batch) over tensor t with its own strides (bf16, box
// 64 x 128 x 1 x 1, 128-byte swizzle); x8[t] its contiguous E4M3 output, scales[t] its
// [BH, ceil(N/128)] block scales, post[t] the factor on the stored scale, transform[t] != 0 to
// apply H_d D (signs: d entries +-1).  rope (NULL: none) marks
// the tensors whose rows are first rotated with the frequency-major [d/2, n_pos] float32 tables
// cos and sin (n_pos >= N).
cudaError_t launch_hadamard_quant(const CUtensorMap* tm, int ntensors, uint8_t* const* x8, float* const* scales,
                                  const float* post, const int* transform, const signed char* signs, int BH, int H,
                                  int N, int d, const int* rope, const float* cos, const float* sin, int n_pos,
                                  int num_sms, int* status, cudaStream_t stream);

// The same for packed batches: tensor t is [total[t], H, d] (tm[t] a 4-D map (d, rows, heads, 1)),
// sequence b owning rows cu[t][b] .. cu[t][b+1]-1 (device offsets), quantised in 128-row blocks
// of each sequence; x8[t] is [total[t], H, d] contiguous, scales[t] [B, H, ceil(max_len[t]/128)].
cudaError_t launch_hadamard_quant_varlen(const CUtensorMap* tm, int ntensors, uint8_t* const* x8, float* const* scales,
                                         const float* post, const int* transform, const signed char* signs, int B,
                                         int H, const int* const* cu, const int* total, const int* max_len, int d,
                                         int num_sms, int* status, cudaStream_t stream);

// Sets the pre-kernel's shared-memory attributes on the current device.
cudaError_t setup_hadamard_quant_kernels();

}  // namespace ea
