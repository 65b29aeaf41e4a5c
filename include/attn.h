/*
 * exact_attention_100_b200 -- C ABI of the exact attention forward for NVIDIA B200 (sm_100a).
 *
 * What is computed (cited by page title and section):
 *   O = softmax(scale * Q K^T) V per (batch, head)        "FlashAttention-3", intro formula and
 *                                                           section "数学对象没变"
 *   LSE_i = log sum_j exp(scale * q_i . k_j)              "Flash Attention V3 解析", section 2.2
 *                                                           (only the logsumexp is kept per row)
 *   tiled, with a running row max m and row sum l, never   "FlashAttention-2/3", sections
 *   writing the N x N score matrix to memory               "在线 Softmax" and "技术原理"
 *   causal masking with all-masked blocks skipped          "Flash Attention V3 解析", section 2.2
 *   FP8 path: x~ = H D x (random-sign Hadamard) on Q, K    "FlashAttention-3", section
 *   before E4M3 quantisation with per-block scales         "FP8 路径与低精度误差"; "FlashAttention-2/3",
 *                                                           section "FA-3：拥抱 Hopper", features 2-3
 *
 * Conventions shared by every entry point
 *   - Pointers to tensors are DEVICE pointers (cudaMalloc'd or equivalent) on the current CUDA
 *     device, unless an argument says otherwise.  The caller owns every tensor.
 *   - Tensors are contiguous [B, H, N, d] (row-major, d fastest); LSE is contiguous [B, H, N]
 *     float32; per-block scales are contiguous [B, H, ceil(N/128)] float32 -- except where an
 *     entry point states its own layout (the *_strided, *_varlen and merge entry points).
 *   - Every tensor pointer must be 16-byte aligned unless the entry point states otherwise.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously; the call returns once it is enqueued.
 *   - Arguments are checked before any CUDA call; a bad argument returns an error status and
 *     enqueues nothing.  No entry point allocates memory per call.  The library keeps one small
 *     per-device workspace (a device status word), created on first use, and the forward's
 *     per-shape work lists (attn_fwd_schedule), created on the first launch of a shape; both
 *     are released by attn_shutdown().
 *   - Calls on the same device may come from several host threads; the library's per-device
 *     set-up is guarded by a mutex.
 *   - Errors of the device-side work itself (a bounded wait inside a kernel that ran out) are
 *     reported by attn_device_status(), not by the launching call.
 */
#ifndef EXACT_ATTENTION_100_B200_ATTN_H
#define EXACT_ATTENTION_100_B200_ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every int-returning entry point. */
typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* NULL or misaligned pointer, non-positive size, bad scale/flag   */
  ATTN_ERR_UNSUPPORTED = 2, /* head dim / dtype combination not built, or device not sm_100  */
  ATTN_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed (no device, launch error) */
  ATTN_ERR_TIMEOUT = 4      /* a kernel's bounded wait ran out (from attn_device_status)      */
} attn_status;

/* Element types. */
typedef enum {
  ATTN_BF16 = 0, /* bfloat16                       */
  ATTN_FP32 = 1, /* float32                        */
  ATTN_E4M3 = 2  /* OCP FP8 E4M3FN (max 448, no inf) */
} attn_dtype;

/*
 * attn_fwd -- exact attention forward, bf16 inputs.
 *
 *   q, k, v  [B, H, N, d] bf16, device.  K and V have the same length N as Q.
 *   o        [B, H, N, d] of o_dtype (ATTN_BF16 or ATTN_FP32), device, written.
 *   lse      [B, H, N] float32, device, written: natural-log logsumexp of the scaled scores
 *            of each row over its visible keys.  May be NULL (not written).
 *   B, H, N  >= 1;  B*H < 2^31;  N < 2^31.
 *   d        head dimension: 64, 128 or 256.
 *   scale    score scale (softmax(scale * Q K^T)); finite and > 0; usually 1/sqrt(d).
 *   causal   0: every key visible.  1: key j visible to query i iff j <= i (queries and keys
 *            have equal length, so top-left and bottom-right alignment coincide).
 *   dtype    must be ATTN_BF16.
 *   o_dtype  ATTN_BF16 or ATTN_FP32.
 *   stream   cudaStream_t.
 * Arithmetic: bf16 products accumulated in float32 (tensor cores); softmax in float32 with
 * exp2; P rounded to bf16 before the P.V product; the running sum l is summed from the float32
 * values of P.  Returns ATTN_OK once the kernel is enqueued.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int H, int N, int d, float scale, int causal,
             int dtype, int o_dtype, void* stream);

/*
 * attn_fwd_qk -- attn_fwd with a key/value length Nk that may differ from the query length Nq.
 *
 *   q           [B, H, Nq, d] bf16, device.     k, v   [B, H, Nk, d] bf16, device.
 *   o           [B, H, Nq, d] of o_dtype, written.   lse [B, H, Nq] float32 or NULL, written.
 *   Nq, Nk      >= 1.
 *   causal      1: key j is visible to query i iff j <= i + (Nk - Nq) (bottom-right alignment,
 *               the reading taken where the pages are silent); a query row with no visible key
 *               (only when Nq > Nk) gets O = 0 and LSE = -inf.
 * Other arguments, arithmetic and errors as for attn_fwd, which is attn_fwd_qk with
 * Nq = Nk = N.
 */
int attn_fwd_qk(const void* q, const void* k, const void* v, void* o, float* lse,
                int B, int H, int Nq, int Nk, int d, float scale, int causal,
                int dtype, int o_dtype, void* stream);

/*
 * attn_fwd_strided -- attn_fwd_qk on tensors laid out with arbitrary strides, e.g. the
 * [B, N, H, d] (sequence-major) layout of a fused QKV projection, without a transpose copy.
 *
 *   q, k, v, o  logical [B, H, N, d] tensors (N = Nq for q and o, Nk for k and v); element
 *               (b, h, n, c) of tensor t sits at  base_t + b*sb_t + h*sh_t + n*sn_t + c
 *               elements: the head dimension is contiguous.
 *   strides     HOST pointer to 12 int64 values, read during the call and not kept:
 *               {sb, sh, sn} for q, then k, v and o, in elements.  Each stride of a dimension
 *               of extent > 1 must be a positive multiple of 8 below 2^36 (16-byte rows for the
 *               tensor-memory-access unit); the stride of an extent-1 dimension is ignored.
 *               Outputs must not overlap the inputs or one another.
 *   lse         [B, H, Nq] float32, contiguous, or NULL.
 * Other arguments, causal alignment, arithmetic and errors as for attn_fwd_qk, which is
 * attn_fwd_strided with contiguous strides; a bad stride returns ATTN_ERR_INVALID_ARG.
 */
int attn_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int Nq, int Nk, int d, const long long* strides,
                     float scale, int causal, int dtype, int o_dtype, void* stream);

/*
 * attn_fwd_varlen -- attention over a packed batch of B sequences of different lengths, each an
 * independent problem ("FlashAttention-2/3" motivates long and variable contexts; the packing
 * is this library's).
 *
 *   q, o        [total_q, H, d] (bf16; o of o_dtype), device: sequence b owns rows
 *               cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1.
 *   k, v        [total_k, H, d] bf16, device: sequence b owns rows cu_seqlens_k[b] .. [b+1]-1.
 *   lse         [H, total_q] float32 or NULL, written for every row of every sequence.
 *   cu_seqlens_q, cu_seqlens_k   DEVICE int32 arrays of B + 1 non-decreasing offsets with
 *               cu[B] <= total (cu[0] is normally 0); lengths may be 0.
 *   max_seqlen_q  >= every query length cu_seqlens_q[b+1] - cu_seqlens_q[b]; the launch is
 *               sized for it (no device-to-host read of the offsets).
 *   strides     HOST pointer to 8 int64 values {row stride, head stride} for q, k, v and o, in
 *               elements, each a positive multiple of 8 below 2^36 (head stride of H = 1
 *               ignored); the head dimension is contiguous.
 *   causal      per sequence, bottom-right aligned as in attn_fwd_qk (key j visible to query
 *               i iff j <= i + Nk_b - Nq_b); rows with no visible key get O = 0, LSE = -inf.
 * Rows of another sequence that share a 128-row block with this sequence's last keys are read
 * and weighted by exact zeros, so all of k and v must be finite.  Offsets that break the
 * rules above are found on the device: that sequence is skipped (its rows are not written)
 * and the next attn_device_status() returns ATTN_ERR_INVALID_ARG.
 * Other arguments, arithmetic and host-side errors as for attn_fwd.
 */
int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H,
                    int total_q, int total_k, int max_seqlen_q, int d,
                    const long long* strides, float scale, int causal,
                    int dtype, int o_dtype, void* stream);

/*
 * attn_hadamard_quant -- random-sign Hadamard transform plus per-block E4M3 quantisation.
 *
 *   x       [B, H, N, d] bf16, device (read).
 *   x8      [B, H, N, d] E4M3 bytes, device (written).
 *   scales  [B, H, ceil(N/128)] float32, device (written): dequantisation scale per block of
 *           128 rows of one (batch, head), so that x8 * scale approximates the transformed row.
 *   signs   d int8 entries, each +1 or -1, device (read): the diagonal D of the transform.
 *           NULL = no transform (plain per-block quantisation, as for V).
 *   d       64, 128 or 256.
 * Definition: with y = H_d (D x) (unnormalised Sylvester Hadamard, float32 butterflies of
 * stride 1, 2, 4, ...; y = x when signs is NULL), per block s_u = max(max|y| / 448, 2^-126),
 * x8 = E4M3(y * (1/s_u)) rounded to nearest even with saturation, and
 * scale = s_u * (1/sqrt(d)) (or s_u without the transform), all in IEEE float32.  The
 * normalised transform (1/sqrt(d)) H_d D is orthogonal, so scores computed from transformed Q
 * and K are unchanged.  Entries of `signs` other than +-1 are not checked on the device; an
 * entry that is not -1 counts as +1.
 */
int attn_hadamard_quant(const void* x, void* x8, float* scales, const signed char* signs,
                        int B, int H, int N, int d, void* stream);

/*
 * attn_hadamard_quant_qkv -- attn_hadamard_quant of Q and K (with the transform) and of V
 * (without it) in one launch: the pre-processing of the FP8 path in one call.
 *
 *   q, k, v                     [B, H, N, d] bf16, device (read).
 *   q8, k8, v8                  [B, H, N, d] E4M3 bytes, device (written).
 *   q_scale, k_scale, v_scale   [B, H, ceil(N/128)] float32, device (written).
 *   signs                       d int8 entries +-1, device (read); must not be NULL.
 *   d                           64, 128 or 256.
 * Each output is bit-identical to the corresponding attn_hadamard_quant call (signs for Q and
 * K, NULL for V).
 */
int attn_hadamard_quant_qkv(const void* q, const void* k, const void* v, void* q8, void* k8, void* v8,
                            float* q_scale, float* k_scale, float* v_scale, const signed char* signs,
                            int B, int H, int N, int d, void* stream);

/*
 * attn_hadamard_quant_qkv_strided -- attn_hadamard_quant_qkv reading Q, K and V laid out with
 * arbitrary strides (e.g. the head views of one fused [B, N, 3, H, d] projection), without a
 * transpose copy.
 *
 *   q, k, v     logical [B, H, N, d] bf16 tensors, device (read): element (b, h, n, c) of tensor
 *               t at base_t + b*sb_t + h*sh_t + n*sn_t + c elements (d contiguous).
 *   strides     HOST pointer to 9 int64 values, read during the call and not kept: {sb, sh, sn}
 *               for q, then k and v, in elements, with the rules of attn_fwd_strided (positive
 *               multiples of 8 below 2^36; the stride of an extent-1 dimension is ignored).
 *   q8, k8, v8, q_scale, k_scale, v_scale   contiguous outputs as for attn_hadamard_quant_qkv.
 * Each output is bit-identical to attn_hadamard_quant_qkv on contiguous copies of the inputs;
 * a bad stride returns ATTN_ERR_INVALID_ARG.  Other arguments and errors as there.
 */
int attn_hadamard_quant_qkv_strided(const void* q, const void* k, const void* v, void* q8, void* k8,
                                    void* v8, float* q_scale, float* k_scale, float* v_scale,
                                    const signed char* signs, int B, int H, int N, int d,
                                    const long long* strides, void* stream);

/*
 * attn_hadamard_quant_qkv_varlen -- attn_hadamard_quant_qkv for a packed batch of B sequences of
 * different lengths (the layout of attn_fwd_varlen), quantised in 128-row blocks of each
 * sequence, so that no block (and no scale) mixes two sequences.
 *
 *   q           [total_q, H, d] bf16, device (read): sequence b owns rows cu_seqlens_q[b] ..
 *               cu_seqlens_q[b+1]-1.
 *   k, v        [total_k, H, d] bf16, device (read): sequence b owns rows cu_seqlens_k[b] .. [b+1]-1.
 *   strides     HOST pointer to 6 int64 values: {row stride, head stride} for q, k, v, in
 *               elements, with the rules of attn_fwd_varlen (the head dimension is contiguous).
 *   q8          [total_q, H, d] E4M3 bytes, contiguous, device (written for the rows of each sequence).
 *   k8, v8      [total_k, H, d] E4M3 bytes, contiguous, device (written likewise).
 *   q_scale     [B, H, ceil(max_seqlen_q / 128)] float32, device: entry [b, h, j] is the scale
 *               of rows 128j .. 128j+127 of sequence b (entries past a sequence's last block are
 *               not written).
 *   k_scale, v_scale   [B, H, ceil(max_seqlen_k / 128)] float32, device, likewise.
 *   cu_seqlens_q, cu_seqlens_k   DEVICE int32 arrays of B + 1 offsets, as for attn_fwd_varlen.
 *   max_seqlen_q, max_seqlen_k   >= every query / key length: they size the scale arrays.
 *   signs, d    as for attn_hadamard_quant_qkv (Q and K transformed, V not).
 * For each sequence, codes and scales are bit-identical to attn_hadamard_quant_qkv on that
 * sequence alone.  A block's rows past its sequence's end (the next sequence's rows) count as
 * zero for its scale and are not written.  A sequence whose offsets break their rules (or that
 * is longer than its max_seqlen) is skipped and reported by attn_device_status() as
 * ATTN_ERR_INVALID_ARG.  Other errors as for attn_hadamard_quant_qkv.
 */
int attn_hadamard_quant_qkv_varlen(const void* q, const void* k, const void* v, void* q8, void* k8,
                                   void* v8, float* q_scale, float* k_scale, float* v_scale,
                                   const signed char* signs, const int* cu_seqlens_q,
                                   const int* cu_seqlens_k, int B, int H, int total_q, int total_k,
                                   int max_seqlen_q, int max_seqlen_k, int d, const long long* strides,
                                   void* stream);

/*
 * attn_rope_hadamard_quant_qkv -- attn_hadamard_quant_qkv with the rotary position embedding of
 * Q and K fused in front of the transform ("FlashAttention-3", section "为什么 Hadamard 适合放到
 * 内核里": the transform fuses with RoPE, another bandwidth-bound step; the pages do not define
 * RoPE, the rotate-half form below is this library's reading).
 *
 *   cos, sin    [d/2, n_pos] float32, device, 16-byte aligned (read), frequency-major (each
 *               frequency's positions contiguous): row n of every sequence rotates
 *               coordinates i and i + d/2 by the angle these tables hold at [i, n]:
 *                 y_i       = x_i       * cos[i,n] - x_{i+d/2} * sin[i,n]
 *                 y_{i+d/2} = x_{i+d/2} * cos[i,n] + x_i       * sin[i,n]
 *               in float32, each product and the sum rounded (no fused multiply-add).
 *   n_pos       positions in the tables (their row length), >= N.
 * Q and K are rotated, then transformed (H D) and quantised; V is quantised as it is.  Other
 * arguments, outputs and errors as for attn_hadamard_quant_qkv.
 */
int attn_rope_hadamard_quant_qkv(const void* q, const void* k, const void* v, void* q8, void* k8, void* v8,
                                 float* q_scale, float* k_scale, float* v_scale, const signed char* signs,
                                 const float* cos, const float* sin, int n_pos,
                                 int B, int H, int N, int d, void* stream);

/*
 * attn_fwd_fp8 -- exact-attention forward on per-block E4M3 inputs (approximate: the inputs
 * and P carry E4M3 rounding).
 *
 *   q8, k8, v8     [B, H, N, d] E4M3 bytes, device (from attn_hadamard_quant; Q and K with the
 *                  same sign vector, V usually without the transform).
 *   q_scale, k_scale, v_scale   [B, H, ceil(N/128)] float32 block scales, device.
 *   o              [B, H, N, d] of o_dtype (ATTN_BF16 or ATTN_FP32), device, written.
 *   lse            [B, H, N] float32 or NULL, as for attn_fwd.
 *   d              64, 128 or 256 (at d = 64 the E4M3 rows are 64 bytes: 64-byte TMA boxes
 *                  and swizzle).
 *   scale, causal, stream   as for attn_fwd.
 * Arithmetic: E4M3 products accumulated in float32; the Q/K block scales are folded into the
 * softmax scale of each tile pair; P is scaled by 2^(8-tau) * s_v(block) / max_block s_v (tau = 6,
 * the lazy-rescale threshold in base 2, so the scaled P stays <= 256 < 448) and
 * rounded to E4M3 before the P.V product; O is divided by l and rescaled at the end.
 */
int attn_fwd_fp8(const void* q8, const void* k8, const void* v8,
                 const float* q_scale, const float* k_scale, const float* v_scale,
                 void* o, float* lse, int B, int H, int N, int d, float scale, int causal,
                 int o_dtype, void* stream);

/*
 * attn_fwd_fp8_qk -- attn_fwd_fp8 with a key/value length Nk that may differ from the query
 * length Nq: q8 [B, H, Nq, d] with q_scale [B, H, ceil(Nq/128)], k8 and v8 [B, H, Nk, d] with
 * k_scale, v_scale [B, H, ceil(Nk/128)] (from attn_hadamard_quant on each tensor).  Causal
 * masking bottom-right aligned and rows with no visible key as in attn_fwd_qk; other
 * arguments, arithmetic and errors as for attn_fwd_fp8, which is attn_fwd_fp8_qk with
 * Nq = Nk = N.
 */
int attn_fwd_fp8_qk(const void* q8, const void* k8, const void* v8,
                    const float* q_scale, const float* k_scale, const float* v_scale,
                    void* o, float* lse, int B, int H, int Nq, int Nk, int d, float scale,
                    int causal, int o_dtype, void* stream);

/*
 * attn_fwd_fp8_strided -- attn_fwd_fp8_qk on E4M3 inputs and an output laid out with arbitrary
 * strides (e.g. O written straight into a sequence-major [B, Nq, H, d] buffer).
 *
 *   q8, k8, v8, o   logical [B, H, N, d] tensors (N = Nq for q8 and o, Nk for k8 and v8):
 *                   element (b, h, n, c) at base + b*sb + h*sh + n*sn + c elements.
 *   strides     HOST pointer to 12 int64 values, read during the call and not kept: {sb, sh, sn}
 *               for q8, k8, v8 and o, in elements, below 2^36; those of q8, k8, v8 positive
 *               multiples of 16, those of o positive multiples of 8 (16-byte rows for the
 *               tensor-memory-access unit); the stride of an extent-1 dimension is ignored.
 *               o must not overlap the inputs.
 *   q_scale, k_scale, v_scale, lse   contiguous, as for attn_fwd_fp8_qk.
 * Results are bit-identical to attn_fwd_fp8_qk on contiguous copies; a bad stride returns
 * ATTN_ERR_INVALID_ARG.  Other arguments, arithmetic and errors as for attn_fwd_fp8_qk.
 */
int attn_fwd_fp8_strided(const void* q8, const void* k8, const void* v8,
                         const float* q_scale, const float* k_scale, const float* v_scale,
                         void* o, float* lse, int B, int H, int Nq, int Nk, int d,
                         const long long* strides, float scale, int causal, int o_dtype, void* stream);

/*
 * attn_fwd_schedule -- the work lists the persistent forward kernels follow for a fixed-length
 * launch (introspection: every forward entry point builds them itself).  Host only: no CUDA
 * call is made.
 *
 * A unit is one (batch*head, group of Q tiles): unit u covers bh = u % (B*H) and the Q tiles
 * [t0, t0 + T) with T = 2 (d = 64, 128) or 1 (d = 256), r = u / (B*H), and t0 = T * r, or
 * T * (n_pairs - 1 - r) when causal (n_pairs = ceil(ceil(Nq / 128) / T)).  The units are
 * ordered longest first within groups of heads (the K and V of a group fit a 32 MB share of the
 * 126 MB L2, unless that leaves fewer than two units per CTA in a group) and dealt by greedy list
 * scheduling under a cost of K/V blocks per unit ("FlashAttention-2/3", FA-2 improvement 3:
 * parallelism over the sequence; longest first balances causal units of unequal length).
 *
 *   B, H, Nq, Nk, d, causal   the launch, as for attn_fwd_qk.
 *   dtype       ATTN_BF16 (attn_fwd*) or ATTN_E4M3 (attn_fwd_fp8*: K/V elements of one byte).
 *   num_ctas    the persistent grid: the device's SM count (fewer if there are fewer units).
 *   out, cap    host int32 array of cap entries, written if cap >= *needed: [num_ctas + 1]
 *               list offsets, then the unit ids; CTA b computes out[num_ctas + 1 + i] for i in
 *               [out[b], out[b + 1]), in that order.
 *   needed      host: entries of the table, or 0 if the launch keeps the kernels' round-robin
 *               order (more than 2^20 units; packed batches always do).
 * Returns ATTN_OK, ATTN_ERR_INVALID_ARG or ATTN_ERR_UNSUPPORTED as the forward call would.
 * The tables are built on the first launch of a shape (one allocation and one synchronous copy)
 * and kept until attn_shutdown; a launch inside a stream capture of a shape not seen before,
 * and attn_fwd_noalloc, use the round-robin order, with identical results.
 */
int attn_fwd_schedule(int B, int H, int Nq, int Nk, int d, int causal, int dtype, int num_ctas,
                      int* out, long long cap, long long* needed);

/*
 * attn_fwd_fp8_varlen -- attn_fwd_fp8 over a packed batch of B sequences of different lengths,
 * each an independent problem, on the outputs of attn_hadamard_quant_qkv_varlen.
 *
 *   q8          [total_q, H, d] E4M3 bytes, contiguous, device; sequence b owns rows
 *               cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1.
 *   k8, v8      [total_k, H, d] E4M3 bytes, contiguous, device; rows cu_seqlens_k[b] .. [b+1]-1.
 *   q_scale     [B, H, ceil(max_seqlen_q / 128)] float32 per-sequence block scales, device.
 *   k_scale, v_scale   [B, H, ceil(max_seqlen_k / 128)] float32, device.
 *   o           [total_q, H, d] of o_dtype, contiguous, device, written for every row of every
 *               sequence.
 *   lse         [H, total_q] float32 or NULL.
 *   cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k   as for attn_hadamard_quant_qkv_varlen
 *               (the same values: they index the scales).
 *   d           64, 128 or 256.
 * Per sequence: bit-identical to attn_fwd_fp8_qk on that sequence's codes and scales alone
 * (causal alignment, rows with no visible key, arithmetic).  Offsets that break the rules of
 * attn_fwd_varlen, or a key sequence longer than max_seqlen_k, skip that sequence and are
 * reported by attn_device_status() as ATTN_ERR_INVALID_ARG.  Errors otherwise as attn_fwd_fp8.
 */
int attn_fwd_fp8_varlen(const void* q8, const void* k8, const void* v8,
                        const float* q_scale, const float* k_scale, const float* v_scale,
                        void* o, float* lse, const int* cu_seqlens_q, const int* cu_seqlens_k,
                        int B, int H, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                        int d, float scale, int causal, int o_dtype, void* stream);

/*
 * attn_bwd_workspace_bytes -- size of the float32 workspace attn_bwd needs:
 * 2 * B * H * ceil(N / 128) * 128 * 4 bytes (per row, padded to whole 128-row blocks: the
 * rowsum D of dO * O and LSE * log2 e).  Returns 0 if a size is not positive.
 */
unsigned long long attn_bwd_workspace_bytes(int B, int H, int N);

/*
 * attn_bwd -- backward pass of attn_fwd, bf16.  "FlashAttention-3" (section on scope and
 * limits) has the backward for FP16/BF16; "Flash Attention V3 解析" (section 2.1) recomputes
 * the softmax in it instead of storing P.  With S = scale Q K^T and P = exp(S - LSE):
 *     dV = P^T dO,  dP = dO V^T,  dS = P (dP - D) with D_i = sum_c dO_ic O_ic,
 *     dQ = scale dS K,  dK = scale dS^T Q.
 *
 *   q, k, v     [B, H, N, d] bf16, device: the forward's inputs.
 *   o           [B, H, N, d] bf16, device: the forward's output (attn_fwd with o_dtype bf16).
 *   dout        [B, H, N, d] bf16, device: gradient of the loss with respect to O.
 *   lse         [B, H, N] float32, device: the forward's LSE.
 *   dq, dk, dv  [B, H, N, d] of g_dtype (ATTN_BF16 or ATTN_FP32), device, written.
 *   workspace   device, 16-byte aligned, attn_bwd_workspace_bytes(B, H, N) bytes; owned by the
 *               caller and overwritten.
 *   d           64 or 128 (256: ATTN_ERR_UNSUPPORTED, dK and dV alone would fill TMEM).
 *   scale, causal, stream   as for attn_fwd; the same values as the forward call.
 * Arithmetic: S and dP recomputed by tensor cores (bf16 products, float32 accumulation); P and
 * dS in float32, rounded to bf16 before the three accumulating products (float32 accumulation).
 * No atomics: the result does not depend on scheduling.  Three kernel launches.  Returns
 * ATTN_OK once they are enqueued.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, void* workspace,
             int B, int H, int N, int d, float scale, int causal, int g_dtype, void* stream);

/*
 * attn_bwd_qk -- attn_bwd for attn_fwd_qk: queries (q, o, dout, lse, dq) of length Nq, keys and
 * values (k, v, dk, dv) of length Nk; causal masking bottom-right aligned as in attn_fwd_qk.
 * Keys that no query sees get dK = dV = 0; queries that see no key get dQ = 0.  The workspace
 * is attn_bwd_workspace_bytes(B, H, Nq) bytes.  attn_bwd is attn_bwd_qk with Nq = Nk = N.
 */
int attn_bwd_qk(const void* q, const void* k, const void* v, const void* o, const void* dout,
                const float* lse, void* dq, void* dk, void* dv, void* workspace,
                int B, int H, int Nq, int Nk, int d, float scale, int causal, int g_dtype,
                void* stream);

/*
 * attn_bwd_ds_workspace_bytes -- size of the workspace attn_bwd_ds needs: the float32 rows of
 * attn_bwd_workspace_bytes (rounded up to 1024 bytes), then one bf16 128 x 128 tile of dS per
 * (batch, head, query block, visible key block): B * H * n (n + 1) / 2 tiles causal, B * H * n^2
 * otherwise, n = ceil(N / 128), 32 KB each (2.2 GB at B=2 H=16 N=8192 causal).  Returns 0 if a
 * size is not positive or there are 2^31 - 1 tiles or more.
 */
unsigned long long attn_bwd_ds_workspace_bytes(int B, int H, int N, int causal);

/*
 * attn_bwd_ds -- attn_bwd that keeps dS instead of recomputing it: the dK/dV kernel writes each
 * bf16 dS tile (the one its dK product uses) into the workspace, and a third kernel streams them
 * with the K tiles through the tensor cores, dQ = scale dS K ("Flash Attention V3 解析", section
 * 4.2: dQ accumulates over the key blocks; here in a fixed order, without atomics).  Five
 * products instead of attn_bwd's seven, for O(N^2) workspace.
 *
 *   workspace   device, 16-byte aligned, attn_bwd_ds_workspace_bytes(B, H, N, causal) bytes;
 *               owned by the caller and overwritten.
 *   Other arguments as for attn_bwd (d 64 or 128, equal query and key lengths, contiguous).
 * dK and dV are bit-identical to attn_bwd's; dQ agrees with it within the rounding of the two
 * ways of forming dS (the bounds of attn_bwd hold for both).  Deterministic.  Returns
 * ATTN_ERR_INVALID_ARG also when attn_bwd_ds_workspace_bytes would return 0.
 */
int attn_bwd_ds(const void* q, const void* k, const void* v, const void* o, const void* dout,
                const float* lse, void* dq, void* dk, void* dv, void* workspace,
                int B, int H, int N, int d, float scale, int causal, int g_dtype, void* stream);

/*
 * attn_bwd_strided -- attn_bwd_qk on tensors laid out with arbitrary strides (the backward of
 * attn_fwd_strided).
 *
 *   q, k, v, o, dout, dq, dk, dv   logical [B, H, N, d] tensors (N = Nq for q, o, dout, dq;
 *               Nk for k, v, dk, dv); element (b, h, n, c) at base + b*sb + h*sh + n*sn + c.
 *   strides     HOST pointer to 24 int64 values: {sb, sh, sn} for q, k, v, o, dout, dq, dk, dv in
 *               that order, in elements, with the rules of attn_fwd_strided.  The gradients
 *               must not overlap the inputs or one another.
 *   lse         [B, H, Nq] float32, contiguous (as attn_fwd_strided writes it).
 * Other arguments, arithmetic and errors as for attn_bwd_qk, which is attn_bwd_strided with
 * contiguous strides.
 */
int attn_bwd_strided(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, void* workspace,
                     int B, int H, int Nq, int Nk, int d, const long long* strides,
                     float scale, int causal, int g_dtype, void* stream);

/*
 * attn_bwd_varlen -- the backward of attn_fwd_varlen: a packed batch of B sequences.
 *
 *   q, o, dout, dq   [total_q, H, d]; k, v, dk, dv [total_k, H, d] (bf16 inputs; gradients of
 *               g_dtype), device; sequence b owns query rows cu_seqlens_q[b] .. [b+1]-1 and key
 *               rows cu_seqlens_k[b] .. [b+1]-1.
 *   lse         [H, total_q] float32 from attn_fwd_varlen.
 *   cu_seqlens_q, cu_seqlens_k   DEVICE int32 arrays of B + 1 offsets, as for attn_fwd_varlen.
 *   max_seqlen_q, max_seqlen_k   >= every query / key length; the launches are sized for them.
 *   strides     HOST pointer to 16 int64 values: {row stride, head stride} for q, k, v, o, dout,
 *               dq, dk, dv in that order, in elements, with the rules of attn_fwd_varlen.
 *   workspace   attn_bwd_workspace_bytes(B, H, max_seqlen_q) bytes, device.
 * Per sequence the arithmetic, the zero gradients of unseen keys and key-less queries, and the
 * finiteness requirement on rows read past a sequence's end are those of attn_bwd_qk and
 * attn_fwd_varlen; a sequence whose offsets break the rules is skipped and reported by
 * attn_device_status() as ATTN_ERR_INVALID_ARG.
 */
int attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, void* workspace,
                    const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H,
                    int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                    const long long* strides, float scale, int causal, int g_dtype, void* stream);

/*
 * attn_bwd_varlen_ds_workspace_bytes -- size of the workspace attn_bwd_varlen_ds needs: the
 * float32 rows of attn_bwd_workspace_bytes(B, H, max_seqlen_q) rounded up to 1024 bytes, then
 * B * H * ceil(max_seqlen_q / 128) * ceil(max_seqlen_k / 128) bf16 tiles of 32 KB (a rectangle
 * per sequence and head, whatever the sequences' lengths; only the visible tiles are written).
 * Returns 0 if a size is not positive or there are 2^31 - 1 tiles or more.
 */
unsigned long long attn_bwd_varlen_ds_workspace_bytes(int B, int H, int max_seqlen_q, int max_seqlen_k);

/*
 * attn_bwd_varlen_ds -- attn_bwd_varlen that keeps dS in the workspace and forms dQ from it, as
 * attn_bwd_ds does for fixed lengths (five products instead of seven).
 *   workspace   device, 16-byte aligned, attn_bwd_varlen_ds_workspace_bytes(B, H, max_seqlen_q,
 *               max_seqlen_k) bytes; owned by the caller and overwritten.
 * Other arguments, offsets rules and their reporting as for attn_bwd_varlen.  dK and dV are
 * bit-identical to attn_bwd_varlen's; the bounds of attn_bwd hold for every sequence.
 */
int attn_bwd_varlen_ds(const void* q, const void* k, const void* v, const void* o, const void* dout,
                       const float* lse, void* dq, void* dk, void* dv, void* workspace,
                       const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H,
                       int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                       const long long* strides, float scale, int causal, int g_dtype, void* stream);

/*
 * attn_fwd_noalloc -- attn_fwd for callers that cannot allocate device memory.  The pages have
 * no counterpart; it exists for this library's users.
 *
 * Same arguments, arithmetic and results as attn_fwd.  attn_fwd creates a small per-device
 * workspace with cudaMalloc on its first call; runtimes that own all device memory through
 * their own pool, hosts with a fixed memory budget and latency-critical loops that must never
 * reach cudaMalloc (it can synchronise the device) cannot allow that.  This entry point calls
 * no cudaMalloc, cudaFree or other allocating routine: the kernel's scratch (its device status
 * word, 4 bytes) lives in a static device array of 256 bytes that every GPU loading this
 * library holds until the process exits.  The scratch needed does not depend on B, H, N or d;
 * a call needing more than the array holds would be refused with ATTN_ERR_INVALID_ARG.
 *   - The first call on each device does a one-time set-up (device address of the array,
 *     kernel attributes); make that first call before any stream capture.
 *   - Every call shares the array.  Its status word is sticky: a call ORs into it the failures
 *     of its kernel (a bounded wait that ran out), and only attn_noalloc_status reads and
 *     clears it.  Calls that overlap on the GPU (different streams) race on the word: a
 *     failure is reported to whichever caller reads it first.
 *   - attn_device_status() does not see these calls; attn_noalloc_status() does.
 *   - Calls through this entry point are not counted by attn_num_kernel_launches().
 */
int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int N, int d, float scale, int causal,
                     int dtype, int o_dtype, void* stream);

/*
 * attn_noalloc_status -- synchronises `stream`, returns the status word of attn_fwd_noalloc
 * (the static array on the current device) and clears it; allocates nothing.  The pages have no
 * counterpart.  ATTN_OK if no call since the last read reported a problem; ATTN_ERR_TIMEOUT if
 * a bounded wait inside one ran out (that call's O and LSE are undefined; the context stays
 * usable); ATTN_ERR_CUDA if the copy or the synchronisation failed.  Like attn_fwd_noalloc, its
 * first call on a device does the one-time set-up.
 */
int attn_noalloc_status(void* stream);

/*
 * attn_noalloc_selftest_wait_timeout -- attn_selftest_wait_timeout pointed at the status word
 * of attn_fwd_noalloc: one thread waits on an mbarrier that nothing arrives at, gives up after
 * the bound (2 s) and records a timeout there; the next attn_noalloc_status(stream) returns
 * ATTN_ERR_TIMEOUT.  Allocates nothing.  Returns ATTN_OK once the kernel is enqueued.
 */
int attn_noalloc_selftest_wait_timeout(void* stream);

/*
 * attn_device_status -- synchronises `stream`, returns the current device's status word and
 * clears it.  ATTN_OK if no kernel of this library reported a problem since the last call;
 * ATTN_ERR_TIMEOUT if a bounded wait inside a kernel ran out (that kernel's outputs are then
 * undefined, the CUDA context stays usable); otherwise ATTN_ERR_INVALID_ARG if attn_fwd_varlen
 * found sequence offsets that break their rules; ATTN_ERR_CUDA if synchronising failed.
 */
int attn_device_status(void* stream);

/*
 * attn_merge_partials -- merge of two attention results of the same queries over disjoint key
 * sets, in place: (o_acc, lse_acc) <- the result over the union of their keys.  With
 * l = exp(LSE) the softmax denominator of a part, O = (l_a O_a + l_b O_b) / (l_a + l_b) and
 * LSE = log(l_a + l_b) ("FlashAttention-2/3", section "技术原理": the running rescale applied to
 * two finished parts); the step a sequence-sharded (ring) attention takes after each hop.
 *
 *   o_acc       [rows, d] float32, device, read and written (start from zeros).
 *   lse_acc     [rows] float32, device, read and written (start from -inf: no key yet).
 *   o_part      [rows, d] of part_dtype (ATTN_BF16 or ATTN_FP32), device: O of the new part.
 *   lse_part    [rows] float32, device: its natural-log LSE (-inf: the row sees no key there).
 *   rows        1 .. 2^40; any [B, H, N] of contiguous rows.   d  4 .. 1024, a multiple of 4.
 * Arithmetic: float32, weights exp(LSE - max) so neither exponential overflows.  A row whose
 * two LSEs are -inf keeps O = 0, LSE = -inf.  o_acc and o_part 16-byte aligned; the LSE arrays
 * 4-byte aligned.  Returns ATTN_OK once the kernel is enqueued.
 */
int attn_merge_partials(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                        long long rows, int d, int part_dtype, void* stream);

/*
 * attn_selftest_wait_timeout -- diagnostic of the failure detection every kernel relies on: one
 * thread waits on an mbarrier that nothing arrives at, with the bounded wait the kernels use.
 * After the bound (2 s) the wait gives up and records a timeout; the kernel returns.  The next
 * attn_device_status(stream) returns ATTN_ERR_TIMEOUT, and the CUDA context stays usable.
 * Returns ATTN_OK once the kernel is enqueued.
 */
int attn_selftest_wait_timeout(void* stream);

/* attn_status_string -- static, human-readable name of a status code (never NULL). */
const char* attn_status_string(int status);

/* attn_num_kernel_launches -- number of kernels this library has launched in this process
 * (all devices), for launch accounting in benchmarks. */
unsigned long long attn_num_kernel_launches(void);

/* attn_shutdown -- frees the library's per-device workspaces.  Call with no work of this
 * library pending; later calls re-create what they need. */
void attn_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_100_B200_ATTN_H */
