// C ABI of the library (declared in include/attn.h): argument checks, per-device state,
// TMA tensor-map encoding and kernel launches.  Every argument is checked before the first
// CUDA call, so a bad call returns a status without touching the device.

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <vector>

#include "../../include/attn.h"
#include "attn_kernels.h"
#include "attn_merge.h"
#include "attn_selftest.h"

namespace ea {
cudaError_t setup_fwd_bf16_kernels();
cudaError_t setup_fwd_fp8_kernels();
}  // namespace ea

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  int* status = nullptr;  // device status word (library-owned workspace)
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
std::atomic<unsigned long long> g_launches{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device set-up (under the mutex): device properties, the status word, kernel attributes.
int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (major != 10 || minor != 0) return ATTN_ERR_UNSUPPORTED;
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q{};
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return ATTN_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    if (st.status == nullptr) {
      if (cudaMalloc(&st.status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
      if (cudaMemset(st.status, 0, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    }
    if (ea::setup_fwd_bf16_kernels() != cudaSuccess) return ATTN_ERR_CUDA;
    if (ea::setup_fwd_fp8_kernels() != cudaSuccess) return ATTN_ERR_CUDA;
    if (ea::setup_hadamard_quant_kernels() != cudaSuccess) return ATTN_ERR_CUDA;
    if (ea::setup_bwd_kernels() != cudaSuccess) return ATTN_ERR_CUDA;
    st.num_sms = sms;
    st.ready = true;
  }
  *out = &st;
  return ATTN_OK;
}

// 4-D tiled map for the forward kernels: dims (d, rows, heads, batch) with the caller's element
// strides of a row, a head and a batch entry (d contiguous); box = 128 bytes x 128 rows x 1 x 1,
// 128-byte swizzle (64 bytes and 64-byte swizzle where a row has only 64 bytes: E4M3 at d = 64),
// zero fill past the last row.
bool encode_fwd_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, int d, int N, int H,
                    int B, long long sn, long long sh, long long sb) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(sn) * elem_bytes, static_cast<cuuint64_t>(sh) * elem_bytes,
                                 static_cast<cuuint64_t>(sb) * elem_bytes};
  const int box_row = d * elem_bytes < 128 ? d * elem_bytes : 128;
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_row / elem_bytes), 128u, 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return g_encode(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  box_row == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D tiled map over O for the forward's TMA stores: dims (d, rows, heads, batch), the caller's
// element strides, box = 64 bytes x 128 rows x 1 x 1 (32 bf16 or 16 f32 columns), 64-byte swizzle;
// rows past the last one are not written.
bool encode_o_map(CUtensorMap* map, void* base, int o_dtype, int d, int N, int H, int B, long long sn, long long sh,
                  long long sb) {
  const bool f32 = o_dtype == ATTN_FP32;
  const int eb = f32 ? 4 : 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(sn) * eb, static_cast<cuuint64_t>(sh) * eb,
                                 static_cast<cuuint64_t>(sb) * eb};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(64 / eb), 128u, 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return g_encode(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Element strides (batch, head, row) of one [B, H, N, d] tensor; the forward's maps and its O
// stores take any strides that are positive multiples of 16 bytes (8 bf16 elements, 16 E4M3
// codes) below 2^36 elements.  A stride of a dimension of extent 1 is never used to address
// anything and is replaced by that multiple.
struct Strides {
  long long sb, sh, sn;
};

Strides contiguous_strides(int H, int N, int d) {
  const long long sn = d, sh = sn * N;
  return {sh * H, sh, sn};
}

bool canonical_strides(const long long* s, int B, int H, int N, Strides* out, long long align = 8) {
  long long v[3] = {s[0], s[1], s[2]};
  const int ext[3] = {B, H, N};
  for (int i = 0; i < 3; ++i) {
    if (ext[i] == 1) v[i] = align;
    if (v[i] <= 0 || v[i] % align != 0 || v[i] >= (1ll << 36)) return false;
  }
  *out = {v[0], v[1], v[2]};
  return true;
}

// The persistent kernels index their work units with int: B * H * ceil(N / 128) must fit.
bool units_fit(int B, int H, int N) {
  return static_cast<long long>(B) * H * ((static_cast<long long>(N) + 127) / 128) < 0x7FFFFFFFLL;
}

int check_common(int B, int H, int N, float scale, int causal, int o_dtype) {
  if (B <= 0 || H <= 0 || N <= 0) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7FFFFFFFLL) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (o_dtype != ATTN_BF16 && o_dtype != ATTN_FP32) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

void fill_params(ea::FwdParams& p, void* o, float* lse, int* status, int B, int H, int N, int Nk, int q_tiles,
                 float scale, int causal, int o_dtype) {
  p.o = o;
  p.lse = lse;
  p.status = status;
  p.q_scale = p.k_scale = p.v_scale = nullptr;
  p.cu_q = p.cu_k = nullptr;
  p.total_q = p.total_k = 0;
  p.vl_sched = 0;
  p.unit_tab = nullptr;
  p.max_nk = Nk;
  p.N = N;
  p.BH = B * H;
  p.H = H;
  p.o_sn = 0;  // set by the caller
  p.o_sh = 0;
  p.o_sb = 0;
  p.n_blocks = (N + 127) / 128;
  p.Nk = Nk;
  p.nbk = (Nk + 127) / 128;
  p.kv_sstride = p.nbk;
  p.off = Nk - N;
  p.n_pairs = (p.n_blocks + q_tiles - 1) / q_tiles;
  p.num_units = p.BH * p.n_pairs;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.causal = causal;
  p.o_fp32 = o_dtype == ATTN_FP32 ? 1 : 0;
}

}  // namespace

extern "C" {

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK:
      return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG:
      return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED:
      return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_CUDA:
      return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT:
      return "ATTN_ERR_TIMEOUT";
    default:
      return "ATTN_ERR_UNKNOWN";
  }
}

unsigned long long attn_num_kernel_launches(void) { return g_launches.load(); }

int attn_selftest_wait_timeout(void* stream) {
  DeviceState* st = nullptr;
  const int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  if (ea::launch_wait_selftest(st->status, static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return ATTN_OK;
}

int attn_merge_partials(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, long long rows,
                        int d, int part_dtype, void* stream) {
  if (!o_acc || !lse_acc || !o_part || !lse_part) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o_acc) || !aligned16(o_part) || (reinterpret_cast<uintptr_t>(lse_acc) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(lse_part) & 3u) != 0)
    return ATTN_ERR_INVALID_ARG;
  if (rows <= 0 || rows > (1ll << 40) || d < 4 || d > 1024 || (d & 3) != 0) return ATTN_ERR_INVALID_ARG;
  if (part_dtype != ATTN_BF16 && part_dtype != ATTN_FP32) return ATTN_ERR_INVALID_ARG;
  if (ea::launch_merge_partials(o_acc, lse_acc, o_part, lse_part, rows, d, part_dtype == ATTN_FP32 ? 1 : 0,
                                static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return ATTN_OK;
}

}  // extern "C"

namespace {

// attn_fwd, attn_fwd_qk and attn_fwd_strided: queries [B, H, Nq, d], keys and values
// [B, H, Nk, d], output [B, H, Nq, d], each with element strides st[0..3] (q, k, v, o).
int fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk, int d,
             const Strides* st4, float scale, int causal, int dtype, int o_dtype, void* stream) {
  if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return ATTN_ERR_INVALID_ARG;
  int rc = check_common(B, H, Nq, scale, causal, o_dtype);
  if (rc != ATTN_OK) return rc;
  if (Nk <= 0 || !units_fit(B, H, Nq)) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_BF16) return dtype == ATTN_E4M3 || dtype == ATTN_FP32 ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;

  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  const Strides &sq = st4[0], &sk = st4[1], &sv = st4[2], &so = st4[3];
  CUtensorMap mq, mk, mv, mo;
  if (!encode_fwd_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Nq, H, B, sq.sn, sq.sh, sq.sb) ||
      !encode_fwd_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Nk, H, B, sk.sn, sk.sh, sk.sb) ||
      !encode_fwd_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Nk, H, B, sv.sn, sv.sh, sv.sb) ||
      !encode_o_map(&mo, o, o_dtype, d, Nq, H, B, so.sn, so.sh, so.sb))
    return ATTN_ERR_CUDA;
  ea::FwdParams p;
  fill_params(p, o, lse, st->status, B, H, Nq, Nk, ea::fwd_units_per_tile_pair(d), scale, causal, o_dtype);
  p.o_sb = so.sb;
  p.o_sh = so.sh;
  p.o_sn = so.sn;
  p.unit_tab = ea::fwd_unit_table(p, ea::fwd_units_per_tile_pair(d), d, 2, ea::fwd_grid(p, st->num_sms),
                                  static_cast<cudaStream_t>(stream));
  if (ea::launch_attn_fwd_bf16(d, mq, mk, mv, mo, p, st->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
             float scale, int causal, int dtype, int o_dtype, void* stream) {
  const Strides s = contiguous_strides(H, N, d);
  const Strides st4[4] = {s, s, s, s};
  return fwd_bf16(q, k, v, o, lse, B, H, N, N, d, st4, scale, causal, dtype, o_dtype, stream);
}

int attn_fwd_qk(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                int d, float scale, int causal, int dtype, int o_dtype, void* stream) {
  const Strides sq = contiguous_strides(H, Nq, d), sk = contiguous_strides(H, Nk, d);
  const Strides st4[4] = {sq, sk, sk, sq};
  return fwd_bf16(q, k, v, o, lse, B, H, Nq, Nk, d, st4, scale, causal, dtype, o_dtype, stream);
}

int attn_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                     int d, const long long* strides, float scale, int causal, int dtype, int o_dtype,
                     void* stream) {
  if (strides == nullptr || B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0) return ATTN_ERR_INVALID_ARG;
  Strides st4[4];
  for (int t = 0; t < 4; ++t)
    if (!canonical_strides(strides + 3 * t, B, H, t == 1 || t == 2 ? Nk : Nq, &st4[t])) return ATTN_ERR_INVALID_ARG;
  return fwd_bf16(q, k, v, o, lse, B, H, Nq, Nk, d, st4, scale, causal, dtype, o_dtype, stream);
}

int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens_q,
                    const int* cu_seqlens_k, int B, int H, int total_q, int total_k, int max_seqlen_q, int d,
                    const long long* strides, float scale, int causal, int dtype, int o_dtype, void* stream) {
  if (!q || !k || !v || !o || !cu_seqlens_q || !cu_seqlens_k || !strides) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) != 0 || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) != 0)
    return ATTN_ERR_INVALID_ARG;
  int rc = check_common(B, H, max_seqlen_q, scale, causal, o_dtype);
  if (rc != ATTN_OK) return rc;
  // row coordinates (offset + 128 * tile) stay inside int
  constexpr int kMaxRows = 0x7FFFFFFF - (1 << 20);
  if (total_q <= 0 || total_k <= 0 || total_q > kMaxRows || total_k > kMaxRows || max_seqlen_q > kMaxRows)
    return ATTN_ERR_INVALID_ARG;
  if (max_seqlen_q > total_q) max_seqlen_q = total_q;  // no sequence is longer than the tensor
  if (!units_fit(B, H, max_seqlen_q)) return ATTN_ERR_INVALID_ARG;
  Strides st4[4];
  for (int t = 0; t < 4; ++t) {
    const long long s3[3] = {8, strides[2 * t + 1], strides[2 * t]};  // {batch (unused), head, row}
    if (!canonical_strides(s3, 1, H, t == 1 || t == 2 ? total_k : total_q, &st4[t])) return ATTN_ERR_INVALID_ARG;
  }
  if (dtype != ATTN_BF16) return dtype == ATTN_E4M3 || dtype == ATTN_FP32 ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;

  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  const Strides &sq = st4[0], &sk = st4[1], &sv = st4[2], &so = st4[3];
  CUtensorMap mq, mk, mv, mo;
  if (!encode_fwd_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, total_q, H, 1, sq.sn, sq.sh, sq.sb) ||
      !encode_fwd_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, total_k, H, 1, sk.sn, sk.sh, sk.sb) ||
      !encode_fwd_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, total_k, H, 1, sv.sn, sv.sh, sv.sb) ||
      !encode_o_map(&mo, o, o_dtype, d, total_q, H, 1, so.sn, so.sh, so.sb))
    return ATTN_ERR_CUDA;
  ea::FwdParams p;
  // sized for B sequences of max_seqlen_q queries each; shorter ones skip the surplus units
  fill_params(p, o, lse, st->status, B, H, max_seqlen_q, total_k, ea::fwd_units_per_tile_pair(d), scale, causal,
              o_dtype);
  p.o_sb = 0;
  p.o_sh = so.sh;
  p.o_sn = so.sn;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.total_q = total_q;
  p.total_k = total_k;
  // the in-kernel schedule's shared-memory tables hold up to 1024 sequences and 1023 pairs
  p.vl_sched = (B <= 1024 && p.n_pairs <= 1023) ? 1 : 0;
  if (ea::launch_attn_fwd_bf16(d, mq, mk, mv, mo, p, st->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return ATTN_OK;
}

int attn_hadamard_quant(const void* x, void* x8, float* scales, const signed char* signs, int B, int H, int N, int d,
                        void* stream) {
  if (!x || !x8 || !scales) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x8) || !aligned16(scales) || (signs && !aligned16(signs)))
    return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0 || static_cast<long long>(B) * H > 0x7FFFFFFFLL) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  const float post = signs ? static_cast<float>(1.0 / std::sqrt(static_cast<double>(d))) : 1.0f;
  const Strides c = contiguous_strides(H, N, d);
  CUtensorMap mx;
  if (!encode_fwd_map(&mx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, H, B, c.sn, c.sh, c.sb)) return ATTN_ERR_CUDA;
  uint8_t* out = static_cast<uint8_t*>(x8);
  const int transform = signs != nullptr ? 1 : 0;
  if (ea::launch_hadamard_quant(&mx, 1, &out, &scales, &post, &transform, signs, B * H, H, N, d, nullptr, nullptr,
                                nullptr, 0, st->num_sms, st->status,
                               static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return ATTN_OK;
}

}  // extern "C"

namespace {

// attn_hadamard_quant_qkv, attn_hadamard_quant_qkv_strided and attn_rope_hadamard_quant_qkv
// (cos/sin NULL: no rotation; st3 NULL: contiguous inputs, else their element strides).
int hq_qkv(const void* q, const void* k, const void* v, void* q8, void* k8, void* v8, float* q_scale, float* k_scale,
           float* v_scale, const signed char* signs, const float* cos, const float* sin, int n_pos, int B, int H, int N,
           int d, const Strides* st3, void* stream) {
  const void* in[3] = {q, k, v};
  void* out[3] = {q8, k8, v8};
  float* sc[3] = {q_scale, k_scale, v_scale};
  for (int t = 0; t < 3; ++t) {
    if (!in[t] || !out[t] || !sc[t]) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(in[t]) || !aligned16(out[t]) || !aligned16(sc[t])) return ATTN_ERR_INVALID_ARG;
  }
  if (!signs || !aligned16(signs)) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0 || static_cast<long long>(B) * H > 0x7FFFFFFFLL) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  CUtensorMap maps[3];
  const Strides c = contiguous_strides(H, N, d);
  for (int t = 0; t < 3; ++t) {
    const Strides& st = st3 ? st3[t] : c;
    if (!encode_fwd_map(&maps[t], in[t], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, H, B, st.sn, st.sh, st.sb))
      return ATTN_ERR_CUDA;
  }
  const float rsd = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  uint8_t* o8[3] = {static_cast<uint8_t*>(q8), static_cast<uint8_t*>(k8), static_cast<uint8_t*>(v8)};
  const float post[3] = {rsd, rsd, 1.0f};
  const int transform[3] = {1, 1, 0};
  const int rope[3] = {1, 1, 0};  // Q and K rotated, V not
  if (ea::launch_hadamard_quant(maps, 3, o8, sc, post, transform, signs, B * H, H, N, d, cos ? rope : nullptr, cos, sin,
                                n_pos, st->num_sms, st->status, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_hadamard_quant_qkv(const void* q, const void* k, const void* v, void* q8, void* k8, void* v8,
                            float* q_scale, float* k_scale, float* v_scale, const signed char* signs, int B, int H,
                            int N, int d, void* stream) {
  return hq_qkv(q, k, v, q8, k8, v8, q_scale, k_scale, v_scale, signs, nullptr, nullptr, 0, B, H, N, d, nullptr,
                stream);
}

int attn_hadamard_quant_qkv_strided(const void* q, const void* k, const void* v, void* q8, void* k8, void* v8,
                                    float* q_scale, float* k_scale, float* v_scale, const signed char* signs, int B,
                                    int H, int N, int d, const long long* strides, void* stream) {
  if (strides == nullptr || B <= 0 || H <= 0 || N <= 0) return ATTN_ERR_INVALID_ARG;
  Strides st3[3];
  for (int t = 0; t < 3; ++t)
    if (!canonical_strides(strides + 3 * t, B, H, N, &st3[t])) return ATTN_ERR_INVALID_ARG;
  return hq_qkv(q, k, v, q8, k8, v8, q_scale, k_scale, v_scale, signs, nullptr, nullptr, 0, B, H, N, d, st3, stream);
}

int attn_hadamard_quant_qkv_varlen(const void* q, const void* k, const void* v, void* q8, void* k8, void* v8,
                                   float* q_scale, float* k_scale, float* v_scale, const signed char* signs,
                                   const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H, int total_q,
                                   int total_k, int max_seqlen_q, int max_seqlen_k, int d, const long long* strides,
                                   void* stream) {
  const void* in[3] = {q, k, v};
  void* out[3] = {q8, k8, v8};
  float* sc[3] = {q_scale, k_scale, v_scale};
  for (int t = 0; t < 3; ++t) {
    if (!in[t] || !out[t] || !sc[t]) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(in[t]) || !aligned16(out[t]) || !aligned16(sc[t])) return ATTN_ERR_INVALID_ARG;
  }
  if (!signs || !aligned16(signs) || !cu_seqlens_q || !cu_seqlens_k || !strides) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) != 0 || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) != 0)
    return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || static_cast<long long>(B) * H > 0x7FFFFFFFLL) return ATTN_ERR_INVALID_ARG;
  constexpr int kMaxRows = 0x7FFFFFFF - (1 << 20);  // row coordinates (offset + 128 * block) stay inside int
  const int tot[3] = {total_q, total_k, total_k};
  const int mx[3] = {max_seqlen_q, max_seqlen_k, max_seqlen_k};
  long long units = 0;
  Strides st3[3];
  for (int t = 0; t < 3; ++t) {
    if (tot[t] <= 0 || tot[t] > kMaxRows || mx[t] <= 0 || mx[t] > kMaxRows) return ATTN_ERR_INVALID_ARG;
    units += static_cast<long long>(B) * H * ((mx[t] + 127) / 128);
    const long long s3[3] = {8, strides[2 * t + 1], strides[2 * t]};  // {batch (unused), head, row}
    if (!canonical_strides(s3, 1, H, tot[t], &st3[t])) return ATTN_ERR_INVALID_ARG;
  }
  if (units > 0x7FFFFFFFLL - 65536) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  CUtensorMap maps[3];
  for (int t = 0; t < 3; ++t)
    if (!encode_fwd_map(&maps[t], in[t], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, tot[t], H, 1, st3[t].sn, st3[t].sh,
                        st3[t].sb))
      return ATTN_ERR_CUDA;
  const float rsd = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  uint8_t* o8[3] = {static_cast<uint8_t*>(q8), static_cast<uint8_t*>(k8), static_cast<uint8_t*>(v8)};
  const float post[3] = {rsd, rsd, 1.0f};
  const int transform[3] = {1, 1, 0};
  const int* cu[3] = {cu_seqlens_q, cu_seqlens_k, cu_seqlens_k};
  if (ea::launch_hadamard_quant_varlen(maps, 3, o8, sc, post, transform, signs, B, H, cu, tot, mx, d, st->num_sms,
                                       st->status, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return ATTN_OK;
}

int attn_rope_hadamard_quant_qkv(const void* q, const void* k, const void* v, void* q8, void* k8, void* v8,
                                 float* q_scale, float* k_scale, float* v_scale, const signed char* signs,
                                 const float* cos, const float* sin, int n_pos, int B, int H, int N, int d,
                                 void* stream) {
  if (!cos || !sin || !aligned16(cos) || !aligned16(sin) || n_pos < N) return ATTN_ERR_INVALID_ARG;
  return hq_qkv(q, k, v, q8, k8, v8, q_scale, k_scale, v_scale, signs, cos, sin, n_pos, B, H, N, d, nullptr, stream);
}

}  // extern "C"

namespace {

// attn_fwd_fp8, attn_fwd_fp8_qk and attn_fwd_fp8_strided: E4M3 Q [B, H, Nq, d], K and V
// [B, H, Nk, d]; st4 (NULL: contiguous) the element strides of q8, k8, v8 and o.
int fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale, const float* k_scale,
            const float* v_scale, void* o, float* lse, int B, int H, int Nq, int Nk, int d, const Strides* st4,
            float scale, int causal, int o_dtype, void* stream) {
  if (!q8 || !k8 || !v8 || !q_scale || !k_scale || !v_scale || !o) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || (lse && !aligned16(lse)) ||
      !aligned16(q_scale) || !aligned16(k_scale) || !aligned16(v_scale))
    return ATTN_ERR_INVALID_ARG;
  int rc = check_common(B, H, Nq, scale, causal, o_dtype);
  if (rc != ATTN_OK) return rc;
  if (Nk <= 0 || !units_fit(B, H, Nq)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  const Strides cq = contiguous_strides(H, Nq, d), ck = contiguous_strides(H, Nk, d);
  const Strides sq = st4 ? st4[0] : cq, sk = st4 ? st4[1] : ck, sv = st4 ? st4[2] : ck, so = st4 ? st4[3] : cq;
  CUtensorMap mq, mk, mv, mo;
  if (!encode_fwd_map(&mq, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, Nq, H, B, sq.sn, sq.sh, sq.sb) ||
      !encode_fwd_map(&mk, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, Nk, H, B, sk.sn, sk.sh, sk.sb) ||
      !encode_fwd_map(&mv, v8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, Nk, H, B, sv.sn, sv.sh, sv.sb) ||
      !encode_o_map(&mo, o, o_dtype, d, Nq, H, B, so.sn, so.sh, so.sb))
    return ATTN_ERR_CUDA;
  ea::FwdParams p;
  fill_params(p, o, lse, st->status, B, H, Nq, Nk, ea::fwd_units_per_tile_pair(d), scale, causal, o_dtype);
  p.o_sb = so.sb;
  p.o_sh = so.sh;
  p.o_sn = so.sn;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.unit_tab = ea::fwd_unit_table(p, ea::fwd_units_per_tile_pair(d), d, 1, ea::fwd_grid(p, st->num_sms),
                                  static_cast<cudaStream_t>(stream));
  if (ea::launch_attn_fwd_fp8(d, mq, mk, mv, mo, p, st->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale, const float* k_scale,
                 const float* v_scale, void* o, float* lse, int B, int H, int N, int d, float scale, int causal,
                 int o_dtype, void* stream) {
  return fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, H, N, N, d, nullptr, scale, causal, o_dtype,
                 stream);
}

int attn_fwd_fp8_qk(const void* q8, const void* k8, const void* v8, const float* q_scale, const float* k_scale,
                    const float* v_scale, void* o, float* lse, int B, int H, int Nq, int Nk, int d, float scale,
                    int causal, int o_dtype, void* stream) {
  return fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, H, Nq, Nk, d, nullptr, scale, causal, o_dtype,
                 stream);
}

int attn_fwd_fp8_strided(const void* q8, const void* k8, const void* v8, const float* q_scale,
                         const float* k_scale, const float* v_scale, void* o, float* lse, int B, int H, int Nq,
                         int Nk, int d, const long long* strides, float scale, int causal, int o_dtype,
                         void* stream) {
  if (strides == nullptr || B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0) return ATTN_ERR_INVALID_ARG;
  Strides st4[4];
  for (int t = 0; t < 4; ++t)
    if (!canonical_strides(strides + 3 * t, B, H, t == 1 || t == 2 ? Nk : Nq, &st4[t], t < 3 ? 16 : 8))
      return ATTN_ERR_INVALID_ARG;
  return fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, H, Nq, Nk, d, st4, scale, causal, o_dtype,
                 stream);
}

int attn_fwd_fp8_varlen(const void* q8, const void* k8, const void* v8, const float* q_scale, const float* k_scale,
                        const float* v_scale, void* o, float* lse, const int* cu_seqlens_q, const int* cu_seqlens_k,
                        int B, int H, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                        float scale, int causal, int o_dtype, void* stream) {
  if (!q8 || !k8 || !v8 || !q_scale || !k_scale || !v_scale || !o || !cu_seqlens_q || !cu_seqlens_k)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || (lse && !aligned16(lse)) ||
      !aligned16(q_scale) || !aligned16(k_scale) || !aligned16(v_scale) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) != 0 || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) != 0)
    return ATTN_ERR_INVALID_ARG;
  int rc = check_common(B, H, max_seqlen_q, scale, causal, o_dtype);
  if (rc != ATTN_OK) return rc;
  constexpr int kMaxRows = 0x7FFFFFFF - (1 << 20);
  if (total_q <= 0 || total_k <= 0 || total_q > kMaxRows || total_k > kMaxRows || max_seqlen_q > kMaxRows ||
      max_seqlen_k <= 0 || max_seqlen_k > kMaxRows)
    return ATTN_ERR_INVALID_ARG;
  if (!units_fit(B, H, max_seqlen_q)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  // [total, H, d] contiguous: row stride H*d, head stride d
  const long long sn = static_cast<long long>(H) * d;
  CUtensorMap mq, mk, mv, mo;
  if (!encode_fwd_map(&mq, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, total_q, H, 1, sn, d, 16) ||
      !encode_fwd_map(&mk, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, total_k, H, 1, sn, d, 16) ||
      !encode_fwd_map(&mv, v8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, total_k, H, 1, sn, d, 16) ||
      !encode_o_map(&mo, o, o_dtype, d, total_q, H, 1, sn, d, 8))
    return ATTN_ERR_CUDA;
  ea::FwdParams p;
  // sized for B sequences of max_seqlen_q queries each; shorter ones skip the surplus units
  fill_params(p, o, lse, st->status, B, H, max_seqlen_q, total_k, ea::fwd_units_per_tile_pair(d), scale, causal,
              o_dtype);
  p.o_sb = 0;
  p.o_sh = d;
  p.o_sn = sn;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.total_q = total_q;
  p.total_k = total_k;
  p.vl_sched = (B <= 1024 && p.n_pairs <= 1023) ? 1 : 0;
  p.kv_sstride = (max_seqlen_k + 127) / 128;
  p.max_nk = max_seqlen_k;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  if (ea::launch_attn_fwd_fp8(d, mq, mk, mv, mo, p, st->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return ATTN_OK;
}

int attn_fwd_schedule(int B, int H, int Nq, int Nk, int d, int causal, int dtype, int num_ctas, int* out,
                      long long cap, long long* needed) {
  if (needed == nullptr || cap < 0 || (cap > 0 && out == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0 || num_ctas <= 0 || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7FFFFFFFLL || !units_fit(B, H, Nq)) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_BF16 && dtype != ATTN_E4M3) return dtype == ATTN_FP32 ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  const int tiles = ea::fwd_units_per_tile_pair(d);
  ea::FwdParams p;
  fill_params(p, nullptr, nullptr, nullptr, B, H, Nq, Nk, tiles, 1.0f, causal, ATTN_BF16);
  std::vector<int> t;
  *needed = 0;
  if (!ea::fwd_unit_schedule(p, tiles, d, dtype == ATTN_E4M3 ? 1 : 2, ea::fwd_grid(p, num_ctas), &t)) return ATTN_OK;
  *needed = static_cast<long long>(t.size());
  if (static_cast<long long>(t.size()) <= cap)
    for (size_t i = 0; i < t.size(); ++i) out[i] = t[i];
  return ATTN_OK;
}

unsigned long long attn_bwd_workspace_bytes(int B, int H, int N) {
  if (B <= 0 || H <= 0 || N <= 0) return 0ull;
  const unsigned long long n_pad = (static_cast<unsigned long long>(N) + 127ull) / 128ull * 128ull;
  return 2ull * static_cast<unsigned long long>(B) * static_cast<unsigned long long>(H) * n_pad * 4ull;
}

}  // extern "C"

namespace {

// Packed-batch description for the backward (nullptr: fixed-length batch).
struct Packed {
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
};

// attn_bwd, attn_bwd_qk, attn_bwd_strided and attn_bwd_varlen.  st8: element strides of q, k, v,
// o, dout, dq, dk, dv.  Fixed-length batches: Nq, Nk are the lengths; packed ones: the longest.
// Bytes of the dS-mode workspace: D and LSE * log2 e (padded rows), rounded up to 1024, then the
// bf16 dS^T tiles of every (batch, head): n_b (n_b + 1) / 2 causal, n_b^2 otherwise, 32 KB each.
// 0 if a size is not positive or the tiles cannot be indexed with int.
// The same for packed batches: a rectangle of ceil(max_q / 128) x ceil(max_k / 128) tiles per
// (sequence, head).
unsigned long long bwd_varlen_ds_workspace_bytes(int B, int H, int max_q, int max_k) {
  if (B <= 0 || H <= 0 || max_q <= 0 || max_k <= 0) return 0ull;
  const unsigned long long bh = static_cast<unsigned long long>(B) * static_cast<unsigned long long>(H);
  const unsigned long long nb = (static_cast<unsigned long long>(max_q) + 127ull) / 128ull;
  const unsigned long long nbk = (static_cast<unsigned long long>(max_k) + 127ull) / 128ull;
  if (bh * nb * nbk >= 0x7FFFFFFFull) return 0ull;
  const unsigned long long head = (2ull * bh * nb * 128ull * 4ull + 1023ull) / 1024ull * 1024ull;
  return head + bh * nb * nbk * 128ull * 128ull * 2ull;
}

unsigned long long bwd_ds_workspace_bytes(int B, int H, int N, int causal) {
  if (B <= 0 || H <= 0 || N <= 0 || (causal != 0 && causal != 1)) return 0ull;
  const unsigned long long bh = static_cast<unsigned long long>(B) * static_cast<unsigned long long>(H);
  const unsigned long long nb = (static_cast<unsigned long long>(N) + 127ull) / 128ull;
  const unsigned long long tiles = causal ? nb * (nb + 1ull) / 2ull : nb * nb;
  if (bh * tiles >= 0x7FFFFFFFull) return 0ull;
  const unsigned long long head = (2ull * bh * nb * 128ull * 4ull + 1023ull) / 1024ull * 1024ull;
  return head + bh * tiles * 128ull * 128ull * 2ull;
}

int bwd_bf16(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
             void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk, int d, const Strides* st8,
             const Packed* pk, float scale, int causal, int g_dtype, void* stream, bool ds_mode = false) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return ATTN_ERR_INVALID_ARG;
  int rc = check_common(B, H, Nq, scale, causal, g_dtype);
  if (rc != ATTN_OK) return rc;
  if (Nk <= 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  const long long n_blocks = (static_cast<long long>(Nq) + 127) / 128;
  const long long nbk = (static_cast<long long>(Nk) + 127) / 128;
  if (static_cast<long long>(B) * H * n_blocks > 0x7FFFFFFFLL || static_cast<long long>(B) * H * nbk > 0x7FFFFFFFLL ||
      n_blocks * 128 > 0x7FFFFFFFLL)
    return ATTN_ERR_INVALID_ARG;

  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  const int rows_q = pk ? pk->total_q : Nq, rows_k = pk ? pk->total_k : Nk, nbat = pk ? 1 : B;
  const Strides &sq = st8[0], &sk = st8[1], &sv = st8[2], &so = st8[3], &sdo = st8[4];
  CUtensorMap mq, mk, mv, mdo;
  if (!encode_fwd_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, rows_q, H, nbat, sq.sn, sq.sh, sq.sb) ||
      !encode_fwd_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, rows_k, H, nbat, sk.sn, sk.sh, sk.sb) ||
      !encode_fwd_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, rows_k, H, nbat, sv.sn, sv.sh, sv.sb) ||
      !encode_fwd_map(&mdo, dout, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, rows_q, H, nbat, sdo.sn, sdo.sh, sdo.sb))
    return ATTN_ERR_CUDA;
  ea::BwdParams p;
  p.lse = lse;
  p.o = o;
  p.dout = dout;
  p.BH = B * H;
  p.H = H;
  p.N = Nq;
  p.n_blocks = static_cast<int>(n_blocks);
  p.n_pad = static_cast<int>(n_blocks * 128);
  p.Nk = Nk;
  p.nbk = static_cast<int>(nbk);
  p.off = Nk - Nq;
  p.delta = static_cast<float*>(workspace);
  p.lse2 = static_cast<float*>(workspace) + static_cast<size_t>(p.BH) * p.n_pad;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.status = st->status;
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.causal = causal;
  p.g_fp32 = g_dtype == ATTN_FP32 ? 1 : 0;
  p.o_sb = so.sb, p.o_sh = so.sh, p.o_sn = so.sn;
  p.do_sb = sdo.sb, p.do_sh = sdo.sh, p.do_sn = sdo.sn;
  p.dq_sb = st8[5].sb, p.dq_sh = st8[5].sh, p.dq_sn = st8[5].sn;
  p.dk_sb = st8[6].sb, p.dk_sh = st8[6].sh, p.dk_sn = st8[6].sn;
  p.dv_sb = st8[7].sb, p.dv_sh = st8[7].sh, p.dv_sn = st8[7].sn;
  p.cu_q = pk ? pk->cu_q : nullptr;
  p.cu_k = pk ? pk->cu_k : nullptr;
  p.total_q = pk ? pk->total_q : 0;
  p.total_k = pk ? pk->total_k : 0;
  p.ds = nullptr;
  p.ds_tiles = 0;
  p.ds_rect = 0;
  p.ds_nbk = 0;
  p.kv_tab = p.q_tab = nullptr;
  if (ds_mode) {
    // the dS^T tiles follow D and LSE in the workspace (bwd_ds_workspace_bytes): a triangle or a
    // square of tiles per (batch, head); packed batches: a rectangle of n_blocks x nbk tiles per
    // (sequence, head), whatever each sequence's lengths
    const long long nb = n_blocks;
    if (pk != nullptr) {
      p.ds_rect = 1;
      p.ds_nbk = static_cast<int>(nbk);
      p.ds_tiles = nb * nbk;
    } else {
      p.ds_tiles = causal ? nb * (nb + 1) / 2 : nb * nb;
    }
    const size_t head = (2ull * static_cast<size_t>(p.BH) * p.n_pad * 4ull + 1023ull) / 1024ull * 1024ull;
    p.ds = static_cast<uint8_t*>(workspace) + head;
    if (pk == nullptr) {
      // work lists: the units of groups of heads whose streamed tensors fit L2 run together
      const int kv_units = p.BH * p.nbk, q_units = p.BH * p.n_blocks;
      p.kv_tab = ea::bwd_unit_table(p, 1, d, kv_units < st->num_sms ? kv_units : st->num_sms,
                                    static_cast<cudaStream_t>(stream));
      p.q_tab = ea::bwd_unit_table(p, 2, d, q_units < st->num_sms ? q_units : st->num_sms,
                                   static_cast<cudaStream_t>(stream));
    }
    if (ea::launch_attn_bwd_ds(d, mq, mk, mv, mdo, p, st->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
      return ATTN_ERR_CUDA;
    g_launches.fetch_add(3);
    return ATTN_OK;
  }
  if (ea::launch_attn_bwd(d, mq, mk, mv, mdo, p, st->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_launches.fetch_add(3);
  return ATTN_OK;
}

}  // namespace

extern "C" {

unsigned long long attn_bwd_ds_workspace_bytes(int B, int H, int N, int causal) {
  return bwd_ds_workspace_bytes(B, H, N, causal);
}

int attn_bwd_ds(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                void* dq, void* dk, void* dv, void* workspace, int B, int H, int N, int d, float scale, int causal,
                int g_dtype, void* stream) {
  if (B <= 0 || H <= 0 || N <= 0 || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (bwd_ds_workspace_bytes(B, H, N, causal) == 0ull) return ATTN_ERR_INVALID_ARG;  // too many tiles for int
  const Strides s = contiguous_strides(H, N, d);
  const Strides st8[8] = {s, s, s, s, s, s, s, s};
  return bwd_bf16(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, N, N, d, st8, nullptr, scale, causal, g_dtype,
                  stream, true);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
             void* dq, void* dk, void* dv, void* workspace, int B, int H, int N, int d, float scale, int causal,
             int g_dtype, void* stream) {
  const Strides s = contiguous_strides(H, N, d);
  const Strides st8[8] = {s, s, s, s, s, s, s, s};
  return bwd_bf16(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, N, N, d, st8, nullptr, scale, causal, g_dtype,
                  stream);
}

int attn_bwd_qk(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk, int d, float scale,
                int causal, int g_dtype, void* stream) {
  const Strides a = contiguous_strides(H, Nq, d), c = contiguous_strides(H, Nk, d);
  const Strides st8[8] = {a, c, c, a, a, a, c, c};
  return bwd_bf16(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Nq, Nk, d, st8, nullptr, scale, causal, g_dtype,
                  stream);
}

int attn_bwd_strided(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                     void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk, int d,
                     const long long* strides, float scale, int causal, int g_dtype, void* stream) {
  if (strides == nullptr || B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0) return ATTN_ERR_INVALID_ARG;
  Strides st8[8];
  for (int t = 0; t < 8; ++t) {
    const bool key_side = t == 1 || t == 2 || t == 6 || t == 7;  // k, v, dk, dv
    if (!canonical_strides(strides + 3 * t, B, H, key_side ? Nk : Nq, &st8[t])) return ATTN_ERR_INVALID_ARG;
  }
  return bwd_bf16(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Nq, Nk, d, st8, nullptr, scale, causal, g_dtype,
                  stream);
}

int attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                    void* dq, void* dk, void* dv, void* workspace, const int* cu_seqlens_q, const int* cu_seqlens_k,
                    int B, int H, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                    const long long* strides, float scale, int causal, int g_dtype, void* stream) {
  if (!cu_seqlens_q || !cu_seqlens_k || !strides || B <= 0 || H <= 0) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) != 0 || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) != 0)
    return ATTN_ERR_INVALID_ARG;
  constexpr int kMaxRows = 0x7FFFFFFF - (1 << 20);
  if (total_q <= 0 || total_k <= 0 || total_q > kMaxRows || total_k > kMaxRows || max_seqlen_q <= 0 ||
      max_seqlen_k <= 0 || max_seqlen_q > kMaxRows || max_seqlen_k > kMaxRows)
    return ATTN_ERR_INVALID_ARG;
  if (max_seqlen_q > total_q) max_seqlen_q = total_q;  // no sequence is longer than its tensor
  if (max_seqlen_k > total_k) max_seqlen_k = total_k;
  Strides st8[8];
  for (int t = 0; t < 8; ++t) {
    const bool key_side = t == 1 || t == 2 || t == 6 || t == 7;
    const long long s3[3] = {8, strides[2 * t + 1], strides[2 * t]};  // {batch (unused), head, row}
    if (!canonical_strides(s3, 1, H, key_side ? total_k : total_q, &st8[t])) return ATTN_ERR_INVALID_ARG;
  }
  const Packed pk{cu_seqlens_q, cu_seqlens_k, total_q, total_k};
  return bwd_bf16(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, max_seqlen_q, max_seqlen_k, d, st8, &pk, scale,
                  causal, g_dtype, stream);
}

unsigned long long attn_bwd_varlen_ds_workspace_bytes(int B, int H, int max_seqlen_q, int max_seqlen_k) {
  return bwd_varlen_ds_workspace_bytes(B, H, max_seqlen_q, max_seqlen_k);
}

int attn_bwd_varlen_ds(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                       void* dq, void* dk, void* dv, void* workspace, const int* cu_seqlens_q, const int* cu_seqlens_k,
                       int B, int H, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                       const long long* strides, float scale, int causal, int g_dtype, void* stream) {
  if (!cu_seqlens_q || !cu_seqlens_k || !strides || B <= 0 || H <= 0) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) != 0 || (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) != 0)
    return ATTN_ERR_INVALID_ARG;
  constexpr int kMaxRows = 0x7FFFFFFF - (1 << 20);
  if (total_q <= 0 || total_k <= 0 || total_q > kMaxRows || total_k > kMaxRows || max_seqlen_q <= 0 ||
      max_seqlen_k <= 0 || max_seqlen_q > kMaxRows || max_seqlen_k > kMaxRows)
    return ATTN_ERR_INVALID_ARG;
  if (bwd_varlen_ds_workspace_bytes(B, H, max_seqlen_q, max_seqlen_k) == 0ull) return ATTN_ERR_INVALID_ARG;
  if (max_seqlen_q > total_q) max_seqlen_q = total_q;  // no sequence is longer than its tensor
  if (max_seqlen_k > total_k) max_seqlen_k = total_k;
  Strides st8[8];
  for (int t = 0; t < 8; ++t) {
    const bool key_side = t == 1 || t == 2 || t == 6 || t == 7;
    const long long s3[3] = {8, strides[2 * t + 1], strides[2 * t]};  // {batch (unused), head, row}
    if (!canonical_strides(s3, 1, H, key_side ? total_k : total_q, &st8[t])) return ATTN_ERR_INVALID_ARG;
  }
  const Packed pk{cu_seqlens_q, cu_seqlens_k, total_q, total_k};
  return bwd_bf16(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, max_seqlen_q, max_seqlen_k, d, st8, &pk, scale,
                  causal, g_dtype, stream, true);
}

int attn_device_status(void* stream) {
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host = 0;
  if (cudaMemcpyAsync(&host, st->status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_CUDA;
  if (host != 0) {
    if (cudaMemsetAsync(st->status, 0, sizeof(int), s) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_CUDA;
    return (host & ea::kDevStatusTimeout) ? ATTN_ERR_TIMEOUT : ATTN_ERR_INVALID_ARG;
  }
  return ATTN_OK;
}

void attn_shutdown(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  int cur = 0;
  const bool have_dev = cudaGetDevice(&cur) == cudaSuccess;
  for (int dev = 0; dev < kMaxDevices; ++dev) {
    DeviceState& st = g_dev[dev];
    if (st.status != nullptr && cudaSetDevice(dev) == cudaSuccess) cudaFree(st.status);
    st = DeviceState{};
  }
  if (have_dev) cudaSetDevice(cur);
  ea::free_unit_tables();
}

}  // extern "C"
