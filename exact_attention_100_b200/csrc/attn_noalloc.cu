// attn_fwd_noalloc: the bf16 attention forward for callers that cannot allocate device memory.
//
// attn_fwd keeps its device status word in a workspace that the library cudaMalloc's on the
// first call on each device.  Some callers cannot allow that: runtimes whose device memory is
// owned by their own pool allocator and forbid allocations outside it, hosts that hand the
// library a fixed memory budget, and latency-critical loops that must never reach cudaMalloc,
// which can synchronise the whole device.  This entry point runs the same kernel with that
// scratch placed in a file-scope static __device__ array instead, so it never calls
// cudaMalloc, cudaFree or any allocating library routine.
//
// The first call on each device does a one-time set-up (the device address of the array via
// cudaGetSymbolAddress, the kernel's shared-memory attribute, the tensor-map encoder); make
// that first call before any stream capture.
//
// The array is kNoAllocScratchBytes (256 bytes) per GPU, resident on every GPU that loads this
// library until the process exits.  The kernel needs one int of it per call (its status word),
// whatever B, H, N and d are; a call that would need more than the array holds is refused with
// ATTN_ERR_INVALID_ARG.
//
// The status word is sticky: every call ORs its failures into it (a bounded wait that ran out)
// and nothing clears it except attn_noalloc_status, which reads and clears it on a stream.  It
// starts at zero when the library is loaded.  Calls that overlap on the GPU (different streams)
// share the word, so a failure is reported to whichever caller reads it first.
//
// In host code `g_noalloc_scratch` is only a host-side stand-in for the device array: its
// device address is obtained once per device with cudaGetSymbolAddress (with that device
// current) during the first call on the device, and that address is what the kernel receives.

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "attn_kernels.h"
#include "attn_selftest.h"

namespace ea {
cudaError_t setup_fwd_bf16_kernels();
}

namespace {

constexpr int kNoAllocScratchInts = 64;
constexpr size_t kNoAllocScratchBytes = kNoAllocScratchInts * sizeof(int);  // 256 bytes
constexpr size_t kScratchNeededBytes = sizeof(int);  // the kernel's status word
constexpr int kMaxDevices = 64;

__device__ __align__(256) int g_noalloc_scratch[kNoAllocScratchInts];

struct NoAllocDevice {
  bool ready = false;
  int num_sms = 0;
  int* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};

std::mutex g_mu;
NoAllocDevice g_state[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode_fn = nullptr;

bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Once per device, with that device current: device checks, the tensor-map encoder, the
// kernel attributes and the device address of the static scratch.  No allocation.
int noalloc_setup(NoAllocDevice** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  NoAllocDevice& st = g_state[dev];
  if (!st.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (major != 10 || minor != 0) return ATTN_ERR_UNSUPPORTED;
    if (g_encode_fn == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q{};
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return ATTN_ERR_CUDA;
      g_encode_fn = reinterpret_cast<EncodeTiledFn>(fn);
    }
    int* ptr = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return ATTN_ERR_CUDA;
    if (ea::setup_fwd_bf16_kernels() != cudaSuccess) return ATTN_ERR_CUDA;
    st.scratch = ptr;
    st.num_sms = sms;
    st.ready = true;
  }
  *out = &st;
  return ATTN_OK;
}

// Contiguous [B, H, N, d] bf16 as the forward kernel's 4-D map (d, rows, heads, batch).
bool encode_bf16_rows(CUtensorMap* map, const void* base, int d, int N, int H, int B) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t row = static_cast<cuuint64_t>(d) * 2;
  const cuuint64_t strides[3] = {row, row * static_cast<cuuint64_t>(N),
                                 row * static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(H)};
  const cuuint32_t box[4] = {64u, 128u, 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return g_encode_fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Contiguous [B, H, N, d] O (bf16 or f32) as the map of the kernel's TMA stores: box of 64 bytes
// x 128 rows, 64-byte swizzle.
bool encode_o_rows(CUtensorMap* map, void* base, bool f32, int d, int N, int H, int B) {
  const cuuint64_t eb = f32 ? 4 : 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t row = static_cast<cuuint64_t>(d) * eb;
  const cuuint64_t strides[3] = {row, row * static_cast<cuuint64_t>(N),
                                 row * static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(H)};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(64 / eb), 128u, 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return g_encode_fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                                int d, float scale, int causal, int dtype, int o_dtype, void* stream) {
  if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
  if (!is_aligned16(q) || !is_aligned16(k) || !is_aligned16(v) || !is_aligned16(o) || (lse && !is_aligned16(lse)))
    return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0 || static_cast<long long>(B) * H > 0x7FFFFFFFLL) return ATTN_ERR_INVALID_ARG;
  // the persistent kernel indexes its work units with int: B * H * ceil(N / 128) must fit
  if (static_cast<long long>(B) * H * ((static_cast<long long>(N) + 127) / 128) >= 0x7FFFFFFFLL)
    return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (o_dtype != ATTN_BF16 && o_dtype != ATTN_FP32) return ATTN_ERR_INVALID_ARG;
  if (dtype != ATTN_BF16) return dtype == ATTN_E4M3 || dtype == ATTN_FP32 ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  if (kScratchNeededBytes > kNoAllocScratchBytes) return ATTN_ERR_INVALID_ARG;

  NoAllocDevice* st = nullptr;
  int rc = noalloc_setup(&st);
  if (rc != ATTN_OK) return rc;
  CUtensorMap mq, mk, mv, mo;
  if (!encode_bf16_rows(&mq, q, d, N, H, B) || !encode_bf16_rows(&mk, k, d, N, H, B) ||
      !encode_bf16_rows(&mv, v, d, N, H, B) || !encode_o_rows(&mo, o, o_dtype == ATTN_FP32, d, N, H, B))
    return ATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  ea::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.status = st->scratch;
  p.q_scale = p.k_scale = p.v_scale = nullptr;
  p.cu_q = p.cu_k = nullptr;
  p.total_q = p.total_k = 0;
  p.vl_sched = 0;
  p.unit_tab = nullptr;  // the round-robin order: a table would need device memory
  p.N = N;
  p.BH = B * H;
  p.H = H;
  p.o_sn = d;
  p.o_sh = static_cast<long long>(d) * N;
  p.o_sb = p.o_sh * H;
  p.n_blocks = (N + 127) / 128;
  p.Nk = N;
  p.nbk = p.n_blocks;
  p.kv_sstride = p.nbk;
  p.max_nk = N;
  p.off = 0;
  const int tiles = ea::fwd_units_per_tile_pair(d);
  p.n_pairs = (p.n_blocks + tiles - 1) / tiles;
  p.num_units = p.BH * p.n_pairs;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.causal = causal;
  p.o_fp32 = o_dtype == ATTN_FP32 ? 1 : 0;
  if (ea::launch_attn_fwd_bf16(d, mq, mk, mv, mo, p, st->num_sms, s) != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

extern "C" int attn_noalloc_status(void* stream) {
  NoAllocDevice* st = nullptr;
  int rc = noalloc_setup(&st);
  if (rc != ATTN_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host = 0;  // pageable host memory: the copy completes before cudaMemcpyAsync returns or at the sync
  if (cudaMemcpyAsync(&host, st->scratch, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_CUDA;
  if (host == 0) return ATTN_OK;
  if (cudaMemsetAsync(st->scratch, 0, sizeof(int), s) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_CUDA;
  return (host & ea::kDevStatusTimeout) ? ATTN_ERR_TIMEOUT : ATTN_ERR_INVALID_ARG;
}

extern "C" int attn_noalloc_selftest_wait_timeout(void* stream) {
  NoAllocDevice* st = nullptr;
  int rc = noalloc_setup(&st);
  if (rc != ATTN_OK) return rc;
  return ea::launch_wait_selftest(st->scratch, static_cast<cudaStream_t>(stream)) == cudaSuccess ? ATTN_OK
                                                                                              : ATTN_ERR_CUDA;
}
