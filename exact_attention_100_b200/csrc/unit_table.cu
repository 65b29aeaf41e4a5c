// Work lists of the persistent forward kernels for fixed-length batches: which units (one
// batch*head and one group of 128-row Q tiles, the kernel's decode_unit) each CTA computes, in
// which order; likewise for the two main kernels of the backward's dS mode (units of one
// batch*head and one key block, or one query block).
//
// Units run longest first ("FlashAttention-2/3", FA-2 improvement 3: parallelism over the
// sequence, with causal blocks skipped, leaves units of very different lengths), dealt by greedy
// list scheduling: the next unit goes to the CTA whose list is shortest so far under a cost
// model of K/V blocks per unit.  The order is also grouped by heads: all units of a group of
// heads come before the next group, so that the K and V the running units read (every unit
// streams its head's keys from the first block on) stay in the 126 MB L2 instead of being read
// from HBM once per unit.  The group holds as many heads as fit kGroupKvBytes of K and V,
// and at least enough units for two per CTA, which keeps the greedy lists balanced.
//
// The tables live in device memory, built on the first launch of a shape and kept until
// attn_shutdown (a captured CUDA graph may hold one); launches that are too large to tabulate,
// launches during a stream capture of a shape not seen before, and packed batches keep the
// kernel's built-in round-robin order.

#include <algorithm>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <utility>
#include <vector>

#include "attn_kernels.h"

namespace ea {

namespace {

constexpr long long kGroupKvBytes = 32ll << 20;  // K and V of the heads whose units run together
constexpr long long kMaxTableUnits = 1ll << 20;  // larger launches keep the round-robin order
constexpr size_t kMaxTables = 4096;              // cached shapes per process; later ones too
constexpr int kUnitOverhead = 2;                 // fixed cost of a unit (fill, epilogue), in blocks

// K/V blocks the kernel visits for Q tile t (decode_unit, fixed-length batches)
int blocks_of_tile(const FwdParams& p, int t) {
  if (t >= p.n_blocks) return 0;
  if (!p.causal) return p.nbk;
  const int last = std::min(t * 128 + 127, p.N - 1) + p.off;
  return last < 0 ? 0 : std::min(last / 128 + 1, p.nbk);
}

// kind (0 forward, 1 backward dK/dV, 2 backward dQ from stored dS), device, shape, grid
using Key = std::tuple<int, int, int, int, int, int, int, int, int, int, int, int>;

std::mutex g_tab_mutex;
std::map<Key, int*> g_tabs;  // device tables (nullptr: the shape keeps the round-robin order)

// Heads per group: their streamed bytes within kGroupKvBytes, but at least 2 * grid units per
// group, and groups of nearly equal size.
long long group_heads(int BH, int R, long long bytes_per_head, int grid) {
  long long g_l2 = bytes_per_head > 0 ? kGroupKvBytes / bytes_per_head : BH;
  if (g_l2 < 1) g_l2 = 1;
  const long long g_bal = (2ll * grid + R - 1) / R;
  long long G = std::min<long long>(BH, std::max(g_l2, g_bal));
  const long long n_groups = (BH + G - 1) / G;
  return (BH + n_groups - 1) / n_groups;
}

// Greedy list scheduling of the units u = r * BH + bh (rounds r = 0 .. R-1, numbered longest
// first by the caller, cost[r] each) over `grid` CTAs, group by group of G heads:
// out = [grid + 1 list offsets][unit ids].
void greedy_lists(int BH, int R, const std::vector<long long>& cost, long long G, int grid, std::vector<int>* out) {
  using Slot = std::pair<long long, int>;  // (load so far, CTA): ties go to the lower CTA
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int b = 0; b < grid; ++b) heap.push({0, b});
  std::vector<std::vector<int>> lists(grid);
  for (long long g0 = 0; g0 < BH; g0 += G) {
    const long long g1 = std::min<long long>(BH, g0 + G);
    for (int r = 0; r < R; ++r) {
      for (long long bh = g0; bh < g1; ++bh) {
        Slot s = heap.top();
        heap.pop();
        lists[s.second].push_back(static_cast<int>(static_cast<long long>(r) * BH + bh));
        s.first += cost[r];
        heap.push(s);
      }
    }
  }
  const long long units = static_cast<long long>(BH) * R;
  out->assign(static_cast<size_t>(grid) + 1 + units, 0);
  int pos = 0;
  for (int b = 0; b < grid; ++b) {
    (*out)[b] = pos;
    for (int u : lists[b]) (*out)[grid + 1 + pos++] = u;
  }
  (*out)[grid] = pos;
}

// The cached device copy of a table built by `build` (nullptr: no table for this launch).
template <class Build>
const int* cached_table(const Key& key, cudaStream_t stream, Build build) {
  std::lock_guard<std::mutex> lock(g_tab_mutex);
  const auto it = g_tabs.find(key);
  if (it != g_tabs.end()) return it->second;
  // a new shape: build its table, unless the stream is being captured (no allocation or
  // synchronous copy may join a capture) or the cache is full
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return nullptr;
  if (g_tabs.size() >= kMaxTables) return nullptr;
  std::vector<int> host;
  int* table = nullptr;
  if (build(&host)) {
    const size_t bytes = host.size() * sizeof(int);
    if (cudaMalloc(&table, bytes) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    // synchronous: the table is on the device before the kernel that reads it is launched
    if (cudaMemcpy(table, host.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaFree(table);
      return nullptr;
    }
  }
  g_tabs.emplace(key, table);
  return table;
}

int current_device() {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

}  // namespace

int fwd_grid(const FwdParams& p, int num_sms) { return p.num_units < num_sms ? p.num_units : num_sms; }

bool fwd_unit_schedule(const FwdParams& p, int nq, int d, int elem_bytes, int grid, std::vector<int>* out) {
  if (p.cu_q != nullptr || grid <= 0 || p.num_units <= 0 || p.num_units > kMaxTableUnits) return false;
  const int BH = p.BH, P = p.n_pairs;
  // the kernel's round r holds pair P - 1 - r (causal, longest first) or r; the cost of a unit
  // is the K/V blocks of its longest tile
  std::vector<long long> cost(P);
  for (int r = 0; r < P; ++r) {
    const int pr = p.causal ? P - 1 - r : r;
    int n_max = 0;
    for (int q = 0; q < nq; ++q) n_max = std::max(n_max, blocks_of_tile(p, pr * nq + q));
    cost[r] = n_max + kUnitOverhead;
  }
  // units of groups of heads whose K and V fit kGroupKvBytes
  greedy_lists(BH, P, cost, group_heads(BH, P, 2ll * p.Nk * d * elem_bytes, grid), grid, out);
  return true;
}

const int* fwd_unit_table(const FwdParams& p, int nq, int d, int elem_bytes, int grid, cudaStream_t stream) {
  const int dev = current_device();
  if (dev < 0) return nullptr;
  const Key key{0, dev, p.BH, p.H, p.N, p.Nk, p.causal, nq, d, elem_bytes, grid, p.n_pairs};
  return cached_table(key, stream, [&](std::vector<int>* out) { return fwd_unit_schedule(p, nq, d, elem_bytes, grid, out); });
}

bool bwd_unit_schedule(const BwdParams& p, int kind, int d, int grid, std::vector<int>* out) {
  if (p.cu_q != nullptr || grid <= 0) return false;
  const int BH = p.BH;
  const int R = kind == 1 ? p.nbk : p.n_blocks;
  if (static_cast<long long>(BH) * R > kMaxTableUnits || BH * R <= 0) return false;
  std::vector<long long> cost(R);
  for (int r = 0; r < R; ++r) {
    int n;
    if (kind == 1) {
      // dK/dV unit: key block r and the query blocks from the first one that sees it
      const int first_q = r * 128 - p.off;
      const int i0 = (!p.causal || first_q <= 0) ? 0 : first_q / 128;
      n = std::max(0, p.n_blocks - i0);
    } else {
      // dQ unit: query block n_blocks - 1 - r (causal) or r and its visible key blocks
      const int qb = p.causal ? p.n_blocks - 1 - r : r;
      if (!p.causal) {
        n = p.nbk;
      } else {
        const int last = std::min(qb * 128 + 127, p.N - 1) + p.off;
        n = last < 0 ? 0 : std::min(last / 128 + 1, p.nbk);
      }
    }
    cost[r] = n + kUnitOverhead;
  }
  // the tensors every unit of a head streams: Q and dO (dK/dV) or K (dQ from stored dS)
  const long long bytes = kind == 1 ? 2ll * p.N * d * 2 : static_cast<long long>(p.Nk) * d * 2;
  greedy_lists(BH, R, cost, group_heads(BH, R, bytes, grid), grid, out);
  return true;
}

const int* bwd_unit_table(const BwdParams& p, int kind, int d, int grid, cudaStream_t stream) {
  const int dev = current_device();
  if (dev < 0) return nullptr;
  const Key key{kind, dev, p.BH, p.H, p.N, p.Nk, p.causal, d, 2, grid, 0, 0};
  return cached_table(key, stream, [&](std::vector<int>* out) { return bwd_unit_schedule(p, kind, d, grid, out); });
}

void free_unit_tables() {
  std::lock_guard<std::mutex> lock(g_tab_mutex);
  int cur = 0;
  const bool have_dev = cudaGetDevice(&cur) == cudaSuccess;
  for (auto& kv : g_tabs) {
    if (kv.second != nullptr && cudaSetDevice(std::get<1>(kv.first)) == cudaSuccess) cudaFree(kv.second);
  }
  g_tabs.clear();
  if (have_dev) cudaSetDevice(cur);
}

}  // namespace ea
