// Host-memory tier: the n-gram table stays in pinned host memory and the
// rows a batch touches are brought to the GPU ahead of its lookup (the
// pages' CPU offload of the n-gram table "with asynchronous prefetch": prime-rl
// pull request "add native Qwen3.8 Flash Next", Summary and Overview,
// ngram_embedding_cpu_offload).
//
// ple_prefetch hashes the batch (the same rows as ple_hash), sorts the rows
// (the gradient's radix sort), and for the distinct rows, in ascending order:
//   uniq_rows[u] = the u-th distinct row, cache[u] = host_table[uniq_rows[u]],
//   slots[i] = u for every hit i of that row.
// Each distinct row crosses the host link once, however often the batch
// hits it.  The copies are plain 16-byte loads from mapped pinned memory
// (zero-copy), many in flight per warp.  Called on a side stream for batch
// k+1 while batch k computes, the transfer overlaps the compute; the lookup
// of the batch is then a gather from the cache by slot, and its backward a
// deterministic gradient of the slots into a [cache_rows, head_dim] buffer
// (whose row u belongs to table row uniq_rows[u]).
#include "common.cuh"
#include "sort.cuh"

namespace ple {
namespace {

constexpr int kWinWarps = 8;  // 32-position windows per block
constexpr int kScanThreads = 1024;

// Heads of the runs of equal sorted keys among window w's 32 positions.
__device__ __forceinline__ unsigned window_heads(const uint32_t* __restrict__ K, int64_t N, int64_t w,
                                                 uint32_t* key) {
  const int lane = threadIdx.x & 31;
  const int64_t p = w * 32 + lane;
  const uint32_t k = p < N ? K[p] : 0;
  const uint32_t prev = (p > 0 && p < N) ? K[p - 1] : 0;
  *key = k;
  return __ballot_sync(kFull, p < N && (p == 0 || k != prev));
}

// cnt of every block of kWinWarps windows -> bsum[block]
__global__ void __launch_bounds__(kWinWarps * 32)
count_heads_kernel(const uint32_t* __restrict__ K, int64_t N, int64_t nwin, int64_t* __restrict__ bsum,
                   const uint32_t* abort) {
  __shared__ int wsum[kWinWarps];
  wait_for_prior_grid();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kWinWarps + warp;
  uint32_t key;
  // a sort that gave up: no distinct rows (num_unique = 0, nothing copied)
  const bool stop = ld_relaxed(abort) != 0;
  const unsigned m = (w < nwin && !stop) ? window_heads(K, N, w, &key) : 0u;
  if (lane == 0) wsum[warp] = __popc(m);
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t t = 0;
    for (int i = 0; i < kWinWarps; ++i) t += wsum[i];
    bsum[blockIdx.x] = t;
  }
  allow_next_grid();
}

// In-place exclusive scan of bsum[0, nb) by one block; *total = the sum.
__global__ void __launch_bounds__(kScanThreads) scan_kernel(int64_t* __restrict__ bsum, int64_t nb,
                                                            int64_t* __restrict__ total) {
  __shared__ int64_t part[kScanThreads];
  wait_for_prior_grid();
  int64_t carry = 0;
  constexpr int kPer = 8;
  for (int64_t base = 0; base < nb; base += static_cast<int64_t>(kScanThreads) * kPer) {
    const int64_t i0 = base + static_cast<int64_t>(threadIdx.x) * kPer;
    int64_t v[kPer], s = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      v[u] = i0 + u < nb ? bsum[i0 + u] : 0;
      s += v[u];
    }
    part[threadIdx.x] = s;
    __syncthreads();
    for (int d = 1; d < kScanThreads; d <<= 1) {  // inclusive Hillis-Steele scan of the thread sums
      const int64_t y = threadIdx.x >= static_cast<unsigned>(d) ? part[threadIdx.x - d] : 0;
      __syncthreads();
      part[threadIdx.x] += y;
      __syncthreads();
    }
    int64_t run = carry + part[threadIdx.x] - s;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (i0 + u < nb) bsum[i0 + u] = run;
      run += v[u];
    }
    carry += part[kScanThreads - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) *total = carry;
  allow_next_grid();
}

// Slots of every hit, the distinct rows, and the cache rows (copied from the
// host table; a row outside the table gets uniq_rows = -1 and a zero row).
__global__ void __launch_bounds__(kWinWarps * 32)
finalize_kernel(const uint32_t* __restrict__ K, const uint32_t* __restrict__ I, int64_t N, int64_t nwin,
                const int64_t* __restrict__ bpre, int64_t num_rows, const unsigned char* host_table, int32_t row_bytes,
                unsigned char* __restrict__ cache, int64_t* __restrict__ slots, int64_t* __restrict__ uniq_rows,
                const uint32_t* abort) {
  __shared__ int wsum[kWinWarps];
  __shared__ unsigned char head_lane[kWinWarps][32];  // lane of the r-th head of each window
  wait_for_prior_grid();
  if (ld_relaxed(abort) != 0) return;  // the sort gave up: nothing is written
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kWinWarps + warp;
  uint32_t key = 0;
  const unsigned m = w < nwin ? window_heads(K, N, w, &key) : 0u;
  if (lane == 0) wsum[warp] = __popc(m);
  if ((m >> lane) & 1u) head_lane[warp][__popc(m & ((1u << lane) - 1u))] = static_cast<unsigned char>(lane);
  __syncthreads();
  if (w >= nwin) return;
  int64_t base = bpre[blockIdx.x];
  for (int i = 0; i < warp; ++i) base += wsum[i];
  const int64_t p = w * 32 + lane;
  unsigned le;
  asm("mov.u32 %0, %%lanemask_le;" : "=r"(le));
  const int64_t u = base + __popc(m & le) - 1;  // distinct rows up to and including p, minus one
  if (p < N) {
    const uint32_t i = I[p];  // < N for a sorted workspace; no write outside slots whatever it holds
    if (i < N) slots[i] = u;
  }
  const bool bad = key >= num_rows;
  if (((m >> lane) & 1u) != 0) uniq_rows[u] = bad ? -1 : static_cast<int64_t>(key);
  // copy the rows of this window's heads: (head h, 16-byte column c) pairs over the lanes
  const int V = row_bytes >> 4;
  const int nh = __popc(m);
  const int total = nh * V;
  constexpr int kInFlight = 4;
  for (int q0 = 0; q0 < total; q0 += 32 * kInFlight) {
    uint4 v[kInFlight];
    int64_t dst[kInFlight];
#pragma unroll
    for (int r = 0; r < kInFlight; ++r) {
      const int q = q0 + r * 32 + lane;
      const bool valid = q < total;
      const int h = valid ? q / V : 0;
      const int col = valid ? q - h * V : 0;
      const int pos = valid ? head_lane[warp][h] : 0;  // lane of the h-th head
      const uint32_t hk = __shfl_sync(kFull, key, pos);
      const int64_t hu = __shfl_sync(kFull, u, pos);
      dst[r] = -1;
      v[r] = make_uint4(0, 0, 0, 0);
      if (valid) {
        dst[r] = hu * row_bytes + col * 16;
        if (hk < num_rows)
          v[r] = *reinterpret_cast<const uint4*>(host_table + static_cast<int64_t>(hk) * row_bytes + col * 16);
      }
    }
#pragma unroll
    for (int r = 0; r < kInFlight; ++r)
      if (dst[r] >= 0) *reinterpret_cast<uint4*>(cache + dst[r]) = v[r];
  }
}

struct PrefetchLayout {
  SortLayout sort;
  size_t bsum, total_bytes;
  int64_t nwin, nblocks;
};

PrefetchLayout prefetch_layout(int64_t N) {
  PrefetchLayout L{};
  size_t off = 0;
  L.sort = sort_layout(N, &off);
  L.nwin = (N + 31) / 32;
  L.nblocks = (L.nwin + kWinWarps - 1) / kWinWarps;
  L.bsum = off;
  off = align256(off + sizeof(int64_t) * static_cast<size_t>(L.nblocks));
  L.total_bytes = off;
  return L;
}

bool device_readable(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of an unknown pointer
    return false;
  }
  return a.type == cudaMemoryTypeHost || a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

}  // namespace
}  // namespace ple

using namespace ple;

extern "C" {

size_t ple_prefetch_workspace_bytes(const ple_plan_t* plan, int64_t num_tokens) {
  if (plan == nullptr || num_tokens <= 0) return 0;
  return prefetch_layout(num_tokens * plan->hp.num_heads).total_bytes;
}

ple_status_t ple_prefetch(const ple_plan_t* plan, const int64_t* tokens, int64_t T, const int32_t* cu, int32_t S,
                          const void* host_table, void* cache, int64_t cache_rows, int64_t* slots,
                          int64_t* uniq_rows, int64_t* num_unique, void* workspace, size_t ws_bytes, void* stream) {
  if (plan == nullptr || T < 0 || num_unique == nullptr) return PLE_ERR_INVALID_ARG;
  const auto s = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    const cudaError_t e = cudaMemsetAsync(num_unique, 0, sizeof(int64_t), s);
    return e == cudaSuccess ? PLE_OK : cuda_fail(e);
  }
  const int64_t N = T * plan->hp.num_heads;
  if (tokens == nullptr || cu == nullptr || S < 1 || host_table == nullptr || cache == nullptr || slots == nullptr ||
      uniq_rows == nullptr)
    return PLE_ERR_INVALID_ARG;
  if (cache_rows < N) return PLE_ERR_INVALID_ARG;  // room for every hit's row, whatever the repeats
  if (N >= (int64_t{1} << 31) || plan->num_rows >= int64_t{0xffffffff}) return PLE_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(host_table) & 15u) || (reinterpret_cast<uintptr_t>(cache) & 15u) ||
      (reinterpret_cast<uintptr_t>(slots) & 7u) || (reinterpret_cast<uintptr_t>(uniq_rows) & 7u) ||
      (reinterpret_cast<uintptr_t>(num_unique) & 7u))
    return PLE_ERR_ALIGNMENT;
  if (!device_readable(host_table)) return PLE_ERR_INVALID_ARG;  // pageable host memory: not reachable
  const PrefetchLayout L = prefetch_layout(N);
  if (workspace == nullptr || ws_bytes < L.total_bytes) return PLE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PLE_ERR_ALIGNMENT;
  cudaError_t e;
  unsigned int* status = status_word(plan, static_cast<cudaStream_t>(stream), &e);
  if (status == nullptr) return cuda_fail(e);
  // rows of every hit (written into slots, overwritten by the slots at the end)
  ple_status_t st = ple_hash(plan, tokens, T, cu, S, slots, stream);
  if (st != PLE_OK) return st;
  auto* ws = static_cast<unsigned char*>(workspace);
  const uint32_t* K = nullptr;
  const uint32_t* I = nullptr;
  st = launch_sort(slots, N, plan->num_rows, ws, L.sort, nullptr, 0, status, s, &K, &I);
  if (st != PLE_OK) return st;
  auto* bsum = reinterpret_cast<int64_t*>(ws + L.bsum);
  const uint32_t* abort = sort_abort_word(L.sort, ws);
  e = launch_after(count_heads_kernel, dim3(static_cast<unsigned>(L.nblocks)), dim3(kWinWarps * 32), 0, s, K, N,
                   L.nwin, bsum, abort);
  if (e != cudaSuccess) return cuda_fail(e);
  e = launch_after(scan_kernel, dim3(1), dim3(kScanThreads), 0, s, bsum, L.nblocks, num_unique);
  if (e != cudaSuccess) return cuda_fail(e);
  e = launch_after(finalize_kernel, dim3(static_cast<unsigned>(L.nblocks)), dim3(kWinWarps * 32), 0, s, K, I, N,
                   L.nwin, static_cast<const int64_t*>(bsum), plan->num_rows,
                   static_cast<const unsigned char*>(host_table), plan->row_bytes, static_cast<unsigned char*>(cache),
                   slots, uniq_rows, abort);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch();
}

}  // extern "C"
