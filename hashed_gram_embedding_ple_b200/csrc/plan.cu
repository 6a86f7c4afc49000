// Plan creation (host-only validation and constant precomputation), the
// async status words, and error reporting.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <new>
#include <utility>
#include <vector>

#include <cuda.h>

#include "common.cuh"
#include "ple_debug.h"

namespace {

// Async status words, one per plan slot; slot 0 is for calls that take no
// plan (the short convolution).  A kernel sets bit k-1 of its call's word
// for error k (atomicOr); ple_status takes a word with an atomic exchange on
// the device, so no flag raised meanwhile is lost, and one plan's read
// leaves the other plans' words alone.
constexpr int kStatusSlots = 4096;
constexpr int kTakeRing = 1024;  // result slots of concurrent ple_status calls
__device__ unsigned int g_status_words[kStatusSlots];
__device__ unsigned int g_status_taken[kTakeRing];

// Takes (reads and clears) words [first, first + count) and stores their OR.
__global__ void status_take_kernel(unsigned int* words, int first, int count, unsigned int* out) {
  __shared__ unsigned int acc;
  if (threadIdx.x == 0) acc = 0;
  __syncthreads();
  unsigned int bits = 0;
  for (int i = threadIdx.x; i < count; i += blockDim.x) bits |= atomicExch(words + first + i, 0u);
  bits = __reduce_or_sync(0xffffffffu, bits);
  if ((threadIdx.x & 31) == 0 && bits != 0) atomicOr(&acc, bits);
  __syncthreads();
  if (threadIdx.x == 0) *out = acc;
}

thread_local int t_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

// 100 ms: far above any legitimate wait (the tiles a block waits for are
// running and publish within microseconds), and well above a time slice of
// another context sharing the GPU, during which the waiting block and the
// block it waits for are both paused while the global timer runs on.
constexpr uint64_t kDefaultWaitNs = 100ull * 1000 * 1000;
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};

std::mutex g_slot_mu;
std::vector<bool> g_slot_used(kStatusSlots, false);
std::atomic<unsigned> g_take_ticket{0};

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// Device addresses of the status words for one device, valid for the
// context whose id is `ctx` (0: no context id available, one per device).
struct DeviceSyms {
  std::atomic<unsigned long long> ctx{~0ull};
  std::atomic<unsigned int*> words{nullptr};
  std::atomic<unsigned int*> taken{nullptr};
};
DeviceSyms g_syms[kMaxDevices];
std::mutex g_syms_mu;

}  // namespace

namespace ple {

ple_status_t cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return PLE_ERR_CUDA;
}

ple_status_t check_launch() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PLE_OK : cuda_fail(e);
}

bool current_context_id(unsigned long long* id) {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
    cudaGetLastError();  // a missing entry point is not an error of any call
  });
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return false;
  return get_id(c, id) == CUDA_SUCCESS;
}

// Status-word addresses of the current device, looked up again whenever the
// current context differs from the one they were looked up in (the runtime
// loads this library's module anew into a new context, e.g. after
// cudaDeviceReset).
static cudaError_t device_syms(int* dev_out, unsigned long long* ctx_out, unsigned int** words,
                               unsigned int** taken) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  unsigned long long ctx = 0;
  bool have = current_context_id(&ctx);
  DeviceSyms& d = g_syms[dev];
  if (have && d.ctx.load(std::memory_order_acquire) == ctx) {
    *words = d.words.load(std::memory_order_relaxed);
    *taken = d.taken.load(std::memory_order_relaxed);
  } else {
    std::lock_guard<std::mutex> lock(g_syms_mu);
    void* a = nullptr;
    void* b = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&a, g_status_words);  // (creates the context if there is none yet)
    if (e != cudaSuccess) return e;
    e = cudaGetSymbolAddress(&b, g_status_taken);
    if (e != cudaSuccess) return e;
    if (!have) have = current_context_id(&ctx);
    if (!have) ctx = 0;
    d.words.store(static_cast<unsigned int*>(a), std::memory_order_relaxed);
    d.taken.store(static_cast<unsigned int*>(b), std::memory_order_relaxed);
    d.ctx.store(ctx, std::memory_order_release);
    *words = static_cast<unsigned int*>(a);
    *taken = static_cast<unsigned int*>(b);
  }
  *dev_out = dev;
  *ctx_out = ctx;
  return cudaSuccess;
}

unsigned int* status_word(const ple_plan_t* plan, cudaStream_t stream, cudaError_t* err) {
  int dev = 0;
  unsigned long long ctx = 0;
  unsigned int* words = nullptr;
  unsigned int* taken = nullptr;
  *err = device_syms(&dev, &ctx, &words, &taken);
  if (*err != cudaSuccess) return nullptr;
  if (plan == nullptr) return words;
  unsigned int* w = words + plan->status_slot;
  // the slot may hold bits of a destroyed plan that had it before: cleared
  // (in stream order, ahead of this call's kernels) on the plan's first call
  // in each device context, by the one thread that claims that first call
  unsigned long long seen = plan->cleared_ctx[dev].load(std::memory_order_acquire);
  if (seen != ctx && plan->cleared_ctx[dev].compare_exchange_strong(seen, ctx, std::memory_order_acq_rel)) {
    *err = cudaMemsetAsync(w, 0, sizeof(unsigned int), stream);
    if (*err != cudaSuccess) {
      plan->cleared_ctx[dev].store(~0ull, std::memory_order_release);
      return nullptr;
    }
  }
  return w;
}

uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

int sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

}  // namespace ple

extern "C" {

ple_status_t ple_plan_create(const ple_params_t* p, ple_plan_t** out) {
  if (out == nullptr) return PLE_ERR_INVALID_ARG;
  *out = nullptr;
  if (p == nullptr || p->mults == nullptr || p->primes == nullptr || p->offsets == nullptr)
    return PLE_ERR_INVALID_ARG;
  if (p->ngram_size < 2 || p->ngram_size > ple::kMaxOrder || p->heads_per_ngram < 1)
    return PLE_ERR_INVALID_ARG;
  const int64_t H = static_cast<int64_t>(p->ngram_size - 1) * p->heads_per_ngram;
  if (H > ple::kMaxHeads) return PLE_ERR_UNSUPPORTED;
  if (p->num_rows < 1 || p->head_dim < 1) return PLE_ERR_INVALID_ARG;
  if (p->table_dtype != PLE_F32 && p->table_dtype != PLE_BF16 && p->table_dtype != PLE_F8E4M3)
    return PLE_ERR_INVALID_ARG;
  const int64_t elem = p->table_dtype == PLE_F32 ? 4 : p->table_dtype == PLE_BF16 ? 2 : 1;
  const int64_t row_bytes = elem * p->head_dim;
  if (row_bytes % 16 != 0) return PLE_ERR_ALIGNMENT;
  if (row_bytes > (1 << 20)) return PLE_ERR_UNSUPPORTED;

  std::vector<std::pair<int64_t, int64_t>> ranges;
  for (int64_t j = 0; j < H; ++j) {
    const int64_t prime = p->primes[j], off = p->offsets[j];
    if (prime < 2 || prime > (int64_t{1} << 62) || off < 0) return PLE_ERR_INVALID_ARG;
    if (off > p->num_rows - prime) return PLE_ERR_INVALID_ARG;  // off + prime <= num_rows
    ranges.emplace_back(off, off + prime);
  }
  std::sort(ranges.begin(), ranges.end());
  for (size_t k = 1; k < ranges.size(); ++k)
    if (ranges[k].first < ranges[k - 1].second) return PLE_ERR_INVALID_ARG;

  ple_plan* plan = new (std::nothrow) ple_plan();
  if (plan == nullptr) return PLE_ERR_INVALID_ARG;
  {  // a status word of its own
    std::lock_guard<std::mutex> lock(g_slot_mu);
    int slot = 1;
    while (slot < kStatusSlots && g_slot_used[slot]) ++slot;
    if (slot == kStatusSlots) {
      delete plan;
      return PLE_ERR_UNSUPPORTED;  // kStatusSlots - 1 plans alive at once
    }
    g_slot_used[slot] = true;
    plan->status_slot = slot;
  }
  std::memset(&plan->hp, 0, sizeof(plan->hp));
  plan->hp.ngram_size = p->ngram_size;
  plan->hp.heads_per_ngram = p->heads_per_ngram;
  plan->hp.num_heads = static_cast<int32_t>(H);
  plan->hp.eos_id = p->eos_id;
  for (int k = 0; k < p->ngram_size; ++k) plan->hp.mults[k] = p->mults[k];
  for (int64_t j = 0; j < H; ++j) {
    const uint64_t prime = static_cast<uint64_t>(p->primes[j]);
    ple::HeadConst& c = plan->hp.head[j];
    c.prime = prime;
    c.magic = UINT64_MAX / prime;
    c.wrap = (UINT64_MAX % prime + 1) % prime;
    c.offset = p->offsets[j];
  }
  plan->num_rows = p->num_rows;
  plan->head_dim = p->head_dim;
  plan->table_dtype = p->table_dtype;
  plan->row_bytes = static_cast<int32_t>(row_bytes);
  *out = plan;
  return PLE_OK;
}

void ple_plan_destroy(ple_plan_t* plan) {
  if (plan == nullptr) return;
  {
    std::lock_guard<std::mutex> lock(g_slot_mu);
    g_slot_used[plan->status_slot] = false;
  }
  delete plan;
}

int32_t ple_plan_num_heads(const ple_plan_t* plan) { return plan ? plan->hp.num_heads : 0; }

ple_status_t ple_status(const ple_plan_t* plan, void* stream) {
  const auto s = static_cast<cudaStream_t>(stream);
  int dev = 0;
  unsigned long long ctx = 0;
  unsigned int* words = nullptr;
  unsigned int* taken = nullptr;
  cudaError_t e = ple::device_syms(&dev, &ctx, &words, &taken);
  if (e != cudaSuccess) return ple::cuda_fail(e);
  int first = 0, count = kStatusSlots;  // no plan: every word of the device
  if (plan != nullptr) {
    if (plan->cleared_ctx[dev].load(std::memory_order_acquire) != ctx) {
      e = cudaStreamSynchronize(s);  // nothing of this plan ran in this context yet
      return e == cudaSuccess ? PLE_OK : ple::cuda_fail(e);
    }
    first = plan->status_slot;
    count = 1;
  }
  unsigned int* out = taken + g_take_ticket.fetch_add(1, std::memory_order_relaxed) % kTakeRing;
  status_take_kernel<<<1, count == 1 ? 32 : 1024, 0, s>>>(words, first, count, out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return ple::cuda_fail(e);
  unsigned int bits = 0;
  e = cudaMemcpyAsync(&bits, out, sizeof(bits), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return ple::cuda_fail(e);
  for (int k = 0; k < 32; ++k)
    if (bits & (1u << k)) return static_cast<ple_status_t>(k + 1);
  return PLE_OK;
}

const char* ple_strerror(ple_status_t s) {
  switch (s) {
    case PLE_OK: return "ok";
    case PLE_ERR_INVALID_ARG: return "invalid argument";
    case PLE_ERR_UNSUPPORTED: return "unsupported size or parameter";
    case PLE_ERR_ALIGNMENT: return "pointer or row size not 16-byte aligned";
    case PLE_ERR_WORKSPACE: return "workspace missing or too small";
    case PLE_ERR_CUDA: return "CUDA runtime error";
    case PLE_ERR_BAD_ROW: return "row id outside the table (output zeroed or hit dropped)";
    case PLE_ERR_BAD_SEQLENS: return "malformed cu_seqlens";
    case PLE_ERR_TIMEOUT: return "a bounded wait between blocks ran out (that call's gradient or prefetch was not applied)";
  }
  return "unknown status";
}

int ple_last_cuda_error(void) { return t_last_cuda_error; }

uint64_t ple_debug_set_wait_limit_ns(uint64_t ns) {
  return g_wait_ns.exchange(ns, std::memory_order_relaxed);
}

uint64_t ple_debug_default_wait_limit_ns(void) { return kDefaultWaitNs; }

}  // extern "C"
