// Plan creation (host-only validation and constant precomputation), the
// async status word, and error reporting.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <new>
#include <utility>
#include <vector>

#include "common.cuh"

namespace {

__device__ unsigned int g_status_word;

thread_local int t_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
std::atomic<unsigned int*> g_status_ptr[kMaxDevices];
std::atomic<int> g_sm_count[kMaxDevices];

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

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

unsigned int* status_word(cudaError_t* err) {
  *err = cudaSuccess;
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  unsigned int* p = g_status_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    void* addr = nullptr;
    *err = cudaGetSymbolAddress(&addr, g_status_word);
    if (*err != cudaSuccess) return nullptr;
    p = static_cast<unsigned int*>(addr);
    g_status_ptr[dev].store(p, std::memory_order_release);
  }
  return p;
}

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

void ple_plan_destroy(ple_plan_t* plan) { delete plan; }

int32_t ple_plan_num_heads(const ple_plan_t* plan) { return plan ? plan->hp.num_heads : 0; }

ple_status_t ple_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return ple::cuda_fail(e);
  unsigned int* word = ple::status_word(&e);
  if (word == nullptr) return ple::cuda_fail(e);
  unsigned int bits = 0;
  e = cudaMemcpy(&bits, word, sizeof(bits), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return ple::cuda_fail(e);
  if (bits == 0) return PLE_OK;
  const unsigned int zero = 0;
  e = cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice);
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
    case PLE_ERR_TIMEOUT: return "a bounded wait between blocks ran out (results unspecified)";
  }
  return "unknown status";
}

int ple_last_cuda_error(void) { return t_last_cuda_error; }

}  // extern "C"
