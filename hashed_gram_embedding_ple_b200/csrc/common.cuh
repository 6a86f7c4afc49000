// Internal definitions shared by the libple translation units.
#pragma once

#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

#include "ple.h"

namespace ple {

constexpr int kMaxOrder = 8;   // ngram_size limit
constexpr int kMaxHeads = 64;  // H limit

// Per-head remainder constants.  For a modulus p (2 <= p <= 2^62):
//   magic = floor((2^64 - 1) / p), wrap = 2^64 mod p.
// q = mulhi(u, magic) underestimates floor(u / p) by at most 2 (Barrett,
// "Implementing the RSA public key encryption algorithm on a standard
// digital signal processor", CRYPTO 1986, with a one-word reciprocal), so
// u - q*p lies in [0, 3p) and two conditional subtractions finish u mod p.
struct HeadConst {
  uint64_t prime;
  uint64_t magic;
  uint64_t wrap;
  int64_t offset;
};

// Everything a hash kernel needs, passed by value as a kernel parameter.
struct HashParams {
  int32_t ngram_size;
  int32_t heads_per_ngram;
  int32_t num_heads;
  int32_t pad_;
  int64_t eos_id;
  int64_t mults[kMaxOrder];
  HeadConst head[kMaxHeads];
};

// Floor remainder of a signed 64-bit value: ((h % p) + p) % p.
__device__ __forceinline__ uint64_t floor_mod(int64_t h, const HeadConst& c) {
  const uint64_t u = static_cast<uint64_t>(h);
  const uint64_t q = __umul64hi(u, c.magic);
  uint64_t r = u - q * c.prime;
  if (r >= c.prime) r -= c.prime;
  if (r >= c.prime) r -= c.prime;
  // h < 0: h = u - 2^64, so h mod p = (u mod p - 2^64 mod p) mod p
  if (h < 0) r = (r >= c.wrap) ? r - c.wrap : r + c.prime - c.wrap;
  return r;
}

// Non-coherent table loads (the table is read-only during a call), cached in
// L1: under repeated rows (Zipf-distributed ids) an SM's later hits of a row
// are served by its L1.  Measured on the B200 against L1::no_allocate: the
// backward_stress lookup 140.1 -> 125.0 us, large_table 127.1 -> 125.0 us,
// 64-byte rows 3-6 % faster, no case slower.
__device__ __forceinline__ uint4 ld_nc(const void* p) {
  uint4 r;
  asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// 8-byte form of ld_nc (fp8 codes of one 16-byte output vector).
__device__ __forceinline__ uint2 ld_nc8(const void* p) {
  uint2 r;
  asm("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

// 16-byte streaming store (evict-first: the output is not re-read here).
__device__ __forceinline__ void st_cs(void* p, const uint4& v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Async status bits (bit k-1 for status code k).
__device__ __forceinline__ void raise_flag(unsigned int* status, ple_status_t code) {
  atomicOr(status, 1u << (static_cast<int>(code) - 1));
}

// Index s of the packed sequence holding token t: the last s with
// cu[s] <= t, searched over cu[0..num_seqs) (clamped to [0, num_seqs-1]).
__device__ __forceinline__ int32_t find_sequence(const int32_t* __restrict__ cu, int32_t num_seqs,
                                                 int64_t t) {
  int32_t lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (static_cast<int64_t>(__ldg(cu + mid)) <= t)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// Programmatic dependent launch (sm_90+).  A kernel launched with
// launch_after() may start while its predecessor in the stream is still
// draining; it must call wait_for_prior_grid() before it touches anything the
// predecessor writes (the hardware releases the wait once the predecessor has
// completed and its memory is visible).  allow_next_grid() lets the next
// grid be scheduled early.
__device__ __forceinline__ void wait_for_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_next_grid() { asm volatile("griddepcontrol.launch_dependents;" :::); }

template <typename... Params, typename... Args>
cudaError_t launch_after(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                         Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr{};
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
}

}  // namespace ple

// ---------------------------------------------------------------------------
// Host-side internals (defined in plan.cu)
// ---------------------------------------------------------------------------
struct ple_plan {
  ple::HashParams hp;
  int64_t num_rows;
  int32_t head_dim;
  ple_dtype_t table_dtype;
  int32_t row_bytes;
  int32_t status_slot;  // index of the plan's async status word
  // per device: the id of the context in which the plan's status word was
  // last cleared (~0: never)
  mutable std::atomic<unsigned long long> cleared_ctx[64];
  ple_plan() : status_slot(0) {
    for (auto& c : cleared_ctx) c.store(~0ull, std::memory_order_relaxed);
  }
};

namespace ple {
// Device address of the async status word of `plan` (nullptr: the word of
// calls that take no plan) on the current device; clears the plan's word on
// `stream` at its first use in a device context.
unsigned int* status_word(const ple_plan_t* plan, cudaStream_t stream, cudaError_t* err);
// The current context's id (false if the driver cannot tell).
bool current_context_id(unsigned long long* id);
// Multiprocessor count of the current device (cached).
int sm_count();
// Limit, in nanoseconds, of every bounded wait between the blocks of a
// kernel (the sort's look-back); set by ple_debug_set_wait_limit_ns.
uint64_t wait_limit_ns();
// Record a CUDA error for ple_last_cuda_error and return PLE_ERR_CUDA.
ple_status_t cuda_fail(cudaError_t e);
// PLE_OK, or cuda_fail of the last launch error.
ple_status_t check_launch();
}  // namespace ple
