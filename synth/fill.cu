// Device-side fill for the seeded synthetic table / gradient values.
//
// Implements, independently of the host generator in synth/__init__.py, the
// same counter-based definition: u(seed, i) is the (i+1)-th SplitMix64 output
// (Steele, Lea & Flood, OOPSLA 2014) from state seed * 0xD1B54A32D192ED03; the
// four 16-bit fields of u are summed exactly, centred on 131070 and scaled by
// one fp32 multiply; bf16 is fp32 rounded to nearest-even on its top half.
// This is input generation only and holds none of the lookup's arithmetic.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t sm64_out(uint64_t state0, uint64_t i) {
  uint64_t z = state0 + (i + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ float value_f32(uint64_t state0, uint64_t i, float k) {
  uint64_t u = sm64_out(state0, i);
  int32_t s = (int32_t)(u & 0xFFFF) + (int32_t)((u >> 16) & 0xFFFF) +
              (int32_t)((u >> 32) & 0xFFFF) + (int32_t)(u >> 48);
  return __fmul_rn((float)(s - 131070), k);
}

__device__ __forceinline__ uint32_t bf16_bits(float v) {
  uint32_t b = __float_as_uint(v);
  return (b + 0x7FFFu + ((b >> 16) & 1u)) >> 16;
}

// Each thread writes 16 bytes (4 fp32 or 8 bf16 values) per step.
__global__ void fill_f32(uint64_t state0, uint64_t count, float k, float* __restrict__ dst) {
  const uint64_t nvec = count / 4;
  for (uint64_t v = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; v < nvec;
       v += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t i = v * 4;
    float4 o = make_float4(value_f32(state0, i, k), value_f32(state0, i + 1, k),
                           value_f32(state0, i + 2, k), value_f32(state0, i + 3, k));
    reinterpret_cast<float4*>(dst)[v] = o;
  }
  for (uint64_t i = nvec * 4 + blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < count;
       i += (uint64_t)gridDim.x * blockDim.x)
    dst[i] = value_f32(state0, i, k);
}

__global__ void fill_bf16(uint64_t state0, uint64_t count, float k, uint16_t* __restrict__ dst) {
  const uint64_t nvec = count / 8;
  for (uint64_t v = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; v < nvec;
       v += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t i = v * 8;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      w[q] = bf16_bits(value_f32(state0, i + 2 * q, k)) |
             (bf16_bits(value_f32(state0, i + 2 * q + 1, k)) << 16);
    reinterpret_cast<uint4*>(dst)[v] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  for (uint64_t i = nvec * 8 + blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < count;
       i += (uint64_t)gridDim.x * blockDim.x)
    dst[i] = (uint16_t)bf16_bits(value_f32(state0, i, k));
}

// fp8 e4m3 codes: byte (i mod 8) of u(seed, i / 8), NaN codes moved to the
// largest finite code of their sign; each thread writes 16 codes.
__global__ void fill_e4m3(uint64_t state0, uint64_t count, unsigned char* __restrict__ dst) {
  const uint64_t nvec = count / 16;
  for (uint64_t v = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; v < nvec;
       v += (uint64_t)gridDim.x * blockDim.x) {
    uint32_t w[4];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint64_t u = sm64_out(state0, v * 2 + half);
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const uint32_t byte = (u >> (8 * b)) & 0xFF;
        if ((byte & 0x7F) == 0x7F) u ^= (1ull << (8 * b));
      }
      w[half * 2] = (uint32_t)u;
      w[half * 2 + 1] = (uint32_t)(u >> 32);
    }
    reinterpret_cast<uint4*>(dst)[v] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  for (uint64_t i = nvec * 16 + blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < count;
       i += (uint64_t)gridDim.x * blockDim.x) {
    uint32_t byte = (sm64_out(state0, i / 8) >> (8 * (i % 8))) & 0xFF;
    if ((byte & 0x7F) == 0x7F) byte ^= 1u;
    dst[i] = (unsigned char)byte;
  }
}

}  // namespace

extern "C" {

// Fill dst[0..count) with the generator's values for indices 0..count-1.
// dtype 0 = fp32, 1 = bf16 (bit patterns), 2 = fp8 e4m3 codes.  dst must be
// 16-byte aligned.
// Returns 0 on success, else the cudaError_t of the launch.
int synth_fill(uint64_t seed, uint64_t count, float k, int dtype, void* dst, cudaStream_t stream) {
  if (count == 0) return 0;
  if (dst == nullptr || (reinterpret_cast<uintptr_t>(dst) & 15u) != 0) return -1;
  const uint64_t state0 = seed * 0xD1B54A32D192ED03ull;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned grid = (unsigned)sms * 8u;
  if (dtype == 0)
    fill_f32<<<grid, 256, 0, stream>>>(state0, count, k, static_cast<float*>(dst));
  else if (dtype == 1)
    fill_bf16<<<grid, 256, 0, stream>>>(state0, count, k, static_cast<uint16_t*>(dst));
  else if (dtype == 2)
    fill_e4m3<<<grid, 256, 0, stream>>>(state0, count, static_cast<unsigned char*>(dst));
  else
    return -2;
  return (int)cudaGetLastError();
}

}  // extern "C"
