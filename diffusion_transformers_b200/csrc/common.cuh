// common.cuh — shared internals of libbinattn (one translation unit).
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace binattn {

// Device status word. Kernels that abandon a bounded wait write a non-zero
// code here; binattn_device_status() reads and clears it.
__device__ int g_device_status;

enum DeviceStatusCode : int {
  kDevOk = 0,
  kDevTimeoutMbarrier = 1,
};

__device__ __forceinline__ void report_device_status(int code) {
  atomicCAS(&g_device_status, 0, code);
}

// bf16 bit pattern <-> float (exact widening; RNE narrowing via the intrinsic).
__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}

__host__ __device__ constexpr int words_for(int d) { return (d + 31) / 32; }

// One-time set-up of a kernel (function attributes) is per device: `done`
// holds one bit per device ordinal below 64. needs_setup is true while the
// current device's bit is clear (always, for ordinals it cannot track);
// mark_setup sets it once the set-up has succeeded. Two host threads may both
// run the set-up for one device; it is idempotent.
inline bool needs_setup(const std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return true;
  return !(done.load(std::memory_order_acquire) & (1ull << dev));
}
inline void mark_setup(std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64)
    done.fetch_or(1ull << dev, std::memory_order_release);
}

// The binary score of one (query, key) pair from packed sign bits:
// S = d - 2 * popcount(q XOR k) over W words. Pad bits (channels >= d) are 0
// in both operands, so their XOR is 0 and they add nothing.
// This routine is shared by the SIMT and POPC_TC forward kernels and by the
// debug-scores kernel of those engines.
template <int W>
__device__ __forceinline__ int binary_score(const uint32_t (&q)[W], const uint32_t* k, int d) {
  int pc = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) pc += __popc(q[w] ^ k[w]);
  return d - 2 * pc;
}

}  // namespace binattn
