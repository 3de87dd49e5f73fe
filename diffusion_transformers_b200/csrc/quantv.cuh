// quantv.cuh — the per-channel 8-bit code of V for the 8-bit P.V forward.
//
// Source: "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
// Transformers", §2 hybrid quantisation (values in a per-channel 8-bit code)
// and the hardware-aware implementation bullet (mma.s32.u8.s8.s32). Read as:
// per (b, h, channel c), s_c = max_j |V_jc| / 127 and vq_jc = rint(V_jc / s_c)
// (ties to even, clamped to [-127, 127]), in fp32; s_c = 0 gives vq = 0.
//
// One CTA per (b, h), d % 8 == 0: thread t reads 16-byte chunk g = t % (d/8)
// of tokens t / (d/8), + kQvLanes, ..., so a warp's loads are consecutive
// chunks; the channel maxima go through shared memory, then the same threads
// read their chunks again and write the codes.
//
// Tiled layout (the K-major B operand of tcgen05.mma kind::i8 for O += P V,
// with N = DV channels and K = 64 keys per tile, no swizzle): tile kt of
// (b, h) is DV * 64 bytes at ((bh * nkt + kt) * DV * 64); within it byte
// (channel n, key jj) sits at (n / 8) * 512 + (jj / 16) * 128 + (n % 8) * 16 +
// jj % 16, i.e. 16-byte rows of 16 keys, core matrices of 8 channels
// (LBO = 128 between key groups, SBO = 512 between channel groups). Channel d
// holds 1 for every key < N (the row-sum column), channels d + 1 .. DV - 1 and
// keys >= N hold 0, so one contiguous copy fills a shared-memory stage.
#pragma once
#include "common.cuh"

namespace binattn {

constexpr int kQvThreads = 256;

// The 8-bit code of one value at scale s (fp32, as the reading states).
__device__ __forceinline__ int vcode(float v, float s) {
  if (!(s > 0.f)) return 0;
  const int q = __float2int_rn(__fdiv_rn(v, s));
  return q > 127 ? 127 : (q < -127 ? -127 : q);
}

// Byte offset of (channel n, key jj) inside one tile of the tiled layout.
__host__ __device__ __forceinline__ size_t vq_tile_offset(int n, int jj) {
  return static_cast<size_t>(n / 8) * 512 + (jj / 16) * 128 + (n % 8) * 16 + (jj % 16);
}

// tiled != null: write the tiled layout (DV columns, nkt = ceil(N / 64)
// tiles per (b, h)); plain != null: write vq [B,H,N,d] row-major. scale: [B,H,d].
__global__ void __launch_bounds__(kQvThreads)
quantize_v_kernel(const uint16_t* __restrict__ v, int N, int d, int DV, int8_t* __restrict__ tiled,
                  int8_t* __restrict__ plain, float* __restrict__ scale) {
  __shared__ int smax[128];  // |V| maxima as int bit patterns (non-negative floats order as ints)
  const int bh = blockIdx.x;
  const int ng = d / 8;
  const int lanes = kQvThreads / ng;  // tokens in flight per pass
  const int g = threadIdx.x % ng, lane = threadIdx.x / ng;
  const bool active = lane < lanes;
  for (int c = threadIdx.x; c < d; c += kQvThreads) smax[c] = 0;
  __syncthreads();
  const uint4* src = reinterpret_cast<const uint4*>(v + static_cast<size_t>(bh) * N * d);
  float mx[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (active) {
    for (int j = lane; j < N; j += lanes) {
      const uint4 ch = __ldg(src + static_cast<size_t>(j) * ng + g);
      const uint32_t w[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        mx[2 * e] = fmaxf(mx[2 * e], fabsf(__uint_as_float(w[e] << 16)));
        mx[2 * e + 1] = fmaxf(mx[2 * e + 1], fabsf(__uint_as_float(w[e] & 0xFFFF0000u)));
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) atomicMax(&smax[8 * g + e], __float_as_int(mx[e]));
  }
  __syncthreads();
  if (scale) {
    for (int c = threadIdx.x; c < d; c += kQvThreads)
      scale[static_cast<size_t>(bh) * d + c] = __fdiv_rn(__int_as_float(smax[c]), 127.f);
  }
  float s[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) s[e] = __fdiv_rn(__int_as_float(smax[8 * g + e]), 127.f);
  const int nkt = (N + 63) / 64;
  int8_t* tile0 = tiled ? tiled + static_cast<size_t>(bh) * nkt * DV * 64 : nullptr;
  if (active) {
    for (int j = lane; j < N; j += lanes) {
      const uint4 ch = __ldg(src + static_cast<size_t>(j) * ng + g);
      const uint32_t w[4] = {ch.x, ch.y, ch.z, ch.w};
      int q[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        q[2 * e] = vcode(__uint_as_float(w[e] << 16), s[2 * e]);
        q[2 * e + 1] = vcode(__uint_as_float(w[e] & 0xFFFF0000u), s[2 * e + 1]);
      }
      if (plain) {
        uint2 packed;
        packed.x = (q[0] & 0xFF) | (q[1] & 0xFF) << 8 | (q[2] & 0xFF) << 16 | static_cast<uint32_t>(q[3] & 0xFF) << 24;
        packed.y = (q[4] & 0xFF) | (q[5] & 0xFF) << 8 | (q[6] & 0xFF) << 16 | static_cast<uint32_t>(q[7] & 0xFF) << 24;
        *reinterpret_cast<uint2*>(plain + (static_cast<size_t>(bh) * N + j) * d + 8 * g) = packed;
      }
      if (tile0) {
        int8_t* t = tile0 + static_cast<size_t>(j / 64) * DV * 64;
#pragma unroll
        for (int e = 0; e < 8; ++e) t[vq_tile_offset(8 * g + e, j % 64)] = static_cast<int8_t>(q[e]);
      }
    }
  }
  if (tile0) {
    // the row-sum column and the pad channels of every key < N, and every
    // channel of the keys >= N of the last tile
    const int npad = DV - d;
    for (int e = threadIdx.x; e < N * npad; e += kQvThreads) {
      const int j = e / npad, n = d + e % npad;
      tile0[static_cast<size_t>(j / 64) * DV * 64 + vq_tile_offset(n, j % 64)] = n == d ? 1 : 0;
    }
    const int ntail = nkt * 64 - N;
    for (int e = threadIdx.x; e < ntail * DV; e += kQvThreads) {
      const int j = N + e / DV, n = e % DV;
      tile0[static_cast<size_t>(j / 64) * DV * 64 + vq_tile_offset(n, j % 64)] = 0;
    }
  }
}

}  // namespace binattn
