// quantv.cuh — the per-channel 8-bit code of V for the 8-bit P.V forward.
//
// Source: "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
// Transformers", §2 hybrid quantisation (values in a per-channel 8-bit code)
// and the hardware-aware implementation bullet (mma.s32.u8.s8.s32). Read as:
// per (b, h, channel c), s_c = max_j |V_jc| / 127 and vq_jc = rint(V_jc / s_c)
// (ties to even, clamped to [-127, 127]), in fp32; s_c = 0 gives vq = 0.
//
// Three kernels, d % 8 == 0: vmax_kernel finds every channel's max |V|
// (thread t reads 16-byte chunk t % (d/8) of its tokens, so a warp's loads
// are consecutive chunks), vquant_kernel codes one 64-key tile per CTA and
// writes it, vscale_kernel turns the maxima into the scales.
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

// First kernel: the maximum |V| of every (b, h, channel), as the bit pattern
// of a non-negative float (which orders like the integer), into maxbits
// [B*H, d], zeroed beforehand. grid = (B*H, ceil(N / kQvThreads)): each CTA
// reduces its tokens in shared memory and merges them with atomicMax.
__global__ void __launch_bounds__(kQvThreads)
vmax_kernel(const uint16_t* __restrict__ v, int N, int d, int* __restrict__ maxbits) {
  __shared__ int smax[128];
  const int bh = blockIdx.x;
  const int ng = d / 8;
  const int lanes = kQvThreads / ng;  // tokens per pass
  const int g = threadIdx.x % ng, lane = threadIdx.x / ng;
  for (int c = threadIdx.x; c < d; c += kQvThreads) smax[c] = 0;
  __syncthreads();
  const int j0 = blockIdx.y * kQvThreads;
  const int j1 = min(N, j0 + kQvThreads);
  const uint4* src = reinterpret_cast<const uint4*>(v + static_cast<size_t>(bh) * N * d);
  float mx[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (lane < lanes) {
    for (int j = j0 + lane; j < j1; j += lanes) {
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
  for (int c = threadIdx.x; c < d; c += kQvThreads) atomicMax(&maxbits[static_cast<size_t>(bh) * d + c], smax[c]);
}

// Second kernel: the codes of one 64-key tile per CTA, grid = (B*H, nkt).
// The tile's bf16 rows are staged in shared memory, coded at
// s_c = max_c / 127, and written as whole 16-byte rows of the tiled layout
// (tiled != null; with the row-sum channel and zero pads) and / or to the
// row-major plain [B,H,N,d] (plain != null).
__global__ void __launch_bounds__(kQvThreads)
vquant_kernel(const uint16_t* __restrict__ v, int N, int d, int DV, const int* __restrict__ maxbits,
              int8_t* __restrict__ tiled, int8_t* __restrict__ plain) {
  __shared__ float s_sc[128];
  __shared__ __align__(16) int8_t code[64][128 + 16];  // [key][channel], a row pitch off the bank period
  const int bh = blockIdx.x, kt = blockIdx.y;
  const int ng = d / 8;
  for (int c = threadIdx.x; c < d; c += kQvThreads)
    s_sc[c] = __fdiv_rn(__int_as_float(maxbits[static_cast<size_t>(bh) * d + c]), 127.f);
  __syncthreads();
  const int j0 = kt * 64;
  const uint4* src = reinterpret_cast<const uint4*>(v + static_cast<size_t>(bh) * N * d);
  for (int e = threadIdx.x; e < 64 * ng; e += kQvThreads) {
    const int jj = e / ng, g = e % ng, j = j0 + jj;
    int q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (j < N) {
      const uint4 ch = __ldg(src + static_cast<size_t>(j) * ng + g);
      const uint32_t w[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        q[2 * k] = vcode(__uint_as_float(w[k] << 16), s_sc[8 * g + 2 * k]);
        q[2 * k + 1] = vcode(__uint_as_float(w[k] & 0xFFFF0000u), s_sc[8 * g + 2 * k + 1]);
      }
      if (plain) {
        uint2 packed;
        packed.x = (q[0] & 0xFF) | (q[1] & 0xFF) << 8 | (q[2] & 0xFF) << 16 | static_cast<uint32_t>(q[3] & 0xFF) << 24;
        packed.y = (q[4] & 0xFF) | (q[5] & 0xFF) << 8 | (q[6] & 0xFF) << 16 | static_cast<uint32_t>(q[7] & 0xFF) << 24;
        *reinterpret_cast<uint2*>(plain + (static_cast<size_t>(bh) * N + j) * d + 8 * g) = packed;
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) code[jj][8 * g + k] = static_cast<int8_t>(q[k]);
  }
  if (!tiled) return;
  // the row-sum channel d (1 for keys < N) and zero pad channels up to DV
  for (int e = threadIdx.x; e < 64 * (DV - d); e += kQvThreads) {
    const int jj = e / (DV - d), n = d + e % (DV - d);
    code[jj][n] = (n == d && j0 + jj < N) ? 1 : 0;
  }
  __syncthreads();
  // 16-byte rows: (channel n, key group kg) = the codes of keys 16 kg .. + 15
  int8_t* tile = tiled + (static_cast<size_t>(bh) * gridDim.y + kt) * DV * 64;
  for (int e = threadIdx.x; e < DV * 4; e += kQvThreads) {
    const int n = e >> 2, kg = e & 3;
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w[k] = (code[16 * kg + 4 * k][n] & 0xFF) | (code[16 * kg + 4 * k + 1][n] & 0xFF) << 8 |
             (code[16 * kg + 4 * k + 2][n] & 0xFF) << 16 | static_cast<uint32_t>(code[16 * kg + 4 * k + 3][n] & 0xFF) << 24;
    *reinterpret_cast<uint4*>(tile + vq_tile_offset(n, 16 * kg)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Third kernel: scale = max / 127 for n entries (may work in place, over the
// maxima).
__global__ void __launch_bounds__(256) vscale_kernel(const int* maxbits, long long n, float* scale) {
  const long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  if (i < n) scale[i] = __fdiv_rn(__int_as_float(maxbits[i]), 127.f);
}

}  // namespace binattn
