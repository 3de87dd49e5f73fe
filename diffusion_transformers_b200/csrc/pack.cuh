// pack.cuh — sign bits and per-token scale (binattn_pack).
//
// Source: "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
// Transformers", §2 scaled binary representations (s_i = mu_q * sign(q_i),
// t_j = mu_k * sign(k_j)); mu is the per-token mean |x|.
//
// One block handles kPackTokens consecutive tokens. Their bytes are one
// contiguous range, staged into shared memory with 128-bit coalesced loads
// (when a token is a whole number of 16-byte chunks). Then each warp takes a
// token at a time: lane c looks at channel 32*w + c, __ballot_sync(x >= 0)
// is packed word w, and the lanes' |x| partial sums are warp-reduced into alpha.
#pragma once
#include "common.cuh"

namespace binattn {

constexpr int kPackThreads = 256;
constexpr int kPackTokens = 64;

template <typename T> __device__ __forceinline__ float load_as_float(const T* p);
template <> __device__ __forceinline__ float load_as_float<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float load_as_float<uint16_t>(const uint16_t* p) {
  return bf16_bits_to_float(*p);
}

// kVec: token size d * sizeof(T) is a multiple of 16 bytes (and x is 16-byte
// aligned, which the API checks), so the block's range is whole uint4 chunks.
template <typename T, bool kVec>
__global__ void __launch_bounds__(kPackThreads)
pack_kernel(const T* __restrict__ x, long long n_tokens, int d, int W,
            uint32_t* __restrict__ bits, float* __restrict__ alpha) {
  extern __shared__ uint4 pack_smem[];
  const long long t0 = static_cast<long long>(blockIdx.x) * kPackTokens;
  const int ntok = static_cast<int>(min(static_cast<long long>(kPackTokens), n_tokens - t0));
  const T* src = x + t0 * d;
  const T* tile = src;
  if constexpr (kVec) {
    const int nchunks = static_cast<int>((static_cast<long long>(ntok) * d * sizeof(T)) / 16);
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    for (int c = threadIdx.x; c < nchunks; c += kPackThreads) pack_smem[c] = __ldg(&s4[c]);
    __syncthreads();
    tile = reinterpret_cast<const T*>(pack_smem);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int tk = warp; tk < ntok; tk += kPackThreads / 32) {
    const T* row = tile + static_cast<size_t>(tk) * d;
    float acc = 0.f;
    uint32_t myword = 0;
    for (int w = 0; w < W; ++w) {
      const int c = w * 32 + lane;
      const bool in = c < d;
      const float v = in ? load_as_float(row + c) : 0.f;
      // x >= 0 is true for +0.0 and -0.0; pad lanes contribute 0 bits.
      const uint32_t word = __ballot_sync(0xffffffffu, in && v >= 0.f);
      if (lane == w) myword = word;
      acc += fabsf(v);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const long long t = t0 + tk;
    if (lane < W) bits[t * W + lane] = myword;
    if (lane == 0) alpha[t] = acc / static_cast<float>(d);
  }
}


// Sign words and alpha of one bf16 row with d % 8 == 0 from its 16-byte
// chunks v[0 .. d/8) (chunks beyond d/8 are ignored): the sign words come from
// x >= 0 compares (8 channels per chunk, 4 chunks per word), and |x| is summed
// in eight partial sums (one per position in a chunk) combined by a tree, so
// alpha is a sum of depth <= d/8 + 2 in fp32. binattn_pack and the forward that
// binarises Q itself both call this, so their bits and alpha are identical.
template <int W>
__device__ __forceinline__ void pack_row_chunks(const uint4 (&v)[4 * W], int d, uint32_t* words, float& alpha) {
  const int ng = d / 8;  // 16-byte chunks per token
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int w = 0; w < W; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int g = 4 * w + j;
      if (g < ng) {
        const uint32_t pr[4] = {v[g].x, v[g].y, v[g].z, v[g].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // channel 8g + 2k in the low half, 8g + 2k + 1 in the high half
          const float lo = __uint_as_float(pr[k] << 16);
          const float hi = __uint_as_float(pr[k] & 0xFFFF0000u);
          word |= (lo >= 0.f ? 1u : 0u) << (8 * j + 2 * k);
          word |= (hi >= 0.f ? 1u : 0u) << (8 * j + 2 * k + 1);
          acc[2 * k] += fabsf(lo);
          acc[2 * k + 1] += fabsf(hi);
        }
      }
    }
    words[w] = word;
  }
  const float sum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
  alpha = sum / static_cast<float>(d);
}

// The same for a row read straight from global memory (16-byte aligned): all
// of the row's 16-byte loads are issued at once.
template <int W>
__device__ __forceinline__ void pack_row_bf16(const uint16_t* __restrict__ row, int d, uint32_t* words,
                                              float& alpha) {
  const uint4* src = reinterpret_cast<const uint4*>(row);
  const int ng = d / 8;
  uint4 v[4 * W];
#pragma unroll
  for (int g = 0; g < 4 * W; ++g) v[g] = g < ng ? __ldg(src + g) : make_uint4(0, 0, 0, 0);
  pack_row_chunks<W>(v, d, words, alpha);
}

// The same for a row with W = ceil(d / 32) <= 3 known only at run time.
__device__ __forceinline__ void pack_row_bf16_w(const uint16_t* __restrict__ row, int d, int W, uint32_t* words,
                                                float& alpha) {
  switch (W) {
    case 1: pack_row_bf16<1>(row, d, words, alpha); break;
    case 2: pack_row_bf16<2>(row, d, words, alpha); break;
    default: pack_row_bf16<3>(row, d, words, alpha); break;
  }
}

// bf16 rows with d % 8 == 0 (every token a whole number of 16-byte chunks):
// one thread per token (pack_row_bf16), all of its row's 16-byte loads in
// flight at once.
constexpr int kRowsTokens = 256;
template <int W>
__global__ void __launch_bounds__(kRowsTokens)
pack_bf16_rows_kernel(const uint16_t* __restrict__ x, long long n_tokens, int d,
                      uint32_t* __restrict__ bits, float* __restrict__ alpha) {
  const long long t = static_cast<long long>(blockIdx.x) * kRowsTokens + threadIdx.x;
  if (t >= n_tokens) return;
  uint32_t words[W];
  float a;
  pack_row_bf16<W>(x + t * d, d, words, a);
#pragma unroll
  for (int w = 0; w < W; ++w) bits[t * W + w] = words[w];
  alpha[t] = a;
}

inline size_t pack_smem_bytes(int d, int esize, bool vec) {
  return vec ? static_cast<size_t>(kPackTokens) * d * esize : 0;
}

}  // namespace binattn
