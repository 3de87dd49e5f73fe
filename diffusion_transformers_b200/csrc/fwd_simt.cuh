// fwd_simt.cuh — CUDA-core engine (binattn_forward_engine(..., SIMT)) and the
// debug-scores kernel of the __popc score routine.
//
// One thread per query row; keys are staged through shared memory in tiles of
// kSimtKeys. Scores come from binary_score() (popcount of XOR over the packed
// words), logits are scaled and biased in fp32, and the softmax is kept online
// per key (running max m, sum l, accumulator rescaled when m grows), in the
// FlashAttention manner the method's kernel follows (§2 hardware-aware
// implementation). P stays fp32 here; V is widened from bf16.
#pragma once
#include "common.cuh"

namespace binattn {

constexpr int kSimtRows = 64;
constexpr int kSimtKeys = 32;

template <int W, bool kBias>
__global__ void __launch_bounds__(kSimtRows)
fwd_simt_kernel(const uint32_t* __restrict__ qb, const uint32_t* __restrict__ kb,
                const float* __restrict__ aq, const float* __restrict__ ak,
                const uint16_t* __restrict__ bias, const uint16_t* __restrict__ v,
                float scale, int H, int N, int d, uint16_t* __restrict__ out) {
  constexpr int DMAX = W * 32;
  __shared__ uint32_t s_kb[kSimtKeys][W];
  __shared__ float s_ak[kSimtKeys];
  __shared__ float s_v[kSimtKeys][DMAX];

  const int bh = blockIdx.y;
  const int h = bh % H;
  const int i = blockIdx.x * kSimtRows + threadIdx.x;
  const bool active = i < N;
  const size_t tok0 = static_cast<size_t>(bh) * N;

  uint32_t q[W];
  float ci = 0.f;
#pragma unroll
  for (int w = 0; w < W; ++w) q[w] = active ? qb[(tok0 + i) * W + w] : 0u;
  if (active) ci = scale * aq[tok0 + i];

  float o[DMAX];
#pragma unroll
  for (int c = 0; c < DMAX; ++c) o[c] = 0.f;
  float m = -INFINITY, l = 0.f;

  for (int j0 = 0; j0 < N; j0 += kSimtKeys) {
    __syncthreads();
    for (int e = threadIdx.x; e < kSimtKeys * W; e += kSimtRows) {
      const int jj = e / W, w = e % W, j = j0 + jj;
      s_kb[jj][w] = j < N ? kb[(tok0 + j) * W + w] : 0u;
    }
    for (int jj = threadIdx.x; jj < kSimtKeys; jj += kSimtRows) {
      const int j = j0 + jj;
      s_ak[jj] = j < N ? ak[tok0 + j] : 0.f;
    }
    for (int e = threadIdx.x; e < kSimtKeys * d; e += kSimtRows) {
      const int jj = e / d, c = e % d, j = j0 + jj;
      s_v[jj][c] = j < N ? bf16_bits_to_float(v[(tok0 + j) * d + c]) : 0.f;
    }
    __syncthreads();
    if (!active) continue;
    const int nk = min(kSimtKeys, N - j0);
    const uint16_t* brow = kBias ? bias + (static_cast<size_t>(h) * N + i) * N + j0 : nullptr;
    for (int jj = 0; jj < nk; ++jj) {
      const int s = binary_score<W>(q, s_kb[jj], d);
      float x = ci * s_ak[jj] * static_cast<float>(s);
      if (kBias) x += bf16_bits_to_float(brow[jj]);
      if (x > m) {
        const float corr = expf(m - x);  // m = -inf on the first key gives 0
        l *= corr;
#pragma unroll
        for (int c = 0; c < DMAX; ++c) o[c] *= corr;
        m = x;
      }
      const float p = expf(x - m);
      l += p;
#pragma unroll
      for (int c = 0; c < DMAX; ++c)
        if (c < d) o[c] = fmaf(p, s_v[jj][c], o[c]);
    }
  }
  if (active) {
    const float inv = 1.f / l;
    uint16_t* orow = out + (tok0 + i) * d;
#pragma unroll
    for (int c = 0; c < DMAX; ++c)
      if (c < d) orow[c] = float_to_bf16_bits(o[c] * inv);
  }
}

// S[bh, i, j] for every pair, with the same binary_score() routine.
// grid.x = ceil(N / 256) * N (key tile, query row), grid.y = B*H.
template <int W>
__global__ void __launch_bounds__(256)
scores_popc_kernel(const uint32_t* __restrict__ qb, const uint32_t* __restrict__ kb,
                   int N, int d, int32_t* __restrict__ S) {
  const int tiles = (N + 255) / 256;
  const int i = blockIdx.x / tiles;
  const int j = (blockIdx.x % tiles) * 256 + threadIdx.x;
  const size_t tok0 = static_cast<size_t>(blockIdx.y) * N;
  if (j >= N) return;
  uint32_t q[W];
#pragma unroll
  for (int w = 0; w < W; ++w) q[w] = qb[(tok0 + i) * W + w];
  S[(tok0 + i) * N + j] = binary_score<W>(q, kb + (tok0 + j) * W, d);
}

}  // namespace binattn
