// bwd_simt.cuh — the backward of the binary forward on CUDA cores: for an
// upstream gradient dO, the gradients of V, of the scaled binary Q and K
// (s_i = alpha_q_i sign(q_i), t_j = alpha_k_j sign(k_j)) and of the bias.
//
// Source: "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
// Transformers", §2 methodology: the scaled binary representations, the
// learnable bias added to the logits, softmax and P.V define the forward; the
// training bullet (quantisation-aware training with self-distillation) needs
// its gradients. The pages give no estimator through sign and the mean, so
// the gradients stop at s and t.
//
// With c = softmax_scale, logit_ij = c alpha_q_i alpha_k_j S_ij + bias[h,i,j]
// and P = softmax_j(logit):
//   dP_ij = <dO_i, V_j>,  D_i = sum_j P_ij dP_ij,  dL_ij = P_ij (dP_ij - D_i)
//   dV_j = sum_i P_ij dO_i
//   ds_i = c sum_j dL_ij t_j,  dt_j = c sum_i dL_ij s_i
//   dbias[h,i,j] = sum_b dL_bhij
//
// Two kernels, fp32 throughout, P recomputed from the packed bits:
//  - bwd_rows_kernel: one thread per query row (b,h,i). Pass 1 over the keys
//    keeps the online max m, the sum l and the rescaled sum of exp(.) dP, and
//    writes LSE_i = m + log l and D_i; pass 2 recomputes P and dL and
//    accumulates ds_i.
//  - bwd_cols_kernel: one thread per key (h, j), looping over the batch: for
//    each b it accumulates dV_j and dt_j over the query rows and adds dL_bhij
//    into dbias[h, i, j]. Only this thread touches column j of head h, so the
//    sum over b is in order b and needs no atomics.
// Shared-memory arrays indexed by [channel][thread] use a pitch of 65 floats,
// so that both the thread-wise reads and the row-wise staging stores are free
// of bank conflicts.
#pragma once
#include <string>

#include "common.cuh"

namespace binattn {
namespace bwd {

constexpr int kT = 64;       // threads per block: query rows (rows kernel) or keys (cols kernel)
constexpr int kTile = 64;    // keys (rows kernel) or query rows (cols kernel) staged per tile
constexpr int kPitch = 65;   // pitch of the [channel][thread] arrays

// Dynamic shared memory of each kernel, in bytes, for head dim d (at most 4
// sign words per token).
inline size_t rows_smem_bytes(int d) {
  const size_t floats = 2 * static_cast<size_t>(d) * kPitch  // dO^T, ds accumulators
                        + static_cast<size_t>(kTile) * d     // V of the key tile
                        + static_cast<size_t>(kTile) * kPitch  // bias tile, [key][row]
                        + kTile                              // alpha_k
                        + static_cast<size_t>(kTile) * 4;    // key sign words (W <= 4)
  return floats * 4;
}
inline size_t cols_smem_bytes(int d) {
  const size_t floats = 3 * static_cast<size_t>(d) * kPitch  // V^T of own keys, dV and dt accumulators
                        + static_cast<size_t>(kTile) * d     // dO of the query tile
                        + static_cast<size_t>(kTile) * kT    // bias tile, [row][key]
                        + 3 * kTile                          // alpha_q, LSE, D
                        + static_cast<size_t>(kTile) * 4;    // query sign words
  return floats * 4;
}

template <int W>
__global__ void __launch_bounds__(kT)
bwd_rows_kernel(const uint32_t* __restrict__ qb, const uint32_t* __restrict__ kb,
                const float* __restrict__ aq, const float* __restrict__ ak,
                const uint16_t* __restrict__ bias, const uint16_t* __restrict__ v,
                const uint16_t* __restrict__ dO, float scale, int H, int N, int d,
                float* __restrict__ lse, float* __restrict__ Dg, float* __restrict__ ds) {
  extern __shared__ float sm[];
  float* dOt = sm;                         // [d][kPitch]: dO[i0 + r][c] at c * kPitch + r
  float* acc = dOt + d * kPitch;           // [d][kPitch]: ds accumulators
  float* Vt = acc + d * kPitch;            // [kTile][d]: V[j0 + jj][c] at jj * d + c
  float* bt = Vt + kTile * d;              // [kTile][kPitch]: bias[i0 + r][j0 + jj] at jj * kPitch + r
  float* akt = bt + kTile * kPitch;        // [kTile]
  uint32_t* kbt = reinterpret_cast<uint32_t*>(akt + kTile);  // [kTile][W]

  const int t = threadIdx.x;
  const int bh = blockIdx.y;
  const int h = bh % H;
  const int i0 = blockIdx.x * kT;
  const int i = i0 + t;
  const bool valid = i < N;
  const size_t tok0 = static_cast<size_t>(bh) * N;  // token of (b, h, 0)

  uint32_t qw[W];
#pragma unroll
  for (int w = 0; w < W; ++w) qw[w] = valid ? qb[(tok0 + i) * W + w] : 0u;
  const float ci = valid ? scale * aq[tok0 + i] : 0.f;

  // this block's rows of dO, transposed; zero accumulators
  for (int e = t; e < kT * d; e += kT) {
    const int r = e / d, c = e % d;
    dOt[c * kPitch + r] = i0 + r < N ? bf16_bits_to_float(dO[(tok0 + i0 + r) * d + c]) : 0.f;
    acc[c * kPitch + r] = 0.f;
  }

  const int ntiles = (N + kTile - 1) / kTile;
  auto stage = [&](int j0) {
    __syncthreads();  // the previous tile is no longer read
    for (int e = t; e < kTile * d; e += kT) {
      const int jj = e / d, c = e % d;
      Vt[e] = j0 + jj < N ? bf16_bits_to_float(v[(tok0 + j0 + jj) * d + c]) : 0.f;
    }
    for (int e = t; e < kTile * W; e += kT) {
      const int jj = e / W, w = e % W;
      kbt[e] = j0 + jj < N ? kb[(tok0 + j0 + jj) * W + w] : 0u;
    }
    for (int jj = t; jj < kTile; jj += kT) akt[jj] = j0 + jj < N ? ak[tok0 + j0 + jj] : 0.f;
    if (bias) {
      for (int e = t; e < kT * kTile; e += kT) {
        const int r = e / kTile, jj = e % kTile;
        bt[jj * kPitch + r] = (i0 + r < N && j0 + jj < N)
                                  ? bf16_bits_to_float(bias[(static_cast<size_t>(h) * N + i0 + r) * N + j0 + jj])
                                  : 0.f;
      }
    }
    __syncthreads();
  };
  // logit and dP of key jj of the staged tile for this thread's row
  auto logit_dp = [&](int jj, float& L, float& dP) {
    const int S = binary_score<W>(qw, kbt + jj * W, d);
    L = ci * akt[jj] * static_cast<float>(S);
    if (bias) L += bt[jj * kPitch + t];
    float p = 0.f;
    for (int c = 0; c < d; ++c) p = fmaf(dOt[c * kPitch + t], Vt[jj * d + c], p);
    dP = p;
  };

  // pass 1: m, l and sum exp(L - m) dP, online
  float m = -INFINITY, l = 0.f, aD = 0.f;
  for (int kt = 0; kt < ntiles; ++kt) {
    const int j0 = kt * kTile;
    stage(j0);
    if (valid) {
      const int nj = min(kTile, N - j0);
      for (int jj = 0; jj < nj; ++jj) {
        float L, dP;
        logit_dp(jj, L, dP);
        const float mn = fmaxf(m, L);
        const float r = expf(m - mn);  // 0 while m is -inf
        const float e = expf(L - mn);
        l = l * r + e;
        aD = aD * r + e * dP;
        m = mn;
      }
    }
  }
  const float LSE = valid ? m + logf(l) : 0.f;
  const float D = valid ? aD / l : 0.f;
  if (valid) {
    lse[tok0 + i] = LSE;
    Dg[tok0 + i] = D;
  }

  // pass 2: P and dL again, ds_ic = c sum_j dL_ij alpha_k_j sign(k_jc)
  for (int kt = 0; kt < ntiles; ++kt) {
    const int j0 = kt * kTile;
    stage(j0);
    if (valid) {
      const int nj = min(kTile, N - j0);
      for (int jj = 0; jj < nj; ++jj) {
        float L, dP;
        logit_dp(jj, L, dP);
        const float P = expf(L - LSE);
        const float g = scale * (P * (dP - D)) * akt[jj];
        const uint32_t* kw = kbt + jj * W;
        for (int c = 0; c < d; ++c) {
          const bool pos = (kw[c >> 5] >> (c & 31)) & 1u;
          acc[c * kPitch + t] += pos ? g : -g;
        }
      }
    }
  }
  __syncthreads();
  for (int e = t; e < kT * d; e += kT) {
    const int r = e / d, c = e % d;
    if (i0 + r < N) ds[(tok0 + i0 + r) * d + c] = acc[c * kPitch + r];
  }
}

template <int W>
__global__ void __launch_bounds__(kT)
bwd_cols_kernel(const uint32_t* __restrict__ qb, const uint32_t* __restrict__ kb,
                const float* __restrict__ aq, const float* __restrict__ ak,
                const uint16_t* __restrict__ bias, const uint16_t* __restrict__ v,
                const uint16_t* __restrict__ dO, float scale, int B, int H, int N, int d,
                const float* __restrict__ lse, const float* __restrict__ Dg, float* __restrict__ dV,
                float* __restrict__ dt, float* __restrict__ dbias) {
  extern __shared__ float sm[];
  float* Vt = sm;                          // [d][kPitch]: V[j0 + r][c] at c * kPitch + r (own keys)
  float* dVa = Vt + d * kPitch;            // [d][kPitch]
  float* dta = dVa + d * kPitch;           // [d][kPitch]
  float* dOq = dta + d * kPitch;           // [kTile][d]: dO[i0 + ii][c] at ii * d + c
  float* bt = dOq + kTile * d;             // [kTile][kT]: bias[i0 + ii][j0 + r] at ii * kT + r
  float* aqt = bt + kTile * kT;            // [kTile]
  float* lset = aqt + kTile;               // [kTile]
  float* Dt = lset + kTile;                // [kTile]
  uint32_t* qbt = reinterpret_cast<uint32_t*>(Dt + kTile);  // [kTile][W]

  const int t = threadIdx.x;
  const int h = blockIdx.y;
  const int j0 = blockIdx.x * kT;
  const int j = j0 + t;
  const bool valid = j < N;
  const int ntiles = (N + kTile - 1) / kTile;

  for (int b = 0; b < B; ++b) {
    const size_t tok0 = (static_cast<size_t>(b) * H + h) * N;  // token of (b, h, 0)
    __syncthreads();  // the previous batch entry's accumulators are written out
    for (int e = t; e < kT * d; e += kT) {
      const int r = e / d, c = e % d;
      Vt[c * kPitch + r] = j0 + r < N ? bf16_bits_to_float(v[(tok0 + j0 + r) * d + c]) : 0.f;
      dVa[c * kPitch + r] = 0.f;
      dta[c * kPitch + r] = 0.f;
    }
    uint32_t kw[W];
#pragma unroll
    for (int w = 0; w < W; ++w) kw[w] = valid ? kb[(tok0 + j) * W + w] : 0u;
    const float akj = valid ? ak[tok0 + j] : 0.f;

    for (int it = 0; it < ntiles; ++it) {
      const int i0 = it * kTile;
      __syncthreads();  // the previous query tile is no longer read
      for (int e = t; e < kTile * d; e += kT) {
        const int ii = e / d, c = e % d;
        dOq[e] = i0 + ii < N ? bf16_bits_to_float(dO[(tok0 + i0 + ii) * d + c]) : 0.f;
      }
      for (int e = t; e < kTile * W; e += kT) {
        const int ii = e / W, w = e % W;
        qbt[e] = i0 + ii < N ? qb[(tok0 + i0 + ii) * W + w] : 0u;
      }
      for (int ii = t; ii < kTile; ii += kT) {
        const bool in = i0 + ii < N;
        aqt[ii] = in ? aq[tok0 + i0 + ii] : 0.f;
        lset[ii] = in ? lse[tok0 + i0 + ii] : 0.f;
        Dt[ii] = in ? Dg[tok0 + i0 + ii] : 0.f;
      }
      if (bias) {
        for (int e = t; e < kTile * kT; e += kT) {
          const int ii = e / kT, r = e % kT;
          bt[e] = (i0 + ii < N && j0 + r < N)
                      ? bf16_bits_to_float(bias[(static_cast<size_t>(h) * N + i0 + ii) * N + j0 + r])
                      : 0.f;
        }
      }
      __syncthreads();
      if (valid) {
        const int ni = min(kTile, N - i0);
        for (int ii = 0; ii < ni; ++ii) {
          const uint32_t* qw = qbt + ii * W;
          int pc = 0;
#pragma unroll
          for (int w = 0; w < W; ++w) pc += __popc(qw[w] ^ kw[w]);
          float L = scale * aqt[ii] * akj * static_cast<float>(d - 2 * pc);
          if (bias) L += bt[ii * kT + t];
          const float P = expf(L - lset[ii]);
          float dP = 0.f;
          for (int c = 0; c < d; ++c) dP = fmaf(dOq[ii * d + c], Vt[c * kPitch + t], dP);
          const float dL = P * (dP - Dt[ii]);
          const float g = scale * dL * aqt[ii];
          for (int c = 0; c < d; ++c) {
            dVa[c * kPitch + t] = fmaf(P, dOq[ii * d + c], dVa[c * kPitch + t]);
            const bool pos = (qw[c >> 5] >> (c & 31)) & 1u;
            dta[c * kPitch + t] += pos ? g : -g;
          }
          if (dbias) {
            float* db = dbias + (static_cast<size_t>(h) * N + i0 + ii) * N + j;
            *db = b == 0 ? dL : *db + dL;
          }
        }
      }
    }
    __syncthreads();
    for (int e = t; e < kT * d; e += kT) {
      const int r = e / d, c = e % d;
      if (j0 + r < N) {
        dV[(tok0 + j0 + r) * d + c] = dVa[c * kPitch + r];
        dt[(tok0 + j0 + r) * d + c] = dta[c * kPitch + r];
      }
    }
  }
}

// Launches the two kernels on `st`. lse, D: workspace floats [B * H * N] each.
// The kernels' set-up (their dynamic shared memory) is done once per device.
template <int W>
inline int backward_w(const uint32_t* qb, const uint32_t* kb, const float* aq, const float* ak,
                      const uint16_t* bias, const uint16_t* v, const uint16_t* dO, float scale, int B, int H,
                      int N, int d, float* dV, float* ds, float* dt, float* dbias, float* lse, float* D,
                      cudaStream_t st, std::string* msg) {
  const size_t rs = rows_smem_bytes(d), cs = cols_smem_bytes(d);
  static std::atomic<uint64_t> configured{0};
  if (needs_setup(configured)) {
    cudaError_t e = cudaFuncSetAttribute(bwd_rows_kernel<W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(rows_smem_bytes(W * 32)));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bwd_cols_kernel<W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(cols_smem_bytes(W * 32)));
    if (e != cudaSuccess) {
      *msg = std::string("cudaFuncSetAttribute (backward): ") + cudaGetErrorString(e);
      return 1;
    }
    mark_setup(configured);
  }
  const dim3 grid_rows((N + kT - 1) / kT, B * H);
  bwd_rows_kernel<W><<<grid_rows, kT, rs, st>>>(qb, kb, aq, ak, bias, v, dO, scale, H, N, d, lse, D, ds);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *msg = std::string("bwd_rows_kernel launch: ") + cudaGetErrorString(e);
    return 1;
  }
  const dim3 grid_cols((N + kT - 1) / kT, H);
  bwd_cols_kernel<W><<<grid_cols, kT, cs, st>>>(qb, kb, aq, ak, bias, v, dO, scale, B, H, N, d, lse, D, dV, dt,
                                                 dbias);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *msg = std::string("bwd_cols_kernel launch: ") + cudaGetErrorString(e);
    return 1;
  }
  return 0;
}

inline int backward(const uint32_t* qb, const uint32_t* kb, const float* aq, const float* ak, const uint16_t* bias,
                    const uint16_t* v, const uint16_t* dO, float scale, int B, int H, int N, int d, float* dV,
                    float* ds, float* dt, float* dbias, float* lse, float* D, cudaStream_t st, std::string* msg) {
  switch (words_for(d)) {
    case 1: return backward_w<1>(qb, kb, aq, ak, bias, v, dO, scale, B, H, N, d, dV, ds, dt, dbias, lse, D, st, msg);
    case 2: return backward_w<2>(qb, kb, aq, ak, bias, v, dO, scale, B, H, N, d, dV, ds, dt, dbias, lse, D, st, msg);
    case 3: return backward_w<3>(qb, kb, aq, ak, bias, v, dO, scale, B, H, N, d, dV, ds, dt, dbias, lse, D, st, msg);
    case 4: return backward_w<4>(qb, kb, aq, ak, bias, v, dO, scale, B, H, N, d, dV, ds, dt, dbias, lse, D, st, msg);
    default:
      *msg = "head dim above 128";
      return 1;
  }
}

}  // namespace bwd
}  // namespace binattn
