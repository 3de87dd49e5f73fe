// fwd_tc.cuh — tensor-core engines of binattn_forward (TC and POPC_TC) and the
// debug-scores kernel of the TC engine.
//
// Source: "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
// Transformers", §2 methodology: scaled binary Q/K, XNOR/popcount similarity,
// additive learnable bias, softmax, P.V; FlashAttention2-style tiling from the
// hardware-aware implementation bullet. The tiling here is new for sm_100a.
//
// One CTA (12 warps, one per SM) owns 256 query rows of one (b, h) as two
// 128-row tiles t = 0, 1, and streams all keys in tiles of 128:
//   warps 0-7   softmax: warpgroup t (warps 4t..4t+3), thread = one query row.
//   warp 8      MMA issuer (one thread): tcgen05.mma, tcgen05.commit.
//   warps 9-11  producers: per key tile, alpha_k, the key sign bits (expanded to
//               +-1 bf16 for TC, copied as words for POPC_TC) and V, into a
//               two-stage shared-memory ring.
// Tensor memory (512 columns): S_t at column 128t (fp32, 128 keys), P_t written
// back over the first 64 columns of S_t as bf16 pairs, O_t at 256 + 128t.
//
// TC engine: S_t = Q_t K^T on the tensor core with +-1 bf16 operands. Pad
// channels of Q are 0, so every product is +-1 or 0 and the fp32 accumulator
// holds the exact integer score d - 2 popcount(q XOR k).
// POPC_TC engine: the softmax threads compute S with __popc over the packed
// words (binary_score), the tensor core does P.V only.
//
// Softmax (per row, fp32, online over key tiles): logit = (S * alpha_k) *
// (scale * alpha_q) + bias; running max m and sum l; O_t in TMEM is rescaled by
// exp(m_old - m_new) when m grows; P = exp(logit - m) rounded to bf16 for the
// P.V MMA; the epilogue divides by l and writes bf16.
//
// Every mbarrier wait is bounded (sm100::mbar_wait); on a timeout the CTA
// records a device status code, leaves its loops, waits for its own MMAs and
// frees its tensor memory.
#pragma once
#include <string>
#include "binattn.h"
#include "common.cuh"
#include "sm100.cuh"

namespace binattn {

inline bool tc_supported(int d) { return d % 8 == 0 && d <= 128; }
inline bool tc_built() { return true; }

namespace tc {

using namespace sm100;

constexpr int kRows = 128;       // query rows per softmax warpgroup (MMA M)
constexpr int kKeys = 128;       // keys per tile (QK MMA N, PV MMA K)
constexpr int kStages = 2;
constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
constexpr int kMmaWarp = 8;
constexpr int kProdWarp0 = 9;
constexpr int kProdThreads = 96;
constexpr int kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// Shared-memory map (byte offsets). An "operand tile" is 128 rows x KDIM bf16.
//  Q_t, K_s  (K-major, no swizzle): 16-byte chunk (row r, channel group c) at
//            (r / 8) * (KDIM * 16) + c * 128 + (r % 8) * 16
//            -> descriptor LBO = 128 (next channel group), SBO = KDIM * 16 (next 8 rows).
//  V_s       (MN-major, no swizzle): chunk (key j, d group g) at g * 2048 + j * 16
//            -> descriptor LBO = 128 (next 8 keys), SBO = 2048 (next 8 d values).
template <int KDIM>
struct Layout {
  static constexpr int kTile = kKeys * KDIM * 2;
  static constexpr int kLut = 0;                               // 256 x 16 B
  static constexpr int kQ = 4096;                              // 2 tiles
  static constexpr int kK = kQ + 2 * kTile;                    // kStages tiles
  static constexpr int kV = kK + kStages * kTile;              // kStages tiles
  static constexpr int kAk = kV + kStages * kTile;             // kStages x 128 fp32
  static constexpr int kKb = kAk + kStages * kKeys * 4;        // kStages x 128 x 4 words
  static constexpr int kBar = kKb + kStages * kKeys * 16;      // mbarriers
  static constexpr int kNumBars = 2 * kStages + 7;
  static constexpr int kMisc = kBar + 8 * kNumBars;            // tmem base, abort flag
  static constexpr int kBytes = kMisc + 16;
  // at least this much dynamic shared memory, so that one CTA occupies an SM
  // (each CTA allocates all 512 TMEM columns)
  static constexpr int kLaunchBytes = kBytes > 120 * 1024 ? kBytes : 120 * 1024;
};

struct Params {
  const uint32_t* qb;
  const uint32_t* kb;
  const float* aq;
  const float* ak;
  const uint16_t* bias;
  const uint16_t* v;
  uint16_t* out;
  int32_t* S;  // debug scores (dump mode)
  float scale;
  int H, N, d;
};

template <int KDIM, bool kTcQK, bool kBias, bool kDump>
__global__ void __launch_bounds__(kThreads, 1) fwd_tc_kernel(const Params p) {
  using L = Layout<KDIM>;
  constexpr int W = (KDIM + 31) / 32;  // packed words per token (= ceil(d / 32))
  constexpr int KCH = KDIM / 8;        // 16-byte channel groups per operand row
  constexpr uint32_t kIdescQK = idesc_bf16(kRows, kKeys, false);
  constexpr uint32_t kIdescPV = idesc_bf16(kRows, KDIM, true);

  extern __shared__ __align__(1024) uint8_t smem[];
  uint4* lut = reinterpret_cast<uint4*>(smem + L::kLut);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars;                  // [kStages] producers -> consumers
  uint64_t* kv_empty = bars + kStages;       // [kStages] MMA commit -> producers
  uint64_t* s_full = bars + 2 * kStages;     // [2] QK commit -> softmax t
  uint64_t* p_full = s_full + 2;             // [2] softmax t (128 arrivals) -> MMA
  uint64_t* o_done = p_full + 2;             // [2] PV commit -> softmax t
  uint64_t* drain = o_done + 2;              // error path only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, h = bh % p.H;
  const int N = p.N, d = p.d;
  const size_t tok0 = static_cast<size_t>(bh) * N;
  const int q0 = blockIdx.x * 2 * kRows;
  const int ntiles = (N + kKeys - 1) / kKeys;

  // ---------------------------------------------------------------- setup
  // LUT: 8 sign bits -> 8 bf16 values, element e = +1.0 if bit e is set, else -1.0.
  for (int b = threadIdx.x; b < 256; b += kThreads) {
    uint32_t w[4];
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      const uint32_t lo = ((b >> (2 * pr)) & 1) ? 0x3F80u : 0xBF80u;
      const uint32_t hi = ((b >> (2 * pr + 1)) & 1) ? 0x3F80u : 0xBF80u;
      w[pr] = lo | (hi << 16);
    }
    lut[b] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], kProdThreads);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], kRows);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();

  // Softmax threads: this thread's query row, and (TC) its +-1 row of Q_t.
  const int t = warp >> 2;                      // warpgroup (valid for warps 0-7)
  const int r = ((warp & 3) << 5) | lane;       // row within the tile = TMEM lane
  const int row = q0 + t * kRows + r;
  const bool row_valid = warp < 8 && row < N;
  uint32_t qw[W];
#pragma unroll
  for (int w = 0; w < W; ++w) qw[w] = row_valid ? p.qb[(tok0 + row) * W + w] : 0u;
  if (kTcQK && warp < 8) {
    uint8_t* qs = smem + L::kQ + t * L::kTile;
#pragma unroll
    for (int c = 0; c < KCH; ++c) {
      uint4 val = make_uint4(0, 0, 0, 0);  // pad channels (c >= d) are 0
      if (8 * c < d) val = lut[(qw[c >> 2] >> (8 * (c & 3))) & 0xFFu];
      *reinterpret_cast<uint4*>(qs + (r >> 3) * (KDIM * 16) + c * 128 + (r & 7) * 16) = val;
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kProdWarp0) {
    // ------------------------------------------------------------ producers
    const int pt = threadIdx.x - kProdWarp0 * 32;
    const int dgroups = d / 8;
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kStages;
      if (j >= kStages && !mbar_wait(&kv_empty[s], ((j / kStages) - 1) & 1, abort)) break;
      const int j0 = j * kKeys;
      if constexpr (!kDump) {  // the debug-scores variant gets no alpha_k / V
        float* aks = reinterpret_cast<float*>(smem + L::kAk) + s * kKeys;
        for (int kk = pt; kk < kKeys; kk += kProdThreads)
          aks[kk] = (j0 + kk < N) ? p.ak[tok0 + j0 + kk] : 0.f;
      }
      if constexpr (kTcQK) {
        uint8_t* ks = smem + L::kK + s * L::kTile;
        for (int e = pt; e < kKeys * KCH; e += kProdThreads) {
          const int kk = e / KCH, c = e % KCH, key = j0 + kk;
          uint4 val = make_uint4(0, 0, 0, 0);
          if (key < N && 8 * c < d)
            val = lut[(p.kb[(tok0 + key) * W + (c >> 2)] >> (8 * (c & 3))) & 0xFFu];
          *reinterpret_cast<uint4*>(ks + (kk >> 3) * (KDIM * 16) + c * 128 + (kk & 7) * 16) = val;
        }
      } else {
        uint32_t* kbs = reinterpret_cast<uint32_t*>(smem + L::kKb) + s * kKeys * 4;
        for (int e = pt; e < kKeys * W; e += kProdThreads) {
          const int kk = e / W, w = e % W, key = j0 + kk;
          kbs[kk * 4 + w] = key < N ? p.kb[(tok0 + key) * W + w] : 0u;
        }
      }
      if constexpr (!kDump) {
        uint8_t* vs = smem + L::kV + s * L::kTile;
        constexpr int kVIters = (kKeys * KCH + kProdThreads - 1) / kProdThreads;
        uint4 vbuf[kVIters];
#pragma unroll
        for (int it = 0; it < kVIters; ++it) {
          const int e = pt + it * kProdThreads;
          const int kk = e / KCH, g = e % KCH, key = j0 + kk;
          vbuf[it] = make_uint4(0, 0, 0, 0);
          if (e < kKeys * KCH && key < N && g < dgroups)
            vbuf[it] = __ldg(reinterpret_cast<const uint4*>(p.v + (tok0 + key) * d + 8 * g));
        }
#pragma unroll
        for (int it = 0; it < kVIters; ++it) {
          const int e = pt + it * kProdThreads;
          if (e < kKeys * KCH) {
            const int kk = e / KCH, g = e % KCH;
            *reinterpret_cast<uint4*>(vs + g * 2048 + kk * 16) = vbuf[it];
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&kv_full[s]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_u32(smem + L::kQ);
      const uint32_t k_base = smem_u32(smem + L::kK);
      const uint32_t v_base = smem_u32(smem + L::kV);
      auto issue_qk = [&](int tt, int s) {
#pragma unroll
        for (int ks = 0; ks < KDIM / 16; ++ks) {
          const uint64_t a = smem_desc(q_base + tt * L::kTile + ks * 256, 128, KDIM * 16);
          const uint64_t b = smem_desc(k_base + s * L::kTile + ks * 256, 128, KDIM * 16);
          mma_ss(tmem + tt * 128, a, b, kIdescQK, ks > 0);
        }
        mma_commit(&s_full[tt]);
      };
      bool ok = true;
      if constexpr (kTcQK) {
        ok = mbar_wait(&kv_full[0], 0, abort);
        if (ok) {
          tc_fence_after();
          issue_qk(0, 0);
          issue_qk(1, 0);
        }
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        const int s = j % kStages;
        if (!kTcQK) {
          if (!(ok = mbar_wait(&kv_full[s], (j / kStages) & 1, abort))) break;
          tc_fence_after();
        }
        for (int tt = 0; tt < 2; ++tt) {
          if (!(ok = mbar_wait(&p_full[tt], j & 1, abort))) break;
          tc_fence_after();
          if constexpr (!kDump) {
#pragma unroll
            for (int ks = 0; ks < kKeys / 16; ++ks) {
              const uint64_t b = smem_desc(v_base + s * L::kTile + ks * 256, 128, 2048);
              mma_ts(tmem + 256 + tt * 128, tmem + tt * 128 + ks * 8, b, kIdescPV, (j > 0 || ks > 0));
            }
            mma_commit(&o_done[tt]);
          }
          if (kTcQK && j + 1 < ntiles) {
            const int s1 = (j + 1) % kStages;
            if (tt == 0) {
              if (!(ok = mbar_wait(&kv_full[s1], ((j + 1) / kStages) & 1, abort))) break;
              tc_fence_after();
            }
            issue_qk(tt, s1);
          }
        }
        mma_commit(&kv_empty[s]);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax
    const float ci = (!kDump && row_valid) ? p.scale * p.aq[tok0 + row] : 0.f;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + t * 128;
    const uint32_t o_col = tmem + lane_base + 256 + t * 128;
    const uint16_t* brow = kBias && row_valid ? p.bias + (static_cast<size_t>(h) * N + row) * N : nullptr;
    const bool bias_vec = (N % 8) == 0;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // Waits are made warp-uniform: the tcgen05.ld/st below are warp-collective.
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
    };
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kStages;
      const int j0 = j * kKeys;
      float x[kKeys];
      if (!(ok = wait_all(&kv_full[s], (j / kStages) & 1))) break;
      if constexpr (kTcQK) {
        if (!(ok = wait_all(&s_full[t], j & 1))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kKeys; c += 32) tmem_ld32(s_col + c, reinterpret_cast<uint32_t*>(x + c));
        tmem_ld_wait();
      } else {
        const uint32_t* kbs = reinterpret_cast<const uint32_t*>(smem + L::kKb) + s * kKeys * 4;
#pragma unroll
        for (int c = 0; c < kKeys; ++c)
          x[c] = static_cast<float>(binary_score<W>(qw, kbs + c * 4, d));
      }
      if constexpr (kDump) {
        if (row_valid) {
          int32_t* srow = p.S + (tok0 + row) * N + j0;
#pragma unroll 8
          for (int c = 0; c < kKeys; ++c)
            if (j0 + c < N) srow[c] = static_cast<int32_t>(x[c]);
        }
        tc_fence_before();
        mbar_arrive(&p_full[t]);
        continue;
      }
      // logits = S * alpha_k * (scale * alpha_q) + bias, keys >= N masked
      const float* aks = reinterpret_cast<const float*>(smem + L::kAk) + s * kKeys;
      const bool tail = j0 + kKeys > N;
      float mx = -INFINITY;
#pragma unroll
      for (int c0 = 0; c0 < kKeys; c0 += 8) {
        float bv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) bv[e] = 0.f;
        if (kBias && row_valid) {
          if (bias_vec && !tail) {
            const uint4 raw = *reinterpret_cast<const uint4*>(brow + j0 + c0);
            const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              bv[2 * e] = __uint_as_float(rw[e] << 16);
              bv[2 * e + 1] = __uint_as_float(rw[e] & 0xFFFF0000u);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (j0 + c0 + e < N) bv[e] = bf16_bits_to_float(brow[j0 + c0 + e]);
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = c0 + e;
          float lg = fmaf(x[c] * aks[c], ci, bv[e]);
          if (tail && j0 + c >= N) lg = -INFINITY;
          x[c] = lg;
          mx = fmaxf(mx, lg);
        }
      }
      const float m_new = fmaxf(m, mx);
      const float corr = ex2((m - m_new) * kLog2e);  // 0 on the first tile
      if (j > 0) {
        // O_t must hold PV of tile j-1 before it is rescaled (and before P_t
        // is overwritten, which the MMA ordering already guarantees).
        if (!(ok = wait_all(&o_done[t], (j - 1) & 1))) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll
          for (int c = 0; c < KDIM; c += 16) {
            uint32_t ov[16];
            tmem_ld16(o_col + c, ov);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
            tmem_st16(o_col + c, ov);
          }
        }
      }
      l *= corr;
      m = m_new;
      const float nm = -m * kLog2e;
      uint32_t pk[kKeys / 2];
#pragma unroll
      for (int c = 0; c < kKeys; c += 2) {
        const float p0 = ex2(fmaf(x[c], kLog2e, nm));
        const float p1 = ex2(fmaf(x[c + 1], kLog2e, nm));
        l += p0 + p1;
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      tmem_st32(s_col, pk);
      tmem_st32(s_col + 32, pk + 32);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    if constexpr (!kDump) {
      if (ok && wait_all(&o_done[t], (ntiles - 1) & 1)) {
        tc_fence_after();
        const float inv = 1.f / l;
        uint16_t* orow = p.out + (tok0 + row) * d;
#pragma unroll
        for (int c = 0; c < KDIM; c += 16) {
          uint32_t ov[16];
          tmem_ld16(o_col + c, ov);
          tmem_ld_wait();
          if (row_valid) {
#pragma unroll
            for (int e = 0; e < 16; e += 8) {
              if (c + e < d) {
                uint4 o4;
                o4.x = pack_bf16x2(__uint_as_float(ov[e + 0]) * inv, __uint_as_float(ov[e + 1]) * inv);
                o4.y = pack_bf16x2(__uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
                o4.z = pack_bf16x2(__uint_as_float(ov[e + 4]) * inv, __uint_as_float(ov[e + 5]) * inv);
                o4.w = pack_bf16x2(__uint_as_float(ov[e + 6]) * inv, __uint_as_float(ov[e + 7]) * inv);
                *reinterpret_cast<uint4*>(orow + c + e) = o4;
              }
            }
          }
        }
      }
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    if (*abort) {
      // On the error path some MMAs may still be in flight: wait (bounded) for
      // every MMA this CTA issued before freeing tensor memory.
      if (lane == 0) {
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never);
      }
      __syncwarp();
    }
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int KDIM, bool kTcQK, bool kBias, bool kDump>
inline int launch_tc(const Params& prm, int B, int H, int N, cudaStream_t st, std::string* msg) {
  auto kern = fwd_tc_kernel<KDIM, kTcQK, kBias, kDump>;
  const int smem = Layout<KDIM>::kLaunchBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) {
    *msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
    return BINATTN_ERR_CUDA;
  }
  dim3 grid((N + 2 * kRows - 1) / (2 * kRows), B * H);
  kern<<<grid, kThreads, smem, st>>>(prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    *msg = std::string("fwd_tc_kernel launch: ") + cudaGetErrorString(e);
    return BINATTN_ERR_CUDA;
  }
  return BINATTN_OK;
}

template <bool kTcQK, bool kBias, bool kDump>
inline int dispatch_kdim(const Params& prm, int B, int H, int N, int d, cudaStream_t st,
                         std::string* msg) {
  switch ((d + 15) / 16) {
    case 1: return launch_tc<16, kTcQK, kBias, kDump>(prm, B, H, N, st, msg);
    case 2: return launch_tc<32, kTcQK, kBias, kDump>(prm, B, H, N, st, msg);
    case 3: return launch_tc<48, kTcQK, kBias, kDump>(prm, B, H, N, st, msg);
    case 4: return launch_tc<64, kTcQK, kBias, kDump>(prm, B, H, N, st, msg);
    case 5: return launch_tc<80, kTcQK, kBias, kDump>(prm, B, H, N, st, msg);
    case 6: return launch_tc<96, kTcQK, kBias, kDump>(prm, B, H, N, st, msg);
    case 7: return launch_tc<112, kTcQK, kBias, kDump>(prm, B, H, N, st, msg);
    default: return launch_tc<128, kTcQK, kBias, kDump>(prm, B, H, N, st, msg);
  }
}

}  // namespace tc

inline int forward_tc(bool tc_qk, const uint32_t* qb, const uint32_t* kb, const float* aq,
                      const float* ak, const uint16_t* bias, const uint16_t* v, float scale,
                      int B, int H, int N, int d, uint16_t* out, cudaStream_t st, std::string* msg) {
  tc::Params prm{qb, kb, aq, ak, bias, v, out, nullptr, scale, H, N, d};
  if (tc_qk)
    return bias ? tc::dispatch_kdim<true, true, false>(prm, B, H, N, d, st, msg)
                : tc::dispatch_kdim<true, false, false>(prm, B, H, N, d, st, msg);
  return bias ? tc::dispatch_kdim<false, true, false>(prm, B, H, N, d, st, msg)
              : tc::dispatch_kdim<false, false, false>(prm, B, H, N, d, st, msg);
}

inline int scores_tc(const uint32_t* qb, const uint32_t* kb, int B, int H, int N, int d, int32_t* S,
                     cudaStream_t st, std::string* msg) {
  tc::Params prm{qb, kb, nullptr, nullptr, nullptr, nullptr, nullptr, S, 0.f, H, N, d};
  return tc::dispatch_kdim<true, false, true>(prm, B, H, N, d, st, msg);
}

inline int forward_ref_bf16(const uint16_t*, const uint16_t*, const uint16_t*, const uint16_t*, float,
                            int, int, int, int, uint16_t*, cudaStream_t, std::string* msg) {
  *msg = "bf16 reference not built yet";
  return BINATTN_ERR_UNSUPPORTED;
}

}  // namespace binattn
