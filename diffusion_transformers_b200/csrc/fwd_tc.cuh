// fwd_tc.cuh — tensor-core engines of binattn_forward (TC and POPC_TC), the
// debug-scores kernel of the TC engine, and the bf16 reference attention.
//
// Source: "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
// Transformers", §2 methodology: scaled binary Q/K, XNOR/popcount similarity,
// additive learnable bias, softmax, P.V; FlashAttention2-style tiling from the
// hardware-aware implementation bullet. The tiling here is new for sm_100a.
//
// One CTA (12 warps, one per SM) owns 256 query rows of one (b, h) as two
// 128-row tiles t = 0, 1 and streams the keys in tiles of 64:
//   warps 0-7   softmax: warpgroup t (warps 4t..4t+3), thread = one query row.
//   warp 8      MMA issuer (one thread): tcgen05.mma, tcgen05.commit.
//   warps 9-11  loaders, in one of two modes:
//     TMA mode (KDIM <= 80, N % 8 == 0): warp 9 issues TMA / bulk copies of V
//       and alpha_k (and of the sign words for POPC_TC, of K for the reference);
//       warp 10 issues the bias tiles, each as soon as its stage is free;
//       warp 11 loads the key sign words and expands them to +-1 bf16 operand
//       tiles (TC engine). Q_t lives in tensor memory next to O_t.
//     load mode (other shapes): warps 9-11 load the same data with batched
//       plain loads; Q_t lives in shared memory; softmax threads read the bias.
//
// Tensor memory, 256 columns per warpgroup t (base 256t): two score buffers
// S_t^0, S_t^1 (64 fp32 columns each), O_t (KDIM columns) at +128 and, in TMA
// mode, Q_t (KDIM/2 columns of bf16 pairs) at +128+KDIM. P_t of key tile kt is
// written back as bf16 pairs over the first 32 columns of S_t^(kt%2). With two
// score buffers the MMA warp issues S_t(kt+2) = Q_t K(kt+2)^T right after
// O_t += P_t(kt) V(kt), so the scores of the next tile are ready while the
// softmax threads still work on the current one.
//
// TC engine: S_t = Q_t K^T on the tensor core with +-1 bf16 operands. Pad
// channels of Q are 0, so every product is +-1 or 0 and the fp32 accumulator
// holds the exact integer score d - 2 popcount(q XOR k).
// POPC_TC engine: the softmax threads compute S with __popc over the packed
// words (binary_score); the tensor core does P.V only.
//
// Softmax (per row, fp32, online over key tiles): logit = (S * alpha_k) *
// (scale * alpha_q) + bias; running max m and sum l; O_t in TMEM is rescaled
// only when the tile max exceeds m by more than 8 (log2 units); P =
// exp(logit - m) rounded to bf16 for the P.V MMA; the epilogue divides by l and
// writes bf16.
//
// Every mbarrier wait is bounded (sm100::mbar_wait); on a timeout the CTA
// records a device status code, leaves its loops, waits for its own MMAs and
// frees its tensor memory.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cstring>
#include <mutex>
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
constexpr int kKeys = 64;        // keys per tile (QK MMA N, PV MMA K)
constexpr int kKS = 4;           // stages of the K / V / alpha_k / sign-word ring
constexpr int kBS = 3;           // stages of the bias ring (per warpgroup)
constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp0 = 9;
constexpr int kLoadThreads = 96;     // load mode: warps 9-11
constexpr int kBiasWarp = 10;        // TMA mode: bias tile issuer
constexpr int kExpandWarp0 = 11;     // TMA mode: warp 11 expands signs
constexpr int kExpandThreads = 32;
constexpr int kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 5.545177444479562f;  // 8 * ln 2: rescale O only past 2^8

__host__ __device__ constexpr bool tma_mode_kdim(int kdim) { return kdim <= 80; }

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}

// Shared-memory map (byte offsets).
//  Q_t (load mode) 128 rows x KDIM bf16, K-major, no swizzle: 16-byte chunk
//           (row r, channel group c) at (r / 8) * (KDIM * 16) + c * 128 + (r % 8) * 16
//           -> descriptor LBO = 128 (next channel group), SBO = KDIM * 16 (next 8 rows).
//  K_s     64 keys x KDIM bf16. Binary: the same layout as Q_t. Reference:
//           chunk (key j, channel group c) at c * 1024 + j * 16 (one TMA box of
//           8 channels x 64 keys per group) -> LBO = 1024, SBO = 128.
//  V_s     64 keys x KDIM bf16, MN-major, no swizzle: chunk (key j, d group g)
//           at g * 1024 + j * 16 (one TMA box per group)
//           -> LBO = 128 (next 8 keys), SBO = 1024 (next 8 d values).
//  bias    (TMA mode) per stage and warpgroup: 128 rows x 64 keys bf16 as one
//           128B-swizzled box: key k of row r at r * 128 + ((k / 8) ^ (r % 8)) * 16 + (k % 8) * 2.
//  kb_s    sign words of the tile's keys, contiguous: key j word w at j * W + w.
template <int KDIM, bool kTma>
struct Layout {
  static constexpr int kQTile = kRows * KDIM * 2;
  static constexpr int kKTile = kKeys * KDIM * 2;
  static constexpr int kBiasTile = kRows * kKeys * 2;            // 16 KB
  static constexpr int kLut = 0;                                 // 256 x 16 B
  static constexpr int kQ = 4096;                                // load mode: 2 Q tiles
  static constexpr int kK = kQ + (kTma ? 0 : 2 * kQTile);        // kKS tiles
  static constexpr int kV = kK + kKS * kKTile;                   // kKS tiles
  static constexpr int kBias = (kV + kKS * kKTile + 1023) / 1024 * 1024;  // TMA: [kBS][2]
  static constexpr int kAk = kBias + (kTma ? kBS * 2 * kBiasTile : 0);   // kKS x 64 fp32
  static constexpr int kKb = kAk + kKS * kKeys * 4;              // kKS x 64 x 4 words
  static constexpr int kBar = kKb + kKS * kKeys * 16;
  static constexpr int kNumBars = 64;
  static constexpr int kMisc = kBar + 8 * kNumBars;              // tmem base, abort flag
  static constexpr int kBytes = kMisc + 16;
  // at least this much, so that one CTA occupies an SM (each CTA allocates all
  // 512 TMEM columns)
  static constexpr int kLaunchBytes = kBytes > 120 * 1024 ? kBytes : 120 * 1024;
};

struct Params {
  const uint32_t* qb;
  const uint32_t* kb;
  const uint16_t* q;  // bf16 reference attention: Q [B,H,N,d]
  const uint16_t* k;  // bf16 reference attention: K [B,H,N,d]
  const float* aq;
  const float* ak;
  const uint16_t* bias;
  const uint16_t* v;
  uint16_t* out;
  int32_t* S;  // debug scores (dump mode)
  float scale;
  int B, H, N, d;
  int bias_ld;  // elements between bias rows (N, or the padded row length); 0 means N
  // 64-key TMA-fed pipeline only: CTAs cover 256-row pairs pair_base + blockIdx.x
  // (split == 0), or, with split == 1, CTA 2i + h covers key half h of pair
  // pair_base + i and writes partial results to `part`.
  int pair_base;
  int split;
  float* part;
  // bf16 Q [B,H,N,d] for a forward that binarises Q itself (TMA-fed pipelines
  // only): each row's sign words and alpha_q come from pack_row_bf16 in the
  // kernel, and qb / aq are not read. Null: qb / aq from binattn_pack.
  const uint16_t* qh = nullptr;
  // Test only (the entry point that makes a bounded wait run out): with
  // stall_after >= 0 the TMA producer of the 64-key pipeline issues nothing
  // from key tile stall_after on, so the stage's consumers time out.
  int stall_after = -1;
  // 8-bit P.V (64-key pipeline): V's per-channel 8-bit code in the tiled
  // operand layout (quantv.cuh), its scales [B,H,d], and the exact row max of
  // the logits [B,H,N] (written by the row-max pass, read by the 8-bit pass).
  const int8_t* vq8 = nullptr;
  const float* vscale = nullptr;
  float* mrow = nullptr;
  // Position-sensitive bias (64-key pipeline): the relative-position table
  // bf16 [H, rel_R] of a rel_gh x rel_gw patch grid after rel_ncls (0 or 1)
  // class tokens, rel_R = (2 gh - 1)(2 gw - 1) + 3 ncls.
  const uint16_t* rel_table = nullptr;
  int rel_gh = 0, rel_gw = 0, rel_ncls = 0, rel_R = 0;
  // 64-key pipeline without split: the launch covers pairs pair_base ..
  // pair_base + npairs - 1, CTA c taking c, c + gridDim.x, ... (a persistent
  // launch of fewer CTAs than pairs); 0: one pair per CTA.
  int npairs = 0;
  // 64-key pipeline, dense bias: 1 when each batch entry has its own bias
  // [B, H, N rows] (a context-aware bias, computed per sample), read at row
  // (b * H + h) * N + i; 0 when the batch shares one bias [H, N rows].
  int bias_per_sample = 0;
};

// Named barrier 1 over the load-mode loader warps with an AND reduction.
__device__ __forceinline__ bool loaders_all(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "n"(kLoadThreads)
      : "memory");
  return r != 0;
}

// Score sources (template parameter kQK).
constexpr int kQkPopc = 0;  // __popc in the softmax threads (POPC_TC engine)
constexpr int kQkTc = 1;    // tcgen05.mma on +-1 operands expanded from sign bits (TC engine)
constexpr int kQkRef = 2;   // tcgen05.mma on bf16 Q, K: full-precision reference attention

template <int KDIM, bool kTma, int kQK, bool kBias, bool kDump>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const Params p, const __grid_constant__ CUtensorMap tm_v,
              const __grid_constant__ CUtensorMap tm_ak, const __grid_constant__ CUtensorMap tm_bias,
              const __grid_constant__ CUtensorMap tm_k) {
  constexpr bool kTcQK = kQK != kQkPopc;  // QK^T on the tensor core
  constexpr bool kRef = kQK == kQkRef;
  constexpr uint32_t kKLbo = kRef ? 1024 : 128;
  constexpr uint32_t kKSbo = kRef ? 128 : KDIM * 16;
  using L = Layout<KDIM, kTma>;
  constexpr int W = (KDIM + 31) / 32;  // packed words per token (= ceil(d / 32))
  constexpr int KCH = KDIM / 8;        // 16-byte channel groups per operand row
  constexpr uint32_t kIdescQK = idesc_bf16(kRows, kKeys, false);
  constexpr uint32_t kIdescPV = idesc_bf16(kRows, KDIM, true);
  static_assert(!kTma || tma_mode_kdim(KDIM), "TMA mode keeps Q in TMEM: KDIM <= 80");
  static_assert(KCH % 2 == 0, "KDIM is a multiple of 16");

  extern __shared__ __align__(1024) uint8_t smem[];
  uint4* lut = reinterpret_cast<uint4*>(smem + L::kLut);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars + 0;     // [kKS] V + alpha_k (+ load mode: K, sign words)
  uint64_t* kv_empty = bars + 4;    // [kKS] MMA commit after the stage's P.V
  uint64_t* kb_full = bars + 8;     // [kKS] TMA mode POPC_TC: sign-word bulk copy
  uint64_t* k_full = bars + 12;     // [kKS] TMA mode: K operand ready
  uint64_t* k_empty = bars + 16;    // [kKS] TMA mode: MMA commit after the stage's QK
  uint64_t* b_full = bars + 20;     // [kBS * 2] bias tile landed (stage, t)
  uint64_t* b_empty = bars + 26;    // [kBS * 2] warpgroup t done with the bias tile
  uint64_t* s_full = bars + 32;     // [2 t][2 buf] QK commit -> softmax t
  uint64_t* p_full = bars + 36;     // [2 t][2 buf] softmax t (128 arrivals) -> MMA
  // [2 t][2 buf] PV commit -> softmax t. Two barriers per warpgroup (by tile
  // parity) so that every wait has at most one phase in flight: with double-
  // buffered scores the softmax can be two tiles ahead of P.V, and a single
  // barrier's parity would then be ambiguous.
  uint64_t* o_done = bars + 40;
  uint64_t* drain = bars + 44;      // error path only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Batch entries sharing a bias tile (same h and query tile) are adjacent in
  // launch order, so the bias tile is fetched from HBM once.
  const int b = blockIdx.x % p.B;
  const int qt = blockIdx.x / p.B;
  const int h = blockIdx.y;
  const int bh = b * p.H + h;
  const int N = p.N, d = p.d;
  const size_t tok0 = static_cast<size_t>(bh) * N;
  const int q0 = qt * 2 * kRows;
  const int nkt = (N + kKeys - 1) / kKeys;
  const int dgroups = d / 8;

  // ---------------------------------------------------------------- setup
  // LUT: 8 sign bits -> 8 bf16 values, element e = +1.0 if bit e is set, else -1.0.
  for (int i = threadIdx.x; i < 256; i += kThreads) {
    uint32_t w[4];
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      const uint32_t lo = ((i >> (2 * pr)) & 1) ? 0x3F80u : 0xBF80u;
      const uint32_t hi = ((i >> (2 * pr + 1)) & 1) ? 0x3F80u : 0xBF80u;
      w[pr] = lo | (hi << 16);
    }
    lut[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if constexpr (kTma && !kDump) {
    // Pad groups (g >= d / 8) of V (and of the reference K) are never written
    // by TMA: zero them once so that no stale shared memory enters an MMA.
    const int npad = (KCH - dgroups) * kKeys;
    for (int e = threadIdx.x; e < kKS * npad; e += kThreads) {
      const int s = e / npad, rem = e % npad;
      const int g = dgroups + rem / kKeys, kk = rem % kKeys;
      *reinterpret_cast<uint4*>(smem + L::kV + s * L::kKTile + g * 1024 + kk * 16) = make_uint4(0, 0, 0, 0);
      if (kRef)
        *reinterpret_cast<uint4*>(smem + L::kK + s * L::kKTile + g * 1024 + kk * 16) = make_uint4(0, 0, 0, 0);
    }
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKS; ++s) {
      mbar_init(&kv_full[s], kTma ? 1 : kLoadThreads);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&kb_full[s], 1);
      mbar_init(&k_full[s], kRef ? 1 : kExpandThreads);
      mbar_init(&k_empty[s], 1);
    }
    for (int i = 0; i < kBS * 2; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], kRows);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kRows);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&o_done[i], 1);
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
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Softmax threads: this thread's query row and its operand row of Q_t.
  const int t = warp >> 2;                      // warpgroup (valid for warps 0-7)
  const int r = ((warp & 3) << 5) | lane;       // row within the tile = TMEM lane
  const int row = q0 + t * kRows + r;
  const bool row_valid = warp < 8 && row < N;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  uint32_t qw[W];
#pragma unroll
  for (int w = 0; w < W; ++w) qw[w] = (!kRef && row_valid) ? p.qb[(tok0 + row) * W + w] : 0u;
  // Channel group c (8 channels, 16 bytes) of this row's Q operand row.
  auto q_group = [&](int c) -> uint4 {
    uint4 val = make_uint4(0, 0, 0, 0);  // pad channels (>= d) are 0
    if (8 * c < d) {
      if constexpr (kRef) {
        if (row_valid) val = *reinterpret_cast<const uint4*>(p.q + (tok0 + row) * d + 8 * c);
      } else {
        val = lut[(qw[c >> 2] >> (8 * (c & 3))) & 0xFFu];
      }
    }
    return val;
  };
  if (kTcQK && warp < 8) {
    if constexpr (kTma) {
      // Q_t row in TMEM at column 256t + 128 + KDIM: column c2 holds channels
      // 2*c2 (low half) and 2*c2 + 1.
      const uint32_t qcol = tmem + lane_base + 256 * t + 128 + KDIM;
#pragma unroll
      for (int c = 0; c < KCH; c += 2) {
        uint32_t wv[8];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const uint4 val = q_group(c + h2);
          wv[4 * h2 + 0] = val.x;
          wv[4 * h2 + 1] = val.y;
          wv[4 * h2 + 2] = val.z;
          wv[4 * h2 + 3] = val.w;
        }
        tmem_st8(qcol + 4 * c, wv);
      }
      tmem_st_wait();
      tc_fence_before();
    } else {
      uint8_t* qs = smem + L::kQ + t * L::kQTile;
#pragma unroll
      for (int c = 0; c < KCH; ++c)
        *reinterpret_cast<uint4*>(qs + (r >> 3) * (KDIM * 16) + c * 128 + (r & 7) * 16) = q_group(c);
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  tc_fence_after();

  if (warp >= kLoadWarp0) {
    if constexpr (kTma) {
      if (warp == kLoadWarp0) {
        // --------------------------------- V / alpha_k (/ K, sign words) issuer
        if (lane == 0) {
          for (int kt = 0; kt < nkt; ++kt) {
            const int s = kt % kKS;
            const uint32_t ph_prev = ((kt / kKS) - 1) & 1;
            const int j0 = kt * kKeys;
            const int nk = min(kKeys, N - j0);
            // Stage s is free once tile kt - kKS is done with it: its QK MMAs
            // (reference K) and its P.V MMAs (V, alpha_k, and for POPC_TC the
            // sign words read by the softmax threads before P was published).
            if (kt >= kKS) {
              if (kRef && !mbar_wait(&k_empty[s], ph_prev, abort)) break;
              if (!kDump && !mbar_wait(&kv_empty[s], ph_prev, abort)) break;
            }
            if constexpr (kRef) {  // bf16 K: one box of 8 channels x 64 keys per group
              mbar_arrive_expect_tx(&k_full[s], dgroups * 1024);
              for (int g = 0; g < dgroups; ++g)
                tma_load_3d(smem + L::kK + s * L::kKTile + g * 1024, &tm_k, 8 * g, j0, bh, &k_full[s]);
            } else if constexpr (!kTcQK) {
              // POPC_TC: sign words for the softmax threads, nk keys x W words,
              // contiguous and 16-byte aligned (N % 8 == 0). (For TC the
              // expander warp loads the words itself.)
              const uint32_t nbytes = static_cast<uint32_t>(nk * W * 4);
              mbar_arrive_expect_tx(&kb_full[s], nbytes);
              bulk_load(smem + L::kKb + s * kKeys * 16, p.kb + (tok0 + j0) * W, nbytes, &kb_full[s]);
            }
            if constexpr (!kDump) {
              mbar_arrive_expect_tx(&kv_full[s], dgroups * 1024 + (kRef ? 0 : kKeys * 4));
              for (int g = 0; g < dgroups; ++g)
                tma_load_3d(smem + L::kV + s * L::kKTile + g * 1024, &tm_v, 8 * g, j0, bh, &kv_full[s]);
              if (!kRef) tma_load_2d(smem + L::kAk + s * kKeys * 4, &tm_ak, j0, bh, &kv_full[s]);
            }
          }
        }
        __syncwarp();
      } else if (warp == kBiasWarp) {
        // ------------------------------------------------ bias issuer (one thread)
        // The bias tile (128 rows x 64 keys of warpgroup t) is the largest
        // stream; each is requested as soon as warpgroup t released the stage.
        if (kBias && !kDump && lane == 0) {
          for (int kt = 0; kt < nkt; ++kt) {
            const int bs = kt % kBS;
            bool ok = true;
            for (int tt = 0; tt < 2; ++tt) {
              uint64_t* bf = &b_full[bs * 2 + tt];
              if (kt >= kBS && !(ok = mbar_wait(&b_empty[bs * 2 + tt], ((kt / kBS) - 1) & 1, abort)))
                break;
              mbar_arrive_expect_tx(bf, L::kBiasTile);
              tma_load_3d(smem + L::kBias + (bs * 2 + tt) * L::kBiasTile, &tm_bias, kt * kKeys,
                          q0 + tt * kRows, h, bf);
            }
            if (!ok) break;
          }
        }
        __syncwarp();
      } else if (kTcQK && !kRef) {
        // ------------------------------------------------ sign expander warp
        // Thread et owns keys et and et + 32 of every tile: it loads their sign
        // words itself (the next tile's words are in flight while it waits for
        // the stage) and writes their +-1 rows; consecutive threads write
        // consecutive keys, which keeps the 16-byte stores conflict-free.
        constexpr int kPer = kKeys / kExpandThreads;
        const int et = threadIdx.x - kExpandWarp0 * 32;
        uint32_t wd[kPer][W];
        auto load_words = [&](int kt) {
#pragma unroll
          for (int u = 0; u < kPer; ++u) {
            const int key = kt * kKeys + et + u * kExpandThreads;
#pragma unroll
            for (int w = 0; w < W; ++w) wd[u][w] = key < N ? p.kb[(tok0 + key) * W + w] : 0u;
          }
        };
        load_words(0);
        for (int kt = 0; kt < nkt; ++kt) {
          const int s = kt % kKS;
          if (kt >= kKS && !mbar_wait(&k_empty[s], ((kt / kKS) - 1) & 1, abort)) break;
          uint8_t* ks = smem + L::kK + s * L::kKTile;
#pragma unroll
          for (int u = 0; u < kPer; ++u) {
            const int kk = et + u * kExpandThreads;
#pragma unroll
            for (int c = 0; c < KCH; ++c) {
              uint4 val = make_uint4(0, 0, 0, 0);
              if (8 * c < d) val = lut[(wd[u][c >> 2] >> (8 * (c & 3))) & 0xFFu];
              *reinterpret_cast<uint4*>(ks + (kk >> 3) * (KDIM * 16) + c * 128 + (kk & 7) * 16) = val;
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(&k_full[s]);
          if (kt + 1 < nkt) load_words(kt + 1);
        }
      }
    } else {
      // -------------------------------------------- loaders (load mode)
      // Per key tile: (A) issue every global load of the tile at once (sign
      // words, alpha_k, V, reference K), (B) store them into the stage, (C, TC)
      // once all loaders have stored, expand the sign words to +-1 bf16.
      const int pt = threadIdx.x - kLoadWarp0 * 32;
      constexpr int kKbIters = (kKeys * W + kLoadThreads - 1) / kLoadThreads;
      constexpr int kAkIters = (kKeys + kLoadThreads - 1) / kLoadThreads;
      constexpr int kVIters = (kKeys * KCH + kLoadThreads - 1) / kLoadThreads;
      for (int kt = 0; kt < nkt; ++kt) {
        const int s = kt % kKS;
        // All 96 loaders agree (barrier with AND reduction) so that either all
        // reach the named barrier below or all leave the loop.
        const bool ok = kt < kKS || mbar_wait(&kv_empty[s], ((kt / kKS) - 1) & 1, abort);
        if (!loaders_all(ok)) break;
        const int j0 = kt * kKeys;
        const int nk = min(kKeys, N - j0);
        uint32_t kbuf[kKbIters];
#pragma unroll
        for (int it = 0; it < kKbIters; ++it) {
          const int e = pt + it * kLoadThreads;
          kbuf[it] = (!kRef && e < nk * W) ? p.kb[(tok0 + j0) * W + e] : 0u;
        }
        float abuf[kAkIters];
        uint4 vbuf[kDump ? 1 : kVIters];
        uint4 krow[kRef ? kVIters : 1];
        if constexpr (!kDump) {  // the debug-scores variant gets no alpha_k / V
#pragma unroll
          for (int it = 0; it < kAkIters; ++it) {
            const int kk = pt + it * kLoadThreads;
            abuf[it] = (!kRef && kk < nk) ? p.ak[tok0 + j0 + kk] : 0.f;
          }
#pragma unroll
          for (int it = 0; it < kVIters; ++it) {
            const int e = pt + it * kLoadThreads;
            const int kk = e / KCH, g = e % KCH;
            vbuf[it] = make_uint4(0, 0, 0, 0);
            if (kk < nk && g < dgroups)
              vbuf[it] = __ldg(reinterpret_cast<const uint4*>(p.v + (tok0 + j0 + kk) * d + 8 * g));
          }
        }
        if constexpr (kRef) {
#pragma unroll
          for (int it = 0; it < kVIters; ++it) {
            const int e = pt + it * kLoadThreads;
            const int kk = e / KCH, g = e % KCH;
            krow[it] = make_uint4(0, 0, 0, 0);
            if (kk < nk && g < dgroups)
              krow[it] = __ldg(reinterpret_cast<const uint4*>(p.k + (tok0 + j0 + kk) * d + 8 * g));
          }
        }
        uint32_t* kbs = reinterpret_cast<uint32_t*>(smem + L::kKb + s * kKeys * 16);
#pragma unroll
        for (int it = 0; it < kKbIters; ++it) {
          const int e = pt + it * kLoadThreads;
          if (e < kKeys * W) kbs[e] = kbuf[it];
        }
        if constexpr (!kDump) {
          float* aks = reinterpret_cast<float*>(smem + L::kAk) + s * kKeys;
#pragma unroll
          for (int it = 0; it < kAkIters; ++it) {
            const int kk = pt + it * kLoadThreads;
            if (kk < kKeys) aks[kk] = abuf[it];
          }
          uint8_t* vs = smem + L::kV + s * L::kKTile;
#pragma unroll
          for (int it = 0; it < kVIters; ++it) {
            const int e = pt + it * kLoadThreads;
            if (e < kKeys * KCH) {
              const int kk = e / KCH, g = e % KCH;
              *reinterpret_cast<uint4*>(vs + g * 1024 + kk * 16) = vbuf[it];
            }
          }
        }
        if constexpr (kRef) {
          uint8_t* ks = smem + L::kK + s * L::kKTile;
#pragma unroll
          for (int it = 0; it < kVIters; ++it) {
            const int e = pt + it * kLoadThreads;
            if (e < kKeys * KCH) {
              const int kk = e / KCH, g = e % KCH;
              *reinterpret_cast<uint4*>(ks + g * 1024 + kk * 16) = krow[it];
            }
          }
        }
        if constexpr (kTcQK && !kRef) {
          asm volatile("bar.sync 1, %0;" ::"n"(kLoadThreads) : "memory");  // stores of (B) done
          uint8_t* ks = smem + L::kK + s * L::kKTile;
#pragma unroll 4
          for (int e = pt; e < kKeys * KCH; e += kLoadThreads) {
            const int c = e / kKeys, kk = e % kKeys;  // consecutive threads: consecutive keys
            uint4 val = make_uint4(0, 0, 0, 0);
            if (8 * c < d) val = lut[(kbs[kk * W + (c >> 2)] >> (8 * (c & 3))) & 0xFFu];
            *reinterpret_cast<uint4*>(ks + (kk >> 3) * (KDIM * 16) + c * 128 + (kk & 7) * 16) = val;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&kv_full[s]);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_u32(smem + L::kQ);
      const uint32_t k_base = smem_u32(smem + L::kK);
      const uint32_t v_base = smem_u32(smem + L::kV);
      uint64_t* kready = kTma ? k_full : kv_full;  // "K operand of stage s is ready"
      // S_t^(kt%2) = Q_t K(kt)^T
      auto issue_qk = [&](int tt, int kt) {
        const int s = kt % kKS;
        const uint32_t s_tmem = tmem + 256 * tt + 64 * (kt & 1);
#pragma unroll
        for (int ks = 0; ks < KDIM / 16; ++ks) {
          const uint64_t bdesc = smem_desc(k_base + s * L::kKTile + ks * 2 * kKLbo, kKLbo, kKSbo);
          if constexpr (kTma) {
            mma_ts(s_tmem, tmem + 256 * tt + 128 + KDIM + ks * 8, bdesc, kIdescQK, ks > 0);
          } else {
            const uint64_t adesc = smem_desc(q_base + tt * L::kQTile + ks * 256, 128, KDIM * 16);
            mma_ss(s_tmem, adesc, bdesc, kIdescQK, ks > 0);
          }
        }
        mma_commit(&s_full[tt * 2 + (kt & 1)]);
      };
      bool ok = true;
      if constexpr (kTcQK) {
        for (int kt = 0; ok && kt < 2 && kt < nkt; ++kt) {
          if (!(ok = mbar_wait(&kready[kt % kKS], (kt / kKS) & 1, abort))) break;
          tc_fence_after();
          issue_qk(0, kt);
          issue_qk(1, kt);
          if (kTma) mma_commit(&k_empty[kt % kKS]);
        }
      }
      for (int kt = 0; ok && kt < nkt; ++kt) {
        const int s = kt % kKS;
        if (!kDump && (kTma || !kTcQK)) {  // V ready (load mode TC: implied by kready)
          if (!(ok = mbar_wait(&kv_full[s], (kt / kKS) & 1, abort))) break;
          tc_fence_after();
        }
        for (int tt = 0; tt < 2; ++tt) {
          if (!(ok = mbar_wait(&p_full[tt * 2 + (kt & 1)], (kt >> 1) & 1, abort))) break;
          tc_fence_after();
          if constexpr (!kDump) {
            // O_t += P_t(kt) V(kt): A = P from TMEM (32 columns of bf16 pairs)
#pragma unroll
            for (int ks = 0; ks < kKeys / 16; ++ks) {
              const uint64_t bdesc = smem_desc(v_base + s * L::kKTile + ks * 256, 128, 1024);
              mma_ts(tmem + 256 * tt + 128, tmem + 256 * tt + 64 * (kt & 1) + ks * 8, bdesc, kIdescPV,
                     (kt > 0 || ks > 0));
            }
            mma_commit(&o_done[tt * 2 + (kt & 1)]);
          }
          if (kTcQK && kt + 2 < nkt) {
            // S_t^(kt%2) is free again: P_t(kt) was consumed by the MMA just
            // issued (the tensor pipe executes in issue order).
            if (tt == 0) {
              if (!(ok = mbar_wait(&kready[(kt + 2) % kKS], ((kt + 2) / kKS) & 1, abort))) break;
              tc_fence_after();
            }
            issue_qk(tt, kt + 2);
            if (kTma && tt == 1) mma_commit(&k_empty[(kt + 2) % kKS]);
          }
        }
        mma_commit(&kv_empty[s]);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax
    // per-row factor of the logit: scale * alpha_q (binary) or scale (reference)
    const float ci = kRef ? p.scale : ((!kDump && row_valid) ? p.scale * p.aq[tok0 + row] : 0.f);
    const uint32_t o_col = tmem + lane_base + 256 * t + 128;
    const uint16_t* brow =
        (kBias && !kTma && row_valid) ? p.bias + (static_cast<size_t>(h) * N + row) * N : nullptr;
    const bool bias_vec = (N % 8) == 0;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // Waits are made warp-uniform: the tcgen05.ld/st below are warp-collective.
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
    };
    for (int kt = 0; kt < nkt; ++kt) {
      const int s = kt % kKS;
      const int buf = kt & 1;
      const int j0 = kt * kKeys;
      const uint32_t s_col = tmem + lane_base + 256 * t + 64 * buf;
      float2 xs[kKeys / 2];  // this row's 64 scores, then logits (8-byte aligned storage)
      float* x = reinterpret_cast<float*>(xs);
      if (!kRef && (!kDump || !kTma)) {  // alpha_k (and in load mode sign words) of stage s
        if (!(ok = wait_all(&kv_full[s], (kt / kKS) & 1))) break;
      }
      if constexpr (kTcQK) {
        if (!(ok = wait_all(&s_full[t * 2 + buf], (kt >> 1) & 1))) break;
        tc_fence_after();
        tmem_ld32(s_col, reinterpret_cast<uint32_t*>(x));
        tmem_ld32(s_col + 32, reinterpret_cast<uint32_t*>(x + 32));
        tmem_ld_wait();
      } else {
        if (kTma && !(ok = wait_all(&kb_full[s], (kt / kKS) & 1))) break;
        const uint32_t* kbs = reinterpret_cast<const uint32_t*>(smem + L::kKb + s * kKeys * 16);
#pragma unroll
        for (int c = 0; c < kKeys; ++c)
          x[c] = static_cast<float>(binary_score<W>(qw, kbs + c * W, d));
      }
      if constexpr (kDump) {
        if (row_valid) {
          int32_t* srow = p.S + (tok0 + row) * N + j0;
#pragma unroll
          for (int c = 0; c < kKeys; ++c)
            if (j0 + c < N) srow[c] = static_cast<int32_t>(x[c]);
        }
        tc_fence_before();
        mbar_arrive(&p_full[t * 2 + buf]);
        continue;
      }
      // logits = S * alpha_k * (scale * alpha_q) + bias (packed fp32 pairs)
      const float* aks = reinterpret_cast<const float*>(smem + L::kAk) + s * kKeys;
      const int bs = kt % kBS;
      const uint8_t* bsm = smem + L::kBias + (bs * 2 + t) * L::kBiasTile + r * 128;
      if (kBias && kTma) {
        if (!(ok = wait_all(&b_full[bs * 2 + t], (kt / kBS) & 1))) break;
      }
      const float2 ci2 = make_float2(ci, ci);
#pragma unroll
      for (int c0 = 0; c0 < kKeys; c0 += 8) {
        float2 bv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) bv[e] = make_float2(0.f, 0.f);
        if constexpr (kBias) {
          uint4 raw = make_uint4(0, 0, 0, 0);
          bool have = false;
          if constexpr (kTma) {
            raw = *reinterpret_cast<const uint4*>(bsm + (((c0 >> 3) ^ (r & 7)) << 4));
            have = true;
          } else if (row_valid) {
            if (bias_vec && j0 + c0 + 8 <= N) {
              raw = *reinterpret_cast<const uint4*>(brow + j0 + c0);
              have = true;
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                if (j0 + c0 + 2 * e < N) bv[e].x = bf16_bits_to_float(brow[j0 + c0 + 2 * e]);
                if (j0 + c0 + 2 * e + 1 < N) bv[e].y = bf16_bits_to_float(brow[j0 + c0 + 2 * e + 1]);
              }
            }
          }
          if (have) {
            const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              bv[e] = make_float2(__uint_as_float(rw[e] << 16), __uint_as_float(rw[e] & 0xFFFF0000u));
          }
        }
        if constexpr (kRef) {
#pragma unroll
          for (int e = 0; e < 4; ++e) xs[c0 / 2 + e] = __ffma2_rn(xs[c0 / 2 + e], ci2, bv[e]);
        } else {
          const float4 a0 = *reinterpret_cast<const float4*>(aks + c0);
          const float4 a1 = *reinterpret_cast<const float4*>(aks + c0 + 4);
          const float2 av[4] = {make_float2(a0.x, a0.y), make_float2(a0.z, a0.w),
                                make_float2(a1.x, a1.y), make_float2(a1.z, a1.w)};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            xs[c0 / 2 + e] = __ffma2_rn(__fmul2_rn(xs[c0 / 2 + e], av[e]), ci2, bv[e]);
        }
      }
      if (kBias && kTma) mbar_arrive(&b_empty[bs * 2 + t]);
      if (j0 + kKeys > N) {  // last tile: keys >= N take no part (warp-uniform branch)
#pragma unroll
        for (int c = 0; c < kKeys; ++c)
          if (j0 + c >= N) x[c] = -INFINITY;
      }
      // row max of the tile: four independent 3-input max chains
      float mx4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
      for (int c = 4; c < kKeys; c += 8) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          mx4[e] = max3f(mx4[e], x[c + e], x[c + 4 + e < kKeys ? c + 4 + e : c + e]);
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      // Lazy rescale: the running max m only moves when the tile max exceeds it
      // by more than kRescale (natural-log units, = 8 in log2 units). Until then
      // every p = exp(logit - m) <= 2^8, exact enough in fp32 and bf16, and the
      // final division by l (summed against the same m) cancels the offset.
      const bool grow = mx > m + kRescale;
      const float m_new = grow ? mx : m;
      const float corr = grow ? ex2((m - m_new) * kLog2e) : 1.f;  // 0 on the first tile
      // P.V of tile kt-1 done: needed before O_t is rescaled, and (POPC_TC)
      // before P_t(kt) overwrites the buffer that P.V of tile kt-2 read. (For
      // TC the tensor pipe order already guarantees the latter: S_t(kt) was
      // written after P.V of tile kt-2.) Completion of the previous phase of the
      // same barrier (tile kt-3) is known here, so the parity is unambiguous.
      auto wait_pv_prev = [&]() {
        return wait_all(&o_done[t * 2 + ((kt - 1) & 1)], ((kt - 1) >> 1) & 1);
      };
      if (!kTcQK && kt >= 2) {
        if (!(ok = wait_pv_prev())) break;
        tc_fence_after();
      }
      if (kt > 0 && __any_sync(0xffffffffu, grow)) {
        // O_t must hold P.V of tile kt-1 before it is rescaled; P.V of tile kt
        // cannot start before this warpgroup publishes P_t(kt).
        if (!(ok = wait_pv_prev())) break;
        tc_fence_after();
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
      l *= corr;
      m = m_new;
      // P = exp(logit - m) as bf16 pairs into TMEM over S_t^buf
      const float2 l2e2 = make_float2(kLog2e, kLog2e);
      const float2 nm2 = make_float2(-m * kLog2e, -m * kLog2e);
      float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
#pragma unroll
      for (int c0 = 0; c0 < kKeys; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 a = __ffma2_rn(xs[c0 / 2 + e], l2e2, nm2);
          pk[e] = pack_bf16x2(ex2(a.x), ex2(a.y));
          // l sums the bf16 P the P.V MMA multiplies, so that the weights of
          // O = (P V) / l sum to one exactly
          ls[e & 3] = __fadd2_rn(ls[e & 3], make_float2(__uint_as_float(pk[e] << 16),
                                                        __uint_as_float(pk[e] & 0xFFFF0000u)));
        }
        tmem_st16(s_col + c0 / 2, pk);
      }
      l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y) + (ls[2].x + ls[2].y) + (ls[3].x + ls[3].y);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t * 2 + buf]);
    }
    if constexpr (!kDump) {
      if (ok && wait_all(&o_done[t * 2 + ((nkt - 1) & 1)], ((nkt - 1) >> 1) & 1)) {
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

// ------------------------------------------------------------------- host
using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

struct TensorMaps {
  CUtensorMap v, ak, bias, k;
};

// One [BH][N][d] bf16 tensor as boxes of 8 channels x box_keys keys: each box
// is one column of 16-byte chunks of the no-swizzle operand layouts of the
// tensor-core pipelines. Keys >= N of the last tile are outside the box's
// (b, h) plane and read as 0. Every TMA-fed pipeline builds its V (and
// reference K) maps here.
inline bool make_rows_map(EncodeTiledFn enc, CUtensorMap* tm, const uint16_t* base, cuuint64_t BH,
                          cuuint64_t N, cuuint64_t d, const char* what, std::string* msg,
                          cuuint32_t box_keys = kKeys) {
  if (!enc) {
    *msg = "cuTensorMapEncodeTiled entry point unavailable";
    return false;
  }
  const cuuint32_t es[3] = {1, 1, 1};
  const cuuint64_t dims[3] = {d, N, BH};
  const cuuint64_t strides[2] = {d * 2, N * d * 2};
  const cuuint32_t box[3] = {8, box_keys, 1};
  CUresult rc = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (rc != CUDA_SUCCESS) {
    *msg = std::string("tensor map (") + what + ") rejected: " + std::to_string(rc);
    return false;
  }
  return true;
}

// Tensor maps of one call. Returns false (with a message) if the driver rejects one.
inline bool make_maps(const Params& p, bool with_bias, bool ref, TensorMaps* tm, std::string* msg) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    *msg = "cuTensorMapEncodeTiled entry point unavailable";
    return false;
  }
  const cuuint32_t es[3] = {1, 1, 1};
  const cuuint64_t BH = static_cast<cuuint64_t>(p.B) * p.H, N = p.N, d = p.d;
  if (!make_rows_map(enc, &tm->v, p.v, BH, N, d, "V", msg)) return false;
  if (ref) {
    if (!make_rows_map(enc, &tm->k, p.k, BH, N, d, "K", msg)) return false;
  } else {  // alpha_k [BH][N] fp32: box 64 keys
    const cuuint64_t dims[2] = {N, BH};
    const cuuint64_t strides[1] = {N * 4};
    const cuuint32_t box[2] = {kKeys, 1};
    CUresult rc = enc(&tm->ak, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(p.ak), dims,
                      strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                      CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (rc != CUDA_SUCCESS) { *msg = "tensor map (alpha_k) rejected: " + std::to_string(rc); return false; }
  }
  if (with_bias) {  // bias [H][N rows][N keys] bf16: box 64 keys x 128 rows, 128B swizzle
    const cuuint64_t dims[3] = {N, N, static_cast<cuuint64_t>(p.H)};
    const cuuint64_t strides[2] = {N * 2, N * N * 2};
    const cuuint32_t box[3] = {kKeys, kRows, 1};
    CUresult rc = enc(&tm->bias, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(p.bias),
                      dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (rc != CUDA_SUCCESS) { *msg = "tensor map (bias) rejected: " + std::to_string(rc); return false; }
  }
  return true;
}

template <int KDIM, bool kTma, int kQK, bool kBias, bool kDump>
inline int launch_tc(const Params& prm, const TensorMaps& tm, cudaStream_t st, std::string* msg) {
  auto kern = fwd_tc_kernel<KDIM, kTma, kQK, kBias, kDump>;
  constexpr int smem = Layout<KDIM, kTma>::kLaunchBytes;
  static_assert(smem <= 227 * 1024, "shared memory over the sm_100 per-CTA limit");
  static std::atomic<uint64_t> configured{0};  // attribute set once per device and instantiation
  if (needs_setup(configured)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) {
      *msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
      return BINATTN_ERR_CUDA;
    }
    mark_setup(configured);
  }
  dim3 grid(static_cast<unsigned>(prm.B * ((prm.N + 2 * kRows - 1) / (2 * kRows))), prm.H);
  kern<<<grid, kThreads, smem, st>>>(prm, tm.v, tm.ak, tm.bias, tm.k);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *msg = std::string("fwd_tc_kernel launch: ") + cudaGetErrorString(e);
    return BINATTN_ERR_CUDA;
  }
  return BINATTN_OK;
}

template <int KDIM, int kQK, bool kBias, bool kDump>
inline int launch_mode(const Params& prm, cudaStream_t st, std::string* msg) {
  TensorMaps tm;
  std::memset(&tm, 0, sizeof tm);
  if constexpr (tma_mode_kdim(KDIM)) {
    if (prm.N % 8 == 0) {
      std::string why;
      if (make_maps(prm, kBias, kQK == kQkRef, &tm, &why))
        return launch_tc<KDIM, true, kQK, kBias, kDump>(prm, tm, st, msg);
      std::memset(&tm, 0, sizeof tm);  // the driver refused a map: use the load mode
    }
  }
  return launch_tc<KDIM, false, kQK, kBias, kDump>(prm, tm, st, msg);
}

template <int kQK, bool kBias, bool kDump>
inline int dispatch_kdim(const Params& prm, cudaStream_t st, std::string* msg) {
  switch ((prm.d + 15) / 16) {
    case 1: return launch_mode<16, kQK, kBias, kDump>(prm, st, msg);
    case 2: return launch_mode<32, kQK, kBias, kDump>(prm, st, msg);
    case 3: return launch_mode<48, kQK, kBias, kDump>(prm, st, msg);
    case 4: return launch_mode<64, kQK, kBias, kDump>(prm, st, msg);
    case 5: return launch_mode<80, kQK, kBias, kDump>(prm, st, msg);
    case 6: return launch_mode<96, kQK, kBias, kDump>(prm, st, msg);
    case 7: return launch_mode<112, kQK, kBias, kDump>(prm, st, msg);
    default: return launch_mode<128, kQK, kBias, kDump>(prm, st, msg);
  }
}

}  // namespace tc

inline int forward_tc(bool tc_qk, const uint32_t* qb, const uint32_t* kb, const float* aq,
                      const float* ak, const uint16_t* bias, const uint16_t* v, float scale,
                      int B, int H, int N, int d, uint16_t* out, cudaStream_t st, std::string* msg) {
  tc::Params prm{qb, kb, nullptr, nullptr, aq, ak, bias, v, out, nullptr, scale, B, H, N, d, 0, 0, 0, nullptr};
  if (tc_qk)
    return bias ? tc::dispatch_kdim<tc::kQkTc, true, false>(prm, st, msg)
                : tc::dispatch_kdim<tc::kQkTc, false, false>(prm, st, msg);
  return bias ? tc::dispatch_kdim<tc::kQkPopc, true, false>(prm, st, msg)
              : tc::dispatch_kdim<tc::kQkPopc, false, false>(prm, st, msg);
}

inline int scores_tc(const uint32_t* qb, const uint32_t* kb, int B, int H, int N, int d, int32_t* S,
                     cudaStream_t st, std::string* msg) {
  tc::Params prm{qb,      kb,      nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, S,
                 0.f,     B,       H,       N,       d,       0,       0,       0,       nullptr};
  return tc::dispatch_kdim<tc::kQkTc, false, true>(prm, st, msg);
}

// Full-precision softmax attention on the same tile pipeline (the speed
// reference): S = Q K^T as a bf16 tcgen05.mma, logit = scale * S + bias.
inline int forward_ref_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* bias,
                            const uint16_t* v, float scale, int B, int H, int N, int d, uint16_t* out,
                            cudaStream_t st, std::string* msg) {
  tc::Params prm{nullptr, nullptr, q, k, nullptr, nullptr, bias, v, out, nullptr, scale, B, H, N, d, 0, 0, 0, nullptr};
  return bias ? tc::dispatch_kdim<tc::kQkRef, true, false>(prm, st, msg)
              : tc::dispatch_kdim<tc::kQkRef, false, false>(prm, st, msg);
}

}  // namespace binattn
