// fwd_tc3.cuh — the binary forward with 128-key tiles (e4m3 +-1 operands for
// QK^T). It serves the forward without a bias, where it measured as fast as
// the 64-key pipeline of fwd_tc2.cuh or a little faster.
//
// Source: "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
// Transformers", §2 methodology (scaled binary Q/K, XNOR/popcount similarity,
// additive learnable bias, softmax, P.V) and the hardware-aware implementation
// bullet (FlashAttention2-style tiling). The tiling below is new for sm_100a.
//
// Shapes: d % 8 == 0, d <= 80; with a bias the row stride of the bias is a
// multiple of 8 elements (the bias rows are TMA rows). One CTA (12 warps, one
// per SM) owns 256 query rows of one (b, h) as two 128-row tiles t = 0, 1 and
// streams the keys in tiles of 128:
//   warps 0-7  softmax: warps 4t..4t+3 for tile t, one thread per query row
//              (TMEM lane).
//   warp 8, 9  MMA issuers, one thread each: warp 8 + t issues for tile t.
//   warp 10    TMA: V and the bias boxes (two 64-key boxes per tile), and L2
//              prefetches of the bias two key tiles ahead.
//   warp 11    expands the key sign words to e4m3 +-1 operand rows and stages
//              alpha_k, with the loads two tiles ahead.
// A warpgroup register split (setmaxnreg) gives the softmax warps 216
// registers, enough for the 128 fp32 logits of a row.
//
// Shared memory holds Q_t as an e4m3 +-1 operand (pad channels 0), written
// once by the softmax threads; with Params::qh set they binarise bf16 Q
// themselves (pack_row_bf16, the same code and order as binattn_pack).
//
// Tensor memory, 256 columns per tile t (base 256 t):
//   S_t  [0, 128)        fp32 scores of the current key tile; part A of P_t
//                         (bf16 pairs, keys 2c and 2c + 1 in column c, the
//                         first KA keys) overwrites its first KA / 2 columns;
//   O_t  [128, 128 + DV) fp32 accumulator, DV >= d + 1 (column d holds l);
//   P_B  [128 + DV, 256) part B of P_t: the remaining KB keys (96 for d <= 72).
//
// One score buffer per tile. The issuer of tile t runs, per key tile kt:
//   1. waits for the operands of tile kt + 1;
//   2. O_t += P_A V once part A is published;
//   3. S_t = Q_t K(kt + 1)^T into S_t right behind it (one thread's MMAs run
//      in issue order, and part B is not in S_t);
//   4. O_t += P_B V once part B is published.
// So the turnaround from P to the next scores overlaps the exps of part B.
// Because QK^T(kt) is issued after P.V part A of kt - 1, the scores' commit
// proves that part complete; part B's own commit (pb_free) covers the rest
// before O_t is rescaled or P_B is rewritten.
//
// Softmax per row, fp32: logit = (S alpha_k)(scale alpha_q) + bias; the tile
// max is settled before any exp; the running max m moves only when the tile max
// exceeds it by more than 8 ln 2, and then O_t (with l in column d) is
// rescaled; P = exp(logit - m) rounded to bf16. The two tiles take turns on
// their part-A exp phases through named barriers 3 and 4. Channel d of every V
// stage is 1.0, so O_t column d sums the bf16 P actually multiplied. The
// epilogue divides O by l and writes bf16 (or, for a split key half, the
// unnormalised partials that combine_halves_kernel joins).
//
// Every mbarrier wait is bounded (sm100::mbar_wait); on a timeout the CTA
// records a device status code, leaves its loops, waits for its own MMAs and
// frees its tensor memory.
#pragma once
#include "fwd_tc2.cuh"

namespace binattn {
namespace tc3 {

using namespace sm100;
using tc2::e4m3_bytes;
using tc2::e4m3_nibble;
using tc2::idesc_e4m3;
using tc2::max3f;
using tc2::named_arrive;
using tc2::named_sync;
using tc2::tmem_ld8;

constexpr int kRows = 128;    // query rows per tile (MMA M)
constexpr int kKeys = 128;    // keys per tile (QK MMA N, P.V K)
constexpr int kHalf = 64;     // keys per bias box (a 128B-swizzled box spans 64 bf16 keys)
constexpr int kSoftmaxPerTile = 128;
constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
constexpr int kSoftmaxWarps = 8;
constexpr int kMmaWarp0 = 8;
constexpr int kTmaWarp = 10;
constexpr int kExpandWarp = 11;
constexpr int kTmemCols = 512;
constexpr int kLaunchRegs = 168;   // __launch_bounds__(384, 1): 65536 / 384, rounded down to 8
constexpr int kSoftmaxRegs = 216;  // warps 0-7 after the split
constexpr int kOtherRegs = 72;     // warps 8-11 after the split
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs, "register split");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 5.545177444479562f;  // 8 ln 2

constexpr int kModeBin = 0;   // binary forward
constexpr int kModeDump = 2;  // binary scores only (debug): the same QK^T, S written to global memory

inline bool supported(int d, int N, bool with_bias, int bias_ld = 0) {
  if (d % 8 != 0 || d > 80) return false;
  if (with_bias && (bias_ld > 0 ? bias_ld : N) % 8 != 0) return false;
  return true;
}

// Shared-memory map (byte offsets).
//  bias [kBS][2 t][2 halves] boxes of 128 rows x 64 keys bf16, 128B swizzle
//       (16 KB): key k of row r at r * 128 + ((k / 8) ^ (r % 8)) * 16 + (k % 8) * 2.
//  K    [kKS] binary: 128 keys x 32W e4m3, K-major, no swizzle: 16-byte chunk
//       (key j, channel group c of 16) at (j / 8) * (8 * 32W) + c * 128 + (j % 8) * 16
//       -> LBO = 128, SBO = 8 * 32W. Reference: one TMA box of 8 channels x
//       128 keys per group: chunk (key j, group c of 8) at c * 2048 + j * 16
//       -> LBO = 2048, SBO = 128.
//  V    [kKS] 128 keys x DV bf16, MN-major: chunk (key j, group g of 8) at
//       g * 2048 + j * 16 -> LBO = 128 (next 8 keys), SBO = 2048 (next 8 channels).
//  ak   [kKS] 128 fp32.
template <int DV, int kMode, bool kBias>
struct Layout {
  static constexpr int kBS = 2;
  static constexpr int kBiasBox = kRows * 64 * 2;  // 16 KB
  static constexpr int kKTile = kKeys * 96;
  static constexpr int kQTile = kRows * 96;  // e4m3 Q operand of one 128-row tile
  static constexpr int kVTile = kKeys * DV * 2;
  static constexpr int kBiasBytes = kBias ? kBS * 2 * 2 * kBiasBox : 0;
  // as many K / V stages (up to 4) as fit beside the bias stages and Q in 227 KB
  static constexpr int kStageBytes = kKTile + kVTile + kKeys * 4;
  static constexpr int kKSFit = (227 * 1024 - kBiasBytes - 2 * kQTile - 512) / kStageBytes;
  static constexpr int kKS = kKSFit > 4 ? 4 : kKSFit;
  static constexpr int kBiasOff = 0;
  static constexpr int kQ = kBiasOff + kBiasBytes;
  static constexpr int kK = kQ + 2 * kQTile;
  static constexpr int kV = kK + kKS * kKTile;
  static constexpr int kAk = kV + kKS * kVTile;
  static constexpr int kBar = kAk + kKS * kKeys * 4;
  static constexpr int kNumBars = 32;
  static constexpr int kMisc = kBar + 8 * kNumBars;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kLaunchBytes = kBytes > 120 * 1024 ? kBytes : 120 * 1024;
  // Tensor-memory columns of a tile: S [0, 128), O [128, 128 + DV), P part B
  // from kPB0 to the end of the tile's 256 columns.
  static constexpr int kPB0 = 128 + DV;
  // keys of part B (P in its own columns), a multiple of 16, at most 96; part
  // A (P over the first S columns) takes the rest
  static constexpr int kKB = (2 * (256 - kPB0)) / 16 * 16 > 96 ? 96 : (2 * (256 - kPB0)) / 16 * 16;
  static constexpr int kKA = kKeys - kKB;
};

// D[tmem] (+)= A[smem] * B[smem], e4m3 operands (kind::f8f6f4).
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16-byte shared-memory loads, kept in program order (the chunked logits
// issue the next chunk's loads before the current chunk's arithmetic).
__device__ __forceinline__ float4 lds_f4(const float* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ uint4 lds_u4(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p)));
  return v;
}

// P = exp(logit - m) of keys [K0, K1) of a row, rounded to bf16 pairs (keys
// K0 + 2c and K0 + 2c + 1 in column c from col): every exp is computed before
// the first store, so the exp unit is fed without a break.
template <int K0, int K1>
__device__ __forceinline__ void exps_part(const float* x, float m, uint32_t col) {
  constexpr int kCols = (K1 - K0) / 2;
  static_assert(kCols % 8 == 0, "whole 8-column stores");
  const float2 l2e2 = make_float2(kLog2e, kLog2e);
  const float2 nm2 = make_float2(-m * kLog2e, -m * kLog2e);
  uint32_t pk[kCols];
#pragma unroll
  for (int e = 0; e < kCols; ++e) {
    const float2 a = __ffma2_rn(make_float2(x[K0 + 2 * e], x[K0 + 2 * e + 1]), l2e2, nm2);
    pk[e] = pack_bf16x2(ex2(a.x), ex2(a.y));
  }
  constexpr int k32 = kCols / 32 * 32;
  constexpr int k16 = (kCols - k32) / 16 * 16;
#pragma unroll
  for (int c = 0; c < k32; c += 32) tmem_st32(col + c, pk + c);
  if constexpr (k16 > 0) tmem_st16(col + k32, pk + k32);
  if constexpr (kCols - k32 - k16 > 0) tmem_st8(col + k32 + k16, pk + k32 + k16);
}

template <int DV, int kMode, bool kBias>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc3_kernel(const tc::Params p, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_bias) {
  using L = Layout<DV, kMode, kBias>;
  constexpr int kKS = L::kKS, kBS = L::kBS;
  static_assert(DV % 16 == 0 && DV <= 96, "P.V N");
  static_assert(kMode == kModeBin || kMode == kModeDump, "binary forward or its scores");
  constexpr bool kDump = kMode == kModeDump;
  static_assert(L::kKA >= 16 && L::kKB >= 16, "both parts of P hold keys");
  static_assert(kKS >= 2 && kKS <= 4 && kBS <= 2, "stages / barrier slots");

  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars + 0;    // [kKS] V (+ reference K) landed; binary: K expanded, alpha_k staged
  uint64_t* kv_empty = bars + 4;   // [kKS] both issuers' commits after the tile's P.V
  uint64_t* b_full = bars + 8;     // [kBS][2 t] both bias boxes of (stage, t) landed
  uint64_t* b_empty = bars + 12;   // [kBS][2 t] the 128 softmax threads of t read them
  uint64_t* s_full = bars + 16;    // [2 t] QK^T commit + issuer arrive -> softmax t
  uint64_t* pa_full = bars + 20;   // [2 t] softmax t published P part A (over S)
  uint64_t* pb_full = bars + 22;   // [2 t] softmax t published P part B
  uint64_t* pb_free = bars + 24;   // [2 t] commit of P.V part B: its columns are free, O is whole
  uint64_t* o_done = bars + 26;    // [2 t] commit of the last P.V
  uint64_t* drain = bars + 28;     // [2 t] error path and teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 256-row pair of this CTA (b fastest, then the query tile, then h): the B
  // CTAs that read the same bias rows run next to one another.
  const int nq = (p.N + 2 * kRows - 1) / (2 * kRows);
  const int pidx = p.pair_base + (p.split ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x));
  const int half = p.split ? static_cast<int>(blockIdx.x & 1) : 0;
  const int b = pidx % p.B;
  const int qt = (pidx / p.B) % nq;
  const int h = pidx / (p.B * nq);
  const int bh = b * p.H + h;
  const int N = p.N, d = p.d;
  const int W = (d + 31) / 32;
  const size_t tok0 = static_cast<size_t>(bh) * N;
  const int q0 = qt * 2 * kRows;
  const int nkt_all = (N + kKeys - 1) / kKeys;
  const int kt_begin = p.split && half ? nkt_all / 2 : 0;
  const int nkt = p.split ? (half ? nkt_all - nkt_all / 2 : nkt_all / 2) : nkt_all;
  const int key0 = kt_begin * kKeys;
  const int dgroups = d / 8;

  // ---------------------------------------------------------------- setup
  {
    // Channels >= d of every V stage (never written by TMA): channel d is 1.0
    // (the row-sum column), the rest 0. Reference K: pad channels 0.
    const int npad = (DV / 8 - dgroups) * kKeys;
    for (int e = threadIdx.x; e < kKS * npad; e += kThreads) {
      const int s = e / npad, rem = e % npad;
      const int g = dgroups + rem / kKeys, kk = rem % kKeys;
      *reinterpret_cast<uint4*>(smem + L::kV + s * L::kVTile + g * 2048 + kk * 16) =
          make_uint4(g == dgroups ? 0x3F80u : 0u, 0u, 0u, 0u);
    }
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKS; ++s) {
      mbar_init(&kv_full[s], kDump ? 32 : 33);  // the expander's lanes (+ the V copy's arrive)
      mbar_init(&kv_empty[s], 2);
    }
    for (int i = 0; i < kBS * 2; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], kSoftmaxPerTile);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 2);  // the QK^T commit + the issuer's arrive (operands, bias landed)
      mbar_init(&pa_full[i], kSoftmaxPerTile);
      mbar_init(&pb_full[i], kSoftmaxPerTile);
      mbar_init(&pb_free[i], 1);
      mbar_init(&o_done[i], 1);
      mbar_init(&drain[i], 1);
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int t = warp >> 2;
  const int r = ((warp & 3) << 5) | lane;
  const int row = q0 + t * kRows + r;
  const bool row_valid = warp < kSoftmaxWarps && row < N;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  float aq_row = 0.f;  // alpha_q of this thread's row
  if (warp < kSoftmaxWarps) {
    // Q_t operand row r in shared memory, e4m3 +-1 with pad channels (>= d)
    // 0, K-major like K: 16-byte chunk (row r, channel group c of 16) at
    // (r / 8) * (8 * 32W) + c * 128 + (r % 8) * 16.
    uint8_t* qrow = smem + L::kQ + t * L::kQTile + (r >> 3) * (8 * 32 * W) + (r & 7) * 16;
    uint32_t qw[3] = {0u, 0u, 0u};
    if (row_valid) {
      if (p.qh) {
        pack_row_bf16_w(p.qh + (tok0 + row) * d, d, W, qw, aq_row);  // Q binarised here
      } else {
        for (int w = 0; w < W; ++w) qw[w] = p.qb[(tok0 + row) * W + w];
        if (!kDump) aq_row = p.aq[tok0 + row];  // the score dump has no alphas
      }
    }
    for (int w = 0; w < W; ++w) {
      const uint32_t word = w == 0 ? qw[0] : w == 1 ? qw[1] : qw[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint4 v4;
        v4.x = row_valid ? e4m3_bytes(word, 16 * h2 + 0, 32 * w + 16 * h2 + 0, d, true) : 0u;
        v4.y = row_valid ? e4m3_bytes(word, 16 * h2 + 4, 32 * w + 16 * h2 + 4, d, true) : 0u;
        v4.z = row_valid ? e4m3_bytes(word, 16 * h2 + 8, 32 * w + 16 * h2 + 8, d, true) : 0u;
        v4.w = row_valid ? e4m3_bytes(word, 16 * h2 + 12, 32 * w + 16 * h2 + 12, d, true) : 0u;
        *reinterpret_cast<uint4*>(qrow + (2 * w + h2) * 128) = v4;
      }
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  tc_fence_after();

  // Register split: the launch gives every thread kLaunchRegs; warpgroup 2
  // (issuers, TMA, expander) returns registers and the two softmax
  // warpgroups take them: 2 * 128 * kSoftmaxRegs + 128 * kOtherRegs equals
  // the launch's 384 * kLaunchRegs, so the increase always finds its registers.
  // Each role runs inside its warpgroup's branch, so that the compiler knows
  // the register budget of every instruction.
  if (warp >= kSoftmaxWarps) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
   if (warp == kTmaWarp) {
    // ------------------------------------ V (and reference K), bias boxes
    if (lane == 0 && !kDump) {
      bool ok = true;
      for (int kt = 0; ok && kt < nkt; ++kt) {
        const int j0 = key0 + kt * kKeys;
        const int s = kt % kKS;
        if (kt >= kKS && !(ok = mbar_wait(&kv_empty[s], ((kt / kKS) - 1) & 1, abort))) break;
        mbar_arrive_expect_tx(&kv_full[s], static_cast<uint32_t>(dgroups * 2048));
        for (int g = 0; g < dgroups; ++g)
          tma_load_3d(smem + L::kV + s * L::kVTile + g * 2048, &tm_v, 8 * g, j0, bh, &kv_full[s]);
        if constexpr (kBias) {
          // the bias rows of tile kt + 2 into L2 now, so that their TMA loads
          // (issued once a stage frees) do not wait on HBM
          if (kt + 2 < nkt) {
            for (int t2 = 0; t2 < 2; ++t2) {
              tma_prefetch_l2_3d(&tm_bias, j0 + 2 * kKeys, q0 + t2 * kRows, h);
              tma_prefetch_l2_3d(&tm_bias, j0 + 2 * kKeys + kHalf, q0 + t2 * kRows, h);
            }
          }
          for (int t2 = 0; t2 < 2; ++t2) {
            const int i = (kt % kBS) * 2 + t2;
            if (kt >= kBS && !(ok = mbar_wait(&b_empty[i], ((kt / kBS) - 1) & 1, abort))) break;
            mbar_arrive_expect_tx(&b_full[i], 2 * L::kBiasBox);
            uint8_t* dst = smem + L::kBiasOff + i * 2 * L::kBiasBox;
            tma_load_3d(dst, &tm_bias, j0, q0 + t2 * kRows, h, &b_full[i]);
            tma_load_3d(dst + L::kBiasBox, &tm_bias, j0 + kHalf, q0 + t2 * kRows, h, &b_full[i]);
          }
        }
      }
    }
  } else if (warp == kExpandWarp) {
    // ------------------- binary: key sign words -> e4m3 +-1 rows, alpha_k
    {
      const int kb_row = 32 * W;  // operand bytes per key
      struct TileRegs {
        uint32_t wd[4][3];
        float ak[4];
      };
      auto load_tile = [&](int kt, TileRegs& tr) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int key = key0 + kt * kKeys + lane + 32 * u;
          const bool in = kt < nkt && key < N;
#pragma unroll
          for (int w = 0; w < 3; ++w) tr.wd[u][w] = (in && w < W) ? __ldg(p.kb + (tok0 + key) * W + w) : 0u;
          tr.ak[u] = (!kDump && in) ? __ldg(p.ak + tok0 + key) : 0.f;  // the score dump has no alphas
        }
      };
      TileRegs cur, n1;
      load_tile(0, cur);
      load_tile(1, n1);
      for (int kt = 0; kt < nkt; ++kt) {
        TileRegs n2;
        load_tile(kt + 2, n2);
        const int s = kt % kKS;
        const bool ok = kt < kKS || mbar_wait(&kv_empty[s], ((kt / kKS) - 1) & 1, abort);
        if (!__all_sync(0xffffffffu, ok)) break;
        uint8_t* ks = smem + L::kK + s * L::kKTile;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int rr = lane + 32 * u;
          uint8_t* dst = ks + (rr >> 3) * (8 * kb_row) + (rr & 7) * 16;
#pragma unroll
          for (int c = 0; c < 6; ++c) {
            if (c < 2 * W) {
              const uint32_t hw = cur.wd[u][c >> 1] >> (16 * (c & 1));
              *reinterpret_cast<uint4*>(dst + c * 128) =
                  make_uint4(e4m3_nibble(hw), e4m3_nibble(hw >> 4), e4m3_nibble(hw >> 8), e4m3_nibble(hw >> 12));
            }
          }
        }
        float* aks = reinterpret_cast<float*>(smem + L::kAk) + s * kKeys;
#pragma unroll
        for (int u = 0; u < 4; ++u) aks[lane + 32 * u] = cur.ak[u];
        fence_proxy_async_smem();
        mbar_arrive(&kv_full[s]);
        cur = n1;
        n1 = n2;
      }
    }
  } else {
    // ----------------------------------------------- MMA issuer of tile tt
    const int tt = warp - kMmaWarp0;
    if (lane == 0) {
      constexpr int KA = L::kKA, KB = L::kKB;
      constexpr uint32_t kIdPV = idesc_bf16(kRows, DV, true);
      const uint32_t kb_sbo = static_cast<uint32_t>(8 * 32 * W);
      const uint32_t q_base = smem_u32(smem + L::kQ + tt * L::kQTile);
      const uint32_t base_t = tmem + 256 * tt;
      // S_tt = Q_tt K(kt)^T: both operands K-major e4m3 in shared memory
      auto issue_qk = [&](int kt, uint32_t idesc) {
        const uint32_t k_base = smem_u32(smem + L::kK + (kt % kKS) * L::kKTile);
        for (int ks = 0; ks < W; ++ks)
          mma_ss_f8(base_t, smem_desc(q_base + ks * 256, 128, kb_sbo), smem_desc(k_base + ks * 256, 128, kb_sbo),
                    idesc, ks > 0);
      };
      constexpr uint32_t kIdAll = idesc_e4m3(kRows, kKeys);
      // Tile kt's operands and softmax inputs are in shared memory (the K / V
      // stage with alpha_k and, with a bias, both bias boxes of this tile):
      // the issuer waits for them and arrives on s_full itself, so the
      // softmax threads' single wait on s_full covers them all.
      auto stage_ready = [&](int kt) {
        if (!mbar_wait(&kv_full[kt % kKS], (kt / kKS) & 1, abort)) return false;
        if (kBias && !mbar_wait(&b_full[(kt % kBS) * 2 + tt], (kt / kBS) & 1, abort)) return false;
        mbar_arrive(&s_full[tt]);
        tc_fence_after();
        return true;
      };
      bool ok = stage_ready(0);
      if (ok) {
        issue_qk(0, kIdAll);
        mma_commit(&s_full[tt]);
      }
      for (int kt = 0; ok && kt < nkt; ++kt) {
        const int s = kt % kKS;
        const bool more = kt + 1 < nkt;
        const uint32_t v_base = smem_u32(smem + L::kV + s * L::kVTile);
        // the operands of tile kt + 1, checked before P(kt) is awaited
        if (more && !(ok = stage_ready(kt + 1))) break;
        // O_tt += P_A V(keys 0 .. KA): P part A over S columns [0, KA / 2)
        if (!(ok = mbar_wait(&pa_full[tt], kt & 1, abort))) break;
        tc_fence_after();
        if constexpr (!kDump) {
          for (int ks = 0; ks < KA / 16; ++ks)
            mma_ts(base_t + 128, base_t + ks * 8, smem_desc(v_base + ks * 256, 128, 2048), kIdPV,
                   (kt > 0 || ks > 0));
        }
        // then QK^T(kt + 1) over all of S: part A of P has been read (the
        // tensor pipe runs this thread's MMAs in order) and part B is elsewhere
        if (more) {
          issue_qk(kt + 1, kIdAll);
          mma_commit(&s_full[tt]);
        }
        // O_tt += P_B V(keys KA .. 128): P part B in its own columns
        if (!(ok = mbar_wait(&pb_full[tt], kt & 1, abort))) break;
        tc_fence_after();
        if constexpr (!kDump) {
          for (int ks = 0; ks < KB / 16; ++ks)
            mma_ts(base_t + 128, base_t + L::kPB0 + ks * 8, smem_desc(v_base + (KA / 16 + ks) * 256, 128, 2048),
                   kIdPV, 1u);
        }
        mma_commit(&kv_empty[s]);  // this issuer's last use of stage s
        mma_commit(&pb_free[tt]);
        if (!more) mma_commit(&o_done[tt]);
      }
      {  // wait (bounded) for every MMA of this thread before TMEM is freed
        mma_commit(&drain[tt]);
        volatile int never = 0;
        mbar_wait(&drain[tt], 0, &never);
      }
    }
    __syncwarp();
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ---------------------------------------------------------------- softmax
    constexpr int KA = L::kKA;
    const float ci = row_valid ? p.scale * aq_row : 0.f;
    const uint32_t s_col = tmem + lane_base + 256 * t;
    const uint32_t o_col = s_col + 128;
    const int r7 = r & 7;
    float m = -INFINITY;
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
    };

    if constexpr (kDump) {
      // Scores only: every tile's S is loaded, written out as integers and
      // both parts are handed back at once. As in the forward, part B of
      // tile kt is handed on only after the issuer's part-B commit of tile
      // kt - 1, so these threads never run two phases ahead of its waits.
      for (int kt = 0; kt < nkt; ++kt) {
        if (ok) ok = wait_all(&s_full[t], kt & 1);
        tc_fence_after();
        if (ok) {
          uint32_t xr[kKeys];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(s_col + 32 * c, xr + 32 * c);
          tmem_ld_wait();
          tc_fence_before();
          if (row_valid) {
            const int jt = key0 + kt * kKeys;
            int32_t* srow = p.S + (tok0 + row) * N + jt;
#pragma unroll
            for (int e = 0; e < kKeys; ++e)
              if (jt + e < N) srow[e] = static_cast<int32_t>(__uint_as_float(xr[e]));
          }
          mbar_arrive(&pa_full[t]);
          if (kt > 0) ok = wait_all(&pb_free[t], (kt - 1) & 1);
          if (ok) mbar_arrive(&pb_full[t]);
        }
        ok = __all_sync(0xffffffffu, ok);
      }
    } else {
    // The loop runs every key tile even after an error (with the work
    // skipped), so that each thread takes its part in every named barrier.
    if (t == 1) named_arrive(3, 2 * kSoftmaxPerTile);  // tile 0 takes the first exp turn
    for (int kt = 0; kt < nkt; ++kt) {
      const int s = kt % kKS;
      const int bs = kt % kBS;
      float x[kKeys];
      // scores, alpha_k and the bias boxes of kt (see the issuer's stage_ready)
      if (ok) ok = wait_all(&s_full[t], kt & 1);
      tc_fence_after();
      if (ok) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_col + 32 * c, reinterpret_cast<uint32_t*>(x + 32 * c));
        tmem_ld_wait();
        // logits: S * alpha_k * (scale * alpha_q) + bias, in chunks of 32 keys;
        // the shared-memory inputs of chunk c + 1 are loaded before chunk c is
        // computed, so their latency overlaps the arithmetic
        const uint8_t* bsm = smem + L::kBiasOff + (bs * 2 + t) * 2 * L::kBiasBox + r * 128;
        const float* aks = reinterpret_cast<const float*>(smem + L::kAk) + s * kKeys;
        const float2 ci2 = make_float2(ci, ci);
        struct ChunkIn {
          float4 ak[8];
          uint4 bias[4];
        };
        auto load_chunk = [&](int c, ChunkIn& in) {
#pragma unroll
          for (int i = 0; i < 8; ++i) in.ak[i] = lds_f4(aks + 32 * c + 4 * i);
          if constexpr (kBias) {
            // box c / 2 holds keys 64 (c / 2) ..; 16-byte units 4 (c % 2) + q of this row
#pragma unroll
            for (int q = 0; q < 4; ++q)
              in.bias[q] = lds_u4(bsm + (c >> 1) * L::kBiasBox + (((4 * (c & 1) + q) ^ r7) << 4));
          }
        };
        auto logits_chunk = [&](int c, const ChunkIn& in) {
          float2* xs = reinterpret_cast<float2*>(x + 32 * c);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t rw[4] = {in.bias[q].x, in.bias[q].y, in.bias[q].z, in.bias[q].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 bv = kBias ? make_float2(__uint_as_float(rw[e] << 16), __uint_as_float(rw[e] & 0xFFFF0000u))
                                      : make_float2(0.f, 0.f);
              float2& xv = xs[4 * q + e];
              const float4 a4 = in.ak[2 * q + (e >> 1)];
              const float2 av = (e & 1) ? make_float2(a4.z, a4.w) : make_float2(a4.x, a4.y);
              xv = __ffma2_rn(__fmul2_rn(xv, av), ci2, bv);
            }
          }
        };
        ChunkIn in0, in1;
        load_chunk(0, in0);
        load_chunk(1, in1);
        logits_chunk(0, in0);
        load_chunk(2, in0);
        logits_chunk(1, in1);
        load_chunk(3, in1);
        logits_chunk(2, in0);
        logits_chunk(3, in1);
        if (kBias) mbar_arrive(&b_empty[bs * 2 + t]);  // bias boxes read
        const int jt = key0 + kt * kKeys;
        if (jt + kKeys > N) {  // keys >= N take no part (warp-uniform branch)
#pragma unroll
          for (int e = 0; e < kKeys; ++e)
            if (jt + e >= N) x[e] = -INFINITY;
        }
        // tile max: four independent 3-input max chains
        float mc[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float* xf = x + 32 * c;
          float a = max3f(xf[0], xf[1], xf[2]);
#pragma unroll
          for (int e = 3; e < 31; e += 2) a = max3f(a, xf[e], xf[e + 1]);
          mc[c] = fmaxf(a, xf[31]);
        }
        const float tmax = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
        // Lazy rescale: m moves only when the tile max exceeds it by more than
        // kRescale; until then every p = exp(logit - m) <= 2^8, and the final
        // division by l (summed against the same m) cancels the offset. O_t
        // is whole once P.V part B of tile kt - 1 has completed (part A's
        // completion precedes this tile's scores).
        const bool grow = tmax > m + kRescale;
        if (__any_sync(0xffffffffu, grow)) {
          const float m_new = grow ? tmax : m;
          const float corr = grow ? ex2((m - m_new) * kLog2e) : 1.f;  // 0 while m is -inf
          if (kt > 0 && (ok = wait_all(&pb_free[t], (kt - 1) & 1))) {
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < DV; cc += 16) {
              uint32_t ov[16];
              tmem_ld16(o_col + cc, ov);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
              tmem_st16(o_col + cc, ov);
            }
          }
          m = m_new;
        }
      }
      // Exp token: the part-A exp phases of the two tiles alternate (named
      // barriers 3 and 4 over both tiles' softmax threads), so one tile's
      // exps run while the other waits for its scores and computes its logits.
      // Every iteration passes the token exactly once, also after an error.
      named_sync(3 + t, 2 * kSoftmaxPerTile);
      const bool ok_at_a = ok;
      if (ok) {
        // part A over S columns [0, KA / 2): P.V of it and the rest of the
        // next QK^T can start while part B is computed
        exps_part<0, KA>(x, m, s_col);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&pa_full[t]);
        // the token passes once part A is out: the other tile's exps overlap
        // this tile's part B and the wait for its next scores
        if (!(t == 1 && kt == nkt - 1)) named_arrive(4 - t, 2 * kSoftmaxPerTile);
        // part B into its own columns, free once P.V part B of tile kt - 1 is done
        if (kt > 0) ok = wait_all(&pb_free[t], (kt - 1) & 1);
        tc_fence_after();
        if (ok) {
          exps_part<KA, kKeys>(x, m, s_col + L::kPB0);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&pb_full[t]);
        }
      }
      if (!ok_at_a && !(t == 1 && kt == nkt - 1)) named_arrive(4 - t, 2 * kSoftmaxPerTile);  // error path
    }
    if (ok && wait_all(&o_done[t], 0)) {
      tc_fence_after();
      uint32_t lbits;  // l = O_t column d
      asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(lbits) : "r"(o_col + d));
      tmem_ld_wait();
      if (p.split) {
        // Partial result of this key half: unnormalised O (d fp32), then m,
        // then l, channel-major: value c of row r256 of (pair slot, half) at
        // ((slot * 2 + half) * (d + 2) + c) * 256 + r256.
        const int r256 = t * kRows + r;
        float* dst = p.part + static_cast<size_t>((pidx - p.pair_base) * 2 + half) * (d + 2) * (2 * kRows) + r256;
        for (int cc = 0; cc < d; cc += 8) {  // warp-uniform trip count: the loads are collective
          uint32_t ov[8];
          tmem_ld8(o_col + cc, ov);
          tmem_ld_wait();
          if (row_valid) {
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[(cc + e) * (2 * kRows)] = __uint_as_float(ov[e]);
          }
        }
        if (row_valid) {
          dst[d * (2 * kRows)] = m;
          dst[(d + 1) * (2 * kRows)] = __uint_as_float(lbits);
        }
      } else {
        const float inv = 1.f / __uint_as_float(lbits);
        uint16_t* orow = p.out + (tok0 + row) * d;
#pragma unroll
        for (int cc = 0; cc < DV; cc += 16) {
          if (cc < d) {  // warp-uniform
            uint32_t ov[16];
            tmem_ld16(o_col + cc, ov);
            tmem_ld_wait();
            if (row_valid) {
#pragma unroll
              for (int e = 0; e < 16; e += 8) {
                if (cc + e < d) {
                  uint4 o4;
                  o4.x = pack_bf16x2(__uint_as_float(ov[e + 0]) * inv, __uint_as_float(ov[e + 1]) * inv);
                  o4.y = pack_bf16x2(__uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
                  o4.z = pack_bf16x2(__uint_as_float(ov[e + 4]) * inv, __uint_as_float(ov[e + 5]) * inv);
                  o4.w = pack_bf16x2(__uint_as_float(ov[e + 6]) * inv, __uint_as_float(ov[e + 7]) * inv);
                  *reinterpret_cast<uint4*>(orow + cc + e) = o4;
                }
              }
            }
          }
        }
      }
    }
    }  // the forward (not kDump)
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------- host
// V as boxes of 8 channels x 128 keys (tc::make_rows_map).
inline bool make_rows_map(CUtensorMap* tm, const uint16_t* base, cuuint64_t BH, cuuint64_t N, cuuint64_t d,
                          const char* what, std::string* msg) {
  return tc::make_rows_map(tc::encode_fn(), tm, base, BH, N, d, what, msg, kKeys);
}

template <int DV, int kMode, bool kBias>
inline int launch(const tc::Params& prm, int ctas, cudaStream_t st, std::string* msg) {
  CUtensorMap tm_v, tm_bias;
  std::memset(&tm_v, 0, sizeof tm_v);
  std::memset(&tm_bias, 0, sizeof tm_bias);
  const cuuint64_t BH = static_cast<cuuint64_t>(prm.B) * prm.H;
  if (kMode != kModeDump && !make_rows_map(&tm_v, prm.v, BH, prm.N, prm.d, "V", msg)) return BINATTN_ERR_CUDA;
  if (kBias && !tc2::make_bias_map(&tm_bias, prm.bias, prm.H, prm.N, prm.bias_ld > 0 ? prm.bias_ld : prm.N, msg))
    return BINATTN_ERR_CUDA;
  auto kern = fwd_tc3_kernel<DV, kMode, kBias>;
  constexpr int smem = Layout<DV, kMode, kBias>::kLaunchBytes;
  static_assert(smem <= 227 * 1024, "shared memory over the sm_100 per-CTA limit");
  static std::atomic<uint64_t> configured{0};  // set-up once per device
  if (needs_setup(configured)) {
    // The register split assumes the launch gives kLaunchRegs per thread: with
    // fewer, the softmax warpgroups' setmaxnreg.inc could not be satisfied.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) {
      *msg = std::string("cudaFuncGetAttributes: ") + cudaGetErrorString(e);
      return BINATTN_ERR_CUDA;
    }
    if (fa.numRegs != kLaunchRegs) {
      *msg = "fwd_tc3_kernel built with " + std::to_string(fa.numRegs) + " registers per thread, not " +
             std::to_string(kLaunchRegs) + ": the register split would not fit";
      return BINATTN_ERR_CUDA;
    }
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) {
      *msg = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
      return BINATTN_ERR_CUDA;
    }
    mark_setup(configured);
  }
  kern<<<static_cast<unsigned>(ctas), kThreads, smem, st>>>(prm, tm_v, tm_bias);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *msg = std::string("fwd_tc3_kernel launch: ") + cudaGetErrorString(e);
    return BINATTN_ERR_CUDA;
  }
  return BINATTN_OK;
}

template <int kMode, bool kBias>
inline int dispatch_dv(const tc::Params& prm, int ctas, cudaStream_t st, std::string* msg) {
  switch (tc2::dv_for(prm.d)) {
    case 32: return launch<32, kMode, kBias>(prm, ctas, st, msg);
    case 64: return launch<64, kMode, kBias>(prm, ctas, st, msg);
    case 80: return launch<80, kMode, kBias>(prm, ctas, st, msg);
    default: return launch<96, kMode, kBias>(prm, ctas, st, msg);
  }
}

}  // namespace tc3

// Integer scores S [B,H,N,N] as the 128-key pipeline computes them (its QK^T
// with Q and K both e4m3 in shared memory), for d % 8 == 0, d <= 80.
inline int scores_tc3(const uint32_t* qb, const uint32_t* kb, int B, int H, int N, int d, int32_t* S,
                      cudaStream_t st, std::string* msg) {
  tc::Params prm{qb, kb, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, S, 0.f, B, H, N, d, 0, 0, 0,
                 nullptr};
  return tc3::launch<32, tc3::kModeDump, false>(prm, tc2::total_pairs(B, H, N), st, msg);
}

// Binary forward on the 128-key pipeline. part: workspace for the tail split
// (tc2::split_part_bytes), or null for no split. The split plan, the partial
// layout and the combine kernel are those of the 64-key pipeline.
// qh: bf16 Q for a forward that binarises Q itself (qb, aq then unused), or null.
inline int forward_tc3(const uint32_t* qb, const uint32_t* kb, const float* aq, const float* ak,
                       const uint16_t* bias, const uint16_t* v, float scale, int B, int H, int N, int d,
                       uint16_t* out, cudaStream_t st, std::string* msg, int bias_ld = 0,
                       float* part = nullptr, const uint16_t* qh = nullptr) {
  tc::Params prm{qb, kb, nullptr, nullptr, aq, ak, bias, v, out, nullptr, scale, B, H, N, d, bias_ld, 0, 0,
                 nullptr, qh};
  auto run = [&](int ctas) {
    return bias ? tc3::dispatch_dv<tc3::kModeBin, true>(prm, ctas, st, msg)
                : tc3::dispatch_dv<tc3::kModeBin, false>(prm, ctas, st, msg);
  };
  // one pair per CTA (this pipeline has no persistent loop)
  return tc2::run_pairs(prm, part, false, run, st, msg);
}

}  // namespace binattn
