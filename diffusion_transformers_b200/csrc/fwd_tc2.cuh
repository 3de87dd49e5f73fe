// fwd_tc2.cuh — the TMA-fed forward pipeline with e4m3 +-1 operands for the
// binary QK^T: the binary forward (with a dense bias shared over the batch or
// one per batch entry, a relative-position table bias, or none), its 8-bit P.V
// passes, its debug-scores variant, and the bf16 reference attention on the
// same pipeline.
//
// Source: "BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
// Transformers", §2 methodology (scaled binary Q/K, XNOR/popcount similarity,
// additive learnable bias, softmax, P.V) and the hardware-aware implementation
// bullet (FlashAttention2-style tiling). The tiling below is new for sm_100a.
//
// Shapes: d % 8 == 0, d <= 80; with a bias also N % 8 == 0 (the bias rows are
// TMA rows). One CTA (12 warps, one per SM) owns 256 query rows of one (b, h)
// as two 128-row tiles t = 0, 1 and streams the keys in tiles of 64. A launch
// of fewer CTAs than such pairs (one per SM) is persistent: each CTA takes
// several pairs in turn, keeping its tensor memory and barriers, and its
// shared-memory rings run on from one pair's key tiles into the next's.
//   warps 0-7  softmax: warps 4t..4t+3 for tile t, one thread per query row
//              (TMEM lane).
//   warp 8, 9  MMA issuers, one thread each: warp 8 + t issues for tile t.
//   warp 10    TMA: V (and the bf16 K of the reference attention), bias tiles.
//   warp 11    binary engines: expands the key sign words to e4m3 +-1 operand
//              rows and stages alpha_k, loading both two tiles ahead.
//
// Tensor memory, 256 columns per warpgroup t (base 256t):
//   S_t^b  columns [64b, 64b + 64), b = 0, 1: fp32 scores of key tile kt with
//          kt % 2 == b; P_t(kt) is written back as bf16 pairs over the first
//          32 columns of S_t^b;
//   O_t    columns [128, 128 + DV): fp32 accumulator, DV = P.V MMA N >= d + 1;
//   Q_t    binary: e4m3 bytes, 4 channels per column, columns [224, 224 + 8W);
//          reference: bf16 pairs, columns [128 + DV, 128 + DV + DV/2).
// Channel d of V is 1 in every key row (the stage's pad channels are written
// once and never by TMA), so O_t column d accumulates the row sum l of the
// bf16 P actually multiplied, and every rescale of O rescales l with it.
//
// Issuer t, per key tile kt: once P_t(kt) is published, O_t += P_t(kt) V(kt);
// then S_t^b = Q_t K(kt+2)^T into the buffer just read (the tensor pipe runs
// one thread's MMAs in issue order), committed to s_full[t][b]. So the scores
// of tile kt+1 are ready while the softmax threads work on tile kt, and the
// commit of QK^T(kt+2) also proves P.V(kt) complete.
//
// Binary scores: Q and K bits become e4m3 +1.0 (0x38) / -1.0 (0xB8), pad
// channels of Q are 0, and the fp32 accumulator holds the exact integer
// d - 2 popcount(q XOR k) (kind::f8f6f4, K = 32 channels per MMA).
//
// Per pair the softmax threads stage Q_t (its sign words loaded one pair
// ahead) and hand it to the issuer through q_ready; the issuer then starts
// the pair's first two QK^T.
//
// Softmax per row, fp32, one thread per row: logit = (S alpha_k)
// (scale alpha_q) + bias; the tile's max is settled before any exp; the
// running max m moves only when the tile max exceeds it by more than 8 (log2
// units), and then O_t (with l) is rescaled; P = exp(logit - m) rounded to
// bf16. The two 128-row tiles take turns on their exp phases (named barriers),
// so one tile's exps overlap the other's logits. The epilogue divides O by l
// (column d) and writes bf16.
//
// Every mbarrier wait is bounded (sm100::mbar_wait); on a timeout the CTA
// records a device status code, leaves its loops, waits for its own MMAs and
// frees its tensor memory.
#pragma once
#include "fwd_tc.cuh"
#include "pack.cuh"

namespace binattn {
namespace tc2 {

using namespace sm100;

constexpr int kRows = 128;    // query rows per warpgroup (MMA M)
constexpr int kKeys = 64;     // keys per tile (QK MMA N, P.V K)
constexpr int kChunk = 32;    // keys per softmax chunk
constexpr int kSoftmaxWarps = 8;     // 4 per 128-row tile: one thread per row
constexpr int kSoftmaxPerTile = 128;  // softmax threads per 128-row tile
constexpr int kWarps = 12;
constexpr int kThreads = kWarps * 32;
constexpr int kMmaWarp0 = 8;  // warps 8, 9: MMA issuers for t = 0, 1
constexpr int kTmaWarp = 10;
constexpr int kExpandWarp = 11;
constexpr int kTmemCols = 512;
constexpr int kQColBin = 224;  // binary Q operand columns (<= 24)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 5.545177444479562f;  // 8 ln 2: rescale only past a 2^8 growth

// Score sources.
constexpr int kModeBin = 0;   // binary forward
constexpr int kModeRef = 1;   // bf16 reference attention
constexpr int kModeDump = 2;  // binary scores only (debug)
constexpr int kModeMax = 3;   // 8-bit P.V, first pass: the exact row max of the logits
constexpr int kModeI8 = 4;    // 8-bit P.V, second pass: u8 P (against that max) times s8 V

// Shapes this pipeline takes (the caller falls back to the load-mode pipeline otherwise).
// bias_ld: elements between bias rows (N, or a padded length; TMA needs % 8 == 0).
inline bool supported(int d, int N, bool with_bias, bool ref, int bias_ld = 0) {
  if (d % 8 != 0 || d > 80) return false;
  if (with_bias && (bias_ld > 0 ? bias_ld : N) % 8 != 0) return false;
  if (ref && d > 72) return false;  // Q_t of the reference needs DV/2 more columns
  return true;
}
// P.V N: a multiple of 16 with room for the ones channel d.
inline int dv_for(int d) { return d < 32 ? 32 : d < 64 ? 64 : d < 80 ? 80 : 96; }

// Shared-memory map (byte offsets).
//  bias   [kBS][2 t] 128 rows x 64 keys bf16 as one 128B-swizzled box (16 KB):
//         key k of row r at r * 128 + ((k / 8) ^ (r % 8)) * 16 + (k % 8) * 2.
//  K      [kKS] binary: 64 keys x 32W e4m3, K-major, no swizzle: 16-byte chunk
//         (key j, channel group c of 16) at (j / 8) * (8 * 32W) + c * 128 + (j % 8) * 16
//         -> LBO = 128, SBO = 8 * 32W. Reference: 64 keys x DV bf16, one TMA
//         box of 8 channels x 64 keys per group: chunk (key j, group c of 8)
//         at c * 1024 + j * 16 -> LBO = 1024, SBO = 128.
//  V      [kKS] 64 keys x DV bf16, MN-major: chunk (key j, group g of 8) at
//         g * 1024 + j * 16 -> LBO = 128 (next 8 keys), SBO = 1024 (next 8 channels).
//  ak     [kKS] 64 fp32.
// Bias kinds of the 64-key pipeline.
constexpr int kNoBias = 0;
constexpr int kDenseBias = 1;   // bf16 [H, N, N] (rows bias_ld apart), TMA boxes
constexpr int kRelPosBias = 2;     // relative-position table [H, R] gathered from shared memory
constexpr int kRelPosBiasCls = 3;  // the same with one class token before the patches
constexpr int kRelPosBiasRows = 4; // no class token, grid rows a multiple of 32 keys: one run per chunk
constexpr int kRelTabMax = 20480;  // table entries per head that fit beside the stages (fp32)
constexpr int kClsKey = -(1 << 30);  // key offset that marks a class key

template <int DV, int kMode, int kBiasKind>
struct Layout {
  static constexpr bool kBias = kBiasKind == kDenseBias;
  static constexpr bool kRel = kBiasKind == kRelPosBias || kBiasKind == kRelPosBiasCls ||
                               kBiasKind == kRelPosBiasRows;
  static constexpr int kKS = (kBias || kRel) ? 4 : 8;            // K / V / alpha_k stages
  static constexpr int kBS = 4;                                  // bias stages (per t)
  static constexpr int kBiasTile = kRows * kKeys * 2;            // 16 KB
  static constexpr int kKTile = kMode == kModeRef ? kKeys * DV * 2 : kKeys * 96;
  static constexpr int kVTile = (kMode == kModeDump || kMode == kModeMax) ? 0
                                : kMode == kModeI8 ? kKeys * DV : kKeys * DV * 2;
  static constexpr int kBiasOff = 0;
  static constexpr int kK = kBiasOff + (kBias ? kBS * 2 * kBiasTile : 0);
  static constexpr int kV = kK + kKS * kKTile;
  static constexpr int kAk = kV + kKS * kVTile;
  static constexpr int kKo = kAk + kKS * kKeys * 4;               // relative-position key offsets
  static constexpr int kTab = kKo + (kRel ? kKS * kKeys * 4 : 0);  // relative-position table (fp32)
  static constexpr int kBar = kTab + (kRel ? kRelTabMax * 4 : 0);
  static constexpr int kNumBars = 48;
  static constexpr int kMisc = kBar + 8 * kNumBars;  // tmem base, abort flag
  static constexpr int kBytes = kMisc + 16;
  // at least this much, so that one CTA occupies an SM (each CTA allocates all
  // 512 TMEM columns)
  static constexpr int kLaunchBytes = kBytes > 120 * 1024 ? kBytes : 120 * 1024;
};

// Instruction descriptor for kind::f8f6f4 with e4m3 A and B (format 0), fp32 D,
// both operands K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem], 8-bit floating-point operands.
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor for kind::i8: unsigned 8-bit A, signed 8-bit B, s32 D,
// both operands K-major.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4) | (0u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem], 8-bit integer operands (s32 accumulate).
__device__ __forceinline__ void mma_ts_i8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Named barrier `id` over `n` threads (a multiple of 32): wait, or arrive only.
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// 32 lanes x 32 bits x 8 columns: thread i gets columns [col, col + 8) of lane base + i.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr));
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}

// Four e4m3 operand bytes from the low 4 bits of x, lowest bit first: +1.0
// (0x38) for a set bit, -1.0 (0xB8) for a clear one. The multiply places bit
// e of x at bit 8e (the shifted copies of x do not overlap, so no carries).
__device__ __forceinline__ uint32_t e4m3_nibble(uint32_t x) {
  const uint32_t spread = (x & 0xFu) * 0x00204081u;
  return ((spread << 7) & 0x80808080u) ^ 0xB8B8B8B8u;
}

// Four e4m3 operand bytes from bits [j0, j0 + 4) of a sign word: +1 for a set
// bit, -1 for a clear one; channels c >= d are 0 when zero_pad is set.
__device__ __forceinline__ uint32_t e4m3_bytes(uint32_t word, int j0, int c0, int d, bool zero_pad) {
  uint32_t v = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t byte = ((word >> (j0 + j)) & 1u) ? 0x38u : 0xB8u;
    if (zero_pad && c0 + j >= d) byte = 0;
    v |= byte << (8 * j);
  }
  return v;
}

template <int DV, int kMode, int kBiasKind>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc2_kernel(const tc::Params p, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_bias, const __grid_constant__ CUtensorMap tm_k) {
  using L = Layout<DV, kMode, kBiasKind>;
  constexpr bool kBias = L::kBias;  // dense bias
  constexpr bool kRel = L::kRel;    // relative-position table
  constexpr bool kRelCls = kBiasKind == kRelPosBiasCls;    // ... with a class token
  constexpr bool kRelRows = kBiasKind == kRelPosBiasRows;  // ... read by runs of the table
  constexpr bool kRef = kMode == kModeRef;
  constexpr bool kDump = kMode == kModeDump;
  constexpr bool kMax = kMode == kModeMax;
  constexpr bool kI8 = kMode == kModeI8;
  constexpr bool kF16PV = kMode == kModeBin || kRef;  // bf16 P.V from TMA-loaded V
  constexpr bool kNoPV = kDump || kMax;
  constexpr int kKS = L::kKS, kBS = L::kBS;
  static_assert(DV % 16 == 0 && DV <= 96, "P.V N");
  static_assert(!kRef || DV <= 80, "reference Q_t columns");
  static_assert(kKS <= 8 && kBS <= 4, "barrier slots");

  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars + 0;    // [kKS] V (+ reference K) landed; binary: K expanded, alpha_k staged
  uint64_t* kv_empty = bars + 8;   // [kKS] both issuers' commits after the tile's P.V
  uint64_t* b_full = bars + 16;    // [kBS][2 t] bias tile landed
  uint64_t* b_empty = bars + 24;   // [kBS][2 t] the 128 softmax threads of t are done with it
  uint64_t* s_full = bars + 32;    // [2 t][2 b] QK^T commit + issuer arrive -> softmax t
  uint64_t* p_full = bars + 36;    // [2 t][2 b] softmax t published P (128 arrivals) -> issuer t
  uint64_t* o_done = bars + 40;    // [2 t][2 b] P.V commit of the last two tiles (no QK^T follows)
  uint64_t* drain = bars + 44;     // [2 t] error path only
  uint64_t* q_ready = bars + 46;   // [2 t] softmax t staged the pair's Q_t (128 arrivals) -> issuer t
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work items are 256-row pairs, numbered b fastest, then the query tile,
  // then h: batch entries sharing a bias tile (same h and query tile) are
  // adjacent, so CTAs running side by side fetch it from HBM once.
  // Without split, CTA c takes pairs pair_base + c + i * gridDim.x, i = 0, 1,
  // ..., below pair_base + npairs (npairs == 0: one pair per CTA). A CTA that
  // takes several pairs keeps its tensor memory, barriers and staged pads,
  // and its shared-memory rings run on across pairs, so the next pair's first
  // tiles load while the current pair finishes. With split, CTA 2i + half
  // takes one key half of pair pair_base + i. The position-sensitive bias
  // stages one head's table once, so its launches take one pair per CTA.
  const int nq = (p.N + 2 * kRows - 1) / (2 * kRows);
  const int half = p.split ? static_cast<int>(blockIdx.x & 1) : 0;
  const int G = static_cast<int>(gridDim.x);
  const int npairs = p.npairs > 0 ? p.npairs : G;
  const int n_items = (p.split || kRel) ? 1 : max(0, (npairs - static_cast<int>(blockIdx.x) + G - 1) / G);
  struct Item {
    int pidx, h, bh, q0;
    size_t tok0;
  };
  auto item = [&](int it) {
    Item w;
    w.pidx = p.pair_base + (p.split ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x) + it * G);
    const int b = w.pidx % p.B;
    const int qt = (w.pidx / p.B) % nq;
    w.h = w.pidx / (p.B * nq);
    w.bh = b * p.H + w.h;
    w.tok0 = static_cast<size_t>(w.bh) * p.N;
    w.q0 = qt * 2 * kRows;
    return w;
  };
  const int N = p.N, d = p.d;
  const int W = (d + 31) / 32;                 // sign words per token (binary)
  const int nkt_all = (N + kKeys - 1) / kKeys;
  const int kt_begin = p.split && half ? nkt_all / 2 : 0;
  const int nkt = p.split ? (half ? nkt_all - nkt_all / 2 : nkt_all / 2) : nkt_all;  // tiles of this CTA
  const int key0 = kt_begin * kKeys;  // first key of this CTA
  const int dgroups = d / 8;                   // 8-channel groups written by TMA
  const int kq16 = (d + 15) / 16;              // reference QK^T MMAs (16 channels each)

  // ---------------------------------------------------------------- setup
  if constexpr (kF16PV) {
    // Channels >= d of every V stage (never written by TMA): channel d is 1.0
    // (the row-sum column), the rest 0. Reference K: pad channels 0.
    const int npad = (DV / 8 - dgroups) * kKeys;
    for (int e = threadIdx.x; e < kKS * npad; e += kThreads) {
      const int s = e / npad, rem = e % npad;
      const int g = dgroups + rem / kKeys, kk = rem % kKeys;
      *reinterpret_cast<uint4*>(smem + L::kV + s * L::kVTile + g * 1024 + kk * 16) =
          make_uint4(g == dgroups ? 0x3F80u : 0u, 0u, 0u, 0u);
    }
    if constexpr (kRef) {
      const int kpad = (2 * kq16 - dgroups) * kKeys;
      for (int e = threadIdx.x; e < kKS * kpad; e += kThreads) {
        const int s = e / kpad, rem = e % kpad;
        const int g = dgroups + rem / kKeys, kk = rem % kKeys;
        *reinterpret_cast<uint4*>(smem + L::kK + s * L::kKTile + g * 1024 + kk * 16) = make_uint4(0, 0, 0, 0);
      }
    }
  }
  if constexpr (kRel) {
    // this head's relative-position table, widened to fp32 once
    float* tab = reinterpret_cast<float*>(smem + L::kTab);
    const uint16_t* src_t = p.rel_table + static_cast<size_t>(item(0).h) * p.rel_R;
    for (int e = threadIdx.x; e < p.rel_R; e += kThreads) tab[e] = bf16_bits_to_float(src_t[e]);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKS; ++s) {
      // the expander's 32 lanes, plus the arrive of the V copy
      mbar_init(&kv_full[s], kRef ? 1 : (kNoPV ? 32 : 33));
      mbar_init(&kv_empty[s], 2);
    }
    for (int i = 0; i < kBS * 2; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], kSoftmaxPerTile);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 2);  // the QK^T commit + the issuer's arrive (alpha_k, bias landed)
      mbar_init(&p_full[i], kSoftmaxPerTile);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(&q_ready[0], kSoftmaxPerTile);
    mbar_init(&q_ready[1], kSoftmaxPerTile);
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

  // Softmax warp w < 8: tile t = w / 4, rows 32 (w % 4) .. + 31 (the warp's
  // TMEM lane quadrant), one thread per row.
  const int t = warp >> 2;
  const int r = ((warp & 3) << 5) | lane;    // row within the tile = TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  // Softmax threads, once per pair: this thread's row of Q_t into TMEM, and
  // alpha_q of the row (binary forward), returned. A binary forward from
  // binattn_pack's output takes the row's sign words and alpha_q in qw / aq,
  // loaded one pair ahead (fetch_qbits below).
  auto stage_q = [&](const Item& w, int row, bool row_valid, const uint32_t (&qw_in)[3], float aq_in) {
    float aq_row = 0.f;
    if constexpr (kRef) {
      // bf16 pairs: column c2 holds channels 2 c2 (low half) and 2 c2 + 1
      const uint32_t qcol = tmem + lane_base + 256 * t + 128 + DV;
      for (int c = 0; c < 2 * kq16; c += 2) {
        uint32_t wv[8];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint4 val = make_uint4(0, 0, 0, 0);
          if (row_valid && 8 * (c + h2) < d)
            val = *reinterpret_cast<const uint4*>(p.q + (w.tok0 + row) * d + 8 * (c + h2));
          wv[4 * h2 + 0] = val.x;
          wv[4 * h2 + 1] = val.y;
          wv[4 * h2 + 2] = val.z;
          wv[4 * h2 + 3] = val.w;
        }
        tmem_st8(qcol + 4 * c, wv);
      }
    } else {
      // e4m3 bytes: column c4 holds channels 4 c4 .. 4 c4 + 3 (lowest byte first);
      // pad channels (>= d) are 0 so they add nothing to the score.
      const uint32_t qcol = tmem + lane_base + 256 * t + kQColBin;
      uint32_t qw[3] = {qw_in[0], qw_in[1], qw_in[2]};
      aq_row = aq_in;
      if (row_valid && !kDump && p.qh)
        pack_row_bf16_w(p.qh + (w.tok0 + row) * d, d, W, qw, aq_row);  // Q binarised here
      for (int k = 0; k < W; ++k) {
        const uint32_t word = k == 0 ? qw[0] : k == 1 ? qw[1] : qw[2];
        uint32_t wv[8];
#pragma unroll
        // four channels per column (e4m3_nibble); d % 8 == 0, so a column is
        // wholly below d or wholly padding (0)
        for (int j = 0; j < 8; ++j) wv[j] = (row_valid && 32 * k + 4 * j < d) ? e4m3_nibble(word >> (4 * j)) : 0u;
        tmem_st8(qcol + 8 * k, wv);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    return aq_row;
  };
  fence_proxy_async_smem();
  __syncthreads();
  tc_fence_after();

  if (warp == kTmaWarp) {
    // --------------------------- V (and reference K), bias: one thread issues
    // Ring slots and phases follow the tile count g over all of the CTA's
    // pairs (g = it * nkt + kt), as in every role below.
    if (lane == 0 && (!kNoPV || kBias)) {
      bool ok = true;
      for (int it = 0; ok && it < n_items; ++it) {
        const Item w = item(it);
        for (int kt = 0; ok && kt < nkt; ++kt) {
          const int g = it * nkt + kt;
          if (p.stall_after >= 0 && g >= p.stall_after) {  // test only
            ok = false;
            break;
          }
          const int j0 = key0 + kt * kKeys;
          if constexpr (kF16PV) {
            const int s = g % kKS;
            if (g >= kKS && !(ok = mbar_wait(&kv_empty[s], ((g / kKS) - 1) & 1, abort))) break;
            mbar_arrive_expect_tx(&kv_full[s], static_cast<uint32_t>(dgroups * 1024 * (kRef ? 2 : 1)));
            for (int c = 0; c < dgroups; ++c)
              tma_load_3d(smem + L::kV + s * L::kVTile + c * 1024, &tm_v, 8 * c, j0, w.bh, &kv_full[s]);
            if constexpr (kRef) {
              for (int c = 0; c < dgroups; ++c)
                tma_load_3d(smem + L::kK + s * L::kKTile + c * 1024, &tm_k, 8 * c, j0, w.bh, &kv_full[s]);
            }
          } else if constexpr (kI8) {
            // the tile's 8-bit V operand is one contiguous block of the tiled layout
            const int s = g % kKS;
            if (g >= kKS && !(ok = mbar_wait(&kv_empty[s], ((g / kKS) - 1) & 1, abort))) break;
            mbar_arrive_expect_tx(&kv_full[s], static_cast<uint32_t>(L::kVTile));
            bulk_load(smem + L::kV + s * L::kVTile,
                      p.vq8 + (static_cast<size_t>(w.bh) * nkt_all + kt_begin + kt) * L::kVTile,
                      static_cast<uint32_t>(L::kVTile), &kv_full[s]);
          }
          if constexpr (kBias) {
            for (int t2 = 0; t2 < 2; ++t2) {
              const int i = (g % kBS) * 2 + t2;
              if (g >= kBS && !(ok = mbar_wait(&b_empty[i], ((g / kBS) - 1) & 1, abort))) break;
              mbar_arrive_expect_tx(&b_full[i], L::kBiasTile);
              tma_load_3d(smem + L::kBiasOff + i * L::kBiasTile, &tm_bias, j0, w.q0 + t2 * kRows,
                          p.bias_per_sample ? w.bh : w.h, &b_full[i]);
            }
          }
        }
      }
    }
  } else if (warp == kExpandWarp) {
    // ------------------- binary: key sign words -> e4m3 +-1 rows, alpha_k
    // The sign words and alpha_k of tile kt + 2 are loaded into registers
    // before tile kt is expanded, so the global-load latency overlaps two tile
    // periods instead of sitting between the stage's release and its refill.
    if constexpr (!kRef) {
      const int kb_row = 32 * W;  // operand bytes per key
      struct TileRegs {
        uint32_t wd[2][3];
        float ak[2];
        int ko[2];
      };
      // The tiles of the CTA's sequence in order: key tile kt_l of pair it_l
      // is loaded next (tok_l: the pair's first token), past the end zeros.
      const int g_end = n_items * nkt;
      int it_l = 0, kt_l = 0;
      size_t tok_l = n_items > 0 ? item(0).tok0 : 0;
      auto load_next = [&](TileRegs& tr) {
        const bool live = it_l < n_items;
        const size_t tok0 = tok_l;
        const int kt = kt_l;
        if (live && ++kt_l == nkt) {
          kt_l = 0;
          if (++it_l < n_items) tok_l = item(it_l).tok0;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int key = key0 + kt * kKeys + lane + 32 * u;
          const bool in = live && key < N;
#pragma unroll
          for (int w = 0; w < 3; ++w) tr.wd[u][w] = (in && w < W) ? __ldg(p.kb + (tok0 + key) * W + w) : 0u;
          tr.ak[u] = (!kDump && in) ? __ldg(p.ak + tok0 + key) : 0.f;
          if constexpr (kRel && !kRelRows) {
            // -(y_j (2 gw - 1) + x_j) for a patch key, so that a patch query's
            // base plus it is the table entry of their displacement
            const int pj = key - p.rel_ncls;
            tr.ko[u] = !in ? 0 : pj < 0 ? kClsKey : -((pj / p.rel_gw) * (2 * p.rel_gw - 1) + pj % p.rel_gw);
          }
        }
      };
      TileRegs cur, n1;
      load_next(cur);
      load_next(n1);
      for (int g = 0; g < g_end; ++g) {
        TileRegs n2;
        load_next(n2);
        const int s = g % kKS;
        const bool ok = g < kKS || mbar_wait(&kv_empty[s], ((g / kKS) - 1) & 1, abort);
        if (!__all_sync(0xffffffffu, ok)) break;
        uint8_t* ks = smem + L::kK + s * L::kKTile;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int rr = lane + 32 * u;
          uint8_t* dst = ks + (rr >> 3) * (8 * kb_row) + (rr & 7) * 16;
#pragma unroll
          for (int c = 0; c < 6; ++c) {
            if (c < 2 * W) {
              const uint32_t half = cur.wd[u][c >> 1] >> (16 * (c & 1));
              *reinterpret_cast<uint4*>(dst + c * 128) =
                  make_uint4(e4m3_nibble(half), e4m3_nibble(half >> 4), e4m3_nibble(half >> 8), e4m3_nibble(half >> 12));
            }
          }
        }
        if constexpr (!kDump) {
          float* aks = reinterpret_cast<float*>(smem + L::kAk) + s * kKeys;
#pragma unroll
          for (int u = 0; u < 2; ++u) aks[lane + 32 * u] = cur.ak[u];
          if constexpr (kRel && !kRelRows) {
            int* kos = reinterpret_cast<int*>(smem + L::kKo) + s * kKeys;
#pragma unroll
            for (int u = 0; u < 2; ++u) kos[lane + 32 * u] = cur.ko[u];
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&kv_full[s]);
        cur = n1;
        n1 = n2;
      }
    }
  } else if (warp >= kMmaWarp0) {
    // ----------------------------------------------- MMA issuer of tile tt
    const int tt = warp - kMmaWarp0;
    if (lane == 0) {
      constexpr uint32_t kIdQK = kRef ? idesc_bf16(kRows, kKeys, false) : idesc_e4m3(kRows, kKeys);
      constexpr uint32_t kIdPV = idesc_bf16(kRows, DV, true);
      const uint32_t kb_sbo = kRef ? 128u : static_cast<uint32_t>(8 * 32 * W);
      const uint32_t base_t = tmem + 256 * tt;
      // S_tt^(g%2) = Q_tt K(g)^T for tile g of the CTA's sequence
      auto issue_qk = [&](int g) {
        const uint32_t k_base = smem_u32(smem + L::kK + (g % kKS) * L::kKTile);
        const uint32_t d_col = base_t + 64 * (g & 1);
        if constexpr (kRef) {
          for (int ks = 0; ks < kq16; ++ks)
            mma_ts(d_col, base_t + 128 + DV + ks * 8, smem_desc(k_base + ks * 2048, 1024, kb_sbo), kIdQK, ks > 0);
        } else {
          for (int ks = 0; ks < W; ++ks)
            mma_ts_f8(d_col, base_t + kQColBin + ks * 8, smem_desc(k_base + ks * 256, 128, kb_sbo), kIdQK, ks > 0);
        }
      };
      bool ok = true;
      // Tile kt's operands and softmax inputs are in shared memory: the K / V
      // stage with alpha_k and, with a bias, this tile's bias box. The issuer
      // waits for them and then arrives on s_full itself (release), so the
      // softmax threads' single wait on s_full also covers alpha_k and the bias.
      auto stage_ready = [&](int g) {
        if (!mbar_wait(&kv_full[g % kKS], (g / kKS) & 1, abort)) return false;
        if (kBias && !mbar_wait(&b_full[(g % kBS) * 2 + tt], (g / kBS) & 1, abort)) return false;
        mbar_arrive(&s_full[tt * 2 + (g & 1)]);
        tc_fence_after();
        return true;
      };
      for (int it = 0; ok && it < n_items; ++it) {
        // Q_tt of the pair is in TMEM (and, from the second pair on, the
        // softmax threads have read the previous pair's O)
        if (!(ok = mbar_wait(&q_ready[tt], it & 1, abort))) break;
        tc_fence_after();
        const int g0 = it * nkt;
        for (int kt = 0; ok && kt < 2 && kt < nkt; ++kt) {
          if (!(ok = stage_ready(g0 + kt))) break;
          issue_qk(g0 + kt);
          mma_commit(&s_full[tt * 2 + ((g0 + kt) & 1)]);
        }
        for (int kt = 0; ok && kt < nkt; ++kt) {
          const int g = g0 + kt;
          const int s = g % kKS;
          const int bf = g & 1;
          if (!(ok = mbar_wait(&p_full[tt * 2 + bf], (g >> 1) & 1, abort))) break;
          tc_fence_after();
          if constexpr (kF16PV) {
            // O_tt += P_tt(kt) V(kt): A = P (bf16 pairs, 8 columns per 16 keys)
            const uint32_t v_base = smem_u32(smem + L::kV + s * L::kVTile);
#pragma unroll
            for (int ks = 0; ks < kKeys / 16; ++ks)
              mma_ts(base_t + 128, base_t + 64 * bf + ks * 8, smem_desc(v_base + ks * 256, 128, 1024), kIdPV,
                     (kt > 0 || ks > 0));
          } else if constexpr (kI8) {
            // O_tt (s32) += P_tt(kt) V(kt): A = u8 P (4 keys per column, 8
            // columns per 32 keys), B = s8 V, K-major, 32 keys per MMA
            const uint32_t v_base = smem_u32(smem + L::kV + s * L::kVTile);
#pragma unroll
            for (int ks = 0; ks < kKeys / 32; ++ks)
              mma_ts_i8(base_t + 128, base_t + 64 * bf + ks * 8, smem_desc(v_base + ks * 256, 128, 512),
                        idesc_i8(kRows, DV), (kt > 0 || ks > 0));
          }
          mma_commit(&kv_empty[s]);  // this issuer's last use of stage s
          if (kt + 2 < nkt) {
            if (!(ok = stage_ready(g + 2))) break;
            issue_qk(g + 2);
            mma_commit(&s_full[tt * 2 + bf]);
          } else if constexpr (!kNoPV) {
            mma_commit(&o_done[tt * 2 + bf]);
          }
        }
      }
      {  // wait (bounded) for every MMA of this thread before TMEM is freed
        mma_commit(&drain[tt]);
        volatile int never = 0;
        mbar_wait(&drain[tt], 0, &never);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax
    const uint32_t o_col = tmem + lane_base + 256 * t + 128;
    const int r7 = r & 7;
    // Per pair (set at the top of each): the thread's row, the per-row factor
    // of the logit (scale * alpha_q, binary; scale, reference) and the running
    // max (in the 8-bit pass, the row's exact max from the first pass).
    int row = 0;
    bool row_valid = false;
    size_t tok0 = 0;
    float ci = 0.f;
    float m = -INFINITY;
    bool ok = true;
    // Waits are made warp-uniform: the tcgen05.ld/st below are warp-collective.
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
    };
    // o_done[t][b] completes once per pair for each b when a pair has two or
    // more key tiles; with one, the pairs alternate between the two buffers.
    auto od_parity = [&](int it) { return static_cast<uint32_t>((nkt >= 2 ? it : it >> 1) & 1); };
    // P.V of tile g - 1 (key tile kt - 1 of pair it) is complete once
    // QK^T(g + 1) (issued after it by the same thread) is, or, for the pair's
    // last tile, once its own commit lands.
    auto wait_pv_prev = [&](int g, int kt, int it) {
      const bool r1 = kt + 1 < nkt ? wait_all(&s_full[t * 2 + ((g + 1) & 1)], ((g + 1) >> 1) & 1)
                                   : wait_all(&o_done[t * 2 + ((g - 1) & 1)], od_parity(it));
      tc_fence_after();
      return r1;
    };
    // logits of chunk c (32 keys, in place): S * alpha_k * (scale * alpha_q) + bias
    // Position-sensitive bias: a patch query i reads table entry
    // rel_base + ko_j for a patch key j (ko_j staged by the expander); a class
    // query (and a row >= N, whose result is not stored) reads one fixed entry
    // for every patch key; a class key reads rel_cls_key.
    int rel_base = 0, rel_fixed = -1, rel_cls_key = 0;
    auto rel_setup = [&]() {
      const int R0 = (2 * p.rel_gh - 1) * (2 * p.rel_gw - 1);
      const int pi = row - p.rel_ncls;
      // a row >= N takes patch 0's base (its result is not stored; every
      // index it forms is still inside the table)
      const int pb = (row_valid && pi >= 0) ? pi : 0;
      rel_base = (pb / p.rel_gw + p.rel_gh - 1) * (2 * p.rel_gw - 1) + pb % p.rel_gw + p.rel_gw - 1;
      if constexpr (kRelCls) {
        if (row_valid && pi >= 0) {
          rel_cls_key = R0 + 1;
        } else {
          rel_fixed = row_valid ? R0 : 0;
          rel_cls_key = row_valid ? R0 + 2 : 0;
        }
      }
    };
    const float* rel_tab = reinterpret_cast<const float*>(smem + L::kTab);
    auto logits = [&](uint32_t* xr, int c, const uint8_t* bsm, const float* aks, int jtile) {
      float2* xs = reinterpret_cast<float2*>(xr);
      const float2 ci2 = make_float2(ci, ci);
#pragma unroll
      for (int q = 0; q < kChunk / 8; ++q) {
        float2 bv[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        if constexpr (kBias) {
          const int u = 4 * c + q;  // 16-byte unit of the row in the 64-key box
          const uint4 raw = *reinterpret_cast<const uint4*>(bsm + ((u ^ r7) << 4));
          const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            bv[e] = make_float2(__uint_as_float(rw[e] << 16), __uint_as_float(rw[e] & 0xFFFF0000u));
        } else if constexpr (kRel) {
          if constexpr (kRelRows) {
            // the chunk's 32 keys lie in one grid row, so key e of the chunk
            // reads entry rp - e; a chunk beyond N (wholly masked) reads the
            // last real chunk's entries instead
            const int jc = min(jtile + kChunk * c, N - kChunk);
            const float* rp = rel_tab + rel_base - (jc / p.rel_gw) * (2 * p.rel_gw - 1) - jc % p.rel_gw;
#pragma unroll
            for (int e = 0; e < 4; ++e) bv[e] = make_float2(rp[-(8 * q + 2 * e)], rp[-(8 * q + 2 * e + 1)]);
          } else {
          // the stage's key offsets follow its alpha_k (Layout: kKo = kAk + kKS * 64 * 4)
          const int* kos = reinterpret_cast<const int*>(aks + kKS * kKeys) + kChunk * c + 8 * q;
          const int4 o0 = *reinterpret_cast<const int4*>(kos);
          const int4 o1 = *reinterpret_cast<const int4*>(kos + 4);
          const int o[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
          float bb[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if constexpr (kRelCls)
              bb[e] = rel_tab[o[e] == kClsKey ? rel_cls_key : (rel_fixed >= 0 ? rel_fixed : rel_base + o[e])];
            else
              bb[e] = rel_tab[rel_base + o[e]];
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) bv[e] = make_float2(bb[2 * e], bb[2 * e + 1]);
          }
        }
        if constexpr (kRef) {
#pragma unroll
          for (int e = 0; e < 4; ++e) xs[4 * q + e] = __ffma2_rn(xs[4 * q + e], ci2, bv[e]);
        } else {
          const float4 a0 = *reinterpret_cast<const float4*>(aks + kChunk * c + 8 * q);
          const float4 a1 = *reinterpret_cast<const float4*>(aks + kChunk * c + 8 * q + 4);
          const float2 av[4] = {make_float2(a0.x, a0.y), make_float2(a0.z, a0.w), make_float2(a1.x, a1.y),
                                make_float2(a1.z, a1.w)};
#pragma unroll
          for (int e = 0; e < 4; ++e) xs[4 * q + e] = __ffma2_rn(__fmul2_rn(xs[4 * q + e], av[e]), ci2, bv[e]);
        }
      }
    };
    // P = exp(logit - m) of a chunk as bf16 pairs into 16 TMEM columns
    auto exps = [&](const uint32_t* xr, uint32_t p_col) {
      const float2* xs = reinterpret_cast<const float2*>(xr);
      const float2 l2e2 = make_float2(kLog2e, kLog2e);
      const float2 nm2 = make_float2(-m * kLog2e, -m * kLog2e);
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float2 a = __ffma2_rn(xs[e], l2e2, nm2);
        pk[e] = pack_bf16x2(ex2(a.x), ex2(a.y));
      }
      tmem_st16(p_col, pk);
    };

    // 8-bit pass: u = rint(255 exp(logit - m)) of a 32-key chunk (m the row's
    // exact max, so u <= 255), four keys per 32-bit TMEM column, lowest key in
    // the lowest byte: the unsigned 8-bit A operand of the kind::i8 P.V
    // The rounding runs on the FMA pipe: y = 255 p + 1.5 * 2^23 (one fused
    // multiply-add, rounded to nearest even) holds rint(255 p) in its low
    // mantissa bits, since 0 <= 255 p <= 255 sits where the ulp is 1; the low
    // bytes of four such words are then gathered by byte permutes.
    auto exps_u8 = [&](const uint32_t* xr, uint32_t p_col) {
      const float2* xs = reinterpret_cast<const float2*>(xr);
      const float2 l2e2 = make_float2(kLog2e, kLog2e);
      const float2 nm2 = make_float2(-m * kLog2e, -m * kLog2e);
      const float2 k255 = make_float2(255.f, 255.f);
      const float2 magic = make_float2(12582912.f, 12582912.f);
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float2 a0 = __ffma2_rn(xs[2 * e], l2e2, nm2);
        const float2 a1 = __ffma2_rn(xs[2 * e + 1], l2e2, nm2);
        const float2 y0 = __ffma2_rn(make_float2(ex2(a0.x), ex2(a0.y)), k255, magic);
        const float2 y1 = __ffma2_rn(make_float2(ex2(a1.x), ex2(a1.y)), k255, magic);
        const uint32_t lo = __byte_perm(__float_as_uint(y0.x), __float_as_uint(y0.y), 0x0040);
        const uint32_t hi = __byte_perm(__float_as_uint(y1.x), __float_as_uint(y1.y), 0x0040);
        pk[e] = __byte_perm(lo, hi, 0x5410);
      }
      tmem_st8(p_col, pk);
    };

    // The loop runs every key tile even after an error (with the work
    // skipped), so that each thread takes its part in every named barrier.
    if (!kNoPV && t == 1 && n_items > 0) named_arrive(3, 2 * kSoftmaxPerTile);  // tile 0 takes the first exp turn
    const int g_end = n_items * nkt;
    // the sign words and alpha_q of this thread's row in pair it2 (zeros for
    // a row >= N, past the last pair, and where stage_q does not take them)
    uint32_t qn[3];
    float aqn;
    auto fetch_qbits = [&](int it2, uint32_t (&qw)[3], float& a) {
      qw[0] = qw[1] = qw[2] = 0u;
      a = 0.f;
      if (kRef || p.qh != nullptr || it2 >= n_items) return;
      const Item w2 = item(it2);
      const int row2 = w2.q0 + t * kRows + r;
      if (row2 < N) {
#pragma unroll
        for (int k = 0; k < 3; ++k)
          if (k < W) qw[k] = __ldg(p.qb + (w2.tok0 + row2) * W + k);
        if (!kDump) a = __ldg(p.aq + w2.tok0 + row2);
      }
    };
    fetch_qbits(0, qn, aqn);
    for (int it = 0; it < n_items; ++it) {
    const Item w = item(it);
    tok0 = w.tok0;
    row = w.q0 + t * kRows + r;
    row_valid = row < N;
    {
      // Q_t of the pair into TMEM; the issuer waits for all 128 rows. From
      // the second pair on, the previous pair's epilogue has read O_t (its
      // last P.V waited for), so the pair's first P.V may overwrite it.
      const float aq_row = ok ? stage_q(w, row, row_valid, qn, aqn) : 0.f;
      mbar_arrive(&q_ready[t]);
      ci = kRef ? p.scale : ((!kDump && row_valid) ? p.scale * aq_row : 0.f);
      fetch_qbits(it + 1, qn, aqn);  // in flight through this pair
    }
    m = -INFINITY;
    if constexpr (kI8) m = row_valid ? p.mrow[tok0 + row] : 0.f;
    if constexpr (kRel) rel_setup();
    for (int kt = 0; kt < nkt; ++kt) {
      const int g = it * nkt + kt;  // tile of the CTA's sequence: ring slots and phases
      const int s = g % kKS;
      const int bf = g & 1;
      const int bs = g % kBS;
      // scores, alpha_k and the bias tile of g (see the issuer's stage_ready)
      if (ok) ok = wait_all(&s_full[t * 2 + bf], (g >> 1) & 1);
      tc_fence_after();
      const uint32_t s_col = tmem + lane_base + 256 * t + 64 * bf;
      uint32_t xa[kChunk], xb[kChunk];
      if (ok) {
        tmem_ld32(s_col, xa);
        tmem_ld32(s_col + kChunk, xb);
        tmem_ld_wait();
      }
      if constexpr (kDump) {
        if (ok && row_valid) {
          int32_t* srow = p.S + (tok0 + row) * N + key0 + kt * kKeys;
#pragma unroll
          for (int e = 0; e < kChunk; ++e) {
            if (key0 + kt * kKeys + e < N) srow[e] = static_cast<int32_t>(__uint_as_float(xa[e]));
            if (key0 + kt * kKeys + kChunk + e < N) srow[kChunk + e] = static_cast<int32_t>(__uint_as_float(xb[e]));
          }
        }
      } else {
        if (ok) {
          const uint8_t* bsm = smem + L::kBiasOff + (bs * 2 + t) * L::kBiasTile + r * 128;
          const float* aks = reinterpret_cast<const float*>(smem + L::kAk) + s * kKeys;
          logits(xa, 0, bsm, aks, key0 + kt * kKeys);
          logits(xb, 1, bsm, aks, key0 + kt * kKeys);
          float* x0 = reinterpret_cast<float*>(xa);
          float* x1 = reinterpret_cast<float*>(xb);
          const int jt = key0 + kt * kKeys;
          if (jt + kKeys > N) {  // keys >= N take no part (warp-uniform branch)
#pragma unroll
            for (int e = 0; e < kChunk; ++e) {
              if (jt + e >= N) x0[e] = -INFINITY;
              if (jt + kChunk + e >= N) x1[e] = -INFINITY;
            }
          }
          // tile max: four independent 3-input max chains over both chunks
          float mc[4];
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            float a = max3f(x0[k4], x0[k4 + 4], x0[k4 + 8]);
            a = max3f(a, x0[k4 + 12], x0[k4 + 16]);
            a = max3f(a, x0[k4 + 20], x0[k4 + 24]);
            a = max3f(a, x0[k4 + 28], x1[k4]);
            a = max3f(a, x1[k4 + 4], x1[k4 + 8]);
            a = max3f(a, x1[k4 + 12], x1[k4 + 16]);
            a = max3f(a, x1[k4 + 20], x1[k4 + 24]);
            mc[k4] = fmaxf(a, x1[k4 + 28]);
          }
          const float tmax = fmaxf(max3f(mc[0], mc[1], mc[2]), mc[3]);
          // Lazy rescale: m moves only when the tile max exceeds it by more
          // than kRescale; until then every p = exp(logit - m) <= 2^8, and the
          // final division by l (summed against the same m) cancels the
          // offset. O_t holds l in column d, so one rescale covers both.
          // The row-max pass only keeps the max; the 8-bit pass has it already.
          const bool grow = kF16PV && tmax > m + kRescale;
          if constexpr (kMax) m = fmaxf(m, tmax);
          if (__any_sync(0xffffffffu, grow)) {
            const float m_new = grow ? tmax : m;
            const float corr = grow ? ex2((m - m_new) * kLog2e) : 1.f;  // 0 while m is -inf
            if (kt > 0 && (ok = wait_pv_prev(g, kt, it))) {
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
        // MUFU token: the exp phases of the two tiles alternate (named barriers
        // 3 and 4 over both tiles' softmax threads), so one tile's exps run
        // while the other computes its logits.
        if constexpr (kMax) {
          if (ok && kBias) mbar_arrive(&b_empty[bs * 2 + t]);
        } else {
          named_sync(3 + t, 2 * kSoftmaxPerTile);
          if (ok) {
            if constexpr (kI8) {
              exps_u8(xa, s_col);
              exps_u8(xb, s_col + 8);
            } else {
              exps(xa, s_col);
              exps(xb, s_col + 16);
            }
            if (kBias) mbar_arrive(&b_empty[bs * 2 + t]);
          }
          if (!(t == 1 && g == g_end - 1)) named_arrive(4 - t, 2 * kSoftmaxPerTile);  // pass the token on
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[t * 2 + bf]);
      }
    }
    if constexpr (kMax) {
      if (ok && row_valid) p.mrow[tok0 + row] = m;
    } else if constexpr (kI8) {
      if (ok && wait_all(&o_done[t * 2 + ((it * nkt + nkt - 1) & 1)], od_parity(it))) {
        tc_fence_after();
        // O_c = s_c * acc_c / l with the s32 sums acc_c = sum_j u_j vq_jc and
        // l = sum_j u_j (column d, the ones channel of the 8-bit V)
        uint32_t lbits;
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(lbits) : "r"(o_col + d));
        tmem_ld_wait();
        const float inv = 1.f / static_cast<float>(static_cast<int>(lbits));
        const float* vs = p.vscale + static_cast<size_t>(item(it).bh) * d;
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
                  float f[8];
#pragma unroll
                  for (int k = 0; k < 8; ++k)
                    f[k] = __ldg(vs + cc + e + k) * static_cast<float>(static_cast<int>(ov[e + k])) * inv;
                  *reinterpret_cast<uint4*>(orow + cc + e) =
                      make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                 pack_bf16x2(f[6], f[7]));
                }
              }
            }
          }
        }
      }
    } else if constexpr (!kDump) {
      if (ok && wait_all(&o_done[t * 2 + ((it * nkt + nkt - 1) & 1)], od_parity(it))) {
        tc_fence_after();
        uint32_t lbits;  // l = O_t column d
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(lbits) : "r"(o_col + d));
        tmem_ld_wait();
        if (p.split) {
          // Partial result of this key half: unnormalised O (d fp32), then m, then l.
          // channel-major: value c of row r256 of (pair slot, half) at
          // ((slot * 2 + half) * (d + 2) + c) * 256 + r256, so that a warp's 32
          // rows store (and the combine kernel loads) 128 contiguous bytes
          const int r256 = t * kRows + r;
          // (a split launch takes one pair per CTA: pair_base + blockIdx.x / 2)
          float* dst = p.part + static_cast<size_t>((blockIdx.x >> 1) * 2 + half) * (d + 2) * (2 * kRows) + r256;
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
        // two column blocks of 16 per wait, so that the tensor-memory latency
        // is paid once per 32 columns
#pragma unroll
        for (int cc = 0; cc < DV; cc += 32) {
          if (cc < d) {  // warp-uniform: d is the same for every thread
            uint32_t ov[32];
            tmem_ld16(o_col + cc, *reinterpret_cast<uint32_t(*)[16]>(ov));
            if (cc + 16 < DV && cc + 16 < d) tmem_ld16(o_col + cc + 16, *reinterpret_cast<uint32_t(*)[16]>(ov + 16));
            tmem_ld_wait();
            if (row_valid) {
#pragma unroll
              for (int e = 0; e < 32; e += 8) {
                if (cc + e < DV && cc + e < d) {
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
    }
    }  // pairs
  }

  // ------------------------------------------------------------- teardown
  // Both issuers waited for their own MMAs; every TMEM access of the softmax
  // threads is complete (wait::ld / wait::st) before this barrier.
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Bias rows padded to ld elements (ld % 8 == 0, pad 0), so that they are TMA
// rows: out[(h * N + i) * ld + j] = j < N ? bias[(h * N + i) * src_ld + j] : 0.
// One warp per row (grid-stride over rows): lane c writes 16-byte chunk c of
// the padded row (out is 16-byte aligned, ld % 8 == 0), reading its 8 source
// elements with consecutive 2-byte loads across the warp (a source row starts
// at any element).
__global__ void __launch_bounds__(256) pad_bias_rows_kernel(const uint16_t* __restrict__ bias,
                                                            long long rows, int N, int src_ld, int ld,
                                                            uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  const int chunks = ld / 8;
  for (long long row = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); row < rows;
       row += nwarps) {
    const uint16_t* src = bias + row * src_ld;
    uint4* dst = reinterpret_cast<uint4*>(out + row * ld);
    for (int c = lane; c < chunks; c += 32) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 8 * c + 2 * e;
        const uint32_t lo = j < N ? __ldg(src + j) : 0u;
        const uint32_t hi = j + 1 < N ? __ldg(src + j + 1) : 0u;
        w[e] = lo | (hi << 16);
      }
      dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}
// Launches pad_bias_rows_kernel over rows rows: 8 warps per block, at most
// 8 blocks per SM of a 148-SM part (the kernel strides over the rest).
inline void pad_bias_rows(const uint16_t* bias, long long rows, int N, int src_ld, int ld, uint16_t* out,
                          cudaStream_t st) {
  const long long blocks = (rows + 7) / 8;
  const unsigned grid = static_cast<unsigned>(blocks < 148 * 8 ? blocks : 148 * 8);
  pad_bias_rows_kernel<<<grid, 256, 0, st>>>(bias, rows, N, src_ld, ld, out);
}

// Joins the two key halves of split pairs: for row i with partials (O_h, m_h,
// l_h), M = max(m_0, m_1), w_h = exp(m_h - M), O = (w_0 O_0 + w_1 O_1) /
// (w_0 l_0 + w_1 l_1), rounded to bf16. One thread per row of the split pairs.
__global__ void __launch_bounds__(256) combine_halves_kernel(const float* __restrict__ part, int pair_base,
                                                             int npairs, int B, int H, int N, int d,
                                                             uint16_t* __restrict__ out) {
  const int i = blockIdx.x * 256 + threadIdx.x;  // row of the split pairs
  if (i >= npairs * 2 * kRows) return;
  const int pidx = pair_base + i / (2 * kRows);
  const int rr = i % (2 * kRows);
  const int nq = (N + 2 * kRows - 1) / (2 * kRows);
  const int b = pidx % B, qt = (pidx / B) % nq, h = pidx / (B * nq);
  const int row = qt * 2 * kRows + rr;
  if (row >= N) return;
  // channel-major partials (see the split epilogue): value c of half h at p_h[c * 256]
  constexpr int kS = 2 * kRows;
  const float* p0 = part + static_cast<size_t>(i / kS) * 2 * (d + 2) * kS + rr;
  const float* p1 = p0 + static_cast<size_t>(d + 2) * kS;
  const float m0 = p0[d * kS], m1 = p1[d * kS];
  const float M = fmaxf(m0, m1);
  const float w0 = ex2((m0 - M) * kLog2e), w1 = ex2((m1 - M) * kLog2e);
  const float inv = 1.f / (w0 * p0[(d + 1) * kS] + w1 * p1[(d + 1) * kS]);
  uint16_t* orow = out + ((static_cast<size_t>(b) * H + h) * N + row) * d;
  for (int c = 0; c < d; c += 8) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w[e] = pack_bf16x2((w0 * p0[(c + 2 * e) * kS] + w1 * p1[(c + 2 * e) * kS]) * inv,
                         (w0 * p0[(c + 2 * e + 1) * kS] + w1 * p1[(c + 2 * e + 1) * kS]) * inv);
    *reinterpret_cast<uint4*>(orow + c) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ------------------------------------------------------------------- host
// V (and the reference's K) as boxes of 8 channels x 64 keys (tc::make_rows_map).
inline bool make_rows_map(CUtensorMap* tm, const uint16_t* base, cuuint64_t BH, cuuint64_t N, cuuint64_t d,
                          const char* what, std::string* msg) {
  return tc::make_rows_map(tc::encode_fn(), tm, base, BH, N, d, what, msg, kKeys);
}

// bias [H][N rows][N keys] bf16 (or [B * H][N][N], one bias per batch entry),
// rows ld elements apart (ld % 8 == 0), as boxes of 64 keys x 128 rows, 128B
// swizzle.
inline bool make_bias_map(CUtensorMap* tm, const uint16_t* bias, cuuint64_t H, cuuint64_t N,
                          cuuint64_t ld, std::string* msg) {
  tc::EncodeTiledFn enc = tc::encode_fn();
  if (!enc) {
    *msg = "cuTensorMapEncodeTiled entry point unavailable";
    return false;
  }
  const cuuint32_t es[3] = {1, 1, 1};
  const cuuint64_t dims[3] = {N, N, H};
  const cuuint64_t strides[2] = {ld * 2, N * ld * 2};
  const cuuint32_t box[3] = {64, kRows, 1};
  CUresult rc = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(bias), dims, strides, box,
                    es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (rc != CUDA_SUCCESS) {
    *msg = "tensor map (bias) rejected: " + std::to_string(rc);
    return false;
  }
  return true;
}

template <int DV, int kMode, int kBiasKind>
inline int launch(const tc::Params& prm, int ctas, cudaStream_t st, std::string* msg) {
  constexpr bool kBias = kBiasKind == kDenseBias;
  CUtensorMap tm_v, tm_bias, tm_k;
  std::memset(&tm_v, 0, sizeof tm_v);
  std::memset(&tm_bias, 0, sizeof tm_bias);
  std::memset(&tm_k, 0, sizeof tm_k);
  const cuuint64_t BH = static_cast<cuuint64_t>(prm.B) * prm.H;
  if ((kMode == kModeBin || kMode == kModeRef) && !make_rows_map(&tm_v, prm.v, BH, prm.N, prm.d, "V", msg))
    return BINATTN_ERR_CUDA;
  if (kMode == kModeRef && !make_rows_map(&tm_k, prm.k, BH, prm.N, prm.d, "K", msg)) return BINATTN_ERR_CUDA;
  if (kBias && !make_bias_map(&tm_bias, prm.bias, prm.bias_per_sample ? BH : prm.H, prm.N,
                              prm.bias_ld > 0 ? prm.bias_ld : prm.N, msg))
    return BINATTN_ERR_CUDA;
  auto kern = fwd_tc2_kernel<DV, kMode, kBiasKind>;
  constexpr int smem = Layout<DV, kMode, kBiasKind>::kLaunchBytes;
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
  kern<<<static_cast<unsigned>(ctas), kThreads, smem, st>>>(prm, tm_v, tm_bias, tm_k);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *msg = std::string("fwd_tc2_kernel launch: ") + cudaGetErrorString(e);
    return BINATTN_ERR_CUDA;
  }
  return BINATTN_OK;
}

template <int kMode, int kBiasKind>
inline int dispatch_dv(const tc::Params& prm, int ctas, cudaStream_t st, std::string* msg) {
  switch (dv_for(prm.d)) {
    case 32: return launch<32, kMode, kBiasKind>(prm, ctas, st, msg);
    case 64: return launch<64, kMode, kBiasKind>(prm, ctas, st, msg);
    case 80: return launch<80, kMode, kBiasKind>(prm, ctas, st, msg);
    default:
      if constexpr (kMode == kModeRef) {
        *msg = "the reference attention on this pipeline needs d <= 72";
        return BINATTN_ERR_UNSUPPORTED;
      } else {
        return launch<96, kMode, kBiasKind>(prm, ctas, st, msg);
      }
  }
}

// 256-row pairs of a call (one CTA each without a split).
inline int total_pairs(int B, int H, int N) { return B * H * ((N + 2 * kRows - 1) / (2 * kRows)); }

// Tail split: with P pairs on S SMs, the first floor(P / S) * S pairs run as
// whole CTAs; when that is at least one wave, the remaining R pairs fill at
// most one wave twice over (2R <= S) and there are at least 32 key tiles (a
// measured threshold: with 16 or fewer the split costs more than it saves), each
// of the R pairs runs as two CTAs that take one half of the key tiles each,
// and a combine kernel joins the halves. Without a device to ask, no split.
struct SplitPlan {
  int full, tail;
};
inline SplitPlan split_plan(int B, int H, int N) {
  const int P = total_pairs(B, H, N);
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      nsm <= 0) {
    cudaGetLastError();
    return {P, 0};
  }
  const int full = P / nsm * nsm, tail = P - full;
  // worth it only behind at least one whole wave and with enough key tiles
  // that half of them outweighs the extra launch and the combine
  if (full == 0 || tail == 0 || 2 * tail > nsm || (N + kKeys - 1) / kKeys < 32) return {P, 0};
  return {full, tail};
}
// The grid of a launch over P whole pairs: with more pairs than SMs it is
// persistent, one CTA per SM (each CTA holds all of its SM's tensor memory),
// CTA c taking pairs c, c + S, ...; sets prm.npairs and returns the CTA
// count. Otherwise, or without a device to ask, one pair per CTA (npairs = 0).
// Measured on one B200 against one pair per CTA: DeiT-B -16%, ViT-L/16 -9%,
// DiT-XL/2 512 px -6%, DiT-XL/2 1024 px (its 444 whole pairs) -1%, and the
// same or better for both 8-bit P.V passes.
inline int grid_for(tc::Params& prm, int P) {
  prm.npairs = 0;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      nsm <= 0) {
    cudaGetLastError();
    return P;
  }
  if (P <= nsm) return P;
  prm.npairs = P;
  return nsm;
}
// Bytes of the partial results of the split pairs (fp32 O, m, l per row and half).
inline size_t split_part_bytes(int B, int H, int N, int d) {
  const SplitPlan pl = split_plan(B, H, N);
  return static_cast<size_t>(pl.tail) * 2 * kRows * 2 * (d + 2) * 4;
}

// One forward over all pairs of a call. With `part` (split_part_bytes of
// workspace) and a split plan, the whole pairs run as one launch and the tail
// pairs as two key halves each, joined by combine_halves_kernel; without,
// every pair runs whole. run(ctas) launches the kernel with prm. persistent:
// the whole-pair launch may take several pairs per CTA (grid_for); a kernel
// that stages per-head data keeps one pair per CTA.
template <class Run>
inline int run_pairs(tc::Params& prm, float* part, bool persistent, Run run, cudaStream_t st, std::string* msg) {
  const int B = prm.B, H = prm.H, N = prm.N, d = prm.d;
  const SplitPlan plan = part ? split_plan(B, H, N) : SplitPlan{total_pairs(B, H, N), 0};
  if (plan.full > 0) {  // (a split launch takes one pair per CTA and ignores npairs)
    prm.npairs = 0;
    if (int rc = run(persistent ? grid_for(prm, plan.full) : plan.full)) return rc;
  }
  if (plan.tail > 0) {
    prm.pair_base = plan.full;
    prm.split = 1;
    prm.part = part;
    if (int rc = run(2 * plan.tail)) return rc;
    const int rows = plan.tail * 2 * kRows;
    combine_halves_kernel<<<(rows + 255) / 256, 256, 0, st>>>(part, plan.full, plan.tail, B, H, N, d, prm.out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      *msg = std::string("combine_halves_kernel launch: ") + cudaGetErrorString(e);
      return BINATTN_ERR_CUDA;
    }
  }
  return BINATTN_OK;
}

}  // namespace tc2

// part: workspace for the tail split (tc2::split_part_bytes), or null for no split.
// qh: bf16 Q for a forward that binarises Q itself (qb, aq then unused), or null.
// bias_per_sample: the bias is [B, H, N, N] (one per batch entry), not [H, N, N].
inline int forward_tc2(const uint32_t* qb, const uint32_t* kb, const float* aq, const float* ak,
                       const uint16_t* bias, const uint16_t* v, float scale, int B, int H, int N, int d,
                       uint16_t* out, cudaStream_t st, std::string* msg, int bias_ld = 0,
                       float* part = nullptr, const uint16_t* qh = nullptr, int stall_after = -1,
                       bool bias_per_sample = false) {
  tc::Params prm{qb, kb, nullptr, nullptr, aq, ak, bias, v, out, nullptr, scale, B, H, N, d, bias_ld, 0, 0,
                 nullptr, qh, stall_after};
  prm.bias_per_sample = bias_per_sample ? 1 : 0;
  auto run = [&](int ctas) {
    return bias ? tc2::dispatch_dv<tc2::kModeBin, tc2::kDenseBias>(prm, ctas, st, msg)
                : tc2::dispatch_dv<tc2::kModeBin, tc2::kNoBias>(prm, ctas, st, msg);
  };
  return tc2::run_pairs(prm, part, true, run, st, msg);
}

// The binary forward with the position-sensitive bias: table bf16
// [H, (2gh - 1)(2gw - 1) + 3 ncls] of a gh x gw patch grid after ncls class
// tokens (N = ncls + gh * gw), gathered per key from shared memory instead of
// a dense [H, N, N] read. part: as for forward_tc2 (tail split), or null.
inline int forward_tc2_relpos(const uint32_t* qb, const uint32_t* kb, const float* aq, const float* ak,
                              const uint16_t* table, int gh, int gw, int ncls, const uint16_t* v, float scale,
                              int B, int H, int N, int d, uint16_t* out, cudaStream_t st, std::string* msg,
                              float* part) {
  tc::Params prm{qb, kb, nullptr, nullptr, aq, ak, nullptr, v, out, nullptr, scale, B, H, N, d, 0, 0, 0, nullptr};
  prm.rel_table = table;
  prm.rel_gh = gh;
  prm.rel_gw = gw;
  prm.rel_ncls = ncls;
  prm.rel_R = (2 * gh - 1) * (2 * gw - 1) + 3 * ncls;
  // grid rows a whole number of 32-key chunks and no class token: every chunk
  // of keys is one run of the table (N is then a multiple of 32, so a chunk is
  // wholly below N or wholly beyond it)
  const bool rows = ncls == 0 && gw % tc2::kChunk == 0;
  auto run = [&](int ctas) {
    return ncls   ? tc2::dispatch_dv<tc2::kModeBin, tc2::kRelPosBiasCls>(prm, ctas, st, msg)
           : rows ? tc2::dispatch_dv<tc2::kModeBin, tc2::kRelPosBiasRows>(prm, ctas, st, msg)
                  : tc2::dispatch_dv<tc2::kModeBin, tc2::kRelPosBias>(prm, ctas, st, msg);
  };
  // one pair per CTA: the kernel stages one head's table
  return tc2::run_pairs(prm, part, false, run, st, msg);
}

// The 8-bit P.V forward on the 64-key pipeline: the row-max pass writes the
// exact max of every row's logits to mrow, then the 8-bit pass forms
// u = rint(255 exp(logit - max)) and O = s * (u . vq) / sum u with V's tiled
// 8-bit code vq8 and scales vscale (quantize_v_kernel). No tail split.
inline int forward_tc2_int8(const uint32_t* qb, const uint32_t* kb, const float* aq, const float* ak,
                            const uint16_t* bias, int bias_ld, const int8_t* vq8, const float* vscale, float* mrow,
                            float scale, int B, int H, int N, int d, uint16_t* out, cudaStream_t st,
                            std::string* msg) {
  tc::Params prm{qb, kb, nullptr, nullptr, aq, ak, bias, nullptr, out, nullptr, scale, B, H, N, d, bias_ld, 0, 0,
                 nullptr};
  prm.vq8 = vq8;
  prm.vscale = vscale;
  prm.mrow = mrow;
  const int ctas = tc2::grid_for(prm, tc2::total_pairs(B, H, N));
  if (int rc = bias ? tc2::dispatch_dv<tc2::kModeMax, tc2::kDenseBias>(prm, ctas, st, msg)
                    : tc2::dispatch_dv<tc2::kModeMax, tc2::kNoBias>(prm, ctas, st, msg))
    return rc;
  return bias ? tc2::dispatch_dv<tc2::kModeI8, tc2::kDenseBias>(prm, ctas, st, msg)
              : tc2::dispatch_dv<tc2::kModeI8, tc2::kNoBias>(prm, ctas, st, msg);
}

inline int scores_tc2(const uint32_t* qb, const uint32_t* kb, int B, int H, int N, int d, int32_t* S,
                      cudaStream_t st, std::string* msg) {
  tc::Params prm{qb, kb, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, S, 0.f, B, H, N, d, 0, 0, 0,
                 nullptr};
  return tc2::launch<32, tc2::kModeDump, tc2::kNoBias>(prm, tc2::grid_for(prm, tc2::total_pairs(B, H, N)), st,
                                                       msg);
}

// part: workspace for the tail split (tc2::split_part_bytes), or null.
inline int forward_ref_tc2(const uint16_t* q, const uint16_t* k, const uint16_t* bias, const uint16_t* v,
                           float scale, int B, int H, int N, int d, uint16_t* out, cudaStream_t st,
                           std::string* msg, float* part = nullptr) {
  tc::Params prm{nullptr, nullptr, q, k, nullptr, nullptr, bias, v, out, nullptr, scale, B, H, N, d, 0, 0, 0,
                 nullptr};
  auto run = [&](int ctas) {
    return bias ? tc2::dispatch_dv<tc2::kModeRef, tc2::kDenseBias>(prm, ctas, st, msg)
                : tc2::dispatch_dv<tc2::kModeRef, tc2::kNoBias>(prm, ctas, st, msg);
  };
  return tc2::run_pairs(prm, part, true, run, st, msg);
}

}  // namespace binattn
