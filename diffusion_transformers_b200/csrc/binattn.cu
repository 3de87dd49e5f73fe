// binattn.cu — the C ABI of libbinattn (declared in include/binattn.h).
//
// Host-side argument validation, engine dispatch and status reporting. All
// kernels are compiled into this one translation unit from the .cuh files.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "binattn.h"
#include "common.cuh"
#include "pack.cuh"
#include "fwd_simt.cuh"
#include "fwd_tc.cuh"
#include "fwd_tc2.cuh"
#include "quantv.cuh"
#include "bwd_simt.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int status, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

int ok() {
  g_last_error.clear();
  return BINATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1)
    return fail(BINATTN_ERR_SHAPE, "B, H, N, d must be >= 1 (got %d, %d, %d, %d)", B, H, N, d);
  if (d > 128) return fail(BINATTN_ERR_SHAPE, "d = %d > 128 is not supported", d);
  if (static_cast<long long>(B) * H > 65535)
    return fail(BINATTN_ERR_SHAPE, "B*H = %lld > 65535", static_cast<long long>(B) * H);
  if (N > 65535) return fail(BINATTN_ERR_SHAPE, "N = %d > 65535", N);
  return BINATTN_OK;
}

#define BINATTN_CHECK_PTR(p)                                                 \
  do {                                                                       \
    if (!(p)) return fail(BINATTN_ERR_NULL, "%s is NULL", #p);               \
    if (!aligned16(p)) return fail(BINATTN_ERR_ALIGN, "%s is not 16-byte aligned", #p); \
  } while (0)

int launch_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(BINATTN_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
  return ok();
}

int check_forward_args(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                       const float* alpha_k, const uint16_t* bias, const uint16_t* v,
                       float softmax_scale, int B, int H, int N, int d, const uint16_t* out) {
  BINATTN_CHECK_PTR(q_bits);
  BINATTN_CHECK_PTR(k_bits);
  BINATTN_CHECK_PTR(alpha_q);
  BINATTN_CHECK_PTR(alpha_k);
  BINATTN_CHECK_PTR(v);
  BINATTN_CHECK_PTR(out);
  if (bias && !aligned16(bias)) return fail(BINATTN_ERR_ALIGN, "bias is not 16-byte aligned");
  if (!std::isfinite(softmax_scale)) return fail(BINATTN_ERR_ARG, "softmax_scale is not finite");
  return check_shape(B, H, N, d);
}

template <int W>
int launch_simt(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                const float* alpha_k, const uint16_t* bias, const uint16_t* v, float scale,
                int B, int H, int N, int d, uint16_t* out, cudaStream_t st) {
  dim3 grid((N + binattn::kSimtRows - 1) / binattn::kSimtRows, B * H);
  if (bias)
    binattn::fwd_simt_kernel<W, true><<<grid, binattn::kSimtRows, 0, st>>>(
        q_bits, k_bits, alpha_q, alpha_k, bias, v, scale, H, N, d, out);
  else
    binattn::fwd_simt_kernel<W, false><<<grid, binattn::kSimtRows, 0, st>>>(
        q_bits, k_bits, alpha_q, alpha_k, nullptr, v, scale, H, N, d, out);
  return launch_status("fwd_simt_kernel");
}

int forward_simt(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                 const float* alpha_k, const uint16_t* bias, const uint16_t* v, float scale,
                 int B, int H, int N, int d, uint16_t* out, cudaStream_t st) {
  switch (binattn::words_for(d)) {
    case 1: return launch_simt<1>(q_bits, k_bits, alpha_q, alpha_k, bias, v, scale, B, H, N, d, out, st);
    case 2: return launch_simt<2>(q_bits, k_bits, alpha_q, alpha_k, bias, v, scale, B, H, N, d, out, st);
    case 3: return launch_simt<3>(q_bits, k_bits, alpha_q, alpha_k, bias, v, scale, B, H, N, d, out, st);
    default: return launch_simt<4>(q_bits, k_bits, alpha_q, alpha_k, bias, v, scale, B, H, N, d, out, st);
  }
}

template <int W>
int launch_scores_popc(const uint32_t* q_bits, const uint32_t* k_bits, int B, int H, int N,
                       int d, int32_t* S, cudaStream_t st) {
  const long long gx = static_cast<long long>((N + 255) / 256) * N;
  dim3 grid(static_cast<unsigned>(gx), B * H);
  binattn::scores_popc_kernel<W><<<grid, 256, 0, st>>>(q_bits, k_bits, N, d, S);
  return launch_status("scores_popc_kernel");
}

}  // namespace

extern "C" {

int binattn_abi_version(void) { return BINATTN_ABI_VERSION; }

const char* binattn_strerror(int status) {
  switch (status) {
    case BINATTN_OK: return "success";
    case BINATTN_ERR_NULL: return "a required pointer is NULL";
    case BINATTN_ERR_SHAPE: return "B, H, N or d out of range";
    case BINATTN_ERR_DTYPE: return "unknown dtype";
    case BINATTN_ERR_ALIGN: return "pointer not 16-byte aligned";
    case BINATTN_ERR_UNSUPPORTED: return "engine or shape not supported by this build";
    case BINATTN_ERR_CUDA: return "CUDA error";
    case BINATTN_ERR_TIMEOUT: return "a kernel abandoned a bounded wait";
    case BINATTN_ERR_ARG: return "invalid argument";
    default: return "unknown status";
  }
}

const char* binattn_last_error_message(void) { return g_last_error.c_str(); }

int binattn_pack(const void* x, int dtype, int B, int H, int N, int d, uint32_t* bits,
                 float* alpha, void* stream) {
  BINATTN_CHECK_PTR(x);
  BINATTN_CHECK_PTR(bits);
  BINATTN_CHECK_PTR(alpha);
  if (dtype != BINATTN_F32 && dtype != BINATTN_BF16)
    return fail(BINATTN_ERR_DTYPE, "dtype %d is neither BINATTN_F32 nor BINATTN_BF16", dtype);
  if (int rc = check_shape(B, H, N, d)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long n_tokens = static_cast<long long>(B) * H * N;
  const int W = binattn::words_for(d);
  const int esize = dtype == BINATTN_F32 ? 4 : 2;
  const bool vec = (d * esize) % 16 == 0;
  const size_t smem = binattn::pack_smem_bytes(d, esize, vec);
  const unsigned grid = static_cast<unsigned>((n_tokens + binattn::kPackTokens - 1) / binattn::kPackTokens);
  if (dtype == BINATTN_F32) {
    const float* xf = static_cast<const float*>(x);
    if (vec) binattn::pack_kernel<float, true><<<grid, binattn::kPackThreads, smem, st>>>(xf, n_tokens, d, W, bits, alpha);
    else binattn::pack_kernel<float, false><<<grid, binattn::kPackThreads, 0, st>>>(xf, n_tokens, d, W, bits, alpha);
  } else if (d % 8 == 0) {  // whole 16-byte chunks per token: one thread per token
    const uint16_t* xb = static_cast<const uint16_t*>(x);
    constexpr int kT = binattn::kRowsTokens;
    const unsigned rgrid = static_cast<unsigned>((n_tokens + kT - 1) / kT);
    switch (W) {
      case 1: binattn::pack_bf16_rows_kernel<1><<<rgrid, kT, 0, st>>>(xb, n_tokens, d, bits, alpha); break;
      case 2: binattn::pack_bf16_rows_kernel<2><<<rgrid, kT, 0, st>>>(xb, n_tokens, d, bits, alpha); break;
      case 3: binattn::pack_bf16_rows_kernel<3><<<rgrid, kT, 0, st>>>(xb, n_tokens, d, bits, alpha); break;
      default: binattn::pack_bf16_rows_kernel<4><<<rgrid, kT, 0, st>>>(xb, n_tokens, d, bits, alpha); break;
    }
  } else {
    const uint16_t* xb = static_cast<const uint16_t*>(x);
    if (vec) binattn::pack_kernel<uint16_t, true><<<grid, binattn::kPackThreads, smem, st>>>(xb, n_tokens, d, W, bits, alpha);
    else binattn::pack_kernel<uint16_t, false><<<grid, binattn::kPackThreads, 0, st>>>(xb, n_tokens, d, W, bits, alpha);
  }
  return launch_status("pack_kernel");
}

int binattn_forward_engine(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                           const float* alpha_k, const uint16_t* bias, const uint16_t* v,
                           float softmax_scale, int B, int H, int N, int d, uint16_t* out,
                           int engine, void* stream) {
  if (int rc = check_forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out))
    return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (engine == BINATTN_ENGINE_AUTO)
    engine = binattn::tc_built() && binattn::tc_supported(d) ? BINATTN_ENGINE_TC : BINATTN_ENGINE_SIMT;
  switch (engine) {
    case BINATTN_ENGINE_SIMT:
      return forward_simt(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out, st);
    case BINATTN_ENGINE_POPC_TC:
    case BINATTN_ENGINE_TC: {
      if (!binattn::tc_supported(d))
        return fail(BINATTN_ERR_UNSUPPORTED, "engine %d needs d %% 8 == 0 (d = %d)", engine, d);
      std::string msg;
      // TC: e4m3 +-1 operands on the TMA-fed 64-key pipeline where the shape
      // allows (with or without a bias); other shapes use bf16 +-1 operands
      int rc;
      if (engine == BINATTN_ENGINE_TC && binattn::tc2::supported(d, N, bias != nullptr, false))
        rc = binattn::forward_tc2(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out, st,
                                  &msg);
      else
        rc = binattn::forward_tc(engine == BINATTN_ENGINE_TC, q_bits, k_bits, alpha_q, alpha_k, bias, v,
                                 softmax_scale, B, H, N, d, out, st, &msg);
      if (rc) return fail(rc, "%s", msg.c_str());
      return ok();
    }
    default:
      return fail(BINATTN_ERR_ARG, "unknown engine %d", engine);
  }
}

int binattn_forward(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                    const float* alpha_k, const uint16_t* bias, const uint16_t* v,
                    float softmax_scale, int B, int H, int N, int d, uint16_t* out, void* stream) {
  return binattn_forward_engine(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N,
                                d, out, BINATTN_ENGINE_AUTO, stream);
}

namespace {
// Workspace of binattn_forward_ws, for calls that run on the TMA-fed pipeline:
//  [0, pad)          the bias with rows padded to ld = roundup(N, 8) elements,
//                    when N % 8 != 0 (bias rows must be TMA rows);
//  [pad, pad + part) partial results of the split tail pairs (tc2::split_plan).
// pad is rounded up to 256 bytes.
int padded_bias_ld(int N) { return (N + 7) / 8 * 8; }
bool ws_path(int d, int N, bool has_bias) {
  return binattn::tc2::supported(d, N, has_bias, false, has_bias ? padded_bias_ld(N) : 0);
}
// Bytes of the padded bias copy: needed when the bias rows (bias_ld elements
// apart) are not TMA rows. bias_heads: H for a shared bias [H, N, N], B * H
// for one bias per batch entry.
size_t ws_pad_bytes(long long bias_heads, int N, bool has_bias, int bias_ld) {
  if (!has_bias || bias_ld % 8 == 0) return 0;
  return (static_cast<size_t>(bias_heads) * N * padded_bias_ld(N) * 2 + 255) / 256 * 256;
}
size_t ws_bytes(int B, int H, int N, int d, bool has_bias, int bias_ld, bool per_sample = false) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || !ws_path(d, N, has_bias)) return 0;
  const long long bias_heads = per_sample ? static_cast<long long>(B) * H : H;
  return ws_pad_bytes(bias_heads, N, has_bias, bias_ld) + binattn::tc2::split_part_bytes(B, H, N, d);
}
}  // namespace

size_t binattn_forward_workspace_bytes(int B, int H, int N, int d, int has_bias) {
  return ws_bytes(B, H, N, d, has_bias != 0, N);
}

int binattn_padded_bias_ld(int N) { return N < 1 ? 0 : padded_bias_ld(N); }

size_t binattn_forward_bias_ld_workspace_bytes(int B, int H, int N, int d, int bias_ld) {
  if (bias_ld < N) return 0;
  return ws_bytes(B, H, N, d, true, bias_ld);
}

namespace {
// The TMA-fed forward with a workspace (ws_path(d, N, bias) holds): bias rows
// padded into the workspace when N % 8 != 0, a short last wave split by key
// halves, and with qh set, Q binarised inside the kernel.
// bias_ld: elements between the caller's bias rows (>= N). per_sample: the
// bias is [B, H, N, bias_ld] (one per batch entry), not [H, N, bias_ld].
int forward_tma_ws(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q, const float* alpha_k,
                   const uint16_t* bias, int bias_ld, const uint16_t* v, float softmax_scale, int B, int H, int N,
                   int d, uint16_t* out, void* workspace, size_t need, const uint16_t* qh, cudaStream_t st,
                   bool per_sample = false) {
  const long long bias_heads = per_sample ? static_cast<long long>(B) * H : H;
  const size_t pad = ws_pad_bytes(bias_heads, N, bias != nullptr, bias_ld);
  const uint16_t* fbias = bias;
  int ld = bias_ld == N ? 0 : bias_ld;
  if (pad) {
    ld = padded_bias_ld(N);
    uint16_t* padded = static_cast<uint16_t*>(workspace);
    binattn::tc2::pad_bias_rows(bias, bias_heads * N, N, bias_ld, ld, padded, st);
    if (int rc = launch_status("pad_bias_rows_kernel")) return rc;
    fbias = padded;
  }
  float* part = need > pad ? reinterpret_cast<float*>(static_cast<char*>(workspace) + pad) : nullptr;
  std::string msg;
  int rc = binattn::forward_tc2(q_bits, k_bits, alpha_q, alpha_k, fbias, v, softmax_scale, B, H, N, d, out, st,
                                &msg, ld, part, qh, -1, per_sample);
  if (rc) return fail(rc, "%s", msg.c_str());
  return ok();
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Whether binattn_forward_fused_ws binarises Q inside the forward kernel.
bool fused_path(int q_dtype, int d, int N, bool has_bias) { return q_dtype == BINATTN_BF16 && ws_path(d, N, has_bias); }
}  // namespace

int binattn_forward_ws(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                       const float* alpha_k, const uint16_t* bias, const uint16_t* v,
                       float softmax_scale, int B, int H, int N, int d, uint16_t* out,
                       void* workspace, size_t workspace_bytes, void* stream) {
  if (int rc = check_forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out))
    return rc;
  const size_t need = binattn_forward_workspace_bytes(B, H, N, d, bias != nullptr);
  if (need == 0)
    return binattn_forward_engine(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out,
                                  BINATTN_ENGINE_AUTO, stream);
  BINATTN_CHECK_PTR(workspace);
  if (workspace_bytes < need)
    return fail(BINATTN_ERR_ARG, "workspace of %zu bytes is below the %zu this shape needs", workspace_bytes, need);
  return forward_tma_ws(q_bits, k_bits, alpha_q, alpha_k, bias, N, v, softmax_scale, B, H, N, d, out, workspace,
                        need, nullptr, static_cast<cudaStream_t>(stream));
}

int binattn_forward_bias_ld_ws(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                               const float* alpha_k, const uint16_t* bias, int bias_ld, const uint16_t* v,
                               float softmax_scale, int B, int H, int N, int d, uint16_t* out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  BINATTN_CHECK_PTR(bias);
  if (int rc = check_forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out))
    return rc;
  if (bias_ld < N) return fail(BINATTN_ERR_ARG, "bias_ld = %d is below N = %d", bias_ld, N);
  if (bias_ld == N)
    return binattn_forward_ws(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out, workspace,
                              workspace_bytes, stream);
  const size_t need = binattn_forward_bias_ld_workspace_bytes(B, H, N, d, bias_ld);
  if (!ws_path(d, N, true))
    return fail(BINATTN_ERR_UNSUPPORTED, "a strided bias needs the TMA-fed pipeline (d %% 8 == 0, d <= 80); d = %d", d);
  if (need) {
    BINATTN_CHECK_PTR(workspace);
    if (workspace_bytes < need)
      return fail(BINATTN_ERR_ARG, "workspace of %zu bytes is below the %zu this shape needs", workspace_bytes,
                  need);
  }
  return forward_tma_ws(q_bits, k_bits, alpha_q, alpha_k, bias, bias_ld, v, softmax_scale, B, H, N, d, out,
                        workspace, need, nullptr, static_cast<cudaStream_t>(stream));
}

size_t binattn_forward_sample_bias_workspace_bytes(int B, int H, int N, int d, int bias_ld) {
  if (bias_ld < N) return 0;
  return ws_bytes(B, H, N, d, true, bias_ld, true);
}

int binattn_forward_sample_bias_ws(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                                   const float* alpha_k, const uint16_t* bias, int bias_ld, const uint16_t* v,
                                   float softmax_scale, int B, int H, int N, int d, uint16_t* out, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  BINATTN_CHECK_PTR(bias);
  if (int rc = check_forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out))
    return rc;
  if (bias_ld < N) return fail(BINATTN_ERR_ARG, "bias_ld = %d is below N = %d", bias_ld, N);
  if (!ws_path(d, N, true))
    return fail(BINATTN_ERR_UNSUPPORTED,
                "a per-sample bias needs the TMA-fed pipeline (d %% 8 == 0, d <= 80); d = %d", d);
  const size_t need = binattn_forward_sample_bias_workspace_bytes(B, H, N, d, bias_ld);
  if (need) {
    BINATTN_CHECK_PTR(workspace);
    if (workspace_bytes < need)
      return fail(BINATTN_ERR_ARG, "workspace of %zu bytes is below the %zu this shape needs", workspace_bytes,
                  need);
  }
  return forward_tma_ws(q_bits, k_bits, alpha_q, alpha_k, bias, bias_ld, v, softmax_scale, B, H, N, d, out,
                        workspace, need, nullptr, static_cast<cudaStream_t>(stream), true);
}

size_t binattn_forward_fused_workspace_bytes(int B, int H, int N, int d, int q_dtype, int has_bias) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
  const size_t fw = binattn_forward_workspace_bytes(B, H, N, d, has_bias);
  if (fused_path(q_dtype, d, N, has_bias != 0)) return fw;
  const size_t tokens = static_cast<size_t>(B) * H * N;
  return round256(fw) + round256(tokens * binattn::words_for(d) * 4) + round256(tokens * 4);
}

int binattn_forward_fused_ws(const void* q, int q_dtype, const uint32_t* k_bits, const float* alpha_k,
                             const uint16_t* bias, const uint16_t* v, float softmax_scale, int B, int H, int N,
                             int d, uint16_t* out, void* workspace, size_t workspace_bytes, void* stream) {
  BINATTN_CHECK_PTR(q);
  if (q_dtype != BINATTN_F32 && q_dtype != BINATTN_BF16)
    return fail(BINATTN_ERR_DTYPE, "q_dtype %d is neither BINATTN_F32 nor BINATTN_BF16", q_dtype);
  // k_bits stands in for the absent q_bits / alpha_q in the common checks
  if (int rc = check_forward_args(k_bits, k_bits, alpha_k, alpha_k, bias, v, softmax_scale, B, H, N, d, out))
    return rc;
  const size_t need = binattn_forward_fused_workspace_bytes(B, H, N, d, q_dtype, bias != nullptr);
  if (need) {
    BINATTN_CHECK_PTR(workspace);
    if (workspace_bytes < need)
      return fail(BINATTN_ERR_ARG, "workspace of %zu bytes is below the %zu this shape needs", workspace_bytes,
                  need);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t fw = binattn_forward_workspace_bytes(B, H, N, d, bias != nullptr);
  if (fused_path(q_dtype, d, N, bias != nullptr))
    return forward_tma_ws(nullptr, k_bits, nullptr, alpha_k, bias, N, v, softmax_scale, B, H, N, d, out, workspace,
                          fw, static_cast<const uint16_t*>(q), st);
  // Other shapes and fp32 Q: binattn_pack into the workspace, then the forward.
  char* ws = static_cast<char*>(workspace);
  const size_t tokens = static_cast<size_t>(B) * H * N;
  uint32_t* q_bits = reinterpret_cast<uint32_t*>(ws + round256(fw));
  float* alpha_q = reinterpret_cast<float*>(ws + round256(fw) + round256(tokens * binattn::words_for(d) * 4));
  if (int rc = binattn_pack(q, q_dtype, B, H, N, d, q_bits, alpha_q, stream)) return rc;
  return binattn_forward_ws(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out,
                            fw ? workspace : nullptr, fw, stream);
}

namespace {
// Scratch of binattn_forward_static_ws: a file-scope device array, so the call
// needs no allocation. Every device that loads the library holds it until the
// process exits. Host code cannot pass the array's name to a kernel (on the
// host it names a stand-in, not device memory): the device address is looked
// up once per device, with that device current, and kept in g_static_addr.
constexpr size_t kStaticWorkspaceBytes = size_t(32) << 20;
__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];
constexpr int kStaticMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_addr[kStaticMaxDevices];  // null until the device's first call

// Device address of g_static_workspace on the current device.
int static_workspace_addr(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(BINATTN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kStaticMaxDevices)
    return fail(BINATTN_ERR_UNSUPPORTED, "device %d is beyond the %d the static workspace tracks", dev,
                kStaticMaxDevices);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return fail(BINATTN_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_static_addr[dev] = p;
  }
  *addr = g_static_addr[dev];
  return BINATTN_OK;
}
}  // namespace

// Nothing in the workspace has to start at zero: every byte a call reads from
// it (the padded bias copy, the partials of split pairs) is written earlier in
// the same call, so the previous call's contents never leak into a result.
int binattn_forward_static_ws(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                              const float* alpha_k, const uint16_t* bias, const uint16_t* v,
                              float softmax_scale, int B, int H, int N, int d, uint16_t* out,
                              void* stream) {
  if (int rc = check_forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out))
    return rc;
  const size_t need = binattn_forward_workspace_bytes(B, H, N, d, bias != nullptr);
  if (need > kStaticWorkspaceBytes)
    return fail(BINATTN_ERR_UNSUPPORTED, "this shape needs %zu bytes of workspace; the static one holds %zu",
                need, kStaticWorkspaceBytes);
  void* ws = nullptr;
  if (int rc = static_workspace_addr(&ws)) return rc;
  return binattn_forward_ws(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out, ws,
                            kStaticWorkspaceBytes, stream);
}

namespace {
// V's 8-bit code: the channel maxima into maxbits (zeroed first), the codes
// (tiled with DV columns and / or plain), then the scales.
int quantize_v_launch(const uint16_t* v, int B, int H, int N, int d, int DV, int* maxbits, int8_t* tiled,
                      int8_t* plain, float* scale, cudaStream_t st) {
  const size_t nmax = static_cast<size_t>(B) * H * d;
  cudaError_t e = cudaMemsetAsync(maxbits, 0, nmax * sizeof(int), st);
  if (e != cudaSuccess) return fail(BINATTN_ERR_CUDA, "memset of the V maxima: %s", cudaGetErrorString(e));
  const dim3 gmax(static_cast<unsigned>(B * H), static_cast<unsigned>((N + binattn::kQvThreads - 1) / binattn::kQvThreads));
  binattn::vmax_kernel<<<gmax, binattn::kQvThreads, 0, st>>>(v, N, d, maxbits);
  if (int rc = launch_status("vmax_kernel")) return rc;
  const dim3 gq(static_cast<unsigned>(B * H), static_cast<unsigned>((N + 63) / 64));
  binattn::vquant_kernel<<<gq, binattn::kQvThreads, 0, st>>>(v, N, d, DV, maxbits, tiled, plain);
  if (int rc = launch_status("vquant_kernel")) return rc;
  binattn::vscale_kernel<<<static_cast<unsigned>((nmax + 255) / 256), 256, 0, st>>>(maxbits, static_cast<long long>(nmax), scale);
  return launch_status("vscale_kernel");
}
}  // namespace

int binattn_quantize_v(const uint16_t* v, int B, int H, int N, int d, int8_t* vq, float* scale, void* stream) {
  BINATTN_CHECK_PTR(v);
  BINATTN_CHECK_PTR(vq);
  BINATTN_CHECK_PTR(scale);
  if (int rc = check_shape(B, H, N, d)) return rc;
  if (d % 8 != 0) return fail(BINATTN_ERR_UNSUPPORTED, "the 8-bit V code needs d %% 8 == 0 (d = %d)", d);
  // the scales' buffer holds the maxima until the codes are written
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return quantize_v_launch(v, B, H, N, d, 0, reinterpret_cast<int*>(scale), nullptr, vq, scale, st);
}

namespace {
// Workspace of binattn_forward_int8: V's tiled 8-bit code, its scales, the row
// maxima, and with N % 8 != 0 the bias with padded rows.
struct Int8Ws {
  size_t vq, scale, mrow, vmax, pad, total;
};
Int8Ws int8_ws(int B, int H, int N, int d, bool has_bias) {
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t nkt = (static_cast<size_t>(N) + 63) / 64;
  Int8Ws w;
  w.vq = round256(BH * nkt * binattn::tc2::dv_for(d) * 64);
  w.scale = round256(BH * d * 4);
  w.mrow = round256(BH * N * 4);
  w.vmax = round256(BH * d * 4);
  w.pad = ws_pad_bytes(H, N, has_bias, N);
  w.total = w.vq + w.scale + w.mrow + w.vmax + w.pad;
  return w;
}
bool int8_path(int d, int N, bool has_bias) {
  return binattn::tc2::supported(d, N, has_bias, false, has_bias ? padded_bias_ld(N) : 0);
}
}  // namespace

size_t binattn_forward_int8_workspace_bytes(int B, int H, int N, int d, int has_bias) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || !int8_path(d, N, has_bias != 0)) return 0;
  return int8_ws(B, H, N, d, has_bias != 0).total;
}

int binattn_forward_int8(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q, const float* alpha_k,
                         const uint16_t* bias, const uint16_t* v, float softmax_scale, int B, int H, int N, int d,
                         uint16_t* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (int rc = check_forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out))
    return rc;
  if (!int8_path(d, N, bias != nullptr))
    return fail(BINATTN_ERR_UNSUPPORTED, "the 8-bit P.V forward needs d %% 8 == 0 and d <= 80 (d = %d)", d);
  BINATTN_CHECK_PTR(workspace);
  const Int8Ws w = int8_ws(B, H, N, d, bias != nullptr);
  if (workspace_bytes < w.total)
    return fail(BINATTN_ERR_ARG, "workspace of %zu bytes is below the %zu this shape needs", workspace_bytes, w.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int8_t* vq8 = reinterpret_cast<int8_t*>(ws);
  float* vscale = reinterpret_cast<float*>(ws + w.vq);
  float* mrow = reinterpret_cast<float*>(ws + w.vq + w.scale);
  int* vmax = reinterpret_cast<int*>(ws + w.vq + w.scale + w.mrow);
  const uint16_t* fbias = bias;
  int ld = 0;
  if (w.pad) {
    ld = padded_bias_ld(N);
    uint16_t* padded = reinterpret_cast<uint16_t*>(ws + w.vq + w.scale + w.mrow + w.vmax);
    binattn::tc2::pad_bias_rows(bias, static_cast<long long>(H) * N, N, N, ld, padded, st);
    if (int rc = launch_status("pad_bias_rows_kernel")) return rc;
    fbias = padded;
  }
  if (int rc = quantize_v_launch(v, B, H, N, d, binattn::tc2::dv_for(d), vmax, vq8, nullptr, vscale, st)) return rc;
  std::string msg;
  if (int rc = binattn::forward_tc2_int8(q_bits, k_bits, alpha_q, alpha_k, fbias, ld, vq8, vscale, mrow,
                                         softmax_scale, B, H, N, d, out, st, &msg))
    return fail(rc, "%s", msg.c_str());
  return ok();
}

size_t binattn_forward_relpos_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || !binattn::tc2::supported(d, N, false, false)) return 0;
  return binattn::tc2::split_part_bytes(B, H, N, d);
}

int binattn_forward_relpos(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                           const float* alpha_k, const uint16_t* table, int gh, int gw, int n_cls,
                           const uint16_t* v, float softmax_scale, int B, int H, int N, int d, uint16_t* out,
                           void* workspace, size_t workspace_bytes, void* stream) {
  BINATTN_CHECK_PTR(table);
  if (int rc = check_forward_args(q_bits, k_bits, alpha_q, alpha_k, nullptr, v, softmax_scale, B, H, N, d, out))
    return rc;
  if (gh < 1 || gw < 1 || (n_cls != 0 && n_cls != 1) || static_cast<long long>(gh) * gw + n_cls != N)
    return fail(BINATTN_ERR_SHAPE, "N = %d is not n_cls + gh * gw (%d + %d * %d)", N, n_cls, gh, gw);
  const long long R = static_cast<long long>(2 * gh - 1) * (2 * gw - 1) + 3 * n_cls;
  if (R > binattn::tc2::kRelTabMax)
    return fail(BINATTN_ERR_UNSUPPORTED, "a %lld-entry table is more than the %d that fit in shared memory", R,
                binattn::tc2::kRelTabMax);
  if (!binattn::tc2::supported(d, N, false, false))
    return fail(BINATTN_ERR_UNSUPPORTED, "the position-sensitive bias needs d %% 8 == 0 and d <= 80 (d = %d)", d);
  const size_t need = binattn_forward_relpos_workspace_bytes(B, H, N, d);
  if (need) {
    BINATTN_CHECK_PTR(workspace);
    if (workspace_bytes < need)
      return fail(BINATTN_ERR_ARG, "workspace of %zu bytes is below the %zu this shape needs", workspace_bytes,
                  need);
  }
  std::string msg;
  if (int rc = binattn::forward_tc2_relpos(q_bits, k_bits, alpha_q, alpha_k, table, gh, gw, n_cls, v,
                                           softmax_scale, B, H, N, d, out, static_cast<cudaStream_t>(stream), &msg,
                                           need ? static_cast<float*>(workspace) : nullptr))
    return fail(rc, "%s", msg.c_str());
  return ok();
}

int binattn_scores_debug(const uint32_t* q_bits, const uint32_t* k_bits, int B, int H, int N,
                         int d, int32_t* S, int engine, void* stream) {
  BINATTN_CHECK_PTR(q_bits);
  BINATTN_CHECK_PTR(k_bits);
  BINATTN_CHECK_PTR(S);
  if (int rc = check_shape(B, H, N, d)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (engine == BINATTN_ENGINE_AUTO)
    engine = binattn::tc_built() && binattn::tc_supported(d) ? BINATTN_ENGINE_TC : BINATTN_ENGINE_SIMT;
  switch (engine) {
    case BINATTN_ENGINE_SIMT:
    case BINATTN_ENGINE_POPC_TC:
      switch (binattn::words_for(d)) {
        case 1: return launch_scores_popc<1>(q_bits, k_bits, B, H, N, d, S, st);
        case 2: return launch_scores_popc<2>(q_bits, k_bits, B, H, N, d, S, st);
        case 3: return launch_scores_popc<3>(q_bits, k_bits, B, H, N, d, S, st);
        default: return launch_scores_popc<4>(q_bits, k_bits, B, H, N, d, S, st);
      }
    case BINATTN_ENGINE_TC:
    case BINATTN_ENGINE_TC_BIASED: {
      if (!binattn::tc_supported(d))
        return fail(BINATTN_ERR_UNSUPPORTED, "engine TC needs d %% 8 == 0 (d = %d)", d);
      // the kernel the TC forward runs for this shape: the TMA-fed 64-key
      // pipeline, else the load-mode one
      std::string msg;
      int rc;
      if (binattn::tc2::supported(d, N, false, false))
        rc = binattn::scores_tc2(q_bits, k_bits, B, H, N, d, S, st, &msg);
      else
        rc = binattn::scores_tc(q_bits, k_bits, B, H, N, d, S, st, &msg);
      if (rc) return fail(rc, "%s", msg.c_str());
      return ok();
    }
    default:
      return fail(BINATTN_ERR_ARG, "unknown engine %d", engine);
  }
}

static int ref_bf16_forward(const uint16_t* q, const uint16_t* k, const uint16_t* bias, const uint16_t* v,
                            float softmax_scale, int B, int H, int N, int d, uint16_t* out, float* part,
                            void* stream) {
  BINATTN_CHECK_PTR(q);
  BINATTN_CHECK_PTR(k);
  BINATTN_CHECK_PTR(v);
  BINATTN_CHECK_PTR(out);
  if (bias && !aligned16(bias)) return fail(BINATTN_ERR_ALIGN, "bias is not 16-byte aligned");
  if (!std::isfinite(softmax_scale)) return fail(BINATTN_ERR_ARG, "softmax_scale is not finite");
  if (int rc = check_shape(B, H, N, d)) return rc;
  if (!binattn::tc_supported(d))
    return fail(BINATTN_ERR_UNSUPPORTED, "the bf16 reference needs d %% 8 == 0 (d = %d)", d);
  std::string msg;
  int rc = binattn::tc2::supported(d, N, bias != nullptr, true)
               ? binattn::forward_ref_tc2(q, k, bias, v, softmax_scale, B, H, N, d, out,
                                          static_cast<cudaStream_t>(stream), &msg, part)
               : binattn::forward_ref_bf16(q, k, bias, v, softmax_scale, B, H, N, d, out,
                                           static_cast<cudaStream_t>(stream), &msg);
  if (rc) return fail(rc, "%s", msg.c_str());
  return ok();
}

int binattn_ref_bf16_forward(const uint16_t* q, const uint16_t* k, const uint16_t* bias,
                             const uint16_t* v, float softmax_scale, int B, int H, int N, int d,
                             uint16_t* out, void* stream) {
  return ref_bf16_forward(q, k, bias, v, softmax_scale, B, H, N, d, out, nullptr, stream);
}

size_t binattn_ref_bf16_forward_workspace_bytes(int B, int H, int N, int d, int has_bias) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || !binattn::tc2::supported(d, N, has_bias != 0, true)) return 0;
  return binattn::tc2::split_part_bytes(B, H, N, d);
}

int binattn_ref_bf16_forward_ws(const uint16_t* q, const uint16_t* k, const uint16_t* bias, const uint16_t* v,
                                float softmax_scale, int B, int H, int N, int d, uint16_t* out,
                                void* workspace, size_t workspace_bytes, void* stream) {
  const size_t need = (B >= 1 && H >= 1 && N >= 1 && d >= 1)
                          ? binattn_ref_bf16_forward_workspace_bytes(B, H, N, d, bias != nullptr)
                          : 0;
  if (need) {
    BINATTN_CHECK_PTR(workspace);
    if (workspace_bytes < need)
      return fail(BINATTN_ERR_ARG, "workspace of %zu bytes is below the %zu this shape needs", workspace_bytes,
                  need);
  }
  return ref_bf16_forward(q, k, bias, v, softmax_scale, B, H, N, d, out,
                          need ? static_cast<float*>(workspace) : nullptr, stream);
}

int binattn_test_wait_timeout(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q,
                              const float* alpha_k, const uint16_t* bias, const uint16_t* v,
                              float softmax_scale, int B, int H, int N, int d, uint16_t* out,
                              int stall_after, void* stream) {
  if (int rc = check_forward_args(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out))
    return rc;
  if (!binattn::tc2::supported(d, N, bias != nullptr, false))
    return fail(BINATTN_ERR_UNSUPPORTED, "the 64-key pipeline does not take d = %d, N = %d", d, N);
  if (stall_after < 0) return fail(BINATTN_ERR_ARG, "stall_after must be >= 0");
  std::string msg;
  const int rc = binattn::forward_tc2(q_bits, k_bits, alpha_q, alpha_k, bias, v, softmax_scale, B, H, N, d, out,
                                      static_cast<cudaStream_t>(stream), &msg, 0, nullptr, nullptr, stall_after);
  if (rc) return fail(rc, "%s", msg.c_str());
  return ok();
}

size_t binattn_backward_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || d > 128 || static_cast<long long>(B) * H > 65535 || N > 65535) return 0;
  // LSE and D, one float each per query row
  return (2 * static_cast<size_t>(B) * H * N * sizeof(float) + 255) / 256 * 256;
}

int binattn_backward(const uint32_t* q_bits, const uint32_t* k_bits, const float* alpha_q, const float* alpha_k,
                     const uint16_t* bias, const uint16_t* v, const uint16_t* dO, float softmax_scale, int B, int H,
                     int N, int d, float* dV, float* ds, float* dt, float* dbias, void* workspace,
                     size_t workspace_bytes, void* stream) {
  BINATTN_CHECK_PTR(q_bits);
  BINATTN_CHECK_PTR(k_bits);
  BINATTN_CHECK_PTR(alpha_q);
  BINATTN_CHECK_PTR(alpha_k);
  BINATTN_CHECK_PTR(v);
  BINATTN_CHECK_PTR(dO);
  BINATTN_CHECK_PTR(dV);
  BINATTN_CHECK_PTR(ds);
  BINATTN_CHECK_PTR(dt);
  BINATTN_CHECK_PTR(workspace);
  if (bias && !aligned16(bias)) return fail(BINATTN_ERR_ALIGN, "bias is not 16-byte aligned");
  if (dbias && !aligned16(dbias)) return fail(BINATTN_ERR_ALIGN, "dbias is not 16-byte aligned");
  if (!std::isfinite(softmax_scale)) return fail(BINATTN_ERR_ARG, "softmax_scale is not finite");
  if (int rc = check_shape(B, H, N, d)) return rc;
  const size_t need = binattn_backward_workspace_bytes(B, H, N, d);
  if (workspace_bytes < need)
    return fail(BINATTN_ERR_ARG, "workspace of %zu bytes is below the %zu this shape needs", workspace_bytes, need);
  float* lse = static_cast<float*>(workspace);
  float* D = lse + static_cast<size_t>(B) * H * N;
  std::string msg;
  if (binattn::bwd::backward(q_bits, k_bits, alpha_q, alpha_k, bias, v, dO, softmax_scale, B, H, N, d, dV, ds, dt,
                             dbias, lse, D, static_cast<cudaStream_t>(stream), &msg))
    return fail(BINATTN_ERR_CUDA, "%s", msg.c_str());
  return ok();
}

int binattn_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(BINATTN_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  int status = 0;
  e = cudaMemcpyFromSymbol(&status, binattn::g_device_status, sizeof(int));
  if (e != cudaSuccess) return fail(BINATTN_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  const int zero = 0;
  e = cudaMemcpyToSymbol(binattn::g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return fail(BINATTN_ERR_CUDA, "status clear: %s", cudaGetErrorString(e));
  if (status != 0) return fail(BINATTN_ERR_TIMEOUT, "device status code %d", status);
  return ok();
}

}  // extern "C"
