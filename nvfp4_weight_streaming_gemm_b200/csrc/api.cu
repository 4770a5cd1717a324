// The C ABI of libnvfp4ws (include/nvfp4ws.h): argument validation, workspace
// sizing, kernel-path dispatch and error reporting. Every check runs on the host
// before anything is enqueued.
#include "common.cuh"
#include "fp8.h"
#include "kernels.h"
#include "mma.h"

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <vector>

namespace nvfp4ws {

static thread_local char g_last_error[512] = "";
__device__ unsigned int g_device_error = 0u;

int set_error(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

void clear_error() { g_last_error[0] = 0; }

static std::atomic<unsigned long long> g_launches{0};

int check_launch(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(NVFP4WS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return NVFP4WS_OK;
}

unsigned int* device_error_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  return static_cast<unsigned int*>(p);
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared validation of the GEMM-shaped calls.
static int validate_gemm(const void* X, const uint8_t* q, const uint8_t* sf, const float* ts, int64_t M,
                         int64_t N, int64_t K, const char* who) {
  if (!X || !q || !sf || !ts) return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: null input pointer", who);
  if (M < 1 || N < 1 || K < 1) return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: M, N, K must be >= 1", who);
  if (M > NVFP4WS_MAX_M)
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "%s: M=%lld exceeds %d", who, (long long)M, NVFP4WS_MAX_M);
  if (K % 32 != 0) return set_error(NVFP4WS_ERR_UNSUPPORTED, "%s: K=%lld is not a multiple of 32", who, (long long)K);
  if (N > (int64_t)0x7fffffff || K > ((int64_t)1 << 24))
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "%s: N or K too large", who);
  if (!aligned16(X) || !aligned16(q) || !aligned16(sf))
    return set_error(NVFP4WS_ERR_MISALIGNED, "%s: X, q and sf must be 16-byte aligned", who);
  return NVFP4WS_OK;
}

// Kernel actually used for a request: MMA means the block-scaled kernel when the
// shape allows it, else the f16 tensor-core kernel.
// MXF4_ROWS: the block-scaled kernel over consecutive slices of X's rows, one launch each.
enum { KPATH_GEMV = 1, KPATH_MXF4 = 2, KPATH_GEMV_REGS = 3, KPATH_MMA_F16 = 4, KPATH_MXF4_ROWS = 5, KPATH_NONE = 0 };

// Rows per launch when a GEMM's M exceeds what one block-scaled launch serves (M * 5 <= 352):
// ceil(M / 70) slices of equal size. Each slice re-reads the weight, but at these M the f16
// kernel is bound by its MMA issue rate (measured on the 27B gate+up shape: 204 us at M = 128
// against 59 us at M = 68 on the block-scaled kernel), and past M = 128 only the GEMV is left.
static int64_t mxf4_slice_rows(int64_t M) {
  const int64_t cap = 352 / kGemmTerms;
  const int64_t n = (M + cap - 1) / cap;
  return (M + n - 1) / n;
}

// terms: activation terms of the block-scaled kernel for this call (a GEMM's or the verify's).
// row_slices: AUTO may run the block-scaled kernel over slices of X's rows (GEMMs only).
static int resolve_path(int path, int64_t M, int64_t K, int terms = kGemmTerms, bool row_slices = false) {
  switch (path) {
    case NVFP4WS_PATH_AUTO:
      // The block-scaled tensor-core kernel whenever it applies, M = 1 included: on B200 a
      // CUDA-core GEMV spends ~3.4 instructions per weight element on dequantisation and
      // products, more than an SM can issue at HBM rate (measured: 1.5 of 4 per cycle, 0.3-0.5
      // of HBM), while kind::mxf4nvf4 takes the packed weights with no per-element work.
      if (mxf4_supported(M, K, terms)) return KPATH_MXF4;
      if (row_slices && mxf4_supported(mxf4_slice_rows(M), K, terms)) return KPATH_MXF4_ROWS;
      if (M >= mma_min_m() && mma_supported(M, K)) return KPATH_MMA_F16;
      return KPATH_GEMV;
    case NVFP4WS_PATH_GEMV: return KPATH_GEMV;
    case NVFP4WS_PATH_GEMV_REGS: return KPATH_GEMV_REGS;
    case NVFP4WS_PATH_MMA:
      if (mxf4_supported(M, K, terms)) return KPATH_MXF4;
      return mma_supported(M, K) ? KPATH_MMA_F16 : KPATH_NONE;
    case NVFP4WS_PATH_MMA_F16: return mma_supported(M, K) ? KPATH_MMA_F16 : KPATH_NONE;
    default: return KPATH_NONE;
  }
}

// Workspace that serves every path supporting the shape.
static size_t gemm_ws_any(int64_t M, int64_t N, int64_t K) {
  size_t a = mma_supported(M, K) ? mma_gemm_workspace_bytes(M, N, K) : 0;
  size_t b = mxf4_supported(M, K) ? mxf4_workspace_bytes(M, N, K) : 0;
  const int64_t mr = mxf4_slice_rows(M);
  size_t c = (!mxf4_supported(M, K) && mxf4_supported(mr, K)) ? mxf4_workspace_bytes(mr, N, K) : 0;
  return std::max(a, std::max(b, c));
}

}  // namespace nvfp4ws

using namespace nvfp4ws;

extern "C" {

const char* nvfp4ws_status_string(int status) {
  switch (status) {
    case NVFP4WS_OK: return "NVFP4WS_OK";
    case NVFP4WS_ERR_INVALID_ARG: return "NVFP4WS_ERR_INVALID_ARG";
    case NVFP4WS_ERR_UNSUPPORTED: return "NVFP4WS_ERR_UNSUPPORTED";
    case NVFP4WS_ERR_MISALIGNED: return "NVFP4WS_ERR_MISALIGNED";
    case NVFP4WS_ERR_WORKSPACE: return "NVFP4WS_ERR_WORKSPACE";
    case NVFP4WS_ERR_CUDA: return "NVFP4WS_ERR_CUDA";
    case NVFP4WS_ERR_DEVICE_TIMEOUT: return "NVFP4WS_ERR_DEVICE_TIMEOUT";
    default: return "NVFP4WS_UNKNOWN_STATUS";
  }
}

const char* nvfp4ws_last_error(void) { return g_last_error; }

int nvfp4ws_version(void) { return 201; }

int nvfp4ws_sm_count(void) { return device_sm_count(); }

unsigned long long nvfp4ws_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int nvfp4_pack(const float* W, int64_t N, int64_t K, uint8_t* q, uint8_t* sf, float* tensor_scale,
               const float* tensor_scale_in, nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  if (!W || !q || !sf || !tensor_scale) return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pack: null pointer");
  if (N < 1 || K < 16 || K % 16 != 0)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pack: need N >= 1 and K a positive multiple of 16");
  if (!aligned16(W) || !aligned16(q))
    return set_error(NVFP4WS_ERR_MISALIGNED, "nvfp4_pack: W and q must be 16-byte aligned");
  if (((uintptr_t)tensor_scale & 3u) || ((uintptr_t)tensor_scale_in & 3u))
    return set_error(NVFP4WS_ERR_MISALIGNED, "nvfp4_pack: tensor scales must be 4-byte aligned");
  return launch_pack(W, N, K, q, sf, tensor_scale, tensor_scale_in, (cudaStream_t)stream);
}

size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 32) return 0;
  return gemm_ws_any(M, N, K);   // enough for every path that supports the shape, so a forced path works too
}

int nvfp4_gemm_skinny_path(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale,
                           int64_t M, int64_t N, int64_t K, void* Y, int y_dtype, void* workspace,
                           size_t workspace_bytes, int path, nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  if (int e = validate_gemm(X, q, sf, tensor_scale, M, N, K, "nvfp4_gemm_skinny")) return e;
  if (!Y) return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_gemm_skinny: Y is null");
  if (!aligned16(Y)) return set_error(NVFP4WS_ERR_MISALIGNED, "nvfp4_gemm_skinny: Y must be 16-byte aligned");
  if (y_dtype != NVFP4WS_Y_F32 && y_dtype != NVFP4WS_Y_BF16)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_gemm_skinny: bad y_dtype %d", y_dtype);
  if (path < NVFP4WS_PATH_AUTO || path > NVFP4WS_PATH_MMA_F16)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_gemm_skinny: bad path %d", path);
  const int kp = resolve_path(path, M, K, kGemmTerms, true);
  cudaStream_t s = (cudaStream_t)stream;
  if (kp == KPATH_NONE)
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "nvfp4_gemm_skinny: the tensor-core paths need K %% 256 == 0 and "
                     "M <= 128 (M=%lld K=%lld)", (long long)M, (long long)K);
  if (kp == KPATH_MXF4_ROWS) {
    // The slices run one after another on the stream and share the workspace: each launch's
    // prep kernel waits for the previous GEMM to finish before it rewrites the images, and
    // every launch leaves its tickets zero.
    const int64_t mr = mxf4_slice_rows(M);
    size_t need = mxf4_workspace_bytes(mr, N, K);
    if (workspace == nullptr || workspace_bytes < need)
      return set_error(NVFP4WS_ERR_WORKSPACE, "nvfp4_gemm_skinny: workspace needs %zu bytes", need);
    if (!aligned16(workspace))
      return set_error(NVFP4WS_ERR_MISALIGNED, "nvfp4_gemm_skinny: workspace must be 16-byte aligned");
    const size_t ysz = y_dtype == NVFP4WS_Y_BF16 ? 2 : 4;
    for (int64_t m0 = 0; m0 < M; m0 += mr) {
      const int64_t m = std::min(mr, M - m0);
      if (int e = launch_mxf4_gemm(static_cast<const uint16_t*>(X) + m0 * K, q, sf, tensor_scale, m, N, K,
                                   static_cast<char*>(Y) + (size_t)(m0 * N) * ysz, y_dtype, workspace, s))
        return e;
    }
    return NVFP4WS_OK;
  }
  if (kp == KPATH_MXF4) {
    size_t need = mxf4_workspace_bytes(M, N, K);
    if (workspace == nullptr || workspace_bytes < need)
      return set_error(NVFP4WS_ERR_WORKSPACE, "nvfp4_gemm_skinny: workspace needs %zu bytes", need);
    if (!aligned16(workspace))
      return set_error(NVFP4WS_ERR_MISALIGNED, "nvfp4_gemm_skinny: workspace must be 16-byte aligned");
    return launch_mxf4_gemm(static_cast<const uint16_t*>(X), q, sf, tensor_scale, M, N, K, Y, y_dtype, workspace, s);
  }
  if (kp == KPATH_MMA_F16) {
    size_t need = mma_gemm_workspace_bytes(M, N, K);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need))
      return set_error(NVFP4WS_ERR_WORKSPACE, "nvfp4_gemm_skinny: workspace needs %zu bytes", need);
    if (need > 0 && !aligned16(workspace))
      return set_error(NVFP4WS_ERR_MISALIGNED, "nvfp4_gemm_skinny: workspace must be 16-byte aligned");
    return launch_mma_gemm(static_cast<const uint16_t*>(X), q, sf, tensor_scale, M, N, K, Y, y_dtype,
                           workspace, workspace_bytes, s);
  }
  if (!gemv_supported(K))
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "nvfp4_gemm_skinny: GEMV path supports K <= 65536");
  GemvArgs a{};
  a.X = static_cast<const uint16_t*>(X);
  a.q = q; a.sf = sf; a.ts = tensor_scale;
  a.M = M; a.N = N; a.K = K;
  a.Y = Y; a.y_bf16 = (y_dtype == NVFP4WS_Y_BF16);
  return launch_gemv(a, false, kp == KPATH_GEMV_REGS, s);
}

int nvfp4_gemm_skinny(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale, int64_t M,
                      int64_t N, int64_t K, void* Y, int y_dtype, void* workspace, size_t workspace_bytes,
                      nvfp4ws_stream_t stream) {
  return nvfp4_gemm_skinny_path(X, q, sf, tensor_scale, M, N, K, Y, y_dtype, workspace, workspace_bytes,
                                NVFP4WS_PATH_AUTO, stream);
}

size_t nvfp4_gemm_w4a4_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > NVFP4WS_MAX_M || N < 1) return 0;
  return mxf4_workspace_bytes(M, N, K, 1);
}

int nvfp4_gemm_w4a4(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale, int64_t M,
                    int64_t N, int64_t K, void* Y, int y_dtype, void* workspace, size_t workspace_bytes,
                    nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  if (int e = validate_gemm(X, q, sf, tensor_scale, M, N, K, "nvfp4_gemm_w4a4")) return e;
  if (!Y) return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_gemm_w4a4: Y is null");
  if (!aligned16(Y)) return set_error(NVFP4WS_ERR_MISALIGNED, "nvfp4_gemm_w4a4: Y must be 16-byte aligned");
  if (y_dtype != NVFP4WS_Y_F32 && y_dtype != NVFP4WS_Y_BF16)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_gemm_w4a4: bad y_dtype %d", y_dtype);
  if (!mxf4_supported(M, K, 1))
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "nvfp4_gemm_w4a4: needs K %% 256 == 0, 256 <= K <= 32768 (K=%lld)",
                     (long long)K);
  const size_t need = mxf4_workspace_bytes(M, N, K, 1);
  if (workspace == nullptr || workspace_bytes < need)
    return set_error(NVFP4WS_ERR_WORKSPACE, "nvfp4_gemm_w4a4: workspace needs %zu bytes", need);
  if (!aligned16(workspace)) return set_error(NVFP4WS_ERR_MISALIGNED, "nvfp4_gemm_w4a4: workspace must be 16-byte aligned");
  return launch_mxf4_gemm(static_cast<const uint16_t*>(X), q, sf, tensor_scale, M, N, K, Y, y_dtype, workspace,
                          (cudaStream_t)stream, 1);
}

// Largest partial-argmax grid of the two GEMV variants, so either fits the workspace.
static int gemv_verify_grid(int64_t M, int64_t N, int64_t K) {
  GemvPlan a = gemv_plan(M, N, K, false), b = gemv_plan(M, N, K, true);
  return a.grid > b.grid ? a.grid : b.grid;
}

static size_t gemv_verify_workspace(int64_t M, int64_t N, int64_t K) {
  return 2 * align_up((size_t)gemv_verify_grid(M, N, K) * (size_t)M * 4, 256);
}

size_t lmhead_verify_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 32) return 0;
  size_t w = gemv_verify_workspace(M, N, K);
  size_t m = mma_supported(M, K) ? mma_verify_workspace_bytes(M, N, K) : 0;
  size_t x = mxf4_supported(M, K, kVerifyTerms) ? mxf4_workspace_bytes(M, N, K, kVerifyTerms) : 0;
  if (m > w) w = m;
  return x > w ? x : w;
}

}  // extern "C"

// The lm_head GEMM and its fused verify, chain (v.parents == null) or tree.
static int verify_impl(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale, int64_t M,
                       int64_t N, int64_t K, const VerifyRule& v, void* workspace, size_t workspace_bytes, int path,
                       cudaStream_t s) {
  const int32_t* drafts = v.drafts;
  const int32_t B = v.B, D = v.D;
  int32_t *argmax = v.argmax, *accept_len = v.accept_len;
  if (int e = validate_gemm(X, q, sf, tensor_scale, M, N, K, "lmhead_verify")) return e;
  if (B < 1 || D < 0) return set_error(NVFP4WS_ERR_INVALID_ARG, "lmhead_verify: need B >= 1 and D >= 0");
  if ((int64_t)B * (D + 1) != M)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "lmhead_verify: M=%lld must equal B*(D+1)=%lld", (long long)M,
                     (long long)B * (D + 1));
  if (D > 0 && !drafts) return set_error(NVFP4WS_ERR_INVALID_ARG, "lmhead_verify: drafts is null");
  if (!argmax || !accept_len) return set_error(NVFP4WS_ERR_INVALID_ARG, "lmhead_verify: null output pointer");
  if (path < NVFP4WS_PATH_AUTO || path > NVFP4WS_PATH_MMA_F16)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "lmhead_verify: bad path %d", path);
  const int kp = resolve_path(path, M, K, kVerifyTerms);
  if (kp == KPATH_NONE)
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "lmhead_verify: the tensor-core paths need K %% 256 == 0 and "
                     "M <= 128 (M=%lld K=%lld)", (long long)M, (long long)K);
  if (kp == KPATH_MXF4) {
    size_t need = mxf4_workspace_bytes(M, N, K, kVerifyTerms);
    if (workspace == nullptr || workspace_bytes < need)
      return set_error(NVFP4WS_ERR_WORKSPACE, "lmhead_verify: workspace needs %zu bytes", need);
    if (!aligned16(workspace)) return set_error(NVFP4WS_ERR_MISALIGNED, "lmhead_verify: workspace must be 16-byte aligned");
    return launch_mxf4_verify(static_cast<const uint16_t*>(X), q, sf, tensor_scale, M, N, K, v, workspace, s);
  }
  if (kp == KPATH_MMA_F16) {
    size_t need = mma_verify_workspace_bytes(M, N, K);
    if (workspace == nullptr || workspace_bytes < need)
      return set_error(NVFP4WS_ERR_WORKSPACE, "lmhead_verify: workspace needs %zu bytes", need);
    if (!aligned16(workspace)) return set_error(NVFP4WS_ERR_MISALIGNED, "lmhead_verify: workspace must be 16-byte aligned");
    return launch_mma_verify(static_cast<const uint16_t*>(X), q, sf, tensor_scale, M, N, K, v, workspace, s);
  }
  if (!gemv_supported(K)) return set_error(NVFP4WS_ERR_UNSUPPORTED, "lmhead_verify: GEMV path supports K <= 65536");
  size_t need = gemv_verify_workspace(M, N, K);
  if (workspace == nullptr || workspace_bytes < need)
    return set_error(NVFP4WS_ERR_WORKSPACE, "lmhead_verify: workspace needs %zu bytes", need);
  if (!aligned16(workspace)) return set_error(NVFP4WS_ERR_MISALIGNED, "lmhead_verify: workspace must be 16-byte aligned");
  const bool regs_only = (kp == KPATH_GEMV_REGS);
  GemvPlan p = gemv_plan(M, N, K, regs_only);
  const int pgrid = gemv_verify_grid(M, N, K);
  GemvArgs a{};
  a.X = static_cast<const uint16_t*>(X);
  a.q = q; a.sf = sf; a.ts = tensor_scale;
  a.M = M; a.N = N; a.K = K;
  a.part_val = static_cast<float*>(workspace);
  a.part_idx = reinterpret_cast<int*>(static_cast<char*>(workspace) + align_up((size_t)pgrid * M * 4, 256));
  if (int e = launch_gemv(a, true, regs_only, s)) return e;
  return launch_verify_stage2(a.part_val, a.part_idx, p.grid, (int)M, v, s);
}

extern "C" {

int lmhead_verify_argmax_accept_path(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale,
                                     int64_t M, int64_t N, int64_t K, const int32_t* drafts, int32_t B, int32_t D,
                                     int32_t* argmax, int32_t* accept_len, float* max_logit, void* workspace,
                                     size_t workspace_bytes, int path, nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  const VerifyRule v{drafts, nullptr, B, D, argmax, accept_len, nullptr, max_logit};
  return verify_impl(X, q, sf, tensor_scale, M, N, K, v, workspace, workspace_bytes, path, (cudaStream_t)stream);
}

int lmhead_verify_tree(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale, int64_t M,
                       int64_t N, int64_t K, const int32_t* drafts, const int32_t* parents, int32_t B, int32_t D,
                       int32_t* argmax, int32_t* accept_len, int32_t* accept_node, float* max_logit, void* workspace,
                       size_t workspace_bytes, nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  if (D > 0 && !parents) return set_error(NVFP4WS_ERR_INVALID_ARG, "lmhead_verify_tree: parents is null");
  const VerifyRule v{drafts, D > 0 ? parents : nullptr, B, D, argmax, accept_len, accept_node, max_logit};
  return verify_impl(X, q, sf, tensor_scale, M, N, K, v, workspace, workspace_bytes, NVFP4WS_PATH_AUTO,
                     (cudaStream_t)stream);
}

int lmhead_verify_argmax_accept(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale,
                                int64_t M, int64_t N, int64_t K, const int32_t* drafts, int32_t B, int32_t D,
                                int32_t* argmax, int32_t* accept_len, float* max_logit, void* workspace,
                                size_t workspace_bytes, nvfp4ws_stream_t stream) {
  return lmhead_verify_argmax_accept_path(X, q, sf, tensor_scale, M, N, K, drafts, B, D, argmax, accept_len,
                                          max_logit, workspace, workspace_bytes, NVFP4WS_PATH_AUTO, stream);
}

// ------------------------------------------------------------------ weight passes

// A caller built against another version of the header passes structs of another size: refuse
// them before reading any member past struct_size.
static int check_problem_sizes(const nvfp4_gemm_problem* problems, int32_t count, const char* who) {
  for (int32_t i = 0; i < count; ++i)
    if (problems[i].struct_size != NVFP4WS_GEMM_PROBLEM_SIZE)
      return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: problem %d: struct_size %u, this library expects %u (rebuild "
                       "against this nvfp4ws.h)", who, i, problems[i].struct_size, NVFP4WS_GEMM_PROBLEM_SIZE);
  return NVFP4WS_OK;
}

static int check_verify_size(const nvfp4_verify_spec* v, const char* who) {
  if (v->struct_size != NVFP4WS_VERIFY_SPEC_SIZE)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: verify struct_size %u, this library expects %u (rebuild against "
                     "this nvfp4ws.h)", who, v->struct_size, NVFP4WS_VERIFY_SPEC_SIZE);
  return NVFP4WS_OK;
}

static int to_host_problems(const nvfp4_gemm_problem* problems, int32_t count, int64_t M, int verify_last,
                            std::vector<MxHostProblem>* out, const char* who, int terms) {
  if (!problems || count < 1) return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: need count >= 1 problems", who);
  if (int e = check_problem_sizes(problems, count, who)) return e;
  // a verify problem takes more activation terms than the GEMMs, so fewer tokens fit
  const int max_m = std::min(352 / (verify_last ? std::max(terms, kVerifyTerms) : terms), NVFP4WS_MAX_M);
  if (M < 1 || M > max_m || !mxf4_supported(M, 256, terms))
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "%s: M=%lld outside 1..%d", who, (long long)M, max_m);
  out->clear();
  for (int32_t i = 0; i < count; ++i) {
    const nvfp4_gemm_problem& p = problems[i];
    const bool v = verify_last && i == count - 1;
    if (int e = validate_gemm(p.X, p.q, p.sf, p.tensor_scale, M, p.N, p.K, who)) return e;
    if (!mxf4_supported(M, p.K, terms))
      return set_error(NVFP4WS_ERR_UNSUPPORTED, "%s: problem %d: K=%lld must be a multiple of 256 in [256, 32768]",
                       who, i, (long long)p.K);
    if (!v) {
      if (!p.Y) return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: problem %d: Y is null", who, i);
      if (!aligned16(p.Y)) return set_error(NVFP4WS_ERR_MISALIGNED, "%s: problem %d: Y must be 16-byte aligned", who, i);
      if (p.y_dtype != NVFP4WS_Y_F32 && p.y_dtype != NVFP4WS_Y_BF16)
        return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: problem %d: bad y_dtype %d", who, i, p.y_dtype);
    }
    MxHostProblem h{static_cast<const uint16_t*>(p.X), p.q, p.sf, p.tensor_scale, p.N, p.K,
                    v ? nullptr : p.Y, (!v && p.y_dtype == NVFP4WS_Y_BF16) ? 1 : 0, v ? 1 : 0};
    out->push_back(h);
  }
  return NVFP4WS_OK;
}

static constexpr uint32_t kPassFlags = NVFP4WS_PASS_BATCH_INVARIANT | NVFP4WS_PASS_W4A4 | NVFP4WS_PASS_FOUR_TERMS;
static int pass_terms(uint32_t flags) {
  return (flags & NVFP4WS_PASS_W4A4) ? 1 : (flags & NVFP4WS_PASS_FOUR_TERMS) ? kGemmTermsFast : kGemmTerms;
}
static bool pass_flags_ok(uint32_t flags) {
  return (flags & ~kPassFlags) == 0 && (flags & (NVFP4WS_PASS_W4A4 | NVFP4WS_PASS_FOUR_TERMS)) !=
                                           (NVFP4WS_PASS_W4A4 | NVFP4WS_PASS_FOUR_TERMS);
}

size_t nvfp4_pass_workspace_bytes_ex(const nvfp4_gemm_problem* problems, int32_t count, int64_t M,
                                     int32_t verify_last, uint32_t flags) {
  std::vector<MxHostProblem> hp;
  if (!pass_flags_ok(flags) || ((flags & NVFP4WS_PASS_W4A4) && verify_last)) return 0;
  if (to_host_problems(problems, count, M, verify_last, &hp, "nvfp4_pass_workspace_bytes", pass_terms(flags)) !=
      NVFP4WS_OK)
    return 0;
  return mxf4_pass_workspace_bytes(hp.data(), count, M, (flags & NVFP4WS_PASS_BATCH_INVARIANT) != 0,
                                   pass_terms(flags));
}

size_t nvfp4_pass_workspace_bytes(const nvfp4_gemm_problem* problems, int32_t count, int64_t M, int32_t verify_last) {
  return nvfp4_pass_workspace_bytes_ex(problems, count, M, verify_last, 0u);
}

int nvfp4_pass_init(nvfp4_pass* pass, const nvfp4_gemm_problem* problems, int32_t count, int64_t M,
                    const nvfp4_verify_spec* verify, void* workspace, size_t workspace_bytes) {
  return nvfp4_pass_init_ex(pass, problems, count, M, verify, 0u, workspace, workspace_bytes);
}

int nvfp4_pass_init_ex(nvfp4_pass* pass, const nvfp4_gemm_problem* problems, int32_t count, int64_t M,
                       const nvfp4_verify_spec* verify, uint32_t flags, void* workspace, size_t workspace_bytes) {
  g_last_error[0] = 0;
  if (!pass_flags_ok(flags))
    return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pass_init: unknown flags or W4A4 with four terms (0x%x)", flags);
  if ((flags & NVFP4WS_PASS_W4A4) && verify)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pass_init: a W4A4 pass runs no verify");
  static_assert(sizeof(nvfp4_pass) >= kMxPassStateBytes, "nvfp4_pass is too small for the pass state");
  if (!pass) return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pass_init: pass is null");
  std::memset(pass, 0, sizeof(nvfp4_pass));
  if (verify)
    if (int e = check_verify_size(verify, "nvfp4_pass_init")) return e;
  std::vector<MxHostProblem> hp;
  if (int e = to_host_problems(problems, count, M, verify != nullptr, &hp, "nvfp4_pass_init", pass_terms(flags)))
    return e;
  VerifyRule vs{};
  if (verify) {
    if (verify->B < 1 || verify->D < 0)
      return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pass_init: verify needs B >= 1 and D >= 0");
    if ((int64_t)verify->B * (verify->D + 1) != M)
      return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pass_init: M=%lld must equal B*(D+1)=%lld", (long long)M,
                       (long long)verify->B * (verify->D + 1));
    if (verify->D > 0 && !verify->drafts) return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pass_init: drafts is null");
    if (!verify->argmax || !verify->accept_len)
      return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pass_init: null verify output pointer");
    vs = VerifyRule{verify->drafts, verify->parents, verify->B, verify->D, verify->argmax, verify->accept_len,
                    verify->accept_node, verify->max_logit};
  }
  if (!workspace) return set_error(NVFP4WS_ERR_WORKSPACE, "nvfp4_pass_init: workspace is null");
  if (!aligned16(workspace)) return set_error(NVFP4WS_ERR_MISALIGNED, "nvfp4_pass_init: workspace must be 16-byte aligned");
  return mxf4_pass_init(pass->opaque, hp.data(), count, M, verify ? &vs : nullptr,
                        (flags & NVFP4WS_PASS_BATCH_INVARIANT) != 0, pass_terms(flags), workspace, workspace_bytes);
}

int nvfp4_pass_run(const nvfp4_pass* pass, nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  if (!pass) return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pass_run: pass is null");
  return mxf4_pass_run(pass->opaque, (cudaStream_t)stream);
}

// ------------------------------------------------------------------ FP8 weights

int fp8_pack(const float* W, int64_t N, int64_t K, uint8_t* q, float* scales, nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  if (!W || !q || !scales) return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pack: null pointer");
  if (N < 1 || K < 16 || K % 16 != 0 || K > (int64_t)65535 * kFp8Block || N > (int64_t)0x7fffffff * kFp8Block)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pack: need N >= 1 and K a multiple of 16 in [16, 8388480]");
  if (!aligned16(W) || !aligned16(q)) return set_error(NVFP4WS_ERR_MISALIGNED, "fp8_pack: W and q must be 16-byte aligned");
  if ((uintptr_t)scales & 3u) return set_error(NVFP4WS_ERR_MISALIGNED, "fp8_pack: scales must be 4-byte aligned");
  return launch_fp8_pack(W, N, K, q, scales, (cudaStream_t)stream);
}

// Enough for either FP8 kernel, so a forced path works with the same buffer.
size_t fp8_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return std::max(fp8_gemm_workspace_bytes_int(M, N, K), fp8q_workspace_bytes_int(M, N, K, false));
}

size_t fp8_lmhead_verify_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return std::max(fp8_verify_workspace_bytes_int(M, N, K), fp8q_workspace_bytes_int(M, N, K, true));
}

static int validate_fp8(const void* X, const uint8_t* q, const float* scales, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t workspace_bytes, size_t need, const char* who) {
  if (!X || !q || !scales) return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: null input pointer", who);
  if (M < 1 || N < 1 || K < 1) return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: M, N, K must be >= 1", who);
  if (N > (int64_t)0x7fffffff) return set_error(NVFP4WS_ERR_UNSUPPORTED, "%s: N too large", who);
  if (!fp8_supported(M, K))
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "%s: needs 1 <= M <= 128 and K a positive multiple of 128 (M=%lld K=%lld)",
                     who, (long long)M, (long long)K);
  if (!aligned16(X) || !aligned16(q)) return set_error(NVFP4WS_ERR_MISALIGNED, "%s: X and q must be 16-byte aligned", who);
  if ((uintptr_t)scales & 3u) return set_error(NVFP4WS_ERR_MISALIGNED, "%s: scales must be 4-byte aligned", who);
  if (workspace == nullptr || workspace_bytes < need)
    return set_error(NVFP4WS_ERR_WORKSPACE, "%s: workspace needs %zu bytes", who, need);
  if (!aligned16(workspace)) return set_error(NVFP4WS_ERR_MISALIGNED, "%s: workspace must be 16-byte aligned", who);
  return NVFP4WS_OK;
}

int fp8_gemm_skinny_path(const void* X, const uint8_t* q, const float* scales, int64_t M, int64_t N, int64_t K,
                         void* Y, int y_dtype, void* workspace, size_t workspace_bytes, int path,
                         nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  if (!Y) return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_gemm_skinny: Y is null");
  if (y_dtype != NVFP4WS_Y_F32 && y_dtype != NVFP4WS_Y_BF16)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_gemm_skinny: bad y_dtype %d", y_dtype);
  if (path != NVFP4WS_FP8_DEQUANT_F16 && path != NVFP4WS_FP8_E4M3_TERMS)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_gemm_skinny: bad path %d", path);
  if (int e = validate_fp8(X, q, scales, M, N, K, workspace, workspace_bytes, fp8_gemm_workspace_bytes(M, N, K),
                           "fp8_gemm_skinny"))
    return e;
  if (!aligned16(Y)) return set_error(NVFP4WS_ERR_MISALIGNED, "fp8_gemm_skinny: Y must be 16-byte aligned");
  if (path == NVFP4WS_FP8_E4M3_TERMS)
    return launch_fp8q_gemm(static_cast<const uint16_t*>(X), q, scales, M, N, K, Y, y_dtype, workspace,
                            (cudaStream_t)stream);
  return launch_fp8_gemm(static_cast<const uint16_t*>(X), q, scales, M, N, K, Y, y_dtype, workspace,
                         (cudaStream_t)stream);
}

int fp8_gemm_skinny(const void* X, const uint8_t* q, const float* scales, int64_t M, int64_t N, int64_t K, void* Y,
                    int y_dtype, void* workspace, size_t workspace_bytes, nvfp4ws_stream_t stream) {
  return fp8_gemm_skinny_path(X, q, scales, M, N, K, Y, y_dtype, workspace, workspace_bytes,
                              NVFP4WS_FP8_DEQUANT_F16, stream);
}

int fp8_lmhead_verify(const void* X, const uint8_t* q, const float* scales, int64_t M, int64_t N, int64_t K,
                      const nvfp4_verify_spec* verify, void* workspace, size_t workspace_bytes,
                      nvfp4ws_stream_t stream) {
  return fp8_lmhead_verify_path(X, q, scales, M, N, K, verify, workspace, workspace_bytes, NVFP4WS_FP8_DEQUANT_F16,
                                stream);
}

int fp8_lmhead_verify_path(const void* X, const uint8_t* q, const float* scales, int64_t M, int64_t N, int64_t K,
                           const nvfp4_verify_spec* verify, void* workspace, size_t workspace_bytes, int path,
                           nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  if (path != NVFP4WS_FP8_DEQUANT_F16 && path != NVFP4WS_FP8_E4M3_TERMS)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_lmhead_verify: bad path %d", path);
  if (!verify) return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_lmhead_verify: verify is null");
  if (int e = check_verify_size(verify, "fp8_lmhead_verify")) return e;
  const int32_t B = verify->B, D = verify->D;
  if (B < 1 || D < 0) return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_lmhead_verify: need B >= 1 and D >= 0");
  if ((int64_t)B * (D + 1) != M)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_lmhead_verify: M=%lld must equal B*(D+1)=%lld", (long long)M,
                     (long long)B * (D + 1));
  if (D > 0 && !verify->drafts) return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_lmhead_verify: drafts is null");
  if (!verify->argmax || !verify->accept_len)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_lmhead_verify: null output pointer");
  if (int e = validate_fp8(X, q, scales, M, N, K, workspace, workspace_bytes,
                           fp8_lmhead_verify_workspace_bytes(M, N, K), "fp8_lmhead_verify"))
    return e;
  const VerifyRule v{verify->drafts, D > 0 ? verify->parents : nullptr, B, D, verify->argmax, verify->accept_len,
                     verify->accept_node, verify->max_logit};
  if (path == NVFP4WS_FP8_E4M3_TERMS)
    return launch_fp8q_verify(static_cast<const uint16_t*>(X), q, scales, M, N, K, v, workspace, (cudaStream_t)stream);
  return launch_fp8_verify(static_cast<const uint16_t*>(X), q, scales, M, N, K, v, workspace, (cudaStream_t)stream);
}

static int fp8_host_problems(const fp8_gemm_problem* problems, int32_t count, int64_t M, int verify_last,
                             std::vector<Fp8HostProblem>* out, const char* who) {
  if (!problems || count < 1) return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: need count >= 1 problems", who);
  for (int32_t i = 0; i < count; ++i)
    if (problems[i].struct_size != NVFP4WS_FP8_PROBLEM_SIZE)
      return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: problem %d: struct_size %u, this library expects %u (rebuild "
                       "against this nvfp4ws.h)", who, i, problems[i].struct_size, NVFP4WS_FP8_PROBLEM_SIZE);
  out->clear();
  for (int32_t i = 0; i < count; ++i) {
    const fp8_gemm_problem& p = problems[i];
    const bool v = verify_last && i == count - 1;
    if (!p.X || !p.q || !p.scales) return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: problem %d: null input", who, i);
    if (p.N < 1 || p.N > (int64_t)0x7fffffff)
      return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: problem %d: N=%lld out of range", who, i, (long long)p.N);
    if (!fp8_supported(M, p.K))
      return set_error(NVFP4WS_ERR_UNSUPPORTED, "%s: problem %d: needs 1 <= M <= 128 and K a positive multiple of 128 "
                       "(M=%lld K=%lld)", who, i, (long long)M, (long long)p.K);
    if (!aligned16(p.X) || !aligned16(p.q))
      return set_error(NVFP4WS_ERR_MISALIGNED, "%s: problem %d: X and q must be 16-byte aligned", who, i);
    if ((uintptr_t)p.scales & 3u)
      return set_error(NVFP4WS_ERR_MISALIGNED, "%s: problem %d: scales must be 4-byte aligned", who, i);
    if (!v) {
      if (!p.Y) return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: problem %d: Y is null", who, i);
      if (!aligned16(p.Y)) return set_error(NVFP4WS_ERR_MISALIGNED, "%s: problem %d: Y must be 16-byte aligned", who, i);
      if (p.y_dtype != NVFP4WS_Y_F32 && p.y_dtype != NVFP4WS_Y_BF16)
        return set_error(NVFP4WS_ERR_INVALID_ARG, "%s: problem %d: bad y_dtype %d", who, i, p.y_dtype);
    }
    out->push_back(Fp8HostProblem{static_cast<const uint16_t*>(p.X), p.q, p.scales, p.N, p.K, v ? nullptr : p.Y,
                                  (!v && p.y_dtype == NVFP4WS_Y_BF16) ? 1 : 0, v ? 1 : 0});
  }
  return NVFP4WS_OK;
}

size_t fp8_pass_workspace_bytes_path(const fp8_gemm_problem* problems, int32_t count, int64_t M, int32_t verify_last,
                                     int path) {
  std::vector<Fp8HostProblem> hp;
  if (path != NVFP4WS_FP8_DEQUANT_F16 && path != NVFP4WS_FP8_E4M3_TERMS) return 0;
  if (fp8_host_problems(problems, count, M, verify_last, &hp, "fp8_pass_workspace_bytes") != NVFP4WS_OK) return 0;
  return path == NVFP4WS_FP8_E4M3_TERMS ? fp8q_pass_workspace_bytes_int(hp.data(), count, M)
                                        : fp8_pass_workspace_bytes_int(hp.data(), count, M);
}

size_t fp8_pass_workspace_bytes(const fp8_gemm_problem* problems, int32_t count, int64_t M, int32_t verify_last) {
  return fp8_pass_workspace_bytes_path(problems, count, M, verify_last, NVFP4WS_FP8_DEQUANT_F16);
}

int fp8_pass_init_path(nvfp4_pass* pass, const fp8_gemm_problem* problems, int32_t count, int64_t M,
                       const nvfp4_verify_spec* verify, int path, void* workspace, size_t workspace_bytes) {
  g_last_error[0] = 0;
  static_assert(sizeof(nvfp4_pass) >= kFp8PassStateBytes, "nvfp4_pass is too small for the FP8 pass state");
  if (!pass) return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pass_init: pass is null");
  std::memset(pass, 0, sizeof(nvfp4_pass));
  if (path != NVFP4WS_FP8_DEQUANT_F16 && path != NVFP4WS_FP8_E4M3_TERMS)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pass_init: bad path %d", path);
  if (verify)
    if (int e = check_verify_size(verify, "fp8_pass_init")) return e;
  std::vector<Fp8HostProblem> hp;
  if (int e = fp8_host_problems(problems, count, M, verify != nullptr, &hp, "fp8_pass_init")) return e;
  VerifyRule vs{};
  if (verify) {
    if (verify->B < 1 || verify->D < 0)
      return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pass_init: verify needs B >= 1 and D >= 0");
    if ((int64_t)verify->B * (verify->D + 1) != M)
      return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pass_init: M=%lld must equal B*(D+1)=%lld", (long long)M,
                       (long long)verify->B * (verify->D + 1));
    if (verify->D > 0 && !verify->drafts) return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pass_init: drafts is null");
    if (!verify->argmax || !verify->accept_len)
      return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pass_init: null verify output pointer");
    vs = VerifyRule{verify->drafts, verify->D > 0 ? verify->parents : nullptr, verify->B, verify->D, verify->argmax,
                    verify->accept_len, verify->accept_node, verify->max_logit};
  }
  if (!workspace) return set_error(NVFP4WS_ERR_WORKSPACE, "fp8_pass_init: workspace is null");
  if (!aligned16(workspace)) return set_error(NVFP4WS_ERR_MISALIGNED, "fp8_pass_init: workspace must be 16-byte aligned");
  if (path == NVFP4WS_FP8_E4M3_TERMS)
    return fp8q_pass_init_int(pass->opaque, hp.data(), count, M, verify ? &vs : nullptr, workspace, workspace_bytes);
  return fp8_pass_init_int(pass->opaque, hp.data(), count, M, verify ? &vs : nullptr, workspace, workspace_bytes);
}

int fp8_pass_init(nvfp4_pass* pass, const fp8_gemm_problem* problems, int32_t count, int64_t M,
                  const nvfp4_verify_spec* verify, void* workspace, size_t workspace_bytes) {
  return fp8_pass_init_path(pass, problems, count, M, verify, NVFP4WS_FP8_DEQUANT_F16, workspace, workspace_bytes);
}

int fp8_pass_run(const nvfp4_pass* pass, nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  if (!pass) return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pass_run: pass is null");
  if (fp8q_pass_owns(pass->opaque)) return fp8q_pass_run_int(pass->opaque, (cudaStream_t)stream);
  return fp8_pass_run_int(pass->opaque, (cudaStream_t)stream);
}

int nvfp4ws_check(nvfp4ws_stream_t stream) {
  g_last_error[0] = 0;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return set_error(NVFP4WS_ERR_CUDA, "nvfp4ws_check: %s", cudaGetErrorString(e));
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e != cudaSuccess) return set_error(NVFP4WS_ERR_CUDA, "nvfp4ws_check: %s", cudaGetErrorString(e));
  if (v != 0) {
    unsigned int zero = 0;
    cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    if (v & kDevErrWaitTimeout)
      return set_error(NVFP4WS_ERR_DEVICE_TIMEOUT, "a bounded device wait gave up (code 0x%x)", v);
    return set_error(NVFP4WS_ERR_INVALID_ARG, "a draft tree had a parent outside [0, k-1] (code 0x%x)", v);
  }
  return NVFP4WS_OK;
}

}  // extern "C"
