/*
 * nvfp4ws.h -- C ABI of libnvfp4ws.so: NVFP4 weight-streaming skinny GEMM and
 * fused greedy verify for NVIDIA B200 (sm_100a).
 *
 * The operation comes from these web pages, cited by title and section:
 *   - "Qwen3.8 on DGX Spark (GB10)", "The seven targets, and switching between
 *     them": the weights are NVFP4 group-16.
 *   - The same page, introduction: the target verifies drafted tokens over the
 *     full 248,320-row vocabulary; the draft head may be a 65,536-row slice.
 *   - "TandemLLM", introduction: accept drafted tokens up to the first one the
 *     target disagrees with, then emit the target's own token (greedy verify).
 *     The same paragraph gives the one-ulp near-tie caveat.
 *   - "TandemLLM", "How it works": one decode step reads every weight once.
 *   - "ling-engine", introduction: 16 drafted tokens per step, and 2-4 sequences
 *     that share one weight read.
 *
 * Conventions common to every entry point
 *   - Pointers. All tensor pointers are DEVICE pointers unless a comment says
 *     otherwise. The caller owns every buffer. The library never allocates
 *     device or host memory.
 *   - Layouts. All layouts are row-major and dense (leading dimension = row
 *     length).
 *   - Asynchrony. Work is enqueued on `stream` (NULL = the legacy default
 *     stream) and runs asynchronously. The call returns once it is enqueued.
 *   - Validation. Argument checks are synchronous, on the host, and enqueue
 *     nothing when they fail. The return value is an nvfp4ws_status; the last
 *     error text of the calling thread is available from nvfp4ws_last_error().
 *   - Errors. A launch failure returns NVFP4WS_ERR_CUDA. No C++ exception
 *     crosses this interface.
 *   - Device errors. Kernels that wait for other CTAs give up after a bounded
 *     number of polls and record a code in a device error word. The
 *     next call of nvfp4ws_check() reports it.
 *   - Threads. The entry points are reentrant. Concurrent calls must not share
 *     a workspace.
 */
#ifndef NVFP4WS_H_
#define NVFP4WS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream). Kept opaque so this header needs no CUDA header. */
typedef void* nvfp4ws_stream_t;

typedef enum {
  NVFP4WS_OK = 0,
  NVFP4WS_ERR_INVALID_ARG = 1,    /* null pointer, bad size or bad enum value */
  NVFP4WS_ERR_UNSUPPORTED = 2,    /* shape outside what the kernels support (e.g. K % 32 != 0, M > 256) */
  NVFP4WS_ERR_MISALIGNED = 3,     /* a pointer does not have the alignment the call requires */
  NVFP4WS_ERR_WORKSPACE = 4,      /* workspace missing or smaller than the *_workspace_bytes query */
  NVFP4WS_ERR_CUDA = 5,           /* a CUDA runtime call or kernel launch failed */
  NVFP4WS_ERR_DEVICE_TIMEOUT = 6  /* a bounded device-side wait gave up (see nvfp4ws_check) */
} nvfp4ws_status;

/* Output element type of nvfp4_gemm_skinny. */
typedef enum { NVFP4WS_Y_F32 = 0, NVFP4WS_Y_BF16 = 1 } nvfp4ws_ydtype;

/* Kernel path of the GEMM. AUTO takes the block-scaled tensor-core kernel when K % 256 == 0: in one
   launch for M <= 70, and for larger M in ceil(M/70) equal slices of X's rows, one launch each
   (nvfp4_gemm_skinny only; the verify takes the f16 tensor-core kernel for 70 < M <= 128). When
   K % 256 != 0 it takes the GEMV. The others force a path. */
typedef enum {
  NVFP4WS_PATH_AUTO = 0,
  NVFP4WS_PATH_GEMV = 1,          /* CUDA-core streaming GEMV: dequantises in registers; rows staged by
                                     cp.async.bulk when K % 256 == 0, else register prefetch */
  NVFP4WS_PATH_MMA = 2,           /* tcgen05 tensor-core path: block-scaled kind::mxf4nvf4 on the packed
                                     weights when M*5 <= 352 (activations as 5 residual NVFP4 terms),
                                     else the f16 kernel below */
  NVFP4WS_PATH_GEMV_REGS = 3,     /* the register-prefetch GEMV variant at any K (for comparisons) */
  NVFP4WS_PATH_MMA_F16 = 4        /* tcgen05 kind::f16 on weights dequantised exactly to f16 in TMEM */
} nvfp4ws_path;

/* Human-readable name of a status code. Never NULL. Static storage. */
const char* nvfp4ws_status_string(int status);

/* Detail text of the last failing call on this host thread ("" if none). Thread-local storage. */
const char* nvfp4ws_last_error(void);

/* Library version as major*10000 + minor*100 + patch. 200 added struct_size to
 * nvfp4_gemm_problem and nvfp4_verify_spec. 201 added NVFP4WS_PASS_FOUR_TERMS. */
int nvfp4ws_version(void);

/* Largest M (rows of X) accepted by the GEMM and verify entry points. */
#define NVFP4WS_MAX_M 256

/*
 * nvfp4_pack -- quantise an fp32 weight to NVFP4 (two-level scaling) and pack it.
 *
 * Passage: "Qwen3.8 on DGX Spark (GB10)", "The seven targets ...": NVFP4
 * group-16. The pages give no bit-level definition. This library reads it as:
 *   ts   = fp32( amax(|W|) / (6 * 448) )                    per tensor
 *   S    = E4M3_rne_satfinite( amax(|block|) / (6 * ts) )    per 16 consecutive k
 *   code = E2M1_rne_satfinite( w / (S * ts) )                per element; sign kept
 * Both quotients are formed in float64 and rounded once (ties to even). If
 * ts == 0 or S == 0, the affected codes are +0.
 *
 * Arguments
 *   W               fp32 [N, K] row-major, device, 16-byte aligned. Read only.
 *   N, K            N >= 1, K >= 16, K % 16 == 0.
 *   q               out: uint8 [N, K/2], device. Byte (n, j) holds code(n, 2j) in
 *                   bits 0..3 and code(n, 2j+1) in bits 4..7.
 *   sf              out: uint8 [N, K/16], device. E4M3 bits of each block scale.
 *   tensor_scale    out: fp32 [1], device. The ts used.
 *   tensor_scale_in in: fp32 [1], device, or NULL. When non-NULL, this ts is used
 *                   instead of amax/2688, and copied to tensor_scale.
 * Returns NVFP4WS_OK, or INVALID_ARG / MISALIGNED / CUDA.
 */
int nvfp4_pack(const float* W, int64_t N, int64_t K, uint8_t* q, uint8_t* sf,
               float* tensor_scale, const float* tensor_scale_in, nvfp4ws_stream_t stream);

/*
 * nvfp4_gemm_workspace_bytes -- device workspace needed by nvfp4_gemm_skinny (any
 * path) for this shape; 0 when none is needed. Pass at least this many bytes.
 */
size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * nvfp4_gemm_skinny -- Y[M, N] = X[M, K] . dequant(W)[N, K]^T.
 *
 * Passage: "TandemLLM", "How it works" (each step reads every weight once, at
 * NVFP4), and the veloGB10 page, "Unique aspects: Engineered to the roofline"
 * (the pass is weight-bandwidth bound). M = 1 is plain decode, 17 is 16 drafts
 * + 1, and 68 is four sequences sharing one read.
 *
 * Arithmetic of the GEMV and f16 tensor-core paths: each row of X is multiplied by a
 * power of two 2^-e, with e chosen from the row's amax so that amax * 2^-e lies in
 * [2^14, 2^15), and converted to f16. That is exact for every value above 2^-25 * amax
 * (smaller ones round to f16 subnormals), and nothing saturates. Each product
 * x * (e2m1 * S) is then exact, sums are fp32, and the result is multiplied by ts and
 * by 2^e, in fp32.
 * Arithmetic of the block-scaled path (the default when K % 256 == 0; M > 70 in row slices):
 * X is first written as 5 residual NVFP4 terms. Each is a per-row fp32 scale, an
 * E4M3 scale per 16 and E2M1 codes; each term quantises what the previous ones left.
 * The tensor core then multiplies the packed weights by those terms exactly, with
 * fp32 accumulation. Measured error against the exact product is ~1e-5 of max|y|.
 *
 * Arguments
 *   X       bf16 [M, K] row-major, device, 16-byte aligned.
 *   q, sf   packed NVFP4 weight as produced by nvfp4_pack, device, 16-byte aligned.
 *   tensor_scale  fp32 [1], device.
 *   M       1 <= M <= NVFP4WS_MAX_M.   N >= 1.   K >= 32, K % 32 == 0.
 *   Y       out: [M, N] row-major, device, 16-byte aligned; fp32 or bf16 per y_dtype.
 *   workspace, workspace_bytes  device scratch of at least
 *           nvfp4_gemm_workspace_bytes(M, N, K) bytes, 16-byte aligned (may be NULL
 *           when that is 0). It must be zero-filled before its first use. Every
 *           completed call leaves the part that needs it zero again, so a buffer
 *           can be reused across calls and shapes without clearing.
 * Returns NVFP4WS_OK, or INVALID_ARG / UNSUPPORTED / MISALIGNED / WORKSPACE / CUDA.
 */
int nvfp4_gemm_skinny(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale,
                      int64_t M, int64_t N, int64_t K, void* Y, int y_dtype,
                      void* workspace, size_t workspace_bytes, nvfp4ws_stream_t stream);

/* As nvfp4_gemm_skinny, with an explicit kernel path (nvfp4ws_path). Used by the M sweep and the tests. */
int nvfp4_gemm_skinny_path(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale,
                           int64_t M, int64_t N, int64_t K, void* Y, int y_dtype,
                           void* workspace, size_t workspace_bytes, int path, nvfp4ws_stream_t stream);

/*
 * nvfp4_gemm_w4a4 -- the W4A4 product for prefill-sized M: X is quantised to NVFP4 too,
 * and both operands go through the block-scaled tensor cores.
 *
 * Passages: "Qwen3.8 on DGX Spark (GB10)", introduction (NVFP4 on the block-scaled
 * tensor cores) and "TandemLLM", "The parts" (4-bit projections). The pages give no
 * activation recipe; this library applies the weights' two-level NVFP4 scheme (the rule of
 * nvfp4_pack) to each row of X, with the row's amax in place of the tensor's:
 *   g[m]   = fp32(amax_k |x[m,k]| / 2688)
 *   S      = E4M3_rne_satfinite(amax_block / (6 g[m]))        per 16 elements
 *   c      = E2M1_rne_satfinite(x / (S g[m]))                 (+0 where S g = 0; sign kept)
 *   Y[m,n] = sum_k (e2m1(c)·S·g[m])[m,k] · dequant(W)[n,k], accumulated in fp32,
 * with both quotients exact and rounded once.
 * This is not the exact bf16 product nvfp4_gemm_skinny computes: each activation
 * carries up to half an E2M1 step of quantisation error.
 *
 * Arguments as nvfp4_gemm_skinny; 1 <= M <= NVFP4WS_MAX_M; K a multiple of 256 in
 * [256, 32768]; workspace of at least nvfp4_gemm_w4a4_workspace_bytes(M, N, K) bytes,
 * zero-filled before its first use.
 */
size_t nvfp4_gemm_w4a4_workspace_bytes(int64_t M, int64_t N, int64_t K);
int nvfp4_gemm_w4a4(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale,
                    int64_t M, int64_t N, int64_t K, void* Y, int y_dtype,
                    void* workspace, size_t workspace_bytes, nvfp4ws_stream_t stream);

/* Workspace needed by lmhead_verify_argmax_accept for this shape. */
size_t lmhead_verify_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * lmhead_verify_argmax_accept -- lm_head GEMM with fused greedy verify.
 *
 * Passages: "TandemLLM", introduction (accept drafts up to the first
 * disagreement, then the target's token) and "How it works" (keep the longest
 * agreeing path). "Qwen3.8 on DGX Spark (GB10)", introduction (verify over the
 * whole vocabulary).
 *
 * The logits y = X . dequant(W)^T are computed exactly as in nvfp4_gemm_skinny
 * but never written to memory. Per row m:
 *   argmax[m] = the smallest n with y[m, n] == max_n y[m, n]
 * Rows are grouped per sequence: M = B * (D + 1), and row b*(D+1)+i is the
 * target's prediction for draft slot i of sequence b. Then:
 *   accept_len[b] = min{ i in [0, D) : drafts[b, i] != argmax[b*(D+1) + i] }, or D
 * The committed tokens of sequence b are argmax[b*(D+1) .. b*(D+1) + accept_len[b]]:
 * the accepted drafts followed by the target's correction (or bonus) token.
 *
 * Arguments
 *   X, q, sf, tensor_scale, N, K   as in nvfp4_gemm_skinny (N = vocabulary rows).
 *   M           must equal B * (D + 1); 1 <= M <= NVFP4WS_MAX_M.
 *   drafts      int32 [B, D] row-major, device (may be NULL when D == 0).
 *   B, D        B >= 1, D >= 0.
 *   argmax      out: int32 [M], device.
 *   accept_len  out: int32 [B], device.
 *   max_logit   out: fp32 [M], device, or NULL to skip (the winning logit, for tie diagnostics).
 *   workspace   device scratch of at least lmhead_verify_workspace_bytes(M, N, K) bytes,
 *               16-byte aligned, zero-filled before its first use (as for the GEMM).
 * Returns NVFP4WS_OK, or INVALID_ARG / UNSUPPORTED / MISALIGNED / WORKSPACE / CUDA.
 * Logits that are NaN make argmax undefined.
 */
int lmhead_verify_argmax_accept(const void* X, const uint8_t* q, const uint8_t* sf,
                                const float* tensor_scale, int64_t M, int64_t N, int64_t K,
                                const int32_t* drafts, int32_t B, int32_t D,
                                int32_t* argmax, int32_t* accept_len, float* max_logit,
                                void* workspace, size_t workspace_bytes, nvfp4ws_stream_t stream);

/*
 * lmhead_verify_tree -- lm_head GEMM with fused greedy verify of a draft TREE.
 *
 * Passage: "TandemLLM", "How it works" (the drafters propose a tree, the target
 * verifies the whole tree in one pass, and the longest path it agrees with is kept).
 *
 * Each sequence b has nodes 0..D. Node 0 is the committed context. Node k >= 1 holds
 * the draft token drafts[b, k-1] and hangs under node parents[b, k-1], which must lie
 * in [0, k-1] (a parent precedes its children). Row b*(D+1)+k of X is the target's
 * input after the root-to-k path, so argmax[b*(D+1)+k] is its greedy next token there.
 * Node k is accepted when its parent is accepted and
 *   drafts[b, k-1] == argmax[b*(D+1) + parents[b, k-1]]      (node 0 always is).
 * The kept path ends at the accepted node of greatest depth (the lowest node index
 * among equals): accept_node[b] is that node and accept_len[b] its depth. The
 * committed tokens are the drafts on the root-to-accept_node path, in path order,
 * followed by argmax[b*(D+1) + accept_node[b]]. With parents[b, k-1] = k-1 for every
 * k (a chain) the result is lmhead_verify_argmax_accept's.
 *
 * Arguments as lmhead_verify_argmax_accept, plus
 *   parents      int32 [B, D] row-major, device (may be NULL when D == 0).
 *   accept_node  out: int32 [B], device, or NULL to skip.
 * A parent outside [0, k-1] rejects its node and sets the device error word, which the
 * next nvfp4ws_check reports as NVFP4WS_ERR_INVALID_ARG.
 */
int lmhead_verify_tree(const void* X, const uint8_t* q, const uint8_t* sf, const float* tensor_scale,
                       int64_t M, int64_t N, int64_t K, const int32_t* drafts, const int32_t* parents,
                       int32_t B, int32_t D, int32_t* argmax, int32_t* accept_len, int32_t* accept_node,
                       float* max_logit, void* workspace, size_t workspace_bytes, nvfp4ws_stream_t stream);

/* As lmhead_verify_argmax_accept, with an explicit kernel path (nvfp4ws_path). */
int lmhead_verify_argmax_accept_path(const void* X, const uint8_t* q, const uint8_t* sf,
                                     const float* tensor_scale, int64_t M, int64_t N, int64_t K,
                                     const int32_t* drafts, int32_t B, int32_t D,
                                     int32_t* argmax, int32_t* accept_len, float* max_logit,
                                     void* workspace, size_t workspace_bytes, int path,
                                     nvfp4ws_stream_t stream);

/*
 * Weight passes -- a list of independent GEMMs that share M, run by ONE persistent
 * launch, optionally ending with the fused lm_head verify.
 *
 * Passage: "TandemLLM", "How it works" (one decode step reads every weight once)
 * and the veloGB10 page, "Unique aspects: Engineered to the roofline" (the pass is
 * bound by weight bandwidth). On B200 a single GEMM of a 27B layer streams for
 * only 5-15 us, about as long as launching, filling and draining a persistent
 * kernel. A pass therefore streams the whole list as one sequence of (problem,
 * 128-row tile, 256-wide K-chunk) units, split evenly across the SMs: each SM's
 * weight stream runs from its first unit to its last without a drain.
 *
 * Each problem computes Y_i[M, N_i] = X_i[M, K_i] . dequant(W_i)^T exactly as
 * nvfp4_gemm_skinny's block-scaled path does (same arithmetic and error). The
 * problems run concurrently in no particular order: no problem's X may be another
 * problem's Y. With `verify` non-NULL the LAST problem is the lm_head: its Y is
 * ignored and the step ends with the argmax over its N rows and the accept lengths,
 * as lmhead_verify_argmax_accept computes them.
 *
 * nvfp4_pass_workspace_bytes -- device workspace for this list (verify_last != 0
 *   when the last problem is the verify problem); 0 when the list is invalid.
 * nvfp4_pass_init -- validates the list, lays out the workspace and writes the
 *   problems' descriptors into it with a SYNCHRONOUS copy: call it at set-up, not
 *   while a stream is being captured, and not while a run on this workspace is in
 *   flight. The workspace must be zero-filled before the first run; every run
 *   leaves the part that needs it zero again. The pointers given (X, W, Y, verify
 *   buffers, workspace) are baked into the pass: later runs read and write the
 *   same buffers, so refill X in place between runs.
 * nvfp4_pass_run -- enqueues the pass on `stream` (3 kernels with verify, else 2; a
 *   NVFP4WS_PASS_FOUR_TERMS pass with a verify after GEMMs: 5).
 *   It can be captured in a CUDA graph.
 *
 * Arguments
 *   problems[i]   X: bf16 [M, K], device, 16-byte aligned.  q, sf, tensor_scale: as
 *                 produced by nvfp4_pack.  N >= 1.  K a multiple of 256, 256 <= K <=
 *                 32768.  Y: [M, N] fp32 or bf16 per y_dtype (ignored for the verify
 *                 problem).
 *   count         >= 1.
 *   M             1 <= M <= 70 (the block-scaled path's limit: M times the 5 activation
 *                 terms fits 352 B rows; 88 for a NVFP4WS_PASS_FOUR_TERMS pass without verify).
 *   verify        NULL, or the verify buffers: M must equal B * (D + 1); drafts int32
 *                 [B, D] (may be NULL when D == 0); argmax int32 [M]; accept_len int32
 *                 [B]; max_logit fp32 [M] or NULL; parents int32 [B, D] for a tree
 *                 verify as lmhead_verify_tree computes it, or NULL for the chain rule;
 *                 accept_node int32 [B] or NULL (the kept path's end node).
 *   pass          caller-owned host state, filled by nvfp4_pass_init.
 * Returns NVFP4WS_OK, or INVALID_ARG / UNSUPPORTED / MISALIGNED / WORKSPACE / CUDA.
 */
/* Both structs below open with struct_size, which the caller sets to the struct's size as
 * compiled (NVFP4WS_GEMM_PROBLEM_SIZE, NVFP4WS_VERIFY_SPEC_SIZE). A call that gets any other
 * value returns NVFP4WS_ERR_INVALID_ARG before it reads a further member, so code built
 * against another version of this header is refused on the host instead of having its
 * struct read past its end. */
typedef struct nvfp4_gemm_problem {
  uint32_t struct_size;    /* = NVFP4WS_GEMM_PROBLEM_SIZE */
  const void* X;
  const uint8_t* q;
  const uint8_t* sf;
  const float* tensor_scale;
  int64_t N;
  int64_t K;
  void* Y;
  int32_t y_dtype;
} nvfp4_gemm_problem;

typedef struct nvfp4_verify_spec {
  uint32_t struct_size;    /* = NVFP4WS_VERIFY_SPEC_SIZE */
  const int32_t* drafts;
  int32_t B;
  int32_t D;
  int32_t* argmax;
  int32_t* accept_len;
  float* max_logit;
  const int32_t* parents;
  int32_t* accept_node;
} nvfp4_verify_spec;

#define NVFP4WS_GEMM_PROBLEM_SIZE ((uint32_t)sizeof(nvfp4_gemm_problem))
#define NVFP4WS_VERIFY_SPEC_SIZE ((uint32_t)sizeof(nvfp4_verify_spec))

typedef struct nvfp4_pass {
  uint64_t opaque[32];
} nvfp4_pass;

size_t nvfp4_pass_workspace_bytes(const nvfp4_gemm_problem* problems, int32_t count, int64_t M,
                                  int32_t verify_last);
int nvfp4_pass_init(nvfp4_pass* pass, const nvfp4_gemm_problem* problems, int32_t count, int64_t M,
                    const nvfp4_verify_spec* verify, void* workspace, size_t workspace_bytes);

/*
 * Batch-invariant passes.
 *
 * Passage: "TandemLLM", "The parts" (the projection kernels give a row the same bits
 * whatever other rows share the batch) and its feature list ("--probe-binv (batch
 * invariance)"). With NVFP4WS_PASS_BATCH_INVARIANT a pass gives every row of Y (and of
 * the verify's logits) the same bits for any M in [1, 70] with the same problem list:
 * the work is split into the same units at the same points, summed in the same order,
 * whatever M is. (A row's activation terms depend on that row alone.) It costs
 * bandwidth at small M, where the default plan uses larger units.
 *
 * nvfp4_pass_workspace_bytes_ex / nvfp4_pass_init_ex -- as the calls above, with
 *   `flags`, an OR of NVFP4WS_PASS_BATCH_INVARIANT, NVFP4WS_PASS_W4A4 and
 *   NVFP4WS_PASS_FOUR_TERMS (other bits, or W4A4 with FOUR_TERMS, are INVALID_ARG, and
 *   the workspace query returns 0). Pass the same flags to both.
 */
#define NVFP4WS_PASS_BATCH_INVARIANT 1u
/* A W4A4 pass: every problem as nvfp4_gemm_w4a4 computes it (M up to NVFP4WS_MAX_M, no
 * verify problem). */
#define NVFP4WS_PASS_W4A4 2u
/* The GEMMs of the pass write X as 4 residual NVFP4 terms instead of 5: their error against
 * the exact product is ~1e-4 of a row's max|y| instead of ~1e-5 (a float64 model of the terms
 * leaves 7e-5 to 1e-4 on the 27B layer shapes), and the tensor core, the image copies and the
 * scale copies do a fifth less work per weight byte. Where a row has few outputs (N of a few
 * columns) the per-row bar of 2e-3 of max|y| can then be missed on an output near zero. A
 * verify problem keeps 5 terms (its argmax compares logits that may lie 1e-3 apart) and runs as
 * a second persistent launch after the GEMMs' launch, whose weight loads may start while the
 * GEMMs' last tiles finish. M up to 88 without a verify. */
#define NVFP4WS_PASS_FOUR_TERMS 4u
size_t nvfp4_pass_workspace_bytes_ex(const nvfp4_gemm_problem* problems, int32_t count, int64_t M,
                                     int32_t verify_last, uint32_t flags);
int nvfp4_pass_init_ex(nvfp4_pass* pass, const nvfp4_gemm_problem* problems, int32_t count, int64_t M,
                       const nvfp4_verify_spec* verify, uint32_t flags, void* workspace, size_t workspace_bytes);
int nvfp4_pass_run(const nvfp4_pass* pass, nvfp4ws_stream_t stream);

/*
 * FP8 weights -- E4M3 codes with one fp32 scale per 128 x 128 block (rows x K).
 *
 * Passages: "TandemLLM", "The parts" (the lm_head is kept in FP8 E4M3, as the vendor's
 * checkpoint ships it) and "Qwen3.8 on DGX Spark (GB10)" (block-scaled FP8 projections). The
 * pages give neither the block shape nor the scale rule. This library reads them as
 *   s[i, j] = fp32( amax|W[128i .. 128i+127, 128j .. 128j+127]| / 448 )   0 for a zero block
 *   code    = E4M3_rne_satfinite( w / s ), sign kept                   +0 where s = 0
 * with the quotient formed in float64 and rounded once. Blocks at the right and bottom
 * edges cover what remains of W.
 *
 * fp8_pack -- quantise an fp32 weight.
 *   W        fp32 [N, K] row-major, device, 16-byte aligned. Read only.
 *   N, K     N >= 1; K >= 16, K % 16 == 0, K <= 8388480.
 *   q        out: uint8 [N, K] row-major, device, 16-byte aligned: E4M3 bits per element.
 *   scales   out: fp32 [ceil(N/128), ceil(K/128)] row-major, device, 4-byte aligned.
 * Returns NVFP4WS_OK, or INVALID_ARG / MISALIGNED / CUDA.
 *
 * fp8_gemm_skinny -- Y[M, N] = X[M, K] . dequant(W)^T, with
 *   dequant(W)[n, k] = e4m3(q[n, k]) * scales[n / 128, k / 128].
 *   X is converted to f16 as in nvfp4_gemm_skinny, so each product x * e4m3(q) is exact;
 *   each block's 128 products are summed in fp32, multiplied by the block's scale and
 *   added to the row's sum in K order, in fp32.
 *   X        bf16 [M, K], device, 16-byte aligned.   1 <= M <= 128.
 *   q, scales  as written by fp8_pack.   N >= 1.   K a positive multiple of 128.
 *   Y        out: [M, N], device, 16-byte aligned; fp32 or bf16 per y_dtype.
 *   workspace  at least fp8_gemm_workspace_bytes(M, N, K) bytes, 16-byte aligned, zero-filled
 *            before its first use; every completed call leaves it reusable.
 * Returns NVFP4WS_OK, or INVALID_ARG / UNSUPPORTED / MISALIGNED / WORKSPACE / CUDA.
 *
 * fp8_lmhead_verify -- the FP8 lm_head with the fused greedy verify. The logits are
 *   fp8_gemm_skinny's and are never written to memory. `verify` gives the rule and its
 *   buffers as for a weight pass: the chain rule of lmhead_verify_argmax_accept when
 *   verify->parents is NULL, else the tree rule of lmhead_verify_tree. M must equal
 *   verify->B * (verify->D + 1). Workspace: fp8_lmhead_verify_workspace_bytes(M, N, K).
 */
int fp8_pack(const float* W, int64_t N, int64_t K, uint8_t* q, float* scales, nvfp4ws_stream_t stream);

/* FP8 kernel of fp8_gemm_skinny_path / fp8_lmhead_verify_path. DEQUANT_F16 (the default of the
 * calls without _path): the codes are converted to f16 (exact) for tcgen05 kind::f16, and every
 * product is exact. E4M3_TERMS: the codes go straight into kind::f8f6f4, and each row of X is
 * written as two residual E4M3 terms under one power-of-two scale g = 2^(e-8), amax|x| in
 * [2^(e-1), 2^e): exact except for elements whose low bits fall below E4M3's subnormal step in
 * the second term (absolute error below 2^-14 g per element). */
#define NVFP4WS_FP8_DEQUANT_F16 0
#define NVFP4WS_FP8_E4M3_TERMS 1
size_t fp8_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
int fp8_gemm_skinny(const void* X, const uint8_t* q, const float* scales, int64_t M, int64_t N, int64_t K,
                    void* Y, int y_dtype, void* workspace, size_t workspace_bytes, nvfp4ws_stream_t stream);
int fp8_gemm_skinny_path(const void* X, const uint8_t* q, const float* scales, int64_t M, int64_t N, int64_t K,
                         void* Y, int y_dtype, void* workspace, size_t workspace_bytes, int path,
                         nvfp4ws_stream_t stream);
size_t fp8_lmhead_verify_workspace_bytes(int64_t M, int64_t N, int64_t K);
int fp8_lmhead_verify(const void* X, const uint8_t* q, const float* scales, int64_t M, int64_t N, int64_t K,
                      const nvfp4_verify_spec* verify, void* workspace, size_t workspace_bytes,
                      nvfp4ws_stream_t stream);
int fp8_lmhead_verify_path(const void* X, const uint8_t* q, const float* scales, int64_t M, int64_t N, int64_t K,
                           const nvfp4_verify_spec* verify, void* workspace, size_t workspace_bytes, int path,
                           nvfp4ws_stream_t stream);

/*
 * FP8 weight passes -- a list of independent FP8 GEMMs that share M, run by ONE persistent
 * launch, optionally ending with the fused verify over an FP8 lm_head.
 *
 * Passages: "TandemLLM", "How it works" (one decode step reads every weight once) and "The
 * parts" (the FP8 attention projections and head beside the 4-bit weights). As for NVFP4
 * passes, the units of all the problems (128-row tile x 128- or 256-wide K range) form one
 * sequence split evenly across the SMs. Each problem computes what fp8_gemm_skinny computes.
 * The problems run concurrently in no particular order: no problem's X may be another
 * problem's Y. With `verify` non-NULL the LAST problem is the lm_head: its Y is ignored and
 * the pass ends with the argmax and accept rule of fp8_lmhead_verify. An NVFP4 pass and an
 * FP8 pass can be enqueued back to back (or captured in one CUDA graph) to stream a model
 * whose matrices use both formats.
 *
 * fp8_pass_workspace_bytes -- device workspace for this list (verify_last != 0 when the last
 *   problem is the verify problem); 0 when the list is invalid.
 * fp8_pass_init -- validates the list, lays out the workspace and writes the problems'
 *   descriptors into it with a SYNCHRONOUS copy (call it at set-up, outside stream capture).
 *   The workspace must be zero-filled before the first run; every run leaves it reusable.
 *   The pointers given are baked into the pass.
 * fp8_pass_run -- enqueues the pass on `stream` (2 kernels with verify, else 1). It can be
 *   captured in a CUDA graph.
 *
 * Arguments
 *   problems[i]   X: bf16 [M, K], device, 16-byte aligned.  q, scales: as written by fp8_pack.
 *                 N >= 1.  K a positive multiple of 128.  Y: [M, N] fp32 or bf16 per y_dtype,
 *                 16-byte aligned (ignored for the verify problem).
 *   count         >= 1.
 *   M             1 <= M <= 128.
 *   verify        NULL, or the verify rule and buffers (nvfp4_verify_spec): M must equal
 *                 B * (D + 1); parents NULL for the chain rule.
 *   pass          caller-owned host state, filled by fp8_pass_init (an nvfp4_pass handle;
 *                 nvfp4_pass_run refuses it).
 * Returns NVFP4WS_OK, or INVALID_ARG / UNSUPPORTED / MISALIGNED / WORKSPACE / CUDA.
 */
typedef struct fp8_gemm_problem {
  uint32_t struct_size;    /* = NVFP4WS_FP8_PROBLEM_SIZE (see nvfp4_gemm_problem) */
  const void* X;
  const uint8_t* q;
  const float* scales;
  int64_t N;
  int64_t K;
  void* Y;
  int32_t y_dtype;
} fp8_gemm_problem;

#define NVFP4WS_FP8_PROBLEM_SIZE ((uint32_t)sizeof(fp8_gemm_problem))

size_t fp8_pass_workspace_bytes(const fp8_gemm_problem* problems, int32_t count, int64_t M, int32_t verify_last);
int fp8_pass_init(nvfp4_pass* pass, const fp8_gemm_problem* problems, int32_t count, int64_t M,
                  const nvfp4_verify_spec* verify, void* workspace, size_t workspace_bytes);
int fp8_pass_run(const nvfp4_pass* pass, nvfp4ws_stream_t stream);

/* As fp8_pass_workspace_bytes / fp8_pass_init, with the FP8 kernel chosen by `path`
 * (NVFP4WS_FP8_DEQUANT_F16, the default of the calls above, or NVFP4WS_FP8_E4M3_TERMS with the
 * arithmetic fp8_gemm_skinny_path describes for it). Pass the same path to both; fp8_pass_run
 * runs whichever kernel the pass was initialised with. */
size_t fp8_pass_workspace_bytes_path(const fp8_gemm_problem* problems, int32_t count, int64_t M, int32_t verify_last,
                                     int path);
int fp8_pass_init_path(nvfp4_pass* pass, const fp8_gemm_problem* problems, int32_t count, int64_t M,
                       const nvfp4_verify_spec* verify, int path, void* workspace, size_t workspace_bytes);

/*
 * nvfp4_gemm_skinny_noalloc -- the tensor-core GEMM of nvfp4_gemm_skinny for callers
 * that cannot allocate device memory and so cannot pass a workspace. Examples are a
 * host that fixes its device-memory plan at start-up and forbids later allocation,
 * code running under another framework's pooling allocator, and a plugin interface
 * that provides no scratch buffer. (The pages have no counterpart: this is a
 * packaging choice of this library.)
 *
 * Scratch comes from one built-in device array of 16 MiB. Every GPU that loads the
 * library holds it until the process exits. The first call on a device looks up the
 * array's address (cudaGetSymbolAddress), so make that first call before any
 * stream capture. Every call shares the array and leaves its last contents in it.
 * Each call clears the part that must start at zero (cudaMemsetAsync on `stream`).
 * Calls whose work overlaps on the GPU race on the array.
 * Nothing is allocated: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * It always runs the f16 tensor-core kernel (NVFP4WS_PATH_MMA_F16), whatever M is, with
 * that kernel's arithmetic as nvfp4_gemm_skinny describes it (rows of X shifted by a power
 * of two, exact f16 products, fp32 sums). Arguments and result are as for
 * nvfp4_gemm_skinny on that path: 1 <= M <= 128, K a positive multiple of 256, N >= 1.
 * Returns NVFP4WS_ERR_UNSUPPORTED for a shape outside that range, or whose scratch
 * (nvfp4_gemm_workspace_bytes) exceeds the 16 MiB array; otherwise as nvfp4_gemm_skinny.
 */
int nvfp4_gemm_skinny_noalloc(const void* X, const uint8_t* q, const uint8_t* sf,
                              const float* tensor_scale, int64_t M, int64_t N, int64_t K,
                              void* Y, int y_dtype, nvfp4ws_stream_t stream);

/*
 * nvfp4ws_check -- synchronise `stream`, then read and clear the device error word
 * of the current device. Returns NVFP4WS_OK, NVFP4WS_ERR_DEVICE_TIMEOUT (a bounded
 * wait gave up; the detail is in nvfp4ws_last_error) or NVFP4WS_ERR_CUDA.
 */
int nvfp4ws_check(nvfp4ws_stream_t stream);

/* Number of SMs the kernels size their grids for (the current device's count). -1 on error. */
int nvfp4ws_sm_count(void);

/* Kernels (and memset nodes) this process has enqueued through the library so far, all
   devices and threads together. During CUDA-graph capture this counts what the graph holds. */
unsigned long long nvfp4ws_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4WS_H_ */
