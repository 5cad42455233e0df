/*
 * specv — batched verification and acceptance of block-diffusion
 * speculative drafts on one NVIDIA B200 (sm_100a).
 *
 * C ABI. Every pointer argument is a DEVICE pointer owned by the caller,
 * unless stated otherwise; the library never allocates, frees or
 * synchronises, and every call is stream-ordered on `stream`. A negative
 * return value means the call was rejected on the host before any launch
 * (nothing was written); SPEC_ERR_CUDA means a launch failed.
 *
 * Logit layout: row-major, vocabulary innermost; a row is V contiguous
 * elements, fp32 or bf16 (dtype). Base pointers must be 16-byte aligned
 * when V * element size is a multiple of 16 (the vectorised path);
 * otherwise any element-aligned pointer works (scalar path).
 *
 * Workspaces. Calls that merge work across thread blocks take a caller-owned
 * workspace of at least the size its *_workspace_size function returns.
 * It must be zeroed once (spec_workspace_init) before its first use; after
 * that it is self-resetting, so one fixed-address workspace serves every
 * later call and every replay of a captured CUDA graph. Word 0 of the
 * workspace is a sticky device status: the OR of SPEC_DEV_* flags raised by
 * any call since the last spec_workspace_init. It is readable after the
 * stream is synchronised. Calls that overlap on the GPU must not share a
 * workspace.
 *
 * Sources (cited by page title and section):
 *  [DBLAST] "DBLAST: Dependent Block Drafting for Stochastic Speculative
 *           Decoding", Pith review: "What carries the argument" (Eq. 5,
 *           latent-mixture proposal and category-posterior verification),
 *           "Assumptions" (rejection-corrected speculative sampling is
 *           lossless for any proposal; same sampling filter for target),
 *           "What would settle it" (temperature-scaled target sampling).
 *  [DSCALE] "DScale: Scaling Block-Diffusion Speculative Decoding with
 *           Adaptive Verification", Abstract (DVL allocation into half the
 *           native verification capacity; fixed-address workspaces that
 *           carry changing boundaries through verification while captured
 *           graphs are reused).
 *  [QA]     "Why does throughput collapse under high concurrency?" (block-
 *           diffusion failure-mode Q&A): verify lengths from prefix
 *           survival probabilities.
 */
#ifndef SPECV_H
#define SPECV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* spec_stream_t; /* same object as cudaStream_t; NULL = legacy default stream */

typedef enum {
  SPEC_OK = 0,
  SPEC_ERR_ARG = -1,          /* null pointer, bad size, misalignment, T <= 0, budget < B ... */
  SPEC_ERR_UNSUPPORTED = -2,  /* shape outside the supported range (K > 8, L > 32, B > 4096 ...) */
  SPEC_ERR_CUDA = -3,         /* a kernel launch failed */
  SPEC_ERR_WORKSPACE = -4     /* workspace missing or smaller than required */
} spec_status;

typedef enum { SPEC_F32 = 0, SPEC_BF16 = 1 } spec_dtype;

/* Device status flags (workspace word 0). */
#define SPEC_DEV_TOKEN_RANGE 1  /* a drafted token outside [0, V): that request gets accept_len = -1 */
#define SPEC_DEV_NONFINITE 2    /* a needed row had a non-finite max or normaliser: accept_len = -1 */
#define SPEC_DEV_VERIFY_LEN 4   /* verify_len[b] outside [0, L]: accept_len = -1 */
#define SPEC_DEV_SCORES 8       /* a survival score outside [0, 1] or NaN */

/* Limits. */
#define SPEC_MAX_L 32
#define SPEC_MAX_K 8
#define SPEC_MAX_B 4096
#define SPEC_MAX_V 1048576      /* vocabulary of the verify calls (terminal token packed in 20 bits) */
#define SPEC_MAX_DVL_ELEMS 16384 /* B * L for dvl_allocate_pack */
#define SPEC_NOALLOC_MAX_ROWS 4096 /* rows of spec_softmax_T_noalloc (fixed 48 KiB scratch) */

/* Human-readable name of a spec_status value. Host only; never fails. */
const char* spec_status_string(int status);

/* Workspace sizes in bytes (host only; pure arithmetic, no CUDA call).
 * Return 0 for arguments outside the supported range. */
size_t spec_softmax_workspace_size(int64_t rows);
size_t spec_verify_workspace_size(int B, int L, int K, int64_t V);
size_t spec_dvl_workspace_size(int B);

/* Zero a workspace (cudaMemsetAsync on `stream`). Call once per workspace
 * before its first use, and again to clear the sticky status word. */
int spec_workspace_init(void* workspace, size_t ws_bytes, spec_stream_t stream);

/*
 * spec_softmax_T — temperature softmax statistics of `rows` logit rows
 * ([DBLAST] "What would settle it": target sampling at temperature T; the
 * same T scales target and draft logits).
 *   logits     [rows, row_stride] elements of `dtype`; row r starts at
 *              logits + r * row_stride; only the first V are read.
 *   row_stride elements, >= V; a multiple of 16 bytes for the vector path.
 *   T          > 0. With z = x / T:
 *   row_max    [rows] fp32 out: max_v z_v
 *   row_lse    [rows] fp32 out: log sum_v exp(z_v)
 *   probs      [rows, V] fp32 out (nullable): exp(z_v - row_lse)
 *   workspace  >= spec_softmax_workspace_size(rows) bytes.
 * Non-finite rows produce non-finite outputs (no status flag).
 */
int spec_softmax_T(const void* logits, int dtype, int64_t rows, int64_t V, int64_t row_stride,
                   float T, float* row_max, float* row_lse, float* probs,
                   void* workspace, size_t ws_bytes, spec_stream_t stream);

/*
 * spec_softmax_T_noalloc — spec_softmax_T for callers that cannot allocate
 * device memory. The paper has no counterpart: this entry point exists only
 * for such callers. Arguments, results and numerics are those of
 * spec_softmax_T without the workspace; the call allocates nothing
 * (no cudaMalloc, cudaFree or allocating library routine).
 * Scratch: the statistics partials live in one fixed array inside the library
 * (static __device__, 256-byte aligned, (2048 + SPEC_NOALLOC_MAX_ROWS) * 8
 * bytes = 48 KiB on each device).
 *   rows  0 <= rows <= SPEC_NOALLOC_MAX_ROWS; larger returns
 *         SPEC_ERR_UNSUPPORTED before anything is launched.
 * Set-up: the first call on a device looks up the array's device address with
 * cudaGetSymbolAddress, with that device current (the current device must be
 * the stream's device), and caches it under the id of the current CUDA
 * context; a failed lookup returns SPEC_ERR_CUDA. Make that first call on
 * each device before any stream capture begins. A device reset ends the
 * context, so the first call after it looks the address up again (again
 * outside any capture).
 * Sharing: every call on a device uses the same array. Nothing in it has to
 * start at zero (each call writes every slot before it reads it), but calls
 * whose kernels overlap on the GPU (different streams, or different host
 * threads) race on the array and return wrong statistics: issue them in order
 * on one stream.
 */
int spec_softmax_T_noalloc(const void* logits, int dtype, int64_t rows, int64_t V, int64_t row_stride,
                           float T, float* row_max, float* row_lse, float* probs, spec_stream_t stream);

/*
 * spec_verify_block — lossless speculative-sampling verification of B
 * independently drafted blocks ([DBLAST] "Assumptions"; the independent
 * K = 1 proposal q(x_{1:L}|y) = prod_i q_i(x_i|y)).
 * For request b with verify length l = verify_len[b] (L if NULL):
 *   position i < l is accepted iff u[b,i] < min(1, p_i(x_i) / q_i(x_i)),
 *   p_i = softmax(target row i / T), q_i = softmax(draft row i / T);
 *   j = first rejected position, or l if none (found with a warp ballot);
 *   if j < l the terminal token is argmax_v log(p_j(v) - q_j(v)) + g[b,j,v]
 *   over {v : p_j(v) > q_j(v)} (Gumbel-max draw from norm(max(0, p_j - q_j)));
 *   if j = l it is argmax_v log p_l(v) + g[b,l,v] (the bonus token).
 *   Ties go to the lowest v.
 * Arguments:
 *   target_logits  dense [B, L+1, V] when target_row_off == NULL; otherwise
 *                  packed rows [*, V] where the row of (b, i) is
 *                  target_row_off[b] + i (e.g. offsets from dvl_allocate_pack).
 *   target_row_off [B] int32 (nullable), read on the device.
 *   draft_logits   [B, L, V] of the same dtype.
 *                  (draft_logits, draft_tokens and uniforms may be NULL when L == 0.)
 *   draft_tokens   [B, L] int32 x_i. A token outside [0, V) raises
 *                  SPEC_DEV_TOKEN_RANGE and that request gets accept_len = -1
 *                  and out_tokens = -1; nothing is read out of bounds.
 *   verify_len     [B] int32 (nullable -> L), read on the device.
 *   uniforms       [B, L] fp32 in [0, 1).
 *   gumbel         [B, L+1, V] fp32 noise, indexed by (request, terminal
 *                  position); only row j of each request is read.
 *   T              > 0.
 *   accept_len     [B] int32 out: j (number of accepted draft tokens).
 *   out_tokens     [B, L+1] int32 out: x_0..x_{j-1}, terminal token, then -1.
 *   workspace      >= spec_verify_workspace_size(B, L, 1, V) bytes, zeroed once.
 * Limits: 1 <= B <= SPEC_MAX_B, 0 <= L <= SPEC_MAX_L, 1 <= V <= SPEC_MAX_V.
 * Execution: the two stages of spec_verify_window_stats and
 * spec_verify_accept, chained with programmatic dependent launch.
 */
int spec_verify_block(const void* target_logits, const int32_t* target_row_off,
                      const void* draft_logits, int dtype,
                      const int32_t* draft_tokens, const int32_t* verify_len,
                      const float* uniforms, const float* gumbel,
                      int B, int L, int64_t V, float T,
                      int32_t* accept_len, int32_t* out_tokens,
                      void* workspace, size_t ws_bytes, spec_stream_t stream);

/*
 * spec_verify_mixture — verification of latent-mixture (dependent) drafts
 * ([DBLAST] "What carries the argument", Eq. 5:
 *   q_dep(x_{1:L}|y) = sum_z q(z|y) prod_i q_i(x_i|y,z)).
 * The proposal at position i is the mixture marginal under the category
 * posterior updated by the accepted prefix:
 *   log pi_i(z) = log w_z + sum_{k<i} log q_k(x_k|y,z) - normaliser,
 *   q_i(v) = sum_z pi_i(z) q_i(v|y,z);
 * the accept test, residual and bonus draws are those of spec_verify_block
 * with this q_i. With K = 1 and w = 1 the results are bit-identical to
 * spec_verify_block.
 *   draft_logits  [B, K, L, V]; mix_weights [B, K] fp32 probabilities q(z|y)
 *                 (any positive scale; zero excludes a category).
 *   workspace     >= spec_verify_workspace_size(B, L, K, V) bytes.
 * Other arguments as spec_verify_block. Limits: 1 <= K <= SPEC_MAX_K.
 */
int spec_verify_mixture(const void* target_logits, const int32_t* target_row_off,
                        const void* draft_logits, const float* mix_weights, int K, int dtype,
                        const int32_t* draft_tokens, const int32_t* verify_len,
                        const float* uniforms, const float* gumbel,
                        int B, int L, int64_t V, float T,
                        int32_t* accept_len, int32_t* out_tokens,
                        void* workspace, size_t ws_bytes, spec_stream_t stream);

/*
 * spec_verify_block_top_p, spec_verify_mixture_top_p — the same
 * verification with every row filtered to its top-p nucleus ([DBLAST]
 * "What would settle it": target sampling at T = 1.5 with top-p 0.95;
 * "Assumptions": target probabilities under the same sampling filter, here
 * applied to the target rows and to every draft category alike).
 * The nucleus of a row (temperature softmax of x / T) is the shortest run of
 * its tokens, ordered by probability descending and index ascending, whose
 * probability mass reaches top_p; kept tokens are renormalised by that mass
 * and every other token has probability 0. Then, as in spec_verify_block /
 * spec_verify_mixture with the filtered rows:
 *   a drafted token outside target row i's nucleus is rejected (p = 0);
 *   one that the filtered proposal gives probability 0 is accepted;
 *   the residual max(0, p_j - q_j) and the bonus row l are the filtered ones.
 * A request whose accepted tokens have probability 0 under every filtered
 * draft category (impossible when the drafts were sampled from the filtered
 * proposal) has no posterior: SPEC_DEV_NONFINITE, accept_len = -1.
 *   top_p      in (0, 1]; 1 is the unfiltered call (same results as
 *              spec_verify_block / spec_verify_mixture); NaN or <= 0:
 *              SPEC_ERR_ARG.
 *   workspace  >= spec_verify_top_p_workspace_size(B, L, K, V) bytes, zeroed
 *              once (it also serves the unfiltered calls of the same shape).
 * Other arguments and limits as spec_verify_block / spec_verify_mixture
 * (K = 1 and w = 1 for the block variant).
 * Execution: launches chained with programmatic dependent launch, over the
 * verify window plus each request's bonus row. For bf16 rows of 16-byte
 * vectors with V >= 4096 a windowed nucleus kernel finds each row's
 * normaliser and cut from one pass (the keys near the cut, chosen from a
 * strided sample, counted per value; every token's mass summed); the exact
 * nucleus kernel then takes only the rows it hands over (a NaN or an
 * infinity, or a crossing outside its window twice). Other rows go to the
 * exact kernel alone (bf16 value counts, or for fp32 a radix descent over
 * the logits' order keys with exact fixed-point masses, then the tie cut by
 * token index). The accept / sample stage follows with the filtered rows.
 */
size_t spec_verify_top_p_workspace_size(int B, int L, int K, int64_t V);

int spec_verify_block_top_p(const void* target_logits, const int32_t* target_row_off,
                            const void* draft_logits, int dtype,
                            const int32_t* draft_tokens, const int32_t* verify_len,
                            const float* uniforms, const float* gumbel,
                            int B, int L, int64_t V, float T, float top_p,
                            int32_t* accept_len, int32_t* out_tokens,
                            void* workspace, size_t ws_bytes, spec_stream_t stream);

int spec_verify_mixture_top_p(const void* target_logits, const int32_t* target_row_off,
                              const void* draft_logits, const float* mix_weights, int K, int dtype,
                              const int32_t* draft_tokens, const int32_t* verify_len,
                              const float* uniforms, const float* gumbel,
                              int B, int L, int64_t V, float T, float top_p,
                              int32_t* accept_len, int32_t* out_tokens,
                              void* workspace, size_t ws_bytes, spec_stream_t stream);

/*
 * The two stages that spec_verify_block / spec_verify_mixture launch, for
 * callers that schedule them separately (e.g. to time or overlap them).
 *
 * spec_verify_window_stats — stage 1, the fused temperature softmax over the
 * verify window ([DBLAST] "What would settle it"; same T for target and
 * draft): for every request b, target rows 0..l_b-1 and the K draft rows of
 * positions 0..l_b-1 (l_b = verify_len[b], L if NULL) are streamed once and
 * their (max, normaliser) statistics, and each row's logit at the drafted
 * token, are written into the workspace. Target row l_b (the bonus row)
 * needs no normaliser and is not read here. With L == 0 nothing is launched;
 * draft_logits and draft_tokens may then be NULL.
 *
 * spec_verify_accept — stage 2: category posterior (K > 1), accept tests,
 * first rejection, residual / bonus Gumbel-max draw and outputs, exactly as
 * described for spec_verify_block / spec_verify_mixture (mix_weights may be
 * NULL only when K == 1, meaning w = 1). It must follow stage 1 on the same
 * stream with the same target, draft, verify_len, B, L, K, V, T, dtype and
 * workspace, with no other call using that workspace in between.
 * Arguments and limits as spec_verify_mixture.
 */
int spec_verify_window_stats(const void* target_logits, const int32_t* target_row_off,
                             const void* draft_logits, int K, int dtype,
                             const int32_t* draft_tokens, const int32_t* verify_len,
                             int B, int L, int64_t V, float T,
                             void* workspace, size_t ws_bytes, spec_stream_t stream);

int spec_verify_accept(const void* target_logits, const int32_t* target_row_off,
                       const void* draft_logits, const float* mix_weights, int K, int dtype,
                       const int32_t* draft_tokens, const int32_t* verify_len,
                       const float* uniforms, const float* gumbel,
                       int B, int L, int64_t V, float T,
                       int32_t* accept_len, int32_t* out_tokens,
                       void* workspace, size_t ws_bytes, spec_stream_t stream);

/*
 * dvl_allocate_pack — dynamic verify-length allocation ([DSCALE] Abstract;
 * [QA] prefix survival probabilities).
 *   scores        [B, L] fp32 per-position survival scores s[b,i] in [0, 1]
 *                 (outside: SPEC_DEV_SCORES, results unspecified but in range;
 *                 NULL allowed when L == 0).
 *   P[b,i] = s[b,0] * ... * s[b,i] in fp64, left to right (non-increasing in i).
 *   budget        total verify slots, >= B; slots used = min(budget, B*(L+1)).
 *                 Every request keeps its root slot; the other
 *                 min(budget, B*(L+1)) - B slots go to the largest P overall,
 *                 ordered (P desc, b asc, i asc). Half capacity is
 *                 budget = floor(B*(L+1)/2).
 *   verify_len    [B] int32 out: number of positions selected in row b.
 *   offsets       [B+1] int32 out: exclusive scan of verify_len + 1
 *                 (offsets[B] = slots used).
 *   slot_map      [budget] int32 out (nullable): slot -> b*(L+1) + i, -1 if unused.
 *   dense_target  [B, L+1, V] (nullable) and packed_target [budget, V]
 *                 (nullable; both or neither): copies row (b, i), i <= verify_len[b],
 *                 to packed row offsets[b] + i. Unused packed rows are untouched.
 *   dtype, V      of the packed rows (ignored without packing).
 *   workspace     >= spec_dvl_workspace_size(B) bytes, zeroed once.
 * The outputs live at fixed addresses and feed spec_verify_* (verify_len,
 * target_row_off = offsets) on the device, so one captured graph serves
 * every allocation. Limits: B * L <= SPEC_MAX_DVL_ELEMS, L <= SPEC_MAX_L.
 * Execution: one thread block; a radix select over the products' 64-bit
 * keys finds the cut, so the work is O(B * L).
 */
int dvl_allocate_pack(const float* scores, int B, int L, int budget,
                      int32_t* verify_len, int32_t* offsets, int32_t* slot_map,
                      const void* dense_target, void* packed_target, int dtype, int64_t V,
                      void* workspace, size_t ws_bytes, spec_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SPECV_H */
