/*
 * Plain CPU fp64 oracle for block-draft speculative verification.
 *
 * TEST INFRASTRUCTURE ONLY. This library is the slow, obviously-correct
 * definition that the CUDA path is checked against. Only the test-suite,
 * the smoke check and the benchmark's CPU-baseline leg may load it; the
 * product library never links or calls it, and the two share no code.
 *
 * Every input is read exactly (bf16 bits widened to fp32, then to fp64);
 * all arithmetic is fp64 with libm exp/log, summed in ascending index order.
 *
 * Sources restated here (cited by page title and section):
 *  - "DBLAST: Dependent Block Drafting for Stochastic Speculative Decoding"
 *    (Pith review): "What carries the argument" (the latent-mixture proposal
 *    q_dep, Eq. 5, and verification conditioned on the accepted prefix
 *    through the category posterior); "Assumptions" (speculative sampling
 *    with rejection correction preserves the target distribution for any
 *    proposal, from the cited works of Leviathan et al. and Chen et al.);
 *    "What would settle it" (temperature-scaled target sampling).
 *  - "DScale: Scaling Block-Diffusion Speculative Decoding with Adaptive
 *    Verification", Abstract: dynamic verify-length (DVL) allocation packs
 *    scored prefixes into half the native verification capacity, into
 *    fixed-address workspaces.
 *  - "Why does throughput collapse under high concurrency?" (block-diffusion
 *    failure-mode Q&A): verify lengths tailored from prefix survival
 *    probabilities.
 */
#ifndef SPECV_ORACLE_H
#define SPECV_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1 };

enum {
  ORC_OK = 0,
  ORC_ERR_ARG = -1,
  /* per-request data errors (accept_len[b] = -1); the call still completes */
  ORC_FLAG_TOKEN_RANGE = 1,
  ORC_FLAG_NONFINITE = 2,
  ORC_FLAG_VERIFY_LEN = 4,
  ORC_FLAG_SCORES = 8
};

/* Optional per-request diagnostics of oracle_verify. Every pointer may be
 * NULL. Arrays indexed [b*L + i] hold NaN (or -1) for positions not tested. */
typedef struct {
  double* lp;            /* [B*L] log p_i(x_i): target log-prob of the drafted token */
  double* lq;            /* [B*L] log q_i(x_i): proposal log-prob (posterior marginal if K>1) */
  double* rho;           /* [B*L] rho_i = exp(lp_i - lq_i) */
  double* accept_margin; /* [B*L] |u_i - min(1, rho_i)| for every tested position */
  int32_t* terminal_row; /* [B] j: position whose distribution the last token is drawn from */
  int32_t* terminal_kind;/* [B] 0 = residual, 1 = bonus (all accepted), 2 = empty residual fallback */
  double* argmax_gap;    /* [B] fp64 gap between the two best terminal scores (+inf if one candidate) */
  double* argmax_kappa;  /* [B] max(1, kappa of the two best); kappa_v = p_v / (p_v - q_v) */
  double* terminal_dist; /* [B*V] normalised distribution the terminal token is a Gumbel-max draw from */
  double* nucleus_margin;/* [B] top_p < 1: smallest distance between top_p and the cumulative masses on
                            either side of the nucleus cut, over the rows the outputs depend on (+inf
                            for top_p = 1): below 1e-6 the nucleus itself is a low-margin decision */
} oracle_diag;

/* Temperature softmax of each row: z = x / T, row_max = max z,
 * row_lse = row_max + log sum exp(z - row_max), probs = exp(z - row_lse).
 * x rows start at x + r*row_stride (elements). probs (nullable) is [rows, V]. */
int oracle_softmax_T(const void* x, int dtype, int64_t rows, int64_t V, int64_t row_stride,
                     double T, double* row_max, double* row_lse, double* probs);

/* Speculative verification of B drafted blocks of length L.
 *  target:  dense [B, L+1, V] (target_row_off == NULL) or packed rows, where the
 *           target row of request b, position i is row target_row_off[b] + i.
 *  draft:   [B, K, L, V]; for K == 1 this is the independent block proposal.
 *  mix_w:   [B, K] category probabilities q(z|y); NULL means w = 1 (K must be 1).
 *  tokens:  [B, L] drafted tokens x_i; u: [B, L] uniforms in [0, 1);
 *  g:       [B, L+1, V] Gumbel noise, indexed by (request, terminal position).
 *  verify_len: [B] (nullable -> L) number of positions that are tested.
 *  top_p:   in (0, 1]; below 1 every row's temperature softmax is filtered to
 *           its nucleus before use (the smallest set of most probable tokens,
 *           ties to the lower index, whose mass reaches top_p, renormalised;
 *           other tokens get probability 0), for the target and for every
 *           draft category alike. 1 leaves the rows unfiltered.
 *  Outputs: accept_len [B], out_tokens [B, L+1] (accepted prefix, the
 *  terminal token, then -1). Returns ORC_ERR_ARG, or the OR of per-request flags. */
int oracle_verify(const void* target, const int32_t* target_row_off, const void* draft, int dtype,
                  const int32_t* tokens, const int32_t* verify_len, const float* u, const float* g,
                  const float* mix_w, int K, int B, int L, int64_t V, double T, double top_p, int n_threads,
                  int32_t* accept_len, int32_t* out_tokens, const oracle_diag* diag);

/* DVL allocation: prefix-survival products P[b,i] = s[b,0]*...*s[b,i] (fp64,
 * left to right), greedy global top-(budget' - B) over P with order
 * (P desc, b asc, i asc) where budget' = min(budget, B*(L+1)); verify_len[b]
 * = number selected in row b; offsets = exclusive scan of verify_len+1
 * ([B+1]); slot_map[budget]: packed slot -> dense row b*(L+1)+i, -1 unused.
 * prefix (nullable) receives P. */
int oracle_dvl_allocate(const float* scores, int B, int L, int budget,
                        int32_t* verify_len, int32_t* offsets, int32_t* slot_map, double* prefix);

/* Copy dense target rows [B, L+1, V] into the packed buffer:
 * packed[offsets[b] + i] = dense[b, i] for i <= verify_len[b]. */
int oracle_pack(const void* dense, int dtype, int B, int L, int64_t V,
                const int32_t* verify_len, const int32_t* offsets, void* packed);

#ifdef __cplusplus
}
#endif
#endif
