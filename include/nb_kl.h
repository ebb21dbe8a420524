/*
 * nb_kl — full-vocabulary hidden-state distillation loss on NVIDIA B200 (sm_100a).
 *
 * C ABI. Every pointer argument named h_*, W_*, labels, loss_*, lse_*, aux, n_valid,
 * grad_out, dh_s, dW_s and workspace is a DEVICE pointer; shapes are passed by value in
 * a host-side nb_kl_shape. Nothing here allocates device memory: the caller owns every
 * buffer, including the workspace. All calls are asynchronous on `stream` (a
 * cudaStream_t passed as void*; NULL = legacy default stream).
 *
 * What is computed ("Nitrobrew tweet analysis", sections "Nitrobrew 的两个动作" and
 * "工程落地"; "03 White-box OPD", sections 1 and 2.3):
 *   z_s = h_s W_s^T, z_t = h_t W_t^T, rebuilt one vocabulary block at a time and never
 *   stored; u = z / tau (temperature inside the softmax); S = softmax(u_s),
 *   T = softmax(u_t);
 *   beta == 0:   loss_n = KL(T || S)              (forward KL)
 *   beta == 1:   loss_n = KL(S || T)              (reverse KL, the OPD objective)
 *   0 < beta < 1: loss_n = beta KL(T || M) + (1 - beta) KL(S || M),
 *                 M = (1 - beta) S + beta T       (generalized JSD)
 *   loss_mean = sum over rows with label != ignore_index of loss_n / N_v
 *   (a per-token mean; 0 when N_v == 0).
 * The teacher is frozen: the backward returns dL/dh_s and dL/dW_s only.
 *
 * Layouts: h_s [n_tokens, d_s], h_t [n_tokens, d_t] row-major (bf16 or fp32, see
 * nb_kl_shape.h_dtype); W_s [vocab, d_s], W_t [vocab, d_t] row-major bf16; labels
 * [n_tokens] int64; every per-token output [n_tokens] fp32; dh_s [n_tokens, d_s] fp32;
 * dW_s [vocab, d_s] fp32. Row n of h_s, h_t and labels is one position (no shift).
 *
 * Requirements (NB_ERR_INVALID_ARG otherwise): d_s and d_t multiples of 8 in [8, 65536];
 * 1 <= vocab <= 2^30; 0 <= n_tokens <= 2^30 (n_tokens may be 0); reserved == 0; chunk_v a
 * multiple of 256 or 0; h_*, W_* and the workspace 16-byte aligned; 0 <= beta <= 1; tau > 0
 * and finite. A workspace smaller than nb_kl_workspace_size(shape, beta) gives
 * NB_ERR_WORKSPACE.
 *
 * Errors: invalid arguments are reported synchronously by the return value and launch
 * nothing. Device-side failures (a bounded wait that ran out) are written to a status
 * word inside the workspace; nb_kl_device_status() reads it. Every forward/backward call
 * clears that word when it starts.
 */
#ifndef NB_KL_H
#define NB_KL_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NB_KL_API __attribute__((visibility("default")))
#else
#define NB_KL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nb_status {
  NB_OK = 0,
  NB_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, bad size, beta or tau out of range */
  NB_ERR_UNSUPPORTED = -2,  /* no sm_100 device, or a size beyond what the kernels index */
  NB_ERR_WORKSPACE = -3,    /* workspace smaller than nb_kl_workspace_size() */
  NB_ERR_CUDA = -4,         /* a CUDA runtime / driver call failed */
  NB_ERR_TIMEOUT = -5       /* a bounded device-side wait ran out (device status word) */
} nb_status;

typedef enum nb_dtype { NB_BF16 = 0, NB_F32 = 1 } nb_dtype;

typedef struct nb_kl_shape {
  int64_t n_tokens;     /* N = B * T rows of h_s, h_t, labels */
  int64_t vocab;        /* V */
  int64_t d_s;          /* student hidden width */
  int64_t d_t;          /* teacher hidden width (or the rank of a compressed teacher code) */
  int32_t h_dtype;      /* nb_dtype of h_s and h_t; W_s and W_t are always bf16 */
  int32_t reserved;     /* must be 0 */
  int64_t ignore_index; /* label of masked positions, normally -100 */
  int64_t chunk_v;      /* backward vocabulary chunk (multiple of 256); 0 = library default */
} nb_kl_shape;

/* Bytes of scratch the calls need for this shape: O(n_tokens * (d_s + d_t + chunk_v))
 * plus O(n_tokens * vocab / 2048) floats of split-V state — never O(n_tokens * vocab).
 * Returns 0 for an invalid shape. */
NB_KL_API size_t nb_kl_workspace_size(const nb_kl_shape* shape, float beta);

/* Vocabulary columns per backward chunk for this shape: shape->chunk_v, or the library's
 * default when it is 0: the vocabulary cut into equal chunks, each a multiple of 256 columns
 * of at most max(2048, min(131072, max(24576 gradient tiles of 128 x 256 for the padded token
 * count, 4 d_s))) columns (at most ~1.5 GB of bf16 gradient chunk). 0 for an invalid shape. */
NB_KL_API int64_t nb_kl_chunk_columns(const nb_kl_shape* shape);

/* Forward ("Nitrobrew 的两个动作": block GEMMs + online log-sum-exp + KL numerator).
 * Outputs (device, caller-owned): loss_tok, lse_s, lse_t, aux [n_tokens] fp32 —
 * lse_* are natural-log LSEs of the tempered logits u = z / tau; aux is the per-token KL
 * for beta in {0, 1} and KL(S || M) for 0 < beta < 1 (the backward needs it); masked rows
 * get 0 in all four. loss_mean: one fp32; n_valid: one int64 (N_v). */
NB_KL_API nb_status nb_kl_forward(const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t,
                        const void* W_t, const int64_t* labels, float beta, float tau, float* loss_tok,
                        float* lse_s, float* lse_t, float* aux, float* loss_mean, int64_t* n_valid,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Forward plus per-token side outputs of the student from the same sweep
 * ("01 · 论文精读与参考实现全景映射", section 1: Eq. 6, the per-token entropy H_t that the
 * peak-entropy scheduler of section 3.5 ranks; Eq. 8, log pi_theta(y_t | .) of the
 * student's own sampled token). Both are taken under the tempered student softmax
 * S = softmax(z_s / tau) that the loss uses, in nats:
 *   entropy_s[n]  = -sum_v S[n,v] ln S[n,v]
 *   logp_label[n] = ln S[n, labels[n]]   (NaN when labels[n] is outside [0, vocab))
 * entropy_s and logp_label are device fp32 [n_tokens], caller-owned; either may be NULL
 * (both NULL is nb_kl_forward). Masked rows get 0 in both. Every other argument and result
 * is that of nb_kl_forward, with the same workspace. */
NB_KL_API nb_status nb_kl_forward_side(const nb_kl_shape* shape, const void* h_s, const void* W_s,
                             const void* h_t, const void* W_t, const int64_t* labels, float beta, float tau,
                             float* loss_tok, float* lse_s, float* lse_t, float* aux, float* loss_mean,
                             int64_t* n_valid, float* entropy_s, float* logp_label, void* workspace,
                             size_t workspace_bytes, void* stream);

/* ---- Vocabulary-parallel forward (the unembeddings split by rows across ranks) ----------
 * "Nitrobrew tweet analysis", section "工程落地": under tensor parallelism the unembedding is
 * sharded, and the full-vocabulary loss then needs one exchange per token. Each rank holds
 * rows [vocab_offset, vocab_offset + shape->vocab) of W_s and W_t (W_s / W_t point at the
 * shard) and the full h_s, h_t and labels. The per-token online softmax state of a shard is
 * merged across shards with the same log-sum-exp merge the single-GPU call uses between its
 * vocabulary splits, so the result equals the unsharded call up to summation order.
 *
 * Flow on every rank (the exchange is the caller's, e.g. an all-gather over NCCL):
 *   nb_kl_vp_state      -> state  [NB_KL_VP_FIELDS][n_tokens]      (local shard)
 *   all-gather          -> states [n_parts][NB_KL_VP_FIELDS][n_tokens] (parts in rank order)
 *   nb_kl_vp_combine    -> lse_s, lse_t, entropy_s, logp_label; for beta in {0, 1} also
 *                          loss_tok, aux, loss_mean, n_valid (final)
 *   for 0 < beta < 1:  nb_kl_vp_jsd_partial (local shard, global lse_s / lse_t)
 *                      -> part [2][n_tokens];  all-gather -> parts [n_parts][2][n_tokens];
 *                      nb_kl_vp_jsd_combine -> loss_tok, aux, loss_mean, n_valid
 * The backward needs no new call: nb_kl_backward on the shard with the global lse_s, lse_t
 * and aux gives this shard's rows of dW_s exactly and its term of dh_s; dh_s is the sum of
 * the ranks' terms (an all-reduce).
 *
 * State layout: fp32, field-major, base-2 tempered units (x = z log2(e) / tau): the running
 * maxima and rescaled sums of both models (m_s, l_s, m_t, l_t), the KL numerator a (beta in
 * {0, 1}), the student entropy accumulator e, and the student's x at the row's label (NaN
 * when the label is not in this shard). Masked rows hold 0 and are never read. */
#define NB_KL_VP_FIELDS 7

/* First part on one shard. shape->vocab is the shard's row count; the workspace is sized by
 * nb_kl_workspace_size(shape, beta). Labels keep their global values. 0 <= vocab_offset <= 2^30. */
NB_KL_API nb_status nb_kl_vp_state(const nb_kl_shape* shape, int64_t vocab_offset, const void* h_s,
                         const void* W_s, const void* h_t, const void* W_t, const int64_t* labels, float beta,
                         float tau, float* state, void* workspace, size_t workspace_bytes, void* stream);

/* Merge of n_parts (1 to 4096) gathered shard states (device, [n_parts][NB_KL_VP_FIELDS][n_tokens])
 * in part order, in fp64. Outputs as nb_kl_forward_side (entropy_s / logp_label may be NULL);
 * for 0 < beta < 1, loss_tok and aux are written as 0 and loss_mean / n_valid are those of
 * the zero losses: nb_kl_vp_jsd_combine replaces them. No workspace. */
NB_KL_API nb_status nb_kl_vp_combine(int64_t n_tokens, int n_parts, const float* states, const int64_t* labels,
                           int64_t ignore_index, float beta, float* loss_tok, float* lse_s, float* lse_t,
                           float* aux, float* entropy_s, float* logp_label, float* loss_mean, int64_t* n_valid,
                           void* stream);

/* Second JSD sweep on one shard (0 < beta < 1 only) with the merged natural-log lse_s /
 * lse_t [n_tokens]: part[0][n] = the shard's terms of the divergence of row n, part[1][n] =
 * its terms of KL(S || M), in nats (device fp32 [2][n_tokens]; masked rows 0). */
NB_KL_API nb_status nb_kl_vp_jsd_partial(const nb_kl_shape* shape, const void* h_s, const void* W_s,
                               const void* h_t, const void* W_t, const int64_t* labels, float beta, float tau,
                               const float* lse_s, const float* lse_t, float* part, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Sum of n_parts gathered JSD partials ([n_parts][2][n_tokens]) in part order, in fp64:
 * loss_tok, aux [n_tokens], loss_mean, n_valid. No workspace. */
NB_KL_API nb_status nb_kl_vp_jsd_combine(int64_t n_tokens, int n_parts, const float* parts,
                               const int64_t* labels, int64_t ignore_index, float* loss_tok, float* aux,
                               float* loss_mean, int64_t* n_valid, void* stream);

/* ---- Spectral-compression front end ----------------------------------------------------
 * "Nitrobrew tweet analysis": thread item 6/8 (spectral compression shrinks the hidden state
 * below d_model, no longer exactly) and the evaluation table's "SVD-Nitrobrew" row (k floats
 * per token). With the thin SVD W_t = U S V^T and V_k the right singular vectors of the k
 * largest singular values, the teacher sends h_t' = V_k^T h_t and the loss uses
 * W_t' = W_t V_k = U_k S_k with d_t = k: its teacher logits are those of the best rank-k
 * approximation of W_t. Both products are nb_kl_project; V_k comes from the eigenvectors of
 * the Gram matrix nb_kl_gram(W_t) (the small d_t x d_t eigendecomposition is the caller's,
 * once per teacher checkpoint). Both run on the same tcgen05 GEMM as the backward.
 *
 * Workspace of both calls: NB_KL_SMALL_WORKSPACE_BYTES of device memory (status word), 16-byte
 * aligned; nb_kl_device_status reads it. Pointers are device pointers, 16-byte aligned. */
#define NB_KL_SMALL_WORKSPACE_BYTES 256

/* G = X^T X: X [rows, d] bf16 row-major, G [d, d] fp32 (overwritten; fp32 accumulation).
 * d a multiple of 8, 8 <= d <= 65536, 1 <= rows <= 2^30. */
NB_KL_API nb_status nb_kl_gram(const void* X, int64_t rows, int64_t d, float* G, void* workspace, void* stream);

/* Y = X B: X [rows, d] bf16, B [d, k] bf16 (row-major: k contiguous), Y [rows, k] bf16, the
 * fp32 sum rounded to nearest even. d and k multiples of 8 (>= 8, <= 65536). Teacher codes
 * (X = h_t, B = V_k) and the compressed unembedding (X = W_t, B = V_k). */
NB_KL_API nb_status nb_kl_project(const void* X, int64_t rows, int64_t d, const void* B, int64_t k, void* Y,
                        void* workspace, void* stream);

/* Rank-k basis from the eigenpairs of G = W_t^T W_t ("Nitrobrew tweet analysis", thread item 6/8
 * and the evaluation table's "SVD-Nitrobrew" row: the code keeps the right singular vectors of
 * the k largest singular values of W_t). evals [d] fp64 and evecs [d, d] fp64 row-major with
 * eigenvector i in column i (the layout of a symmetric eigensolver's output; any eigenvalue
 * order). Writes V_k [d, k] bf16 row-major: column r is the eigenvector of the r-th largest
 * eigenvalue (ties by index, NaN last), rounded to nearest even from fp64 once; sigma [k] fp64:
 * sqrt(max(lambda, 0)), the singular values of W_t (NaN stays NaN); and, unless NULL, V_k_f64 [d, k] fp64, the
 * same columns unrounded. 1 <= k <= d <= 65536; all buffers on the device, caller-owned. */
NB_KL_API nb_status nb_kl_spectral_select(const double* evals, const double* evecs, int64_t d, int64_t k,
                                          void* V_k, double* sigma, double* V_k_f64, void* stream);

/* ---- Teacher -> student hand-off of hidden states -----------------------------------------
 * "Nitrobrew tweet analysis", thread items 3/8 and 4/8 and section "OPD 为什么更痛": when teacher
 * and student sit on different GPUs, what must cross to the loss is the teacher's final hidden
 * state (d_t values per token, or the rank-k code) instead of V logits. src is the teacher's
 * [n_rows, row_bytes] buffer as this process sees it: another GPU's memory reached through peer
 * access (nb_kl_enable_peer_access) or a CUDA IPC mapping, or local memory. The kernel reads it
 * with plain 16-byte loads (no TMA, no multicast) and writes dst (local, [n_rows, row_bytes]);
 * with labels (device int64 [n_rows]) only rows whose label is not ignore_index cross the link
 * and the other dst rows keep their contents. Both pointers 16-byte aligned, row_bytes a
 * multiple of 16 (at most 2^24). The loss can also take src directly as h_t: its row gather
 * then reads the valid rows over the link in each call (forward and backward), where one
 * hand-off into local memory reads them once. */
NB_KL_API nb_status nb_kl_handoff_rows(const void* src, void* dst, int64_t n_rows, int64_t row_bytes,
                             const int64_t* labels, int64_t ignore_index, void* stream);

/* Enable this device's access to peer_device's memory (cudaDeviceEnablePeerAccess; already
 * enabled is not an error). NB_ERR_UNSUPPORTED when the devices cannot reach each other. */
NB_KL_API nb_status nb_kl_enable_peer_access(int peer_device);

/* Backward ("仓库实现": recompute the logit blocks; gradients reach h_s and W_s only).
 * Inputs lse_s, lse_t, aux are the forward's outputs for the same arguments; grad_out is
 * one fp32 on the device (dOut/dloss_mean). Writes dh_s [n_tokens, d_s] (masked rows 0)
 * and dW_s [vocab, d_s]: overwritten, or added to when accumulate_dW != 0. */
NB_KL_API nb_status nb_kl_backward(const nb_kl_shape* shape, const void* h_s, const void* W_s, const void* h_t,
                         const void* W_t, const int64_t* labels, float beta, float tau, const float* lse_s,
                         const float* lse_t, const float* aux, const float* grad_out, float* dh_s, float* dW_s,
                         int accumulate_dW, void* workspace, size_t workspace_bytes, void* stream);

/* Size of the fixed device scratch behind nb_kl_forward_noalloc (64 MiB per device). */
#define NB_KL_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* Forward without a caller-supplied workspace, for callers that cannot allocate device
 * memory themselves: code that runs under a memory manager owning every device byte (a raw
 * cudaMalloc would escape its accounting or fail its budget), or code that must not call
 * cudaMalloc/cudaFree at all because those calls can synchronise the device. The pages have
 * no counterpart; this is a deployment convenience.
 * Same arguments and results as nb_kl_forward minus the workspace. The scratch is one fixed
 * array of NB_KL_NOALLOC_SCRATCH_BYTES in the library's device image; every device that loads
 * the library holds it until the process exits. Shapes whose nb_kl_workspace_size exceeds it
 * return NB_ERR_WORKSPACE without launching anything. Nothing is allocated: the first call on
 * a device looks up the array's device address (cudaGetSymbolAddress, with that device
 * current) and caches it, so make that first call before any stream capture. All calls share
 * the one array and it keeps the previous call's contents (the call clears what must start
 * at zero): calls that may overlap on the GPU — from several streams or threads — race and
 * must be serialised by the caller. */
NB_KL_API nb_status nb_kl_forward_noalloc(const nb_kl_shape* shape, const void* h_s, const void* W_s,
                                          const void* h_t, const void* W_t, const int64_t* labels, float beta,
                                          float tau, float* loss_tok, float* lse_s, float* lse_t, float* aux,
                                          float* loss_mean, int64_t* n_valid, void* stream);

/* Device status word of nb_kl_forward_noalloc's fixed scratch on the current device, read the
 * way nb_kl_device_status reads a caller's workspace: synchronises `stream`, then returns NB_OK,
 * or NB_ERR_TIMEOUT when a bounded pipeline wait of the last call ran out (its outputs are then
 * not valid), or NB_ERR_CUDA. Like every other use of the shared array, call it after the
 * forward it checks and before the next nb_kl_forward_noalloc on this device: the next call
 * clears the word. The pages have no counterpart. */
NB_KL_API nb_status nb_kl_noalloc_device_status(void* stream);

/* Static text for a status code. */
NB_KL_API const char* nb_kl_status_string(nb_status status);

/* Synchronises `stream`, then returns the device status word of `workspace`
 * (NB_OK, or NB_ERR_TIMEOUT after a bounded wait ran out), or NB_ERR_CUDA. */
NB_KL_API nb_status nb_kl_device_status(void* workspace, void* stream);

/* ---- test hooks (no counterpart on the pages) ---------------------------------------- */

/* C[M, N] = sum_k A[m, k] B[n, k] in fp32 with the library's tcgen05 GEMM. A is stored
 * row-major as [M, K] (a_mn_major = 0) or [K, M] (a_mn_major = 1); B as [N, K]
 * (b_mn_major = 0) or [K, N] (b_mn_major = 1); bf16, 16-byte aligned, leading
 * dimensions multiples of 8. workspace needs 256 bytes (status word). */
NB_KL_API nb_status nb_kl_debug_gemm(const void* A, int a_mn_major, const void* B, int b_mn_major, int64_t M, int64_t N,
                           int64_t K, float* C, void* workspace, void* stream);

/* Launches a kernel whose mbarrier wait can never complete, bounded by limit_ns (at most 5 s),
 * so that the timeout path can be exercised without hanging the GPU: sleeping != 0 waits with
 * the sleeping barrier tests of the pipeline kernels (the limit is checked every 16 suspensions
 * of at most 1 ms), sleeping == 0 by polling. Afterwards nb_kl_device_status(workspace) reports
 * NB_ERR_TIMEOUT. workspace: 256 bytes, device memory. */
NB_KL_API nb_status nb_kl_debug_wait_timeout(void* workspace, uint64_t limit_ns, int sleeping, void* stream);

/* Number of kernel launches the last forward / backward call on this thread made. */
NB_KL_API int nb_kl_last_launch_count(void);

/* ---- measurement hooks (no counterpart on the pages) --------------------------------- */

/* Kernel categories of the timing hook. */
enum {
  NB_KL_KERNEL_SWEEP_FWD = 0,   /* forward vocabulary sweep (block GEMMs + online LSE/KL) */
  NB_KL_KERNEL_SWEEP_JSD = 1,   /* second forward sweep of the JSD */
  NB_KL_KERNEL_SWEEP_GRAD = 2,  /* backward recompute sweep writing the gradient chunk */
  NB_KL_KERNEL_GEMM_BWD = 3,    /* backward dh_s / dW_s GEMMs */
  NB_KL_KERNEL_ROWOPS = 4,      /* compaction, merges, mean */
  NB_KL_KERNEL_GEMM_PROJ = 5,   /* spectral front end: Gram and projection GEMMs */
  NB_KL_KERNEL_HANDOFF = 6,     /* hand-off copy of hidden rows */
  NB_KL_KERNEL_CATEGORIES = 7
};

/* Per calling thread: when on, every launch is bracketed by two CUDA events recorded on
 * its stream (no synchronisation is added). Off by default. */
NB_KL_API void nb_kl_timing_enable(int on);

/* Waits for the recorded events, writes the summed milliseconds and launch counts per
 * category into ms[ncat] / launches[ncat] (either may be NULL), clears the record and
 * returns the number of launches read. */
NB_KL_API int nb_kl_timing_read(double* ms, int* launches, int ncat);

#ifdef __cplusplus
}
#endif

#endif /* NB_KL_H */
