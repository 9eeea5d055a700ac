/*
 * safe_attn.h - C ABI of the SAFE-DiT attention hot path for NVIDIA B200
 * (sm_100a). Library: libsafe_attn.so (mask_free_b200/).
 *
 * Source of every operation: "SAFE-DiT: Semantics-Aware Fast-path Execution
 * for High-Resolution Diffusion Transformers" (arXiv 2606.29360), cited below
 * by equation number.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers marked "device" are caller-owned device memory on the current
 *    CUDA device; pointers marked "host" are host memory. The library
 *    allocates no device memory. It keeps state between calls in two
 *    places only: the device status word (safe_get_device_status) and the
 *    fixed scratch array of the allocation-free entry point
 *    safe_pcsp_topk_noalloc, which holds the last such call's per-head
 *    partial scores.
 *  - bf16 tensors are passed as `const void*` / `void*` and must be 16-byte
 *    aligned and contiguous in the layouts stated (row-major, innermost last):
 *      image tensors Q, K, V, O, Kc, Vc    [B, N, H, d]
 *      compact row tensors (rows of S)     [B, k, H, d]
 *      text tensors Ky, Vy                 [B, M, H, d]
 *      hidden states X (row-wise layers)   [B, N, d_in], weights W^T [d_out, d_in]
 *  - Supported head dims d (attention): 64, 96, 128. `scale` is the logit scale (the
 *    paper uses 1/sqrt(d), Eq. (2)); it must be finite and positive, else
 *    SAFE_ERR_INVALID_ARG.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Every
 *    call is asynchronous on `stream` unless it says "synchronises".
 *  - Errors: arguments are validated on the host before any launch and a
 *    violation returns SAFE_ERR_INVALID_ARG (or SAFE_ERR_UNSUPPORTED for a
 *    legal but unimplemented shape) without touching device memory. A failed
 *    launch returns SAFE_ERR_CUDA. Problems only visible on the device (an
 *    index out of range, a non-ascending S, a valid length outside [1, M], a
 *    NaN score, a pipeline wait that timed out) never fault or hang: the
 *    kernel skips the offending access and sets a bit in the device status
 *    word, read with safe_get_device_status.
 */
#ifndef SAFE_ATTN_H
#define SAFE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAFE_OK = 0,
  SAFE_ERR_INVALID_ARG = 1,
  SAFE_ERR_UNSUPPORTED = 2,
  SAFE_ERR_CUDA = 3,
  SAFE_ERR_TIMEOUT = 4,      /* device-side: a pipeline wait exceeded its limit */
  SAFE_ERR_DEVICE_CHECK = 5  /* device-side: an input failed a device check */
} safe_status;

typedef enum { SAFE_BOOL = 0, SAFE_U8 = 1, SAFE_F32 = 2, SAFE_F16 = 3, SAFE_BF16 = 4 } safe_dtype;

/* ABI version of this header (bumped on any signature or entry-point change): 7. */
int safe_abi_version(void);
const char* safe_status_string(int status);

/*
 * Row-constant mask classifier: Eq. (6) (class R) applied independently to
 * every broadcast query row, as stated after Eq. (6); Eq. (7) shows such rows
 * leave softmax unchanged, so a mask in R may be dropped (Eq. (8)).
 *
 *  mask     device, the mask's first element.
 *  dtype    SAFE_BOOL / SAFE_U8: nonzero = key visible; a row is in R iff
 *           every key is visible. SAFE_F32 / SAFE_F16 / SAFE_BF16: additive
 *           bias; a row is in R iff every entry is finite and equal (by value,
 *           -0 == +0) to the others.
 *  sizes    host, 4 sizes of the view [B, H, n_q, n_k] (each >= 1).
 *  strides  host, 4 strides in ELEMENTS (>= 0). A dimension with stride 0 is
 *           a broadcast dimension: its rows are the same stored row and count
 *           once (its size is treated as 1 for counting and indexing).
 *  d_result device, int64[3] written by the call: {verdict (1 = every row in
 *           R, the mask is removable; 0 = keep the original masked call),
 *           nfail = number of distinct rows not in R, first_fail = smallest
 *           flat index b*H'*Q' + h*Q' + i of a failing row over the distinct
 *           extents H', Q' (-1 if none)}.
 * The mask is read once. Deliberate departure from the paper, which
 * certifies masks by provenance and never scans them (text after Eq. (8)):
 * a caller with provenance simply skips this call.
 */
safe_status safe_mask_classify(const void* mask, int dtype, const int64_t sizes[4], const int64_t strides[4],
                               int64_t* d_result, void* stream);

/* As safe_mask_classify, then synchronises `stream` and copies the result to
 * host h_result[3] (same order). d_result is device scratch of 3 int64. */
safe_status safe_mask_classify_sync(const void* mask, int dtype, const int64_t sizes[4],
                                    const int64_t strides[4], int64_t* d_result, int64_t* h_result,
                                    void* stream);

/*
 * Mask-free image self-attention, Eq. (3) with m_img elided (Eq. (8)):
 *   O[b,i,h,:] = sum_j softmax_j(scale * <Q[b,i,h,:], K[b,j,h,:]>) V[b,j,h,:]
 * over all N keys.
 *  Q, K, V  device bf16 [B, N, H, d];  O device bf16 [B, N, H, d] (written).
 *  lse      device fp32 [B, H, N] natural-log log-sum-exp of the scaled
 *           logits, or NULL.
 *  ws       device workspace of safe_attn_workspace_bytes(B, N, N, H, d)
 *           bytes (256-byte aligned), or NULL. With it, the units of the
 *           last, partial wave of CTAs are split into key ranges whose
 *           partial results a second small kernel merges (balances the
 *           wave); without it every CTA takes all keys. The parts keep
 *           their O / l in bf16 beside their fp32 running max and sum, so a
 *           split row carries one more bf16 rounding (2^-9 relative) than
 *           an unsplit one. Contents need no initialisation; the size is 0
 *           when no split pays off.
 * fp32 accumulation and softmax; O is rounded to bf16 (nearest even).
 */
size_t safe_attn_workspace_bytes(int B, int n_q, int N, int H, int d);
safe_status safe_attn_self(const void* Q, const void* K, const void* V, void* O, float* lse, int B, int N, int H,
                           int d, float scale, void* ws, size_t ws_bytes, void* stream);

/*
 * Image->text cross-attention keeping the text padding mask, Eq. (4), and its
 * row-selective form Eq. (17):
 *   O[b,r,h,:] = sum_{j < valid_len[b]} softmax_j(scale * <Q[b,i_r,h,:], Ky[b,j,h,:]>) Vy[b,j,h,:]
 * Padding is the per-sample valid key length (keys j < valid_len[b] are
 * valid; right padding); it is never materialised as a mask, and padding
 * key/value rows are never read (they may hold any bytes, NaN included).
 *  Q        device bf16 [B, N, H, d].
 *  q_idx    device int32 [B, nq] query rows i_r (the sensitive set S,
 *           ascending, values in [0, N)), or NULL for all rows (nq == N).
 *  Ky, Vy   device bf16 [B, M, H, d], M <= 256.
 *  valid_len device int32 [B], each in [1, M] (clamped and flagged if not).
 *  O        device bf16 [B, nq, H, d] (written).
 */
safe_status safe_attn_cross(const void* Q, const int32_t* q_idx, int nq, const void* Ky, const void* Vy,
                            const int32_t* valid_len, void* O, int B, int N, int M, int H, int d, float scale,
                            void* stream);

/*
 * PCSP sensitivity scores and top-k partition, Eq. (9), (10), (12):
 *   scores[b,i] (+)= (1/H) * sum_h sum_{j < valid_len[b]} w[b,j] * A_{b,h}[i,j]
 * where A is the exact image->text attention probability of Eq. (9) (same
 * arithmetic as safe_attn_cross; the head sum runs in a fixed order, so the
 * scores are bit-reproducible). Then, if k > 0, the top-k split of Eq. (12)
 * on the resulting scores (see safe_topk_partition).
 *  Q, Ky, valid_len  as safe_attn_cross; Q may be NULL to skip scoring and
 *           only partition the given scores.
 *  w        device fp32 [B, M] content weights (>= 0, zero on padding), or
 *           NULL for uniform 1/valid_len[b] weights on the valid keys.
 *  scores   device fp32 [B, N], in/out. accumulate = 1 adds this call's
 *           scores (one warm-up step and layer of Eq. (10)) to the buffer;
 *           0 overwrites it. The 1/(|W||L|) mean over calls is left to the
 *           caller (a positive constant does not change the top-k).
 *  k        0 = scores only; else 1 <= k <= N, S device int32 [B, k] and C
 *           device int32 [B, N-k] (C may be NULL), each strictly ascending.
 *  ws       device workspace of at least safe_pcsp_workspace_bytes(B, N, H)
 *           bytes (per-head partial scores), 256-byte aligned.
 */
size_t safe_pcsp_workspace_bytes(int B, int N, int H);
safe_status safe_pcsp_topk(const void* Q, const void* Ky, const int32_t* valid_len, const float* w, int B, int N,
                           int M, int H, int d, float scale, float* scores, int accumulate, int k, int32_t* S,
                           int32_t* C, void* ws, size_t ws_bytes, void* stream);

/*
 * Allocation-free variant of safe_pcsp_topk (the paper has no counterpart:
 * this is an interface for callers, not a step of the method).
 *
 * Some callers cannot allocate device memory: code hosted inside another
 * framework that owns every device allocation and hands its plugins no
 * workspace, and latency-critical loops whose memory plan is fixed at
 * start-up, where a cudaMalloc would synchronise the device or fail. This
 * entry point takes the same arguments as safe_pcsp_topk minus the workspace
 * and allocates nothing: the per-head partial scores go to a fixed 8 MiB
 * array inside the library (2^21 floats), which every GPU that loads the
 * library holds until the process exits.
 *  - Limit: B * H * N <= 2^21 (e.g. B = 2, H = 24, N <= 43690). Larger
 *    sizes return SAFE_ERR_UNSUPPORTED before any launch.
 *  - Set-up: the first call on a device (with that device current) looks up
 *    the array's device address once; make that first call before any stream
 *    capture.
 *  - Sharing: all calls on a device share the one array and it keeps the last
 *    call's contents (each call overwrites the part it reads, so nothing has
 *    to be cleared). Calls that overlap on the GPU (e.g. on two streams at
 *    once) race on it: serialise them.
 */
safe_status safe_pcsp_topk_noalloc(const void* Q, const void* Ky, const int32_t* valid_len, const float* w, int B,
                                   int N, int M, int H, int d, float scale, float* scores, int accumulate, int k,
                                   int32_t* S, int32_t* C, void* stream);

/*
 * Cross-attention and PCSP scores in one pass over the queries (the scores
 * of Eq. (10) are taken from the probabilities of the cross-attention call
 * itself, Eq. (9)): O exactly as safe_attn_cross with q_idx = NULL, and
 * scores / S / C exactly as safe_pcsp_topk with the same Q, Ky, valid_len,
 * w, accumulate and k (same arithmetic, bit-identical results).
 *  Arguments as those two calls; ws sized safe_pcsp_workspace_bytes(B, N, H).
 */
safe_status safe_attn_cross_pcsp(const void* Q, const void* Ky, const void* Vy, const int32_t* valid_len,
                                 const float* w, void* O, int B, int N, int M, int H, int d, float scale,
                                 float* scores, int accumulate, int k, int32_t* S, int32_t* C, void* ws,
                                 size_t ws_bytes, void* stream);

/*
 * Top-k partition of Eq. (12) on given scores: S[b] = the k tokens with the
 * largest score, ordered by (score descending, index ascending) so ties go to
 * the lower index; -0.0 ranks as +0.0; C[b] = the other N-k tokens. Both are
 * written sorted ascending. Exact (integer radix select on order-preserving
 * keys). A NaN score is flagged (SAFE_ERR_DEVICE_CHECK) and ranks lowest.
 *  scores device fp32 [B, N]; S device int32 [B, k]; C device int32 [B, N-k]
 *  or NULL.
 */
safe_status safe_topk_partition(const float* scores, int B, int N, int k, int32_t* S, int32_t* C, void* stream);

/*
 * SRSU selective self-attention, Eq. (16):
 *   O_S[b,r,h,:] = sum_j softmax_j(scale * <Q_S[b,r,h,:], Kc[b,j,h,:]>) Vc[b,j,h,:]
 * over all N keys of the global K/V (Kc, Vc: current sensitive rows and cached
 * context rows in original token order, i.e. after safe_ctx_cache_scatter).
 *  Q        device bf16: q_compact = 0: [B, N, H, d], rows gathered by S on
 *           the device (TMA gather); q_compact = 1: [B, k, H, d] already
 *           compact (S only documents the rows).
 *  S        device int32 [B, k], strictly ascending, values in [0, N).
 *  Kc, Vc   device bf16 [B, N, H, d].
 *  O_S      device bf16 [B, k, H, d] (written); lse device fp32 [B, H, k] or NULL.
 *  ws       device workspace (16-byte aligned, caller-owned, contents
 *           undefined after the call) of ws_bytes bytes, or NULL:
 *           safe_srsu_workspace_bytes(B, k, N, H, d) bytes: with
 *           q_compact = 0 the rows of S are first copied out of Q into it as a
 *           compact [B, k, H, d] tensor (faster than gathering them inside
 *           the attention kernel), and the rest serves the key split;
 *           safe_attn_workspace_bytes(B, k, N, H, d) bytes: the key split
 *           only; less: neither (every result is the same bit for bit).
 */
size_t safe_srsu_workspace_bytes(int B, int k, int N, int H, int d);
safe_status safe_srsu_attn(const void* Q, int q_compact, const int32_t* S, int k, const void* Kc, const void* Vc,
                           void* O_S, float* lse, int B, int N, int H, int d, float scale, void* ws, size_t ws_bytes,
                           void* stream);

/*
 * SRSU with the global keys assembled in the kernel, Eq. (14), (16): the key
 * and value rows of S come from the current sensitive rows, all other rows
 * from the context cache, in original token order; the cache is only read.
 * The result is bit-identical to safe_ctx_cache_scatter(Kcur, Vcur,
 * cur_compact, S, ...) into the cache followed by safe_srsu_attn on it, without
 * the scatter pass and without writing the cache (between anchors its rows of
 * S are never read as context, Eq. (14), (19)).
 *  Q          as safe_srsu_attn.
 *  S          device int32 [B, k], strictly ascending (as safe_topk_partition
 *             writes it), values in [0, N): it locates the rows of S inside
 *             each key tile. A row met out of order is skipped and sets bit
 *             (1 << SAFE_ERR_DEVICE_CHECK) in the device status word.
 *  Kcur, Vcur device bf16: cur_compact = 1: [B, k, H, d] (row r holds token
 *             S[b, r]); cur_compact = 0: [B, N, H, d] (rows S[b, r] are used).
 *  Kc, Vc     device bf16 [B, N, H, d], the context cache (read only).
 *  O_S, lse, ws, scale: as safe_srsu_attn.
 */
safe_status safe_srsu_attn_assembled(const void* Q, int q_compact, const int32_t* S, int k, const void* Kcur,
                                     const void* Vcur, int cur_compact, const void* Kc, const void* Vc, void* O_S,
                                     float* lse, int B, int N, int H, int d, float scale, void* ws, size_t ws_bytes,
                                     void* stream);

/*
 * Context-cache update, Eq. (14), (16), (19): write the current sensitive
 * rows into the cache in original token order (in place):
 *   Kc[b, S[b,r], :, :] = Ksrc[b, r or S[b,r], :, :]   (same for V)
 * S == NULL is the anchor refresh of Eq. (19): the whole cache becomes the
 * source (k ignored). Every other byte of the cache is left unchanged.
 *  Ksrc, Vsrc device bf16: src_compact = 1: [B, k, H, d]; 0: [B, N, H, d].
 *  S          device int32 [B, k] (values in [0, N); out-of-range rows are
 *             skipped and flagged), or NULL.
 *  Kc, Vc     device bf16 [B, N, H, d], updated in place.
 */
safe_status safe_ctx_cache_scatter(const void* Ksrc, const void* Vsrc, int src_compact, const int32_t* S, int k,
                                   void* Kc, void* Vc, int B, int N, int H, int d, void* stream);

/*
 * Sensitivity field of Eq. (11):  s = Norm(G_sigma * s~)  per sample.
 * The N = grid_h * grid_w scores of a sample (e.g. from safe_pcsp_topk) lie
 * on the latent token grid in row-major order (token i = y * grid_w + x).
 * G_sigma: the separable Gaussian exp(-t^2 / (2 sigma^2)) at integer offsets
 * |t| <= r = floor(truncate * sigma + 1/2), normalised to sum 1 (sigma = 0:
 * no smoothing); borders by half-sample reflection. Norm: per-sample min-max
 * map onto [0, 1]; a flat field maps to 0. The paper gives neither sigma nor
 * the border rule; both are inputs / stated readings. fp32 arithmetic.
 *  scores  device fp32 [B, N] (read); s device fp32 [B, N] (written; may
 *          not alias scores).
 *  ws      device workspace of safe_sensitivity_workspace_bytes(B, N) bytes
 *          (256-byte aligned); contents need no initialisation.
 *  sigma >= 0 and truncate > 0, finite, with r <= 128 (else
 *  SAFE_ERR_UNSUPPORTED). Top-k of s (Eq. (12)) with safe_topk_partition.
 */
size_t safe_sensitivity_workspace_bytes(int B, int N);
safe_status safe_sensitivity_field(const float* scores, float* s, int B, int grid_h, int grid_w, float sigma,
                                   float truncate, void* ws, size_t ws_bytes, void* stream);

/*
 * Binary sensitivity field of the SW-CFG binary variant (after Eq. (21)):
 * s[b, i] = 1 for i in S[b], 0 for the context tokens C.
 *  S  device int32 [B, k], strictly ascending, values in [0, N) (violations
 *     are flagged, SAFE_ERR_DEVICE_CHECK); s device fp32 [B, N] (written).
 */
safe_status safe_partition_indicator(const int32_t* S, int k, float* s, int B, int N, void* stream);

/*
 * Sensitivity-weighted classifier-free guidance, Eq. (20), (21):
 *   gamma_i = gamma_ctx + (gamma_sens - gamma_ctx) * s[b, i]
 *   out[b, i, c] = f_u[b, i, c] + gamma_i * (f_c[b, i, c] - f_u[b, i, c])
 * gamma_sens == gamma_ctx is standard CFG with that scale.
 *  f_c, f_u  device [B, N, C] conditional / unconditional predictions
 *            (token-major, C values per token), dtype SAFE_F32 or SAFE_BF16
 *            (naturally aligned; 16-byte vectors are used when every row
 *            and pointer allows).
 *  s         device fp32 [B, N] (e.g. from safe_sensitivity_field or
 *            safe_partition_indicator).
 *  out       device [B, N, C], same dtype; may alias f_c or f_u.
 * fp32 arithmetic; bf16 output rounded to nearest even.
 */
safe_status safe_sw_cfg(const void* f_c, const void* f_u, const float* s, void* out, int dtype, int B, int N, int C,
                        float gamma_ctx, float gamma_sens, void* stream);

/*
 * A row-wise layer of the row-selective block B^S (Eq. (15)) on the
 * sensitive rows only; with the row selection P_S of Eq. (13):
 *   Y[b, r, :] = act( X[b, S[b, r], :] W^T + bias ),   r < k
 * S == NULL: every row in order (r < N; the dense block of Eq. (18)), k
 * ignored. bf16 operands, fp32 accumulation on the tensor cores, bf16 result.
 * The projections and the MLP of the block are such layers; the paper names
 * no activation: act 0 = none, 1 = GELU in its tanh form
 * 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).
 *  X     device bf16 [B, N, d_in], token-major.
 *  S     device int32 [B, k] rows of X (any order; an index outside [0, N) is
 *        replaced by row 0 and flagged), or NULL.
 *  Wt    device bf16 [d_out, d_in] (the weight of y = x W^T + b).
 *  bias  device fp32 [d_out] (4-byte aligned) or NULL.
 *  Y     device bf16 [B, k or N, d_out] (written; may not overlap X or Wt).
 *  ws    device workspace of safe_gather_linear_workspace_bytes(B, k, d_in)
 *        bytes (16-byte aligned; caller-owned, contents undefined after the
 *        call), used with S only: the rows of S are first copied into it as
 *        a compact [B, k, d_in] matrix, which the GEMM then reads by tiled
 *        copies. NULL (or ws_bytes too small): the GEMM gathers the rows of
 *        S itself, correct but slower. Ignored when S == NULL.
 *        Every row (S == NULL or the compact copy) runs on CTA pairs
 *        (clusters of two SMs, 256 x 256 output tiles); the gathered form
 *        on single SMs (128 x 256 tiles). Both give the same bits.
 *  d_in >= 64 and d_out >= 8, both multiples of 8; X, Wt, Y 16-byte aligned.
 */
size_t safe_gather_linear_workspace_bytes(int B, int k, int d_in);
safe_status safe_gather_linear(const void* X, const int32_t* S, int k, const void* Wt, const float* bias, int act,
                               void* Y, int B, int N, int d_in, int d_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Device status word: synchronises `stream`, writes to *h_status (host) the
 * OR of (1 << code) over every device-side error code raised since the last
 * read, and clears the word. 0 = no device-side error.
 */
safe_status safe_get_device_status(int* h_status, void* stream);

/*
 * Self-test of the bounded device waits (no counterpart in the paper):
 * launches one CTA that waits on a barrier nothing ever arrives on, with a
 * limit of limit_ns nanoseconds (1 <= limit_ns <= 1e9). The wait gives up,
 * the kernel returns normally, and the next safe_get_device_status reports
 * bit (1 << SAFE_ERR_TIMEOUT). Used to test the timeout path without hanging
 * or faulting the GPU.
 */
safe_status safe_selftest_wait_timeout(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SAFE_ATTN_H */
