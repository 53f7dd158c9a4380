/*
 * lla.h — C ABI of the B200 (sm_100a) Looped Latent Attention library.
 *
 * Looped Latent Attention (LLA) compresses the loop-indexed K/V cache of a
 * weight-tied looped Transformer.  For each cached token, layer, head and axis
 * (K or V) the T per-loop vectors x = [x_1; ...; x_T] are replaced by one
 * latent c = (x - mu) W_down, and loop t's vector is rebuilt on read as
 * x_hat_t = c W_up,t^T + mu_t.
 *   Source: "Looped Latent Attention: Cross-Loop KV Compression for Looped
 *   Transformers" (O'Neill & Reid, arXiv 2607.15456), §3 eqs. (1)-(4),
 *   "RoPE and reconstruction", "LLA-2D variant".
 *
 * Conventions shared by every entry point
 *   - bf16 data is passed as raw bfloat16 bit patterns (uint16_t).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Device pointers are the caller's: the library never frees them.  All
 *     launches are asynchronous on `stream`.  Argument errors are detected
 *     on the host before anything is launched, and reported as a status.
 *   - Errors never cross the ABI as exceptions.  Device-side range problems
 *     (a seq_len above max_tokens, a position outside the RoPE table) are
 *     clamped and recorded in a status word inside the workspace, readable
 *     with lla_workspace_flags().
 *   - Device pointers used by the decode kernels must be 16-byte aligned;
 *     otherwise LLA_ERR_ALIGNMENT.
 */
#ifndef LLA_B200_H
#define LLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LLA_OK = 0,
    LLA_ERR_INVALID_ARG = 1,       /* null pointer, negative size, index out of range   */
    LLA_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside what the kernels implement           */
    LLA_ERR_ALIGNMENT = 3,         /* a device pointer is not 16-byte aligned             */
    LLA_ERR_CUDA = 4,              /* a CUDA runtime call or kernel launch failed         */
    LLA_ERR_OOM = 5,               /* device allocation for the codec failed              */
    LLA_ERR_WORKSPACE = 6          /* workspace missing or smaller than required          */
} lla_status;

/* Human-readable text for a status code (static storage). */
const char* lla_status_string(lla_status status);

/* Library version string, e.g. "lla-b200 0.1". */
const char* lla_version(void);

/*
 * Codec description.
 *   D layers, T loops, H heads of width d_head; latent ranks r_k (keys) and
 *   r_v (values) [LLA §3 eq. (2), "asymmetric ranks"].
 *   variant 0 = per-head LLA: one (r_k + r_v) latent per token, layer, head.
 *   variant 1 = LLA-2D: one (r_k + r_v) latent per token and layer decodes all
 *               H heads [LLA §3, "LLA-2D variant"].
 *   rope_base: RoPE base (rotate-half pairs (i, i + d_head/2), frequencies
 *               base^(-2i/d_head)); RoPE is applied after reconstruction
 *               [LLA §3, "RoPE and reconstruction"].
 *   max_pos:   keys and queries may sit at positions [0, max_pos).
 */
typedef struct {
    int D, T, H, d_head, r_k, r_v;
    int variant;
    float rope_base;
    int max_pos;
} lla_codec_desc;

typedef struct lla_codec lla_codec; /* opaque; owns device copies of the codec */

/*
 * lla_create_codec — copy codec matrices (host, float32) to the device.
 *   Per-head (variant 0), with S = T*d_head:
 *     w_down_k [D][H][S][r_k], w_down_v [D][H][S][r_v]      (eq. (2))
 *     w_up_k   [D][H][T][d_head][r_k], w_up_v [.. r_v]       (eq. (3), W_up,t)
 *     mu_k, mu_v [D][H][S]                                   (mu; mu_t = loop slice)
 *   LLA-2D (variant 1), with S2 = T*H*d_head, stacks ordered (loop, head, d):
 *     w_down_k [D][S2][r_k], w_down_v [D][S2][r_v]
 *     w_up_k   [D][T][H][d_head][r_k], w_up_v [.. r_v]
 *     mu_k, mu_v [D][S2]
 *   The device copy keeps W_down as bf16 (an encode GEMM operand), W_up and mu
 *   as float32, b = mu W_down as float32, and RoPE tables built in double
 *   precision.  Returns LLA_ERR_OOM if device memory runs out.  The call
 *   synchronises `stream` before returning.  W_down and W_up are independent
 *   inputs (equal only at SVD initialisation).
 */
lla_status lla_create_codec(lla_codec** out, const lla_codec_desc* desc,
                            const float* w_down_k, const float* w_down_v,
                            const float* w_up_k, const float* w_up_v,
                            const float* mu_k, const float* mu_v, void* stream);

/* Free the codec's device memory (synchronous).  NULL is accepted. */
lla_status lla_destroy_codec(lla_codec* codec);

/* Copy out the description a codec was created with. */
lla_status lla_codec_get_desc(const lla_codec* codec, lla_codec_desc* out);

/*
 * lla_store_bytes — exact size of a latent store.
 *   Layout (bf16, no padding):
 *     per-head: store[batch][D][max_tokens][H][r_k + r_v]
 *     LLA-2D:   store[batch][D][max_tokens][r_k + r_v]
 *   Within a token's (head's) row the K latent (r_k) precedes the V latent
 *   (r_v).  Size = batch*D*max_tokens*(r_k+r_v)*H*2 bytes (per-head) or
 *   without H (2D), so the compression ratio of eq. (4) holds exactly.
 *   Returns 0 for an invalid description or negative sizes.
 */
size_t lla_store_bytes(const lla_codec_desc* desc, int batch, int max_tokens);

/*
 * lla_encode — write latents c = (x - mu) W_down into the store [LLA §3 eq. (2)].
 *   x         device bf16, per-head: [n][num_layers][H][2][S] (axis 0 = K, 1 = V);
 *             LLA-2D: [n][num_layers][2][S2].  Row i is the loop stack of
 *             token i for layers layer_begin .. layer_begin+num_layers-1.
 *   seq_idx, tok_idx  device int32 [n]: destination sequence and token slot
 *             of row i (0 <= seq_idx < batch, 0 <= tok_idx < max_tokens; rows
 *             out of range are skipped and flagged in *nothing*: they are
 *             simply not written).
 *   store     device bf16 latent store (layout of lla_store_bytes).
 *   Accumulation is float32 from bf16 operands; the result is rounded to
 *   bf16 (round-to-nearest-even).
 */
lla_status lla_encode(const lla_codec* codec, const uint16_t* x, int n,
                      int layer_begin, int num_layers,
                      const int32_t* seq_idx, const int32_t* tok_idx,
                      uint16_t* store, int batch, int max_tokens, void* stream);

/*
 * lla_decode_workspace_bytes — device scratch the decode calls need for a
 * given batch (split partials, query-side operands, status word).  Depends on
 * the codec and batch, and on max_tokens only through the split count.
 */
size_t lla_decode_workspace_bytes(const lla_codec* codec, int batch, int max_tokens);

/*
 * lla_decode_attn — per-head LLA decode attention for one (layer, loop) call.
 *   For every sequence b and head h, with n = seq_lens[b] cached tokens
 *   (token j at RoPE position j) and the query at position q_pos[b]:
 *     k_hat_j = c^K_j W^K_up,t^T + mu^K_t,   v_hat_j = c^V_j W^V_up,t^T + mu^V_t
 *     s_j = softmax_scale * <RoPE_{q_pos}(q_bh), RoPE_j(k_hat_j)>
 *     out_bh = sum_j softmax(s)_j v_hat_j          (zero when n == 0)
 *   [LLA §3 eq. (3), "RoPE and reconstruction"].  The V side is summed in
 *   latent space, (sum_j p_j c^V_j) W^V_up,t^T + mu^V_t, which is exact since
 *   the normalised p_j sum to one.
 *   store     device bf16 [batch][D][max_tokens][H][r_k + r_v]
 *   q         device float32 [batch][H][d_head], before RoPE
 *   q_pos     device int32 [batch]; seq_lens device int32 [batch] (<= max_tokens)
 *   out       device float32 [batch][H][d_head]
 *   workspace device, >= lla_decode_workspace_bytes(codec, batch, max_tokens),
 *             16-byte aligned; the library owns its contents during the call.
 *             They need no initialisation and carry nothing from one call to
 *             the next (only the status word is read afterwards).
 *   Concurrent calls must use distinct workspaces.
 */
lla_status lla_decode_attn(const lla_codec* codec, const uint16_t* store, int batch,
                           int max_tokens, int layer, int loop, const float* q,
                           const int32_t* q_pos, const int32_t* seq_lens,
                           float softmax_scale, float* out, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * lla_decode_attn_2d — LLA-2D decode attention [LLA §3, "LLA-2D variant"].
 *   Same arguments as lla_decode_attn; the codec must have variant 1 and the
 *   store is [batch][D][max_tokens][r_k + r_v]: one latent per token decodes
 *   all H heads through per-(loop, head) up-projections.  On the tcgen05
 *   kernel the latent-space V sum is a tensor-core GEMM whose attention
 *   weights are bf16 (the softmax denominator sums the same rounded weights).
 */
lla_status lla_decode_attn_2d(const lla_codec* codec, const uint16_t* store, int batch,
                              int max_tokens, int layer, int loop, const float* q,
                              const int32_t* q_pos, const int32_t* seq_lens,
                              float softmax_scale, float* out, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Kernel selection for tests and measurements.
 *   impl: 0 = best available, 1 = CUDA-core reference kernel (no tensor
 *         cores), 2 = tcgen05/TMA kernel (LLA_ERR_UNSUPPORTED_SHAPE when the
 *         shape is outside it).
 *   num_ctas: 0 = automatic; otherwise the number of context splits (impl 1)
 *         or persistent CTAs (impl 2).  Results do not depend on it beyond
 *         float32 rounding.
 *   ev_begin, ev_end: optional cudaEvent_t handles (NULL = none), recorded on
 *         `stream` immediately before and after the main attention kernel,
 *         so a caller can time that kernel alone (the query prologue and the
 *         split-combine launch fall outside the pair).
 */
typedef struct {
    int impl;
    int num_ctas;
    void* ev_begin;
    void* ev_end;
} lla_decode_opts;

lla_status lla_decode_attn_ex(const lla_codec* codec, const uint16_t* store, int batch,
                              int max_tokens, int layer, int loop, const float* q,
                              const int32_t* q_pos, const int32_t* seq_lens,
                              float softmax_scale, float* out, void* workspace,
                              size_t workspace_bytes, const lla_decode_opts* opts,
                              void* stream);

/*
 * Paged latent stores.  A pool of pages, each holding LLA_PAGE_TOKENS consecutive
 * tokens of one sequence for every layer:
 *   per-head: pool[num_pages][D][LLA_PAGE_TOKENS][H][r_k + r_v]
 *   LLA-2D:   pool[num_pages][D][LLA_PAGE_TOKENS][r_k + r_v]
 * and a block table, device int32 [batch][max_pages]: token j of sequence b
 * lives in pool page block_table[b][j / LLA_PAGE_TOKENS], slot
 * j % LLA_PAGE_TOKENS.  A sequence's logical capacity is
 * max_pages * LLA_PAGE_TOKENS tokens; its pages need not be contiguous or in
 * order, and entries past its length are not read.  The method is unchanged
 * [LLA §3 eqs. (2)-(3)]: only where a latent row is kept differs (serving
 * systems page their caches; the paper's store is the contiguous layout).
 */
#define LLA_PAGE_TOKENS 128

/* Bytes of a pool of num_pages pages (0 for an invalid description). */
size_t lla_paged_store_bytes(const lla_codec_desc* desc, int num_pages);

/*
 * lla_encode_paged — lla_encode into a paged store.  Rows whose sequence,
 *   token (>= max_pages * LLA_PAGE_TOKENS) or page index (outside
 *   [0, num_pages)) is out of range are not written.
 *   pool        device bf16, lla_paged_store_bytes(desc, num_pages) bytes
 *   block_table device int32 [batch][max_pages]
 */
lla_status lla_encode_paged(const lla_codec* codec, const uint16_t* x, int n,
                            int layer_begin, int num_layers,
                            const int32_t* seq_idx, const int32_t* tok_idx,
                            uint16_t* pool, int num_pages, const int32_t* block_table,
                            int max_pages, int batch, void* stream);

/*
 * lla_decode_attn_paged — decode attention (either codec variant) over a paged
 *   store, with an optional self slot (k_self and v_self both NULL: none; see
 *   lla_decode_attn_self).  Results equal those of the contiguous store
 *   holding the same rows.  seq_lens[b] <= max_pages * LLA_PAGE_TOKENS; a
 *   block-table entry outside [0, num_pages) among a sequence's pages cuts the
 *   sequence before that page and sets LLA_FLAG_PAGE_INVALID (4) in the
 *   workspace status.  The workspace is sized by
 *   lla_decode_workspace_bytes(codec, batch, max_pages * LLA_PAGE_TOKENS).
 */
lla_status lla_decode_attn_paged(const lla_codec* codec, const uint16_t* pool, int num_pages,
                                 const int32_t* block_table, int max_pages, int batch,
                                 int layer, int loop, const float* q, const int32_t* q_pos,
                                 const int32_t* seq_lens, const float* k_self,
                                 const float* v_self, float softmax_scale, float* out,
                                 void* workspace, size_t workspace_bytes,
                                 const lla_decode_opts* opts, void* stream);

/*
 * Comparator: decode attention over a full (uncompressed) K/V cache, the
 * "fast path" that keeps every cached token's loop-t key and value themselves
 * [LLA summary, "Serving Capacity"; LLA §3, "Teacher cache"].  Not part of
 * LLA; it is here so that both paths can be timed on the same GPU where the
 * full cache fits.
 *   s_j = softmax_scale * <RoPE_{q_pos}(q_bh), k_bhj>,  out_bh = sum_j softmax(s)_j v_bhj
 *   with keys cached already rotated at their positions (zero when n == 0).
 *   k_cache, v_cache  device bf16, head-major: sequence b's head h, token j at
 *             element b * seq_stride + (h * max_tokens + j) * d_head (seq_stride >=
 *             H*max_tokens*d_head, a multiple of 8: a slice of a larger
 *             [batch][layers][loops][...] cache)
 *   q, q_pos, seq_lens, out, workspace  as lla_decode_attn (no codec: H, d_head
 *             and rope_base are given); d_head must be 128.
 *   num_ctas  0 = one persistent CTA per SM; otherwise that many.
 */
size_t lla_full_decode_workspace_bytes(int H, int d_head, int batch);
lla_status lla_full_decode_attn(int H, int d_head, float rope_base, const uint16_t* k_cache,
                                const uint16_t* v_cache, long long seq_stride, int batch,
                                int max_tokens, const float* q, const int32_t* q_pos,
                                const int32_t* seq_lens, float softmax_scale, float* out,
                                void* workspace, size_t workspace_bytes, int num_ctas,
                                void* stream);

/*
 * lla_reconstruct_cache — the fast path's cache: rebuild the loop-t keys and values of every
 *   cached token once from the latent store and keep them [LLA summary, "Serving Capacity"],
 *   for one (layer, loop):
 *     k_hat_j = RoPE_j(c^K_j W^K_up,t^T + mu^K_t),   v_hat_j = c^V_j W^V_up,t^T + mu^V_t
 *   [LLA §3 eq. (3); RoPE after reconstruction, "RoPE and reconstruction"], rounded to bf16
 *   (nearest-even), written in the layout lla_full_decode_attn reads (keys already rotated).
 *   Either codec variant (2D: head h reconstructs from the token's one latent).
 *   store      device bf16 latent store (layout of lla_store_bytes), 16-byte aligned
 *   seq_lens   device int32 [batch]: tokens j < min(seq_lens[b], max_tokens) are written; the
 *              other rows of the cache are left as they are
 *   k_cache, v_cache  device bf16, 16-byte aligned: sequence b's head h, token j at element
 *              b * seq_stride + (h * cache_tokens + j) * d_head; seq_stride a multiple of 8,
 *              >= H * cache_tokens * d_head; cache_tokens >= max_tokens
 *   impl       0 = best available, 1 = CUDA-core kernel (any shape), 2 = tcgen05 kernel
 *              (d_head 128 with r_k/r_v 16/32 or 96/160 per head, or 64/128 for LLA-2D; it
 *              multiplies by a bf16 copy of W_up, the CUDA-core kernel by the fp32 one)
 *   Requires max_tokens <= the codec's max_pos (positions of the RoPE table); otherwise
 *   LLA_ERR_INVALID_ARG.  Asynchronous on `stream`.
 */
lla_status lla_reconstruct_cache(const lla_codec* codec, const uint16_t* store, int batch, int max_tokens,
                                 int layer, int loop, const int32_t* seq_lens, uint16_t* k_cache,
                                 uint16_t* v_cache, long long seq_stride, int cache_tokens, int impl,
                                 void* stream);

/*
 * lla_decode_attn_self — decode attention with the current token as a self slot
 *   [LLA §3 eq. (2)-(3)]: a token's latent is written only after its last loop
 *   (eq. (2) encodes the whole loop stack), so while it is being decoded its
 *   own loop-t key and value are the loop's exact vectors.  They join the
 *   softmax as one more slot at the query's position:
 *     out_bh = sum over the n cached tokens and the self slot of
 *              softmax(s)_j v_j,  s_self = softmax_scale * <q_bh, k_self_bh>
 *   (query and self key share one rotation, which cancels in the product).
 *   Arguments as lla_decode_attn (either codec variant: per-head or 2D store),
 *   plus
 *   k_self    device float32 [batch][H][d_head], the current token's loop-t
 *             key before RoPE, 16-byte aligned
 *   v_self    device float32 [batch][H][d_head], its loop-t value
 *   opts      as lla_decode_attn_ex, or NULL.
 *   With n == 0 the output is v_self.  Errors as lla_decode_attn; a NULL
 *   k_self or v_self with batch > 0 is LLA_ERR_INVALID_ARG.
 */
lla_status lla_decode_attn_self(const lla_codec* codec, const uint16_t* store, int batch,
                                int max_tokens, int layer, int loop, const float* q,
                                const int32_t* q_pos, const int32_t* seq_lens,
                                const float* k_self, const float* v_self,
                                float softmax_scale, float* out, void* workspace,
                                size_t workspace_bytes, const lla_decode_opts* opts,
                                void* stream);

/*
 * Codec fit on the GPU — the SVD initialisation of W_down [LLA §3,
 * "Initialisation and conversion"]: for each of `problems` independent
 * (layer, head, axis) slots, the calibration stacks X (n x S; S = T*d_head,
 * or T*H*d_head for the 2D variant) are centred with their mean and W_down is
 * the top-r right singular vectors of X - mu, each column flipped so that its
 * entry of largest magnitude is positive.  The loop-t up-projection is then
 * the loop-t row slice of W_down, and mu_t the loop-t slice of mu.
 *   Computed in fp64: the Gram matrix of the smaller side, subspace iteration
 *   with a block of min(n, S, max(2r, r+16)) columns orthonormalised by shifted
 *   CholeskyQR3, then Rayleigh-Ritz with cyclic Jacobi rotations.  The
 *   singular values and the fitted subspace converge with the iteration count
 *   (24 by default; ~1e-8 relative on smooth low-rank-plus-noise stacks).
 *   X        device float32 [problems][n][S]
 *   mu       device float32 [problems][S] (out)
 *   w_down   device float32 [problems][S][r] (out)
 *   sigma    device float32 [problems][r] (out, the top singular values), or NULL
 *   iters    subspace iterations; 0 selects the default (24)
 *   workspace  device, 16-byte aligned, >= lla_fit_codec_workspace_bytes() bytes;
 *            its first word is a status word (lla_workspace_flags): bit 3 (8)
 *            means a Cholesky pivot was not positive (a rank-deficient block;
 *            the result is then not reliable).
 * Requires 1 <= r <= min(n, S) (else LLA_ERR_INVALID_ARG) and a block of at
 * most 1024 columns with min(n, S) <= 32768 and problems <= 65535 (else
 * LLA_ERR_UNSUPPORTED_SHAPE).
 * lla_fit_codec_workspace_bytes returns 0 for arguments lla_fit_codec rejects.
 */
size_t lla_fit_codec_workspace_bytes(int problems, int n, int S, int r);
lla_status lla_fit_codec(int problems, int n, int S, int r, const float* X, float* mu, float* w_down,
                         float* sigma, int iters, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * lla_workspace_flags — read the device status word of a decode workspace
 * (synchronises `stream`).  Bit 0: a seq_len was above max_tokens (clamped);
 * bit 1: a key or query position was outside [0, max_pos) (clamped).  The
 * word is cleared at the start of every decode call.
 */
lla_status lla_workspace_flags(const void* workspace, uint32_t* flags, void* stream);

/*
 * lla_decode_attn_noalloc — lla_decode_attn (or its LLA-2D form, chosen by
 * the codec's variant) for callers that cannot allocate device memory.
 *   The paper has no counterpart: this is a deployment convenience.  Some
 *   hosts may not call cudaMalloc once they are running (the call can stall
 *   every stream of the device), or have handed all device memory to their
 *   own pool; they can pass inputs and outputs but not a workspace.  This
 *   entry point runs the CUDA-core decode kernel and its split-combine with
 *   their scratch in an 8 MiB array compiled into the library, which every
 *   GPU that loads the library holds until the process exits.  It calls no
 *   allocator of any kind.
 *   Limit: the scratch of one call is a 256-byte header plus the split records,
 *   batch x splits x H x (r_v + 2) floats, where splits is the automatic
 *   split count: ceil(4 x SMs / (batch x H)), at least 1 and at most
 *   ceil(max_tokens / 128).  A call whose scratch exceeds 8 MiB is rejected
 *   with LLA_ERR_WORKSPACE before anything is launched.  Once batch x H
 *   reaches 4 x SMs (592 on a 148-SM B200) splits is 1, so with H 16 and
 *   r_v 32 (2176 bytes per sequence) batches up to 3854 fit; the per-head
 *   workload with batch 768 needs about 1.6 MiB.
 *   The first call on each device looks up the array's device address (with
 *   that device current) and caches it; make that first call before any
 *   stream capture.  cudaDeviceReset on a device after a call here leaves the
 *   cached address stale: this entry point must not be used on that device
 *   again in the same process.
 *   All calls on a device share the one array and it keeps the last call's
 *   contents: the status word is cleared at the start of each call, the
 *   split records are rewritten.  Calls that overlap on the GPU (different
 *   streams, or different host threads without ordering) race on it.
 *   The status word is not readable by the caller (the array has no address
 *   the caller can pass to lla_workspace_flags): a seq_len above max_tokens
 *   or a position outside [0, max_pos) is clamped as in lla_decode_attn, but
 *   silently.  Callers that need the flags use lla_decode_attn.
 *   Arguments and results are those of lla_decode_attn without the
 *   workspace.
 */
lla_status lla_decode_attn_noalloc(const lla_codec* codec, const uint16_t* store, int batch,
                                   int max_tokens, int layer, int loop, const float* q,
                                   const int32_t* q_pos, const int32_t* seq_lens,
                                   float softmax_scale, float* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LLA_B200_H */
