/*
 * bd_attn.h -- C ABI of the B200 (sm_100a) block-diffusion attention library
 * (libbdattn.so).
 *
 * Two operations, both exact masked softmax attention with a natural-log
 * log-sum-exp side output:
 *
 *   bd_attn_fwd     training / prefill form over the sequence [x_t ; x_0].
 *   bd_attn_decode  block-decode form: a block of b noisy queries over a
 *                   clean KV cache plus the block itself.
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers owned by the caller, contiguous
 *     row-major, 16-byte aligned.  bf16 tensors are IEEE bfloat16 bit patterns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and return right after the launch.  They never synchronise the
 *     host, never allocate (except bd_attn_decode with workspace == NULL, see
 *     there) and never free.
 *   - No exception or abort crosses the ABI: every error is a bd_status.
 *     Argument errors are detected on the host before anything is launched;
 *     nothing is written to any output in that case.
 *   - Grouped-query attention: q-head h reads kv-head h / (Hq / Hkv).
 *   - lse is ln( sum over visible keys of exp(scale * q.k) ).
 */
#ifndef BD_ATTN_H
#define BD_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *` */

#if defined(__GNUC__)
#define BD_API __attribute__((visibility("default")))
#else
#define BD_API
#endif

typedef enum {
    BD_OK = 0,
    BD_ERR_INVALID_ARG = 1,     /* null/misaligned pointer, bad size or mode */
    BD_ERR_UNSUPPORTED = 2,     /* valid request this build does not handle */
    BD_ERR_CUDA = 3,            /* a CUDA runtime/driver call failed */
    BD_ERR_DEVICE_TIMEOUT = 4   /* a bounded device wait ran out, a
                                   device-side range check failed, or two
                                   launches shared a work counter pair */
} bd_status;

/*
 * Training / prefill block-diffusion attention.
 *
 * Defines: the three-part mask of "Nemotron-Labs-Diffusion-8B-Base 3x decoding
 * speed-up" (doido.pw), section 1 "Block Diffusion Attention" -- block
 * diagonal M_BD, offset block-causal M_OBC, block-causal M_BC -- read with the
 * BDLM objective of "LLaDA2.0-Uni" (discuss.pytorch.kr), section "Training
 * objective and loss function", eq. L_BDLM, which predicts x_{0,k} from
 * x_{0,<k} and x_{t,k} with K = L_total / L_B blocks.
 *
 * Each (batch, head) slice is a sequence of N = 2L rows: rows 0..L-1 are the
 * noisy tokens x_t, rows L..2L-1 the clean tokens x_0, each half cut into L/b
 * blocks of b rows.  A noisy row of block k sees the noisy rows of block k
 * (bidirectionally) and the clean rows of blocks < k; a clean row of block k
 * sees the clean rows of blocks <= k; no row sees a noisy row of another
 * block, and clean rows see no noisy row.
 *
 *   q    [B, Hq,  2L, d] bf16      (read)
 *   k, v [B, Hkv, 2L, d] bf16      (read)
 *   out  [B, Hq,  2L, d] bf16      (written: softmax(scale q k^T) v, rounded
 *                                   to nearest even)
 *   lse  [B, Hq,  2L]    fp32      (written)
 *   scale: softmax scale applied to q.k (typically 1/sqrt(d)); finite, > 0.
 *
 * Errors: BD_ERR_INVALID_ARG for a null or non-16-byte-aligned pointer, any
 * size <= 0, Hq % Hkv != 0, L % b != 0, or a non-finite/non-positive scale;
 * BD_ERR_UNSUPPORTED for d not in {32, 64, 128}; BD_ERR_CUDA if the launch
 * fails.
 *
 * Kernels: every head dim runs on the tcgen05 / TMA kernels (d = 64 and 32
 * on tiles read zero-extended to 128 columns).
 *
 * Concurrency: the launch is one persistent CTA per SM that takes
 * its work items from one of 64 counter pairs in device memory, chosen
 * round-robin when the call is made (and so fixed inside a captured CUDA
 * graph) and reset by the launch's last CTA.  Launches sharing a pair must
 * not overlap in time: keep fewer than 64 calls in flight per device, and do
 * not run two replays of one captured graph at the same time.  Each CTA
 * counts itself into the pair before its first fetch; a count beyond the
 * launch's own CTAs means such an overlap, and the device status word then
 * records BD_ERR_DEVICE_TIMEOUT (the outputs of the overlapping launches are
 * unreliable).
 */
BD_API bd_status bd_attn_fwd(const void *q, const void *k, const void *v, void *out,
                      float *lse, int B, int Hq, int Hkv, int L, int b, int d,
                      float scale, struct CUstream_st *stream);

/*
 * Backward of the training / prefill block-diffusion attention.
 *
 * Defines: the gradient that the BDLM training objective of "LLaDA2.0-Uni"
 * (discuss.pytorch.kr), section "Training objective and loss function", eq.
 * L_BDLM, sends through the attention of bd_attn_fwd (same mask, same
 * layouts).  For every visible (query i, key j) pair of one head, with
 * P_ij = exp(scale q_i.k_j - lse_i) and D_i = dout_i . out_i:
 *     dv_j = sum_i P_ij dout_i,
 *     dS_ij = P_ij (dout_i . v_j - D_i),
 *     dq_i = scale sum_j dS_ij k_j,   dk_j = scale sum_i dS_ij q_i;
 * the q-heads of a GQA group add into their kv-head's dk and dv.  The lse
 * side output of the forward is treated as a constant (no gradient into it).
 *
 *   q, out, dout [B, Hq,  2L, d] bf16   (read; out and lse as written by
 *   lse          [B, Hq,  2L]    fp32    bd_attn_fwd for these q, k, v)
 *   k, v         [B, Hkv, 2L, d] bf16   (read)
 *   dq           [B, Hq,  2L, d] bf16   (written)
 *   dk, dv       [B, Hkv, 2L, d] bf16   (written)
 *   workspace    DEVICE scratch of bd_attn_bwd_workspace_bytes(B, Hq, L)
 *                bytes, 256-byte aligned (per-row D and lse * log2 e)
 *
 * Three kernels on `stream`: a per-row pass, a dK/dV pass over key tiles and
 * a dQ pass over query tiles; nothing is allocated and no atomics are used,
 * so results are deterministic.  Concurrency as for bd_attn_fwd (each pass
 * takes one of the 64 scheduling counter pairs).
 *
 * Errors: as bd_attn_fwd, plus BD_ERR_INVALID_ARG for a null or misaligned
 * workspace or one smaller than required; BD_ERR_UNSUPPORTED for d != 128.
 */
BD_API bd_status bd_attn_bwd(const void *q, const void *k, const void *v,
                             const void *out, const float *lse,
                             const void *dout, void *dq, void *dk, void *dv,
                             int B, int Hq, int Hkv, int L, int b, int d,
                             float scale, struct CUstream_st *stream,
                             void *workspace, size_t workspace_bytes);

/* Bytes of scratch bd_attn_bwd needs (0 on bad sizes).  Host only. */
BD_API size_t bd_attn_bwd_workspace_bytes(int B, int Hq, int L);

/*
 * Block-decode block-diffusion attention.
 *
 * Defines: a block of b noisy queries attends to the cached clean prefix and
 * to its own block, bidirectionally while denoising a draft and causally when
 * verifying it against the same cache: "Nemotron-Labs-Diffusion-8B-Base 3x
 * decoding speed-up", section 2 "Linear Speculative Decoding";
 * "Nemotron-Labs-Diffusion-VLM-8B", section "Multi-mode decoding";
 * "Nemotron-Labs-Diffusion-3B", section "What it is" (guess a run of tokens
 * and check them in the same cache memory).
 *
 * The caller has already written the block's own K/V into the caches at
 * positions cache_len[i] .. cache_len[i]+b-1; cache_len counts the clean
 * prefix only.  Block row j of sequence i sees cache positions
 * 0 .. cache_len[i]-1 and block positions cache_len[i]+j' for every j' < b
 * (intra_block_mode 0, bidirectional denoise) or every j' <= j
 * (intra_block_mode 1, causal verify).  intra_block_mode 2 is cross-attention
 * only: the b rows are the canvas of an encoder-decoder model and see the
 * encoder's cache positions 0 .. cache_len[i]-1 and nothing of themselves
 * ("DiffusionGemma" pipeline page of the diffusers docs, introduction and
 * pipeline class description: a bidirectional decoder cross-attends to the
 * KV cache a causal encoder wrote, to denoise a canvas of canvas_length
 * tokens); with cache_len[i] = 0 such rows see nothing and get out = 0,
 * lse = -inf.  Softmax scale is 1/sqrt(d).
 *
 *   q_blk            [B, Hq, b, d]        bf16 (read)
 *   k_cache, v_cache [B, Hkv, S_cap, d]   bf16 (read; rows beyond
 *                                               cache_len[i]+b never read)
 *   cache_len        [B] int32, DEVICE memory (read on the device only, so
 *                    the call never waits for the host and can be captured in
 *                    a CUDA graph)
 *   out              [B, Hq, b, d]        bf16 (written)
 *   lse              [B, Hq, b]           fp32 (written)
 *   S_cap            row capacity of the caches (>= b in modes 0 and 1)
 *   workspace        device scratch of at least
 *                    bd_attn_decode_workspace_bytes(B, Hq, Hkv, b, d, S_cap)
 *                    bytes (19.6 MB, the same for every size: the partial
 *                    results of at most two cut units per persistent CTA),
 *                    256-byte aligned; its contents on entry do not matter.
 *                    NULL makes the library use an internal buffer of the
 *                    current device, allocated by the first such call (so
 *                    that call must not be inside a stream capture) and
 *                    never freed, so graphs captured with it stay valid.
 *                    Every NULL-workspace call on a device shares that
 *                    buffer: calls whose kernels may overlap on the GPU (two
 *                    streams without ordering between them) race on it and
 *                    give wrong results -- order them, or
 *                    pass each stream its own workspace.
 *
 * Errors: BD_ERR_INVALID_ARG for a null or misaligned pointer, any size <= 0,
 * Hq % Hkv != 0, S_cap < b in modes 0 and 1, intra_block_mode not 0/1/2, or
 * a workspace smaller than required; BD_ERR_UNSUPPORTED for d not in {32,
 * 64, 128}; BD_ERR_CUDA if the launch (or the internal workspace allocation)
 * fails.  A cache_len[i] outside [0, S_cap - b] (modes 0 and 1) or [0, S_cap]
 * (mode 2) is caught on the device: that sequence's rows are written as NaN
 * with lse NaN, and the device status word (see bd_attn_get_device_status)
 * records BD_ERR_DEVICE_TIMEOUT.
 */
BD_API bd_status bd_attn_decode(const void *q_blk, const void *k_cache,
                         const void *v_cache, const int32_t *cache_len,
                         void *out, float *lse, int B, int Hq, int Hkv, int b,
                         int d, int intra_block_mode,
                         struct CUstream_st *stream, int S_cap,
                         void *workspace, size_t workspace_bytes);

/* Size of the fixed scratch array bd_attn_decode_noalloc works in. */
#define BD_ATTN_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * Block decode that never allocates device memory (no counterpart on the
 * source pages; it exists for callers that cannot allocate).
 *
 * Some callers cannot call cudaMalloc at the point where they decode: a
 * serving loop whose device memory is owned entirely by another allocator
 * (a framework's caching allocator, a fixed memory budget), code running
 * inside a stream capture where allocation is not allowed, or real-time code
 * that forbids allocation after start-up.  This call computes exactly what
 * bd_attn_decode computes, with the same arguments, layouts and errors, but
 * takes no workspace: its scratch (bd_attn_decode_workspace_bytes, 19.6 MB
 * for every size) lives in a fixed array of BD_ATTN_NOALLOC_SCRATCH_BYTES
 * bytes compiled into the library's device code.  Every GPU on which the
 * library's kernels are loaded holds that array until the process exits.
 *
 * - The first call on a device looks up the array's device address (with
 *   that device current) and caches it; make that first call before any
 *   stream capture.
 * - The array holds the scratch of every size (checked when the library is
 *   built); a size whose scratch exceeded it would be rejected with
 *   BD_ERR_UNSUPPORTED before anything is launched.
 * - All calls share the one array and it keeps whatever the last call left
 *   there; nothing in it needs to start at zero.  Calls whose kernels overlap
 *   on the GPU (for example on two streams without ordering between them)
 *   race on the array and give wrong results: order them on one stream or
 *   with events.
 * - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
BD_API bd_status bd_attn_decode_noalloc(const void *q_blk, const void *k_cache,
                                        const void *v_cache,
                                        const int32_t *cache_len, void *out,
                                        float *lse, int B, int Hq, int Hkv,
                                        int b, int d, int intra_block_mode,
                                        struct CUstream_st *stream, int S_cap);

/*
 * Speculative decoding: accepted prefix length.
 *
 * Defines: "Nemotron-Labs-Diffusion-8B-Base 3x decoding speed-up", section 2
 * "Linear Speculative Decoding": a block drafted with bidirectional attention
 * is validated with causal attention and its longest matching prefix is
 * accepted.
 *
 *   draft, target  [B, b] int32 tokens, DEVICE memory (read): the drafted
 *                  block and the verifier's token for each block position
 *   n_accept       [B] int32, DEVICE memory (written): the length of the
 *                  longest prefix j = 0 .. n-1 with draft[i][j] == target[i][j]
 *
 * Errors: BD_ERR_INVALID_ARG for a null or non-4-byte-aligned pointer or a
 * size <= 0; BD_ERR_CUDA if the launch fails.
 */
BD_API bd_status bd_spec_accept(const int32_t *draft, const int32_t *target,
                                int32_t *n_accept, int B, int b,
                                struct CUstream_st *stream);

/*
 * Append accepted rows to the KV cache and advance its length, on the device.
 *
 * Defines: the "update the KV cache" step of linear speculative decoding,
 * "Nemotron-Labs-Diffusion-8B-Base 3x decoding speed-up", section 2.
 *
 *   k_cache, v_cache  [B, Hkv, S_cap, d] bf16 (read and written in place)
 *   cache_len         [B] int32, DEVICE memory (read, then advanced by
 *                     n_new[i])
 *   k_new, v_new      [B, Hkv, b, d] bf16 (read): the block's K/V; rows
 *                     0 .. n_new[i]-1 are copied to cache positions
 *                     cache_len[i] .. cache_len[i]+n_new[i]-1.  Both NULL:
 *                     the rows are already there (the usual case: the block's
 *                     K/V were written at the cache tail before the causal
 *                     verification), so only the length advances.
 *   n_new             [B] int32, DEVICE memory (read), e.g. from
 *                     bd_spec_accept
 *
 * Nothing is allocated; the call can be captured in a CUDA graph.  A
 * sequence with n_new[i] outside [0, b] or cache_len[i] + n_new[i] > S_cap is
 * left untouched and the device status word records BD_ERR_DEVICE_TIMEOUT.
 * Errors: BD_ERR_INVALID_ARG for a null pointer (k_new and v_new must be both
 * NULL or both set), a misaligned pointer or a size <= 0;
 * BD_ERR_UNSUPPORTED for d not in {32, 64, 128}; BD_ERR_CUDA if the launch
 * fails.
 */
BD_API bd_status bd_cache_append(void *k_cache, void *v_cache, int32_t *cache_len,
                                 const void *k_new, const void *v_new,
                                 const int32_t *n_new, int B, int Hkv, int b,
                                 int d, int S_cap, struct CUstream_st *stream);

/*
 * Crop the KV cache to at most max_len positions: cache_len[i] =
 * min(cache_len[i], max_len), on the device (the cache rows stay where they
 * are).  Defines: "Nemotron-Labs-Diffusion-8B-Base 3x decoding speed-up",
 * section "KV cache strategy" (the cache is cropped to a maximum length
 * during generation).  cache_len: [B] int32 in DEVICE memory.
 * Errors: BD_ERR_INVALID_ARG for a null or misaligned pointer, B <= 0 or
 * max_len < 0; BD_ERR_CUDA if the launch fails.
 */
BD_API bd_status bd_cache_crop(int32_t *cache_len, int B, int max_len,
                               struct CUstream_st *stream);

/*
 * Sparse prefix retention (SPRINT): prune the cached prefix once at the start
 * of a block.
 *
 * Defines: "LLaDA2.0-Uni" (discuss.pytorch.kr), section "SPRINT: training-free
 * inference acceleration", paragraph "Sparse Prefix Retention".  Each prefix
 * position p < cache_len[i] gets the score
 *     s_p = alpha * I_p + (1 - alpha) * conf[i][p],
 *     I_p = |k_p|_2 / mean over the prefix of |k_j|_2,
 * where |k_p|_2 is the norm of position p's key over all kv-heads and dims
 * of this cache (0 for all p if that mean is 0), and conf is the caller's
 * top-1 softmax confidence.  Each modality (modality[i][p] == 0: text, else
 * image) with n prefix positions keeps floor(r * n + 1/2) of them, r =
 * keep_text or keep_image: those with the highest score, ties to the lower
 * position.  The page uses alpha = 0.5, keep_image = 0.8, keep_text = 1.0.
 * The kept positions, in their original order, become the new prefix.
 * Scores are computed in double precision.
 *
 *   k_cache, v_cache  [B, Hkv, S_cap, d] bf16 (read)
 *   cache_len         [B] int32, DEVICE (read)
 *   conf              [B, S_cap] fp32, DEVICE (read; entries < cache_len[i])
 *   modality          [B, S_cap] uint8, DEVICE (read; entries < cache_len[i])
 *   k_out, v_out      [B, Hkv, S_cap, d] bf16 (written: rows 0 ..
 *                     new_len[i]-1 are the kept rows; later rows untouched).
 *                     Must not overlap the input caches.
 *   kept              [B, S_cap] int32, DEVICE (written: kept positions in
 *                     increasing order, then -1)
 *   new_len           [B] int32, DEVICE (written; the prefix length to pass to
 *                     bd_attn_decode as cache_len afterwards)
 *   score             [B, S_cap] fp64, DEVICE (written for p < cache_len[i])
 *                     or NULL
 *   workspace         DEVICE scratch of bd_sprint_workspace_bytes(B, S_cap)
 *                     bytes, 256-byte aligned
 *
 * Errors: BD_ERR_INVALID_ARG for a null (other than score) or misaligned
 * pointer, a size <= 0, alpha or a keep ratio outside [0, 1], aliasing
 * outputs, or a short workspace; BD_ERR_UNSUPPORTED for d not in {32, 64,
 * 128} or S_cap > 65536; BD_ERR_CUDA if a launch fails.  A cache_len[i]
 * outside [0, S_cap] gives new_len[i] = 0 and records BD_ERR_DEVICE_TIMEOUT
 * in the device status word.
 */
BD_API bd_status bd_sprint_prune(const void *k_cache, const void *v_cache,
                                 const int32_t *cache_len, const float *conf,
                                 const uint8_t *modality, float alpha,
                                 float keep_text, float keep_image,
                                 void *k_out, void *v_out, int32_t *kept,
                                 int32_t *new_len, double *score, int B,
                                 int Hkv, int d, int S_cap,
                                 struct CUstream_st *stream, void *workspace,
                                 size_t workspace_bytes);

/* Bytes of scratch bd_sprint_prune needs (0 on bad sizes).  Host only. */
BD_API size_t bd_sprint_workspace_bytes(int B, int S_cap);

/* Bytes of scratch bd_attn_decode needs for these sizes (0 on bad sizes).
 * Pure host arithmetic; needs no GPU. */
BD_API size_t bd_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int b, int d,
                                      int S_cap);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: BD_OK, or BD_ERR_DEVICE_TIMEOUT if a kernel gave up a
 * bounded wait, rejected a device-resident size, or found its work counter
 * pair in use by another launch since the last call;
 * BD_ERR_CUDA if the synchronisation itself failed. */
BD_API bd_status bd_attn_get_device_status(struct CUstream_st *stream);

/* Static, NUL-terminated description of a status code. */
BD_API const char *bd_attn_status_string(bd_status status);

#ifdef __cplusplus
}
#endif

#endif /* BD_ATTN_H */
