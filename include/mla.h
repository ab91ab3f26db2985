/*
 * mla.h -- C ABI of a decode-time Multi-head Latent Attention (MLA) library
 * for NVIDIA B200 (sm_100a).
 *
 * What is computed (the method's equations):
 *   "DeepSeek-V3 Technical Report" reading note (dogely.com), MLA section:
 *     c^KV_t = W^DKV h_t,  k^R_t = RoPE(W^KR h_t),  k_{t,i} = [W^UK_i c^KV_t ; k^R_t],
 *     v_{t,i} = W^UV_i c^KV_t,
 *     o_{t,i} = sum_{j<=t} Softmax_j(q_{t,i}^T k_{j,i} / sqrt(d_h + d_h^R)) v_{j,i},
 *     u_t = W^O [o_{t,1}; ...; o_{t,n_h}].
 *   "DeepSeek-V2: Strong, Economical, Efficient" (translation), §2.1.2-§2.1.3
 *     (only [c^KV_t ; k^R_t] is cached: d_c + d_h^R elements per token per layer)
 *     and Appendix C (W^UK is absorbed into the query and W^UV into the output
 *     side, so attention runs on the cached rows directly).
 *
 * The decode step is five calls, all asynchronous on the caller's stream:
 *   mla_cache_append    write [c^KV ; k^R] rows for new tokens
 *   mla_absorb_q        q_abs_i = [W^UK_i^T q^C_i ; RoPE(q^R_i, pos)]
 *   mla_decode_attn     split-KV softmax over the latent rows -> partials
 *   mla_combine_splits  log-sum-exp merge of the partials -> ctx_lat
 *   mla_out_proj        o_i = W^UV_i ctx_lat_i  (and optionally u = W^O o)
 * and, ahead of mla_absorb_q when the caller starts from the hidden state,
 *   mla_query_proj      q^C, q^R (unrotated) from h, with or without W^DQ
 *
 * Conventions for every call
 *   - Tensor pointers are DEVICE memory owned by the caller, row-major and
 *     contiguous, element type = cfg.dtype (bf16 or fp32), unless stated.
 *     Integer tensors (positions, lengths, block tables) are device int32.
 *   - Weights are row-major [out_features, in_features]:
 *       W_DKV [d_c, d_model]     W_KR [d_r, d_model]
 *       W_UK, W_UV [n_h*d_h, d_c] (rows i*d_h .. i*d_h+d_h-1 belong to head i)
 *       W_O [d_model, n_h*d_h]
 *   - The latent cache row of a token is D = d_c + d_r elements [c^KV | k^R].
 *     Contiguous cache (cfg.page_size == 0): cache = [B, cache_len, D], where
 *       cache_len is the per-sequence capacity in tokens; block_table = NULL.
 *     Paged cache (cfg.page_size > 0): cache = pool [cache_len, page_size, D],
 *       cache_len = number of blocks in the pool; block_table = [B,
 *       max_blocks_per_seq] int32 block ids; token p of sequence b lives in block
 *       block_table[b*max_blocks_per_seq + p/page_size], row p%page_size.
 *   - RoPE rotates consecutive pairs (x_2k, x_2k+1) of the d_r-wide rotary part
 *     by angle pos*theta_k, theta_k = rope_base^(-2k/d_r) (RoFormer form; the
 *     angle keeps double-precision accuracy: formed in double on the CUDA
 *     cores; in the tensor-core GEMMs as the exact product pos*theta_hi plus
 *     pos*theta_lo for a float pair theta_hi + theta_lo = theta_k, reduced by
 *     2 pi in three parts before the sine and cosine).
 *   - Host-side argument checks return an error before anything is launched.
 *     Checks that need device data (positions, lengths, block ids beyond the
 *     table or pool) are made in the kernels: an offending access is skipped
 *     and a flag is set in the handle's status word, which
 *     mla_get_device_status() reports.  Every device-side wait is bounded; a
 *     wait that runs out sets MLA_ERR_TIMEOUT in the same word.
 *   - The library allocates device memory only in mla_create (the handle's
 *     status word and RoPE table).  The decode calls use the caller's workspace
 *     (mla_decode_attn_combine_noalloc uses a fixed array in the device image
 *     instead; see its declaration).
 *   - A sequence with ctx_len = 0 produces a zero ctx_lat row and lse = -inf.
 *   - Results are deterministic for a fixed num_parts (no floating-point atomics).
 *   - A handle may be used from one host thread at a time.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Identical to cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *mla_stream_t;

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,   /* a host-checked argument is out of range or NULL */
  MLA_ERR_UNSUPPORTED = 2,   /* shape or dtype this build has no kernel for */
  MLA_ERR_WORKSPACE = 3,     /* workspace pointer NULL, misaligned or too small */
  MLA_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
  MLA_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out */
  MLA_ERR_DEVICE_BOUNDS = 6  /* a device-side index check failed (access skipped) */
} mla_status;

typedef enum { MLA_BF16 = 0, MLA_FP32 = 1 } mla_dtype;

typedef struct {
  int n_h;          /* attention heads */
  int d_h;          /* per-head width of q^C / v */
  int d_c;          /* KV compression width (latent c^KV) */
  int d_r;          /* decoupled RoPE width d_h^R (even) */
  int d_model;      /* model width d */
  int page_size;    /* 0 = contiguous cache; else tokens per block (64 for the fast paths) */
  double rope_base; /* RoPE base, e.g. 10000 */
  int dtype;        /* mla_dtype: storage and input type of every tensor */
} mla_config;

typedef struct mla_handle mla_handle;

/* Human-readable name of a status code.  Never NULL. */
const char *mla_status_string(int status);

/* Host-only check of a configuration (no CUDA calls): MLA_OK,
 * MLA_ERR_INVALID_ARG (non-positive or odd d_r, NULL) or MLA_ERR_UNSUPPORTED. */
int mla_config_validate(const mla_config *cfg);

/* Create a handle on the current CUDA device.  Allocates the status word and
 * the RoPE frequency table (theta_k in double precision), and looks up the
 * device address of the scratch array that mla_decode_attn_combine_noalloc
 * uses (that lookup loads the part of the library's device image holding the
 * array, which is when the array's memory is reserved on this device).  On
 * failure *out is NULL.  Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
int mla_create(const mla_config *cfg, mla_handle **out);

/* Release a handle (synchronises nothing; the caller must not have work in
 * flight that uses it).  NULL is accepted. */
void mla_destroy(mla_handle *handle);

/* Long-context scaling of the rotary part (YaRN): V2 §3.2.4 extends the 4K
 * window to 128K with YaRN on the decoupled key k^R only, s = 40, alpha = 1,
 * beta = 32, and a length-scaling factor sqrt(t) = c ln s + 1 (c = 0.0707 in
 * the V2 paper, 0.1 in the V3 note's context-extension section).
 *   factor        s >= 1 (1 turns the scaling off: plain RoPE, t = 1)
 *   original_ctx  the window the frequencies were trained on (> 0)
 *   alpha, beta   0 <= alpha < beta: a rotary pair that turns more than beta
 *                 times over original_ctx keeps its frequency, one that turns
 *                 fewer than alpha times is slowed by s, linear in between
 *   mscale_coef   c >= 0; every score (content and rotary part) is multiplied
 *                 by t = (c ln s + 1)^2, i.e. sqrt(t) scales query and key
 * Replaces the handle's frequency table (synchronously, on the handle's
 * device) and its score scale; applies to the calls made afterwards on this
 * handle (mla_cache_append, mla_absorb_q, mla_decode_attn).  Rows already in
 * a cache were rotated with the previous table, so set the scaling before
 * filling the cache.  Errors: INVALID_ARG (NULL handle, bad values, wrong
 * current device), CUDA. */
int mla_set_rope_scaling(mla_handle *handle, double factor, int original_ctx, double alpha,
                         double beta, double mscale_coef);

/* Strict tensor-core mode (off by default).  A bf16 configuration of the
 * DeepSeek-V2 attention shapes runs its append, absorption, attention, output
 * projection and query projection on tcgen05 kernels; when one of those
 * kernels cannot take a call's arguments (a pointer that is not 16-byte
 * aligned, a cache of 2^31 rows or more, a tensor map the driver rejects) the
 * call normally runs the CUDA-core kernel instead, with the same results.
 * With strict mode on, such a call returns MLA_ERR_UNSUPPORTED before
 * launching anything.  Calls for which the configuration has no tensor-core
 * kernel at all (fp32, other shapes, the FP8 cache at 128 heads) are not
 * affected.  Meant for tests and benchmarks that must run the tensor-core
 * path.  Errors: INVALID_ARG (NULL handle). */
int mla_set_strict(mla_handle *handle, int strict);

/* Cache append (V3 note, MLA equations: c^KV_t = W^DKV h_t, k^R_t = RoPE(W^KR h_t);
 * V2 §2.1.3: the cached row is [c^KV_t ; k^R_t]).
 *   h          [B, T, d_model] hidden states of T new tokens per sequence
 *   start_pos  device int32 [B]: token t of sequence b is written at position
 *              start_pos[b] + t and rotated by that position
 *   w_dkv      [d_c, d_model], w_kr [d_r, d_model]
 *   cache, cache_len, block_table, max_blocks_per_seq: see the conventions above
 * Positions outside the cache (or unmapped blocks) are skipped and flagged
 * MLA_ERR_DEVICE_BOUNDS.  T may be large (bulk fill) or 1 (decode step). */
int mla_cache_append(mla_handle *handle, const void *h, int B, int T, const int *start_pos,
                     const void *w_dkv, const void *w_kr, void *cache, long long cache_len,
                     const int *block_table, int max_blocks_per_seq, mla_stream_t stream);

/* Query projection of the current token, before absorption (V2 §2.1.2 query
 * compression, c^Q_t = W^DQ h_t, q^C_t = W^UQ c^Q_t; §2.1.3 q^R_t = W^QR c^Q_t,
 * rotated later by mla_absorb_q; Appendix B: V2-Lite has no query compression,
 * q^C_t = W^Q h_t and q^R_t = W^QR h_t):
 *   x      [B, d_model] hidden state of each sequence's new token
 *   w_dq   [d_cq, d_model] (W^DQ), or NULL for the uncompressed form
 *   d_cq   query compression width d_c' (ignored when w_dq is NULL)
 *   w_uq   [n_h*d_h, d_cq] (W^UQ), or W^Q [n_h*d_h, d_model] when w_dq is NULL
 *   w_qr   [n_h*d_r, d_cq], or [n_h*d_r, d_model] when w_dq is NULL
 *   c_q    [B, d_cq] (out) the compressed query, or NULL when w_dq is NULL
 *   q_nope [B, n_h, d_h] (out), q_rope [B, n_h, d_r] (out, not yet rotated):
 *          the inputs mla_absorb_q takes.
 * No normalisation is applied to c^Q.  Every product accumulates in fp32; c_q
 * is stored in cfg.dtype and the up-projections read that stored value. */
int mla_query_proj(mla_handle *handle, const void *x, int B, const void *w_dq, int d_cq,
                   const void *w_uq, const void *w_qr, void *c_q, void *q_nope, void *q_rope,
                   mla_stream_t stream);

/* Query absorption (V2 Appendix C; V3 note q_{t,i} = [q^C_{t,i} ; q^R_{t,i}]):
 *   q_abs[b,i,:d_c]  = W^UK_i^T q_nope[b,i,:]        (W^UK_i = rows i*d_h.. of W^UK)
 *   q_abs[b,i,d_c:]  = RoPE(q_rope[b,i,:], pos[b])
 *   q_nope [B, n_h, d_h], q_rope [B, n_h, d_r] (before rotation), pos device int32 [B]
 *   (the query's own position, normally ctx_len-1), q_abs [B, n_h, d_c+d_r]. */
int mla_absorb_q(mla_handle *handle, const void *q_nope, const void *q_rope, const int *pos,
                 const void *w_uk, void *q_abs, int B, mla_stream_t stream);

/* Bytes of workspace mla_decode_attn/mla_combine_splits need for batch B with
 * num_parts work partitions (0 = the default for this handle's kernel).
 * Returns 0 on invalid arguments. */
size_t mla_decode_workspace_size(const mla_handle *handle, int B, int num_parts);

/* Default number of work partitions for this handle (depends on the kernel
 * selected for the configuration and on the device's SM count); 0 for a NULL
 * handle. */
int mla_default_num_parts(const mla_handle *handle);

/* Split-KV decode attention over the latent cache (V3 note: o_{t,i} with the
 * softmax over j = 1..t, scale 1/sqrt(d_h + d_r); absorbed form of V2 App. C).
 * The batch's KV tokens, in tiles of mla_plan_tile(handle, 0) tokens (the
 * attention kernel's own tile: 256, 128 or 64), are cut into num_parts equal
 * shares;
 * each share is processed by one worker (one CTA, or one CTA pair for 128
 * heads) and yields, per (sequence, share) piece, the normalised partial
 * ctx_lat and its log-sum-exp, written into the workspace.
 *   q_abs   [B, n_h, d_c+d_r] absorbed queries
 *   ctx_len device int32 [B], ctx_len[b] tokens of sequence b are attended.
 *           A length below 0 or above what the cache can address for one
 *           sequence (cache_len for a contiguous cache, max_blocks_per_seq *
 *           page_size for a paged one) sets MLA_ERR_DEVICE_BOUNDS in the status
 *           word and is clamped to that range, for the split plan and for the
 *           attention alike.
 *   workspace >= mla_decode_workspace_size(handle, B, num_parts) bytes, 256-byte
 *   aligned, device memory; its contents are overwritten. */
int mla_decode_attn(mla_handle *handle, const void *q_abs, const void *cache, long long cache_len,
                    const int *block_table, int max_blocks_per_seq, const int *ctx_len, int B,
                    int num_parts, void *workspace, size_t ws_bytes, mla_stream_t stream);

/* Decode attention over a token range of each sequence: tokens
 * ctx_begin[b] .. ctx_len[b]-1 of sequence b instead of 0 .. ctx_len[b]-1;
 * otherwise as mla_decode_attn (same workspace, same partials, merged by
 * mla_combine_splits or mla_combine_splits_f32).  This is the per-device step
 * of split-KV across devices for long contexts: each device holds and attends
 * one token range of every sequence, and the per-range results are merged
 * with mla_merge_ranges (the "DeepSeek-V3" note's decode deployment runs
 * attention data-parallel with sequence parallelism; the merge is the
 * log-sum-exp algebra of the split combine).
 *   ctx_begin device int32 [B]; each value a multiple of 64 in [0, ctx_len[b]].
 *             Other values set MLA_ERR_DEVICE_BOUNDS in the status word and are
 *             clamped into that range and rounded down to a multiple of 64.
 *   With a paged cache the block table needs entries only for the blocks of
 *   the range (the others may be -1): a device's pool can hold just its range.
 * Errors as mla_decode_attn; INVALID_ARG for a NULL ctx_begin. */
int mla_decode_attn_range(mla_handle *handle, const void *q_abs, const void *cache, long long cache_len,
                          const int *block_table, int max_blocks_per_seq, const int *ctx_begin,
                          const int *ctx_len, int B, int num_parts, void *workspace, size_t ws_bytes,
                          mla_stream_t stream);

/* Merge the partials of the preceding mla_decode_attn on the same workspace:
 * m = max_s lse_s, ctx_lat = sum_s e^(lse_s - m) O_s / sum_s e^(lse_s - m),
 * lse = m + log sum_s e^(lse_s - m).
 *   ctx_lat [B, n_h, d_c] (cfg.dtype), lse [B, n_h] float32 or NULL.
 * B and num_parts must equal those given to mla_decode_attn. */
int mla_combine_splits(mla_handle *handle, const void *workspace, size_t ws_bytes, int B,
                       int num_parts, void *ctx_lat, float *lse, mla_stream_t stream);

/* The same merge written in float32 whatever cfg.dtype: ctx_lat [B, n_h, d_c]
 * float32 and lse [B, n_h] float32 (not NULL), the per-range result that
 * devices exchange before mla_merge_ranges. */
int mla_combine_splits_f32(mla_handle *handle, const void *workspace, size_t ws_bytes, int B,
                           int num_parts, float *ctx_lat, float *lse, mla_stream_t stream);

/* Merge the results of R token ranges of the same B sequences (split-KV across
 * devices), in range order, with the combine's algebra: per (b, i),
 * m = max_r lse_r, ctx_lat = sum_r e^(lse_r - m) ctx_r / sum_r e^(lse_r - m),
 * lse = m + log sum_r e^(lse_r - m); a range with lse = -inf (no tokens)
 * carries no weight, and if every range is empty the row is zero with
 * lse = -inf.
 *   ctx_parts [R, B, n_h, d_c] float32, lse_parts [R, B, n_h] float32 (device)
 *   ctx_lat [B, n_h, d_c] (cfg.dtype), lse [B, n_h] float32 or NULL.
 * Errors: INVALID_ARG (NULL pointers, R <= 0 with B > 0), CUDA. */
int mla_merge_ranges(mla_handle *handle, const float *ctx_parts, const float *lse_parts, int R, int B,
                     void *ctx_lat, float *lse, mla_stream_t stream);

/* Output projection (V2 App. C, W^UV absorbed to the output side; V3 note u_t):
 *   o[b,i,:] = W^UV_i ctx_lat[b,i,:]      o [B, n_h, d_h]
 *   if w_o != NULL: u[b,:] = W^O o[b,:,:] (flattened)   u [B, d_model]
 * w_uv [n_h*d_h, d_c], w_o [d_model, n_h*d_h] or NULL (then u is ignored). */
int mla_out_proj(mla_handle *handle, const void *ctx_lat, const void *w_uv, const void *w_o,
                 void *o, void *u, int B, mla_stream_t stream);

/* mla_combine_splits followed by mla_out_proj as one step: the partials of
 * the preceding mla_decode_attn on the same workspace are merged inside the
 * output projection (the log-sum-exp algebra of mla_combine_splits, then
 * o[b,i,:] = W^UV_i ctx_lat[b,i,:], V2 App. C), so the merged latents do not
 * make a round trip through device memory.
 *   w_uv [n_h*d_h, d_c]; o [B, n_h, d_h]; w_o / u as mla_out_proj.
 *   ctx_lat [B, n_h, d_c] (cfg.dtype) or NULL: when given it receives the
 *   merged latents, the same values mla_combine_splits writes; lse [B, n_h]
 *   float32 or NULL likewise.
 * B and num_parts must equal those given to mla_decode_attn.  The merged
 * latents enter the projection rounded to cfg.dtype, as with the two calls.
 * bf16 with d_h a multiple of 128 and d_c a multiple of 128 up to 512 runs one
 * tcgen05 kernel; other shapes run a CUDA-core kernel (refused under strict
 * mode where the tensor-core kernel exists but cannot take the arguments).
 * Errors: INVALID_ARG (NULL handle, w_uv or o; w_o without u; negative B or
 * num_parts), WORKSPACE, UNSUPPORTED, CUDA. */
int mla_combine_out_proj(mla_handle *handle, const void *workspace, size_t ws_bytes, int B, int num_parts,
                         const void *w_uv, const void *w_o, void *o, void *u, void *ctx_lat, float *lse,
                         mla_stream_t stream);

/* Self-test of the device-side time-out path: launches one wait on a barrier
 * that nothing completes, which gives up after limit_ns nanoseconds (1e3 ..
 * 1e9) and sets the time-out bit in the handle's status word, exactly as a
 * wait in the decode kernels does past its 2 s limit.  The next
 * mla_get_device_status then returns MLA_ERR_TIMEOUT; the context stays
 * usable.  MLA_ERR_INVALID_ARG for a NULL handle or a limit out of range. */
int mla_selftest_wait_timeout(mla_handle *handle, long long limit_ns, mla_stream_t stream);

/* Synchronise `stream`, read and clear the handle's device status word.
 * Returns MLA_OK, MLA_ERR_TIMEOUT, MLA_ERR_DEVICE_BOUNDS or MLA_ERR_CUDA. */
int mla_get_device_status(mla_handle *handle, mla_stream_t stream);

/* Host mirror of the split plan with 64-token tiles, the plan of the CUDA-core
 * kernels (no CUDA calls); mla_plan_pieces_tiled with mla_plan_tile(handle, fp8)
 * mirrors the plan any handle uses.
 *   ctx_len host int32 [B]; num_parts as for mla_decode_attn (must be > 0 here).
 *   piece_base host int64 [B+1] (out): pieces of sequence b are
 *   piece_base[b] .. piece_base[b+1]-1.  Returns the total number of pieces,
 *   or -1 on invalid arguments. */
long long mla_plan_pieces(const int *ctx_len, int B, int num_parts, long long *piece_base);

/* The same plan with tiles of tile_tokens tokens (a multiple of 64):
 * sequence b contributes ceil(ctx_len[b] / tile_tokens) tiles, and the batch's
 * tiles are cut into num_parts equal shares.  mla_plan_pieces is this with 64.
 * Returns -1 on invalid arguments. */
long long mla_plan_pieces_tiled(const int *ctx_len, int B, int num_parts, int tile_tokens, long long *piece_base);

/* Tokens per tile of the split plan mla_decode_attn (fp8 = 0) or
 * mla_decode_attn_fp8 (fp8 = 1) uses with this handle: the MMA tile of the
 * attention kernel it runs (256 for 128 heads in bf16, 128 for 16 or 32
 * heads, 64 on the CUDA cores), so that a share pays for no partial tile
 * inside a sequence.  -1 for a NULL handle. */
int mla_plan_tile(const mla_handle *handle, int fp8);

/* Allocation-free variant of mla_decode_attn followed by mla_combine_splits.
 * The pages have no counterpart: this entry point exists for callers that
 * cannot allocate device memory where attention runs (code inside an
 * allocator or memory-pool callback, runtimes that forbid cudaMalloc after
 * start-up, embeddings that only lend the library buffers they already own).
 * Instead of a caller workspace, the split partials live in one fixed scratch
 * array of mla_noalloc_scratch_bytes() bytes (32 MiB) inside the library's
 * device image; every GPU that loads the library holds it until exit.
 *   Arguments as for mla_decode_attn, plus ctx_lat [B, n_h, d_c] (cfg.dtype)
 *   and lse [B, n_h] float32 or NULL as for mla_combine_splits.
 *   num_parts = 0 picks the default split count, lowered until the partials
 *   fit the array; an explicit num_parts (or a batch) whose partials do not
 *   fit is rejected with MLA_ERR_WORKSPACE before anything is launched.
 * No cudaMalloc/cudaFree or allocating library call is made.  The array's
 * device address is looked up once, by mla_create on the handle's device
 * (cudaGetSymbolAddress with that device current); that lookup is also what
 * loads the array onto the device, so creating the handle is the step that
 * reserves its memory, and this call itself allocates nothing.  The handle's
 * device must be current.
 * All calls share the array and leave their partials in it; calls whose work
 * overlaps on the GPU (unordered streams) race on it.  The array needs no
 * zeroing: each call writes everything it reads. */
int mla_decode_attn_combine_noalloc(mla_handle *handle, const void *q_abs, const void *cache,
                                    long long cache_len, const int *block_table,
                                    int max_blocks_per_seq, const int *ctx_len, int B, int num_parts,
                                    void *ctx_lat, float *lse, mla_stream_t stream);

/* Size in bytes of the scratch array mla_decode_attn_combine_noalloc uses. */
size_t mla_noalloc_scratch_bytes(void);

/* ---------------------------------------------------------------------------
 * FP8 latent cache ("DeepSeek-V2" §3.2.3: the deployed KV cache is quantised
 * to about 6 bits per element, format not given; "DeepSeek-V3" note, FP8
 * section: activations are quantised tile-wise, per token and per 128
 * channels, scaled by the group's absolute maximum).
 *
 * Format.  A token's row of D = d_c + d_r elements [c^KV | k^R] is stored as
 * D one-byte OCP FP8 E4M3 codes, in the same row layout as the cfg.dtype
 * cache (contiguous [B, cache_len, D] or paged [cache_len, page_size, D]).
 * The row is cut into scale groups of 128 channels over c^KV, then over k^R
 * (the last group of each part may be narrower); G = mla_fp8_scale_groups()
 * (5 at d_c = 512, d_r = 64).  kv_scale is float32 [rows, G] with the same
 * row indexing as the codes.  For a group with absolute maximum a (float32):
 * sigma = a / 448 and code = E4M3(x / sigma), both divisions rounded to
 * nearest in float32, the conversion rounding to nearest even and saturating
 * at 448; a group of zeros has sigma = 0 and zero codes.  The stored value is
 * code * sigma.
 * ------------------------------------------------------------------------- */

/* G, the number of scale groups per row (0 for a NULL handle). */
int mla_fp8_scale_groups(const mla_handle *handle);

/* Bytes of workspace mla_cache_append_fp8 needs for B sequences of T new
 * tokens (float32 rows before quantisation); 0 on invalid arguments. */
size_t mla_cache_append_fp8_workspace_size(const mla_handle *handle, int B, int T);

/* mla_cache_append into an FP8 cache: the rows [c^KV ; RoPE(k^R)] are formed
 * in float32 exactly as mla_cache_append forms them, then quantised.
 *   cache       uint8 codes, layout as for mla_cache_append
 *   kv_scale    float32 [rows, G]
 *   workspace   >= mla_cache_append_fp8_workspace_size(handle, B, T) bytes of
 *               device memory, 256-byte aligned; overwritten.
 * Other arguments and errors as for mla_cache_append; MLA_ERR_WORKSPACE for a
 * missing, misaligned or short workspace. */
int mla_cache_append_fp8(mla_handle *handle, const void *h, int B, int T, const int *start_pos,
                         const void *w_dkv, const void *w_kr, void *cache, float *kv_scale,
                         long long cache_len, const int *block_table, int max_blocks_per_seq,
                         void *workspace, size_t ws_bytes, mla_stream_t stream);

/* Quantise n_rows rows [n_rows, D] (cfg.dtype; e.g. rows of an existing
 * cache) into codes [n_rows, D] (uint8) and kv_scale [n_rows, G], row i to
 * row i.  Rows are independent, so a contiguous cache converts in one call
 * and a paged pool by passing the whole pool as rows. */
int mla_quantize_rows_fp8(mla_handle *handle, const void *rows, long long n_rows, void *codes,
                          float *kv_scale, mla_stream_t stream);

/* mla_decode_attn over an FP8 cache (codes and kv_scale as above).  The
 * partials, the workspace and mla_combine_splits are those of
 * mla_decode_attn.  16 or 32 heads at d_c = 512, d_r = 64 run on the tensor
 * cores (the codes are widened to bf16 in shared memory, code * sigma rounded
 * to bf16); every other shape, 128 heads included, on the CUDA-core kernel,
 * which is functional but hundreds of times slower than the bf16 tensor-core
 * path at DeepSeek-V2 shapes.  kv_scale NULL is MLA_ERR_INVALID_ARG. */
int mla_decode_attn_fp8(mla_handle *handle, const void *q_abs, const void *cache, const float *kv_scale,
                        long long cache_len, const int *block_table, int max_blocks_per_seq,
                        const int *ctx_len, int B, int num_parts, void *workspace, size_t ws_bytes,
                        mla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
