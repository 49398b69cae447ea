/*
 * head_attention_streaming_b200 — C ABI of the fused attention forward for
 * NVIDIA B200 (sm_100a).
 *
 * The library computes, per batch b, query head hq and query row i,
 *
 *     O[b,i,hq,:] = sum_j softmax_j( scale * Q[b,i,hq,:] . K[b,j,hkv,:] ) V[b,j,hkv,:]
 *
 * over the keys j visible to row i. This is the per-head scaled dot-product
 * attention of the flashdreams.accelerated developer guide ("Optimized Multi
 * Head Attention" -> "Multi Head Attention Definition", the equation for A_h),
 * with the scale given explicitly (1/sqrt(d) there), for the token-major
 * [batch, seq, heads, head_dim] layout that page and the FlashAttention-4
 * runtime page ("FLASH4.md", H3 call layout) use.
 *
 * All functions are plain C. Pointers named "device" must point to CUDA device
 * memory of the current device; the library allocates no device memory and
 * owns no buffer. Every function returns an attn_status_t value (as int).
 */
#ifndef HEAD_ATTENTION_STREAMING_B200_ATTN_H_
#define HEAD_ATTENTION_STREAMING_B200_ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,   /* an argument breaks the contract below; nothing was launched */
  ATTN_ERR_UNSUPPORTED = 2,   /* valid by the pages' contract but not built (head_dim, device) */
  ATTN_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (launch, descriptor encode) */
  ATTN_ERR_TIMEOUT = 4,       /* a device-side wait ran past its limit (see attn_device_fault) */
  ATTN_ERR_SCRATCH_LIMIT = 5  /* the request needs more than the library's fixed-size scratch
                                 (attn_fwd_splitkv_static); nothing was launched */
} attn_status_t;

typedef enum { ATTN_DTYPE_BF16 = 0, ATTN_DTYPE_FP16 = 1 } attn_dtype_t;

typedef enum {
  ATTN_MASK_NONE = 0,    /* every key visible (cross-attention, full self-attention) */
  ATTN_MASK_CAUSAL = 1,  /* key j visible to row i iff j <= kv_offset + i */
  ATTN_MASK_CHUNK = 2    /* streaming chunk: key j visible iff j < kv_offset + Lq */
} attn_mask_t;

/*
 * attn_fwd — fused attention forward, asynchronous on `stream`.
 *
 * Operation: scaled dot-product attention (developer guide, "Multi Head
 * Attention Definition"); grouped K/V heads as in the skill page
 * "optimizing-attention-flash", "Workflow 2" Step 3 (multi-query attention),
 * with query head hq reading K/V head hq / (Hq / Hkv); the causal flag of the
 * same page's flash-attn call; and the streaming self-attention step of the
 * developer guide's "Generic Multi Head Attention Interface" and the user
 * guide's "Cache lifecycle", where the current chunk's K/V are already in the
 * rolling cache when the chunk is queried and the chunk attends to the whole
 * visible cache.
 *
 * Arguments (all tensors contiguous, row-major, 16-byte aligned base):
 *   q    device, [B, Lq, Hq, d]  of dtype            (read)
 *   k    device, [B, Lk, Hkv, d] of dtype            (read)
 *   v    device, [B, Lk, Hkv, d] of dtype            (read)
 *   o    device, [B, Lq, Hq, d]  of dtype            (written; must not overlap q, k, v)
 *   lse  device, [B, Hq, Lq] float32, natural log of sum_j exp(scale * s_ij)
 *        over visible keys; may be NULL (then not written)
 *   B, Lq, Lk, Hq, Hkv  >= 1, Hq % Hkv == 0
 *   d    head_dim, a power of two 16..256 (the pages' range): 16 and 32 run
 *        through the 64-wide kernel (its TMA boxes read the columns past d as
 *        zero and store only d columns); 256 runs one 128-row query tile per
 *        work unit (its tensor memory holds S twice and O once)
 *   scale  finite, >= 0 (1/sqrt(d) in the pages)
 *   causal attn_mask_t: 0 none, 1 causal, 2 streaming chunk
 *   kv_offset  cache position of query row 0: 0 for mask 0; for masks 1 and 2,
 *        0 <= kv_offset and kv_offset + Lq <= Lk (a causal call with
 *        kv_offset = Lk - Lq aligns the diagonal bottom-right)
 *   dtype  attn_dtype_t, the element type of q, k, v and o
 *   stream cudaStream_t (NULL = legacy default stream)
 *
 * Errors: every argument is checked before any CUDA call; a violation returns
 * ATTN_ERR_INVALID_ARG (or ATTN_ERR_UNSUPPORTED for a head_dim or device this
 * build does not run) and launches nothing. There is no fallback to another
 * kernel or to the CPU. A failed launch returns ATTN_ERR_CUDA. The call does
 * not synchronize; a device-side timeout is reported by attn_device_fault.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int Lq, int Lk, int Hq, int Hkv, int d, float scale,
             int causal, int kv_offset, int dtype, void* stream);

/*
 * attn_fwd_window — attn_fwd with a sliding window (local attention): query
 * row i, at key position p = kv_offset + i, sees keys p - window_left <= j <=
 * p + window_right; -1 leaves that side unbounded (skill page
 * "optimizing-attention-flash", "Sliding window attention": flash-attn's
 * window_size=(left, right)). (-1, 0) is causal, (-1, -1) is no mask. KV tiles
 * outside every row's window are neither loaded nor multiplied.
 * Arguments as attn_fwd with 0 <= kv_offset, kv_offset + Lq <= Lk, and
 * window_left, window_right >= -1 (so every row sees its own position).
 */
int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Lq,
                    int Lk, int Hq, int Hkv, int d, float scale, int window_left, int window_right,
                    int kv_offset, int dtype, void* stream);

/*
 * Unscaled FP8 attention (developer guide, "OptimizedImplConfig":
 * quantized_sdpa casts Q, K and V directly to float8_e4m3fn, keeps the K/V
 * cache in that type, and uses FP8 probabilities for the P V product).
 *
 * attn_fp8_cast — y[i] = e4m3(x[i]) for n 16-bit values (dtype), rounded to
 * nearest even and saturated at +-448. n % 8 == 0; x 16-byte and y 8-byte
 * aligned; no overlap. Asynchronous on `stream`.
 *
 * attn_fp8_cast_vt — V [B, Lk, Hkv, d] (16-bit, dtype) to e4m3 transposed:
 * vt[b, h, c, j] = e4m3(v[b, j, h, c]) in [B, Hkv, d, pitch] bytes, pitch >= Lk
 * and a multiple of 16 (bytes j >= Lk of a row are not written); d a power of
 * two 16..256. The transposed layout makes V's tiles the K-major operand of P V.
 *
 * attn_fwd_fp8 — attention forward on e4m3 operands: q8 [B, Lq, Hq, d] and
 * k8 [B, Lk, Hkv, d] e4m3, vt8 as written by attn_fp8_cast_vt (pitch
 * vt_pitch); S = scale q8 k8^T and the softmax in float32; P rounded to e4m3
 * for the P V product (the row sum uses the unrounded P); o [B, Lq, Hq, d]
 * bfloat16 and lse as attn_fwd. Masks, GQA, kv_offset and errors as attn_fwd;
 * d = 16, 32, 64, 128, 256 (below 128 through the 128-wide kernel, whose
 * 128-byte TMA boxes read the columns of Q, K and the rows of V^T past d as
 * zero, with the O chunks past d not stored; 256 through the one-tile kernel).
 */
int attn_fp8_cast(const void* x, void* y, long long n, int dtype, void* stream);
int attn_fp8_cast_vt(const void* v, void* vt, int B, int Lk, int Hkv, int d, int pitch, int dtype,
                     void* stream);
int attn_fwd_fp8(const void* q8, const void* k8, const void* vt8, void* o, float* lse, int B, int Lq,
                 int Lk, int vt_pitch, int Hq, int Hkv, int d, float scale, int causal, int kv_offset,
                 void* stream);

/*
 * Per-token scaled FP8 attention (developer guide, "Quantization Toolkit":
 * slice scales s = max(max |x| / 448, eps) in float32 with eps = 2^-126,
 * codes e4m3(x / s) clipped to +-448; "Quantized GEMM", inner-dimension rule:
 * the scales of each GEMM operand stay constant along its reduction axis).
 *
 * attn_fp8_quantize_tokens — one scale per (batch, token, head) of x
 * [B, L, H, d] (16-bit, dtype): s[b, h, l] at s[(b H + h) s_pitch + l]
 * (float32, s_pitch >= L), codes y [B, L, H, d] e4m3. d a power of two in
 * 16..256; x 16-byte, y 8-byte, s 4-byte aligned; no overlap.
 *
 * attn_fp8_quantize_vt — one scale per (batch, head, channel) of V
 * [B, Lk, Hkv, d] (the max runs over the keys): sv [B, Hkv, d] float32, codes
 * written transposed like attn_fp8_cast_vt ([B, Hkv, d, pitch]). d a power of
 * two in 16..256. Four launches on `stream` (zero sv, column maxima, codes,
 * maxima to scales); sv holds the scales once they complete.
 *
 * attn_fwd_fp8_scaled — attn_fwd_fp8 on scaled codes: the score of row i and
 * key j is scale * sq[b, hq, i] * sk[b, hkv, j] * (q8_i . k8_j) (sq
 * [B, Hq, sq_pitch], sk [B, Hkv, sk_pitch] as attn_fp8_quantize_tokens writes
 * them, sk_pitch a multiple of 4, sk 16-byte aligned), and column c of O is
 * multiplied by sv[b, hkv, c] ([B, Hkv, d], 16-byte aligned; NULL: V cast
 * without scales). P is rounded to e4m3 as in attn_fwd_fp8. Head dims as
 * attn_fwd_fp8.
 */
int attn_fp8_quantize_tokens(const void* x, void* y, float* s, int B, int L, int H, int d, int s_pitch,
                             int dtype, void* stream);
int attn_fp8_quantize_vt(const void* v, void* vt, float* sv, int B, int Lk, int Hkv, int d, int pitch,
                         int dtype, void* stream);
int attn_fwd_fp8_scaled(const void* q8, const void* k8, const void* vt8, const float* sq,
                        const float* sk, const float* sv, void* o, float* lse, int B, int Lq, int Lk,
                        int vt_pitch, int sq_pitch, int sk_pitch, int Hq, int Hkv, int d, float scale,
                        int causal, int kv_offset, void* stream);

/*
 * attn_fwd_cache — attn_fwd with K and V read from the first Lk tokens of a
 * [B, S, Hkv, d] cache (the rolling block cache of streaming self-attention,
 * whose valid tokens are a prefix of its S slots): batch b's keys start at
 * k_cache + b * S * Hkv * d. Lk <= S. Everything else as attn_fwd.
 */
int attn_fwd_cache(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                   int B, int Lq, int Lk, int S, int Hq, int Hkv, int d, float scale, int causal,
                   int kv_offset, int dtype, void* stream);

/*
 * attn_fwd_splitkv — attn_fwd with the visible keys of every query tile split
 * into ranges that different CTAs process at once, then merged: for few query
 * rows over many keys (a short chunk against a long cache), where one CTA per
 * 256-row query pair would leave most SMs idle.
 *
 * Operation: attention over disjoint key ranges, combined exactly through the
 * per-range log-sum-exp: lse = ln sum_g exp(lse_g), O = sum_g exp(lse_g - lse)
 * O_g (the softmax of the developer guide's "Multi Head Attention Definition"
 * with its normaliser summed range by range). All three masks: under the
 * causal mask a query tile takes only the tiles of a range it can see, and a
 * row that sees no key of a range contributes an empty partial (O = 0,
 * lse_g = -inf, weight 0); range 0 always holds key 0, which every row sees.
 * Under masks 1 and 2 the ranges cover keys below kv_offset + Lq only.
 *
 * Arguments as attn_fwd, plus:
 *   n_splits   requested number of key ranges, >= 1, or 0 to choose one from
 *              the shape and the SM count (causal: only while the unsplit
 *              units are fewer than the SMs, since causal units differ in
 *              length and a second wave of them costs more than it saves). Ranges are whole 128-key tiles,
 *              ceil(tiles / n_splits) each, so the count used can be lower than
 *              requested (4 tiles asked for 3 ranges give 2); never an empty range
 *   workspace  device float32 buffer of at least
 *              attn_splitkv_workspace_bytes(B, Lq, Hq, d, n) bytes for the n
 *              ranges used (partial O and LSE), 16-byte aligned, overlapping no
 *              operand; may be NULL when no split happens (n = 1)
 *   splits_used  if not NULL, receives n (written before any launch)
 * With n = 1 the call is attn_fwd. Two launches otherwise (the split forward,
 * then the merge), asynchronous on `stream`. The workspace is the caller's and
 * must not be reused before the call's work on `stream` has completed.
 */
size_t attn_splitkv_workspace_bytes(int B, int Lq, int Hq, int d, int n_splits);
int attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                     float* workspace, size_t workspace_bytes, int n_splits, int B, int Lq, int Lk,
                     int Hq, int Hkv, int d, float scale, int causal, int kv_offset, int dtype,
                     int* splits_used, void* stream);

/*
 * attn_fwd_splitkv_static — attn_fwd_splitkv for callers that cannot allocate
 * device memory: no workspace argument, and the call allocates nothing (no
 * cudaMalloc, no cudaFree, no allocating library routine). It exists for
 * code that is handed only its input and output buffers, such as a plugin
 * slot of a host framework with no workspace argument, or a step loop that
 * must not call cudaMalloc because that call can synchronize the device. The
 * pages describe no counterpart: it is a packaging of attn_fwd_splitkv.
 *
 * Scratch: the float32 partial outputs and LSEs live in one file-scope device
 * array of 64 MB (16 Mi floats) inside this library. Every GPU that loads the
 * library holds those 64 MB until the process exits. The first call on a
 * device looks up the array's device address there (cudaGetSymbolAddress,
 * with that device current) and keeps it; make that first call before any
 * stream capture. Every call shares the one array and overwrites it: calls
 * that overlap on the GPU (two streams, two host threads) race and must be
 * ordered by the caller. Each call writes every partial it reads before
 * reading it, so nothing is cleared between calls.
 *
 * Limit: with n_splits = 0 the split count is chosen as for attn_fwd_splitkv
 * and then lowered until attn_splitkv_workspace_bytes(B, Lq, Hq, d, count)
 * <= 64 MB (down to one range, which runs attn_fwd and needs no scratch). An
 * explicit n_splits > 1 whose partials need more than 64 MB is refused with
 * ATTN_ERR_SCRATCH_LIMIT before anything is launched. *splits_used reports
 * the count used. Other arguments and errors as attn_fwd_splitkv.
 */
int attn_fwd_splitkv_static(const void* q, const void* k, const void* v, void* o, float* lse,
                            int n_splits, int B, int Lq, int Lk, int Hq, int Hkv, int d, float scale,
                            int causal, int kv_offset, int dtype, int* splits_used, void* stream);

/*
 * attn_fwd_host — the same forward for operands in host memory: copies q, k, v
 * from host to the caller's device buffers, runs attn_fwd, and copies o (and
 * lse when both lse pointers are given) back to host memory. The copies
 * overlap the computation: the call is cut into at most 16 chunks with at
 * least 2 MB of q each (attn_host_chunks gives the plan) — whole batches per
 * chunk when there are at least as many batches as chunks, else each batch's
 * query rows in ranges of whole 256-row pairs. Per chunk the k and v of its
 * batches (first chunk of a batch only) and its q rows are copied in, its
 * forward starts once they have landed, and its o (and lse) go back while the
 * next chunk computes. Chunks hold whole work units of attn_fwd and every
 * chunk takes the whole call's choice of schedule, so o and lse are
 * bit-identical to one attn_fwd call. Host-to-device and
 * device-to-host copies run on two streams the library creates once per
 * device; the forwards run on `stream`, which waits for everything before the
 * call returns control of it: synchronize `stream` before reading o_host, and
 * keep every host buffer allocated and unchanged until then (use pinned host
 * memory: pageable memory serializes the copies). Calls on one
 * device are queued one at a time (a per-device lock while queueing).
 * Shapes, dtype, mask and errors as attn_fwd; additionally every host pointer
 * but lse_host must be non-NULL, and lse_host and lse_dev must be both NULL
 * or both non-NULL. Device buffers are owned by the caller and sized as
 * attn_fwd's q, k, v, o, lse; lse_dev is used as scratch (after the call it
 * holds each chunk's [nb, Hq, rows] block at the chunk's place, which is the
 * [B, Hq, Lq] layout of lse_host only when every chunk holds whole batches).
 */
int attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                  float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                  float* lse_dev, int B, int Lq, int Lk, int Hq, int Hkv, int d, float scale,
                  int causal, int kv_offset, int dtype, void* stream);

/*
 * attn_host_chunks — the chunk plan attn_fwd_host uses for a call of these
 * sizes (host logic only, no CUDA call). Writes 4 ints per chunk into plan
 * (room for 16 chunks = 64 ints, caller-owned): first batch b0, batches nb,
 * first query row r0, rows n; chunk c covers rows [r0, r0 + n) of batches
 * [b0, b0 + nb). Returns the number of chunks (1..16), or
 * -ATTN_ERR_INVALID_ARG for a NULL plan or a size below 1.
 */
int attn_host_chunks(int B, int Lq, int Hq, int d, int* plan);

typedef enum {
  ATTN_NORM_NONE = 0,   /* Q and K unchanged */
  ATTN_NORM_HEAD = 1,   /* RMSNorm over each head's d features (m = d) */
  ATTN_NORM_INNER = 2   /* RMSNorm over all H*d features of a token (m = H d) */
} attn_norm_scope_t;

typedef enum {
  ATTN_ROPE_NONE = 0,        /* no rotation */
  ATTN_ROPE_INTERLEAVED = 1, /* pair r = features (2r, 2r + 1) */
  ATTN_ROPE_SPLIT = 2        /* pair r = features (r, r + d/2) */
} attn_rope_style_t;

/*
 * attn_qk_prologue — Q/K RMS normalisation followed by rotary position
 * embedding, for Q and (optionally) the new K chunk in one launch,
 * asynchronous on `stream`.
 *
 * Operation (developer guide, "Multi Head Attention Definition"): for every
 * token, RMSNorm_gamma(z) = gamma * z / sqrt(mean(z^2) + eps) over each head
 * (ATTN_NORM_HEAD) or over the whole token (ATTN_NORM_INNER); then feature
 * pair r of the token at sequence index p is rotated by the angle
 * angles[p * d + a_r], where a_r is the pair's first feature (2r interleaved,
 * r split-half): (z_a, z_b) -> (z_a cos - z_b sin, z_a sin + z_b cos). The
 * page normalises before RoPE; so does this call. Arithmetic in float32 from
 * the 16-bit inputs, one round-to-nearest to dtype at the end. V is not
 * touched.
 *
 * Arguments (tensors contiguous, row-major; 16-bit tensors 16-byte aligned,
 * float arrays 4-byte aligned):
 *   q      device, [B, Lq, Hq, d] of dtype                   (read)
 *   q_out  device, [B, Lq, Hq, d] of dtype (written; may equal q for in place,
 *          must not otherwise overlap any other operand)
 *   k, k_out  as q / q_out with [B, Lk, Hkv, d]; both NULL to process Q only
 *   gamma_q, gamma_k  device float32 weights of length d (head scope) or
 *          Hq*d / Hkv*d (inner scope); NULL means all ones; ignored for
 *          ATTN_NORM_NONE
 *   angles_q, angles_k  device float32 [Lq, d] / [Lk, d]: the expanded angle
 *          table rope_freqs[L, 1, 1, d] of the pages, one angle per feature
 *          (row p is sequence index p of every batch); NULL iff
 *          rope_style == ATTN_ROPE_NONE
 *   d      a power of two, 16..256
 *   norm_scope  attn_norm_scope_t; eps finite, >= 0 (1e-6 in the pages)
 *   rope_style  attn_rope_style_t
 *   dtype  attn_dtype_t of q, q_out, k, k_out
 *
 * Errors: every argument is checked before any CUDA call; a violation returns
 * ATTN_ERR_INVALID_ARG (ATTN_ERR_UNSUPPORTED for another head_dim) and
 * launches nothing. A failed launch returns ATTN_ERR_CUDA. No allocation, no
 * synchronisation.
 */
int attn_qk_prologue(const void* q, void* q_out, const void* k, void* k_out,
                     const float* gamma_q, const float* gamma_k, const float* angles_q,
                     const float* angles_k, int B, int Lq, int Lk, int Hq, int Hkv, int d,
                     int norm_scope, float eps, int rope_style, int dtype, void* stream);

/*
 * attn_stream_update — the K/V cache update of one streaming self-attention
 * step, with the query prologue, in one launch, asynchronous on `stream`.
 *
 * Operation (developer guide, "Generic Multi Head Attention Interface"; user
 * guide, "Cache lifecycle"): the current chunk's K/V are written into the
 * rolling block cache before the chunk is queried, keys with before-cache
 * RoPE already rotated. For every batch b and chunk token i < L:
 *   k_cache[b, slot + i] = RoPE(RMSNorm(k[b, i]))   (as attn_qk_prologue)
 *   v_cache[b, slot + i] = v[b, i]                  (copied; V is never
 *                                                    normalised or rotated)
 *   q_out[b, i]          = RoPE(RMSNorm(q[b, i]))   (when q is given)
 * The angle row of token i is i (the tables hold the chunk's positions).
 *
 * Arguments (16-bit tensors contiguous and 16-byte aligned):
 *   q, q_out  device [B, L, Hq, d] of dtype, or both NULL; q_out may equal q
 *   k, v      device [B, L, Hkv, d] of dtype (read)
 *   k_cache, v_cache  device [B, S, Hkv, d] of dtype; tokens slot .. slot+L-1
 *             of every batch are written, nothing else is touched
 *   gamma_*, angles_*, norm_scope, eps, rope_style, d  as attn_qk_prologue
 *             (angles_q / angles_k: [L, d])
 *   0 <= slot and slot + L <= S
 * Errors as attn_qk_prologue; additionally the caches may overlap no input and
 * not each other. No allocation, no synchronisation.
 */
int attn_stream_update(const void* q, void* q_out, const void* k, const void* v, void* k_cache,
                       void* v_cache, const float* gamma_q, const float* gamma_k,
                       const float* angles_q, const float* angles_k, int B, int L, int S, int slot,
                       int Hq, int Hkv, int d, int norm_scope, float eps, int rope_style, int dtype,
                       void* stream);

/*
 * attn_rope_after_cache — RoPE after the K/V cache update (developer guide,
 * "Multi Head Attention Definition": the cache keeps unrotated keys, and right
 * before attention the current queries and every visible cached key are
 * rotated with the angles of their current positions, again at every step).
 *
 *   q, q_out   device [B, Lq, Hq, d] (16-bit, dtype): queries, rotated with
 *              angle rows q_row0 .. q_row0 + Lq - 1; q_out may be q (in place)
 *   k_cache    device [B, S, Hkv, d]: its first Lk slots are read
 *   k_rot      device [B, S, Hkv, d]: slot s < Lk receives k_cache slot s
 *              rotated with angle row k_rows[s] (device int32 [Lk]; NULL: row
 *              s); other slots are not written
 *   angles     device float32 [n_angle_rows, d], the expanded per-feature
 *              angle table of positions 0 .. n_angle_rows - 1 (the pages'
 *              cache-relative rope_freqs); rows read from k_rows are clamped
 *              to the table
 *   rope_style ATTN_ROPE_INTERLEAVED or ATTN_ROPE_SPLIT; no normalisation
 *              (the cache holds keys already normalised)
 * One launch, asynchronous on `stream`. Errors: arguments checked before any
 * CUDA call (ATTN_ERR_INVALID_ARG; ATTN_ERR_UNSUPPORTED for d outside the
 * powers of two 16..256); k_rot may overlap nothing else.
 */
int attn_rope_after_cache(const void* q, void* q_out, const void* k_cache, void* k_rot,
                          const float* angles, int n_angle_rows, int q_row0, const int* k_rows, int B,
                          int Lq, int Lk, int S, int Hq, int Hkv, int d, int rope_style, int dtype,
                          void* stream);

/* Short English text of a status code (static storage). */
const char* attn_status_string(int status);

/*
 * attn_device_fault — synchronizes the current device, then returns in *bits
 * the device fault word that kernels of this library set when a bounded wait
 * on a shared-memory barrier ran out (0: none). Each bit names the wait that
 * gave up. With clear != 0 the word is reset to 0. Returns ATTN_ERR_TIMEOUT
 * when *bits != 0, else ATTN_OK (or ATTN_ERR_CUDA).
 */
int attn_device_fault(unsigned int* bits, int clear);

/*
 * attn_debug_fault_site — synchronizes the current device, then returns in
 * *site the site number of the first index check that failed in any kernel of
 * this library since the last clear (0: none). Only the debug build
 * (libattn_sm100_debug.so, compiled with -DATTN_DEBUG) checks: there every
 * kernel tests the global-memory rows, shared-memory offsets and TMA
 * coordinates it computes (tensor-memory columns are checked at compile time)
 * against the shapes of the call before using them; a failed check sets
 * bit 11 (0x800) of the fault word (attention kernels), records its site
 * and skips that access, so the launch ends normally with a wrong result. In
 * the release build *site is always 0. With clear != 0 the site words are
 * reset. Returns ATTN_OK, ATTN_ERR_INVALID_ARG for a NULL site, or ATTN_ERR_CUDA.
 * Sites: 1 Q tile coordinates, 2 K/V tile coordinates, 3 O store coordinates,
 * 4 LSE index, 5 key-split partial row, 6 per-token scale rows, 7 V channel
 * scales, 8 O staging row, 9 d = 256 output row, 10 key-split merge columns,
 * 21 prologue token / cache slot, 31-33 FP8 cast and quantizer rows.
 */
int attn_debug_fault_site(unsigned int* site, int clear);

/* 1 in the debug build (-DATTN_DEBUG), 0 in the release build. */
int attn_debug_build(void);

/*
 * attn_set_wait_timeout_ns — limit, in nanoseconds, of every device-side
 * barrier wait in kernels launched after this call (default 4e9). A wait that
 * runs out sets its bit in the fault word, stops its CTA's pipeline, waits
 * briefly for its own copies and MMAs in flight, frees its tensor memory and
 * exits. Values below 1e6 are raised to 1e6.
 */
int attn_set_wait_timeout_ns(unsigned long long ns);

/*
 * Diagnostics, used by the tests to check the building blocks of attn_fwd on
 * the device. None is needed to compute attention.
 *
 * attn_selftest_mma — one 128x128 tile through the same tensor-core path as
 * attn_fwd: TMA loads of q, k, v ([128, 128] row-major, dtype), S = q k^T
 * accumulated in tensor memory and copied to s_out ([128,128] float32), then
 * P = round_dtype(S / 16) written back to tensor memory and O = P v copied to
 * o_out ([128,128] float32). Synchronous.
 *
 * attn_selftest_wait_timeout — launches one CTA that waits on a barrier
 * nothing completes, with the given limit in nanoseconds (1e6..1e10); returns
 * ATTN_ERR_TIMEOUT when the wait gave up as designed (and clears the fault
 * word), ATTN_OK if it did not. Synchronous.
 */
int attn_selftest_mma(const void* q, const void* k, const void* v, float* s_out, float* o_out,
                      int dtype, void* stream);
int attn_selftest_wait_timeout(unsigned long long timeout_ns, void* stream);

/*
 * attn_selftest_exp2 — y[i] = 2^x[i] for i < n (device float32 arrays) through
 * the FMA-pipe exponential attn_fwd uses for part of its softmax exponentials:
 * relative error within 7.6e-5 of 2^x for -125 <= x <= 8 (the softmax's
 * exponent arguments never exceed 8); arguments below -125 give about 2^-125.
 * The same softmax definition as attn_fwd's (developer guide, "Multi Head
 * Attention Definition"); this entry exists to test that arithmetic.
 * Synchronous.
 */
int attn_selftest_exp2(const float* x, float* y, int n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HEAD_ATTENTION_STREAMING_B200_ATTN_H_ */
