/*
 * attn_b200.h -- C ABI of the B200 (sm_100a) exact-attention library, libattn_b200.so.
 *
 * Operations (sources are docs.rs source pages, cited as crate version, file, Rust item):
 *   attn_fwd     exact scaled-dot-product attention O = softmax(Q K^T * scale + mask) V with
 *                the per-row logsumexp, grouped-query head sharing and an optional causal mask.
 *                scirs2-neural 0.4.3 src/layers/flash_attention.rs (flash_attention_forward,
 *                online_softmax_update); scirs2-neural 0.4.4 src/layers/grouped_query_attention.rs
 *                (GroupedQueryAttention::forward_with_cache: head groups, causal mask with a
 *                cache offset).
 *   attn_fwd_ex  attn_fwd with rotary position embedding applied to Q and K first.
 *                scirs2-neural 0.4.4 grouped_query_attention.rs (RotaryPositionEmbedding::apply).
 *   attn_fwd_masked  attn_fwd_ex with an additive score mask.  whisper-apr 0.3.1
 *                attention_generated.rs (compute_block_scores, scaled_dot_product_attention).
 *   attn_decode  one query token per (sequence, q head) against a KV cache, split along the keys
 *                and merged by logsumexp.  oxibonsai-model 0.1.4 src/layers/flash_decode.rs
 *                (flash_decode_tile, combine_tile_outputs, flash_decode_single_head);
 *                whisper-apr 0.3.1 src/model/lfm2/gqa.rs (attention_cached).
 *   rope_apply   the rotation alone, in place.  RotaryPositionEmbedding::apply as above.
 *   attn_bwd     gradients of the forward wrt q, k, v.  flash_attention.rs (flash_backward_head);
 *                grouped_query_attention.rs (backward).
 *   attn_kv_append  decode-step cache append with the new keys and queries rotated at their
 *                positions.  grouped_query_attention.rs (forward_with_cache); whisper-apr KvCache.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers (CUDA global memory), row-major and contiguous in
 *     the layouts stated below, 16-byte aligned.  The caller owns every buffer; the library
 *     allocates no memory on these paths.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     No call synchronises the device.  Arguments are validated on the host before any launch;
 *     an invalid call returns an error status and launches nothing.
 *   - ATTN_ERR_CUDA means a launch or driver call failed; the CUDA error is left for the caller's
 *     next cudaGetLastError() / synchronisation to report as well.
 *   - Kernels never trap.  Device-side anomalies (a bounded wait that gave up, a decode length
 *     outside [1, Smax]) set bits in a device status word read by attn_read_device_status().
 *   - Softmax semantics: s_ij = scale * <q_i, k_j>; with `causal`, key j is masked for query
 *     row i when j > i + (Skv - Sq) (bottom-right alignment: the last query row sees every key).
 *     lse_i = ln sum_j exp(s_ij) over unmasked keys (natural log, scaled scores).  A row with no
 *     unmasked key gets o_i = 0 and lse_i = -inf.
 *   - GQA: q head h reads kv head h / (Hq / Hkv); Hq must be a multiple of Hkv (Hkv == Hq is
 *     multi-head, Hkv == 1 is multi-query attention).
 *   - Head dims: D in {64, 128} run natively.  attn_fwd_ex and attn_bwd also take any other
 *     even D < 128: q, k, v (and dout) are zero-padded to 64 or 128 in the
 *     workspace (zero dims add nothing to q.k; the scale is the caller's, so no correction is
 *     needed; RoPE keeps the frequencies of D) and the outputs are copied back without the
 *     padding.  whisper-apr 0.3.1 src/model/lfm2/gqa.rs (GqaConfig::pad_head_dim_to,
 *     padded_head_dim) pads a head dim up to a multiple for aligned computation (36 -> 40 for
 *     Moonshine); here the multiple is the kernels' tile width.  attn_fwd,
 *     which has no workspace, returns ATTN_ERR_UNSUPPORTED for them, as does attn_decode; odd
 *     head dims are unsupported.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,    /* a size <= 0, a NULL required pointer, a bad flag          */
    ATTN_ERR_DIM_MISMATCH = 2,   /* Hq not a multiple of Hkv; odd D with RoPE                 */
    ATTN_ERR_EMPTY_KV = 3,       /* Skv == 0 / Smax == 0: no key to attend to                 */
    ATTN_ERR_UNSUPPORTED = 4,    /* valid request outside what the kernels implement          */
    ATTN_ERR_WORKSPACE = 5,      /* workspace NULL or smaller than the *_workspace_size query */
    ATTN_ERR_CUDA = 6,           /* a CUDA launch or driver call failed                       */
    ATTN_ERR_DEVICE_TIMEOUT = 7  /* reserved for status-word decoding by callers              */
} attn_status;

typedef enum {
    ATTN_BF16 = 0,        /* q, k, v, o, x stored as bfloat16; fp32 accumulation              */
    ATTN_FP32 = 1,        /* q, k, v, o, x stored as float32; fp32 arithmetic (no TF32)       */
    ATTN_BF16_OUT_F32 = 2 /* q, k, v bfloat16; o written as float32 (attn_fwd*, attn_decode).
                             bf16 storage of o has a spacing of 2^-6 at |o| >= 2, so callers
                             that need o to better than that take it in float32.              */
} attn_dtype;

typedef void* attn_stream_t; /* a cudaStream_t */

/*
 * attn_fwd -- exact attention forward (prefill).
 *   q    [B, Sq, Hq, D]   dtype          read
 *   k, v [B, Skv, Hkv, D] dtype          read
 *   o    [B, Sq, Hq, D]   dtype (float32 with ATTN_BF16_OUT_F32)   written
 *   lse  [B, Hq, Sq]      float32        written; may be NULL (not produced)
 *   scale                  the score multiplier (commonly 1/sqrt(D)); must be finite and > 0
 *   causal                 0 or 1
 * Returns ATTN_OK, or INVALID_ARG / DIM_MISMATCH / EMPTY_KV / UNSUPPORTED / CUDA.
 * bf16 path: QK^T and PV on tcgen05 tensor cores, P rounded to bf16, fp32 accumulators; O is
 * normalised by the sum of the rounded P values (the weights the PV product used) and lse by
 * the fp32 sum.
 */
attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                     int Hkv, int Sq, int Skv, int D, float scale, int causal, attn_dtype dtype,
                     attn_stream_t stream);

/*
 * attn_fwd_ex -- attn_fwd with RoPE on Q and K (rope_base > 0; rope_base <= 0 is attn_fwd).
 *   Query row i is rotated at position q_pos0 + i, key j at position j:
 *   theta_p = pos * rope_base^(-2p/D) for pair p; (x_2p, x_2p+1) -> (x_2p cos - x_2p+1 sin,
 *   x_2p sin + x_2p+1 cos).  Angles are formed in double precision.  q_pos0 >= 0; D even.
 *   workspace / workspace_bytes: device scratch of at least attn_fwd_ex_workspace_size(...)
 *   bytes, owned by the caller; its contents are overwritten.  With rope_base <= 0 the
 *   workspace may be NULL: the call then runs as attn_fwd.  A non-NULL workspace smaller
 *   than the size query returns ATTN_ERR_WORKSPACE.
 * Key splits: a bf16 problem whose 128-row query tiles (ceil(Sq/128) * B * Hq of them) fill at
 * most half of the 148 SMs divides each tile's key tiles among attn_fwd_kv_splits(...) CTAs
 * (contiguous near-equal chunks) and merges their normalised partial outputs by logsumexp,
 * L = log sum_s e^(lse_s), O = sum_s e^(lse_s - L) o_s, in a second kernel launched as a
 * programmatic dependent (the split-KV combine of the decode path: oxibonsai-model 0.1.4
 * src/layers/flash_decode.rs, combine_tile_outputs).  This needs the workspace (the partials
 * live there); attn_fwd and a NULL workspace run unsplit.  The result is the same attention
 * up to rounding.
 * bf16 path: rotated Q and K are carried as a pair of bf16 values (hi + lo) each, so the
 * rotated operands keep about 16 mantissa bits; QK^T runs as three bf16 MMA chains.  K is
 * rotated once per call by a pre-pass into the workspace; with ATTN_ROPE_K_FORM=fused in the
 * environment (read at every call) the prefill kernel rotates each K tile in shared memory
 * instead -- the same result up to rounding, kept as the measured alternative (it is slower).
 */
attn_status attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal,
                        attn_dtype dtype, float rope_base, int q_pos0, void* workspace,
                        size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_fwd_masked -- attn_fwd_ex with an additive mask on the scaled scores:
 *   s_ij = scale * q_i . k_j + mask[b, h, i, j]   (then the causal mask, if causal)
 *   whisper-apr 0.3.1 src/model/attention_generated.rs (compute_block_scores: score = dot *
 *   scale, then score += mask[q, k]; scaled_dot_product_attention adds the mask before the row
 *   softmax).  mask: float32, element (b, h, i, j) at mask[b * mask_batch_stride +
 *   h * mask_head_stride + i * Skv + j] (strides in elements, >= 0; 0 broadcasts, e.g. both 0
 *   for one [Sq, Skv] mask shared by every batch and head), 4-byte aligned, read on the device.
 *   -inf entries remove keys; a row whose scores are all -inf gets o = 0, lse = -inf.  Other
 *   arguments, workspace and errors as attn_fwd_ex (attn_fwd_ex_workspace_size gives the bytes).
 *   At D = 64 without RoPE, with every mask row 16-byte aligned (base, strides and Skv multiples
 *   of 4 elements), the mask is staged into shared memory by TMA; otherwise each thread reads
 *   its mask row with plain loads.
 */
attn_status attn_fwd_masked(const void* q, const void* k, const void* v, const float* mask, int64_t mask_batch_stride,
                            int64_t mask_head_stride, void* o, float* lse, int B, int Hq, int Hkv, int Sq, int Skv,
                            int D, float scale, int causal, attn_dtype dtype, float rope_base, int q_pos0,
                            void* workspace, size_t workspace_bytes, attn_stream_t stream);

/* Bytes of workspace attn_fwd_ex needs for these sizes: with RoPE the cos/sin table and the
 * rotated-K halves; with key splits the fp32 partial outputs and logsumexps,
 * splits * B * Sq * Hq * (D + 1) * 4 bytes (each part rounded up to 256 bytes); for D outside
 * {64, 128} the padded q, k, v, o and the inner call's needs.  0 when none applies.          */
size_t attn_fwd_ex_workspace_size(int B, int Hq, int Hkv, int Sq, int Skv, int D, attn_dtype dtype,
                                  float rope_base, int q_pos0);

/* Key splits attn_fwd_ex uses for these sizes when given its workspace (1: unsplit):
 * n = min(148 / tiles, nkv / 2, 16) for bf16 problems with tiles = ceil(Sq/128) * B * Hq <= 74
 * and nkv = ceil(Skv/128), when n >= 2 and the split spares the longest chunk at least 8 key
 * tiles (nkv - ceil(nkv / n) >= 8); 1 otherwise (and for ATTN_FP32).  Sizes <= 0 give 1.      */
int attn_fwd_kv_splits(int B, int Hq, int Sq, int Skv, attn_dtype dtype);

/*
 * attn_decode -- one query token per (sequence b, q head) against a KV cache, split-KV.
 *   q       [B, Hq, D]          bf16    read
 *   kcache  [B, Smax, Hkv, D]   bf16    read (rows >= seqlens[b] are never read)
 *   vcache  [B, Smax, Hkv, D]   bf16    read
 *   seqlens [B]                 int32   read on the device; values outside [1, Smax] are
 *                                       clamped and flagged in the device status word
 *   o       [B, Hq, D]          bf16    written (float32 with ATTN_BF16_OUT_F32)
 *   lse     [B, Hq]             float32 written; may be NULL
 *   num_splits  upper bound on KV splits per sequence (>= 1); sequence b uses
 *               clamp(seqlens[b] / 512, 1, num_splits) contiguous near-equal splits
 *   workspace   device scratch of >= attn_decode_workspace_size(B, Hq, D, num_splits) bytes
 * No causal mask: the single new token sees the whole cache.  dtype ATTN_BF16 or
 * ATTN_BF16_OUT_F32 (ATTN_FP32 returns ATTN_ERR_UNSUPPORTED).
 */
attn_status attn_decode(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                        void* o, float* lse, int B, int Hq, int Hkv, int Smax, int D, float scale,
                        int num_splits, void* workspace, size_t workspace_bytes, attn_dtype dtype,
                        attn_stream_t stream);

/* Bytes of workspace attn_decode needs (partial outputs and logsumexps of every split).    */
size_t attn_decode_workspace_size(int B, int Hq, int D, int num_splits);

/*
 * attn_decode_noalloc -- attn_decode for callers that cannot allocate device memory.
 *   (Not an operation of the method: the pages have no counterpart.  It is attn_decode with
 *   the split partials kept in scratch memory that the library owns.)
 *   Some callers cannot hand attn_decode a workspace: code inside a host framework that owns
 *   every device allocation and gives it only input and output buffers, or a latency-bound
 *   serving path that must not call cudaMalloc, which can synchronise the device and take an
 *   unbounded time.  This entry point takes the same arguments as attn_decode minus the
 *   workspace and allocates nothing: the partials go to a fixed array of
 *   ATTN_NOALLOC_SCRATCH_BYTES bytes that exists once on every GPU that loads the library and
 *   stays allocated until the process exits.
 *   - Sizes: attn_decode_workspace_size(B, Hq, D, num_splits) must not exceed
 *     ATTN_NOALLOC_SCRATCH_BYTES, else ATTN_ERR_WORKSPACE (attn_last_error() says by how much).
 *   - Set-up: the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, which may load the library's GPU code onto that device).  Failure
 *     returns ATTN_ERR_CUDA.
 *   - Sharing: every call on a device uses the same array, and it keeps the last call's
 *     contents.  Calls that overlap on the GPU (different streams, no ordering between them)
 *     race on it and may return wrong results; order them on one stream or with events.
 *     Nothing in the array needs to start at zero.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (16u << 20)
attn_status attn_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                const int32_t* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                                int Smax, int D, float scale, int num_splits, attn_dtype dtype,
                                attn_stream_t stream);

/*
 * rope_apply -- rotate x in place: x [T, H, D] (dtype), token t at position pos[t]
 * (int32 device array [T]); rotation as in attn_fwd_ex.  D must be even (DIM_MISMATCH).
 */
attn_status rope_apply(void* x, const int32_t* pos, int T, int H, int D, float base, attn_dtype dtype,
                       attn_stream_t stream);

/*
 * attn_bwd -- gradients of attn_fwd / attn_fwd_ex with respect to q, k and v.
 *   scirs2-neural 0.4.3 flash_attention.rs (flash_backward_head: FA-2's backward, recomputing the
 *   probabilities from the saved row statistics); scirs2-neural 0.4.4 grouped_query_attention.rs
 *   (backward: kv-head gradients summed over the group, RoPE undone on dq and dk).
 *   q, o, dout [B, Sq, Hq, D]   read (o: the forward's output; dout: gradient of the loss wrt o)
 *   k, v       [B, Skv, Hkv, D] read
 *   lse        [B, Hq, Sq] fp32 read: the forward's logsumexp (-inf for rows without a key)
 *   dq         [B, Sq, Hq, D]   written;  dk, dv [B, Skv, Hkv, D] written
 *   dtype: ATTN_FP32 (all fp32), ATTN_BF16 (inputs and gradients bf16), ATTN_BF16_OUT_F32
 *   (bf16 inputs, fp32 gradients).  scale, causal, rope_base, q_pos0: as passed to the forward.
 *   workspace: >= attn_bwd_workspace_size(...) bytes of device scratch, contents overwritten.
 * ATTN_FP32 runs in fp32 on the CUDA cores (matches the definition to ~1e-6 relative when o and
 * lse are exact).  The bf16 dtypes run the products on the tensor cores (bf16 operands, fp32
 * accumulation; P and dS are rounded to bf16 as operands, ~2^-9 relative each); with RoPE the
 * scores are recomputed from hi + lo bf16 halves of the rotated q and k, as in the forward.
 * o from the bf16 forward carries its own rounding into D_i = dout . o.
 */
attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                     int causal, attn_dtype dtype, float rope_base, int q_pos0, void* workspace,
                     size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_bwd_masked -- attn_bwd for attn_fwd_masked: the probabilities are recomputed with the
 * same additive mask (same pointer and strides as the forward); mask entries are constants, so
 * no gradient flows to them.  Arguments, workspace (attn_bwd_workspace_size) and errors as
 * attn_bwd.
 */
attn_status attn_bwd_masked(const void* q, const void* k, const void* v, const float* mask, int64_t mask_batch_stride,
                            int64_t mask_head_stride, const void* o, const float* lse, const void* dout, void* dq,
                            void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal,
                            attn_dtype dtype, float rope_base, int q_pos0, void* workspace, size_t workspace_bytes,
                            attn_stream_t stream);

/* Bytes of workspace attn_bwd needs for these sizes and dtype (fp32: fp32 copies of rotated q
 * and k, dout, v; bf16: the rotated q and k as hi/lo bf16 pairs with RoPE; both: the row sums
 * D_i and, with RoPE, the angle table); 0 for invalid sizes.                               */
size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Sq, int Skv, int D, attn_dtype dtype, float rope_base,
                               int q_pos0);

/*
 * attn_kv_append -- the decode step's cache update, fused into one launch: rotate the new keys
 * with RoPE at their positions and write them, with the new values, into the cache right after
 * each sequence's current length; rotate the new queries at the same positions; advance the
 * lengths.  scirs2-neural 0.4.4 grouped_query_attention.rs (forward_with_cache: new K/V follow
 * the cached ones, new Q and K are rotated at the cache offset); whisper-apr 0.3.1
 * src/model/lfm2 KvCache (an append past the capacity is an error).
 *   kcache, vcache [B, Smax, Hkv, D]  bf16   rows [L_b, L_b + T) written (K rotated)
 *   seqlens [B]                       int32  device; read as L_b, advanced to L_b + T
 *   k_new, v_new   [B, T, Hkv, D]     bf16   read
 *   q              [B, T, Hq, D]      bf16   rotated in place at positions L_b + t; may be NULL
 *   rope_base > 0: token t of sequence b is rotated at position L_b + t (angles in double, as in
 *   rope_apply); rope_base <= 0: keys and queries are copied / left unrotated.
 * Overflow: a sequence with L_b < 0 or L_b + T > Smax is left untouched (cache rows, length and
 * its q rows) and bit 8 of the device status word is set; the other sequences are appended.
 * D must be a multiple of 8 (DIM_MISMATCH), all pointers 16-byte aligned.  After the call,
 * attn_decode with the same seqlens lets each new query see the cache including its own key.
 */
attn_status attn_kv_append(void* kcache, void* vcache, int32_t* seqlens, const void* k_new, const void* v_new,
                           void* q, int B, int T, int Hq, int Hkv, int Smax, int D, float rope_base,
                           attn_stream_t stream);

/* Static description of a status code.                                                     */
const char* attn_status_string(attn_status s);

/* Which call failed, and the CUDA error text, for the calling thread's most recent
 * ATTN_ERR_CUDA ("" if none).  The string stays valid until that thread's next failure.     */
const char* attn_last_error(void);

/*
 * attn_selftest_wait_timeout -- check of the kernels' failure reporting: launches one tiny
 * kernel whose only wait (an mbarrier nothing arrives on) can never complete.  The wait gives up
 * after timeout_us microseconds (1 .. 1e6), sets bit 1 in the device status word and the kernel
 * returns normally; attn_read_device_status then reports it.  The same bounded wait guards every
 * wait in the attention kernels (with a 2 s bound), so a logic or hardware stall ends with a
 * status bit rather than a hung GPU.
 */
attn_status attn_selftest_wait_timeout(int timeout_us, attn_stream_t stream);

/*
 * Read and clear the device status word (bit 1: a bounded wait gave up; bit 2: a decode
 * sequence length was clamped; bit 4: tensor memory allocation failed; bit 8: a cache append
 * would have passed the capacity and was skipped).  Synchronises
 * `stream` first.  Returns the bits, or -1 if the read itself failed.
 */
int attn_read_device_status(attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
