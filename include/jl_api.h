/*
 * jl_api.h -- C ABI of the B200 (sm_100a) Dynamic Bifocal RoPE attention
 * library (libjetlong.so).
 *
 * The method (Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal
 * RoPE; Jet-Long review (romaanj.github.io), "Method"; gist.science technical
 * summary, "Methodologie §1-§2"):
 *   G     = max(1, ceil(L / w_pretrained)), from the current length L
 *   f(x)  = floor(x / G)                    remote position map
 *   a causal pair (query i, key j) with i - j < w0 keeps its base RoPE score;
 *   every other causal pair is scored with the query at p_q(i) and the key at
 *   f(j).  Keys stay in the cache rotated at their absolute positions; the
 *   correction rotations R(p_q(i) - i) and R(f(j) - j) are applied on the fly.
 *
 * The pages leave the query-side remote position unstated.  `mode` selects it:
 *   JL_QSHIFT_SELF_EXTEND  p_q(i) = floor(i/G) + (w0 - floor(w0/G))
 *                          (remote distances continue from w0; default)
 *   JL_QSHIFT_NONE         p_q(i) = floor(i/G)
 * Both reduce to base RoPE at G = 1.
 *
 * Conventions shared by every entry point:
 *   - bf16 tensors are row-major and contiguous:
 *       Q, O (prefill) [B, L, Hq, D]; K, V (prefill) [B, L, Hkv, D];
 *       KV cache (decode) [B, Lmax, Hkv, D]; q, o (decode) [B, Hq, D];
 *       LSE fp32: prefill [B, Hq, L], decode [B, Hq] (natural log of the sum
 *       of exp of the scaled scores).
 *   - Q and K hold rows already rotated at their absolute (base) positions with
 *     half-split RoPE pairs (t, t + D/2), theta_t = rope_base^(-2t/D).
 *   - D (head_dim) is 64 or 128; Hq % Hkv == 0; 1 <= L; w0 >= 0;
 *     w_pretrained >= 1.  softmax_scale == 0 means 1/sqrt(D).
 *   - Size limits (JL_ERR_UNSUPPORTED beyond them): L <= 2^30; B and Hkv
 *     <= 65535; one prefill call's query rows <= 65535 * 128 = 8,388,480
 *     (longer prompts go in chunks, jl_bifocal_prefill_chunk), with
 *     Hq * ceil(rows / 128) * B < 2^31.
 *   - Device pointers must be 16-byte aligned.  The caller owns every buffer
 *     (inputs, outputs and scratch); the library never allocates device
 *     memory and never writes its inputs.
 *   - Calls are asynchronous on `stream` (a cudaStream_t, NULL = default
 *     stream).  The return value reports argument checks and launch errors.
 *     Device-side failures are written to *dev_error (a device int, may be
 *     NULL) as a non-zero value -- 1: a pipeline wait ran out of time; 2: a
 *     varlen sequence length out of range; 3: a corrected prefill operand
 *     beyond fp16's range -- and the outputs are then invalid.
 *   - Reentrant; no global state beyond cached kernel attributes, with one
 *     exception: jl_bifocal_decode_noalloc keeps its scratch in a fixed device
 *     array inside the library, shared by every call on a device, so its
 *     calls must be ordered on the GPU (see that entry).
 */
#ifndef JL_API_H
#define JL_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  JL_OK = 0,
  JL_ERR_INVALID_ARG = -1,    /* null pointer, bad size or range */
  JL_ERR_UNSUPPORTED = -2,    /* shape the kernels do not handle (e.g. D not 64/128) */
  JL_ERR_ALIGNMENT = -3,      /* a device pointer is not 16-byte aligned */
  JL_ERR_WORKSPACE = -4,      /* scratch missing or smaller than required */
  JL_ERR_CUDA = -5,           /* a CUDA runtime / driver call failed */
  JL_ERR_DEVICE_TIMEOUT = -6  /* reserved: host-side report of a device timeout */
} jl_status;

typedef enum { JL_QSHIFT_NONE = 0, JL_QSHIFT_SELF_EXTEND = 1 } jl_qshift;

/*
 * Optional prefill flags, OR-ed into `mode` (decode ignores them).
 *
 * The default prefill forms remote scores from fp16 hi + lo operands:
 * S = Q_hi K_hi + Q_hi K_lo + Q_lo K_hi, with x = hi + lo to about 22
 * significant bits, so a score's rounding error is about 2^-21 |q| |k| (in
 * fp32 accumulation).  The correction rotations are computed in fp32 from fp64
 * angles: R(p_q(i) - i) is applied to the query block inside the attention
 * kernel, in registers, on its way into tensor memory; R(f(j) - j) is applied
 * to the key rows once per KV head by a correction pass that writes their hi
 * and lo parts to the workspace (it serves every query head of the KV head).
 * Local (base RoPE) scores and P V use the bf16 inputs as they are.  Corrected
 * values must stay within fp16's range: a query or key component of magnitude
 * 46340 or more can overflow, which is reported as device error 3 (results
 * invalid).
 *
 * JL_PREFILL_KEYS_IN_KERNEL: the same arithmetic, with the key tiles also
 *   corrected inside the attention kernel (a rotation warpgroup, one tile
 *   ahead of the tensor core): no workspace, but slower on B200 (every query
 *   head's CTAs redo the rotation of the shared key tiles).
 * JL_PREFILL_FP16: a correction pass writes R(p_q(i) - i) Q_i and R(f(j) - j) K_j
 *   rounded once to fp16, and the attention kernel forms each remote score
 *   with one fp16 product (two query heads per CTA).  About twice as fast, but
 *   a score's rounding error is about 2^-11 |q| |k|: on rows dominated by one
 *   key of large norm that shows in the LSE (1e-2 on the pages' outlier
 *   workload, against 1e-3 for the default).
 * The two flags are exclusive.  When every pair is local (G = 1 or w0 >= L) no
 * operand is corrected and every mode runs plain causal RoPE attention on the
 * bf16 inputs (two query heads per CTA), needing no workspace.
 */
enum { JL_PREFILL_FP16 = 4, JL_PREFILL_KEYS_IN_KERNEL = 8 };

/* Human-readable name of a status code (static string). */
const char* jl_status_string(int status);

/*
 * Group size G = max(1, ceil(L / w_pretrained)) (Jet-Long review, "Method";
 * gist.science summary, "Methodologie §1").  Host only.
 * Errors: JL_ERR_INVALID_ARG if L < 0, w_pretrained < 1 or G_out is NULL.
 */
int jl_group_size(int64_t L, int64_t w_pretrained, int64_t* G_out);

/*
 * Remote positions for a length-L sequence (host arrays of L int32 each, either
 * may be NULL): q_pos_out[i] = p_q(i) (see `mode`), k_pos_out[j] = f(j).
 * Host only; used to check the position maps bit-exactly.
 * Errors: JL_ERR_INVALID_ARG for L < 1, w0 < 0, w_pretrained < 1, a bad mode,
 * or positions that do not fit int32.
 */
int jl_remote_positions(int64_t L, int64_t w0, int64_t w_pretrained, int mode, int32_t* q_pos_out,
                        int32_t* k_pos_out);

/*
 * Tile schedule of jl_bifocal_prefill over a whole sequence of length L, per
 * (batch, query head), from the same functions the attention kernel runs.
 * A causal pair (i, j) is local when i - j < w0 and remote otherwise (Jet-Long
 * review, "Method"); a 128 x 128 tile holding both kinds gets a local and a
 * remote pass with complementary masks.  When G = 1 or w0 >= L every tile gets
 * one local pass (the method is then exactly base RoPE).  Host only.
 * counts_out[4] (caller-owned): [0] tiles with a local pass only, [1] tiles
 * with both passes, [2] tiles with a remote pass only, [3] passes in total
 * ([0] + 2 [1] + [2]).
 * Errors: JL_ERR_INVALID_ARG for a NULL counts_out, L < 1 or L > 2^30, w0 < 0
 * or w_pretrained < 1.
 */
int jl_prefill_tile_classes(int64_t L, int64_t w0, int64_t w_pretrained, int64_t* counts_out);

/*
 * Scratch bytes jl_bifocal_prefill may need: the larger of the default's
 * (fp16 hi and lo key rows, 4 * B * L * Hkv * D bytes) and JL_PREFILL_FP16's
 * (fp16 corrected query and key rows, 2 * B * L * (Hq + Hkv) * D bytes), each
 * plus alignment.  JL_PREFILL_KEYS_IN_KERNEL needs none.  0 on bad arguments.
 */
size_t jl_prefill_workspace_bytes(int B, int L, int Hq, int Hkv, int head_dim);

/*
 * Fused bifocal causal prefill (self-attention of L new tokens).
 *   q [B, L, Hq, D], k / v [B, L, Hkv, D]: bf16 device, base-rotated, read only.
 *   o [B, L, Hq, D] bf16 device (written); lse [B, Hq, L] fp32 device or NULL.
 *   w0: band width of exact base-RoPE scoring (i - j < w0); w0 >= L, or
 *   L <= w_pretrained (G = 1), gives plain causal RoPE attention.
 *   mode: query shift (jl_qshift) | optional prefill flag (see above).
 *   workspace: device scratch of at least jl_prefill_workspace_bytes(...)
 *   bytes (contents on entry do not matter; overwritten); may be NULL / 0 with
 *   JL_PREFILL_KEYS_IN_KERNEL or when every pair is local.
 * Launches: jl_prefill_correction (one correction-rotation kernel for the
 * keys; with JL_PREFILL_FP16 one for the queries too; none with
 * JL_PREFILL_KEYS_IN_KERNEL or when every pair is local), then
 * jl_prefill_attention (the fused tcgen05 attention kernel).  *dev_error
 * receives 1 (a pipeline wait ran out) or 3 (a corrected value beyond fp16's
 * range).
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED, JL_ERR_ALIGNMENT,
 * JL_ERR_WORKSPACE, JL_ERR_CUDA; nothing is launched on an argument error.
 */
int jl_bifocal_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L,
                       int Hq, int Hkv, int head_dim, int w0, int w_pretrained, double rope_base,
                       float softmax_scale, int mode, void* workspace, size_t workspace_bytes,
                       int* dev_error, void* stream);

/*
 * First stage of jl_bifocal_prefill, exposed so the two stages can be timed or
 * scheduled separately: the correction pass.  Default: writes R(f(j) - j) K_j
 * to the workspace as fp16 hi [B, L, Hkv, D] and, at offset round_up(2 * B *
 * L * Hkv * D, 256), lo (hi + lo carries about 22 significant bits).
 * JL_PREFILL_FP16: writes R(p_q(i) - i) Q_i as fp16 [B, L, Hq, D], followed (at
 * offset round_up(2 * B * L * Hq * D, 256)) by R(f(j) - j) K_j as fp16
 * [B, L, Hkv, D].  JL_PREFILL_KEYS_IN_KERNEL: nothing to do.  Only rows that
 * have a remote partner are written (queries i >= w0, keys j < L - w0).  The
 * correction identity is the additive composition of RoPE rotations
 * (gist.science summary, "§2 On-the-Fly Correctie Rotatie").  A rotated value
 * beyond fp16's range sets *dev_error (a device int, may be NULL) to 3.
 * Launches nothing when every pair is local.  Errors as jl_bifocal_prefill.
 */
int jl_prefill_correction(const void* q, const void* k, int B, int L, int Hq, int Hkv, int head_dim, int w0,
                          int w_pretrained, double rope_base, int mode, void* workspace, size_t workspace_bytes,
                          int* dev_error, void* stream);

/*
 * Second stage of jl_bifocal_prefill: the fused tcgen05 attention kernel
 * (one launch), reading Q, K, V and the corrected rows that
 * jl_prefill_correction left in `workspace` (same w0 / w_pretrained /
 * rope_base / mode).  Errors as jl_bifocal_prefill.
 */
int jl_prefill_attention(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L, int Hq,
                         int Hkv, int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale,
                         int mode, const void* workspace, size_t workspace_bytes, int* dev_error, void* stream);

/*
 * Scratch bytes jl_bifocal_prefill_chunk may need (as
 * jl_prefill_workspace_bytes, with chunk_len query rows and q_offset +
 * chunk_len key rows).  0 on bad arguments.
 */
size_t jl_prefill_chunk_workspace_bytes(int B, int q_offset, int chunk_len, int Hq, int Hkv, int head_dim);

/*
 * Chunked prefill against an existing cache: the chunk's queries sit at
 * positions q_offset .. q_offset + chunk_len - 1 and attend (causally) to
 * cache keys 0 .. q_offset + chunk_len - 1; G comes from the total length
 * q_offset + chunk_len (the current length, Jet-Long review "Method").  With
 * q_offset = 0 and chunk_len = L this is jl_bifocal_prefill on a cache.
 *   q [B, chunk_len, Hq, D]: bf16 device, rotated at its absolute positions.
 *   k_cache / v_cache [B, cache_len, Hkv, D]: bf16 device, already holding the
 *   chunk's own keys and values; read only.  q_offset + chunk_len <= cache_len.
 *   o [B, chunk_len, Hq, D] bf16; lse [B, Hq, chunk_len] fp32 or NULL.
 *   workspace: jl_prefill_chunk_workspace_bytes(...) bytes (NULL / 0 with
 *   JL_PREFILL_KEYS_IN_KERNEL).  Everything else as jl_bifocal_prefill.
 * Note: a cache built by earlier decode steps is not equivalent to re-running
 * prefill over the whole sequence (the keys were rotated once, at their base
 * positions, either way; the hidden states are not recomputed).
 * Launches: as jl_bifocal_prefill.
 */
int jl_bifocal_prefill_chunk(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len, void* o,
                             float* lse, int B, int q_offset, int chunk_len, int Hq, int Hkv, int head_dim, int w0,
                             int w_pretrained, double rope_base, float softmax_scale, int mode, void* workspace,
                             size_t workspace_bytes, int* dev_error, void* stream);

/*
 * Scratch bytes jl_bifocal_prefill_ie needs: the corrected key rows (hi and
 * lo, every row), three fp32 partial outputs [B, L, Hq, D] and their LSEs
 * [B, Hq, L] (`mode` does not change it).
 */
size_t jl_prefill_ie_workspace_bytes(int B, int L, int Hq, int Hkv, int head_dim, int mode);

/*
 * The pages' own prefill formulation, unfused, for comparison with the fused
 * per-tile kernel (Jet-Long review, "Method"; gist.science summary, "§2
 * Inclusie-Exclusie Attention Merge"): three attention calls — (A) the window
 * 0 <= i - j < w0 with base RoPE, (B) every causal pair with remote positions,
 * (C) the window with remote positions — each writing an fp32 output and an
 * fp32 LSE (the default prefill path: hi + lo remote operands; the prefill
 * flags in `mode` are ignored), merged as
 * O = (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C), W_X = exp(LSE_X - max
 * LSE).  Same arguments and result as jl_bifocal_prefill up to rounding, which
 * the subtraction amplifies by (W_A + W_B + W_C) / (W_A + W_B - W_C): without
 * bound on rows where one key inside the window dominates both B and C.
 * workspace: jl_prefill_ie_workspace_bytes(...).  When every pair is local it
 * runs jl_bifocal_prefill.
 * Launches: one correction kernel (every key row), three attention kernels
 * and one merge kernel.
 */
int jl_bifocal_prefill_ie(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L, int Hq,
                          int Hkv, int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale,
                          int mode, void* workspace, size_t workspace_bytes, int* dev_error, void* stream);

/*
 * Scratch bytes jl_bifocal_decode needs on this device (split partials and one
 * ticket counter per (batch, KV head)).  0 on bad arguments.
 */
size_t jl_decode_workspace_bytes(int B, int L, int Hq, int Hkv, int head_dim);

/*
 * Fused bifocal decode: one new query token per sequence at position L - 1
 * against the first L cache entries (L counts the new token's own key).
 *   q [B, Hq, D] bf16 device, rotated at position L - 1.
 *   k_cache / v_cache [B, cache_len, Hkv, D] bf16 device, keys rotated at their
 *   absolute positions; read only, never rewritten; L <= cache_len.
 *   o [B, Hq, D] bf16 device; lse [B, Hq] fp32 device or NULL.
 *   Hq / Hkv <= 8.
 *   workspace: device scratch of at least jl_decode_workspace_bytes(...) bytes.
 *   Its ticket counters must be zero before the first call (allocate it
 *   zero-filled); every call leaves them at zero again.  Calls that share a
 *   workspace must not overlap on the GPU.
 * Launches one kernel.
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED, JL_ERR_ALIGNMENT,
 * JL_ERR_WORKSPACE, JL_ERR_CUDA; nothing is launched on an argument error.
 */
int jl_bifocal_decode(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len, void* o,
                      float* lse, int B, int L, int Hq, int Hkv, int head_dim, int w0, int w_pretrained,
                      double rope_base, float softmax_scale, int mode, void* workspace,
                      size_t workspace_bytes, int* dev_error, void* stream);

/*
 * Varlen (continuous-batch) decode: sequence b has its own length
 * seq_lens[b] (device int32 array, 1 <= seq_lens[b] <= cache_len), hence its
 * own G_b = max(1, ceil(L_b / w_pretrained)), query position L_b - 1 and band.
 * The cache is read as it is: a sequence that crosses a multiple of
 * w_pretrained changes G without any cache rewrite (Jet-Long review, "Method";
 * gist.science summary, "§2 On-the-Fly Correctie Rotatie").
 *   max_len: the largest seq_lens value (host side; it sizes the split count).
 *   Everything else as jl_bifocal_decode; workspace as
 *   jl_decode_workspace_bytes(B, max_len, Hq, Hkv, head_dim).
 *   A length outside [1, cache_len] is clamped and flagged in *dev_error (2).
 * Launches one kernel.
 */
int jl_bifocal_decode_varlen(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len,
                             const int32_t* seq_lens, int max_len, void* o, float* lse, int B, int Hq, int Hkv,
                             int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale, int mode,
                             void* workspace, size_t workspace_bytes, int* dev_error, void* stream);

/*
 * Base RoPE of each sequence's new token and its append to the cache (one
 * launch).  q_raw [B, Hq, D], k_raw / v_new [B, Hkv, D]: bf16 device, not
 * rotated.  positions: device int32 [B], the new token's absolute position
 * p_b (0 <= p_b < cache_len).  Writes q_out [B, Hq, D] = R(p_b) q_raw (the
 * decode query), k_cache[b, p_b] = R(p_b) k_raw and v_cache[b, p_b] = v_new;
 * no other cache row is touched.  Angles p_b * theta_t are formed in fp64.
 * A position out of range skips that sequence and sets *dev_error to 2.
 * Errors: JL_ERR_INVALID_ARG, JL_ERR_UNSUPPORTED, JL_ERR_ALIGNMENT, JL_ERR_CUDA.
 */
int jl_rope_append(const void* q_raw, const void* k_raw, const void* v_new, const int32_t* positions, void* q_out,
                   void* k_cache, void* v_cache, int64_t cache_len, int B, int Hq, int Hkv, int head_dim,
                   double rope_base, int* dev_error, void* stream);

/*
 * Decode over one key range of a longer sequence (sequence-split decode across
 * GPUs): cache rows 0 .. key_count - 1 hold the keys at positions key_offset ..
 * key_offset + key_count - 1 of a sequence of total length total_len, whose new
 * query sits at position total_len - 1; G, the query shift and the band come
 * from total_len.  Writes this range's softmax-normalised o [B, Hq, D] (bf16)
 * and lse [B, Hq] (fp32, required for the combine).  key_offset + key_count
 * <= total_len; key_count <= cache_len.  Workspace as
 * jl_decode_workspace_bytes(B, key_count, ...).  Launches one kernel.
 */
int jl_bifocal_decode_range(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len,
                            int key_offset, int key_count, int total_len, void* o, float* lse, int B, int Hq, int Hkv,
                            int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale, int mode,
                            void* workspace, size_t workspace_bytes, int* dev_error, void* stream);

/*
 * Log-sum-exp combine of `parts` partial decode results over disjoint key
 * ranges (e.g. gathered from the GPUs of a sequence-split decode):
 * o_parts [parts, B, Hq, D] bf16 and lse_parts [parts, B, Hq] fp32 (device),
 * o [B, Hq, D] = sum_r exp(lse_r - M) o_r / sum_r exp(lse_r - M),
 * lse [B, Hq] = M + ln sum_r exp(lse_r - M) (may be NULL).  One launch.
 */
int jl_decode_combine(const void* o_parts, const float* lse_parts, int parts, void* o, float* lse, int B, int Hq,
                      int head_dim, void* stream);

/*
 * Self-test of the failure path every pipeline wait shares (no counterpart on
 * the pages): one tiny kernel waits, with the same bounded mbarrier wait, on a
 * barrier that nothing completes.  After timeout_s seconds (0 < timeout_s <= 10)
 * that wait gives up and writes 1 (the device-timeout code) to *dev_error (a
 * device int); a second warp waiting on another such barrier gives up as soon
 * as the first has aborted.  A wait that returned success would write 99.  The
 * kernel then returns normally, so the context stays usable.  Asynchronous on
 * `stream`; read *dev_error after synchronising.
 * Errors: JL_ERR_INVALID_ARG (null dev_error, timeout out of range), JL_ERR_CUDA.
 */
int jl_wait_timeout_check(int* dev_error, double timeout_s, void* stream);

/*
 * jl_bifocal_decode without a workspace argument, for callers that cannot
 * allocate device memory (e.g. a plugin inside an inference engine whose
 * device memory is wholly owned by the host framework's pool, or a serving
 * loop that must not allocate once it runs).  The paper has no counterpart:
 * this is an interface convenience of this library.
 *   Same arguments, layouts, results and errors as jl_bifocal_decode, minus
 *   the workspace.  Scratch lives in a fixed 4 MiB device array inside the
 *   library (held on every GPU that loads the library until exit), laid out
 *   for the split count the call uses; when that layout would not fit, the
 *   call runs with fewer splits (same results up to the order of the final
 *   sum).  A problem that does not fit with one split per (sequence, KV head)
 *   -- B * Hq * (4 * D + 8) + 4 * B * Hkv bytes plus alignment above 4 MiB,
 *   e.g. more than 126 sequences of 64 query heads at D = 128 -- is rejected
 *   with JL_ERR_WORKSPACE before any launch.
 *   All calls on a device share that array and it keeps the last call's
 *   contents: calls that overlap on the GPU race and give wrong results, so
 *   order them on one stream (or with events).  The ticket counters are
 *   cleared with cudaMemsetAsync before every launch.
 *   The first call on a device (and the first after cudaDeviceReset) looks up
 *   the array's address (cudaGetSymbolAddress, with that device current) and
 *   caches it; make that first call before any stream capture.  Nothing
 *   allocates device memory.
 * Launches one memset and one kernel.
 */
int jl_bifocal_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len, void* o,
                              float* lse, int B, int L, int Hq, int Hkv, int head_dim, int w0, int w_pretrained,
                              double rope_base, float softmax_scale, int mode, int* dev_error, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* JL_API_H */
