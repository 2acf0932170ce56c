// Kernel argument blocks and launchers (internal; the public surface is jl_api.h).
#pragma once

#include "jl_common.cuh"
#include "jl_sched.h"

namespace jl {

constexpr int kMaxHalfDim = 64;  // head_dim <= 128

// Correction rotation of rows [row_begin, row_end) of x [B, x_rows, H, D] (bf16)
// into y / y_lo [B, y_rows, H, D] (fp16); row r sits at position r + pos_off.
struct RotateArgs {
  const __nv_bfloat16* x;
  __half* y;     // fp16 output
  __half* y_lo;  // optional fp16 residual (y + y_lo carries about 22 bits), or null
  int B, x_rows, y_rows, H;
  int pos_off;
  int row_begin, row_end;
  int is_query;      // 1: rotate by p_q(i) - i, 0: by f(j) - j
  int64_t G, shift;  // group size and query shift
  int* dev_error;    // device int or null: set to kDevRange when a rotated value leaves fp16's range
  double theta[kMaxHalfDim];
  double u_hi[kMaxHalfDim], u_lo[kMaxHalfDim];  // theta_t / (2 pi), split for exact turn removal
};
cudaError_t launch_rotate_rows(const RotateArgs& args, int D, cudaStream_t stream);

// Fused bifocal prefill from fp16 corrected rows (tcgen05 + TMEM + TMA; two
// query heads per CTA).
struct PrefillArgs {
  __nv_bfloat16* o;  // [B, Lq, Hq, D]
  float* lse;        // [B, Hq, Lq] or null
  int* dev_error;    // device int or null
  int B, Hq, Hkv, r;
  int q_off;         // position of query row 0 (0 for a whole-sequence prefill)
  int Lq;            // query rows (this chunk)
  int Lk;            // keys: q_off + Lq
  int nh;            // query heads per CTA (1 or 2, same KV head)
  int num_mb;        // ceil(Lq / 128)
  int w0;            // band width; huge when every pair is local
  int all_local;
  float scale_log2;  // softmax scale * log2(e)
};
cudaError_t launch_prefill(const CUtensorMap& tm_q, const CUtensorMap& tm_qr, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_kr, const CUtensorMap& tm_v, const PrefillArgs& a, int D,
                           cudaStream_t stream);

// Fused bifocal prefill with the correction rotation inside the kernel and
// remote scores from fp16 hi + lo operands (tcgen05 + TMEM; one query head per
// CTA).  With rot_k = false the key tiles' hi / lo rows come from the
// correction pass through tm_kh / tm_kl instead of being rotated in the kernel.
struct PrefillHiloArgs {
  const __nv_bfloat16* q;  // [B, Lq, Hq, D], rotated at the absolute positions
  const __nv_bfloat16* k;  // [B, k_rows, Hkv, D]
  __nv_bfloat16* o;        // [B, Lq, Hq, D] bf16 output (when o_f32 is null)
  float* o_f32;            // [B, Lq, Hq, D] fp32 output instead (inclusion-exclusion partials), or null
  float* lse;              // [B, Hq, Lq] or null
  int* dev_error;          // device int or null
  int B, Hq, Hkv, r;
  int q_off;               // position of query row 0
  int Lq;                  // query rows (this chunk)
  int k_rows;              // rows of K / V
  int num_mb;              // ceil(Lq / 128)
  int w0;
  int kind;                // kBifocal, or one call of the inclusion-exclusion formulation
  int64_t G, shift;        // group size and query shift (from the total length q_off + Lq)
  float scale_log2;        // softmax scale * log2(e)
  double theta[kMaxHalfDim];
  double u_hi[kMaxHalfDim], u_lo[kMaxHalfDim];  // theta_t / (2 pi), split for exact turn removal
  float2 t1[kMaxHalfDim * 16];   // R(-theta_t b) for b < 16, [t][b] (cos, sin)
  float2 t16[kMaxHalfDim * 8];   // R(-theta_t 16 a) for a < 8, [t][a]
};
cudaError_t launch_prefill_hilo(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_kh,
                                const CUtensorMap& tm_kl, const PrefillHiloArgs& a, int D, bool rot_k,
                                cudaStream_t stream);

// Split-KV bifocal decode (mma.sync tiles, in-register correction of keys).
struct DecodeArgs {
  const __nv_bfloat16* q;  // [B, Hq, D], rotated at position L_b - 1
  __nv_bfloat16* o;        // [B, Hq, D]
  float* lse;              // [B, Hq] or null
  float2* part_ml;         // [B, Hkv, splits, r] (running max in log2 units, sum)
  float* part_o;           // [B, Hkv, splits, r, D]
  int* counters;           // [B, Hkv], zero between calls
  int* dev_error;
  const int* seq_lens;     // [B] per-sequence L_b (device), or null: every L_b = L
  int B, L, Hq, Hkv, r;    // L: the common length, or the largest L_b
  int64_t cache_len;       // rows of the cache (bound on L_b)
  int key_off;             // position of cache row 0 (a key range of a longer sequence), else 0
  int L_total;             // that sequence's total length (query at L_total - 1), or 0: = L
  int splits;              // CTAs per (batch, KV head); each covers a share of its sequence's tiles
  int w0, w_pretrained, qshift;
  float scale_log2;
  double theta[kMaxHalfDim];
  double u_hi[kMaxHalfDim], u_lo[kMaxHalfDim];  // theta_t / (2 pi), split for exact turn removal
};
// dev_error value for a sequence length outside [1, cache_len] (varlen decode)
constexpr int kDevBadLength = 2;
cudaError_t launch_decode(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const DecodeArgs& a, int D,
                          cudaStream_t stream);
// Resident decode CTAs per SM (occupancy of the D = 128 kernel, cached).
int decode_ctas_per_sm();
// Keys per decode tile (one TMA stage; splits cover whole tiles).
int decode_tile_keys();

// jl_bifocal_decode with its scratch in a caller-given fixed region of
// scratch_bytes (the no-allocation entry point): the region is laid out for the
// split count the call uses, lowered until it fits (JL_ERR_WORKSPACE when even
// one split per (sequence, KV head) does not), and the ticket counters are
// cleared on the stream before the launch.  Same argument checks as the public
// entry points; nothing is launched on an argument error.
int decode_in_fixed_scratch(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len, void* o,
                            float* lse, int B, int L, int Hq, int Hkv, int head_dim, int w0, int w_pretrained,
                            double rope_base, float softmax_scale, int mode, void* scratch, size_t scratch_bytes,
                            int* dev_error, void* stream);

// Inclusion-exclusion merge of three partial prefill outputs.
struct MergeArgs {
  const float* o_x[3];          // O_A, O_B, O_C [B, L, Hq, D] (fp32)
  const float* lse_x[3];        // LSE_A, LSE_B, LSE_C [B, Hq, L] (natural log)
  __nv_bfloat16* o;
  float* lse;                   // or null
  int B, L, Hq;
};
cudaError_t launch_ie_merge(const MergeArgs& a, int D, cudaStream_t stream);

// Log-sum-exp combine of R partial decode results over disjoint key ranges.
struct CombineArgs {
  const __nv_bfloat16* o_parts;  // [R, B, Hq, D]
  const float* lse_parts;        // [R, B, Hq]
  __nv_bfloat16* o;              // [B, Hq, D]
  float* lse;                    // [B, Hq] or null
  int R, B, Hq;
};
cudaError_t launch_lse_combine(const CombineArgs& a, int D, cudaStream_t stream);
cudaError_t launch_wait_timeout_check(int* dev_error, unsigned long long timeout_ns, cudaStream_t stream);

// Base RoPE of one new token per sequence and its append to the KV cache.
struct AppendArgs {
  const __nv_bfloat16* q_raw;  // [B, Hq, D] unrotated
  const __nv_bfloat16* k_raw;  // [B, Hkv, D] unrotated
  const __nv_bfloat16* v_new;  // [B, Hkv, D]
  const int* positions;        // [B] absolute position of the new token (device)
  __nv_bfloat16* q_out;        // [B, Hq, D] rotated at its position
  __nv_bfloat16* k_cache;      // [B, cache_len, Hkv, D]
  __nv_bfloat16* v_cache;
  int64_t cache_len;
  int B, Hq, Hkv;
  int* dev_error;
  double theta[kMaxHalfDim];
  double u_hi[kMaxHalfDim], u_lo[kMaxHalfDim];  // theta_t / (2 pi), split for exact turn removal
};
cudaError_t launch_rope_append(const AppendArgs& a, int D, cudaStream_t stream);

}  // namespace jl
