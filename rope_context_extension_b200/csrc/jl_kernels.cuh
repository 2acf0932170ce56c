// Kernel argument blocks and launchers (internal; the public surface is jl_api.h).
#pragma once

#include "jl_common.cuh"

namespace jl {

constexpr int kMaxHalfDim = 64;  // head_dim <= 128

// Correction rotation of rows [row_begin, row_end) of a [B, L, H, D] bf16 tensor.
struct RotateArgs {
  const __nv_bfloat16* x;
  __half* y;     // fp16 output
  __half* y_lo;  // optional fp16 residual (y + y_lo carries about 22 bits), or null
  int B, L, H;
  int row_begin, row_end;
  int is_query;      // 1: rotate by p_q(i) - i, 0: by f(j) - j
  int64_t G, shift;  // group size and query shift
  double theta[kMaxHalfDim];
};
cudaError_t launch_rotate_rows(const RotateArgs& args, int D, cudaStream_t stream);

// Fused bifocal prefill (tcgen05 + TMEM + TMA).
struct PrefillArgs {
  __nv_bfloat16* o;  // [B, L, Hq, D]
  float* lse;        // [B, Hq, L] or null
  int* dev_error;    // device int or null
  int B, L, Hq, Hkv, r;
  int nh;            // query heads per CTA (1 or 2, same KV head)
  int num_mb;        // ceil(L / 128)
  int w0;            // band width; huge when every pair is local
  int all_local;
  float scale_log2;  // softmax scale * log2(e)
};
cudaError_t launch_prefill(const CUtensorMap& tm_q, const CUtensorMap& tm_qr, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_kr, const CUtensorMap& tm_v, const CUtensorMap& tm_qr_lo,
                           const CUtensorMap& tm_kr_lo, const PrefillArgs& a, int D, bool split,
                           cudaStream_t stream);

// Split-KV bifocal decode (mma.sync tiles, in-register correction of keys).
struct DecodeArgs {
  const __nv_bfloat16* q;  // [B, Hq, D], rotated at position L - 1
  __nv_bfloat16* o;        // [B, Hq, D]
  float* lse;              // [B, Hq] or null
  float2* part_ml;         // [B, Hkv, splits, r] (running max in log2 units, sum)
  float* part_o;           // [B, Hkv, splits, r, D]
  int* counters;           // [B, Hkv], zero between calls
  int* dev_error;
  int B, L, Hq, Hkv, r;
  int splits, ntiles;      // 64-key tiles in [0, L)
  int w0, all_local;
  int64_t G;
  uint32_t g_magic;        // ceil(2^32 / G) for G < 16 (floor(x / G) = umulhi(x, g_magic), x < 32)
  int64_t dq;              // p_q(L - 1) - (L - 1)
  float scale_log2;
  double theta[kMaxHalfDim];
};
cudaError_t launch_decode(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const DecodeArgs& a, int D,
                          cudaStream_t stream);
// Resident decode CTAs per SM (occupancy of the D = 128 kernel, cached).
int decode_ctas_per_sm();

}  // namespace jl
