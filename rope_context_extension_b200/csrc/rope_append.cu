// Base RoPE of the newest token of each sequence and its append to the cache.
//
// A decode step receives the new token's unrotated q, k and v.  Keys enter the
// cache rotated at their absolute position and are never rewritten afterwards
// (Jet-Long review, "Method": the cache stores uncompressed keys at absolute
// positions; gist.science summary, "§2 On-the-Fly Correctie Rotatie": the
// cache stays untouched when the group size changes).  This kernel rotates q
// and k by their position p_b (half-split pairs, theta_t = base^(-2t/D), angle
// p_b * theta_t formed and reduced in fp64), writes the rotated q for the
// decode kernel, and stores the rotated k and the v in cache row p_b.
#include "jl_kernels.cuh"

namespace jl {

namespace {

template <int D>
__global__ void __launch_bounds__(128) rope_append_kernel(const __grid_constant__ AppendArgs a) {
  constexpr int H2 = D / 2;
  __shared__ float2 cs[H2];
  const int b = blockIdx.x;
  const int p = a.positions[b];
  if (p < 0 || (int64_t)p >= a.cache_len) {
    if (threadIdx.x == 0 && a.dev_error) atomicExch(a.dev_error, kDevBadLength);
    return;
  }
  for (int t = threadIdx.x; t < H2; t += blockDim.x) {
    double s, c;
    sincos_int_angle(p, a.u_hi[t], a.u_lo[t], &s, &c);
    cs[t] = make_float2((float)c, (float)s);
  }
  __syncthreads();
  const int nrot = (a.Hq + a.Hkv) * H2;
  for (int idx = threadIdx.x; idx < nrot; idx += blockDim.x) {
    const int h = idx / H2, t = idx % H2;
    const __nv_bfloat16* src;
    __nv_bfloat16* dst;
    if (h < a.Hq) {
      src = a.q_raw + ((size_t)b * a.Hq + h) * D;
      dst = a.q_out + ((size_t)b * a.Hq + h) * D;
    } else {
      const int g = h - a.Hq;
      src = a.k_raw + ((size_t)b * a.Hkv + g) * D;
      dst = a.k_cache + (((size_t)b * a.cache_len + p) * a.Hkv + g) * D;
    }
    const float x = __bfloat162float(src[t]), y = __bfloat162float(src[t + H2]);
    const float2 f = cs[t];
    dst[t] = __float2bfloat16_rn(x * f.x - y * f.y);
    dst[t + H2] = __float2bfloat16_rn(y * f.x + x * f.y);
  }
  for (int idx = threadIdx.x; idx < a.Hkv * D; idx += blockDim.x) {
    const int g = idx / D, e = idx % D;
    a.v_cache[(((size_t)b * a.cache_len + p) * a.Hkv + g) * D + e] = a.v_new[((size_t)b * a.Hkv + g) * D + e];
  }
}

}  // namespace

cudaError_t launch_rope_append(const AppendArgs& a, int D, cudaStream_t stream) {
  if (D == 128)
    rope_append_kernel<128><<<a.B, 128, 0, stream>>>(a);
  else
    rope_append_kernel<64><<<a.B, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace jl
