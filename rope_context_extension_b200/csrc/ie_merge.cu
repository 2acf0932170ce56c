// Log-sum-exp merges: the inclusion-exclusion merge of the three calls of the
// pages' prefill formulation, and the combine of a sequence-split decode.
//
// Inclusion-exclusion merge of the three calls of the pages' prefill
// formulation (Jet-Long review, "Method"):
//   O = (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C),  W_X = exp(LSE_X - M),
//   LSE = M + ln(W_A + W_B - W_C),  M = max(LSE_A, LSE_B, LSE_C),
// where A is the window with base RoPE, B every causal pair with remote
// positions and C the window with remote positions; C removes exactly the part
// of B that A replaces.  The three partial outputs arrive in fp32 (the remote
// calls' scores carry hi + lo operands), so what the subtraction W_B O_B -
// W_C O_C amplifies is fp32 rounding; where W_B and W_C nearly cancel (a key
// that dominates both sits in the window) that still grows without bound, a
// property of the formulation.  One warp per (sequence, row, head).
#include "jl_kernels.cuh"

namespace jl {

namespace {

template <int D>
__global__ void __launch_bounds__(256) ie_merge_kernel(const __grid_constant__ MergeArgs a) {
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)a.B * a.L * a.Hq;
  if (warp_global >= rows) return;
  const int h = (int)(warp_global % a.Hq);
  const int64_t bi = warp_global / a.Hq;
  const int i = (int)(bi % a.L);
  const int b = (int)(bi / a.L);
  const size_t lidx = ((size_t)b * a.Hq + h) * a.L + i;
  const float la = a.lse_x[0][lidx], lb = a.lse_x[1][lidx], lc = a.lse_x[2][lidx];
  const float M = fmaxf(fmaxf(la, lb), lc);
  const float wa = la == -INFINITY ? 0.f : expf(la - M);
  const float wb = lb == -INFINITY ? 0.f : expf(lb - M);
  const float wc = lc == -INFINITY ? 0.f : expf(lc - M);
  const float den = wa + wb - wc;
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const size_t obase = ((size_t)bi * a.Hq + h) * D;
  constexpr int kPer = D / 32;  // elements per lane
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const int d = lane + 32 * e;
    const float oa = a.o_x[0][obase + d];
    const float ob = a.o_x[1][obase + d];
    const float oc = a.o_x[2][obase + d];
    a.o[obase + d] = __float2bfloat16_rn((wa * oa + wb * ob - wc * oc) * inv);
  }
  if (lane == 0 && a.lse != nullptr) a.lse[lidx] = M + logf(den);
}

// O = sum_r exp(LSE_r - M) O_r / sum_r exp(LSE_r - M), LSE = M + ln(sum ...):
// partial results over disjoint key ranges of one query (a sequence-split
// decode), one warp per (sequence, head).
template <int D>
__global__ void __launch_bounds__(256) lse_combine_kernel(const __grid_constant__ CombineArgs a) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = a.B * a.Hq;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int r = 0; r < a.R; ++r) M = fmaxf(M, a.lse_parts[(size_t)r * rows + row]);
  float den = 0.f;
  for (int r = 0; r < a.R; ++r) {
    const float l = a.lse_parts[(size_t)r * rows + row];
    den += l == -INFINITY ? 0.f : expf(l - M);
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  constexpr int kPer = D / 32;
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const int d = lane + 32 * e;
    float acc = 0.f;
    for (int r = 0; r < a.R; ++r) {
      const float l = a.lse_parts[(size_t)r * rows + row];
      const float w = l == -INFINITY ? 0.f : expf(l - M);
      acc += w * __bfloat162float(a.o_parts[((size_t)r * rows + row) * D + d]);
    }
    a.o[(size_t)row * D + d] = __float2bfloat16_rn(acc * inv);
  }
  if (lane == 0 && a.lse != nullptr) a.lse[row] = M + logf(den);
}

// Exercises the pipelines' bounded wait on a barrier that nothing completes:
// warp 0 waits until its limit runs out (it must return false and write the
// timeout code), warp 1 waits on a second such barrier and must give up as soon
// as warp 0 has aborted.  A wait that returned true writes 99 instead.
__global__ void wait_timeout_check_kernel(int* dev_error, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bars[0]), 1);
    mbar_init(smem_addr(&bars[1]), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int w = threadIdx.x >> 5;
  const bool ok = mbar_wait(smem_addr(&bars[w]), 0u, &abort_flag, w == 0 ? dev_error : nullptr,
                            w == 0 ? timeout_ns : 4 * timeout_ns);
  if (ok && (threadIdx.x & 31) == 0) atomicExch(dev_error, 99);
}

}  // namespace

cudaError_t launch_wait_timeout_check(int* dev_error, unsigned long long timeout_ns, cudaStream_t stream) {
  wait_timeout_check_kernel<<<1, 64, 0, stream>>>(dev_error, timeout_ns);
  return cudaGetLastError();
}

cudaError_t launch_lse_combine(const CombineArgs& a, int D, cudaStream_t stream) {
  const int rows = a.B * a.Hq;
  const int blocks = (rows * 32 + 255) / 256;
  if (D == 128)
    lse_combine_kernel<128><<<blocks, 256, 0, stream>>>(a);
  else
    lse_combine_kernel<64><<<blocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ie_merge(const MergeArgs& a, int D, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.B * a.L * a.Hq;
  const int64_t blocks = (rows * 32 + 255) / 256;
  if (D == 128)
    ie_merge_kernel<128><<<(unsigned)blocks, 256, 0, stream>>>(a);
  else
    ie_merge_kernel<64><<<(unsigned)blocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace jl
