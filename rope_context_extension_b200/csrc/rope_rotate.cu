// Correction-rotation pass for bifocal prefill.
//
// For the remote score set each query row i needs R(p_q(i)) q_raw and each key
// j needs R(f(j)) k_raw.  The inputs arrive rotated at their base positions, so
// (RoPE rotations compose additively, gist.science summary "§2 On-the-Fly
// Correctie Rotatie") one rotation by the correction angle dq(i) = p_q(i) - i
// (dk(j) = f(j) - j) turns the base-rotated row into the remote-rotated row.
// This kernel applies that correction once per row and writes the result to
// caller-owned scratch; the input tensors (the KV cache) are never touched.
//
// Angles reach ~1e5 rad at 128K tokens, so they are formed and reduced in fp64
// (one sincos per (row, pair), shared by every head of the row, with the whole
// turns removed exactly first: sincos_int_angle); the rotation
// itself is fp32 and the output is rounded to fp16 (round-to-nearest-even),
// optionally with the rounding residual as a second fp16 row (hi + lo carry
// about 22 significant bits): the rotated rows only feed the score products,
// and fp16 keeps three more mantissa bits than bf16 at the same tensor-core
// rate.  A rotated value beyond fp16's range (|x| >= 65520, reachable from
// inputs of magnitude 46340 or more) cannot be carried: the kernel reports it
// as kDevRange in *dev_error, and the results are invalid.
#include "jl_kernels.cuh"

namespace jl {

namespace {

constexpr int kRotRows = 16;
constexpr int kRotThreads = 256;

template <int D>
__global__ void __launch_bounds__(kRotThreads)
    rotate_rows_kernel(const __grid_constant__ RotateArgs args) {
  constexpr int H2 = D / 2;
  __shared__ float2 cs[kRotRows][H2];

  const int b = blockIdx.y;
  const int row0 = args.row_begin + blockIdx.x * kRotRows;

  for (int idx = threadIdx.x; idx < kRotRows * H2; idx += blockDim.x) {
    const int r = idx / H2, t = idx % H2;
    const int64_t i = row0 + r;
    float2 v = make_float2(1.f, 0.f);
    if (i < args.row_end) {
      const int64_t pos = i + args.pos_off;
      const int64_t target = args.is_query ? query_remote(pos, args.G, args.shift) : key_remote(pos, args.G);
      double s, c;
      sincos_int_angle(target - pos, args.u_hi[t], args.u_lo[t], &s, &c);
      v = make_float2((float)c, (float)s);
    }
    cs[r][t] = v;
  }
  __syncthreads();

  constexpr int kChunks = H2 / 8;  // 8 pairs (16 B of each half) per work item
  const int items = kRotRows * args.H * kChunks;
  uint32_t range = 0;  // bit 15 / 31 set by an fp16 half that is inf or NaN
  for (int w = threadIdx.x; w < items; w += blockDim.x) {
    const int ch = w % kChunks;
    const int h = (w / kChunks) % args.H;
    const int r = w / (kChunks * args.H);
    const int64_t i = row0 + r;
    if (i >= args.row_end) continue;
    const size_t xbase = (((size_t)b * args.x_rows + i) * args.H + h) * D;
    const size_t base = (((size_t)b * args.y_rows + i) * args.H + h) * D;
    const uint4 lo = *reinterpret_cast<const uint4*>(args.x + xbase + ch * 8);
    const uint4 hi = *reinterpret_cast<const uint4*>(args.x + xbase + H2 + ch * 8);
    const uint32_t lw[4] = {lo.x, lo.y, lo.z, lo.w};
    const uint32_t hw[4] = {hi.x, hi.y, hi.z, hi.w};
    float rx[8], ry[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 c0 = cs[r][ch * 8 + 2 * k];
      const float2 c1 = cs[r][ch * 8 + 2 * k + 1];
      const float x0 = bf16lo_to_f32(lw[k]), x1 = bf16hi_to_f32(lw[k]);
      const float y0 = bf16lo_to_f32(hw[k]), y1 = bf16hi_to_f32(hw[k]);
      // (x, y) -> (x cos - y sin, y cos + x sin)
      rx[2 * k] = x0 * c0.x - y0 * c0.y;
      rx[2 * k + 1] = x1 * c1.x - y1 * c1.y;
      ry[2 * k] = y0 * c0.x + x0 * c0.y;
      ry[2 * k + 1] = y1 * c1.x + x1 * c1.y;
    }
    uint32_t lo_out[4], hi_out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      lo_out[k] = pack_f16x2(rx[2 * k], rx[2 * k + 1]);
      hi_out[k] = pack_f16x2(ry[2 * k], ry[2 * k + 1]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      range |= ((lo_out[k] & 0x7FFF7FFFu) + 0x04000400u) | ((hi_out[k] & 0x7FFF7FFFu) + 0x04000400u);
    *reinterpret_cast<uint4*>(args.y + base + ch * 8) = make_uint4(lo_out[0], lo_out[1], lo_out[2], lo_out[3]);
    *reinterpret_cast<uint4*>(args.y + base + H2 + ch * 8) =
        make_uint4(hi_out[0], hi_out[1], hi_out[2], hi_out[3]);
    if (args.y_lo != nullptr) {
      // residuals of the fp16 rounding, themselves rounded to fp16
      uint32_t rl[4], rh[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 a = *reinterpret_cast<const __half2*>(&lo_out[k]);
        const __half2 c = *reinterpret_cast<const __half2*>(&hi_out[k]);
        rl[k] = pack_f16x2(rx[2 * k] - __low2float(a), rx[2 * k + 1] - __high2float(a));
        rh[k] = pack_f16x2(ry[2 * k] - __low2float(c), ry[2 * k + 1] - __high2float(c));
      }
      *reinterpret_cast<uint4*>(args.y_lo + base + ch * 8) = make_uint4(rl[0], rl[1], rl[2], rl[3]);
      *reinterpret_cast<uint4*>(args.y_lo + base + H2 + ch * 8) = make_uint4(rh[0], rh[1], rh[2], rh[3]);
    }
  }
  if ((range & 0x80008000u) != 0u && args.dev_error != nullptr) atomicExch(args.dev_error, kDevRange);
}

}  // namespace

cudaError_t launch_rotate_rows(const RotateArgs& args, int D, cudaStream_t stream) {
  if (args.row_end <= args.row_begin) return cudaSuccess;
  const int rows = args.row_end - args.row_begin;
  dim3 grid((rows + kRotRows - 1) / kRotRows, args.B);
  if (D == 128) {
    rotate_rows_kernel<128><<<grid, kRotThreads, 0, stream>>>(args);
  } else {
    rotate_rows_kernel<64><<<grid, kRotThreads, 0, stream>>>(args);
  }
  return cudaGetLastError();
}

}  // namespace jl
