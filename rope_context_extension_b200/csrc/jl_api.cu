// C ABI of libjetlong.so: argument checks, position maps, scratch layout,
// tensor-map encoding and kernel launches.  See include/jl_api.h.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/jl_api.h"
#include "jl_kernels.cuh"

namespace {

using jl::DecodeArgs;
using jl::PrefillArgs;
using jl::RotateArgs;

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D 16-bit map over [B, rows, H, D] (innermost first: D, H, rows, B) with a
// {64, 1, box_rows, 1} box and 128-byte swizzle.
bool encode_16bit_4d(CUtensorMap* map, const void* base, int D, int H, int64_t rows, int B, int box_rows,
                     CUtensorMapDataType dtype) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)rows * H * D * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_bf16_4d(CUtensorMap* map, const void* base, int D, int H, int64_t rows, int B, int box_rows) {
  return encode_16bit_4d(map, base, D, H, rows, B, box_rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}
bool encode_f16_4d(CUtensorMap* map, const void* base, int D, int H, int64_t rows, int B, int box_rows) {
  return encode_16bit_4d(map, base, D, H, rows, B, box_rows, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

void fill_theta(double* theta, int D, double base) {
  for (int t = 0; t < D / 2; ++t) theta[t] = std::pow(base, -2.0 * t / D);
}

// theta_t / (2 pi) as u_hi + u_lo, u_hi rounded to 22 significant bits (so that
// n * u_hi is exact in fp64 for |n| < 2^31; see sincos_int_angle).
void fill_turns(double* u_hi, double* u_lo, const double* theta, int D) {
  for (int t = 0; t < D / 2; ++t) {
    const double u = theta[t] / 6.283185307179586;
    int e = 0;
    const double m = std::frexp(u, &e);
    u_hi[t] = std::ldexp(std::nearbyint(std::ldexp(m, 22)), e - 22);
    u_lo[t] = u - u_hi[t];
  }
}

constexpr int kMaxGridYZ = 65535;  // CUDA's limit on a grid's y and z dimensions

int common_checks(int B, int L, int Hq, int Hkv, int D, int w0, int w_pretrained, double rope_base, int mode) {
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || w0 < 0 || w_pretrained < 1) return JL_ERR_INVALID_ARG;
  if (!(rope_base > 0.0) || !std::isfinite(rope_base)) return JL_ERR_INVALID_ARG;
  if ((mode & ~(JL_QSHIFT_SELF_EXTEND | JL_PREFILL_FP16 | JL_PREFILL_KEYS_IN_KERNEL)) != 0) return JL_ERR_INVALID_ARG;
  if ((mode & JL_PREFILL_FP16) && (mode & JL_PREFILL_KEYS_IN_KERNEL)) return JL_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return JL_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return JL_ERR_UNSUPPORTED;
  if (L > (1 << 30)) return JL_ERR_UNSUPPORTED;
  if (B > kMaxGridYZ || Hkv > kMaxGridYZ) return JL_ERR_UNSUPPORTED;  // grid y / z dimensions
  return JL_OK;
}

float resolve_scale(float s, int D) { return s == 0.f ? 1.0f / std::sqrt((float)D) : s; }

// Upper bound of the decode split count (sizes the scratch): two CTA waves
// over all (batch, KV head) pairs at two CTAs per SM.  The scratch is then at
// most about 2 * 2 * SMs * r * (D + 2) * 4 bytes (2.5 MB at r = 8, D = 128).
int decode_splits_max(int B, int Hkv) {
  const int slots = 2 * device_sms();
  int s = (2 * slots + B * Hkv - 1) / (B * Hkv);
  if (s < 1) s = 1;
  if (s > 2048) s = 2048;  // the final merge keeps r x splits weights in shared memory
  return s;
}

// Split count for one call: whole decode tiles per split, and the CTA count
// chosen so the last wave on the GPU is as full as possible (at least four
// tiles per split so the per-CTA set-up stays small).
int decode_splits(int B, int Hkv, int ntiles) {
  const int n = B * Hkv;
  const int slots = jl::decode_ctas_per_sm() * device_sms();
  const int smax = std::min(decode_splits_max(B, Hkv), std::max(1, ntiles / 4));
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= smax; ++s) {
    const long ctas = (long)n * s;
    const long waves = (ctas + slots - 1) / slots;
    // time ~ waves x (tiles per split) + a small per-split overhead
    const double per = (double)((ntiles + s - 1) / s) + 2.0;
    const double cost = (double)waves * per;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

struct DecodeLayout {
  size_t counters, ml, o, total;
};
DecodeLayout decode_layout(int B, int Hq, int Hkv, int D, int splits) {
  const int r = Hq / Hkv;
  DecodeLayout lay;
  lay.counters = 0;
  lay.ml = round_up((size_t)B * Hkv * sizeof(int));
  lay.o = lay.ml + round_up((size_t)B * Hkv * splits * r * sizeof(float2));
  lay.total = lay.o + round_up((size_t)B * Hkv * splits * r * D * sizeof(float));
  return lay;
}

}  // namespace

extern "C" {

const char* jl_status_string(int status) {
  switch (status) {
    case JL_OK: return "ok";
    case JL_ERR_INVALID_ARG: return "invalid argument";
    case JL_ERR_UNSUPPORTED: return "unsupported shape";
    case JL_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case JL_ERR_WORKSPACE: return "workspace missing or too small";
    case JL_ERR_CUDA: return "CUDA error";
    case JL_ERR_DEVICE_TIMEOUT: return "device pipeline timeout";
    default: return "unknown status";
  }
}

int jl_group_size(int64_t L, int64_t w_pretrained, int64_t* G_out) {
  if (G_out == nullptr || L < 0 || w_pretrained < 1) return JL_ERR_INVALID_ARG;
  *G_out = jl::group_size(L, w_pretrained);
  return JL_OK;
}

int jl_remote_positions(int64_t L, int64_t w0, int64_t w_pretrained, int mode, int32_t* q_pos_out,
                        int32_t* k_pos_out) {
  if (L < 1 || w0 < 0 || w_pretrained < 1) return JL_ERR_INVALID_ARG;
  if (mode != JL_QSHIFT_NONE && mode != JL_QSHIFT_SELF_EXTEND) return JL_ERR_INVALID_ARG;
  const int64_t G = jl::group_size(L, w_pretrained);
  const int64_t shift = jl::query_shift(w0, G, mode);
  if ((L - 1) / G + shift > INT32_MAX) return JL_ERR_INVALID_ARG;
  for (int64_t i = 0; i < L; ++i) {
    if (q_pos_out) q_pos_out[i] = (int32_t)jl::query_remote(i, G, shift);
    if (k_pos_out) k_pos_out[i] = (int32_t)jl::key_remote(i, G);
  }
  return JL_OK;
}

int jl_prefill_tile_classes(int64_t L, int64_t w0, int64_t w_pretrained, int64_t* counts_out) {
  if (counts_out == nullptr || L < 1 || L > (int64_t(1) << 30) || w0 < 0 || w_pretrained < 1)
    return JL_ERR_INVALID_ARG;
  const int64_t G = jl::group_size(L, w_pretrained);
  const bool al = jl::all_local(L, w0, G);
  // the band width the attention launch hands the kernel
  const int w0k = al ? (1 << 30) : (int)w0;
  int64_t loc_only = 0, both = 0, rem_only = 0, passes = 0;
  for (int mb = 0; mb < (int)((L + 127) / 128); ++mb) {
    const int last = (int)std::min<int64_t>(mb * 128 + 127, L - 1);
    const jl::Sched s = jl::make_sched<jl::kBifocal>(mb * 128, last, w0k, al);
    // local passes visit blocks nb_max - n_loc + 1 .. nb_max, remote passes 0 .. nb_rem_max
    int ov = 0;
    if (s.n_loc > 0 && s.n_rem > 0) {
      const int lo = s.nb_max - s.n_loc + 1;
      const int hi = s.nb_rem_max < s.nb_max ? s.nb_rem_max : s.nb_max;
      ov = hi >= lo ? hi - lo + 1 : 0;
    }
    both += ov;
    loc_only += s.n_loc - ov;
    rem_only += s.n_rem - ov;
    passes += s.n_loc + s.n_rem;
  }
  counts_out[0] = loc_only;
  counts_out[1] = both;
  counts_out[2] = rem_only;
  counts_out[3] = passes;
  return JL_OK;
}

}  // extern "C"

namespace {

// Prefill scratch:
//   default                   corrected key rows as fp16 hi [B, Lk, Hkv, D], then lo
//   JL_PREFILL_FP16           fp16 corrected query rows [B, Lq, Hq, D], then fp16
//                             corrected key rows [B, Lk, Hkv, D]
//   JL_PREFILL_KEYS_IN_KERNEL none (both sides corrected inside the attention kernel)
size_t prefill_ws_fp16(int B, int Lq, int Lk, int Hq, int Hkv, int D) {
  return round_up((size_t)B * Lq * Hq * D * 2) + round_up((size_t)B * Lk * Hkv * D * 2);
}
size_t prefill_ws_prerot(int B, int Lk, int Hkv, int D) { return 2 * round_up((size_t)B * Lk * Hkv * D * 2); }
size_t prefill_ws_any(int B, int Lq, int Lk, int Hq, int Hkv, int D) {
  return std::max(prefill_ws_fp16(B, Lq, Lk, Hq, Hkv, D), prefill_ws_prerot(B, Lk, Hkv, D));
}

}  // namespace

extern "C" {

size_t jl_prefill_workspace_bytes(int B, int L, int Hq, int Hkv, int head_dim) {
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || head_dim < 1) return 0;
  return prefill_ws_any(B, L, L, Hq, Hkv, head_dim);
}

size_t jl_prefill_chunk_workspace_bytes(int B, int q_offset, int chunk_len, int Hq, int Hkv, int head_dim) {
  if (B < 1 || q_offset < 0 || chunk_len < 1 || Hq < 1 || Hkv < 1 || head_dim < 1) return 0;
  return prefill_ws_any(B, chunk_len, q_offset + chunk_len, Hq, Hkv, head_dim);
}

namespace {

// One prefill problem: query rows [q_off, q_off + Lq) of every sequence
// against keys [0, q_off + Lq); Q / O / LSE hold Lq rows, K / V hold k_rows
// rows (>= q_off + Lq).  G comes from the total length q_off + Lq.
struct PrefillProblem {
  const void* q;
  const void* k;
  const void* v;
  int B, q_off, Lq, k_rows, Hq, Hkv, D;
  int Lk() const { return q_off + Lq; }
};

bool prefill_all_local(const PrefillProblem& pp, int w0, int w_pretrained) {
  return jl::all_local(pp.Lk(), w0, jl::group_size(pp.Lk(), w_pretrained));
}

// Scratch the call needs in this mode (0 with the keys corrected inside the
// kernel and whenever every pair is local).
size_t prefill_ws_need(const PrefillProblem& pp, int w0, int w_pretrained, int mode) {
  if (prefill_all_local(pp, w0, w_pretrained)) return 0;
  if (mode & JL_PREFILL_FP16) return prefill_ws_fp16(pp.B, pp.Lq, pp.Lk(), pp.Hq, pp.Hkv, pp.D);
  if (mode & JL_PREFILL_KEYS_IN_KERNEL) return 0;
  return prefill_ws_prerot(pp.B, pp.Lk(), pp.Hkv, pp.D);
}

__half* ws_first(void* ws) { return reinterpret_cast<__half*>(ws); }
__half* ws_second(void* ws, size_t first_bytes) {
  return reinterpret_cast<__half*>(reinterpret_cast<char*>(ws) + round_up(first_bytes));
}

int problem_checks(const PrefillProblem& pp, int w0, int w_pretrained, double rope_base, int mode) {
  int st = common_checks(pp.B, pp.Lk(), pp.Hq, pp.Hkv, pp.D, w0, w_pretrained, rope_base, mode);
  if (st != JL_OK) return st;
  if (pp.q_off < 0 || pp.Lq < 1 || pp.k_rows < pp.Lk()) return JL_ERR_INVALID_ARG;
  // attention grid: (query heads or head pairs, 128-row query blocks, batch),
  // with a 32-bit linear CTA index
  const int64_t blocks = ((int64_t)pp.Lq + 127) / 128;
  if (blocks > kMaxGridYZ || (int64_t)pp.Hq * blocks * pp.B > INT32_MAX) return JL_ERR_UNSUPPORTED;
  if (!pp.q || !pp.k || !pp.v) return JL_ERR_INVALID_ARG;
  if (!aligned16(pp.q) || !aligned16(pp.k) || !aligned16(pp.v)) return JL_ERR_ALIGNMENT;
  return JL_OK;
}

int workspace_checks(const PrefillProblem& pp, int w0, int w_pretrained, int mode, const void* workspace,
                     size_t workspace_bytes) {
  const size_t need = prefill_ws_need(pp, w0, w_pretrained, mode);
  if (need == 0) return JL_OK;
  if (!workspace || workspace_bytes < need) return JL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return JL_ERR_ALIGNMENT;
  return JL_OK;
}

// Correction pass: fp16 hi + lo key rows (default), fp16 query and key rows
// (JL_PREFILL_FP16), nothing with JL_PREFILL_KEYS_IN_KERNEL.  all_keys: every
// key row (the inclusion-exclusion call B scores every causal pair remotely),
// not only those with a remote partner.
int correction_launch(const PrefillProblem& pp, int w0, int w_pretrained, double rope_base, int mode,
                      void* workspace, int* dev_error, cudaStream_t s, bool all_keys = false) {
  if (prefill_all_local(pp, w0, w_pretrained)) return JL_OK;  // nothing to correct
  if (mode & JL_PREFILL_KEYS_IN_KERNEL) return JL_OK;
  const int64_t G = jl::group_size(pp.Lk(), w_pretrained);
  RotateArgs ra;
  std::memset(&ra, 0, sizeof(ra));
  fill_theta(ra.theta, pp.D, rope_base);
  fill_turns(ra.u_hi, ra.u_lo, ra.theta, pp.D);
  ra.G = G;
  ra.shift = jl::query_shift(w0, G, mode & JL_QSHIFT_SELF_EXTEND);
  ra.B = pp.B;
  ra.dev_error = dev_error;
  const size_t kbytes = (size_t)pp.B * pp.Lk() * pp.Hkv * pp.D * 2;
  if (mode & JL_PREFILL_FP16) {
    // queries that have a remote key: positions q_off + r >= w0
    ra.x = reinterpret_cast<const __nv_bfloat16*>(pp.q);
    ra.y = ws_first(workspace);
    ra.y_lo = nullptr;
    ra.x_rows = ra.y_rows = pp.Lq;
    ra.H = pp.Hq;
    ra.pos_off = pp.q_off;
    ra.row_begin = std::max(0, w0 - pp.q_off);
    ra.row_end = pp.Lq;
    ra.is_query = 1;
    if (jl::launch_rotate_rows(ra, pp.D, s) != cudaSuccess) return JL_ERR_CUDA;
  }
  // keys that have a remote query: j <= q_off + Lq - 1 - w0
  ra.x = reinterpret_cast<const __nv_bfloat16*>(pp.k);
  if (mode & JL_PREFILL_FP16) {
    ra.y = ws_second(workspace, (size_t)pp.B * pp.Lq * pp.Hq * pp.D * 2);
    ra.y_lo = nullptr;
  } else {
    ra.y = ws_first(workspace);
    ra.y_lo = ws_second(workspace, kbytes);
  }
  ra.x_rows = pp.k_rows;
  ra.y_rows = pp.Lk();
  ra.H = pp.Hkv;
  ra.pos_off = 0;
  ra.row_begin = 0;
  ra.row_end = all_keys ? pp.Lk() : pp.Lk() - w0;
  ra.is_query = 0;
  if (jl::launch_rotate_rows(ra, pp.D, s) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

// Host tables of the in-kernel correction: R(-theta_t b) for b < 16 and
// R(-theta_t 16 a) for a < 8, formed in fp64 and rounded to fp32.
void fill_hilo_tables(jl::PrefillHiloArgs& a, int D, double rope_base) {
  fill_theta(a.theta, D, rope_base);
  fill_turns(a.u_hi, a.u_lo, a.theta, D);
  for (int t = 0; t < D / 2; ++t) {
    for (int b = 0; b < 16; ++b)
      a.t1[t * 16 + b] = make_float2((float)std::cos(b * a.theta[t]), (float)-std::sin(b * a.theta[t]));
    for (int m = 0; m < 8; ++m)
      a.t16[t * 8 + m] = make_float2((float)std::cos(16.0 * m * a.theta[t]), (float)-std::sin(16.0 * m * a.theta[t]));
  }
}

// The attention launch.  Every pair local: the two-heads-per-CTA kernel on the
// bf16 inputs (plain causal RoPE, no rounding of operands).  JL_PREFILL_FP16:
// the same kernel on the fp16 rows of the correction pass.  Otherwise the hi +
// lo kernel, correcting the query block itself and taking the key rows' hi /
// lo parts from the workspace (or, with JL_PREFILL_KEYS_IN_KERNEL, correcting
// the key tiles itself too).  o_f32 (inclusion-exclusion partials) writes fp32
// instead of bf16 output.
int attention_launch(const PrefillProblem& pp, void* o, float* o_f32, float* lse, int w0, int w_pretrained,
                     double rope_base, float softmax_scale, int mode, const void* workspace, int* dev_error,
                     cudaStream_t stream, int kind = jl::kBifocal) {
  const int D = pp.D;
  const int64_t G = jl::group_size(pp.Lk(), w_pretrained);
  const bool all_local = kind == jl::kBifocal && jl::all_local(pp.Lk(), w0, G);
  const int r = pp.Hq / pp.Hkv;
  const float scale_log2 = resolve_scale(softmax_scale, D) * 1.4426950408889634f;
  CUtensorMap tk, tv;
  if (!encode_bf16_4d(&tk, pp.k, D, pp.Hkv, pp.k_rows, pp.B, 128) ||
      !encode_bf16_4d(&tv, pp.v, D, pp.Hkv, pp.k_rows, pp.B, 128))
    return JL_ERR_CUDA;
  if (all_local || (mode & JL_PREFILL_FP16)) {
    if (kind != jl::kBifocal || o_f32 != nullptr) return JL_ERR_INVALID_ARG;
    CUtensorMap tq, tqr, tkr;
    if (!encode_bf16_4d(&tq, pp.q, D, pp.Hq, pp.Lq, pp.B, 128)) return JL_ERR_CUDA;
    if (!all_local) {
      void* ws = const_cast<void*>(workspace);
      if (!encode_f16_4d(&tqr, ws_first(ws), D, pp.Hq, pp.Lq, pp.B, 128) ||
          !encode_f16_4d(&tkr, ws_second(ws, (size_t)pp.B * pp.Lq * pp.Hq * pp.D * 2), D, pp.Hkv, pp.Lk(), pp.B,
                         128))
        return JL_ERR_CUDA;
    } else {
      tqr = tq;
      tkr = tk;
    }
    PrefillArgs pa;
    std::memset(&pa, 0, sizeof(pa));
    pa.o = reinterpret_cast<__nv_bfloat16*>(o);
    pa.lse = lse;
    pa.dev_error = dev_error;
    pa.B = pp.B;
    pa.Hq = pp.Hq;
    pa.Hkv = pp.Hkv;
    pa.r = r;
    pa.q_off = pp.q_off;
    pa.Lq = pp.Lq;
    pa.Lk = pp.Lk();
    pa.nh = r % 2 == 0 ? 2 : 1;
    pa.num_mb = (pp.Lq + 127) / 128;
    pa.all_local = all_local ? 1 : 0;
    pa.w0 = all_local ? (1 << 30) : w0;
    pa.scale_log2 = scale_log2;
    if (jl::launch_prefill(tq, tqr, tk, tkr, tv, pa, D, stream) != cudaSuccess) return JL_ERR_CUDA;
    return JL_OK;
  }
  const bool rot_k = (mode & JL_PREFILL_KEYS_IN_KERNEL) != 0;
  CUtensorMap tkh = tk, tkl = tk;
  if (!rot_k) {
    void* ws = const_cast<void*>(workspace);
    const size_t kbytes = (size_t)pp.B * pp.Lk() * pp.Hkv * pp.D * 2;
    if (!encode_f16_4d(&tkh, ws_first(ws), D, pp.Hkv, pp.Lk(), pp.B, 128) ||
        !encode_f16_4d(&tkl, ws_second(ws, kbytes), D, pp.Hkv, pp.Lk(), pp.B, 128))
      return JL_ERR_CUDA;
  }
  static_assert(sizeof(jl::PrefillHiloArgs) + 4 * sizeof(CUtensorMap) <= 32764, "kernel parameters too large");
  jl::PrefillHiloArgs ha;
  std::memset(&ha, 0, sizeof(ha));
  ha.q = reinterpret_cast<const __nv_bfloat16*>(pp.q);
  ha.k = reinterpret_cast<const __nv_bfloat16*>(pp.k);
  ha.o = reinterpret_cast<__nv_bfloat16*>(o);
  ha.o_f32 = o_f32;
  ha.lse = lse;
  ha.dev_error = dev_error;
  ha.B = pp.B;
  ha.Hq = pp.Hq;
  ha.Hkv = pp.Hkv;
  ha.r = r;
  ha.q_off = pp.q_off;
  ha.Lq = pp.Lq;
  ha.k_rows = pp.k_rows;
  ha.num_mb = (pp.Lq + 127) / 128;
  ha.w0 = w0;
  ha.kind = kind;
  ha.G = G;
  ha.shift = jl::query_shift(w0, G, mode & JL_QSHIFT_SELF_EXTEND);
  ha.scale_log2 = scale_log2;
  fill_hilo_tables(ha, D, rope_base);
  if (jl::launch_prefill_hilo(tk, tv, tkh, tkl, ha, D, rot_k, stream) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

int prefill_entry(const PrefillProblem& pp, void* o, float* lse, int w0, int w_pretrained, double rope_base,
                  float softmax_scale, int mode, void* workspace, size_t workspace_bytes, int* dev_error,
                  void* stream, bool correct, bool attend) {
  // Validate everything before the first launch.
  int st = problem_checks(pp, w0, w_pretrained, rope_base, mode);
  if (st != JL_OK) return st;
  if (attend) {
    if (!o) return JL_ERR_INVALID_ARG;
    if (!aligned16(o) || (lse && ((uintptr_t)lse & 3u))) return JL_ERR_ALIGNMENT;
  }
  st = workspace_checks(pp, w0, w_pretrained, mode, workspace, workspace_bytes);
  if (st != JL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (correct) {
    st = correction_launch(pp, w0, w_pretrained, rope_base, mode, workspace, dev_error, s);
    if (st != JL_OK) return st;
  }
  if (attend)
    return attention_launch(pp, o, nullptr, lse, w0, w_pretrained, rope_base, softmax_scale, mode, workspace,
                            dev_error, s);
  return JL_OK;
}

}  // namespace

int jl_prefill_correction(const void* q, const void* k, int B, int L, int Hq, int Hkv, int head_dim, int w0,
                          int w_pretrained, double rope_base, int mode, void* workspace, size_t workspace_bytes,
                          int* dev_error, void* stream) {
  const PrefillProblem pp{q, k, k, B, 0, L, L, Hq, Hkv, head_dim};
  return prefill_entry(pp, nullptr, nullptr, w0, w_pretrained, rope_base, 0.f, mode, workspace, workspace_bytes,
                       dev_error, stream, true, false);
}

int jl_prefill_attention(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L, int Hq,
                         int Hkv, int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale,
                         int mode, const void* workspace, size_t workspace_bytes, int* dev_error, void* stream) {
  const PrefillProblem pp{q, k, v, B, 0, L, L, Hq, Hkv, head_dim};
  return prefill_entry(pp, o, lse, w0, w_pretrained, rope_base, softmax_scale, mode, const_cast<void*>(workspace),
                       workspace_bytes, dev_error, stream, false, true);
}

int jl_bifocal_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L, int Hq,
                       int Hkv, int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale,
                       int mode, void* workspace, size_t workspace_bytes, int* dev_error, void* stream) {
  const PrefillProblem pp{q, k, v, B, 0, L, L, Hq, Hkv, head_dim};
  return prefill_entry(pp, o, lse, w0, w_pretrained, rope_base, softmax_scale, mode, workspace, workspace_bytes,
                       dev_error, stream, true, true);
}

int jl_bifocal_prefill_chunk(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len, void* o,
                             float* lse, int B, int q_offset, int chunk_len, int Hq, int Hkv, int head_dim, int w0,
                             int w_pretrained, double rope_base, float softmax_scale, int mode, void* workspace,
                             size_t workspace_bytes, int* dev_error, void* stream) {
  if (cache_len < 1 || cache_len > ((int64_t)1 << 30)) return JL_ERR_INVALID_ARG;
  if (q_offset < 0 || chunk_len < 1 || (int64_t)q_offset + chunk_len > cache_len) return JL_ERR_INVALID_ARG;
  const PrefillProblem pp{q, k_cache, v_cache, B, q_offset, chunk_len, (int)cache_len, Hq, Hkv, head_dim};
  return prefill_entry(pp, o, lse, w0, w_pretrained, rope_base, softmax_scale, mode, workspace, workspace_bytes,
                       dev_error, stream, true, true);
}

namespace {

struct IeLayout {
  size_t keys, o[3], lse[3], total;
};
// Corrected key rows (hi + lo, every row), then three fp32 partial outputs and
// their LSEs.
IeLayout ie_layout(int B, int L, int Hq, int Hkv, int D) {
  IeLayout lay;
  size_t off = 0;
  lay.keys = off;
  off += prefill_ws_prerot(B, L, Hkv, D);
  for (int x = 0; x < 3; ++x) {
    lay.o[x] = off;
    off += round_up((size_t)B * L * Hq * D * 4);
  }
  for (int x = 0; x < 3; ++x) {
    lay.lse[x] = off;
    off += round_up((size_t)B * Hq * L * 4);
  }
  lay.total = off;
  return lay;
}

}  // namespace

size_t jl_prefill_ie_workspace_bytes(int B, int L, int Hq, int Hkv, int head_dim, int mode) {
  (void)mode;
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || head_dim < 1) return 0;
  return ie_layout(B, L, Hq, Hkv, head_dim).total;
}

int jl_bifocal_prefill_ie(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L, int Hq,
                          int Hkv, int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale,
                          int mode, void* workspace, size_t workspace_bytes, int* dev_error, void* stream) {
  const PrefillProblem pp{q, k, v, B, 0, L, L, Hq, Hkv, head_dim};
  int st = problem_checks(pp, w0, w_pretrained, rope_base, mode);
  if (st != JL_OK) return st;
  if (!o) return JL_ERR_INVALID_ARG;
  if (!aligned16(o) || (lse && ((uintptr_t)lse & 3u))) return JL_ERR_ALIGNMENT;
  const int qmode = mode & JL_QSHIFT_SELF_EXTEND;  // the three calls always use the default (hi + lo) path
  const int64_t G = jl::group_size(L, w_pretrained);
  if (jl::all_local(L, w0, G)) {
    // every pair local: the three calls collapse to plain causal attention
    return jl_bifocal_prefill(q, k, v, o, lse, B, L, Hq, Hkv, head_dim, w0, w_pretrained, rope_base, softmax_scale,
                              qmode, nullptr, 0, dev_error, stream);
  }
  const IeLayout lay = ie_layout(B, L, Hq, Hkv, head_dim);
  if (!workspace || workspace_bytes < lay.total) return JL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return JL_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = reinterpret_cast<char*>(workspace);
  st = correction_launch(pp, w0, w_pretrained, rope_base, qmode, ws + lay.keys, dev_error, s, /*all_keys=*/true);
  if (st != JL_OK) return st;
  const int kinds[3] = {jl::kWindowBase, jl::kCausalRemote, jl::kWindowRemote};
  jl::MergeArgs ma;
  std::memset(&ma, 0, sizeof(ma));
  for (int x = 0; x < 3; ++x) {
    float* ox = reinterpret_cast<float*>(ws + lay.o[x]);
    float* lx = reinterpret_cast<float*>(ws + lay.lse[x]);
    st = attention_launch(pp, nullptr, ox, lx, w0, w_pretrained, rope_base, softmax_scale, qmode, ws + lay.keys,
                          dev_error, s, kinds[x]);
    if (st != JL_OK) return st;
    ma.o_x[x] = ox;
    ma.lse_x[x] = lx;
  }
  ma.o = reinterpret_cast<__nv_bfloat16*>(o);
  ma.lse = lse;
  ma.B = B;
  ma.L = L;
  ma.Hq = Hq;
  if (jl::launch_ie_merge(ma, head_dim, s) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

size_t jl_decode_workspace_bytes(int B, int L, int Hq, int Hkv, int head_dim) {
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || head_dim < 1 || Hq % Hkv) return 0;
  return decode_layout(B, Hq, Hkv, head_dim, decode_splits_max(B, Hkv)).total;
}

namespace {

// Shared by the uniform-length and the varlen decode entry points.
// compact = false: the workspace has the layout jl_decode_workspace_bytes sizes
// (room for decode_splits_max splits).  compact = true (fixed scratch of the
// no-allocation entry point): the layout holds exactly the split count this
// call uses, which is lowered until that layout fits in workspace_bytes, and
// the ticket counters are cleared on the stream before the launch.
int decode_launch(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len,
                  const int32_t* seq_lens, int L, void* o, float* lse, int B, int Hq, int Hkv, int D, int w0,
                  int w_pretrained, double rope_base, float softmax_scale, int mode, void* workspace,
                  size_t workspace_bytes, int* dev_error, void* stream, int key_off = 0, int L_total = 0,
                  bool compact = false) {
  int st = common_checks(B, L_total > 0 ? L_total : L, Hq, Hkv, D, w0, w_pretrained, rope_base, mode);
  if (st == JL_OK && L < 1) st = JL_ERR_INVALID_ARG;
  if (st != JL_OK) return st;
  if (!q || !k_cache || !v_cache || !o) return JL_ERR_INVALID_ARG;
  if (cache_len < L || cache_len > (int64_t)1 << 31) return JL_ERR_INVALID_ARG;
  if (Hq / Hkv > 8) return JL_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (lse && ((uintptr_t)lse & 3u)) || (seq_lens && ((uintptr_t)seq_lens & 3u)))
    return JL_ERR_ALIGNMENT;
  const int tk_keys = jl::decode_tile_keys();
  const int ntiles = (L + tk_keys - 1) / tk_keys;
  int splits = decode_splits(B, Hkv, ntiles);
  if (compact) {
    while (splits > 1 && decode_layout(B, Hq, Hkv, D, splits).total > workspace_bytes) --splits;
  }
  const DecodeLayout lay = decode_layout(B, Hq, Hkv, D, compact ? splits : decode_splits_max(B, Hkv));
  if (!workspace || workspace_bytes < lay.total) return JL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return JL_ERR_ALIGNMENT;

  CUtensorMap tk, tv;
  if (!encode_bf16_4d(&tk, k_cache, D, Hkv, cache_len, B, tk_keys) ||
      !encode_bf16_4d(&tv, v_cache, D, Hkv, cache_len, B, tk_keys))
    return JL_ERR_CUDA;

  DecodeArgs a;
  std::memset(&a, 0, sizeof(a));
  char* ws = reinterpret_cast<char*>(workspace);
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.o = reinterpret_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.counters = reinterpret_cast<int*>(ws + lay.counters);
  a.part_ml = reinterpret_cast<float2*>(ws + lay.ml);
  a.part_o = reinterpret_cast<float*>(ws + lay.o);
  a.dev_error = dev_error;
  a.seq_lens = seq_lens;
  a.key_off = key_off;
  a.L_total = L_total;
  a.B = B;
  a.L = L;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.r = Hq / Hkv;
  a.cache_len = cache_len;
  a.splits = splits;
  a.w0 = w0;
  a.w_pretrained = w_pretrained;
  a.qshift = mode & JL_QSHIFT_SELF_EXTEND;
  a.scale_log2 = resolve_scale(softmax_scale, D) * 1.4426950408889634f;
  fill_theta(a.theta, D, rope_base);
  fill_turns(a.u_hi, a.u_lo, a.theta, D);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (compact && cudaMemsetAsync(a.counters, 0, (size_t)B * Hkv * sizeof(int), s) != cudaSuccess)
    return JL_ERR_CUDA;
  if (jl::launch_decode(tk, tv, a, D, s) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

}  // namespace

}  // extern "C"

namespace jl {

int decode_in_fixed_scratch(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len, void* o,
                            float* lse, int B, int L, int Hq, int Hkv, int head_dim, int w0, int w_pretrained,
                            double rope_base, float softmax_scale, int mode, void* scratch, size_t scratch_bytes,
                            int* dev_error, void* stream) {
  return decode_launch(q, k_cache, v_cache, cache_len, nullptr, L, o, lse, B, Hq, Hkv, head_dim, w0, w_pretrained,
                       rope_base, softmax_scale, mode, scratch, scratch_bytes, dev_error, stream, 0, 0,
                       /*compact=*/true);
}

}  // namespace jl

extern "C" {

int jl_bifocal_decode(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len, void* o,
                      float* lse, int B, int L, int Hq, int Hkv, int head_dim, int w0, int w_pretrained,
                      double rope_base, float softmax_scale, int mode, void* workspace, size_t workspace_bytes,
                      int* dev_error, void* stream) {
  return decode_launch(q, k_cache, v_cache, cache_len, nullptr, L, o, lse, B, Hq, Hkv, head_dim, w0, w_pretrained,
                       rope_base, softmax_scale, mode, workspace, workspace_bytes, dev_error, stream);
}

int jl_bifocal_decode_varlen(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len,
                             const int32_t* seq_lens, int max_len, void* o, float* lse, int B, int Hq, int Hkv,
                             int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale, int mode,
                             void* workspace, size_t workspace_bytes, int* dev_error, void* stream) {
  if (seq_lens == nullptr) return JL_ERR_INVALID_ARG;
  return decode_launch(q, k_cache, v_cache, cache_len, seq_lens, max_len, o, lse, B, Hq, Hkv, head_dim, w0,
                       w_pretrained, rope_base, softmax_scale, mode, workspace, workspace_bytes, dev_error, stream);
}

int jl_bifocal_decode_range(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len,
                            int key_offset, int key_count, int total_len, void* o, float* lse, int B, int Hq, int Hkv,
                            int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale, int mode,
                            void* workspace, size_t workspace_bytes, int* dev_error, void* stream) {
  if (key_offset < 0 || key_count < 1 || total_len < 1) return JL_ERR_INVALID_ARG;
  if ((int64_t)key_offset + key_count > total_len || key_count > cache_len) return JL_ERR_INVALID_ARG;
  return decode_launch(q, k_cache, v_cache, cache_len, nullptr, key_count, o, lse, B, Hq, Hkv, head_dim, w0,
                       w_pretrained, rope_base, softmax_scale, mode, workspace, workspace_bytes, dev_error, stream,
                       key_offset, total_len);
}

int jl_decode_combine(const void* o_parts, const float* lse_parts, int parts, void* o, float* lse, int B, int Hq,
                      int head_dim, void* stream) {
  if (parts < 1 || B < 1 || Hq < 1 || !o_parts || !lse_parts || !o) return JL_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return JL_ERR_UNSUPPORTED;
  if (!aligned16(o_parts) || !aligned16(o) || ((uintptr_t)lse_parts & 3u) || (lse && ((uintptr_t)lse & 3u)))
    return JL_ERR_ALIGNMENT;
  jl::CombineArgs a;
  a.o_parts = reinterpret_cast<const __nv_bfloat16*>(o_parts);
  a.lse_parts = lse_parts;
  a.o = reinterpret_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.R = parts;
  a.B = B;
  a.Hq = Hq;
  if (jl::launch_lse_combine(a, head_dim, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

int jl_wait_timeout_check(int* dev_error, double timeout_s, void* stream) {
  if (!dev_error || !(timeout_s > 0.0) || timeout_s > 10.0) return JL_ERR_INVALID_ARG;
  if (jl::launch_wait_timeout_check(dev_error, (unsigned long long)(timeout_s * 1e9),
                                    reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JL_ERR_CUDA;
  return JL_OK;
}

int jl_rope_append(const void* q_raw, const void* k_raw, const void* v_new, const int32_t* positions, void* q_out,
                   void* k_cache, void* v_cache, int64_t cache_len, int B, int Hq, int Hkv, int head_dim,
                   double rope_base, int* dev_error, void* stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || cache_len < 1 || cache_len > (int64_t)1 << 31) return JL_ERR_INVALID_ARG;
  if (!(rope_base > 0.0) || !std::isfinite(rope_base)) return JL_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return JL_ERR_UNSUPPORTED;
  if (!q_raw || !k_raw || !v_new || !positions || !q_out || !k_cache || !v_cache) return JL_ERR_INVALID_ARG;
  if (!aligned16(q_raw) || !aligned16(k_raw) || !aligned16(v_new) || !aligned16(q_out) || !aligned16(k_cache) ||
      !aligned16(v_cache) || ((uintptr_t)positions & 3u))
    return JL_ERR_ALIGNMENT;
  jl::AppendArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q_raw = reinterpret_cast<const __nv_bfloat16*>(q_raw);
  a.k_raw = reinterpret_cast<const __nv_bfloat16*>(k_raw);
  a.v_new = reinterpret_cast<const __nv_bfloat16*>(v_new);
  a.positions = positions;
  a.q_out = reinterpret_cast<__nv_bfloat16*>(q_out);
  a.k_cache = reinterpret_cast<__nv_bfloat16*>(k_cache);
  a.v_cache = reinterpret_cast<__nv_bfloat16*>(v_cache);
  a.cache_len = cache_len;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.dev_error = dev_error;
  fill_theta(a.theta, head_dim, rope_base);
  fill_turns(a.u_hi, a.u_lo, a.theta, head_dim);
  if (jl::launch_rope_append(a, head_dim, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

}  // extern "C"
