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

constexpr int kMaxGridYZ = 65535;  // CUDA's limit on a grid's y and z dimensions

int common_checks(int B, int L, int Hq, int Hkv, int D, int w0, int w_pretrained, double rope_base, int mode) {
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || w0 < 0 || w_pretrained < 1) return JL_ERR_INVALID_ARG;
  if (!(rope_base > 0.0) || !std::isfinite(rope_base)) return JL_ERR_INVALID_ARG;
  if ((mode & ~(JL_QSHIFT_SELF_EXTEND | JL_REMOTE_SPLIT)) != 0) return JL_ERR_INVALID_ARG;
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

size_t jl_prefill_workspace_bytes(int B, int L, int Hq, int Hkv, int head_dim) {
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || head_dim < 1) return 0;
  return round_up((size_t)B * L * Hq * head_dim * 2) + round_up((size_t)B * L * Hkv * head_dim * 2);
}

size_t jl_prefill_chunk_workspace_bytes(int B, int q_offset, int chunk_len, int Hq, int Hkv, int head_dim) {
  if (B < 1 || q_offset < 0 || chunk_len < 1 || Hq < 1 || Hkv < 1 || head_dim < 1) return 0;
  return round_up((size_t)B * chunk_len * Hq * head_dim * 2) +
         round_up((size_t)B * ((size_t)q_offset + chunk_len) * Hkv * head_dim * 2);
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
  size_t base_ws() const { return jl_prefill_chunk_workspace_bytes(B, q_off, Lq, Hq, Hkv, D); }
};

__half* q_rem_ptr(void* ws) { return reinterpret_cast<__half*>(ws); }
__half* k_rem_ptr(void* ws, const PrefillProblem& pp) {
  return reinterpret_cast<__half*>(reinterpret_cast<char*>(ws) + round_up((size_t)pp.B * pp.Lq * pp.Hq * pp.D * 2));
}

int problem_checks(const PrefillProblem& pp, int w0, int w_pretrained, double rope_base, int mode) {
  int st = common_checks(pp.B, pp.Lk(), pp.Hq, pp.Hkv, pp.D, w0, w_pretrained, rope_base, mode);
  if (st != JL_OK) return st;
  if (pp.q_off < 0 || pp.Lq < 1 || pp.k_rows < pp.Lk()) return JL_ERR_INVALID_ARG;
  // attention grid: (query-head groups, 128-row query blocks, batch), with a
  // 32-bit linear CTA index
  const int64_t blocks = ((int64_t)pp.Lq + 127) / 128;
  if (blocks > kMaxGridYZ || (int64_t)pp.Hq * blocks * pp.B > INT32_MAX) return JL_ERR_UNSUPPORTED;
  if (!pp.q || !pp.k || !pp.v) return JL_ERR_INVALID_ARG;
  if (!aligned16(pp.q) || !aligned16(pp.k) || !aligned16(pp.v)) return JL_ERR_ALIGNMENT;
  return JL_OK;
}

int workspace_checks(const PrefillProblem& pp, int w0, int w_pretrained, int mode, const void* workspace,
                     size_t workspace_bytes) {
  const int64_t G = jl::group_size(pp.Lk(), w_pretrained);
  if (jl::all_local(pp.Lk(), w0, G)) return JL_OK;
  const size_t need = ((mode & JL_REMOTE_SPLIT) ? 2 : 1) * pp.base_ws();
  if (!workspace || workspace_bytes < need) return JL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return JL_ERR_ALIGNMENT;
  return JL_OK;
}

int correction_launch(const PrefillProblem& pp, int w0, int w_pretrained, double rope_base, int mode,
                      void* workspace, cudaStream_t s, bool all_rows = false) {
  const int64_t G = jl::group_size(pp.Lk(), w_pretrained);
  if (jl::all_local(pp.Lk(), w0, G)) return JL_OK;  // nothing to correct
  const bool split = (mode & JL_REMOTE_SPLIT) != 0;
  char* lo_base = reinterpret_cast<char*>(workspace) + pp.base_ws();  // split: Q_lo then K_lo
  RotateArgs ra;
  std::memset(&ra, 0, sizeof(ra));
  fill_theta(ra.theta, pp.D, rope_base);
  ra.G = G;
  ra.shift = jl::query_shift(w0, G, mode & JL_QSHIFT_SELF_EXTEND);
  ra.B = pp.B;
  // queries that have a remote key: positions q_off + r >= w0
  ra.x = reinterpret_cast<const __nv_bfloat16*>(pp.q);
  ra.y = q_rem_ptr(workspace);
  ra.y_lo = split ? q_rem_ptr(lo_base) : nullptr;
  ra.x_rows = ra.y_rows = pp.Lq;
  ra.H = pp.Hq;
  ra.pos_off = pp.q_off;
  ra.row_begin = all_rows ? 0 : std::max(0, w0 - pp.q_off);
  ra.row_end = pp.Lq;
  ra.is_query = 1;
  if (jl::launch_rotate_rows(ra, pp.D, s) != cudaSuccess) return JL_ERR_CUDA;
  // keys that have a remote query: j <= q_off + Lq - 1 - w0
  ra.x = reinterpret_cast<const __nv_bfloat16*>(pp.k);
  ra.y = k_rem_ptr(workspace, pp);
  ra.y_lo = split ? k_rem_ptr(lo_base, pp) : nullptr;
  ra.x_rows = pp.k_rows;
  ra.y_rows = pp.Lk();
  ra.H = pp.Hkv;
  ra.pos_off = 0;
  ra.row_begin = 0;
  ra.row_end = all_rows ? pp.Lk() : pp.Lk() - w0;
  ra.is_query = 0;
  if (jl::launch_rotate_rows(ra, pp.D, s) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

int attention_launch(const PrefillProblem& pp, void* o, float* lse, int w0, int w_pretrained, float softmax_scale,
                     int mode, const void* workspace, int* dev_error, cudaStream_t stream, int kind = jl::kBifocal) {
  const int D = pp.D;
  const int64_t G = jl::group_size(pp.Lk(), w_pretrained);
  const bool all_local = kind == jl::kBifocal && jl::all_local(pp.Lk(), w0, G);
  const bool split = !all_local && (mode & JL_REMOTE_SPLIT) != 0;
  CUtensorMap tq, tqr, tk, tkr, tv, tqr_lo, tkr_lo;
  if (!encode_bf16_4d(&tq, pp.q, D, pp.Hq, pp.Lq, pp.B, 128) ||
      !encode_bf16_4d(&tk, pp.k, D, pp.Hkv, pp.k_rows, pp.B, 128) ||
      !encode_bf16_4d(&tv, pp.v, D, pp.Hkv, pp.k_rows, pp.B, 128))
    return JL_ERR_CUDA;
  if (!all_local) {
    void* ws = const_cast<void*>(workspace);
    if (!encode_f16_4d(&tqr, q_rem_ptr(ws), D, pp.Hq, pp.Lq, pp.B, 128) ||
        !encode_f16_4d(&tkr, k_rem_ptr(ws, pp), D, pp.Hkv, pp.Lk(), pp.B, 128))
      return JL_ERR_CUDA;
  } else {
    tqr = tq;
    tkr = tk;
  }
  if (split) {
    void* lo = reinterpret_cast<char*>(const_cast<void*>(workspace)) + pp.base_ws();
    if (!encode_f16_4d(&tqr_lo, q_rem_ptr(lo), D, pp.Hq, pp.Lq, pp.B, 128) ||
        !encode_f16_4d(&tkr_lo, k_rem_ptr(lo, pp), D, pp.Hkv, pp.Lk(), pp.B, 128))
      return JL_ERR_CUDA;
  } else {
    tqr_lo = tqr;
    tkr_lo = tkr;
  }
  const int r = pp.Hq / pp.Hkv;
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
  pa.nh = (!split && r % 2 == 0) ? 2 : 1;
  pa.num_mb = (pp.Lq + 127) / 128;
  pa.all_local = all_local ? 1 : 0;
  pa.w0 = all_local ? (1 << 30) : w0;
  pa.kind = kind;
  pa.scale_log2 = resolve_scale(softmax_scale, D) * 1.4426950408889634f;
  if (jl::launch_prefill(tq, tqr, tk, tkr, tv, tqr_lo, tkr_lo, pa, D, split, stream) != cudaSuccess)
    return JL_ERR_CUDA;
  return JL_OK;
}

}  // namespace

int jl_prefill_correction(const void* q, const void* k, int B, int L, int Hq, int Hkv, int head_dim, int w0,
                          int w_pretrained, double rope_base, int mode, void* workspace, size_t workspace_bytes,
                          void* stream) {
  const PrefillProblem pp{q, k, k, B, 0, L, L, Hq, Hkv, head_dim};
  int st = problem_checks(pp, w0, w_pretrained, rope_base, mode);
  if (st == JL_OK) st = workspace_checks(pp, w0, w_pretrained, mode, workspace, workspace_bytes);
  if (st != JL_OK) return st;
  return correction_launch(pp, w0, w_pretrained, rope_base, mode, workspace, reinterpret_cast<cudaStream_t>(stream));
}

int jl_prefill_attention(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L, int Hq,
                         int Hkv, int head_dim, int w0, int w_pretrained, float softmax_scale, int mode,
                         const void* workspace, size_t workspace_bytes, int* dev_error, void* stream) {
  const PrefillProblem pp{q, k, v, B, 0, L, L, Hq, Hkv, head_dim};
  int st = problem_checks(pp, w0, w_pretrained, 10000.0, mode);
  if (st != JL_OK) return st;
  if (!o) return JL_ERR_INVALID_ARG;
  if (!aligned16(o) || (lse && ((uintptr_t)lse & 3u))) return JL_ERR_ALIGNMENT;
  st = workspace_checks(pp, w0, w_pretrained, mode, workspace, workspace_bytes);
  if (st != JL_OK) return st;
  return attention_launch(pp, o, lse, w0, w_pretrained, softmax_scale, mode, workspace, dev_error,
                          reinterpret_cast<cudaStream_t>(stream));
}

int jl_bifocal_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L, int Hq,
                       int Hkv, int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale,
                       int mode, void* workspace, size_t workspace_bytes, int* dev_error, void* stream) {
  // Validate everything before the first launch.
  const PrefillProblem pp{q, k, v, B, 0, L, L, Hq, Hkv, head_dim};
  int st = problem_checks(pp, w0, w_pretrained, rope_base, mode);
  if (st != JL_OK) return st;
  if (!o) return JL_ERR_INVALID_ARG;
  if (!aligned16(o) || (lse && ((uintptr_t)lse & 3u))) return JL_ERR_ALIGNMENT;
  st = workspace_checks(pp, w0, w_pretrained, mode, workspace, workspace_bytes);
  if (st != JL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = correction_launch(pp, w0, w_pretrained, rope_base, mode, workspace, s);
  if (st != JL_OK) return st;
  return attention_launch(pp, o, lse, w0, w_pretrained, softmax_scale, mode, workspace, dev_error, s);
}

int jl_bifocal_prefill_chunk(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len, void* o,
                             float* lse, int B, int q_offset, int chunk_len, int Hq, int Hkv, int head_dim, int w0,
                             int w_pretrained, double rope_base, float softmax_scale, int mode, void* workspace,
                             size_t workspace_bytes, int* dev_error, void* stream) {
  if (cache_len < 1 || cache_len > ((int64_t)1 << 30)) return JL_ERR_INVALID_ARG;
  if (q_offset < 0 || chunk_len < 1 || (int64_t)q_offset + chunk_len > cache_len) return JL_ERR_INVALID_ARG;
  const PrefillProblem pp{q, k_cache, v_cache, B, q_offset, chunk_len, (int)cache_len, Hq, Hkv, head_dim};
  int st = problem_checks(pp, w0, w_pretrained, rope_base, mode);
  if (st != JL_OK) return st;
  if (!o) return JL_ERR_INVALID_ARG;
  if (!aligned16(o) || (lse && ((uintptr_t)lse & 3u))) return JL_ERR_ALIGNMENT;
  st = workspace_checks(pp, w0, w_pretrained, mode, workspace, workspace_bytes);
  if (st != JL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = correction_launch(pp, w0, w_pretrained, rope_base, mode, workspace, s);
  if (st != JL_OK) return st;
  return attention_launch(pp, o, lse, w0, w_pretrained, softmax_scale, mode, workspace, dev_error, s);
}

namespace {

struct IeLayout {
  size_t o[3], lse[3], total;
};
IeLayout ie_layout(int B, int L, int Hq, int Hkv, int D, int mode) {
  IeLayout lay;
  size_t off = ((mode & JL_REMOTE_SPLIT) ? 2 : 1) * jl_prefill_workspace_bytes(B, L, Hq, Hkv, D);
  for (int x = 0; x < 3; ++x) {
    lay.o[x] = off;
    off += round_up((size_t)B * L * Hq * D * 2);
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
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || head_dim < 1) return 0;
  return ie_layout(B, L, Hq, Hkv, head_dim, mode).total;
}

int jl_bifocal_prefill_ie(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L, int Hq,
                          int Hkv, int head_dim, int w0, int w_pretrained, double rope_base, float softmax_scale,
                          int mode, void* workspace, size_t workspace_bytes, int* dev_error, void* stream) {
  const PrefillProblem pp{q, k, v, B, 0, L, L, Hq, Hkv, head_dim};
  int st = problem_checks(pp, w0, w_pretrained, rope_base, mode);
  if (st != JL_OK) return st;
  if (!o) return JL_ERR_INVALID_ARG;
  if (!aligned16(o) || (lse && ((uintptr_t)lse & 3u))) return JL_ERR_ALIGNMENT;
  const int64_t G = jl::group_size(L, w_pretrained);
  if (jl::all_local(L, w0, G)) {
    // every pair local: the three calls collapse to plain causal attention
    return jl_bifocal_prefill(q, k, v, o, lse, B, L, Hq, Hkv, head_dim, w0, w_pretrained, rope_base, softmax_scale,
                              mode, workspace, workspace_bytes, dev_error, stream);
  }
  const IeLayout lay = ie_layout(B, L, Hq, Hkv, head_dim, mode);
  if (!workspace || workspace_bytes < lay.total) return JL_ERR_WORKSPACE;
  if (!aligned16(workspace)) return JL_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = reinterpret_cast<char*>(workspace);
  // call B scores every causal pair with corrected rows: correct all rows
  st = correction_launch(pp, w0, w_pretrained, rope_base, mode, workspace, s, /*all_rows=*/true);
  if (st != JL_OK) return st;
  const int kinds[3] = {jl::kWindowBase, jl::kCausalRemote, jl::kWindowRemote};
  jl::MergeArgs ma;
  std::memset(&ma, 0, sizeof(ma));
  for (int x = 0; x < 3; ++x) {
    void* ox = ws + lay.o[x];
    float* lx = reinterpret_cast<float*>(ws + lay.lse[x]);
    st = attention_launch(pp, ox, lx, w0, w_pretrained, softmax_scale, mode, workspace, dev_error, s, kinds[x]);
    if (st != JL_OK) return st;
    ma.o_x[x] = reinterpret_cast<const __nv_bfloat16*>(ox);
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
  if (jl::launch_rope_append(a, head_dim, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

}  // extern "C"
