// Bifocal decode for callers that cannot allocate device memory.
//
// Some callers of a decode step are not allowed to call cudaMalloc: a plugin
// running inside an inference engine whose device memory is entirely owned by
// the host framework's pool, or a serving loop that must not allocate (nor take
// the implicit device synchronisation an allocation can bring) once it is
// running.  jl_bifocal_decode_noalloc serves them: it is jl_bifocal_decode with
// its scratch (split partials and ticket counters) placed in a fixed
// file-scope device array instead of a caller-provided workspace.
//
//   * The array holds kNoAllocScratchBytes (4 MiB).  A problem whose decode
//     scratch would exceed that is rejected with JL_ERR_WORKSPACE before any
//     launch.  Every GPU that loads this library keeps the array until the
//     process exits.
//   * All calls on a device share the one array, which keeps the last call's
//     contents.  The ticket counters are cleared (cudaMemsetAsync, no
//     allocation) before each launch; everything else is overwritten before it
//     is read.  Calls that overlap on the GPU (different streams, no ordering
//     between them) race on the array and give wrong results; order them.
//   * The first call on a device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; make that
//     first call before any stream capture.
//   * Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "../../include/jl_api.h"
#include "jl_kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
constexpr int kMaxDevices = 64;

// Host code must never pass this name to a kernel: on the host it is only a
// stand-in for the symbol.  Kernels get the address cached below.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return JL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return JL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return JL_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return JL_OK;
}

}  // namespace

extern "C" int jl_bifocal_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len,
                                         void* o, float* lse, int B, int L, int Hq, int Hkv, int head_dim, int w0,
                                         int w_pretrained, double rope_base, float softmax_scale, int mode,
                                         int* dev_error, void* stream) {
  // The checks jl_bifocal_decode makes before it launches, so that an argument
  // error launches nothing here either (not even the counter clear).
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || w0 < 0 || w_pretrained < 1 || Hq % Hkv != 0)
    return JL_ERR_INVALID_ARG;
  if (!(rope_base > 0.0) || (mode & ~(JL_QSHIFT_SELF_EXTEND | JL_REMOTE_SPLIT)) != 0) return JL_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return JL_ERR_UNSUPPORTED;
  if (Hq / Hkv > 8 || L > (1 << 30)) return JL_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !o || cache_len < L || cache_len > ((int64_t)1 << 31)) return JL_ERR_INVALID_ARG;
  auto mis = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (mis(q) || mis(k_cache) || mis(v_cache) || mis(o) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return JL_ERR_ALIGNMENT;

  const size_t need = jl_decode_workspace_bytes(B, L, Hq, Hkv, head_dim);
  if (need == 0) return JL_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return JL_ERR_WORKSPACE;  // beyond the fixed array

  void* scratch = nullptr;
  int st = scratch_address(&scratch);
  if (st != JL_OK) return st;

  // The ticket counters (one int per (batch, KV head), at the start of the
  // scratch layout) must be zero when the kernel starts.
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, (size_t)B * Hkv * sizeof(int), s) != cudaSuccess) return JL_ERR_CUDA;

  return jl_bifocal_decode(q, k_cache, v_cache, cache_len, o, lse, B, L, Hq, Hkv, head_dim, w0, w_pretrained,
                           rope_base, softmax_scale, mode, scratch, kNoAllocScratchBytes, dev_error, stream);
}
