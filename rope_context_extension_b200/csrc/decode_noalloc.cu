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
//   * The array holds kNoAllocScratchBytes (4 MiB).  The split partials are
//     laid out for the split count the call uses; when that layout would not
//     fit, the call uses fewer splits (same results up to the order of the
//     final sum, slower on a short batch).  A problem that does not fit even
//     with one split per (sequence, KV head) -- B * Hq * (4 D + 8) + 4 B Hkv
//     bytes, plus alignment, above 4 MiB: e.g. more than 126 sequences at 64
//     query heads of D = 128 -- is rejected with JL_ERR_WORKSPACE before any
//     launch.  Every GPU that loads this library keeps the array until the
//     process exits.
//   * All calls on a device share the one array, which keeps the last call's
//     contents.  The ticket counters are cleared (cudaMemsetAsync, no
//     allocation) before each launch; everything else is overwritten before it
//     is read.  Calls that overlap on the GPU (different streams, no ordering
//     between them) race on the array and give wrong results; order them.
//   * The first call on a device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; make that
//     first call before any stream capture.  The cache is keyed by the
//     context's unique id as well, so after cudaDeviceReset (a new primary
//     context) the next call looks the address up again.
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
unsigned long long g_scratch_ctx_id[kMaxDevices] = {};

// Unique id of the calling thread's current context (never reused within the
// process), or 0 when the thread has none yet.  Driver entry points are looked
// up through the runtime, so the library does not link libcuda directly.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_decode_scratch on the current device, looked up once per
// (device, context) and cached.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return JL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return JL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long id = current_context_id();
  if (g_scratch_addr[dev] == nullptr || id == 0 || id != g_scratch_ctx_id[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return JL_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx_id[dev] = current_context_id();  // the runtime has made its context current by now
  }
  *out = g_scratch_addr[dev];
  return JL_OK;
}

}  // namespace

extern "C" int jl_bifocal_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, int64_t cache_len,
                                         void* o, float* lse, int B, int L, int Hq, int Hkv, int head_dim, int w0,
                                         int w_pretrained, double rope_base, float softmax_scale, int mode,
                                         int* dev_error, void* stream) {
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != JL_OK) return st;
  // Argument checks, the split count that fits the array, the ticket clear and
  // the launch (nothing is launched on an argument error).
  return jl::decode_in_fixed_scratch(q, k_cache, v_cache, cache_len, o, lse, B, L, Hq, Hkv, head_dim, w0,
                                     w_pretrained, rope_base, softmax_scale, mode, scratch, kNoAllocScratchBytes,
                                     dev_error, stream);
}
