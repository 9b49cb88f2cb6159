// sparse_attn_topk_noalloc: the fused selection + attention call for callers
// that cannot allocate device memory.  Its scratch (pooled means, block
// scores, kept-block lists, status word) lives in a file-scope __device__ array
// instead of a caller-provided workspace; the caller still passes q, k, v, out
// and the optional mask.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "bsa.h"
#include "bsa_internal.h"

namespace bsa {
namespace {

// 32 MiB, held by every GPU that loads the library until the process exits.
constexpr size_t kStaticScratchBytes = 32ull << 20;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 256;
struct ScratchEntry {
  void* ctx;  // CUDA context the address was looked up in
  void* ptr;  // device address of that context's copy of g_static_scratch
};
std::mutex g_scratch_mu;
ScratchEntry g_scratch[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the current device's copy of g_static_scratch.  In host
// code the symbol's name is only a host-side handle, so the address is looked
// up with cudaGetSymbolAddress (with the device current) and cached per device
// and CUDA context: a new context on the device (after cudaDeviceReset, say)
// reloads the module, so its address is looked up afresh.
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CtxGetCurrentFn get = ctx_get_current_fn();
  if (get == nullptr) return cudaErrorInitializationError;
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return cudaErrorInitializationError;
  if (ctx == nullptr) {
    // No context is current on this thread yet: the symbol lookup initialises
    // the device's primary context (and loads the module), then it is current.
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_static_scratch)) != cudaSuccess) return e;
    if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorInitializationError;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchEntry& s = g_scratch[dev];
  if (s.ptr == nullptr || s.ctx != static_cast<void*>(ctx)) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    s.ptr = p;
    s.ctx = ctx;
  }
  *out = s.ptr;
  return cudaSuccess;
}

bsa_status reject(bsa_status s, const char* msg) {
  set_last_error(msg);
  return s;
}

}  // namespace
}  // namespace bsa

using namespace bsa;

extern "C" bsa_status sparse_attn_topk_noalloc(const void* q, const void* k, const void* v,
                                               bsa_shape s, float topk, int is_causal, void* out,
                                               uint8_t* mask_out, void* stream) {
  set_last_error("");
  if (s.B < 1 || s.H < 1 || s.N < 1 || (s.d != 64 && s.d != 128) || s.N > kBlockK * kMaxKb ||
      static_cast<int64_t>(s.B) * s.H > 65535)
    return reject(BSA_ERR_INVALID_ARG, "bad shape: need B, H, N >= 1, d in {64, 128}, N <= 131072, B*H <= 65535");
  const void* ptrs[4] = {q, k, v, out};
  for (const void* p : ptrs)
    if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) != 0)
      return reject(BSA_ERR_INVALID_ARG, "q, k, v and out must be non-NULL and 16-byte aligned");
  if (!(topk > 0.f) || !(topk <= 1.f)) return reject(BSA_ERR_INVALID_ARG, "topk must lie in (0, 1]");
  {
    const size_t bytes = static_cast<size_t>(s.B) * s.H * s.N * s.d * 2;
    const uintptr_t o = reinterpret_cast<uintptr_t>(out);
    for (const void* in : {q, k, v}) {
      const uintptr_t p = reinterpret_cast<uintptr_t>(in);
      if (o < p + bytes && p < o + bytes)
        return reject(BSA_ERR_INVALID_ARG, "out overlaps q, k or v; the attention output needs its own buffer");
    }
  }
  // The scratch holds the block-score matrices of as many heads at a time as
  // fit (at least one); the selection then runs over the heads in chunks.
  const size_t need = workspace_layout(s.B, s.H, s.N, s.d, nullptr, nullptr, 1);
  if (need > kStaticScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "this shape needs %zu bytes of scratch; the static scratch of the no-allocation call "
             "holds %zu bytes (use sparse_attn_topk with a caller workspace)",
             need, kStaticScratchBytes);
    return reject(BSA_ERR_INVALID_ARG, msg);
  }
  const int BH = s.B * s.H;
  const int score_heads = max_score_heads(s.B, s.H, s.N, s.d, kStaticScratchBytes);
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return reject(BSA_ERR_CUDA, cudaGetErrorString(e));
  Workspace w;
  workspace_layout(s.B, s.H, s.N, s.d, &w, base, score_heads);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int Kb = (s.N + kBlockK - 1) / kBlockK;
  const int causal = is_causal != 0;
  // The status word must start at zero; everything else is overwritten.
  if ((e = cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st)) != cudaSuccess ||
      (e = launch_pool(q, k, BH, s.N, s.d, w.qbar, w.kbar, st)) != cudaSuccess ||
      (e = launch_select(w.qbar, w.kbar, w.scores, w.score_heads, BH, s.N, s.d, keep_count(topk, Kb), topk,
                         causal, mask_out, w.idx, w.cnt, w.status, st)) != cudaSuccess)
    return reject(BSA_ERR_CUDA, cudaGetErrorString(e));
  const char* why = nullptr;
  e = launch_attention(q, k, v, out, BH, s.N, s.d, causal, w.idx, w.cnt, w.status, wait_timeout_ns(), st,
                       &why);
  if (e != cudaSuccess) return reject(BSA_ERR_CUDA, why ? why : cudaGetErrorString(e));
  return BSA_OK;
}

extern "C" bsa_status sparse_attn_topk_noalloc_status(void* stream) {
  set_last_error("");
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return reject(BSA_ERR_CUDA, cudaGetErrorString(e));
  // The status word sits at the start of the scratch, as in a caller workspace.
  return bsa_last_device_status(base, stream);
}
