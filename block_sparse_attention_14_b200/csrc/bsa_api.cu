// C ABI of the library (declared in include/bsa.h): argument validation,
// workspace carve-up and the launch sequences of the three calls.
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "bsa.h"
#include "bsa_internal.h"

namespace bsa {
namespace {

thread_local char g_last_error[512] = {0};
constexpr uint64_t kDefaultTimeoutNs = 10000000000ull;  // 10 s
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};

bsa_status fail(bsa_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
bsa_status fail(bsa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

bsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxN = kBlockK * kMaxKb;  // 131072

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bsa_status check_shape(const bsa_shape& s) {
  if (s.B < 1 || s.H < 1 || s.N < 1)
    return fail(BSA_ERR_INVALID_ARG, "B, H and N must be >= 1 (got B=%d H=%d N=%d)", s.B, s.H, s.N);
  if (s.d != 64 && s.d != 128) return fail(BSA_ERR_INVALID_ARG, "d must be 64 or 128 (got %d)", s.d);
  if (s.N > kMaxN) return fail(BSA_ERR_INVALID_ARG, "N must be <= %d (got %d)", kMaxN, s.N);
  if (static_cast<int64_t>(s.B) * s.H > 65535)
    return fail(BSA_ERR_INVALID_ARG, "B*H must be <= 65535 (got %lld)",
                static_cast<long long>(s.B) * s.H);
  return BSA_OK;
}

bsa_status check_tensor(const void* p, const char* name) {
  if (p == nullptr) return fail(BSA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, 16)) return fail(BSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return BSA_OK;
}

// out must not overlap q, k or v: every CTA of a head reads that head's K and
// V while other CTAs write their output rows.
bsa_status check_out_disjoint(const bsa_shape& s, const void* out, const void* q, const void* k,
                              const void* v) {
  const size_t bytes = static_cast<size_t>(s.B) * s.H * s.N * s.d * 2;
  const uintptr_t o = reinterpret_cast<uintptr_t>(out);
  const void* ins[3] = {q, k, v};
  const char* names[3] = {"q", "k", "v"};
  for (int i = 0; i < 3; ++i) {
    const uintptr_t p = reinterpret_cast<uintptr_t>(ins[i]);
    if (o < p + bytes && p < o + bytes)
      return fail(BSA_ERR_INVALID_ARG, "out overlaps %s; the attention output needs its own buffer", names[i]);
  }
  return BSA_OK;
}

bsa_status check_ws(const bsa_shape& s, void* ws, size_t ws_bytes, Workspace* out) {
  if (ws == nullptr) return fail(BSA_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(ws, 256)) return fail(BSA_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  const size_t need = workspace_layout(s.B, s.H, s.N, s.d, out, ws);
  if (ws_bytes < need)
    return fail(BSA_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  return BSA_OK;
}

bsa_status check_topk(float topk) {
  if (!(topk > 0.f) || !(topk <= 1.f))
    return fail(BSA_ERR_INVALID_ARG, "topk must lie in (0, 1] (got %g)", static_cast<double>(topk));
  return BSA_OK;
}

#define BSA_TRY(x)                          \
  do {                                      \
    bsa_status _s = (x);                    \
    if (_s != BSA_OK) return _s;            \
  } while (0)

#define BSA_CUDA(x, what)                   \
  do {                                      \
    cudaError_t _e = (x);                   \
    if (_e != cudaSuccess) return cuda_fail(_e, what); \
  } while (0)

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bsa_status check_pinned(const void* p, const char* name) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // clear the error state the failed query left
    return fail(BSA_ERR_INVALID_ARG, "%s: pointer attributes unavailable", name);
  }
  if (a.type != cudaMemoryTypeHost)
    return fail(BSA_ERR_INVALID_ARG,
                "%s must be page-locked host memory (cudaHostAlloc or cudaHostRegister)", name);
  return BSA_OK;
}

// Streams and events of one host-pipelined call.  Destroying them while work
// is still pending is allowed: CUDA releases them once that work completes.
struct PipelineResources {
  cudaStream_t copy_in = nullptr, copy_out = nullptr, select = nullptr, attn[2] = {nullptr, nullptr};
  cudaEvent_t events[2 + 3 * 64] = {};
  int n_events = 0;
  cudaError_t event(cudaEvent_t* e) {
    cudaError_t r = cudaEventCreateWithFlags(e, cudaEventDisableTiming);
    if (r == cudaSuccess) events[n_events++] = *e;
    return r;
  }
  ~PipelineResources() {
    for (int i = 0; i < n_events; ++i) cudaEventDestroy(events[i]);
    if (copy_in) cudaStreamDestroy(copy_in);
    if (copy_out) cudaStreamDestroy(copy_out);
    if (select) cudaStreamDestroy(select);
    for (cudaStream_t a : attn)
      if (a) cudaStreamDestroy(a);
  }
};

}  // namespace

uint64_t wait_timeout_ns() { return g_timeout_ns.load(); }

int keep_count(float topk, int Kb) {
  const double t = static_cast<double>(topk);
  long long k = static_cast<long long>(ceil(t * static_cast<double>(Kb)));
  if (k < 1) k = 1;
  if (k > Kb) k = Kb;
  return static_cast<int>(k);
}

int max_score_heads(int B, int H, int N, int d, size_t capacity) {
  const size_t one = workspace_layout(B, H, N, d, nullptr, nullptr, 1);
  if (one > capacity) return 0;
  const size_t Qb = (static_cast<size_t>(N) + kBlockQ - 1) / kBlockQ;
  const size_t Kb = (static_cast<size_t>(N) + kBlockK - 1) / kBlockK;
  const size_t per_head = Qb * padded_kb(static_cast<int>(Kb)) * sizeof(float);
  // Every section is rounded up to 256 bytes, so the layout with SH heads is the
  // layout without the score section plus SH * per_head rounded up to 256.
  const size_t fixed = one - align256(per_head);
  const size_t BH = static_cast<size_t>(B) * H;
  size_t sh = (capacity - fixed) / per_head;
  if (sh > BH) sh = BH;
  return static_cast<int>(sh);
}

void set_last_error(const char* msg) {
  snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
}

size_t workspace_layout(int B, int H, int N, int d, Workspace* ws, void* base, int score_heads) {
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t SH = (score_heads <= 0 || static_cast<size_t>(score_heads) > BH) ? BH : score_heads;
  const size_t Qb = (static_cast<size_t>(N) + kBlockQ - 1) / kBlockQ;
  const size_t Kb = (static_cast<size_t>(N) + kBlockK - 1) / kBlockK;
  size_t off = 0;
  const size_t o_status = off; off = align256(off + sizeof(DeviceStatus));
  const size_t o_qbar = off;   off = align256(off + BH * Qb * d * sizeof(float));
  const size_t o_kbar = off;   off = align256(off + BH * Kb * d * sizeof(float));
  const size_t o_sc = off;     off = align256(off + SH * Qb * padded_kb(static_cast<int>(Kb)) * sizeof(float));
  const size_t o_idx = off;    off = align256(off + BH * Qb * Kb * sizeof(int16_t));
  const size_t o_cnt = off;    off = align256(off + BH * Qb * sizeof(int32_t));
  if (ws != nullptr) {
    char* b = static_cast<char*>(base);
    ws->status = reinterpret_cast<DeviceStatus*>(b + o_status);
    ws->qbar = reinterpret_cast<float*>(b + o_qbar);
    ws->kbar = reinterpret_cast<float*>(b + o_kbar);
    ws->scores = reinterpret_cast<float*>(b + o_sc);
    ws->score_heads = static_cast<int>(SH);
    ws->idx = reinterpret_cast<int16_t*>(b + o_idx);
    ws->cnt = reinterpret_cast<int32_t*>(b + o_cnt);
    ws->bytes = off;
  }
  return off;
}

}  // namespace bsa

using namespace bsa;

extern "C" {

int bsa_abi_version(void) { return 2; }

const char* bsa_status_string(bsa_status s) {
  switch (s) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
    case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT";
  }
  return "BSA_UNKNOWN_STATUS";
}

const char* bsa_last_error_message(void) { return g_last_error; }

void bsa_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : (ns < 1000 ? 1000 : ns));
}

size_t bsa_workspace_bytes(bsa_shape s) {
  if (check_shape(s) != BSA_OK) return 0;
  return workspace_layout(s.B, s.H, s.N, s.d, nullptr, nullptr);
}

bsa_status sparse_attn_block_scores(const void* q, const void* k, bsa_shape s, float* p_out,
                                    void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  BSA_TRY(check_shape(s));
  BSA_TRY(check_tensor(q, "q"));
  BSA_TRY(check_tensor(k, "k"));
  if (p_out == nullptr || !aligned(p_out, 4))
    return fail(BSA_ERR_INVALID_ARG, "p_out is NULL or not 4-byte aligned");
  Workspace w;
  BSA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = s.B * s.H;
  BSA_CUDA(cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st), "status reset");
  BSA_CUDA(launch_pool(q, k, BH, s.N, s.d, w.qbar, w.kbar, st), "pool kernel launch");
  BSA_CUDA(launch_block_scores(w.qbar, w.kbar, w.scores, w.score_heads, BH, s.N, s.d, p_out, w.status, st), "block-score kernel launch");
  return BSA_OK;
}

bsa_status sparse_attn_select(const void* q, const void* k, bsa_shape s, float topk, int is_causal,
                              uint8_t* mask_out, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  BSA_TRY(check_shape(s));
  BSA_TRY(check_tensor(q, "q"));
  BSA_TRY(check_tensor(k, "k"));
  BSA_TRY(check_topk(topk));
  if (mask_out == nullptr) return fail(BSA_ERR_INVALID_ARG, "mask_out is NULL");
  Workspace w;
  BSA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = s.B * s.H;
  const int Kb = (s.N + kBlockK - 1) / kBlockK;
  BSA_CUDA(cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st), "status reset");
  BSA_CUDA(launch_pool(q, k, BH, s.N, s.d, w.qbar, w.kbar, st), "pool kernel launch");
  BSA_CUDA(launch_select(w.qbar, w.kbar, w.scores, w.score_heads, BH, s.N, s.d, keep_count(topk, Kb), topk, is_causal != 0,
                         mask_out, w.idx, w.cnt, w.status, st),
           "select kernel launch");
  return BSA_OK;
}

bsa_status sparse_attn_select_cdf(const void* q, const void* k, bsa_shape s, float threshold,
                                  uint8_t* mask_out, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  BSA_TRY(check_shape(s));
  BSA_TRY(check_tensor(q, "q"));
  BSA_TRY(check_tensor(k, "k"));
  if (!(threshold > 0.f) || !(threshold <= 1.f))
    return fail(BSA_ERR_INVALID_ARG, "threshold must lie in (0, 1] (got %g)", static_cast<double>(threshold));
  if (mask_out == nullptr) return fail(BSA_ERR_INVALID_ARG, "mask_out is NULL");
  Workspace w;
  BSA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = s.B * s.H;
  BSA_CUDA(cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st), "status reset");
  BSA_CUDA(launch_pool(q, k, BH, s.N, s.d, w.qbar, w.kbar, st), "pool kernel launch");
  BSA_CUDA(launch_select_cdf(w.qbar, w.kbar, w.scores, w.score_heads, BH, s.N, s.d, threshold, mask_out, w.idx, w.cnt, w.status, st),
           "cdf select kernel launch");
  return BSA_OK;
}

bsa_status sparse_attn_cdf(const void* q, const void* k, const void* v, bsa_shape s, float threshold,
                           int is_causal, void* out, uint8_t* mask_out, void* ws, size_t ws_bytes,
                           void* stream) {
  g_last_error[0] = 0;
  BSA_TRY(check_shape(s));
  if (is_causal != 0) return fail(BSA_ERR_UNSUPPORTED, "the cdfthreshd mode is non-causal only");
  BSA_TRY(check_tensor(q, "q"));
  BSA_TRY(check_tensor(k, "k"));
  BSA_TRY(check_tensor(v, "v"));
  BSA_TRY(check_tensor(out, "out"));
  BSA_TRY(check_out_disjoint(s, out, q, k, v));
  if (!(threshold > 0.f) || !(threshold <= 1.f))
    return fail(BSA_ERR_INVALID_ARG, "threshold must lie in (0, 1] (got %g)", static_cast<double>(threshold));
  Workspace w;
  BSA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = s.B * s.H;
  BSA_CUDA(cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st), "status reset");
  BSA_CUDA(launch_pool(q, k, BH, s.N, s.d, w.qbar, w.kbar, st), "pool kernel launch");
  BSA_CUDA(launch_select_cdf(w.qbar, w.kbar, w.scores, w.score_heads, BH, s.N, s.d, threshold, mask_out, w.idx, w.cnt, w.status, st),
           "cdf select kernel launch");
  const char* why = nullptr;
  cudaError_t e = launch_attention(q, k, v, out, BH, s.N, s.d, 0, w.idx, w.cnt, w.status,
                                   g_timeout_ns.load(), st, &why);
  if (e != cudaSuccess) return why ? fail(BSA_ERR_CUDA, "%s", why) : cuda_fail(e, "attention kernel launch");
  return BSA_OK;
}

bsa_status block_sparse_attn_fwd(const void* q, const void* k, const void* v, bsa_shape s,
                                 const uint8_t* mask_id, int is_causal, void* out, void* ws,
                                 size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  BSA_TRY(check_shape(s));
  BSA_TRY(check_tensor(q, "q"));
  BSA_TRY(check_tensor(k, "k"));
  BSA_TRY(check_tensor(v, "v"));
  BSA_TRY(check_tensor(out, "out"));
  BSA_TRY(check_out_disjoint(s, out, q, k, v));
  Workspace w;
  BSA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = s.B * s.H;
  BSA_CUDA(cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st), "status reset");
  BSA_CUDA(launch_compact(mask_id, BH, s.N, is_causal != 0, w.idx, w.cnt, st), "compaction kernel launch");
  const char* why = nullptr;
  cudaError_t e = launch_attention(q, k, v, out, BH, s.N, s.d, is_causal != 0, w.idx, w.cnt, w.status,
                                   g_timeout_ns.load(), st, &why);
  if (e != cudaSuccess) return why ? fail(BSA_ERR_CUDA, "%s", why) : cuda_fail(e, "attention kernel launch");
  return BSA_OK;
}

bsa_status sparse_attn_topk(const void* q, const void* k, const void* v, bsa_shape s, float topk,
                            int is_causal, void* out, uint8_t* mask_out, void* ws, size_t ws_bytes,
                            void* stream) {
  g_last_error[0] = 0;
  BSA_TRY(check_shape(s));
  BSA_TRY(check_tensor(q, "q"));
  BSA_TRY(check_tensor(k, "k"));
  BSA_TRY(check_tensor(v, "v"));
  BSA_TRY(check_tensor(out, "out"));
  BSA_TRY(check_out_disjoint(s, out, q, k, v));
  BSA_TRY(check_topk(topk));
  Workspace w;
  BSA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = s.B * s.H;
  const int Kb = (s.N + kBlockK - 1) / kBlockK;
  BSA_CUDA(cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st), "status reset");
  BSA_CUDA(launch_pool(q, k, BH, s.N, s.d, w.qbar, w.kbar, st), "pool kernel launch");
  BSA_CUDA(launch_select(w.qbar, w.kbar, w.scores, w.score_heads, BH, s.N, s.d, keep_count(topk, Kb), topk, is_causal != 0,
                         mask_out, w.idx, w.cnt, w.status, st),
           "select kernel launch");
  const char* why = nullptr;
  cudaError_t e = launch_attention(q, k, v, out, BH, s.N, s.d, is_causal != 0, w.idx, w.cnt, w.status,
                                   g_timeout_ns.load(), st, &why);
  if (e != cudaSuccess) return why ? fail(BSA_ERR_CUDA, "%s", why) : cuda_fail(e, "attention kernel launch");
  return BSA_OK;
}

bsa_status sparse_attn_topk_host(const void* q_host, const void* k_host, const void* v_host,
                                 bsa_shape s, float topk, int is_causal, void* out_host, void* q_dev,
                                 void* k_dev, void* v_dev, void* out_dev, void* ws, size_t ws_bytes,
                                 int chunks, void* stream) {
  g_last_error[0] = 0;
  BSA_TRY(check_shape(s));
  BSA_TRY(check_tensor(q_host, "q_host"));
  BSA_TRY(check_tensor(k_host, "k_host"));
  BSA_TRY(check_tensor(v_host, "v_host"));
  BSA_TRY(check_tensor(out_host, "out_host"));
  BSA_TRY(check_tensor(q_dev, "q_dev"));
  BSA_TRY(check_tensor(k_dev, "k_dev"));
  BSA_TRY(check_tensor(v_dev, "v_dev"));
  BSA_TRY(check_tensor(out_dev, "out_dev"));
  BSA_TRY(check_out_disjoint(s, out_dev, q_dev, k_dev, v_dev));
  BSA_TRY(check_topk(topk));
  Workspace w;
  BSA_TRY(check_ws(s, ws, ws_bytes, &w));
  BSA_TRY(check_pinned(q_host, "q_host"));
  BSA_TRY(check_pinned(k_host, "k_host"));
  BSA_TRY(check_pinned(v_host, "v_host"));
  BSA_TRY(check_pinned(out_host, "out_host"));
  const int BH = s.B * s.H;
  const int Qb = (s.N + kBlockQ - 1) / kBlockQ;
  const int max_chunks = BH < 64 ? BH : 64;
  int nc = chunks;
  if (nc <= 0) {
    // About four waves of attention CTAs (one per SM) per chunk.  A chunk's last
    // wave overlaps the next chunk's selection and first CTAs, so small chunks
    // cost little on the GPU and keep the pipeline's fill and drain (one
    // chunk's copy in and copy out) short.
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
    const int64_t ctas = static_cast<int64_t>(BH) * Qb;
    nc = static_cast<int>((ctas + 2 * sms) / (4 * sms));
  }
  nc = nc < 1 ? 1 : (nc > max_chunks ? max_chunks : nc);
  const int Kb = (s.N + kBlockK - 1) / kBlockK;
  const int kk = keep_count(topk, Kb);
  const size_t head_bytes = static_cast<size_t>(s.N) * s.d * 2;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  PipelineResources r;
  cudaEvent_t e_start = nullptr, e_end = nullptr;
  int prio_low = 0, prio_high = 0;
  BSA_CUDA(cudaDeviceGetStreamPriorityRange(&prio_low, &prio_high), "stream priorities");
  BSA_CUDA(cudaStreamCreateWithFlags(&r.copy_in, cudaStreamNonBlocking), "copy stream");
  BSA_CUDA(cudaStreamCreateWithFlags(&r.copy_out, cudaStreamNonBlocking), "copy stream");
  BSA_CUDA(cudaStreamCreateWithPriority(&r.select, cudaStreamNonBlocking, prio_high), "select stream");
  for (cudaStream_t& a : r.attn) BSA_CUDA(cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking), "attention stream");
  BSA_CUDA(r.event(&e_start), "event");
  BSA_CUDA(r.event(&e_end), "event");
  // Nothing of this call starts before the work already queued on `stream`
  // (the status reset included).
  BSA_CUDA(cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st), "status reset");
  BSA_CUDA(cudaEventRecord(e_start, st), "event record");
  for (cudaStream_t x : {r.copy_in, r.copy_out, r.select, r.attn[0], r.attn[1]})
    BSA_CUDA(cudaStreamWaitEvent(x, e_start, 0), "stream wait");

  // Chunk c: heads [h0, h1) of the flattened B*H.  Copy in on copy_in; selection
  // on the high-priority select stream, into the chunk's own heads of the full
  // workspace layout; attention on attn[c % 2]; copy out on copy_out.  Chunks
  // touch disjoint byte ranges of every buffer, so the selection of chunk c+1
  // runs on the SMs that chunk c's attention leaves idle in its last wave, and
  // chunk c+1's attention starts on SMs as chunk c's last CTAs retire.
  const auto run = [&]() -> bsa_status {
    const char* qh = static_cast<const char*>(q_host);
    const char* kh = static_cast<const char*>(k_host);
    const char* vh = static_cast<const char*>(v_host);
    char* oh = static_cast<char*>(out_host);
    char* qd = static_cast<char*>(q_dev);
    char* kd = static_cast<char*>(k_dev);
    char* vd = static_cast<char*>(v_dev);
    char* od = static_cast<char*>(out_dev);
    // With the default chunking the first and the last chunk hold one head each:
    // the pipeline then fills with one head's copy in and drains with one head's
    // copy out; the other heads split evenly over the middle chunks.
    const bool ramp = chunks <= 0 && nc >= 3 && BH >= nc + 2;
    const auto bound = [&](int c) -> int {
      if (!ramp) return static_cast<int>(static_cast<int64_t>(BH) * c / nc);
      if (c == 0) return 0;
      if (c >= nc) return BH;
      return 1 + static_cast<int>(static_cast<int64_t>(BH - 2) * (c - 1) / (nc - 2));
    };
    for (int c = 0; c < nc; ++c) {
      const int h0 = bound(c);
      const int h1 = bound(c + 1);
      const int bhc = h1 - h0;
      if (bhc == 0) continue;
      const size_t off = static_cast<size_t>(h0) * head_bytes;
      const size_t bytes = static_cast<size_t>(bhc) * head_bytes;
      cudaEvent_t e_in = nullptr, e_sel = nullptr, e_done = nullptr;
      BSA_CUDA(r.event(&e_in), "event");
      BSA_CUDA(r.event(&e_sel), "event");
      BSA_CUDA(r.event(&e_done), "event");
      BSA_CUDA(cudaMemcpyAsync(qd + off, qh + off, bytes, cudaMemcpyHostToDevice, r.copy_in), "q copy in");
      BSA_CUDA(cudaMemcpyAsync(kd + off, kh + off, bytes, cudaMemcpyHostToDevice, r.copy_in), "k copy in");
      BSA_CUDA(cudaMemcpyAsync(vd + off, vh + off, bytes, cudaMemcpyHostToDevice, r.copy_in), "v copy in");
      BSA_CUDA(cudaEventRecord(e_in, r.copy_in), "event record");
      BSA_CUDA(cudaStreamWaitEvent(r.select, e_in, 0), "stream wait");
      const size_t hh = static_cast<size_t>(h0);
      float* qbar = w.qbar + hh * Qb * s.d;
      float* kbar = w.kbar + hh * Kb * s.d;
      float* scores = w.scores + hh * Qb * padded_kb(Kb);
      int16_t* idx = w.idx + hh * Qb * Kb;
      int32_t* cnt = w.cnt + hh * Qb;
      BSA_CUDA(launch_pool(qd + off, kd + off, bhc, s.N, s.d, qbar, kbar, r.select), "pool kernel launch");
      BSA_CUDA(launch_select(qbar, kbar, scores, bhc, bhc, s.N, s.d, kk, topk, is_causal != 0, nullptr, idx, cnt,
                             w.status, r.select),
               "select kernel launch");
      BSA_CUDA(cudaEventRecord(e_sel, r.select), "event record");
      cudaStream_t sa = r.attn[c & 1];
      BSA_CUDA(cudaStreamWaitEvent(sa, e_sel, 0), "stream wait");
      const char* why = nullptr;
      cudaError_t e = launch_attention(qd + off, kd + off, vd + off, od + off, bhc, s.N, s.d, is_causal != 0,
                                       idx, cnt, w.status, g_timeout_ns.load(), sa, &why);
      if (e != cudaSuccess) return why ? fail(BSA_ERR_CUDA, "%s", why) : cuda_fail(e, "attention kernel launch");
      BSA_CUDA(cudaEventRecord(e_done, sa), "event record");
      BSA_CUDA(cudaStreamWaitEvent(r.copy_out, e_done, 0), "stream wait");
      BSA_CUDA(cudaMemcpyAsync(oh + off, od + off, bytes, cudaMemcpyDeviceToHost, r.copy_out), "out copy");
    }
    return BSA_OK;
  };
  const bsa_status status = run();
  // `stream` waits for the last copy out, also after a failure part-way, so
  // that synchronising it covers everything this call queued.
  if (cudaEventRecord(e_end, r.copy_out) == cudaSuccess) cudaStreamWaitEvent(st, e_end, 0);
  return status;
}

bsa_status block_sparse_attn_plan(const uint8_t* mask_id, bsa_shape s, int is_causal, void* ws,
                                  size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  BSA_TRY(check_shape(s));
  Workspace w;
  BSA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  BSA_CUDA(cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st), "status reset");
  BSA_CUDA(launch_compact(mask_id, s.B * s.H, s.N, is_causal != 0, w.idx, w.cnt, st),
           "compaction kernel launch");
  return BSA_OK;
}

bsa_status block_sparse_attn_apply(const void* q, const void* k, const void* v, bsa_shape s,
                                   int is_causal, void* out, void* ws, size_t ws_bytes,
                                   void* stream) {
  g_last_error[0] = 0;
  BSA_TRY(check_shape(s));
  BSA_TRY(check_tensor(q, "q"));
  BSA_TRY(check_tensor(k, "k"));
  BSA_TRY(check_tensor(v, "v"));
  BSA_TRY(check_tensor(out, "out"));
  BSA_TRY(check_out_disjoint(s, out, q, k, v));
  Workspace w;
  BSA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  BSA_CUDA(cudaMemsetAsync(w.status, 0, sizeof(DeviceStatus), st), "status reset");
  const char* why = nullptr;
  cudaError_t e = launch_attention(q, k, v, out, s.B * s.H, s.N, s.d, is_causal != 0, w.idx, w.cnt,
                                   w.status, g_timeout_ns.load(), st, &why);
  if (e != cudaSuccess) return why ? fail(BSA_ERR_CUDA, "%s", why) : cuda_fail(e, "attention kernel launch");
  return BSA_OK;
}

bsa_status bsa_last_device_status(const void* ws, void* stream) {
  g_last_error[0] = 0;
  if (ws == nullptr || !aligned(ws, 256)) return fail(BSA_ERR_INVALID_ARG, "workspace is NULL or unaligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  BSA_CUDA(cudaStreamSynchronize(st), "stream synchronize");
  DeviceStatus h;
  BSA_CUDA(cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost), "status read");
  if (h.code == kDevTimeout)
    return fail(BSA_ERR_TIMEOUT, "a bounded wait ran out (site %u, CTA %u)", h.where, h.block);
  if (h.code != 0) return fail(BSA_ERR_CUDA, "unknown device status %u", h.code);
  return BSA_OK;
}

}  // extern "C"
