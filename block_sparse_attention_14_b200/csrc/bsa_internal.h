// Host-side launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "bsa_common.cuh"

namespace bsa {

// Workspace carve-up (every section 256-byte aligned).
struct Workspace {
  DeviceStatus* status;  // 256 bytes
  float* qbar;           // [B*H, Qb, d]
  float* kbar;           // [B*H, Kb, d]
  float* scores;         // [score_heads, Qb, padded_kb(Kb)]  block dot products Qbar_i . Kbar_j
  int score_heads;       // heads whose score matrices the scores section holds at once
  int16_t* idx;          // [B*H, Qb, Kb]  ascending kept key-block indices (prefix of cnt)
  int32_t* cnt;          // [B*H, Qb]
  size_t bytes;
};

// Carves `base` into the sections above; returns the bytes needed.  The scores
// section holds score_heads heads at a time (<= 0 or > B*H: all B*H); the
// selection launchers then work through the heads in chunks of that many.
size_t workspace_layout(int B, int H, int N, int d, Workspace* ws, void* base, int score_heads = 0);

// Row stride of the block-score matrix: Kb rounded up to a multiple of 4 floats.
inline int padded_kb(int Kb) { return (Kb + 3) & ~3; }

// Current limit of the kernels' bounded waits (bsa_set_wait_timeout_ns).
uint64_t wait_timeout_ns();

// Kept key blocks per row for a top-k fraction: clamp(ceil(topk * Kb), 1, Kb),
// in double precision on the float value of topk.
int keep_count(float topk, int Kb);

// The largest number of heads whose block-score matrices fit, together with the
// rest of the workspace layout, in `capacity` bytes (at most B*H; 0 if not even
// one head fits).
int max_score_heads(int B, int H, int N, int d, size_t capacity);

// Records the message returned by bsa_last_error_message() on this thread.
void set_last_error(const char* msg);

// The driver's cuTensorMapEncodeTiled, looked up once (nullptr if unavailable).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

// (a3) block dot products on the tensor cores (split TF32, fp32-like accuracy):
// S[bh][i][j] = Qbar_i . Kbar_j, rows of padded_kb(Kb) floats.  Its waits are
// bounded by timeout_ns and a timeout is recorded in `status`.
cudaError_t launch_dots_tc(const float* qbar, const float* kbar, int BH, int Qb, int Kb, int d,
                           float* S, DeviceStatus* status, uint64_t timeout_ns, cudaStream_t st);

// (a1, a2) mean-pool q over 128-row blocks and k over 64-row blocks.
cudaError_t launch_pool(const void* q, const void* k, int BH, int N, int d, float* qbar,
                        float* kbar, cudaStream_t st);

// (a3, a4) block scores (into `scores`) and top-k; writes mask (optional), idx
// and cnt.  kkeep is the kept count per row; with causal != 0 each row i
// instead keeps ceil(topk * E_i) of its E_i = min(2i+2, Kb) eligible blocks.
// `status` is the workspace's status word (the block dot products' bounded
// waits record a timeout there).
cudaError_t launch_select(const float* qbar, const float* kbar, float* scores, int score_heads, int BH,
                          int N, int d, int kkeep, float topk, int causal, uint8_t* mask_out,
                          int16_t* idx, int32_t* cnt, DeviceStatus* status, cudaStream_t st);

// cdfthreshd selection: the shortest score-ordered prefix reaching softmax mass
// `threshold`; writes mask (optional), idx and cnt.
cudaError_t launch_select_cdf(const float* qbar, const float* kbar, float* scores, int score_heads,
                              int BH, int N, int d, float threshold, uint8_t* mask_out,
                              int16_t* idx, int32_t* cnt, DeviceStatus* status, cudaStream_t st);

// (a3) block-score map only: p_out = softmax of the scaled block scores.
cudaError_t launch_block_scores(const float* qbar, const float* kbar, float* scores, int score_heads,
                                int BH, int N, int d, float* p_out, DeviceStatus* status,
                                cudaStream_t st);

// (a4') caller mask (NULL = all ones) -> idx and cnt; causal != 0 drops the
// blocks past 2i+1 of row i.
cudaError_t launch_compact(const uint8_t* mask, int BH, int N, int causal, int16_t* idx,
                           int32_t* cnt, cudaStream_t st);

// (a5, a6) block-sparse attention forward over the idx lists.
cudaError_t launch_attention(const void* q, const void* k, const void* v, void* out, int BH, int N,
                             int d, int causal, const int16_t* idx, const int32_t* cnt,
                             DeviceStatus* status, uint64_t timeout_ns, cudaStream_t st,
                             const char** why);

}  // namespace bsa
