// Token reordering around the attention call: a video token permutation that
// makes every 128-row query block and 64-row key block spatially compact
// (4 x 4 x 4 cubes, after the AB-Attention README's "Optional cube layout", or
// a Morton3D / Z-order curve, after the LightX2V page's "Sol-Attn on Wan2.1"),
// and an HBM-bound gather / scatter kernel that applies or undoes it on
// [B, H, N, d] bf16 tensors.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <numeric>
#include <vector>

#include "bsa.h"
#include "bsa_internal.h"

namespace bsa {
namespace {

// dst row n <- src row perm[n] (gather), or dst row perm[n] <- src row n
// (scatter, the inverse permutation).  One thread moves one 16-byte chunk;
// consecutive threads cover consecutive chunks of a row, so both sides are
// accessed in whole 16-byte vectors along contiguous rows.
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ src,
                                                           uint4* __restrict__ dst,
                                                           const int32_t* __restrict__ perm,
                                                           int N, int chunks, long long total,
                                                           int inverse) {
  for (long long e = blockIdx.x * 256ll + threadIdx.x; e < total; e += static_cast<long long>(gridDim.x) * 256) {
    const int c = static_cast<int>(e % chunks);
    const long long rowg = e / chunks;  // bh * N + n
    const int n = static_cast<int>(rowg % N);
    const long long bh = rowg / N;
    const long long other = bh * N + perm[n];
    if (inverse)
      dst[other * chunks + c] = __ldg(src + rowg * chunks + c);
    else
      dst[rowg * chunks + c] = __ldg(src + other * chunks + c);
  }
}

}  // namespace
}  // namespace bsa

using namespace bsa;

extern "C" bsa_status bsa_token_permutation(int T, int Hg, int Wg, int text, int mode,
                                            int32_t* perm_out) {
  set_last_error("");
  if (T < 1 || Hg < 1 || Wg < 1 || text < 0 || perm_out == nullptr || mode < 0 || mode > 2) {
    set_last_error("bad grid, text length, mode or NULL perm_out");
    return BSA_ERR_INVALID_ARG;
  }
  const long long nv = static_cast<long long>(T) * Hg * Wg;
  if (nv + text > (1ll << 31) - 1 || T >= (1 << 20) || Hg >= (1 << 20) || Wg >= (1 << 20)) {
    set_last_error("sequence too long");
    return BSA_ERR_INVALID_ARG;
  }
  for (int i = 0; i < text; ++i) perm_out[i] = i;
  std::vector<int64_t> key(nv);
  for (long long m = 0; m < nv; ++m) {
    const int64_t t = m / (static_cast<long long>(Hg) * Wg), h = (m / Wg) % Hg, w = m % Wg;
    if (mode == 0) {
      key[m] = m;
    } else if (mode == 1) {  // cube: (t/4, h/4, w/4) then (t%4, h%4, w%4), lexicographic
      const int64_t nh = (Hg + 3) / 4, nw = (Wg + 3) / 4;
      const int64_t cube = ((t / 4) * nh + h / 4) * nw + w / 4;
      key[m] = cube * 64 + (t % 4) * 16 + (h % 4) * 4 + (w % 4);
    } else {  // Morton3D: bit b of t, h, w at key bits 3b+2, 3b+1, 3b
      int64_t k = 0;
      for (int b = 0; b < 21; ++b)
        k |= (((t >> b) & 1) << (3 * b + 2)) | (((h >> b) & 1) << (3 * b + 1)) | (((w >> b) & 1) << (3 * b));
      key[m] = k;
    }
  }
  std::vector<int32_t> order(nv);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return key[a] < key[b]; });
  for (long long i = 0; i < nv; ++i) perm_out[text + i] = text + order[i];
  return BSA_OK;
}

extern "C" bsa_status bsa_permute_tokens(const void* src, void* dst, bsa_shape s, const int32_t* perm,
                                         int inverse, void* stream) {
  set_last_error("");
  if (s.B < 1 || s.H < 1 || s.N < 1 || s.d < 8 || s.d % 8 != 0) {
    set_last_error("bad shape: B, H, N >= 1 and d a positive multiple of 8");
    return BSA_ERR_INVALID_ARG;
  }
  if (src == nullptr || dst == nullptr || perm == nullptr || src == dst ||
      (reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(dst) & 15u) ||
      (reinterpret_cast<uintptr_t>(perm) & 3u)) {
    set_last_error("src, dst (16-byte aligned, distinct) and perm (4-byte aligned) must be non-NULL");
    return BSA_ERR_INVALID_ARG;
  }
  const int chunks = s.d / 8;
  const long long total = static_cast<long long>(s.B) * s.H * s.N * chunks;
  const int grid = static_cast<int>(std::min<long long>((total + 255) / 256, 148ll * 16));
  permute_rows_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), perm, s.N, chunks, total, inverse);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e));
    return BSA_ERR_CUDA;
  }
  return BSA_OK;
}
