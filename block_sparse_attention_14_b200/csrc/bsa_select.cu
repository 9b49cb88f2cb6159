// Selection stage: mean pooling of q/k, compressed block scores, top-k key
// blocks per query block (radix select, ties to the lower block index), and
// compaction of a caller mask into per-row kept-block index lists.
//
// Method: "SpargeAttention Documentation" -- spas_sage2_attn_meansim_topk_cuda
// ("meansim", "topk") and the 128 x 64 mask of its "Mask Requirements".
// Pooling reads q and k once with 16-byte loads (HBM-bound); the block dot
// products run on the tensor cores (bsa_dots_tc.cu); the per-row kernels read
// one score row each from L2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bsa_internal.h"

namespace bsa {
namespace {

// ------------------------------------------------------------------ pooling
// One CTA per (query block i, head bh).  Thread (g, c) owns the 16-byte column
// chunk c (8 bf16) of rows g, g + RG, ...; partial sums are combined in shared
// memory in a fixed order, then divided by the number of valid rows.  The
// loads are latency-bound; five resident CTAs per SM (at most 48 registers, no
// spills) measured ~7% faster at Wan2.1-14B size than the four that 51
// registers allowed, and six (with spills) slower.
template <int D>
__global__ void __launch_bounds__(256, 5) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k,
                                                   float* __restrict__ qbar,
                                                   float* __restrict__ kbar, int N, int Qb,
                                                   int Kb) {
  constexpr int TPR = D / 8;       // threads per row: one 16-byte chunk each
  constexpr int RG = 256 / TPR;    // row groups
  constexpr int RPT = 128 / RG;    // rows per thread within the 128-row block
  static_assert(64 % RG == 0, "row groups must split at the 64-row boundary");
  __shared__ float red[3][RG][D];  // partial sums: q, k (rows 0-63), k (rows 64-127)

  const int i = blockIdx.x;
  const int bh = blockIdx.y;
  const int t = threadIdx.x;
  const int c = t % TPR;
  const int g = t / TPR;
  const int rows = min(kBlockQ, N - i * kBlockQ);
  const size_t base = (static_cast<size_t>(bh) * N + static_cast<size_t>(i) * kBlockQ) * D;
  const uint4* q4 = reinterpret_cast<const uint4*>(q + base);
  const uint4* k4 = reinterpret_cast<const uint4*>(k + base);

  uint4 qv[RPT], kv[RPT];
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    const int r = g + RG * m;
    if (r < rows) {
      qv[m] = __ldg(q4 + static_cast<size_t>(r) * TPR + c);
      kv[m] = __ldg(k4 + static_cast<size_t>(r) * TPR + c);
    } else {
      qv[m] = make_uint4(0, 0, 0, 0);
      kv[m] = make_uint4(0, 0, 0, 0);
    }
  }
  float aq[8], ak0[8], ak1[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) aq[e] = ak0[e] = ak1[e] = 0.f;
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    const __nv_bfloat162* qh = reinterpret_cast<const __nv_bfloat162*>(&qv[m]);
    const __nv_bfloat162* kh = reinterpret_cast<const __nv_bfloat162*>(&kv[m]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 qf = __bfloat1622float2(qh[e]);
      const float2 kf = __bfloat1622float2(kh[e]);
      aq[2 * e] += qf.x;
      aq[2 * e + 1] += qf.y;
      if (m < RPT / 2) {
        ak0[2 * e] += kf.x;
        ak0[2 * e + 1] += kf.y;
      } else {
        ak1[2 * e] += kf.x;
        ak1[2 * e + 1] += kf.y;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    red[0][g][c * 8 + e] = aq[e];
    red[1][g][c * 8 + e] = ak0[e];
    red[2][g][c * 8 + e] = ak1[e];
  }
  __syncthreads();
  const int rows_k0 = min(kBlockK, rows);
  const int rows_k1 = rows - kBlockK;  // > 0 only if key block 2i+1 exists
  for (int col = t; col < 3 * D; col += 256) {
    const int which = col / D;
    const int cc = col % D;
    if (which == 2 && rows_k1 <= 0) continue;
    float s = 0.f;
#pragma unroll 8
    for (int gg = 0; gg < RG; ++gg) s += red[which][gg][cc];
    if (which == 0) {
      qbar[(static_cast<size_t>(bh) * Qb + i) * D + cc] = s / static_cast<float>(rows);
    } else if (which == 1) {
      kbar[(static_cast<size_t>(bh) * Kb + 2 * i) * D + cc] = s / static_cast<float>(rows_k0);
    } else {
      kbar[(static_cast<size_t>(bh) * Kb + 2 * i + 1) * D + cc] = s / static_cast<float>(rows_k1);
    }
  }
}

// ------------------------------------------------------------ block scores
// S[bh][i][j] = Qbar_i . Kbar_j for every query block i and key block j, rows
// padded to Kp = Kb rounded up to 4, are computed on the tensor cores by
// launch_dots_tc (bsa_dots_tc.cu): split-TF32 products, fp32-like accuracy.

// Order-preserving map of a float onto uint32 (larger float -> larger key).
// +0 and -0 map to the same key.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The row kernels below run one warp per (bh, i) row, eight rows per CTA; the
// warp first copies its score row into shared memory.
constexpr int kRowWarps = 8;

__device__ __forceinline__ float* stage_row(const float* __restrict__ S, size_t row, int Kp,
                                            float* dst) {
  const int lane = threadIdx.x & 31;
  const float4* src = reinterpret_cast<const float4*>(S + row * Kp);
  for (int j4 = lane; j4 < Kp / 4; j4 += 32) reinterpret_cast<float4*>(dst)[j4] = src[j4];
  __syncwarp();
  return dst;
}

// Top-k of one row of dot products by one warp: a most-significant-digit radix
// select over the float keys finds the kk-th largest key T and how many of the
// keys equal to T are kept; the row is then emitted in ascending block order
// (keys above T, plus the first `need_eq` keys equal to T).  The digits are
// taken of (key - kmin) from the top bit of the row's key range down, so the
// first histogram spreads over all 256 buckets instead of the few that the
// top byte of similar floats falls in (which serialised the shared atomics).
__device__ void warp_topk_row(float* row, int Kb, int kk, uint32_t* hist, uint8_t* mask_row,
                              int16_t* idx_row, int32_t* cnt_out) {
  const int lane = threadIdx.x & 31;
  // The row's scores are replaced by the bit patterns of their keys in place
  // (each lane reads back only the entries it wrote), so the passes below take
  // the keys directly.
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int j = lane; j < Kb; j += 32) {
    const uint32_t u = float_key(row[j]);
    row[j] = __uint_as_float(u);
    kmin = min(kmin, u);
    kmax = max(kmax, u);
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  const int nbits = 32 - __clz(static_cast<int>(kmax - kmin));  // bits of the range (0 if flat)
  const unsigned lt = (1u << lane) - 1u;
  uint32_t prefix = 0, pmask = 0;  // over v = key - kmin
  int remaining = kk;
  for (int hi = nbits; hi > 0;) {
    const int lo = hi > 8 ? hi - 8 : 0;
    const uint32_t dmask = (1u << (hi - lo)) - 1u;
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = lane; j < Kb; j += 32) {
      const uint32_t v = __float_as_uint(row[j]) - kmin;
      if ((v & pmask) == prefix) atomicAdd(&hist[(v >> lo) & dmask], 1u);
    }
    __syncwarp();
    // Lane l owns buckets 255-8l ... 248-8l (descending).
    uint32_t cntb[8];
    uint32_t local = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      cntb[t] = hist[255 - 8 * lane - t];
      local += cntb[t];
    }
    uint32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, incl >= static_cast<uint32_t>(remaining));
    const int src = __ffs(hit) - 1;  // first lane whose running count reaches `remaining`
    uint32_t bucket = 0, above = 0, bcnt = 0;
    if (lane == src) {
      uint32_t run = incl - local;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (run + cntb[t] >= static_cast<uint32_t>(remaining)) {
          bucket = 255 - 8 * lane - t;
          above = run;
          bcnt = cntb[t];
          break;
        }
        run += cntb[t];
      }
    }
    bucket = __shfl_sync(0xffffffffu, bucket, src);
    above = __shfl_sync(0xffffffffu, above, src);
    bcnt = __shfl_sync(0xffffffffu, bcnt, src);
    remaining -= static_cast<int>(above);
    prefix |= bucket << lo;
    pmask |= dmask << lo;
    hi = lo;
    __syncwarp();
    if (hi > 0 && bcnt <= 64) {
      // At most 64 keys share the digits found so far: instead of more passes,
      // gather them (into the histogram's space) and rank them directly.  The
      // threshold is the candidate x with g(x) < remaining <= g(x) + e(x), where
      // g and e count the candidates above and equal to x; every key above x is
      // kept, and remaining - g(x) of the keys equal to x.
      uint32_t* cand = hist;
      int m = 0;
      for (int j0 = 0; j0 < Kb; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t v = (j < Kb) ? __float_as_uint(row[j]) - kmin : 0u;
        const bool in = (j < Kb) && (v & pmask) == prefix;
        const unsigned b = __ballot_sync(0xffffffffu, in);
        if (in) cand[m + __popc(b & lt)] = v;
        m += __popc(b);
      }
      __syncwarp();
      const uint32_t x0 = lane < m ? cand[lane] : 0u;
      const uint32_t x1 = lane + 32 < m ? cand[lane + 32] : 0u;
      int g0 = 0, e0 = 0, g1 = 0, e1 = 0;
      for (int c = 0; c < m; ++c) {
        const uint32_t y = cand[c];
        g0 += y > x0;
        e0 += y == x0;
        g1 += y > x1;
        e1 += y == x1;
      }
      const unsigned h0 = __ballot_sync(0xffffffffu, lane < m && g0 < remaining && remaining <= g0 + e0);
      const unsigned h1 = __ballot_sync(0xffffffffu, lane + 32 < m && g1 < remaining && remaining <= g1 + e1);
      const int s0 = h0 ? __ffs(h0) - 1 : __ffs(h1) - 1;
      const uint32_t xs = __shfl_sync(0xffffffffu, h0 ? x0 : x1, s0);
      const int gs = __shfl_sync(0xffffffffu, h0 ? g0 : g1, s0);
      prefix = xs;
      remaining -= gs;
      break;
    }
  }
  const uint32_t T = prefix + kmin;
  const int need_eq = remaining;  // keys equal to T still to keep, lowest index first
  int eq_seen = 0, kept = 0;
  for (int base = 0; base < Kb; base += 32) {
    const int j = base + lane;
    const uint32_t u = (j < Kb) ? __float_as_uint(row[j]) : 0u;
    const bool eq = (j < Kb) && (u == T);
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool keep = (j < Kb) && (u > T || (eq && eq_seen + __popc(eqb & lt) < need_eq));
    eq_seen += __popc(eqb);
    const unsigned kb = __ballot_sync(0xffffffffu, keep);
    if (keep) idx_row[kept + __popc(kb & lt)] = static_cast<int16_t>(j);
    if (mask_row != nullptr && j < Kb) mask_row[j] = keep ? 1 : 0;
    kept += __popc(kb);
  }
  if (lane == 0) *cnt_out = kept;
}

// cdfthreshd selection of one row by one warp: the shortest prefix, in
// (score descending, index ascending) order, whose softmax mass reaches tau;
// at least one block; every block if rounding leaves the total below tau.
// row[] holds the raw dot products and is overwritten with the probabilities.
// The largest key T whose mass F(T) = sum of P over keys >= T still reaches
// tau is found bit by bit (fp32 sums in a fixed lane-then-shuffle order);
// then every key above T is kept plus the first `need` keys equal to T.
constexpr int kCdfPer = kMaxKb / 32;

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_fsum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ void warp_cdf_row(float* row, int Kb, float scale, float tau, uint8_t* mask_row,
                             int16_t* idx_row, int32_t* cnt_out) {
  const int lane = threadIdx.x & 31;
  const int nper = (Kb + 31) >> 5;
  uint32_t key[kCdfPer];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < kCdfPer; ++i) {
    const int j = i * 32 + lane;
    const bool v = i < nper && j < Kb;
    key[i] = v ? float_key(row[j]) : 0u;  // 0 is below every real key
    if (v) mx = fmaxf(mx, row[j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float z = 0.f;
  for (int j = lane; j < Kb; j += 32) {
    const float e = expf((row[j] - mx) * scale);
    row[j] = e;
    z += e;
  }
  const float inv = 1.f / warp_fsum(z);
  for (int j = lane; j < Kb; j += 32) row[j] *= inv;
  __syncwarp();
  auto mass_at_or_above = [&](uint32_t cand) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < kCdfPer; ++i)
      if (i < nper && key[i] >= cand) m += row[i * 32 + lane];
    return warp_fsum(m);
  };
  uint32_t T = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    if (mass_at_or_above(cand) >= tau) T = cand;
  }
  const unsigned lt = (1u << lane) - 1u;
  int kept = 0;
  if (T == 0) {  // the whole row's mass stays below tau: keep every block
    for (int j = lane; j < Kb; j += 32) {
      idx_row[j] = static_cast<int16_t>(j);
      if (mask_row != nullptr) mask_row[j] = 1;
    }
    if (lane == 0) *cnt_out = Kb;
    return;
  }
  float above = 0.f, p_eq = 0.f;
  int n_eq = 0;
#pragma unroll
  for (int i = 0; i < kCdfPer; ++i) {
    if (i < nper) {
      if (key[i] > T) above += row[i * 32 + lane];
      if (key[i] == T) {
        p_eq = row[i * 32 + lane];
        ++n_eq;
      }
    }
  }
  above = warp_fsum(above);
  p_eq = fmaxf(p_eq, __shfl_xor_sync(0xffffffffu, p_eq, 16));
  p_eq = fmaxf(p_eq, __shfl_xor_sync(0xffffffffu, p_eq, 8));
  p_eq = fmaxf(p_eq, __shfl_xor_sync(0xffffffffu, p_eq, 4));
  p_eq = fmaxf(p_eq, __shfl_xor_sync(0xffffffffu, p_eq, 2));
  p_eq = fmaxf(p_eq, __shfl_xor_sync(0xffffffffu, p_eq, 1));
  n_eq = warp_sum(n_eq);
  int need = p_eq > 0.f ? static_cast<int>(ceilf((tau - above) / p_eq)) : n_eq;
  need = max(1, min(n_eq, need));
  int eq_seen = 0;
#pragma unroll
  for (int i = 0; i < kCdfPer; ++i) {
    if (i >= nper) break;
    const int j = i * 32 + lane;
    const uint32_t u = key[i];
    const bool valid = j < Kb;
    const bool eq = valid && u == T;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool keep = valid && (u > T || (eq && eq_seen + __popc(eqb & lt) < need));
    eq_seen += __popc(eqb);
    const unsigned kb = __ballot_sync(0xffffffffu, keep);
    if (keep) idx_row[kept + __popc(kb & lt)] = static_cast<int16_t>(j);
    if (mask_row != nullptr && valid) mask_row[j] = keep ? 1 : 0;
    kept += __popc(kb);
  }
  if (lane == 0) *cnt_out = kept;
}

__global__ void __launch_bounds__(32 * kRowWarps) select_cdf_kernel(const float* __restrict__ S,
                                                                   int rows, int Kb, int Kp,
                                                                   float scale, float tau,
                                                                   uint8_t* __restrict__ mask_out,
                                                                   int16_t* __restrict__ idx,
                                                                   int32_t* __restrict__ cnt) {
  extern __shared__ __align__(16) float smem[];
  const int w = threadIdx.x >> 5;
  const size_t row = static_cast<size_t>(blockIdx.x) * kRowWarps + w;
  if (row >= static_cast<size_t>(rows)) return;
  float* r = stage_row(S, row, Kp, smem + w * Kp);
  warp_cdf_row(r, Kb, scale, tau, mask_out ? mask_out + row * Kb : nullptr, idx + row * Kb,
               cnt + row);
}

// Kept count for a fraction of E blocks: clamp(ceil(topk * E), 1, E) in double
// precision on the float value of topk (the host computes the same for the
// non-causal case).
__device__ __forceinline__ int keep_count_dev(float topk, int E) {
  int k = static_cast<int>(ceil(static_cast<double>(topk) * static_cast<double>(E)));
  return max(1, min(E, k));
}

__global__ void __launch_bounds__(32 * kRowWarps) select_kernel(const float* __restrict__ S, int rows,
                                                               int Qb, int Kb, int Kp, int kk,
                                                               float topk, int causal,
                                                               uint8_t* __restrict__ mask_out,
                                                               int16_t* __restrict__ idx,
                                                               int32_t* __restrict__ cnt) {
  extern __shared__ __align__(16) float smem[];  // [kRowWarps][Kp] rows, [kRowWarps][256] hist
  const int w = threadIdx.x >> 5;
  const size_t row = static_cast<size_t>(blockIdx.x) * kRowWarps + w;
  if (row >= static_cast<size_t>(rows)) return;
  float* r = stage_row(S, row, Kp, smem + w * Kp);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + kRowWarps * Kp) + w * 256;
  const int i = static_cast<int>(row % static_cast<size_t>(Qb));
  // Causal: query block i may use key blocks 0 .. 2i+1 only; top-k runs over those.
  const int Ke = causal ? min(2 * i + 2, Kb) : Kb;
  const int k_row = causal ? keep_count_dev(topk, Ke) : kk;
  uint8_t* mrow = mask_out ? mask_out + row * Kb : nullptr;
  warp_topk_row(r, Ke, k_row, hist, mrow, idx + row * Kb, cnt + row);
  if (mrow != nullptr)
    for (int j = Ke + (threadIdx.x & 31); j < Kb; j += 32) mrow[j] = 0;
}

__global__ void __launch_bounds__(32 * kRowWarps) block_scores_kernel(const float* __restrict__ S,
                                                                     int rows, int Kb, int Kp,
                                                                     float scale,
                                                                     float* __restrict__ p_out) {
  extern __shared__ __align__(16) float smem[];
  const int w = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const size_t row = static_cast<size_t>(blockIdx.x) * kRowWarps + w;
  if (row >= static_cast<size_t>(rows)) return;
  const float* r = stage_row(S, row, Kp, smem + w * Kp);
  float mx = -INFINITY;
  for (int j = lane; j < Kb; j += 32) mx = fmaxf(mx, r[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  for (int j = lane; j < Kb; j += 32) sum += expf((r[j] - mx) * scale);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = 1.f / sum;
  float* out = p_out + row * Kb;
  for (int j = lane; j < Kb; j += 32) out[j] = expf((r[j] - mx) * scale) * inv;
}

// ----------------------------------------------------------------- compaction
// One warp per (b, h, i) row: kept block indices in ascending order.
__global__ void __launch_bounds__(256) compact_kernel(const uint8_t* __restrict__ mask, int rows,
                                                      int Qb, int Kb, int causal,
                                                      int16_t* __restrict__ idx,
                                                      int32_t* __restrict__ cnt) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  // Causal: blocks past 2i+1 hold only later keys and are dropped.
  const int limit = causal ? min(2 * (row % Qb) + 2, Kb) : Kb;
  const uint8_t* m = mask ? mask + static_cast<size_t>(row) * Kb : nullptr;
  int16_t* out = idx + static_cast<size_t>(row) * Kb;
  const unsigned lt = (1u << lane) - 1u;
  int kept = 0;
  for (int base = 0; base < Kb; base += 32) {
    const int j = base + lane;
    const bool keep = (j < limit) && (m == nullptr || m[j] != 0);
    const unsigned b = __ballot_sync(0xffffffffu, keep);
    if (keep) out[kept + __popc(b & lt)] = static_cast<int16_t>(j);
    kept += __popc(b);
  }
  if (lane == 0) cnt[row] = kept;
}

size_t row_smem(int Kp, bool with_hist) {
  return sizeof(float) * kRowWarps * static_cast<size_t>(Kp) +
         (with_hist ? sizeof(uint32_t) * kRowWarps * 256 : 0);
}

cudaError_t launch_dots(const float* qbar, const float* kbar, int BH, int Qb, int Kb, int d,
                        float* S, DeviceStatus* status, cudaStream_t st) {
  return launch_dots_tc(qbar, kbar, BH, Qb, Kb, d, S, status, wait_timeout_ns(), st);
}

}  // namespace

cudaError_t launch_pool(const void* q, const void* k, int BH, int N, int d, float* qbar,
                        float* kbar, cudaStream_t st) {
  const int Qb = (N + kBlockQ - 1) / kBlockQ;
  const int Kb = (N + kBlockK - 1) / kBlockK;
  dim3 grid(Qb, BH);
  if (d == 128)
    pool_kernel<128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                           static_cast<const __nv_bfloat16*>(k), qbar, kbar, N,
                                           Qb, Kb);
  else
    pool_kernel<64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                          static_cast<const __nv_bfloat16*>(k), qbar, kbar, N, Qb,
                                          Kb);
  return cudaGetLastError();
}

// The selection launchers work through the heads in chunks of score_heads: the
// dot products of a chunk go to the scores section, then the row kernels of
// that chunk read them.  Everything is stream-ordered, so chunks reuse it.
cudaError_t launch_select(const float* qbar, const float* kbar, float* scores, int score_heads, int BH,
                          int N, int d, int kk, float topk, int causal, uint8_t* mask_out,
                          int16_t* idx, int32_t* cnt, DeviceStatus* status, cudaStream_t st) {
  const int Qb = (N + kBlockQ - 1) / kBlockQ;
  const int Kb = (N + kBlockK - 1) / kBlockK;
  const int Kp = padded_kb(Kb);
  const size_t smem = row_smem(Kp, true);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int sh = (score_heads <= 0 || score_heads > BH) ? BH : score_heads;
  for (int h0 = 0; h0 < BH; h0 += sh) {
    const int nh = BH - h0 < sh ? BH - h0 : sh;
    const size_t r0 = static_cast<size_t>(h0) * Qb;
    e = launch_dots(qbar + r0 * d, kbar + static_cast<size_t>(h0) * Kb * d, nh, Qb, Kb, d, scores, status, st);
    if (e != cudaSuccess) return e;
    const int rows = nh * Qb;
    select_kernel<<<(rows + kRowWarps - 1) / kRowWarps, 32 * kRowWarps, smem, st>>>(
        scores, rows, Qb, Kb, Kp, kk, topk, causal, mask_out ? mask_out + r0 * Kb : nullptr,
        idx + r0 * Kb, cnt + r0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_select_cdf(const float* qbar, const float* kbar, float* scores, int score_heads,
                              int BH, int N, int d, float threshold, uint8_t* mask_out,
                              int16_t* idx, int32_t* cnt, DeviceStatus* status, cudaStream_t st) {
  const int Qb = (N + kBlockQ - 1) / kBlockQ;
  const int Kb = (N + kBlockK - 1) / kBlockK;
  const int Kp = padded_kb(Kb);
  const size_t smem = row_smem(Kp, false);
  const float scale = 1.0f / sqrtf(static_cast<float>(d));
  cudaError_t e = cudaFuncSetAttribute(select_cdf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int sh = (score_heads <= 0 || score_heads > BH) ? BH : score_heads;
  for (int h0 = 0; h0 < BH; h0 += sh) {
    const int nh = BH - h0 < sh ? BH - h0 : sh;
    const size_t r0 = static_cast<size_t>(h0) * Qb;
    e = launch_dots(qbar + r0 * d, kbar + static_cast<size_t>(h0) * Kb * d, nh, Qb, Kb, d, scores, status, st);
    if (e != cudaSuccess) return e;
    const int rows = nh * Qb;
    select_cdf_kernel<<<(rows + kRowWarps - 1) / kRowWarps, 32 * kRowWarps, smem, st>>>(
        scores, rows, Kb, Kp, scale, threshold, mask_out ? mask_out + r0 * Kb : nullptr, idx + r0 * Kb,
        cnt + r0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_block_scores(const float* qbar, const float* kbar, float* scores, int score_heads,
                                int BH, int N, int d, float* p_out, DeviceStatus* status,
                                cudaStream_t st) {
  const int Qb = (N + kBlockQ - 1) / kBlockQ;
  const int Kb = (N + kBlockK - 1) / kBlockK;
  const int Kp = padded_kb(Kb);
  const size_t smem = row_smem(Kp, false);
  const float scale = 1.0f / sqrtf(static_cast<float>(d));
  cudaError_t e = cudaFuncSetAttribute(block_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int sh = (score_heads <= 0 || score_heads > BH) ? BH : score_heads;
  for (int h0 = 0; h0 < BH; h0 += sh) {
    const int nh = BH - h0 < sh ? BH - h0 : sh;
    const size_t r0 = static_cast<size_t>(h0) * Qb;
    e = launch_dots(qbar + r0 * d, kbar + static_cast<size_t>(h0) * Kb * d, nh, Qb, Kb, d, scores, status, st);
    if (e != cudaSuccess) return e;
    const int rows = nh * Qb;
    block_scores_kernel<<<(rows + kRowWarps - 1) / kRowWarps, 32 * kRowWarps, smem, st>>>(
        scores, rows, Kb, Kp, scale, p_out + r0 * Kb);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_compact(const uint8_t* mask, int BH, int N, int causal, int16_t* idx,
                           int32_t* cnt, cudaStream_t st) {
  const int Qb = (N + kBlockQ - 1) / kBlockQ;
  const int Kb = (N + kBlockK - 1) / kBlockK;
  const int rows = BH * Qb;
  compact_kernel<<<(rows + 7) / 8, 256, 0, st>>>(mask, rows, Qb, Kb, causal, idx, cnt);
  return cudaGetLastError();
}

}  // namespace bsa
