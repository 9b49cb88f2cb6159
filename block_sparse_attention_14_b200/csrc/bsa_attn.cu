// Block-sparse attention forward on sm_100a: only the kept 128 x 64 tiles of
// each (head, query block) are visited, following block_sparse_sage2_attn_cuda
// and its "Mask Requirements" ("SpargeAttention Documentation"): non-causal,
// bf16 inputs, scale 1/sqrt(d).
//
// One CTA per (head, query block), 256 threads:
//   warp 0      TMA producer for the Q tile and the kept K tiles
//   warp 1      TMEM owner and MMA issuer (one thread issues tcgen05.mma)
//   warp 2      TMA producer for the kept V tiles
//   warps 4-7   softmax and epilogue; thread t owns query row t, which is TMEM
//               lane t, so row max / row sum need no shuffles
// Kept key blocks are consumed in pairs (128 keys), so S = Q K^T is one
// M=128, N=128 tensor-core tile per pair (N=64 for an odd last block), and
// O += P V runs with K=128.  S is double-buffered in TMEM so QK^T of pair j+1
// overlaps the softmax of pair j.  P is written back to TMEM as bf16 (or to
// shared memory in the kPInTmem=false variant) and O accumulates in TMEM.
// The online softmax works in the exp2 domain and only rescales O when the row
// maximum grows by more than 2^8, which keeps every exponent <= 2^8 and is
// exact because l and O always share the same reference maximum.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "bsa_internal.h"

namespace bsa {
namespace {

enum WaitSite : uint32_t {
  kWaitQ = 1,
  kWaitKFull = 2,
  kWaitKEmpty = 3,
  kWaitVFull = 4,
  kWaitVEmpty = 5,
  kWaitSFull = 6,
  kWaitPFull = 7,
  kWaitODone = 8,
  kWaitFinal = 9,
  kWaitDrain = 10,
};

struct AttnArgs {
  const int16_t* idx;  // [BH, Qb, Kb] kept key blocks, ascending, first cnt valid
  const int32_t* cnt;  // [BH, Qb]
  __nv_bfloat16* out;  // [BH, N, D]
  DeviceStatus* status;
  uint64_t timeout_ns;
  int N, Qb, Kb;
  float scale_log2;  // log2(e) / sqrt(d)
};

template <int D, bool kPInTmem>
struct Cfg {
  static constexpr int kChunk = 16384;           // one 128-row x 64-column bf16 SW128 chunk
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = 128 * D * 2;   // a pair of 64-row key blocks
  static constexpr int kKSt = (D == 128) ? 2 : (kPInTmem ? 4 : 3);
  static constexpr int kVSt = (D == 128) ? (kPInTmem ? 3 : 2) : (kPInTmem ? 4 : 3);
  static constexpr int kPBytes = kPInTmem ? 0 : 128 * 128 * 2;
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + kKSt * kKVBytes;
  static constexpr int kOffP = kOffV + kVSt * kKVBytes;
  static constexpr int kSmem = kOffP + kPBytes + 1024;  // + alignment slack
  // TMEM columns
  static constexpr uint32_t kColS = 0;    // two 128-column S buffers
  static constexpr uint32_t kColO = 256;  // D columns
  static constexpr uint32_t kColP = 384;  // 64 columns of packed bf16 pairs
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static_assert(kSmem > 114 * 1024, "one CTA per SM (it allocates all 512 TMEM columns)");
};

template <int D, bool kPInTmem>
__global__ void __launch_bounds__(256, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using C = Cfg<D, kPInTmem>;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bar_q, bar_kfull[C::kKSt], bar_kempty[C::kKSt],
      bar_vfull[C::kVSt], bar_vempty[C::kVSt], bar_sfull[2], bar_pfull, bar_odone, bar_final;
  __shared__ uint32_t s_tmem;
  __shared__ int16_t s_idx[kMaxKb];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x / a.Qb;
  const int qi = blockIdx.x - bh * a.Qb;
  const size_t row_id = static_cast<size_t>(bh) * a.Qb + qi;
  const int rows_valid = min(kBlockQ, a.N - qi * kBlockQ);
  __nv_bfloat16* out_blk = a.out + (static_cast<size_t>(bh) * a.N + static_cast<size_t>(qi) * kBlockQ) * D;

  // One thread reads the count (and whether an earlier CTA already gave up) so
  // that every thread takes the same early-exit decision.
  __shared__ int s_cnt;
  if (threadIdx.x == 0)
    s_cnt = (*reinterpret_cast<volatile uint32_t*>(&a.status->code) != 0) ? -1 : a.cnt[row_id];
  __syncthreads();
  const int cnt = s_cnt;
  if (cnt < 0) return;
  if (cnt == 0) {  // no kept key block: the defined output is zero
    uint4* o4 = reinterpret_cast<uint4*>(out_blk);
    for (int e = threadIdx.x; e < rows_valid * D / 8; e += blockDim.x) o4[e] = make_uint4(0, 0, 0, 0);
    return;
  }
  for (int t = threadIdx.x; t < cnt; t += blockDim.x) s_idx[t] = a.idx[row_id * a.Kb + t];

  const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
  const uint32_t sQ = base;
  const uint32_t sK0 = base + C::kOffK;
  const uint32_t sV0 = base + C::kOffV;
  const uint32_t sP = base + C::kOffP;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < C::kKSt; ++s) {
      mbar_init(smem_u32(&bar_kfull[s]), 1);
      mbar_init(smem_u32(&bar_kempty[s]), 1);
    }
    for (int s = 0; s < C::kVSt; ++s) {
      mbar_init(smem_u32(&bar_vfull[s]), 1);
      mbar_init(smem_u32(&bar_vempty[s]), 1);
    }
    mbar_init(smem_u32(&bar_sfull[0]), 1);
    mbar_init(smem_u32(&bar_sfull[1]), 1);
    mbar_init(smem_u32(&bar_pfull), 128);
    mbar_init(smem_u32(&bar_odone), 1);
    mbar_init(smem_u32(&bar_final), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int npairs = (cnt + 1) >> 1;
  DeviceStatus* st = a.status;
  const uint64_t tmo = a.timeout_ns;

  // Stage-issue counters, used by the producers to drain in-flight copies.
  uint32_t issued[4] = {0, 0, 0, 0};

  if (warp == 0) {
    // ------------------------------------------------ Q / K producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      mbar_expect_tx(smem_u32(&bar_q), C::kQBytes);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_3d(sQ + c * C::kChunk, &tm_q, smem_u32(&bar_q), c * 64, qi * kBlockQ, bh);
      for (int j = 0; j < npairs; ++j) {
        const int s = j % C::kKSt;
        const int n = j / C::kKSt;
        if (n > 0 && !mbar_wait(smem_u32(&bar_kempty[s]), (n - 1) & 1, st, tmo, kWaitKEmpty)) break;
        const int nb = min(2, cnt - 2 * j);
        const uint32_t bar = smem_u32(&bar_kfull[s]);
        mbar_expect_tx(bar, nb * 64 * D * 2);
        for (int h = 0; h < nb; ++h) {
          const int blk = s_idx[2 * j + h];
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(sK0 + s * C::kKVBytes + c * C::kChunk + h * 8192, &tm_k, bar, c * 64,
                        blk * kBlockK, bh);
        }
        ++issued[s];
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------ V producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_v);
      for (int j = 0; j < npairs; ++j) {
        const int s = j % C::kVSt;
        const int n = j / C::kVSt;
        if (n > 0 && !mbar_wait(smem_u32(&bar_vempty[s]), (n - 1) & 1, st, tmo, kWaitVEmpty)) break;
        const int nb = min(2, cnt - 2 * j);
        const uint32_t bar = smem_u32(&bar_vfull[s]);
        mbar_expect_tx(bar, nb * 64 * D * 2);
        for (int h = 0; h < nb; ++h) {
          const int blk = s_idx[2 * j + h];
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(sV0 + s * C::kKVBytes + c * C::kChunk + h * 8192, &tm_v, bar, c * 64,
                        blk * kBlockK, bh);
        }
        ++issued[s];
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_bf16(128, D, true);
      bool ok = mbar_wait(smem_u32(&bar_q), 0, st, tmo, kWaitQ);
      tc_fence_after();
      auto issue_qk = [&](int j) -> bool {
        const int s = j % C::kKSt;
        if (!mbar_wait(smem_u32(&bar_kfull[s]), (j / C::kKSt) & 1, st, tmo, kWaitKFull)) return false;
        tc_fence_after();
        const int nb = min(2, cnt - 2 * j);
        const uint32_t idesc = idesc_bf16(128, 64 * nb, false);
        const uint32_t dt = tmem + C::kColS + (j & 1) * 128;
        const uint32_t kb = sK0 + s * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kChunk + (kk & 3) * 32;
          umma_ss(dt, sw128_desc(sQ + off, 16, 1024), sw128_desc(kb + off, 16, 1024), idesc, kk > 0);
        }
        umma_commit(smem_u32(&bar_sfull[j & 1]));
        umma_commit(smem_u32(&bar_kempty[s]));
        return true;
      };
      if (ok) ok = issue_qk(0);
      for (int j = 0; ok && j < npairs; ++j) {
        if (j + 1 < npairs && !(ok = issue_qk(j + 1))) break;
        if (!(ok = mbar_wait(smem_u32(&bar_pfull), j & 1, st, tmo, kWaitPFull))) break;
        const int s = j % C::kVSt;
        if (!(ok = mbar_wait(smem_u32(&bar_vfull[s]), (j / C::kVSt) & 1, st, tmo, kWaitVFull))) break;
        tc_fence_after();
        const int nb = min(2, cnt - 2 * j);
        const uint32_t vb = sV0 + s * C::kKVBytes;
        for (int kk = 0; kk < nb * 4; ++kk) {
          const uint64_t bdesc = sw128_desc(vb + kk * 2048, C::kChunk, 1024);
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          if constexpr (kPInTmem) {
            umma_ts(tmem + C::kColO, tmem + C::kColP + kk * 8, bdesc, idesc_pv, acc);
          } else {
            const uint32_t pa = sP + (kk >> 2) * C::kChunk + (kk & 3) * 32;
            umma_ss(tmem + C::kColO, sw128_desc(pa, 16, 1024), bdesc, idesc_pv, acc);
          }
        }
        umma_commit(smem_u32(&bar_odone));
        umma_commit(smem_u32(&bar_vempty[s]));
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ softmax + epilogue
    const int row = threadIdx.x - 128;  // query row in the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    const int kb_last = a.Kb - 1;
    const int tail = a.N - kb_last * kBlockK;  // valid keys in the last key block (1..64)
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < npairs; ++j) {
      ok = mbar_wait(smem_u32(&bar_sfull[j & 1]), (j >> 1) & 1, st, tmo, kWaitSFull);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const int nb = min(2, cnt - 2 * j);
      float s[128];
      const uint32_t sbuf = tmem + lane_off + C::kColS + (j & 1) * 128;
      tmem_ld64(sbuf, s);
      if (nb == 2) {
        tmem_ld64(sbuf + 64, s + 64);
      } else {
#pragma unroll
        for (int c = 64; c < 128; ++c) s[c] = -INFINITY;
      }
      if (tail < 64) {
        const bool last0 = s_idx[2 * j] == kb_last;
        const bool last1 = nb == 2 && s_idx[2 * j + 1] == kb_last;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          if (last0 && c >= tail) s[c] = -INFINITY;
          if (last1 && c >= tail) s[64 + c] = -INFINITY;
        }
      }
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = s[e];
#pragma unroll
      for (int c = 8; c < 128; ++c) mx[c & 7] = fmaxf(mx[c & 7], s[c]);
      const float rmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float m_new = fmaxf(m_run, rmax * sl2);
      const bool need = m_new > m_run + 8.0f;  // always true for the first pair
      const float m_use = need ? m_new : m_run;
      const float alpha = ex2_approx(m_run - m_use);  // 0 for the first pair, 1 if no rescale
      uint32_t pk[64];
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2_approx(fmaf(s[2 * c], sl2, -m_use));
        const float p1 = ex2_approx(fmaf(s[2 * c + 1], sl2, -m_use));
        ps[c & 3] += p0 + p1;
        pk[c] = pack_bf16(p0, p1);
      }
      l_run = l_run * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      if (j > 0) {
        // O and the P buffer are free once the previous P.V has completed.
        ok = mbar_wait(smem_u32(&bar_odone), (j - 1) & 1, st, tmo, kWaitODone);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            float o[32];
            const uint32_t oaddr = tmem + lane_off + C::kColO + cc * 32;
            tmem_ld32(oaddr, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(oaddr, reinterpret_cast<const uint32_t*>(o));
          }
        }
      }
      if constexpr (kPInTmem) {
        tmem_st32(tmem + lane_off + C::kColP, pk);
        if (nb == 2) tmem_st32(tmem + lane_off + C::kColP + 32, pk + 32);
      } else {
        // Row `row` of the K-major, 128-byte-swizzled P tile (keys 0-63 in the
        // first 16 KB chunk, keys 64-127 in the second).
        const uint32_t rbase = sP + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const uint32_t addr = rbase + h * C::kChunk + ((g ^ (row & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                         "r"(pk[h * 32 + g * 4]), "r"(pk[h * 32 + g * 4 + 1]),
                         "r"(pk[h * 32 + g * 4 + 2]), "r"(pk[h * 32 + g * 4 + 3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_pfull));
      m_run = m_use;
    }
    if (ok) {
      ok = mbar_wait(smem_u32(&bar_odone), (npairs - 1) & 1, st, tmo, kWaitODone);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      __nv_bfloat16* orow = out_blk + static_cast<size_t>(row) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        float o[32];
        tmem_ld32(tmem + lane_off + C::kColO + cc * 32, o);
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = pack_bf16(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
        if (row < rows_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  // Every role has left its loop (finished, or gave up after a bounded wait).
  // Drain what may still be in flight before the TMEM is released and the CTA
  // exits: outstanding TMA loads (producers) and tensor-core ops (issuer).
  __syncthreads();
  if ((warp == 0 || warp == 2) && lane == 0) {
    const int nst = (warp == 0) ? C::kKSt : C::kVSt;
    for (int s = 0; s < nst; ++s) {
      if (issued[s] == 0) continue;
      const uint32_t bar = smem_u32(warp == 0 ? &bar_kfull[s] : &bar_vfull[s]);
      uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar, (issued[s] - 1) & 1)) {
        if (globaltimer_ns() - t0 > tmo) {
          atomicCAS(&st->code, 0u, kDevTimeout);
          break;
        }
      }
    }
    if (warp == 0) {
      uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&bar_q), 0)) {
        if (globaltimer_ns() - t0 > tmo) {
          atomicCAS(&st->code, 0u, kDevTimeout);
          break;
        }
      }
    }
  }
  if (warp == 1) {
    if (lane == 0) {
      umma_commit(smem_u32(&bar_final));
      uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&bar_final), 0)) {
        if (globaltimer_ns() - t0 > tmo) {
          atomicCAS(&st->code, 0u, kDevTimeout);
          break;
        }
      }
    }
    __syncwarp();
    tc_fence_after();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [BH, N, D] bf16 viewed as a 3-D tensor (D fastest); box = 64 columns x rows x 1,
// 128-byte swizzle, rows past N read as zero.
bool make_map(CUtensorMap* m, const void* ptr, int BH, int N, int D, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(N) * D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool kPInTmem>
cudaError_t launch_typed(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const AttnArgs& args, int BH, cudaStream_t st) {
  using C = Cfg<D, kPInTmem>;
  auto kern = bsa_fwd_kernel<D, kPInTmem>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(BH) * static_cast<unsigned>(args.Qb);
  kern<<<grid, 256, C::kSmem, st>>>(mq, mk, mv, args);
  return cudaGetLastError();
}

}  // namespace

#ifndef BSA_P_IN_TMEM
#define BSA_P_IN_TMEM 1
#endif

cudaError_t launch_attention(const void* q, const void* k, const void* v, void* out, int BH, int N,
                             int d, const int16_t* idx, const int32_t* cnt, DeviceStatus* status,
                             uint64_t timeout_ns, cudaStream_t st, const char** why) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, BH, N, d, kBlockQ) || !make_map(&mk, k, BH, N, d, kBlockK) ||
      !make_map(&mv, v, BH, N, d, kBlockK)) {
    if (why) *why = "cuTensorMapEncodeTiled failed or is unavailable";
    return cudaErrorInvalidValue;
  }
  AttnArgs args;
  args.idx = idx;
  args.cnt = cnt;
  args.out = static_cast<__nv_bfloat16*>(out);
  args.status = status;
  args.timeout_ns = timeout_ns;
  args.N = N;
  args.Qb = (N + kBlockQ - 1) / kBlockQ;
  args.Kb = (N + kBlockK - 1) / kBlockK;
  args.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(d));
  if (d == 128) return launch_typed<128, BSA_P_IN_TMEM != 0>(mq, mk, mv, args, BH, st);
  return launch_typed<64, BSA_P_IN_TMEM != 0>(mq, mk, mv, args, BH, st);
}

}  // namespace bsa
